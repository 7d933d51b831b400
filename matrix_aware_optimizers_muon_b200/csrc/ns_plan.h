// Planning and launch sequence of the Newton-Schulz path (Muon and the plain
// orthogonaliser): shape buckets, workspace carving, chunking.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>
#include <vector>

#include <cuda_runtime.h>

namespace mo {

constexpr size_t WS_HEADER = 256;   // device status word + reserved

struct NsItem {
  long long rows = 0, cols = 0;   // stored shape
  const float* in = nullptr;      // G (Muon) or input
  float* mom = nullptr;           // momentum (Muon) or nullptr
  float* out = nullptr;           // W (Muon) or output
  int32_t* flag = nullptr;        // nonfinite flag slot
  bool vec = false;               // float4 path allowed
};

struct NsCall {
  bool muon = true;
  float beta = 0.95f;
  bool nesterov = true, ema = false;
  int steps = 5;
  float a = 3.4445f, b = -4.7750f, c = 2.0315f, eps = 1e-7f;
  float lr = 0.f, wd = 0.f;
  int adjust_lr = 0;
};

// Workspace bytes: *min_bytes runs one matrix at a time, *full_bytes runs
// every bucket of equal oriented shape as one batch.
void ns_workspace(const int64_t* rows, const int64_t* cols, int n, size_t* min_bytes, size_t* full_bytes);

// Enqueue the whole call.  On a planning error (workspace too small) sets
// *err and returns cudaSuccess without launching.
cudaError_t ns_run(const std::vector<NsItem>& items, const NsCall& call, char* ws, size_t ws_bytes,
                   cudaStream_t stream, std::string* err);

// The same with the status word and the scratch region given apart (for
// callers that place the Newton-Schulz scratch inside a larger workspace).
cudaError_t ns_run_at(const std::vector<NsItem>& items, const NsCall& call, int* status, char* base,
                      size_t avail, cudaStream_t stream, std::string* err);

}  // namespace mo
