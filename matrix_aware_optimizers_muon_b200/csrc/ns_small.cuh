// Fused small-matrix Newton-Schulz / Muon kernel (m' <= 128, n' <= 256).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mo {

constexpr int SMALL_MAX_M = 128;
constexpr int SMALL_MAX_N = 256;

struct SmallArgs {
  int count;                  // matrices (all with the stored shape rows x cols)
  int rows, cols;
  int tall;                   // rows > cols: transposed when oriented
  int mode;                   // 0: out = O ; 1: Muon (momentum in, W update out)
  float beta;
  int nesterov, ema;
  int steps;
  int vec;                    // 1: cols % 4 == 0 and every matrix 16-byte aligned
  float a, b, c, eps;
  float decay, step;
  const float* const* in;     // device tables of `count` pointers
  float* const* mom;          // null in mode 0
  float* const* out;
  int32_t* const* flag;       // null or table (entries may be null)
  int* status;
  uint32_t cols_magic;        // set by the launcher: ceil(2^32 / cols), row = umulhi(index, magic)
};

// Uploads `n` entries of four pointer tables (in, mom, out, flag) into device
// memory at dst (4 consecutive arrays of `n` pointers).
void launch_upload_tables(void** dst, int n, const void* const* in, const void* const* mom,
                          const void* const* out, const void* const* flag, cudaStream_t s);

// One persistent launch over all matrices (grid: up to three CTAs per SM).
cudaError_t launch_ns_small(const SmallArgs& a, int sm_count, cudaStream_t s);

}  // namespace mo
