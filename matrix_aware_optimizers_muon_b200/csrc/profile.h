// Optional per-launch timing: when a context enables it, every kernel launch
// the library issues is bracketed by a CUDA event pair on its stream, tagged
// with the kernel kind and the launch's executed tensor-core flops.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <vector>

namespace mo {

enum ProfKind {
  PK_PREP = 0,       // Muon momentum / cast / partial norms
  PK_NORM = 1,       // norm finalize
  PK_GRAM = 2,       // A = X X^T
  PK_POLY = 3,       // P = a I + b A + c A A
  PK_UPDATE = 4,     // X' = P X  (P = a I + b A + c A A; small kernel: a X + P X)
  PK_APPLY = 5,      // W update / output store
  PK_SOAP_EW = 6,    // SOAP elementwise kernels
  PK_SOAP_GEMM = 7,  // SOAP tensor-core products
  PK_SOAP_QR = 8,    // SOAP QR (Cholesky / triangular kernels)
  PK_GEMM = 9,       // stand-alone mo_gemm_bf16
  PK_SOAP_EMA = 10,  // SOAP factor EMAs (symmetric products)
  PK_QR_CHOL = 11,   // QR: diagonal-block Cholesky + inverse
  PK_QR_ROWBLK = 12, // QR: panel / TRSM row blocks times the block inverse
  PK_QR_TRAIL = 13,  // QR: tensor-core trailing updates
  PK_SMALL = 14,     // fused small-matrix Newton-Schulz / Muon
  PK_TABLES = 15,    // device pointer-table uploads
  PK_COUNT = 16
};

struct ProfRec {
  cudaEvent_t a = nullptr, b = nullptr;
  int kind = 0;
  double flops = 0;
};

struct Profiler {
  std::vector<ProfRec> recs;
  size_t used = 0;
  bool failed = false;
};

extern thread_local Profiler* g_prof;

// Named host range (NVTX) around a call or a phase, for timeline profilers;
// the calls do nothing unless a profiler is attached to the process.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// RAII bracket around one launch (no-op when profiling is off).
struct ProfScope {
  ProfRec* rec = nullptr;
  cudaStream_t s;
  ProfScope(int kind, cudaStream_t stream, double flops = 0.0);
  ~ProfScope();
};

}  // namespace mo
