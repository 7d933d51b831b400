// Internal host-side interfaces shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <utility>

namespace mo {

// Makes a context's device current for the length of one API call and puts
// the caller's current device back when the call returns, so that calling
// into the library never changes which device the caller's thread uses.
class DeviceScope {
 public:
  DeviceScope() = default;
  DeviceScope(const DeviceScope&) = delete;
  DeviceScope& operator=(const DeviceScope&) = delete;
  cudaError_t enter(int dev) {
    cudaError_t e = cudaGetDevice(&prev_);
    if (e != cudaSuccess) return e;
    if (prev_ != dev) {
      e = cudaSetDevice(dev);
      if (e == cudaSuccess) switched_ = true;
    }
    return e;
  }
  ~DeviceScope() {
    if (switched_) (void)cudaSetDevice(prev_);
  }

 private:
  int prev_ = -1;
  bool switched_ = false;
};

// Device address of the status word at the start of the fixed scratch array
// of ns_orthogonalize_static on device `dev`, or null while no call has set
// the array up there.
int32_t* static_status_word(int dev);

// Allow `bytes` of dynamic shared memory for kernel `func` on the current
// device: set once per (device, kernel), thread-safe.
cudaError_t ensure_smem_attr(const void* func, int bytes);

// Launch `kern` with programmatic stream serialization (and, with cluster2,
// clusters of two CTAs): it may start while the previous kernel of the
// stream runs, so it must call pdl_wait() before touching global memory.
// Per host thread: launches made by launch_pdl leave out programmatic
// stream serialization while set (graph bodies recorded by the library).
inline bool& pdl_off() {
  static thread_local bool off = false;
  return off;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       bool cluster2, Args&&... args) {
  // programmatic serialization unless this thread is recording a graph body
  // that must hold plain kernel nodes (pdl_off())
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (!pdl_off()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster2) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 2;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// One batched GEMM D_b = alpha_b * (A_b B_b) + beta_b * C_b on bf16 (or,
// with ab_f16, fp16) operands.
// Operand storage (row-major, element strides):
//   A: a_mn ? [K rows][M cols] : [M rows][K cols]
//   B: b_mn ? [K rows][N cols] : [N rows][K cols]
// Row strides must be multiples of 8 elements and base pointers 16-byte
// aligned (TMA); C and D may be bf16 or fp32.
struct GemmOp {
  const void* A = nullptr;
  long long lda = 0, strideA = 0;
  int a_mn = 0;
  const void* B = nullptr;
  long long ldb = 0, strideB = 0;
  int b_mn = 0;
  int M = 0, N = 0, K = 0, batch = 1;
  int sym = 0;
  float alpha = 1.f, beta = 0.f;
  const float* scale = nullptr;
  int alpha_pow = 0, beta_pow = 0;
  const void* C = nullptr;
  long long ldc = 0, strideC = 0;
  int c_f32 = 0;
  void* D = nullptr;
  long long ldd = 0, strideD = 0;
  int d_f32 = 0;
  int kind = 9;          // profiling tag (ProfKind)
  // per-matrix pointer tables in device memory (optional)
  const void* const* c_tab = nullptr;
  void* const* d_tab = nullptr;
  float* const* e_tab = nullptr;
  long long lde = 0;
  // epilogue mode: 0 = alpha acc + beta C, 1 = Adam in the rotated basis,
  // 2 = the Muon apply of O = bf16(alpha acc + beta C) to W = e_tab[b]
  int epi = 0;
  float adam_b2 = 0.f, adam_ibc1 = 1.f, adam_ibc2 = 1.f, adam_eps = 0.f;
  // tile order: 0 = chosen by the launcher; n > 0 = bands of n row tiles
  int band = 0;
  // Muon apply (epi 2): W <- ap_decay W - ap_step[tall] O; matrices
  // b >= ap_tall_from store W transposed (N x M), the others as M x N
  float ap_decay = 1.f;
  float ap_step[2] = {0.f, 0.f};
  int ap_tall_from = 0;
  int ap_vec = 0;        // every W: 16-byte aligned base and row stride
  // plane-stacked K (split-precision products): K = nseg * kseg, segment s
  // uses plane pat_a[s] of A and pat_b[s] of B; planes are planeA/planeB
  // elements apart.  kseg must be a multiple of 64 when nseg > 1.
  int nseg = 1;
  unsigned char pat_a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  unsigned char pat_b[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  long long planeA = 0, planeB = 0;
  // bf16 D written as two planes (h, l) d_plane elements apart
  int d_split = 0;
  long long d_plane = 0;
  // per-matrix skip flags in device memory (optional)
  const int* skip = nullptr;
  // A and B hold fp16 values (both; the MMA takes one type for the two)
  int ab_f16 = 0;
  // optional launch gate (device): the whole launch does nothing when
  // *gate >= gate_n (every matrix of a refresh pass already done)
  const int* gate = nullptr;
  int gate_n = 0;
  const int* gate_idx = nullptr;     // optional device index: the gate word is gate[*gate_idx]
  // added to each matrix's diagonal (row == column) before D is rounded
  float diag_add = 0.f;
  // CTA pairs (256 x 256 tiles over two SMs) where the shape allows them,
  // whatever K (measured faster for the SOAP products, slower for the
  // Newton-Schulz chain's long-K products at the power cap)
  int pair = 0;
};

// Launch the tcgen05 GEMM.  Returns cudaSuccess or the launch/encode error.
cudaError_t launch_gemm(const GemmOp& op, int* status, cudaStream_t stream);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Round x up to a multiple of a.
inline long long round_up(long long x, long long a) { return (x + a - 1) / a * a; }

}  // namespace mo
