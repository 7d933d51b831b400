// ns_orthogonalize_static: the Newton-Schulz orthogonaliser for one matrix
// with its scratch in a fixed device array instead of a caller workspace.
//
// Who needs it: callers that cannot allocate device memory at the point of
// the call -- code whose GPU memory is owned by another allocator that
// leaves nothing spare to hand out, a runtime that forbids allocation after
// start-up, or a caller with no access to an allocator at all (a plain C
// host program linking only this library).  They pass their input and output
// buffers; the scratch is the array below, which every GPU that loads this
// library holds (16 MiB) until the process exits.
//
// Set-up: the first call on a device, with that device current, looks up the
// array's device address with cudaGetSymbolAddress and caches it; that first
// call should therefore come before any stream capture.  In host code the
// array's name is only a host-side stand-in, never a device address.
//
// Sharing: every call uses the same array and leaves its contents behind.
// The array starts with a status word where a kernel wait that gives up
// records its code; mo_device_status reads and clears it (with or without
// an attached workspace), so a call that timed out is visible until then.
// Everything else a call reads it first writes.  Calls whose kernels overlap on the GPU (different streams
// without ordering) race on the array.
#include <cmath>
#include <mutex>
#include <string>

#include "../../include/mo.h"
#include "elementwise.cuh"
#include "ns_plan.h"
#include "runtime.h"

static __device__ __align__(256) unsigned char g_ns_scratch[MO_STATIC_SCRATCH_BYTES];

namespace mo {
int ctx_device(const mo_ctx* ctx);
mo_status ctx_fail(mo_ctx* ctx, mo_status st, const std::string& msg);
}

namespace {

constexpr size_t kAlign = 1024;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

std::mutex g_setup_mu;
char* g_scratch_addr[64] = {nullptr};

// Device address of the scratch array on `dev` (which must be current).
cudaError_t scratch_on(int dev, char** out) {
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_ns_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<char*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

namespace mo {
int32_t* static_status_word(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  return reinterpret_cast<int32_t*>(g_scratch_addr[dev]);
}
}  // namespace mo

extern "C" MO_API mo_status ns_orthogonalize_static(mo_ctx* ctx, const float* in, float* out,
                                                    int64_t rows, int64_t cols, const mo_ns_cfg* cfg,
                                                    void* stream) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (in == nullptr || out == nullptr || cfg == nullptr)
    return mo::ctx_fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize_static: null argument");
  if (rows <= 0 || cols <= 0 || rows > (1 << 20) || cols > (1 << 20))
    return mo::ctx_fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize_static: bad shape");
  if (cfg->ns_steps < 1 || cfg->ns_steps > 64 || !std::isfinite(cfg->a) || !std::isfinite(cfg->b) ||
      !std::isfinite(cfg->c) || !std::isfinite(cfg->eps) || cfg->eps < 0.f)
    return mo::ctx_fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize_static: bad Newton-Schulz config");
  if ((reinterpret_cast<uintptr_t>(in) & 3u) || (reinterpret_cast<uintptr_t>(out) & 3u))
    return mo::ctx_fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize_static: pointers must be 4-byte aligned");
  const size_t bytes = (size_t)rows * cols * 4;
  const char* a0 = reinterpret_cast<const char*>(in);
  const char* b0 = reinterpret_cast<const char*>(out);
  if (a0 < b0 + bytes && b0 < a0 + bytes)
    return mo::ctx_fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize_static: in and out overlap");

  // the same oriented layout as the workspace path, for one matrix
  const bool tall = rows > cols;
  const long long mp = tall ? cols : rows, np = tall ? rows : cols;
  const long long ldx = mo::round_up(np, 64), lda = mo::round_up(mp, 64);
  const long long xstride = mp * ldx, astride = mp * lda;
  const long long tiles = ((mp + 63) / 64) * ((np + 63) / 64);
  const size_t need = mo::WS_HEADER + 2 * align_up(xstride * 2) + 2 * align_up(astride * 2) +
                      align_up(tiles * 4) + align_up(4);
  if (need > MO_STATIC_SCRATCH_BYTES)
    return mo::ctx_fail(ctx, MO_ERR_UNSUPPORTED,
                        "ns_orthogonalize_static: a " + std::to_string(rows) + " x " + std::to_string(cols) +
                            " matrix needs " + std::to_string(need) + " bytes of scratch; the fixed array holds " +
                            std::to_string((size_t)MO_STATIC_SCRATCH_BYTES) +
                            " (use ns_orthogonalize with a workspace)");

  const int dev = mo::ctx_device(ctx);
  mo::DeviceScope dev_scope;                     // the caller's device is current again on return
  cudaError_t e = dev_scope.enter(dev);
  char* ws = nullptr;
  if (e == cudaSuccess) e = scratch_on(dev, &ws);
  if (e != cudaSuccess)
    return mo::ctx_fail(ctx, MO_ERR_CUDA, std::string("ns_orthogonalize_static: set-up: ") + cudaGetErrorString(e));
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  int* status = reinterpret_cast<int*>(ws);
  char* p = ws + mo::WS_HEADER;
  __nv_bfloat16* X0 = reinterpret_cast<__nv_bfloat16*>(p); p += align_up(xstride * 2);
  __nv_bfloat16* X1 = reinterpret_cast<__nv_bfloat16*>(p); p += align_up(xstride * 2);
  __nv_bfloat16* A = reinterpret_cast<__nv_bfloat16*>(p); p += align_up(astride * 2);
  __nv_bfloat16* P = reinterpret_cast<__nv_bfloat16*>(p); p += align_up(astride * 2);
  float* part = reinterpret_cast<float*>(p); p += align_up(tiles * 4);
  float* inv = reinterpret_cast<float*>(p);

  // The status word (zero when the library loads) is not cleared here: a
  // timeout code an earlier call recorded stays until mo_device_status reads
  // it.  All other scratch is written before it is read.

  mo::EwTable t;
  t.in[0] = in; t.mom[0] = nullptr; t.out[0] = out;
  t.flag[0] = cfg->nonfinite; t.tall[0] = tall ? 1 : 0;
  const bool vec = (cols % 4 == 0) && !(reinterpret_cast<uintptr_t>(in) & 15u) &&
                   !(reinterpret_cast<uintptr_t>(out) & 15u);
  mo::PrepArgs pa;
  pa.count = 1; pa.mp = (int)mp; pa.np = (int)np;
  pa.tiles_r = (int)((rows + 63) / 64); pa.tiles_c = (int)((cols + 63) / 64);
  pa.beta = 0.f; pa.mode = 0; pa.nesterov = 0; pa.ema = 0; pa.vec = vec;
  pa.X = X0; pa.ldx = ldx; pa.xstride = xstride; pa.partial = part;
  if (e == cudaSuccess) { mo::launch_prep(t, pa, s); e = cudaGetLastError(); }
  mo::FinalizeArgs fa;
  fa.count = 1; fa.tiles = (int)tiles; fa.eps = cfg->eps; fa.partial = part; fa.inv = inv;
  if (e == cudaSuccess) { mo::launch_finalize(t, fa, s); e = cudaGetLastError(); }

  __nv_bfloat16* Xc = X0;
  __nv_bfloat16* Xn = X1;
  for (int it = 0; it < cfg->ns_steps && e == cudaSuccess; ++it) {
    mo::GemmOp g;                                  // A = X X^T
    g.A = Xc; g.lda = ldx; g.strideA = xstride;
    g.B = Xc; g.ldb = ldx; g.strideB = xstride;
    g.M = (int)mp; g.N = (int)mp; g.K = (int)np; g.sym = 1;
    g.scale = inv; g.alpha_pow = it == 0 ? 2 : 0;
    g.D = A; g.ldd = lda; g.strideD = astride;
    e = mo::launch_gemm(g, status, s);
    if (e != cudaSuccess) break;
    const bool fold = mp >= 128;                   // as in the workspace path
    mo::GemmOp q;                                  // P = a I + b A + c A A (or b A + c A A)
    q.A = A; q.lda = lda; q.strideA = astride;
    q.B = A; q.ldb = lda; q.strideB = astride;
    q.M = (int)mp; q.N = (int)mp; q.K = (int)mp; q.sym = 1;
    q.alpha = cfg->c; q.beta = cfg->b; q.diag_add = fold ? cfg->a : 0.f;
    q.C = A; q.ldc = lda; q.strideC = astride;
    q.D = P; q.ldd = lda; q.strideD = astride;
    e = mo::launch_gemm(q, status, s);
    if (e != cudaSuccess) break;
    mo::GemmOp u;                                  // X' = P X (or a X + P X)
    u.A = P; u.lda = lda; u.strideA = astride;
    u.B = Xc; u.ldb = ldx; u.strideB = xstride; u.b_mn = 1;
    u.M = (int)mp; u.N = (int)np; u.K = (int)mp;
    u.scale = inv; u.alpha_pow = it == 0 ? 1 : 0;
    if (!fold) {
      u.beta = cfg->a; u.beta_pow = it == 0 ? 1 : 0;
      u.C = Xc; u.ldc = ldx; u.strideC = xstride;
    }
    u.D = Xn; u.ldd = ldx; u.strideD = xstride;
    e = mo::launch_gemm(u, status, s);
    Xc = Xn;
    Xn = (Xn == X1) ? X0 : X1;
  }
  mo::ApplyArgs aa;
  aa.count = 1; aa.mp = (int)mp; aa.np = (int)np;
  aa.tiles_r = pa.tiles_r; aa.tiles_c = pa.tiles_c;
  aa.mode = 0; aa.decay = 1.f; aa.step = 0.f; aa.vec = vec;
  aa.X = Xc; aa.ldx = ldx; aa.xstride = xstride;
  if (e == cudaSuccess) { mo::launch_apply(t, aa, s); e = cudaGetLastError(); }
  if (e != cudaSuccess)
    return mo::ctx_fail(ctx, MO_ERR_CUDA, std::string("ns_orthogonalize_static: ") + cudaGetErrorString(e));
  return MO_OK;
}
