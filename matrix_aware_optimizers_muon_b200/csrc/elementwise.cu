// HBM-bound kernels of the Muon / Newton-Schulz path.
//
//  prep      B <- beta B + G (or the moving-average form), N = G + beta B
//            (Nesterov) or B; writes B, the bf16 cast of N in the oriented
//            layout (transposed through shared memory for tall matrices) and
//            one partial sum of N^2 per 64 x 64 tile.  Reads G and B once.
//  finalize  per matrix: ||N||_F from the tile partials in a fixed order
//            (bit-reproducible), inv = 1 / (||N||_F + eps), nonfinite flag.
//  apply     W <- (1 - lr wd) W - lr s O with O the bf16 Newton-Schulz
//            output (un-oriented), or out = O for the plain orthogonaliser.
#include "elementwise.cuh"
#include "runtime.h"
#include "ptx.cuh"
#include "profile.h"

namespace mo {

namespace {

constexpr int LDS = EW_TILE + 8;   // shared tile row: 72 bf16 = 144 bytes (16-byte aligned)

__device__ __forceinline__ float momentum_update(float g, float b, float beta, int ema) {
  return ema ? fmaf(beta, b, (1.0f - beta) * g) : fmaf(beta, b, g);
}

__global__ void __launch_bounds__(EW_THREADS) prep_kernel(const EwTable t, const PrepArgs a) {
  __shared__ __align__(16) __nv_bfloat16 xs[EW_TILE][LDS];
  __shared__ float red[EW_THREADS / 32];
  pdl_wait();
  pdl_trigger();

  const int T = a.tiles_r * a.tiles_c;
  const int j = blockIdx.x / T;
  const int tile = blockIdx.x - j * T;
  const bool tall = t.tall[j] != 0;
  const int rows = tall ? a.np : a.mp;        // stored shape
  const int cols = tall ? a.mp : a.np;
  const int tr = tile / a.tiles_c;
  const int tc = tile - tr * a.tiles_c;
  const int r0 = tr * EW_TILE, c0 = tc * EW_TILE;
  const float* __restrict__ G = t.in[j];
  float* __restrict__ B = t.mom[j];
  const float beta = a.beta;
  float ss = 0.0f;

  auto put = [&](int r, int c, float n) {
    const __nv_bfloat16 h = __float2bfloat16_rn(n);
    if (tall) xs[c][r] = h; else xs[r][c] = h;
  };

  if (a.vec) {
    const int cq = (threadIdx.x & 15) * 4;
    const int rr = threadIdx.x >> 4;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int r = rr + 16 * p;
      const int gr = r0 + r, gc = c0 + cq;
      float n[4] = {0.f, 0.f, 0.f, 0.f};
      if (gr < rows && gc < cols) {
        const size_t off = (size_t)gr * cols + gc;
        const float4 g = __ldcs(reinterpret_cast<const float4*>(G + off));
        if (a.mode == 1) {
          const float4 b = __ldcs(reinterpret_cast<const float4*>(B + off));
          float4 bn;
          bn.x = momentum_update(g.x, b.x, beta, a.ema);
          bn.y = momentum_update(g.y, b.y, beta, a.ema);
          bn.z = momentum_update(g.z, b.z, beta, a.ema);
          bn.w = momentum_update(g.w, b.w, beta, a.ema);
          __stcs(reinterpret_cast<float4*>(B + off), bn);
          if (a.nesterov) {
            n[0] = fmaf(beta, bn.x, g.x); n[1] = fmaf(beta, bn.y, g.y);
            n[2] = fmaf(beta, bn.z, g.z); n[3] = fmaf(beta, bn.w, g.w);
          } else {
            n[0] = bn.x; n[1] = bn.y; n[2] = bn.z; n[3] = bn.w;
          }
        } else {
          n[0] = g.x; n[1] = g.y; n[2] = g.z; n[3] = g.w;
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ss = fmaf(n[i], n[i], ss);
        put(r, cq + i, n[i]);
      }
    }
  } else {
    const int c = threadIdx.x & 63;
    const int rr = threadIdx.x >> 6;
#pragma unroll 4
    for (int p = 0; p < 16; ++p) {
      const int r = rr + 4 * p;
      const int gr = r0 + r, gc = c0 + c;
      float n = 0.f;
      if (gr < rows && gc < cols) {
        const size_t off = (size_t)gr * cols + gc;
        const float g = G[off];
        if (a.mode == 1) {
          const float bn = momentum_update(g, B[off], beta, a.ema);
          B[off] = bn;
          n = a.nesterov ? fmaf(beta, bn, g) : bn;
        } else {
          n = g;
        }
      }
      ss = fmaf(n, n, ss);
      put(r, c, n);
    }
  }
  __syncthreads();

  // write the oriented bf16 tile: X row = stored row (wide) or stored col (tall)
  const int orow0 = tall ? c0 : r0;
  const int ocol0 = tall ? r0 : c0;
  __nv_bfloat16* X = a.X + (size_t)j * a.xstride;
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int i = (threadIdx.x >> 3) + 32 * p;
    const int k = (threadIdx.x & 7) * 8;
    const int orow = orow0 + i;
    if (orow < a.mp) {
      const uint4 v = *reinterpret_cast<const uint4*>(&xs[i][k]);
      *reinterpret_cast<uint4*>(X + (size_t)orow * a.ldx + ocol0 + k) = v;
    }
  }

  // deterministic block reduction of the tile's sum of squares
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < EW_THREADS / 32; ++w) s += red[w];
    a.partial[(size_t)j * T + tile] = s;
  }
}

__global__ void finalize_kernel(const EwTable t, const FinalizeArgs a) {
  pdl_wait();
  pdl_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.count) return;
  const float* p = a.partial + (size_t)warp * a.tiles;
  float s = 0.f;
  for (int i = lane; i < a.tiles; i += 32) s += p[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    const float norm = sqrtf(s);
    a.inv[warp] = 1.0f / (norm + a.eps);
    if (t.flag[warp] != nullptr) *t.flag[warp] = isfinite(norm) ? 0 : 1;
  }
}

__global__ void __launch_bounds__(EW_THREADS) apply_kernel(const EwTable t, const ApplyArgs a) {
  __shared__ __align__(16) __nv_bfloat16 xs[EW_TILE][LDS];
  pdl_wait();
  pdl_trigger();

  const int T = a.tiles_r * a.tiles_c;
  const int j = blockIdx.x / T;
  const int tile = blockIdx.x - j * T;
  const bool tall = t.tall[j] != 0;
  const int rows = tall ? a.np : a.mp;
  const int cols = tall ? a.mp : a.np;
  const int tr = tile / a.tiles_c;
  const int tc = tile - tr * a.tiles_c;
  const int r0 = tr * EW_TILE, c0 = tc * EW_TILE;
  const int orow0 = tall ? c0 : r0;
  const int ocol0 = tall ? r0 : c0;
  const __nv_bfloat16* X = a.X + (size_t)j * a.xstride;

#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int i = (threadIdx.x >> 3) + 32 * p;
    const int k = (threadIdx.x & 7) * 8;
    const int orow = orow0 + i;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (orow < a.mp) v = *reinterpret_cast<const uint4*>(X + (size_t)orow * a.ldx + ocol0 + k);
    *reinterpret_cast<uint4*>(&xs[i][k]) = v;
  }
  __syncthreads();

  float* __restrict__ W = t.out[j];
  auto o_at = [&](int r, int c) -> float {
    return __bfloat162float(tall ? xs[c][r] : xs[r][c]);
  };
  if (a.vec) {
    const int cq = (threadIdx.x & 15) * 4;
    const int rr = threadIdx.x >> 4;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int r = rr + 16 * p;
      const int gr = r0 + r, gc = c0 + cq;
      if (gr < rows && gc < cols) {
        const size_t off = (size_t)gr * cols + gc;
        float4 o = make_float4(o_at(r, cq), o_at(r, cq + 1), o_at(r, cq + 2), o_at(r, cq + 3));
        if (a.mode == 1) {
          const float4 w = __ldcs(reinterpret_cast<const float4*>(W + off));
          o.x = fmaf(a.decay, w.x, -a.step * o.x);
          o.y = fmaf(a.decay, w.y, -a.step * o.y);
          o.z = fmaf(a.decay, w.z, -a.step * o.z);
          o.w = fmaf(a.decay, w.w, -a.step * o.w);
        }
        __stcs(reinterpret_cast<float4*>(W + off), o);
      }
    }
  } else {
    const int c = threadIdx.x & 63;
    const int rr = threadIdx.x >> 6;
#pragma unroll 4
    for (int p = 0; p < 16; ++p) {
      const int r = rr + 4 * p;
      const int gr = r0 + r, gc = c0 + c;
      if (gr < rows && gc < cols) {
        const size_t off = (size_t)gr * cols + gc;
        const float o = o_at(r, c);
        W[off] = a.mode == 1 ? fmaf(a.decay, W[off], -a.step * o) : o;
      }
    }
  }
}

}  // namespace

void launch_prep(const EwTable& t, const PrepArgs& a, cudaStream_t s) {
  const long long blocks = (long long)a.count * a.tiles_r * a.tiles_c;
  ProfScope prof(PK_PREP, s);
  if (blocks > 0) launch_pdl(prep_kernel, dim3((unsigned)blocks), dim3(EW_THREADS), 0, s, false, t, a);
}

void launch_finalize(const EwTable& t, const FinalizeArgs& a, cudaStream_t s) {
  const int warps_per_block = 4;
  const int blocks = (a.count + warps_per_block - 1) / warps_per_block;
  ProfScope prof(PK_NORM, s);
  if (blocks > 0) launch_pdl(finalize_kernel, dim3(blocks), dim3(32 * warps_per_block), 0, s, false, t, a);
}

void launch_apply(const EwTable& t, const ApplyArgs& a, cudaStream_t s) {
  const long long blocks = (long long)a.count * a.tiles_r * a.tiles_c;
  ProfScope prof(PK_APPLY, s);
  if (blocks > 0) launch_pdl(apply_kernel, dim3((unsigned)blocks), dim3(EW_THREADS), 0, s, false, t, a);
}

}  // namespace mo
