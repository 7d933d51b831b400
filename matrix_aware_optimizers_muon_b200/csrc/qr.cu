// Kernels of the SOAP basis refresh other than the tensor-core products:
// factor scales, fp16 plane splits, column norms, the per-matrix pass
// control, the 128 x 128 diagonal Cholesky blocks and the row-block solves.
#include <cfloat>

#include "chol_block.cuh"
#include "profile.h"
#include "ptx.cuh"
#include "qr.cuh"
#include "runtime.h"

namespace mo {

namespace {

constexpr size_t A1K = 1024;
size_t a1k(size_t x) { return (x + A1K - 1) / A1K * A1K; }

__global__ void qr_init_kernel(const QrCtl c, int q) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= q) return;
  c.done[b] = 0;
  c.skip[b] = 0;
  c.fail[b] = 0;
  c.mode[b] = -1;
  c.next_shift[b] = 0;
  c.mult[b] = 1.f;
  c.floor[b] = QR_PLAIN_FLOOR;
  c.shift[b] = 0.f;
  c.minpiv[b] = 0x7f800000u;
  c.dev[b] = 0u;
  if (b == 0) {
    for (int p = 0; p < QR_MAX_PASSES; ++p) c.pass_done[p] = 0;
    *c.npass = 0;
  }
}

// One CTA per matrix: the largest diagonal entry, then a power-of-two scale
// that brings it below 2^13 (exponent clamped so that the scale is finite).
__global__ void __launch_bounds__(256) factor_scale_kernel(const FactorScaleArgs a, const QrCtl c) {
  __shared__ float red[8];
  const int b = blockIdx.x;
  const float* F = a.F[b];
  const float d = a.delta ? a.delta[b] : 0.f;
  float m = 0.f;
  for (int i = threadIdx.x; i < a.k; i += blockDim.x) m = fmaxf(m, F[(long long)i * a.k + i] + d);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    m = fmaxf(m, red[0]);
    float sc = 1.f;
    if (m > 0.f && m <= FLT_MAX) {
      int e = 0;
      frexpf(m, &e);                       // m < 2^e
      e = e < -100 ? -100 : (e > 100 ? 100 : e);
      sc = ldexpf(1.f, 13 - e);
    }
    c.fscale[b] = sc;
    c.fiscale[b] = 1.f / sc;
  }
}

__device__ __forceinline__ uint4 pack_half8(const float (&x)[8]) {
  uint4 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h = __floats2half2_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return u;
}

// Two fp16 planes (h, l) of 8 values already multiplied by the plane scale.
__device__ __forceinline__ void store_planes_h8(__half* d, long long plane_stride, const float (&xs)[8]) {
  const uint4 h = pack_half8(xs);
  float r[8];
  const __half* hh = reinterpret_cast<const __half*>(&h);
#pragma unroll
  for (int i = 0; i < 8; ++i) r[i] = xs[i] - __half2float(hh[i]);
  *reinterpret_cast<uint4*>(d) = h;
  *reinterpret_cast<uint4*>(d + plane_stride) = pack_half8(r);
}

// A uniform value in [-1, 1) from a 32-bit integer hash (the finaliser of
// MurmurHash3, Appleby) of the element's coordinates and a seed.
__device__ __forceinline__ float hash_uniform(unsigned b, unsigned r, unsigned c, unsigned seed) {
  unsigned h = (r * 0x9E3779B1u) ^ (c * 0x85EBCA77u) ^ (b * 0xC2B2AE3Du) ^ (seed * 0x27D4EB2Fu);
  h ^= h >> 16;
  h *= 0x85EBCA6Bu;
  h ^= h >> 13;
  h *= 0xC2B2AE35u;
  h ^= h >> 16;
  return (float)(h >> 8) * (2.0f / 16777216.0f) - 1.0f;
}

__device__ __forceinline__ void split16_row(const Split16Args& a, int b, int r, int c0, unsigned seed) {
  const bool rv = r < a.rows_valid;
  const float* src = a.src[b] + (long long)r * a.lds;
  float x[8];
  if (rv && c0 + 8 <= a.cols_valid) {
    const float4 u = *reinterpret_cast<const float4*>(src + c0);
    const float4 v = *reinterpret_cast<const float4*>(src + c0 + 4);
    x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
    x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = (rv && c0 + i < a.cols_valid) ? src[c0 + i] : 0.f;
  }
  const bool noisy = a.noise_on && a.noise_on[b];
  const float namp = noisy ? a.noise_amp * rsqrtf((float)a.cols_pad) : 0.f;
  bool pad[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = c0 + i;
    pad[i] = false;
    if (rv && c < a.cols_valid) {
      if (a.diag_add && r == c) x[i] += a.diag_add[b];
      if (a.col_scale) {
        const float s = a.col_scale[(size_t)b * a.cols_pad + c];
        x[i] = s == 0.f ? (r == c ? 1.f : 0.f) : x[i] * s;     // a zero column becomes e_c
      }
      if (noisy) x[i] = fmaf(namp, hash_uniform(b, r, c, seed), x[i]);
    } else {
      pad[i] = a.pad_identity && r == c;
      x[i] = pad[i] ? 1.f : 0.f;
    }
  }
  if (a.write_back) {
    float* w = a.write_back + (size_t)b * a.wb_stride + (long long)r * a.ldw + c0;
    reinterpret_cast<float4*>(w)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(w)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
  const float sc = a.mscale ? a.mscale[b] : a.cscale;
  const float pad_val = fminf(sc, 16384.f);      // a positive diagonal that fits fp16
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = pad[i] ? pad_val : x[i] * sc;
  store_planes_h8(a.dst + (size_t)b * a.mat_stride + (long long)r * a.ldd + c0, a.plane_stride, x);
}

__global__ void split16_kernel(const Split16Args a) {
  pdl_wait();
  pdl_trigger();
  if (a.gate && *a.gate >= a.gate_n) return;
  const int b = blockIdx.z;
  if (a.skip && a.skip[b]) return;
  const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (c0 >= a.cols_pad) return;
  const unsigned seed = a.seed_dev ? (unsigned)*a.seed_dev : a.noise_seed;
  for (int r = blockIdx.y; r < a.rows_pad; r += gridDim.y) split16_row(a, b, r, c0, seed);
}

// 32 columns x 8 row groups per CTA; the 8 partial sums of a column are
// added in a fixed order (bitwise reproducible).
__global__ void __launch_bounds__(256) colnorm2_kernel(const float* Y, long long ld, long long stride, int rows,
                                                       int cols, float* inv_d, const int* skip, const int* gate,
                                                       int gate_n) {
  __shared__ float part[8][33];
  pdl_wait();
  pdl_trigger();
  if (gate && *gate >= gate_n) return;
  const int b = blockIdx.y;
  if (skip && skip[b]) return;
  const int cx = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + cx;
  float s = 0.f;
  if (c < cols) {
    const float* y = Y + (size_t)b * stride + c;
#pragma unroll 4
    for (int r = g; r < rows; r += 8) {
      const float v = y[(long long)r * ld];
      s = fmaf(v, v, s);
    }
  }
  part[g][cx] = s;
  __syncthreads();
  if (g == 0 && c < cols) {
    float t = part[0][cx];
#pragma unroll
    for (int i = 1; i < 8; ++i) t += part[i][cx];
    inv_d[(size_t)b * cols + c] = t == 0.f ? 0.f : (isinf(t) ? __int_as_float(0x7fc00000) : 1.0f / sqrtf(t));
  }
}

// Partial Gram statistics: block g of matrix b covers rows [g rpb, (g+1) rpb).
__global__ void __launch_bounds__(256) qr_check_kernel(const float* C, long long ld, long long stride, int kp,
                                                       const QrCtl c, const int* gate, int gate_n) {
  __shared__ float red[8];
  pdl_wait();
  pdl_trigger();
  if (gate && *gate >= gate_n) return;
  const int b = blockIdx.y;
  if (c.done[b]) return;
  const int rpb = (kp + QR_CHECK_BLOCKS - 1) / QR_CHECK_BLOCKS;
  const int r0 = blockIdx.x * rpb;
  const int r1 = min(kp, r0 + rpb);
  const float* Cb = C + (size_t)b * stride;
  float dev = 0.f, sq = 0.f;
  bool nan = false;
  const int q4 = kp / 4;
  for (long long e = threadIdx.x; e < (long long)(r1 - r0) * q4; e += blockDim.x) {
    const int r = r0 + (int)(e / q4);
    const int c4 = (int)(e - (long long)(r - r0) * q4) * 4;
    const float4 v = *reinterpret_cast<const float4*>(Cb + (long long)r * ld + c4);
    const float x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float dv = fabsf(x[i] - (r == c4 + i ? 1.f : 0.f));
      if (dv != dv) nan = true;
      dev = fmaxf(dev, dv);
      sq = fmaf(x[i], x[i], sq);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, o));
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  nan = __any_sync(0xffffffffu, nan);
  if ((threadIdx.x & 31) == 0) {
    red[threadIdx.x >> 5] = sq;
    atomicMax(c.dev + b, nan ? 0x7fc00000u : __float_as_uint(dev));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int w = 1; w < 8; ++w) t += red[w];
    c.part[(size_t)b * QR_CHECK_BLOCKS + blockIdx.x] = t;
  }
}

// One CTA per matrix: the outcome of the previous attempt, the check of this
// pass's Gram, the mode of this pass, and the shift of the diagonal.
__global__ void __launch_bounds__(256) qr_decide_kernel(float* C, long long ld, long long stride, int kp,
                                                        const QrCtl c, int pass_host, const int* pass_dev) {
  __shared__ float s_shift;
  pdl_wait();
  pdl_trigger();
  const int pass = pass_dev ? *pass_dev : pass_host;
  const int b = blockIdx.x;
  if (threadIdx.x == 0) {
    float sh = 0.f;
    if (c.done[b]) {
      c.skip[b] = 1;
      c.mode[b] = -1;
    } else {
      const int prev = c.mode[b];
      if (prev >= 0) {
        if (c.fail[b]) {
          c.next_shift[b] = 1;
          if (prev == 1) c.mult[b] = fminf(c.mult[b] * 10.f, 1e6f);
        } else if (prev == 1) {
          c.next_shift[b] = __uint_as_float(c.minpiv[b]) < 10.f * c.shift[b] ? 1 : 0;
        } else {
          c.next_shift[b] = 0;
        }
      }
      const unsigned dbits = c.dev[b];
      if (dbits <= __float_as_uint(QR_TAU_DONE)) {
        c.done[b] = 1;
        c.skip[b] = 1;
        c.mode[b] = -1;
      } else {
        float sq = 0.f;
        for (int g = 0; g < QR_CHECK_BLOCKS; ++g) sq += c.part[(size_t)b * QR_CHECK_BLOCKS + g];
        const int shifted = c.next_shift[b];
        // the shift stays below 10 (of the unit diagonal) so that the
        // factor's entries fit the fp16 planes
        sh = shifted ? fminf(QR_SHIFT_REL * sqrtf(sq) * c.mult[b], 10.f) : 0.f;
        c.mode[b] = shifted;
        c.shift[b] = sh;
        c.floor[b] = shifted ? 0.f : QR_PLAIN_FLOOR;
        c.fail[b] = 0;
        c.skip[b] = 0;
        c.minpiv[b] = 0x7f800000u;
      }
      c.dev[b] = 0u;                        // the next pass's check accumulates from zero
    }
    if (c.done[b]) atomicAdd(c.pass_done + pass, 1);
    s_shift = sh;
  }
  __syncthreads();
  const float sh = s_shift;
  if (sh != 0.f) {
    float* Cb = C + (size_t)b * stride;
    for (int i = threadIdx.x; i < kp; i += blockDim.x) Cb[(long long)i * ld + i] += sh;
  }
}

// One CTA (256 threads) per matrix: Cholesky of the diagonal block with the
// matrix's pivot floor, then the inverse of its lower factor.
__global__ void __launch_bounds__(256) qr_chol_kernel(const float* C, long long ld, long long stride, int k0,
                                                      float* Dinv, const QrCtl c, const int* gate,
                                                      const int* gate_idx, int gate_n) {
  pdl_wait();
  pdl_trigger();
  if (gate && gate[gate_idx ? *gate_idx : 0] >= gate_n) return;
  const int b = blockIdx.x;
  if (c.skip[b]) return;
  extern __shared__ float sm[];
  float* A = sm;                          // [128][129]
  float* X = A + CB * CB_LD;              // [128][129]
  float* T = X + CB * CB_LD;              // [32][97]
  float* inv_diag = T + 32 * CB_T_LD;     // [128]
  __shared__ int bad;
  __shared__ float mp;
  const int tid = threadIdx.x;
  const float* src = C + (size_t)b * stride + (long long)k0 * ld + k0;
  // the 128 x 128 block as 4096 float4 loads, 16 per thread, all in flight
  // before the first shared-memory store (rows of C are 16-byte aligned)
  {
    float4 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = tid + 256 * i, r = e >> 5, c4 = (e & 31) * 4;
      v[i] = *reinterpret_cast<const float4*>(src + (long long)r * ld + c4);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = tid + 256 * i, r = e >> 5, c4 = (e & 31) * 4;
      float* a = A + r * CB_LD + c4;
      a[0] = v[i].x; a[1] = v[i].y; a[2] = v[i].z; a[3] = v[i].w;
    }
  }
  if (tid == 0) {
    bad = 0;
    mp = __int_as_float(0x7f800000);
  }
  __syncthreads();
  chol128_factor(A, inv_diag, &bad, c.floor[b], &mp);
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      c.fail[b] = 1;
      c.skip[b] = 1;
    }
    return;
  }
  if (tid == 0 && mp > 0.f) atomicMin(c.minpiv + b, __float_as_uint(mp));
  chol128_inverse(A, inv_diag, X, T);
  // the inverse transposed: DinvT[p][c] = Dinv[c][p] (nonzero for c >= p), so
  // that the panel kernel stages it with straight float4 copies
  float* dst = Dinv + (size_t)b * CB * CB;
#pragma unroll 4
  for (int i = 0; i < 16; ++i) {
    const int e = tid + 256 * i, pr = e >> 5, c4 = (e & 31) * 4;
    const float* x = X + c4 * CB_LD + pr;
    reinterpret_cast<float4*>(dst)[e] =
        make_float4(c4 >= pr ? x[0] : 0.f, c4 + 1 >= pr ? x[CB_LD] : 0.f, c4 + 2 >= pr ? x[2 * CB_LD] : 0.f,
                    c4 + 3 >= pr ? x[3 * CB_LD] : 0.f);
  }
}

// out = in * Dinv^T for 128 rows x 128 columns per CTA (256 threads), from
// transposed shared copies of the rows and of Dinv (Dinv lower: p <= c; its
// global copy is stored transposed).  Column group g (8 columns) needs p <=
// 8 g + 7 only; lane l of warp w computes rows 4 l .. 4 l + 3 for the groups
// w and 15 - w in turn, so every warp runs the same 136 steps of the p loop
// with all lanes on the same bound.
constexpr int PANEL_ROWS = 128;
constexpr int PANEL_LDD = QR_B + 4;           // Dt[p][c] = Dinv[c][p]
constexpr int PANEL_LDR = PANEL_ROWS + 4;     // Rt[p][r] = in[r0 + r][p]
constexpr int PANEL_SMEM = (QR_B * PANEL_LDD + QR_B * PANEL_LDR) * 4;

__global__ void __launch_bounds__(256, 1) qr_panel_kernel(const PanelArgs a) {
  pdl_wait();
  pdl_trigger();
  if (a.gate && a.gate[a.gate_idx ? *a.gate_idx : 0] >= a.q) return;
  const int b = blockIdx.y;
  if (a.skip[b]) return;
  extern __shared__ float sm[];
  float* Dt = sm;
  float* Rt = sm + QR_B * PANEL_LDD;
  const int r0 = a.r0 + blockIdx.x * PANEL_ROWS;
  const long long col0 = (long long)a.j * QR_B;
  const float* dinv = a.Dinv + (size_t)b * QR_B * QR_B;
  float* cy = a.CY + (size_t)b * a.mat_stride + col0;
  // DinvT (4096 float4) and the 128 x 128 rows (4096 float4) in two halves
  // of 8 + 8 loads per thread, each half's loads issued before its
  // shared-memory stores.  The rows are read with the lanes of a warp on
  // consecutive rows (same 16 bytes of each), so that their transposing
  // stores Rt[p][r] hit consecutive banks.
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    float4 d[8], y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = reinterpret_cast<const float4*>(dinv)[threadIdx.x + 256 * (8 * half + i)];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = threadIdx.x + 256 * (8 * half + i), r = e & (PANEL_ROWS - 1), p4 = (e >> 7) * 4;
      y[i] = (r0 + r < a.r1) ? *reinterpret_cast<const float4*>(cy + (long long)(r0 + r) * a.ld + p4)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = threadIdx.x + 256 * (8 * half + i), pr = e >> 5, c4 = (e & 31) * 4;     // DinvT[pr][c4 ..]
      *reinterpret_cast<float4*>(&Dt[pr * PANEL_LDD + c4]) = d[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = threadIdx.x + 256 * (8 * half + i), r = e & (PANEL_ROWS - 1), p4 = (e >> 7) * 4;
      Rt[(p4 + 0) * PANEL_LDR + r] = y[i].x;
      Rt[(p4 + 1) * PANEL_LDR + r] = y[i].y;
      Rt[(p4 + 2) * PANEL_LDR + r] = y[i].z;
      Rt[(p4 + 3) * PANEL_LDR + r] = y[i].w;
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __half* lq = a.LQ + (size_t)b * a.mat_stride + col0;
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    const int g = h == 0 ? warp : 15 - warp;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[i][k] = 0.f;
    const int pmax = 8 * g + 7;
#pragma unroll 2
    for (int p = 0; p <= pmax; ++p) {
      const float4 rv = *reinterpret_cast<const float4*>(&Rt[p * PANEL_LDR + 4 * lane]);
      const float4 d0 = *reinterpret_cast<const float4*>(&Dt[p * PANEL_LDD + 8 * g]);
      const float4 d1 = *reinterpret_cast<const float4*>(&Dt[p * PANEL_LDD + 8 * g + 4]);
      const float rr[4] = {rv.x, rv.y, rv.z, rv.w};
      const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[i][k] = fmaf(rr[i], dd[k], acc[i][k]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = r0 + 4 * lane + i;
      if (row >= a.r1) continue;
      const int c0 = 8 * g;
      if (row >= a.f32_from) {
        float* o = cy + (long long)row * a.ld + c0;
        reinterpret_cast<float4*>(o)[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        reinterpret_cast<float4*>(o)[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
      }
      float xs[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) xs[k] = acc[i][k] * QR_PLANE_SCALE;
      store_planes_h8(lq + (long long)row * a.ld + c0, a.plane_stride, xs);
    }
  }
}

__global__ void qr_loop_kernel(const QrCtl c, int q, cudaGraphConditionalHandle h) {
  pdl_wait();
  const int p = *c.npass;
  const bool more = c.pass_done[p] < q && p + 1 < QR_MAX_PASSES;
  *c.npass = p + 1;
  cudaGraphSetConditional(h, more ? 1u : 0u);
}

__global__ void qr_finish_flags_kernel(const QrCtl c, const FlagTable f, int q) {
  const int b = threadIdx.x;
  if (b < q && !c.done[b] && f.f[b] != nullptr) *f.f[b] = 1;
}

struct Fallback {
  const float* q[SOAP_MAXB];
};

// Row r of matrix b (one CTA per row): the previous basis, identity-padded.
__global__ void qr_fallback_kernel(const QrCtl c, float* Y, long long ld, long long stride, int k, int kp,
                                   const Fallback f) {
  const int b = blockIdx.y;
  if (c.done[b]) return;
  const int r = blockIdx.x;
  float* y = Y + (size_t)b * stride + (long long)r * ld;
  const float* src = f.q[b] + (long long)r * k;
  for (int col = threadIdx.x; col < kp; col += blockDim.x)
    y[col] = (r < k && col < k) ? src[col] : (r == col ? 1.f : 0.f);
}

}  // namespace

size_t qr_ctl_bytes(int q) {
  // eleven arrays of q words, the partial sums, two scale arrays
  return 13 * a1k((size_t)q * 4) + a1k((size_t)q * QR_CHECK_BLOCKS * 4);
}

QrCtl qr_ctl_at(char* base, int q) {
  const size_t w = a1k((size_t)q * 4);
  QrCtl c;
  c.done = reinterpret_cast<int*>(base + 0 * w);
  c.skip = reinterpret_cast<int*>(base + 1 * w);
  c.fail = reinterpret_cast<int*>(base + 2 * w);
  c.mode = reinterpret_cast<int*>(base + 3 * w);
  c.next_shift = reinterpret_cast<int*>(base + 4 * w);
  c.mult = reinterpret_cast<float*>(base + 5 * w);
  c.floor = reinterpret_cast<float*>(base + 6 * w);
  c.shift = reinterpret_cast<float*>(base + 7 * w);
  c.minpiv = reinterpret_cast<unsigned*>(base + 8 * w);
  c.dev = reinterpret_cast<unsigned*>(base + 9 * w);
  c.fscale = reinterpret_cast<float*>(base + 10 * w);
  c.fiscale = reinterpret_cast<float*>(base + 11 * w);
  c.pass_done = reinterpret_cast<int*>(base + 12 * w);     // QR_MAX_PASSES + 1 <= 256 words
  c.npass = c.pass_done + QR_MAX_PASSES;
  c.part = reinterpret_cast<float*>(base + 13 * w);
  return c;
}

void launch_qr_init(const QrCtl& c, int q, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  qr_init_kernel<<<(q + 127) / 128, 128, 0, s>>>(c, q);
}

void launch_factor_scale(const FactorScaleArgs& a, const QrCtl& c, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  factor_scale_kernel<<<a.count, 256, 0, s>>>(a, c);
}

void launch_split16(const Split16Args& a, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  const int per_block = 256 * 8;
  // up to 256 row groups per matrix, each CTA looping over its rows: a
  // gated-off launch then has few CTAs to retire
  const int ry = a.rows_pad < 256 ? a.rows_pad : 256;
  dim3 grid((a.cols_pad + per_block - 1) / per_block, ry, a.count);
  (void)launch_pdl(split16_kernel, grid, dim3(256), 0, s, false, a);
}

void launch_colnorm2(const float* Y, long long ld, long long mat_stride, int count, int rows, int cols,
                     float* inv_d, const int* skip, const int* gate, int gate_n, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  dim3 grid((cols + 31) / 32, count);
  (void)launch_pdl(colnorm2_kernel, grid, dim3(256), 0, s, false, Y, ld, mat_stride, rows, cols, inv_d, skip, gate,
                   gate_n);
}

void launch_qr_control(const float* C, long long ld, long long mat_stride, int q, int kp, const QrCtl& c,
                       int pass, const int* pass_dev, const int* gate, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  (void)launch_pdl(qr_check_kernel, dim3(QR_CHECK_BLOCKS, q), dim3(256), 0, s, false, C, ld, mat_stride, kp, c, gate,
                   q);
  (void)launch_pdl(qr_decide_kernel, dim3(q), dim3(256), 0, s, false, const_cast<float*>(C), ld, mat_stride, kp, c,
                   pass, pass_dev);
}

void launch_qr_chol(const float* C, long long ld, long long mat_stride, int q, int j, float* Dinv,
                    const QrCtl& c, const int* gate, const int* gate_idx, cudaStream_t s) {
  ProfScope prof(PK_QR_CHOL, s);
  const int smem = (2 * CB * CB_LD + 32 * CB_T_LD + CB) * 4;
  (void)ensure_smem_attr(reinterpret_cast<const void*>(qr_chol_kernel), smem);
  (void)launch_pdl(qr_chol_kernel, dim3(q), dim3(256), (size_t)smem, s, false, C, ld, mat_stride, j * QR_B, Dinv, c,
                   gate, gate_idx, q);
}

void launch_qr_panel(const PanelArgs& a, cudaStream_t s) {
  if (a.r1 <= a.r0) return;
  ProfScope prof(PK_QR_ROWBLK, s);
  (void)ensure_smem_attr(reinterpret_cast<const void*>(qr_panel_kernel), PANEL_SMEM);
  dim3 grid((a.r1 - a.r0 + PANEL_ROWS - 1) / PANEL_ROWS, a.q);
  (void)launch_pdl(qr_panel_kernel, grid, dim3(256), (size_t)PANEL_SMEM, s, false, a);
}

void launch_qr_loop(const QrCtl& c, int q, cudaGraphConditionalHandle h, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  (void)launch_pdl(qr_loop_kernel, dim3(1), dim3(1), 0, s, false, c, q, h);
}

void launch_qr_finish(const QrCtl& c, const FlagTable& flags, int q, float* Y, long long ld,
                      long long mat_stride, int k, int kp, const float* const* Qold, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  qr_finish_flags_kernel<<<1, SOAP_MAXB, 0, s>>>(c, flags, q);
  Fallback f;
  for (int b = 0; b < q && b < SOAP_MAXB; ++b) f.q[b] = Qold[b];
  qr_fallback_kernel<<<dim3(kp, q), 256, 0, s>>>(c, Y, ld, mat_stride, k, kp, f);
}

}  // namespace mo
