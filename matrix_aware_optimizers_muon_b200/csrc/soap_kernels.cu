// Elementwise, splitting and small dense kernels of the SOAP path.
#include "profile.h"
#include "soap_kernels.cuh"
#include "runtime.h"
#include "chol_block.cuh"

namespace mo {

namespace {

constexpr int EWT = 256;

struct PtrUpload {
  int n;
  const void* p[SOAP_MAXB];
};

__global__ void upload_ptrs_kernel(void** dst, const PtrUpload u) {
  const int i = threadIdx.x + blockIdx.x * blockDim.x;
  if (i < u.n) dst[i] = const_cast<void*>(u.p[i]);
}

__device__ __forceinline__ uint2 pack4(float a, float b, float c, float d) {
  const __nv_bfloat162 x = __floats2bfloat162_rn(a, b), y = __floats2bfloat162_rn(c, d);
  uint2 v;
  v.x = *reinterpret_cast<const uint32_t*>(&x);
  v.y = *reinterpret_cast<const uint32_t*>(&y);
  return v;
}

__device__ __forceinline__ float4 widen4(uint2 v) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// Two bf16 planes (h, l) of 4 values at plane[0] / plane[stride].
__device__ __forceinline__ void store_planes4(__nv_bfloat16* d, long long stride, float4 x) {
  const uint2 h = pack4(x.x, x.y, x.z, x.w);
  const float4 hf = widen4(h);
  const uint2 l = pack4(x.x - hf.x, x.y - hf.y, x.z - hf.z, x.w - hf.w);
  *reinterpret_cast<uint2*>(d) = h;
  *reinterpret_cast<uint2*>(d + stride) = l;
}

__global__ void soap_prep_kernel(const SoapPrepArgs a) {
  const int j = blockIdx.y;
  const float* __restrict__ G = a.G[j];
  float* __restrict__ M = a.M[j];
  const long long cols4 = a.cols / 4;
  const long long n4 = a.rows * cols4;
  const float c = 1.0f - a.beta1;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / cols4, q = i - r * cols4;
    const float4 g = __ldcs(reinterpret_cast<const float4*>(G) + i);
    float4 m = reinterpret_cast<const float4*>(M)[i];
    const size_t off = (size_t)j * a.mat_stride + (size_t)r * a.ldp + 4 * q;
    if (a.muon) {
      // Muon momentum (sum form) and the Nesterov numerator
      m.x = fmaf(a.beta1, m.x, g.x);
      m.y = fmaf(a.beta1, m.y, g.y);
      m.z = fmaf(a.beta1, m.z, g.z);
      m.w = fmaf(a.beta1, m.w, g.w);
      reinterpret_cast<float4*>(M)[i] = m;
      float4 nv = m;
      if (a.nesterov)
        nv = make_float4(fmaf(a.beta1, m.x, g.x), fmaf(a.beta1, m.y, g.y), fmaf(a.beta1, m.z, g.z),
                         fmaf(a.beta1, m.w, g.w));
      store_planes4(a.Gp + off, a.plane_stride, g);
      store_planes4(a.Mp + off, a.plane_stride, nv);
      continue;
    }
    m.x = fmaf(a.beta1, m.x, c * g.x);
    m.y = fmaf(a.beta1, m.y, c * g.y);
    m.z = fmaf(a.beta1, m.z, c * g.z);
    m.w = fmaf(a.beta1, m.w, c * g.w);
    reinterpret_cast<float4*>(M)[i] = m;
    store_planes4(a.Gp + off, a.plane_stride, g);
    store_planes4(a.Mp + off, a.plane_stride, m);
  }
}

// x = h + m + l with h = bf16(x), m = bf16(x - h), l = bf16(x - h - m); the
// differences are exact in fp32.
__device__ __forceinline__ void split3(float x, __nv_bfloat16& h, __nv_bfloat16& m, __nv_bfloat16& l) {
  h = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(h);
  m = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(m);
  l = __float2bfloat16_rn(r2);
}

__global__ void split_kernel(const SplitArgs a) {
  const int b = blockIdx.z;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int r = blockIdx.y;
  if (c >= a.cols_pad || r >= a.rows_pad) return;
  float x;
  if (r < a.rows_valid && c < a.cols_valid) {
    x = a.src[b][(long long)r * a.lds + c];
    if (a.diag_add && r == c) x += a.diag_add[b];
    if (a.col_scale) x *= a.col_scale[(size_t)b * a.cols_pad + c];
  } else {
    x = (a.pad_identity && r == c) ? 1.0f : 0.0f;
  }
  if (a.write_back) a.write_back[(size_t)b * a.wb_stride + (long long)r * a.ldw + c] = x;
  __nv_bfloat16* d = a.dst + (size_t)b * a.mat_stride + (long long)r * a.ldd + c;
  if (a.nplanes == 1) {
    *d = __float2bfloat16_rn(x);
  } else if (a.nplanes == 2) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    d[0] = h;
    d[a.plane_stride] = __float2bfloat16_rn(x - __bfloat162float(h));
  } else {
    __nv_bfloat16 h, m, l;
    split3(x, h, m, l);
    d[0] = h;
    d[a.plane_stride] = m;
    d[2 * a.plane_stride] = l;
  }
}

__global__ void __launch_bounds__(256) damping_kernel(const DampArgs a) {
  __shared__ float part[256];
  const int b = blockIdx.x;
  const float* F = a.F[b];
  float t = 0.f;
  for (int i = threadIdx.x; i < a.k; i += 256) t += F[(long long)i * a.k + i];
  part[threadIdx.x] = t;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) a.delta[b] = part[0] != 0.f ? a.rho * part[0] : 1.0f;
}

// Largest |C - I| entry per matrix, as the bit pattern of a non-negative
// float (ordered like the values, so atomicMax on ints is exact); NaN
// compares above everything.
__global__ void __launch_bounds__(256) identity_dev_kernel(const float* C, long long ld, long long stride, int k,
                                                           int* dev) {
  const int b = blockIdx.y;
  const float* c = C + (size_t)b * stride;
  const long long total = (long long)k * k;
  float m = 0.f;
  bool nan = false;
  for (long long e = blockIdx.x * 256LL + threadIdx.x; e < total; e += (long long)gridDim.x * 256) {
    const long long i = e / k, j = e - i * k;
    const float d = fabsf(c[i * ld + j] - (i == j ? 1.0f : 0.0f));
    if (d != d) nan = true;
    else m = fmaxf(m, d);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  nan = __any_sync(0xffffffffu, nan);
  if ((threadIdx.x & 31) == 0) atomicMax(dev + b, nan ? 0x7fc00000 : __float_as_int(m));
}

__global__ void identity_skip_kernel(const int* dev, int count, float tol, int* skip) {
  const int b = threadIdx.x;
  if (b < count) skip[b] = dev[b] <= __float_as_int(tol) ? 1 : 0;
}

__global__ void colnorm_kernel(const float* Y, long long ld, long long stride, int rows, int cols,
                               float* inv_d) {
  const int b = blockIdx.y;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const float* y = Y + (size_t)b * stride + c;
  float s = 0.f;
  for (int r = 0; r < rows; ++r) {
    const float v = y[(long long)r * ld];
    s = fmaf(v, v, s);
  }
  inv_d[(size_t)b * cols + c] = 1.0f / sqrtf(s);
}

__global__ void shift_diag_kernel(float* C, long long ld, long long stride, int n, float shift) {
  const int b = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) C[(size_t)b * stride + (long long)i * ld + i] += shift;
}

// One CTA (256 threads) per matrix: Cholesky of the 128 x 128 diagonal
// block at (k0, k0) and the inverse of its lower factor (chol_block.cuh).
__global__ void __launch_bounds__(256) chol_diag_kernel(const float* C, long long ld, long long stride,
                                                        int k0, float* Dinv, const FlagTable flags,
                                                        const int* skip) {
  if (skip && skip[blockIdx.x]) return;
  extern __shared__ float sm[];
  float* A = sm;                          // [128][129]
  float* X = A + CB * CB_LD;              // [128][129]
  float* T = X + CB * CB_LD;              // [32][97]
  float* inv_diag = T + 32 * CB_T_LD;     // [128]
  __shared__ int bad;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const float* src = C + (size_t)b * stride + (long long)k0 * ld + k0;
  for (int e = tid; e < CB * CB; e += blockDim.x) {
    const int r = e >> 7, c = e & 127;
    A[r * CB_LD + c] = src[(long long)r * ld + c];
  }
  if (tid == 0) bad = 0;
  __syncthreads();
  chol128_factor(A, inv_diag, &bad);
  chol128_inverse(A, inv_diag, X, T);
  const float nanv = __int_as_float(0x7fc00000);
  const bool fail = bad != 0;
  float* dst = Dinv + (size_t)b * CB * CB;
  for (int e = tid; e < CB * CB; e += blockDim.x) {
    const int r = e >> 7, c = e & 127;
    dst[e] = fail ? nanv : (c <= r ? X[r * CB_LD + c] : 0.f);
  }
  if (tid == 0 && fail && flags.f[b] != nullptr) *flags.f[b] = 1;
}

// out[r][c] = sum_{p <= c} in[r][p] Dinv[c][p]   (in * Dinv^T, Dinv lower).
// 64 rows per CTA, 256 threads; thread (ty, tx) computes rows 4 ty .. +3 and
// columns 8 tx .. +7 from transposed shared copies of the rows and of Dinv.
__global__ void __launch_bounds__(256) rowblock_kernel(const RowBlockArgs a) {
  if (a.skip && a.skip[blockIdx.y]) return;
  extern __shared__ float sm[];
  constexpr int LDD = QR_B + 4;        // Dt[p][c] = Dinv[c][p]
  constexpr int LDR = 64 + 4;          // Rt[p][r] = in[r0 + r][p]
  float* Dt = sm;
  float* Rt = sm + QR_B * LDD;
  const int b = blockIdx.y;
  const int r0 = blockIdx.x * 64;
  const float* dinv = a.Dinv + (size_t)b * QR_B * QR_B;
  for (int e = threadIdx.x; e < QR_B * QR_B; e += blockDim.x) {
    const int c = e >> 7, p = e & 127;
    Dt[p * LDD + c] = dinv[e];
  }
  const float* in = a.in + (size_t)b * a.in_stride;
  for (int e = threadIdx.x; e < 64 * QR_B; e += blockDim.x) {
    const int r = e >> 7, p = e & 127;
    Rt[p * LDR + r] = (r0 + r < a.rows) ? in[(long long)(r0 + r) * a.ld_in + p] : 0.f;
  }
  __syncthreads();
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[i][k] = 0.f;
  const int pmax = 8 * tx + 7;         // Dinv is lower: p <= c
  for (int p = 0; p <= pmax; ++p) {
    const float4 rv = *reinterpret_cast<const float4*>(&Rt[p * LDR + 4 * ty]);
    const float4 d0 = *reinterpret_cast<const float4*>(&Dt[p * LDD + 8 * tx]);
    const float4 d1 = *reinterpret_cast<const float4*>(&Dt[p * LDD + 8 * tx + 4]);
    const float rr[4] = {rv.x, rv.y, rv.z, rv.w};
    const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[i][k] = fmaf(rr[i], dd[k], acc[i][k]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long row = r0 + 4 * ty + i;
    if (row >= a.rows) continue;
    const int c0 = 8 * tx;
    if (a.out) {
      float* o = a.out + (size_t)b * a.out_stride + row * a.ld_out + c0;
      reinterpret_cast<float4*>(o)[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      reinterpret_cast<float4*>(o)[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
    }
    if (a.planes) {
      __nv_bfloat16* d = a.planes + (size_t)b * a.mat_stride + row * QR_B + c0;
      union Pack { __nv_bfloat16 h[8]; uint4 u; } hv, mv, lv;
#pragma unroll
      for (int k = 0; k < 8; ++k) split3(acc[i][k], hv.h[k], mv.h[k], lv.h[k]);
      *reinterpret_cast<uint4*>(d) = hv.u;
      *reinterpret_cast<uint4*>(d + a.plane_stride) = mv.u;
      *reinterpret_cast<uint4*>(d + 2 * a.plane_stride) = lv.u;
    }
  }
}

__global__ void copy_out_kernel(const CopyOutArgs a) {
  const int b = blockIdx.z;
  const int r = blockIdx.y;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < a.k) a.dst[b][(long long)r * a.k + c] = a.Y[(size_t)b * a.mat_stride + (long long)r * a.ld + c];
}

__global__ void adam_identity_kernel(const AdamIdArgs a) {
  const int j = blockIdx.y;
  const float* __restrict__ G = a.G[j];
  const float* __restrict__ M = a.M[j];
  float* __restrict__ V = a.V[j];
  float* __restrict__ W = a.W[j];
  const long long n4 = a.elems / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 g = __ldcs(reinterpret_cast<const float4*>(G) + i);
    const float4 m = __ldcs(reinterpret_cast<const float4*>(M) + i);
    float4 v = reinterpret_cast<const float4*>(V)[i];
    const float c = 1.0f - a.beta2;
    if (a.muon) {
      // SOAP-Muon with identity bases: P = N / (sqrt(V / bc2) + eps)
      float4 x = m;
      if (a.nesterov)
        x = make_float4(fmaf(a.mu, m.x, g.x), fmaf(a.mu, m.y, g.y), fmaf(a.mu, m.z, g.z), fmaf(a.mu, m.w, g.w));
      float4 pv;
#define MO_PRE(X)                                                               \
      v.X = fmaf(a.beta2, v.X, c * g.X * g.X);                                  \
      pv.X = (x.X * a.ibc1) / (sqrtf(v.X * a.ibc2) + a.eps);
      MO_PRE(x) MO_PRE(y) MO_PRE(z) MO_PRE(w)
#undef MO_PRE
      reinterpret_cast<float4*>(V)[i] = v;
      reinterpret_cast<float4*>(a.P[j])[i] = pv;
      continue;
    }
    float4 w = reinterpret_cast<const float4*>(W)[i];
#define MO_ADAM(X)                                                              \
    v.X = fmaf(a.beta2, v.X, c * g.X * g.X);                                    \
    w.X = fmaf(a.decay, w.X, -a.lr * ((m.X * a.ibc1) / (sqrtf(v.X * a.ibc2) + a.eps)));
    MO_ADAM(x) MO_ADAM(y) MO_ADAM(z) MO_ADAM(w)
#undef MO_ADAM
    reinterpret_cast<float4*>(V)[i] = v;
    reinterpret_cast<float4*>(W)[i] = w;
  }
}

__global__ void set_flags_kernel(const FlagTable f, int count, int32_t value) {
  const int i = threadIdx.x;
  if (i < count && f.f[i] != nullptr) *f.f[i] = value;
}

int ew_blocks(long long n4) {
  long long b = (n4 + EWT - 1) / EWT;
  return (int)(b < 4096 ? (b > 0 ? b : 1) : 4096);
}

}  // namespace

void launch_upload_ptrs(void** dst, const void* const* src, int n, cudaStream_t s) {
  PtrUpload u;
  u.n = n;
  for (int i = 0; i < n && i < SOAP_MAXB; ++i) u.p[i] = src[i];
  ProfScope prof(PK_TABLES, s);
  upload_ptrs_kernel<<<1, SOAP_MAXB, 0, s>>>(dst, u);
}

void launch_soap_prep(const SoapPrepArgs& a, cudaStream_t s) {
  ProfScope prof(PK_SOAP_EW, s);
  dim3 grid(ew_blocks(a.rows * a.cols / 16 + 1), a.count);
  soap_prep_kernel<<<grid, EWT, 0, s>>>(a);
}

void launch_split(const SplitArgs& a, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  dim3 grid((a.cols_pad + 255) / 256, a.rows_pad, a.count);
  split_kernel<<<grid, 256, 0, s>>>(a);
}

void launch_damping(const DampArgs& a, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  damping_kernel<<<a.count, 256, 0, s>>>(a);
}

void launch_identity_check(const float* C, long long ld, long long mat_stride, int count, int k, float tol,
                           int* dev, int* skip, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  cudaMemsetAsync(dev, 0, sizeof(int) * count, s);
  const long long total = (long long)k * k;
  long long blocks = (total + 256 * 16 - 1) / (256 * 16);
  dim3 grid((unsigned)(blocks < 512 ? blocks : 512), count);
  identity_dev_kernel<<<grid, 256, 0, s>>>(C, ld, mat_stride, k, dev);
  identity_skip_kernel<<<1, SOAP_MAXB, 0, s>>>(dev, count, tol, skip);
}

void launch_colnorm(const float* Y, long long ld, long long mat_stride, int count, int rows, int cols,
                    float* inv_d, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  dim3 grid((cols + 127) / 128, count);
  colnorm_kernel<<<grid, 128, 0, s>>>(Y, ld, mat_stride, rows, cols, inv_d);
}

void launch_shift_diag(float* C, long long ld, long long mat_stride, int count, int n, float shift,
                       cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  dim3 grid((n + 255) / 256, count);
  shift_diag_kernel<<<grid, 256, 0, s>>>(C, ld, mat_stride, n, shift);
}

void launch_chol_diag(const float* C, long long ld, long long mat_stride, int count, int k0,
                      float* Dinv, const FlagTable& flags, cudaStream_t s, const int* skip) {
  ProfScope prof(PK_QR_CHOL, s);
  const int smem = (2 * CB * CB_LD + 32 * CB_T_LD + CB) * 4;
  // a refused attribute makes the launch below fail; the caller's
  // cudaGetLastError() reports it
  (void)ensure_smem_attr(reinterpret_cast<const void*>(chol_diag_kernel), smem);
  chol_diag_kernel<<<count, 256, smem, s>>>(C, ld, mat_stride, k0, Dinv, flags, skip);
}

void launch_rowblock_dinv(const RowBlockArgs& a, cudaStream_t s) {
  ProfScope prof(PK_QR_ROWBLK, s);
  const int smem = (QR_B * (QR_B + 4) + QR_B * (64 + 4)) * 4;
  (void)ensure_smem_attr(reinterpret_cast<const void*>(rowblock_kernel), smem);
  dim3 grid((a.rows + 63) / 64, a.count);
  rowblock_kernel<<<grid, 256, smem, s>>>(a);
}

void launch_copy_out(const CopyOutArgs& a, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  dim3 grid((a.k + 255) / 256, a.k, a.count);
  copy_out_kernel<<<grid, 256, 0, s>>>(a);
}

void launch_adam_identity(const AdamIdArgs& a, cudaStream_t s) {
  ProfScope prof(PK_SOAP_EW, s);
  dim3 grid(ew_blocks(a.elems / 4 / 4 + 1), a.count);
  adam_identity_kernel<<<grid, EWT, 0, s>>>(a);
}

void launch_set_flags(const FlagTable& flags, int count, int32_t value, cudaStream_t s) {
  ProfScope prof(PK_SOAP_EW, s);
  set_flags_kernel<<<1, SOAP_MAXB, 0, s>>>(flags, count, value);
}

}  // namespace mo
