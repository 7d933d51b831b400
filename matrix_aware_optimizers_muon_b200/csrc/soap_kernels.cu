// Elementwise, splitting and small dense kernels of the SOAP path.
#include "profile.h"
#include "soap_kernels.cuh"

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
    m.x = fmaf(a.beta1, m.x, c * g.x);
    m.y = fmaf(a.beta1, m.y, c * g.y);
    m.z = fmaf(a.beta1, m.z, c * g.z);
    m.w = fmaf(a.beta1, m.w, c * g.w);
    reinterpret_cast<float4*>(M)[i] = m;
    const size_t off = (size_t)j * a.mat_stride + (size_t)r * a.ldp + 4 * q;
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

// One CTA (1024 threads) per matrix: Cholesky of a 128 x 128 block in shared
// memory, then the inverse of the lower factor, 8 threads per column.
__global__ void __launch_bounds__(1024) chol_diag_kernel(const float* C, long long ld, long long stride,
                                                         int k0, float* Dinv, const FlagTable flags) {
  extern __shared__ float sm[];
  float* A = sm;                      // [128][129]
  float* X = sm + QR_B * (QR_B + 1);  // [128][129]
  constexpr int LDS = QR_B + 1;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const float* src = C + (size_t)b * stride + (long long)k0 * ld + k0;
  for (int e = tid; e < QR_B * QR_B; e += blockDim.x) {
    const int r = e / QR_B, c = e % QR_B;
    A[r * LDS + c] = src[(long long)r * ld + c];
  }
  __shared__ int bad;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int j = 0; j < QR_B; ++j) {
    if (tid == 0) {
      const float d = A[j * LDS + j];
      if (!(d > 0.f)) bad = 1;
      A[j * LDS + j] = sqrtf(d);
    }
    __syncthreads();
    const float piv = A[j * LDS + j];
    for (int i = j + 1 + tid; i < QR_B; i += blockDim.x) A[i * LDS + j] /= piv;
    __syncthreads();
    // trailing lower update: A[i][c] -= A[i][j] A[c][j] for j < c <= i
    const int n = QR_B - 1 - j;
    const int tot = n * (n + 1) / 2;
    for (int e = tid; e < tot; e += blockDim.x) {
      // e -> (i, c) with 0 <= c <= i < n (row-major lower triangle)
      int i = (int)((sqrtf(8.0f * e + 1.0f) - 1.0f) * 0.5f);
      while ((i + 1) * (i + 2) / 2 <= e) ++i;
      while (i * (i + 1) / 2 > e) --i;
      const int c = e - i * (i + 1) / 2;
      const int ii = i + j + 1, cc = c + j + 1;
      A[ii * LDS + cc] -= A[ii * LDS + j] * A[cc * LDS + j];
    }
    __syncthreads();
  }
  // inverse of the lower factor: X = L^{-1}, row by row; 8 threads per column
  const int col = tid >> 3, part = tid & 7;
  for (int i = 0; i < QR_B; ++i) {
    float s = 0.f;
    if (col < i) {
      for (int p = col + part; p < i; p += 8) s = fmaf(A[i * LDS + p], X[p * LDS + col], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (part == 0) {
      float v;
      if (col < i) v = -s / A[i * LDS + i];
      else if (col == i) v = 1.0f / A[i * LDS + i];
      else v = 0.f;
      X[i * LDS + col] = v;
    }
    __syncthreads();
  }
  const float nanv = __int_as_float(0x7fc00000);
  float* dst = Dinv + (size_t)b * QR_B * QR_B;
  for (int e = tid; e < QR_B * QR_B; e += blockDim.x) {
    const int r = e / QR_B, c = e % QR_B;
    dst[e] = bad ? nanv : X[r * LDS + c];
  }
  if (tid == 0 && bad && flags.f[b] != nullptr) *flags.f[b] = 1;
}

// out[r][c] = sum_{p <= c} in[r][p] Dinv[c][p]   (in * Dinv^T, Dinv lower)
// 64 rows per CTA, 256 threads; Dinv^T and the input rows staged in smem.
__global__ void __launch_bounds__(256) rowblock_kernel(const RowBlockArgs a) {
  extern __shared__ float sm[];
  float* D = sm;                       // Dinv [128][129]
  float* R = sm + QR_B * (QR_B + 1);   // rows [64][129]
  constexpr int LDS = QR_B + 1;
  const int b = blockIdx.y;
  const int r0 = blockIdx.x * 64;
  const float* dinv = a.Dinv + (size_t)b * QR_B * QR_B;
  for (int e = threadIdx.x; e < QR_B * QR_B; e += blockDim.x) D[(e / QR_B) * LDS + e % QR_B] = dinv[e];
  const float* in = a.in + (size_t)b * a.in_stride;
  for (int e = threadIdx.x; e < 64 * QR_B; e += blockDim.x) {
    const int r = e / QR_B, c = e % QR_B;
    R[r * LDS + c] = (r0 + r < a.rows) ? in[(long long)(r0 + r) * a.ld_in + c] : 0.f;
  }
  __syncthreads();
  // thread -> (row group of 4, column c); 256 threads = 64 columns x 4 ... loop over 128 columns
  for (int e = threadIdx.x; e < 64 * QR_B; e += blockDim.x) {
    const int r = e / QR_B, c = e % QR_B;
    if (r0 + r >= a.rows) continue;
    float s = 0.f;
    for (int p = 0; p <= c; ++p) s = fmaf(R[r * LDS + p], D[c * LDS + p], s);
    const long long row = r0 + r;
    if (a.out) a.out[(size_t)b * a.out_stride + row * a.ld_out + c] = s;
    if (a.planes) {
      __nv_bfloat16 h, m, l;
      split3(s, h, m, l);
      __nv_bfloat16* d = a.planes + (size_t)b * a.mat_stride + row * QR_B + c;
      d[0] = h;
      d[a.plane_stride] = m;
      d[2 * a.plane_stride] = l;
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
    float4 w = reinterpret_cast<const float4*>(W)[i];
    const float c = 1.0f - a.beta2;
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
                      float* Dinv, const FlagTable& flags, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  const int smem = 2 * QR_B * (QR_B + 1) * 4;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(chol_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    attr = true;
  }
  chol_diag_kernel<<<count, 1024, smem, s>>>(C, ld, mat_stride, k0, Dinv, flags);
}

void launch_rowblock_dinv(const RowBlockArgs& a, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  const int smem = (QR_B + 64) * (QR_B + 1) * 4;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(rowblock_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    attr = true;
  }
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
  set_flags_kernel<<<1, SOAP_MAXB, 0, s>>>(flags, count, value);
}

}  // namespace mo
