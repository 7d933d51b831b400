// Elementwise, splitting and small dense kernels of the SOAP path.
#include "profile.h"
#include "soap_kernels.cuh"
#include "runtime.h"

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

// four columns per thread: one float4 read of Y (rows are 16-byte aligned,
// ld a multiple of 128), the fp32 copy, and four bf16 of each plane
__global__ void basis_out_kernel(const BasisOutArgs a) {
  const int b = blockIdx.z;
  const int r = blockIdx.y;
  const int kpad = a.kpad[b];
  const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (r >= kpad || c0 >= kpad) return;
  const int k = a.k;
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  if (r < k) {
    const float* y = a.Y + (size_t)b * a.mat_stride + (long long)r * a.ld + c0;
    if (c0 + 4 <= k) {
      const float4 v = *reinterpret_cast<const float4*>(y);
      x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) x[j] = c0 + j < k ? y[j] : 0.f;
    }
    float* q = a.q[b] + (long long)r * k + c0;
    if (a.vec[b] && c0 + 4 <= k) {
      *reinterpret_cast<float4*>(q) = make_float4(x[0], x[1], x[2], x[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (c0 + j < k) q[j] = x[j];
    }
  }
  __nv_bfloat162 h01 = __floats2bfloat162_rn(x[0], x[1]);
  __nv_bfloat162 h23 = __floats2bfloat162_rn(x[2], x[3]);
  const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
  __nv_bfloat162 l01 = __floats2bfloat162_rn(x[0] - f01.x, x[1] - f01.y);
  __nv_bfloat162 l23 = __floats2bfloat162_rn(x[2] - f23.x, x[3] - f23.y);
  __nv_bfloat16* d = a.planes[b] + (long long)r * kpad + c0;     // 8-byte aligned: kpad % 4 == 0
  *reinterpret_cast<uint2*>(d) =
      make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
  *reinterpret_cast<uint2*>(d + a.pst[b]) =
      make_uint2(*reinterpret_cast<const uint32_t*>(&l01), *reinterpret_cast<const uint32_t*>(&l23));
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

void launch_basis_out(const BasisOutArgs& a, cudaStream_t s) {
  ProfScope prof(PK_SOAP_QR, s);
  dim3 grid((a.kpad_max + 1023) / 1024, a.kpad_max, a.count);
  basis_out_kernel<<<grid, 256, 0, s>>>(a);
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
