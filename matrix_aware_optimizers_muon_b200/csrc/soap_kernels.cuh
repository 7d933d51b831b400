// Kernels of the SOAP path other than the tensor-core GEMM.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace mo {

constexpr int SOAP_MAXB = 256;   // matrices per launch (pointer tables in kernel params)
constexpr int QR_B = 128;        // Cholesky diagonal block

// Copy a table of device pointers into device memory (stream ordered).
void launch_upload_ptrs(void** dst, const void* const* src, int n, cudaStream_t s);

struct SoapPrepArgs {
  int count;
  long long rows, cols;            // matrix shape (cols % 4 == 0)
  float beta1;                     // SOAP: M's beta; SOAP-Muon: the momentum mu
  int muon = 0, nesterov = 0;      // SOAP-Muon: B <- mu B + G, planes of N = G + mu B (or B)
  const float* G[SOAP_MAXB];
  float* M[SOAP_MAXB];
  __nv_bfloat16* Gp;               // two planes of G: [2][count][*][ldp]
  __nv_bfloat16* Mp;               // two planes of M
  long long ldp, mat_stride, plane_stride;
};
// M <- b1 M + (1 - b1) G ; two bf16 planes (h, l) of G and of the new M
// (SOAP-Muon: of G and of the Nesterov momentum N)
void launch_soap_prep(const SoapPrepArgs& a, cudaStream_t s);

// Split fp32 matrices into bf16 planes x = h + m + l (nearly exact): plane p
// of matrix b is written to dst + p * plane_stride + b * mat_stride, with row
// stride ldd; rows >= rows_valid or cols >= cols_valid are written as zero
// (or as the identity when `pad_identity`), up to rows_pad x cols_pad.
// Optional: per-column scale (inv_d[b * cols_pad + c]) applied first, and the
// scaled fp32 value written back to the source.
struct SplitArgs {
  int count, rows_valid, cols_valid, rows_pad, cols_pad;
  const float* src[SOAP_MAXB];     // fp32, row stride lds
  long long lds;
  const float* col_scale;          // optional [count][cols_pad]
  float* write_back;               // optional: scaled fp32, [count][rows_pad][ldw]
  long long ldw, wb_stride;
  __nv_bfloat16* dst;
  long long ldd, mat_stride, plane_stride;
  int nplanes;                     // 1 (bf16 cast), 2 (h, l) or 3 (h, m, l)
  int pad_identity;
  const float* diag_add = nullptr; // optional [count]: added to the valid diagonal first
};
void launch_split(const SplitArgs& a, cudaStream_t s);

// Damping of the power step: delta[b] = rho * trace(F[b]) over the k x k
// factor F[b] (row stride k), or 1 when that trace is zero.  The trace is
// summed in a fixed order (per-thread strided sums, then a tree).
struct DampArgs {
  int count, k;
  float rho;
  const float* F[SOAP_MAXB];
  float* delta;
};
void launch_damping(const DampArgs& a, cudaStream_t s);

struct FlagTable {
  int32_t* f[SOAP_MAXB];           // per-matrix flag slots (entries may be null)
};

// Final basis: Qout[b] (caller fp32 k x k) = Y[b][:k, :k]
// The new bases out of the refresh, in one pass over them: job b's k x k
// basis (rows of Y + b * mat_stride, row stride ld) into the caller's q[b]
// (fp32, row stride k) and, zero-padded to kpad[b] x kpad[b] (a multiple of
// 4), as two bf16 planes h = bf16(x), l = bf16(x - h) at planes[b] (row
// stride kpad[b], plane stride pst[b]) for the rotations.  vec[b]: q[b] is
// 16-byte aligned and k % 4 == 0 (float4 stores).
struct BasisOutArgs {
  int count, k, kpad_max;
  const float* Y; long long ld, mat_stride;
  float* q[SOAP_MAXB];
  __nv_bfloat16* planes[SOAP_MAXB];
  int kpad[SOAP_MAXB];
  long long pst[SOAP_MAXB];
  unsigned char vec[SOAP_MAXB];
};
void launch_basis_out(const BasisOutArgs& a, cudaStream_t s);

// Adam step with identity bases (both sides) fused with the apply:
// V <- b2 V + (1-b2) G^2 ; W <- decay W - lr (M / bc1) / (sqrt(V / bc2) + eps)
// SOAP-Muon (muon = 1): M holds the updated momentum B, the numerator is
// N = G + mu B (Nesterov) or B, and the result Dbar goes to P instead of W.
struct AdamIdArgs {
  int count;
  long long elems;
  float beta2, ibc1, ibc2, eps, decay, lr;
  int muon = 0, nesterov = 0;
  float mu = 0.f;
  const float* G[SOAP_MAXB];
  const float* M[SOAP_MAXB];
  float* V[SOAP_MAXB];
  float* W[SOAP_MAXB];
  float* P[SOAP_MAXB];
};
void launch_adam_identity(const AdamIdArgs& a, cudaStream_t s);

// Per-matrix flag reset (the QR pivots report into them)
void launch_set_flags(const FlagTable& flags, int count, int32_t value, cudaStream_t s);

}  // namespace mo
