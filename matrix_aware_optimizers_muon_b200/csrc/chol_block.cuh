// Cholesky factor and its inverse for one 128 x 128 symmetric positive
// definite block in shared memory, blocked by 32:
//   for each 32-column block kb:
//     warp 0 factors the 32 x 32 diagonal block in registers (one row per
//     lane, pivots and columns exchanged by shuffles);
//     the rows below solve against it (one row per thread);
//     every thread updates 4 x 4 tiles of the trailing lower triangle;
//   then four warps invert the four diagonal 32 x 32 factors (one column per
//   lane) and the off-diagonal blocks of the inverse follow block row by
//   block row: X_ij = -X_ii (sum_{j<=k<i} L_ik X_kj).
// 256 threads; A and X are [128][129] fp32 (row stride 129), T is [32][97]
// scratch.  A holds the block on entry (lower triangle read) and L on exit
// (lower triangle); X receives L^{-1} (lower triangle; the upper triangle is
// not written).  Returns through *bad whether a pivot was not above the
// floor (0 by default: not positive; NaN included).
#pragma once

namespace mo {

constexpr int CB = 128;
constexpr int CB_LD = CB + 1;
constexpr int CB_T_LD = 97;

// Step J of the warp-level 32 x 32 factorisation (lane i holds row i in
// r[0..31]); a template so that every register index is a constant.
template <int J>
__device__ __forceinline__ void chol32_step(float (&r)[32], int lane, bool& ok, float* inv_diag, float floor,
                                            float& mp) {
  if constexpr (J < 32) {
    const float d = __shfl_sync(0xffffffffu, r[J], J);
    ok = ok && (d > floor);
    mp = fminf(mp, d);
    const float sq = sqrtf(d);
    const float inv = 1.0f / sq;
    if (lane == J) {
      r[J] = sq;
      inv_diag[J] = inv;
    } else if (lane > J) {
      r[J] *= inv;
    }
#pragma unroll
    for (int c = J + 1; c < 32; ++c) {
      const float lcj = __shfl_sync(0xffffffffu, r[J], c);
      if (c <= lane) r[c] = fmaf(-r[J], lcj, r[c]);
    }
    chol32_step<J + 1>(r, lane, ok, inv_diag, floor, mp);
  }
}

// `floor`: a pivot (diagonal of the Schur complement before its square root)
// at or below it sets *bad; *minpiv (optional, shared) receives the smallest
// pivot met.
__device__ __forceinline__ void chol128_factor(float* A, float* inv_diag, int* bad, float floor = 0.f,
                                               float* minpiv = nullptr) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int kb = 0; kb < 4; ++kb) {
    const int b0 = 32 * kb;
    // ---- diagonal block: lane i holds row b0 + i
    if (warp == 0) {
      float r[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) r[c] = c <= lane ? A[(b0 + lane) * CB_LD + b0 + c] : 0.f;
      bool ok = true;
      float mp = __int_as_float(0x7f800000);
      chol32_step<0>(r, lane, ok, inv_diag + b0, floor, mp);
      if (lane == 0 && minpiv != nullptr) *minpiv = fminf(*minpiv, mp);
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c <= lane) A[(b0 + lane) * CB_LD + b0 + c] = r[c];
      if (lane == 0 && !ok) *bad = 1;
    }
    __syncthreads();
    const int n2 = CB - b0 - 32;                  // rows / columns after this block
    // ---- panel: rows below solve x L_D^T = a (one row per thread)
    if (tid < n2) {
      const int row = b0 + 32 + tid;
      float a[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) a[c] = A[row * CB_LD + b0 + c];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float acc = a[j];
#pragma unroll
        for (int p = 0; p < j; ++p) acc = fmaf(-a[p], A[(b0 + j) * CB_LD + b0 + p], acc);
        a[j] = acc * inv_diag[b0 + j];
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) A[row * CB_LD + b0 + c] = a[c];
    }
    __syncthreads();
    // ---- trailing update of the lower triangle in 4 x 4 tiles
    if (n2 > 0) {
      const int nt = n2 / 4;
      const int tiles = nt * (nt + 1) / 2;
      const int base = b0 + 32;
      for (int t = tid; t < tiles; t += blockDim.x) {
        // tile (tr, tc) with tc <= tr, enumerated row by row
        int tr = (int)((sqrtf(8.0f * t + 1.0f) - 1.0f) * 0.5f);
        while (tr * (tr + 1) / 2 > t) --tr;
        while ((tr + 1) * (tr + 2) / 2 <= t) ++tr;
        const int tc = t - tr * (tr + 1) / 2;
        const int r0 = base + 4 * tr, c0 = base + 4 * tc;
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
        for (int p = 0; p < 32; ++p) {
          float lr[4], lc[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            lr[i] = A[(r0 + i) * CB_LD + b0 + p];
            lc[i] = A[(c0 + i) * CB_LD + b0 + p];
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(lr[i], lc[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (c0 + j <= r0 + i) A[(r0 + i) * CB_LD + c0 + j] -= acc[i][j];
      }
    }
    __syncthreads();
  }
}

__device__ __forceinline__ void chol128_inverse(const float* A, const float* inv_diag, float* X, float* T) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- diagonal blocks: warp w inverts block w; lane c owns column c
  if (warp < 4) {
    const int b0 = 32 * warp;
    float x[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float acc = i == lane ? 1.0f : 0.f;
#pragma unroll
      for (int p = 0; p < i; ++p) acc = fmaf(-A[(b0 + i) * CB_LD + b0 + p], x[p], acc);
      x[i] = i >= lane ? acc * inv_diag[b0 + i] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) X[(b0 + i) * CB_LD + b0 + lane] = x[i];
  }
  __syncthreads();
  // ---- off-diagonal blocks, block row by block row, in 4 x 4 register tiles
  for (int bi = 1; bi < 4; ++bi) {
    const int r0 = 32 * bi;
    const int cols = 32 * bi;                       // columns 0 .. 32 bi - 1 of X
    const int tiles = 8 * (cols / 4);               // 4 x 4 tiles of the 32 x cols block
    // T[i][c] = sum_{block(c) <= k < r0} L[r0 + i][k] X[k][c]  (X[k][c] = 0 above
    // the diagonal block of column c)
    for (int t = tid; t < tiles; t += blockDim.x) {
      const int ti = t / (cols / 4), tc = t - ti * (cols / 4);
      const int i0 = 4 * ti, c0 = 4 * tc;
      const int kstart = c0 & ~31;
      float acc[4][4] = {};
      for (int k = kstart; k < r0; ++k) {
        float a[4], x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          a[u] = A[(r0 + i0 + u) * CB_LD + k];
          x[u] = X[k * CB_LD + c0 + u];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], x[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) T[(i0 + u) * CB_T_LD + c0 + v] = acc[u][v];
    }
    __syncthreads();
    // X[r0 + i][c] = -sum_{p <= i} X[r0 + i][r0 + p] T[p][c]
    for (int t = tid; t < tiles; t += blockDim.x) {
      const int ti = t / (cols / 4), tc = t - ti * (cols / 4);
      const int i0 = 4 * ti, c0 = 4 * tc;
      float acc[4][4] = {};
      for (int p = 0; p < i0 + 4; ++p) {
        float xr[4], tv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          xr[u] = p <= i0 + u ? X[(r0 + i0 + u) * CB_LD + r0 + p] : 0.f;
          tv[u] = T[p * CB_T_LD + c0 + u];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(xr[u], tv[v], acc[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) X[(r0 + i0 + u) * CB_LD + c0 + v] = -acc[u][v];
    }
    __syncthreads();
  }
}

}  // namespace mo
