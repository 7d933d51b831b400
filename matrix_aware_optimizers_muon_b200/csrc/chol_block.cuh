// Cholesky factor and its inverse for one 128 x 128 symmetric positive
// definite block in shared memory (256 threads).
//
// Factor, blocked by 16 (right-looking):
//   for each 16-column block kb:
//     warp 0 factors the 16 x 16 diagonal block in registers (one row per
//     lane, pivots and columns exchanged by shuffles);
//     the rows below solve against it (one row per thread);
//     every thread updates 4 x 4 tiles of the trailing lower triangle.
// Inverse, blocked by 32:
//   warp w inverts diagonal block w from its two 16 x 16 halves,
//     [[X11, 0], [X21, X22]] with X21 = -X22 (L21 X11);
//   the off-diagonal blocks follow block row by block row:
//     X_ij = -X_ii (sum_{j<=k<i} L_ik X_kj).
// The unrolled chains are kept short (16 steps) so that the code of each
// phase stays resident in the instruction cache: a fully unrolled 32-step
// chain is tens of KB of straight-line code, and fetching it dominated the
// block factorisation.
// A and X are [128][129] fp32 (row stride 129), T is [32][97] scratch.  A
// holds the block on entry (lower triangle read) and L on exit (lower
// triangle); X receives L^{-1} (lower triangle; the upper triangle is not
// written).  Returns through *bad whether a pivot was not above the floor (0
// by default: not positive; NaN included).
#pragma once

namespace mo {

constexpr int CB = 128;
constexpr int CB_LD = CB + 1;
constexpr int CB_T_LD = 97;
constexpr int CB_K = 16;                 // column block of the factorisation

// Step J of the warp-level 16 x 16 factorisation (lane i < 16 holds row i in
// r[0..15]; lanes 16-31 carry zeros); a template so that every register
// index is a constant.  The pivot's square root and reciprocal come from
// one reciprocal square root: sqrt(d) = d * rsqrt(d).
template <int J>
__device__ __forceinline__ void chol16_step(float (&r)[CB_K], int lane, bool& ok, float* inv_diag, float floor,
                                            float& mp) {
  if constexpr (J < CB_K) {
    const float d = __shfl_sync(0xffffffffu, r[J], J);
    ok = ok && (d > floor);
    mp = fminf(mp, d);
    const float inv = rsqrtf(d);
    if (lane == J) {
      r[J] = d * inv;
      inv_diag[J] = inv;
    } else if (lane > J) {
      r[J] *= inv;
    }
#pragma unroll
    for (int c = J + 1; c < CB_K; ++c) {
      const float lcj = __shfl_sync(0xffffffffu, r[J], c);
      if (c <= lane) r[c] = fmaf(-r[J], lcj, r[c]);
    }
    chol16_step<J + 1>(r, lane, ok, inv_diag, floor, mp);
  }
}

// `floor`: a pivot (diagonal of the Schur complement before its square root)
// at or below it sets *bad; *minpiv (optional, shared) receives the smallest
// pivot met.
__device__ __forceinline__ void chol128_factor(float* A, float* inv_diag, int* bad, float floor = 0.f,
                                               float* minpiv = nullptr) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll 1
  for (int kb = 0; kb < CB / CB_K; ++kb) {
    const int b0 = CB_K * kb;
    // ---- diagonal block: lane i < 16 holds row b0 + i
    if (warp == 0) {
      float r[CB_K];
#pragma unroll
      for (int c = 0; c < CB_K; ++c) r[c] = (lane < CB_K && c <= lane) ? A[(b0 + lane) * CB_LD + b0 + c] : 0.f;
      bool ok = true;
      float mp = __int_as_float(0x7f800000);
      chol16_step<0>(r, lane, ok, inv_diag + b0, floor, mp);
      if (lane < CB_K) {
#pragma unroll
        for (int c = 0; c < CB_K; ++c)
          if (c <= lane) A[(b0 + lane) * CB_LD + b0 + c] = r[c];
      }
      if (lane == 0) {
        if (minpiv != nullptr) *minpiv = fminf(*minpiv, mp);
        if (!ok) *bad = 1;
      }
    }
    __syncthreads();
    const int n2 = CB - b0 - CB_K;                // rows / columns after this block
    if (n2 == 0) break;
    // ---- panel: rows below solve x L_D^T = a (one row per thread), column
    // by column with the later columns updated as each one is final
    if (tid < n2) {
      const int row = b0 + CB_K + tid;
      float a[CB_K];
#pragma unroll
      for (int c = 0; c < CB_K; ++c) a[c] = A[row * CB_LD + b0 + c];
#pragma unroll
      for (int p = 0; p < CB_K; ++p) {
        a[p] *= inv_diag[b0 + p];
#pragma unroll
        for (int j = p + 1; j < CB_K; ++j) a[j] = fmaf(-a[p], A[(b0 + j) * CB_LD + b0 + p], a[j]);
      }
#pragma unroll
      for (int c = 0; c < CB_K; ++c) A[row * CB_LD + b0 + c] = a[c];
    }
    __syncthreads();
    // ---- trailing update of the lower triangle in 4 x 4 tiles
    {
      const int nt = n2 / 4;
      const int tiles = nt * (nt + 1) / 2;
      const int base = b0 + CB_K;
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
#pragma unroll 4
        for (int p = 0; p < CB_K; ++p) {
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

// Inverse of a 16 x 16 lower factor (rows b0 .. b0 + 15 of A) by one half
// warp: lane c < 16 of the half computes column c, x = L^{-1} e_c, row by
// row with the later rows updated as each entry is final; written to X.
__device__ __forceinline__ void inv16_column(const float* A, const float* inv_diag, float* X, int b0, int c) {
  float x[CB_K];
#pragma unroll
  for (int i = 0; i < CB_K; ++i) x[i] = i == c ? 1.0f : 0.f;
#pragma unroll
  for (int p = 0; p < CB_K; ++p) {
    x[p] = p >= c ? x[p] * inv_diag[b0 + p] : 0.f;
#pragma unroll
    for (int i = p + 1; i < CB_K; ++i) x[i] = fmaf(-A[(b0 + i) * CB_LD + b0 + p], x[p], x[i]);
  }
#pragma unroll
  for (int i = 0; i < CB_K; ++i) X[(b0 + i) * CB_LD + b0 + c] = x[i];
}

__device__ __forceinline__ void chol128_inverse(const float* A, const float* inv_diag, float* X, float* T) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // ---- diagonal blocks: warp w inverts the 32 x 32 block w from its halves
  if (warp < 4) {
    const int b0 = 32 * warp;
    const int half = lane >> 4, c = lane & 15;
    inv16_column(A, inv_diag, X, b0 + CB_K * half, c);         // X11 (half 0), X22 (half 1)
    // the block's upper-right quadrant is zero (the block rows below read
    // whole 32-column blocks of X)
    if (half == 0) {
#pragma unroll
      for (int i = 0; i < CB_K; ++i) X[(b0 + i) * CB_LD + b0 + CB_K + c] = 0.f;
    }
    __syncwarp();
    // S = L21 X11 (16 x 16, S[i][c] = sum_{k >= c} L21[i][k] X11[k][c]):
    // half h computes rows 8 h .. 8 h + 7 of column c
    float* S = T + warp * (CB_K * (CB_K + 1));                 // [16][17] per warp
#pragma unroll 1
    for (int ii = 0; ii < 8; ++ii) {
      const int i = 8 * half + ii;
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < CB_K; ++k)
        if (k >= c) s = fmaf(A[(b0 + CB_K + i) * CB_LD + b0 + k], X[(b0 + k) * CB_LD + b0 + c], s);
      S[i * (CB_K + 1) + c] = s;
    }
    __syncwarp();
    // X21 = -X22 S: half h computes rows 8 h .. 8 h + 7 of column c
#pragma unroll 1
    for (int ii = 0; ii < 8; ++ii) {
      const int i = 8 * half + ii;
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < CB_K; ++q)
        if (q <= i) s = fmaf(X[(b0 + CB_K + i) * CB_LD + b0 + CB_K + q], S[q * (CB_K + 1) + c], s);
      X[(b0 + CB_K + i) * CB_LD + b0 + c] = -s;
    }
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
#pragma unroll 4
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
#pragma unroll 4
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
