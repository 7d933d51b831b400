// Batched bf16 (or fp16) GEMM on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA, with a fused epilogue: D = alpha_b * (A B) + beta_b * C, the
// Adam step of SOAP in the rotated basis (EPI_ADAM), or the Muon apply
// W <- decay W - step bf16(alpha_b A B + beta_b C) into fp32 W (EPI_APPLY).
//
// One persistent CTA per SM (with PAIR, a cluster of two CTAs on two SMs
// shares each 256-row tile through cta_group::2 MMAs), 6 warps:
//   warp 0      TMA producer: fills a ring of shared-memory stages
//   warp 1      MMA issuer: one elected thread issues tcgen05.mma into one
//               of two TMEM accumulators (so the epilogue of tile i overlaps
//               the main loop of tile i+1) and commits stage releases
//   warps 2..5  epilogue: tcgen05.ld the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 = tile rows), apply alpha/beta/C, store
//
// Tiles are 128 x BN (BN = 256 or 128) with BK = 64 (one 128-byte swizzle
// row of bf16).  A is M x K and B is K x N; each may be stored K-major
// (K contiguous) or MN-major (M or N contiguous).  With `sym` set the
// product is known to be symmetric (X X^T, or A A with A symmetric): only
// tiles that touch the upper triangle are computed, and each upper element
// is stored at (r, c) and mirrored to (c, r), so both halves are bit-equal.
// Tiles are taken in column order, or in bands of row tiles when the A
// panel overflows L2 (gemm_decode); the order changes no result.
#pragma once

#include "ptx.cuh"
#include <cuda_bf16.h>

namespace mo {

struct GemmParams {
  int M, N, K;              // per-matrix problem size
  int batch;                // number of independent matrices
  int bm;                   // rows of a tile: 128, or 256 for a CTA pair
  int tiles_m, tiles_n;     // tile grid of one matrix
  int tiles_per_mat;        // tiles enumerated per matrix (fewer when sym)
  int sym;                  // symmetric product: upper tiles + mirror stores
  float alpha, beta;        // epilogue coefficients
  const float* scale;       // optional per-matrix scale s_b (device)
  int alpha_pow, beta_pow;  // alpha_b = alpha * s_b^alpha_pow, beta_b likewise
  const void* C;            // optional epilogue input (may alias D)
  long long ldc, strideC;   // elements
  int c_f32;                // C is fp32 (else bf16)
  void* D;                  // output
  long long ldd, strideD;   // elements
  int d_f32;                // D is fp32 (else bf16)
  int* status;              // device status word (timeouts)
  // optional per-matrix pointer tables (device arrays of `batch` entries);
  // when set they replace base + b * stride for C, D and E
  const void* const* c_tab;
  void* const* d_tab;
  float* const* e_tab;
  int epi;                  // EPI_AXPBY or EPI_ADAM
  // Adam-in-basis epilogue (acc = G'): V = b2 V + (1 - b2) acc^2 (E, fp32,
  // in place); D = bf16((C * ibc1) / (sqrt(V * ibc2) + eps)) with C = M'
  float adam_b2, adam_ibc1, adam_ibc2, adam_eps;
  long long lde, strideE;
  // plane-stacked K: K = nseg * kseg; segment s multiplies plane pat_a[s] of
  // A by plane pat_b[s] of B (split-precision products); nseg == 1: plain
  int nseg, kseg;
  unsigned char pat_a[8], pat_b[8];
  // bf16 output as two planes: D = bf16(x), D + d_plane = bf16(x - bf16(x))
  int d_split;
  long long d_plane;
  // optional per-matrix flags (device): matrices with skip[b] != 0 are left
  // untouched (every role of the kernel skips their tiles)
  const int* skip;
  // bf16 C read by TMA (tensor map tmC, 32 x 32 boxes, 64-byte swizzle)
  int c_tma;
  // full 32 x 32 blocks of a plain bf16 D are written by TMA stores (tensor
  // map tmD, same boxes): non-symmetric with c_tma, from the slot their C
  // block arrived in; otherwise from staging slots (a symmetric product's
  // mirror block by a second store)
  int d_tma;
  // tile order: bands of `band` row tiles, each band column by column; a
  // band of tiles_m rows (or more) is the plain column order
  int band;
  // Muon apply (EPI_APPLY): O = bf16(alpha acc + beta C) is not stored;
  // W <- ap_decay W - ap_step[tall] O instead, with W = e_tab[b] (fp32,
  // contiguous), laid out like the product (M x N) or, for the matrices
  // b >= ap_tall_from, as its transpose (N x M)
  float ap_decay;
  float ap_step[2];
  int ap_tall_from;
  int ap_vec;               // every W of the launch: 16-byte aligned rows
  // launch gate: nothing when gate[gate_idx ? *gate_idx : 0] >= gate_n
  const int* gate;
  int gate_n;
  const int* gate_idx;
  // added to the diagonal elements (row == column) of each matrix's
  // output, before rounding (epilogue AXPBY)
  float diag;
  // A and B hold fp16 (not bf16) values: the same kind::f16 MMA with the
  // operand type fields of the instruction descriptor set to f16
  int ab_f16;
};

enum { EPI_AXPBY = 0, EPI_ADAM = 1, EPI_APPLY = 2 };

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_THREADS = 192;        // producer, MMA issuer, 4 epilogue warps
constexpr int GEMM_THREADS_EPI2 = 320;   // the same with two sets of 4 epilogue warps

// PAIR: a cluster of two CTAs computes a 256 x BN tile with cta_group::2
// MMAs; each CTA stages its 128 rows of A and BN/2 rows (columns of the
// product) of B, so a stage is 32 KB instead of 48 KB per SM.
// EPI2: two sets of four epilogue warps, set s draining accumulator s (the
// MMA issuer alternates the two accumulators tile by tile), for products
// with a short K whose main loop per tile is not longer than one set's
// epilogue; their staging takes one TMA stage fewer.
template <int BN, bool PAIR = false, bool EPI2 = false>
struct GemmCfg {
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK * 2;
  static constexpr int BN_LOCAL = PAIR ? BN / 2 : BN;
  static constexpr int B_BYTES = BN_LOCAL * GEMM_BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = PAIR ? (EPI2 ? 5 : 6) : (BN == 256 ? (EPI2 ? 3 : 4) : (EPI2 ? 5 : 6));
  // fp32 accumulators in tensor memory: two, or four 128-column ones with
  // two epilogue sets (each set then drains every other accumulator, and a
  // tile's epilogue overlaps the next three tiles' main loops)
  static constexpr int NACC = (EPI2 && BN == 128) ? 4 : 2;
  static constexpr int TMEM_COLS = NACC * BN;
  static constexpr int BAR_BYTES = 1024;            // mbarriers; keeps the epilogue stage 1 KB aligned
  static constexpr int EPI_WARPS = EPI2 ? 8 : 4;
  static constexpr int EPI_BYTES = EPI_WARPS * 8192;  // per epilogue warp: output block (or C), its transpose
  static constexpr int THREADS = EPI2 ? GEMM_THREADS_EPI2 : GEMM_THREADS;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + EPI_BYTES + 1024;
};

// Tiles of one matrix in column order (M fastest, so the CTAs in flight
// share B columns in L2).  For a symmetric product only the tiles touching
// the upper triangle are enumerated: column tn holds rows tm with
// tm * BM <= tn * BN + BN - 1, i.e. tm < q (tn + 1) with q = BN / BM (1 or
// 2), so the persistent CTAs get equal shares of computed tiles.
//
// When the A panel of a matrix does not fit in L2 the host may split the
// rows into bands of p.band tiles: band after band, each in column order
// (rows fastest), so that a band's A rows stay in L2 while the B columns
// stream past them once per band.
__device__ __forceinline__ int sym_rows_in_col(const GemmParams& p, int BN, int tn) {
  const int r = (tn * BN + BN - 1) / p.bm + 1;
  return r < p.tiles_m ? r : p.tiles_m;
}

// Upper-triangle tiles of a symmetric product in the band of rows
// [r0, r0 + rows): column tn holds clamp(q (tn + 1) - r0, 0, rows) of them.
// Columns before a hold none, columns from f on hold all `rows`, the ones
// in between a ramp; returned with a and f (both clamped to tiles_n).
__device__ __forceinline__ long long sym_band_tiles(const GemmParams& p, int q, int r0, int rows, int& a,
                                                    int& f) {
  const int tn_all = p.tiles_n;
  a = r0 / q;
  f = (r0 + rows + q - 1) / q - 1;
  if (a > tn_all) a = tn_all;
  if (f > tn_all) f = tn_all;
  if (f < a) f = a;
  // sum over tn in [a, f) of q (tn + 1) - r0, then full columns
  const long long ramp = (long long)q * ((long long)f * (f + 1) - (long long)a * (a + 1)) / 2 -
                         (long long)r0 * (f - a);
  return ramp + (long long)rows * (tn_all - f);
}

__device__ __forceinline__ bool gemm_decode(const GemmParams& p, int BN, int t, int& b, int& tm,
                                            int& tn) {
  b = t / p.tiles_per_mat;
  if (p.skip && p.skip[b]) return false;
  int u = t - b * p.tiles_per_mat;
  if (p.band < p.tiles_m) {
    const int G = p.band;
    if (!p.sym) {
      const int per_band = G * p.tiles_n;
      const int k = u / per_band;
      const int r0 = k * G;
      const int rows = p.tiles_m - r0 < G ? p.tiles_m - r0 : G;
      const int v = u - k * per_band;
      tn = v / rows;
      tm = r0 + (v - tn * rows);
      return true;
    }
    const int q = BN / p.bm;
    for (int r0 = 0; r0 < p.tiles_m; r0 += G) {
      const int rows = p.tiles_m - r0 < G ? p.tiles_m - r0 : G;
      int a, f;
      const long long cnt = sym_band_tiles(p, q, r0, rows, a, f);
      if (u >= cnt) {
        u -= (int)cnt;
        continue;
      }
      for (tn = a; tn < f; ++tn) {
        const int c = q * (tn + 1) - r0;
        if (u < c) {
          tm = r0 + u;
          return true;
        }
        u -= c;
      }
      tn = f + u / rows;
      tm = r0 + (u - (tn - f) * rows);
      return true;
    }
    tm = tn = 0;               // unreachable for t < tiles_per_mat * batch
    return true;
  }
  if (!p.sym) {
    tn = u / p.tiles_m;
    tm = u - tn * p.tiles_m;
    return true;
  }
  for (tn = 0; tn < p.tiles_n; ++tn) {
    const int c = sym_rows_in_col(p, BN, tn);
    if (u < c) break;
    u -= c;
  }
  tm = u;
  return true;
}

__device__ __forceinline__ const void* c_base(const GemmParams& p, int b) {
  if (p.c_tab) return p.c_tab[b];
  return reinterpret_cast<const char*>(p.C) + (size_t)b * p.strideC * (p.c_f32 ? 4 : 2);
}

__device__ __forceinline__ void* d_base(const GemmParams& p, int b) {
  if (p.d_tab) return p.d_tab[b];
  return reinterpret_cast<char*>(p.D) + (size_t)b * p.strideD * (p.d_f32 ? 4 : 2);
}

__device__ __forceinline__ float ipow_scale(const float* s, int b, int pw) {
  if (s == nullptr || pw == 0) return 1.0f;
  const float v = s[b];
  return pw == 1 ? v : v * v;
}

// Load n (<= 32) consecutive values at base + off (fp32 or bf16) into c[0..31];
// the vector path needs n == 32 and 16-byte aligned rows.
__device__ __forceinline__ void load_row32(const char* base, int f32, long long off, int n, float (&c)[32]) {
  if (f32) {
    const float* src = reinterpret_cast<const float*>(base) + off;
    if (n == 32) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 v = reinterpret_cast<const float4*>(src)[i];
        c[4 * i] = v.x; c[4 * i + 1] = v.y; c[4 * i + 2] = v.z; c[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) c[i] = i < n ? src[i] : 0.0f;
    }
  } else {
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(base) + off;
    if (n == 32) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = reinterpret_cast<const uint4*>(src)[i];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
          c[8 * i + 2 * j] = f.x;
          c[8 * i + 2 * j + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) c[i] = i < n ? __bfloat162float(src[i]) : 0.0f;
    }
  }
}

// Store x[lo..hi) at base + off + i (fp32, bf16, or bf16 as two planes).
__device__ __forceinline__ void store_row(const GemmParams& p, char* base, long long off, int hi, int lo,
                                          const float (&x)[32]) {
  if (p.d_f32) {
    float* dst = reinterpret_cast<float*>(base) + off;
    if (lo == 0 && hi == 32) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4*>(dst)[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i >= lo && i < hi) dst[i] = x[i];
    }
    return;
  }
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(base) + off;
  if (lo == 0 && hi == 32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[8 * i + 2 * j], x[8 * i + 2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t*>(&h);
      }
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (p.d_split) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float x0 = x[8 * i + 2 * j], x1 = x[8 * i + 2 * j + 1];
          const float2 hf = __bfloat1622float2(__floats2bfloat162_rn(x0, x1));
          const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
          w[j] = *reinterpret_cast<const uint32_t*>(&l);
        }
        reinterpret_cast<uint4*>(dst + p.d_plane)[i] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i >= lo && i < hi) {
        const __nv_bfloat16 h = __float2bfloat16_rn(x[i]);
        dst[i] = h;
        if (p.d_split) dst[i + p.d_plane] = __float2bfloat16_rn(x[i] - __bfloat162float(h));
      }
    }
  }
}

// Mirror stores of a symmetric product: element (r, c0 + i) also goes to
// (c0 + i, r) for lo <= i < hi with c0 + i > r.  For fixed i the lanes of a
// warp hold consecutive rows r, so each store instruction is contiguous.
__device__ __forceinline__ void store_mirror(const GemmParams& p, char* base, int r, int c0, int lo, int hi,
                                             const float (&x)[32]) {
  if (p.d_f32) {
    float* dst = reinterpret_cast<float*>(base) + r;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i >= lo && i < hi && c0 + i > r) dst[(long long)(c0 + i) * p.ldd] = x[i];
  } else {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(base) + r;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i >= lo && i < hi && c0 + i > r) {
        const __nv_bfloat16 h = __float2bfloat16_rn(x[i]);
        dst[(long long)(c0 + i) * p.ldd] = h;
        if (p.d_split) dst[(long long)(c0 + i) * p.ldd + p.d_plane] = __float2bfloat16_rn(x[i] - __bfloat162float(h));
      }
    }
  }
}

// Coalesced bf16 stores of one warp's 32 x 32 output block through shared
// memory: the block (rows of the warp's lanes, columns c0..c0+31) is staged
// row-major and, for a symmetric product, transposed; then every store
// instruction writes eight full 64-byte rows.  The staging rows are 64 bytes
// with their four 16-byte units XOR-swizzled by (row / 2) % 4, which keeps
// the 16-byte writes, the 2-byte transposed writes and the 16-byte reads
// free of bank conflicts.  drow = &D[r0][c0]; dmir = &D[c0][r0] or null.
__device__ __forceinline__ uint32_t stg_off(int row, int unit) {
  return (uint32_t)(row * 64 + ((unit ^ ((row >> 1) & 3)) << 4));
}

__device__ __forceinline__ void stage_store32(uint8_t* stg, int lane, const float (&x)[32], __nv_bfloat16* drow,
                                              __nv_bfloat16* dmir, long long ldd) {
  uint8_t* srow = stg;
  uint8_t* scol = stg + 2048;
  __syncwarp();                       // the previous block's reads are done
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[8 * u + 2 * j], x[8 * u + 2 * j + 1]);
      w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(srow + stg_off(lane, u)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (dmir) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      *reinterpret_cast<__nv_bfloat16*>(scol + stg_off(i, lane >> 3) + ((lane & 7) << 1)) = __float2bfloat16_rn(x[i]);
  }
  __syncwarp();
  const int u = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int R = 8 * j + (lane >> 2);
    *reinterpret_cast<uint4*>(drow + (long long)R * ldd + 8 * u) = *reinterpret_cast<const uint4*>(srow + stg_off(R, u));
    if (dmir)
      *reinterpret_cast<uint4*>(dmir + (long long)R * ldd + 8 * u) = *reinterpret_cast<const uint4*>(scol + stg_off(R, u));
  }
}

// A 32 x 32 block on the diagonal of a symmetric product: each element
// takes the value computed above the diagonal (its own for c >= r, its
// mirror's for c < r), so both halves are bit-equal, with the same coalesced
// row stores.
// The transpose of the staged 32 x 32 bf16 block `own` into `mir` (both in
// the rows of stg_off(); every lane's row of `own` written before the
// call).  Each 8 x 8 sub-block (I, J) is one 16-byte unit J of rows 8I..8I+7:
// a transposing ldmatrix takes the four sub-blocks (I, 0..3), and stmatrix
// writes sub-block (I, J)^T as rows 8J..8J+7, unit I, of the mirror.
__device__ __forceinline__ void stage_mirror_trans(const uint8_t* own, uint8_t* mir, int lane) {
#pragma unroll
  for (int I = 0; I < 4; ++I) {
    uint32_t r0, r1, r2, r3;
    const uint32_t src = smem_u32(own + stg_off(8 * I + (lane & 7), lane >> 3));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(src)
                 : "memory");
    const uint32_t dst = smem_u32(mir + stg_off(lane, I));
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
  }
}

// For TMA stores of a 32 x 32 bf16 block: this lane's row into `own` and,
// when `mir` is set, its transpose (the mirror block) into `mir`, both in
// the 64-byte-swizzled rows of stg_off().
__device__ __forceinline__ void stage_rows_tma(uint8_t* own, uint8_t* mir, int lane, const float (&x)[32]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[8 * u + 2 * j], x[8 * u + 2 * j + 1]);
      w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(own + stg_off(lane, u)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (mir) {
    __syncwarp();                       // every row of `own` is staged
    stage_mirror_trans(own, mir, lane);
  }
}

// A staged block on the diagonal of a symmetric product (own rows and their
// transpose staged, then a __syncwarp): every element below the diagonal
// takes its mirror's value, in place in `own`; each lane rewrites the
// 16-byte units it reads.
__device__ __forceinline__ void symmetrize_staged(uint8_t* own, const uint8_t* mir, int lane) {
  const int u = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int R = 8 * j + (lane >> 2);
    uint4 a = *reinterpret_cast<const uint4*>(own + stg_off(R, u));
    const uint4 m = *reinterpret_cast<const uint4*>(mir + stg_off(R, u));
    uint16_t* pa = reinterpret_cast<uint16_t*>(&a);
    const uint16_t* pm = reinterpret_cast<const uint16_t*>(&m);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (8 * u + e < R) pa[e] = pm[e];
    *reinterpret_cast<uint4*>(own + stg_off(R, u)) = a;
  }
}

__device__ __forceinline__ void stage_store32_diag(uint8_t* stg, int lane, const float (&x)[32], __nv_bfloat16* drow,
                                                   long long ldd) {
  uint8_t* srow = stg;
  uint8_t* scol = stg + 2048;
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[8 * u + 2 * j], x[8 * u + 2 * j + 1]);
      w[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(srow + stg_off(lane, u)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
#pragma unroll
  for (int i = 0; i < 32; ++i)
    *reinterpret_cast<__nv_bfloat16*>(scol + stg_off(i, lane >> 3) + ((lane & 7) << 1)) = __float2bfloat16_rn(x[i]);
  __syncwarp();
  const int u = lane & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int R = 8 * j + (lane >> 2);
    uint4 a = *reinterpret_cast<const uint4*>(srow + stg_off(R, u));
    const uint4 m = *reinterpret_cast<const uint4*>(scol + stg_off(R, u));
    // columns 8u .. 8u + 7 of row R: below the diagonal (c < R) from the mirror
    uint16_t* pa = reinterpret_cast<uint16_t*>(&a);
    const uint16_t* pm = reinterpret_cast<const uint16_t*>(&m);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (8 * u + e < R) pa[e] = pm[e];
    *reinterpret_cast<uint4*>(drow + (long long)R * ldd + 8 * u) = a;
  }
}

// The fp32 version: 128-byte staging rows with the classic 128-byte XOR
// swizzle (unit ^ row % 8); every store instruction writes four full rows.
__device__ __forceinline__ uint32_t stg32_off(int row, int unit) {
  return (uint32_t)(row * 128 + ((unit ^ (row & 7)) << 4));
}

__device__ __forceinline__ void stage_store32_f32(uint8_t* stg, int lane, const float (&x)[32], float* drow,
                                                  float* dmir, long long ldd, bool streaming = false) {
  uint8_t* srow = stg;
  uint8_t* scol = stg + 4096;
  __syncwarp();                       // earlier reads of the staging rows are done
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<float4*>(srow + stg32_off(lane, u)) = make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
  if (dmir) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      *reinterpret_cast<float*>(scol + stg32_off(i, lane >> 2) + ((lane & 3) << 2)) = x[i];
  }
  __syncwarp();
  const int u = lane & 7;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int R = 4 * j + (lane >> 3);
    const float4 v = *reinterpret_cast<const float4*>(srow + stg32_off(R, u));
    float4* dst = reinterpret_cast<float4*>(drow + (long long)R * ldd + 4 * u);
    if (streaming) __stcs(dst, v);     // written once: evict-first in L2
    else *dst = v;
    if (dmir)
      *reinterpret_cast<float4*>(dmir + (long long)R * ldd + 4 * u) = *reinterpret_cast<const float4*>(scol + stg32_off(R, u));
  }
}

__device__ __forceinline__ void stage_store32_f32_diag(uint8_t* stg, int lane, const float (&x)[32], float* drow,
                                                       long long ldd) {
  uint8_t* srow = stg;
  uint8_t* scol = stg + 4096;
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<float4*>(srow + stg32_off(lane, u)) = make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
#pragma unroll
  for (int i = 0; i < 32; ++i)
    *reinterpret_cast<float*>(scol + stg32_off(i, lane >> 2) + ((lane & 3) << 2)) = x[i];
  __syncwarp();
  const int u = lane & 7;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int R = 4 * j + (lane >> 3);
    float4 a = *reinterpret_cast<const float4*>(srow + stg32_off(R, u));
    const float4 m = *reinterpret_cast<const float4*>(scol + stg32_off(R, u));
    if (4 * u + 0 < R) a.x = m.x;
    if (4 * u + 1 < R) a.y = m.y;
    if (4 * u + 2 < R) a.z = m.z;
    if (4 * u + 3 < R) a.w = m.w;
    *reinterpret_cast<float4*>(drow + (long long)R * ldd + 4 * u) = a;
  }
}

template <int BN, int A_MN, int B_MN, bool PAIR = false, bool EPI2 = false>
__global__ void __launch_bounds__(GemmCfg<BN, PAIR, EPI2>::THREADS, 1) __maxnreg__(EPI2 ? 200 : 255)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                 const GemmParams p) {
  using Cfg = GemmCfg<BN, PAIR, EPI2>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int BM_T = PAIR ? 2 * GEMM_BM : GEMM_BM;     // rows per tile
  constexpr int BN_L = Cfg::BN_LOCAL;                     // B rows staged by this CTA
  constexpr uint32_t IDESC_BF16 = idesc_bf16_f32(BM_T, BN, A_MN, B_MN);
  const uint32_t IDESC = p.ab_f16 ? idesc_as_f16(IDESC_BF16) : IDESC_BF16;

  // a gated launch reads its gate first (after its predecessor) and, when
  // closed, leaves before any setup; the whole grid reads the same word
  if (p.gate != nullptr) {
    pdl_wait();
    if (p.gate[p.gate_idx ? *p.gate_idx : 0] >= p.gate_n) return;
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + Cfg::NACC;
  uint64_t* drain = acc_empty + Cfg::NACC;
  uint64_t* cbar = drain + 1;                 // [epilogue warps][4]: C blocks read by TMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cbar + 4 * Cfg::EPI_WARPS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* consumed = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // a pair: rank 0 issues the MMAs; both CTAs load and run the epilogue
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < Cfg::NACC; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], PAIR ? 256 : 128);   // the epilogue threads of every CTA of the tile
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 4 * Cfg::EPI_WARPS; ++i) mbar_init(&cbar[i], 1);
    *abort_flag = 0;
    *consumed = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if constexpr (PAIR) cluster_sync_all();       // the peer's barriers exist before any remote arrival
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the prologue above touched no global memory: from here on the previous
  // kernel's results are needed
  pdl_wait();
  pdl_trigger();

  const int total = p.tiles_per_mat * p.batch;
  const int nk = (p.K + GEMM_BK - 1) / GEMM_BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = unit; t < total && ok; t += units) {
        int b, tm, tn;
        if (!gemm_decode(p, BN, t, b, tm, tn)) continue;
        const int arow = tm * BM_T + (int)rank * GEMM_BM;      // this CTA's rows of A
        const int bcol = tn * BN + (int)rank * BN_L;           // this CTA's rows of B (columns of D)
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, DEV_TIMEOUT_EMPTY)) {
            ok = false;
            break;
          }
          // a pair counts both CTAs' bytes on the even CTA's barrier
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], PAIR ? 2 * Cfg::STAGE_BYTES : Cfg::STAGE_BYTES);
          const uint32_t full_cl = PAIR ? mapa_shared(&full[stage], 0) : 0u;
          auto load = [&](void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3) {
            if constexpr (PAIR) tma_load_4d_pair(dst, map, full_cl, c0, c1, c2, c3);
            else tma_load_4d(dst, map, &full[stage], c0, c1, c2, c3);
          };
          uint8_t* sa = smem + stage * Cfg::STAGE_BYTES;
          uint8_t* sb = sa + Cfg::A_BYTES;
          int kl = kb * GEMM_BK, pa = 0, pb = 0;
          if (p.nseg > 1) {
            const int seg = kl / p.kseg;
            kl -= seg * p.kseg;
            pa = p.pat_a[seg];
            pb = p.pat_b[seg];
          }
          if (!A_MN) {
            load(sa, &tmA, kl, arow, b, pa);
          } else {
            load(sa, &tmA, arow, kl, b, pa);
            load(sa + GEMM_BK * 128, &tmA, arow + 64, kl, b, pa);
          }
          if (!B_MN) {
            load(sb, &tmB, kl, bcol, b, pb);
          } else {
#pragma unroll
            for (int j = 0; j < BN_L / 64; ++j) load(sb + j * GEMM_BK * 128, &tmB, bcol + 64 * j, kl, b, pb);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && rank == 0) {
        // let every copy already in flight land before the CTA can exit
        // (a pair's copies are counted on the even CTA's barriers)
        for (int i = *consumed; i < issued; ++i)
          mbar_wait_drain(&full[i % STAGES], (uint32_t)((i / STAGES) & 1), p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && rank == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool any = false, ok = true;
      for (int t = unit; t < total && ok; t += units) {
        int b, tm, tn;
        if (!gemm_decode(p, BN, t, b, tm, tn)) continue;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, p.status, DEV_TIMEOUT_ACC_EMPTY)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, DEV_TIMEOUT_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t sb = sa + Cfg::A_BYTES;
#pragma unroll
          for (int k = 0; k < GEMM_BK / 16; ++k) {
            const uint64_t ad = A_MN ? smem_desc_sw128(sa + k * 2048, GEMM_BK * 128, 1024)
                                     : smem_desc_sw128(sa + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? smem_desc_sw128(sb + k * 2048, GEMM_BK * 128, 1024)
                                     : smem_desc_sw128(sb + k * 32, 16, 1024);
            if constexpr (PAIR) tc_mma_f16_pair(d_tmem, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
            else tc_mma_f16(d_tmem, ad, bd, IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          any = true;
          if constexpr (PAIR) tc_commit_pair(&empty[stage], 3);     // frees the stage in both CTAs
          else tc_commit(&empty[stage]);
          *consumed = *consumed + 1;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (PAIR) tc_commit_pair(&acc_full[acc], 3);     // both CTAs' epilogues
        else tc_commit(&acc_full[acc]);
        if (++acc == Cfg::NACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (any) {
        // every MMA issued by this thread must finish before TMEM is freed
        if constexpr (PAIR) tc_commit_pair(drain, 1);
        else tc_commit(drain);
        mbar_wait_drain(drain, 0, p.status);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int ew = warp - 2;                // epilogue warp index
    const int eset = ew >> 2;               // EPI2: the accumulator this warp's set drains
    const int row_in_tile = q * 32 + lane;
    uint8_t* stg = smem + STAGES * Cfg::STAGE_BYTES + Cfg::BAR_BYTES + ew * 8192;
    uint8_t* stc = stg + 4096;              // staged 32 x 32 bf16 block of C
    // C blocks that TMA writes in the 64-byte-swizzled layout stg_off()
    // reads go to 2 KB slots (1 KB aligned) at stg + 2048 slot: slots 2 and
    // 3 while stg holds the output staging rows, all four when the output
    // leaves by TMA stores from the C slots themselves
    uint64_t* cb = cbar + 4 * ew;
    uint32_t cph = 0u;                      // bit i: phase of slot i
    uint32_t cpend = 0u;                    // bit i: a copy into slot i is in flight
    const bool plain_bf16 = !p.d_f32 && !p.d_split;
    const bool plain_f32 = p.d_f32 && !p.d_split;
    const bool has_c = p.C != nullptr || p.c_tab != nullptr;
    const bool adam = p.epi == EPI_ADAM;
    const bool apply = p.epi == EPI_APPLY;
    int ntile = 0;                          // tiles of this CTA so far: accumulator ntile % NACC
    // a pair's epilogue threads release the accumulator on the even CTA's barrier
    const uint32_t acc_empty_cl0 = PAIR ? mapa_shared(&acc_empty[0], 0) : 0u;
    const uint32_t acc_empty_cl1 = PAIR ? mapa_shared(&acc_empty[1], 0) : 0u;
    for (int t = unit; t < total; t += units) {
      int b, tm, tn;
      if (!gemm_decode(p, BN, t, b, tm, tn)) continue;
      const int acc = ntile % Cfg::NACC;
      const uint32_t acc_phase = (uint32_t)(ntile / Cfg::NACC) & 1u;
      ++ntile;
      if (EPI2 && (acc & 1) != eset) continue;    // the other set's tile
      const int r = tm * BM_T + (int)rank * GEMM_BM + row_in_tile;
      const bool row_ok = r < p.M;
      // this matrix's operands, resolved once per tile
      const char* cbase = has_c ? reinterpret_cast<const char*>(c_base(p, b)) : nullptr;
      char* dbase = reinterpret_cast<char*>(d_base(p, b));
      float* vbase = adam ? p.e_tab[b] : nullptr;
      float* wbase = apply ? p.e_tab[b] : nullptr;
      const bool wtall = apply && b >= p.ap_tall_from;
      const long long ldw = wtall ? p.M : p.N;      // W is contiguous: N x M (tall) or M x N
      const float wstep = p.ap_step[wtall ? 1 : 0];
      if (row_ok) {
        // pull this row's epilogue inputs into L2 while the main loop runs,
        // so that the loads after the accumulator wait do not pay DRAM latency
        const int n0 = tn * BN;
        const int nn = p.N - n0 < BN ? p.N - n0 : BN;
        if (has_c && nn > 0) {
          const int es = p.c_f32 ? 4 : 2;
          const char* row = cbase + ((long long)r * p.ldc + n0) * es;
          for (int off = 0; off < nn * es; off += 128) prefetch_l2(row + off);
        }
        if (adam && nn > 0) {
          const char* row = reinterpret_cast<const char*>(vbase + (long long)r * p.lde + n0);
          for (int off = 0; off < nn * 4; off += 128) prefetch_l2(row + off);
        }
        if (apply && !wtall && nn > 0) {
          const char* row = reinterpret_cast<const char*>(wbase + (long long)r * ldw + n0);
          for (int off = 0; off < nn * 4; off += 128) prefetch_l2(row + off);
        }
      }
      // bf16 C of full blocks comes by TMA, the first two 32-column blocks
      // requested now so that they arrive while the main loop runs
      const int r0 = tm * BM_T + (int)rank * GEMM_BM + q * 32;     // this warp's first row
      const int n0 = tn * BN;
      // a symmetric product skips the 32 x 32 blocks below the diagonal
      const int cc_begin = p.sym ? (r0 - n0 > 0 ? r0 - n0 : 0) : 0;
      if (apply && wtall && r0 < p.M) {
        // the transposed W block of this warp: one 128-byte line per W row
        const int nn = p.N - n0 < BN ? p.N - n0 : BN;
        for (int c = lane; c < nn; c += 32) prefetch_l2(wbase + (long long)(n0 + c) * ldw + r0);
      }
      // Muon apply on a full tile: W blocks move with coalesced accesses,
      // 16-byte vectors through shared memory (W laid out like the product)
      // or one 128-byte W row per access (transposed W)
      const bool wfull = apply && n0 + BN <= p.N && __all_sync(0xffffffffu, row_ok);
      const bool wvec = wfull && !wtall && p.ap_vec;
      const bool wtr = wfull && wtall;
      const bool ctma = p.c_tma && !adam && plain_bf16 && n0 + BN <= p.N && __all_sync(0xffffffffu, row_ok);
      // output blocks by TMA store, written over their C block's slot;
      // C requested three blocks ahead
      const bool dtma = ctma && p.d_tma && !p.sym;
      // ... or from the staging slots 0 (own block) and 1 (mirror block)
      const bool dstg = p.d_tma && !dtma && n0 + BN <= p.N && (!has_c || ctma) && __all_sync(0xffffffffu, row_ok);
      auto issue_c = [&](int slot, int cc) {
        mbar_arrive_expect_tx(&cb[slot], 32 * 32 * 2);
        tma_load_3d(stg + 2048 * slot, &tmC, &cb[slot], n0 + cc, r0, b);
        cpend |= 1u << slot;
      };
      if (ctma && lane == 0) {
        fence_proxy_async_smem();              // earlier reads of the slots come first
        if (dtma) {
          bulk_wait_read();                    // the previous tile's stores have read their slots
          for (int i = 0; i < 3; ++i)
            if (cc_begin + 32 * i < BN) issue_c(i, cc_begin + 32 * i);
        } else {
          if (cc_begin < BN) issue_c(2, cc_begin);
          if (cc_begin + 32 < BN) issue_c(3, cc_begin + 32);
        }
      }
      // with TMA stores in the launch, the previous tile's stores must have
      // read their slots before any lane writes the staging area again (the
      // vote after the accumulator wait orders the other lanes after this)
      if (p.d_tma && lane == 0) bulk_wait_read();
      // warp-uniform: tcgen05.ld below must be executed by all 32 lanes
      const bool ok = mbar_wait(&acc_full[acc], acc_phase, abort_flag, p.status, DEV_TIMEOUT_ACC_FULL);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const float alpha = p.alpha * ipow_scale(p.scale, b, p.alpha_pow);
      const float beta = p.beta * ipow_scale(p.scale, b, p.beta_pow);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      // otherwise bf16 C of full blocks (pointer tables): loaded one block
      // ahead with coalesced 16-byte loads (eight 64-byte rows per
      // instruction), then transposed to row-per-lane through shared memory
      const bool cpre = !EPI2 && !ctma && has_c && !adam && !p.c_f32 && plain_bf16 && n0 + BN <= p.N &&
                        __all_sync(0xffffffffu, row_ok);
      const __nv_bfloat16* c16 = reinterpret_cast<const __nv_bfloat16*>(cbase);
      uint4 cnext[4];
      auto load_c = [&](int cc) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int R = 8 * j + (lane >> 2);
          cnext[j] = *reinterpret_cast<const uint4*>(c16 + (long long)(r0 + R) * p.ldc + n0 + cc + 8 * (lane & 3));
        }
      };
      if (cpre && cc_begin < BN) load_c(cc_begin);
      // fp32 C for full blocks: coalesced 16-byte loads issued before the
      // accumulator read, staged in shared memory (the output's staging rows)
      const bool cf32 = has_c && !adam && p.c_f32 && !p.d_split && n0 + BN <= p.N &&
                        __all_sync(0xffffffffu, row_ok);
      const float* c32 = reinterpret_cast<const float*>(cbase);
      // a full tile of a plain product (no C, no mirror, bf16 out by TMA
      // stores): a compact loop, away from the general one's many cases
      const bool plain_tile = dstg && !has_c && !p.sym && !adam && !apply && p.diag == 0.f;
      if (plain_tile) {
#pragma unroll 1
        for (int cc = 0; cc < BN; cc += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + cc, v);
          tmem_ld_wait();
          float x[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = alpha * __uint_as_float(v[i]);
          if (lane == 0) bulk_wait_read();         // the previous block's store has read the slot
          __syncwarp();
          stage_rows_tma(stg, nullptr, lane, x);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmD, stg, n0 + cc, r0, b);
            bulk_commit();
          }
        }
      }
      // a full tile of a symmetric product (Gram; polynomial with C by TMA
      // in slots 2 and 3): blocks on or above the diagonal, each stored with
      // its mirror image (a diagonal block symmetrised in place)
      const bool sym_tile = dstg && p.sym && !adam && !apply;
      if (sym_tile) {
        int kq = 0;
#pragma unroll 1
        for (int cc = cc_begin; cc < BN; cc += 32, ++kq) {
          const int c0 = n0 + cc;
          const bool dg = c0 == r0;
          uint32_t v[32];
          tmem_ld32(taddr + cc, v);
          tmem_ld_wait();
          float x[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = alpha * __uint_as_float(v[i]);
          if (ctma) {
            const int bi = 2 + (kq & 1);
            mbar_wait(&cb[bi], (cph >> bi) & 1u, abort_flag, p.status, DEV_TIMEOUT_ACC_FULL);
            cph ^= 1u << bi;
            cpend &= ~(1u << bi);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 w = *reinterpret_cast<const uint4*>(stg + 2048 * bi + stg_off(lane, u));
              const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws[j]));
                x[8 * u + 2 * j] = fmaf(beta, f.x, x[8 * u + 2 * j]);
                x[8 * u + 2 * j + 1] = fmaf(beta, f.y, x[8 * u + 2 * j + 1]);
              }
            }
            __syncwarp();                         // every lane has read the slot
            if (lane == 0) {
              fence_proxy_async_smem();
              if (cc + 64 < BN) issue_c(bi, cc + 64);
            }
          }
          if (dg && p.diag != 0.f) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c0 + i == r) x[i] += p.diag;
          }
          if (lane == 0) bulk_wait_read();         // the previous block's stores have read slots 0 and 1
          __syncwarp();
          stage_rows_tma(stg, stg + 2048, lane, x);
          if (dg) {
            __syncwarp();
            symmetrize_staged(stg, stg + 2048, lane);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmD, stg, c0, r0, b);
            if (!dg) tma_store_3d(&tmD, stg + 2048, r0, c0, b);
            bulk_commit();
          }
        }
      }
      int kk = 0;                                // 32-column blocks done in this tile
#pragma unroll 1
      for (int cc = (plain_tile || sym_tile) ? BN : cc_begin; cc < BN; cc += 32, ++kk) {
        uint4 ccur[4];
        if (cpre) {
#pragma unroll
          for (int j = 0; j < 4; ++j) ccur[j] = cnext[j];
          if (cc + 32 < BN) load_c(cc + 32);
        }
        float4 cf[8];
        if (cf32) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            cf[j] = *reinterpret_cast<const float4*>(c32 + (long long)(r0 + 4 * j + (lane >> 3)) * p.ldc + n0 + cc +
                                                     4 * (lane & 7));
        } else if (wvec) {
          // W rows r0 .. r0 + 31, columns n0 + cc .. + 31: eight 128-byte rows
          // per load.  W is touched once, so its loads and stores are
          // streaming (evict-first): the product's operands keep L2
#pragma unroll
          for (int j = 0; j < 8; ++j)
            cf[j] = __ldcs(reinterpret_cast<const float4*>(wbase + (long long)(r0 + 4 * j + (lane >> 3)) * ldw + n0 +
                                                           cc + 4 * (lane & 7)));
        } else if (wtr) {
          // transposed W: element (row r0 + lane, column n0 + cc + i) of the
          // product is W[n0 + cc + i][r0 + lane], one 128-byte row per load
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float* w = wbase + (long long)(n0 + cc + 4 * j) * ldw + r0 + lane;
            cf[j] = make_float4(__ldcs(w), __ldcs(w + ldw), __ldcs(w + 2 * ldw), __ldcs(w + 3 * ldw));
          }
        }
        uint32_t v[32];
        tmem_ld32(taddr + cc, v);
        tmem_ld_wait();
        const int c0 = n0 + cc;
        // warp-uniform: every lane holds a full row segment of plain bf16 output
        const bool all_in = __all_sync(0xffffffffu, row_ok && c0 + 32 <= p.N);
        const bool blk_full = all_in && (!p.sym || c0 >= r0 + 32);
        const bool fast = plain_bf16 && blk_full;
        const bool fast32 = plain_f32 && blk_full;
        const bool diag = p.sym && all_in && c0 == r0 && (plain_bf16 || plain_f32);
        if (fast || fast32 || diag || cf32 || (row_ok && c0 < p.N)) {
          const bool full = c0 + 32 <= p.N;
          float x[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = alpha * __uint_as_float(v[i]);
          if (adam) {
            // V <- b2 V + (1 - b2) G'^2 ;  Dbar = (M' / bc1) / (sqrt(V / bc2) + eps)
            float mr[32];
            load_row32(cbase, p.c_f32, (long long)r * p.ldc + c0, full ? 32 : p.N - c0, mr);
            float* vp = vbase + (long long)r * p.lde + c0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (full || c0 + i < p.N) {
                const float g = x[i];
                const float vn = fmaf(p.adam_b2, vp[i], (1.0f - p.adam_b2) * g * g);
                vp[i] = vn;
                x[i] = (mr[i] * p.adam_ibc1) / (sqrtf(vn * p.adam_ibc2) + p.adam_eps);
              }
            }
          } else if (cf32) {
            __syncwarp();                 // the previous block's reads of the staging rows are done
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<float4*>(stg + stg32_off(4 * j + (lane >> 3), lane & 7)) = cf[j];
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float4 w = *reinterpret_cast<const float4*>(stg + stg32_off(lane, u));
              x[4 * u] = fmaf(beta, w.x, x[4 * u]);
              x[4 * u + 1] = fmaf(beta, w.y, x[4 * u + 1]);
              x[4 * u + 2] = fmaf(beta, w.z, x[4 * u + 2]);
              x[4 * u + 3] = fmaf(beta, w.w, x[4 * u + 3]);
            }
          } else if (ctma) {
            const int bi = dtma ? (kk & 3) : 2 + (kk & 1);
            mbar_wait(&cb[bi], (cph >> bi) & 1u, abort_flag, p.status, DEV_TIMEOUT_ACC_FULL);
            cph ^= 1u << bi;
            cpend &= ~(1u << bi);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 w = *reinterpret_cast<const uint4*>(stg + 2048 * bi + stg_off(lane, u));
              const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws[j]));
                x[8 * u + 2 * j] = fmaf(beta, f.x, x[8 * u + 2 * j]);
                x[8 * u + 2 * j + 1] = fmaf(beta, f.y, x[8 * u + 2 * j + 1]);
              }
            }
            if (!dtma) {
              __syncwarp();               // every lane has read the buffer
              if (lane == 0) {
                fence_proxy_async_smem();
                if (cc + 64 < BN) issue_c(bi, cc + 64);
              }
            }
          } else if (cpre) {
            __syncwarp();                 // the previous block's reads of stc are done
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<uint4*>(stc + stg_off(8 * j + (lane >> 2), lane & 3)) = ccur[j];
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 w = *reinterpret_cast<const uint4*>(stc + stg_off(lane, u));
              const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws[j]));
                x[8 * u + 2 * j] = fmaf(beta, f.x, x[8 * u + 2 * j]);
                x[8 * u + 2 * j + 1] = fmaf(beta, f.y, x[8 * u + 2 * j + 1]);
              }
            }
          } else if (has_c) {
            float c[32];
            load_row32(cbase, p.c_f32, (long long)r * p.ldc + c0, full ? 32 : p.N - c0, c);
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = fmaf(beta, c[i], x[i]);
          }
          if (p.diag != 0.f && c0 < r0 + 32 && r0 < c0 + 32) {
            // the block meets the diagonal: lane r adds to its element (r, r)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c0 + i == r) x[i] += p.diag;
          }
          if (apply) {
            // O = bf16(x), as the plain output would hold it; then the Muon
            // apply W <- decay W - step O in fp32
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
            if (wvec) {
              __syncwarp();               // the previous block's reads of the staging rows are done
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(stg + stg32_off(4 * j + (lane >> 3), lane & 7)) = cf[j];
              __syncwarp();
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const float4 w = *reinterpret_cast<const float4*>(stg + stg32_off(lane, u));
                x[4 * u] = fmaf(p.ap_decay, w.x, -wstep * x[4 * u]);
                x[4 * u + 1] = fmaf(p.ap_decay, w.y, -wstep * x[4 * u + 1]);
                x[4 * u + 2] = fmaf(p.ap_decay, w.z, -wstep * x[4 * u + 2]);
                x[4 * u + 3] = fmaf(p.ap_decay, w.w, -wstep * x[4 * u + 3]);
              }
              stage_store32_f32(stg, lane, x, wbase + (long long)r0 * ldw + c0, nullptr, ldw, true);
            } else if (wtr) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                float* w = wbase + (long long)(c0 + 4 * j) * ldw + r0 + lane;
                __stcs(w, fmaf(p.ap_decay, cf[j].x, -wstep * x[4 * j]));
                __stcs(w + ldw, fmaf(p.ap_decay, cf[j].y, -wstep * x[4 * j + 1]));
                __stcs(w + 2 * ldw, fmaf(p.ap_decay, cf[j].z, -wstep * x[4 * j + 2]));
                __stcs(w + 3 * ldw, fmaf(p.ap_decay, cf[j].w, -wstep * x[4 * j + 3]));
              }
            } else if (row_ok) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                if (c0 + i < p.N) {
                  float* w = wbase + (wtall ? (long long)(c0 + i) * ldw + r : (long long)r * ldw + c0 + i);
                  *w = fmaf(p.ap_decay, *w, -wstep * x[i]);
                }
              }
            }
          } else if (dstg && (fast || (diag && plain_bf16))) {
            // the previous block's stores have read the staging slots
            if (lane == 0) bulk_wait_read();
            __syncwarp();
            uint8_t* own = stg;
            uint8_t* mir = stg + 2048;
            stage_rows_tma(own, (p.sym || diag) ? mir : nullptr, lane, x);
            if (diag) {
              __syncwarp();
              symmetrize_staged(own, mir, lane);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmD, own, c0, r0, b);
              if (p.sym && !diag) tma_store_3d(&tmD, mir, r0, c0, b);
              bulk_commit();
            }
          } else if (diag) {
            if (plain_f32)
              stage_store32_f32_diag(stg, lane, x, reinterpret_cast<float*>(dbase) + (long long)r0 * p.ldd + c0, p.ldd);
            else
              stage_store32_diag(stg, lane, x, reinterpret_cast<__nv_bfloat16*>(dbase) + (long long)r0 * p.ldd + c0,
                                 p.ldd);
          } else if (fast32) {
            float* d32 = reinterpret_cast<float*>(dbase);
            stage_store32_f32(stg, lane, x, d32 + (long long)r0 * p.ldd + c0,
                              p.sym ? d32 + (long long)c0 * p.ldd + r0 : nullptr, p.ldd);
          } else if (fast && dtma) {
            // this lane's row of bf16 output over the row of C it read, then
            // one TMA store of the block; the slot of the previous block is
            // free once its store has read it and takes the C block three
            // ahead
            uint8_t* slot = stg + 2048 * (kk & 3);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint32_t w[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(x[8 * u + 2 * j], x[8 * u + 2 * j + 1]);
                w[j] = *reinterpret_cast<const uint32_t*>(&h);
              }
              *reinterpret_cast<uint4*>(slot + stg_off(lane, u)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmD, slot, n0 + cc, r0, b);
              bulk_commit();
              bulk_wait_read_but1();
              if (cc + 96 < BN) issue_c((kk + 3) & 3, cc + 96);
            }
          } else if (fast) {
            __nv_bfloat16* d16 = reinterpret_cast<__nv_bfloat16*>(dbase);
            stage_store32(stg, lane, x, d16 + (long long)r0 * p.ldd + c0,
                          p.sym ? d16 + (long long)c0 * p.ldd + r0 : nullptr, p.ldd);
          } else if (!p.sym) {
            store_row(p, dbase, (long long)r * p.ldd + c0, full ? 32 : p.N - c0, 0, x);
          } else if (c0 + 31 >= r) {
            // upper part of this row chunk: store it, then its mirror image
            const int lo = c0 >= r ? 0 : r - c0;          // first column with c >= r
            const int hi = full ? 32 : p.N - c0;
            store_row(p, dbase, (long long)r * p.ldd + c0, hi, lo, x);
            store_mirror(p, dbase, r, c0, lo, hi, x);
          }
        }
      }
      tc_fence_before();
      if constexpr (PAIR) mbar_arrive_cluster(acc ? acc_empty_cl1 : acc_empty_cl0);
      else mbar_arrive(&acc_empty[acc]);
    }
    // C blocks requested for a tile that was abandoned must land before
    // exit, and the output stores must be complete
    if (lane == 0) {
      for (int bi = 0; bi < 4; ++bi)
        if ((cpend >> bi) & 1u) mbar_wait_drain(&cb[bi], (cph >> bi) & 1u, p.status);
      bulk_wait_all();
    }
  }

  __syncthreads();
  // a pair: the peer's epilogue has read its accumulators and the even CTA's
  // MMAs (which read the peer's shared memory) have drained
  if constexpr (PAIR) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    else tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace mo
