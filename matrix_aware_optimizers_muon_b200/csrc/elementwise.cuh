// Elementwise / reduction kernels of the Muon path (HBM-bound).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace mo {

constexpr int EW_MAX = 256;     // matrices per launch (pointer table in kernel params)
constexpr int EW_TILE = 64;     // 64 x 64 element tiles
constexpr int EW_THREADS = 256;

// Per-launch pointer table.  All matrices of one launch share the oriented
// shape (mp x np, mp <= np); each may be stored as mp x np or np x mp.
struct EwTable {
  const float* in[EW_MAX];      // G (Muon) or the input matrix (plain NS)
  float* mom[EW_MAX];           // momentum buffer (Muon) or nullptr
  float* out[EW_MAX];           // W (Muon apply) or the fp32 output (plain NS)
  int32_t* flag[EW_MAX];        // optional nonfinite flag slot
  unsigned char tall[EW_MAX];   // stored as np x mp (transposed when oriented)
};

struct PrepArgs {
  int count;                  // matrices in this launch
  int mp, np;                 // oriented shape
  int tiles_r, tiles_c;       // 64x64 tiles of the stored matrix (rows, cols)
  float beta;                 // momentum
  int mode;                   // 0: plain (N = in), 1: Muon momentum step
  int nesterov, ema;
  int vec;                    // float4 path allowed (cols % 4 == 0, 16-byte aligned)
  __nv_bfloat16* X;           // oriented bf16 output, [count][mp][ldx]
  long long ldx, xstride;
  float* partial;             // [count][tiles] partial sums of N^2
};

struct FinalizeArgs {
  int count, tiles;
  float eps;
  const float* partial;
  float* inv;                 // 1 / (||N||_F + eps) per matrix
};

struct ApplyArgs {
  int count;
  int mp, np;
  int tiles_r, tiles_c;
  int mode;                   // 0: out = O (plain NS), 1: W = decay W - step O
  float decay, step;
  int vec;
  const __nv_bfloat16* X;
  long long ldx, xstride;
};

void launch_prep(const EwTable& t, const PrepArgs& a, cudaStream_t s);
void launch_finalize(const EwTable& t, const FinalizeArgs& a, cudaStream_t s);
void launch_apply(const EwTable& t, const ApplyArgs& a, cudaStream_t s);

}  // namespace mo
