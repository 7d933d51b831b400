// Fused Newton-Schulz (and Muon step) for small matrices: m' <= 128 and
// n' <= 256 after orientation.  One persistent CTA walks over the matrices;
// for each it keeps X (m' x n') and A = X X^T in shared memory (128-byte-
// swizzled K-major tiles, zero padded to 128 x 256 / 128 x 128), with P =
// b A + c A A written over A row by row once A A is in tensor memory, and
// the fp32 products in tensor memory, so HBM sees only the inputs and the
// outputs.  The arithmetic and rounding points are those of the
// batched path: N = G + beta B (Muon) or the input, Nb = bf16(N),
// inv = 1 / (||N||_F + eps) applied in fp32 inside iteration 0, every stored
// iterate rounded to bf16.
//
// Warps 0-3: workers, thread t owns row t of the oriented matrix (loads,
// norms, tcgen05.ld epilogues, stores).  Warp 4: TMEM allocation and the
// single-thread tcgen05.mma issue.
#include <cuda_bf16.h>

#include "ns_small.cuh"
#include "profile.h"
#include "ptx.cuh"
#include "runtime.h"

namespace mo {

namespace {

constexpr int SM_THREADS = 160;
constexpr int CHUNK = 128 * 128;                 // bytes of one 64-column chunk of 128 rows
constexpr int A_BYTES = 2 * CHUNK;               // 128 x 128
constexpr int VU = 4;                            // float4 accesses in flight per thread
constexpr int STAGE_F = A_BYTES / 4;             // floats of one bulk-copy round (the A region)
constexpr int LU = 2, SU = 2;                    // float4 per thread per batch: bulk load / store rounds

// X holds npad / 64 chunks and A (then P) 2: with npad <= 128 three CTAs fit
// on one SM (shared memory), with 128 tensor-memory columns each.
constexpr int smem_bytes(int npad) { return (npad / 64) * CHUNK + A_BYTES + 1024 + 256; }
// tensor-memory columns: the widest product (128 for A and A A, npad for P X)
__host__ __device__ constexpr uint32_t tmem_cols(int npad) { return npad <= 128 ? 128u : 256u; }

// byte offset of element (r, c) inside a swizzled chunked tile
__device__ __forceinline__ uint32_t swz(int r, int c) {
  const int chunk = c >> 6, cc = c & 63;
  return (uint32_t)(chunk * CHUNK + r * 128 + ((((cc >> 3) ^ (r & 7))) << 4) + ((cc & 7) << 1));
}

// byte offset of the 16-byte unit holding columns [8u, 8u + 8) of row r
__device__ __forceinline__ uint32_t swz_unit(int r, int u) {
  const int chunk = u >> 3, uu = u & 7;
  return (uint32_t)(chunk * CHUNK + r * 128 + ((uu ^ (r & 7)) << 4));
}

// named barrier 1 over the four worker warps, returning whether v held on
// every worker thread
__device__ __forceinline__ bool workers_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// K-major descriptor of a chunked tile, for the k-th 16-wide K step
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int k) {
  return smem_desc_sw128(base + (k >> 2) * CHUNK + (k & 3) * 32, 16, 1024);
}

// MN-major descriptor (B = X with K = rows, N = columns), k-th 16-row K step
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int k) {
  return smem_desc_sw128(base + k * 2048, CHUNK, 1024);
}

__device__ __forceinline__ void store_unit(uint8_t* tile, int r, int u, const float (&x)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
    w[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(tile + swz_unit(r, u)) = make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void unpack_unit(const uint4 v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
    x[2 * j] = f.x;
    x[2 * j + 1] = f.y;
  }
}

// BULK: the matrices go through the bulk-copy path (a separate instantiation
// keeps each variant's register allocation to its own paths)
template <bool BULK>
__global__ void __launch_bounds__(SM_THREADS, 3) ns_small_kernel(const SmallArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int np = a.tall ? a.rows : a.cols;      // oriented cols (<= 256)
  const int npad = (np + 63) & ~63;             // K of the Gram, N of the update
  const int xbytes = (npad >> 6) * CHUNK;
  uint8_t* X = smem;
  uint8_t* A = smem + xbytes;                   // A, then P over it
  uint8_t* P = A;
  const uint32_t TMEM_COLS = tmem_cols(npad);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(A + A_BYTES);
  uint64_t* work_bar = mma_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(work_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(tmem_slot + 4);      // [4] warp partials
  uint64_t* load_bar = mma_bar + 8;                          // bulk copies into the A region

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
  const uint32_t idesc_g = idesc_bf16_f32(128, 128, 0, 0);
  const uint32_t idesc_u = idesc_bf16_f32(128, npad, 0, 1);

  if (tid == 0) {
    mbar_init(mma_bar, 1);
    mbar_init(work_bar, 128);
    mbar_init(load_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();                         // the prologue touched no global memory
  pdl_trigger();
  const uint32_t sX = smem_u32(X), sA = smem_u32(A), sP = smem_u32(P);

  uint32_t mma_phase = 0, work_phase = 0, load_phase = 0;
  uint32_t ncommit = 0;                          // MMA thread: commits issued so far
  bool load_pending = false;                     // thread 0: a bulk load not yet waited for
  uint32_t pend_parity = 0;                      // ... and the phase parity it completes
  bool ok = true;
  // Matrices of at most 64 KB (n' <= 128) with 16-byte rows move through the
  // A region (free while a matrix is loaded and stored) by bulk copies of up
  // to 32 KB per round: one memory latency per round, not one per float4
  // batch of each thread.  Thread 0 issues the copies.
  // the oriented matrix fills the 128 x npad tile: no padding to clear
  const int mo_rows = a.tall ? a.cols : a.rows;
  const bool full_tile = mo_rows == 128 && np == npad;
  for (int mat = blockIdx.x; mat < a.count && ok; mat += gridDim.x) {
    if (warp < 4) {
      // ---- load: momentum, Nesterov, bf16 cast into X (oriented), norm
      // (padding of the previous matrix may hold non-finite values: cleared
      // for every matrix that does not fill the tile)
      if (!full_tile) {
        for (int e = tid; e < xbytes / 16; e += 128) reinterpret_cast<uint4*>(X)[e] = make_uint4(0, 0, 0, 0);
        __syncwarp();
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      const float* G = a.in[mat];
      float* B = a.mom ? a.mom[mat] : nullptr;
      const int total = a.rows * a.cols;
      float ss = 0.f;
      if (BULK && a.mode == 0) {
        // plain NS: 16 float4 loads in flight per thread, straight into
        // registers (no staging traffic in the shared memory the SM's CTAs
        // share): two rounds for a 128 x 128 matrix
        constexpr int RU = 16;
        const float4* G4 = reinterpret_cast<const float4*>(G);
        const int total4 = total >> 2;
        for (int e0 = tid; e0 < total4; e0 += 128 * RU) {
          float4 g[RU];
#pragma unroll
          for (int u = 0; u < RU; ++u) {
            const int e = e0 + u * 128;
            g[u] = e < total4 ? __ldg(G4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < RU; ++u) {
            const int e4 = e0 + u * 128;
            if (e4 >= total4) break;
            const float nv[4] = {g[u].x, g[u].y, g[u].z, g[u].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) ss = fmaf(nv[j], nv[j], ss);
            const int e = 4 * e4;
            const int r = (int)__umulhi((uint32_t)e, a.cols_magic), c = e - r * a.cols;
            if (!a.tall) {
              const __nv_bfloat162 lo = __floats2bfloat162_rn(nv[0], nv[1]);
              const __nv_bfloat162 hi = __floats2bfloat162_rn(nv[2], nv[3]);
              *reinterpret_cast<uint2*>(X + swz(r, c)) =
                  make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<__nv_bfloat16*>(X + swz(c + j, r)) = __float2bfloat16_rn(nv[j]);
            }
          }
        }
      } else if constexpr (BULK) {
        // per round: `per` floats of G (and of B in Muon mode) into A
        const int per = a.mode == 1 ? STAGE_F / 2 : STAGE_F;
        const float* sg = reinterpret_cast<const float*>(A);
        float* sb = reinterpret_cast<float*>(A) + per;
        for (int base = 0; base < total; base += per) {
          const int cnt = total - base < per ? total - base : per;     // a multiple of 4
          if (tid == 0) {
            fence_async_smem();                  // this thread's earlier accesses of A come first
            bulk_wait_read();                    // the previous output's copies have read A
            mbar_arrive_expect_tx(load_bar, (uint32_t)cnt * 4u * (a.mode == 1 ? 2u : 1u));
            bulk_load(A, G + base, (uint32_t)cnt * 4u, load_bar);
            if (a.mode == 1) bulk_load(sb, B + base, (uint32_t)cnt * 4u, load_bar);
            load_pending = true;
            pend_parity = load_phase;
          }
          // a failed wait leaves the values undefined but keeps every
          // barrier of the worker warps in step (the status word has the error)
          const bool got = mbar_wait(load_bar, load_phase, abort_flag, a.status, DEV_TIMEOUT_FULL);
          ok = ok && got;
          if (tid == 0 && got) load_pending = false;
          load_phase ^= 1u;
          // batches of LU float4 per thread, every load of a batch issued
          // before its X stores (the two regions alias for the compiler)
          for (int e40 = tid; e40 < (cnt >> 2); e40 += 128 * LU) {
            float4 gq[LU], bq[LU];
#pragma unroll
            for (int u = 0; u < LU; ++u) {
              const int e4 = e40 + 128 * u;
              if (e4 < (cnt >> 2)) {
                gq[u] = reinterpret_cast<const float4*>(sg)[e4];
                if (a.mode == 1) bq[u] = reinterpret_cast<const float4*>(sb)[e4];
              }
            }
#pragma unroll
            for (int u = 0; u < LU; ++u) {
            const int e4 = e40 + 128 * u;
            if (e4 >= (cnt >> 2)) break;
            float gv[4] = {gq[u].x, gq[u].y, gq[u].z, gq[u].w}, nv[4];
            float bv[4] = {0.f, 0.f, 0.f, 0.f};
            if (a.mode == 1) { bv[0] = bq[u].x; bv[1] = bq[u].y; bv[2] = bq[u].z; bv[3] = bq[u].w; }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float n = gv[j];
              if (a.mode == 1) {
                const float bn = a.ema ? fmaf(a.beta, bv[j], (1.0f - a.beta) * gv[j]) : fmaf(a.beta, bv[j], gv[j]);
                bv[j] = bn;
                n = a.nesterov ? fmaf(a.beta, bn, gv[j]) : bn;
              }
              nv[j] = n;
              ss = fmaf(n, n, ss);
            }
            const int e = base + 4 * e4;
            if (a.mode == 1) *reinterpret_cast<float4*>(B + e) = make_float4(bv[0], bv[1], bv[2], bv[3]);
            const int r = (int)__umulhi((uint32_t)e, a.cols_magic), c = e - r * a.cols;
            if (!a.tall) {
              const __nv_bfloat162 lo = __floats2bfloat162_rn(nv[0], nv[1]);
              const __nv_bfloat162 hi = __floats2bfloat162_rn(nv[2], nv[3]);
              *reinterpret_cast<uint2*>(X + swz(r, c)) =
                  make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<__nv_bfloat16*>(X + swz(c + j, r)) = __float2bfloat16_rn(nv[j]);
            }
            }
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");     // A has been read: the next round may land
        }
      } else if (a.vec) {
        // float4 accesses, VU in flight per thread (cols % 4 == 0, 16-byte
        // aligned matrices): four consecutive columns of one row each
        const float4* G4 = reinterpret_cast<const float4*>(G);
        float4* B4 = reinterpret_cast<float4*>(B);
        const int total4 = total >> 2;
        for (int e0 = tid; e0 < total4; e0 += 128 * VU) {
          float4 g[VU], b[VU];
#pragma unroll
          for (int u = 0; u < VU; ++u) {
            const int e = e0 + u * 128;
            if (e < total4) {
              g[u] = __ldg(G4 + e);
              if (a.mode == 1) b[u] = B4[e];
            }
          }
#pragma unroll
          for (int u = 0; u < VU; ++u) {
            const int e = e0 + u * 128;
            if (e >= total4) break;
            float gv[4] = {g[u].x, g[u].y, g[u].z, g[u].w}, nv[4];
            float bv[4] = {0.f, 0.f, 0.f, 0.f};
            if (a.mode == 1) { bv[0] = b[u].x; bv[1] = b[u].y; bv[2] = b[u].z; bv[3] = b[u].w; }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float n = gv[j];
              if (a.mode == 1) {
                const float bn = a.ema ? fmaf(a.beta, bv[j], (1.0f - a.beta) * gv[j]) : fmaf(a.beta, bv[j], gv[j]);
                bv[j] = bn;
                n = a.nesterov ? fmaf(a.beta, bn, gv[j]) : bn;
              }
              nv[j] = n;
              ss = fmaf(n, n, ss);
            }
            if (a.mode == 1) B4[e] = make_float4(bv[0], bv[1], bv[2], bv[3]);
            const int r = (4 * e) / a.cols, c = 4 * e - r * a.cols;
            if (!a.tall) {
              const __nv_bfloat162 lo = __floats2bfloat162_rn(nv[0], nv[1]);
              const __nv_bfloat162 hi = __floats2bfloat162_rn(nv[2], nv[3]);
              *reinterpret_cast<uint2*>(X + swz(r, c)) =
                  make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
            } else {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<__nv_bfloat16*>(X + swz(c + j, r)) = __float2bfloat16_rn(nv[j]);
            }
          }
        }
      } else {
        for (int e = tid; e < total; e += 128) {
          const int r = e / a.cols, c = e - r * a.cols;
          const float g = G[e];
          float n = g;
          if (a.mode == 1) {
            const float bn = a.ema ? fmaf(a.beta, B[e], (1.0f - a.beta) * g) : fmaf(a.beta, B[e], g);
            B[e] = bn;
            n = a.nesterov ? fmaf(a.beta, bn, g) : bn;
          }
          ss = fmaf(n, n, ss);
          const int xr = a.tall ? c : r, xc = a.tall ? r : c;
          *reinterpret_cast<__nv_bfloat16*>(X + swz(xr, xc)) = __float2bfloat16_rn(n);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) red[warp] = ss;
      fence_async_smem();
      ok = workers_all(ok);                      // a failed load stops every worker warp
      const float norm = sqrtf(((red[0] + red[1]) + red[2]) + red[3]);
      const float inv = 1.0f / (norm + a.eps);
      if (tid == 0 && a.flag && a.flag[mat]) *a.flag[mat] = isfinite(norm) ? 0 : 1;
      tc_fence_before();
      mbar_arrive(work_bar);                     // X ready

      const int r = tid;                         // this thread's row
      const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
      for (int it = 0; it < a.steps && ok; ++it) {
        // ---- A = X X^T (scaled by inv^2 in iteration 0)
        ok = mbar_wait(mma_bar, mma_phase, abort_flag, a.status, DEV_TIMEOUT_ACC_FULL);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        mma_phase ^= 1u;
        tc_fence_after();
        const float ga = it == 0 ? inv * inv : 1.0f;
#pragma unroll 1
        for (int cc = 0; cc < 128; cc += 32) {
          uint32_t v[32];
          tmem_ld32(trow + cc, v);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = ga * __uint_as_float(v[8 * u + j]);
            store_unit(A, r, (cc >> 3) + u, x);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(work_bar);
        // ---- P = b A + c A A, over A: A A has been read into tensor
        // memory, and each thread reads and rewrites only its own row
        ok = mbar_wait(mma_bar, mma_phase, abort_flag, a.status, DEV_TIMEOUT_ACC_FULL);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        mma_phase ^= 1u;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 128; cc += 32) {
          uint32_t v[32];
          tmem_ld32(trow + cc, v);
          tmem_ld_wait();
          // the four units of A first (P is written over them)
          uint4 araw[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) araw[u] = *reinterpret_cast<const uint4*>(A + swz_unit(r, (cc >> 3) + u));
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float av[8], x[8];
            unpack_unit(araw[u], av);
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = fmaf(a.b, av[j], a.c * __uint_as_float(v[8 * u + j]));
            store_unit(P, r, (cc >> 3) + u, x);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(work_bar);
        // ---- X' = a X + P X   (iteration 0: inv (a Nb + P Nb))
        ok = mbar_wait(mma_bar, mma_phase, abort_flag, a.status, DEV_TIMEOUT_ACC_FULL);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        mma_phase ^= 1u;
        tc_fence_after();
        const float s_acc = it == 0 ? inv : 1.0f;
        const float s_x = it == 0 ? a.a * inv : a.a;
#pragma unroll 1
        for (int cc = 0; cc < npad; cc += 32) {
          uint32_t v[32];
          tmem_ld32(trow + cc, v);
          tmem_ld_wait();
          // the four units of X first (X' is written over them)
          uint4 xraw[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) xraw[u] = *reinterpret_cast<const uint4*>(X + swz_unit(r, (cc >> 3) + u));
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float xv[8], x[8];
            unpack_unit(xraw[u], xv);
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = fmaf(s_x, xv[j], s_acc * __uint_as_float(v[8 * u + j]));
            store_unit(X, r, (cc >> 3) + u, x);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(work_bar);
      }
      // ---- the last X is O (a failed wait skips the store; every worker
      // thread meets the consensus barrier, and every thread the block
      // barrier below, which ends the loop)
      ok = workers_all(ok);
      if (ok) {
        float* out = a.out[mat];
        if (BULK && a.mode == 1) {
          // rounds of 32 KB: fp32 O (or, in Muon mode, W <- decay W - step O
          // on W brought in by a bulk load) staged in A, then one bulk store
          float4* st4 = reinterpret_cast<float4*>(A);
          for (int base = 0; base < total; base += STAGE_F) {
            const int cnt = total - base < STAGE_F ? total - base : STAGE_F;
            if (a.mode == 1) {
              if (tid == 0) {
                fence_async_smem();
                bulk_wait_read();                // the previous round's store has read A
                mbar_arrive_expect_tx(load_bar, (uint32_t)cnt * 4u);
                bulk_load(A, out + base, (uint32_t)cnt * 4u, load_bar);
                load_pending = true;
                pend_parity = load_phase;
              }
              const bool got = mbar_wait(load_bar, load_phase, abort_flag, a.status, DEV_TIMEOUT_FULL);
              if (tid == 0 && got) load_pending = false;
              load_phase ^= 1u;
            } else if (base > 0) {
              if (tid == 0) bulk_wait_read();    // the previous round's store has read A
              asm volatile("bar.sync 1, 128;" ::: "memory");
            }
            // batches of SU float4 per thread: the X (and W) reads of a
            // batch before its staging stores
            for (int e40 = tid; e40 < (cnt >> 2); e40 += 128 * SU) {
              float o[SU][4];
              float4 wq[SU];
#pragma unroll
              for (int u = 0; u < SU; ++u) {
                const int e4 = e40 + 128 * u;
                if (e4 < (cnt >> 2)) {
                  const int e = base + 4 * e4;
                  const int rr = (int)__umulhi((uint32_t)e, a.cols_magic), c = e - rr * a.cols;
                  if (!a.tall) {
                    const uint2 v = *reinterpret_cast<const uint2*>(X + swz(rr, c));
                    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
                    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
                    o[u][0] = lo.x; o[u][1] = lo.y; o[u][2] = hi.x; o[u][3] = hi.y;
                  } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                      o[u][j] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(X + swz(c + j, rr)));
                  }
                  if (a.mode == 1) wq[u] = st4[e4];
                }
              }
#pragma unroll
              for (int u = 0; u < SU; ++u) {
                const int e4 = e40 + 128 * u;
                if (e4 >= (cnt >> 2)) break;
                if (a.mode == 1)
                  st4[e4] = make_float4(fmaf(a.decay, wq[u].x, -a.step * o[u][0]), fmaf(a.decay, wq[u].y, -a.step * o[u][1]),
                                        fmaf(a.decay, wq[u].z, -a.step * o[u][2]), fmaf(a.decay, wq[u].w, -a.step * o[u][3]));
                else
                  st4[e4] = make_float4(o[u][0], o[u][1], o[u][2], o[u][3]);
              }
            }
            fence_async_smem();                  // the staged values are visible to the copy
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (tid == 0) {
              bulk_store(out + base, A, (uint32_t)cnt * 4u);
              bulk_commit();
            }
          }
        } else if (a.vec) {
          float4* O4 = reinterpret_cast<float4*>(out);
          const int total4 = total >> 2;
          for (int e0 = tid; e0 < total4; e0 += 128 * VU) {
            float4 w[VU];
            if (a.mode == 1) {
#pragma unroll
              for (int u = 0; u < VU; ++u)
                if (e0 + u * 128 < total4) w[u] = O4[e0 + u * 128];
            }
#pragma unroll
            for (int u = 0; u < VU; ++u) {
              const int e = e0 + u * 128;
              if (e >= total4) break;
              const int r = (4 * e) / a.cols, c = 4 * e - r * a.cols;
              float o[4];
              if (!a.tall) {
                const uint2 v = *reinterpret_cast<const uint2*>(X + swz(r, c));
                const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
                const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
                o[0] = lo.x; o[1] = lo.y; o[2] = hi.x; o[3] = hi.y;
              } else {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  o[j] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(X + swz(c + j, r)));
              }
              if (a.mode == 1)
                O4[e] = make_float4(fmaf(a.decay, w[u].x, -a.step * o[0]), fmaf(a.decay, w[u].y, -a.step * o[1]),
                                    fmaf(a.decay, w[u].z, -a.step * o[2]), fmaf(a.decay, w[u].w, -a.step * o[3]));
              else
                O4[e] = make_float4(o[0], o[1], o[2], o[3]);
            }
          }
        } else {
          for (int e = tid; e < total; e += 128) {
            const int rr = e / a.cols, c = e - rr * a.cols;
            const int xr = a.tall ? c : rr, xc = a.tall ? rr : c;
            const float o = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(X + swz(xr, xc)));
            out[e] = a.mode == 1 ? fmaf(a.decay, out[e], -a.step * o) : o;
          }
        }
      }
    } else if (lane == 0) {
      // ---- MMA issuer: per iteration Gram, A A, P X
      for (int it = 0; it < a.steps && ok; ++it) {
        ok = mbar_wait(work_bar, work_phase, abort_flag, a.status, DEV_TIMEOUT_FULL);
        if (!ok) break;
        work_phase ^= 1u;
        tc_fence_after();
        for (int k = 0; k < npad / 16; ++k)
          tc_mma_f16(tmem, desc_k(sX, k), desc_k(sX, k), idesc_g, k != 0);
        tc_commit(mma_bar);
        ++ncommit;
        ok = mbar_wait(work_bar, work_phase, abort_flag, a.status, DEV_TIMEOUT_FULL);
        if (!ok) break;
        work_phase ^= 1u;
        tc_fence_after();
        for (int k = 0; k < 8; ++k)
          tc_mma_f16(tmem, desc_k(sA, k), desc_k(sA, k), idesc_g, k != 0);
        tc_commit(mma_bar);
        ++ncommit;
        ok = mbar_wait(work_bar, work_phase, abort_flag, a.status, DEV_TIMEOUT_FULL);
        if (!ok) break;
        work_phase ^= 1u;
        tc_fence_after();
        for (int k = 0; k < 8; ++k)
          tc_mma_f16(tmem, desc_k(sP, k), desc_mn(sX, k), idesc_u, k != 0);
        tc_commit(mma_bar);
        ++ncommit;
      }
      if (ok) {
        // the workers' last arrival (after the final X) closes this matrix
        ok = mbar_wait(work_bar, work_phase, abort_flag, a.status, DEV_TIMEOUT_FULL);
        work_phase ^= 1u;
      }
    }
    ok = __syncthreads_and(ok);
  }
  if (tid == 0) {
    // a bulk load whose wait gave up must land before the CTA exits, and
    // the output copies must be complete
    if (load_pending) mbar_wait_drain(load_bar, pend_parity, a.status);
    bulk_wait_all();
  }
  // drain: every MMA issued must finish before TMEM is released
  if (warp == 4 && lane == 0 && ncommit > 0) {
    tc_commit(mma_bar);
    mbar_wait_drain(mma_bar, ncommit & 1u, a.status);
  }
  __syncthreads();
  if (warp == 4) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

constexpr int UPLOAD_N = 960;       // 4 x 960 pointers = 30 KB of kernel parameters

struct TableUpload {
  int n;
  const void* p[4][UPLOAD_N];
};

__global__ void upload_tables_kernel(void** dst, int stride, const TableUpload u) {
  pdl_wait();                         // the previous launch may still read the tables
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < u.n)
    for (int t = 0; t < 4; ++t) dst[t * stride + i] = const_cast<void*>(u.p[t][i]);
}

}  // namespace

void launch_upload_tables(void** dst, int n, const void* const* in, const void* const* mom,
                          const void* const* out, const void* const* flag, cudaStream_t s) {
  for (int first = 0; first < n; first += UPLOAD_N) {
    TableUpload u;
    u.n = n - first < UPLOAD_N ? n - first : UPLOAD_N;
    for (int i = 0; i < u.n; ++i) {
      u.p[0][i] = in[first + i];
      u.p[1][i] = mom[first + i];
      u.p[2][i] = out[first + i];
      u.p[3][i] = flag[first + i];
    }
    ProfScope prof(PK_TABLES, s);
    launch_pdl(upload_tables_kernel, dim3((u.n + 127) / 128), dim3(128), 0, s, false, dst + first, n, u);
  }
}

cudaError_t launch_ns_small(const SmallArgs& args, int sm_count, cudaStream_t s) {
  SmallArgs a = args;
  // element index / cols by a multiply-high: exact for indices below 2^16
  // (a matrix here has at most 128 x 256 elements) and cols < 2^16
  a.cols_magic = a.cols > 1 ? (uint32_t)((((uint64_t)1 << 32) + (uint64_t)a.cols - 1) / (uint64_t)a.cols) : 0u;
  const int np = a.tall ? a.rows : a.cols;
  const int npad = (np + 63) & ~63;
  // matrices of at most 64 KB with rows of 16-byte multiples: bulk copies
  const bool bulk = a.vec && npad <= 128;
  auto kern = bulk ? ns_small_kernel<true> : ns_small_kernel<false>;
  cudaError_t ea = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem_bytes(SMALL_MAX_N));
  if (ea != cudaSuccess) return ea;
  const int smem = smem_bytes(npad);
  // as many CTAs per SM (up to three) as shared and tensor memory hold: one's
  // loads, stores and epilogues then overlap the others' tensor-core phases
  int per_sm = (228 * 1024) / (smem + 1024);
  const int by_tmem = (int)(512 / tmem_cols(npad));
  per_sm = per_sm < by_tmem ? per_sm : by_tmem;
  per_sm = per_sm > 3 ? 3 : (per_sm < 1 ? 1 : per_sm);
  const int grid = a.count < per_sm * sm_count ? a.count : per_sm * sm_count;
  ProfScope prof(PK_SMALL, s, 0.0);
  return launch_pdl(kern, dim3(grid), dim3(SM_THREADS), (size_t)smem, s, false, a);
}

}  // namespace mo
