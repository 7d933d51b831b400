// Host side of the tcgen05 GEMM: TMA descriptor encoding and launch.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "gemm.cuh"
#include "profile.h"
#include "runtime.h"

// products with K up to this many columns use two sets of epilogue warps
#ifndef MO_EPI2_MAX_K
#define MO_EPI2_MAX_K 2048
#endif
// 1: short-K products with two epilogue sets take 128-wide tiles and four
// accumulators
#ifndef MO_SHORTK_NARROW
#define MO_SHORTK_NARROW 0
#endif
// 1: short-K products with two epilogue sets and more than one row tile run
// on CTA pairs (256 x 256 tiles, each CTA staging half of B: a third fewer
// bytes from L2 per flop, the bound of these products)
#ifndef MO_SHORTK_PAIR
#define MO_SHORTK_PAIR 1
#endif
// 1: outputs of non-symmetric products with a TMA-read C leave by TMA stores
#ifndef MO_GEMM_DTMA
#define MO_GEMM_DTMA 1
#endif

namespace mo {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode_fn() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult qres;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) == cudaSuccess &&
      qres == cudaDriverEntryPointSuccess) {
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
}

// 4-D bf16 tensor map over `planes` x `batch` matrices of storage rows x cols
// (row stride ld, matrix stride bstride, plane stride pstride, all in
// elements); box = 64 x box_rows.
bool encode_bf16_4d(CUtensorMap* map, const void* ptr, long long rows, long long cols, long long ld,
                    long long bstride, int batch, long long pstride, int planes, int box_rows, bool f16 = false) {
  std::call_once(g_encode_once, load_encode_fn);
  if (g_encode == nullptr) return false;
  const long long bs = batch > 1 ? bstride : rows * ld;
  const long long ps = planes > 1 ? pstride : bs * batch;
  cuuint64_t dims[4] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch, (cuuint64_t)planes};
  cuuint64_t strides[3] = {(cuuint64_t)(ld * 2), (cuuint64_t)(bs * 2), (cuuint64_t)(ps * 2)};
  cuuint32_t box[4] = {64u, (cuuint32_t)box_rows, 1u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = g_encode(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                        const_cast<void*>(ptr), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over `batch` matrices rows x cols (row stride ld,
// matrix stride bstride, elements) read in 32 x 32 boxes with the 64-byte
// swizzle (the epilogue's C blocks).
bool encode_bf16_c(CUtensorMap* map, const void* ptr, long long rows, long long cols, long long ld,
                   long long bstride, int batch) {
  std::call_once(g_encode_once, load_encode_fn);
  if (g_encode == nullptr) return false;
  const long long bs = batch > 1 ? bstride : rows * ld;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(bs * 2)};
  cuuint32_t box[3] = {32u, 32u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int planes_of(const unsigned char* pat, int nseg) {
  int m = 0;
  for (int i = 0; i < nseg; ++i) m = pat[i] > m ? pat[i] : m;
  return m + 1;
}

// Row tiles per band of the tile order (see gemm_decode).  The plain column
// order re-reads the A panel of a matrix from DRAM once per wave of tiles
// when the panel does not fit in L2; bands of G row tiles read A once and
// the B panel once per band.  Bands are used when the estimate of DRAM bytes
// read drops by more than a third (symmetric products sweep about half of
// the columns per band and of the rows per wave).
int choose_band(int bm, int tiles_m, long long M, long long N, long long kseg, int pa, int pb, bool sym,
                long long tiles_per_mat, long long units) {
  const double budget = 48.0 * 1024 * 1024;         // A rows kept in the 126 MB L2
  const double row_bytes = (double)bm * kseg * pa * 2.0;
  const double a_bytes = (double)M * kseg * pa * 2.0;
  const double b_bytes = (double)N * kseg * pb * 2.0;
  if (a_bytes <= budget) return tiles_m;
  int g = (int)(budget / row_bytes);
  if (g < 1) g = 1;
  if (g >= tiles_m) return tiles_m;
  const int nb = (tiles_m + g - 1) / g;
  const double waves = (double)tiles_per_mat / (double)units;
  const double rereads = sym ? waves / 2 : waves;
  const double plain = b_bytes + a_bytes * (rereads > 1.0 ? rereads : 1.0);
  const double banded = a_bytes + b_bytes * (sym ? (nb + 1) / 2.0 : (double)nb);
  return banded * 1.5 < plain ? g : tiles_m;
}

template <int BN, int A_MN, int B_MN, bool PAIR = false, bool EPI2 = false>
cudaError_t launch_t(const GemmOp& op, int* status, cudaStream_t stream) {
  using Cfg = GemmCfg<BN, PAIR, EPI2>;
  constexpr int BM_T = PAIR ? 2 * GEMM_BM : GEMM_BM;
  CUtensorMap ta, tb, tc, td;
  std::memset(&tc, 0, sizeof(tc));
  std::memset(&td, 0, sizeof(td));
  const int nseg = op.nseg > 1 ? op.nseg : 1;
  if (nseg > 8 || (nseg > 1 && op.K % (nseg * GEMM_BK) != 0)) return cudaErrorInvalidValue;
  const long long kseg = op.K / nseg;
  const int pa = planes_of(op.pat_a, nseg), pb = planes_of(op.pat_b, nseg);
  const bool h = op.ab_f16 != 0;
  const bool ok_a = A_MN ? encode_bf16_4d(&ta, op.A, kseg, op.M, op.lda, op.strideA, op.batch, op.planeA, pa, 64, h)
                         : encode_bf16_4d(&ta, op.A, op.M, kseg, op.lda, op.strideA, op.batch, op.planeA, pa, GEMM_BM,
                                          h);
  const bool ok_b = B_MN ? encode_bf16_4d(&tb, op.B, kseg, op.N, op.ldb, op.strideB, op.batch, op.planeB, pb, 64, h)
                         : encode_bf16_4d(&tb, op.B, op.N, kseg, op.ldb, op.strideB, op.batch, op.planeB, pb,
                                          Cfg::BN_LOCAL, h);
  if (!ok_a || !ok_b) return cudaErrorInvalidValue;

  GemmParams p;
  p.M = op.M; p.N = op.N; p.K = op.K; p.batch = op.batch;
  p.bm = BM_T;
  p.tiles_m = (op.M + BM_T - 1) / BM_T;
  p.tiles_n = (op.N + BN - 1) / BN;
  p.sym = op.sym;
  p.alpha = op.alpha; p.beta = op.beta; p.scale = op.scale;
  p.alpha_pow = op.alpha_pow; p.beta_pow = op.beta_pow;
  p.C = op.C; p.ldc = op.ldc; p.strideC = op.strideC; p.c_f32 = op.c_f32;
  p.D = op.D; p.ldd = op.ldd; p.strideD = op.strideD; p.d_f32 = op.d_f32;
  p.status = status;
  p.c_tab = op.c_tab; p.d_tab = op.d_tab; p.e_tab = op.e_tab;
  p.epi = op.epi;
  p.adam_b2 = op.adam_b2; p.adam_ibc1 = op.adam_ibc1; p.adam_ibc2 = op.adam_ibc2; p.adam_eps = op.adam_eps;
  p.lde = op.lde; p.strideE = 0;
  p.nseg = nseg;
  p.kseg = (int)kseg;
  for (int i = 0; i < 8; ++i) { p.pat_a[i] = op.pat_a[i]; p.pat_b[i] = op.pat_b[i]; }
  p.d_split = op.d_split;
  p.d_plane = op.d_plane;
  p.skip = op.skip;
  p.ap_decay = op.ap_decay;
  p.ap_step[0] = op.ap_step[0];
  p.ap_step[1] = op.ap_step[1];
  p.ap_tall_from = op.ap_tall_from;
  p.ap_vec = op.ap_vec;
  p.ab_f16 = op.ab_f16;
  p.gate = op.gate;
  p.gate_n = op.gate_n;
  p.gate_idx = op.gate_idx;
  p.diag = op.diag_add;
  if (op.diag_add != 0.f && op.epi != EPI_AXPBY) return cudaErrorInvalidValue;
  if (op.epi == EPI_APPLY && (op.sym || op.e_tab == nullptr || op.d_f32 || op.d_split))
    return cudaErrorInvalidValue;
  // a strided bf16 C of the plain (or Muon apply) epilogue is read by TMA
  p.c_tma = 0;
  if (op.C != nullptr && op.c_tab == nullptr && !op.c_f32 && (op.epi == EPI_AXPBY || op.epi == EPI_APPLY) &&
      !op.d_f32 && !op.d_split &&
      (op.batch == 1 || op.strideC % 8 == 0) && op.ldc % 8 == 0 &&
      (reinterpret_cast<uintptr_t>(op.C) & 15) == 0) {
    if (!encode_bf16_c(&tc, op.C, op.M, op.N, op.ldc, op.strideC, op.batch)) return cudaErrorInvalidValue;
    p.c_tma = 1;
  }
  // a strided bf16 D of a plain product whose C (if any) comes by TMA is
  // written by TMA stores: from the slots its C blocks arrived in
  // (non-symmetric with C), else from staging slots
  p.d_tma = 0;
  if ((p.c_tma || (op.C == nullptr && op.c_tab == nullptr)) && op.epi == EPI_AXPBY && !op.d_f32 && !op.d_split && op.d_tab == nullptr &&
      op.D != nullptr &&
      (op.batch == 1 || op.strideD % 8 == 0) && op.ldd % 8 == 0 && (reinterpret_cast<uintptr_t>(op.D) & 15) == 0 &&
      MO_GEMM_DTMA) {
    if (!encode_bf16_c(&td, op.D, op.M, op.N, op.ldd, op.strideD, op.batch)) return cudaErrorInvalidValue;
    p.d_tma = 1;
  }

  auto kern = gemm_bf16_kernel<BN, A_MN, B_MN, PAIR, EPI2>;
  cudaError_t ea = ensure_smem_attr(reinterpret_cast<const void*>(kern), Cfg::SMEM_BYTES);
  if (ea != cudaSuccess) return ea;
  // tiles enumerated per matrix: all, or those touching the upper triangle
  long long tiles = 0;
  for (int tn = 0; tn < p.tiles_n; ++tn) {
    if (!p.sym) { tiles += p.tiles_m; continue; }
    const int r = (tn * BN + BN - 1) / BM_T + 1;
    tiles += r < p.tiles_m ? r : p.tiles_m;
  }
  p.tiles_per_mat = (int)tiles;
  const long long total = tiles * p.batch;
  if (total >= (1ll << 31)) return cudaErrorInvalidValue;
  // one CTA per SM; a pair per two SMs
  const long long units = PAIR ? device_sm_count() / 2 : device_sm_count();
  p.band = op.band > 0 ? op.band
                       : choose_band(BM_T, p.tiles_m, op.M, op.N, kseg, pa, pb, op.sym != 0, tiles, units);
  const int grid = (int)((total < units ? total : units) * (PAIR ? 2 : 1));
  if (grid <= 0) return cudaSuccess;
  // executed tensor-core flops: computed tiles x 128 x BN x padded K x 2
  const double flops = 2.0 * tiles * p.batch * BM_T * BN * (double)round_up(p.K, GEMM_BK);
  ProfScope prof(op.kind, stream, flops);
  return launch_pdl(kern, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM_BYTES, stream, PAIR, ta, tb, tc, td, p);
}

}  // namespace

cudaError_t ensure_smem_attr(const void* func, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({dev, func})) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.insert({dev, func});
  return e;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

namespace {
// CTA pairs (256 x 256 tiles over two SMs) for products with more than 128
// rows and N > 128: for short K with two epilogue sets, for products that
// ask for them (GemmOp::pair, the SOAP products), and for all when
// MO_GEMM_PAIR=1 is set in the environment.  They do the same work in fewer
// cycles, but under the B200's power cap the clock drops by as much or more
// on the Newton-Schulz chain's long-K products (measured), so single-CTA
// 128 x 256 tiles are the default there.
bool pairs_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("MO_GEMM_PAIR");
    return v != nullptr && v[0] == '1';
  }();
  return on;
}
}  // namespace

cudaError_t launch_gemm(const GemmOp& op, int* status, cudaStream_t stream) {
  if (op.M <= 0 || op.N <= 0 || op.K <= 0 || op.batch <= 0) return cudaSuccess;
  // 128-wide N tiles when N is small, or when the product has too few
  // 128 x 256 tiles to occupy a quarter of the SMs (short launches are bound
  // by the per-tile epilogue, which narrower tiles spread over more SMs);
  // 256 otherwise
  const long long wide_tiles = (long long)((op.M + GEMM_BM - 1) / GEMM_BM) * ((op.N + 255) / 256) * op.batch;
  bool narrow = op.N <= 128 || wide_tiles * 4 < device_sm_count();
  // two sets of epilogue warps when K is short and every CTA gets at least
  // two tiles: a tile's main loop (K / 64 steps) is then no longer than one
  // set's epilogue, which would otherwise leave the tensor pipe idle
  // between tiles
  const int bn = narrow ? 128 : 256;
  const long long tiles = (long long)((op.M + GEMM_BM - 1) / GEMM_BM) * ((op.N + bn - 1) / bn) * op.batch;
  const bool epi2 = op.K <= MO_EPI2_MAX_K && tiles >= 2LL * device_sm_count();
  if (!narrow && op.M > GEMM_BM && (pairs_enabled() || op.pair || (epi2 && MO_SHORTK_PAIR))) {
    switch ((epi2 ? 4 : 0) | (op.a_mn ? 2 : 0) | (op.b_mn ? 1 : 0)) {
      case 0: return launch_t<256, 0, 0, true>(op, status, stream);
      case 1: return launch_t<256, 0, 1, true>(op, status, stream);
      case 2: return launch_t<256, 1, 0, true>(op, status, stream);
      case 3: return launch_t<256, 1, 1, true>(op, status, stream);
      case 4: return launch_t<256, 0, 0, true, true>(op, status, stream);
      case 5: return launch_t<256, 0, 1, true, true>(op, status, stream);
      case 6: return launch_t<256, 1, 0, true, true>(op, status, stream);
      default: return launch_t<256, 1, 1, true, true>(op, status, stream);
    }
  }
  // with two epilogue sets, 128-wide tiles get four accumulators: a tile's
  // epilogue then no longer holds up the main loop of the tile after next
  if (epi2 && MO_SHORTK_NARROW) narrow = true;
  const int sel = (epi2 ? 8 : 0) | (narrow ? 4 : 0) | (op.a_mn ? 2 : 0) | (op.b_mn ? 1 : 0);
  switch (sel) {
    case 0: return launch_t<256, 0, 0>(op, status, stream);
    case 1: return launch_t<256, 0, 1>(op, status, stream);
    case 2: return launch_t<256, 1, 0>(op, status, stream);
    case 3: return launch_t<256, 1, 1>(op, status, stream);
    case 4: return launch_t<128, 0, 0>(op, status, stream);
    case 5: return launch_t<128, 0, 1>(op, status, stream);
    case 6: return launch_t<128, 1, 0>(op, status, stream);
    case 7: return launch_t<128, 1, 1>(op, status, stream);
    case 8: return launch_t<256, 0, 0, false, true>(op, status, stream);
    case 9: return launch_t<256, 0, 1, false, true>(op, status, stream);
    case 10: return launch_t<256, 1, 0, false, true>(op, status, stream);
    case 11: return launch_t<256, 1, 1, false, true>(op, status, stream);
    case 12: return launch_t<128, 0, 0, false, true>(op, status, stream);
    case 13: return launch_t<128, 0, 1, false, true>(op, status, stream);
    case 14: return launch_t<128, 1, 0, false, true>(op, status, stream);
    default: return launch_t<128, 1, 1, false, true>(op, status, stream);
  }
}

}  // namespace mo
