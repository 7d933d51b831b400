// SOAP driver: one optimizer step with a per-step basis refresh.
//
// Phase 1 (per group of equal shape and sides):
//   prep:  M <- b1 M + (1-b1) G,  Gb = bf16(G), Mb = bf16(M)
//   EMAs:  L <- bs L + (1-bs) Gb Gb^T ; R <- bs R + (1-bs) Gb^T Gb
//          (symmetric tcgen05 products written into the caller's L / R)
// Phase 2 (per bucket of equal factor size k, all sides of all matrices):
//   the refresh Q <- qr(F Q) of qr.cuh: the power step as an fp16
//   two-plane product, then CholeskyQR passes (left-looking blocked
//   Cholesky of the Gram with the solve for Q in the same products), plain
//   or shifted per matrix as the conditioning needs, until the basis is
//   orthonormal -> Q (unique QR, diag(R) > 0) into the caller's Q and bf16(Q)
// Phase 3 (per group): rotations with two-plane bf16 operands (x = h + l,
//   three bf16 MMAs lh + hl + hh per product), Adam in the rotated basis
//   fused into the epilogue of the G' product, rotation back fused with
//   W <- (1 - lr wd) W - lr D.
// SOAP-Muon runs phase 1, the rotations with the stored bases (writing the
// preconditioned momentum P instead of applying), the Muon engine on P, and
// the refresh last.
#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "ns_plan.h"
#include "profile.h"
#include "qr.cuh"
#include "runtime.h"
#include "soap_kernels.cuh"
#include "soap_plan.h"

namespace mo {

namespace {

constexpr size_t AL = 1024;
size_t al(size_t x) { return (x + AL - 1) / AL * AL; }

// The refresh's pass loop as a CUDA graph: a conditional while node whose
// body is one pass ending in launch_qr_loop, so that only the passes a step
// needs are executed (a warm step needs two of the eight allowed).  One
// instantiated graph per (device, workspace, bucket layout), kept while the
// same workspace and shapes come back; its kernels hold workspace pointers
// only.
struct PassGraph {
  int dev = -1;
  const char* ws = nullptr;
  size_t cy = 0, lq = 0, dinv = 0, invd = 0, ctl = 0;
  int q = 0;
  long long kp = 0, k = 0;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};
std::mutex g_pass_graph_mu;
std::vector<PassGraph> g_pass_graphs;                  // most recent last, at most 16
constexpr size_t PASS_GRAPH_KEEP = 16;

cudaStream_t pass_capture_stream(int dev) {
  static cudaStream_t streams[64] = {};
  if (dev < 0 || dev >= 64) return nullptr;
  if (streams[dev] == nullptr && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess) {
    streams[dev] = nullptr;
    (void)cudaGetLastError();
  }
  return streams[dev];
}

// Launches the pass-loop graph of `key` on s, recording it first with
// `record(stream, handle)` when it is not cached.  Returns false (nothing
// launched, errors cleared) when a graph cannot be made, so that the caller
// launches the passes directly.
template <class Record>
bool launch_pass_graph(PassGraph key, Record&& record, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_pass_graph_mu);
  for (size_t i = 0; i < g_pass_graphs.size(); ++i) {
    const PassGraph& g = g_pass_graphs[i];
    if (g.dev == key.dev && g.ws == key.ws && g.cy == key.cy && g.lq == key.lq && g.dinv == key.dinv &&
        g.invd == key.invd && g.ctl == key.ctl && g.q == key.q && g.kp == key.kp && g.k == key.k) {
      if (cudaGraphLaunch(g.exec, s) == cudaSuccess) return true;
      // a graph that no longer launches (its context was reset) is dropped
      (void)cudaGetLastError();
      g_pass_graphs.erase(g_pass_graphs.begin() + (long)i);
      return false;
    }
  }
  cudaStream_t cs = pass_capture_stream(key.dev);
  if (cs == nullptr) return false;
  cudaGraph_t graph = nullptr;
  if (cudaGraphCreate(&graph, 0) != cudaSuccess) return (void)cudaGetLastError(), false;
  auto give_up = [&]() {
    cudaGraphDestroy(graph);
    (void)cudaGetLastError();
    return false;
  };
  cudaGraphConditionalHandle h;
  if (cudaGraphConditionalHandleCreate(&h, graph, 1u, cudaGraphCondAssignDefault) != cudaSuccess) return give_up();
  cudaGraphNodeParams np = {};
  np.type = cudaGraphNodeTypeConditional;
  np.conditional.handle = h;
  np.conditional.type = cudaGraphCondTypeWhile;
  np.conditional.size = 1;
  cudaGraphNode_t node;
  if (cudaGraphAddNode(&node, graph, nullptr, 0, &np) != cudaSuccess) return give_up();
  cudaGraph_t body = np.conditional.phGraph_out[0];
  if (cudaStreamBeginCaptureToGraph(cs, body, nullptr, nullptr, 0, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
    return give_up();
  pdl_off() = true;
  const cudaError_t er = record(cs, h);
  pdl_off() = false;
  cudaGraph_t captured = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(cs, &captured);
  if (er != cudaSuccess || ec != cudaSuccess) return give_up();
  cudaGraphExec_t exec = nullptr;
  if (cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) return give_up();
  key.graph = graph;
  key.exec = exec;
  if (g_pass_graphs.size() >= PASS_GRAPH_KEEP) {
    cudaGraphExecDestroy(g_pass_graphs.front().exec);
    cudaGraphDestroy(g_pass_graphs.front().graph);
    g_pass_graphs.erase(g_pass_graphs.begin());
  }
  g_pass_graphs.push_back(key);
  return cudaGraphLaunch(exec, s) == cudaSuccess || ((void)cudaGetLastError(), false);
}

// two-plane products: x = h + l, x y ~ lh + hl + hh (bf16 planes for the
// rotations, fp16 planes with ab_f16 for the refresh).  The small products
// are accumulated first and hh last: the tensor core's fp32 accumulation
// loses low-order bits of each addend that is small next to the running sum.
void set_planes2(GemmOp& g, long long planeA, long long planeB) {
  const unsigned char pa[3] = {1, 0, 0}, pb[3] = {0, 1, 0};
  g.nseg = 3;
  for (int i = 0; i < 3; ++i) { g.pat_a[i] = pa[i]; g.pat_b[i] = pb[i]; }
  g.planeA = planeA;
  g.planeB = planeB;
}

// Per group (equal shape and sides).  Operands of the rotations are two bf16
// planes (h, l) in buffers padded to multiples of 64 (zero padding, so the
// padded K contributes nothing): gp, mp_ [2][c][mpad][npad], tp (T and S),
// dp (Dbar), qlp [2][c][mpad][mpad], qrp [2][c][npad][npad]; mr is M' fp32.
struct Group {
  long long m, n, mpad, npad;
  bool left, right;
  std::vector<int> items;
  size_t gp, mpl, tp, mr, dp, qlp, qrp, tabs, pb;
};

struct Job {
  int item, group, pos;
  bool left;       // left factor (k = m) or right (k = n)
};

// Per bucket of equal factor side k (kp = k rounded up to 128): the stacked
// fp32 [C; Y] and fp16 planes [L; Q] of the refresh ([q][2 kp][kp] each, two
// planes), the diagonal-block inverses, column scales, the optional damping
// and the pass-control state.
struct Bucket {
  long long k, kp;
  std::vector<Job> jobs;
  size_t cy, lq, dinv, invd, damp, ctl;
};

struct Plan {
  std::vector<Group> groups;
  std::vector<Bucket> buckets;
  size_t total = 0;
};

// with_p: SOAP-Muon, which also needs an fp32 P (m x n) per matrix.
Plan make_plan(const std::vector<SoapItem>& items, bool with_p = false) {
  Plan P;
  std::map<std::tuple<long long, long long, bool, bool>, int> gid;
  for (int i = 0; i < (int)items.size(); ++i) {
    const mo_soap_mat& m = items[i].m;
    auto key = std::make_tuple((long long)m.rows, (long long)m.cols, m.L != nullptr, m.R != nullptr);
    auto it = gid.find(key);
    if (it == gid.end() || P.groups[it->second].items.size() >= (size_t)SOAP_MAXB) {
      Group g;
      g.m = m.rows; g.n = m.cols; g.left = m.L != nullptr; g.right = m.R != nullptr;
      g.mpad = round_up(g.m, 64); g.npad = round_up(g.n, 64);
      P.groups.push_back(g);
      gid[key] = (int)P.groups.size() - 1;
      it = gid.find(key);
    }
    P.groups[it->second].items.push_back(i);
  }
  size_t off = WS_HEADER;
  for (Group& g : P.groups) {
    const size_t c = g.items.size(), mn = (size_t)g.m * g.n, pn = (size_t)g.mpad * g.npad;
    g.gp = off; off += al(2 * c * pn * 2);
    g.mpl = off; off += al(2 * c * pn * 2);
    g.tp = off; off += al(2 * c * pn * 2);
    g.mr = off; off += al(c * mn * 4);
    g.dp = off; off += al(2 * c * pn * 2);
    g.qlp = off; off += g.left ? al(2 * c * g.mpad * g.mpad * 2) : 0;
    g.qrp = off; off += g.right ? al(2 * c * g.npad * g.npad * 2) : 0;
    g.tabs = off; off += al(5 * SOAP_MAXB * sizeof(void*));
    g.pb = off; off += with_p ? al(c * mn * 4) : 0;
  }
  std::map<long long, int> bid;
  for (int gi = 0; gi < (int)P.groups.size(); ++gi) {
    const Group& g = P.groups[gi];
    for (int side = 0; side < 2; ++side) {
      if (side == 0 && !g.left) continue;
      if (side == 1 && !g.right) continue;
      const long long k = side == 0 ? g.m : g.n;
      for (int pos = 0; pos < (int)g.items.size(); ++pos) {
        auto it = bid.find(k);
        if (it == bid.end() || P.buckets[it->second].jobs.size() >= (size_t)SOAP_MAXB) {
          Bucket b;
          b.k = k;
          b.kp = round_up(k, QR_B);
          P.buckets.push_back(b);
          bid[k] = (int)P.buckets.size() - 1;
          it = bid.find(k);
        }
        P.buckets[it->second].jobs.push_back({g.items[pos], gi, pos, side == 0});
      }
    }
  }
  for (Bucket& b : P.buckets) {
    const size_t q = b.jobs.size(), kk = (size_t)b.kp * b.kp;
    b.cy = off; off += al(q * 2 * kk * 4);
    b.lq = off; off += al(2 * q * 2 * kk * 2);
    b.dinv = off; off += al(q * QR_B * QR_B * 4);
    b.invd = off; off += al(q * b.kp * 4);
    b.damp = off; off += al(q * 4);
    b.ctl = off; off += al(qr_ctl_bytes((int)q));
  }
  P.total = off;
  return P;
}

template <typename T>
T* at(char* ws, size_t off) { return reinterpret_cast<T*>(ws + off); }

// Newton-Schulz scratch of SOAP-Muon (all matrices as one batch per shape),
// without the status header that the SOAP workspace already holds.
size_t ns_bytes_for(const std::vector<SoapItem>& items) {
  std::vector<int64_t> rows, cols;
  for (const SoapItem& it : items) { rows.push_back(it.m.rows); cols.push_back(it.m.cols); }
  size_t mn = 0, full = 0;
  ns_workspace(rows.data(), cols.data(), (int)rows.size(), &mn, &full);
  return full - WS_HEADER;
}

// SOAP-Muon's Newton-Schulz stage: P (preconditioned momentum, fp32 in the
// workspace) -> O -> W <- (1 - lr wd) W - lr s O.  The Muon engine runs with
// momentum 0 on P (B = 0 B + P = P, N = P + 0 B = P, both exact), so the
// orthogonaliser and the apply are those of muon_step.
cudaError_t soap_muon_ns(const std::vector<SoapItem>& items, const Plan& P, const SoapMuonExt& ext,
                         const mo_soap_cfg& cfg, char* ws, size_t ws_bytes, cudaStream_t s, std::string* err) {
  std::vector<NsItem> ns;
  for (const Group& g : P.groups) {
    const size_t mn = (size_t)g.m * g.n;
    for (int j = 0; j < (int)g.items.size(); ++j) {
      const SoapItem& it = items[g.items[j]];
      float* p = reinterpret_cast<float*>(ws + g.pb) + (size_t)j * mn;
      NsItem x;
      x.rows = g.m; x.cols = g.n;
      x.in = p; x.mom = p; x.out = it.m.W; x.flag = it.flag;
      x.vec = true;        // cols % 8 == 0, P 16-byte aligned, W checked by the caller
      ns.push_back(x);
    }
  }
  NsCall call = ext.ns;
  call.muon = true;
  call.beta = 0.f; call.nesterov = true; call.ema = false;
  call.lr = cfg.lr; call.wd = cfg.weight_decay;
  return ns_run_at(ns, call, reinterpret_cast<int*>(ws), ws + P.total, ws_bytes - P.total, s, err);
}

}  // namespace

void soap_workspace(const int64_t* rows, const int64_t* cols, int n, size_t* min_bytes, size_t* full_bytes) {
  // shapes only: assume both factor sides are kept
  std::vector<SoapItem> items(n);
  std::vector<float> dummy(1);
  for (int i = 0; i < n; ++i) {
    items[i].m.rows = rows[i];
    items[i].m.cols = cols[i];
    items[i].m.L = items[i].m.R = dummy.data();
  }
  const Plan P = make_plan(items);
  *min_bytes = P.total;
  *full_bytes = P.total;
}

size_t soap_workspace_exact(const std::vector<SoapItem>& items, bool soap_muon) {
  return make_plan(items, soap_muon).total + (soap_muon ? ns_bytes_for(items) : 0);
}

cudaError_t soap_run(const std::vector<SoapItem>& items, const mo_soap_cfg& cfg, int64_t step, char* ws,
                     size_t ws_bytes, cudaStream_t s, std::string* err, const SoapMuonExt* ext) {
  const Plan P = make_plan(items, ext != nullptr);
  const size_t need = P.total + (ext ? ns_bytes_for(items) : 0);
  if (need > ws_bytes) {
    *err = "workspace too small: need " + std::to_string(need) + " bytes";
    return cudaSuccess;
  }
  int* status = reinterpret_cast<int*>(ws);
  const float b1 = ext ? ext->mu : cfg.beta1, b2 = cfg.beta2, bs = cfg.shampoo_beta;
  // SOAP-Muon divides the (uncorrected) Muon momentum: no first-moment correction
  const double bc1 = (cfg.bias_correction && !ext) ? 1.0 - std::pow((double)b1, (double)step) : 1.0;
  const double bc2 = cfg.bias_correction ? 1.0 - std::pow((double)b2, (double)step) : 1.0;
  const float decay = (float)(1.0 - (double)cfg.lr * (double)cfg.weight_decay);
  cudaError_t e = cudaSuccess;

  // ---------------------------------------------------------------- phase 1
  // factor EMAs, first moment (SOAP-Muon: the Muon momentum), planes of G and M/N
  auto phase1 = [&]() -> cudaError_t {
    for (const Group& g : P.groups) {
      const int c = (int)g.items.size();
      void** tab = at<void*>(ws, g.tabs);       // [L | R | V | W | P] pointer tables
      const void* ptrs[SOAP_MAXB];
      for (int k = 0; k < (ext ? 5 : 4); ++k) {
        for (int j = 0; j < c; ++j) {
          const mo_soap_mat& m = items[g.items[j]].m;
          ptrs[j] = k == 0 ? (const void*)m.L : k == 1 ? (const void*)m.R : k == 2 ? (const void*)m.V
                  : k == 3 ? (const void*)m.W : (const void*)(ws + g.pb + (size_t)j * g.m * g.n * 4);
        }
        launch_upload_ptrs(tab + k * SOAP_MAXB, ptrs, c, s);
      }
      if (cfg.nonfinite) {
        FlagTable ft;
        for (int j = 0; j < c; ++j) ft.f[j] = items[g.items[j]].flag;
        launch_set_flags(ft, c, 0, s);
      }
      const long long pn = g.mpad * g.npad;
      if (g.mpad != g.m || g.npad != g.n) {   // zero padding of the plane buffers
        e = cudaMemsetAsync(ws + g.gp, 0, g.mr - g.gp, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(ws + g.dp, 0, al(2 * c * pn * 2), s);
        if (e != cudaSuccess) return e;
      }
      SoapPrepArgs pa;
      pa.count = c; pa.rows = g.m; pa.cols = g.n; pa.beta1 = b1;
      pa.muon = ext ? 1 : 0; pa.nesterov = ext && ext->nesterov ? 1 : 0;
      for (int j = 0; j < c; ++j) { pa.G[j] = items[g.items[j]].m.G; pa.M[j] = items[g.items[j]].m.M; }
      pa.Gp = at<__nv_bfloat16>(ws, g.gp);
      pa.Mp = at<__nv_bfloat16>(ws, g.mpl);
      pa.ldp = g.npad; pa.mat_stride = pn; pa.plane_stride = (long long)c * pn;
      launch_soap_prep(pa, s);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      if (g.left) {          // L <- bs L + (1 - bs) Gb Gb^T   (Gb = plane h of G)
        GemmOp op;
        op.pair = 1;
        op.A = pa.Gp; op.lda = g.npad; op.strideA = pn;
        op.B = pa.Gp; op.ldb = g.npad; op.strideB = pn;
        op.M = (int)g.m; op.N = (int)g.m; op.K = (int)g.n; op.batch = c; op.sym = 1;
        op.alpha = 1.f - bs; op.beta = bs;
        op.C = tab; op.c_tab = (const void* const*)(tab + 0 * SOAP_MAXB); op.ldc = g.m; op.c_f32 = 1;
        op.D = tab; op.d_tab = (void* const*)(tab + 0 * SOAP_MAXB); op.ldd = g.m; op.d_f32 = 1;
        op.kind = PK_SOAP_EMA;
        if ((e = launch_gemm(op, status, s)) != cudaSuccess) return e;
      }
      if (g.right) {         // R <- bs R + (1 - bs) Gb^T Gb
        GemmOp op;
        op.pair = 1;
        op.A = pa.Gp; op.lda = g.npad; op.strideA = pn; op.a_mn = 1;
        op.B = pa.Gp; op.ldb = g.npad; op.strideB = pn; op.b_mn = 1;
        op.M = (int)g.n; op.N = (int)g.n; op.K = (int)g.m; op.batch = c; op.sym = 1;
        op.alpha = 1.f - bs; op.beta = bs;
        op.C = tab; op.c_tab = (const void* const*)(tab + 1 * SOAP_MAXB); op.ldc = g.n; op.c_f32 = 1;
        op.D = tab; op.d_tab = (void* const*)(tab + 1 * SOAP_MAXB); op.ldd = g.n; op.d_f32 = 1;
        op.kind = PK_SOAP_EMA;
        if ((e = launch_gemm(op, status, s)) != cudaSuccess) return e;
      }
    }
    return cudaGetLastError();
  };

  // ---------------------------------------------------------------- phase 2
  // keep the stored bases: only their two bf16 planes are needed for the rotations
  auto old_bases = [&]() -> cudaError_t {
    for (const Group& g : P.groups) {
      const int c = (int)g.items.size();
      for (int side = 0; side < 2; ++side) {
        if ((side == 0 && !g.left) || (side == 1 && !g.right)) continue;
        const long long k = side == 0 ? g.m : g.n;
        const long long kpad = side == 0 ? g.mpad : g.npad;
        SplitArgs sq;
        sq.count = c; sq.rows_valid = (int)k; sq.cols_valid = (int)k;
        sq.rows_pad = (int)kpad; sq.cols_pad = (int)kpad;
        for (int j = 0; j < c; ++j) {
          const mo_soap_mat& m = items[g.items[j]].m;
          sq.src[j] = side == 0 ? m.QL : m.QR;
        }
        sq.lds = k; sq.col_scale = nullptr; sq.write_back = nullptr; sq.ldw = 0; sq.wb_stride = 0;
        sq.dst = at<__nv_bfloat16>(ws, side == 0 ? g.qlp : g.qrp);
        sq.ldd = kpad; sq.mat_stride = kpad * kpad; sq.plane_stride = (long long)c * kpad * kpad;
        sq.nplanes = 2; sq.pad_identity = 0;
        launch_split(sq, s);
      }
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return cudaGetLastError();
  };
  // the per-step refresh Q <- qr(F Q) per bucket (qr.cuh): the power step,
  // then CholeskyQR passes until the basis is orthonormal
  auto refresh = [&]() -> cudaError_t {
    for (const Bucket& bk : P.buckets) {
      const int q = (int)bk.jobs.size();
      const long long k = bk.k, kp = bk.kp, kk = kp * kp, ms = 2 * kk, pst = (long long)q * ms;
      float* CY = at<float>(ws, bk.cy);           // [C; Y]
      __half* LQ = at<__half>(ws, bk.lq);         // planes of [L; Q]
      float* Dinv = at<float>(ws, bk.dinv);
      float* invd = at<float>(ws, bk.invd);
      const QrCtl ctl = qr_ctl_at(ws + bk.ctl, q);
      FlagTable flags;
      for (int j = 0; j < q; ++j) flags.f[j] = items[bk.jobs[j].item].flag;
      auto factor_of = [&](int j) -> const float* {
        const mo_soap_mat& m = items[bk.jobs[j].item].m;
        return bk.jobs[j].left ? m.L : m.R;
      };
      auto basis_of = [&](int j) -> const float* {
        const mo_soap_mat& m = items[bk.jobs[j].item].m;
        return bk.jobs[j].left ? m.QL : m.QR;
      };
      launch_qr_init(ctl, q, s);

      // power step Y = F Q_old (F + d I with the optional damping), both as
      // fp16 planes padded with the identity; F's planes scaled per matrix
      const float* delta = nullptr;
      if (cfg.damping > 0.f) {
        DampArgs da;
        da.count = q; da.k = (int)k; da.rho = cfg.damping; da.delta = at<float>(ws, bk.damp);
        for (int j = 0; j < q; ++j) da.F[j] = factor_of(j);
        launch_damping(da, s);
        delta = da.delta;
      }
      FactorScaleArgs fs;
      fs.count = q; fs.k = (int)k; fs.delta = delta;
      for (int j = 0; j < q; ++j) fs.F[j] = factor_of(j);
      launch_factor_scale(fs, ctl, s);
      Split16Args sp;
      sp.count = q; sp.rows_valid = sp.cols_valid = (int)k; sp.rows_pad = sp.cols_pad = (int)kp;
      sp.lds = k; sp.dst = LQ; sp.ldd = kp; sp.mat_stride = ms; sp.plane_stride = pst; sp.pad_identity = 1;
      for (int j = 0; j < q; ++j) sp.src[j] = factor_of(j);
      sp.diag_add = delta;
      sp.mscale = ctl.fscale;
      launch_split16(sp, s);
      for (int j = 0; j < q; ++j) sp.src[j] = basis_of(j);
      sp.diag_add = nullptr;
      sp.mscale = nullptr;
      sp.cscale = QR_Y_SCALE;
      sp.dst = LQ + kk;
      launch_split16(sp, s);
      {
        GemmOp op;
        op.pair = 1;
        op.A = LQ; op.lda = kp; op.strideA = ms;                           // F [i][p]: K-major
        op.B = LQ + kk; op.ldb = kp; op.strideB = ms; op.b_mn = 1;        // Q_old [p][j]: MN-major
        set_planes2(op, pst, pst);
        op.ab_f16 = 1;
        op.M = (int)kp; op.N = (int)kp; op.K = (int)(3 * kp); op.batch = q;
        op.alpha = 1.f / QR_Y_SCALE; op.scale = ctl.fiscale; op.alpha_pow = 1;
        op.D = CY + kk; op.ldd = kp; op.strideD = ms; op.d_f32 = 1;
        op.kind = PK_SOAP_QR;
        if ((e = launch_gemm(op, status, s)) != cudaSuccess) return e;
      }

      const int nb = (int)(kp / QR_B);
      // One CholeskyQR pass.  Launched directly (pass >= 0), later launches
      // are gated on the device by the matrices done after the previous
      // pass's decision; recorded into the pass-loop graph (pass < 0), the
      // pass index is the device word ctl.npass and the loop itself stops.
      auto enqueue_pass = [&](int pass, cudaStream_t st) -> cudaError_t {
        const bool graph = pass < 0;
        const int* gate_in = (!graph && pass > 0) ? ctl.pass_done + (pass - 1) : nullptr;
        const int* gate_steps = graph ? ctl.pass_done : ctl.pass_done + pass;
        const int* gate_idx = graph ? ctl.npass : nullptr;
        cudaError_t er;
        // normalise Y's columns (a zero column becomes e_c), planes of the
        // result into the Q part of [L; Q], C = Y^T Y into the C part
        launch_colnorm2(CY + kk, kp, ms, q, (int)kp, (int)kp, invd, ctl.done, gate_in, q, st);
        Split16Args sy;
        sy.count = q; sy.rows_valid = sy.cols_valid = sy.rows_pad = sy.cols_pad = (int)kp;
        for (int j = 0; j < q; ++j) sy.src[j] = CY + (size_t)j * ms + kk;
        sy.lds = kp; sy.col_scale = invd; sy.cscale = QR_Y_SCALE;
        sy.write_back = CY + kk; sy.ldw = kp; sy.wb_stride = ms;
        sy.dst = LQ + kk; sy.ldd = kp; sy.mat_stride = ms; sy.plane_stride = pst;
        sy.skip = ctl.done;
        sy.noise_on = ctl.fail;                  // set by a failed attempt of the previous pass
        sy.noise_amp = QR_NOISE;
        sy.noise_seed = graph ? 0u : (unsigned)pass;
        sy.seed_dev = graph ? ctl.npass : nullptr;
        sy.gate = gate_in; sy.gate_n = q;
        launch_split16(sy, st);
        {
          GemmOp g;
          g.pair = 1;
          g.A = LQ + kk; g.lda = kp; g.strideA = ms; g.a_mn = 1;
          g.B = LQ + kk; g.ldb = kp; g.strideB = ms; g.b_mn = 1;
          set_planes2(g, pst, pst);
          g.ab_f16 = 1;
          g.M = (int)kp; g.N = (int)kp; g.K = (int)(3 * kp); g.batch = q; g.sym = 1;
          g.alpha = 1.f / (QR_Y_SCALE * QR_Y_SCALE);
          g.D = CY; g.ldd = kp; g.strideD = ms; g.d_f32 = 1;
          g.kind = PK_SOAP_QR;
          g.skip = ctl.done;
          g.gate = gate_in; g.gate_n = q;
          if ((er = launch_gemm(g, status, st)) != cudaSuccess) return er;
        }
        // done / plain / shifted per matrix, the shift on C's diagonal
        launch_qr_control(CY, kp, ms, q, (int)kp, ctl, graph ? 0 : pass, graph ? ctl.npass : nullptr, gate_in, st);
        for (int j = 0; j < nb; ++j) {
          const long long r0 = (long long)j * QR_B;
          if (j > 0) {     // [C; Y][r0 :, j] -= [L; Q][r0 :, < j] L[j, < j]^T
            GemmOp t;
            t.pair = 1;
            t.A = LQ + r0 * kp; t.lda = kp; t.strideA = ms;
            t.B = LQ + r0 * kp; t.ldb = kp; t.strideB = ms;
            set_planes2(t, pst, pst);
            t.ab_f16 = 1;
            t.M = (int)(2 * kp - r0); t.N = QR_B; t.K = (int)(3 * r0); t.batch = q;
            t.alpha = -1.f / (QR_PLANE_SCALE * QR_PLANE_SCALE); t.beta = 1.f;
            t.C = CY + r0 * kp + r0; t.ldc = kp; t.strideC = ms; t.c_f32 = 1;
            t.D = CY + r0 * kp + r0; t.ldd = kp; t.strideD = ms; t.d_f32 = 1;
            t.kind = PK_QR_TRAIL;
            t.skip = ctl.skip;
            t.gate = gate_steps; t.gate_n = q; t.gate_idx = gate_idx;
            if ((er = launch_gemm(t, status, st)) != cudaSuccess) return er;
          }
          launch_qr_chol(CY, kp, ms, q, j, Dinv, ctl, gate_steps, gate_idx, st);
          PanelArgs pa;
          pa.q = q; pa.j = j; pa.r0 = (int)(r0 + QR_B); pa.r1 = (int)(2 * kp); pa.f32_from = (int)kp;
          pa.CY = CY; pa.ld = kp; pa.mat_stride = ms; pa.Dinv = Dinv;
          pa.LQ = LQ; pa.plane_stride = pst; pa.skip = ctl.skip;
          pa.gate = gate_steps; pa.gate_idx = gate_idx;
          launch_qr_panel(pa, st);
        }
        return cudaGetLastError();
      };
      // the graph holds no event brackets: with profiling on, or inside a
      // caller's capture, the passes are launched directly
      cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
      const bool direct_passes = g_prof != nullptr || cudaStreamIsCapturing(s, &cap) != cudaSuccess ||
                                 cap != cudaStreamCaptureStatusNone;
      bool in_graph = false;
      if (!direct_passes) {
        PassGraph key;
        (void)cudaGetDevice(&key.dev);
        key.ws = ws; key.cy = bk.cy; key.lq = bk.lq; key.dinv = bk.dinv; key.invd = bk.invd; key.ctl = bk.ctl;
        key.q = q; key.kp = kp; key.k = k;
        in_graph = launch_pass_graph(
            key,
            [&](cudaStream_t cs, cudaGraphConditionalHandle h) -> cudaError_t {
              cudaError_t er = enqueue_pass(-1, cs);
              if (er != cudaSuccess) return er;
              launch_qr_loop(ctl, q, h, cs);
              return cudaGetLastError();
            },
            s);
      }
      if (!in_graph)
        for (int pass = 0; pass < QR_MAX_PASSES; ++pass)
          if ((e = enqueue_pass(pass, s)) != cudaSuccess) return e;
      {
        const float* qold[SOAP_MAXB];
        for (int j = 0; j < q; ++j) qold[j] = basis_of(j);
        launch_qr_finish(ctl, flags, q, CY + kk, kp, ms, (int)k, (int)kp, qold, s);
      }
      BasisOutArgs bo;
      bo.count = q; bo.k = (int)k; bo.kpad_max = 0;
      bo.Y = CY + kk; bo.ld = kp; bo.mat_stride = ms;
      for (int j = 0; j < q; ++j) {
        const Job& jb = bk.jobs[j];
        const Group& g = P.groups[jb.group];
        const mo_soap_mat& m = items[jb.item].m;
        const long long kpad = jb.left ? g.mpad : g.npad;
        bo.q[j] = jb.left ? m.QL : m.QR;
        bo.vec[j] = (k % 4 == 0 && (reinterpret_cast<uintptr_t>(bo.q[j]) & 15) == 0) ? 1 : 0;
        bo.kpad[j] = (int)kpad;
        bo.planes[j] = at<__nv_bfloat16>(ws, jb.left ? g.qlp : g.qrp) + (size_t)jb.pos * kpad * kpad;
        bo.pst[j] = (long long)g.items.size() * kpad * kpad;
        bo.kpad_max = std::max(bo.kpad_max, (int)kpad);
      }
      // the new bases: fp32 into the caller's Q, two bf16 planes into the
      // group buffers for the rotations, in one pass
      launch_basis_out(bo, s);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaGetLastError();
  };

  // ---------------------------------------------------------------- phase 3
  // rotations with Adam in the basis; SOAP applies W, SOAP-Muon writes P
  auto rotate = [&]() -> cudaError_t {
    for (const Group& g : P.groups) {
      const int c = (int)g.items.size();
      const long long m = g.m, n = g.n, mn = m * n;
      const long long mp = g.mpad, np = g.npad, pn = mp * np;
      void** tab = at<void*>(ws, g.tabs);
      __nv_bfloat16* Gp = at<__nv_bfloat16>(ws, g.gp);
      __nv_bfloat16* Mp = at<__nv_bfloat16>(ws, g.mpl);
      __nv_bfloat16* Tp = at<__nv_bfloat16>(ws, g.tp);
      float* Mr = at<float>(ws, g.mr);
      __nv_bfloat16* Dp = at<__nv_bfloat16>(ws, g.dp);
      __nv_bfloat16* QLp = at<__nv_bfloat16>(ws, g.qlp);
      __nv_bfloat16* QRp = at<__nv_bfloat16>(ws, g.qrp);
      const long long ppn = (long long)c * pn, pmm = (long long)c * mp * mp, pnn = (long long)c * np * np;
      if (!g.left && !g.right) {
        AdamIdArgs a;
        a.count = c; a.elems = mn; a.beta2 = b2; a.ibc1 = (float)(1.0 / bc1); a.ibc2 = (float)(1.0 / bc2);
        a.eps = cfg.eps; a.decay = decay; a.lr = cfg.lr;
        a.muon = ext ? 1 : 0; a.nesterov = ext && ext->nesterov ? 1 : 0; a.mu = b1;
        for (int j = 0; j < c; ++j) {
          const mo_soap_mat& mm = items[g.items[j]].m;
          a.G[j] = mm.G; a.M[j] = mm.M; a.V[j] = mm.V; a.W[j] = mm.W;
          a.P[j] = ext ? reinterpret_cast<float*>(ws + g.pb + (size_t)j * mn * 4) : nullptr;
        }
        launch_adam_identity(a, s);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        continue;
      }
      // product with the left basis transposed: out = QL^T X  (X: [mp][np] planes)
      auto left_t = [&](GemmOp& op, const __nv_bfloat16* X) {
        op.A = QLp; op.lda = mp; op.strideA = mp * mp; op.a_mn = 1;
        op.B = X; op.ldb = np; op.strideB = pn; op.b_mn = 1;
        set_planes2(op, pmm, ppn);
        op.M = (int)m; op.N = (int)n; op.K = (int)(3 * mp);
      };
      // out = X QR  (X as K-major planes [mp][np])
      auto right_n = [&](GemmOp& op, const __nv_bfloat16* X) {
        op.A = X; op.lda = np; op.strideA = pn;
        op.B = QRp; op.ldb = np; op.strideB = np * np; op.b_mn = 1;
        set_planes2(op, ppn, pnn);
        op.M = (int)m; op.N = (int)n; op.K = (int)(3 * np);
      };
      auto to_planes = [&](GemmOp& op, __nv_bfloat16* D) {
        op.D = D; op.ldd = np; op.strideD = pn; op.d_f32 = 0; op.d_split = 1; op.d_plane = ppn;
      };
      // rotate X into the basis: M' (fp32) or, with the Adam epilogue, V and Dbar
      auto rotate_in = [&](const __nv_bfloat16* X, bool adam) -> cudaError_t {
        GemmOp op;
        op.pair = 1;
        op.kind = PK_SOAP_GEMM;
        op.batch = c;
        if (g.left && g.right) {
          GemmOp t;                       // T = QL^T X, kept as two planes
          t.pair = 1;
          t.kind = PK_SOAP_GEMM; t.batch = c;
          left_t(t, X);
          to_planes(t, Tp);
          cudaError_t r = launch_gemm(t, status, s);
          if (r != cudaSuccess) return r;
          right_n(op, Tp);                // T QR
        } else if (g.left) {
          left_t(op, X);
        } else {
          right_n(op, X);
        }
        if (!adam) {
          op.D = Mr; op.ldd = n; op.strideD = mn; op.d_f32 = 1;
        } else {
          op.epi = 1;                     // Adam-in-basis epilogue
          op.C = Mr; op.ldc = n; op.strideC = mn; op.c_f32 = 1;
          op.e_tab = reinterpret_cast<float* const*>(tab + 2 * SOAP_MAXB); op.lde = n;
          op.adam_b2 = b2; op.adam_ibc1 = (float)(1.0 / bc1); op.adam_ibc2 = (float)(1.0 / bc2);
          op.adam_eps = cfg.eps;
          to_planes(op, Dp);
        }
        return launch_gemm(op, status, s);
      };
      if ((e = rotate_in(Mp, false)) != cudaSuccess) return e;     // M'
      if ((e = rotate_in(Gp, true)) != cudaSuccess) return e;      // G', V, Dbar
      // rotate back and apply: W <- decay W - lr QL Dbar QR^T
      GemmOp op;
      op.pair = 1;
      op.kind = PK_SOAP_GEMM;
      op.batch = c;
      auto left_n = [&](GemmOp& g2, const __nv_bfloat16* X) {      // QL X
        g2.A = QLp; g2.lda = mp; g2.strideA = mp * mp;
        g2.B = X; g2.ldb = np; g2.strideB = pn; g2.b_mn = 1;
        set_planes2(g2, pmm, ppn);
        g2.M = (int)m; g2.N = (int)n; g2.K = (int)(3 * mp);
      };
      auto right_t = [&](GemmOp& g2, const __nv_bfloat16* X) {     // X QR^T
        g2.A = X; g2.lda = np; g2.strideA = pn;
        g2.B = QRp; g2.ldb = np; g2.strideB = np * np;
        set_planes2(g2, ppn, pnn);
        g2.M = (int)m; g2.N = (int)n; g2.K = (int)(3 * np);
      };
      if (g.left && g.right) {
        GemmOp t;                         // S = QL Dbar, kept as two planes
        t.pair = 1;
        t.kind = PK_SOAP_GEMM; t.batch = c;
        left_n(t, Dp);
        to_planes(t, Tp);
        if ((e = launch_gemm(t, status, s)) != cudaSuccess) return e;
        right_t(op, Tp);
      } else if (g.left) {
        left_n(op, Dp);
      } else {
        right_t(op, Dp);
      }
      if (ext) {                        // SOAP-Muon: P = QL Dbar QR^T (fp32)
        op.D = ws + g.pb; op.ldd = n; op.strideD = mn; op.d_f32 = 1;
      } else {                          // SOAP: W <- decay W - lr QL Dbar QR^T
        op.alpha = -cfg.lr; op.beta = decay;
        op.C = tab; op.c_tab = (const void* const*)(tab + 3 * SOAP_MAXB); op.ldc = n; op.c_f32 = 1;
        op.D = tab; op.d_tab = (void* const*)(tab + 3 * SOAP_MAXB); op.ldd = n; op.d_f32 = 1;
      }
      if ((e = launch_gemm(op, status, s)) != cudaSuccess) return e;
    }
    return cudaGetLastError();
  };

  // each phase under its own profiler range
  auto ranged = [](const char* name, auto&& fn) -> cudaError_t {
    NvtxRange nvtx(name);
    return fn();
  };
  if ((e = ranged("mo soap factors + first moment", phase1)) != cudaSuccess) return e;
  if (ext == nullptr) {
    if ((e = cfg.skip_refresh ? ranged("mo soap bases kept", old_bases) : ranged("mo soap basis refresh", refresh)) !=
        cudaSuccess)
      return e;
    return ranged("mo soap rotate + adam + apply", rotate);
  }
  // SOAP-Muon: precondition with the previous bases, orthogonalise and apply,
  // then refresh the bases for the next step
  if ((e = ranged("mo soap previous bases", old_bases)) != cudaSuccess) return e;
  if ((e = ranged("mo soap precondition", rotate)) != cudaSuccess) return e;
  if ((e = soap_muon_ns(items, P, *ext, cfg, ws, ws_bytes, s, err)) != cudaSuccess || !err->empty()) return e;
  if (cfg.skip_refresh) return cudaGetLastError();
  return ranged("mo soap basis refresh", refresh);
}

}  // namespace mo
