// SOAP driver: one optimizer step with a per-step basis refresh.
//
// Phase 1 (per group of equal shape and sides):
//   prep:  M <- b1 M + (1-b1) G,  Gb = bf16(G), Mb = bf16(M)
//   EMAs:  L <- bs L + (1-bs) Gb Gb^T ; R <- bs R + (1-bs) Gb^T Gb
//          (symmetric tcgen05 products written into the caller's L / R)
// Phase 2 (per bucket of equal factor size k, all sides of all matrices):
//   power: Y = (L + d I) Q, d = damping * trace(L), fp32-accurate
//          (3-plane bf16 split, 6 plane products)
//   QR:    shifted CholeskyQR3: up to three passes of
//            column-normalise Y, C = Y^T Y (fp32-accurate), [shift C],
//            blocked Cholesky C = L L^T with 128-wide diagonal blocks and
//            Y <- Y L^{-T} (right-looking, tensor-core trailing updates);
//          the third pass is skipped per matrix when its Gram is already
//          within 5e-5 of the identity (every warm step)
//          -> Q (unique QR, diag(R) > 0) into the caller's Q and bf16(Q)
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
#include <tuple>

#include "ns_plan.h"
#include "profile.h"
#include "runtime.h"
#include "soap_kernels.cuh"
#include "soap_plan.h"

namespace mo {

namespace {

constexpr size_t AL = 1024;
size_t al(size_t x) { return (x + AL - 1) / AL * AL; }

// plane products of the fp32-accurate GEMMs: x = h + m + l, and
// x y ~ hh + hm + mh + hl + lh + mm  (dropped terms are below 2^-24).  The
// small products are accumulated first and hh last: the tensor core's fp32
// accumulation loses low-order bits of each addend that is small next to
// the running sum, so adding the small terms into an accumulator that
// already holds hh would cost most of their accuracy.
const unsigned char PAT_A[6] = {1, 2, 0, 1, 0, 0};
const unsigned char PAT_B[6] = {1, 0, 2, 0, 1, 0};

void set_planes(GemmOp& g, long long planeA, long long planeB) {
  g.nseg = 6;
  for (int i = 0; i < 6; ++i) { g.pat_a[i] = PAT_A[i]; g.pat_b[i] = PAT_B[i]; }
  g.planeA = planeA;
  g.planeB = planeB;
}

// two-plane products of the rotations: x = h + l, x y ~ lh + hl + hh
// (small products first, as above)
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

struct Bucket {
  long long k, kp;
  std::vector<Job> jobs;
  size_t y, c, ypl, qpl, ppl, qjpl, dinv, invd, damp, qdev, qskip;
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
    b.y = off; off += al(q * kk * 4);
    b.c = off; off += al(q * kk * 4);
    b.ypl = off; off += al(3 * q * kk * 2);
    b.qpl = off; off += al(3 * q * kk * 2);
    b.ppl = off; off += al(3 * q * b.kp * QR_B * 2);
    b.qjpl = off; off += al(3 * q * b.kp * QR_B * 2);
    b.dinv = off; off += al(q * QR_B * QR_B * 4);
    b.invd = off; off += al(q * b.kp * 4);
    b.damp = off; off += al(q * 4);
    b.qdev = off; off += al(q * 4);
    b.qskip = off; off += al(q * 4);
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
  // the per-step refresh: damped power step + shifted CholeskyQR3 per bucket
  auto refresh = [&]() -> cudaError_t {
    for (const Bucket& bk : P.buckets) {
      const int q = (int)bk.jobs.size();
      const long long k = bk.k, kp = bk.kp, kk = kp * kp;
      float* Y = at<float>(ws, bk.y);
      float* C = at<float>(ws, bk.c);
      __nv_bfloat16* Ypl = at<__nv_bfloat16>(ws, bk.ypl);
      __nv_bfloat16* Qpl = at<__nv_bfloat16>(ws, bk.qpl);
      __nv_bfloat16* Ppl = at<__nv_bfloat16>(ws, bk.ppl);
      __nv_bfloat16* Qjpl = at<__nv_bfloat16>(ws, bk.qjpl);
      float* Dinv = at<float>(ws, bk.dinv);
      float* invd = at<float>(ws, bk.invd);
      FlagTable flags;
      for (int j = 0; j < q; ++j) flags.f[j] = items[bk.jobs[j].item].flag;

      // power step: Y = (L + d I) Q, d = damping * trace(L) (planes of the
      // damped L into Ypl, planes of the old Q into Qpl)
      float* damp = at<float>(ws, bk.damp);
      {
        DampArgs da;
        da.count = q; da.k = (int)k; da.rho = cfg.damping; da.delta = damp;
        for (int j = 0; j < q; ++j) {
          const mo_soap_mat& m = items[bk.jobs[j].item].m;
          da.F[j] = bk.jobs[j].left ? m.L : m.R;
        }
        launch_damping(da, s);
      }
      SplitArgs sa;
      sa.count = q; sa.rows_valid = (int)k; sa.cols_valid = (int)k; sa.rows_pad = (int)kp; sa.cols_pad = (int)kp;
      sa.lds = k; sa.col_scale = nullptr; sa.write_back = nullptr; sa.ldw = 0; sa.wb_stride = 0;
      sa.ldd = kp; sa.mat_stride = kk; sa.plane_stride = (long long)q * kk; sa.nplanes = 3; sa.pad_identity = 1;
      for (int j = 0; j < q; ++j) {
        const mo_soap_mat& m = items[bk.jobs[j].item].m;
        sa.src[j] = bk.jobs[j].left ? m.L : m.R;
      }
      sa.dst = Ypl;
      sa.diag_add = damp;
      launch_split(sa, s);
      sa.diag_add = nullptr;
      for (int j = 0; j < q; ++j) {
        const mo_soap_mat& m = items[bk.jobs[j].item].m;
        sa.src[j] = bk.jobs[j].left ? m.QL : m.QR;
      }
      sa.dst = Qpl;
      launch_split(sa, s);
      {
        GemmOp op;
        op.A = Ypl; op.lda = kp; op.strideA = kk;          // L [i][p]: K-major
        op.B = Qpl; op.ldb = kp; op.strideB = kk; op.b_mn = 1;   // Q [p][j]: MN-major
        set_planes(op, (long long)q * kk, (long long)q * kk);
        op.M = (int)kp; op.N = (int)kp; op.K = (int)(6 * kp); op.batch = q;
        op.D = Y; op.ldd = kp; op.strideD = kk; op.d_f32 = 1;
        op.kind = PK_SOAP_QR;
        if ((e = launch_gemm(op, status, s)) != cudaSuccess) return e;
      }

      // shifted CholeskyQR3
      const int nb = (int)(kp / QR_B);
      for (int pass = 0; pass < 3; ++pass) {
        launch_colnorm(Y, kp, kk, q, (int)kp, (int)kp, invd, s);
        SplitArgs sy;
        sy.count = q; sy.rows_valid = (int)kp; sy.cols_valid = (int)kp; sy.rows_pad = (int)kp; sy.cols_pad = (int)kp;
        for (int j = 0; j < q; ++j) sy.src[j] = Y + (size_t)j * kk;
        sy.lds = kp; sy.col_scale = invd; sy.write_back = Y; sy.ldw = kp; sy.wb_stride = kk;
        sy.dst = Ypl; sy.ldd = kp; sy.mat_stride = kk; sy.plane_stride = (long long)q * kk;
        sy.nplanes = 3; sy.pad_identity = 0;
        launch_split(sy, s);
        {   // C = Y^T Y, fp32-accurate, symmetric
          GemmOp op;
          op.A = Ypl; op.lda = kp; op.strideA = kk; op.a_mn = 1;
          op.B = Ypl; op.ldb = kp; op.strideB = kk; op.b_mn = 1;
          set_planes(op, (long long)q * kk, (long long)q * kk);
          op.M = (int)kp; op.N = (int)kp; op.K = (int)(6 * kp); op.batch = q; op.sym = 1;
          op.D = C; op.ldd = kp; op.strideD = kk; op.d_f32 = 1;
          op.kind = PK_SOAP_QR;
          if ((e = launch_gemm(op, status, s)) != cudaSuccess) return e;
        }
        // The first pass shifts the Gram matrix (unit diagonal, trace kp) by
        // 1e-5 of its trace, above its fp32 rounding error.  With the damped
        // factor, cond(Y) <= 1 + 1 / damping (1e5 at the default), and the
        // shifted pass leaves a Q whose Gram the two unshifted passes
        // factor safely (cond(Q) below the fp32 limit of Cholesky QR).
        if (pass == 0) launch_shift_diag(C, kp, kk, q, (int)kp, 1e-5f * (float)kp, s);
        // The last pass only corrects what is left of the previous pass's
        // rounding.  A basis whose Gram is within 5e-5 of the identity keeps
        // its (column-normalised) Q and every kernel of the pass skips it:
        // the tensor core's fp32 accumulation leaves the Gram of an exactly
        // orthonormal 4096-column basis about 2e-5 off the identity, so the
        // pass could not lower the error below that floor, and the two-plane
        // rotations that use the basis resolve 2^-16 = 1.5e-5.  Cold starts
        // (deviation 1e-2 and more after the shifted pass) run all three.
        const int* skip = nullptr;
        if (pass == 2) {
          launch_identity_check(C, kp, kk, q, (int)kp, 5e-5f, at<int>(ws, bk.qdev), at<int>(ws, bk.qskip), s);
          skip = at<int>(ws, bk.qskip);
        }
        for (int jb = 0; jb < nb; ++jb) {
          const long long k0 = (long long)jb * QR_B;
          const long long rem = kp - k0 - QR_B;
          launch_chol_diag(C, kp, kk, q, (int)k0, Dinv, flags, s, skip);
          if (rem > 0) {      // panel L21 = C21 L11^{-T}, kept only as planes
            RowBlockArgs ra;
            ra.count = q; ra.rows = (int)rem;
            ra.in = C + (k0 + QR_B) * kp + k0; ra.ld_in = kp; ra.in_stride = kk;
            ra.out = nullptr; ra.ld_out = 0; ra.out_stride = 0;
            ra.Dinv = Dinv;
            ra.planes = Ppl; ra.plane_stride = (long long)q * kp * QR_B; ra.mat_stride = kp * QR_B;
            ra.skip = skip;
            launch_rowblock_dinv(ra, s);
          }
          {                   // Q_j = Y_j L_jj^{-T} (in place) and its planes
            RowBlockArgs ra;
            ra.count = q; ra.rows = (int)kp;
            ra.in = Y + k0; ra.ld_in = kp; ra.in_stride = kk;
            ra.out = Y + k0; ra.ld_out = kp; ra.out_stride = kk;
            ra.Dinv = Dinv;
            ra.planes = Qjpl; ra.plane_stride = (long long)q * kp * QR_B; ra.mat_stride = kp * QR_B;
            ra.skip = skip;
            launch_rowblock_dinv(ra, s);
          }
          if (rem > 0) {
            GemmOp op;        // C22 -= L21 L21^T
            op.A = Ppl; op.lda = QR_B; op.strideA = kp * QR_B;
            op.B = Ppl; op.ldb = QR_B; op.strideB = kp * QR_B;
            set_planes(op, (long long)q * kp * QR_B, (long long)q * kp * QR_B);
            op.M = (int)rem; op.N = (int)rem; op.K = 6 * QR_B; op.batch = q; op.sym = 1;
            op.alpha = -1.f; op.beta = 1.f;
            float* c22 = C + (k0 + QR_B) * kp + (k0 + QR_B);
            op.C = c22; op.ldc = kp; op.strideC = kk; op.c_f32 = 1;
            op.D = c22; op.ldd = kp; op.strideD = kk; op.d_f32 = 1;
            op.kind = PK_QR_TRAIL;
            op.skip = skip;
            if ((e = launch_gemm(op, status, s)) != cudaSuccess) return e;
            GemmOp t;         // Y[:, k0+128:] -= Q_j L21^T
            t.A = Qjpl; t.lda = QR_B; t.strideA = kp * QR_B;
            t.B = Ppl; t.ldb = QR_B; t.strideB = kp * QR_B;
            set_planes(t, (long long)q * kp * QR_B, (long long)q * kp * QR_B);
            t.M = (int)kp; t.N = (int)rem; t.K = 6 * QR_B; t.batch = q;
            t.alpha = -1.f; t.beta = 1.f;
            float* yr = Y + (k0 + QR_B);
            t.C = yr; t.ldc = kp; t.strideC = kk; t.c_f32 = 1;
            t.D = yr; t.ldd = kp; t.strideD = kk; t.d_f32 = 1;
            t.kind = PK_QR_TRAIL;
            t.skip = skip;
            if ((e = launch_gemm(t, status, s)) != cudaSuccess) return e;
          }
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
      }
      // the new bases: fp32 into the caller's Q, bf16 into the group buffers
      CopyOutArgs co;
      co.count = q; co.k = (int)k; co.Y = Y; co.ld = kp; co.mat_stride = kk;
      for (int j = 0; j < q; ++j) {
        const mo_soap_mat& m = items[bk.jobs[j].item].m;
        co.dst[j] = bk.jobs[j].left ? m.QL : m.QR;
      }
      launch_copy_out(co, s);
      // two bf16 planes of each new basis into its group's buffer (one launch
      // per job: the group buffers are not uniformly strided across the bucket)
      for (int j = 0; j < q; ++j) {
        const Job& jb = bk.jobs[j];
        const Group& g = P.groups[jb.group];
        const long long kpad = jb.left ? g.mpad : g.npad;
        SplitArgs one;
        one.count = 1; one.rows_valid = (int)k; one.cols_valid = (int)k;
        one.rows_pad = (int)kpad; one.cols_pad = (int)kpad;
        one.src[0] = Y + (size_t)j * kk; one.lds = kp;
        one.col_scale = nullptr; one.write_back = nullptr; one.ldw = 0; one.wb_stride = 0;
        one.dst = at<__nv_bfloat16>(ws, jb.left ? g.qlp : g.qrp) + (size_t)jb.pos * kpad * kpad;
        one.ldd = kpad; one.mat_stride = 0;
        one.plane_stride = (long long)g.items.size() * kpad * kpad;
        one.nplanes = 2; one.pad_identity = 0;
        launch_split(one, s);
      }
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
        op.kind = PK_SOAP_GEMM;
        op.batch = c;
        if (g.left && g.right) {
          GemmOp t;                       // T = QL^T X, kept as two planes
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
