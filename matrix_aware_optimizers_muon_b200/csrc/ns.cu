// Newton-Schulz driver: buckets matrices by oriented shape (m' <= n') and,
// per bucket chunk, launches
//   prep (momentum, Nesterov, bf16 cast + orientation, tile partials of N^2)
//   finalize (||N||_F -> 1 / (||N||_F + eps))
//   ns_steps x { A = X X^T          (symmetric: upper tiles + mirror)
//                P = a I + b A + c A A  (symmetric: upper tiles + mirror)
//                X' = P X }         (= a X + (b A + c A A) X; with fewer
//                                    than 128 rows P = b A + c A A and
//                                    X' = a X + P X; iteration 0 folds the
//                                    1/(||N||+eps) scale into the fp32
//                                    epilogues)
//   apply (W <- (1 - lr wd) W - lr s O, un-oriented; or out = O); for Muon
//   the apply runs in the epilogue of the last update product instead, so
//   O is never stored
#include <algorithm>
#include <cmath>
#include <map>

#include "elementwise.cuh"
#include "ns_small.cuh"
#include "ns_plan.h"
#include "profile.h"
#include "runtime.h"

namespace mo {

namespace {

constexpr size_t ALIGN = 1024;

size_t al(size_t x) { return (x + ALIGN - 1) / ALIGN * ALIGN; }

struct Shape {
  long long mp, np;   // oriented: mp <= np
  bool operator<(const Shape& o) const { return mp != o.mp ? mp < o.mp : np < o.np; }
};

Shape oriented(long long rows, long long cols) {
  return rows > cols ? Shape{cols, rows} : Shape{rows, cols};
}

struct Layout {
  long long ldx, lda, xstride, astride, tiles;
  size_t x_bytes, a_bytes, part_bytes, inv_bytes, tab_bytes;
  size_t total(int cnt) const {
    return 2 * al(x_bytes * cnt) + 2 * al(a_bytes * cnt) + al(part_bytes * cnt) + al(inv_bytes * cnt) +
           al(tab_bytes * cnt);
  }
};

Layout layout_of(const Shape& s) {
  Layout L;
  L.ldx = round_up(s.np, 64);
  L.lda = round_up(s.mp, 64);
  L.xstride = s.mp * L.ldx;
  L.astride = s.mp * L.lda;
  L.tiles = ((s.mp + 63) / 64) * ((s.np + 63) / 64);
  L.x_bytes = (size_t)L.xstride * 2;
  L.a_bytes = (size_t)L.astride * 2;
  L.part_bytes = (size_t)L.tiles * 4;
  L.inv_bytes = 4;
  L.tab_bytes = 4 * sizeof(void*);     // device pointer tables (in, mom, out, flag)
  return L;
}

}  // namespace

void ns_workspace(const int64_t* rows, const int64_t* cols, int n, size_t* min_bytes, size_t* full_bytes) {
  std::map<Shape, int> count;
  for (int i = 0; i < n; ++i) count[oriented(rows[i], cols[i])]++;
  size_t mn = 0, full = 0;
  for (auto& kv : count) {
    const Layout L = layout_of(kv.first);
    mn = std::max(mn, L.total(1));
    full = std::max(full, L.total(std::min(kv.second, 1 << 16)));
  }
  *min_bytes = WS_HEADER + mn;
  *full_bytes = WS_HEADER + full;
}

cudaError_t ns_run(const std::vector<NsItem>& items, const NsCall& call, char* ws, size_t ws_bytes,
                   cudaStream_t stream, std::string* err) {
  return ns_run_at(items, call, reinterpret_cast<int*>(ws), ws + WS_HEADER,
                   ws_bytes > WS_HEADER ? ws_bytes - WS_HEADER : 0, stream, err);
}

cudaError_t ns_run_at(const std::vector<NsItem>& items, const NsCall& call, int* status, char* base,
                      size_t avail, cudaStream_t stream, std::string* err) {
  std::map<Shape, std::vector<int>> buckets;
  for (int i = 0; i < (int)items.size(); ++i)
    buckets[oriented(items[i].rows, items[i].cols)].push_back(i);
  auto is_tall = [&](int i) { return items[i].rows > items[i].cols; };

  for (auto& kv : buckets) {
    const Shape s = kv.first;
    std::vector<int> idx = kv.second;
    // wide (or square) matrices first, then tall ones: every elementwise
    // launch below covers a contiguous run of one orientation
    std::stable_partition(idx.begin(), idx.end(), [&](int i) { return !is_tall(i); });
    const Layout L = layout_of(s);
    if (s.mp <= SMALL_MAX_M && s.np <= SMALL_MAX_N) {
      // small matrices: one fused launch per orientation, no iterate buffers
      const size_t need = 4 * idx.size() * sizeof(void*);
      if (need > avail) {
        *err = "workspace too small for the pointer tables of " + std::to_string(idx.size()) + " matrices";
        return cudaSuccess;
      }
      void** tab = reinterpret_cast<void**>(base);
      for (int pass = 0; pass < 2; ++pass) {
        std::vector<const void*> in, mom, out, flg;
        long long rows = 0, cols = 0;
        for (int i : idx) {
          if (is_tall(i) != (pass == 1)) continue;
          in.push_back(items[i].in); mom.push_back(items[i].mom);
          out.push_back(items[i].out); flg.push_back(items[i].flag);
          rows = items[i].rows; cols = items[i].cols;
        }
        const int n = (int)in.size();
        if (n == 0) continue;
        bool vec = cols % 4 == 0;
        for (int j = 0; j < n && vec; ++j) {
          auto al16 = [](const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
          vec = al16(in[j]) && al16(out[j]) && (!call.muon || al16(mom[j]));
        }
        launch_upload_tables(tab, n, in.data(), mom.data(), out.data(), flg.data(), stream);
        NvtxRange nvtx_small("mo newton-schulz small matrices");
        SmallArgs sa;
        sa.count = n; sa.rows = (int)rows; sa.cols = (int)cols; sa.tall = pass;
        sa.mode = call.muon ? 1 : 0;
        sa.beta = call.beta; sa.nesterov = call.nesterov; sa.ema = call.ema;
        sa.steps = call.steps; sa.vec = vec ? 1 : 0; sa.a = call.a; sa.b = call.b; sa.c = call.c; sa.eps = call.eps;
        const double m = (double)rows, nn = (double)cols;
        const double scale = call.adjust_lr == 0 ? 0.2 * std::sqrt(std::max(m, nn)) : std::sqrt(std::max(1.0, m / nn));
        sa.decay = (float)(1.0 - (double)call.lr * (double)call.wd);
        sa.step = (float)((double)call.lr * scale);
        sa.in = reinterpret_cast<const float* const*>(tab);
        sa.mom = call.muon ? reinterpret_cast<float* const*>(tab + n) : nullptr;
        sa.out = reinterpret_cast<float* const*>(tab + 2 * n);
        sa.flag = reinterpret_cast<int32_t* const*>(tab + 3 * n);
        sa.status = status;
        cudaError_t e = launch_ns_small(sa, device_sm_count(), stream);
        if (e != cudaSuccess) return e;
        // the next launch may reuse the tables only after this one is done
        // reading them; both run on one stream, so stream order suffices
      }
      continue;
    }
    if (L.total(1) > avail) {
      *err = "workspace too small for a " + std::to_string(s.mp) + " x " + std::to_string(s.np) +
             " matrix (need " + std::to_string(L.total(1) + WS_HEADER) + " bytes)";
      return cudaSuccess;
    }
    int chunk = (int)idx.size();
    while (chunk > 1 && L.total(chunk) > avail) chunk = std::max(1, (int)(chunk * (double)avail / L.total(chunk)));
    while (chunk > 1 && L.total(chunk) > avail) --chunk;

    for (int c0 = 0; c0 < (int)idx.size(); c0 += chunk) {
      NvtxRange nvtx_chunk("mo newton-schulz bucket chunk");
      const int cnt = std::min(chunk, (int)idx.size() - c0);
      char* p = base;
      __nv_bfloat16* X0 = reinterpret_cast<__nv_bfloat16*>(p); p += al(L.x_bytes * cnt);
      __nv_bfloat16* X1 = reinterpret_cast<__nv_bfloat16*>(p); p += al(L.x_bytes * cnt);
      __nv_bfloat16* A = reinterpret_cast<__nv_bfloat16*>(p); p += al(L.a_bytes * cnt);
      __nv_bfloat16* P = reinterpret_cast<__nv_bfloat16*>(p); p += al(L.a_bytes * cnt);
      float* part = reinterpret_cast<float*>(p); p += al(L.part_bytes * cnt);
      float* inv = reinterpret_cast<float*>(p); p += al(L.inv_bytes * cnt);
      void** tab = reinterpret_cast<void**>(p);

      // runs [first, first + count) of equal orientation, at most EW_MAX long
      struct Run { int first, count; bool tall; };
      std::vector<Run> runs;
      for (int k = 0; k < cnt;) {
        const bool t = is_tall(idx[c0 + k]);
        int e = k;
        while (e < cnt && e - k < EW_MAX && is_tall(idx[c0 + e]) == t) ++e;
        runs.push_back({k, e - k, t});
        k = e;
      }
      auto table = [&](const Run& r) {
        EwTable t;
        bool vec = true;
        for (int k = 0; k < r.count; ++k) {
          const NsItem& it = items[idx[c0 + r.first + k]];
          t.in[k] = it.in; t.mom[k] = it.mom; t.out[k] = it.out; t.flag[k] = it.flag;
          t.tall[k] = r.tall ? 1 : 0;
          vec = vec && it.vec;
        }
        return std::make_pair(t, vec);
      };

      // pass 1: momentum / cast / orientation / tile partials, then the norms
      for (const Run& r : runs) {
        auto tv = table(r);
        PrepArgs pa;
        pa.count = r.count;
        pa.mp = (int)s.mp; pa.np = (int)s.np;
        pa.tiles_r = (int)(((r.tall ? s.np : s.mp) + 63) / 64);   // tiles of the stored matrix
        pa.tiles_c = (int)(((r.tall ? s.mp : s.np) + 63) / 64);
        pa.beta = call.beta;
        pa.mode = call.muon ? 1 : 0;
        pa.nesterov = call.nesterov;
        pa.ema = call.ema;
        pa.vec = tv.second;
        pa.X = X0 + (size_t)r.first * L.xstride;
        pa.ldx = L.ldx; pa.xstride = L.xstride;
        pa.partial = part + (size_t)r.first * L.tiles;
        launch_prep(tv.first, pa, stream);
        FinalizeArgs fa;
        fa.count = r.count;
        fa.tiles = (int)L.tiles;
        fa.eps = call.eps;
        fa.partial = pa.partial;
        fa.inv = inv + r.first;
        launch_finalize(tv.first, fa, stream);
      }
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;

      // Muon: the last update's epilogue applies O to W, through a device
      // table of the chunk's W pointers (wide matrices first, then tall)
      const bool fused_apply = call.muon && call.steps > 0;
      int tall_from = cnt;
      bool w_vec = true;
      float decay = 1.f, step_of[2] = {0.f, 0.f};
      if (fused_apply) {
        std::vector<const void*> tin(cnt), tmom(cnt), tout(cnt), tflg(cnt);
        for (int k = 0; k < cnt; ++k) {
          const NsItem& it = items[idx[c0 + k]];
          tin[k] = it.in; tmom[k] = it.mom; tout[k] = it.out; tflg[k] = it.flag;
          if (is_tall(idx[c0 + k]) && tall_from == cnt) tall_from = k;
          w_vec = w_vec && it.vec;
        }
        launch_upload_tables(tab, cnt, tin.data(), tmom.data(), tout.data(), tflg.data(), stream);
        decay = (float)(1.0 - (double)call.lr * (double)call.wd);
        for (int t = 0; t < 2; ++t) {
          const double m = (double)(t ? s.np : s.mp), n = (double)(t ? s.mp : s.np);   // stored shape
          const double scale = call.adjust_lr == 0 ? 0.2 * std::sqrt(std::max(m, n))
                                                   : std::sqrt(std::max(1.0, m / n));
          step_of[t] = (float)((double)call.lr * scale);
        }
      }

      // Newton-Schulz iterations on the oriented bf16 batch
      __nv_bfloat16* Xc = X0;
      __nv_bfloat16* Xn = X1;
      for (int it = 0; it < call.steps; ++it) {
        NvtxRange nvtx_it("mo newton-schulz iteration");
        GemmOp g;                      // A = X X^T
        g.A = Xc; g.lda = L.ldx; g.strideA = L.xstride; g.a_mn = 0;
        g.B = Xc; g.ldb = L.ldx; g.strideB = L.xstride; g.b_mn = 0;
        g.M = (int)s.mp; g.N = (int)s.mp; g.K = (int)s.np; g.batch = cnt; g.sym = 1;
        g.alpha = 1.f; g.scale = inv; g.alpha_pow = it == 0 ? 2 : 0;
        g.D = A; g.ldd = L.lda; g.strideD = L.astride; g.d_f32 = 0; g.kind = PK_GRAM;
        e = launch_gemm(g, status, stream);
        if (e != cudaSuccess) return e;

        // P = a I + b A + c A A   (A symmetric: A A = A A^T); a on the
        // diagonal lets the update X' = a X + (b A + c A A) X be one product.
        // With fewer than 128 rows a row of X carries a large share of the
        // norm, P's diagonal is of the order of a, and rounding a + P_ii to
        // bf16 costs more than it does with a X kept apart: there P =
        // b A + c A A and the update reads X as C
        const bool fold = s.mp >= 128;
        GemmOp q;
        q.A = A; q.lda = L.lda; q.strideA = L.astride; q.a_mn = 0;
        q.B = A; q.ldb = L.lda; q.strideB = L.astride; q.b_mn = 0;
        q.M = (int)s.mp; q.N = (int)s.mp; q.K = (int)s.mp; q.batch = cnt; q.sym = 1;
        q.alpha = call.c; q.beta = call.b; q.diag_add = fold ? call.a : 0.f;
        q.C = A; q.ldc = L.lda; q.strideC = L.astride; q.c_f32 = 0;
        q.D = P; q.ldd = L.lda; q.strideD = L.astride; q.d_f32 = 0; q.kind = PK_POLY;
        e = launch_gemm(q, status, stream);
        if (e != cudaSuccess) return e;

        GemmOp u;                      // X' = P X, or a X + P X   (X stored [K = m'][N = n'])
        u.A = P; u.lda = L.lda; u.strideA = L.astride; u.a_mn = 0;
        u.B = Xc; u.ldb = L.ldx; u.strideB = L.xstride; u.b_mn = 1;
        u.M = (int)s.mp; u.N = (int)s.np; u.K = (int)s.mp; u.batch = cnt; u.sym = 0;
        u.alpha = 1.f; u.beta = fold ? 0.f : call.a;
        u.scale = inv; u.alpha_pow = it == 0 ? 1 : 0; u.beta_pow = (!fold && it == 0) ? 1 : 0;
        if (!fold) { u.C = Xc; u.ldc = L.ldx; u.strideC = L.xstride; u.c_f32 = 0; }
        u.D = Xn; u.ldd = L.ldx; u.strideD = L.xstride; u.d_f32 = 0; u.kind = PK_UPDATE;
        if (fused_apply && it == call.steps - 1) {
          u.epi = 2;                   // Muon apply epilogue
          u.e_tab = reinterpret_cast<float* const*>(tab + 2 * cnt);
          u.ap_decay = decay;
          u.ap_step[0] = step_of[0];
          u.ap_step[1] = step_of[1];
          u.ap_tall_from = tall_from;
          u.ap_vec = w_vec ? 1 : 0;
        }
        e = launch_gemm(u, status, stream);
        if (e != cudaSuccess) return e;
        std::swap(Xc, Xn);
      }

      // pass 2: store O (plain), or apply the scaled update when no update
      // product ran (zero iterations)
      for (const Run& r : runs) {
        if (fused_apply) break;
        auto tv = table(r);
        const NsItem& it0 = items[idx[c0 + r.first]];
        const double m = (double)it0.rows, n = (double)it0.cols;
        const double scale = call.adjust_lr == 0 ? 0.2 * std::sqrt(std::max(m, n))
                                                 : std::sqrt(std::max(1.0, m / n));
        ApplyArgs aa;
        aa.count = r.count;
        aa.mp = (int)s.mp; aa.np = (int)s.np;
        aa.tiles_r = (int)(((r.tall ? s.np : s.mp) + 63) / 64);
        aa.tiles_c = (int)(((r.tall ? s.mp : s.np) + 63) / 64);
        aa.mode = call.muon ? 1 : 0;
        aa.decay = (float)(1.0 - (double)call.lr * (double)call.wd);
        aa.step = (float)((double)call.lr * scale);
        aa.vec = tv.second;
        aa.X = Xc + (size_t)r.first * L.xstride;
        aa.ldx = L.ldx; aa.xstride = L.xstride;
        launch_apply(tv.first, aa, stream);
      }
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

}  // namespace mo
