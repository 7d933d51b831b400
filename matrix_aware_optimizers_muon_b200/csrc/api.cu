// C ABI entry points: validation, workspace planning, shape bucketing and the
// per-bucket launch sequences of the Muon and Newton-Schulz paths.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <utility>
#include <vector>

#include "../../include/mo.h"
#include "elementwise.cuh"
#include "ns_plan.h"
#include "profile.h"
#include "runtime.h"
#include "soap_plan.h"

struct mo_ctx {
  int device = 0;
  char* ws = nullptr;
  size_t ws_bytes = 0;
  int32_t detached_status = 0;   // status word of a workspace detached before it was read
  std::string err;
  bool profiling = false;
  mo::Profiler prof;
};

namespace {

mo_status fail(mo_ctx* ctx, mo_status st, const std::string& msg) {
  if (ctx) ctx->err = msg;
  return st;
}

mo_status cuda_fail(mo_ctx* ctx, cudaError_t e, const char* where) {
  return fail(ctx, MO_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

bool finite_nonneg(float x) { return std::isfinite(x) && x >= 0.f; }

// Routes the library's launch brackets to this context's profiler for the
// duration of one API call.
struct ProfBind {
  explicit ProfBind(mo_ctx* c) { mo::g_prof = (c && c->profiling) ? &c->prof : nullptr; }
  ~ProfBind() { mo::g_prof = nullptr; }
};

// device of the context must be current for launches; `scope` restores the
// caller's device when the entry point returns
mo_status enter(mo_ctx* ctx, mo::DeviceScope& scope) {
  cudaError_t e = scope.enter(ctx->device);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "cudaSetDevice");
  return MO_OK;
}

}  // namespace

extern "C" {

const char* mo_version(void) { return "mo 0.1 (sm_100a)"; }

mo_status mo_ctx_create(mo_ctx** ctx, int device) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  *ctx = nullptr;
  if (device < 0) return MO_ERR_INVALID_ARG;
  mo_ctx* c = new mo_ctx();
  c->device = device;
  *ctx = c;
  return MO_OK;
}

void mo_ctx_destroy(mo_ctx* ctx) { delete ctx; }

const char* mo_last_error(const mo_ctx* ctx) { return ctx ? ctx->err.c_str() : "null context"; }

mo_status mo_workspace_bytes(mo_ctx* ctx, int op, const int64_t* rows, const int64_t* cols, int n,
                             size_t* min_bytes, size_t* full_bytes) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && (rows == nullptr || cols == nullptr)))
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_workspace_bytes: null shape arrays");
  for (int i = 0; i < n; ++i)
    if (rows[i] <= 0 || cols[i] <= 0 || rows[i] > (1 << 20) || cols[i] > (1 << 20))
      return fail(ctx, MO_ERR_INVALID_ARG, "mo_workspace_bytes: bad shape at index " + std::to_string(i));
  size_t mn = 0, full = 0;
  if (op == 0 || op == 2) {
    mo::ns_workspace(rows, cols, n, &mn, &full);
  } else if (op == 1) {
    mo::soap_workspace(rows, cols, n, &mn, &full);
  } else {
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_workspace_bytes: op must be 0, 1 or 2");
  }
  if (min_bytes) *min_bytes = mn;
  if (full_bytes) *full_bytes = full;
  return MO_OK;
}

mo_status mo_set_workspace(mo_ctx* ctx, void* dev_ptr, size_t bytes, void* stream) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (dev_ptr == nullptr && bytes == 0) {
    // detach: keep the status word in the context, then forget the buffer
    if (ctx->ws == nullptr) return MO_OK;
    mo::DeviceScope dev_scope;
    mo_status st = enter(ctx, dev_scope);
    if (st != MO_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cap);
    if (e == cudaSuccess && cap == cudaStreamCaptureStatusNone) {
      int32_t v = 0;
      e = cudaMemcpyAsync(&v, ctx->ws, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
      if (e == cudaSuccess) e = cudaStreamSynchronize(s);
      if (e == cudaSuccess) ctx->detached_status |= v;
    }
    ctx->ws = nullptr;
    ctx->ws_bytes = 0;
    if (e != cudaSuccess) return cuda_fail(ctx, e, "mo_set_workspace (detach)");
    return MO_OK;
  }
  if (dev_ptr == nullptr || bytes < mo::WS_HEADER)
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_set_workspace: null or too small (< 256 bytes)");
  if (reinterpret_cast<uintptr_t>(dev_ptr) % 256 != 0)
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_set_workspace: pointer must be 256-byte aligned");
  mo::DeviceScope dev_scope;
  mo_status st = enter(ctx, dev_scope);
  if (st != MO_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* old = ctx->ws;
  char* ws = static_cast<char*>(dev_ptr);
  cudaError_t e = cudaSuccess;
  if (old != ws) {
    e = cudaMemsetAsync(ws, 0, mo::WS_HEADER, s);
    // a timeout code the old workspace still holds stays readable through
    // mo_device_status after the switch
    if (e == cudaSuccess && old != nullptr)
      e = cudaMemcpyAsync(ws, old, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
  }
  if (e != cudaSuccess) return cuda_fail(ctx, e, "mo_set_workspace");
  ctx->ws = ws;
  ctx->ws_bytes = bytes;
  return MO_OK;
}

mo_status mo_device_status(mo_ctx* ctx, void* stream, int32_t* status) {
  if (ctx == nullptr || status == nullptr) return MO_ERR_INVALID_ARG;
  // the attached workspace's word and the word of the fixed scratch array
  // that ns_orthogonalize_static uses on this device (once it has been set up)
  int32_t* words[2] = {reinterpret_cast<int32_t*>(ctx->ws), mo::static_status_word(ctx->device)};
  if (words[0] == nullptr && words[1] == nullptr && ctx->detached_status == 0)
    return fail(ctx, MO_ERR_NO_WORKSPACE, "mo_device_status: no workspace attached and no static call made");
  mo::DeviceScope dev_scope;
  mo_status st = enter(ctx, dev_scope);
  if (st != MO_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t got[2] = {0, 0};
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < 2 && e == cudaSuccess; ++i)
    if (words[i]) e = cudaMemcpyAsync(&got[i], words[i], sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  for (int i = 0; i < 2 && e == cudaSuccess; ++i)
    if (words[i]) e = cudaMemsetAsync(words[i], 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "mo_device_status");
  const int32_t v = got[0] | got[1] | ctx->detached_status;
  ctx->detached_status = 0;
  *status = v;
  if (v != 0) return fail(ctx, MO_ERR_DEVICE, "device status " + std::to_string(v) + ": a kernel wait timed out");
  return MO_OK;
}

// ---------------------------------------------------------------- profiling

mo_status mo_profile_enable(mo_ctx* ctx, int enable) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  ctx->profiling = enable != 0;
  ctx->prof.used = 0;
  ctx->prof.failed = false;
  return MO_OK;
}

mo_status mo_profile_read(mo_ctx* ctx, double* ms, double* flops, int64_t* launches, int nkinds) {
  if (ctx == nullptr || nkinds < 0 || (nkinds > 0 && (ms == nullptr || flops == nullptr || launches == nullptr)))
    return MO_ERR_INVALID_ARG;
  mo::DeviceScope dev_scope;
  mo_status st = enter(ctx, dev_scope);
  if (st != MO_OK) return st;
  for (int k = 0; k < nkinds; ++k) { ms[k] = 0; flops[k] = 0; launches[k] = 0; }
  if (ctx->prof.failed) return fail(ctx, MO_ERR_CUDA, "mo_profile_read: an event could not be created or recorded");
  for (size_t i = 0; i < ctx->prof.used; ++i) {
    mo::ProfRec& r = ctx->prof.recs[i];
    cudaError_t e = cudaEventSynchronize(r.b);
    float t = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "mo_profile_read");
    if (r.kind >= 0 && r.kind < nkinds) {
      ms[r.kind] += t;
      flops[r.kind] += r.flops;
      launches[r.kind] += 1;
    }
  }
  ctx->prof.used = 0;
  return MO_OK;
}

// ---------------------------------------------------------------- Muon / NS

static mo_status check_ns_coeffs(mo_ctx* ctx, int steps, float a, float b, float c, float eps,
                                 const char* who) {
  if (steps < 1 || steps > 64)
    return fail(ctx, MO_ERR_INVALID_ARG, std::string(who) + ": ns_steps must be in 1..64");
  if (!std::isfinite(a) || !std::isfinite(b) || !std::isfinite(c))
    return fail(ctx, MO_ERR_INVALID_ARG, std::string(who) + ": coefficients must be finite");
  if (!finite_nonneg(eps)) return fail(ctx, MO_ERR_INVALID_ARG, std::string(who) + ": eps must be finite and >= 0");
  return MO_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

mo_status muon_step(mo_ctx* ctx, const mo_muon_mat* mats, int n, const mo_muon_cfg* cfg, void* stream) {
  ProfBind prof_bind(ctx);
  mo::NvtxRange nvtx("mo muon_step");
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0) return fail(ctx, MO_ERR_INVALID_ARG, "muon_step: n < 0");
  if (n == 0) return MO_OK;
  if (mats == nullptr || cfg == nullptr) return fail(ctx, MO_ERR_INVALID_ARG, "muon_step: null mats or cfg");
  if (!finite_nonneg(cfg->lr) || !finite_nonneg(cfg->weight_decay))
    return fail(ctx, MO_ERR_INVALID_ARG, "muon_step: lr and weight_decay must be finite and >= 0");
  if (!(cfg->momentum >= 0.f && cfg->momentum < 1.f))
    return fail(ctx, MO_ERR_INVALID_ARG, "muon_step: momentum must be in [0, 1)");
  if (cfg->adjust_lr != 0 && cfg->adjust_lr != 1)
    return fail(ctx, MO_ERR_INVALID_ARG, "muon_step: adjust_lr must be 0 or 1");
  mo_status st = check_ns_coeffs(ctx, cfg->ns_steps, cfg->a, cfg->b, cfg->c, cfg->eps, "muon_step");
  if (st != MO_OK) return st;

  std::vector<mo::NsItem> items;
  items.reserve(n);
  for (int i = 0; i < n; ++i) {
    const mo_muon_mat& m = mats[i];
    if (m.G == nullptr) continue;
    if (m.rows <= 0 || m.cols <= 0 || m.rows > (1 << 20) || m.cols > (1 << 20))
      return fail(ctx, MO_ERR_INVALID_ARG, "muon_step: bad shape at index " + std::to_string(i));
    if (m.W == nullptr || m.momentum == nullptr)
      return fail(ctx, MO_ERR_INVALID_ARG, "muon_step: null W or momentum at index " + std::to_string(i));
    if (!aligned4(m.W) || !aligned4(m.G) || !aligned4(m.momentum))
      return fail(ctx, MO_ERR_INVALID_ARG, "muon_step: pointers must be 4-byte aligned (index " + std::to_string(i) + ")");
    mo::NsItem it;
    it.rows = m.rows; it.cols = m.cols;
    it.in = m.G; it.mom = m.momentum; it.out = m.W;
    it.flag = cfg->nonfinite ? cfg->nonfinite + i : nullptr;
    it.vec = (m.cols % 4 == 0) && aligned16(m.W) && aligned16(m.G) && aligned16(m.momentum);
    items.push_back(it);
  }
  if (items.empty()) return MO_OK;
  if (ctx->ws == nullptr) return fail(ctx, MO_ERR_NO_WORKSPACE, "muon_step: no workspace attached");
  mo::DeviceScope dev_scope;
  st = enter(ctx, dev_scope);
  if (st != MO_OK) return st;

  mo::NsCall call;
  call.muon = true;
  call.beta = cfg->momentum;
  call.nesterov = cfg->nesterov != 0;
  call.ema = cfg->momentum_ema != 0;
  call.steps = cfg->ns_steps;
  call.a = cfg->a; call.b = cfg->b; call.c = cfg->c; call.eps = cfg->eps;
  call.lr = cfg->lr; call.wd = cfg->weight_decay; call.adjust_lr = cfg->adjust_lr;
  std::string err;
  cudaError_t e = mo::ns_run(items, call, ctx->ws, ctx->ws_bytes, static_cast<cudaStream_t>(stream), &err);
  if (!err.empty()) return fail(ctx, MO_ERR_NO_WORKSPACE, "muon_step: " + err);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "muon_step");
  return MO_OK;
}

mo_status ns_orthogonalize(mo_ctx* ctx, const float* const* in, float* const* out, const int64_t* rows,
                           const int64_t* cols, int n, const mo_ns_cfg* cfg, void* stream) {
  ProfBind prof_bind(ctx);
  mo::NvtxRange nvtx("mo ns_orthogonalize");
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0) return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize: n < 0");
  if (n == 0) return MO_OK;
  if (in == nullptr || out == nullptr || rows == nullptr || cols == nullptr || cfg == nullptr)
    return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize: null argument array");
  mo_status st = check_ns_coeffs(ctx, cfg->ns_steps, cfg->a, cfg->b, cfg->c, cfg->eps, "ns_orthogonalize");
  if (st != MO_OK) return st;
  std::vector<mo::NsItem> items;
  for (int i = 0; i < n; ++i) {
    if (rows[i] <= 0 || cols[i] <= 0 || rows[i] > (1 << 20) || cols[i] > (1 << 20))
      return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize: bad shape at index " + std::to_string(i));
    if (in[i] == nullptr || out[i] == nullptr)
      return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize: null matrix at index " + std::to_string(i));
    if (!aligned4(in[i]) || !aligned4(out[i]))
      return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize: pointers must be 4-byte aligned");
    const char* a0 = reinterpret_cast<const char*>(in[i]);
    const char* b0 = reinterpret_cast<const char*>(out[i]);
    const size_t bytes = (size_t)rows[i] * cols[i] * 4;
    if (a0 < b0 + bytes && b0 < a0 + bytes)
      return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize: in and out overlap at index " + std::to_string(i));
    mo::NsItem it;
    it.rows = rows[i]; it.cols = cols[i];
    it.in = in[i]; it.mom = nullptr; it.out = out[i];
    it.flag = cfg->nonfinite ? cfg->nonfinite + i : nullptr;
    it.vec = (cols[i] % 4 == 0) && aligned16(in[i]) && aligned16(out[i]);
    items.push_back(it);
  }
  if (ctx->ws == nullptr) return fail(ctx, MO_ERR_NO_WORKSPACE, "ns_orthogonalize: no workspace attached");
  mo::DeviceScope dev_scope;
  st = enter(ctx, dev_scope);
  if (st != MO_OK) return st;
  mo::NsCall call;
  call.muon = false;
  call.steps = cfg->ns_steps;
  call.a = cfg->a; call.b = cfg->b; call.c = cfg->c; call.eps = cfg->eps;
  std::string err;
  cudaError_t e = mo::ns_run(items, call, ctx->ws, ctx->ws_bytes, static_cast<cudaStream_t>(stream), &err);
  if (!err.empty()) return fail(ctx, MO_ERR_NO_WORKSPACE, "ns_orthogonalize: " + err);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "ns_orthogonalize");
  return MO_OK;
}

// Strided batches of equal shape: the per-matrix pointer lists are built
// here, so the caller passes O(1) arguments for any number of matrices.
mo_status ns_orthogonalize_strided(mo_ctx* ctx, const float* in, int64_t in_stride, float* out,
                                   int64_t out_stride, int64_t rows, int64_t cols, int n, const mo_ns_cfg* cfg,
                                   void* stream) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0) return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize_strided: n < 0");
  if (n == 0) return MO_OK;
  if (in == nullptr || out == nullptr || cfg == nullptr)
    return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize_strided: null argument");
  if (rows <= 0 || cols <= 0 || (n > 1 && (in_stride < rows * cols || out_stride < rows * cols)))
    return fail(ctx, MO_ERR_INVALID_ARG, "ns_orthogonalize_strided: bad shape or a stride below rows * cols");
  std::vector<const float*> ins(n);
  std::vector<float*> outs(n);
  std::vector<int64_t> r(n, rows), c(n, cols);
  for (int i = 0; i < n; ++i) {
    ins[i] = in + (size_t)i * in_stride;
    outs[i] = out + (size_t)i * out_stride;
  }
  return ns_orthogonalize(ctx, ins.data(), outs.data(), r.data(), c.data(), n, cfg, stream);
}

mo_status muon_step_strided(mo_ctx* ctx, float* W, const float* G, float* momentum, int64_t stride, int64_t rows,
                            int64_t cols, int n, const mo_muon_cfg* cfg, void* stream) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0) return fail(ctx, MO_ERR_INVALID_ARG, "muon_step_strided: n < 0");
  if (n == 0) return MO_OK;
  if (W == nullptr || G == nullptr || momentum == nullptr || cfg == nullptr)
    return fail(ctx, MO_ERR_INVALID_ARG, "muon_step_strided: null argument");
  if (rows <= 0 || cols <= 0 || (n > 1 && stride < rows * cols))
    return fail(ctx, MO_ERR_INVALID_ARG, "muon_step_strided: bad shape or a stride below rows * cols");
  std::vector<mo_muon_mat> mats(n);
  for (int i = 0; i < n; ++i) {
    const size_t off = (size_t)i * stride;
    mats[i].rows = rows;
    mats[i].cols = cols;
    mats[i].W = W + off;
    mats[i].G = G + off;
    mats[i].momentum = momentum + off;
  }
  return muon_step(ctx, mats.data(), n, cfg, stream);
}

// ---------------------------------------------------------------- SOAP

namespace {

// Validation and launch shared by soap_step and soap_muon_step (ext != null;
// then M is the Muon momentum B).
mo_status soap_impl(mo_ctx* ctx, const mo_soap_mat* mats, int n, const mo_soap_cfg* cfg, int64_t step,
                    void* stream, const mo::SoapMuonExt* ext) {
  const std::string fn = ext ? "soap_muon_step" : "soap_step";
  if (step < 1) return fail(ctx, MO_ERR_INVALID_ARG, fn + ": step must be >= 1");
  if (!finite_nonneg(cfg->lr) || !finite_nonneg(cfg->weight_decay) || !finite_nonneg(cfg->eps))
    return fail(ctx, MO_ERR_INVALID_ARG, fn + ": lr, weight_decay and eps must be finite and >= 0");
  auto beta_ok = [](float b) { return b >= 0.f && b < 1.f; };
  if (!beta_ok(cfg->beta1) || !beta_ok(cfg->beta2) || !beta_ok(cfg->shampoo_beta))
    return fail(ctx, MO_ERR_INVALID_ARG, fn + ": betas must be in [0, 1)");
  if (!(cfg->damping >= 0.f && cfg->damping <= 1e-2f))
    return fail(ctx, MO_ERR_INVALID_ARG, fn + ": damping must be in [0, 1e-2]");
  std::vector<mo::SoapItem> items;
  for (int i = 0; i < n; ++i) {
    const mo_soap_mat& m = mats[i];
    if (m.G == nullptr) continue;
    if (m.rows <= 0 || m.cols <= 0 || m.rows > (1 << 16) || m.cols > (1 << 20))
      return fail(ctx, MO_ERR_INVALID_ARG, fn + ": bad shape at index " + std::to_string(i));
    if (m.W == nullptr || m.M == nullptr || m.V == nullptr)
      return fail(ctx, MO_ERR_INVALID_ARG, fn + ": null W, M or V at index " + std::to_string(i));
    if ((m.L == nullptr) != (m.QL == nullptr) || (m.R == nullptr) != (m.QR == nullptr))
      return fail(ctx, MO_ERR_INVALID_ARG, fn + ": a side needs both its factor and its basis (index " + std::to_string(i) + ")");
    if ((m.L && m.rows > 16384) || (m.R && m.cols > 16384))
      return fail(ctx, MO_ERR_UNSUPPORTED, fn + ": factor sides above 16384 are not supported; pass NULL for an identity basis");
    const void* ptrs[8] = {m.W, m.G, m.M, m.V, m.L, m.QL, m.R, m.QR};
    for (const void* p : ptrs)
      if (p && !aligned16(p))
        return fail(ctx, MO_ERR_INVALID_ARG, fn + ": pointers must be 16-byte aligned (index " + std::to_string(i) + ")");
    if (m.cols % 8 != 0 || m.rows % 8 != 0)
      return fail(ctx, MO_ERR_UNSUPPORTED, fn + ": rows and cols must be multiples of 8 (index " + std::to_string(i) + ")");
    mo::SoapItem it;
    it.m = m;
    it.flag = cfg->nonfinite ? cfg->nonfinite + i : nullptr;
    items.push_back(it);
  }
  if (items.empty()) return MO_OK;
  if (ctx->ws == nullptr) return fail(ctx, MO_ERR_NO_WORKSPACE, fn + ": no workspace attached");
  mo::DeviceScope dev_scope;
  mo_status st = enter(ctx, dev_scope);
  if (st != MO_OK) return st;
  std::string err;
  cudaError_t e = mo::soap_run(items, *cfg, step, ctx->ws, ctx->ws_bytes, static_cast<cudaStream_t>(stream), &err, ext);
  if (!err.empty()) return fail(ctx, e == cudaErrorNotSupported ? MO_ERR_UNSUPPORTED : MO_ERR_NO_WORKSPACE, fn + ": " + err);
  if (e != cudaSuccess) return cuda_fail(ctx, e, fn.c_str());
  return MO_OK;
}

mo_soap_mat as_soap_mat(const mo_soap_muon_mat& a) {
  mo_soap_mat m;
  m.rows = a.rows; m.cols = a.cols; m.W = a.W; m.G = a.G; m.M = a.B; m.V = a.V;
  m.L = a.L; m.QL = a.QL; m.R = a.R; m.QR = a.QR;
  return m;
}

}  // namespace

mo_status soap_step(mo_ctx* ctx, const mo_soap_mat* mats, int n, const mo_soap_cfg* cfg, int64_t step,
                    void* stream) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0) return fail(ctx, MO_ERR_INVALID_ARG, "soap_step: n < 0");
  ProfBind prof_bind(ctx);
  mo::NvtxRange nvtx("mo soap_step");
  if (n == 0) return MO_OK;
  if (mats == nullptr || cfg == nullptr) return fail(ctx, MO_ERR_INVALID_ARG, "soap_step: null mats or cfg");
  return soap_impl(ctx, mats, n, cfg, step, stream, nullptr);
}

mo_status soap_muon_step(mo_ctx* ctx, const mo_soap_muon_mat* mats, int n, const mo_soap_muon_cfg* cfg,
                         int64_t step, void* stream) {
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0) return fail(ctx, MO_ERR_INVALID_ARG, "soap_muon_step: n < 0");
  ProfBind prof_bind(ctx);
  mo::NvtxRange nvtx("mo soap_muon_step");
  if (n == 0) return MO_OK;
  if (mats == nullptr || cfg == nullptr) return fail(ctx, MO_ERR_INVALID_ARG, "soap_muon_step: null mats or cfg");
  if (!(cfg->momentum >= 0.f && cfg->momentum < 1.f))
    return fail(ctx, MO_ERR_INVALID_ARG, "soap_muon_step: momentum must be in [0, 1)");
  if (cfg->adjust_lr != 0 && cfg->adjust_lr != 1)
    return fail(ctx, MO_ERR_INVALID_ARG, "soap_muon_step: adjust_lr must be 0 or 1");
  mo_status st = check_ns_coeffs(ctx, cfg->ns_steps, cfg->a, cfg->b, cfg->c, cfg->ns_eps, "soap_muon_step");
  if (st != MO_OK) return st;
  std::vector<mo_soap_mat> sm(n);
  for (int i = 0; i < n; ++i) sm[i] = as_soap_mat(mats[i]);
  mo_soap_cfg sc;
  sc.lr = cfg->lr; sc.beta1 = cfg->momentum; sc.beta2 = cfg->beta2; sc.shampoo_beta = cfg->shampoo_beta;
  sc.eps = cfg->eps; sc.weight_decay = cfg->weight_decay; sc.bias_correction = cfg->bias_correction;
  sc.nonfinite = cfg->nonfinite; sc.skip_refresh = cfg->skip_refresh; sc.damping = cfg->damping;
  mo::SoapMuonExt ext;
  ext.mu = cfg->momentum;
  ext.nesterov = cfg->nesterov != 0;
  ext.ns.steps = cfg->ns_steps;
  ext.ns.a = cfg->a; ext.ns.b = cfg->b; ext.ns.c = cfg->c; ext.ns.eps = cfg->ns_eps;
  ext.ns.adjust_lr = cfg->adjust_lr;
  return soap_impl(ctx, sm.data(), n, &sc, step, stream, &ext);
}

mo_status mo_soap_workspace_bytes(mo_ctx* ctx, const mo_soap_mat* mats, int n, size_t* bytes) {
  if (ctx == nullptr || bytes == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && mats == nullptr)) return fail(ctx, MO_ERR_INVALID_ARG, "mo_soap_workspace_bytes: bad arguments");
  std::vector<mo::SoapItem> items;
  for (int i = 0; i < n; ++i) {
    if (mats[i].rows <= 0 || mats[i].cols <= 0 || mats[i].rows > (1 << 16) || mats[i].cols > (1 << 20))
      return fail(ctx, MO_ERR_INVALID_ARG, "mo_soap_workspace_bytes: bad shape at index " + std::to_string(i));
    mo::SoapItem it;
    it.m = mats[i];
    items.push_back(it);
  }
  *bytes = mo::soap_workspace_exact(items);
  return MO_OK;
}

mo_status mo_soap_muon_workspace_bytes(mo_ctx* ctx, const mo_soap_muon_mat* mats, int n, size_t* bytes) {
  if (ctx == nullptr || bytes == nullptr) return MO_ERR_INVALID_ARG;
  if (n < 0 || (n > 0 && mats == nullptr))
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_soap_muon_workspace_bytes: bad arguments");
  std::vector<mo::SoapItem> items;
  for (int i = 0; i < n; ++i) {
    if (mats[i].rows <= 0 || mats[i].cols <= 0 || mats[i].rows > (1 << 16) || mats[i].cols > (1 << 20))
      return fail(ctx, MO_ERR_INVALID_ARG, "mo_soap_muon_workspace_bytes: bad shape at index " + std::to_string(i));
    mo::SoapItem it;
    it.m = as_soap_mat(mats[i]);
    items.push_back(it);
  }
  *bytes = mo::soap_workspace_exact(items, true);
  return MO_OK;
}

// ---------------------------------------------------------------- GEMM block

mo_status mo_gemm_bf16(mo_ctx* ctx, const mo_gemm_desc* d, void* stream) {
  ProfBind prof_bind(ctx);
  mo::NvtxRange nvtx("mo gemm_bf16");
  if (ctx == nullptr) return MO_ERR_INVALID_ARG;
  if (d == nullptr) return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: null descriptor");
  if (d->M <= 0 || d->N <= 0 || d->K <= 0 || d->batch <= 0)
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: M, N, K and batch must be positive");
  if (d->A == nullptr || d->B == nullptr || d->D == nullptr)
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: null A, B or D");
  if (d->sym && d->M != d->N) return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: sym needs M == N");
  if (!aligned16(d->A) || !aligned16(d->B) || d->lda % 8 || d->ldb % 8 || d->strideA % 8 || d->strideB % 8)
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: A/B need 16-byte aligned bases and strides that are multiples of 8");
  const long long a_cols = d->a_mn ? d->M : d->K;
  const long long b_cols = d->b_mn ? d->N : d->K;
  if (d->lda < a_cols || d->ldb < b_cols || d->ldd < d->N || (d->C && d->ldc < d->N))
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: leading dimension smaller than the row length");
  const int eb = d->d_f32 ? 4 : 2;
  const int cb = d->c_f32 ? 4 : 2;
  if (!aligned16(d->D) || (d->ldd * eb) % 16 || (d->strideD * eb) % 16 ||
      (d->C && (!aligned16(d->C) || (d->ldc * cb) % 16 || (d->strideC * cb) % 16)))
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: C/D need 16-byte aligned bases and rows");
  if (d->alpha_pow < 0 || d->alpha_pow > 2 || d->beta_pow < 0 || d->beta_pow > 2)
    return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: alpha_pow and beta_pow must be 0, 1 or 2");
  if (d->band < 0) return fail(ctx, MO_ERR_INVALID_ARG, "mo_gemm_bf16: band must be >= 0");
  if (ctx->ws == nullptr) return fail(ctx, MO_ERR_NO_WORKSPACE, "mo_gemm_bf16: no workspace attached (status word)");
  mo::DeviceScope dev_scope;
  mo_status st = enter(ctx, dev_scope);
  if (st != MO_OK) return st;
  mo::GemmOp op;
  op.A = d->A; op.lda = d->lda; op.strideA = d->strideA; op.a_mn = d->a_mn;
  op.B = d->B; op.ldb = d->ldb; op.strideB = d->strideB; op.b_mn = d->b_mn;
  op.M = d->M; op.N = d->N; op.K = d->K; op.batch = d->batch; op.sym = d->sym;
  op.alpha = d->alpha; op.beta = d->beta; op.scale = d->scale;
  op.alpha_pow = d->alpha_pow; op.beta_pow = d->beta_pow;
  op.C = d->C; op.ldc = d->ldc; op.strideC = d->strideC; op.c_f32 = d->c_f32;
  op.D = d->D; op.ldd = d->ldd; op.strideD = d->strideD; op.d_f32 = d->d_f32;
  op.band = d->band;
  cudaError_t e = mo::launch_gemm(op, reinterpret_cast<int*>(ctx->ws), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(ctx, e, "mo_gemm_bf16");
  return MO_OK;
}

}  // extern "C"

// Accessors for entry points defined in other translation units.
namespace mo {
int ctx_device(const mo_ctx* ctx) { return ctx->device; }
mo_status ctx_fail(mo_ctx* ctx, mo_status st, const std::string& msg) { return fail(ctx, st, msg); }
}  // namespace mo
