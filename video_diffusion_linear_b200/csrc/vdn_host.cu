// C ABI of libvdn: argument validation, the workspace plan and the launch
// sequence of the branch on the caller's stream.  See include/vdn.h.
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "image.cuh"
#include "internal.h"

using namespace vdn;

namespace vdn {

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

#ifndef VDN_HAVE_TC
#define VDN_HAVE_TC 1
#endif

bool use_tc(const vdn_shape& sh, int impl) {
  bool ok = sh.dtype == VDN_DTYPE_BF16 && sh.d == 128;
  if (impl == VDN_IMPL_SIMT) return false;
  if (impl == VDN_IMPL_AUTO && !VDN_HAVE_TC) return false;
  return ok;
}

WsPlan plan_workspace(const vdn_shape& sh, int /*rule*/, bool tc) {
  WsPlan p;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t d = (size_t)sh.d;
  const size_t NF = (size_t)sh.B * sh.H * sh.F;
  const size_t frame_mats = NF * d * d * sizeof(float);
  p.status = take(256);
  p.pexp = take(NF * sizeof(int));
  p.qexp = take(NF * sizeof(int));
  p.wexp = take(NF * sizeof(int));
  if (!tc) {
    const size_t feat = (size_t)sh.B * sh.F * sh.S * sh.H * d * sizeof(float);
    p.qf = take(feat);
    p.kf = take(feat);
    p.vf = take(feat);
    p.A = take(frame_mats);
    p.Bm = take(frame_mats);
    p.Nm = take(frame_mats);
    p.P = take(frame_mats);
    p.Q = take(frame_mats);
    p.W = take(frame_mats);
  } else {
    const size_t slots = NF + kStatsGrid;
    p.part = take(slots * d * 2 * d * sizeof(float));
    p.Bm = take(frame_mats);
    p.nimg = take(NF * (size_t)kImgBytes);
    p.P = take(frame_mats);
    p.Q = take(frame_mats);
    p.wimg = take(NF * (size_t)kWImgBytes);
    p.wbexp = take(NF * kWRowBlocks * sizeof(int));
  }
  p.total = off;
  return p;
}

}  // namespace vdn

namespace {

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

struct Range {
  uintptr_t lo, hi;
};
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

vdn_status check_shape(const vdn_shape* sh) {
  if (!sh) return VDN_ERR_INVALID_ARG;
  if (sh->B < 1 || sh->H < 1 || sh->F < 1 || sh->S < 1 || sh->d < 1 || sh->conv_width < 1)
    return VDN_ERR_INVALID_ARG;
  if (sh->dtype != VDN_DTYPE_F32 && sh->dtype != VDN_DTYPE_BF16) return VDN_ERR_INVALID_ARG;
  if (sh->d != 16 && sh->d != 128) return VDN_ERR_UNSUPPORTED;
  if (sh->conv_width != 1 && sh->conv_width != 3) return VDN_ERR_UNSUPPORTED;
  if (sh->dtype == VDN_DTYPE_BF16 && sh->d != 128) return VDN_ERR_UNSUPPORTED;
  // index ranges used by the kernels: tokens of one batch element and frame
  // triples must fit in int32, and the whole tensor in 2^62 bytes.
  long long N = (long long)sh->F * sh->S;
  long long NF = (long long)sh->B * sh->H * sh->F;
  if (N > 0x7fffffffLL || NF > 0x7fffffffLL || 2LL * sh->B * sh->H > 0x7fffffffLL) return VDN_ERR_UNSUPPORTED;
  double bytes = (double)sh->B * N * sh->H * sh->d * 4.0;
  if (bytes > 4.0e18) return VDN_ERR_UNSUPPORTED;
  return VDN_OK;
}

size_t elem_size(int dtype) { return dtype == VDN_DTYPE_BF16 ? 2 : 4; }

vdn_status validate(const vdn_shape* sh, const void* q, const void* k, const void* v, const float* beta,
                    const float* alpha, const void* gate, const float* rms_w, const float* conv_k_w,
                    const float* conv_v_w, const float* text_state, int rule, float c, int chunk, int radius,
                    void* workspace, size_t workspace_bytes, void* out, int impl) {
  vdn_status s = check_shape(sh);
  if (s != VDN_OK) return s;
  if (rule < VDN_RULE_SANA_SCALED || rule > VDN_RULE_ADDITIVE) return VDN_ERR_INVALID_ARG;
  if (impl < VDN_IMPL_AUTO || impl > VDN_IMPL_TC) return VDN_ERR_INVALID_ARG;
  if (impl == VDN_IMPL_TC && !(sh->dtype == VDN_DTYPE_BF16 && sh->d == 128)) return VDN_ERR_UNSUPPORTED;
  if (chunk < 1 || radius < 0 || !std::isfinite(c)) return VDN_ERR_INVALID_ARG;
  if (!q || !k || !v || !beta || !alpha || !gate || !rms_w || !out || !workspace) return VDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, out};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return VDN_ERR_ALIGNMENT;
  if (!aligned(workspace, 256)) return VDN_ERR_ALIGNMENT;
  WsPlan plan = plan_workspace(*sh, rule, use_tc(*sh, impl));
  if (workspace_bytes < plan.total) return VDN_ERR_WORKSPACE;
  // out must not overlap any input nor the workspace
  const size_t es = elem_size(sh->dtype);
  const size_t tok = (size_t)sh->B * sh->F * sh->S * sh->H;
  const size_t big = tok * sh->d * es;
  const size_t d = (size_t)sh->d;
  Range ro{(uintptr_t)out, (uintptr_t)out + big};
  Range rin[] = {
      {(uintptr_t)q, (uintptr_t)q + big},
      {(uintptr_t)k, (uintptr_t)k + big},
      {(uintptr_t)v, (uintptr_t)v + big},
      {(uintptr_t)gate, (uintptr_t)gate + big},
      {(uintptr_t)beta, (uintptr_t)beta + tok * 4},
      {(uintptr_t)alpha, (uintptr_t)alpha + (size_t)sh->B * sh->F * sh->H * d * 4},
      {(uintptr_t)rms_w, (uintptr_t)rms_w + d * 4},
      {(uintptr_t)conv_k_w, conv_k_w ? (uintptr_t)conv_k_w + (size_t)sh->H * d * sh->conv_width * 4 : 0},
      {(uintptr_t)conv_v_w, conv_v_w ? (uintptr_t)conv_v_w + (size_t)sh->H * d * sh->conv_width * 4 : 0},
      {(uintptr_t)text_state, text_state ? (uintptr_t)text_state + (size_t)sh->H * d * d * 4 : 0},
      {(uintptr_t)workspace, (uintptr_t)workspace + plan.total},
  };
  for (const Range& r : rin)
    if (r.hi > r.lo && overlap(ro, r)) return VDN_ERR_INVALID_ARG;
  return VDN_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

#define VDN_LAUNCH(expr)                   \
  do {                                     \
    cudaError_t e_ = (expr);               \
    if (e_ != cudaSuccess) return VDN_ERR_CUDA; \
  } while (0)

vdn_status run_forward(const Args& a, void* ws, int impl, void* const* events = nullptr) {
  const bool tc = use_tc(a.sh, impl);
  int ev = 0;
  auto mark = [&]() -> cudaError_t {
    if (!events) return cudaSuccess;
    return cudaEventRecord((cudaEvent_t)events[ev++], a.stream);
  };
  WsPlan p = plan_workspace(a.sh, a.rule, tc);
  const vdn_debug_out* dbg = a.dbg;
  uint32_t* status = at<uint32_t>(ws, p.status);
  VDN_LAUNCH(cudaMemsetAsync(status, 0, sizeof(uint32_t), a.stream));
  VDN_LAUNCH(mark());
  if (!tc) {
    float *qf = at<float>(ws, p.qf), *kf = at<float>(ws, p.kf), *vf = at<float>(ws, p.vf);
    float *A = at<float>(ws, p.A), *Bm = at<float>(ws, p.Bm), *Nm = at<float>(ws, p.Nm);
    float *P = at<float>(ws, p.P), *Q = at<float>(ws, p.Q), *W = at<float>(ws, p.W);
    int *pexp = at<int>(ws, p.pexp), *qexp = at<int>(ws, p.qexp), *wexp = at<int>(ws, p.wexp);
    VDN_LAUNCH(launch_features_simt(a, qf, kf, vf));
    VDN_LAUNCH(mark());
    VDN_LAUNCH(launch_stats_simt(a, kf, vf, A, Bm));
    VDN_LAUNCH(mark());
    VDN_LAUNCH(launch_solve(a, A, Nm, nullptr, nullptr, nullptr, nullptr));
    VDN_LAUNCH(mark());
    VDN_LAUNCH(launch_scan_simt(a, Bm, Nm, P, Q, pexp, qexp));
    VDN_LAUNCH(mark());
    VDN_LAUNCH(launch_gather(a, P, Q, pexp, qexp, W, nullptr, wexp, nullptr));
    VDN_LAUNCH(mark());
    VDN_LAUNCH(launch_readout_simt(a, qf, W, wexp));
    VDN_LAUNCH(mark());
    if (dbg) {
      if (dbg->A) VDN_LAUNCH(launch_copy_frames(a, A, dbg->A));
      if (dbg->B) VDN_LAUNCH(launch_copy_frames(a, Bm, dbg->B));
      if (dbg->N) VDN_LAUNCH(launch_copy_frames(a, Nm, dbg->N));
      if (dbg->P) VDN_LAUNCH(launch_copy_frames(a, P, dbg->P, pexp));
      if (dbg->Q) VDN_LAUNCH(launch_copy_frames(a, Q, dbg->Q, qexp));
      if (dbg->W) VDN_LAUNCH(launch_copy_frames(a, W, dbg->W, wexp));
    }
    return VDN_OK;
  }
  float* part = at<float>(ws, p.part);
  float* Bsum = at<float>(ws, p.Bm);
  uint16_t* nimg = at<uint16_t>(ws, p.nimg);
  float *P = at<float>(ws, p.P), *Q = at<float>(ws, p.Q);
  uint16_t* wimg = at<uint16_t>(ws, p.wimg);
  int* wbexp = at<int>(ws, p.wbexp);
  int *pexp = at<int>(ws, p.pexp), *qexp = at<int>(ws, p.qexp), *wexp = at<int>(ws, p.wexp);
  bool all_frames = dbg && (dbg->P || dbg->Q);
  // the debug export of W: the gather writes 2^-wexp W_t into dbg->W, rescaled in place below
  VDN_LAUNCH(launch_stats_tc(a, part, status));
  VDN_LAUNCH(mark());
  VDN_LAUNCH(launch_solve(a, nullptr, dbg ? dbg->N : nullptr, nimg, part, Bsum, dbg ? dbg->A : nullptr));
  VDN_LAUNCH(mark());
  VDN_LAUNCH(launch_scan_tc(a, Bsum, nimg, P, Q, pexp, qexp, all_frames, status));
  VDN_LAUNCH(mark());
  VDN_LAUNCH(launch_gather(a, P, Q, pexp, qexp, dbg ? dbg->W : nullptr, wimg, wexp, wbexp));
  VDN_LAUNCH(mark());
  VDN_LAUNCH(launch_readout_tc(a, wimg, wexp, wbexp, status));
  VDN_LAUNCH(mark());
  if (dbg) {
    if (dbg->B) VDN_LAUNCH(launch_copy_frames(a, Bsum, dbg->B));
    if (dbg->P) VDN_LAUNCH(launch_copy_frames(a, P, dbg->P, pexp));
    if (dbg->Q) VDN_LAUNCH(launch_copy_frames(a, Q, dbg->Q, qexp));
    if (dbg->W) VDN_LAUNCH(launch_copy_frames(a, dbg->W, dbg->W, wexp));
  }
  return VDN_OK;
}

vdn_status forward_common(const vdn_shape* shape, const void* q, const void* k, const void* v, const float* beta,
                          const float* alpha, const void* gate, const float* rms_w, const float* conv_k_w,
                          const float* conv_v_w, const float* text_state, int rule, float c, int chunk, int radius,
                          void* workspace, size_t workspace_bytes, void* out, void* stream,
                          const vdn_debug_out* dbg, void* const* events = nullptr, int n_events = 0) {
  int impl = dbg ? dbg->impl : VDN_IMPL_AUTO;
  vdn_status s = validate(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                          radius, workspace, workspace_bytes, out, impl);
  if (s != VDN_OK) return s;
  if (dbg) {
    const float* dp[] = {dbg->A, dbg->B, dbg->N, dbg->P, dbg->Q, dbg->W};
    for (const float* p : dp)
      if (p && !aligned(p, 16)) return VDN_ERR_ALIGNMENT;
  }
  Args a;
  a.sh = *shape;
  a.q = q; a.k = k; a.v = v;
  a.beta = beta; a.alpha = alpha; a.gate = gate; a.rms_w = rms_w;
  a.conv_k_w = conv_k_w; a.conv_v_w = conv_v_w; a.text_state = text_state;
  a.rule = rule; a.c = (rule == VDN_RULE_VDN_SOLVE || rule == VDN_RULE_ADDITIVE) ? 1.0f : c;
  a.chunk = chunk; a.radius = radius;
  a.out = out;
  a.stream = (cudaStream_t)stream;
  a.dbg = dbg;
  if (events) {
    const int need = (use_tc(a.sh, impl) ? 5 : 6) + 1;
    if (n_events < need) return VDN_ERR_INVALID_ARG;
    for (int i = 0; i < need; ++i)
      if (!events[i]) return VDN_ERR_INVALID_ARG;
  }
  return run_forward(a, workspace, impl, events);
}

vdn_status check_softmax_args(const vdn_shape* sh, const void* qr, const void* kr, const void* v, int chunk,
                              int radius, float scale, int accumulate, const void* workspace,
                              size_t workspace_bytes, size_t need, const void* out) {
  vdn_status s = check_shape(sh);
  if (s != VDN_OK) return s;
  if (chunk < 1 || radius < 0 || !std::isfinite(scale) || (accumulate != 0 && accumulate != 1))
    return VDN_ERR_INVALID_ARG;
  if (!qr || !kr || !v || !out || !workspace) return VDN_ERR_INVALID_ARG;
  const void* ptrs[] = {qr, kr, v, out};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return VDN_ERR_ALIGNMENT;
  if (!aligned(workspace, 256)) return VDN_ERR_ALIGNMENT;
  if (workspace_bytes < need) return VDN_ERR_WORKSPACE;
  const size_t big = (size_t)sh->B * sh->F * sh->S * sh->H * sh->d * elem_size(sh->dtype);
  const Range ro{(uintptr_t)out, (uintptr_t)out + big};
  const Range rin[] = {{(uintptr_t)qr, (uintptr_t)qr + big},
                       {(uintptr_t)kr, (uintptr_t)kr + big},
                       {(uintptr_t)v, (uintptr_t)v + big},
                       {(uintptr_t)workspace, (uintptr_t)workspace + need}};
  for (const Range& r : rin)
    if (overlap(ro, r)) return VDN_ERR_INVALID_ARG;
  return VDN_OK;
}

vdn_status run_window_softmax(const vdn_shape& sh, const void* qr, const void* kr, const void* v, int chunk,
                              int radius, float scale, int accumulate, uint32_t* status, void* out,
                              cudaStream_t stream) {
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt((float)sh.d);
  cudaError_t e = (sh.dtype == VDN_DTYPE_BF16 && sh.d == 128 && VDN_HAVE_TC)
                      ? launch_window_softmax_tc(sh, qr, kr, v, chunk, radius, sc, accumulate, out, status, stream)
                      : launch_window_softmax_simt(sh, qr, kr, v, chunk, radius, sc, accumulate, out, stream);
  return e == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t vdn_branch_workspace_size_impl(const vdn_shape* shape, int rule, int impl) {
  if (check_shape(shape) != VDN_OK) return 0;
  if (rule < VDN_RULE_SANA_SCALED || rule > VDN_RULE_ADDITIVE) return 0;
  if (impl < VDN_IMPL_AUTO || impl > VDN_IMPL_TC) return 0;
  if (impl == VDN_IMPL_TC && !(shape->dtype == VDN_DTYPE_BF16 && shape->d == 128)) return 0;
  return plan_workspace(*shape, rule, use_tc(*shape, impl)).total;
}

size_t vdn_branch_workspace_size(const vdn_shape* shape, int rule) {
  return vdn_branch_workspace_size_impl(shape, rule, VDN_IMPL_AUTO);
}

size_t vdn_branch_backward_workspace_size(const vdn_shape* shape, int rule) {
  if (check_shape(shape) != VDN_OK) return 0;
  if (rule < VDN_RULE_SANA_SCALED || rule > VDN_RULE_ADDITIVE) return 0;
  return plan_backward(*shape, rule).total;
}

}  // extern "C"

namespace {
vdn_status backward_common(const vdn_shape* shape, const void* q, const void* k, const void* v, const float* beta,
                           const float* alpha, const void* gate, const float* rms_w, const float* conv_k_w,
                           const float* conv_v_w, const float* text_state, int rule, float c, int chunk, int radius,
                           const void* dout, void* workspace, size_t workspace_bytes, void* dq, void* dk, void* dv,
                           float* dbeta, float* dalpha, void* dgate, float* drms_w, float* dconv_k_w,
                           float* dconv_v_w, float* dtext_state, void* stream, void* const* events, int n_events,
                           const void* saved = nullptr, size_t saved_bytes = 0) {
  // the forward's checks, with dq standing for the output (it must not overlap an input either);
  // the backward's own workspace size is checked below
  if (check_shape(shape) != VDN_OK) return check_shape(shape);
  const bool recompute = saved == nullptr;
  const BwdPlan plan = plan_backward(*shape, rule < VDN_RULE_SANA_SCALED || rule > VDN_RULE_ADDITIVE
                                                 ? VDN_RULE_VDN_SOLVE : rule, recompute);
  vdn_status s = validate(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                          radius, workspace, SIZE_MAX, dq, VDN_IMPL_AUTO);
  if (s != VDN_OK) return s;
  if (workspace_bytes < plan.total) return VDN_ERR_WORKSPACE;
  const SavedPlan sp = plan_saved(*shape);
  if (!recompute && (saved_bytes < sp.total || !aligned(saved, 256))) return saved_bytes < sp.total
                                                                              ? VDN_ERR_WORKSPACE
                                                                              : VDN_ERR_ALIGNMENT;
  if (!dout || !dk || !dv || !dbeta || !dalpha || !dgate || !drms_w) return VDN_ERR_INVALID_ARG;
  // a gradient exists exactly for the optional inputs that were given
  if ((conv_k_w == nullptr) != (dconv_k_w == nullptr) || (conv_v_w == nullptr) != (dconv_v_w == nullptr) ||
      (text_state == nullptr) != (dtext_state == nullptr))
    return VDN_ERR_INVALID_ARG;
  const void* ptrs[] = {dout, dk, dv, dbeta, dalpha, dgate, drms_w, dconv_k_w, dconv_v_w, dtext_state};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return VDN_ERR_ALIGNMENT;
  // gradients must not overlap each other, an input or the workspace
  const size_t es = elem_size(shape->dtype);
  const size_t tok = (size_t)shape->B * shape->F * shape->S * shape->H;
  const size_t big = tok * shape->d * es;
  const size_t d = (size_t)shape->d;
  const size_t nal = (size_t)shape->B * shape->F * shape->H * d * 4;
  const size_t ntap = (size_t)shape->H * d * shape->conv_width * 4;
  const Range outs[] = {
      {(uintptr_t)dq, (uintptr_t)dq + big}, {(uintptr_t)dk, (uintptr_t)dk + big},
      {(uintptr_t)dv, (uintptr_t)dv + big}, {(uintptr_t)dgate, (uintptr_t)dgate + big},
      {(uintptr_t)dbeta, (uintptr_t)dbeta + tok * 4}, {(uintptr_t)dalpha, (uintptr_t)dalpha + nal},
      {(uintptr_t)drms_w, (uintptr_t)drms_w + d * 4},
      {(uintptr_t)dconv_k_w, dconv_k_w ? (uintptr_t)dconv_k_w + ntap : 0},
      {(uintptr_t)dconv_v_w, dconv_v_w ? (uintptr_t)dconv_v_w + ntap : 0},
      {(uintptr_t)dtext_state, dtext_state ? (uintptr_t)dtext_state + (size_t)shape->H * d * d * 4 : 0},
  };
  const Range ins[] = {
      {(uintptr_t)q, (uintptr_t)q + big}, {(uintptr_t)k, (uintptr_t)k + big}, {(uintptr_t)v, (uintptr_t)v + big},
      {(uintptr_t)gate, (uintptr_t)gate + big}, {(uintptr_t)dout, (uintptr_t)dout + big},
      {(uintptr_t)beta, (uintptr_t)beta + tok * 4}, {(uintptr_t)alpha, (uintptr_t)alpha + nal},
      {(uintptr_t)rms_w, (uintptr_t)rms_w + d * 4},
      {(uintptr_t)conv_k_w, conv_k_w ? (uintptr_t)conv_k_w + ntap : 0},
      {(uintptr_t)conv_v_w, conv_v_w ? (uintptr_t)conv_v_w + ntap : 0},
      {(uintptr_t)text_state, text_state ? (uintptr_t)text_state + (size_t)shape->H * d * d * 4 : 0},
      {(uintptr_t)workspace, (uintptr_t)workspace + plan.total},
      {(uintptr_t)saved, saved ? (uintptr_t)saved + sp.total : 0},
  };
  const int no = sizeof(outs) / sizeof(outs[0]), ni = sizeof(ins) / sizeof(ins[0]);
  for (int i = 0; i < no; ++i) {
    if (outs[i].hi <= outs[i].lo) continue;
    for (int j = 0; j < ni; ++j)
      if (ins[j].hi > ins[j].lo && overlap(outs[i], ins[j])) return VDN_ERR_INVALID_ARG;
    for (int j = i + 1; j < no; ++j)
      if (outs[j].hi > outs[j].lo && overlap(outs[i], outs[j])) return VDN_ERR_INVALID_ARG;
  }
  char* ws = static_cast<char*>(workspace);
  if (!recompute && ws + plan.total > static_cast<const char*>(saved) &&
      static_cast<const char*>(saved) + sp.total > ws)
    return VDN_ERR_INVALID_ARG;
  Args a;
  a.sh = *shape;
  a.q = q; a.k = k; a.v = v;
  a.beta = beta; a.alpha = alpha; a.gate = gate; a.rms_w = rms_w;
  a.conv_k_w = conv_k_w; a.conv_v_w = conv_v_w; a.text_state = text_state;
  a.rule = rule; a.c = (rule == VDN_RULE_VDN_SOLVE || rule == VDN_RULE_ADDITIVE) ? 1.0f : c;
  a.chunk = chunk; a.radius = radius;
  a.stream = (cudaStream_t)stream;
  a.dbg = nullptr;
  if (events) {
    if (n_events < kBwdKernels + 2) return VDN_ERR_INVALID_ARG;
    for (int i = 0; i < kBwdKernels + 2; ++i)
      if (!events[i]) return VDN_ERR_INVALID_ARG;
    if (cudaEventRecord((cudaEvent_t)events[0], a.stream) != cudaSuccess) return VDN_ERR_CUDA;
  }
  BwdState st;
  if (recompute) {
    // forward with the per-frame export into the backward workspace
    vdn_debug_out dbg;
    dbg.impl = VDN_IMPL_AUTO;
    dbg.A = at<float>(ws, plan.A);
    dbg.B = at<float>(ws, plan.Bm);
    dbg.N = at<float>(ws, plan.Nm);
    dbg.P = at<float>(ws, plan.P);
    dbg.Q = at<float>(ws, plan.Q);
    dbg.W = at<float>(ws, plan.W);
    a.out = ws + plan.out;
    a.dbg = &dbg;
    s = run_forward(a, ws + plan.fwd, VDN_IMPL_AUTO);
    if (s != VDN_OK) return s;
    a.dbg = nullptr;
    st = {dbg.A, dbg.B, dbg.N, dbg.P, dbg.Q, dbg.W,
          use_tc(*shape, VDN_IMPL_AUTO)
              ? at<uint16_t>(ws, plan.fwd + plan_workspace(*shape, rule, true).nimg) : nullptr};
  } else {
    if (cudaMemsetAsync(ws + plan.status, 0, sizeof(uint32_t), a.stream) != cudaSuccess) return VDN_ERR_CUDA;
    char* sv = const_cast<char*>(static_cast<const char*>(saved));
    st = {at<float>(sv, sp.A), at<float>(sv, sp.Bm), at<float>(sv, sp.Nm), at<float>(sv, sp.P),
          at<float>(sv, sp.Q), at<float>(sv, sp.W), sp.nimg || use_tc(*shape, VDN_IMPL_AUTO)
                                                         ? at<uint16_t>(sv, sp.nimg) : nullptr};
  }
  if (events && cudaEventRecord((cudaEvent_t)events[1], a.stream) != cudaSuccess) return VDN_ERR_CUDA;
  BwdGrads g{dout, dq, dk, dv, dbeta, dalpha, dgate, drms_w, dconv_k_w, dconv_v_w, dtext_state};
  if (run_backward(a, g, st, ws, plan, events) != cudaSuccess) return VDN_ERR_CUDA;
  return VDN_OK;
}
}  // namespace

extern "C" {

vdn_status vdn_branch_backward(const vdn_shape* shape, const void* q, const void* k, const void* v,
                               const float* beta, const float* alpha, const void* gate, const float* rms_w,
                               const float* conv_k_w, const float* conv_v_w, const float* text_state, int rule,
                               float c, int chunk, int radius, const void* dout, void* workspace,
                               size_t workspace_bytes, void* dq, void* dk, void* dv, float* dbeta, float* dalpha,
                               void* dgate, float* drms_w, float* dconv_k_w, float* dconv_v_w,
                               float* dtext_state, void* stream) {
  return backward_common(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                         radius, dout, workspace, workspace_bytes, dq, dk, dv, dbeta, dalpha, dgate, drms_w,
                         dconv_k_w, dconv_v_w, dtext_state, stream, nullptr, 0);
}

size_t vdn_branch_saved_size(const vdn_shape* shape) {
  if (check_shape(shape) != VDN_OK) return 0;
  return plan_saved(*shape).total;
}

size_t vdn_branch_backward_saved_workspace_size(const vdn_shape* shape, int rule) {
  if (check_shape(shape) != VDN_OK) return 0;
  if (rule < VDN_RULE_SANA_SCALED || rule > VDN_RULE_ADDITIVE) return 0;
  return plan_backward(*shape, rule, false).total;
}

vdn_status vdn_branch_forward_train(const vdn_shape* shape, const void* q, const void* k, const void* v,
                                    const float* beta, const float* alpha, const void* gate, const float* rms_w,
                                    const float* conv_k_w, const float* conv_v_w, const float* text_state, int rule,
                                    float c, int chunk, int radius, void* workspace, size_t workspace_bytes,
                                    void* out, void* saved, size_t saved_bytes, void* stream) {
  vdn_status s = check_shape(shape);
  if (s != VDN_OK) return s;
  if (!saved) return VDN_ERR_INVALID_ARG;
  if (!aligned(saved, 256)) return VDN_ERR_ALIGNMENT;
  const SavedPlan sp = plan_saved(*shape);
  if (saved_bytes < sp.total) return VDN_ERR_WORKSPACE;
  // the saved state must not overlap an input, the output or the workspace
  const size_t big = (size_t)shape->B * shape->F * shape->S * shape->H * shape->d * elem_size(shape->dtype);
  const Range rs{(uintptr_t)saved, (uintptr_t)saved + sp.total};
  const Range others[] = {{(uintptr_t)q, (uintptr_t)q + big}, {(uintptr_t)k, (uintptr_t)k + big},
                          {(uintptr_t)v, (uintptr_t)v + big}, {(uintptr_t)gate, (uintptr_t)gate + big},
                          {(uintptr_t)out, (uintptr_t)out + big},
                          {(uintptr_t)workspace, (uintptr_t)workspace + workspace_bytes}};
  for (const Range& r : others)
    if (r.hi > r.lo && overlap(rs, r)) return VDN_ERR_INVALID_ARG;
  char* sv = static_cast<char*>(saved);
  vdn_debug_out dbg;
  dbg.impl = VDN_IMPL_AUTO;
  dbg.A = at<float>(sv, sp.A);
  dbg.B = at<float>(sv, sp.Bm);
  dbg.N = at<float>(sv, sp.Nm);
  dbg.P = at<float>(sv, sp.P);
  dbg.Q = at<float>(sv, sp.Q);
  dbg.W = at<float>(sv, sp.W);
  s = forward_common(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                     radius, workspace, workspace_bytes, out, stream, &dbg);
  if (s != VDN_OK) return s;
  if (sp.nimg) {
    // the tensor-core path's operand images of N_f, which the backward's adjoint products read
    const size_t nimg_off = plan_workspace(*shape, rule, true).nimg;
    const size_t bytes = (size_t)shape->B * shape->H * shape->F * kImgBytes;
    if (cudaMemcpyAsync(sv + sp.nimg, static_cast<char*>(workspace) + nimg_off, bytes, cudaMemcpyDeviceToDevice,
                        (cudaStream_t)stream) != cudaSuccess)
      return VDN_ERR_CUDA;
  }
  return VDN_OK;
}

vdn_status vdn_branch_backward_saved(const vdn_shape* shape, const void* q, const void* k, const void* v,
                                     const float* beta, const float* alpha, const void* gate, const float* rms_w,
                                     const float* conv_k_w, const float* conv_v_w, const float* text_state,
                                     int rule, float c, int chunk, int radius, const void* dout, const void* saved,
                                     size_t saved_bytes, void* workspace, size_t workspace_bytes, void* dq,
                                     void* dk, void* dv, float* dbeta, float* dalpha, void* dgate, float* drms_w,
                                     float* dconv_k_w, float* dconv_v_w, float* dtext_state, void* stream) {
  if (!saved) return VDN_ERR_INVALID_ARG;
  return backward_common(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                         radius, dout, workspace, workspace_bytes, dq, dk, dv, dbeta, dalpha, dgate, drms_w,
                         dconv_k_w, dconv_v_w, dtext_state, stream, nullptr, 0, saved, saved_bytes);
}

vdn_status vdn_branch_backward_timed(const vdn_shape* shape, const void* q, const void* k, const void* v,
                                     const float* beta, const float* alpha, const void* gate, const float* rms_w,
                                     const float* conv_k_w, const float* conv_v_w, const float* text_state,
                                     int rule, float c, int chunk, int radius, const void* dout, void* workspace,
                                     size_t workspace_bytes, void* dq, void* dk, void* dv, float* dbeta,
                                     float* dalpha, void* dgate, float* drms_w, float* dconv_k_w,
                                     float* dconv_v_w, float* dtext_state, void* stream, void* const* events,
                                     int n_events) {
  if (!events) return VDN_ERR_INVALID_ARG;
  return backward_common(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                         radius, dout, workspace, workspace_bytes, dq, dk, dv, dbeta, dalpha, dgate, drms_w,
                         dconv_k_w, dconv_v_w, dtext_state, stream, events, n_events);
}

vdn_status vdn_branch_forward(const vdn_shape* shape, const void* q, const void* k, const void* v,
                              const float* beta, const float* alpha, const void* gate, const float* rms_w,
                              const float* conv_k_w, const float* conv_v_w, const float* text_state, int rule,
                              float c, int chunk, int radius, void* workspace, size_t workspace_bytes, void* out,
                              void* stream) {
  return forward_common(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                        radius, workspace, workspace_bytes, out, stream, nullptr);
}

vdn_status vdn_branch_forward_debug(const vdn_shape* shape, const void* q, const void* k, const void* v,
                                    const float* beta, const float* alpha, const void* gate, const float* rms_w,
                                    const float* conv_k_w, const float* conv_v_w, const float* text_state,
                                    int rule, float c, int chunk, int radius, void* workspace,
                                    size_t workspace_bytes, void* out, void* stream, const vdn_debug_out* dbg) {
  return forward_common(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                        radius, workspace, workspace_bytes, out, stream, dbg);
}

int vdn_branch_launch_count(const vdn_shape* shape, int impl) {
  if (check_shape(shape) != VDN_OK || impl < VDN_IMPL_AUTO || impl > VDN_IMPL_TC) return 0;
  if (impl == VDN_IMPL_TC && !(shape->dtype == VDN_DTYPE_BF16 && shape->d == 128)) return 0;
  return use_tc(*shape, impl) ? 5 : 6;
}

vdn_status vdn_branch_forward_timed(const vdn_shape* shape, const void* q, const void* k, const void* v,
                                    const float* beta, const float* alpha, const void* gate, const float* rms_w,
                                    const float* conv_k_w, const float* conv_v_w, const float* text_state,
                                    int rule, float c, int chunk, int radius, void* workspace,
                                    size_t workspace_bytes, void* out, void* stream, void* const* events,
                                    int n_events) {
  if (!events) return VDN_ERR_INVALID_ARG;
  return forward_common(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                        radius, workspace, workspace_bytes, out, stream, nullptr, events, n_events);
}

vdn_status vdn_feature_prep(const vdn_shape* shape, const void* q, const void* k, const void* v,
                            const float* conv_k_w, const float* conv_v_w, void* q_out, void* k_out, void* v_out,
                            void* stream) {
  vdn_status s = check_shape(shape);
  if (s != VDN_OK) return s;
  if (!q || !k || !v || !q_out || !k_out || !v_out) return VDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, conv_k_w, conv_v_w, q_out, k_out, v_out};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return VDN_ERR_ALIGNMENT;
  const size_t big = (size_t)shape->B * shape->F * shape->S * shape->H * shape->d * elem_size(shape->dtype);
  const void* ins[] = {q, k, v};
  void* outs[] = {q_out, k_out, v_out};
  for (void* o : outs)
    for (const void* i : ins)
      if (overlap({(uintptr_t)o, (uintptr_t)o + big}, {(uintptr_t)i, (uintptr_t)i + big})) return VDN_ERR_INVALID_ARG;
  if (overlap({(uintptr_t)q_out, (uintptr_t)q_out + big}, {(uintptr_t)k_out, (uintptr_t)k_out + big}) ||
      overlap({(uintptr_t)q_out, (uintptr_t)q_out + big}, {(uintptr_t)v_out, (uintptr_t)v_out + big}) ||
      overlap({(uintptr_t)k_out, (uintptr_t)k_out + big}, {(uintptr_t)v_out, (uintptr_t)v_out + big}))
    return VDN_ERR_INVALID_ARG;
  cudaError_t e = launch_feature_prep(*shape, q, k, v, conv_k_w, conv_v_w, q_out, k_out, v_out, (cudaStream_t)stream);
  return e == cudaSuccess ? VDN_OK : VDN_ERR_CUDA;
}

size_t vdn_window_softmax_workspace_size(const vdn_shape* shape) {
  return check_shape(shape) == VDN_OK ? 256 : 0;
}

vdn_status vdn_window_softmax_forward(const vdn_shape* shape, const void* q_rope, const void* k_rope, const void* v,
                                      int chunk, int radius, float scale, int accumulate, void* workspace,
                                      size_t workspace_bytes, void* out, void* stream) {
  vdn_status s = check_softmax_args(shape, q_rope, k_rope, v, chunk, radius, scale, accumulate, workspace,
                                    workspace_bytes, 256, out);
  if (s != VDN_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return VDN_ERR_CUDA;
  return run_window_softmax(*shape, q_rope, k_rope, v, chunk, radius, scale, accumulate,
                            static_cast<uint32_t*>(workspace), out, st);
}

vdn_status vdn_hybrid_forward(const vdn_shape* shape, const void* q_rope, const void* k_rope, const void* q,
                              const void* k, const void* v, const float* beta, const float* alpha, const void* gate,
                              const float* rms_w, const float* conv_k_w, const float* conv_v_w,
                              const float* text_state, int rule, float c, int chunk, int radius, float scale,
                              void* workspace, size_t workspace_bytes, void* out, void* stream) {
  vdn_status s = check_softmax_args(shape, q_rope, k_rope, v, chunk, radius, scale, 1, workspace, workspace_bytes,
                                    256, out);
  if (s != VDN_OK) return s;
  // the linear branch validates the rest and writes out; the softmax branch adds to it
  s = forward_common(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                     radius, workspace, workspace_bytes, out, stream, nullptr);
  if (s != VDN_OK) return s;
  return run_window_softmax(*shape, q_rope, k_rope, v, chunk, radius, scale, 1, static_cast<uint32_t*>(workspace),
                            out, (cudaStream_t)stream);
}

vdn_status vdn_window_bounds(int t, int F, int chunk, int radius, int* lo, int* hi) {
  if (!lo || !hi || F < 1 || t < 0 || t >= F || chunk < 1 || radius < 0) return VDN_ERR_INVALID_ARG;
  vdn::window_bounds(t, F, chunk, radius, *lo, *hi);
  return VDN_OK;
}

vdn_status vdn_workspace_status(const void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < 256) return VDN_ERR_INVALID_ARG;
  uint32_t word = 0;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return VDN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return VDN_ERR_CUDA;
  return word == 0 ? VDN_OK : VDN_ERR_TIMEOUT;
}

const char* vdn_status_string(int status) {
  switch (status) {
    case VDN_OK: return "ok";
    case VDN_ERR_INVALID_ARG: return "invalid argument";
    case VDN_ERR_UNSUPPORTED: return "unsupported size or type";
    case VDN_ERR_ALIGNMENT: return "misaligned pointer";
    case VDN_ERR_WORKSPACE: return "workspace too small";
    case VDN_ERR_CUDA: return "CUDA error";
    case VDN_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------- frame sharding
namespace {

struct FramePart {
  int f0 = 0, F_local = 0, nch_total = 0, nch_stride = 0;
};

// rank's frames: a contiguous run of whole chunks (the clip's last chunk may be short)
vdn_status frame_part(int F_total, int world, int rank, int chunk, FramePart& fp) {
  if (F_total < 1 || chunk < 1 || world < 1 || rank < 0 || rank >= world) return VDN_ERR_INVALID_ARG;
  const long long C = ((long long)F_total + chunk - 1) / chunk;
  if (world > C) return VDN_ERR_INVALID_ARG;   // every rank owns at least one chunk
  int c0, c1;
  chunk_range((int)C, world, rank, c0, c1);
  const long long f1 = (long long)c1 * chunk < F_total ? (long long)c1 * chunk : F_total;
  fp.f0 = (int)((long long)c0 * chunk);
  fp.F_local = (int)(f1 - fp.f0);
  fp.nch_total = (int)C;
  fp.nch_stride = (int)((C + world - 1) / world);
  return VDN_OK;
}

// a rank's map buffer: the maps [B*H][2][nch][G | O][d][d] fp32, then their exponents
// [B*H][2][nch][G | O] int32, padded to 16 bytes
size_t frame_map_floats(const vdn_shape& sh, const FramePart& fp) {
  return (size_t)sh.B * sh.H * 2 * fp.nch_stride * 2 * sh.d * sh.d;
}
size_t frame_map_bytes(const vdn_shape& sh, const FramePart& fp) {
  const size_t exps = (size_t)sh.B * sh.H * 2 * fp.nch_stride * 2;
  return (frame_map_floats(sh, fp) * sizeof(float) + exps * sizeof(int) + 15) & ~(size_t)15;
}

// workspace of the second phase: the clip's chunk-edge states and the rank's read-out images
struct FramesPlan {
  size_t status = 0, P = 0, Q = 0, pexp = 0, qexp = 0, wimg = 0, wexp = 0, wbexp = 0, total = 0;
};
FramesPlan plan_frames(const vdn_shape& local, int F_total) {
  FramesPlan p;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t BH = (size_t)local.B * local.H, d = (size_t)local.d;
  const size_t NFg = BH * F_total, NFl = BH * local.F;
  p.status = take(256);
  p.P = take(NFg * d * d * sizeof(float));
  p.Q = take(NFg * d * d * sizeof(float));
  p.pexp = take(NFg * sizeof(int));
  p.qexp = take(NFg * sizeof(int));
  p.wimg = take(NFl * (size_t)kWImgBytes);
  p.wexp = take(NFl * sizeof(int));
  p.wbexp = take(NFl * kWRowBlocks * sizeof(int));
  p.total = off;
  return p;
}

// shape, partition and scalar checks shared by both phases
vdn_status check_frames(const vdn_shape* local, int F_total, int world, int rank, int rule, float c, int chunk,
                        FramePart& fp) {
  vdn_status s = check_shape(local);
  if (s != VDN_OK) return s;
  if (local->dtype != VDN_DTYPE_BF16 || local->d != 128) return VDN_ERR_UNSUPPORTED;   // tensor-core path only
  if (chunk > kGatherMaxChunk) return VDN_ERR_UNSUPPORTED;
  if (rule < VDN_RULE_SANA_SCALED || rule > VDN_RULE_ADDITIVE || !std::isfinite(c)) return VDN_ERR_INVALID_ARG;
  s = frame_part(F_total, world, rank, chunk, fp);
  if (s != VDN_OK) return s;
  if (local->F != fp.F_local) return VDN_ERR_INVALID_ARG;
  vdn_shape g = *local;
  g.F = F_total;
  return check_shape(&g);   // the clip-wide banks obey the same index limits
}

size_t frames_workspace(const vdn_shape& local, int F_total, int rule) {
  size_t a = plan_workspace(local, rule, true).total, b = plan_frames(local, F_total).total;
  return a > b ? a : b;
}

Args frame_args(const vdn_shape& sh, int rule, float c, int chunk, int radius, void* stream) {
  Args a{};
  a.sh = sh;
  a.rule = rule;
  a.c = (rule == VDN_RULE_VDN_SOLVE || rule == VDN_RULE_ADDITIVE) ? 1.0f : c;
  a.chunk = chunk;
  a.radius = radius;
  a.stream = (cudaStream_t)stream;
  return a;
}

}  // namespace

extern "C" {

vdn_status vdn_frame_range(int F_total, int world, int rank, int chunk, int* f0, int* f1) {
  if (!f0 || !f1) return VDN_ERR_INVALID_ARG;
  FramePart fp;
  vdn_status s = frame_part(F_total, world, rank, chunk, fp);
  if (s != VDN_OK) return s;
  *f0 = fp.f0;
  *f1 = fp.f0 + fp.F_local;
  return VDN_OK;
}

vdn_status vdn_frame_owner(int F_total, int world, int chunk, int frame, int* rank) {
  if (!rank || frame < 0 || frame >= F_total) return VDN_ERR_INVALID_ARG;
  FramePart fp;
  vdn_status s = frame_part(F_total, world, 0, chunk, fp);
  if (s != VDN_OK) return s;
  int j;
  chunk_owner(frame / chunk, fp.nch_total, world, *rank, j);
  return VDN_OK;
}

size_t vdn_frames_map_bytes(const vdn_shape* shape, int F_total, int world, int rank, int chunk) {
  FramePart fp;
  if (check_frames(shape, F_total, world, rank, VDN_RULE_VDN_SOLVE, 1.0f, chunk, fp) != VDN_OK) return 0;
  return frame_map_bytes(*shape, fp);
}

size_t vdn_frames_workspace_size(const vdn_shape* shape, int F_total, int world, int rank, int rule, int chunk) {
  FramePart fp;
  if (check_frames(shape, F_total, world, rank, rule, 1.0f, chunk, fp) != VDN_OK) return 0;
  return frames_workspace(*shape, F_total, rule);
}

vdn_status vdn_frames_maps(const vdn_shape* shape, int F_total, int world, int rank, const void* k, const void* v,
                           const float* beta, const float* alpha, const float* conv_k_w, const float* conv_v_w,
                           int rule, float c, int chunk, void* workspace, size_t workspace_bytes, float* maps,
                           size_t maps_bytes, void* stream) {
  FramePart fp;
  vdn_status s = check_frames(shape, F_total, world, rank, rule, c, chunk, fp);
  if (s != VDN_OK) return s;
  if (!k || !v || !beta || !alpha || !maps || !workspace) return VDN_ERR_INVALID_ARG;
  const void* ptrs[] = {k, v, beta, alpha, conv_k_w, conv_v_w, maps};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return VDN_ERR_ALIGNMENT;
  if (!aligned(workspace, 256)) return VDN_ERR_ALIGNMENT;
  const size_t need = frames_workspace(*shape, F_total, rule);
  if (workspace_bytes < need) return VDN_ERR_WORKSPACE;
  const size_t mb = frame_map_bytes(*shape, fp);
  if (maps_bytes < mb) return VDN_ERR_INVALID_ARG;
  const size_t tok = (size_t)shape->B * shape->F * shape->S * shape->H, d = (size_t)shape->d;
  const size_t big = tok * d * 2;
  Range rm{(uintptr_t)maps, (uintptr_t)maps + mb};
  Range rin[] = {
      {(uintptr_t)k, (uintptr_t)k + big},
      {(uintptr_t)v, (uintptr_t)v + big},
      {(uintptr_t)beta, (uintptr_t)beta + tok * 4},
      {(uintptr_t)alpha, (uintptr_t)alpha + (size_t)shape->B * shape->F * shape->H * d * 4},
      {(uintptr_t)conv_k_w, conv_k_w ? (uintptr_t)conv_k_w + (size_t)shape->H * d * shape->conv_width * 4 : 0},
      {(uintptr_t)conv_v_w, conv_v_w ? (uintptr_t)conv_v_w + (size_t)shape->H * d * shape->conv_width * 4 : 0},
      {(uintptr_t)workspace, (uintptr_t)workspace + need},
  };
  for (const Range& r : rin)
    if (r.hi > r.lo && overlap(rm, r)) return VDN_ERR_INVALID_ARG;

  Args a = frame_args(*shape, rule, c, chunk, 0, stream);
  a.k = k; a.v = v; a.beta = beta; a.alpha = alpha;
  a.conv_k_w = conv_k_w; a.conv_v_w = conv_v_w;
  WsPlan p = plan_workspace(*shape, rule, true);
  uint32_t* status = at<uint32_t>(workspace, p.status);
  float* part = at<float>(workspace, p.part);
  float* Bsum = at<float>(workspace, p.Bm);
  uint16_t* nimg = at<uint16_t>(workspace, p.nimg);
  VDN_LAUNCH(cudaMemsetAsync(status, 0, sizeof(uint32_t), a.stream));
  VDN_LAUNCH(launch_stats_tc(a, part, status));
  VDN_LAUNCH(launch_solve(a, nullptr, nullptr, nimg, part, Bsum, nullptr));
  int* map_exp = reinterpret_cast<int*>(maps + frame_map_floats(*shape, fp));
  VDN_LAUNCH(launch_scan_tc(a, Bsum, nimg, nullptr, nullptr, nullptr, nullptr, false, status, kScanSegZero, maps,
                            map_exp, fp.nch_stride));
  VDN_LAUNCH(launch_scan_tc(a, Bsum, nimg, nullptr, nullptr, nullptr, nullptr, false, status, kScanSegIdentity, maps,
                            map_exp, fp.nch_stride));
  return VDN_OK;
}

vdn_status vdn_frames_finish(const vdn_shape* shape, int F_total, int world, int rank, const void* q,
                             const float* alpha_all, const void* gate, const float* rms_w, const float* text_state,
                             int rule, float c, int chunk, int radius, const float* maps_all, size_t maps_all_bytes,
                             void* workspace, size_t workspace_bytes, void* out, void* stream) {
  FramePart fp;
  vdn_status s = check_frames(shape, F_total, world, rank, rule, c, chunk, fp);
  if (s != VDN_OK) return s;
  if (radius < 0) return VDN_ERR_INVALID_ARG;
  if (!q || !alpha_all || !gate || !rms_w || !maps_all || !workspace || !out) return VDN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, alpha_all, gate, rms_w, text_state, maps_all, out};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return VDN_ERR_ALIGNMENT;
  if (!aligned(workspace, 256)) return VDN_ERR_ALIGNMENT;
  const size_t need = frames_workspace(*shape, F_total, rule);
  if (workspace_bytes < need) return VDN_ERR_WORKSPACE;
  const size_t mb = frame_map_bytes(*shape, fp) * (size_t)world;
  if (maps_all_bytes < mb) return VDN_ERR_INVALID_ARG;
  const size_t tok = (size_t)shape->B * shape->F * shape->S * shape->H, d = (size_t)shape->d;
  const size_t big = tok * d * 2;
  Range ro{(uintptr_t)out, (uintptr_t)out + big};
  Range rin[] = {
      {(uintptr_t)q, (uintptr_t)q + big},
      {(uintptr_t)gate, (uintptr_t)gate + big},
      {(uintptr_t)alpha_all, (uintptr_t)alpha_all + (size_t)shape->B * F_total * shape->H * d * 4},
      {(uintptr_t)rms_w, (uintptr_t)rms_w + d * 4},
      {(uintptr_t)text_state, text_state ? (uintptr_t)text_state + (size_t)shape->H * d * d * 4 : 0},
      {(uintptr_t)maps_all, (uintptr_t)maps_all + mb},
      {(uintptr_t)workspace, (uintptr_t)workspace + need},
  };
  for (const Range& r : rin)
    if (r.hi > r.lo && overlap(ro, r)) return VDN_ERR_INVALID_ARG;
  // the fold reads the maps while it writes the workspace's state banks
  if (overlap(Range{(uintptr_t)maps_all, (uintptr_t)maps_all + mb}, Range{(uintptr_t)workspace, (uintptr_t)workspace + need}))
    return VDN_ERR_INVALID_ARG;

  vdn_shape g = *shape;
  g.F = F_total;
  Args ag = frame_args(g, rule, c, chunk, radius, stream);   // the clip: fold and gather
  ag.alpha = alpha_all;
  ag.text_state = text_state;
  Args al = frame_args(*shape, rule, c, chunk, radius, stream);   // the rank's frames: read-out
  al.q = q; al.gate = gate; al.rms_w = rms_w; al.out = out;
  FramesPlan p = plan_frames(*shape, F_total);
  uint32_t* status = at<uint32_t>(workspace, p.status);
  float *P = at<float>(workspace, p.P), *Q = at<float>(workspace, p.Q);
  int *pexp = at<int>(workspace, p.pexp), *qexp = at<int>(workspace, p.qexp);
  uint16_t* wimg = at<uint16_t>(workspace, p.wimg);
  int *wexp = at<int>(workspace, p.wexp), *wbexp = at<int>(workspace, p.wbexp);
  // the status word is not cleared here: with the workspace of vdn_frames_maps it keeps that
  // phase's report, and an expired wait of either phase stays visible afterwards
  VDN_LAUNCH(launch_fold_maps(ag, maps_all, frame_map_bytes(*shape, fp), frame_map_floats(*shape, fp) * sizeof(float),
                              world, fp.nch_stride, P, Q, pexp, qexp));
  VDN_LAUNCH(launch_gather_frames(ag, fp.f0, fp.F_local, P, Q, pexp, qexp, nullptr, wimg, wexp, wbexp));
  VDN_LAUNCH(launch_readout_tc(al, wimg, wexp, wbexp, status));
  return VDN_OK;
}

}  // extern "C"
