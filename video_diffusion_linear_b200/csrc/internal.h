// Internal interface between the C-ABI host code and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "vdn.h"

namespace vdn {

struct Args {
  vdn_shape sh;
  const void* q; const void* k; const void* v;
  const float* beta; const float* alpha;
  const void* gate; const float* rms_w;
  const float* conv_k_w; const float* conv_v_w;
  const float* text_state;
  int rule; float c; int chunk; int radius;
  void* out;
  cudaStream_t stream;
  const vdn_debug_out* dbg;   // may be NULL
  long long N() const { return (long long)sh.F * sh.S; }
  long long NF() const { return (long long)sh.B * sh.H * sh.F; }   // (batch, head, frame) triples
};

// CTAs of the persistent frame-statistics kernel of the tensor-core path.  A
// fixed count (the SM count of a B200) keeps the workspace a pure function of
// the shape; correctness does not depend on it.
constexpr int kStatsGrid = 148;
constexpr int kStatsTokens = 96;     // tokens per statistics block

// Byte offsets of the workspace regions (each 256-byte aligned).
struct WsPlan {
  size_t status = 0;
  // SIMT path
  size_t qf = 0, kf = 0, vf = 0;        // fp32 [B, N, H, d]
  size_t A = 0, Bm = 0, Nm = 0;         // fp32 [B, H, F, d, d]
  size_t P = 0, Q = 0, W = 0;           // fp32 [B, H, F, d, d]
  // block exponents: a stored state X means 2^e X (int32 [B, H, F] each)
  size_t pexp = 0, qexp = 0, wexp = 0;
  // tensor-core path
  size_t part = 0;                      // fp32 [slots][2d][d]: partial sums laid out [A; B]
  size_t nimg = 0;                      // bf16 [B,H,F][2][d][d] operand images (hi, lo) of N_f
  size_t wimg = 0;                      // fp16 [B,H,F][d][d] read-out operand images of W_t
  size_t wbexp = 0;                     // int32 [B,H,F][4] row-block exponents of those images
  size_t total = 0;
};

bool use_tc(const vdn_shape& sh, int impl);
WsPlan plan_workspace(const vdn_shape& sh, int rule, bool tc);

// ---- launchers; each returns cudaSuccess or the launch error
// SIMT path (any supported d, fp32 or bf16 I/O)
cudaError_t launch_features_simt(const Args& a, float* qf, float* kf, float* vf);
cudaError_t launch_stats_simt(const Args& a, const float* kf, const float* vf, float* A, float* Bm);
cudaError_t launch_solve(const Args& a, const float* A, float* Nm, uint16_t* nimg, const float* partials,
                         float* Bsum, float* Aout);
cudaError_t launch_scan_simt(const Args& a, const float* Bm, const float* Nm, float* P, float* Q, int* pexp,
                             int* qexp);
cudaError_t launch_gather(const Args& a, const float* P, const float* Q, const int* pexp, const int* qexp, float* W,
                          uint16_t* wimg, int* wexp, int* wbexp);
cudaError_t launch_readout_simt(const Args& a, const float* qf, const float* W, const int* wexp);
// longest chunk the per-chunk gather of the tensor-core path takes (frame sharding requires it)
constexpr int kGatherMaxChunk = 16;
// frame sharding (tensor-core path): the gather for query frames fq0 .. fq0 + Fq - 1 of the
// a.sh.F-frame clip (P, Q, exponents and alpha cover the clip; W_t lands at index t - fq0)
cudaError_t launch_gather_frames(const Args& a, int fq0, int Fq, const float* P, const float* Q, const int* pexp,
                                 const int* qexp, float* W, uint16_t* wimg, int* wexp, int* wbexp);
// the fold of every chunk's affine maps into the chunk-edge states P (chunk ends) and Q (chunk
// starts) of the a.sh.F-frame clip, from 0.5 x the text state (frames.cu)
// maps_all holds `world` rank buffers of rank_bytes each, every one the maps followed (at
// exp_off_bytes) by their int32 exponents; the folded states get exponents in pexp / qexp.
cudaError_t launch_fold_maps(const Args& a, const float* maps_all, size_t rank_bytes, size_t exp_off_bytes, int world,
                             int nch_stride, float* P, float* Q, int* pexp, int* qexp);
// dst = src * 2^expo[frame] (expo may be NULL)
cudaError_t launch_copy_frames(const Args& a, const float* src, float* dst, const int* expo = nullptr);

// ---- backward pass of the branch (backward.cu)
constexpr int kBwdConvBlocks = 148;   // blocks per head of the conv-reversal kernel
// Byte offsets of the backward workspace (each 256-byte aligned): the forward's own workspace,
// a scratch output, the forward's per-frame export and the adjoint buffers.
struct BwdPlan {
  size_t status = 0;                                   // device status word (first bytes of the workspace)
  size_t fwd = 0, out = 0;                             // forward recompute only
  size_t A = 0, Bm = 0, Nm = 0, P = 0, Q = 0, W = 0;   // fp32 [B, H, F, d, d]
  size_t dW = 0;                                       // fp32 [B, H, F, d, d]
  size_t dPin = 0, dQin = 0;                           // fp32 [B, H, F + 1, d, d]
  size_t dA2 = 0, dB2 = 0;                             // fp32 [2][B, H, F, d, d] (prefix, suffix scan)
  size_t dalpha_g = 0, dalpha2 = 0;                    // fp32 [B, H, F, d], [2][B, H, F, d]
  size_t dseed2 = 0;                                   // fp32 [2][B, H, d, d]
  size_t scan_scratch = 0;                             // fp32 [B, H, 2][2][d, d] (running adjoint, seed)
  size_t lam_all = 0, dX_all = 0;                      // fp32 [2][B, H, F, d, d]: adjoint and dX per step
  size_t Xbuf = 0;                                     // fp32 [2][B, H, F, d, d] (sana_scaled only)
  size_t rms_part = 0;                                 // fp32 [B, H, F][d]
  size_t dW_slots = 0, rms_slots = 0;                  // tensor-core read-out reversal's partial slots:
                                                       // fp32 [B H F + kBwdReadoutGrid][d, d] and [..][d]
  size_t dkc = 0, dvc = 0;                             // [B, N, H, d] in the inputs' element type
  size_t tap_part = 0;                                 // fp32 [H][kBwdConvBlocks][2][d][3]
  size_t fwd_bytes = 0, total = 0;
};
struct BwdGrads {
  const void* dout;
  void* dq; void* dk; void* dv;
  float* dbeta; float* dalpha;
  void* dgate;
  float* drms_w;
  float* dconv_k_w; float* dconv_v_w;
  float* dtext_state;
};
// recompute = false: the forward's per-frame state comes from a saved buffer (no fwd, out, A .. W)
BwdPlan plan_backward(const vdn_shape& sh, int rule, bool recompute = true);
// The forward's per-frame state that the backward reads (fp32 [B, H, F, d, d] each, and on the
// tensor-core path the hi/lo operand images of N_f): where vdn_branch_forward_train saves it.
struct SavedPlan {
  size_t A = 0, Bm = 0, Nm = 0, P = 0, Q = 0, W = 0, nimg = 0, total = 0;
};
SavedPlan plan_saved(const vdn_shape& sh);
struct BwdState {
  const float *A, *Bm, *Nm, *P, *Q, *W;
  const uint16_t* nimg;   // tensor-core path only
};
// the backward kernels, after the forward has filled the plan's A .. W regions; when `events` is
// not NULL, events[2 .. kBwdKernels + 1] are recorded after each of them (events[0] and events[1] bracket
// the forward recompute)
constexpr int kBwdKernels = 6;
// tensor-core versions of the read-out and statistics reversals (bf16, d = 128; tc_backward.cu)
// the read-out reversal runs two CTAs per SM over the (frame, tile) units; each (CTA, frame)
// pair it touches leaves partial dW_t and RMS-weight sums in slot (CTA + frame), which the launch
// then adds per frame into dW and rms_part (slots: B H F + kBwdReadoutGrid, of d^2 and d floats)
constexpr int kBwdReadoutGrid = 296;
cudaError_t launch_bwd_readout_tc(const Args& a, const void* dout, const float* W, float* dW, float* rms_part,
                                  float* dW_slots, float* rms_slots, void* dq, void* dgate, uint32_t* status);
cudaError_t launch_bwd_stats_tc(const Args& a, int K, const float* dA2, const float* dB2, void* dkc, void* dvc,
                                float* dbeta, uint32_t* status);
cudaError_t launch_bwd_scan_tc(const Args& a, const uint16_t* nimg, const float* dPin, const float* dQin,
                               float* lam_all, float* dX_all, float* dseed2, uint32_t* status);
cudaError_t run_backward(const Args& a, const BwdGrads& g, const BwdState& st, void* ws, const BwdPlan& p,
                         void* const* events);

// standalone step 1 (dtype in, dtype out)
cudaError_t launch_feature_prep(const vdn_shape& sh, const void* q, const void* k, const void* v,
                                const float* wk, const float* wv, void* qo, void* ko, void* vo,
                                cudaStream_t st);

// tensor-core path (bf16, d = 128)
cudaError_t launch_stats_tc(const Args& a, float* partials, uint32_t* status);
// scan modes: the whole clip from the text seed, or per-chunk affine maps (frame sharding)
constexpr int kScanWhole = 0, kScanSegZero = 1, kScanSegIdentity = 2;
// segment modes write map (b, h, direction, chunk j, G | O) of the rank's chunks to
// maps[((((b H + h) 2 + dir) nch_stride + j) 2 + (0 G | 1 O))][128][128] and its exponent to
// map_exp at the same index
cudaError_t launch_scan_tc(const Args& a, const float* Bsum, const uint16_t* nimg, float* P, float* Q, int* pexp,
                           int* qexp, bool all_frames, uint32_t* status, int seg_mode = kScanWhole,
                           float* maps = nullptr, int* map_exp = nullptr, int nch_stride = 0);
cudaError_t launch_window_softmax_simt(const vdn_shape& sh, const void* qr, const void* kr, const void* v, int chunk,
                                       int radius, float scale, int accumulate, void* out, cudaStream_t stream);
cudaError_t launch_window_softmax_tc(const vdn_shape& sh, const void* qr, const void* kr, const void* v, int chunk,
                                     int radius, float scale, int accumulate, void* out, uint32_t* status,
                                     cudaStream_t stream);
cudaError_t launch_readout_tc(const Args& a, const uint16_t* wimg, const int* wexp, const int* wbexp,
                              uint32_t* status);

}  // namespace vdn
