// Device helpers shared by the libvdn kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "vdn.h"

namespace vdn {

constexpr float kL2Eps = 1e-12f;     // q', k' = x / sqrt(sum x^2 + 1e-12)
constexpr float kRmsEps = 1e-6f;     // RMSNorm over d
constexpr float kTextStateScale = 0.5f;

// ---------------------------------------------------------------- element access
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// bf16x2 packed in a 32-bit word -> two floats (exact)
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// two floats -> bf16x2 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^x by the hardware approximation (one MUFU op; relative error about 2^-22,
// 2^-inf = 0), for the softmax weights that are rounded to bf16 afterwards
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^e for e in [-126, 127], built from the exponent field (exact)
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// two floats -> f16x2 (round to nearest even), lo in the low half
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// SiLU with the accurate exponential (SIMT paths, fp32 parity).
__device__ __forceinline__ float silu_precise(float x) { return x / (1.0f + expf(-x)); }

// SiLU through the identity sigmoid(x) = (1 + tanh(x/2)) / 2 and the hardware
// tanh approximation (one MUFU op); used where operands are rounded to bf16.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float silu_fast(float x) {
  float hx = 0.5f * x;
  return fmaf(hx, tanh_approx(hx), hx);
}

// tanh of a pair of floats.  Default: two hardware tanh.approx.f32 ops.
// With VDN_TANH_F16X2 defined, one packed tanh.approx.f16x2 op (f16 keeps an
// 11-bit mantissa, below the bf16 rounding of the tensor-core operands).
__device__ __forceinline__ float2 tanh2(float2 h) {
#ifdef VDN_TANH_F16X2
  uint32_t hp, tp;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(hp) : "f"(h.y), "f"(h.x));
  asm("tanh.approx.f16x2 %0, %1;" : "=r"(tp) : "r"(hp));
  float t0, t1;
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
      : "=f"(t0), "=f"(t1) : "r"(tp));
  return make_float2(t0, t1);
#else
  return make_float2(tanh_approx(h.x), tanh_approx(h.y));
#endif
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- window geometry
// Chunk-aligned softmax window of query frame t (page: "what is the far field").
__host__ __device__ __forceinline__ void window_bounds(int t, int F, int chunk, int radius, int& lo, int& hi) {
  int c = t / chunk;
  long long l = (long long)chunk * (c - radius);
  long long h = (long long)chunk * (c + radius + 1) - 1;
  lo = l < 0 ? 0 : (int)l;
  hi = h > F - 1 ? F - 1 : (int)h;
}

// Frame sharding: C chunks split into `world` contiguous runs, the first C % world
// ranks taking one chunk more.  chunk_range gives rank r's chunks [c0, c1);
// chunk_owner the rank of chunk c and its index j there (requires world <= C).
__host__ __device__ __forceinline__ void chunk_range(int C, int world, int r, int& c0, int& c1) {
  const int base = C / world, extra = C % world;
  c0 = r * base + (r < extra ? r : extra);
  c1 = c0 + base + (r < extra ? 1 : 0);
}
__host__ __device__ __forceinline__ void chunk_owner(int c, int C, int world, int& r, int& j) {
  const int base = C / world, extra = C % world;
  if (c < extra * (base + 1)) {
    r = c / (base + 1);
    j = c - r * (base + 1);
  } else {   // base >= 1 here: world <= C
    r = extra + (c - extra * (base + 1)) / base;
    j = c - (r * base + extra);
  }
}

// Coefficients of the generic step  S_f = (S_{f-1} D_f + cpre B_f) N_f + cpost B_f,
// which covers the three rules of the page plus the additive test rule.
struct RuleCoef {
  float cpre, cpost, c2;   // c2: scale of A inside N_f
  bool solve;              // N_f = (I + c2 A)^-1 (else I - c2 A, or I for additive)
  bool identity;
};
__host__ __device__ __forceinline__ RuleCoef rule_coef(int rule, float c) {
  RuleCoef r;
  switch (rule) {
    case VDN_RULE_VDN_SOLVE: r = {1.f, 0.f, 1.f, true, false}; break;
    case VDN_RULE_VDN_SCALED: r = {c, 0.f, c * c, true, false}; break;
    case VDN_RULE_SANA_SCALED: r = {0.f, c, c * c, false, false}; break;
    default: r = {1.f, 0.f, 0.f, false, true}; break;   // additive
  }
  return r;
}

// Block exponent of the scan states.  A rule whose per-frame operator has
// eigenvalues beyond 1 in magnitude (sana_scaled with c^2 |A| > 2) makes the
// state grow without bound; the scans keep X with true state 2^e X and rescale
// X by 2^-32 (exactly) whenever an entry passes 2^32.  One step multiplies a
// row norm by at most |D| |N| <= 1 + c^2 sum_s beta_s |k'_s|^2 <= 1 + c^2 S
// (about 2^12 for S = 4096), and a row norm is at most sqrt(128) times the
// largest entry, so stored states stay below 2^48 and the read-out's sum of
// squares of o = W_t q' (|q'| = 1, below 2^111) cannot overflow.  Its RMSNorm is scale-free up to eps,
// which is scaled by 2^(-2e) accordingly.
constexpr float kRenormAbove = 4294967296.0f;               // 2^32
constexpr float kRenormScale = 2.3283064365386963e-10f;    // 2^-32
constexpr int kRenormExp = 32;

// ---------------------------------------------------------------- device status word
// Written only by bounded waits that gave up; read by vdn_workspace_status().
constexpr uint32_t kStatusTimeout = 0x7100u;

}  // namespace vdn
