// Tensor-core kernels of the backward pass (bf16 inputs, d = 128): the two
// per-token contractions of the branch's gradients and the adjoint recurrence of
// the scans.  The per-token kernels work in tiles of 128 tokens of one (batch,
// head, frame), two threads per token (TMEM lane = token, one column half each),
// and are persistent: each CTA walks a contiguous range of the (frame, tile) units.
//
//   k_bwd_readout_tc  (Step 5 reversed)  O = Q' W_t^T      (A = Q' K-major, B = W_t K-major)
//                                        dQ' = DO W_t       (A = DO K-major, B = W_t read MN-major)
//                                        dW_t += DO^T Q'    (A = DO MN-major, B = Q' MN-major)
//                     296 CTAs (two per SM); the partial dW_t and RMS-weight sums of each
//                     (CTA, frame) pair go to slot CTA + frame, added per frame in CTA order by
//                     k_bwd_sum_slots
//   k_bwd_stats_tc    (Step 2 reversed)  U = K' (dA + dA^T), Z = K' dB^T   (B images K-major)
//                                        V' dB                          (dB image read MN-major)
//                     148 CTAs; raw k, v rows (+ halo) staged in shared memory, the conv
//                     unrolled over its taps; dk', dv' written in bf16 by TMA store
//   k_bwd_scan_tc     (Step 4 scans reversed)  dX_f = lam_f N_f, one CTA per (batch, head,
//                     direction), lam split into bf16 hi + lo against the forward's hi/lo N_f
//
// Operands are bf16 images in the 128-byte-swizzled layout of image.cuh written by
// the threads (q', do, k', v' per tile; W_t, dA + dA^T, dB where a CTA's range
// enters a frame); accumulators fp32 in TMEM.  The elementwise parts (RMSNorm and
// gate reversed, L2 norm and SiLU reversed, the conv recomputed from the raw
// tokens) run in the epilogues in fp32, as in the SIMT kernels of backward.cu.
// Every wait is bounded and reports through the device status word.
#include <cuda_bf16.h>

#include "common.cuh"
#include "image.cuh"
#include "internal.h"
#include "tc.cuh"
#include "tmap.h"

namespace vdn {
namespace {

constexpr int kBT = 128;                                                   // tokens per tile
constexpr uint32_t kIdKK = tc::idesc_bf16_f32(128, 128, false, false);    // A, B K-major
constexpr uint32_t kIdKM = tc::idesc_bf16_f32(128, 128, false, true);     // A K-major, B MN-major
constexpr uint32_t kIdMM = tc::idesc_bf16_f32(128, 128, true, true);      // A, B MN-major

__device__ __forceinline__ void store_chunk_bf16(uint8_t* img, int n, int k, const float* v) {
  *reinterpret_cast<uint4*>(img + img_offset(0, n, k)) =
      make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// D (+)= A B over K = 128 for 128 x 128 bf16 operand tiles in the image layout.
// K-major tile: rows are M (or N), 128-byte rows of K; its K step of 16 is +32 B within a
// 64-element half, halves 16 KB apart.  MN-major: rows are K, 16 rows (2 KB) per K step.
__device__ __forceinline__ void mma_kk(uint32_t d, uint32_t a, uint32_t b, bool acc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
    tc::umma_bf16(d, tc::smem_desc(a + off, 16, 1024), tc::smem_desc(b + off, 16, 1024), kIdKK,
                  (acc || kk > 0) ? 1u : 0u);
  }
}
__device__ __forceinline__ void mma_km(uint32_t d, uint32_t a, uint32_t b, bool acc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    tc::umma_bf16(d, tc::smem_desc(a + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                  tc::smem_desc(b + kk * 2048, 16384, 1024), kIdKM, (acc || kk > 0) ? 1u : 0u);
}
__device__ __forceinline__ void mma_mm(uint32_t d, uint32_t a, uint32_t b, bool acc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    tc::umma_bf16(d, tc::smem_desc(a + kk * 2048, 16384, 1024), tc::smem_desc(b + kk * 2048, 16384, 1024), kIdMM,
                  (acc || kk > 0) ? 1u : 0u);
}

// lane l receives the sum over the warp's lanes of v[l] (v[] is consumed)
__device__ __forceinline__ float transpose_sum32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = bf16lo(w[e]);
    v[2 * e + 1] = bf16hi(w[e]);
  }
}
__device__ __forceinline__ void unpack_bf16x8(uint4 u, float* v) {
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}
__device__ __forceinline__ void store8_bf16(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<uint4*>(p) =
      make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}
// sigma(x) = 1/2 + 1/2 tanh(x/2) by the hardware tanh (one MUFU op, relative error about 2^-11,
// below the bf16 rounding of every gradient these kernels write), as the forward's tensor-core
// kernels evaluate SiLU; silu(x) = x sigma(x), d silu = sigma (1 + x (1 - sigma)) dx
__device__ __forceinline__ float sigm_fast(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }
__device__ __forceinline__ float silu_f(float x) { return x * sigm_fast(x); }
__device__ __forceinline__ float silu_grad_f(float x, float g) {
  const float s = sigm_fast(x);
  return g * s * fmaf(x, 1.f - s, 1.f);
}

constexpr int kReadoutThreads = 256;   // two threads per token row (column halves)
struct ReadoutTcSmem {
  uint8_t w[32768];     // W_t image (rows i, K = j)
  uint8_t qf[32768];    // Q' tile (rows tokens, K = j)
  uint8_t dov[32768];   // DO tile (rows tokens, K = i)
  float rms[8][128];    // per-warp RMS-weight partials (zero outside the warp's column half)
  float red[4][2][128]; // per-token partial sums of the two column halves
  uint64_t bar;
  uint32_t tmem_base;
  int abort;
};

// ---------------------------------------------------------------- Step 5 reversed
// Two threads per token row: the warps w and w + 4 share TMEM lanes 32 (w % 4) .. and take the
// column halves 64 hf .. 64 hf + 63 (hf = w / 4); per-token sums are combined in shared memory.
// Persistent: CTA i takes the contiguous range [i T / G, (i + 1) T / G) of the (frame, tile)
// units, T = B H F x tiles per frame, so no wave is left partly empty.  Where its range enters a
// frame it builds that frame's W_t image; where it leaves one (or ends) it writes the partial
// dW_t accumulated in TMEM and its RMS-weight partial sums to slot (i + frame) -- distinct for
// every (CTA, frame) pair, as in the forward statistics -- and k_bwd_sum_slots adds each frame's
// slots in a fixed order.
__device__ __forceinline__ long long bwd_unit_owner(long long x, long long T, long long G) {
  return ((x + 1) * G + T - 1) / T - 1;   // the largest i with i T / G <= x
}

__global__ void __launch_bounds__(kReadoutThreads, 2) k_bwd_readout_tc(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ gate,
    const __nv_bfloat16* __restrict__ dout, const float* __restrict__ rms_w, const float* __restrict__ Wall,
    float* __restrict__ dWslot, float* __restrict__ rms_slot, __nv_bfloat16* __restrict__ dq,
    __nv_bfloat16* __restrict__ dgate, int H, int F, int S, long long NFt, uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  ReadoutTcSmem& sm = tc::smem_align<ReadoutTcSmem>(smem_raw);
  const long long N = (long long)F * S;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, hf = warp >> 2;
  const int m = 32 * quarter + lane;                // token of the tile = TMEM lane
  volatile int* abort_flag = &sm.abort;
  if (tid == 0) {
    tc::mbar_init(&sm.bar, 1);
    sm.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&sm.tmem_base, 256);
    tc::tmem_relinquish();
  }
  for (int e = tid; e < 8 * 128; e += kReadoutThreads) (&sm.rms[0][0])[e] = 0.f;
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;        // O / dQ' at columns 0..127, dW at 128..255
  const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
  const uint32_t aw = tc::smem_u32(sm.w), aq = tc::smem_u32(sm.qf), ad = tc::smem_u32(sm.dov);
  auto ld_row = [&](int p, uint32_t (&r)[32]) {     // columns 32 p .. 32 p + 31 of this token's row
    tc::tmem_ld32(tmem + 32 * p + lane_off, r);
    tc::tmem_ld_wait();
  };
  const int ntile = (S + kBT - 1) / kBT;
  const long long T = NFt * ntile, G = gridDim.x;
  const long long u0 = (long long)blockIdx.x * T / G, u1 = ((long long)blockIdx.x + 1) * T / G;
  float racc[2] = {0.f, 0.f};
  uint32_t ph = 0;
  bool ok = true;
  int tile = 0;
  long long cur = -1;
  for (long long u = u0; u < u1 && ok; ++u, ++tile) {
    const long long fi = u / ntile;
    const int s0 = (int)(u - fi * ntile) * kBT;
    const int f = (int)(fi % F);
    const long long bh = fi / F;
    const int h = (int)(bh % H);
    const long long b = bh / H;
    if (fi != cur) {
      // W_t image of the frame: thread (m, hf) writes the 8 chunks of its half of row m
      const float* wr = Wall + fi * 16384 + m * 128;
#pragma unroll 4
      for (int c = 8 * hf; c < 8 * hf + 8; ++c) {
        const float4 a = *reinterpret_cast<const float4*>(wr + 8 * c);
        const float4 bq = *reinterpret_cast<const float4*>(wr + 8 * c + 4);
        const float v[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
        store_chunk_bf16(sm.w, m, 8 * c, v);
      }
      racc[0] = racc[1] = 0.f;
      tile = 0;
      cur = fi;
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncthreads();
      tc::tc_fence_after();
    }
    {
    const int s = s0 + m;
    const bool valid = s < S;
    const long long row = ((b * N + (long long)f * S + (valid ? s : 0)) * H + h) * 128;
    // x = silu(q) into the Q' tile (q' = x / |x|: the 1/|x| is folded into O, DO and dQ' below)
    float ss = 0.f;
    {
      uint4 qu[8];   // this thread's 64 channels, all loads issued before any use
#pragma unroll
      for (int c = 0; c < 8; ++c)
        qu[c] = valid ? __ldg(reinterpret_cast<const uint4*>(q + row + 8 * (8 * hf + c))) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float v[8];
        unpack_bf16x8(qu[c], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[e] = valid ? silu_f(v[e]) : 0.f;
          ss = fmaf(v[e], v[e], ss);
        }
        store_chunk_bf16(sm.qf, m, 8 * (8 * hf + c), v);
      }
    }
    sm.red[0][hf][m] = ss;
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (tid == 0) {
      mma_kk(tmem, aq, aw, false);             // O |x| = X W_t^T
      tc::umma_commit(&sm.bar);
    }
    if (!(ok = tc::mbar_wait(&sm.bar, ph, abort_flag, status))) break;
    ph ^= 1;
    tc::tc_fence_after();
    const float sst = sm.red[0][0][m] + sm.red[0][1][m] + kL2Eps;
    const float inv = rsqrtf(sst), nrm = sst * inv;   // 1/|x|, |x|
    // RMSNorm and gate reversed
    float so2 = 0.f;
#pragma unroll 1
    for (int p = 2 * hf; p < 2 * hf + 2; ++p) {
      uint32_t o[32];
      ld_row(p, o);
#pragma unroll
      for (int c = 0; c < 32; ++c) so2 = fmaf(__uint_as_float(o[c]), __uint_as_float(o[c]), so2);
    }
    sm.red[1][hf][m] = so2;
    __syncthreads();
    const float rr = rsqrtf((sm.red[1][0][m] + sm.red[1][1][m]) * inv * inv * (1.f / 128.f) + kRmsEps);
    float so = 0.f;
#pragma unroll 1
    for (int pp = 0; pp < 2; ++pp) {
      const int p = 2 * hf + pp;
      uint4 gou[4], gau[4];   // dout, gate of this half of the row, issued before the TMEM load
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        const int c0 = 32 * p + 8 * c8;
        gou[c8] = valid ? __ldg(reinterpret_cast<const uint4*>(dout + row + c0)) : make_uint4(0, 0, 0, 0);
        gau[c8] = valid ? __ldg(reinterpret_cast<const uint4*>(gate + row + c0)) : make_uint4(0, 0, 0, 0);
      }
      uint32_t o[32];
      ld_row(p, o);
      float red[32];
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        const int c0 = 32 * p + 8 * c8;
        float go[8], g[8], dyv[8];
        unpack_bf16x8(gou[c8], go);
        unpack_bf16x8(gau[c8], g);
        float dg[8], rw8[8];
        *reinterpret_cast<float4*>(rw8) = __ldg(reinterpret_cast<const float4*>(rms_w + c0));
        *reinterpret_cast<float4*>(rw8 + 4) = __ldg(reinterpret_cast<const float4*>(rms_w + c0 + 4));
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float ov = inv * __uint_as_float(o[8 * c8 + e]);
          const float oh = ov * rr;
          const float dy = go[e] * g[e];
          dyv[e] = dy;
          dg[e] = go[e] * oh * rw8[e];
          red[8 * c8 + e] = dy * oh;
          so = fmaf(dy * rw8[e], ov, so);
        }
        if (valid) store8_bf16(dgate + row + c0, dg);
        store_chunk_bf16(sm.dov, m, c0, dyv);   // dy for the next pass, where DO then overwrites it
      }
      racc[pp] += transpose_sum32(red, lane);
    }
    sm.red[2][hf][m] = so;
    __syncthreads();
    const float k3 = rr * rr * rr * (sm.red[2][0][m] + sm.red[2][1][m]) * (1.f / 128.f);
#pragma unroll 1
    for (int p = 2 * hf; p < 2 * hf + 2; ++p) {
      uint32_t o[32];
      ld_row(p, o);
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        const int c0 = 32 * p + 8 * c8;
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (valid) {
          float dy[8], rw8[8];
          load8_bf16(reinterpret_cast<const __nv_bfloat16*>(sm.dov + img_offset(0, m, c0)), dy);
          *reinterpret_cast<float4*>(rw8) = __ldg(reinterpret_cast<const float4*>(rms_w + c0));
          *reinterpret_cast<float4*>(rw8 + 4) = __ldg(reinterpret_cast<const float4*>(rms_w + c0 + 4));
          // the tile holds do / |x| (so that DO^T X sums do q'^T)
#pragma unroll
          for (int e = 0; e < 8; ++e)
            v[e] = inv * (rr * dy[e] * rw8[e] - k3 * inv * __uint_as_float(o[8 * c8 + e]));
        }
        store_chunk_bf16(sm.dov, m, c0, v);
      }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (tid == 0) {
      mma_km(tmem, ad, aw, false);               // dQ' / |x| = (DO / |x|) W_t
      mma_mm(tmem + 128, ad, aq, tile > 0);      // dW_t += (DO / |x|)^T X = DO^T Q'
      tc::umma_commit(&sm.bar);
    }
    if (!(ok = tc::mbar_wait(&sm.bar, ph, abort_flag, status))) break;
    ph ^= 1;
    tc::tc_fence_after();
    // q' = l2n(silu(q)) reversed: dx = (g - x (x.g) / |x|^2) / |x| with x = silu(q), g = dq';
    // x.g from the tile's x (bf16), then dq = silu'(q) dx
    float xg = 0.f;
#pragma unroll 1
    for (int p = 2 * hf; p < 2 * hf + 2; ++p) {
      uint32_t o[32];
      ld_row(p, o);
      if (!valid) continue;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float x[8];
        load8_bf16(reinterpret_cast<const __nv_bfloat16*>(sm.qf + img_offset(0, m, 32 * p + 8 * c8)), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) xg = fmaf(x[e], nrm * __uint_as_float(o[8 * c8 + e]), xg);
      }
    }
    sm.red[3][hf][m] = xg;
    __syncthreads();
    xg = sm.red[3][0][m] + sm.red[3][1][m];
#pragma unroll 1
    for (int p = 2 * hf; p < 2 * hf + 2; ++p) {
      uint4 qu[4];   // issued before the TMEM load
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8)
        qu[c8] = valid ? __ldg(reinterpret_cast<const uint4*>(q + row + 32 * p + 8 * c8)) : make_uint4(0, 0, 0, 0);
      uint32_t o[32];
      ld_row(p, o);
      if (!valid) continue;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float v[8], r8[8];
        unpack_bf16x8(qu[c8], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float sg = sigm_fast(v[e]);
          const float x = v[e] * sg;
          const float dx = (nrm * __uint_as_float(o[8 * c8 + e]) - x * xg * inv * inv) * inv;
          r8[e] = dx * sg * fmaf(v[e], 1.f - sg, 1.f);
        }
        store8_bf16(dq + row + 32 * p + 8 * c8, r8);
      }
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    }
    if (u + 1 == u1 || (u + 1) % ntile == 0) {
      // the range leaves the frame: its partial dW_t (row i = m, this thread's column half) and
      // RMS-weight sums to slot (blockIdx.x + frame)
      const long long slot = (long long)blockIdx.x + fi;
      float* dW = dWslot + slot * 16384 + m * 128;
#pragma unroll
      for (int p = 2 * hf; p < 2 * hf + 2; ++p) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + 128 + 32 * p + lane_off, r);
        tc::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dW + 32 * p + e) =
              make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                          __uint_as_float(r[e + 3]));
      }
      sm.rms[warp][32 * (2 * hf) + lane] = racc[0];
      sm.rms[warp][32 * (2 * hf + 1) + lane] = racc[1];
      tc::tc_fence_before();
      __syncthreads();
      if (tid < 128) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) acc += sm.rms[w][tid];
        rms_slot[slot * 128 + tid] = acc;
      }
      __syncthreads();
      tc::tc_fence_after();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 256);
  }
}

// Each frame's dW_t and RMS-weight partial sums: the slots (i + frame) of the read-out reversal's
// CTAs i whose ranges covered the frame, added in CTA order.  Block (frame, part): 256 threads,
// one float4 of dW_t each per part of 1024 floats; part 0 also sums the 128 RMS-weight entries.
__global__ void __launch_bounds__(256) k_bwd_sum_slots(const float* __restrict__ dWslot,
                                                       const float* __restrict__ rms_slot, int ntile, long long T,
                                                       long long G, float* __restrict__ dW,
                                                       float* __restrict__ rms_part) {
  const long long fi = blockIdx.x;
  const long long c0 = bwd_unit_owner(fi * ntile, T, G), c1 = bwd_unit_owner(fi * ntile + ntile - 1, T, G);
  const int e4 = blockIdx.y * 256 + threadIdx.x;   // float4 index within the frame's 4096
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long c = c0; c <= c1; ++c) {
    const float4 v = reinterpret_cast<const float4*>(dWslot + (c + fi) * 16384)[e4];
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  reinterpret_cast<float4*>(dW + fi * 16384)[e4] = acc;
  if (blockIdx.y == 0 && threadIdx.x < 128) {
    float r = 0.f;
    for (long long c = c0; c <= c1; ++c) r += rms_slot[(c + fi) * 128 + threadIdx.x];
    rms_part[fi * 128 + threadIdx.x] = r;
  }
}

// ---------------------------------------------------------------- Step 2 reversed
constexpr int kRawStride = 272;     // bytes per staged token row (256 + 16: conflict-free 16-byte reads)
constexpr int kRawRows = kBT + 2;    // the tile's tokens and one halo token on each side
struct StatsTcSmem {
  uint8_t da[32768];    // (dA + dA^T) image (rows i, K = j)
  uint8_t db[32768];    // dB image (rows i, K = j)
  uint8_t kf[32768];    // K' tile
  uint8_t vf[32768];    // V' tile
  uint8_t kraw[kRawRows * kRawStride];   // raw k rows s0 - 1 .. s0 + 128 (bf16; zero outside the frame)
  uint8_t vraw[kRawRows * kRawStride];
  float taps[2][3][128];                 // [k, v][tap][channel] of this head (identity: centre tap 1)
  float red[3][2][128];                  // per-token partial sums of the two column halves
  uint64_t bar;
  uint32_t tmem_base;
  int abort;
};

// the short conv of one channel chunk (8 channels c0..c0+7) of the tile's token t (frame index s),
// in-frame taps, from the staged rows (row t + 1 holds token t) and the staged taps tp[tap][channel]
// (the staged rows are zero outside the frame, so every tap is applied: an outside row adds 0)
template <int KT>
__device__ __forceinline__ void conv8(const uint8_t* raw, const float (*tp)[128], int t, int c0, float* out) {
  constexpr int PAD = (KT - 1) / 2;
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = 0.f;
#pragma unroll
  for (int j = 0; j < KT; ++j) {
    float v[8];
    load8_bf16(reinterpret_cast<const __nv_bfloat16*>(raw + (t + 1 + j - PAD) * kRawStride + 2 * c0), v);
    const float4 w0 = *reinterpret_cast<const float4*>(&tp[j][c0]);
    const float4 w1 = *reinterpret_cast<const float4*>(&tp[j][c0 + 4]);
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = fmaf(wv[e], v[e], out[e]);
  }
}

// Two threads per token row: the warps w and w + 4 share TMEM lanes 32 (w % 4) .. and take the
// column halves 64 hf .. 64 hf + 63 (hf = w / 4); per-token sums are combined in shared memory.
constexpr int kStatsThreads = 256;

template <int KT>   // taps of the staged convs (a missing conv: the identity, one centre tap)
__global__ void __launch_bounds__(kStatsThreads) k_bwd_stats_tc(const __grid_constant__ CUtensorMap tmDK,
                                                                const __grid_constant__ CUtensorMap tmDV,
                                                                const __nv_bfloat16* __restrict__ k,
                                                                const __nv_bfloat16* __restrict__ v,
                                                                const float* __restrict__ beta,
                                                                const float* __restrict__ wk,
                                                                const float* __restrict__ wv,
                                                                const float* __restrict__ dA2,
                                                                const float* __restrict__ dB2,
                                                                __nv_bfloat16* __restrict__ dkc,
                                                                __nv_bfloat16* __restrict__ dvc,
                                                                float* __restrict__ dbeta, int H, int F, int S,
                                                                long long NFt, uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  StatsTcSmem& sm = tc::smem_align<StatsTcSmem>(smem_raw);
  const long long N = (long long)F * S;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, hf = warp >> 2;
  const int m = 32 * quarter + lane;                       // token of the tile = TMEM lane
  volatile int* abort_flag = &sm.abort;
  if (tid == 0) {
    tc::mbar_init(&sm.bar, 1);
    sm.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&sm.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;        // U |x| at 0, Z |x| at 128, V' dB at 256
  const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
  const uint32_t a_da = tc::smem_u32(sm.da), a_db = tc::smem_u32(sm.db), a_k = tc::smem_u32(sm.kf),
                 a_v = tc::smem_u32(sm.vf);
  // persistent: CTA i takes the contiguous range [i T / G, (i + 1) T / G) of the (frame, tile)
  // units, T = B H F x tiles per frame, so no wave is left partly empty; the frame's operand
  // images and taps are rebuilt whenever the range enters a new frame
  const int ntile = (S + kBT - 1) / kBT;
  const long long T = NFt * ntile, G = gridDim.x;
  const long long u0 = (long long)blockIdx.x * T / G, u1 = ((long long)blockIdx.x + 1) * T / G;
  long long cur = -1;
  uint32_t ph = 0;
  bool ok = true;
  for (long long u = u0; u < u1 && ok; ++u) {
    const long long fi = u / ntile;
    const int s0 = (int)(u - fi * ntile) * kBT;
    const int f = (int)(fi % F);
    const long long bh = fi / F;
    const int h = (int)(bh % H);
    const long long b = bh / H;
    const long long frame_row0 = b * N + (long long)f * S;   // token row of s = 0
    if (fi != cur) {
      // images of dA + dA^T (threads 0..127, row = tid) and dB (threads 128..255), both scans'
      // parts summed (the previous tile's products and reads of them are complete)
      const int i = tid & 127;
      const float* x0 = (tid < 128 ? dA2 : dB2) + fi * 16384;
      const float* x1 = (tid < 128 ? dA2 : dB2) + (NFt + fi) * 16384;
      uint8_t* img = tid < 128 ? sm.da : sm.db;
      for (int c = 0; c < 16; ++c) {
        float va[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 8 * c + e;
          va[e] = x0[i * 128 + j] + x1[i * 128 + j];
          if (tid < 128) va[e] += x0[j * 128 + i] + x1[j * 128 + i];
        }
        store_chunk_bf16(img, i, 8 * c, va);
      }
      // taps of this head, [tensor][tap][channel]; a missing conv is the identity (one centre tap)
      if (tid < 128)
        for (int j = 0; j < 3; ++j) {
          const bool centre = j == (KT - 1) / 2;
          sm.taps[0][j][i] = j < KT ? (wk ? wk[((long long)h * 128 + i) * KT + j] : (centre ? 1.f : 0.f)) : 0.f;
          sm.taps[1][j][i] = j < KT ? (wv ? wv[((long long)h * 128 + i) * KT + j] : (centre ? 1.f : 0.f)) : 0.f;
        }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncthreads();
      tc::tc_fence_after();
      cur = fi;
    }
    const int s = s0 + m;
    const bool valid = s < S;
    const long long tok = frame_row0 * H + (long long)(valid ? s : 0) * H + h;
    const float bt = valid ? __ldg(beta + tok) : 0.f;   // issued here, used after the product
    // stage the raw k, v rows of tokens s0 - 1 .. s0 + 128 (zero outside the frame): sixteen
    // threads per row, so each warp reads two whole 256-byte rows; all loads issued first
    {
      constexpr int kChunks = kRawRows * 16, kIt = (kChunks + kStatsThreads - 1) / kStatsThreads;
      uint4 kb[kIt], vb[kIt];
#pragma unroll
      for (int u = 0; u < kIt; ++u) {
        const int idx = tid + u * kStatsThreads, r = idx >> 4, c = idx & 15;
        const int sr = s0 - 1 + r;
        const bool in = idx < kChunks && sr >= 0 && sr < S;
        const long long off = ((frame_row0 + (in ? sr : 0)) * H + h) * 128 + 8 * c;
        kb[u] = in ? *reinterpret_cast<const uint4*>(k + off) : make_uint4(0, 0, 0, 0);
        vb[u] = in ? *reinterpret_cast<const uint4*>(v + off) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kIt; ++u) {
        const int idx = tid + u * kStatsThreads, r = idx >> 4, c = idx & 15;
        if (idx < kChunks) {
          *reinterpret_cast<uint4*>(sm.kraw + r * kRawStride + 16 * c) = kb[u];
          *reinterpret_cast<uint4*>(sm.vraw + r * kRawStride + 16 * c) = vb[u];
        }
      }
    }
    if (tid == 0) tc::bulk_wait_read_all();   // the previous tile's gradient stores left kf / vf
    __syncthreads();
    // x = silu(conv k) (k' = x / |x|: the 1/|x| is applied to U and Z in the epilogue) and
    // v' = silu(conv v) into the K', V' tiles: this thread's 8 chunks of its token
    float ss = 0.f;
#pragma unroll 2
    for (int c = 8 * hf; c < 8 * hf + 8; ++c) {
      float kv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, vv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (valid) {
        conv8<KT>(sm.kraw, sm.taps[0], m, 8 * c, kv);
        conv8<KT>(sm.vraw, sm.taps[1], m, 8 * c, vv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          kv[e] = silu_f(kv[e]);
          ss = fmaf(kv[e], kv[e], ss);
          vv[e] = silu_f(vv[e]);
        }
      }
      store_chunk_bf16(sm.kf, m, 8 * c, kv);
      store_chunk_bf16(sm.vf, m, 8 * c, vv);
    }
    sm.red[0][hf][m] = ss;
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (tid == 0) {
      mma_kk(tmem, a_k, a_da, false);            // U |x|: X (dA + dA^T)
      mma_kk(tmem + 128, a_k, a_db, false);      // Z |x|: z_i |x| = sum_j dB[i][j] x_j
      mma_km(tmem + 256, a_v, a_db, false);      // w_i = sum_j dB[j][i] v'_j
      tc::umma_commit(&sm.bar);
    }
    if (!(ok = tc::mbar_wait(&sm.bar, ph, abort_flag, status))) break;
    ph ^= 1;
    tc::tc_fence_after();
    const float inv = rsqrtf(sm.red[0][0][m] + sm.red[0][1][m] + kL2Eps);
    // the TMEM loads are warp-collective: every thread loads, only valid tokens compute
    // pass 1: d beta and x . dk' over this thread's half, from the tiles' x and v' (bf16)
    float dbt = 0.f, xg = 0.f;
#pragma unroll 1
    for (int p = 2 * hf; p < 2 * hf + 2; ++p) {
      uint32_t u[32], z[32], w[32];
      tc::tmem_ld32(tmem + 32 * p + lane_off, u);
      tc::tmem_ld32(tmem + 128 + 32 * p + lane_off, z);
      tc::tmem_ld32(tmem + 256 + 32 * p + lane_off, w);
      tc::tmem_ld_wait();
      if (!valid) continue;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float xk[8], xv[8];
        load8_bf16(reinterpret_cast<const __nv_bfloat16*>(sm.kf + img_offset(0, m, 32 * p + 8 * c8)), xk);
        load8_bf16(reinterpret_cast<const __nv_bfloat16*>(sm.vf + img_offset(0, m, 32 * p + 8 * c8)), xv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int q8 = 8 * c8 + e;
          const float uu = inv * __uint_as_float(u[q8]), zz = inv * __uint_as_float(z[q8]);
          const float ww = __uint_as_float(w[q8]);
          // d beta = 1/2 k'^T (dA + dA^T) k' + v'^T dB k'
          dbt = fmaf(0.5f * xk[e] * inv, uu, dbt);
          dbt = fmaf(xv[e], zz, dbt);
          xg = fmaf(xk[e], bt * (uu + ww), xg);
        }
      }
    }
    sm.red[1][hf][m] = dbt;
    sm.red[2][hf][m] = xg;
    __syncthreads();
    xg = sm.red[2][0][m] + sm.red[2][1][m];
    if (valid && hf == 0) dbeta[tok] = sm.red[1][0][m] + sm.red[1][1][m];
    // pass 2: dkc = silu'(kc) (dk' - x (x . dk') / |x|^2) / |x|, dvc = silu'(vc) beta z
#pragma unroll 1
    for (int p = 2 * hf; p < 2 * hf + 2; ++p) {
      uint32_t u[32], z[32], w[32];
      tc::tmem_ld32(tmem + 32 * p + lane_off, u);
      tc::tmem_ld32(tmem + 128 + 32 * p + lane_off, z);
      tc::tmem_ld32(tmem + 256 + 32 * p + lane_off, w);
      tc::tmem_ld_wait();
      if (!valid) continue;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        const int c0 = 32 * p + 8 * c8;
        float kc[8], vc[8], gk[8], gv[8];
        conv8<KT>(sm.kraw, sm.taps[0], m, c0, kc);
        conv8<KT>(sm.vraw, sm.taps[1], m, c0, vc);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int q8 = 8 * c8 + e;
          const float sg = sigm_fast(kc[e]);
          const float x = kc[e] * sg;
          const float dk = bt * (inv * __uint_as_float(u[q8]) + __uint_as_float(w[q8]));
          gk[e] = (dk - x * xg * inv * inv) * inv * sg * fmaf(kc[e], 1.f - sg, 1.f);
          gv[e] = silu_grad_f(vc[e], bt * inv * __uint_as_float(z[q8]));
        }
        // bf16, as the gradients they feed (dk, dv) are written: into the (read) K', V'
        // tiles, which leave through TMA stores in the same layout
        store_chunk_bf16(sm.kf, m, c0, gk);
        store_chunk_bf16(sm.vf, m, c0, gv);
      }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (tid == 0) {   // rows past the frame end are clipped by the tensor maps
      const int fb = (int)(b * F + f);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tc::tma_store_4d(&tmDK, sm.kf + hh * 16384, 64 * hh, h, s0, fb);
        tc::tma_store_4d(&tmDV, sm.vf + hh * 16384, 64 * hh, h, s0, fb);
      }
      tc::bulk_commit();
    }
  }
  if (tid == 0) tc::bulk_wait_all();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- Steps 3-4 reversed: the adjoint scans
// One CTA per (batch, head, direction) walks the frames in the reverse order of absorption:
//     lam_f = lam + g_f                      (g_f: the bridge's gradient of the state after frame f)
//     dX_f = lam_f N_f^T = lam_f N_f         (N_f symmetric for every rule; tcgen05, bf16 hi/lo)
//     lam  = dX_f D_f
// storing lam_f and dX_f for the batched kernel that forms dA, dB, d alpha.  The product splits
// lam into bf16 hi + lo and uses the forward's hi/lo image of N_f (three MMAs per K step, about 16
// significant bits per term, fp32 accumulation), as the forward scan does.
struct __align__(1024) BwdScanSmem {
  uint8_t aop[2][32768];     // lam hi, lam lo: K-major SW128 A operands
  uint8_t nimg[65536];       // N_f hi | lo image
  float alpha[128];
  uint64_t bar_n, bar_mma, bar_nhi;
  uint32_t tmem_base;
  int abort;
};
constexpr int kBwdScanThreads = 256;   // two threads per state row (column halves)

__device__ __forceinline__ void split_pair_bf16(float2 x, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(x.x, x.y);
  lo = pack_bf16x2(x.x - bf16lo(hi), x.y - bf16hi(hi));
}

__global__ void __launch_bounds__(kBwdScanThreads, 1) k_bwd_scan_tc(const uint16_t* __restrict__ nimg_g,
                                                                    const float* __restrict__ alpha,
                                                                    const float* __restrict__ dPin,
                                                                    const float* __restrict__ dQin,
                                                                    float* __restrict__ lam_all,
                                                                    float* __restrict__ dX_all,
                                                                    float* __restrict__ dseed2, int H, int F,
                                                                    uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  BwdScanSmem& sm = tc::smem_align<BwdScanSmem>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m = 32 * (warp & 3) + lane;     // state row = TMEM lane
  const int k0 = 64 * (tid >> 7);           // column half
  const int dir = blockIdx.y;
  const long long bh = blockIdx.x;
  const long long BH = gridDim.x;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const long long DD = 128 * 128;
  volatile int* abort_flag = &sm.abort;
  if (tid == 0) {
    tc::mbar_init(&sm.bar_n, 1);
    tc::mbar_init(&sm.bar_mma, 1);
    tc::mbar_init(&sm.bar_nhi, 1);
    sm.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&sm.tmem_base, 128);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t t_row = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + k0;
  const float* din = (dir == 0 ? dPin : dQin) + bh * (F + 1) * DD;
  auto frame_of = [&](int step) { return dir == 0 ? F - 1 - step : step; };
  auto load_n_part = [&](int step, int part) {
    const long long fi = bh * F + frame_of(step);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(nimg_g + fi * (kImgBytes / 2)) + part * 32768;
    if (part == 0) tc::mbar_arrive_expect_tx(&sm.bar_n, kImgBytes);
#pragma unroll
    for (int j = 0; j < 2; ++j) tc::bulk_load(sm.nimg + part * 32768 + j * 16384, src + j * 16384, 16384, &sm.bar_n);
  };
  if (tid == 0) {
    load_n_part(0, 0);
    load_n_part(0, 1);
  }
  float2 s[32];   // the running adjoint, row m, columns k0 .. k0 + 63
#pragma unroll
  for (int p = 0; p < 32; ++p) s[p] = make_float2(0.f, 0.f);
  const uint32_t a_hi = tc::smem_u32(sm.aop[0]), a_lo = tc::smem_u32(sm.aop[1]);
  const uint32_t n_hi = tc::smem_u32(sm.nimg), n_lo = n_hi + 32768;
  uint32_t ph = 0;
  for (int step = 0; step < F; ++step) {
    const int f = frame_of(step);
    const long long fi = bh * F + f;
    const long long go = ((long long)dir * BH * F + fi) * DD + (long long)m * 128 + k0;
    if (tid < 128) sm.alpha[tid] = alpha[((b * F + f) * H + h) * 128 + tid];
    // lam_f = lam + g_f: stored, and split into the A operands
    const float* g = din + (long long)(dir == 0 ? f + 1 : f) * DD + (long long)m * 128 + k0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 g0 = *reinterpret_cast<const float4*>(g + 8 * c);
      const float4 g1 = *reinterpret_cast<const float4*>(g + 8 * c + 4);
      s[4 * c + 0] = make_float2(s[4 * c + 0].x + g0.x, s[4 * c + 0].y + g0.y);
      s[4 * c + 1] = make_float2(s[4 * c + 1].x + g0.z, s[4 * c + 1].y + g0.w);
      s[4 * c + 2] = make_float2(s[4 * c + 2].x + g1.x, s[4 * c + 2].y + g1.y);
      s[4 * c + 3] = make_float2(s[4 * c + 3].x + g1.z, s[4 * c + 3].y + g1.w);
      *reinterpret_cast<float4*>(lam_all + go + 8 * c) = make_float4(s[4 * c].x, s[4 * c].y, s[4 * c + 1].x, s[4 * c + 1].y);
      *reinterpret_cast<float4*>(lam_all + go + 8 * c + 4) =
          make_float4(s[4 * c + 2].x, s[4 * c + 2].y, s[4 * c + 3].x, s[4 * c + 3].y);
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) split_pair_bf16(s[4 * c + q], hw[q], lw[q]);
      const uint32_t off = img_offset(0, m, k0 + 8 * c);
      *reinterpret_cast<uint4*>(sm.aop[0] + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sm.aop[1] + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (tid == 0) {
      if (tc::mbar_wait(&sm.bar_n, ph, abort_flag, status)) {
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint64_t bhd = tc::smem_desc(n_hi + koff, 16, 1024);
          tc::umma_bf16(tmem, tc::smem_desc(a_hi + koff, 16, 1024), bhd, kIdKK, kk > 0 ? 1u : 0u);
          tc::umma_bf16(tmem, tc::smem_desc(a_lo + koff, 16, 1024), bhd, kIdKK, 1u);
        }
        tc::umma_commit(&sm.bar_nhi);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::umma_bf16(tmem, tc::smem_desc(a_hi + koff, 16, 1024), tc::smem_desc(n_lo + koff, 16, 1024), kIdKK, 1u);
        }
        tc::umma_commit(&sm.bar_mma);
        if (step + 1 < F && tc::mbar_wait(&sm.bar_nhi, ph, abort_flag, status)) load_n_part(step + 1, 0);
      }
    }
    if (!tc::mbar_wait(&sm.bar_mma, ph, abort_flag, status)) break;
    tc::tc_fence_after();
    if (tid == 0 && step + 1 < F) load_n_part(step + 1, 1);   // the product that read N_lo is complete
    // dX_f: stored; the next adjoint is dX_f D_f
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t r[32];
      tc::tmem_ld32(t_row + 32 * j, r);
      tc::tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const int p = 16 * j + e / 2;
        const int kc = k0 + 32 * j + e;
        const float4 dx = make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                                      __uint_as_float(r[e + 3]));
        *reinterpret_cast<float4*>(dX_all + go + 32 * j + e) = dx;
        const float4 al = *reinterpret_cast<const float4*>(&sm.alpha[kc]);
        s[p] = make_float2(dx.x * al.x, dx.y * al.y);
        s[p + 1] = make_float2(dx.z * al.z, dx.w * al.w);
      }
    }
    tc::tc_fence_before();
    __syncthreads();            // accumulator read, alpha slot and A operands free
    ph ^= 1;
  }
  // the gradient of the seed: the final adjoint plus the bridge's direct use of the seed
  {
    const float* g0 = din + (long long)(dir == 0 ? 0 : F) * DD + (long long)m * 128 + k0;
    float* ds = dseed2 + ((long long)dir * BH + bh) * DD + (long long)m * 128 + k0;
#pragma unroll
    for (int p = 0; p < 32; ++p) {
      const float2 gg = *reinterpret_cast<const float2*>(g0 + 2 * p);
      *reinterpret_cast<float2*>(ds + 2 * p) = make_float2(s[p].x + gg.x, s[p].y + gg.y);
    }
  }
  // teardown: make sure no copy or product of ours is still in flight
  __syncthreads();
  if (sm.abort && tid == 0) tc::mbar_wait(&sm.bar_n, ph, abort_flag, nullptr);
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

}  // namespace

cudaError_t launch_bwd_readout_tc(const Args& a, const void* dout, const float* W, float* dW, float* rms_part,
                                  float* dW_slots, float* rms_slots, void* dq, void* dgate, uint32_t* status) {
  const size_t smem = sizeof(ReadoutTcSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_bwd_readout_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ntile = (a.sh.S + kBT - 1) / kBT;
  const long long T = a.NF() * ntile;
  const long long G = T < kBwdReadoutGrid ? T : kBwdReadoutGrid;
  k_bwd_readout_tc<<<(unsigned)G, kReadoutThreads, smem, a.stream>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.gate),
      static_cast<const __nv_bfloat16*>(dout), a.rms_w, W, dW_slots, rms_slots, static_cast<__nv_bfloat16*>(dq),
      static_cast<__nv_bfloat16*>(dgate), a.sh.H, a.sh.F, a.sh.S, a.NF(), status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_bwd_sum_slots<<<dim3((unsigned)a.NF(), 16), 256, 0, a.stream>>>(dW_slots, rms_slots, ntile, T, G, dW, rms_part);
  return cudaGetLastError();
}

cudaError_t launch_bwd_stats_tc(const Args& a, int K, const float* dA2, const float* dB2, void* dkc, void* dvc,
                                float* dbeta, uint32_t* status) {
  const size_t smem = sizeof(StatsTcSmem) + 1024;
  CUtensorMap tdk, tdv;
  const long long BF = (long long)a.sh.B * a.sh.F;
  if (!tmap_tokens_bf16(&tdk, dkc, a.sh.d, a.sh.H, a.sh.S, BF, kBT) ||
      !tmap_tokens_bf16(&tdv, dvc, a.sh.d, a.sh.H, a.sh.S, BF, kBT))
    return cudaErrorInvalidValue;
  if (K != 1 && K != 3) return cudaErrorInvalidValue;
  auto kern = K == 3 ? k_bwd_stats_tc<3> : k_bwd_stats_tc<1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long units = a.NF() * ((a.sh.S + kBT - 1) / kBT);
  const unsigned grid = (unsigned)(units < kStatsGrid ? units : kStatsGrid);   // one CTA per SM
  kern<<<grid, kStatsThreads, smem, a.stream>>>(
      tdk, tdv, static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v), a.beta, a.conv_k_w,
      a.conv_v_w, dA2, dB2, static_cast<__nv_bfloat16*>(dkc), static_cast<__nv_bfloat16*>(dvc), dbeta, a.sh.H,
      a.sh.F, a.sh.S, a.NF(), status);
  return cudaGetLastError();
}

cudaError_t launch_bwd_scan_tc(const Args& a, const uint16_t* nimg, const float* dPin, const float* dQin,
                               float* lam_all, float* dX_all, float* dseed2, uint32_t* status) {
  const size_t smem = sizeof(BwdScanSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_bwd_scan_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_bwd_scan_tc<<<dim3((unsigned)((long long)a.sh.B * a.sh.H), 2), kBwdScanThreads, smem, a.stream>>>(
      nimg, a.alpha, dPin, dQin, lam_all, dX_all, dseed2, a.sh.H, a.sh.F, status);
  return cudaGetLastError();
}

}  // namespace vdn
