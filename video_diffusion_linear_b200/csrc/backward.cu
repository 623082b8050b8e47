// Backward pass of the VDN-H3 linear branch: the gradients of the five steps of
// "VDN-Minimax-H3 bidirectional linear branch in five steps" and of the
// text-state seeds, taken in reverse order (the page trains the branch, stages
// A1/A2, but prints no backward; this is the exact gradient of the forward).
//
// The forward runs first with its per-frame export (A_f, B_f, N_f, P_f, Q_f, W_t
// in fp32); then, in fp32 SIMT kernels (fp32 inputs, d = 16 and 128; for bf16 at
// d = 128 the read-out, statistics and scan reversals run on the tensor cores in
// tc_backward.cu and the conv reversal in k_bwd_conv128):
//   k_bwd_readout  (batch, head, frame): recompute q', o = W_t q', RMSNorm; write
//                  dgate and dq; dW_t = sum_s do_s q'_s^T; RMS-weight partials
//   k_bwd_gather   (batch, head, column block): dW_t onto the boundary states P_{lo-1} and
//                  Q_{hi+1} (or the seed at a clip edge), d alpha of the bridge
//   k_bwd_scan     (batch, head, direction): the adjoint recurrence of each scan,
//                  frame by frame in reverse order of absorption, storing lam_f, dX_f
//   k_bwd_scan_grads (batch, head, frame, direction): dA, dB, d alpha of each step
//   k_bwd_stats    (batch, head, frame): dk', dv', d beta from dA_f, dB_f; L2-norm
//                  and SiLU reversed into the gradients of the conv outputs
//   k_bwd_conv     the short conv reversed (dk, dv, tap partials); k_bwd_conv128
//                  the bf16, d = 128 form (8 channels x a run of 32 tokens per thread)
//   k_bwd_finish   reductions over CTAs, heads and batch; d alpha summed
#include <cuda_bf16.h>

#include <type_traits>

#include "common.cuh"
#include "image.cuh"
#include "internal.h"

namespace vdn {
namespace {

constexpr int kBT = 256;   // threads of every backward block
constexpr int kBwdMaxWindow = 64;   // frames of a window whose alpha the gather reversal stages
constexpr int kTok = 32;   // tokens per tile of the per-token kernels

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + expf(-x)); }
// d silu(x) = sigma(x) (1 + x (1 - sigma(x))) dx
__device__ __forceinline__ float silu_grad(float x, float g) {
  const float s = sigmoidf_(x);
  return g * s * (1.f + x * (1.f - s));
}

// ---------------------------------------------------------------- per-token helpers (one warp per token)
// Lane `lane` holds channels c = lane + 32 r, r < PER (d = 16: lanes 16..31 hold nothing).
template <int D>
struct Lanes {
  static constexpr int PER = D >= 32 ? D / 32 : 1;
  __device__ static bool has(int lane, int r) { return lane + 32 * r < D; }
};

// x_hat = x / n, n = sqrt(sum x^2 + eps): dx = (g - x_hat (x_hat . g)) / n
template <int D>
__device__ __forceinline__ void l2n_grad(const float (&x)[Lanes<D>::PER], const float (&g)[Lanes<D>::PER],
                                         float (&dx)[Lanes<D>::PER], int lane) {
  constexpr int PER = Lanes<D>::PER;
  float ss = 0.f;
#pragma unroll
  for (int r = 0; r < PER; ++r) ss += Lanes<D>::has(lane, r) ? x[r] * x[r] : 0.f;
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss + kL2Eps);
  float xg = 0.f;
#pragma unroll
  for (int r = 0; r < PER; ++r) xg += Lanes<D>::has(lane, r) ? x[r] * inv * g[r] : 0.f;
  xg = warp_sum(xg);
#pragma unroll
  for (int r = 0; r < PER; ++r) dx[r] = (g[r] - x[r] * inv * xg) * inv;
}

// ---------------------------------------------------------------- tile products in shared memory
// out[t][i] = sum_j in[t][j] M(i, j) over a tile of kTok tokens, with M(i, j) read
// from a row-padded (stride D + 1) shared matrix as m[i (D+1) + j] or, transposed,
// m[j (D+1) + i].  Thread tid owns token t = tid / 8 and channels i = tid % 8 + 8 u.
template <int D, bool kTrans>
__device__ __forceinline__ void tile_matvec(float* out, const float* in, const float* m) {
  constexpr int U = D / 8;
  const int t = threadIdx.x >> 3, i0 = threadIdx.x & 7;
  float acc[U];
#pragma unroll
  for (int u = 0; u < U; ++u) acc[u] = 0.f;
  const float* x = in + t * (D + 1);
  for (int j = 0; j < D; ++j) {
    const float xj = x[j];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + 8 * u;
      acc[u] = fmaf(xj, kTrans ? m[j * (D + 1) + i] : m[i * (D + 1) + j], acc[u]);
    }
  }
#pragma unroll
  for (int u = 0; u < U; ++u) out[t * (D + 1) + i0 + 8 * u] = acc[u];
}

// C = alpha op(A) op(B) for D x D row-major matrices in global memory, by the whole
// block (kBT threads; thread (ty, tx) owns rows ty + 16 r and columns tx + 16 s).
// `slab` is 2 * 16 * (D + 1) floats of shared memory.  Ends with a block barrier.
template <int D>
__device__ void cta_mm(float* __restrict__ C, const float* __restrict__ A, bool tA, const float* __restrict__ Bm,
                       bool tB, float alpha, float* slab) {
  constexpr int R = D / 16;
  float* As = slab;                 // As[kk][i] = op(A)[i][k0 + kk]
  float* Bs = slab + 16 * (D + 1);  // Bs[kk][j] = op(B)[k0 + kk][j]
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[R][R];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int s = 0; s < R; ++s) acc[r][s] = 0.f;
  // the next 16-wide slab is read into registers while this one is multiplied
  constexpr int NL = 16 * D / kBT;   // elements of each operand per thread and slab
  float na[NL], nb[NL];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int u = 0; u < NL; ++u) {
      const int e = tid + u * kBT, kk = e / D, i = e % D, k = k0 + kk;
      na[u] = tA ? A[k * D + i] : A[i * D + k];
      nb[u] = tB ? Bm[i * D + k] : Bm[k * D + i];
    }
  };
  fetch(0);
  for (int k0 = 0; k0 < D; k0 += 16) {
#pragma unroll
    for (int u = 0; u < NL; ++u) {
      const int e = tid + u * kBT, kk = e / D, i = e % D;
      As[kk * (D + 1) + i] = na[u];
      Bs[kk * (D + 1) + i] = nb[u];
    }
    __syncthreads();
    if (k0 + 16 < D) fetch(k0 + 16);
#pragma unroll 4
    for (int kk = 0; kk < 16; ++kk) {
      float a[R], b[R];
#pragma unroll
      for (int r = 0; r < R; ++r) a[r] = As[kk * (D + 1) + ty + 16 * r];
#pragma unroll
      for (int s = 0; s < R; ++s) b[s] = Bs[kk * (D + 1) + tx + 16 * s];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int s = 0; s < R; ++s) acc[r][s] = fmaf(a[r], b[s], acc[r][s]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int s = 0; s < R; ++s) C[(ty + 16 * r) * D + tx + 16 * s] = alpha * acc[r][s];
  __syncthreads();
}

// ---------------------------------------------------------------- step 5 reversed
template <int D>
struct ReadoutSmem {
  float W[D * (D + 1)];     // W_t, rows padded
  float qf[kTok * (D + 1)];
  float dov[kTok * (D + 1)];
  float o[kTok * (D + 1)];  // o, then dq'
  float rms[kBT / 32][D];   // per-warp RMS-weight partials
};

template <int D, typename T>
__global__ void __launch_bounds__(kBT) k_bwd_readout(const T* __restrict__ q, const T* __restrict__ gate,
                                                     const T* __restrict__ dout, const float* __restrict__ rms_w,
                                                     const float* __restrict__ Wall, float* __restrict__ dWall,
                                                     float* __restrict__ rms_part, T* __restrict__ dq,
                                                     T* __restrict__ dgate, int H, int F, int S) {
  constexpr int PER = Lanes<D>::PER;
  extern __shared__ float smem_f[];
  ReadoutSmem<D>& sm = *reinterpret_cast<ReadoutSmem<D>*>(smem_f);
  const long long fi = blockIdx.x;             // (b, h, f)
  const int f = (int)(fi % F);
  const long long bh = fi / F;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const long long N = (long long)F * S;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* Wt = Wall + fi * D * D;
  for (int e = tid; e < D * D; e += kBT) sm.W[(e / D) * (D + 1) + e % D] = Wt[e];
  float rw[PER], racc[PER];
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    rw[r] = Lanes<D>::has(lane, r) ? rms_w[lane + 32 * r] : 0.f;
    racc[r] = 0.f;
  }
  constexpr int R = D / 16;
  float dW[R][R];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int s = 0; s < R; ++s) dW[r][s] = 0.f;
  __syncthreads();

  for (int s0 = 0; s0 < S; s0 += kTok) {
    // q' of the tile's tokens (zero rows past the frame)
    for (int t = warp; t < kTok; t += kBT / 32) {
      const int s = s0 + t;
      float qs[PER];
      float ss = 0.f;
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        qs[r] = 0.f;
        if (s < S && Lanes<D>::has(lane, r))
          qs[r] = silu_precise(to_f32(q[((b * N + (long long)f * S + s) * H + h) * D + lane + 32 * r]));
        ss += qs[r] * qs[r];
      }
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss + kL2Eps);
#pragma unroll
      for (int r = 0; r < PER; ++r)
        if (Lanes<D>::has(lane, r)) sm.qf[t * (D + 1) + lane + 32 * r] = s < S ? qs[r] * inv : 0.f;
    }
    __syncthreads();
    tile_matvec<D, false>(sm.o, sm.qf, sm.W);          // o = W_t q'
    __syncthreads();
    // RMSNorm and gate reversed: dgate, d rms_w, do
    for (int t = warp; t < kTok; t += kBT / 32) {
      const int s = s0 + t;
      if (s >= S) {
#pragma unroll
        for (int r = 0; r < PER; ++r)
          if (Lanes<D>::has(lane, r)) sm.dov[t * (D + 1) + lane + 32 * r] = 0.f;
        continue;
      }
      const long long row = ((b * N + (long long)f * S + s) * H + h) * D;
      float o[PER], dy[PER];
      float ss = 0.f;
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        o[r] = Lanes<D>::has(lane, r) ? sm.o[t * (D + 1) + lane + 32 * r] : 0.f;
        ss += o[r] * o[r];
      }
      ss = warp_sum(ss);
      const float rr = rsqrtf(ss / D + kRmsEps);
      float so = 0.f;
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        if (!Lanes<D>::has(lane, r)) {
          dy[r] = 0.f;
          continue;
        }
        const int c = lane + 32 * r;
        const float go = to_f32(dout[row + c]), g = to_f32(gate[row + c]);
        const float oh = o[r] * rr;
        dgate[row + c] = from_f32<T>(go * oh * rw[r]);
        dy[r] = go * g;
        racc[r] = fmaf(dy[r], oh, racc[r]);
        so += dy[r] * rw[r] * o[r];
      }
      so = warp_sum(so);
      const float k3 = rr * rr * rr * so / D;
#pragma unroll
      for (int r = 0; r < PER; ++r)
        if (Lanes<D>::has(lane, r)) sm.dov[t * (D + 1) + lane + 32 * r] = rr * dy[r] * rw[r] - k3 * o[r];
    }
    __syncthreads();
    tile_matvec<D, true>(sm.o, sm.dov, sm.W);          // dq' = W_t^T do
    // dW_t += do q'^T over the tile
    {
      const int ty = tid >> 4, tx = tid & 15;
      for (int t = 0; t < kTok; ++t) {
        float a[R], c[R];
#pragma unroll
        for (int r = 0; r < R; ++r) a[r] = sm.dov[t * (D + 1) + ty + 16 * r];
#pragma unroll
        for (int s = 0; s < R; ++s) c[s] = sm.qf[t * (D + 1) + tx + 16 * s];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int s = 0; s < R; ++s) dW[r][s] = fmaf(a[r], c[s], dW[r][s]);
      }
    }
    __syncthreads();
    // q' = l2n(silu(q)) reversed
    for (int t = warp; t < kTok; t += kBT / 32) {
      const int s = s0 + t;
      if (s >= S) continue;
      const long long row = ((b * N + (long long)f * S + s) * H + h) * D;
      float x[PER], qs[PER], g[PER], dqs[PER];
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        x[r] = Lanes<D>::has(lane, r) ? to_f32(q[row + lane + 32 * r]) : 0.f;
        qs[r] = Lanes<D>::has(lane, r) ? silu_precise(x[r]) : 0.f;
        g[r] = Lanes<D>::has(lane, r) ? sm.o[t * (D + 1) + lane + 32 * r] : 0.f;
      }
      l2n_grad<D>(qs, g, dqs, lane);
#pragma unroll
      for (int r = 0; r < PER; ++r)
        if (Lanes<D>::has(lane, r)) dq[row + lane + 32 * r] = from_f32<T>(silu_grad(x[r], dqs[r]));
    }
    __syncthreads();
  }
  {
    const int ty = tid >> 4, tx = tid & 15;
    float* dWt = dWall + fi * D * D;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int s = 0; s < R; ++s) dWt[(ty + 16 * r) * D + tx + 16 * s] = dW[r][s];
  }
#pragma unroll
  for (int r = 0; r < PER; ++r)
    if (Lanes<D>::has(lane, r)) sm.rms[warp][lane + 32 * r] = racc[r];
  __syncthreads();
  for (int c = tid; c < D; c += kBT) {
    float sacc = 0.f;
    for (int w = 0; w < kBT / 32; ++w) sacc += sm.rms[w][c];
    rms_part[fi * D + c] = sacc;
  }
}

// ---------------------------------------------------------------- step 4 (gather + bridge) reversed
// dPin[b, h][0] receives the gradient of the seed as P_{-1}, dPin[b, h][f + 1] that of P_f;
// dQin[b, h][f] that of Q_f, dQin[b, h][F] that of the seed as Q_F.  dalpha_g [B, H, F, D].
// Block (b·h, column block): columns are independent here, so each block owns CB columns for
// every query frame t (its updates of the boundary slots are ordered), rows split over RG groups.
template <int D>
__global__ void __launch_bounds__(kBT) k_bwd_gather(const float* __restrict__ P, const float* __restrict__ Q,
                                                    const float* __restrict__ alpha,
                                                    const float* __restrict__ text_state,
                                                    const float* __restrict__ dWall, float* __restrict__ dPin,
                                                    float* __restrict__ dQin, float* __restrict__ dalpha_g, int H,
                                                    int F, int chunk, int radius) {
  constexpr int CB = D < 32 ? D : 32;      // columns per block
  constexpr int RG = kBT / CB;             // row groups
  constexpr int RPT = D / RG;              // rows per thread
  __shared__ float red[2][RG][CB];
  // alpha of the current window's frames (a chunk's frames share the window), and the suffix
  // products used for "the product of the other factors"
  __shared__ float aw[kBwdMaxWindow][CB], rt[kBwdMaxWindow][CB];
  const long long bh = blockIdx.x;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const int jj = threadIdx.x % CB, rg = threadIdx.x / CB;
  const int j = blockIdx.y * CB + jj;
  const long long DD = (long long)D * D;
  float* dP = dPin + bh * (F + 1) * DD;
  float* dQ = dQin + bh * (F + 1) * DD;
  float* dal = dalpha_g + bh * F * D;
  auto alpha_at = [&](int f) { return alpha[((b * F + f) * H + h) * D + j]; };
  int wlo = -1, whi = -1;
  for (int t = 0; t < F; ++t) {
    int lo, hi;
    window_bounds(t, F, chunk, radius, lo, hi);
    const bool staged = hi - lo + 1 <= kBwdMaxWindow;   // uniform over the block
    if (staged && (lo != wlo || hi != whi)) {   // stage the window's alpha (all loads issued together)
      __syncthreads();
      for (int e = threadIdx.x; e < (hi - lo + 1) * CB; e += kBT) {
        const int f = lo + e / CB, c = e % CB;
        aw[f - lo][c] = alpha[((b * F + f) * H + h) * D + blockIdx.y * CB + c];
      }
      wlo = lo;
      whi = hi;
      __syncthreads();
    }
    auto al = [&](int f) { return staged ? aw[f - lo][jj] : alpha_at(f); };
    float a = 1.f, bb = 1.f;
    for (int f = lo; f <= t; ++f) a *= al(f);
    for (int f = t; f <= hi; ++f) bb *= al(f);
    const float* dW = dWall + (bh * F + t) * DD;
    const float* pre = lo == 0 ? nullptr : P + (bh * F + lo - 1) * DD;
    const float* suf = hi == F - 1 ? nullptr : Q + (bh * F + hi + 1) * DD;
    float* dpre = dP + (long long)lo * DD;          // slot lo: P_{lo-1} (slot 0: the seed)
    float* dsuf = dQ + (long long)(hi + 1) * DD;    // slot hi + 1: Q_{hi+1} (slot F: the seed)
    float da = 0.f, db = 0.f;
#pragma unroll 4
    for (int r = 0; r < RPT; ++r) {
      const int i = rg + RG * r;
      const long long e = (long long)i * D + j;
      const float g = dW[e];
      dpre[e] += g * a;
      dsuf[e] += g * bb;
      const float sd = text_state ? 0.5f * text_state[(long long)h * DD + e] : 0.f;
      da = fmaf(pre ? pre[e] : sd, g, da);
      db = fmaf(suf ? suf[e] : sd, g, db);
    }
    red[0][rg][jj] = da;
    red[1][rg][jj] = db;
    __syncthreads();
    if (rg == 0) {
      da = db = 0.f;
      for (int r = 0; r < RG; ++r) {
        da += red[0][r][jj];
        db += red[1][r][jj];
      }
      // d prod / d alpha_f = product of the other factors = (left of f) x (right of f); a window
      // wider than the staging buffer takes the products factor by factor
      if (!staged) {
        for (int f = lo; f <= t; ++f) {
          float pr = 1.f;
          for (int g2 = lo; g2 <= t; ++g2)
            if (g2 != f) pr *= alpha_at(g2);
          dal[f * D + j] += da * pr;
        }
        for (int f = t; f <= hi; ++f) {
          float pr = 1.f;
          for (int g2 = t; g2 <= hi; ++g2)
            if (g2 != f) pr *= alpha_at(g2);
          dal[f * D + j] += db * pr;
        }
      }
      if (staged) {
        float right = 1.f;
        for (int f = t; f >= lo; --f) {
          rt[f - lo][jj] = right;
          right *= aw[f - lo][jj];
        }
        float left = 1.f;
        for (int f = lo; f <= t; ++f) {
          dal[f * D + j] += da * (left * rt[f - lo][jj]);
          left *= aw[f - lo][jj];
        }
        right = 1.f;
        for (int f = hi; f >= t; --f) {
          rt[f - lo][jj] = right;
          right *= aw[f - lo][jj];
        }
        left = 1.f;
        for (int f = t; f <= hi; ++f) {
          dal[f * D + j] += db * (left * rt[f - lo][jj]);
          left *= aw[f - lo][jj];
        }
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- steps 3-4 (scans) reversed
// Block (b, h, dir): dir 0 reverses the prefix scan P_f = step(P_{f-1}, f) from f = F-1 down,
// dir 1 the suffix scan Q_f = step(Q_{f+1}, f) from f = 0 up.  For the generic step
// S_out = (S_in D + cpre B) N + cpost B the recurrence needs only
//   lam_f = (gradient reaching S_out) ,  dX_f = lam_f N^T (N symmetric) ,  next lam = dX_f D;
// lam_f and dX_f of every frame are stored for k_bwd_scan_grads, which forms dA, dB, d alpha.
// scratch: 2 D x D per block (the running lam, the seed).
template <int D>
__global__ void __launch_bounds__(kBT) k_bwd_scan(const float* __restrict__ Nm, const float* __restrict__ alpha,
                                                  const float* __restrict__ text_state,
                                                  const float* __restrict__ dPin, const float* __restrict__ dQin,
                                                  float* __restrict__ lam_all, float* __restrict__ dX_all,
                                                  float* __restrict__ dseed2, float* __restrict__ scratch, int H,
                                                  int F) {
  __shared__ float slab[2 * 16 * (D + 1)];
  const long long bh = blockIdx.x;
  const int dir = blockIdx.y;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const long long DD = (long long)D * D;
  const long long BH = gridDim.x;
  const int tid = threadIdx.x;
  float* lam = scratch + (bh * 2 + dir) * 2 * DD;
  float* seed = lam + DD;
  const float* din = (dir == 0 ? dPin : dQin) + bh * (F + 1) * DD;
  for (long long e = tid; e < DD; e += kBT) {
    seed[e] = text_state ? 0.5f * text_state[(long long)h * DD + e] : 0.f;
    lam[e] = 0.f;
  }
  __syncthreads();
  for (int it = 0; it < F; ++it) {
    const int f = dir == 0 ? F - 1 - it : it;
    const long long fo = (bh * F + f) * DD;
    const long long go = ((long long)dir * BH * F + bh * F + f) * DD;
    const float* gin = din + (long long)(dir == 0 ? f + 1 : f) * DD;
    float* lf = lam_all + go;
    for (long long e = tid; e < DD; e += kBT) lf[e] = lam[e] + gin[e];
    __syncthreads();
    cta_mm<D>(dX_all + go, lf, false, Nm + fo, true, 1.f, slab);
    const float* dX = dX_all + go;
    for (long long e = tid; e < DD; e += kBT) {
      const int jj = (int)(e % D);
      lam[e] = dX[e] * alpha[((b * F + f) * H + h) * D + jj];
    }
    __syncthreads();
  }
  const float* g0 = din + (long long)(dir == 0 ? 0 : F) * DD;
  for (long long e = tid; e < DD; e += kBT) dseed2[((long long)dir * BH + bh) * DD + e] = lam[e] + g0[e];
}

// Block (b h f, dir): the step's gradients from lam_f and dX_f,
//   dB = cpre dX + cpost lam, d alpha_j = sum_i S_in[i][j] dX[i][j],
//   dA = -c2 S_out^T dX (N = (I + c2 A)^-1) or -c2 X^T lam with X = S_in D + cpre B (N = I - c2 A).
// Xbuf: one D x D per block.
template <int D>
__global__ void __launch_bounds__(kBT) k_bwd_scan_grads(const float* __restrict__ Bm, const float* __restrict__ P,
                                                        const float* __restrict__ Q,
                                                        const float* __restrict__ alpha, RuleCoef rc,
                                                        const float* __restrict__ lam_all,
                                                        const float* __restrict__ dX_all,
                                                        const float* __restrict__ text_state,
                                                        float* __restrict__ dA2, float* __restrict__ dB2,
                                                        float* __restrict__ dalpha2, float* __restrict__ Xbuf, int H,
                                                        int F) {
  __shared__ float slab[2 * 16 * (D + 1)];
  const long long fi = blockIdx.x;            // (b, h, f)
  const int dir = blockIdx.y;
  const long long NFt = gridDim.x;
  const int f = (int)(fi % F);
  const long long bh = fi / F;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const long long DD = (long long)D * D;
  const int tid = threadIdx.x;
  const long long fo = fi * DD;
  const long long go = ((long long)dir * NFt + fi) * DD;
  const float* S = dir == 0 ? P : Q;
  const float* S_out = S + fo;
  // S_in: the neighbouring state, or the seed 0.5 T at the clip edge (read elementwise only)
  const bool edge = dir == 0 ? f == 0 : f == F - 1;
  const float* S_nb = dir == 0 ? S + fo - DD : S + fo + DD;
  auto s_in = [&](long long e) {
    return edge ? (text_state ? 0.5f * text_state[(long long)h * DD + e] : 0.f) : S_nb[e];
  };
  const float* lam = lam_all + go;
  const float* dX = dX_all + go;
  float* dA = dA2 + go;
  float* dB = dB2 + go;
  if (rc.solve) {
    cta_mm<D>(dA, S_out, true, dX, false, -rc.c2, slab);
  } else if (rc.c2 != 0.f) {
    float* X = Xbuf + go;
    for (long long e = tid; e < DD; e += kBT) {
      const int jj = (int)(e % D);
      X[e] = s_in(e) * alpha[((b * F + f) * H + h) * D + jj] + rc.cpre * Bm[fo + e];
    }
    __syncthreads();
    cta_mm<D>(dA, X, true, lam, false, -rc.c2, slab);
  } else {
    for (long long e = tid; e < DD; e += kBT) dA[e] = 0.f;
  }
  for (long long e = tid; e < DD; e += kBT) dB[e] = rc.cpre * dX[e] + rc.cpost * lam[e];
  if (tid < D) {
    float acc = 0.f;
    for (int i = 0; i < D; ++i) acc = fmaf(s_in((long long)i * D + tid), dX[i * D + tid], acc);
    dalpha2[((long long)dir * NFt + fi) * D + tid] = acc;
  }
}

// ---------------------------------------------------------------- step 2 reversed (+ step 1 up to the conv)
template <int D>
struct StatsSmem {
  float dAs[D * (D + 1)];   // dA + dA^T
  float dB[D * (D + 1)];
  float kf[kTok * (D + 1)];
  float vf[kTok * (D + 1)];
  float u[kTok * (D + 1)];  // (dA + dA^T) k'
  float w[kTok * (D + 1)];  // dB^T v'
  float z[kTok * (D + 1)];  // dB k'
};

template <int D, typename T>
__global__ void __launch_bounds__(kBT) k_bwd_stats(const T* __restrict__ k, const T* __restrict__ v,
                                                   const float* __restrict__ beta, const float* __restrict__ wk,
                                                   const float* __restrict__ wv, int K,
                                                   const float* __restrict__ dA2, const float* __restrict__ dB2,
                                                   T* __restrict__ dkc, T* __restrict__ dvc,
                                                   float* __restrict__ dbeta, int H, int F, int S) {
  constexpr int PER = Lanes<D>::PER;
  constexpr int TPW = kTok / (kBT / 32);      // tokens per warp and tile
  extern __shared__ float smem_f[];
  StatsSmem<D>& sm = *reinterpret_cast<StatsSmem<D>*>(smem_f);
  const long long fi = blockIdx.x;
  const int f = (int)(fi % F);
  const long long bh = fi / F;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const long long N = (long long)F * S;
  const long long DD = (long long)D * D;
  const long long BHF = (long long)gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (long long e = tid; e < DD; e += kBT) {
    const int i = (int)(e / D), j = (int)(e % D);
    const float a_ij = dA2[fi * DD + e] + dA2[(BHF + fi) * DD + e];
    const float a_ji = dA2[fi * DD + j * D + i] + dA2[(BHF + fi) * DD + j * D + i];
    sm.dAs[i * (D + 1) + j] = a_ij + a_ji;
    sm.dB[i * (D + 1) + j] = dB2[fi * DD + e] + dB2[(BHF + fi) * DD + e];
  }
  const int pad = (K - 1) / 2;
  for (int s0 = 0; s0 < S; s0 += kTok) {
    // features of the tile's tokens; the pre-activations stay in registers
    float kc[TPW][PER], vc[TPW][PER];
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
      const int t = warp * TPW + tt, s = s0 + t;
      float ks[PER];
      float ss = 0.f;
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        kc[tt][r] = vc[tt][r] = ks[r] = 0.f;
        const int c = lane + 32 * r;
        if (s < S && Lanes<D>::has(lane, r)) {
          float ak = 0.f, av = 0.f;
          const long long base = ((b * N + (long long)f * S + s) * H + h) * D + c;
          if (wk == nullptr) ak = to_f32(k[base]);
          if (wv == nullptr) av = to_f32(v[base]);
          for (int j = 0; j < K; ++j) {
            const int sj = s + j - pad;
            if (sj < 0 || sj >= S) continue;
            const long long nb = ((b * N + (long long)f * S + sj) * H + h) * D + c;
            if (wk) ak = fmaf(wk[((long long)h * D + c) * K + j], to_f32(k[nb]), ak);
            if (wv) av = fmaf(wv[((long long)h * D + c) * K + j], to_f32(v[nb]), av);
          }
          kc[tt][r] = ak;
          vc[tt][r] = av;
          ks[r] = silu_precise(ak);
        }
        ss += ks[r] * ks[r];
      }
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss + kL2Eps);
#pragma unroll
      for (int r = 0; r < PER; ++r)
        if (Lanes<D>::has(lane, r)) {
          sm.kf[t * (D + 1) + lane + 32 * r] = ks[r] * inv;
          sm.vf[t * (D + 1) + lane + 32 * r] = s < S ? silu_precise(vc[tt][r]) : 0.f;
        }
    }
    __syncthreads();
    tile_matvec<D, false>(sm.u, sm.kf, sm.dAs);   // u_i = sum_j dAs[i][j] k'_j
    tile_matvec<D, true>(sm.w, sm.vf, sm.dB);     // w_i = sum_j dB[j][i] v'_j
    tile_matvec<D, false>(sm.z, sm.kf, sm.dB);    // z_i = sum_j dB[i][j] k'_j
    __syncthreads();
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
      const int t = warp * TPW + tt, s = s0 + t;
      if (s >= S) continue;                        // warp-uniform
      const long long tok = (b * N + (long long)f * S + s) * H + h;
      const float bt = beta[tok];
      float ks[PER], dkf[PER], dks[PER];
      float kb = 0.f;
#pragma unroll
      for (int r = 0; r < PER; ++r) {
        const int c = lane + 32 * r;
        ks[r] = dkf[r] = 0.f;
        if (!Lanes<D>::has(lane, r)) continue;
        const float kfc = sm.kf[t * (D + 1) + c], vfc = sm.vf[t * (D + 1) + c];
        const float u = sm.u[t * (D + 1) + c], w = sm.w[t * (D + 1) + c], z = sm.z[t * (D + 1) + c];
        // d beta = k'^T dA k' + v'^T dB k' = 1/2 k'^T (dA + dA^T) k' + v' . (dB k')
        kb += 0.5f * kfc * u + vfc * z;
        dkf[r] = bt * (u + w);
        ks[r] = silu_precise(kc[tt][r]);
        dvc[tok * D + c] = from_f32<T>(silu_grad(vc[tt][r], bt * z));
      }
      kb = warp_sum(kb);
      if (lane == 0) dbeta[tok] = kb;
      l2n_grad<D>(ks, dkf, dks, lane);
#pragma unroll
      for (int r = 0; r < PER; ++r)
        if (Lanes<D>::has(lane, r)) dkc[tok * D + lane + 32 * r] = from_f32<T>(silu_grad(kc[tt][r], dks[r]));
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- step 1 conv reversed
template <typename T> __device__ __forceinline__ void load8t(const T* p, float* v);
template <> __device__ __forceinline__ void load8t<float>(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <> __device__ __forceinline__ void load8t<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = bf16lo(w[e]);
    v[2 * e + 1] = bf16hi(w[e]);
  }
}
template <typename T> __device__ __forceinline__ void store8t(T* p, const float* v);
template <> __device__ __forceinline__ void store8t<float>(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
template <> __device__ __forceinline__ void store8t<__nv_bfloat16>(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<uint4*>(p) =
      make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

template <typename T> __device__ __forceinline__ void load4t(const T* p, float* v);
template <> __device__ __forceinline__ void load4t<float>(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <> __device__ __forceinline__ void load4t<__nv_bfloat16>(const __nv_bfloat16* p, float* v) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
}
template <typename T> __device__ __forceinline__ void store4t(T* p, const float* v);
template <> __device__ __forceinline__ void store4t<float>(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <> __device__ __forceinline__ void store4t<__nv_bfloat16>(__nv_bfloat16* p, const float* v) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}

// Thread = (token, group of 4 channels), grid-stride over the tokens of head h = blockIdx.y:
// dk[s] = sum_j w[j] dkc[s - j + p] over in-frame indices (out[s'] reads x[s' + j - p]), and the
// tap partials sum_s dkc[s] k[s + j - p], reduced per block.  A missing conv is the identity
// (centre tap 1); KT is the tap count of the staged convs.
template <int D, typename T, int KT>
__global__ void __launch_bounds__(kBT, 2) k_bwd_conv(const T* __restrict__ k, const T* __restrict__ v,
                                                  const float* __restrict__ wk, const float* __restrict__ wv,
                                                  const T* __restrict__ dkc, const T* __restrict__ dvc,
                                                  T* __restrict__ dk, T* __restrict__ dv,
                                                  float* __restrict__ tap_part, int B, int H, int F, int S) {
  constexpr int CW = 4;                    // channels per thread
  constexpr int G = D / CW;                // channel groups
  constexpr int TPI = kBT / G;             // tokens per block and iteration
  constexpr int PAD = (KT - 1) / 2;
  __shared__ float red[kBT / 32][G][2][KT][CW];
  const int h = blockIdx.y;
  const int tid = threadIdx.x, cg = tid % G, tl = tid / G, warp = tid >> 5, lane = tid & 31;
  const int c0 = CW * cg;
  const long long N = (long long)F * S, total = (long long)B * N;
  float wkr[KT][CW], wvr[KT][CW], tk[KT][CW], tv[KT][CW];
#pragma unroll
  for (int j = 0; j < KT; ++j)
#pragma unroll
    for (int e = 0; e < CW; ++e) {
      wkr[j][e] = wk ? wk[((long long)h * D + c0 + e) * KT + j] : (j == PAD ? 1.f : 0.f);
      wvr[j][e] = wv ? wv[((long long)h * D + c0 + e) * KT + j] : (j == PAD ? 1.f : 0.f);
      tk[j][e] = tv[j][e] = 0.f;
    }
  for (long long tokn = (long long)blockIdx.x * TPI + tl; tokn < total; tokn += (long long)gridDim.x * TPI) {
    const long long b = tokn / N, n = tokn % N;
    const int s = (int)(n % S);
    const long long row = (b * N + n) * H + h;     // token row (times D)
    float ck[CW], cv[CW], gk[CW], gv[CW];
    load4t(dkc + row * D + c0, ck);
    load4t(dvc + row * D + c0, cv);
#pragma unroll
    for (int e = 0; e < CW; ++e) gk[e] = gv[e] = 0.f;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
      const int so = s - j + PAD;                  // out[so] reads x[s] through tap j
      if (so >= 0 && so < S) {
        float a[CW], c[CW];
        if (so == s) {
#pragma unroll
          for (int e = 0; e < CW; ++e) {
            a[e] = ck[e];
            c[e] = cv[e];
          }
        } else {
          load4t(dkc + (row + (long long)(so - s) * H) * D + c0, a);
          load4t(dvc + (row + (long long)(so - s) * H) * D + c0, c);
        }
#pragma unroll
        for (int e = 0; e < CW; ++e) {
          gk[e] = fmaf(wkr[j][e], a[e], gk[e]);
          gv[e] = fmaf(wvr[j][e], c[e], gv[e]);
        }
      }
      const int sx = s + j - PAD;                  // tap j of out[s] reads x[sx]
      if (sx >= 0 && sx < S) {
        float x[CW], y[CW];
        load4t(k + (row + (long long)(sx - s) * H) * D + c0, x);
        load4t(v + (row + (long long)(sx - s) * H) * D + c0, y);
#pragma unroll
        for (int e = 0; e < CW; ++e) {
          tk[j][e] = fmaf(ck[e], x[e], tk[j][e]);
          tv[j][e] = fmaf(cv[e], y[e], tv[j][e]);
        }
      }
    }
    store4t(dk + row * D + c0, gk);
    store4t(dv + row * D + c0, gv);
  }
  // tap partials: lanes with the same channel group within the warp, then the block's warps
#pragma unroll
  for (int off = G; off < 32; off <<= 1)   // (no-op once a warp holds one token's groups)
#pragma unroll
    for (int j = 0; j < KT; ++j)
#pragma unroll
      for (int e = 0; e < CW; ++e) {
        tk[j][e] += __shfl_xor_sync(0xffffffffu, tk[j][e], off);
        tv[j][e] += __shfl_xor_sync(0xffffffffu, tv[j][e], off);
      }
  if (lane < G)
#pragma unroll
    for (int j = 0; j < KT; ++j)
#pragma unroll
      for (int e = 0; e < CW; ++e) {
        red[warp][cg][0][j][e] = tk[j][e];
        red[warp][cg][1][j][e] = tv[j][e];
      }
  __syncthreads();
  for (int idx = tid; idx < G * 2 * KT * CW; idx += kBT) {
    const int e = idx % CW, j = (idx / CW) % KT, m = (idx / (CW * KT)) % 2, g2 = idx / (2 * CW * KT);
    float acc = 0.f;
    for (int w = 0; w < kBT / 32; ++w) acc += red[w][g2][m][j][e];
    tap_part[(((long long)h * gridDim.x + blockIdx.x) * 2 + m) * D * 3 + (CW * g2 + e) * 3 + j] = acc;
  }
}

// bf16, d = 128: thread = (tensor, 8 channels, run of 32 tokens of one frame).  The 16 threads
// of a channel row read it as one 256-byte line, and each thread slides a window of rows along its
// run (rows loaded four tokens ahead, each row of x and of the conv-output gradient read once), so
// the kernel streams k, v, dkc, dvc once and writes dk, dv once.  Same sums as k_bwd_conv:
// dx[s] = sum_j w[j] g[s - j + p], taps sum_s g[s] x[s + j - p], rows outside the frame zero.
constexpr int kConvRun = 32;
__device__ __forceinline__ void unpack_row8(uint4 u, float (&x)[8]) {
  x[0] = bf16lo(u.x); x[1] = bf16hi(u.x); x[2] = bf16lo(u.y); x[3] = bf16hi(u.y);
  x[4] = bf16lo(u.z); x[5] = bf16hi(u.z); x[6] = bf16lo(u.w); x[7] = bf16hi(u.w);
}
template <int KT>
__global__ void __launch_bounds__(512, 1) k_bwd_conv128(const __nv_bfloat16* __restrict__ k,
                                                        const __nv_bfloat16* __restrict__ v,
                                                        const float* __restrict__ wk, const float* __restrict__ wv,
                                                        const __nv_bfloat16* __restrict__ dkc,
                                                        const __nv_bfloat16* __restrict__ dvc,
                                                        __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                                                        float* __restrict__ tap_part, int B, int H, int F, int S) {
  constexpr int PAD = (KT - 1) / 2;
  __shared__ float red[8][2][16][KT][8];     // [warp of the tensor][tensor][channel group][tap][channel]
  const int tid = threadIdx.x, lane = tid & 31;
  const int ten = tid >> 8;                  // 0: k, 1: v
  const int g = tid & 15;                    // channels 8 g .. 8 g + 7
  const int sl = (tid >> 4) & 15;            // run slot of the block
  const int h = blockIdx.y;
  const __nv_bfloat16* x = ten ? v : k;
  const __nv_bfloat16* gx = ten ? dvc : dkc;
  __nv_bfloat16* out = ten ? dv : dk;
  const float* wg = ten ? wv : wk;
  float w[KT][8], tp[KT][8];
#pragma unroll
  for (int j = 0; j < KT; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      w[j][e] = wg ? wg[((long long)h * 128 + 8 * g + e) * KT + j] : (j == PAD ? 1.f : 0.f);
      tp[j][e] = 0.f;
    }
  const int nrun = (S + kConvRun - 1) / kConvRun;
  const long long runs = (long long)B * F * nrun;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (long long r = (long long)blockIdx.x * 16 + sl; r < runs; r += (long long)gridDim.x * 16) {
    const long long fb = r / nrun;                         // b F + f
    const int s0 = (int)(r - fb * nrun) * kConvRun, s1 = min(S, s0 + kConvRun);
    auto at = [&](int s) { return ((fb * S + s) * H + h) * 128 + 8 * g; };
    auto ld = [&](const __nv_bfloat16* p, int s) {
      return (s >= 0 && s < S) ? __ldg(reinterpret_cast<const uint4*>(p + at(s))) : z;
    };
    uint4 gw[6], xw[6];                                    // rows s - 1 .. s + 4 of the batch at s
    gw[0] = ld(gx, s0 - 1); xw[0] = ld(x, s0 - 1);
    gw[1] = ld(gx, s0);     xw[1] = ld(x, s0);
    for (int s = s0; s < s1; s += 4) {
#pragma unroll
      for (int i = 2; i < 6; ++i) {
        gw[i] = ld(gx, s - 1 + i);
        xw[i] = KT > 1 ? ld(x, s - 1 + i) : z;
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (s + t >= s1) break;
        float gm[8], gc[8], gp[8], xm[8], xc[8], xp[8];
        unpack_row8(gw[t], gm); unpack_row8(gw[t + 1], gc); unpack_row8(gw[t + 2], gp);
        unpack_row8(xw[t], xm); unpack_row8(xw[t + 1], xc); unpack_row8(xw[t + 2], xp);
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (KT == 3) {
            o[e] = fmaf(w[0][e], gp[e], fmaf(w[1][e], gc[e], w[2][e] * gm[e]));
            tp[0][e] = fmaf(gc[e], xm[e], tp[0][e]);
            tp[1][e] = fmaf(gc[e], xc[e], tp[1][e]);
            tp[2][e] = fmaf(gc[e], xp[e], tp[2][e]);
          } else {
            o[e] = w[0][e] * gc[e];
            tp[0][e] = fmaf(gc[e], xc[e], tp[0][e]);
          }
        }
        *reinterpret_cast<uint4*>(out + at(s + t)) =
            make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                       pack_bf16x2(o[6], o[7]));
      }
      gw[0] = gw[4]; xw[0] = xw[4];
      gw[1] = gw[5]; xw[1] = xw[5];
    }
  }
  // tap partials: the two run slots of a warp (lanes l and l + 16), then the tensor's 8 warps
#pragma unroll
  for (int j = 0; j < KT; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) tp[j][e] += __shfl_xor_sync(0xffffffffu, tp[j][e], 16);
  const int wt = (tid >> 5) & 7;
  if (lane < 16)
#pragma unroll
    for (int j = 0; j < KT; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) red[wt][ten][g][j][e] = tp[j][e];
  __syncthreads();
  for (int idx = tid; idx < 2 * 16 * KT * 8; idx += 512) {
    const int e = idx % 8, j = (idx / 8) % KT, g2 = (idx / (8 * KT)) % 16, m = idx / (8 * KT * 16);
    float acc = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2) acc += red[w2][m][g2][j][e];
    tap_part[(((long long)h * gridDim.x + blockIdx.x) * 2 + m) * 128 * 3 + (8 * g2 + e) * 3 + j] = acc;
  }
}

// ---------------------------------------------------------------- reductions
template <int D>
__global__ void __launch_bounds__(kBT) k_bwd_finish(const float* __restrict__ rms_part, long long nfr,
                                                    const float* __restrict__ tap_part, int conv_blocks, int K,
                                                    const float* __restrict__ dseed2,
                                                    const float* __restrict__ dalpha_g,
                                                    const float* __restrict__ dalpha2, float* __restrict__ drms_w,
                                                    float* __restrict__ dwk, float* __restrict__ dwv,
                                                    float* __restrict__ dtext, float* __restrict__ dalpha, int B,
                                                    int H, int F) {
  const long long DD = (long long)D * D;
  const long long BH = (long long)B * H;
  const long long gtid = (long long)blockIdx.x * kBT + threadIdx.x;
  const long long gsize = (long long)gridDim.x * kBT;
  // d rms_w: sum over every (b, h, f) block of the read-out
  for (long long c = gtid; c < D; c += gsize) {
    float acc = 0.f;
    for (long long i = 0; i < nfr; ++i) acc += rms_part[i * D + c];
    drms_w[c] = acc;
  }
  // conv taps: sum over the conv blocks of each head
  for (long long e = gtid; e < (long long)H * D * K; e += gsize) {
    const int h = (int)(e / (D * K)), c = (int)((e / K) % D), j = (int)(e % K);
    float ak = 0.f, av = 0.f;
    for (int blk = 0; blk < conv_blocks; ++blk) {
      const long long base = (((long long)h * conv_blocks + blk) * 2) * D * 3;
      ak += tap_part[base + c * 3 + j];
      av += tap_part[base + D * 3 + c * 3 + j];
    }
    if (dwk) dwk[e] = ak;
    if (dwv) dwv[e] = av;
  }
  // text state: 0.5 (d seed of the prefix scan + d seed of the suffix scan), summed over the batch
  if (dtext)
    for (long long e = gtid; e < (long long)H * DD; e += gsize) {
      const int h = (int)(e / DD);
      const long long m = e % DD;
      float acc = 0.f;
      for (int b = 0; b < B; ++b) {
        const long long bh = (long long)b * H + h;
        acc += dseed2[bh * DD + m] + dseed2[(BH + bh) * DD + m];
      }
      dtext[e] = 0.5f * acc;
    }
  // d alpha [B, F, H, D] = bridge + prefix-scan + suffix-scan parts ([B, H, F, D] each)
  for (long long e = gtid; e < BH * F * D; e += gsize) {
    const int c = (int)(e % D);
    const int f = (int)((e / D) % F);
    const long long bh = e / ((long long)F * D);
    const int h = (int)(bh % H);
    const long long b = bh / H;
    const float acc = dalpha_g[e] + dalpha2[e] + dalpha2[BH * F * D + e];
    dalpha[((b * F + f) * H + h) * D + c] = acc;
  }
}

}  // namespace

// ---------------------------------------------------------------- host side
SavedPlan plan_saved(const vdn_shape& sh) {
  SavedPlan p;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const long long NF = (long long)sh.B * sh.H * sh.F, DD = (long long)sh.d * sh.d;
  p.A = take(NF * DD * 4);
  p.Bm = take(NF * DD * 4);
  p.Nm = take(NF * DD * 4);
  p.P = take(NF * DD * 4);
  p.Q = take(NF * DD * 4);
  p.W = take(NF * DD * 4);
  p.nimg = use_tc(sh, VDN_IMPL_AUTO) ? take(NF * (size_t)kImgBytes) : 0;
  p.total = off;
  return p;
}

BwdPlan plan_backward(const vdn_shape& sh, int rule, bool recompute) {
  BwdPlan p;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const bool tc = use_tc(sh, VDN_IMPL_AUTO);
  const size_t fwd = plan_workspace(sh, rule, tc).total;
  const long long BH = (long long)sh.B * sh.H, NF = BH * sh.F, DD = (long long)sh.d * sh.d;
  const long long tokens = (long long)sh.B * sh.F * sh.S * sh.H;
  const size_t el = sh.dtype == VDN_DTYPE_BF16 ? 2 : 4;
  if (recompute) {
    p.fwd = take(fwd);                 // its first bytes hold the forward's status word
    p.out = take(tokens * sh.d * el);
    p.A = take(NF * DD * 4);
    p.Bm = take(NF * DD * 4);
    p.Nm = take(NF * DD * 4);
    p.P = take(NF * DD * 4);
    p.Q = take(NF * DD * 4);
    p.W = take(NF * DD * 4);
  } else {
    p.status = take(256);
  }
  p.dW = take(NF * DD * 4);
  p.dPin = take(BH * (sh.F + 1) * DD * 4);
  p.dQin = take(BH * (sh.F + 1) * DD * 4);
  p.dA2 = take(2 * NF * DD * 4);
  p.dB2 = take(2 * NF * DD * 4);
  p.dalpha_g = take(NF * sh.d * 4);
  p.dalpha2 = take(2 * NF * sh.d * 4);
  p.dseed2 = take(2 * BH * DD * 4);
  p.scan_scratch = take(BH * 2 * 2 * DD * 4);
  p.lam_all = take(2 * NF * DD * 4);
  p.dX_all = take(2 * NF * DD * 4);
  p.Xbuf = rule == VDN_RULE_SANA_SCALED ? take(2 * NF * DD * 4) : 0;
  p.rms_part = take(NF * sh.d * 4);
  if (sh.d == 128 && sh.dtype == VDN_DTYPE_BF16) {   // the tensor-core read-out reversal's slots
    p.dW_slots = take((NF + kBwdReadoutGrid) * DD * 4);
    p.rms_slots = take((NF + kBwdReadoutGrid) * sh.d * 4);
  }
  p.dkc = take(tokens * sh.d * el);          // the inputs' element type (bf16 on the tensor-core path)
  p.dvc = take(tokens * sh.d * el);
  p.tap_part = take((size_t)sh.H * kBwdConvBlocks * 2 * sh.d * 3 * 4);
  p.fwd_bytes = fwd;
  p.total = off;
  return p;
}

template <int D, typename T>
static cudaError_t run_backward_t(const Args& a, const BwdGrads& g, const BwdState& st, void* ws,
                                  const BwdPlan& p, void* const* events) {
  int ev = 2;   // events[0], events[1]: before and after the forward recompute
  auto mark = [&]() -> cudaError_t {
    return events ? cudaEventRecord((cudaEvent_t)events[ev++], a.stream) : cudaSuccess;
  };
  cudaError_t e;
  auto at = [&](size_t o) { return reinterpret_cast<float*>(static_cast<char*>(ws) + o); };
  const vdn_shape& sh = a.sh;
  const long long BH = (long long)sh.B * sh.H, NF = BH * sh.F;
  const int K = (a.conv_k_w || a.conv_v_w) ? sh.conv_width : 1;
  // bf16 at d = 128: the two per-token contractions on the tensor cores
  constexpr bool kTc = D == 128 && std::is_same<T, __nv_bfloat16>::value;
  uint32_t* status = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + p.status);   // first word of the workspace
  // step 5 reversed
  if (kTc) {
    if ((e = launch_bwd_readout_tc(a, g.dout, st.W, at(p.dW), at(p.rms_part), at(p.dW_slots), at(p.rms_slots),
                                   g.dq, g.dgate, status)) != cudaSuccess)
      return e;
  } else {
    const size_t smem = sizeof(ReadoutSmem<D>);
    e = cudaFuncSetAttribute(k_bwd_readout<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_bwd_readout<D, T><<<(unsigned)NF, kBT, smem, a.stream>>>(
        static_cast<const T*>(a.q), static_cast<const T*>(a.gate), static_cast<const T*>(g.dout), a.rms_w, st.W,
        at(p.dW), at(p.rms_part), static_cast<T*>(g.dq), static_cast<T*>(g.dgate), sh.H, sh.F, sh.S);
  }
  if ((e = mark()) != cudaSuccess) return e;
  // step 4 (gather + bridge) reversed
  k_bwd_gather<D><<<dim3((unsigned)BH, D < 32 ? 1 : D / 32), kBT, 0, a.stream>>>(
      st.P, st.Q, a.alpha, a.text_state, at(p.dW), at(p.dPin), at(p.dQin), at(p.dalpha_g), sh.H, sh.F, a.chunk,
      a.radius);
  if ((e = mark()) != cudaSuccess) return e;
  // steps 3-4 (scans) reversed
  if (kTc) {
    // the forward's hi/lo operand images of N_f (tensor-core path) serve the adjoint products
    const uint16_t* nimg = st.nimg;
    if ((e = launch_bwd_scan_tc(a, nimg, at(p.dPin), at(p.dQin), at(p.lam_all), at(p.dX_all), at(p.dseed2),
                                status)) != cudaSuccess)
      return e;
  } else {
    k_bwd_scan<D><<<dim3((unsigned)BH, 2), kBT, 0, a.stream>>>(st.Nm, a.alpha, a.text_state, at(p.dPin),
                                                                 at(p.dQin), at(p.lam_all), at(p.dX_all),
                                                                 at(p.dseed2), at(p.scan_scratch), sh.H, sh.F);
  }
  k_bwd_scan_grads<D><<<dim3((unsigned)NF, 2), kBT, 0, a.stream>>>(
      st.Bm, st.P, st.Q, a.alpha, rule_coef(a.rule, a.c), at(p.lam_all), at(p.dX_all), a.text_state,
      at(p.dA2), at(p.dB2), at(p.dalpha2), at(p.Xbuf), sh.H, sh.F);
  if ((e = mark()) != cudaSuccess) return e;
  // step 2 reversed
  if (kTc) {
    if ((e = launch_bwd_stats_tc(a, K, at(p.dA2), at(p.dB2), reinterpret_cast<void*>(at(p.dkc)),
                                 reinterpret_cast<void*>(at(p.dvc)), g.dbeta, status)) != cudaSuccess)
      return e;
  } else {
    const size_t smem = sizeof(StatsSmem<D>);
    e = cudaFuncSetAttribute(k_bwd_stats<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_bwd_stats<D, T><<<(unsigned)NF, kBT, smem, a.stream>>>(
        static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.beta, a.conv_k_w, a.conv_v_w, K, at(p.dA2),
        at(p.dB2), reinterpret_cast<T*>(at(p.dkc)), reinterpret_cast<T*>(at(p.dvc)), g.dbeta, sh.H, sh.F, sh.S);
  }
  if ((e = mark()) != cudaSuccess) return e;
  // step 1 (conv) reversed
  if (kTc && K == 3)
    k_bwd_conv128<3><<<dim3(kBwdConvBlocks, sh.H), 512, 0, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v), a.conv_k_w, a.conv_v_w,
        reinterpret_cast<const __nv_bfloat16*>(at(p.dkc)), reinterpret_cast<const __nv_bfloat16*>(at(p.dvc)),
        static_cast<__nv_bfloat16*>(g.dk), static_cast<__nv_bfloat16*>(g.dv), at(p.tap_part), sh.B, sh.H, sh.F, sh.S);
  else if (kTc)
    k_bwd_conv128<1><<<dim3(kBwdConvBlocks, sh.H), 512, 0, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v), a.conv_k_w, a.conv_v_w,
        reinterpret_cast<const __nv_bfloat16*>(at(p.dkc)), reinterpret_cast<const __nv_bfloat16*>(at(p.dvc)),
        static_cast<__nv_bfloat16*>(g.dk), static_cast<__nv_bfloat16*>(g.dv), at(p.tap_part), sh.B, sh.H, sh.F, sh.S);
  else if (K == 3)
    k_bwd_conv<D, T, 3><<<dim3(kBwdConvBlocks, sh.H), kBT, 0, a.stream>>>(
        static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.conv_k_w, a.conv_v_w,
        reinterpret_cast<const T*>(at(p.dkc)), reinterpret_cast<const T*>(at(p.dvc)),
        static_cast<T*>(g.dk), static_cast<T*>(g.dv), at(p.tap_part), sh.B, sh.H, sh.F, sh.S);
  else
    k_bwd_conv<D, T, 1><<<dim3(kBwdConvBlocks, sh.H), kBT, 0, a.stream>>>(
        static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.conv_k_w, a.conv_v_w,
        reinterpret_cast<const T*>(at(p.dkc)), reinterpret_cast<const T*>(at(p.dvc)),
        static_cast<T*>(g.dk), static_cast<T*>(g.dv), at(p.tap_part), sh.B, sh.H, sh.F, sh.S);
  if ((e = mark()) != cudaSuccess) return e;
  k_bwd_finish<D><<<148, kBT, 0, a.stream>>>(at(p.rms_part), NF, at(p.tap_part), kBwdConvBlocks, K, at(p.dseed2),
                                             at(p.dalpha_g), at(p.dalpha2), g.drms_w, g.dconv_k_w, g.dconv_v_w,
                                             g.dtext_state, g.dalpha, sh.B, sh.H, sh.F);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return mark();
}

cudaError_t run_backward(const Args& a, const BwdGrads& g, const BwdState& st, void* ws, const BwdPlan& p,
                         void* const* events) {
  const vdn_shape& sh = a.sh;
  const long long BH = (long long)sh.B * sh.H, DD = (long long)sh.d * sh.d;
  char* base = static_cast<char*>(ws);
  cudaError_t e;
  if ((e = cudaMemsetAsync(base + p.dPin, 0, BH * (sh.F + 1) * DD * 4, a.stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(base + p.dQin, 0, BH * (sh.F + 1) * DD * 4, a.stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(base + p.dalpha_g, 0, BH * sh.F * sh.d * 4, a.stream)) != cudaSuccess) return e;
  const bool bf = sh.dtype == VDN_DTYPE_BF16;
  if (sh.d == 16) return bf ? run_backward_t<16, __nv_bfloat16>(a, g, st, ws, p, events) : run_backward_t<16, float>(a, g, st, ws, p, events);
  return bf ? run_backward_t<128, __nv_bfloat16>(a, g, st, ws, p, events) : run_backward_t<128, float>(a, g, st, ws, p, events);
}

}  // namespace vdn
