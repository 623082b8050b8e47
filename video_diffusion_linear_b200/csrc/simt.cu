// SIMT (CUDA-core) kernels of the branch: the fp32 path for every supported d,
// and the reference-grade GPU path used for per-stage checks.
//
// Steps follow the page "VDN-Minimax-H3 bidirectional linear branch in five
// steps": Step 1 (NoPE features), Step 2 (frame statistics), Step 3/4 (delta
// rule, bidirectional scan) and Step 5 (read-out, RMSNorm, output gate).
#include "common.cuh"
#include "internal.h"

namespace vdn {

// ---------------------------------------------------------------- Step 1
// One warp per (batch, token, head); lane handles channels lane + 32 r.
// k, v: depthwise conv over the frame's tokens (centred, zero padding at the
// frame edge), SiLU; q: SiLU; q and k L2-normalised.
template <typename TI, typename TO, int D>
__global__ void __launch_bounds__(256) k_features_simt(const TI* __restrict__ q, const TI* __restrict__ k,
                                                       const TI* __restrict__ v, const float* __restrict__ wk,
                                                       const float* __restrict__ wv, int K, TO* __restrict__ qo,
                                                       TO* __restrict__ ko, TO* __restrict__ vo, int B, int F,
                                                       int S, int H) {
  constexpr int PER = (D + 31) / 32;
  long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  long long N = (long long)F * S;
  long long total = (long long)B * N * H;
  if (warp >= total) return;
  int h = (int)(warp % H);
  long long bn = warp / H;
  long long n = bn % N;
  long long b = bn / N;
  int s = (int)(n % S);
  int pad = (K - 1) / 2;
  float qv[PER], kv[PER], vv[PER];
  float sq = 0.f, sk = 0.f;
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    int c = lane + 32 * r;
    qv[r] = kv[r] = vv[r] = 0.f;
    if (c < D) {
      long long base = ((b * N + n) * H + h) * D + c;
      float x = to_f32(q[base]);
      qv[r] = silu_precise(x);
      float ak = 0.f, av = 0.f;
      if (wk == nullptr) ak = to_f32(k[base]);
      if (wv == nullptr) av = to_f32(v[base]);
      for (int j = 0; j < K; ++j) {
        int ss = s + j - pad;
        if (ss < 0 || ss >= S) continue;
        long long nb = ((b * N + (n - s + ss)) * H + h) * D + c;
        if (wk) ak = fmaf(wk[((long long)h * D + c) * K + j], to_f32(k[nb]), ak);
        if (wv) av = fmaf(wv[((long long)h * D + c) * K + j], to_f32(v[nb]), av);
      }
      kv[r] = silu_precise(ak);
      vv[r] = silu_precise(av);
      sq += qv[r] * qv[r];
      sk += kv[r] * kv[r];
    }
  }
  sq = warp_sum(sq);
  sk = warp_sum(sk);
  float iq = rsqrtf(sq + kL2Eps), ik = rsqrtf(sk + kL2Eps);
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    int c = lane + 32 * r;
    if (c < D) {
      long long base = ((b * N + n) * H + h) * D + c;
      qo[base] = from_f32<TO>(qv[r] * iq);
      ko[base] = from_f32<TO>(kv[r] * ik);
      vo[base] = from_f32<TO>(vv[r]);
    }
  }
}

template <typename TI, typename TO>
static cudaError_t features_dispatch(const vdn_shape& sh, const void* q, const void* k, const void* v,
                                     const float* wk, const float* wv, void* qo, void* ko, void* vo,
                                     cudaStream_t st) {
  long long warps = (long long)sh.B * sh.F * sh.S * sh.H;
  long long blocks = (warps * 32 + 255) / 256;
  int K = (wk || wv) ? sh.conv_width : 1;
  auto go = [&](auto kern) {
    kern<<<(unsigned)blocks, 256, 0, st>>>((const TI*)q, (const TI*)k, (const TI*)v, wk, wv, K, (TO*)qo, (TO*)ko,
                                           (TO*)vo, sh.B, sh.F, sh.S, sh.H);
  };
  if (sh.d == 16) go(k_features_simt<TI, TO, 16>);
  else go(k_features_simt<TI, TO, 128>);
  return cudaGetLastError();
}

cudaError_t launch_features_simt(const Args& a, float* qf, float* kf, float* vf) {
  if (a.sh.dtype == VDN_DTYPE_BF16)
    return features_dispatch<__nv_bfloat16, float>(a.sh, a.q, a.k, a.v, a.conv_k_w, a.conv_v_w, qf, kf, vf,
                                                   a.stream);
  return features_dispatch<float, float>(a.sh, a.q, a.k, a.v, a.conv_k_w, a.conv_v_w, qf, kf, vf, a.stream);
}

// ---------------------------------------------------------------- Step 2
// A_f = sum_s beta_s k'_s k'_s^T, B_f = sum_s beta_s v'_s k'_s^T.
// Block: one TLxTL tile of A or B of one (batch, head, frame); 16x16 threads,
// each accumulating an MTxMT micro-tile over the frame's tokens.
template <int D>
__global__ void __launch_bounds__(256) k_stats_simt(const float* __restrict__ kf, const float* __restrict__ vf,
                                                    const float* __restrict__ beta, float* __restrict__ A,
                                                    float* __restrict__ Bm, int H, int F, int S) {
  constexpr int TL = D < 64 ? D : 64;
  constexpr int NT = D / TL;
  constexpr int MT = TL / 16;
  constexpr int CH = 32;
  __shared__ float xs[CH][TL + 1];
  __shared__ float ys[CH][TL + 1];
  long long fi = blockIdx.x;
  int tile = blockIdx.y;
  int mat = tile / (NT * NT), ti = (tile / NT) % NT, tj = tile % NT;
  int f = (int)(fi % F);
  long long bh = fi / F;
  int h = (int)(bh % H);
  long long b = bh / H;
  long long N = (long long)F * S;
  const float* X = mat == 0 ? kf : vf;
  int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[MT][MT];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int n = 0; n < MT; ++n) acc[m][n] = 0.f;
  for (int s0 = 0; s0 < S; s0 += CH) {
    for (int e = tid; e < CH * TL; e += 256) {
      int r = e / TL, cc = e % TL, s = s0 + r;
      float xv = 0.f, yv = 0.f;
      if (s < S) {
        long long n = (long long)f * S + s;
        long long base = ((b * N + n) * H + h) * D;
        xv = X[base + ti * TL + cc];
        yv = beta[(b * N + n) * H + h] * kf[base + tj * TL + cc];
      }
      xs[r][cc] = xv;
      ys[r][cc] = yv;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < CH; ++r) {
      float xr[MT], yr[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        xr[m] = xs[r][ty * MT + m];
        yr[m] = ys[r][tx * MT + m];
      }
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < MT; ++n) acc[m][n] = fmaf(xr[m], yr[n], acc[m][n]);
    }
    __syncthreads();
  }
  float* out = (mat == 0 ? A : Bm) + fi * D * D;
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int n = 0; n < MT; ++n) out[(ti * TL + ty * MT + m) * D + tj * TL + tx * MT + n] = acc[m][n];
}

cudaError_t launch_stats_simt(const Args& a, const float* kf, const float* vf, float* A, float* Bm) {
  dim3 grid((unsigned)a.NF(), a.sh.d == 16 ? 2 : 8);
  if (a.sh.d == 16) k_stats_simt<16><<<grid, 256, 0, a.stream>>>(kf, vf, a.beta, A, Bm, a.sh.H, a.sh.F, a.sh.S);
  else k_stats_simt<128><<<grid, 256, 0, a.stream>>>(kf, vf, a.beta, A, Bm, a.sh.H, a.sh.F, a.sh.S);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- Step 3/4
// Bidirectional scan, one block per (batch, head, direction):
//   S_f = (S_{f-1} D_f + cpre B_f) N_f + cpost B_f,
// forward over f = 0..F-1 (prefix P_f) and backward over f = F-1..0 (suffix
// Q_f), both seeded with 0.5 * text_state.  Thread (ty, tx) owns state
// elements (ty + 16 ia, tx + 16 ib).
template <int D>
__global__ void __launch_bounds__(256) k_scan_simt(const float* __restrict__ Bm, const float* __restrict__ Nm,
                                                   const float* __restrict__ alpha, const float* __restrict__ text,
                                                   RuleCoef rc, float* __restrict__ P, float* __restrict__ Q,
                                                   int* __restrict__ pexp, int* __restrict__ qexp, int H, int F) {
  constexpr int R = D / 16;
  constexpr int LD = D + 1;
  extern __shared__ float sm[];
  float* X = sm;
  float* Ns = sm + D * LD;
  int dir = blockIdx.x & 1;
  long long bh = blockIdx.x >> 1;
  int h = (int)(bh % H);
  long long b = bh / H;
  int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float s[R][R];
#pragma unroll
  for (int ia = 0; ia < R; ++ia)
#pragma unroll
    for (int ib = 0; ib < R; ++ib) {
      int i = ty + 16 * ia, k = tx + 16 * ib;
      s[ia][ib] = text ? kTextStateScale * text[((long long)h * D + i) * D + k] : 0.f;
    }
  int ex = 0;   // block exponent: the true state is 2^ex s
  for (int step = 0; step < F; ++step) {
    int f = dir == 0 ? step : F - 1 - step;
    long long fi = bh * F + f;
    const float cpre = ldexpf(rc.cpre, -ex), cpost = ldexpf(rc.cpost, -ex);
    const float* Bf = Bm + fi * D * D;
    const float* Nf = Nm + fi * D * D;
    const float* al = alpha + ((b * F + f) * H + h) * D;
    for (int e = tid; e < D * D; e += 256) Ns[(e / D) * LD + (e % D)] = Nf[e];
#pragma unroll
    for (int ia = 0; ia < R; ++ia)
#pragma unroll
      for (int ib = 0; ib < R; ++ib) {
        int i = ty + 16 * ia, k = tx + 16 * ib;
        X[i * LD + k] = fmaf(s[ia][ib], al[k], cpre * Bf[i * D + k]);
      }
    __syncthreads();
    float acc[R][R];
#pragma unroll
    for (int ia = 0; ia < R; ++ia)
#pragma unroll
      for (int ib = 0; ib < R; ++ib) acc[ia][ib] = 0.f;
    for (int j = 0; j < D; ++j) {
      float xr[R], nr[R];
#pragma unroll
      for (int ia = 0; ia < R; ++ia) xr[ia] = X[(ty + 16 * ia) * LD + j];
#pragma unroll
      for (int ib = 0; ib < R; ++ib) nr[ib] = Ns[j * LD + tx + 16 * ib];
#pragma unroll
      for (int ia = 0; ia < R; ++ia)
#pragma unroll
        for (int ib = 0; ib < R; ++ib) acc[ia][ib] = fmaf(xr[ia], nr[ib], acc[ia][ib]);
    }
    float* dst = (dir == 0 ? P : Q) + fi * D * D;
    float amax = 0.f;
#pragma unroll
    for (int ia = 0; ia < R; ++ia)
#pragma unroll
      for (int ib = 0; ib < R; ++ib) {
        int i = ty + 16 * ia, k = tx + 16 * ib;
        s[ia][ib] = fmaf(cpost, Bf[i * D + k], acc[ia][ib]);
        dst[i * D + k] = s[ia][ib];
        amax = fmaxf(amax, fabsf(s[ia][ib]));
      }
    if (tid == 0) (dir == 0 ? pexp : qexp)[fi] = ex;
    if (__syncthreads_or(amax > kRenormAbove)) {
#pragma unroll
      for (int ia = 0; ia < R; ++ia)
#pragma unroll
        for (int ib = 0; ib < R; ++ib) s[ia][ib] *= kRenormScale;
      ex += kRenormExp;
    }
  }
}

cudaError_t launch_scan_simt(const Args& a, const float* Bm, const float* Nm, float* P, float* Q, int* pexp,
                             int* qexp) {
  RuleCoef rc = rule_coef(a.rule, a.c);
  unsigned grid = (unsigned)(2LL * a.sh.B * a.sh.H);
  if (a.sh.d == 16) {
    size_t smem = 2 * 16 * 17 * sizeof(float);
    k_scan_simt<16><<<grid, 256, smem, a.stream>>>(Bm, Nm, a.alpha, a.text_state, rc, P, Q, pexp, qexp, a.sh.H,
                                                    a.sh.F);
  } else {
    size_t smem = 2 * 128 * 129 * sizeof(float);
    cudaFuncSetAttribute(k_scan_simt<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_scan_simt<128><<<grid, 256, smem, a.stream>>>(Bm, Nm, a.alpha, a.text_state, rc, P, Q, pexp, qexp, a.sh.H,
                                                     a.sh.F);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- Step 5
// One block per (batch, head, frame, 64-token tile); W_t in shared memory,
// one warp per token: o = W_t q', RMSNorm over d, times rms_w and the gate.
template <typename T, int D>
__global__ void __launch_bounds__(256) k_readout_simt(const float* __restrict__ qf, const T* __restrict__ gate,
                                                      const float* __restrict__ rms_w, const float* __restrict__ W,
                                                      const int* __restrict__ wexp, T* __restrict__ out, int H, int F,
                                                      int S) {
  constexpr int LD = D + 1;
  constexpr int PER = (D + 31) / 32;
  constexpr int TT = 64;
  extern __shared__ float sm[];
  float* Ws = sm;
  float* qs = sm + D * LD;   // [8][D]
  long long fi = blockIdx.x;
  int f = (int)(fi % F);
  long long bh = fi / F;
  int h = (int)(bh % H);
  long long b = bh / H;
  long long N = (long long)F * S;
  const float* Wt = W + fi * D * D;
  const float eps = ldexpf(kRmsEps, -2 * wexp[fi]);   // W_t is stored as 2^-e W_t
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) Ws[(e / D) * LD + (e % D)] = Wt[e];
  __syncthreads();
  int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* qrow = qs + warp * D;
  int s_end = min(S, (int)(blockIdx.y + 1) * TT);
  for (int s = blockIdx.y * TT + warp; s < s_end; s += 8) {
    long long n = (long long)f * S + s;
    long long base = ((b * N + n) * H + h) * D;
    for (int c = lane; c < D; c += 32) qrow[c] = qf[base + c];
    __syncwarp();
    float o[PER];
    float ss = 0.f;
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      int i = lane + 32 * r;
      float acc = 0.f;
      if (i < D) {
        for (int j = 0; j < D; ++j) acc = fmaf(Ws[i * LD + j], qrow[j], acc);
      }
      o[r] = acc;
      ss += acc * acc;
    }
    ss = warp_sum(ss);
    float inv = rsqrtf(ss / D + eps);
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      int i = lane + 32 * r;
      if (i < D) out[base + i] = from_f32<T>(o[r] * inv * rms_w[i] * to_f32(gate[base + i]));
    }
    __syncwarp();
  }
}

cudaError_t launch_readout_simt(const Args& a, const float* qf, const float* W, const int* wexp) {
  dim3 grid((unsigned)a.NF(), (unsigned)((a.sh.S + 63) / 64));
  int d = a.sh.d;
  size_t smem = ((size_t)d * (d + 1) + 8 * d) * sizeof(float);
  auto go = [&](auto kern, auto tag) {
    using T = decltype(tag);
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, 256, smem, a.stream>>>(qf, (const T*)a.gate, a.rms_w, W, wexp, (T*)a.out, a.sh.H, a.sh.F, a.sh.S);
  };
  if (a.sh.dtype == VDN_DTYPE_BF16) {
    if (d == 16) go(k_readout_simt<__nv_bfloat16, 16>, __nv_bfloat16());
    else go(k_readout_simt<__nv_bfloat16, 128>, __nv_bfloat16());
  } else {
    if (d == 16) go(k_readout_simt<float, 16>, float());
    else go(k_readout_simt<float, 128>, float());
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- standalone Step 1, bf16, d = 128
// A streaming kernel: it reads q, k, v once and writes q', k', v' once, so it is
// bound by HBM bandwidth.  A block of 256 threads serves one head: its 16
// half-warps each own one (batch, frame) and a run of kFpRun consecutive tokens
// of that frame, and lane c of a half-warp holds channels 8c .. 8c + 7, so every
// load and store of a token row is one coalesced 16-byte access per lane (a
// 256-byte row per half-warp).  The run is swept kFpStep tokens at a time with a
// sliding window of rows, so the conv's neighbour rows are read once (plus one
// row at each end of the run).  The head's conv taps sit in shared memory.  q and
// k are normalised with a 16-lane shuffle reduction; SiLU uses the hardware tanh
// (x sigmoid(x) = h + h tanh h, h = x/2), whose error is far below the bf16
// rounding of the outputs.
namespace {
constexpr int kFpRun = 64;    // tokens per half-warp run
constexpr int kFpStep = 2;    // tokens per step

__device__ __forceinline__ void unpack8(uint4 u, float (&x)[8]) {
  x[0] = bf16lo(u.x); x[1] = bf16hi(u.x); x[2] = bf16lo(u.y); x[3] = bf16hi(u.y);
  x[4] = bf16lo(u.z); x[5] = bf16hi(u.z); x[6] = bf16lo(u.w); x[7] = bf16hi(u.w);
}
__device__ __forceinline__ uint4 pack8(const float (&x)[8], float s) {
  return make_uint4(pack_bf16x2(x[0] * s, x[1] * s), pack_bf16x2(x[2] * s, x[3] * s), pack_bf16x2(x[4] * s, x[5] * s),
                    pack_bf16x2(x[6] * s, x[7] * s));
}
__device__ __forceinline__ float silu_h(float hx) { return fmaf(hx, tanh_approx(hx), hx); }   // hx = x / 2
}  // namespace

__global__ void __launch_bounds__(256, 2) k_features128(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                                        const uint4* __restrict__ v, const float* __restrict__ wk,
                                                        const float* __restrict__ wv, int K, uint4* __restrict__ qo,
                                                        uint4* __restrict__ ko, uint4* __restrict__ vo, int F, int S,
                                                        int H, int nrun, long long runs) {
  __shared__ __align__(16) float taps[2][3][128];   // [k|v][tap][channel] / 2
  const int h = blockIdx.y;
  for (int e = threadIdx.x; e < 2 * 3 * 128; e += blockDim.x) {
    const int ten = e / 384, j = (e / 128) % 3, ch = e % 128;
    const float* wg = ten == 0 ? wk : wv;
    const long long i = (long long)h * 128 + ch;
    const float val = wg ? (K == 3 ? wg[i * 3 + j] : (j == 1 ? wg[i] : 0.f)) : (j == 1 ? 1.f : 0.f);
    taps[ten][j][ch] = 0.5f * val;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, c = lane & 15;
  const long long g = (long long)blockIdx.x * (blockDim.x >> 4) + (threadIdx.x >> 4);   // this half-warp's run
  const bool live = g < runs;                   // a dead half-warp still joins the warp's shuffles
  const long long gg = live ? g : 0;
  const int run = (int)(gg % nrun);
  const long long bf = gg / nrun;               // b * F + f
  const int s0 = run * kFpRun, s1 = min(S, s0 + kFpRun);
  const long long row0 = bf * (long long)S;     // token row of the frame's first token
  auto at = [&](int s) { return ((row0 + s) * H + h) * 16 + c; };   // uint4 index of (token s, lane chunk)
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  auto ld = [&](const uint4* p, int s) { return (live && s >= 0 && s < S) ? __ldg(p + at(s)) : z; };
  // window: rows s - 1 .. s + kFpStep of k and v for the step starting at token s
  uint4 kw[kFpStep + 2], vw[kFpStep + 2];
  kw[0] = ld(k, s0 - 1);
  vw[0] = ld(v, s0 - 1);
  kw[1] = ld(k, s0);
  vw[1] = ld(v, s0);
  for (int s = s0; s < s1; s += kFpStep) {
    uint4 qw[kFpStep];
#pragma unroll
    for (int i = 0; i < kFpStep; ++i) {
      kw[i + 2] = s + i + 1 < s1 + 1 ? ld(k, s + 1 + i) : z;
      vw[i + 2] = s + i + 1 < s1 + 1 ? ld(v, s + 1 + i) : z;
      qw[i] = s + i < s1 ? ld(q, s + i) : z;
    }
#pragma unroll
    for (int i = 0; i < kFpStep; ++i) {
      float k0[8], k1[8], k2[8], v0[8], v1[8], v2[8], qx[8];
      unpack8(kw[i], k0); unpack8(kw[i + 1], k1); unpack8(kw[i + 2], k2);
      unpack8(vw[i], v0); unpack8(vw[i + 1], v1); unpack8(vw[i + 2], v2);
      unpack8(qw[i], qx);
      float yk[8], yv[8], yq[8];
      float ssk = 0.f, ssq = 0.f;
#pragma unroll
      for (int e = 0; e < 8; e += 4) {
        const float4 a0 = *reinterpret_cast<const float4*>(&taps[0][0][8 * c + e]);
        const float4 a1 = *reinterpret_cast<const float4*>(&taps[0][1][8 * c + e]);
        const float4 a2 = *reinterpret_cast<const float4*>(&taps[0][2][8 * c + e]);
        const float4 b0 = *reinterpret_cast<const float4*>(&taps[1][0][8 * c + e]);
        const float4 b1 = *reinterpret_cast<const float4*>(&taps[1][1][8 * c + e]);
        const float4 b2 = *reinterpret_cast<const float4*>(&taps[1][2][8 * c + e]);
        const float ta[3][4] = {{a0.x, a0.y, a0.z, a0.w}, {a1.x, a1.y, a1.z, a1.w}, {a2.x, a2.y, a2.z, a2.w}};
        const float tb[3][4] = {{b0.x, b0.y, b0.z, b0.w}, {b1.x, b1.y, b1.z, b1.w}, {b2.x, b2.y, b2.z, b2.w}};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float hk = fmaf(ta[0][u], k0[e + u], fmaf(ta[1][u], k1[e + u], ta[2][u] * k2[e + u]));
          const float hv = fmaf(tb[0][u], v0[e + u], fmaf(tb[1][u], v1[e + u], tb[2][u] * v2[e + u]));
          yk[e + u] = silu_h(hk);
          yv[e + u] = silu_h(hv);
          yq[e + u] = silu_h(0.5f * qx[e + u]);
          ssk = fmaf(yk[e + u], yk[e + u], ssk);
          ssq = fmaf(yq[e + u], yq[e + u], ssq);
        }
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) {
        ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
        ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
      }
      const int si = s + i;
      if (live && si < s1) {
        const long long o = at(si);
        ko[o] = pack8(yk, rsqrtf(ssk + kL2Eps));
        qo[o] = pack8(yq, rsqrtf(ssq + kL2Eps));
        vo[o] = pack8(yv, 1.f);
      }
    }
    // slide the window by kFpStep rows
    kw[0] = kw[kFpStep];
    vw[0] = vw[kFpStep];
    kw[1] = kw[kFpStep + 1];
    vw[1] = vw[kFpStep + 1];
  }
}

cudaError_t launch_feature_prep(const vdn_shape& sh, const void* q, const void* k, const void* v,
                                const float* wk, const float* wv, void* qo, void* ko, void* vo,
                                cudaStream_t st) {
  if (sh.dtype == VDN_DTYPE_BF16 && sh.d == 128) {
    const int nrun = (sh.S + kFpRun - 1) / kFpRun;
    const long long runs = (long long)sh.B * sh.F * nrun;   // per head
    const dim3 grid((unsigned)((runs + 15) / 16), (unsigned)sh.H);
    const int K = (wk || wv) ? sh.conv_width : 1;
    k_features128<<<grid, 256, 0, st>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, wk, wv, K, (uint4*)qo,
                                        (uint4*)ko, (uint4*)vo, sh.F, sh.S, sh.H, nrun, runs);
    return cudaGetLastError();
  }
  if (sh.dtype == VDN_DTYPE_BF16)
    return features_dispatch<__nv_bfloat16, __nv_bfloat16>(sh, q, k, v, wk, wv, qo, ko, vo, st);
  return features_dispatch<float, float>(sh, q, k, v, wk, wv, qo, ko, vo, st);
}

// ---------------------------------------------------------------- debug copies
__global__ void k_copy(const float* __restrict__ s, float* __restrict__ d, const int* __restrict__ expo,
                       long long per_frame, long long n) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    d[i] = expo ? ldexpf(s[i], expo[i / per_frame]) : s[i];
}

cudaError_t launch_copy_frames(const Args& a, const float* src, float* dst, const int* expo) {
  long long per = (long long)a.sh.d * a.sh.d;
  long long n = a.NF() * per;
  k_copy<<<1184, 256, 0, a.stream>>>(src, dst, expo, per, n);
  return cudaGetLastError();
}

}  // namespace vdn
