// Per-frame operator (page "Step 3") and window gather + bridge (page "Step 4").
//
// k_solve builds, for every (batch, head, frame), the matrix N_f of the generic
// step  S_f = (S_{f-1} D_f + cpre B_f) N_f + cpost B_f:
//   vdn_solve / vdn_scaled:  N_f = (I + c^2 A_f)^-1   (exact inverse, fp32)
//   sana_scaled:             N_f = I - c^2 A_f
//   additive (test rule):    N_f = I
// The inverse is done once per frame, independent of the state, so each scan
// step is a plain d x d product.  I + c^2 A is symmetric positive definite
// (A = sum beta k k^T with beta > 0), so Gauss-Jordan elimination without
// pivoting is stable here: every pivot is a Schur complement of an SPD matrix.
#include "common.cuh"
#include "image.cuh"
#include "internal.h"

namespace vdn {

// Stream-K split of the statistics kernel (tensor-core path): CTA i of G owns
// statistics blocks [floor(i T / G), floor((i+1) T / G)).
__host__ __device__ __forceinline__ long long sk_begin(long long i, long long T, long long G) { return (i * T) / G; }
// The CTA whose range holds block x: the largest i with sk_begin(i) <= x.
__host__ __device__ __forceinline__ int sk_owner(long long x, long long T, long long G) {
  return (int)(((x + 1) * G + T - 1) / T) - 1;
}

template <int D>
__global__ void __launch_bounds__(256) k_solve(const float* __restrict__ A, const float* __restrict__ part,
                                               long long Tblocks, int nb, int G, RuleCoef rc,
                                               float* __restrict__ Nm, uint16_t* __restrict__ nimg,
                                               float* __restrict__ Bsum, float* __restrict__ Aout, int H, int F) {
  constexpr int R = D / 16;
  constexpr int LD = D + 1;
  extern __shared__ float sm[];
  float* stage = sm;             // [D][LD]
  float* colv = sm + D * LD;     // [2][D]
  float* rowv = colv + 2 * D;    // [2][D]
  long long fi = blockIdx.x;     // (b * H + h) * F + f
  int f = (int)(fi % F);
  long long bh = fi / F;
  int h = (int)(bh % H);
  long long b = bh / H;
  int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float a[R][R];

  if (part == nullptr) {
    const float* Af = A + fi * D * D;
#pragma unroll
    for (int ia = 0; ia < R; ++ia)
#pragma unroll
      for (int ib = 0; ib < R; ++ib) a[ia][ib] = Af[(ty + 16 * ia) * D + tx + 16 * ib];
  } else {
    // Sum the partial [A | B^T] rows written by the statistics CTAs that
    // covered this frame (frames are processed in (b, f, h) order there).
    long long pf = ((long long)b * F + f) * H + h;
    long long x0 = pf * nb, x1 = x0 + nb - 1;
    int i0 = sk_owner(x0, Tblocks, G), i1 = sk_owner(x1, Tblocks, G);
#pragma unroll
    for (int ia = 0; ia < R; ++ia)
#pragma unroll
      for (int ib = 0; ib < R; ++ib) a[ia][ib] = 0.f;
    for (int e = tid; e < D * D; e += 256) stage[(e / D) * LD + (e % D)] = 0.f;
    for (int ci = i0; ci <= i1; ++ci) {
      const float* p = part + (long long)(ci + pf) * (D * 2 * D);
#pragma unroll
      for (int ia = 0; ia < R; ++ia)
#pragma unroll
        for (int ib = 0; ib < R; ++ib) a[ia][ib] += p[(ty + 16 * ia) * (2 * D) + tx + 16 * ib];
      for (int e = tid; e < D * D; e += 256) stage[(e / D) * LD + (e % D)] += p[(e / D) * (2 * D) + D + (e % D)];
    }
    __syncthreads();
    float* Bf = Bsum + fi * D * D;   // B[i][j] = (B^T)[j][i]
    for (int e = tid; e < D * D; e += 256) Bf[e] = stage[(e % D) * LD + (e / D)];
    if (Aout) {
#pragma unroll
      for (int ia = 0; ia < R; ++ia)
#pragma unroll
        for (int ib = 0; ib < R; ++ib) Aout[fi * D * D + (ty + 16 * ia) * D + tx + 16 * ib] = a[ia][ib];
    }
    __syncthreads();
  }

#pragma unroll
  for (int ia = 0; ia < R; ++ia)
#pragma unroll
    for (int ib = 0; ib < R; ++ib) {
      float diag = (ty + 16 * ia == tx + 16 * ib) ? 1.f : 0.f;
      float x = a[ia][ib];
      a[ia][ib] = rc.identity ? diag : (rc.solve ? fmaf(rc.c2, x, diag) : fmaf(-rc.c2, x, diag));
    }

  if (rc.solve) {
    // In-place Gauss-Jordan inversion; one barrier per pivot (double-buffered
    // pivot row / column vectors).
#pragma unroll
    for (int jb = 0; jb < R; ++jb) {
      for (int jt = 0; jt < 16; ++jt) {
        int j = 16 * jb + jt;
        float* cv = colv + (j & 1) * D;
        float* rv = rowv + (j & 1) * D;
        if (tx == jt) {
#pragma unroll
          for (int ia = 0; ia < R; ++ia) cv[ty + 16 * ia] = a[ia][jb];
        }
        if (ty == jt) {
#pragma unroll
          for (int ib = 0; ib < R; ++ib) rv[tx + 16 * ib] = a[jb][ib];
        }
        __syncthreads();
        float r = 1.0f / cv[j];
        float cr[R], rk[R];
#pragma unroll
        for (int ia = 0; ia < R; ++ia) cr[ia] = cv[ty + 16 * ia] * r;
#pragma unroll
        for (int ib = 0; ib < R; ++ib) rk[ib] = rv[tx + 16 * ib];
#pragma unroll
        for (int ia = 0; ia < R; ++ia)
#pragma unroll
          for (int ib = 0; ib < R; ++ib) a[ia][ib] = fmaf(-cr[ia], rk[ib], a[ia][ib]);
        if (ty == jt) {
#pragma unroll
          for (int ib = 0; ib < R; ++ib) a[jb][ib] = rk[ib] * r;
        }
        if (tx == jt) {
#pragma unroll
          for (int ia = 0; ia < R; ++ia) a[ia][jb] = -cr[ia];
        }
        if (ty == jt && tx == jt) a[jb][jb] = r;
      }
    }
  }

  if (Nm) {
#pragma unroll
    for (int ia = 0; ia < R; ++ia)
#pragma unroll
      for (int ib = 0; ib < R; ++ib) Nm[fi * D * D + (ty + 16 * ia) * D + tx + 16 * ib] = a[ia][ib];
  }
  if constexpr (D == 128) {
    if (nimg) {
#pragma unroll
      for (int ia = 0; ia < R; ++ia)
#pragma unroll
        for (int ib = 0; ib < R; ++ib) stage[(ty + 16 * ia) * LD + tx + 16 * ib] = a[ia][ib];
      __syncthreads();
      // B operand of the scan: element (n, k) = N_f[k][n]
      write_image128(stage, LD, true, nimg + fi * (kImgBytes / 2));
    }
  }
}

cudaError_t launch_solve(const Args& a, const float* A, float* Nm, uint16_t* nimg, const float* partials,
                         float* Bsum, float* Aout) {
  RuleCoef rc = rule_coef(a.rule, a.c);
  int d = a.sh.d;
  size_t smem = ((size_t)d * (d + 1) + 4 * d) * sizeof(float);
  int nb = (a.sh.S + kStatsTokens - 1) / kStatsTokens;
  long long T = a.NF() * nb;
  int G = (int)(T < kStatsGrid ? T : kStatsGrid);
  if (d == 16) {
    k_solve<16><<<(unsigned)a.NF(), 256, smem, a.stream>>>(A, partials, T, nb, G, rc, Nm, nimg, Bsum, Aout,
                                                           a.sh.H, a.sh.F);
  } else {
    cudaFuncSetAttribute(k_solve<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_solve<128><<<(unsigned)a.NF(), 256, smem, a.stream>>>(A, partials, T, nb, G, rc, Nm, nimg, Bsum, Aout,
                                                            a.sh.H, a.sh.F);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- gather + bridge
// Query frame t with window [lo, hi]:
//   W_t = P_{lo-1} diag(prod_{g=lo..t} alpha_g) + Q_{hi+1} diag(prod_{g=t..hi} alpha_g),
// where P_{-1} = Q_F = 0.5 * text_state (zero without one).
// States carry block exponents (true state = 2^e X); the two sides are brought
// to the larger exponent, the sum is scaled by the power of two that puts its
// largest entry in [0.5, 1), and W_t is stored as 2^-e_w W_t with e_w in wexp.
// Power-of-two scaling is exact, so for states that never needed rescaling the
// stored W_t differs from the plain sum only in its exponent; the read-out never
// sees entries that could overflow its sum of squares.
template <int D>
__global__ void __launch_bounds__(256) k_gather(const float* __restrict__ P, const float* __restrict__ Q,
                                                const int* __restrict__ pexp, const int* __restrict__ qexp,
                                                const float* __restrict__ alpha, const float* __restrict__ text,
                                                int H, int F, int chunk, int radius, float* __restrict__ W,
                                                uint16_t* __restrict__ wimg, int* __restrict__ wexp) {
  constexpr int LD = D + 1;
  extern __shared__ float sm[];
  float* dpre = sm;
  float* dsuf = sm + D;
  float* stage = sm + 2 * D;
  long long fi = blockIdx.x;
  int t = (int)(fi % F);
  long long bh = fi / F;
  int h = (int)(bh % H);
  long long b = bh / H;
  int lo, hi;
  window_bounds(t, F, chunk, radius, lo, hi);
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float dp = 1.f, ds = 1.f;
    for (int g = lo; g <= t; ++g) dp *= alpha[((b * F + g) * H + h) * D + c];
    for (int g = t; g <= hi; ++g) ds *= alpha[((b * F + g) * H + h) * D + c];
    dpre[c] = dp;
    dsuf[c] = ds;
  }
  __syncthreads();
  const float* pre = lo > 0 ? P + (bh * F + (lo - 1)) * D * D : nullptr;
  const float* suf = hi < F - 1 ? Q + (bh * F + (hi + 1)) * D * D : nullptr;
  const float* seed = text ? text + (long long)h * D * D : nullptr;
  const int ep = pre ? pexp[bh * F + (lo - 1)] : 0;
  const int eq = suf ? qexp[bh * F + (hi + 1)] : 0;
  const int ew = ep > eq ? ep : eq;
  const float sp = ldexpf(1.f, ep - ew), sq = ldexpf(1.f, eq - ew);
  constexpr int PER = D * D / 256;     // blockDim.x == 256
  float wv[PER];
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    const int e = threadIdx.x + 256 * r, k = e % D;
    float pv = pre ? pre[e] : (seed ? kTextStateScale * seed[e] : 0.f);
    float sv = suf ? suf[e] : (seed ? kTextStateScale * seed[e] : 0.f);
    wv[r] = fmaf(pv * sp, dpre[k], sv * sq * dsuf[k]);
    amax = fmaxf(amax, fabsf(wv[r]));
  }
  float* red = stage + (D == 128 && wimg ? D * LD : 0);   // 8 floats after the staging tile
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w8 = 1; w8 < 8; ++w8) amax = fmaxf(amax, red[w8]);
  int ek = 0;
  if (amax > 0.f) frexpf(amax, &ek);
  if (threadIdx.x == 0) wexp[fi] = ew + ek;
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    const int e = threadIdx.x + 256 * r, i = e / D, k = e % D;
    const float w = ldexpf(wv[r], -ek);
    if (W) W[fi * D * D + e] = w;
    if (D == 128 && wimg) stage[i * LD + k] = w;
  }
  if constexpr (D == 128) {
    if (wimg) {
      __syncthreads();
      // B operand of the read-out: element (n, k) = W_t[n][k]
      write_image128(stage, LD, false, wimg + fi * (kImgBytes / 2));
    }
  }
}

cudaError_t launch_gather(const Args& a, const float* P, const float* Q, const int* pexp, const int* qexp, float* W,
                          uint16_t* wimg, int* wexp) {
  int d = a.sh.d;
  size_t smem = (2 * (size_t)d + (wimg ? (size_t)d * (d + 1) : 0) + 8) * sizeof(float);
  if (d == 16) {
    k_gather<16><<<(unsigned)a.NF(), 256, smem, a.stream>>>(P, Q, pexp, qexp, a.alpha, a.text_state, a.sh.H, a.sh.F,
                                                            a.chunk, a.radius, W, nullptr, wexp);
  } else {
    cudaFuncSetAttribute(k_gather<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k_gather<128><<<(unsigned)a.NF(), 256, smem, a.stream>>>(P, Q, pexp, qexp, a.alpha, a.text_state, a.sh.H,
                                                             a.sh.F, a.chunk, a.radius, W, wimg, wexp);
  }
  return cudaGetLastError();
}

}  // namespace vdn
