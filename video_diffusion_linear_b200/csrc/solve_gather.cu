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
    // Sum the partial slots ([A; B], 256 rows of 128) written by the statistics
    // CTAs that covered this frame (frames are processed in (b, f, h) order there).
    long long pf = ((long long)b * F + f) * H + h;
    long long x0 = pf * nb, x1 = x0 + nb - 1;
    int i0 = sk_owner(x0, Tblocks, G), i1 = sk_owner(x1, Tblocks, G);
#pragma unroll
    for (int ia = 0; ia < R; ++ia)
#pragma unroll
      for (int ib = 0; ib < R; ++ib) a[ia][ib] = 0.f;
    for (int e = tid; e < D * D; e += 256) stage[(e / D) * LD + (e % D)] = 0.f;
    for (int ci = i0; ci <= i1; ++ci) {
      const float* p = part + (long long)(ci + pf) * (2 * D * D);
#pragma unroll
      for (int ia = 0; ia < R; ++ia)
#pragma unroll
        for (int ib = 0; ib < R; ++ib) a[ia][ib] += p[(ty + 16 * ia) * D + tx + 16 * ib];
      // B rows of the slot: float4 loads, all issued before use
      constexpr int NV4 = D * D / 4, NV = (NV4 + 255) / 256;
      float4 bv[NV];
#pragma unroll
      for (int r = 0; r < NV; ++r) {
        const int e4 = tid + 256 * r, row = e4 / (D / 4), c4 = e4 % (D / 4);
        if (e4 < NV4) bv[r] = *reinterpret_cast<const float4*>(p + D * D + row * D + 4 * c4);
      }
#pragma unroll
      for (int r = 0; r < NV; ++r) {
        const int e4 = tid + 256 * r, row = e4 / (D / 4), c4 = e4 % (D / 4);
        if (e4 < NV4) {
          float* st = stage + row * LD + 4 * c4;
          st[0] += bv[r].x; st[1] += bv[r].y; st[2] += bv[r].z; st[3] += bv[r].w;
        }
      }
    }
    __syncthreads();
    float* Bf = Bsum + fi * D * D;
    for (int e = tid; e < D * D; e += 256) Bf[e] = stage[(e / D) * LD + (e % D)];
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

// d = 128 solve by the symmetric sweep operator.  N_f^-1 = I + c^2 A_f is
// symmetric positive definite; sweeping pivot k (d = a_kk):
//   a_ij <- a_ij - a_ik a_kj / d   (i, j != k),   a_ik, a_kj <- a_ik / d, a_kj / d,   a_kk <- -1 / d
// keeps the matrix symmetric, and sweeping every pivot in turn leaves -M^-1
// (Gauss-Jordan elimination without pivoting, with every pivot a Schur
// complement of an SPD matrix, so positive).  Symmetry halves the work: the
// 136 threads that own the upper-triangle 8x8 blocks (I <= J) of a 16 x 16 block
// grid do all of it, one pivot per barrier, with pivot row k broadcast through
// shared memory (its entries left of the diagonal block come from column k of
// the blocks above it).  Updates run on packed fp32 pairs; the pivot reciprocal
// is the hardware approximation refined by one Newton step (relative error near
// 2^-23, the same as a correctly rounded division up to one unit).  Three frames
// share an SM.  The scan's operand image and the debug copies are written from
// the blocks directly, each off-diagonal block once as itself and once
// transposed.
constexpr int kSolveThreads = 160;     // 136 block owners + 24 that only help with the sums
constexpr int kSolveBlocks = 136;      // 16 * 17 / 2

__device__ __forceinline__ void store_chunk_image(uint8_t* img, int n, int c, const float (&v)[8]) {
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    __nv_bfloat16 h0, l0, h1, l1;
    split_bf16(v[e], h0, l0);
    split_bf16(v[e + 1], h1, l1);
    hw[e / 2] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
    lw[e / 2] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
  }
  const uint32_t off = img_offset(0, n, 8 * c);
  *reinterpret_cast<uint4*>(img + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  *reinterpret_cast<uint4*>(img + 32768 + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

__global__ void __launch_bounds__(kSolveThreads, 3) k_solve128(const float* __restrict__ part, long long Tblocks,
                                                              int nb, int G, RuleCoef rc, float* __restrict__ Nm,
                                                              uint16_t* __restrict__ nimg, float* __restrict__ Bsum,
                                                              float* __restrict__ Aout, int H, int F) {
  constexpr int D = 128;
  __shared__ __align__(16) float rowv[2][D];      // pivot row, double-buffered
  const long long fi = blockIdx.x;
  const int f = (int)(fi % F);
  const long long bh = fi / F;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const int tid = threadIdx.x;
  const bool owner = tid < kSolveBlocks;
  // block (I, J), I <= J, row-major over the upper triangle
  int I = 0, J = 0;
  {
    int t = owner ? tid : 0;
    while (t >= 16 - I) { t -= 16 - I; ++I; }
    J = I + t;
  }
  const int r0 = 8 * I, c0 = 8 * J;
  float2 a[8][4];                      // a[i][p] = (A[r0+i][c0+2p], A[r0+i][c0+2p+1])

  const long long pf = ((long long)b * F + f) * H + h;
  const long long x0 = pf * nb, x1 = x0 + nb - 1;
  const int i0 = sk_owner(x0, Tblocks, G), i1 = sk_owner(x1, Tblocks, G);

  // ---- B: rows 128 .. 255 of the frame's partial slots ([A; B], 256 rows of 128),
  // summed with coalesced 16-byte accesses, eight in flight per thread and slot
  {
    constexpr int NV4 = D * D / 4;
    float4* Bf = reinterpret_cast<float4*>(Bsum + fi * D * D);
    for (int e0 = tid; e0 < NV4; e0 += 8 * kSolveThreads) {
      float4 acc[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int ci = i0; ci <= i1; ++ci) {
        const float4* src = reinterpret_cast<const float4*>(part + (long long)(ci + pf) * (2 * D * D) + D * D);
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e4 = e0 + u * kSolveThreads;
          v[u] = e4 < NV4 ? src[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          acc[u].x += v[u].x; acc[u].y += v[u].y; acc[u].z += v[u].z; acc[u].w += v[u].w;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e4 = e0 + u * kSolveThreads;
        if (e4 < NV4) Bf[e4] = acc[u];
      }
    }
  }

  // ---- A: sum this block of the A rows (0 .. 127) of the frame's partial slots
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int p = 0; p < 4; ++p) a[i][p] = make_float2(0.f, 0.f);
  if (owner) {
    for (int ci = i0; ci <= i1; ++ci) {
      const float* pp = part + (long long)(ci + pf) * (2 * D * D) + r0 * D + c0;
#pragma unroll
      for (int ih = 0; ih < 8; ih += 4) {   // four rows (8 float4) in flight
        float4 v[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[i][0] = *reinterpret_cast<const float4*>(pp + (ih + i) * D);
          v[i][1] = *reinterpret_cast<const float4*>(pp + (ih + i) * D + 4);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[ih + i][0] = __fadd2_rn(a[ih + i][0], make_float2(v[i][0].x, v[i][0].y));
          a[ih + i][1] = __fadd2_rn(a[ih + i][1], make_float2(v[i][0].z, v[i][0].w));
          a[ih + i][2] = __fadd2_rn(a[ih + i][2], make_float2(v[i][1].x, v[i][1].y));
          a[ih + i][3] = __fadd2_rn(a[ih + i][3], make_float2(v[i][1].z, v[i][1].w));
        }
      }
    }
    if (Aout) {
      float* Af = Aout + fi * D * D;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        *reinterpret_cast<float4*>(Af + (r0 + i) * D + c0) = make_float4(a[i][0].x, a[i][0].y, a[i][1].x, a[i][1].y);
        *reinterpret_cast<float4*>(Af + (r0 + i) * D + c0 + 4) = make_float4(a[i][2].x, a[i][2].y, a[i][3].x, a[i][3].y);
      }
      if (I != J) {   // the mirror block
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          float cvv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) cvv[i] = (m & 1) ? a[i][m >> 1].y : a[i][m >> 1].x;
          *reinterpret_cast<float4*>(Af + (c0 + m) * D + r0) = make_float4(cvv[0], cvv[1], cvv[2], cvv[3]);
          *reinterpret_cast<float4*>(Af + (c0 + m) * D + r0 + 4) = make_float4(cvv[4], cvv[5], cvv[6], cvv[7]);
        }
      }
    }
  }

  // ---- N^-1 = I + c^2 A (solve rules); N = I - c^2 A (sana) or I (additive)
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float d0 = (r0 + i == c0 + 2 * p) ? 1.f : 0.f, d1 = (r0 + i == c0 + 2 * p + 1) ? 1.f : 0.f;
      const float s = rc.solve ? rc.c2 : -rc.c2;
      a[i][p] = rc.identity ? make_float2(d0, d1) : make_float2(fmaf(s, a[i][p].x, d0), fmaf(s, a[i][p].y, d1));
    }

  float sign = 1.f;
  if (rc.solve) {
    sign = -1.f;                       // the sweep leaves -N
    for (int K = 0; K < 16; ++K) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int k = 8 * K + kk;
        float* rv = rowv[kk & 1];
        if (owner && I == K) {         // row kk of the blocks right of (and at) the diagonal
          *reinterpret_cast<float4*>(rv + c0) = make_float4(a[kk][0].x, a[kk][0].y, a[kk][1].x, a[kk][1].y);
          *reinterpret_cast<float4*>(rv + c0 + 4) = make_float4(a[kk][2].x, a[kk][2].y, a[kk][3].x, a[kk][3].y);
        } else if (owner && J == K) {  // column kk of the blocks above the diagonal (a_ik = a_ki)
          float cvv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) cvv[i] = (kk & 1) ? a[i][kk >> 1].y : a[i][kk >> 1].x;
          *reinterpret_cast<float4*>(rv + r0) = make_float4(cvv[0], cvv[1], cvv[2], cvv[3]);
          *reinterpret_cast<float4*>(rv + r0 + 4) = make_float4(cvv[4], cvv[5], cvv[6], cvv[7]);
        }
        __syncthreads();
        if (owner) {
          const float pv = rv[k];
          float r;
          asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(pv));
          r = r * fmaf(-pv, r, 2.0f);                   // one Newton step
          const float4 ra = *reinterpret_cast<const float4*>(rv + r0);
          const float4 rb = *reinterpret_cast<const float4*>(rv + r0 + 4);
          const float4 ca = *reinterpret_cast<const float4*>(rv + c0);
          const float4 cb = *reinterpret_cast<const float4*>(rv + c0 + 4);
          const float cr[8] = {ra.x * r, ra.y * r, ra.z * r, ra.w * r, rb.x * r, rb.y * r, rb.z * r, rb.w * r};
          const float2 rk[4] = {make_float2(ca.x, ca.y), make_float2(ca.z, ca.w), make_float2(cb.x, cb.y),
                                make_float2(cb.z, cb.w)};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 m = make_float2(-cr[i], -cr[i]);
#pragma unroll
            for (int p = 0; p < 4; ++p) a[i][p] = __ffma2_rn(m, rk[p], a[i][p]);
          }
          if (I == K) {                // row k: a_kj / d
#pragma unroll
            for (int p = 0; p < 4; ++p) a[kk][p] = make_float2(rk[p].x * r, rk[p].y * r);
          }
          if (J == K) {                // column k: a_ik / d
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (kk & 1) a[i][kk >> 1].y = cr[i];
              else a[i][kk >> 1].x = cr[i];
            }
          }
          if (I == K && J == K) {
            if (kk & 1) a[kk][kk >> 1].y = -r;
            else a[kk][kk >> 1].x = -r;
          }
        }
      }
    }
  }

  if (owner) {
    uint8_t* img = nimg ? reinterpret_cast<uint8_t*>(nimg + fi * (kImgBytes / 2)) : nullptr;
    float* Nf = Nm ? Nm + fi * D * D : nullptr;
    // B operand image of the scan: row n holds N_f[n][k] (N_f symmetric)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v[8] = {sign * a[i][0].x, sign * a[i][0].y, sign * a[i][1].x, sign * a[i][1].y,
                          sign * a[i][2].x, sign * a[i][2].y, sign * a[i][3].x, sign * a[i][3].y};
      if (img) store_chunk_image(img, r0 + i, J, v);
      if (Nf) {
        *reinterpret_cast<float4*>(Nf + (r0 + i) * D + c0) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(Nf + (r0 + i) * D + c0 + 4) = make_float4(v[4], v[5], v[6], v[7]);
      }
    }
    if (I != J) {
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = sign * ((m & 1) ? a[i][m >> 1].y : a[i][m >> 1].x);
        if (img) store_chunk_image(img, c0 + m, I, v);
        if (Nf) {
          *reinterpret_cast<float4*>(Nf + (c0 + m) * D + r0) = make_float4(v[0], v[1], v[2], v[3]);
          *reinterpret_cast<float4*>(Nf + (c0 + m) * D + r0 + 4) = make_float4(v[4], v[5], v[6], v[7]);
        }
      }
    }
  }
}

cudaError_t launch_solve(const Args& a, const float* A, float* Nm, uint16_t* nimg, const float* partials,
                         float* Bsum, float* Aout) {
  if (a.sh.d == 128 && partials) {
    RuleCoef rc = rule_coef(a.rule, a.c);
    int nb = (a.sh.S + kStatsTokens - 1) / kStatsTokens;
    long long T = a.NF() * nb;
    int G = (int)(T < kStatsGrid ? T : kStatsGrid);
    k_solve128<<<(unsigned)a.NF(), kSolveThreads, 0, a.stream>>>(partials, T, nb, G, rc, Nm, nimg, Bsum, Aout, a.sh.H,
                                                          a.sh.F);
    return cudaGetLastError();
  }
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

// d = 128: 512 threads, four per row of W_t (32 columns each).  The state rows
// are loaded first (float4), the decay vectors meanwhile by one thread per
// channel, then each thread writes its part of the bf16 hi/lo operand image
// directly (four 16-byte chunks per part, 128-byte swizzle).
__global__ void __launch_bounds__(512) k_gather128(const float* __restrict__ P, const float* __restrict__ Q,
                                                   const int* __restrict__ pexp, const int* __restrict__ qexp,
                                                   const float* __restrict__ alpha, const float* __restrict__ text,
                                                   int H, int F, int chunk, int radius, float* __restrict__ W,
                                                   uint16_t* __restrict__ wimg, int* __restrict__ wexp,
                                                   int* __restrict__ wbexp) {
  constexpr int D = 128;
  __shared__ float dpre[D], dsuf[D], red[16];
  const int tid = threadIdx.x, n = tid >> 2, k0 = (tid & 3) * 32;
  const long long fi = blockIdx.x;
  const int t = (int)(fi % F);
  const long long bh = fi / F;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  int lo, hi;
  window_bounds(t, F, chunk, radius, lo, hi);
  const float* pre = lo > 0 ? P + (bh * F + (lo - 1)) * D * D : nullptr;
  const float* suf = hi < F - 1 ? Q + (bh * F + (hi + 1)) * D * D : nullptr;
  const float* seed = text ? text + (long long)h * D * D : nullptr;
  float4 pv[8], sv[8];
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int off = n * D + k0 + 4 * j;
    pv[j] = pre ? *reinterpret_cast<const float4*>(pre + off) : (seed ? *reinterpret_cast<const float4*>(seed + off) : z);
    sv[j] = suf ? *reinterpret_cast<const float4*>(suf + off) : (seed ? *reinterpret_cast<const float4*>(seed + off) : z);
  }
  if (tid < D) {
    float dp = 1.f, ds = 1.f;
    const float* al = alpha + (b * F * H + h) * D + tid;   // alpha[b][g][h][c] = al[g * H * D]
    for (int g0 = lo; g0 <= hi; g0 += 8) {
      float av[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) av[u] = (g0 + u <= hi) ? al[(long long)(g0 + u) * H * D] : 1.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int g = g0 + u;
        if (g <= t) dp *= av[u];
        if (g >= t) ds *= av[u];
      }
    }
    dpre[tid] = dp;
    dsuf[tid] = ds;
  }
  const int ep = pre ? pexp[bh * F + (lo - 1)] : 0;
  const int eq = suf ? qexp[bh * F + (hi + 1)] : 0;
  const int ew = ep > eq ? ep : eq;
  const float sp = (pre ? 1.f : (seed ? kTextStateScale : 0.f)) * ldexpf(1.f, ep - ew);
  const float sq = (suf ? 1.f : (seed ? kTextStateScale : 0.f)) * ldexpf(1.f, eq - ew);
  __syncthreads();
  float w[32];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int k = k0 + 4 * j;
    w[4 * j + 0] = fmaf(pv[j].x * sp, dpre[k + 0], sv[j].x * sq * dsuf[k + 0]);
    w[4 * j + 1] = fmaf(pv[j].y * sp, dpre[k + 1], sv[j].y * sq * dsuf[k + 1]);
    w[4 * j + 2] = fmaf(pv[j].z * sp, dpre[k + 2], sv[j].z * sq * dsuf[k + 2]);
    w[4 * j + 3] = fmaf(pv[j].w * sp, dpre[k + 3], sv[j].w * sq * dsuf[k + 3]);
#pragma unroll
    for (int u = 0; u < 4; ++u) amax = fmaxf(amax, fabsf(w[4 * j + u]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int u = 1; u < 16; ++u) amax = fmaxf(amax, red[u]);
  int ek = 0;
  if (amax > 0.f) frexpf(amax, &ek);
  if (tid == 0) wexp[fi] = ew + ek;
#pragma unroll
  for (int u = 0; u < 32; ++u) w[u] = ldexpf(w[u], -ek);
  if (W) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(W + fi * D * D + n * D + k0 + 4 * j) =
          make_float4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
  if (wimg) {   // fp16 image; W is already normalised as a whole, so every row block has exponent 0
    uint8_t* img = reinterpret_cast<uint8_t*>(wimg) + fi * kWImgBytes;
#pragma unroll
    for (int cch = 0; cch < 4; ++cch) store_chunk_f16(img, n, k0 + 8 * cch, &w[8 * cch]);
    if (tid < kWRowBlocks) wbexp[fi * kWRowBlocks + tid] = 0;
  }
}

// d = 128: one CTA per (batch, head, window chunk, block of 32 rows).  Every
// query frame of a chunk has the same window [lo, hi], hence the same two
// boundary states; their rows are read once and each frame's W_t differs only
// in its two decay vectors.  The sides are aligned to the larger block exponent
// (stored states are below 2^48, see the scans' block exponent), W_t is stored as 2^-e W_t.
// Frame sharding: the query frames are fq0 .. fq0 + Fq - 1 of an F-frame clip
// (fq0 a multiple of chunk), P, Q, their exponents and alpha cover the whole
// clip, and W_t is written at the query frame's local index t - fq0.
constexpr int kGatherRows = 32;
static_assert(kWBlockRows == kGatherRows, "one gather CTA per row block of the W image");

__global__ void __launch_bounds__(128) k_gather128_chunk(const float* __restrict__ P, const float* __restrict__ Q,
                                                         const int* __restrict__ pexp, const int* __restrict__ qexp,
                                                         const float* __restrict__ alpha,
                                                         const float* __restrict__ text, int H, int F, int chunk,
                                                         int radius, int fq0, int Fq, float* __restrict__ W,
                                                         uint16_t* __restrict__ wimg, int* __restrict__ wexp,
                                                         int* __restrict__ wbexp) {
  constexpr int D = 128;
  __shared__ float dpre[kGatherMaxChunk][D], dsuf[kGatherMaxChunk][D];
  __shared__ float red[2][4];
  const int tid = threadIdx.x, n = blockIdx.z * kGatherRows + (tid >> 2), k0 = (tid & 3) * 32;
  const long long bh = blockIdx.x;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const int t0 = fq0 + blockIdx.y * chunk, t1 = min(fq0 + Fq, t0 + chunk);   // query frames of this chunk
  int lo, hi;
  window_bounds(t0, F, chunk, radius, lo, hi);
  const float* pre = lo > 0 ? P + (bh * F + (lo - 1)) * D * D : nullptr;
  const float* suf = hi < F - 1 ? Q + (bh * F + (hi + 1)) * D * D : nullptr;
  const float* seed = text ? text + (long long)h * D * D : nullptr;
  float4 pv[8], sv[8];
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int off = n * D + k0 + 4 * j;
    pv[j] = pre ? *reinterpret_cast<const float4*>(pre + off) : (seed ? *reinterpret_cast<const float4*>(seed + off) : z);
    sv[j] = suf ? *reinterpret_cast<const float4*>(suf + off) : (seed ? *reinterpret_cast<const float4*>(seed + off) : z);
  }
  {
    // dpre[t] = prod_{g=lo..t} alpha_g,  dsuf[t] = prod_{g=t..hi} alpha_g  (one channel per thread)
    const float* al = alpha + (b * F * H + h) * D + tid;
    float dp = 1.f;
    for (int g = lo; g < t0; ++g) dp *= al[(long long)g * H * D];
    for (int t = t0; t < t1; ++t) {
      dp *= al[(long long)t * H * D];
      dpre[t - t0][tid] = dp;
    }
    float ds = 1.f;
    for (int g = hi; g >= t1; --g) ds *= al[(long long)g * H * D];
    for (int t = t1 - 1; t >= t0; --t) {
      ds *= al[(long long)t * H * D];
      dsuf[t - t0][tid] = ds;
    }
  }
  const int ep = pre ? pexp[bh * F + (lo - 1)] : 0;
  const int eq = suf ? qexp[bh * F + (hi + 1)] : 0;
  const int ew = ep > eq ? ep : eq;
  const float sp = (pre ? 1.f : (seed ? kTextStateScale : 0.f)) * ldexpf(1.f, ep - ew);
  const float sq = (suf ? 1.f : (seed ? kTextStateScale : 0.f)) * ldexpf(1.f, eq - ew);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    pv[j].x *= sp; pv[j].y *= sp; pv[j].z *= sp; pv[j].w *= sp;
    sv[j].x *= sq; sv[j].y *= sq; sv[j].z *= sq; sv[j].w *= sq;
  }
  __syncthreads();
  for (int t = t0; t < t1; ++t) {
    const float* dp = dpre[t - t0];
    const float* ds = dsuf[t - t0];
    const long long fi = bh * Fq + (t - fq0);
    if (tid == 0 && blockIdx.z == 0) wexp[fi] = ew;
    float w[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int k = k0 + 4 * j;
      const float4 a = *reinterpret_cast<const float4*>(dp + k);
      const float4 c = *reinterpret_cast<const float4*>(ds + k);
      w[4 * j + 0] = fmaf(pv[j].x, a.x, sv[j].x * c.x);
      w[4 * j + 1] = fmaf(pv[j].y, a.y, sv[j].y * c.y);
      w[4 * j + 2] = fmaf(pv[j].z, a.z, sv[j].z * c.z);
      w[4 * j + 3] = fmaf(pv[j].w, a.w, sv[j].w * c.w);
    }
    if (W) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(W + fi * D * D + n * D + k0 + 4 * j) =
            make_float4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    }
    if (wimg) {
      // this CTA's 32 rows form one row block of the fp16 image: scale it by the
      // power of two that puts its largest entry in [0.5, 1)
      float amax = 0.f;
#pragma unroll
      for (int u = 0; u < 32; ++u) amax = fmaxf(amax, fabsf(w[u]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      float* rb = red[(t - t0) & 1];   // double-buffered: one barrier per frame
      if ((tid & 31) == 0) rb[tid >> 5] = amax;
      __syncthreads();
      amax = fmaxf(fmaxf(rb[0], rb[1]), fmaxf(rb[2], rb[3]));
      int eb = 0;
      if (amax > 0.f) frexpf(amax, &eb);
      eb = min(max(eb, -125), 126);    // 2^-eb stays a normal float
      if (tid == 0) wbexp[fi * kWRowBlocks + blockIdx.z] = eb;
      const float sc = pow2f(-eb);
      uint8_t* img = reinterpret_cast<uint8_t*>(wimg) + fi * kWImgBytes;
#pragma unroll
      for (int cch = 0; cch < 4; ++cch) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = w[8 * cch + e] * sc;
        store_chunk_f16(img, n, k0 + 8 * cch, v);
      }
    }
  }
}

cudaError_t launch_gather_frames(const Args& a, int fq0, int Fq, const float* P, const float* Q, const int* pexp,
                                 const int* qexp, float* W, uint16_t* wimg, int* wexp, int* wbexp) {
  if (a.sh.d != 128 || a.chunk > kGatherMaxChunk || fq0 % a.chunk != 0 || Fq < 1 || fq0 + Fq > a.sh.F)
    return cudaErrorInvalidValue;
  dim3 grid((unsigned)((long long)a.sh.B * a.sh.H), (unsigned)((Fq + a.chunk - 1) / a.chunk), 128 / kGatherRows);
  k_gather128_chunk<<<grid, 128, 0, a.stream>>>(P, Q, pexp, qexp, a.alpha, a.text_state, a.sh.H, a.sh.F, a.chunk,
                                                 a.radius, fq0, Fq, W, wimg, wexp, wbexp);
  return cudaGetLastError();
}

cudaError_t launch_gather(const Args& a, const float* P, const float* Q, const int* pexp, const int* qexp, float* W,
                          uint16_t* wimg, int* wexp, int* wbexp) {
  if (a.sh.d == 128 && a.chunk <= kGatherMaxChunk) return launch_gather_frames(a, 0, a.sh.F, P, Q, pexp, qexp, W, wimg,
                                                                               wexp, wbexp);
  if (a.sh.d == 128) {
    k_gather128<<<(unsigned)a.NF(), 512, 0, a.stream>>>(P, Q, pexp, qexp, a.alpha, a.text_state, a.sh.H, a.sh.F,
                                                        a.chunk, a.radius, W, wimg, wexp, wbexp);
    return cudaGetLastError();
  }
  size_t smem = (2 * 16 + 8) * sizeof(float);
  k_gather<16><<<(unsigned)a.NF(), 256, smem, a.stream>>>(P, Q, pexp, qexp, a.alpha, a.text_state, a.sh.H, a.sh.F,
                                                          a.chunk, a.radius, W, nullptr, wexp);
  return cudaGetLastError();
}

}  // namespace vdn
