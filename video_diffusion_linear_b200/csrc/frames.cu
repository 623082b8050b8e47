// Frame sharding of the branch: the fold of the per-chunk affine maps (page
// sections "Step 3" and "Step 4").
//
// Each rule's frame step is affine in the state, S_out = S_in G_f + B'_f, so a
// chunk of frames composes into one map S -> S G_c + O_c per scan direction
// (the segment mode of the scan writes them).  Once every rank holds every
// chunk's maps, the chunk-edge states the window gather reads follow by folding
// the maps in scan order from the seed:
//     prefix: S <- S G_c + O_c for c = 0, 1, ..;       P at the last frame of chunk c
//     suffix: S <- S G_c + O_c for c = C-1, C-2, ..;   Q at the first frame of chunk c
// One CTA per (batch, head, direction); each step is a 128 x 128 x 128 product in
// fp32 on the CUDA cores (a handful of steps per clip).  Maps and states carry
// power-of-two block exponents (true value = 2^e x stored value), as the scans'
// states do, so rules whose frame operators grow the state (sana_scaled with
// c^2 |A| > 2) stay finite over any number of chunks.
#include "common.cuh"
#include "internal.h"

namespace vdn {

namespace {

constexpr int kFoldThreads = 256;
constexpr int kD = 128;

}  // namespace

// maps_all: [world] rank buffers of frames_map_bytes each, laid out as
//   [B*H][2 directions][nch_stride][G_c | O_c][128][128] fp32, then
//   [B*H][2 directions][nch_stride][G_c | O_c] int32 exponents.
// P, Q: [B*H][F][128][128] with exponents pexp, qexp [B*H][F]; only chunk-edge
// frames are written.
__global__ void __launch_bounds__(kFoldThreads, 1) k_fold_maps(const float* __restrict__ maps_all,
                                                               long long rank_floats, long long exp_off, int world,
                                                               int nch_stride, int nch_total, long long BH,
                                                               const float* __restrict__ text, int H, int F,
                                                               int chunk, float* __restrict__ P,
                                                               float* __restrict__ Q, int* __restrict__ pexp,
                                                               int* __restrict__ qexp) {
  extern __shared__ float4 fold_smem[];
  float* S = reinterpret_cast<float*>(fold_smem);   // state [128][128]
  float* G = S + kD * kD;                           // G_c [128][128]
  const int tid = threadIdx.x;
  const int dir = blockIdx.x & 1;
  const long long bh = blockIdx.x >> 1;
  const int h = (int)(bh % H);
  const int r0 = (tid >> 4) * 8, c0 = (tid & 15) * 8;   // this thread's 8 x 8 block of the product

  const float* T = text ? text + (long long)h * kD * kD : nullptr;
  for (int i = tid * 4; i < kD * kD; i += kFoldThreads * 4) {
    float4 v = T ? *reinterpret_cast<const float4*>(T + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    v.x *= kTextStateScale; v.y *= kTextStateScale; v.z *= kTextStateScale; v.w *= kTextStateScale;
    *reinterpret_cast<float4*>(S + i) = v;
  }
  int es = 0;   // exponent of the state
  for (int step = 0; step + 1 < nch_total; ++step) {
    const int c = dir == 0 ? step : nch_total - 1 - step;
    int r, j;
    chunk_owner(c, nch_total, world, r, j);
    const long long slot = ((bh * 2 + dir) * nch_stride + j) * 2;   // G_c; O_c is slot + 1
    const float* rank_base = maps_all + r * rank_floats;
    const float* Gc = rank_base + slot * (long long)kD * kD;
    const float* Oc = Gc + kD * kD;
    const int* ex = reinterpret_cast<const int*>(rank_base + exp_off) + slot;
    // S G_c + O_c = 2^e (sg X_S X_G + so X_O), e the larger of the two terms' exponents
    const int eg = es + ex[0], eo = ex[1];
    const int e = eg > eo ? eg : eo;
    const float sg = ldexpf(1.f, eg - e), so = ldexpf(1.f, eo - e);
    __syncthreads();   // the previous step's reads of G and writes of S are done
    for (int i = tid * 4; i < kD * kD; i += kFoldThreads * 4)
      *reinterpret_cast<float4*>(G + i) = *reinterpret_cast<const float4*>(Gc + i);
    __syncthreads();
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int bb = 0; bb < 8; ++bb) acc[a][bb] = 0.f;
#pragma unroll 4
    for (int k = 0; k < kD; ++k) {
      const float4 g0 = *reinterpret_cast<const float4*>(G + k * kD + c0);
      const float4 g1 = *reinterpret_cast<const float4*>(G + k * kD + c0 + 4);
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float sa = S[(r0 + a) * kD + k];
        acc[a][0] = fmaf(sa, g0.x, acc[a][0]); acc[a][1] = fmaf(sa, g0.y, acc[a][1]);
        acc[a][2] = fmaf(sa, g0.z, acc[a][2]); acc[a][3] = fmaf(sa, g0.w, acc[a][3]);
        acc[a][4] = fmaf(sa, g1.x, acc[a][4]); acc[a][5] = fmaf(sa, g1.y, acc[a][5]);
        acc[a][6] = fmaf(sa, g1.z, acc[a][6]); acc[a][7] = fmaf(sa, g1.w, acc[a][7]);
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const float4 o0 = *reinterpret_cast<const float4*>(Oc + (r0 + a) * kD + c0);
      const float4 o1 = *reinterpret_cast<const float4*>(Oc + (r0 + a) * kD + c0 + 4);
      const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
      for (int bb = 0; bb < 8; ++bb) {
        acc[a][bb] = fmaf(sg, acc[a][bb], so * ov[bb]);
        amax = fmaxf(amax, fabsf(acc[a][bb]));
      }
    }
    es = e;
    // every read of the old state is done; rescale as the scans do past 2^32
    if (__syncthreads_or(amax > kRenormAbove)) {
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int bb = 0; bb < 8; ++bb) acc[a][bb] *= kRenormScale;
      es += kRenormExp;
    }
    const int f = dir == 0 ? (c + 1) * chunk - 1 : c * chunk;   // in [0, F): c <= C - 2 resp. c >= 1
    float* dst = (dir == 0 ? P : Q) + (bh * F + f) * (long long)kD * kD;
    if (tid == 0) (dir == 0 ? pexp : qexp)[bh * F + f] = es;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const float4 v0 = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
      const float4 v1 = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
      *reinterpret_cast<float4*>(S + (r0 + a) * kD + c0) = v0;
      *reinterpret_cast<float4*>(S + (r0 + a) * kD + c0 + 4) = v1;
      *reinterpret_cast<float4*>(dst + (r0 + a) * kD + c0) = v0;
      *reinterpret_cast<float4*>(dst + (r0 + a) * kD + c0 + 4) = v1;
    }
  }
}

cudaError_t launch_fold_maps(const Args& a, const float* maps_all, size_t rank_bytes, size_t exp_off_bytes, int world,
                             int nch_stride, float* P, float* Q, int* pexp, int* qexp) {
  if (a.sh.d != kD || world < 1 || a.chunk < 1) return cudaErrorInvalidValue;
  const int nch_total = (a.sh.F + a.chunk - 1) / a.chunk;
  if (world > nch_total || nch_stride < (nch_total + world - 1) / world) return cudaErrorInvalidValue;
  if (rank_bytes % 16 || exp_off_bytes % 16) return cudaErrorInvalidValue;
  const long long BH = (long long)a.sh.B * a.sh.H;
  const size_t smem = 2 * (size_t)kD * kD * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_fold_maps, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_fold_maps<<<(unsigned)(2 * BH), kFoldThreads, smem, a.stream>>>(
      maps_all, (long long)(rank_bytes / 4), (long long)(exp_off_bytes / 4), world, nch_stride, nch_total, BH,
      a.text_state, a.sh.H, a.sh.F, a.chunk, P, Q, pexp, qexp);
  return cudaGetLastError();
}

}  // namespace vdn
