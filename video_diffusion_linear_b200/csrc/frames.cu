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
// fp32 on the CUDA cores (a handful of steps per clip).
#include "common.cuh"
#include "internal.h"

namespace vdn {

namespace {

constexpr int kFoldThreads = 256;
constexpr int kD = 128;

}  // namespace

// maps_all: [world][B*H][2 directions][nch_stride][G_c | O_c][128][128] fp32 (true scale).
// P, Q: [B*H][F][128][128]; only chunk-edge frames are written.
__global__ void __launch_bounds__(kFoldThreads, 1) k_fold_maps(const float* __restrict__ maps_all, int world,
                                                               int nch_stride, int nch_total, long long BH,
                                                               const float* __restrict__ text, int H, int F,
                                                               int chunk, float* __restrict__ P,
                                                               float* __restrict__ Q) {
  extern __shared__ float4 fold_smem[];
  float* S = reinterpret_cast<float*>(fold_smem);   // state [128][128]
  float* G = S + kD * kD;                           // G_c [128][128]
  const int tid = threadIdx.x;
  const int dir = blockIdx.x & 1;
  const long long bh = blockIdx.x >> 1;
  const int h = (int)(bh % H);
  const int r0 = (tid >> 4) * 8, c0 = (tid & 15) * 8;   // this thread's 8 x 8 block of the product
  const long long rank_stride = BH * 2 * nch_stride * 2 * (long long)kD * kD;

  const float* T = text ? text + (long long)h * kD * kD : nullptr;
  for (int i = tid * 4; i < kD * kD; i += kFoldThreads * 4) {
    float4 v = T ? *reinterpret_cast<const float4*>(T + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    v.x *= kTextStateScale; v.y *= kTextStateScale; v.z *= kTextStateScale; v.w *= kTextStateScale;
    *reinterpret_cast<float4*>(S + i) = v;
  }
  for (int step = 0; step + 1 < nch_total; ++step) {
    const int c = dir == 0 ? step : nch_total - 1 - step;
    int r, j;
    chunk_owner(c, nch_total, world, r, j);
    const float* Gc = maps_all + r * rank_stride + (((bh * 2 + dir) * nch_stride + j) * 2) * (long long)kD * kD;
    const float* Oc = Gc + kD * kD;
    __syncthreads();   // the previous step's reads of G and writes of S are done
    for (int i = tid * 4; i < kD * kD; i += kFoldThreads * 4)
      *reinterpret_cast<float4*>(G + i) = *reinterpret_cast<const float4*>(Gc + i);
    __syncthreads();
    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const float4 o0 = *reinterpret_cast<const float4*>(Oc + (r0 + a) * kD + c0);
      const float4 o1 = *reinterpret_cast<const float4*>(Oc + (r0 + a) * kD + c0 + 4);
      acc[a][0] = o0.x; acc[a][1] = o0.y; acc[a][2] = o0.z; acc[a][3] = o0.w;
      acc[a][4] = o1.x; acc[a][5] = o1.y; acc[a][6] = o1.z; acc[a][7] = o1.w;
    }
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
    __syncthreads();   // every read of the old state is done
    const int f = dir == 0 ? (c + 1) * chunk - 1 : c * chunk;   // in [0, F): c <= C - 2 resp. c >= 1
    float* dst = (dir == 0 ? P : Q) + (bh * F + f) * (long long)kD * kD;
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

cudaError_t launch_fold_maps(const Args& a, const float* maps_all, int world, int nch_stride, float* P, float* Q) {
  if (a.sh.d != kD || world < 1 || a.chunk < 1) return cudaErrorInvalidValue;
  const int nch_total = (a.sh.F + a.chunk - 1) / a.chunk;
  if (world > nch_total || nch_stride < (nch_total + world - 1) / world) return cudaErrorInvalidValue;
  const long long BH = (long long)a.sh.B * a.sh.H;
  const size_t smem = 2 * (size_t)kD * kD * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(k_fold_maps, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_fold_maps<<<(unsigned)(2 * BH), kFoldThreads, smem, a.stream>>>(maps_all, world, nch_stride, nch_total, BH,
                                                                    a.text_state, a.sh.H, a.sh.F, a.chunk, P, Q);
  return cudaGetLastError();
}

}  // namespace vdn
