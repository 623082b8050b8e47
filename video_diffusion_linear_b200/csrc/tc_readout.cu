// Read-out, RMSNorm and output gate on the tensor cores (page section "Step 5").
//
// Persistent kernel: CTA i owns a contiguous range of 128-token tiles in the
// order (batch, head, frame, tile), so W_t changes only at frame boundaries.
// Per tile, O[128 tokens x 128] = Q'[128 x 128] W_t^T runs as tcgen05 MMAs with
// the accumulator in TMEM (two buffers), Q' = L2(SiLU(q)) produced in place in
// shared memory.  The product runs on fp16 operands, one MMA per K step: Q'
// (unit rows) and W_t, whose image the gather writes in fp16 with a power-of-two
// exponent per block of 32 rows (its largest entry in [0.5, 1)); the epilogue
// folds 2^e of each row block into the RMSNorm.  The gate / output tiles have
// three stages, so the store of a tile has a whole tile's time to read its
// buffer before that buffer is handed back to the gate loads.
// The epilogue reads one token row per thread from TMEM (32x32b layout), so the
// RMSNorm needs no cross-thread reduction; it multiplies rms_w and the gate and
// writes bf16 through shared memory and a TMA store.
//
// Warp roles (608 threads): 0 TMA producer of W and q, 1 MMA issuer (and TMEM
// owner), 2-9 q transform and 10-17 epilogue, two threads per token row (64
// channels each; the row sums of squares meet in shared memory), 18 TMA
// producer of the gate tiles (its buffers free up later, after the output
// store, so it runs apart from the q loads).
#include "common.cuh"
#include "image.cuh"
#include "internal.h"
#include "tc.cuh"
#include "tmap.h"

namespace vdn {

namespace {

constexpr int kQS = 2;      // q stages
constexpr int kGS = 3;      // gate stages

struct __align__(1024) ReadSmem {
  uint8_t wimg[32768];     // W_t, fp16 (K-major SW128 B operand)
  uint8_t qt[kQS][32768];  // raw q tile -> Q' (K-major SW128 A operand)
  uint8_t gt[kGS][32768];  // gate tile -> output tile
  float rms_w[128];
  float ssq_t[kQS][2][128];  // [stage][channel half][row] partial sums of the q transform
  float ssq_e[2][2][128];  // same for the epilogue
  uint64_t bar_w_full, bar_w_empty;
  uint64_t bar_q_full[kQS], bar_q_ready[kQS], bar_q_empty[kQS];
  uint64_t bar_g_full[kGS], bar_g_empty[kGS];
  uint64_t bar_acc_full[2], bar_acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

constexpr uint32_t kIdesc = tc::idesc_f16_f32(128, 128, false, false);
constexpr int kThreads = 608;

// swizzled byte offset of 16-byte chunk c (0..15) of row r in a [128 x 128] bf16 tile
__device__ __forceinline__ uint32_t row_chunk(int r, int c) {
  return (c >> 3) * 16384 + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) k_readout_tc(const __grid_constant__ CUtensorMap tmQ,
                                                           const __grid_constant__ CUtensorMap tmG,
                                                           const __grid_constant__ CUtensorMap tmO,
                                                           const uint16_t* __restrict__ wimg_g,
                                                           const int* __restrict__ wexp,
                                                           const int* __restrict__ wbexp,
                                                           const float* __restrict__ rms_w, int H, int F,
                                                           int ntile, long long T, uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  ReadSmem& sm = tc::smem_align<ReadSmem>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = &sm.abort;
  const long long G = gridDim.x;
  const long long x0 = (long long)blockIdx.x * T / G, x1 = ((long long)blockIdx.x + 1) * T / G;

  if (tid == 0) {
    tc::mbar_init(&sm.bar_w_full, 1);
    tc::mbar_init(&sm.bar_w_empty, 1);
    for (int s = 0; s < kQS; ++s) {
      tc::mbar_init(&sm.bar_q_full[s], 1);
      tc::mbar_init(&sm.bar_q_ready[s], 256);
      tc::mbar_init(&sm.bar_q_empty[s], 1);
    }
    for (int s = 0; s < kGS; ++s) {
      tc::mbar_init(&sm.bar_g_full[s], 1);
      tc::mbar_init(&sm.bar_g_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&sm.bar_acc_full[s], 1);
      tc::mbar_init(&sm.bar_acc_empty[s], 256);
    }
    sm.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&sm.tmem_base, 256);
    tc::tmem_relinquish();
  }
  if (tid >= 320 && tid < 448) sm.rms_w[tid - 320] = rms_w[tid - 320];
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // tile x = ((b H + h) F + t) ntile + j; each role decodes its first tile once
  // and then steps the counters, so the loops carry no 64-bit division
  struct Tile {
    long long fi;   // (b H + h) F + t: the W_t slot
    int j, t, h, b;
  };
  auto tile_at = [&](long long x) {
    Tile u;
    u.fi = x / ntile;
    u.j = (int)(x - u.fi * ntile);
    const long long bh = u.fi / F;
    u.t = (int)(u.fi - bh * F);
    u.b = (int)(bh / H);
    u.h = (int)(bh - (long long)u.b * H);
    return u;
  };
  auto tile_next = [&](Tile& u) {
    if (++u.j == ntile) {
      u.j = 0;
      ++u.fi;
      if (++u.t == F) {
        u.t = 0;
        if (++u.h == H) {
          u.h = 0;
          ++u.b;
        }
      }
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      long long cur = -1;
      uint32_t wph = 0;
      int it = 0;
      Tile u = tile_at(x0);
      for (long long x = x0; x < x1; ++x, ++it, tile_next(u)) {
        const long long fi = u.fi;
        if (fi != cur) {
          if (cur >= 0) {
            if (!tc::mbar_wait(&sm.bar_w_empty, wph, abort_flag, status)) break;
            wph ^= 1;
          }
          const uint8_t* src = reinterpret_cast<const uint8_t*>(wimg_g) + fi * kWImgBytes;
          tc::mbar_arrive_expect_tx(&sm.bar_w_full, kWImgBytes);
          for (int q = 0; q < 2; ++q) tc::bulk_load(sm.wimg + q * 16384, src + q * 16384, 16384, &sm.bar_w_full);
          cur = fi;
        }
        const int h = u.h, s0 = u.j * 128, fb = u.b * F + u.t;
        const int st = it % kQS;
        const uint32_t ph = (it / kQS) & 1;
        if (!tc::mbar_wait(&sm.bar_q_empty[st], ph ^ 1, abort_flag, status)) break;
        tc::mbar_arrive_expect_tx(&sm.bar_q_full[st], 32768);
        tc::tma_load_4d(&tmQ, &sm.bar_q_full[st], sm.qt[st], 0, h, s0, fb);
        tc::tma_load_4d(&tmQ, &sm.bar_q_full[st], sm.qt[st] + 16384, 64, h, s0, fb);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      long long cur = -1;
      uint32_t wph = 0;
      int it = 0;
      const uint32_t w = tc::smem_u32(sm.wimg);
      Tile u = tile_at(x0);
      for (long long x = x0; x < x1; ++x, ++it, tile_next(u)) {
        const long long fi = u.fi;
        if (fi != cur) {
          if (!tc::mbar_wait(&sm.bar_w_full, wph, abort_flag, status)) break;
          wph ^= 1;
          cur = fi;
        }
        const int qs = it % kQS, ab = it & 1;
        const uint32_t qph = (it / kQS) & 1, aph = (it >> 1) & 1;
        if (!tc::mbar_wait(&sm.bar_q_ready[qs], qph, abort_flag, status)) break;
        if (!tc::mbar_wait(&sm.bar_acc_empty[ab], aph ^ 1, abort_flag, status)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + ab * 128;
        const uint32_t a = tc::smem_u32(sm.qt[qs]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::umma_bf16(d, tc::smem_desc(a + koff, 16, 1024), tc::smem_desc(w + koff, 16, 1024), kIdesc,
                        kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(&sm.bar_q_empty[qs]);
        tc::umma_commit(&sm.bar_acc_full[ab]);
        if (x + 1 == x1 || u.j + 1 == ntile) tc::umma_commit(&sm.bar_w_empty);
      }
    }
  } else if (warp == 18) {
    // ------------------------------------------------------------ gate producer
    if (lane == 0) {
      int it = 0;
      Tile u = tile_at(x0);
      for (long long x = x0; x < x1; ++x, ++it, tile_next(u)) {
        const int h = u.h, s0 = u.j * 128, fb = u.b * F + u.t;
        const int st = it % kGS;
        const uint32_t ph = (it / kGS) & 1;
        if (!tc::mbar_wait(&sm.bar_g_empty[st], ph ^ 1, abort_flag, status)) break;
        tc::mbar_arrive_expect_tx(&sm.bar_g_full[st], 32768);
        tc::tma_load_4d(&tmG, &sm.bar_g_full[st], sm.gt[st], 0, h, s0, fb);
        tc::tma_load_4d(&tmG, &sm.bar_g_full[st], sm.gt[st] + 16384, 64, h, s0, fb);
      }
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ q' = L2(SiLU(q)), in place
    const int tt = tid - 64;
    const int r = tt & 127, hf = tt >> 7;   // row, channel half (chunks 8 hf .. 8 hf + 7)
    int it = 0;
    for (long long x = x0; x < x1; ++x, ++it) {
      const int st = it % kQS;
      const uint32_t ph = (it / kQS) & 1;
      if (!tc::mbar_wait(&sm.bar_q_full[st], ph, abort_flag, status)) break;
      uint8_t* base = sm.qt[st];
      float2 v[32];
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int cq = 0; cq < 8; ++cq) {
        const uint4 w = *reinterpret_cast<const uint4*>(base + row_chunk(r, 8 * hf + cq));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a = make_float2(silu_fast(bf16lo(ws[e])), silu_fast(bf16hi(ws[e])));
          v[4 * cq + e] = a;
          acc = __ffma2_rn(a, a, acc);
        }
      }
      sm.ssq_t[st][hf][r] = acc.x + acc.y;
      tc::named_bar(2, 256);
      const float inv = rsqrtf(sm.ssq_t[st][0][r] + sm.ssq_t[st][1][r] + kL2Eps);
      const float2 iv = make_float2(inv, inv);
#pragma unroll
      for (int cq = 0; cq < 8; ++cq) {
        uint32_t o4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 y = __fmul2_rn(v[4 * cq + e], iv);
          o4[e] = pack_f16x2(y.x, y.y);
        }
        *reinterpret_cast<uint4*>(base + row_chunk(r, 8 * hf + cq)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&sm.bar_q_ready[st]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // thread (row m = TMEM lane, channel half hf) keeps its 64 accumulator values
    // in registers; the two halves' sums of squares meet in shared memory
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;
    const int hf = (warp - 10) >> 2;
    const bool leader = tid == 320;
    int it = 0;
    Tile u = tile_at(x0);
    for (long long x = x0; x < x1; ++x, ++it, tile_next(u)) {
      const int st = it & 1;
      const uint32_t ph = (it >> 1) & 1;
      if (leader && it > 1) {
        tc::bulk_wait_read<1>();                        // the store of tile it - 2 has read its buffer
        tc::mbar_arrive(&sm.bar_g_empty[(it - 2) % kGS]);
      }
      // exponents of W_t (issued before the wait, used after it): the whole
      // matrix (RMSNorm eps) and the two row blocks of this channel half
      const long long fi = u.fi;
      const int ew = wexp[fi];
      const int eb0 = wbexp[fi * kWRowBlocks + 2 * hf], eb1 = wbexp[fi * kWRowBlocks + 2 * hf + 1];
      if (!tc::mbar_wait(&sm.bar_acc_full[st], ph, abort_flag, status)) break;
      tc::tc_fence_after();
      const uint32_t taddr = tmem + st * 128 + 64 * hf + ((uint32_t)(quarter * 32) << 16);
      uint32_t o[64];
      {
        uint32_t (&o0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&o[0]);
        uint32_t (&o1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&o[32]);
        tc::tmem_ld32(taddr, o0);
        tc::tmem_ld32(taddr + 32, o1);
        tc::tmem_ld_wait();
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&sm.bar_acc_empty[st]);
      // the true channel j of this half is 2^eb o_j, eb = eb0 for the first 32
      // channels, eb1 for the last 32 (row blocks of the fp16 image): the scales
      // enter the two partial sums of squares and the per-channel multiplier
      const float sc0 = pow2f(eb0), sc1 = pow2f(eb1);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float2 a = make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1]));
        acc0 = __ffma2_rn(a, a, acc0);
        const float2 c = make_float2(__uint_as_float(o[e + 32]), __uint_as_float(o[e + 33]));
        acc1 = __ffma2_rn(c, c, acc1);
      }
      sm.ssq_e[st][hf][m] = (acc0.x + acc0.y) * (sc0 * sc0) + (acc1.x + acc1.y) * (sc1 * sc1);
      tc::named_bar(1, 256);
      // W_t is stored as 2^-e W_t: the RMSNorm eps scales by 2^-2e
      const float ss = sm.ssq_e[st][0][m] + sm.ssq_e[st][1][m];
      const float inv = rsqrtf(ss * (1.0f / 128.0f) + ldexpf(kRmsEps, -2 * ew));
      const float inv0 = inv * sc0, inv1 = inv * sc1;
      const int gs = it % kGS;
      if (!tc::mbar_wait(&sm.bar_g_full[gs], (it / kGS) & 1, abort_flag, status)) break;
      uint8_t* base = sm.gt[gs];
#pragma unroll
      for (int cq = 0; cq < 8; ++cq) {
        const int c = 8 * hf + cq;
        const uint4 g = *reinterpret_cast<const uint4*>(base + row_chunk(m, c));
        const uint32_t gs[4] = {g.x, g.y, g.z, g.w};
        const float4 w0 = *reinterpret_cast<const float4*>(&sm.rms_w[8 * c]);
        const float4 w1 = *reinterpret_cast<const float4*>(&sm.rms_w[8 * c + 4]);
        const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        const float iv = cq < 4 ? inv0 : inv1;   // chunks 0-3: first row block of the half
        uint32_t outw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 8 * cq + 2 * e;
          const float2 y = __fmul2_rn(__fmul2_rn(make_float2(__uint_as_float(o[j]), __uint_as_float(o[j + 1])),
                                                 make_float2(iv * wv[2 * e], iv * wv[2 * e + 1])),
                                      make_float2(bf16lo(gs[e]), bf16hi(gs[e])));
          outw[e] = pack_bf16x2(y.x, y.y);
        }
        *reinterpret_cast<uint4*>(base + row_chunk(m, c)) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
      }
      tc::fence_proxy_async_smem();
      tc::named_bar(1, 256);
      if (leader) {
        const int h = u.h, s0 = u.j * 128, fb = u.b * F + u.t;
        tc::tma_store_4d(&tmO, base, 0, h, s0, fb);
        tc::tma_store_4d(&tmO, base + 16384, 64, h, s0, fb);
        tc::bulk_commit();
      }
    }
    if (leader) tc::bulk_wait_all();
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 256);
  }
}

cudaError_t launch_readout_tc(const Args& a, const uint16_t* wimg, const int* wexp, const int* wbexp,
                              uint32_t* status) {
  const vdn_shape& sh = a.sh;
  CUtensorMap tq, tg, to;
  long long BF = (long long)sh.B * sh.F;
  if (!tmap_tokens_bf16(&tq, a.q, sh.d, sh.H, sh.S, BF, 128) ||
      !tmap_tokens_bf16(&tg, a.gate, sh.d, sh.H, sh.S, BF, 128) ||
      !tmap_tokens_bf16(&to, a.out, sh.d, sh.H, sh.S, BF, 128))
    return cudaErrorInvalidValue;
  int ntile = (sh.S + 127) / 128;
  long long T = a.NF() * ntile;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long G = T < sms ? T : sms;
  size_t smem = sizeof(ReadSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_readout_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_readout_tc<<<(unsigned)G, kThreads, smem, a.stream>>>(tq, tg, to, wimg, wexp, wbexp, a.rms_w, sh.H, sh.F, ntile, T,
                                                             status);
  return cudaGetLastError();
}

}  // namespace vdn
