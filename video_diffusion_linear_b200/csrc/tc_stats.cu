// Frame statistics on the tensor cores (page sections "Step 1" and "Step 2").
//
// For every (batch, head, frame):  A_f = sum_s beta_s k'_s k'_s^T,
//                                  B_f = sum_s beta_s v'_s k'_s^T,
// a dense contraction over the frame's S tokens.  With X = sqrt(beta) k' and
// Y = sqrt(beta) v' (tokens x channels) one MMA of M = 128, N = 256 per 16
// tokens gives  X^T [X | Y] = [A | B^T]  in a TMEM accumulator, so beta is
// applied once, while the operands are produced, and no operand is written
// twice.  The k/v feature prep of Step 1 (short conv within the frame, SiLU,
// L2 normalisation of k) is fused into that operand production: raw bf16 rows
// arrive by TMA (96 tokens plus one halo row on each side, zero outside the
// frame), the transform warps compute X and Y in fp32 and store them as bf16 in
// the MN-major 128-byte-swizzled layout the tensor cores read.  Y needs no
// reduction across threads, so it is computed first and stored as soon as the
// tensor cores release the operand buffer; X follows once the norms of k are
// known.
//
// Work split: the (frame, 96-token block) pairs, frames ordered (batch, frame,
// head), are cut into gridDim.x contiguous ranges (stream-K).  A CTA flushes its
// accumulator whenever its range leaves a frame, into partial slot
// (blockIdx.x + frame), laid out [A; B] (256 rows of 128 floats); the per-frame
// solve adds the slots of each frame in a fixed order, so the result is
// deterministic.
//
// Warp roles (448 threads): 0 TMA producer, 1 MMA issuer (TMEM owner),
// 2-13 transform (4 tokens x 8 channels per thread); transform warps 2-5 (one
// per TMEM lane quarter) also flush the accumulator when a frame segment ends.
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"
#include "tmap.h"

namespace vdn {

namespace {

constexpr int kTPT = 4;                               // tokens per transform thread
constexpr int kTransformWarps = 12;
constexpr int kBT = 2 * kTPT * kTransformWarps;       // tokens per block
static_assert(kBT == kStatsTokens, "block size");
static_assert(kBT % 32 == 0, "block size");
constexpr int kRS = 2;                                // raw TMA stages
constexpr int kOS = 2;                                // operand stages: the transform fills one while
                                                      // the tensor cores read the other
constexpr int kRawRows = kBT + 2;
constexpr int kRawHalf = (kRawRows * 128 + 1023) / 1024 * 1024;
constexpr int kRawBytes = 4 * kRawRows * 128;         // k and v, two channel halves each
constexpr int kTransformThreads = 32 * kTransformWarps;
constexpr int kThreads = 64 + kTransformThreads;
constexpr int kKAtoms = kBT / 8;                      // 8-token swizzle atoms along K
constexpr int kOpHalf = kKAtoms * 2048;               // X (or Y): 128 channels x kBT bf16
constexpr int kMnAtomStride = kKAtoms * 1024;         // descriptor leading offset: next 64 channels

struct __align__(1024) StatsSmem {
  uint8_t raw[kRS][2][2][kRawHalf];    // [stage][k|v][channel half]
  uint8_t op[kOS][2 * kOpHalf];        // X | Y, MN-major SW128
  float taps[kRS][2][3][128];          // [stage][k|v][tap][channel, permuted as staged] conv taps / 2 of the stage's head
  float sqb[kRS][kBT];                 // [stage][token] sqrt(beta), 0 past the frame end
  uint64_t raw_full[kRS], raw_empty[kRS];
  uint64_t op_full[kOS], op_empty[kOS];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
  int abort;
};

constexpr uint32_t kIdesc = tc::idesc_bf16_f32(128, 256, true, true);

// Work unit x = pf * nb + j: block j of frame segment pf = (b * F + f) * H + h.  The
// loops advance it by increments: 64-bit division in every iteration would put a long
// dependent instruction chain on each role's critical path.
struct Unit {
  long long pf;
  int j, h, f, b;
};
__device__ __forceinline__ Unit unit_at(long long x, int nb, int H, int F) {
  Unit u;
  u.pf = x / nb;
  u.j = (int)(x - u.pf * nb);
  const long long fb = u.pf / H;
  u.h = (int)(u.pf - fb * H);
  u.b = (int)(fb / F);
  u.f = (int)(fb - (long long)u.b * F);
  return u;
}
__device__ __forceinline__ void unit_next(Unit& u, int nb, int H, int F) {
  if (++u.j == nb) {
    u.j = 0;
    ++u.pf;
    if (++u.h == H) {
      u.h = 0;
      if (++u.f == F) {
        u.f = 0;
        ++u.b;
      }
    }
  }
}


// byte offset of the 16-byte chunk holding channels 8c..8c+7 of token t in an
// MN-major SW128 operand of 128 channels x kBT tokens (atoms of 64 channels x
// 8 tokens, 1 KB each; K atoms contiguous, channel halves kMnAtomStride apart)
__device__ __forceinline__ uint32_t op_chunk(int c, int t) {
  return (c >> 3) * kMnAtomStride + (t >> 3) * 1024 + (t & 7) * 128 + ((((c & 7) ^ (t & 7))) << 4);
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) k_stats_tc(const __grid_constant__ CUtensorMap tmK,
                                                         const __grid_constant__ CUtensorMap tmV,
                                                         const float* __restrict__ beta,
                                                         const float* __restrict__ wk_g, const float* __restrict__ wv_g,
                                                         int K, int H, int F, int S, int nb, long long T,
                                                         float* __restrict__ part, uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  StatsSmem& sm = tc::smem_align<StatsSmem>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = &sm.abort;
  const long long G = gridDim.x;
  const long long x0 = (long long)blockIdx.x * T / G, x1 = ((long long)blockIdx.x + 1) * T / G;

  if (tid == 0) {
    for (int s = 0; s < kRS; ++s) {
      tc::mbar_init(&sm.raw_full[s], 1);
      tc::mbar_init(&sm.raw_empty[s], kTransformWarps);
    }
    for (int s = 0; s < kOS; ++s) {
      tc::mbar_init(&sm.op_full[s], kTransformWarps);
      tc::mbar_init(&sm.op_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&sm.acc_full[s], 1);
      tc::mbar_init(&sm.acc_empty[s], 128);
    }
    sm.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&sm.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // the last block of a frame segment: the frame's last block or the CTA's last unit
  auto seg_last = [&](long long x, const Unit& u) { return x + 1 == x1 || u.j + 1 == nb; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    // lane 0 issues the TMA copies; all lanes stage sqrt(beta) of the block's
    // tokens and, when the stage's head changes, the conv taps of that head.
    // beta of the next block is loaded one iteration ahead, so its latency
    // overlaps the wait for a free stage.
    const long long N = (long long)F * S;
    int slot_head[kRS];
#pragma unroll
    for (int r = 0; r < kRS; ++r) slot_head[r] = -1;
    constexpr int BU = kBT / 32;
    float bnext[BU];
    auto load_beta = [&](const Unit& un) {
      const long long nbase = (long long)un.b * N + (long long)un.f * S;
#pragma unroll
      for (int u = 0; u < BU; ++u) {
        const int s = un.j * kBT + lane + 32 * u;
        bnext[u] = s < S ? beta[(nbase + s) * H + un.h] : 0.f;
      }
    };
    Unit un = unit_at(x0, nb, H, F);
    if (x0 < x1) load_beta(un);
    int it = 0;
    for (long long x = x0; x < x1; ++x, ++it) {
      const Unit u = un;
      unit_next(un, nb, H, F);          // the next unit: its beta is loaded during this one
      const int h = u.h, fb = u.b * F + u.f, s0 = u.j * kBT;
      const int rs = it % kRS;
      const uint32_t ph = (it / kRS) & 1;
      if (!tc::mbar_wait(&sm.raw_empty[rs], ph ^ 1, abort_flag, status)) break;
      if (lane == 0) {
        for (int hf = 0; hf < 2; ++hf) {
          tc::tma_load_4d(&tmK, &sm.raw_full[rs], sm.raw[rs][0][hf], 64 * hf, h, s0 - 1, fb);
          tc::tma_load_4d(&tmV, &sm.raw_full[rs], sm.raw[rs][1][hf], 64 * hf, h, s0 - 1, fb);
        }
      }
#pragma unroll
      for (int u = 0; u < BU; ++u) sm.sqb[rs][lane + 32 * u] = sqrtf(bnext[u]);
      if (x + 1 < x1) load_beta(un);
      int cached = slot_head[0];
#pragma unroll
      for (int r = 0; r < kRS; ++r)
        if (r == rs) cached = slot_head[r];
      if (cached != h) {
        for (int e = lane; e < 2 * 3 * 128; e += 32) {
          const int ten = e / 384, tap = (e / 128) % 3, ch = e % 128;
          const float* wg = ten == 0 ? wk_g : wv_g;
          float val;
          if (!wg) val = tap == 1 ? 1.f : 0.f;                       // identity
          else if (K == 3) val = wg[((long long)h * 128 + ch) * 3 + tap];
          else val = tap == 1 ? wg[(long long)h * 128 + ch] : 0.f;   // one tap: centre
          // [tap][quad parity][chunk]: a quarter warp's 8 chunks are 128 contiguous bytes
          sm.taps[rs][ten][tap][((ch >> 2) & 1) * 64 + (ch >> 3) * 4 + (ch & 3)] = 0.5f * val;
        }
#pragma unroll
        for (int r = 0; r < kRS; ++r)
          if (r == rs) slot_head[r] = h;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_expect_tx(&sm.raw_full[rs], kRawBytes);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, seg = 0;
      bool first = true;
      Unit u = unit_at(x0, nb, H, F);
      for (long long x = x0; x < x1; ++x, ++it, unit_next(u, nb, H, F)) {
        const int os = it % kOS;
        const uint32_t oph = (it / kOS) & 1;
        const int ab = seg & 1;
        if (first) {
          if (!tc::mbar_wait(&sm.acc_empty[ab], ((seg >> 1) & 1) ^ 1, abort_flag, status)) break;
        }
        if (!tc::mbar_wait(&sm.op_full[os], oph, abort_flag, status)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + ab * 256;
        const uint32_t base = tc::smem_u32(sm.op[os]);
#pragma unroll
        for (int kk = 0; kk < kBT / 16; ++kk) {
          uint64_t desc = tc::smem_desc(base + kk * 2048, kMnAtomStride, 1024);
          tc::umma_bf16(d, desc, desc, kIdesc, (first && kk == 0) ? 0u : 1u);
        }
        tc::umma_commit(&sm.op_empty[os]);
        first = false;
        if (seg_last(x, u)) {
          tc::umma_commit(&sm.acc_full[ab]);
          ++seg;
          first = true;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ transform (+ flush)
    const int tt = tid - 64;
    const int w = tt >> 5, tg = (tt >> 4) & 1, c = tt & 15;
    const int half = c >> 3, cc = c & 7;
    const int tok0 = 2 * kTPT * w + kTPT * tg;   // first of this thread's kTPT tokens in the block
    const bool flusher = w < 4;                  // warps 2-5: TMEM lane quarters 2, 3, 0, 1
    const int quarter = warp & 3;
    int seg = 0;
    int it = 0;
    Unit u = unit_at(x0, nb, H, F);
    for (long long x = x0; x < x1; ++x, ++it, unit_next(u, nb, H, F)) {
      const int rs = it % kRS;
      const uint32_t rph = (it / kRS) & 1;
      const int os = it % kOS;
      const uint32_t oph = (it / kOS) & 1;
      if (!tc::mbar_wait(&sm.raw_full[rs], rph, abort_flag, status)) break;
      float sb[kTPT];
#pragma unroll
      for (int i = 0; i < kTPT; i += 4) {
        const float4 q4 = *reinterpret_cast<const float4*>(&sm.sqb[rs][tok0 + i]);
        sb[i] = q4.x; sb[i + 1] = q4.y; sb[i + 2] = q4.z; sb[i + 3] = q4.w;
      }

      // y = SiLU(conv(x)) = h + h tanh(h), h = conv(x) / 2 (the taps carry the 1/2);
      // ss = sum of y^2 over this thread's channels
      auto conv_silu = [&](int ten, float2 (&y)[kTPT][4], float (&ss)[kTPT]) {
        float2 w3[3][4];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const float4 a = *reinterpret_cast<const float4*>(&sm.taps[rs][ten][j][4 * c]);
          const float4 b = *reinterpret_cast<const float4*>(&sm.taps[rs][ten][j][64 + 4 * c]);
          w3[j][0] = make_float2(a.x, a.y); w3[j][1] = make_float2(a.z, a.w);
          w3[j][2] = make_float2(b.x, b.y); w3[j][3] = make_float2(b.z, b.w);
        }
        float2 r[kTPT + 2][4];
        const uint8_t* src = sm.raw[rs][ten][half];
#pragma unroll
        for (int rr = 0; rr < kTPT + 2; ++rr) {
          const int row = tok0 + rr;
          const uint4 q = *reinterpret_cast<const uint4*>(src + row * 128 + ((cc ^ (row & 7)) << 4));
          r[rr][0] = make_float2(bf16lo(q.x), bf16hi(q.x));
          r[rr][1] = make_float2(bf16lo(q.y), bf16hi(q.y));
          r[rr][2] = make_float2(bf16lo(q.z), bf16hi(q.z));
          r[rr][3] = make_float2(bf16lo(q.w), bf16hi(q.w));
        }
        float2 hx[kTPT][4];
#pragma unroll
        for (int i = 0; i < kTPT; ++i)
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            float2 a = __fmul2_rn(w3[2][p], r[i + 2][p]);
            a = __ffma2_rn(w3[1][p], r[i + 1][p], a);
            hx[i][p] = __ffma2_rn(w3[0][p], r[i][p], a);
          }
        float2 th[kTPT][4];
#pragma unroll
        for (int i = 0; i < kTPT; ++i)
#pragma unroll
          for (int p = 0; p < 4; ++p) th[i][p] = tanh2(hx[i][p]);
#pragma unroll
        for (int i = 0; i < kTPT; ++i) {
          float2 acc = make_float2(0.f, 0.f);
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            y[i][p] = __ffma2_rn(hx[i][p], th[i][p], hx[i][p]);
            acc = __ffma2_rn(y[i][p], y[i][p], acc);
          }
          ss[i] = acc.x + acc.y;
        }
      };
      auto store = [&](const float2 (&y)[kTPT][4], const float (&scale)[kTPT], uint8_t* dst) {
#pragma unroll
        for (int i = 0; i < kTPT; ++i) {
          const float2 s2 = make_float2(scale[i], scale[i]);
          uint32_t wv[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 a = __fmul2_rn(y[i][p], s2);
            wv[p] = pack_bf16x2(a.x, a.y);
          }
          *reinterpret_cast<uint4*>(dst + op_chunk(c, tok0 + i)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
      };

      if (!tc::mbar_wait(&sm.op_empty[os], oph ^ 1, abort_flag, status)) break;
      {
        float2 vy[kTPT][4];
        float unused[kTPT];
        conv_silu(1, vy, unused);
        store(vy, sb, sm.op[os] + kOpHalf);      // Y = sqrt(beta) v'
      }
      float2 ky[kTPT][4];
      float ssq[kTPT];
      conv_silu(0, ky, ssq);
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.raw_empty[rs]);      // one arrival per warp
#pragma unroll
      for (int i = 0; i < kTPT; ++i) {
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) ssq[i] += __shfl_xor_sync(0xffffffffu, ssq[i], o);
        ssq[i] = sb[i] * rsqrtf(ssq[i] + kL2Eps);
      }
      store(ky, ssq, sm.op[os]);                  // X = sqrt(beta) k'
      tc::fence_proxy_async_smem();   // each thread's stores, then one arrival per warp
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.op_full[os]);
      const bool last = seg_last(x, u);
      if (flusher && last) {
        // the segment of this frame is complete once its last block's MMA is: copy
        // the accumulator to partial slot (blockIdx.x + frame) as [A; B], 256 rows of
        // 128: TMEM lane m holds row m of [A | B^T], i.e. column m of A (symmetric) and
        // of B, which the warp's lanes write as consecutive floats of each slot row
        const int ab = seg & 1;
        if (!tc::mbar_wait(&sm.acc_full[ab], (seg >> 1) & 1, abort_flag, status)) break;
        tc::tc_fence_after();
        const long long pf = u.pf;
        const int m = quarter * 32 + lane;
        float* dstp = part + ((long long)blockIdx.x + pf) * (256 * 128) + m;
        const uint32_t taddr = tmem + ab * 256 + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
        for (int j = 0; j < 8; ++j) {
          uint32_t r[32];
          tc::tmem_ld32(taddr + 32 * j, r);
          tc::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) dstp[(32 * j + e) * 128] = __uint_as_float(r[e]);
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&sm.acc_empty[ab]);
      }
      if (last) ++seg;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_stats_tc(const Args& a, float* partials, uint32_t* status) {
  const vdn_shape& sh = a.sh;
  CUtensorMap tk, tv;
  long long BF = (long long)sh.B * sh.F;
  if (!tmap_tokens_bf16(&tk, a.k, sh.d, sh.H, sh.S, BF, kRawRows) ||
      !tmap_tokens_bf16(&tv, a.v, sh.d, sh.H, sh.S, BF, kRawRows))
    return cudaErrorInvalidValue;
  int nb = (sh.S + kStatsTokens - 1) / kStatsTokens;
  long long T = a.NF() * nb;
  long long G = T < kStatsGrid ? T : kStatsGrid;
  size_t smem = sizeof(StatsSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_stats_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int K = (a.conv_k_w || a.conv_v_w) ? sh.conv_width : 1;
  k_stats_tc<<<(unsigned)G, kThreads, smem, a.stream>>>(tk, tv, a.beta, a.conv_k_w, a.conv_v_w, K, sh.H, sh.F, sh.S,
                                                       nb, T, partials, status);
  return cudaGetLastError();
}

}  // namespace vdn
