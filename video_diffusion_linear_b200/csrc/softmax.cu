// Windowed softmax branch of the hybrid attention layer (page sections on why
// video models stall on attention and what the far field is): every query token
// of frame t attends, through the RoPE-rotated q / k, to all tokens of frames
// lo..hi of its chunk-aligned window, o = softmax(q k^T * scale) v; the linear
// branch covers the frames outside the window and the layer adds the two.
//
// SIMT path (any dtype, d = 16 or 128): a block takes up to 128 query tokens of
// one window chunk (all share the window), stages 32 keys at a time in shared
// memory, and every query keeps a running maximum, normaliser and output
// (online softmax, fp32, exp2 with log2(e) folded into the scale).  A query is
// spread over d / 16 threads of 16 channels each; its dot products meet by
// shuffles within those threads.
//
// Tensor-core path (bf16, d = 128): one CTA per tile of 128 query tokens of a
// window chunk, two passes over the window's key tiles of 128.  Pass 1: the
// tensor cores write S = Q K^T to TMEM (two buffers), the softmax warps read it
// and keep each row's running maximum and normaliser.  Pass 2: S is computed
// again; the softmax warps turn it into P = exp(S - m) / l, stored in bf16 as
// the K-major A operand of O += P V, which accumulates in TMEM.  With the row
// statistics final before pass 2, O never needs rescaling.  Warp roles (320
// threads): 0 TMA producer (Q once, then K tiles, and V tiles in pass 2), 1
// MMA issuer (TMEM owner), 2-9 softmax and epilogue, two threads per query row
// (64 key columns each; their statistics merge once, after pass 1).
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"
#include "tmap.h"

namespace vdn {

namespace {

constexpr int kSoftThreads = 128;
constexpr int kSoftKeys = 32;
constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

template <int D, typename T>
__global__ void __launch_bounds__(kSoftThreads) k_wsoft_simt(const T* __restrict__ qr, const T* __restrict__ kr,
                                                            const T* __restrict__ v, int H, int F, int S, int chunk,
                                                            int radius, int tiles_per_chunk, float scale,
                                                            int accumulate, T* __restrict__ out) {
  constexpr int CPT = 16, TPQ = D / CPT, QPB = kSoftThreads / TPQ;
  __shared__ float ks[kSoftKeys][D], vs[kSoftKeys][D];
  const int tid = threadIdx.x, qi = tid / TPQ, part = tid % TPQ;
  const long long bh = blockIdx.x;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const int c = blockIdx.y / tiles_per_chunk, tile = blockIdx.y % tiles_per_chunk;
  const int f0 = c * chunk;
  if (f0 >= F) return;
  const long long N = (long long)F * S;
  const long long cq0 = (long long)f0 * S, cq1 = (long long)min(F, f0 + chunk) * S;   // queries of the chunk
  const long long n = cq0 + (long long)tile * QPB + qi;
  if (cq0 + (long long)tile * QPB >= cq1) return;       // tile past the (shorter) last chunk: whole block leaves
  const bool valid = n < cq1;
  int lo, hi;
  window_bounds(f0, F, chunk, radius, lo, hi);
  const long long k0 = (long long)lo * S, k1 = (long long)(hi + 1) * S;
  const float sc = scale * kLog2e;

  float q[CPT], o[CPT];
  const long long row = ((b * N + (valid ? n : cq0)) * H + h) * D + part * CPT;
#pragma unroll
  for (int e = 0; e < CPT; ++e) {
    q[e] = to_f32(qr[row + e]) * sc;
    o[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (long long kb = k0; kb < k1; kb += kSoftKeys) {
    const int nk = (int)min((long long)kSoftKeys, k1 - kb);
    __syncthreads();
    for (int e = tid; e < kSoftKeys * D; e += kSoftThreads) {
      const int j = e / D, ch = e % D;
      float kv = 0.f, vv = 0.f;
      if (j < nk) {
        const long long off = ((b * N + kb + j) * H + h) * D + ch;
        kv = to_f32(kr[off]);
        vv = to_f32(v[off]);
      }
      ks[j][ch] = kv;
      vs[j][ch] = vv;
    }
    __syncthreads();
    for (int j = 0; j < nk; ++j) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < CPT; ++e) s = fmaf(q[e], ks[j][part * CPT + e], s);
#pragma unroll
      for (int w = 1; w < TPQ; w <<= 1) s += __shfl_xor_sync(0xffffffffu, s, w);
      const float mn = fmaxf(m, s);
      const float corr = exp2f(m - mn), p = exp2f(s - mn);
      l = fmaf(l, corr, p);
#pragma unroll
      for (int e = 0; e < CPT; ++e) o[e] = fmaf(o[e], corr, p * vs[j][part * CPT + e]);
      m = mn;
    }
  }
  if (!valid) return;
  const float inv = 1.f / l;
  const long long orow = ((b * N + n) * H + h) * D + part * CPT;
#pragma unroll
  for (int e = 0; e < CPT; ++e) {
    float y = o[e] * inv;
    if (accumulate) y += to_f32(out[orow + e]);
    out[orow + e] = from_f32<T>(y);
  }
}

cudaError_t launch_window_softmax_simt(const vdn_shape& sh, const void* qr, const void* kr, const void* v, int chunk,
                                       int radius, float scale, int accumulate, void* out, cudaStream_t stream) {
  const int nchunks = (sh.F + chunk - 1) / chunk;
  const int qpb = kSoftThreads / (sh.d / 16);
  const int tiles = (int)(((long long)chunk * sh.S + qpb - 1) / qpb);
  if ((long long)nchunks * tiles > 65535) return cudaErrorInvalidConfiguration;
  dim3 grid((unsigned)((long long)sh.B * sh.H), (unsigned)(nchunks * tiles));
#define VDN_WSOFT(D_, T_)                                                                                       \
  k_wsoft_simt<D_, T_><<<grid, kSoftThreads, 0, stream>>>(                                                   \
      static_cast<const T_*>(qr), static_cast<const T_*>(kr), static_cast<const T_*>(v), sh.H, sh.F, sh.S, chunk, \
      radius, tiles, scale, accumulate, static_cast<T_*>(out))
  if (sh.dtype == VDN_DTYPE_BF16) {
    VDN_WSOFT(128, __nv_bfloat16);
  } else if (sh.d == 16) {
    VDN_WSOFT(16, float);
  } else {
    VDN_WSOFT(128, float);
  }
#undef VDN_WSOFT
  return cudaGetLastError();
}

namespace {

constexpr int kTcThreads = 320;
constexpr int kKS = 2, kVS = 2;            // K and V tile stages
constexpr float kRescaleAbove = 8.f;      // log2 units: a reference maximum moves only when a score exceeds it by 2^8
constexpr uint32_t kIdescQK = tc::idesc_bf16_f32(128, 128, false, false);   // Q, K tiles: K-major
constexpr uint32_t kIdescPV = tc::idesc_bf16_f32(128, 128, false, true);    // P K-major, V MN-major

// Key tiles alternate between two groups of four softmax warps (group g takes the tiles j with
// j % 2 == g).  Each group has its own S buffer, P buffer and O accumulator, so the two warps that
// share an SM sub-partition (same TMEM lanes, one per group) work one Q K^T apart: one computes
// exponentials while the other loads, reduces and stores.
struct __align__(1024) WsoftSmem {
  uint8_t q[32768];          // Q tile: [channel half][128 rows x 128 B], SW128 (K-major A operand)
  uint8_t k[kKS][32768];     // K tiles: same layout (K-major B operand)
  uint8_t v[kVS][32768];     // V tiles: same layout (MN-major B operand of P V)
  uint8_t p[2][32768];       // P per group: [key half][128 rows x 128 B], SW128 (K-major A operand)
  uint64_t q_full, k_full[kKS], k_empty[kKS], v_full[kVS], v_empty[kVS];
  uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2], o_full;
  uint32_t tmem_base;
  int abort;
};
// after the last MMA the K stages hold the groups' reference maxima and normalisers
struct WsoftStats {
  float m[2][128], l[2][128];   // [group][row]
};
static_assert(sizeof(WsoftStats) <= kKS * 32768, "statistics fit in the K stages");

// byte offset of the 16-byte chunk c (0..15) of row r in a 128 x 128 bf16 SW128 tile
__device__ __forceinline__ uint32_t tile_chunk(int r, int c) {
  return (c >> 3) * 16384 + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

}  // namespace

__global__ void __launch_bounds__(kTcThreads, 1) k_wsoft_tc(const __grid_constant__ CUtensorMap tmQ,
                                                           const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV, int H, int F,
                                                           int S, int chunk, int radius, int tiles_per_chunk,
                                                           float scale, int accumulate,
                                                           __nv_bfloat16* __restrict__ out,
                                                           uint32_t* __restrict__ status) {
  // consecutive CTAs take consecutive query tiles of one (batch, head, chunk): the CTAs resident
  // at a time share one K/V window in L2
  const long long bh = blockIdx.y;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  const int c = blockIdx.x / tiles_per_chunk, tile = blockIdx.x % tiles_per_chunk;
  const int f0 = c * chunk;
  if (f0 >= F) return;
  const long long N = (long long)F * S;
  const long long cq1 = (long long)min(F, f0 + chunk) * S;
  const long long q0 = (long long)f0 * S + 128LL * tile;      // first query token of the tile
  if (q0 >= cq1) return;                                     // past the (shorter) last chunk
  int lo, hi;
  window_bounds(f0, F, chunk, radius, lo, hi);
  const long long k0 = (long long)lo * S, k1 = (long long)(hi + 1) * S;
  const int nkt = (int)((k1 - k0 + 127) / 128);

  extern __shared__ uint8_t smem_raw[];
  WsoftSmem& sm = tc::smem_align<WsoftSmem>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = &sm.abort;
  if (tid == 0) {
    tc::mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kKS; ++s) {
      tc::mbar_init(&sm.k_full[s], 1);
      tc::mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kVS; ++s) {
      tc::mbar_init(&sm.v_full[s], 1);
      tc::mbar_init(&sm.v_empty[s], 1);
    }
    for (int g = 0; g < 2; ++g) {
      tc::mbar_init(&sm.s_full[g], 1);
      tc::mbar_init(&sm.s_empty[g], 4);
      tc::mbar_init(&sm.p_full[g], 4);
      tc::mbar_init(&sm.p_empty[g], 1);
    }
    tc::mbar_init(&sm.o_full, 1);
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
  const uint32_t tmem = sm.tmem_base;       // S of group g at columns 128 g, O of group g at 256 + 128 g
  const int rowq = (int)(b * N + q0), rowk = (int)(b * N + k0);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // K runs two tiles ahead of V: Q K^T for tile j+2 is issued before P V for tile j
    if (lane == 0) {
      auto load_k = [&](int t) -> bool {
        const int ks = t % kKS;
        if (!tc::mbar_wait(&sm.k_empty[ks], ((t / kKS) & 1) ^ 1, abort_flag, status)) return false;
        tc::mbar_arrive_expect_tx(&sm.k_full[ks], 32768);
        tc::tma_load_3d(&tmK, &sm.k_full[ks], sm.k[ks], 0, h, rowk + 128 * t);
        tc::tma_load_3d(&tmK, &sm.k_full[ks], sm.k[ks] + 16384, 64, h, rowk + 128 * t);
        return true;
      };
      auto load_v = [&](int t) -> bool {
        const int vs = t % kVS;
        if (!tc::mbar_wait(&sm.v_empty[vs], ((t / kVS) & 1) ^ 1, abort_flag, status)) return false;
        tc::mbar_arrive_expect_tx(&sm.v_full[vs], 32768);
        tc::tma_load_3d(&tmV, &sm.v_full[vs], sm.v[vs], 0, h, rowk + 128 * t);
        tc::tma_load_3d(&tmV, &sm.v_full[vs], sm.v[vs] + 16384, 64, h, rowk + 128 * t);
        return true;
      };
      tc::mbar_arrive_expect_tx(&sm.q_full, 32768);
      tc::tma_load_3d(&tmQ, &sm.q_full, sm.q, 0, h, rowq);
      tc::tma_load_3d(&tmQ, &sm.q_full, sm.q + 16384, 64, h, rowq);
      bool ok = load_k(0) && (nkt < 2 || load_k(1)) && load_v(0);
      for (int j = 0; j < nkt && ok; ++j) {
        if (j + 2 < nkt) ok = load_k(j + 2);
        if (ok && j + 1 < nkt) ok = load_v(j + 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t aq = tc::smem_u32(sm.q);
      bool ok = tc::mbar_wait(&sm.q_full, 0, abort_flag, status);
      auto qk = [&](int t) -> bool {   // S_t = Q K_t^T into the S buffer of group t % 2
        const int ks = t % kKS, g = t % 2;
        if (!tc::mbar_wait(&sm.k_full[ks], (t / kKS) & 1, abort_flag, status)) return false;
        if (!tc::mbar_wait(&sm.s_empty[g], ((t / 2) & 1) ^ 1, abort_flag, status)) return false;
        tc::tc_fence_after();
        const uint32_t bk = tc::smem_u32(sm.k[ks]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::umma_bf16(tmem + g * 128, tc::smem_desc(aq + off, 16, 1024), tc::smem_desc(bk + off, 16, 1024),
                        kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(&sm.s_full[g]);
        tc::umma_commit(&sm.k_empty[ks]);
        return true;
      };
      auto pv = [&](int j) -> bool {   // O_g += P_j V_j, g = j % 2
        const int vs = j % kVS, g = j % 2;
        if (!tc::mbar_wait(&sm.v_full[vs], (j / kVS) & 1, abort_flag, status)) return false;
        if (!tc::mbar_wait(&sm.p_full[g], (j / 2) & 1, abort_flag, status)) return false;
        tc::tc_fence_after();
        const uint32_t ap = tc::smem_u32(sm.p[g]), bv = tc::smem_u32(sm.v[vs]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          tc::umma_bf16(tmem + 256 + 128 * g, tc::smem_desc(ap + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                        tc::smem_desc(bv + kk * 2048, 16384, 1024), kIdescPV, (j >= 2 || kk > 0) ? 1u : 0u);
        }
        tc::umma_commit(&sm.p_empty[g]);
        tc::umma_commit(&sm.v_empty[vs]);
        return true;
      };
      ok = ok && qk(0) && (nkt < 2 || qk(1));
      for (int j = 0; j < nkt && ok; ++j) {
        if (j + 2 < nkt) ok = qk(j + 2);
        if (ok) ok = pv(j);
      }
      if (ok) tc::umma_commit(&sm.o_full);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3, g = (warp - 2) >> 2;
    const int m = 32 * quarter + lane;                 // query row = TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    // mref: the reference maximum (log2 units) that every exponent of this row in this group is taken
    // against; it moves only when a tile's maximum exceeds it by more than 2^8, and then O_g and l are
    // rescaled
    float mref = -INFINITY, lrun = 0.f;
    bool ok = true;
    for (int j = g, n = 0; j < nkt && ok; j += 2, ++n) {
      // this group's n-th tile: its S buffer, then the tile maximum
      if (!(ok = tc::mbar_wait(&sm.s_full[g], n & 1, abort_flag, status))) break;
      tc::tc_fence_after();
      uint32_t r[128];
#pragma unroll
      for (int part = 0; part < 4; ++part)
        tc::tmem_ld32(tmem + g * 128 + 32 * part + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * part]));
      tc::tmem_ld_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.s_empty[g]);
      const int nvalid = (int)min(128LL, k1 - (k0 + 128LL * j));
      float tmax;
      if (nvalid == 128) {                    // every tile but the window's last: a tree of maxima
        float t8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) t8[a] = __uint_as_float(r[a]);
#pragma unroll
        for (int e = 8; e < 128; ++e) t8[e & 7] = fmaxf(t8[e & 7], __uint_as_float(r[e]));
        tmax = fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])), fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7])));
      } else {
        tmax = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e < nvalid) tmax = fmaxf(tmax, __uint_as_float(r[e]));
      }
      const float mt = tmax * scale;
      float corr = 1.f;
      const bool move = mt > mref + kRescaleAbove;
      if (move) {
        corr = mref == -INFINITY ? 0.f : ex2_approx(mref - mt);
        lrun *= corr;
        mref = mt;
      }
      uint32_t pw[64];
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
      if (nvalid == 128) {
#pragma unroll
        for (int e = 0; e < 128; e += 2) {
          const float p0 = ex2_approx(__uint_as_float(r[e]) * scale - mref);
          const float p1 = ex2_approx(__uint_as_float(r[e + 1]) * scale - mref);
          sum[(e >> 1) & 3] += p0 + p1;
          pw[e / 2] = pack_bf16x2(p0, p1);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 128; e += 2) {
          const float p0 = e < nvalid ? ex2_approx(__uint_as_float(r[e]) * scale - mref) : 0.f;
          const float p1 = e + 1 < nvalid ? ex2_approx(__uint_as_float(r[e + 1]) * scale - mref) : 0.f;
          sum[(e >> 1) & 3] += p0 + p1;
          pw[e / 2] = pack_bf16x2(p0, p1);
        }
      }
      lrun += (sum[0] + sum[1]) + (sum[2] + sum[3]);
      // this group's previous P V has completed once its P buffer is free
      if (!(ok = tc::mbar_wait(&sm.p_empty[g], (n & 1) ^ 1, abort_flag, status))) break;
      // tcgen05.ld/st are warp-collective: the warp rescales its O rows together when any of its
      // rows moved (corr = 1 for the others)
      if (__any_sync(0xffffffffu, move) && n > 0) {
        tc::tc_fence_after();
#pragma unroll
        for (int part = 0; part < 4; ++part) {
          uint32_t o[32];
          const uint32_t taddr = tmem + 256 + 128 * g + 32 * part + lane_off;
          tc::tmem_ld32(taddr, o);
          tc::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
          tc::tmem_st32(taddr, o);
        }
        tc::tmem_st_wait();
        tc::tc_fence_before();
      }
#pragma unroll
      for (int cq = 0; cq < 16; ++cq)
        *reinterpret_cast<uint4*>(sm.p[g] + tile_chunk(m, cq)) =
            make_uint4(pw[4 * cq], pw[4 * cq + 1], pw[4 * cq + 2], pw[4 * cq + 3]);
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.p_full[g]);
    }
    // epilogue, once every MMA has completed (the K stages are then free for the statistics):
    // O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)); a group that saw
    // no tile (m = -inf) adds nothing and its accumulator is never read
    if (ok) ok = tc::mbar_wait(&sm.o_full, 0, abort_flag, status);
    WsoftStats& st = *reinterpret_cast<WsoftStats*>(sm.k[0]);
    if (ok) {
      st.m[g][m] = mref;
      st.l[g][m] = lrun;
    }
    tc::named_bar(2 + quarter, 64);
    if (ok) {
      tc::tc_fence_after();
      const float m0 = st.m[0][m], m1 = st.m[1][m];
      const float mx = fmaxf(m0, m1);
      const float w0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - mx), w1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - mx);
      const float inv_l = 1.f / (st.l[0][m] * w0 + st.l[1][m] * w1);
      const float c0 = w0 * inv_l, c1 = w1 * inv_l;
      const bool use1 = nkt > 1;
      float o[64];       // this thread's 64 output channels (64 g .. 64 g + 63) of its row
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        uint32_t a0[32], a1[32];
        tc::tmem_ld32(tmem + 256 + 64 * g + 32 * part + lane_off, a0);
        tc::tmem_ld32(tmem + 384 + 64 * g + 32 * part + lane_off, a1);
        tc::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e)
          o[32 * part + e] = __uint_as_float(a0[e]) * c0 + (use1 ? __uint_as_float(a1[e]) * c1 : 0.f);
      }
      if (q0 + m < cq1) {
        uint4* dst = reinterpret_cast<uint4*>(out + ((b * N + q0 + m) * H + h) * 128 + 64 * g);
#pragma unroll
        for (int cq = 0; cq < 8; ++cq) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = o[8 * cq + e];
          if (accumulate) {
            const uint4 prev = dst[cq];
            const uint32_t pv4[4] = {prev.x, prev.y, prev.z, prev.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              y[2 * e] += bf16lo(pv4[e]);
              y[2 * e + 1] += bf16hi(pv4[e]);
            }
          }
          dst[cq] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                               pack_bf16x2(y[6], y[7]));
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_window_softmax_tc(const vdn_shape& sh, const void* qr, const void* kr, const void* v, int chunk,
                                     int radius, float scale, int accumulate, void* out, uint32_t* status,
                                     cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  const long long rows = (long long)sh.B * sh.F * sh.S;
  if (rows > 0x7fffffffLL - 256) return cudaErrorInvalidValue;
  if (!tmap_token_rows_bf16(&tq, qr, sh.d, sh.H, rows, 128) || !tmap_token_rows_bf16(&tk, kr, sh.d, sh.H, rows, 128) ||
      !tmap_token_rows_bf16(&tv, v, sh.d, sh.H, rows, 128))
    return cudaErrorInvalidValue;
  const int nchunks = (sh.F + chunk - 1) / chunk;
  const int tiles = (int)(((long long)chunk * sh.S + 127) / 128);
  if ((long long)sh.B * sh.H > 65535) return cudaErrorInvalidConfiguration;
  const size_t smem = sizeof(WsoftSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_wsoft_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(nchunks * tiles), (unsigned)((long long)sh.B * sh.H));
  k_wsoft_tc<<<grid, kTcThreads, smem, stream>>>(tq, tk, tv, sh.H, sh.F, sh.S, chunk, radius, tiles,
                                                 scale * kLog2e, accumulate, static_cast<__nv_bfloat16*>(out),
                                                 status);
  return cudaGetLastError();
}

}  // namespace vdn
