// Bidirectional scan of the delta rule on the tensor cores (page sections
// "Step 3" and "Step 4": the forward prefix scan and backward suffix scan over
// frames, each seeded with 0.5 x the text state).
//
// One CTA per (batch, head, direction) walks the frames serially:
//     X_f = S_{f-1} D_f + cpre B_f            (fp32, two threads per state row)
//     S_f = X_f N_f + cpost B_f               (tcgen05, 128x128x128)
// The product runs in bf16 with hi/lo splitting of both operands
// (X = Xh + Xl, N = Nh + Nl; D = Xh Nl + Xh Nh + Xl Nh), which keeps about 16
// significant bits in every term and accumulates in fp32 in TMEM, so the state
// stays an fp32 quantity at tensor-core speed.  N_f arrives as a pre-swizzled
// operand image (written by the per-frame solve) through bulk copies, its hi and
// lo halves on barriers of their own: the Xh Nl terms run first, so the next
// frame's N_lo can be requested a third of the way into the product (by a thread
// other than the one issuing the MMAs, which stays blocked in the MMA queue).
// B_f comes through TMA with a 128-byte swizzle so that each thread reads its own
// row without bank conflicts.  Only the states the window gather needs are
// stored: P at chunk ends, Q at chunk starts (or every frame for the debug
// export), staged in the free X buffers and written by TMA store.
//
// Segment mode (frame sharding): the state restarts at every chunk, from zero
// with the rule's own coefficients (the chunk's offset O_c) or from the identity
// with cpre = cpost = 0 (the chunk's linear part G_c = prod D_f N_f), and the
// state at the chunk's last step in scan order is stored with its block
// exponent as the chunk's affine map S -> S G_c + O_c.
#include "common.cuh"
#include "image.cuh"
#include "internal.h"
#include "tc.cuh"
#include "tmap.h"

namespace vdn {

namespace {

struct __align__(1024) ScanSmem {
  uint8_t aop[2][32768];     // X hi, X lo: K-major SW128 A operands
  uint8_t nimg[65536];       // N_f hi | lo image
  float bf[4][128 * 32];     // B_f, four swizzled [128 rows][32 cols] boxes
  float alpha[128];
  uint64_t bar_n[2], bar_b, bar_mma, bar_nlo;   // bar_n[part]: N_f hi / lo landed; bar_nlo: N_lo read
  uint32_t tmem_base;
  int abort;
};

constexpr uint32_t kIdesc = tc::idesc_bf16_f32(128, 128, false, false);

// byte offset of B_f[row][col] inside the swizzled box array
__device__ __forceinline__ uint32_t bf_offset(int row, int col) {
  int box = col >> 5, c16 = (col & 31) >> 2;
  return box * 16384 + row * 128 + ((c16 ^ (row & 7)) << 4) + (col & 3) * 4;
}

}  // namespace

// Two threads per state row: thread t owns row m = 32 (warp % 4) + lane (the
// TMEM lane quarter its warp may read) and columns 64 ch .. 64 ch + 63, ch = t / 128.
constexpr int kScanThreads = 256;

// bf16 hi/lo split of a pair: hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split_pair(float2 x, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(x.x, x.y);
  const float2 hf = make_float2(bf16lo(hi), bf16hi(hi));
  const float2 r = __fadd2_rn(x, make_float2(-hf.x, -hf.y));
  lo = pack_bf16x2(r.x, r.y);
}

// kMode: kScanWhole (the clip, from the text seed) or a segment mode; a template parameter so that
// the whole-clip instantiation carries none of the segment mode's work
template <int kMode>
__global__ void __launch_bounds__(kScanThreads, 1) k_scan_tc(const __grid_constant__ CUtensorMap tmB,
                                                            const __grid_constant__ CUtensorMap tmP,
                                                            const __grid_constant__ CUtensorMap tmQ,
                                                            const uint16_t* __restrict__ nimg_g,
                                                            const float* __restrict__ alpha,
                                                            const float* __restrict__ text, RuleCoef rc,
                                                            float* __restrict__ P, float* __restrict__ Q,
                                                            int* __restrict__ pexp, int* __restrict__ qexp, int H,
                                                            int F, int chunk, int all_frames,
                                                            float* __restrict__ maps, int* __restrict__ map_exp,
                                                            int nch_stride, uint32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  ScanSmem& sm = tc::smem_align<ScanSmem>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int m = 32 * (warp & 3) + lane;     // state row (v channel) = TMEM lane
  const int ch = tid >> 7;                   // column half
  const int k0 = 64 * ch;
  const int dir = blockIdx.x & 1;
  const long long bh = blockIdx.x >> 1;
  const int h = (int)(bh % H);
  const long long b = bh / H;
  volatile int* abort_flag = &sm.abort;

  if (tid == 0) {
    tc::mbar_init(&sm.bar_n[0], 1);
    tc::mbar_init(&sm.bar_n[1], 1);
    tc::mbar_init(&sm.bar_b, 1);
    tc::mbar_init(&sm.bar_mma, 1);
    tc::mbar_init(&sm.bar_nlo, 1);
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

  float2 s[32];   // s[p] = state[m][k0 + 2p .. k0 + 2p + 1]
  {
    const float* T = text ? text + ((long long)h * 128 + m) * 128 + k0 : nullptr;
#pragma unroll
    for (int p = 0; p < 32; p += 2) {   // the text state is 16-byte aligned (checked on entry)
      const float4 t4 = T ? *reinterpret_cast<const float4*>(T + 2 * p) : make_float4(0.f, 0.f, 0.f, 0.f);
      s[p] = make_float2(kTextStateScale * t4.x, kTextStateScale * t4.y);
      s[p + 1] = make_float2(kTextStateScale * t4.z, kTextStateScale * t4.w);
    }
  }

  auto frame_of = [&](int step) { return dir == 0 ? step : F - 1 - step; };
  // segment mode: first and last frame of a chunk in this direction's order
  auto seg_first = [&](int f) { return dir == 0 ? f % chunk == 0 : ((f + 1) % chunk == 0 || f == F - 1); };
  auto seg_last = [&](int f) { return dir == 0 ? ((f + 1) % chunk == 0 || f == F - 1) : f % chunk == 0; };
  // N_f image: the hi part (first 32 KB) and the lo part each land on their own
  // barrier and are requested as soon as their buffer is free
  auto load_n_part = [&](int step, int part) {
    long long fi = bh * F + frame_of(step);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(nimg_g + fi * (kImgBytes / 2)) + part * 32768;
    tc::mbar_arrive_expect_tx(&sm.bar_n[part], kImgBytes / 2);
#pragma unroll
    for (int j = 0; j < 2; ++j)
      tc::bulk_load(sm.nimg + part * 32768 + j * 16384, src + j * 16384, 16384, &sm.bar_n[part]);
  };
  auto load_b = [&](int step) {
    long long fi = bh * F + frame_of(step);
    tc::mbar_arrive_expect_tx(&sm.bar_b, 65536);
#pragma unroll
    for (int j = 0; j < 4; ++j) tc::tma_load_2d(&tmB, &sm.bar_b, sm.bf[j], 32 * j, (int)(fi * 128));
  };
  auto prefetch = [&](int step) {   // next frame's operands into L2 (hint only)
    long long fi = bh * F + frame_of(step);
    tc::prefetch_l2(reinterpret_cast<const uint8_t*>(nimg_g + fi * (kImgBytes / 2)), kImgBytes);
  };
  if (tid == 0) {
    load_n_part(0, 0);
    load_n_part(0, 1);
    load_b(0);
    if (F > 1) prefetch(1);
  }

  const bool early_b = rc.cpost == 0.f;   // B_f is only read before the product
  uint32_t ph = 0;
  const uint32_t a_hi = tc::smem_u32(sm.aop[0]), a_lo = tc::smem_u32(sm.aop[1]);
  const uint32_t n_hi = tc::smem_u32(sm.nimg), n_lo = n_hi + 32768;
  const uint8_t* bfb = reinterpret_cast<const uint8_t*>(sm.bf);

  int ex = 0;   // block exponent: the true state is 2^ex s
  float a_next = tid < 128 ? alpha[((b * F + frame_of(0)) * H + h) * 128 + tid] : 0.f;
  for (int step = 0; step < F; ++step) {
    const int f = frame_of(step);
    const long long fi = bh * F + f;
    if (kMode != kScanWhole && seg_first(f)) {   // restart: zero, or the identity
#pragma unroll
      for (int p = 0; p < 32; ++p)
        s[p] = kMode == kScanSegIdentity ? make_float2(k0 + 2 * p == m ? 1.f : 0.f, k0 + 2 * p + 1 == m ? 1.f : 0.f)
                                         : make_float2(0.f, 0.f);
      ex = 0;
    }
    const float cpre = ldexpf(rc.cpre, -ex), cpost = ldexpf(rc.cpost, -ex);
    if (tid < 128) {
      sm.alpha[tid] = a_next;
      if (step + 1 < F) a_next = alpha[((b * F + frame_of(step + 1)) * H + h) * 128 + tid];   // used next step
    }
    if (tid == 0 && step + 2 < F) prefetch(step + 2);
    if (tid == 0) tc::bulk_wait_read_all();   // a state store still reading the X buffers
    __syncthreads();
    if (!tc::mbar_wait(&sm.bar_b, ph, abort_flag, status)) break;

    // X = S D + cpre B  ->  bf16 hi / lo A operands (row m, columns k0 .. k0 + 63)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int k = k0 + 8 * c;
      const float4 al0 = *reinterpret_cast<const float4*>(&sm.alpha[k]);
      const float4 al1 = *reinterpret_cast<const float4*>(&sm.alpha[k + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(bfb + bf_offset(m, k));
      const float4 b1 = *reinterpret_cast<const float4*>(bfb + bf_offset(m, k + 4));
      const float2 cp = make_float2(cpre, cpre);
      float2 x[4];
      x[0] = __ffma2_rn(s[4 * c + 0], make_float2(al0.x, al0.y), __fmul2_rn(cp, make_float2(b0.x, b0.y)));
      x[1] = __ffma2_rn(s[4 * c + 1], make_float2(al0.z, al0.w), __fmul2_rn(cp, make_float2(b0.z, b0.w)));
      x[2] = __ffma2_rn(s[4 * c + 2], make_float2(al1.x, al1.y), __fmul2_rn(cp, make_float2(b1.x, b1.y)));
      x[3] = __ffma2_rn(s[4 * c + 3], make_float2(al1.z, al1.w), __fmul2_rn(cp, make_float2(b1.z, b1.w)));
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) split_pair(x[q], hw[q], lw[q]);
      const uint32_t off = img_offset(0, m, k);
      *reinterpret_cast<uint4*>(sm.aop[0] + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sm.aop[1] + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    if (tid == 0) {
      if (early_b && step + 1 < F) load_b(step + 1);
      // Xh Nl first: N_lo is free a third of the product in, and the next frame's
      // N_lo loads meanwhile; the next frame's N_hi, requested once the whole
      // product is done, has until after that frame's Xh Nl terms
      if (tc::mbar_wait(&sm.bar_n[1], ph, abort_flag, status)) {
        tc::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::umma_bf16(tmem, tc::smem_desc(a_hi + koff, 16, 1024), tc::smem_desc(n_lo + koff, 16, 1024), kIdesc,
                        kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(&sm.bar_nlo);
        if (tc::mbar_wait(&sm.bar_n[0], ph, abort_flag, status)) {
          tc::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
            uint64_t ah = tc::smem_desc(a_hi + koff, 16, 1024), al = tc::smem_desc(a_lo + koff, 16, 1024);
            uint64_t bhd = tc::smem_desc(n_hi + koff, 16, 1024);
            tc::umma_bf16(tmem, ah, bhd, kIdesc, 1u);
            tc::umma_bf16(tmem, al, bhd, kIdesc, 1u);
          }
          tc::umma_commit(&sm.bar_mma);
        }
      }
    } else if (tid == 32 && step + 1 < F) {
      // the copies are requested by a thread of their own: the issuing thread stays
      // blocked in the MMA queue until its last product is accepted
      if (tc::mbar_wait(&sm.bar_nlo, ph, abort_flag, status)) load_n_part(step + 1, 1);
    }
    if (!tc::mbar_wait(&sm.bar_mma, ph, abort_flag, status)) break;
    tc::tc_fence_after();
    if (tid == 32 && step + 1 < F) load_n_part(step + 1, 0);   // the product that read N_hi is complete

    // S_f = X_f N_f (the TMEM accumulator) + cpost B_f
    const bool seg_store = kMode != kScanWhole && seg_last(f);
    const bool store = kMode == kScanWhole && (all_frames || (dir == 0 ? ((f + 1) % chunk == 0) : (f % chunk == 0)));
    // whole clip: the stored state goes out through the (now free) X buffers and a TMA
    // store, row-major and coalesced, in the swizzled [rows][32 cols] boxes of bf_offset
    uint8_t* stage = sm.aop[0];
    // segment mode: map slot [b, h][dir][chunk][G_c | O_c][row][col]; the map is 2^ex times the stored state
    const long long mslot = ((bh * 2 + dir) * nch_stride + f / chunk) * 2 + (kMode == kScanSegIdentity ? 0 : 1);
    float* mdst = kMode == kScanWhole ? nullptr : maps + (mslot * 128 + m) * 128 + k0;
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t r[32];
      tc::tmem_ld32(t_row + 32 * j, r);
      tc::tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const int p = 16 * j + e / 2;
        // with early_b the buffer already receives B_{f+1}: do not read it
        const float4 bv = early_b ? make_float4(0.f, 0.f, 0.f, 0.f)
                                  : *reinterpret_cast<const float4*>(bfb + bf_offset(m, k0 + 32 * j + e));
        const float2 cq = make_float2(cpost, cpost);
        s[p] = __ffma2_rn(cq, make_float2(bv.x, bv.y), make_float2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])));
        s[p + 1] = __ffma2_rn(cq, make_float2(bv.z, bv.w),
                              make_float2(__uint_as_float(r[e + 2]), __uint_as_float(r[e + 3])));
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(s[p].x), fabsf(s[p].y)), fmaxf(fabsf(s[p + 1].x), fabsf(s[p + 1].y))));
        if (store)
          *reinterpret_cast<float4*>(stage + bf_offset(m, k0 + 32 * j + e)) =
              make_float4(s[p].x, s[p].y, s[p + 1].x, s[p + 1].y);
        if (seg_store)
          *reinterpret_cast<float4*>(mdst + 32 * j + e) = make_float4(s[p].x, s[p].y, s[p + 1].x, s[p + 1].y);
      }
    }
    if (store && tid == 0) (dir == 0 ? pexp : qexp)[fi] = ex;
    if (seg_store && tid == 0) map_exp[mslot] = ex;
    if (store) tc::fence_proxy_async_smem();   // the staged rows, before the barrier and the TMA store
    tc::tc_fence_before();
    // accumulator and B_f reads done, alpha slot free; rescale if any entry passed
    // kRenormAbove (2^32)
    if (__syncthreads_or(amax > kRenormAbove)) {
#pragma unroll
      for (int p = 0; p < 32; ++p) s[p] = __fmul2_rn(s[p], make_float2(kRenormScale, kRenormScale));
      ex += kRenormExp;
    }
    if (store && tid == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) tc::tma_store_2d(dir == 0 ? &tmP : &tmQ, stage + j * 16384, 32 * j, (int)(fi * 128));
      tc::bulk_commit();
    }
    if (tid == 0 && !early_b && step + 1 < F) load_b(step + 1);
    ph ^= 1;
  }

  // teardown: make sure no copy or product of ours is still in flight
  if (tid == 0) tc::bulk_wait_all();
  __syncthreads();
  if (sm.abort && tid == 0) {
    tc::mbar_wait(&sm.bar_n[0], ph, abort_flag, nullptr);
    tc::mbar_wait(&sm.bar_n[1], ph, abort_flag, nullptr);
    tc::mbar_wait(&sm.bar_b, ph, abort_flag, nullptr);
  }
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

cudaError_t launch_scan_tc(const Args& a, const float* Bsum, const uint16_t* nimg, float* P, float* Q, int* pexp,
                           int* qexp, bool all_frames, uint32_t* status, int seg_mode, float* maps, int* map_exp,
                           int nch_stride) {
  CUtensorMap tmB, tmP, tmQ;
  if (!tmap_rows_f32(&tmB, Bsum, a.NF() * 128)) return cudaErrorInvalidValue;
  // P / Q: [B H F][128][128] fp32 state stores (segment modes store maps directly: placeholders)
  if (!tmap_rows_f32(&tmP, P ? (const void*)P : (const void*)Bsum, a.NF() * 128) ||
      !tmap_rows_f32(&tmQ, Q ? (const void*)Q : (const void*)Bsum, a.NF() * 128))
    return cudaErrorInvalidValue;
  size_t smem = sizeof(ScanSmem) + 1024;
  cudaError_t e;
  RuleCoef rc = rule_coef(a.rule, a.c);
  if (seg_mode == kScanSegIdentity) rc.cpre = rc.cpost = 0.f;   // the linear part alone
  auto kern = seg_mode == kScanSegZero ? k_scan_tc<kScanSegZero>
              : seg_mode == kScanSegIdentity ? k_scan_tc<kScanSegIdentity> : k_scan_tc<kScanWhole>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(2LL * a.sh.B * a.sh.H), kScanThreads, smem, a.stream>>>(
      tmB, tmP, tmQ, nimg, a.alpha, a.text_state, rc, P, Q, pexp, qexp, a.sh.H, a.sh.F, a.chunk, all_frames ? 1 : 0, maps,
      map_exp, nch_stride, status);
  return cudaGetLastError();
}

}  // namespace vdn
