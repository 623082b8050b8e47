// Operand images for tcgen05.mma: a 128 x 128 matrix stored as bf16 "hi" and
// "lo" halves (x = hi + lo + O(2^-17 |x|)) in the K-major, 128-byte-swizzled
// canonical layout, so a kernel can bring it into shared memory with one bulk
// copy and hand it to the tensor cores unchanged.
//
// Image of X (row n = N index, column k = K index), 64 KB:
//   byte(part, n, k) = part * 32768 + (k / 64) * 16384 + n * 128
//                      + (((k % 64) / 8) ^ (n % 8)) * 16 + (k % 8) * 2
// part 0 = hi, part 1 = lo.  Within each 16 KB K-half the rows sit 128 bytes
// apart and groups of 8 rows 1024 bytes apart (the descriptor's stride offset).
#pragma once

#include <stdint.h>
#include <cuda_bf16.h>

namespace vdn {

constexpr int kImgBytes = 2 * 128 * 128 * 2;   // hi + lo

__host__ __device__ __forceinline__ uint32_t img_offset(int part, int n, int k) {
  return part * 32768u + (k >> 6) * 16384u + n * 128u + ((((k & 63) >> 3) ^ (n & 7)) << 4) + (k & 7) * 2u;
}

// Read-out operand image of W_t: one fp16 part in the same layout (32 KB), each
// block of 32 rows b scaled by 2^-e_b so its largest entry lies in [0.5, 1)
// (e_b stored beside the image; power-of-two scaling is exact).  fp16 keeps 11
// significant bits against 8 for bf16, which the read-out's RMSNorm needs when
// a dominant component of W_t cancels in W_t q'.
constexpr int kWImgBytes = 128 * 128 * 2;
constexpr int kWRowBlocks = 4;
constexpr int kWBlockRows = 128 / kWRowBlocks;

__device__ __forceinline__ void store_chunk_f16(uint8_t* img, int n, int k, const float* v) {
  uint32_t hw[4];
#pragma unroll
  for (int e = 0; e < 8; e += 2) asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(hw[e / 2]) : "f"(v[e + 1]), "f"(v[e]));
  *reinterpret_cast<uint4*>(img + img_offset(0, n, k)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
}

__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// Writes the image of a 128x128 fp32 matrix held in shared memory with leading
// dimension ld.  Element (n, k) of the image is src[n*ld + k], or src[k*ld + n]
// when `transposed`.  All threads of the block take part.
__device__ __forceinline__ void write_image128(const float* src, int ld, bool transposed, uint16_t* img) {
  uint4* dst = reinterpret_cast<uint4*>(img);
  for (int idx = threadIdx.x; idx < 128 * 16; idx += blockDim.x) {
    int n = idx >> 4, c = idx & 15;
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      int k = 8 * c + e;
      float x0 = transposed ? src[k * ld + n] : src[n * ld + k];
      float x1 = transposed ? src[(k + 1) * ld + n] : src[n * ld + k + 1];
      __nv_bfloat16 h0, l0, h1, l1;
      split_bf16(x0, h0, l0);
      split_bf16(x1, h1, l1);
      hw[e / 2] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lw[e / 2] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
    }
    uint32_t off = img_offset(0, n, 8 * c) >> 4;
    dst[off] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    dst[off + 2048] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

}  // namespace vdn
