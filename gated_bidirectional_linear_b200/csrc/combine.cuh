// Deterministic combine of the split-N state partials.
//
// For head bh the contributing CTAs are c_lo .. c_hi of the state partition;
// their partials sit in slots c + bh.  The combined state is
//   S = (((S_in + P_{c_lo}) + P_{c_lo+1}) + ... ) + P_{c_hi}
// in that fixed order (S_in = 0 for the bidirectional call, the carried state
// for a block-causal step), so the result does not depend on scheduling.
// Besides S (fp32) the kernel can write the fp16 image of S that the tensor
// read-out kernel copies into shared memory as its B operand: two K-blocks of
// [d rows][64 columns], rows of 128 bytes, 16-byte chunks XOR-swizzled by
// (row & 7) - the canonical K-major 128-byte-swizzle layout of tcgen05.
// Row a of the image holds S[a][:] * 2^e_a with e_a chosen so the row's
// largest magnitude lands in [2^13, 2^14) (far inside the fp16 range, full
// fp16 precision for the entries that matter); S_rs[a] = 2^-e_a undoes it in
// the read-out epilogue.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace gla {

struct CombineParams {
  Partition part;
  int d;
  int zparts;            // z partials per slot (summed in index order)
  const float* part_S;   // [slots][d][d]
  const float* part_z;   // [slots][zparts][d]
  const float* S_in;     // optional carried state (may alias S_out)
  const float* z_in;     // optional carried key sum (may alias z_out)
  float* S_out;          // [BH][d][d]
  float* z_out;          // [BH][d]
  __half* S_img;         // optional [BH][d*d] swizzled fp16 image (d = 128)
  float* S_rs;           // [BH][d] inverse row scales of the image
};

constexpr int kCombineThreads = 256;
constexpr int kCombineElems = 1024;  // state elements per CTA

// Byte offset of S[a][c] (a = row = output feature, c = reduction index) in
// the swizzled image of a 128 x 128 16-bit matrix.
__host__ __device__ inline uint32_t simg_offset(int a, int c) {
  const int kb = c >> 6;
  const int byte_in_row = (c & 63) * 2;
  const int chunk = byte_in_row >> 4;
  return (uint32_t)(kb * 16384 + a * 128 + (((chunk ^ (a & 7)) << 4) | (byte_in_row & 15)));
}

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineParams p) {
  const int bh = blockIdx.y;
  const int d = p.d;
  const long long tph = p.part.tiles_per_head;
  const int c_lo = part_cta_of(p.part, (long long)bh * tph);
  const int c_hi = part_cta_of(p.part, (long long)(bh + 1) * tph - 1);
  const size_t dd = (size_t)d * d;
  const int e0 = blockIdx.x * kCombineElems;

  for (int e = e0 + threadIdx.x * 4; e < e0 + kCombineElems && e < (int)dd; e += kCombineThreads * 4) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p.S_in) s = *reinterpret_cast<const float4*>(p.S_in + bh * dd + e);
    for (int c = c_lo; c <= c_hi; ++c) {
      const float4 t = *reinterpret_cast<const float4*>(p.part_S + ((size_t)c + bh) * dd + e);
      s.x += t.x; s.y += t.y; s.z += t.z; s.w += t.w;
    }
    *reinterpret_cast<float4*>(p.S_out + bh * dd + e) = s;
    if (p.S_img) {
      // One warp holds one full row (d = 128: 32 threads x 4 elements).
      float m = fmaxf(fmaxf(fabsf(s.x), fabsf(s.y)), fmaxf(fabsf(s.z), fabsf(s.w)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      // m = f * 2^E, f in [0.5, 1): scale by 2^(14 - E).
      int E = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 126;
      if (m == 0.f || E < -100) E = -100;
      if (E > 140) E = 140;
      const float sc = __uint_as_float((uint32_t)(127 + 14 - E) << 23);
      const int a = e / d, cc = e % d;
      if ((threadIdx.x & 31) == 0) p.S_rs[(size_t)bh * d + a] = __uint_as_float((uint32_t)(127 - 14 + E) << 23);
      unsigned char* img = reinterpret_cast<unsigned char*>(p.S_img + bh * dd);
      __half2 lo = __floats2half2_rn(s.x * sc, s.y * sc);
      __half2 hi = __floats2half2_rn(s.z * sc, s.w * sc);
      // c .. c+3 stay inside one 16-byte chunk (c is a multiple of 4).
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(img + simg_offset(a, cc)) = pk;
    }
  }
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e < d; e += kCombineThreads) {
      float s = p.z_in ? p.z_in[(size_t)bh * d + e] : 0.f;
      for (int c = c_lo; c <= c_hi; ++c)
        for (int zp = 0; zp < p.zparts; ++zp)
          s += p.part_z[(((size_t)c + bh) * p.zparts + zp) * d + e];
      p.z_out[(size_t)bh * d + e] = s;
    }
  }
}

}  // namespace gla
