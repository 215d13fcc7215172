// Deterministic combine of the split-N state partials.
//
// For head bh the contributing CTAs are c_lo .. c_hi of the state partition;
// their partials sit in slots c + bh.  The combined state is
//   S = (((S_in + P_{c_lo}) + P_{c_lo+1}) + ... ) + P_{c_hi}
// in that fixed order (S_in = 0 for the bidirectional call, the carried state
// for a block-causal step), so the result does not depend on scheduling.
//
// One cluster of kCombineCluster CTAs handles one head; each CTA sums a slice
// of S.  combine_bulk_kernel brings all of its slices in at once by bulk
// copies (tensor path, heads of up to kCombineBulkSlots slots);
// combine_kernel loads them into registers a few slots per round.  Both add
// in the order above.  For the tensor read-out they also write the fp16 image
// of S that the read-out copies into shared memory as its B operand: two K-blocks
// of [128 rows][64 columns], rows of 128 bytes, 16-byte chunks XOR-swizzled by
// (row & 7) -- the canonical K-major 128-byte-swizzle layout of tcgen05.  The
// image is S * 2^e with one power of two per head, chosen from the head's
// largest |S| (exchanged across the cluster through distributed shared
// memory) so that it lands in [2^13, 2^14): every entry that matters is a
// normal fp16 number with full fp16 precision.  S_scale[bh][0] = 2^e.
#pragma once

#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace gla {

constexpr int kCombineCluster = 8;
constexpr int kMaxZPartsCombined = 4 * kCombineCluster;   // z partials per slot it can add
constexpr int kCombineThreads = 256;   // >= d, so one thread per z element

struct CombineParams {
  Partition part;
  int d;
  int zparts;            // z partials per slot (summed in index order)
  const float* part_S;   // [slots][d][d]
  const float* part_z;   // [slots][zparts][d]
  const float* S_in;     // optional carried state (may alias S_out)
  const float* z_in;     // optional carried key sum (may alias z_out)
  float* S_out;          // optional [BH][d][d] (null: only the image is needed)
  int chunked;           // partials in the tensor path's chunk-major layout (d = 128)
  float* z_out;          // [BH][d]
  __half* S_img;         // optional [BH][128*128] swizzled fp16 image (d = 128)
  float* S_scale;        // [BH][4]: [0] = scale of the image
};

// Byte offset of S[a][c] (a = row = output feature, c = reduction index) in
// the swizzled image of a 128 x 128 16-bit matrix.
__host__ __device__ inline uint32_t simg_offset(int a, int c) {
  const int kb = c >> 6;
  const int byte_in_row = (c & 63) * 2;
  const int chunk = byte_in_row >> 4;
  return (uint32_t)(kb * 16384 + a * 128 + (((chunk ^ (a & 7)) << 4) | (byte_in_row & 15)));
}

// Row-major offset S[a][c] of partial element e.  The tensor path drains its
// accumulator chunk-major (8 columns of all 128 rows after another, so that a
// warp's stores are contiguous): e = (c/8 * 128 + a) * 8 + c%8.
__device__ __forceinline__ int row_major(const CombineParams& p, int e) {
  if (!p.chunked) return e;
  return ((e >> 3) & 127) * 128 + ((e >> 10) << 3) + (e & 7);
}

__device__ __forceinline__ void add4(float4& s, const float4 t) {
  s.x += t.x; s.y += t.y; s.z += t.z; s.w += t.w;
}

// The part both combine kernels share, from the summed slice on: S_out, the
// head maximum and z through one exchange in distributed shared memory, the
// image scale and the fp16 image of this rank's slice.
__device__ __forceinline__ void combine_finish(const CombineParams& p,
                                               cooperative_groups::cluster_group& cluster,
                                               int bh, int rank, const float4 (&acc)[2],
                                               const bool (&live)[2], float zacc) {
  __shared__ float red[kCombineThreads / 32];
  const int d = p.d;
  const size_t dd = (size_t)d * d;
  const int chunk = (int)(dd / kCombineCluster);
  const int e_base = rank * chunk;
  const bool zlive = (int)threadIdx.x < d;
  float m = 0.f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    if (!live[k]) continue;
    const int e = e_base + 4 * threadIdx.x + 4 * kCombineThreads * k;
    if (p.S_out) *reinterpret_cast<float4*>(p.S_out + bh * dd + row_major(p, e)) = acc[k];
    m = fmaxf(m, fmaxf(fmaxf(fabsf(acc[k].x), fabsf(acc[k].y)),
                       fmaxf(fabsf(acc[k].z), fabsf(acc[k].w))));
  }

  // One exchange through distributed shared memory and one cluster barrier:
  // every rank stores its z sums into rank 0's zsum_all[rank] and its |S|
  // maximum into every rank's max_all[rank]; then rank 0 adds the z sums in
  // rank order and each rank takes the head maximum from its own copy.  No
  // rank touches another's shared memory after the barrier, so any may exit.
  __shared__ float zsum_all[kCombineCluster][128];
  __shared__ float max_all[kCombineCluster];
  if (zlive) *cluster.map_shared_rank(&zsum_all[rank][threadIdx.x], 0) = zacc;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < kCombineCluster) {
    float mm = red[0];
    for (int w = 1; w < kCombineThreads / 32; ++w) mm = fmaxf(mm, red[w]);
    *cluster.map_shared_rank(&max_all[rank], (int)threadIdx.x) = mm;
  }
  cluster.sync();
  if (rank == 0 && zlive) {
    float zs = p.z_in ? p.z_in[(size_t)bh * d + threadIdx.x] : 0.f;
    for (int r = 0; r < kCombineCluster; ++r) zs += zsum_all[r][threadIdx.x];
    p.z_out[(size_t)bh * d + threadIdx.x] = zs;
  }
  float hm = 0.f;
  if (p.S_img != nullptr)
    for (int r = 0; r < kCombineCluster; ++r) hm = fmaxf(hm, max_all[r]);

  if (p.S_img == nullptr) return;     // uniform over the whole grid

  // hm = f * 2^E with f in [0.5, 1): scale by 2^(14 - E).
  int E = (int)((__float_as_uint(hm) >> 23) & 0xFFu) - 126;
  if (hm == 0.f || E < -100) E = -100;
  if (E > 140) E = 140;
  const float sc = __uint_as_float((uint32_t)(127 + 14 - E) << 23);
  if (rank == 0 && threadIdx.x == 0) {
    p.S_scale[(size_t)bh * 4 + 0] = sc;
    p.S_scale[(size_t)bh * 4 + 1] = 0.f;
    p.S_scale[(size_t)bh * 4 + 2] = 0.f;
    p.S_scale[(size_t)bh * 4 + 3] = 0.f;
  }
  unsigned char* img = reinterpret_cast<unsigned char*>(p.S_img + bh * dd);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = e_base + 4 * threadIdx.x + 4 * kCombineThreads * k;
    if (e >= e_base + chunk) continue;
    const int rm = row_major(p, e);
    const int a = rm / d, cc = rm % d;
    __half2 lo = __floats2half2_rn(acc[k].x * sc, acc[k].y * sc);
    __half2 hi = __floats2half2_rn(acc[k].z * sc, acc[k].w * sc);
    uint2 pk;   // cc .. cc+3 stay inside one 16-byte chunk (cc is a multiple of 4)
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(img + simg_offset(a, cc)) = pk;
  }
}

__global__ void __cluster_dims__(kCombineCluster, 1, 1) __launch_bounds__(kCombineThreads)
    combine_kernel(CombineParams p) {
  namespace cg = cooperative_groups;
  // Launched as a programmatic dependent of the state reduction: wait for its
  // partials, and let the read-out kernel start its own prologue meanwhile.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cg::cluster_group cluster = cg::this_cluster();

  const int bh = blockIdx.y;
  const int rank = (int)cluster.block_rank();
  const int d = p.d;
  const long long tph = p.part.tiles_per_head;
  const int c_lo = part_cta_of(p.part, (long long)bh * tph);
  const int c_hi = part_cta_of(p.part, (long long)(bh + 1) * tph - 1);
  const size_t dd = (size_t)d * d;
  const int chunk = (int)(dd / kCombineCluster);        // 2048 for d = 128
  const int e_base = rank * chunk;

  // Each thread owns up to two float4 groups of S (e = e_base + 4*tid + 1024*k)
  // and, for d <= 128, one element e = tid of the z partials this rank adds
  // (partials rank, rank + 8, ... of each slot).  All loads of a batch of
  // slots are issued before any is added, then added in slot order.
  constexpr int kBatch = 4;
  float4 acc[2];
  float zacc = 0.f;
  bool live[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = e_base + 4 * threadIdx.x + 4 * kCombineThreads * k;
    live[k] = e < e_base + chunk;
    acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (live[k] && p.S_in)
      acc[k] = *reinterpret_cast<const float4*>(p.S_in + bh * dd + row_major(p, e));
  }
  const bool zlive = (int)threadIdx.x < d;
  for (int c0 = c_lo; c0 <= c_hi; c0 += kBatch) {
    float4 t[kBatch][2];
    float zt[kBatch][4];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int c = c0 + b;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = e_base + 4 * threadIdx.x + 4 * kCombineThreads * k;
        t[b][k] = (c <= c_hi && live[k])
                      ? *reinterpret_cast<const float4*>(p.part_S + ((size_t)c + bh) * dd + e)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int zp = rank + kCombineCluster * q;
        zt[b][q] = (c <= c_hi && zlive && zp < p.zparts)
                       ? p.part_z[(((size_t)c + bh) * p.zparts + zp) * d + threadIdx.x]
                       : 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      if (c0 + b > c_hi) break;
      add4(acc[0], t[b][0]);
      add4(acc[1], t[b][1]);
      zacc += zt[b][0]; zacc += zt[b][1]; zacc += zt[b][2]; zacc += zt[b][3];
    }
  }
  combine_finish(p, cluster, bh, rank, acc, live, zacc);
}

// The same combine with every partial of the head brought in at once: one
// warp issues bulk copies of each slot's slice of S (8 KB) and of the z
// partials this rank adds into shared memory, all completing on one mbarrier,
// so the loads take one round trip however many slots the head has.  The
// sums then run from shared memory in the same order as combine_kernel's, so
// the two kernels give the same bits.  For the tensor path's chunk-major
// partials (d = 128) and heads of at most kCombineBulkSlots slots.
constexpr int kCombineBulkSlots = 20;
constexpr uint32_t kCombineSliceBytes = 128 * 128 / kCombineCluster * 4;   // 8 KB
constexpr uint32_t kCombineZBytes = 128 * 4;                                // one z partial

inline size_t combine_bulk_smem(int slots) {
  return (size_t)slots * (kCombineSliceBytes + 4 * kCombineZBytes);
}

__global__ void __cluster_dims__(kCombineCluster, 1, 1) __launch_bounds__(kCombineThreads)
    combine_bulk_kernel(CombineParams p) {
  namespace cg = cooperative_groups;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(128) unsigned char cb_smem[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;

  const int bh = blockIdx.y;
  const int rank = (int)cluster.block_rank();
  const long long tph = p.part.tiles_per_head;
  const int c_lo = part_cta_of(p.part, (long long)bh * tph);
  const int c_hi = part_cta_of(p.part, (long long)(bh + 1) * tph - 1);
  const int nslots = c_hi - c_lo + 1;
  const size_t dd = 128 * 128;
  const int e_base = rank * (int)(dd / kCombineCluster);
  float* sl = reinterpret_cast<float*>(cb_smem);                       // [slot][2048]
  float* zs = sl + (size_t)nslots * (kCombineSliceBytes / 4);          // [slot][4][128]
  int nq = 0;   // z partials this rank adds per slot: rank, rank + 8, ...
  for (int q = 0; q < 4; ++q)
    if (rank + kCombineCluster * q < p.zparts) nq = q + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    if (threadIdx.x == 0)
      mbar_arrive_expect_tx(&bar, (uint32_t)nslots * (kCombineSliceBytes + nq * kCombineZBytes));
    __syncwarp();
    for (int i = threadIdx.x; i < nslots; i += 32) {
      const size_t slot = (size_t)c_lo + i + bh;
      bulk_load(sl + (size_t)i * (kCombineSliceBytes / 4), p.part_S + slot * dd + e_base,
                kCombineSliceBytes, &bar);
      for (int q = 0; q < nq; ++q)
        bulk_load(zs + ((size_t)i * 4 + q) * 128,
                  p.part_z + (slot * p.zparts + rank + kCombineCluster * q) * 128,
                  kCombineZBytes, &bar);
    }
  }

  float4 acc[2];
  const bool live[2] = {true, true};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = e_base + 4 * threadIdx.x + 4 * kCombineThreads * k;
    acc[k] = p.S_in ? *reinterpret_cast<const float4*>(p.S_in + bh * dd + row_major(p, e))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float zacc = 0.f;
  if (mbar_wait(&bar, 0u, &abort_flag)) {
    for (int i = 0; i < nslots; ++i) {
      const float* si = sl + (size_t)i * (kCombineSliceBytes / 4);
#pragma unroll
      for (int k = 0; k < 2; ++k)
        add4(acc[k], *reinterpret_cast<const float4*>(si + 4 * threadIdx.x + 4 * kCombineThreads * k));
      if (threadIdx.x < 128)
        for (int q = 0; q < nq; ++q) zacc += zs[((size_t)i * 4 + q) * 128 + threadIdx.x];
    }
  } else {
    // Timed out (recorded in the device error word): let the copies land
    // before this CTA's shared memory is released; the result is void.
    int dummy = 0;
    mbar_wait(&bar, 0u, reinterpret_cast<volatile int*>(&dummy));
  }
  combine_finish(p, cluster, bh, rank, acc, live, zacc);
}

}  // namespace gla
