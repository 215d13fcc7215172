// bf16 GEMM on tcgen05 for the layer around the operator: C = A B^T with A
// [M][K] and B [N][K] row-major bf16 (K contiguous: both operands K-major),
// fp32 accumulation in TMEM.
//
//   gemm_kernel  persistent: each CTA walks 128 x 256 output tiles (N fastest,
//                so a band of A rows is reused from L2 across the N tiles while
//                all of B stays in L2).  Warp 0 streams 64-wide K slices of A
//                and B by TMA (128-byte swizzle) into a 4-stage ring, one thread
//                of warp 1 issues tcgen05.mma (M 128, N 256, K 16) into one of
//                two TMEM accumulators, and warps 2..5 (one per TMEM lane
//                quarter) drain the finished accumulator.
//
// Epilogues:
//   kGemmPlain   C [M][N] bf16, row stride N.
//   kGemmSplit   the operator's inputs straight from the projection: columns
//                [0, 4 HD) of the product go to q, k, v and g ([M][HD] each, HD
//                = heads * head_dim) and columns [4 HD, 4 HD + heads) to beta
//                [M][heads] after a sigmoid.
#pragma once

#include "ptx.cuh"
#include "tc.cuh"

namespace gla {

constexpr int kGmBM = 128, kGmBN = 256, kGmBK = 64;
constexpr int kGmStages = 4;
constexpr uint32_t kGmABytes = kGmBM * kGmBK * 2;     // 16 KB
constexpr uint32_t kGmBBytes = kGmBN * kGmBK * 2;     // 32 KB
constexpr uint32_t kGmStageBytes = kGmABytes + kGmBBytes;
constexpr int kGmThreads = 6 * 32;
enum { kGemmPlain = 0, kGemmSplit = 1 };

struct GemmParams {
  int M, N, K;
  int tiles_m, tiles_n;
  int mode;
  __nv_bfloat16* C;            // kGemmPlain
  __nv_bfloat16* dst[4];       // kGemmSplit: q, k, v, g
  __nv_bfloat16* beta;         // kGemmSplit
  int HD, heads;               // kGemmSplit
};

struct GemmSmem {
  static constexpr uint32_t RING = 0;
  static constexpr uint32_t BAR = kGmStages * kGmStageBytes;
  static constexpr uint32_t NBAR = 2 * kGmStages + 5;
  static constexpr uint32_t MISC = BAR + NBAR * 8;
  static constexpr uint32_t END = MISC + 16;
};

__device__ __forceinline__ void stg128_bf(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                GemmParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + GemmSmem::BAR);
  uint64_t* full = bars;
  uint64_t* empty = bars + kGmStages;
  uint64_t* accfull = bars + 2 * kGmStages;
  uint64_t* accempty = accfull + 2;
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + GemmSmem::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + GemmSmem::MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = p.tiles_m * p.tiles_n;
  const int kblocks = (p.K + kGmBK - 1) / kGmBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accfull[a], 1);
      mbar_init(&accempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      pdl_wait();   // A may be the previous kernel's output
      const uint64_t pol_a = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      RingPos<kGmStages> rp;
      int issued = 0;
      long long it = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int tm = t / p.tiles_n, tn = t - tm * p.tiles_n;
        for (int kb = 0; kb < kblocks; ++kb, rp.next(), ++it) {
          if (!mbar_wait(&empty[rp.s], rp.ph ^ 1u, abort_flag)) goto done;
          unsigned char* st = sm + GemmSmem::RING + rp.s * kGmStageBytes;
          mbar_arrive_expect_tx(&full[rp.s], kGmStageBytes);
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
              ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(st)),
              "l"(reinterpret_cast<uint64_t>(&tmA)), "r"(smem_u32(&full[rp.s])), "r"(kb * kGmBK),
              "r"(tm * kGmBM), "l"(pol_a)
              : "memory");
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
              ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(st + kGmABytes)),
              "l"(reinterpret_cast<uint64_t>(&tmB)), "r"(smem_u32(&full[rp.s])), "r"(kb * kGmBK),
              "r"(tn * kGmBN), "l"(pol_b)
              : "memory");
          ++issued;
        }
      }
    done:
      if (*abort_flag) {
        // Let the copies in flight land before shared memory is released.
        for (long long i2 = it - (issued < kGmStages ? issued : kGmStages); i2 < it; ++i2) {
          int dummy = 0;
          mbar_wait(&full[i2 % kGmStages], (uint32_t)((i2 / kGmStages) & 1),
                    reinterpret_cast<volatile int*>(&dummy));
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kGmBM, kGmBN, false, false);
      RingPos<kGmStages> rp;
      RingPos<2> ra;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ra.next()) {
        if (!mbar_wait(&accempty[ra.s], ra.ph ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)ra.s * kGmBN;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb, rp.next()) {
          if (!mbar_wait(&full[rp.s], rp.ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = sbase + GemmSmem::RING + rp.s * kGmStageBytes;
          const uint32_t b = a + kGmABytes;
#pragma unroll
          for (int kk = 0; kk < kGmBK / 16; ++kk)
            umma_f16kind(acc, sdesc_sw128(a + kk * 32, 16, 1024), sdesc_sw128(b + kk * 32, 16, 1024),
                         idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[rp.s]);
        }
        if (!ok) break;
        umma_commit(&accfull[ra.s]);
      }
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy));
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    RingPos<2> ra;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ra.next()) {
      if (!mbar_wait_warp(&accfull[ra.s], ra.ph, abort_flag)) break;
      tc_fence_after();
      const int tm = t / p.tiles_n, tn = t - tm * p.tiles_n;
      const int row = tm * kGmBM + q4 * 32 + lane;
      const bool rvalid = row < p.M;
      const uint32_t acc = tmem + (uint32_t)ra.s * kGmBN + lane_off;
#pragma unroll 1
      for (int ch = 0; ch < kGmBN / 32; ++ch) {
        float v[32];
        tmem_ld32(acc + ch * 32, v);
        tmem_wait_ld();
        const int col0 = tn * kGmBN + ch * 32;
        if (!rvalid || col0 >= p.N) continue;
        if (p.mode == kGemmSplit && col0 >= 4 * p.HD) {
          __nv_bfloat16* bd = p.beta + (size_t)row * p.heads;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int cb = col0 + i - 4 * p.HD;
            if (cb < p.heads) bd[cb] = __float2bfloat16_rn(1.f / (1.f + expf(-v[i])));
          }
          continue;
        }
        __nv_bfloat16* dst;
        if (p.mode == kGemmSplit) {
          const int seg = col0 / p.HD;
          dst = p.dst[seg] + (size_t)row * p.HD + (col0 - seg * p.HD);
        } else {
          dst = p.C + (size_t)row * p.N + col0;
        }
        if (col0 + 32 <= p.N) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            stg128_bf(dst + 8 * q, make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]),
                                              pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                              pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                                              pack_bf16(v[8 * q + 6], v[8 * q + 7])));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (col0 + i < p.N) dst[i] = __float2bfloat16_rn(v[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[ra.s]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// [rows][K] bf16 row-major as a 2D map (K, rows) with boxes of 64 x box_rows,
// 128-byte swizzle, zero fill outside.
inline bool make_kmajor_map(CUtensorMap* m, const void* ptr, int rows, int K, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kGmBK, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launches gemm_kernel for C = A B^T (p carries M, N, K, the mode and the
// destinations), as a programmatic dependent of the previous kernel.
inline gla_status run_gemm(const void* A, const void* B, GemmParams p, int sms,
                           cudaStream_t stream) {
  if (sms <= 0) return GLA_ERR_CUDA;
  CUtensorMap mA, mB;
  if (!make_kmajor_map(&mA, A, p.M, p.K, kGmBM) || !make_kmajor_map(&mB, B, p.N, p.K, kGmBN))
    return GLA_ERR_CUDA;
  p.tiles_m = (p.M + kGmBM - 1) / kGmBM;
  p.tiles_n = (p.N + kGmBN - 1) / kGmBN;
  const int tiles = p.tiles_m * p.tiles_n;
  const size_t smem = 1024 + GemmSmem::END;
  if (!ensure_max_smem(gemm_kernel, 0)) return GLA_ERR_CUDA;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(tiles < sms ? tiles : sms);
  lc.blockDim = dim3(kGmThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = stream;
  lc.attrs = pdl;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, gemm_kernel, mA, mB, p) == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

}  // namespace gla
