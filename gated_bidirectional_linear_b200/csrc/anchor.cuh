// The gated softmax anchor of the hybrid stack: bidirectional softmax
// attention with QK RMSNorm, 3D RoPE and a sigmoid output gate,
//   o_j = sigmoid(g_j) * sum_n softmax_n(q_til_j . k_til_n / sqrt(d)) v_n,
// q_til = RoPE3D(RMSNorm(q)), k_til = RoPE3D(RMSNorm(k)), head dim 128, bf16 in
// and out.
//
//   anchor_prep_kernel  q_til * log2(e) / sqrt(d) and k_til as fp16 in the
//                       [B][N][Hh][128] layout (one warp per token-head).
//   anchor_attn_kernel  one CTA per 128 queries of a head: TMA streams the
//                       head's key / value tiles (128 tokens) through a 2-slot
//                       ring; one thread issues S = Q K^T (fp16) into one of two
//                       TMEM score buffers, so the next tile's scores run while
//                       the softmax warps (one query row per thread) take the
//                       row maximum, exp2 and the running sum of this one and
//                       write P (bf16) to shared memory; O += P V (bf16)
//                       accumulates in TMEM, rescaled by the softmax warps when
//                       a row maximum grows.  The epilogue divides by the row
//                       sum, applies the gate and stores bf16 rows.
#pragma once

#include "tc.cuh"

namespace gla {

constexpr int kAnWarpsPrep = 8;

struct AnchorPrepParams {
  Geom g;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  __half* qt;          // [B][N][Hh][128] fp16, times log2(e) / sqrt(128)
  __half* kt;
};

__global__ void __launch_bounds__(kAnWarpsPrep * 32) anchor_prep_kernel(AnchorPrepParams p) {
  pdl_launch_dependents();   // the attention CTAs may set up meanwhile
  const Geom& g = p.g;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kAnWarpsPrep + (threadIdx.x >> 5);
  const long long rows = (long long)g.B * g.N * g.Hh;
  if (row >= rows) return;
  const long long bn = row / g.Hh;
  const int n = (int)(bn % g.N);
  const int HW = g.H * g.W;
  const int f = n / HW, hh = (n / g.W) % g.H, ww = n % g.W;
  // Lane l: channels 4l .. 4l+3, rotation pairs 2l and 2l+1.
  const size_t off = (size_t)row * 128 + 4 * lane;
  const uint2 qr = *reinterpret_cast<const uint2*>(p.q + off);
  const uint2 kr = *reinterpret_cast<const uint2*>(p.k + off);
  float qx[4] = {bf_lo(qr.x), bf_hi(qr.x), bf_lo(qr.y), bf_hi(qr.y)};
  float kx[4] = {bf_lo(kr.x), bf_hi(kr.x), bf_lo(kr.y), bf_hi(kr.y)};
  float sq = 0.f, sk = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    sq = fmaf(qx[i], qx[i], sq);
    sk = fmaf(kx[i], kx[i], sk);
  }
  sq = warp_sum(sq);
  sk = warp_sum(sk);
  const float rq = rsqrtf(sq * (1.f / 128.f) + kRmsEps) * 0.12751743f;   // log2(e) / sqrt(128)
  const float rk = rsqrtf(sk * (1.f / 128.f) + kRmsEps);
  uint32_t qo[2], ko[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int pr = 2 * lane + i;
    float c = 1.f, s = 0.f;
    if (g.rope_on) {
      const double x = pr < g.pt ? (double)(g.t0 + f) : (pr < g.pt + g.ph ? (double)hh : (double)ww);
      const float2 cs = rope_entry(x, g.freq[pr]);
      c = cs.x;
      s = cs.y;
    }
    const float q0 = qx[2 * i] * rq, q1 = qx[2 * i + 1] * rq;
    const float k0 = kx[2 * i] * rk, k1 = kx[2 * i + 1] * rk;
    qo[i] = pack_f16(fmaf(-q1, s, q0 * c), fmaf(q1, c, q0 * s));
    ko[i] = pack_f16(fmaf(-k1, s, k0 * c), fmaf(k1, c, k0 * s));
  }
  *reinterpret_cast<uint2*>(p.qt + off) = make_uint2(qo[0], qo[1]);
  *reinterpret_cast<uint2*>(p.kt + off) = make_uint2(ko[0], ko[1]);
}

// ------------------------------------------------------------- attention

constexpr int kAnTile = 128;
constexpr int kAnThreads = 6 * 32;      // producer, MMA, 4 softmax warps
constexpr uint32_t kAnS = 0, kAnO = 256; // TMEM columns: two score buffers, O

struct AnchorSmem {
  static constexpr uint32_t Q = 0;                        // q_til tile (fp16)
  static constexpr uint32_t K = Q + kTileBytes;           // [2] k_til tiles (fp16)
  static constexpr uint32_t V = K + 2 * kTileBytes;       // [2] v tiles (bf16)
  static constexpr uint32_t P = V + 2 * kTileBytes;       // [2] P tiles (bf16)
  static constexpr uint32_t BAR = P + 2 * kTileBytes;
  static constexpr uint32_t NBAR = 1 + 6 * 2 + 1;
  static constexpr uint32_t MISC = BAR + NBAR * 8;
  static constexpr uint32_t END = MISC + 16;
};

struct AnchorParams {
  Geom g;
  const __nv_bfloat16* gate;
  __nv_bfloat16* out;
};

__global__ void __launch_bounds__(kAnThreads, 1)
    anchor_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, AnchorParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + AnchorSmem::BAR);
  uint64_t* qfull = bars;
  uint64_t* kvfull = bars + 1;     // [2]
  uint64_t* kvfree = bars + 3;     // [2]
  uint64_t* sfull = bars + 5;      // [2]
  uint64_t* sfree = bars + 7;      // [2]
  uint64_t* pready = bars + 9;     // [2]
  uint64_t* pvdone = bars + 11;    // [2]
  uint64_t* drain = bars + 13;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + AnchorSmem::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + AnchorSmem::MISC + 4);

  const Geom& g = p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, b = bh / g.Hh, h = bh - b * g.Hh;
  const int q0 = blockIdx.x * kAnTile;
  const int nkv = (g.N + kAnTile - 1) / kAnTile;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kvfull[s], 1);
      mbar_init(&kvfree[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&sfree[s], 4);
      mbar_init(&pready[s], 4);
      mbar_init(&pvdone[s], 1);
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
      pdl_wait();   // q_til, k_til come from the prep kernel
      const uint64_t pol = policy_evict_last();   // k, v tiles are read by every query tile
      mbar_arrive_expect_tx(qfull, kTileBytes);
      tma_load_3d(sm + AnchorSmem::Q, &tmQ, qfull, h * 128, q0, b, policy_evict_first());
      tma_load_3d(sm + AnchorSmem::Q + kBox, &tmQ, qfull, h * 128 + 64, q0, b, policy_evict_first());
      RingPos<2> rs;
      int issued = 0;
      for (int j = 0; j < nkv; ++j, rs.next()) {
        if (!mbar_wait(&kvfree[rs.s], rs.ph ^ 1u, abort_flag)) break;
        unsigned char* kt = sm + AnchorSmem::K + rs.s * kTileBytes;
        unsigned char* vt = sm + AnchorSmem::V + rs.s * kTileBytes;
        mbar_arrive_expect_tx(&kvfull[rs.s], 2 * kTileBytes);
        tma_load_3d(kt, &tmK, &kvfull[rs.s], h * 128, j * kAnTile, b, pol);
        tma_load_3d(kt + kBox, &tmK, &kvfull[rs.s], h * 128 + 64, j * kAnTile, b, pol);
        tma_load_3d(vt, &tmV, &kvfull[rs.s], h * 128, j * kAnTile, b, pol);
        tma_load_3d(vt + kBox, &tmV, &kvfull[rs.s], h * 128 + 64, j * kAnTile, b, pol);
        ++issued;
      }
      if (*abort_flag) {
        int dummy = 0;
        volatile int* nd = reinterpret_cast<volatile int*>(&dummy);
        mbar_wait(qfull, 0u, nd);
        for (int i2 = issued - (issued < 2 ? issued : 2); i2 < issued; ++i2)
          mbar_wait(&kvfull[i2 & 1], (uint32_t)((i2 >> 1) & 1), nd);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 128, false, false);
      constexpr uint32_t idPV = idesc_bf16(128, 128, false, true);
      const uint32_t qt = sbase + AnchorSmem::Q;
      auto scores = [&](int j) {
        const int s = j & 1;
        const uint32_t kt = sbase + AnchorSmem::K + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32;
          umma_f16kind(tmem + kAnS + s * 128, sdesc_sw128(qt + koff, 16, 1024),
                       sdesc_sw128(kt + koff, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sfull[s]);
      };
      bool ok = mbar_wait(qfull, 0u, abort_flag) && mbar_wait(&kvfull[0], 0u, abort_flag);
      if (ok) {
        tc_fence_after();
        scores(0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j & 1;
        if (j + 1 < nkv) {
          const int s1 = (j + 1) & 1;
          // the next tile's keys, and the score buffer the softmax warps
          // released after tile j - 1
          if (!mbar_wait(&kvfull[s1], (uint32_t)(((j + 1) >> 1) & 1), abort_flag)) break;
          if (j >= 1 && !mbar_wait(&sfree[s1], (uint32_t)(((j - 1) >> 1) & 1), abort_flag)) break;
          tc_fence_after();
          scores(j + 1);
        }
        if (!mbar_wait(&pready[s], (uint32_t)((j >> 1) & 1), abort_flag)) break;
        tc_fence_after();
        const uint32_t pt = sbase + AnchorSmem::P + s * kTileBytes;
        const uint32_t vt = sbase + AnchorSmem::V + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t poff = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32;
          umma_f16kind(tmem + kAnO, sdesc_sw128(pt + poff, 16, 1024),
                       sdesc_sw128(vt + kk * 2048, kBox, 1024), idPV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&pvdone[s]);
        umma_commit(&kvfree[s]);
      }
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy));
    }
  } else {
    // --------------------------------------------------------- softmax warps
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tmem + kAnO + lane_off;
    const uint32_t sw = (uint32_t)(row & 7);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      const uint32_t tS = tmem + kAnS + s * 128 + lane_off;
      if (!mbar_wait_warp(&sfull[s], (uint32_t)((j >> 1) & 1), abort_flag)) { ok = false; break; }
      tc_fence_after();
      const int kcount = g.N - j * kAnTile;   // valid keys in this tile (>= 1)
      // pass 1: the row maximum of this tile
      float mt = -INFINITY;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float v[32];
        tmem_ld32(tS + cb * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (cb * 32 + i < kcount) mt = fmaxf(mt, v[i]);
      }
      const float mn = fmaxf(m, mt);
      const float alpha = exp2f(m - mn);      // 0 on the first tile (m = -inf)
      // the P buffer of this tile was read by PV(j - 2)
      if (j >= 2 && !mbar_wait_warp(&pvdone[s], (uint32_t)(((j - 2) >> 1) & 1), abort_flag)) {
        ok = false;
        break;
      }
      // pass 2: p = exp2(s - mn) to P (bf16), the row sum
      const uint32_t pt = sbase + AnchorSmem::P + s * kTileBytes;
      float ls = 0.f;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float v[32];
        tmem_ld32(tS + cb * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = cb * 32 + q * 8 + 2 * e;
            const float p0 = c < kcount ? exp2f(v[q * 8 + 2 * e] - mn) : 0.f;
            const float p1 = c + 1 < kcount ? exp2f(v[q * 8 + 2 * e + 1] - mn) : 0.f;
            ls += p0 + p1;
            w4[e] = pack_bf16(p0, p1);
          }
          const int k = cb * 4 + q;       // 16-byte chunk: keys 8k .. 8k+7
          sts128(pt + (uint32_t)(k >> 3) * kBox + (uint32_t)row * 128u +
                     ((((uint32_t)(k & 7)) ^ sw) << 4),
                 make_uint4(w4[0], w4[1], w4[2], w4[3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sfree[s]);
      l = l * alpha + ls;
      m = mn;
      // O holds the sum up to tile j - 1 at the old maximum: rescale it once
      // PV(j - 1) has landed, when some row of the warp has a new maximum.
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!mbar_wait_warp(&pvdone[(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
          float o[32];
          tmem_ld32(tO + cb * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + cb * 32, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[s]);
    }
    // epilogue: O / l, the gate, bf16 rows
    if (ok && mbar_wait_warp(&pvdone[(nkv - 1) & 1], (uint32_t)(((nkv - 1) >> 1) & 1), abort_flag)) {
      tc_fence_after();
      const int n = q0 + row;
      const bool valid = n < g.N;
      const size_t rowoff = (((size_t)b * g.N + (valid ? n : 0)) * g.Hh + h) * 128;
      const float inv = 1.f / l;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float o[32];
        tmem_ld32(tO + cb * 32, o);
        uint4 gv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          gv[q] = valid ? *reinterpret_cast<const uint4*>(p.gate + rowoff + cb * 32 + 8 * q)
                        : make_uint4(0u, 0u, 0u, 0u);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t wv[4] = {gv[q].x, gv[q].y, gv[q].z, gv[q].w};
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float g0 = bf_lo(wv[e]), g1 = bf_hi(wv[e]);
            const float s0 = fmaf(0.5f, tanh_approx(0.5f * g0), 0.5f);
            const float s1 = fmaf(0.5f, tanh_approx(0.5f * g1), 0.5f);
            w4[e] = pack_bf16(o[q * 8 + 2 * e] * inv * s0, o[q * 8 + 2 * e + 1] * inv * s1);
          }
          if (valid)
            *reinterpret_cast<uint4*>(p.out + rowoff + cb * 32 + 8 * q) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The anchor: prep (q_til, k_til into the workspace), then the attention, a
// programmatic dependent of the prep.  Head dim 128, bf16.  `events` (may be
// NULL): recorded before the prep, after it and after the attention.
inline gla_status run_anchor(const Geom& g, const void* q, const void* k, const void* v,
                             const void* gate, void* out, __half* qt, __half* kt,
                             cudaStream_t stream, void* const* events) {
  auto rec = [&](int i) -> cudaError_t {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream);
  };
  if (rec(0) != cudaSuccess) return GLA_ERR_CUDA;
  AnchorPrepParams pp;
  pp.g = g;
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.qt = qt;
  pp.kt = kt;
  const long long rows = (long long)g.B * g.N * g.Hh;
  anchor_prep_kernel<<<(unsigned)((rows + kAnWarpsPrep - 1) / kAnWarpsPrep), kAnWarpsPrep * 32, 0,
                       stream>>>(pp);
  if (cudaGetLastError() != cudaSuccess || rec(1) != cudaSuccess) return GLA_ERR_CUDA;

  CUtensorMap mQ, mK, mV;
  if (!make_act_map(&mQ, qt, g, kAnTile) || !make_act_map(&mK, kt, g, kAnTile) ||
      !make_act_map(&mV, v, g, kAnTile))
    return GLA_ERR_CUDA;
  AnchorParams ap;
  ap.g = g;
  ap.gate = static_cast<const __nv_bfloat16*>(gate);
  ap.out = static_cast<__nv_bfloat16*>(out);
  if (!ensure_max_smem(anchor_attn_kernel, 0)) return GLA_ERR_CUDA;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((g.N + kAnTile - 1) / kAnTile, g.B * g.Hh);
  lc.blockDim = dim3(kAnThreads);
  lc.dynamicSmemBytes = 1024 + AnchorSmem::END;
  lc.stream = stream;
  lc.attrs = pdl;
  lc.numAttrs = 1;
  if (cudaLaunchKernelEx(&lc, anchor_attn_kernel, mQ, mK, mV, ap) != cudaSuccess)
    return GLA_ERR_CUDA;
  return rec(2) == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

}  // namespace gla
