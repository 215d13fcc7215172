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

// One token-head row: RMSNorm, the rotation (c[i], s[i] of this lane's pairs
// 2l, 2l+1), the scale; lane l holds channels 4l .. 4l+3.
__device__ __forceinline__ uint2 an_prep_row(uint2 r, const float (&c)[2], const float (&s)[2],
                                             float scale) {
  const float x[4] = {bf_lo(r.x), bf_hi(r.x), bf_lo(r.y), bf_hi(r.y)};
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) ss = fmaf(x[i], x[i], ss);
  const float rs = rsqrtf(warp_sum(ss) * (1.f / 128.f) + kRmsEps) * scale;
  uint32_t o[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float a = x[2 * i] * rs, b = x[2 * i + 1] * rs;
    o[i] = pack_f16(fmaf(-b, s[i], a * c[i]), fmaf(b, c[i], a * s[i]));
  }
  return make_uint2(o[0], o[1]);
}

// A grid-stride loop over tokens; one warp per token takes every head of it
// (the rotation depends on the token only), two heads per step.
__global__ void __launch_bounds__(kAnWarpsPrep * 32) anchor_prep_kernel(AnchorPrepParams p) {
  pdl_launch_dependents();   // the attention CTAs may set up meanwhile
  const Geom& g = p.g;
  const int lane = threadIdx.x & 31;
  const long long tokens = (long long)g.B * g.N;
  const long long nwarps = (long long)gridDim.x * kAnWarpsPrep;
  const int HW = g.H * g.W;
  constexpr float kQScale = 0.12751743f;   // log2(e) / sqrt(128)
  for (long long bn = (long long)blockIdx.x * kAnWarpsPrep + (threadIdx.x >> 5); bn < tokens;
       bn += nwarps) {
    const int n = (int)(bn % g.N);
    const int f = n / HW, hh = (n / g.W) % g.H, ww = n % g.W;
    float c[2] = {1.f, 1.f}, sn[2] = {0.f, 0.f};
    if (g.rope_on) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int pr = 2 * lane + i;
        const double x =
            pr < g.pt ? (double)(g.t0 + f) : (pr < g.pt + g.ph ? (double)hh : (double)ww);
        const float2 cs = rope_entry(x, g.freq[pr]);
        c[i] = cs.x;
        sn[i] = cs.y;
      }
    }
    const size_t base = (size_t)bn * g.Hh * 128 + 4 * lane;
    int h = 0;
    for (; h + 2 <= g.Hh; h += 2) {
      const size_t o0 = base + (size_t)h * 128, o1 = o0 + 128;
      const uint2 q0 = *reinterpret_cast<const uint2*>(p.q + o0);
      const uint2 q1 = *reinterpret_cast<const uint2*>(p.q + o1);
      const uint2 k0 = *reinterpret_cast<const uint2*>(p.k + o0);
      const uint2 k1 = *reinterpret_cast<const uint2*>(p.k + o1);
      *reinterpret_cast<uint2*>(p.qt + o0) = an_prep_row(q0, c, sn, kQScale);
      *reinterpret_cast<uint2*>(p.qt + o1) = an_prep_row(q1, c, sn, kQScale);
      *reinterpret_cast<uint2*>(p.kt + o0) = an_prep_row(k0, c, sn, 1.f);
      *reinterpret_cast<uint2*>(p.kt + o1) = an_prep_row(k1, c, sn, 1.f);
    }
    if (h < g.Hh) {
      const size_t o0 = base + (size_t)h * 128;
      const uint2 q0 = *reinterpret_cast<const uint2*>(p.q + o0);
      const uint2 k0 = *reinterpret_cast<const uint2*>(p.k + o0);
      *reinterpret_cast<uint2*>(p.qt + o0) = an_prep_row(q0, c, sn, kQScale);
      *reinterpret_cast<uint2*>(p.kt + o0) = an_prep_row(k0, c, sn, 1.f);
    }
  }
}

// ------------------------------------------------------------- attention
//
// One CTA takes two 128-query tiles of a head (t = 0, 1) and streams the
// head's keys and values in 128-token tiles.  Warp 0 issues TMA (q tiles
// once; k and v through rings of two), warp 1 issues the MMAs, warps 2-5 and
// 6-9 are the softmax warpgroups of query tiles 0 and 1 (one query row per
// thread: warp w reads TMEM lane quarter w % 4).
//
// TMEM (512 columns): S_t = q_til_t k_til^T (fp32, 128 columns) at t*128; the
// softmax weights P_t (bf16 pairs, 64 columns) overwrite the first half of
// S_t and feed O_t += P_t V from tensor memory; O_t (fp32) at 256 + t*128.
// The MMA order S_0(j), S_1(j), PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), ... lets
// one warpgroup's softmax run while the tensor cores work for the other.  A
// tcgen05.commit tracks every MMA issued before it, so S_t(j) landing also
// means PV_t(j-1) has: the softmax may then rescale O_t without another wait.
//
// Running maximum: a row keeps the maximum it last rescaled to and rescales
// (O, the row sum) only when a tile's maximum exceeds it by more than 2^8, so
// that weights stay below 256; the normalisation at the end is the same for
// any such reference point.  exp2 runs on the MUFU unit for 3 of every 4
// weight pairs and as a polynomial on the FMA pipes for the 4th.

constexpr int kAnTile = 128;
constexpr int kAnQT = 2;                          // query tiles per CTA
constexpr int kAnSW0 = 2;                         // first softmax warp
constexpr int kAnThreads = (kAnSW0 + 4 * kAnQT) * 32;
constexpr uint32_t kAnO = 256;                    // TMEM column of O_0
constexpr float kAnLazy = 8.f;                    // log2 of the largest weight

struct AnchorSmem {
  static constexpr uint32_t Q = 0;                        // [2] q_til tiles (fp16)
  static constexpr uint32_t K = Q + kAnQT * kTileBytes;   // [2] k_til tiles (fp16)
  static constexpr uint32_t V = K + 2 * kTileBytes;       // [2] v tiles (bf16)
  static constexpr uint32_t BAR = V + 2 * kTileBytes;
  static constexpr uint32_t NBAR = 1 + 2 * 7 + 1;
  static constexpr uint32_t MISC = BAR + NBAR * 8;
  static constexpr uint32_t END = MISC + 16;
};

struct AnchorParams {
  Geom g;
  const __nv_bfloat16* gate;
  __nv_bfloat16* out;
};

// D[tmem] (+)= A[tmem] x B[smem desc], kind::f16: A (M rows = TMEM lanes, K
// packed in pairs per 32-bit column) read from tensor memory.
__device__ __forceinline__ void umma_f16kind_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 2^x on the MUFU unit (ex2.approx: flushes subnormals, 2^-inf = 0).
__device__ __forceinline__ float an_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipes: x = i + f with i = floor(x), f in [0, 1);
// 2^f ~ 1 + f (c1 + f (c2 + f c3)), a degree-3 fit with the constant term
// fixed at 1, relative error below 8.6e-5 on [0, 1) (the coefficients minimise
// the largest relative error, by iteratively reweighted least squares); the
// integer part is added to the exponent field.  x >= -126 (callers clamp).
__device__ __forceinline__ float an_ex2_poly(float x) {
  const float xi = floorf(x);
  const float f = x - xi;
  const float p = fmaf(fmaf(fmaf(0.07706520f, f, 0.22764701f), f, 0.69511634f), f, 1.f);
  return __int_as_float(__float_as_int(p) + (int)((uint32_t)(int)xi << 23));
}

__device__ __forceinline__ void tmem_ld32_at(uint32_t taddr, float* r) {
  tmem_ld32(taddr, *reinterpret_cast<float(*)[32]>(r));
}

// Half a tile of one query row (keys 64*kHalf .. 64*kHalf + 63): the weights
// 2^(s - m) as bf16 pairs into w[32] (as float bit patterns for tcgen05.st),
// the fp32 sum of the rounded weights returned.  kMask: keys at or past `kcount` get weight 0.
template <bool kMask, int kHalf>
__device__ __forceinline__ float an_weights(const float (&s)[128], float m, int kcount,
                                            float (&w)[32]) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int k = 64 * kHalf + 2 * i;
    const float x0 = s[k] - m, x1 = s[k + 1] - m;
    float p0, p1;
    if ((i & 3) == 3) {
      p0 = an_ex2_poly(fmaxf(x0, -126.f));
      p1 = an_ex2_poly(fmaxf(x1, -126.f));
    } else {
      p0 = an_ex2(x0);
      p1 = an_ex2(x1);
    }
    if (kMask) {
      if (k >= kcount) p0 = 0.f;
      if (k + 1 >= kcount) p1 = 0.f;
    }
    // The row sum adds the rounded weights, the ones P V multiplies: the
    // normalised output is then a convex combination of v rows whatever the
    // reference point (a row's largest weight is not exact in bf16 when the
    // reference point lags the maximum).
    const uint32_t pk = pack_bf16(p0, p1);
    acc[i & 3] += __uint_as_float(pk << 16) + __uint_as_float(pk & 0xFFFF0000u);
    w[i] = __uint_as_float(pk);
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// Both halves of a row's weights into P (TMEM columns tP .. tP + 63).
template <bool kMask>
__device__ __forceinline__ float an_weights_to_tmem(const float (&s)[128], float m, int kcount,
                                                    uint32_t tP) {
  float w[32];
  float l = an_weights<kMask, 0>(s, m, kcount, w);
  tmem_st32(tP, w);
  l += an_weights<kMask, 1>(s, m, kcount, w);
  tmem_st32(tP + 32, w);
  return l;
}

template <bool kMask>
__device__ __forceinline__ float an_rowmax(float (&s)[128], int kcount) {
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
  for (int i = 0; i < 128; ++i) {
    if (kMask && i >= kcount) s[i] = -INFINITY;
    mx[i & 7] = fmaxf(mx[i & 7], s[i]);
  }
  return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

// 10 warps: three share one SM sub-partition's 16 K registers, so at most
// 168 registers a thread.
__global__ void __launch_bounds__(kAnThreads, 1)
    anchor_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, AnchorParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + AnchorSmem::BAR);
  uint64_t* qfull = bars;
  uint64_t* kfull = bars + 1;      // [2]
  uint64_t* kfree = bars + 3;      // [2]
  uint64_t* vfull = bars + 5;      // [2]
  uint64_t* vfree = bars + 7;      // [2]
  uint64_t* sfull = bars + 9;      // [2]: per query tile
  uint64_t* pready = bars + 11;    // [2]
  uint64_t* odone = bars + 13;     // [2]
  uint64_t* drain = bars + 15;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + AnchorSmem::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + AnchorSmem::MISC + 4);

  const Geom& g = p.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, b = bh / g.Hh, h = bh - b * g.Hh;
  const int q0 = blockIdx.x * (kAnQT * kAnTile);
  const int nkv = (g.N + kAnTile - 1) / kAnTile;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kfree[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&vfree[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&pready[s], 4);
      mbar_init(&odone[s], 1);
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
      mbar_arrive_expect_tx(qfull, kAnQT * kTileBytes);
      for (int t = 0; t < kAnQT; ++t) {
        unsigned char* qt = sm + AnchorSmem::Q + t * kTileBytes;
        tma_load_3d(qt, &tmQ, qfull, h * 128, q0 + t * kAnTile, b, policy_evict_first());
        tma_load_3d(qt + kBox, &tmQ, qfull, h * 128 + 64, q0 + t * kAnTile, b,
                    policy_evict_first());
      }
      int nk = 0, nv = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j & 1;
        const uint32_t ph = (uint32_t)((j >> 1) & 1);
        if (!mbar_wait(&kfree[s], ph ^ 1u, abort_flag)) break;
        unsigned char* kt = sm + AnchorSmem::K + s * kTileBytes;
        mbar_arrive_expect_tx(&kfull[s], kTileBytes);
        tma_load_3d(kt, &tmK, &kfull[s], h * 128, j * kAnTile, b, pol);
        tma_load_3d(kt + kBox, &tmK, &kfull[s], h * 128 + 64, j * kAnTile, b, pol);
        ++nk;
        if (!mbar_wait(&vfree[s], ph ^ 1u, abort_flag)) break;
        unsigned char* vt = sm + AnchorSmem::V + s * kTileBytes;
        mbar_arrive_expect_tx(&vfull[s], kTileBytes);
        tma_load_3d(vt, &tmV, &vfull[s], h * 128, j * kAnTile, b, pol);
        tma_load_3d(vt + kBox, &tmV, &vfull[s], h * 128 + 64, j * kAnTile, b, pol);
        ++nv;
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA exits
        int dummy = 0;
        volatile int* nd = reinterpret_cast<volatile int*>(&dummy);
        mbar_wait(qfull, 0u, nd);
        for (int i2 = nk - (nk < 2 ? nk : 2); i2 < nk; ++i2)
          mbar_wait(&kfull[i2 & 1], (uint32_t)((i2 >> 1) & 1), nd);
        for (int i2 = nv - (nv < 2 ? nv : 2); i2 < nv; ++i2)
          mbar_wait(&vfull[i2 & 1], (uint32_t)((i2 >> 1) & 1), nd);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, 128, false, false);
      constexpr uint32_t idPV = idesc_bf16(128, 128, false, true);
      auto scores = [&](int t, int j) {   // S_t = q_til_t k_til_j^T
        const uint32_t qt = sbase + AnchorSmem::Q + t * kTileBytes;
        const uint32_t kt = sbase + AnchorSmem::K + (j & 1) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32;
          umma_f16kind(tmem + t * 128, sdesc_sw128(qt + koff, 16, 1024),
                       sdesc_sw128(kt + koff, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sfull[t]);
      };
      auto pv = [&](int t, int j) {       // O_t += P_t v_j, P_t from TMEM
        const uint32_t vt = sbase + AnchorSmem::V + (j & 1) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16kind_ta(tmem + kAnO + t * 128, tmem + t * 128 + kk * 8,
                          sdesc_sw128(vt + kk * 2048, kBox, 1024), idPV,
                          (j > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(qfull, 0u, abort_flag) && mbar_wait(&kfull[0], 0u, abort_flag);
      if (ok) {
        tc_fence_after();
        scores(0, 0);
        scores(1, 0);
        umma_commit(&kfree[0]);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j & 1;
        if (!(ok = mbar_wait(&vfull[s], (uint32_t)((j >> 1) & 1), abort_flag))) break;
        for (int t = 0; t < kAnQT; ++t) {
          if (!(ok = mbar_wait(&pready[t], (uint32_t)(j & 1), abort_flag))) break;
          tc_fence_after();
          pv(t, j);
          if (t == kAnQT - 1) umma_commit(&vfree[s]);
          if (j + 1 < nkv) {
            const int s1 = (j + 1) & 1;
            if (t == 0 && !(ok = mbar_wait(&kfull[s1], (uint32_t)(((j + 1) >> 1) & 1),
                                           abort_flag)))
              break;
            tc_fence_after();
            scores(t, j + 1);
            if (t == kAnQT - 1) umma_commit(&kfree[s1]);
          }
        }
      }
      if (ok)
        for (int t = 0; t < kAnQT; ++t) umma_commit(&odone[t]);
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy));
    }
  } else {
    // --------------------------------------------------------- softmax warps
    const int t = (warp - kAnSW0) >> 2;       // query tile
    const int q4 = warp & 3;                  // TMEM lane quarter
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + t * 128 + lane_off;
    const uint32_t tO = tmem + kAnO + t * 128 + lane_off;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait_warp(&sfull[t], (uint32_t)(j & 1), abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32_at(tS + c * 32, s + c * 32);
      tmem_wait_ld();
      const int kcount = g.N - j * kAnTile;
      const float mt = kcount < kAnTile ? an_rowmax<true>(s, kcount) : an_rowmax<false>(s, kcount);
      const bool grow = mt > m + kAnLazy;
      float alpha = 1.f;
      const bool rescale = __any_sync(0xffffffffu, grow) && j > 0;
      if (grow) {
        alpha = an_ex2(m - mt);   // 0 on the first tile
        l *= alpha;
        m = mt;
      }
      l += kcount < kAnTile ? an_weights_to_tmem<true>(s, m, kcount, tS)
                            : an_weights_to_tmem<false>(s, m, kcount, tS);
      if (rescale) {
        // O_t holds the tiles before j at the old reference point; PV_t(j-1)
        // landed before S_t(j) did, and PV_t(j) waits for this warp's arrival.
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[t]);
    }
    // epilogue: O / l, the gate, bf16 rows
    if (ok && mbar_wait_warp(&odone[t], 0u, abort_flag)) {
      tc_fence_after();
      const int n = q0 + t * kAnTile + row;
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
                             const void* gate, void* out, __half* qt, __half* kt, int sms,
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
  const long long tokens = (long long)g.B * g.N;
  const long long blocks = (tokens + kAnWarpsPrep - 1) / kAnWarpsPrep;
  const int grid = (int)(blocks < 8LL * sms ? blocks : 8LL * sms);
  anchor_prep_kernel<<<grid, kAnWarpsPrep * 32, 0, stream>>>(pp);
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
  lc.gridDim = dim3((g.N + kAnQT * kAnTile - 1) / (kAnQT * kAnTile), g.B * g.Hh);
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
