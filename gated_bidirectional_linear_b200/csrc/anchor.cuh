// The gated softmax anchor of the hybrid stack: bidirectional softmax
// attention with QK RMSNorm, 3D RoPE and a sigmoid output gate,
//   o_j = sigmoid(g_j) * sum_n softmax_n(q_til_j . k_til_n / sqrt(d)) v_n,
// q_til = RoPE3D(RMSNorm(q)), k_til = RoPE3D(RMSNorm(k)), head dim 128, bf16 in
// and out.
//
//   anchor_prep_kernel  q_til * log2(e) / sqrt(d) and k_til as fp16 in the
//                       [B][N][Hh][128] layout (one warp per token, every head).
//   anchor_attn_kernel  one CTA per two 128-query tiles of a head: TMA streams
//                       the head's key / value tiles (128 tokens); one thread
//                       issues S = Q K^T (fp16) and O += P V (bf16, P read from
//                       TMEM); two softmax warpgroups (one query row per thread)
//                       turn each tile's scores into bf16 weights in TMEM while
//                       the tensor cores work for the other query tile.  The
//                       epilogue divides by the row sum, applies the gate and
//                       stores bf16 rows.
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

// 8-byte read-only global load.
__device__ __forceinline__ uint2 ldg_u2(const __nv_bfloat16* p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

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
// (the rotation depends on the token only), four heads per step.  The loads of
// the next step (the next four heads, or the first four of the warp's next
// token) are issued before the current step is processed.
__global__ void __launch_bounds__(kAnWarpsPrep * 32) anchor_prep_kernel(AnchorPrepParams p) {
  pdl_launch_dependents();   // the attention CTAs may set up meanwhile
  const Geom& g = p.g;
  const int lane = threadIdx.x & 31;
  const long long tokens = (long long)g.B * g.N;
  const long long nwarps = (long long)gridDim.x * kAnWarpsPrep;
  const int HW = g.H * g.W;
  constexpr float kQScale = 0.12751743f;   // log2(e) / sqrt(128)
  long long bn = (long long)blockIdx.x * kAnWarpsPrep + (threadIdx.x >> 5);
  if (bn >= tokens) return;
  uint2 qn[4], kn[4];     // the next step's rows
  auto load = [&](long long tok, int h0) {
    const size_t base = (size_t)tok * g.Hh * 128 + 4 * lane;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const size_t o = base + (size_t)(h0 + u < g.Hh ? h0 + u : h0) * 128;
      qn[u] = ldg_u2(p.q + o);
      kn[u] = ldg_u2(p.k + o);
    }
  };
  load(bn, 0);
  for (; bn < tokens; bn += nwarps) {
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
    for (int h0 = 0; h0 < g.Hh; h0 += 4) {
      uint2 qr[4], kr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        qr[u] = qn[u];
        kr[u] = kn[u];
      }
      if (h0 + 4 < g.Hh) {
        load(bn, h0 + 4);
      } else if (bn + nwarps < tokens) {
        load(bn + nwarps, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (h0 + u >= g.Hh) break;
        const size_t o = base + (size_t)(h0 + u) * 128;
        *reinterpret_cast<uint2*>(p.qt + o) = an_prep_row(qr[u], c, sn, kQScale);
        *reinterpret_cast<uint2*>(p.kt + o) = an_prep_row(kr[u], c, sn, 1.f);
      }
    }
  }
}

// ------------------------------------------------------------- attention
//
// One CTA takes two 128-query tiles of a head (t = 0, 1) and streams the
// head's keys and values in 128-token tiles.  Warp 0 issues TMA (q tiles
// once; k through a ring of two slots, v through a ring of three), warp 1
// issues the MMAs, warps 2-5 and 6-9 are the softmax warpgroups of query
// tiles 0 and 1 (one query row per thread: warp w reads TMEM lane quarter
// w % 4).
//
// TMEM (512 columns): S_t = q_til_t k_til^T (fp32, 128 columns) at t*128; the
// softmax weights P_t (bf16 pairs, 64 columns) overwrite the first half of
// S_t and feed O_t += P_t V from tensor memory; O_t (fp32) at 256 + t*128.
// The MMA order S_0(j), S_1(j), PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), ... lets
// one warpgroup's softmax run while the tensor cores work for the other.  A
// tcgen05.commit tracks every MMA issued before it, so S_t(j) landing also
// means PV_t(j-1) has, and the softmax may overwrite P_t.
//
// No running maximum: q_til and k_til are RMS-normalised and rotated, so
// |q_til| = |k_til| <= sqrt(d) and every score in base 2,
// q_til . k_til * log2(e) / sqrt(d), lies within +-sqrt(d) log2(e) = +-16.33
// (d = 128).  The weights 2^s then lie in [2^-16.4, 2^16.4], normal in bf16 and
// fp32, and the normalisation O / l at the end is the softmax for any common
// shift of the scores: no maximum, no rescale of O.  exp2 runs on the MUFU
// unit for three of every four weight pairs and as a polynomial on the FMA
// pipes for the fourth.

constexpr int kAnTile = 128;
constexpr int kAnQT = 2;                          // query tiles per CTA
constexpr int kAnSW0 = 2;                         // first softmax warp
constexpr int kAnThreads = (kAnSW0 + 4 * kAnQT) * 32;
constexpr uint32_t kAnO = 256;                    // TMEM column of O_0
constexpr int kAnVS = 3;                          // v ring slots
constexpr int kAnPolyPairs = 1;                   // of every 4 weight pairs, by polynomial
static_assert(kAnQT == 2, "the MMA issue order interleaves exactly two query tiles");

struct AnchorSmem {
  static constexpr uint32_t Q = 0;                        // [2] q_til tiles (fp16)
  static constexpr uint32_t K = Q + kAnQT * kTileBytes;   // [2] k_til tiles (fp16)
  static constexpr uint32_t V = K + 2 * kTileBytes;       // [3] v tiles (bf16)
  static constexpr uint32_t BAR = V + kAnVS * kTileBytes;
  static constexpr uint32_t NBAR = 1 + 2 * 2 + 2 * kAnVS + 3 * kAnQT + 1;
  static constexpr uint32_t MISC = BAR + NBAR * 8;
  static constexpr uint32_t END = MISC + 16;
};
// Descriptors are advanced by adding 16-byte units to their 14-bit address
// field, which therefore must not overflow for any tile.
static_assert(1024 + 1024 + AnchorSmem::BAR < (1u << 18), "descriptor address field");

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

// One lane of the (fully active) warp gets true.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// 2^x on the MUFU unit (ex2.approx: flushes subnormals, 2^-inf = 0).
__device__ __forceinline__ float an_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (one f32x2 instruction for both halves).
__device__ __forceinline__ f2_t an_f2_add(f2_t a, f2_t b) {
  f2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for a pair, on the FMA pipes (f32x2), none of it on the MUFU /
// conversion unit: x = n + f with n = round(x) (adding 1.5 * 2^23 leaves n in
// the low mantissa bits) and f in [-1/2, 1/2]; 2^f ~ 1 + f (c1 + f (c2 + f (c3
// + f c4))), a degree-4 fit with the constant term fixed at 1, relative error
// below 2.9e-6 on [-1/2, 1/2] (the coefficients minimise the largest relative
// error, by iteratively reweighted least squares), so that a weight rounds to
// the same bf16 as the MUFU's ex2 nearly always; n enters the exponent field
// as (bits of x + 1.5 * 2^23) * 2^23, the magic number's low nine bits being
// zero.  |x| < 126.
__device__ __forceinline__ void an_ex2_poly2(f2_t x, float& p0, float& p1) {
  const f2_t magic = f2(12582912.f, 12582912.f), nmagic = f2(-12582912.f, -12582912.f);
  const f2_t t = an_f2_add(x, magic);
  const f2_t xr = an_f2_add(t, nmagic);
  const f2_t f = f2_fma(xr, f2(-1.f, -1.f), x);
  f2_t p = f2_fma(f2(0.0095828352f, 0.0095828352f), f, f2(0.055906396f, 0.055906396f));
  p = f2_fma(p, f, f2(0.24024099f, 0.24024099f));
  p = f2_fma(p, f, f2(0.69312418f, 0.69312418f));
  p = f2_fma(p, f, f2(1.f, 1.f));
  p0 = __int_as_float(__float_as_int(f2_lo(p)) +
                      (int)((uint32_t)__float_as_int(f2_lo(t)) << 23));
  p1 = __int_as_float(__float_as_int(f2_hi(p)) +
                      (int)((uint32_t)__float_as_int(f2_hi(t)) << 23));
}

__device__ __forceinline__ void tmem_ld32_at(uint32_t taddr, float* r) {
  tmem_ld32(taddr, *reinterpret_cast<float(*)[32]>(r));
}

// a0 += low bf16 half of w, a1 += high half (exact: fp32 sums of the rounded
// weights, the ones P V multiplies).
__device__ __forceinline__ void an_add_bf16x2(float& a0, float& a1, uint32_t w) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(w));
}

// 16 consecutive 32-bit TMEM columns of this warp's lane quarter.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&u)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]),
      "r"(u[8]), "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]),
      "r"(u[15])
      : "memory");
}

// One 32-key chunk c of a row's scores s (base 2, |s| <= 16.33): the weights
// 2^s as bf16 pairs into w (the last kAnPolyPairs pairs of every four by the
// polynomial), the rounded weights added to acc.  kMask: keys at or past
// kcount get weight 0.
template <bool kMask>
__device__ __forceinline__ void an_chunk(const float (&s)[32], int c, int kcount,
                                         float (&acc)[4], uint32_t (&w)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int k0 = 32 * c + 2 * i;
    float p0, p1;
    if ((i & 3) >= 4 - kAnPolyPairs) {
      an_ex2_poly2(f2(s[2 * i], s[2 * i + 1]), p0, p1);
      if (kMask) {
        if (k0 >= kcount) p0 = 0.f;
        if (k0 + 1 >= kcount) p1 = 0.f;
      }
    } else {
      p0 = an_ex2(kMask && k0 >= kcount ? -INFINITY : s[2 * i]);
      p1 = an_ex2(kMask && k0 + 1 >= kcount ? -INFINITY : s[2 * i + 1]);
    }
    const uint32_t pk = pack_bf16(p0, p1);
    an_add_bf16x2(acc[(i & 1) * 2], acc[(i & 1) * 2 + 1], pk);
    w[i] = pk;
  }
}

// A row's weights for one tile: the 128 scores come from TMEM (tS) in four
// 32-column chunks, each load issued before the previous chunk is processed;
// chunk c's 16 packed weight columns go to tS + 16c, over score columns that
// are already in registers.  Returns the sum of the rounded weights.
template <bool kMask>
__device__ __forceinline__ float an_tile(uint32_t tS, int kcount) {
  float sa[32], sb[32];
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  tmem_ld32(tS, sa);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (c < 3) tmem_ld32(tS + 32 * (c + 1), (c & 1) ? sa : sb);
    uint32_t w[16];
    an_chunk<kMask>((c & 1) ? sb : sa, c, kcount, acc, w);
    tmem_st16(tS + 16 * c, w);
    if (c < 3) tmem_wait_ld();
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
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
  uint64_t* vfull = bars + 5;      // [3]
  uint64_t* vfree = vfull + kAnVS; // [3]
  uint64_t* sfull = vfree + kAnVS; // [2]: per query tile
  uint64_t* pready = sfull + kAnQT;
  uint64_t* odone = pready + kAnQT;
  uint64_t* drain = odone + kAnQT;
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
    }
    for (int s = 0; s < kAnVS; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&vfree[s], 1);
    }
    for (int t = 0; t < kAnQT; ++t) {
      mbar_init(&sfull[t], 1);
      mbar_init(&pready[t], 4);
      mbar_init(&odone[t], 1);
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
        const int sv = j % kAnVS;
        if (!mbar_wait(&vfree[sv], (uint32_t)((j / kAnVS) & 1) ^ 1u, abort_flag)) break;
        unsigned char* vt = sm + AnchorSmem::V + sv * kTileBytes;
        mbar_arrive_expect_tx(&vfull[sv], kTileBytes);
        tma_load_3d(vt, &tmV, &vfull[sv], h * 128, j * kAnTile, b, pol);
        tma_load_3d(vt + kBox, &tmV, &vfull[sv], h * 128 + 64, j * kAnTile, b, pol);
        ++nv;
      }
      if (*abort_flag) {
        // let the copies in flight land before the CTA exits
        int dummy = 0;
        volatile int* nd = reinterpret_cast<volatile int*>(&dummy);
        mbar_wait(qfull, 0u, nd);
        for (int i2 = nk - (nk < 2 ? nk : 2); i2 < nk; ++i2)
          mbar_wait(&kfull[i2 & 1], (uint32_t)((i2 >> 1) & 1), nd);
        for (int i2 = nv - (nv < kAnVS ? nv : kAnVS); i2 < nv; ++i2)
          mbar_wait(&vfull[i2 % kAnVS], (uint32_t)((i2 / kAnVS) & 1), nd);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    {
      // The whole warp runs the loop (warp-uniform control and descriptor
      // arithmetic) and one elected lane issues: the warp shares its
      // scheduler with two softmax warps, so the issue path is kept short.
      // Shared-memory descriptors are built once per slot, and a K step only
      // adds its offset (16-byte units) to them.
      constexpr uint32_t idS = idesc_f16(128, 128, false, false);
      constexpr uint32_t idPV = idesc_bf16(128, 128, false, true);
      const bool leader = elect_one();
      const uint64_t dQ0 = sdesc_sw128(sbase + AnchorSmem::Q, 16, 1024);
      const uint64_t dQ1 = dQ0 + (kTileBytes >> 4);
      const uint64_t dK0 = sdesc_sw128(sbase + AnchorSmem::K, 16, 1024);
      const uint64_t dK1 = dK0 + (kTileBytes >> 4);
      const uint64_t dV0 = sdesc_sw128(sbase + AnchorSmem::V, kBox, 1024);
      auto scores = [&](uint32_t d, uint64_t dq, uint64_t dk, uint64_t* bar) {   // S = q_til k_til^T
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (uint32_t)(kk >> 2) * (kBox >> 4) + (uint32_t)(kk & 3) * 2;
            umma_f16kind(d, dq + koff, dk + koff, idS, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar);
        }
        __syncwarp();
      };
      auto pv = [&](uint32_t d, uint32_t a, uint64_t dv, uint32_t acc0) {   // O += P v
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16kind_ta(d, a + kk * 8, dv + (uint32_t)kk * (2048 >> 4), idPV,
                            kk > 0 ? 1u : acc0);
        }
        __syncwarp();
      };
      auto commit = [&](uint64_t* bar) {
        if (leader) umma_commit(bar);
        __syncwarp();
      };
      bool ok = mbar_wait_warp(qfull, 0u, abort_flag) && mbar_wait_warp(&kfull[0], 0u, abort_flag);
      if (ok) {
        tc_fence_after();
        scores(tmem, dQ0, dK0, &sfull[0]);
        scores(tmem + 128, dQ1, dK0, &sfull[1]);
        commit(&kfree[0]);
      }
      int sv = 0;                 // v slot of tile j
      uint32_t phv = 0;           // its fill parity
      for (int j = 0; ok && j < nkv; ++j) {
        if (!(ok = mbar_wait_warp(&vfull[sv], phv, abort_flag))) break;
        const uint64_t dv = dV0 + (uint32_t)sv * (kTileBytes >> 4);
        const uint32_t acc0 = j > 0 ? 1u : 0u;
        const bool more = j + 1 < nkv;
        const uint64_t dk = ((j + 1) & 1) ? dK1 : dK0;     // k slot of tile j + 1
        // query tile 0: O_0 += P_0 v_j, then S_0 of tile j + 1
        if (!(ok = mbar_wait_warp(&pready[0], (uint32_t)(j & 1), abort_flag))) break;
        tc_fence_after();
        pv(tmem + kAnO, tmem, dv, acc0);
        if (more) {
          if (!(ok = mbar_wait_warp(&kfull[(j + 1) & 1], (uint32_t)(((j + 1) >> 1) & 1),
                                    abort_flag)))
            break;
          tc_fence_after();
          scores(tmem, dQ0, dk, &sfull[0]);
        }
        // query tile 1
        if (!(ok = mbar_wait_warp(&pready[1], (uint32_t)(j & 1), abort_flag))) break;
        tc_fence_after();
        pv(tmem + kAnO + 128, tmem + 128, dv, acc0);
        commit(&vfree[sv]);
        if (more) {
          scores(tmem + 128, dQ1, dk, &sfull[1]);
          commit(&kfree[(j + 1) & 1]);
        }
        if (++sv == kAnVS) {
          sv = 0;
          phv ^= 1u;
        }
      }
      if (ok)
        for (int t = 0; t < kAnQT; ++t) commit(&odone[t]);
      commit(drain);
      int dummy = 0;
      mbar_wait_warp(drain, 0, reinterpret_cast<volatile int*>(&dummy));
    }
  } else {
    // --------------------------------------------------------- softmax warps
    const int t = (warp - kAnSW0) >> 2;       // query tile
    const int q4 = warp & 3;                  // TMEM lane quarter
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + t * 128 + lane_off;
    const uint32_t tO = tmem + kAnO + t * 128 + lane_off;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait_warp(&sfull[t], (uint32_t)(j & 1), abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int kcount = g.N - j * kAnTile;
      l += kcount < kAnTile ? an_tile<true>(tS, kcount) : an_tile<false>(tS, kcount);
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
  // One wave of resident blocks: the grid-stride loop spreads the tokens.
  static std::atomic<int> resident{0};
  int per_sm = resident.load(std::memory_order_relaxed);
  if (per_sm <= 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, anchor_prep_kernel,
                                                      kAnWarpsPrep * 32, 0) != cudaSuccess ||
        per_sm <= 0)
      return GLA_ERR_CUDA;
    resident.store(per_sm, std::memory_order_relaxed);
  }
  const long long cap = (long long)per_sm * sms;
  const int grid = (int)(blocks < cap ? blocks : cap);
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
