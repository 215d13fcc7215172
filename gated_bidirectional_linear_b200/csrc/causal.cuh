// Token-level causal variant: token j is read out against the running sums,
// over tokens 0..j of the call (itself included) plus a carried-in state, of
// the per-token states v_n (beta_n k_til_n)^T and of the key features k_pls_n
// (SANA-Video notes, key design 2: causal linear attention needs only these two
// running sums).  A call continues a sequence: the caller's (S, z) come in as
// the state before the call's first token and leave as the state after its
// last.
//
// Tensor path (bf16, head dim 128), three kernels on the state partition (the
// 96-token tiles of tc_state_kernel):
//   tc_state_kernel        per-CTA partial S and z of every head segment.
//   combine_prefix_kernel  for every partial slot, in slot order, the state
//                          before it: S_start = S_in + sum of the earlier
//                          slots of its head (likewise z_start); and the state
//                          after the call, S_out = S_in + all of them.
//   tc_causal_kernel       each CTA walks its tiles again, chunk by chunk, from
//                          its slot's S_start: per 96-token chunk
//                            A   = Q_til (beta K_til)^T         (fp16 operands)
//                            U   = Q_til S_img^T + mask(A) V    (fp16 / bf16)
//                            S  += V^T (beta K_til)             (bf16)
//                          with the denominator from a running prefix sum of
//                          k_pls kept in fp32 by the transform warps.
// CUDA-core path (fp32 arithmetic, any supported head dim): simt_causal_kernel,
// one CTA per head walking its tokens in order.
#pragma once

#include "tc.cuh"

namespace gla {

// ------------------------------------------------------------ CUDA-core path

struct SimtCausalParams {
  Geom g;
  const void *q, *k, *v, *beta, *gate;
  void* out;
  float* S;          // [BH][d][d] in/out (row-major, S[a][c])
  float* z;          // [BH][d] in/out
  float* den_out;    // optional [B][N][Hh]
  float* x_out;      // optional [B][N][Hh][d]
};

constexpr int kSimtCausalThreads = 256;

template <int D>
inline size_t simt_causal_smem() {
  return ((size_t)D * (D + 1) + 9 * D + 8) * 4 + (size_t)(D / 2) * 8;
}

// One CTA per (batch, head): the state lives in shared memory (rows padded to
// D + 1 floats so that a row per thread reads without bank conflicts) and the
// tokens are taken in order: features of token j, S += v_j (beta_j k_til_j)^T,
// z += k_pls_j, then the read-out of token j against the updated sums.
template <int D, typename Tin>
__global__ void __launch_bounds__(kSimtCausalThreads) simt_causal_kernel(SimtCausalParams p) {
  constexpr int M = D / 32;
  constexpr int P = D / 2;
  constexpr int SP = D + 1;
  extern __shared__ __align__(16) float scs[];
  float* S = scs;               // [D][SP]
  float* z = S + D * SP;        // [D]
  float* kb = z + D;            // beta * k_til
  float* kp = kb + D;           // k_pls
  float* qt = kp + D;           // q_til
  float* qp = qt + D;           // q_pls
  float* vv = qp + D;
  float* gg = vv + D;
  float* u = gg + D;            // S q_til
  float* misc = u + D;          // [0] = den
  float2* cs = reinterpret_cast<float2*>(misc + 8);   // (cos, sin) of the token's pairs

  const Geom& g = p.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, b = bh / g.Hh, h = bh - b * g.Hh;
  const Tin* qin = static_cast<const Tin*>(p.q);
  const Tin* kin = static_cast<const Tin*>(p.k);
  const Tin* vin = static_cast<const Tin*>(p.v);
  const Tin* gin = static_cast<const Tin*>(p.gate);
  const Tin* bin = static_cast<const Tin*>(p.beta);
  Tin* oout = static_cast<Tin*>(p.out);

  for (int e = tid; e < D * D; e += blockDim.x) S[(e / D) * SP + e % D] = p.S[(size_t)bh * D * D + e];
  for (int e = tid; e < D; e += blockDim.x) z[e] = p.z[(size_t)bh * D + e];
  const int HW = g.H * g.W;

  for (int j = 0; j < g.N; ++j) {
    const size_t row = ((size_t)b * g.N + j) * g.Hh + h;
    const int f = j / HW, hh = (j / g.W) % g.H, ww = j % g.W;
    if (tid < P && g.rope_on) {
      const int pr = tid;
      const double x = pr < g.pt ? (double)(g.t0 + f) : (pr < g.pt + g.ph ? (double)hh : (double)ww);
      cs[pr] = rope_entry(x, g.freq[pr]);
    }
    __syncthreads();   // also: the previous token's read-out is done with gg, u, misc
    if (warp < 2) {
      // warp 0: key row -> k_pls, beta * k_til; warp 1: query row -> q_pls, q_til
      const Tin* src = (warp == 0 ? kin : qin) + row * D;
      float x[M];
      float ss = 0.f;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        x[m] = to_f32<Tin>(src[lane + 32 * m]);
        ss = fmaf(x[m], x[m], ss);
      }
      const float rstd = rsqrtf(warp_sum(ss) / (float)D + kRmsEps);
      const float scl = warp == 0 ? to_f32<Tin>(bin[row]) : 1.f;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const int e = lane + 32 * m;
        const float xp = fmaxf(x[m] * rstd, 0.f);
        const float other = __shfl_xor_sync(0xffffffffu, xp, 1);
        float xt = xp;
        if (g.rope_on) {
          const float2 c = cs[e >> 1];
          xt = (e & 1) ? fmaf(other, c.y, xp * c.x) : fmaf(-other, c.y, xp * c.x);
        }
        if (warp == 0) {
          kp[e] = xp;
          kb[e] = xt * scl;
        } else {
          qp[e] = xp;
          qt[e] = xt;
        }
      }
    } else if (warp == 2) {
#pragma unroll
      for (int m = 0; m < M; ++m) vv[lane + 32 * m] = to_f32<Tin>(vin[row * D + lane + 32 * m]);
    } else if (warp == 3) {
#pragma unroll
      for (int m = 0; m < M; ++m) gg[lane + 32 * m] = to_f32<Tin>(gin[row * D + lane + 32 * m]);
    }
    __syncthreads();
    for (int e = tid; e < D * D; e += blockDim.x) {
      const int a = e / D, c = e - a * D;
      S[a * SP + c] = fmaf(vv[a], kb[c], S[a * SP + c]);
    }
    for (int e = tid; e < D; e += blockDim.x) z[e] += kp[e];
    __syncthreads();
    if (tid < D) {
      float acc = 0.f;
      for (int c = 0; c < D; ++c) acc = fmaf(S[tid * SP + c], qt[c], acc);
      u[tid] = acc;
    }
    if (warp == kSimtCausalThreads / 32 - 1) {
      float dsum = 0.f;
      for (int c = lane; c < D; c += 32) dsum = fmaf(z[c], qp[c], dsum);
      dsum = warp_sum(dsum);
      if (lane == 0) misc[0] = dsum + g.eps;
    }
    __syncthreads();
    if (warp == 0) {
      const float den = misc[0];
      float x[M], ss = 0.f;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const int e = lane + 32 * m;
        const float sg = 1.f / (1.f + expf(-gg[e]));
        x[m] = sg * (u[e] / den);
        ss = fmaf(x[m], x[m], ss);
      }
      const float rstd = rsqrtf(warp_sum(ss) / (float)D + kRmsEps);
#pragma unroll
      for (int m = 0; m < M; ++m) oout[row * D + lane + 32 * m] = from_f32<Tin>(x[m] * rstd);
      if (p.x_out) {
#pragma unroll
        for (int m = 0; m < M; ++m) p.x_out[row * D + lane + 32 * m] = x[m];
      }
      if (p.den_out && lane == 0) p.den_out[row] = den;
    }
  }
  __syncthreads();
  for (int e = tid; e < D * D; e += blockDim.x) p.S[(size_t)bh * D * D + e] = S[(e / D) * SP + e % D];
  for (int e = tid; e < D; e += blockDim.x) p.z[(size_t)bh * D + e] = z[e];
}

// ------------------------------------------------- prefix of the partials

struct PrefixParams {
  Partition part;
  const float* part_S;   // [slots][128*128] chunk-major partials (tc_state_kernel)
  const float* part_z;   // [slots][kStTW][128], added in index order
  const float* S_in;     // carried state [BH][128][128] row-major (may alias S_out)
  const float* z_in;     // [BH][128] (may alias z_out)
  float* S_start;        // [slots][128*128] chunk-major: the state before the slot
  float* z_start;        // [slots][128]
  float* S_out;          // [BH][128][128] row-major: the state after the call
  float* z_out;          // [BH][128]
};

constexpr int kPrefixSlices = 8;     // CTAs per head, one slice of S each
constexpr int kPrefixThreads = 256;

// For head bh with partial slots c_lo + bh .. c_hi + bh: S_start(c) =
// (((S_in + P_{c_lo}) + ...) + P_{c-1}), the same left-to-right order as the
// bidirectional combine, so every slot's starting state is deterministic.
__global__ void __launch_bounds__(kPrefixThreads) combine_prefix_kernel(PrefixParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int bh = blockIdx.y, slice = blockIdx.x;
  constexpr int dd = 128 * 128;
  const long long tph = p.part.tiles_per_head;
  const int c_lo = part_cta_of(p.part, (long long)bh * tph);
  const int c_hi = part_cta_of(p.part, (long long)(bh + 1) * tph - 1);
  const int e_base = slice * (dd / kPrefixSlices);
  // Chunk-major element e holds S[a][c] with a = (e >> 3) & 127,
  // c = (e >> 10) * 8 + (e & 7).
  auto row_major = [](int e) { return ((e >> 3) & 127) * 128 + ((e >> 10) << 3) + (e & 7); };
  float4 acc[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = e_base + 4 * threadIdx.x + 4 * kPrefixThreads * k;
    acc[k] = p.S_in ? *reinterpret_cast<const float4*>(p.S_in + (size_t)bh * dd + row_major(e))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  constexpr int kBatch = 4;
  for (int c0 = c_lo; c0 <= c_hi; c0 += kBatch) {
    float4 t[kBatch][2];
#pragma unroll
    for (int bb = 0; bb < kBatch; ++bb) {
      const size_t slot = (size_t)(c0 + bb) + bh;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = e_base + 4 * threadIdx.x + 4 * kPrefixThreads * k;
        t[bb][k] = c0 + bb <= c_hi ? *reinterpret_cast<const float4*>(p.part_S + slot * dd + e)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int bb = 0; bb < kBatch; ++bb) {
      if (c0 + bb > c_hi) break;
      const size_t slot = (size_t)(c0 + bb) + bh;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int e = e_base + 4 * threadIdx.x + 4 * kPrefixThreads * k;
        *reinterpret_cast<float4*>(p.S_start + slot * dd + e) = acc[k];
        add4(acc[k], t[bb][k]);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = e_base + 4 * threadIdx.x + 4 * kPrefixThreads * k;
    *reinterpret_cast<float4*>(p.S_out + (size_t)bh * dd + row_major(e)) = acc[k];
  }
  if (slice == 0 && threadIdx.x < 128) {
    // A slot's kStTW z partials are loaded together, then added in order.
    const int t = threadIdx.x;
    float zr = p.z_in ? p.z_in[(size_t)bh * 128 + t] : 0.f;
    for (int c = c_lo; c <= c_hi; ++c) {
      const size_t slot = (size_t)c + bh;
      float zp[kStTW];
#pragma unroll
      for (int w = 0; w < kStTW; ++w) zp[w] = p.part_z[(slot * kStTW + w) * 128 + t];
      p.z_start[slot * 128 + t] = zr;
#pragma unroll
      for (int w = 0; w < kStTW; ++w) zr += zp[w];
    }
    p.z_out[(size_t)bh * 128 + t] = zr;
  }
}

// -------------------------------------------------------- tensor read-out

constexpr int kCaTile = kStTile;                 // tokens per chunk: the state partition's tile
constexpr uint32_t kCaBox = kStBox;              // 96 rows x 128 bytes
constexpr uint32_t kCaTileBytes = kStTileBytes;  // two boxes
// Warp roles: 0 producer, 1 MMA, 2..7 transform, 8..11 chain (P and the
// state image; one per TMEM lane quarter), 12..14 output (lane quarters 0..2:
// rows 0..95).  15 warps keep every scheduler at four warps or fewer, so each
// thread may hold 128 registers (a 16th or 17th warp would cut that).
constexpr int kCaTW = 6;
constexpr int kCaEW0 = 8;
constexpr int kCaEW = 4;
constexpr int kCaOW0 = 12;
constexpr int kCaOW = kCaTile / 32;
constexpr int kCaWarps = kCaOW0 + kCaOW;
constexpr int kCaThreads = kCaWarps * 32;
static_assert(kCaEW0 % 4 == 0 && kCaOW0 % 4 == 0, "role warps start on a lane quarter");
static_assert(2 + kCaTW == kCaEW0, "transform warps 2 .. kCaEW0-1");
// Index of a transform warp (0 .. kCaTW-1), or -1.
__host__ __device__ constexpr int ca_transform_index(int warp) {
  return warp >= 2 && warp < kCaEW0 ? warp - 2 : -1;
}
constexpr int kCaRowsW = kCaTile / kCaTW;         // contiguous rows per transform warp
constexpr int kCaGroups = kCaRowsW / 4;          // its row groups of 4
static_assert(kCaGroups * 4 * kCaTW == kCaTile, "whole row groups per chunk");
static_assert(kCaRowsW % 4 == 0, "row groups start on a multiple of four rows");

// TMEM columns: A = Q_til (beta K_til)^T, two read-out accumulators U, the state.
constexpr uint32_t kCaTmA = 0, kCaTmU = 128, kCaTmS = 384;

struct TcCausalSmem {
  static constexpr uint32_t Q = 0;                              // [2] q tiles -> q_til (fp16) -> P (bf16)
  static constexpr uint32_t K = Q + 2 * kCaTileBytes;           // [2] k tiles -> beta k_til (bf16)
  static constexpr uint32_t KF = K + 2 * kCaTileBytes;          // beta k_til (fp16)
  static constexpr uint32_t V = KF + kCaTileBytes;              // v tile (bf16)
  static constexpr uint32_t SIMG = V + kCaTileBytes;            // fp16 image of S * scale
  static constexpr uint32_t ROWREC = SIMG + kTileBytes;         // [2][96] RoPE row records
  static constexpr uint32_t BETA = ROWREC + 2 * kCaTile * kRecBytes;   // [2][96] f32
  static constexpr uint32_t DEN = BETA + 2 * kCaTile * 4;      // [2][96] f32
  static constexpr uint32_t GTOT = DEN + 2 * kCaTile * 4;      // [2][warp][128] f32 key sums
  static constexpr uint32_t ZRUN = GTOT + 2 * kCaTW * 128 * 4;  // [2][128] f32 key sum before a chunk
  static constexpr uint32_t RED = ZRUN + 2 * 128 * 4;           // [2][4] f32 image maxima
  static constexpr uint32_t SCL = RED + 32;                    // [4] f32 image scale per chunk
  static constexpr uint32_t BAR = SCL + 16;
  static constexpr uint32_t NBAR = 19;
  static constexpr uint32_t MISC = BAR + NBAR * 8;
  static constexpr uint32_t TAB = (MISC + 16 + 15) & ~15u;
};
static_assert(TcCausalSmem::SIMG % 1024 == 0 && TcCausalSmem::KF % 1024 == 0, "swizzle atoms");

struct TcCausalParams {
  Geom g;
  Partition part;
  const __nv_bfloat16* beta;
  const __nv_bfloat16* gate;
  __nv_bfloat16* out;
  const float* S_start;   // [slots][128*128] chunk-major
  const float* z_start;   // [slots][128]
  float* den_out;         // optional [B][N][Hh]
  float* x_out;           // optional [B][N][Hh][128]
  int tab_entries;
};

__device__ __forceinline__ f2_t f2_add(f2_t a, f2_t b) {
  f2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ f2_t shfl_f2(f2_t v, int src) {
  return f2(__shfl_sync(0xffffffffu, f2_lo(v), src), __shfl_sync(0xffffffffu, f2_hi(v), src));
}

// bar.sync with an AND over the participating threads' predicates: every
// thread gets the same answer, so a role leaves its loop together.
__device__ __forceinline__ bool bar_red_and(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred q, r;\n\t"
      "setp.ne.b32 q, %1, 0;\n\t"
      "bar.red.and.pred r, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, r;\n\t}\n"
      : "=r"(r)
      : "r"(pred ? 1 : 0), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint4 ldg_nc128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void stg128(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// The power of two that puts a head maximum hm in [2^13, 2^14) (1 for hm = 0),
// kept within [2^-60, 2^60].
__device__ __forceinline__ float image_scale(float hm) {
  if (!(hm > 0.f)) return 1.f;
  int E = (int)((__float_as_uint(hm) >> 23) & 0xFFu) - 126;
  int s = 14 - E;
  s = s < -60 ? -60 : (s > 60 ? 60 : s);
  return __uint_as_float((uint32_t)(127 + s) << 23);
}

// The fp16 image of the state in TMEM (one row per epilogue thread: row a of
// S is TMEM lane a) as the read-out MMA's B operand: two K-blocks of [128
// rows][64 columns], 16-byte chunks XOR-swizzled by (row & 7).  The four
// epilogue warps agree on the head maximum through shared memory; the barrier
// also carries their wait outcomes (ok), so they leave together on a timeout.
// Returns the scale (power of two) the image carries.
__device__ __forceinline__ float causal_image(uint32_t tS, unsigned char* simg, float* red,
                                              int par, int q4, int lane, bool& ok) {
  const int a = q4 * 32 + lane;
  float m = 0.f;
  if (ok) {
#pragma unroll 1
    for (int blk = 0; blk < 4; ++blk) {
      float v[32];
      tmem_ld32(tS + blk * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[par * 4 + q4] = m;
  ok = bar_red_and(3, kCaEW * 32, ok);
  if (!ok) return 1.f;
  const float hm = fmaxf(fmaxf(red[par * 4 + 0], red[par * 4 + 1]),
                         fmaxf(red[par * 4 + 2], red[par * 4 + 3]));
  const float sc = image_scale(hm);
  const uint32_t sw = (uint32_t)(a & 7);
#pragma unroll 1
  for (int blk = 0; blk < 4; ++blk) {
    float v[32];
    tmem_ld32(tS + blk * 32, v);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = blk * 4 + q;   // 16-byte chunk of the row: columns 8k .. 8k+7
      uint4 o;
      o.x = pack_f16(v[8 * q + 0] * sc, v[8 * q + 1] * sc);
      o.y = pack_f16(v[8 * q + 2] * sc, v[8 * q + 3] * sc);
      o.z = pack_f16(v[8 * q + 4] * sc, v[8 * q + 5] * sc);
      o.w = pack_f16(v[8 * q + 6] * sc, v[8 * q + 7] * sc);
      sts128(smem_u32(simg) + (uint32_t)(k >> 3) * 16384u + (uint32_t)a * 128u +
                 ((((uint32_t)(k & 7)) ^ sw) << 4),
             o);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  return sc;
}

template <bool kDebug>
__global__ void __launch_bounds__(kCaThreads, 1)
    tc_causal_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmG, TcCausalParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + TcCausalSmem::BAR);
  uint64_t* qkfull = bars;          // [2] q, k tiles landed + beta / row records
  uint64_t* qkfree = bars + 2;      // [2] MMAs done with the q / k slot
  uint64_t* vfull = bars + 4;
  uint64_t* vfree = bars + 5;
  uint64_t* tready = bars + 6;      // transform warps done with the chunk
  uint64_t* kffree = bars + 7;      // MMA done with the fp16 key tile
  uint64_t* afull = bars + 8;       // A and the inter-chunk read-out in TMEM
  uint64_t* pready = bars + 9;      // P written (A read)
  uint64_t* imgready = bars + 10;   // the image of the state before the chunk
  uint64_t* ufull = bars + 11;      // [2]
  uint64_t* ufree = bars + 13;      // [2]
  uint64_t* sfull = bars + 15;      // state MMA of the chunk done
  uint64_t* denfree = bars + 16;    // [2]
  uint64_t* drain = bars + 18;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + TcCausalSmem::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + TcCausalSmem::MISC + 4);
  float2* tab = reinterpret_cast<float2*>(sm + TcCausalSmem::TAB);
  float* den_ring = reinterpret_cast<float*>(sm + TcCausalSmem::DEN);
  float* gtot = reinterpret_cast<float*>(sm + TcCausalSmem::GTOT);
  float* zrun = reinterpret_cast<float*>(sm + TcCausalSmem::ZRUN);
  float* red = reinterpret_cast<float*>(sm + TcCausalSmem::RED);

  const Geom& g = p.g;
  const Partition& part = p.part;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long wb = part_begin(part, c), we = part_begin(part, c + 1);
  const RopeWindow win = rope_window(g, part, wb, we - 1);
  const int tph = part.tiles_per_head;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qkfull[s], 2);
      mbar_init(&qkfree[s], 1);
      mbar_init(&ufull[s], 1);
      mbar_init(&ufree[s], kCaOW);
      mbar_init(&denfree[s], kCaOW);
    }
    mbar_init(vfull, 1);
    mbar_init(vfree, 1);
    mbar_init(tready, kCaTW);
    mbar_init(kffree, 1);
    mbar_init(afull, 1);
    mbar_init(pready, kCaEW);
    mbar_init(imgready, kCaEW);
    mbar_init(sfull, 1);
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
    // The inputs were complete before the state kernel started (it waited
    // for them), and this kernel starts only after the prefix kernel, which
    // waited for the state kernel: no grid dependency to wait for here.
    const uint64_t pol = policy_evict_first();
    const uint64_t pol_beta = policy_evict_last();
    long long it = 0;
    int issued_qk = 0, issued_v = 0;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<2> rq;
    uint16_t braw[kCaTile / 32];
    auto fetch_beta = [&](const ItemWalk& w) {
#pragma unroll
      for (int k2 = 0; k2 < kCaTile / 32; ++k2) {
        const int n = w.ti * kCaTile + lane + 32 * k2;
        braw[k2] = n < g.N ? ld_u16_policy(p.beta + ((size_t)w.b * g.N + n) * g.Hh + w.h, pol_beta)
                           : (uint16_t)0;
      }
    };
    if (iw.more()) fetch_beta(iw);
    for (; iw.more(); iw.next(), rq.next(), ++it) {
      const int s = rq.s;
      if (!mbar_wait_warp(&qkfree[s], rq.ph ^ 1u, abort_flag)) break;
      const int b = iw.b, h = iw.h, n0 = iw.ti * kCaTile;
      if (lane == 0) {
        mbar_arrive_expect_tx(&qkfull[s], 2 * kCaTileBytes);
        unsigned char* qt = sm + TcCausalSmem::Q + s * kCaTileBytes;
        unsigned char* kt = sm + TcCausalSmem::K + s * kCaTileBytes;
        tma_load_3d(qt, &tmQ, &qkfull[s], h * 128, n0, b, pol);
        tma_load_3d(qt + kCaBox, &tmQ, &qkfull[s], h * 128 + 64, n0, b, pol);
        tma_load_3d(kt, &tmK, &qkfull[s], h * 128, n0, b, pol);
        tma_load_3d(kt + kCaBox, &tmK, &qkfull[s], h * 128 + 64, n0, b, pol);
        // The epilogue reads this chunk's gate rows with plain loads.
        tma_prefetch_3d(&tmG, h * 128, n0, b);
        tma_prefetch_3d(&tmG, h * 128 + 64, n0, b);
      }
      ++issued_qk;
      float* bs = reinterpret_cast<float*>(sm + TcCausalSmem::BETA + s * kCaTile * 4);
#pragma unroll
      for (int k2 = 0; k2 < kCaTile / 32; ++k2)
        bs[lane + 32 * k2] = __uint_as_float((uint32_t)braw[k2] << 16);
      {
        ItemWalk nx = iw;
        nx.next();
        if (nx.more()) fetch_beta(nx);
      }
      if (g.rope_on)
        tile_rowrec<kCaTile>(g, win, n0, lane, sm + TcCausalSmem::ROWREC + s * kCaTile * kRecBytes);
      __syncwarp();
      if (lane == 0) mbar_arrive(&qkfull[s]);
      if (!mbar_wait_warp(vfree, (uint32_t)((it & 1) ^ 1), abort_flag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(vfull, kCaTileBytes);
        unsigned char* vt = sm + TcCausalSmem::V;
        tma_load_3d(vt, &tmV, vfull, h * 128, n0, b, pol);
        tma_load_3d(vt + kCaBox, &tmV, vfull, h * 128 + 64, n0, b, pol);
      }
      ++issued_v;
    }
    if (*abort_flag && lane == 0) {
      // Let the loads in flight land before shared memory is released.
      int dummy = 0;
      volatile int* nd = reinterpret_cast<volatile int*>(&dummy);
      for (int i2 = issued_qk - (issued_qk < 2 ? issued_qk : 2); i2 < issued_qk; ++i2)
        mbar_wait(&qkfull[i2 & 1], (uint32_t)((i2 >> 1) & 1), nd);
      if (issued_v > 0) mbar_wait(vfull, (uint32_t)((issued_v - 1) & 1), nd);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idA = idesc_f16(128, kCaTile, false, false);
      constexpr uint32_t idI = idesc_f16(128, 128, false, false);
      constexpr uint32_t idPV = idesc_bf16(128, 128, false, true);
      constexpr uint32_t idS = idesc_bf16(128, 128, true, true);
      const uint32_t kf = sbase + TcCausalSmem::KF;
      const uint32_t vt = sbase + TcCausalSmem::V;
      const uint32_t simg = sbase + TcCausalSmem::SIMG;
      ItemWalk iw(wb, we, tph, g.Hh);
      RingPos<2> rq;
      long long i = 0;
      for (; iw.more(); iw.next(), rq.next(), ++i) {
        const uint32_t par = (uint32_t)(i & 1);
        const int s = rq.s;   // q / k slot and read-out accumulator of the chunk
        const uint32_t qt = sbase + TcCausalSmem::Q + s * kCaTileBytes;
        const uint32_t kt = sbase + TcCausalSmem::K + s * kCaTileBytes;
        const uint32_t tU = tmem + kCaTmU + (uint32_t)s * 128u;
        if (!mbar_wait(tready, par, abort_flag)) break;
        tc_fence_after();
        // A = Q_til (beta K_til)^T: M = 128 (rows 96.. unused), N = 96, K = 128 channels.
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)(kk >> 2) * kCaBox + (uint32_t)(kk & 3) * 32;
          umma_f16kind(tmem + kCaTmA, sdesc_sw128(qt + koff, 16, 1024),
                       sdesc_sw128(kf + koff, 16, 1024), idA, kk > 0 ? 1u : 0u);
        }
        umma_commit(kffree);
        if (!mbar_wait(imgready, par, abort_flag)) break;
        if (!mbar_wait(&ufree[s], rq.ph ^ 1u, abort_flag)) break;
        tc_fence_after();
        // U = Q_til S_img^T: the chunk's read-out against the state before it.
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t qoff = (uint32_t)(kk >> 2) * kCaBox + (uint32_t)(kk & 3) * 32;
          const uint32_t soff = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32;
          umma_f16kind(tU, sdesc_sw128(qt + qoff, 16, 1024), sdesc_sw128(simg + soff, 16, 1024),
                       idI, kk > 0 ? 1u : 0u);
        }
        umma_commit(afull);
        if (!mbar_wait(pready, par, abort_flag)) break;
        if (!mbar_wait(vfull, par, abort_flag)) break;
        tc_fence_after();
        // U += P V: the chunk's own tokens, P = mask(A) * scale in the q slot.
#pragma unroll
        for (int kk = 0; kk < kCaTile / 16; ++kk) {
          const uint32_t poff = (uint32_t)(kk >> 2) * kCaBox + (uint32_t)(kk & 3) * 32;
          umma_f16kind(tU, sdesc_sw128(qt + poff, 16, 1024),
                       sdesc_sw128(vt + kk * 2048, kCaBox, 1024), idPV, 1u);
        }
        umma_commit(&ufull[s]);
        // S += V^T (beta K_til): the state after the chunk.
#pragma unroll
        for (int kk = 0; kk < kCaTile / 16; ++kk)
          umma_f16kind(tmem + kCaTmS, sdesc_sw128(vt + kk * 2048, kCaBox, 1024),
                       sdesc_sw128(kt + kk * 2048, kCaBox, 1024), idS, 1u);
        umma_commit(sfull);
        umma_commit(&qkfree[s]);
        umma_commit(vfree);
      }
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy));
    }
  } else if (ca_transform_index(warp) >= 0) {
    // --------------------------------------------------- transform warps
    // q -> q_til (fp16), k -> beta k_til (bf16 in place, fp16 copy), and the
    // denominator of every row from the running sum of k_pls.  Warp tw owns
    // kCaRowsW contiguous rows of the chunk (row groups of four).  A
    // first pass sums the warp's k_pls; after one barrier each warp knows the
    // key sum before its rows (the sum before the chunk plus the earlier
    // warps' sums), and the main pass carries it row group by row group.
    // Warp sums are stored with 16-byte chunk q of lane j at float4 index
    // q * 8 + j, so that the 8 lanes that read one chunk read 128 contiguous
    // bytes.
    const int tw = ca_transform_index(warp);
    rope_build(tab, g, win, tw * 32 + lane, kCaTW * 32);
    named_barrier(1, kCaTW * 32);
    const int rg = tw_row(lane), j = tw_chunk(lane);
    LaneRope lr;
    lane_rope(g, j, smem_u32(tab), lr);
    // The lane's two 16-byte chunks in rows rg and 4 + rg: a row group
    // starting at row R (a multiple of 4) has swizzle phase 4 ((R >> 2) & 1) + rg.
    // (Four scalars chosen by select, not an array indexed by the phase: that
    // would live in local memory and be reloaded for every row group.)
    uint32_t ch0a, ch1a, ch0b, ch1b;
    lane_chunks(0, kCaBox, rg, j, ch0a, ch1a);
    lane_chunks(0, kCaBox, 4 + rg, j, ch0b, ch1b);
    // Lanes of the row group above: rg - 1 (rg = lane bit 2 | lane bit 4 << 1),
    // rg - 2, and the group's last row (rg = 3).
    const int src1 = (rg & 1) ? (lane ^ 4) : (lane ^ 20);
    const int src2 = lane ^ 16;
    const int src3 = lane | 20;
    bool waited_grid = false;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<2> rq;
    long long i = 0;
    for (; iw.more(); iw.next(), rq.next(), ++i) {
      const int s = rq.s;
      const int par = (int)(i & 1);
      bool ok = mbar_wait_warp(&qkfull[s], rq.ph, abort_flag);
      ok = ok && mbar_wait_warp(kffree, (uint32_t)((i & 1) ^ 1), abort_flag);
      ok = ok && mbar_wait_warp(&denfree[s], rq.ph ^ 1u, abort_flag);
      if (!bar_red_and(2, kCaTW * 32, ok && !*abort_flag)) break;
      const uint32_t qt = sbase + TcCausalSmem::Q + s * kCaTileBytes;
      const uint32_t kt = sbase + TcCausalSmem::K + s * kCaTileBytes;
      const uint32_t kf = sbase + TcCausalSmem::KF;
      const float* bs = reinterpret_cast<const float*>(sm + TcCausalSmem::BETA + s * kCaTile * 4);
      const uint32_t rec_s = sbase + TcCausalSmem::ROWREC + s * kCaTile * kRecBytes;
      float* den = den_ring + s * kCaTile;
      const int n0 = iw.ti * kCaTile;
      float* zr_now = zrun + par * 128;
      if (iw.first && tw == 0 && rg == 0) {
        // The key sum of the head starts at its slot's z_start.
        if (!waited_grid) {
          pdl_wait();
          waited_grid = true;
        }
        const float* zs = p.z_start + ((size_t)c + iw.bh) * 128 + 16 * j;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<float4*>(zr_now + 16 * j + 4 * q) =
              *reinterpret_cast<const float4*>(zs + 4 * q);
      }
      // Pass 1: this warp's sum of k_pls over its rows.
      f2_t ta[8];
#pragma unroll
      for (int i2 = 0; i2 < 8; ++i2) ta[i2] = 0ull;
#pragma unroll 1
      for (int u = 0; u < kCaGroups; ++u) {
        const int R = kCaRowsW * tw + 4 * u;
        const uint32_t roff = (uint32_t)(R & ~7) * 128u;
        const int ph = (R >> 2) & 1;
        f2_t x[8];
        unpack8(lds128(kt + (ph ? ch0b : ch0a) + roff), lds128(kt + (ph ? ch1b : ch1a) + roff), x);
        const float rstd = row_rstd(x);
        const f2_t rstd2 = f2(rstd, rstd);
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) ta[i2] = f2_fma(f2_relu(x[i2]), rstd2, ta[i2]);
      }
#pragma unroll
      for (int i2 = 0; i2 < 8; ++i2) {
        ta[i2] = f2_add(ta[i2], shfl_f2(ta[i2], lane ^ 4));
        ta[i2] = f2_add(ta[i2], shfl_f2(ta[i2], lane ^ 16));
      }
      float* gt = gtot + par * (kCaTW * 128);
      if (rg == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<float4*>(gt + tw * 128 + (q * 8 + j) * 4) =
              make_float4(f2_lo(ta[2 * q]), f2_hi(ta[2 * q]), f2_lo(ta[2 * q + 1]),
                          f2_hi(ta[2 * q + 1]));
      }
      named_barrier(2, kCaTW * 32);
      // The key sum before the warp's first row; warp 0 also records the sum
      // after the chunk for the next one.
      f2_t off[8], tot[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 t = *reinterpret_cast<const float4*>(zr_now + 16 * j + 4 * q);
        off[2 * q] = f2(t.x, t.y);
        off[2 * q + 1] = f2(t.z, t.w);
        tot[2 * q] = off[2 * q];
        tot[2 * q + 1] = off[2 * q + 1];
      }
#pragma unroll 1
      for (int w2 = 0; w2 < kCaTW; ++w2) {
        f2_t gv[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 t = *reinterpret_cast<const float4*>(gt + w2 * 128 + (q * 8 + j) * 4);
          gv[2 * q] = f2(t.x, t.y);
          gv[2 * q + 1] = f2(t.z, t.w);
        }
        if (w2 < tw) {
#pragma unroll
          for (int i2 = 0; i2 < 8; ++i2) off[i2] = f2_add(off[i2], gv[i2]);
        }
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) tot[i2] = f2_add(tot[i2], gv[i2]);
      }
      if (tw == 0 && rg == 0) {
        float* zr_next = zrun + (par ^ 1) * 128 + 16 * j;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<float4*>(zr_next + 4 * q) =
              make_float4(f2_lo(tot[2 * q]), f2_hi(tot[2 * q]), f2_lo(tot[2 * q + 1]),
                          f2_hi(tot[2 * q + 1]));
      }
      // Pass 2: the transforms and the denominators, row group by row group.
#pragma unroll 1
      for (int u = 0; u < kCaGroups; ++u) {
        const int R = kCaRowsW * tw + 4 * u;
        const int r = R + rg;
        const uint32_t roff = (uint32_t)(R & ~7) * 128u;
        const int ph = (R >> 2) & 1;
        const uint32_t c0 = (ph ? ch0b : ch0a) + roff, c1 = (ph ? ch1b : ch1a) + roff;
        uint32_t t012 = 0, t345 = 0, t67 = 0;
        if (g.rope_on) lane_rope_row(lr, rec_s + r * kRecBytes, t012, t345, t67);
        const uint4 k0 = lds128(kt + c0), k1 = lds128(kt + c1);
        const uint4 q0 = lds128(qt + c0), q1 = lds128(qt + c1);
        f2_t e[8];
        if (g.rope_on) tab_load8(t012, t345, t67, e);
        const float bet = bs[r];
        // keys
        f2_t kp[8];
        {
          f2_t x[8];
          unpack8(k0, k1, x);
          const float rstd = row_rstd(x);
          const f2_t rstd2 = f2(rstd, rstd);
#pragma unroll
          for (int i2 = 0; i2 < 8; ++i2) {
            x[i2] = f2_relu(x[i2]);
            kp[i2] = f2_mul(x[i2], rstd2);
          }
          uint4 o0, o1;
          rope_scale_pack<false>(g.rope_on, e, x, rstd * bet, o0, o1);
          sts128(kt + c0, o0);
          sts128(kt + c1, o1);
          rope_scale_pack<true>(g.rope_on, e, x, rstd * bet, o0, o1);
          sts128(kf + c0, o0);
          sts128(kf + c1, o1);
        }
        // queries
        f2_t qp[8];
        {
          f2_t y[8];
          unpack8(q0, q1, y);
          const float rstd = row_rstd(y);
          const f2_t rstd2 = f2(rstd, rstd);
#pragma unroll
          for (int i2 = 0; i2 < 8; ++i2) {
            y[i2] = f2_relu(y[i2]);
            qp[i2] = f2_mul(y[i2], rstd2);
          }
          uint4 o0, o1;
          rope_scale_pack<true>(g.rope_on, e, y, rstd, o0, o1);
          sts128(qt + c0, o0);
          sts128(qt + c1, o1);
        }
        // Inclusive prefix of k_pls over the group's four rows (rg order).
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) {
          const f2_t t = shfl_f2(kp[i2], src1);
          if (rg >= 1) kp[i2] = f2_add(kp[i2], t);
        }
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) {
          const f2_t t = shfl_f2(kp[i2], src2);
          if (rg >= 2) kp[i2] = f2_add(kp[i2], t);
        }
        // den = q_pls . (key sum before the group + this row's prefix) + eps
        f2_t dd = 0ull;
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) dd = f2_fma(qp[i2], f2_add(off[i2], kp[i2]), dd);
        const float dn = row_sum(f2_lo(dd) + f2_hi(dd)) + g.eps;
        if (j == 0) {
          den[r] = dn;
          const int n = n0 + r;
          if (kDebug && p.den_out && n < g.N)
            p.den_out[((size_t)iw.b * g.N + n) * g.Hh + iw.h] = dn;
        }
        // The next group starts after this group's last row.
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) off[i2] = f2_add(off[i2], shfl_f2(kp[i2], src3));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(tready);
    }
  } else if (warp < kCaOW0) {
    // -------------------------------------------------------- chain warps (8..11)
    // The two steps the MMA chain waits on: P = mask(A) * scale after the
    // first MMAs of a chunk, and the image of the state after its state MMA
    // (the next chunk's read-out operand).  Thread = TMEM lane = state row;
    // rows 96..127 take part in the image only.
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + kCaTmS + lane_off;
    unsigned char* simg = sm + TcCausalSmem::SIMG;
    float* scl = reinterpret_cast<float*>(sm + TcCausalSmem::SCL);
    bool waited_grid = false;
    bool ok = true;
    uint32_t rpar = 0;
    float cur_scale = 1.f;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<2> rq;
    long long i = 0;
    for (; iw.more(); iw.next(), rq.next(), ++i) {
      const uint32_t par = (uint32_t)(i & 1);
      const int s = rq.s;
      if (iw.first) {
        // The state before the segment: this slot's S_start into TMEM, then
        // its image.  The previous segment's last state MMA was waited for
        // (sfull) in the previous iteration.
        if (!waited_grid) {
          pdl_wait();
          waited_grid = true;
        }
        if (ok) {
          const float* src = p.S_start + ((size_t)c + iw.bh) * 16384 + (size_t)row * 8;
#pragma unroll 1
          for (int blk = 0; blk < 4; ++blk) {
            float v[32];
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
              const float4 a0 = *reinterpret_cast<const float4*>(src + (blk * 4 + cb) * 1024);
              const float4 a1 = *reinterpret_cast<const float4*>(src + (blk * 4 + cb) * 1024 + 4);
              v[8 * cb + 0] = a0.x; v[8 * cb + 1] = a0.y; v[8 * cb + 2] = a0.z; v[8 * cb + 3] = a0.w;
              v[8 * cb + 4] = a1.x; v[8 * cb + 5] = a1.y; v[8 * cb + 6] = a1.z; v[8 * cb + 7] = a1.w;
            }
            tmem_st32(tS + blk * 32, v);
          }
          tmem_wait_st();
        }
        cur_scale = causal_image(tS, simg, red, (int)rpar, q4, lane, ok);
        rpar ^= 1u;
        if (!ok) break;
        if (threadIdx.x == kCaEW0 * 32) scl[i & 3] = cur_scale;
        __syncwarp();
        if (lane == 0) mbar_arrive(imgready);
      }
      // (a) P = mask(A) * scale, over the chunk's q slot.  Wait outcomes are
      // warp-uniform: the tcgen05 loads below are warp-collective.
      ok = ok && mbar_wait_warp(afull, par, abort_flag);
      if (ok && row < kCaTile) {
        tc_fence_after();
        const uint32_t pslot = sbase + TcCausalSmem::Q + s * kCaTileBytes;
        const uint32_t sw = (uint32_t)(row & 7);
#pragma unroll 1
        for (int blk = 0; blk < kCaTile / 32; ++blk) {
          float a[32];
          tmem_ld32(tmem + kCaTmA + lane_off + blk * 32, a);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int k = blk * 4 + q;     // columns (tokens) 8k .. 8k+7
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int n = 8 * k + 2 * e;
              const float lo = n <= row ? a[8 * q + 2 * e] * cur_scale : 0.f;
              const float hi = n + 1 <= row ? a[8 * q + 2 * e + 1] * cur_scale : 0.f;
              w4[e] = pack_bf16(lo, hi);
            }
            sts128(pslot + (uint32_t)(k >> 3) * kCaBox + (uint32_t)row * 128u +
                       ((((uint32_t)(k & 7)) ^ sw) << 4),
                   make_uint4(w4[0], w4[1], w4[2], w4[3]));
          }
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pready);
      // (c) the image of the state after the chunk, for the next chunk of
      // the segment.
      ok = ok && mbar_wait_warp(sfull, par, abort_flag);
      tc_fence_after();
      if (!iw.last) {
        cur_scale = causal_image(tS, simg, red, (int)rpar, q4, lane, ok);
        rpar ^= 1u;
        if (!ok) break;
        if (threadIdx.x == kCaEW0 * 32) scl[(i + 1) & 3] = cur_scale;
        __syncwarp();
        if (lane == 0) mbar_arrive(imgready);
      } else {
        ok = bar_red_and(3, kCaEW * 32, ok);
        if (!ok) break;
      }
    }
  } else if (warp < kCaOW0 + kCaOW) {
    // ------------------------------------------------------- output warps
    // Thread = TMEM lane = token row 0..95 of the chunk:
    // x = sigmoid(g) * U / (den * scale), the output RMSNorm, bf16 stores.
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float* scl = reinterpret_cast<const float*>(sm + TcCausalSmem::SCL);
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<2> rq;
    long long i = 0;
    for (; iw.more(); iw.next(), rq.next(), ++i) {
      const uint32_t par = (uint32_t)(i & 1);
      const int s = rq.s;
      const int b = iw.b, h = iw.h, n0 = iw.ti * kCaTile;
      // den (transform warps) and the scale (chain warps) of the chunk: their
      // barriers have completed for this chunk and at most one chunk more, so
      // waiting on them is immediate and orders the reads after the writes.
      bool ok = mbar_wait_warp(tready, par, abort_flag);
      ok = ok && mbar_wait_warp(imgready, par, abort_flag);
      ok = ok && mbar_wait_warp(&ufull[s], rq.ph, abort_flag);
      if (!ok) break;
      const int n = n0 + row;
      const bool valid = n < g.N;   // per lane: guards global memory only
      tc_fence_after();
      const float hc = 0.5f / (den_ring[s * kCaTile + row] * scl[i & 3]);
      const uint32_t tU = tmem + kCaTmU + (uint32_t)s * 128u + lane_off;
      const size_t rowoff = (((size_t)b * g.N + (valid ? n : 0)) * g.Hh + h) * 128;
      const __nv_bfloat16* grow = p.gate + rowoff;
      const f2_t hc2 = f2(hc, hc), half2 = f2(0.5f, 0.5f);
      f2_t ss2 = 0ull;
      // Gate loads run one 32-channel block ahead of their use (the producer
      // has prefetched the chunk's gate tile into L2).
      uint4 gv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        gv[q] = valid ? ldg_nc128(grow + 8 * q) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        uint4 gn[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          gn[q] = (valid && cb < 3) ? ldg_nc128(grow + (cb + 1) * 32 + 8 * q)
                                    : make_uint4(0u, 0u, 0u, 0u);
        float u[32];
        tmem_ld32(tU + cb * 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 gq = gv[q];
          const uint32_t wv[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const f2_t hg = f2_mul(f2_bf(wv[e]), half2);
            const f2_t t = f2(tanh_approx(f2_lo(hg)), tanh_approx(f2_hi(hg)));
            const f2_t sg = f2_fma(hc2, t, hc2);
            const f2_t x = f2_mul(sg, f2(u[q * 8 + 2 * e], u[q * 8 + 2 * e + 1]));
            ss2 = f2_fma(x, x, ss2);
            u[q * 8 + 2 * e] = f2_lo(x);
            u[q * 8 + 2 * e + 1] = f2_hi(x);
          }
        }
        if (kDebug && p.x_out && valid) {
          float* xo = p.x_out + rowoff + cb * 32;
#pragma unroll
          for (int i2 = 0; i2 < 32; i2 += 4)
            *reinterpret_cast<float4*>(xo + i2) = make_float4(u[i2], u[i2 + 1], u[i2 + 2], u[i2 + 3]);
        }
        tmem_st32(tU + cb * 32, u);
#pragma unroll
        for (int q = 0; q < 4; ++q) gv[q] = gn[q];
      }
      tmem_wait_st();
      const float rstd = rsqrtf((f2_lo(ss2) + f2_hi(ss2)) * (1.f / 128.f) + kRmsEps);
      const f2_t rstd2 = f2(rstd, rstd);
      __nv_bfloat16* orow = p.out + rowoff;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float x[32];
        tmem_ld32(tU + cb * 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const f2_t y = f2_mul(f2(x[q * 8 + 2 * e], x[q * 8 + 2 * e + 1]), rstd2);
            o[e] = pack_bf16(f2_lo(y), f2_hi(y));
          }
          if (valid) stg128(orow + cb * 32 + 8 * q, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ufree[s]);
        mbar_arrive(&denfree[s]);
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

inline size_t tc_causal_smem(int tab_entries) {
  return 1024 + TcCausalSmem::TAB + (size_t)tab_entries * 8;
}

// The tensor path of a causal call: state partials, their prefix, the causal
// read-out, each a programmatic dependent of the kernel before it.  S / z are
// the caller's carried state, read and replaced by the state after the call.
inline gla_status run_causal_tensor(const Geom& g, const void* q, const void* k, const void* v,
                                    const void* beta, const void* gate, void* out, float* S,
                                    float* z, float* part_S, float* part_z, float* S_start,
                                    float* z_start, float* den_dbg, float* x_dbg, int sms,
                                    cudaStream_t stream, void* const* events) {
  auto mark = [&](int i) {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream);
  };
  if (sms <= 0) return GLA_ERR_CUDA;
  if (g.H >= (1 << kPosBits) || g.W >= (1 << kPosBits) || g.T >= (1 << kPosBits))
    return GLA_ERR_UNSUPPORTED;
  if (!tc_rope_lanes_ok(g)) return GLA_ERR_UNSUPPORTED;
  const Partition spart = tc_state_partition(g, sms);
  const int stab = tc_table_entries(g, spart);
  const size_t smem_st = tc_state_smem(stab), smem_ca = tc_causal_smem(stab);
  if (smem_st > kMaxSmem || smem_ca > kMaxSmem) return GLA_ERR_UNSUPPORTED;

  CUtensorMap mK, mV, mQ, mG;
  if (!make_act_map(&mK, k, g, kStTile) || !make_act_map(&mV, v, g, kStTile) ||
      !make_act_map(&mQ, q, g, kStTile) || !make_act_map(&mG, gate, g, kStTile))
    return GLA_ERR_CUDA;

  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;

  TcStateParams sp = {};
  sp.g = g; sp.part = spart;
  sp.beta = static_cast<const __nv_bfloat16*>(beta);
  sp.part_S = part_S; sp.part_z = part_z; sp.tab_entries = stab;
  sp.rope_tab = nullptr;
  sp.wait_ns = kWaitLimitNs;
  sp.stall_item = -1;
  if (!ensure_max_smem(tc_state_kernel, 0)) return GLA_ERR_CUDA;
  cudaLaunchConfig_t sc = {};
  sc.gridDim = dim3(spart.grid);
  sc.blockDim = dim3(kStThreads);
  sc.dynamicSmemBytes = smem_st;
  sc.stream = stream;
  sc.attrs = pdl;
  sc.numAttrs = 1;
  if (mark(0) != cudaSuccess) return GLA_ERR_CUDA;
  if (cudaLaunchKernelEx(&sc, tc_state_kernel, mK, mV, sp) != cudaSuccess || mark(1) != cudaSuccess)
    return GLA_ERR_CUDA;

  PrefixParams pp = {};
  pp.part = spart;
  pp.part_S = part_S; pp.part_z = part_z;
  pp.S_in = S; pp.z_in = z;
  pp.S_start = S_start; pp.z_start = z_start;
  pp.S_out = S; pp.z_out = z;
  cudaLaunchConfig_t pc = {};
  pc.gridDim = dim3(kPrefixSlices, g.B * g.Hh);
  pc.blockDim = dim3(kPrefixThreads);
  pc.stream = stream;
  pc.attrs = pdl;
  pc.numAttrs = 1;
  if (cudaLaunchKernelEx(&pc, combine_prefix_kernel, pp) != cudaSuccess || mark(2) != cudaSuccess)
    return GLA_ERR_CUDA;

  TcCausalParams cp = {};
  cp.g = g; cp.part = spart;
  cp.beta = static_cast<const __nv_bfloat16*>(beta);
  cp.gate = static_cast<const __nv_bfloat16*>(gate);
  cp.out = static_cast<__nv_bfloat16*>(out);
  cp.S_start = S_start; cp.z_start = z_start;
  cp.den_out = den_dbg; cp.x_out = x_dbg; cp.tab_entries = stab;
  const bool dbg = den_dbg != nullptr || x_dbg != nullptr;
  cudaLaunchConfig_t kc = {};
  kc.gridDim = dim3(spart.grid);
  kc.blockDim = dim3(kCaThreads);
  kc.dynamicSmemBytes = smem_ca;
  kc.stream = stream;
  kc.attrs = pdl;
  kc.numAttrs = 1;
  cudaError_t e;
  if (dbg) {
    if (!ensure_max_smem(tc_causal_kernel<true>, 1)) return GLA_ERR_CUDA;
    e = cudaLaunchKernelEx(&kc, tc_causal_kernel<true>, mQ, mK, mV, mG, cp);
  } else {
    if (!ensure_max_smem(tc_causal_kernel<false>, 2)) return GLA_ERR_CUDA;
    e = cudaLaunchKernelEx(&kc, tc_causal_kernel<false>, mQ, mK, mV, mG, cp);
  }
  return e == cudaSuccess && mark(3) == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

}  // namespace gla
