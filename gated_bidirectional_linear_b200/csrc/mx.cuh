// The operator on FP8 (OCP MX) inputs: q, k, v and g arrive as E4M3 codes
// [B][N][Hh][128] (one byte per element) with one E8M0 scale per 32
// consecutive channels ([B][N][Hh][4] bytes); beta stays bf16 and the output is
// bf16.  The decoded value of element i is e4m3(code_i) * 2^(scale - 127);
// every decoded value is exact in bf16 and fp32 (three mantissa bits), so the
// kernels compute the same operator as the bf16 path on the decoded inputs.
//
//   tc_state_mx_kernel  the state reduction of tc_state_kernel with the k and
//                       v tiles arriving as 96 x 128-byte fp8 boxes (3-stage
//                       ring); the transform warps decode both into the bf16
//                       operand tiles the MMA reads (2 slots): beta k_til as
//                       before, and v exactly.
//   combine             unchanged (combine.cuh).
//   tc_apply_mx_kernel  the read-out with 128 x 128-byte fp8 q and g tiles: the
//                       transform warps decode q into the fp16 q_til operand,
//                       the epilogue warps decode g from shared memory and
//                       store the bf16 output rows directly.
//   mx_decode_kernel    E4M3 x scale -> bf16, for the CUDA-core cross-check
//                       path (decode, then the bf16 CUDA-core kernels).
#pragma once

#include <cuda_fp8.h>

#include "tc.cuh"

namespace gla {

// 2^(e - 127) of an E8M0 scale byte (e = 0 gives the fp32 subnormal 2^-127;
// e = 255, which the format reserves for NaN, gives infinity).
__device__ __forceinline__ float e8m0_value(uint32_t e) {
  return e ? __uint_as_float(e << 23) : __uint_as_float(0x00400000u);
}

// 16 E4M3 codes (the lane's 16 channels, first code in the lowest byte) times
// one scale, as 8 fp32 pairs (channels 2i, 2i+1).
__device__ __forceinline__ void mx_decode16(uint4 raw, float scl, f2_t (&x)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  const f2_t s2 = f2(scl, scl);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
          (__nv_fp8x2_storage_t)((w[i] >> (16 * hf)) & 0xFFFFu), __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
      x[2 * i + hf] = f2_mul(f2(f.x, f.y), s2);
    }
  }
}

// Address of the lane's 16-byte chunk j in row r of a 128-byte-row tile with
// 128-byte swizzle (one TMA box of 128 bytes x rows).
__device__ __forceinline__ uint32_t mx_chunk(uint32_t tile, int r, int j) {
  return tile + (uint32_t)r * 128u + ((((uint32_t)j) ^ (uint32_t)(r & 7)) << 4);
}

// --------------------------------------------------------------- state kernel

constexpr int kMxStStages = 3;                       // fp8 input ring
constexpr int kMxStOps = 2;                          // bf16 operand slots
constexpr uint32_t kMxStIn = kStTile * 128;          // one fp8 tile: 96 rows x 128 B
constexpr uint32_t kMxStOpBytes = 2 * kStTileBytes;  // K and V bf16 operand tiles

struct TcStateMxSmem {
  static constexpr uint32_t OP = 0;                                   // [2] K op, V op
  static constexpr uint32_t IN = OP + kMxStOps * kMxStOpBytes;        // [3] k8, v8
  static constexpr uint32_t ROWREC = IN + kMxStStages * 2 * kMxStIn;  // [3][96] records
  static constexpr uint32_t BETA = ROWREC + kMxStStages * kStTile * kRecBytes;  // [3][96] f32
  static constexpr uint32_t SCL = BETA + kMxStStages * kStTile * 4;   // [3][2][96] u32
  static constexpr uint32_t BAR = SCL + kMxStStages * 2 * kStTile * 4;
  static constexpr uint32_t NBAR = 2 * kMxStStages + 2 * kMxStOps + 5;
  static constexpr uint32_t MISC = BAR + NBAR * 8;
  static constexpr uint32_t TAB = (MISC + 16 + 15) & ~15u;
};
static_assert(TcStateMxSmem::IN % 1024 == 0, "swizzle atoms");

struct TcStateMxParams {
  Geom g;
  Partition part;
  const __nv_bfloat16* beta;
  const uint32_t* k_scale;   // [B][N][Hh] words of 4 E8M0 bytes
  const uint32_t* v_scale;
  float* part_S;
  float* part_z;
  float2* rope_tab;          // optional: the call's whole RoPE table for the read-out
  int tab_entries;
};

__global__ void __launch_bounds__(kStThreads, 1)
    tc_state_mx_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, TcStateMxParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + TcStateMxSmem::BAR);
  uint64_t* full = bars;                          // [3] fp8 tiles + scales / beta / records
  uint64_t* empty = bars + kMxStStages;           // [3] transform done with the input stage
  uint64_t* oready = bars + 2 * kMxStStages;      // [2] operand slot written
  uint64_t* ofree = oready + kMxStOps;            // [2] MMA done with the operand slot
  uint64_t* accfull = ofree + kMxStOps;
  uint64_t* accempty = accfull + 2;
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + TcStateMxSmem::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + TcStateMxSmem::MISC + 4);
  float2* tab = reinterpret_cast<float2*>(sm + TcStateMxSmem::TAB);

  const Geom& g = p.g;
  const Partition& part = p.part;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long wb = part_begin(part, c), we = part_begin(part, c + 1);
  const RopeWindow win = rope_window(g, part, wb, we - 1);
  const int tph = part.tiles_per_head;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMxStStages; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], kStTW);
    }
    for (int o = 0; o < kMxStOps; ++o) {
      mbar_init(&oready[o], kStTW);
      mbar_init(&ofree[o], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accfull[a], 1);
      mbar_init(&accempty[a], kStTW);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
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
    pdl_wait();
    const uint64_t pol = policy_evict_first();
    const uint64_t pol_small = policy_evict_last();
    long long it = 0;
    int issued = 0;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<kMxStStages> rp;
    for (; iw.more(); iw.next(), rp.next(), ++it) {
      const int s = rp.s;
      if (!mbar_wait_warp(&empty[s], rp.ph ^ 1u, abort_flag)) break;
      const int b = iw.b, h = iw.h, n0 = iw.ti * kStTile;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], 2 * kMxStIn);
        unsigned char* kt = sm + TcStateMxSmem::IN + (2 * s) * kMxStIn;
        tma_load_3d(kt, &tmK, &full[s], h * 128, n0, b, pol);
        tma_load_3d(kt + kMxStIn, &tmV, &full[s], h * 128, n0, b, pol);
      }
      float* bs = reinterpret_cast<float*>(sm + TcStateMxSmem::BETA + s * kStTile * 4);
      uint32_t* ks = reinterpret_cast<uint32_t*>(sm + TcStateMxSmem::SCL + (2 * s) * kStTile * 4);
      uint32_t* vs = ks + kStTile;
#pragma unroll
      for (int k2 = 0; k2 < kStTile / 32; ++k2) {
        const int r = lane + 32 * k2, n = n0 + r;
        const size_t th = ((size_t)b * g.N + n) * g.Hh + h;
        const bool ok = n < g.N;
        bs[r] = ok ? __uint_as_float((uint32_t)ld_u16_policy(p.beta + th, pol_small) << 16) : 0.f;
        ks[r] = ok ? p.k_scale[th] : 0u;
        vs[r] = ok ? p.v_scale[th] : 0u;
      }
      if (g.rope_on)
        tile_rowrec<kStTile>(g, win, n0, lane, sm + TcStateMxSmem::ROWREC + s * kStTile * kRecBytes);
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
      ++issued;
      if (it == 0 && p.rope_tab != nullptr)
        rope_build_global(p.rope_tab, g, blockIdx.x, gridDim.x, lane, 32);
    }
    if (*abort_flag && lane == 0) {
      long long first = it - (issued < kMxStStages ? issued : kMxStStages);
      for (long long i2 = first; i2 < it; ++i2) {
        int dummy = 0;
        mbar_wait(&full[i2 % kMxStStages], (uint32_t)((i2 / kMxStStages) & 1),
                  reinterpret_cast<volatile int*>(&dummy));
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, true, true);
      int seg = 0;
      ItemWalk iw(wb, we, tph, g.Hh);
      RingPos<kMxStOps> ro;
      for (; iw.more(); iw.next(), ro.next()) {
        const int o = ro.s;
        const bool first = iw.first, last = iw.last;
        const int ab = seg & 1;
        if (first && !mbar_wait(&accempty[ab], (uint32_t)(((seg >> 1) & 1) ^ 1), abort_flag))
          break;
        if (!mbar_wait(&oready[o], ro.ph, abort_flag)) break;
        tc_fence_after();
        const uint32_t kt = sbase + TcStateMxSmem::OP + o * kMxStOpBytes;
        const uint32_t vt = kt + kStTileBytes;
#pragma unroll
        for (int kk = 0; kk < kStTile / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(vt + kk * 2048, kStBox, 1024);
          const uint64_t bd = sdesc_sw128(kt + kk * 2048, kStBox, 1024);
          umma_f16kind(tmem + ab * 128, ad, bd, idesc, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&ofree[o]);
        if (last) {
          umma_commit(&accfull[ab]);
          ++seg;
        }
      }
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy));
    }
  } else {
    // ------------------------- transform warps: decode, k -> beta k_til, v
    rope_build(tab, g, win, threadIdx.x - kStTW0 * 32, kStTW * 32);
    named_barrier(1, kStTW * 32);
    const int tw = warp - kStTW0;
    const int rg = tw_row(lane), j = tw_chunk(lane);
    LaneRope lr;
    lane_rope(g, j, smem_u32(tab), lr);
    uint32_t ch0, ch1;     // the lane's chunks of its first row in a bf16 operand tile
    lane_chunks(0, kStBox, tw * 4 + rg, j, ch0, ch1);
    f2_t zacc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) zacc[i] = 0ull;
    int seg = 0;
    bool ok = true;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<kMxStStages> rp;
    RingPos<kMxStOps> ro;
    for (; iw.more() && ok; iw.next(), rp.next(), ro.next()) {
      const int s = rp.s, o = ro.s;
      const int bh = iw.bh;
      if (!mbar_wait_warp(&full[s], rp.ph, abort_flag)) { ok = false; break; }
      if (!mbar_wait_warp(&ofree[o], ro.ph ^ 1u, abort_flag)) { ok = false; break; }
      const uint32_t k8 = sbase + TcStateMxSmem::IN + (2 * s) * kMxStIn;
      const uint32_t v8 = k8 + kMxStIn;
      const uint32_t kop = sbase + TcStateMxSmem::OP + o * kMxStOpBytes;
      const uint32_t vop = kop + kStTileBytes;
      const float* bs = reinterpret_cast<const float*>(sm + TcStateMxSmem::BETA + s * kStTile * 4);
      const uint32_t* ks =
          reinterpret_cast<const uint32_t*>(sm + TcStateMxSmem::SCL + (2 * s) * kStTile * 4);
      const uint32_t* vs = ks + kStTile;
      const uint32_t rec_s = sbase + TcStateMxSmem::ROWREC + s * kStTile * kRecBytes;
#pragma unroll 1
      for (int u = 0; u < kStRows; ++u) {
        const int r = u * kStRowsPerPass + tw * 4 + rg;
        const uint32_t roff = (uint32_t)(u * kStRowsPerPass) * 128u;
        uint32_t t012 = 0, t345 = 0, t67 = 0;
        if (g.rope_on) lane_rope_row(lr, rec_s + r * kRecBytes, t012, t345, t67);
        const uint4 kraw = lds128(mx_chunk(k8, r, j));
        const uint4 vraw = lds128(mx_chunk(v8, r, j));
        f2_t e[8];
        if (g.rope_on) tab_load8(t012, t345, t67, e);
        const float ksc = e8m0_value((ks[r] >> (8 * (j >> 1))) & 0xFFu);
        const float vsc = e8m0_value((vs[r] >> (8 * (j >> 1))) & 0xFFu);
        const float bet = bs[r];
        {
          f2_t x[8];
          mx_decode16(kraw, ksc, x);
          const float rstd = row_rstd(x);
          const f2_t rstd2 = f2(rstd, rstd);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            x[i] = f2_relu(x[i]);
            zacc[i] = f2_fma(x[i], rstd2, zacc[i]);
          }
          uint4 o0, o1;
          rope_scale_pack<false>(g.rope_on, e, x, rstd * bet, o0, o1);
          sts128(kop + ch0 + roff, o0);
          sts128(kop + ch1 + roff, o1);
        }
        {
          f2_t x[8];
          mx_decode16(vraw, vsc, x);
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) w[i] = pack_bf16(f2_lo(x[i]), f2_hi(x[i]));
          sts128(vop + ch0 + roff, make_uint4(w[0], w[1], w[2], w[3]));
          sts128(vop + ch1 + roff, make_uint4(w[4], w[5], w[6], w[7]));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[s]);
        mbar_arrive(&oready[o]);
      }

      if (iw.last) {
        float zf[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          zf[2 * i] = f2_lo(zacc[i]);
          zf[2 * i + 1] = f2_hi(zacc[i]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          zf[i] += __shfl_xor_sync(0xffffffffu, zf[i], 4);
          zf[i] += __shfl_xor_sync(0xffffffffu, zf[i], 16);
        }
        if (rg == 0) {
          float* zd = p.part_z + (((size_t)c + bh) * kStTW + tw) * 128 + 16 * j;
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(zd + i) = make_float4(zf[i], zf[i + 1], zf[i + 2], zf[i + 3]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) zacc[i] = 0ull;
        {
          const int q4 = warp & 3;
          const int third = tw >> 2;
          const int a = q4 * 32 + lane;
          const int ab = seg & 1;
          if (!mbar_wait_warp(&accfull[ab], (uint32_t)((seg >> 1) & 1), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          float* dst = p.part_S + ((size_t)c + bh) * 128 * 128 + (size_t)a * 8;
#pragma unroll 1
          for (int cb = third; cb < 16; cb += 3) {
            float rr[8];
            tmem_ld8(tmem + (uint32_t)(ab * 128 + cb * 8) + ((uint32_t)(q4 * 32) << 16), rr);
            tmem_wait_ld();
            *reinterpret_cast<float4*>(dst + cb * 1024) = make_float4(rr[0], rr[1], rr[2], rr[3]);
            *reinterpret_cast<float4*>(dst + cb * 1024 + 4) = make_float4(rr[4], rr[5], rr[6], rr[7]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&accempty[ab]);
        }
        ++seg;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// --------------------------------------------------------------- read-out

constexpr uint32_t kMxApIn = kTcTile * 128;          // fp8 tile: 128 rows x 128 B
constexpr int kMxApG = 3;                            // fp8 g ring
constexpr int kMxApThreads = kApEW0 * 32 + kApEW * 32;   // no store warp

struct TcApplyMxSmem {
  static constexpr uint32_t QT = 0;                               // [2] fp16 q_til operand
  static constexpr uint32_t SIMG = QT + kApQ * kTileBytes;        // S image
  static constexpr uint32_t Q8 = SIMG + kTileBytes;               // [2] fp8 q tiles
  static constexpr uint32_t G8 = Q8 + kApQ * kMxApIn;             // [3] fp8 g tiles
  static constexpr uint32_t Z = G8 + kMxApG * kMxApIn;            // z [128] f32
  static constexpr uint32_t SCL = Z + 512;                        // image scale [4] f32
  static constexpr uint32_t DEN = SCL + 16;                       // [kApDen][128]
  static constexpr uint32_t QSC = DEN + kApDen * 512;             // [2][128] q scale words
  static constexpr uint32_t GSC = QSC + kApQ * 512;               // [3][128] g scale words
  static constexpr uint32_t ROWREC = GSC + kMxApG * 512;          // [2][128] records
  static constexpr uint32_t BAR = ROWREC + kApQ * kTcTile * kRecBytes;
  static constexpr uint32_t NBAR = 4 * kApQ + 2 * kMxApG + 2 * kApAcc + 5;
  static constexpr uint32_t MISC = BAR + NBAR * 8;
  static constexpr uint32_t TAB = (MISC + 16 + 15) & ~15u;
};
static_assert(TcApplyMxSmem::Q8 % 1024 == 0 && TcApplyMxSmem::G8 % 1024 == 0, "swizzle atoms");

struct TcApplyMxParams {
  Geom g;
  Partition part;
  const __half* S_img;
  const float* S_scale;
  const float* z;
  const float2* rope_tab;
  const uint32_t* q_scale;   // [B][N][Hh] words of 4 E8M0 bytes
  const uint32_t* g_scale;
  __nv_bfloat16* out;        // [B][N][Hh][128]
  float* den_out;            // optional
  float* x_out;              // optional
  int tab_entries;
};

template <bool kDebug>
__global__ void __launch_bounds__(kMxApThreads, 1)
    tc_apply_mx_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmG, TcApplyMxParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + TcApplyMxSmem::BAR);
  uint64_t* qfull = bars;                 // [2] fp8 q tile + its scales / records
  uint64_t* q8free = qfull + kApQ;        // [2] transform done with the fp8 q tile
  uint64_t* qtfree = q8free + kApQ;       // [2] MMA done with the q_til operand
  uint64_t* qready = qtfree + kApQ;       // [2] q_til written
  uint64_t* gfull = qready + kApQ;        // [3]
  uint64_t* gempty = gfull + kMxApG;      // [3]
  uint64_t* accfull = gempty + kMxApG;
  uint64_t* accempty = accfull + kApAcc;
  uint64_t* sfull = accempty + kApAcc;
  uint64_t* sfree = sfull + 1;
  uint64_t* drain = sfree + 1;
  uint64_t* zfull = drain + 1;
  uint64_t* tfull = zfull + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + TcApplyMxSmem::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + TcApplyMxSmem::MISC + 4);
  float* zs = reinterpret_cast<float*>(sm + TcApplyMxSmem::Z);
  const float* scl_s = reinterpret_cast<const float*>(sm + TcApplyMxSmem::SCL);
  float* den_ring = reinterpret_cast<float*>(sm + TcApplyMxSmem::DEN);
  float2* tab = reinterpret_cast<float2*>(sm + TcApplyMxSmem::TAB);

  const Geom& g = p.g;
  const Partition& part = p.part;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long wb = part_begin(part, c), we = part_begin(part, c + 1);
  const RopeWindow win = rope_window(g, part, wb, we - 1);
  const int tph = part.tiles_per_head;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kApQ; ++s) {
      mbar_init(&qfull[s], 2);      // TMA bytes + the producer's scales / records
      mbar_init(&q8free[s], kApTW);
      mbar_init(&qtfree[s], 1);
      mbar_init(&qready[s], kApTW);
    }
    for (int s = 0; s < kMxApG; ++s) {
      mbar_init(&gfull[s], 2);      // TMA bytes + the producer's scales
      mbar_init(&gempty[s], kApEW);
    }
    for (int a = 0; a < kApAcc; ++a) {
      mbar_init(&accfull[a], 1);
      mbar_init(&accempty[a], kApEW);
    }
    mbar_init(sfull, 1);
    mbar_init(sfree, 1);
    mbar_init(drain, 1);
    mbar_init(zfull, 1);
    mbar_init(tfull, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 256);
    tmem_relinquish();
  }
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    // ------------------------------------------- producer: S image, z, q
    const uint64_t pol = policy_evict_first();
    int seg = 0, issued = 0;
    bool combined = false;
    ItemWalk iw(wb, we, tph, g.Hh);
    ItemWalk ahead = iw;
    ahead.next();
    RingPos<kApQ> rq;
    for (; iw.more(); iw.next(), rq.next()) {
      const int bh = iw.bh, b = iw.b, h = iw.h;
      if (ahead.more()) {
        if (lane == 0) tma_prefetch_3d(&tmQ, ahead.h * 128, ahead.ti * kTcTile, ahead.b);
        ahead.next();
      }
      const int s = rq.s;
      if (!mbar_wait_warp(&q8free[s], rq.ph ^ 1u, abort_flag)) break;
      const int n0 = iw.ti * kTcTile;
      // The tile copy first; the scales and row records land while it flies.
      if (lane == 0) {
        mbar_arrive_expect_tx(&qfull[s], kMxApIn);
        tma_load_3d(sm + TcApplyMxSmem::Q8 + s * kMxApIn, &tmQ, &qfull[s], h * 128, n0, b, pol);
      }
      uint32_t* qs = reinterpret_cast<uint32_t*>(sm + TcApplyMxSmem::QSC + s * 512);
#pragma unroll
      for (int k2 = 0; k2 < kTcTile / 32; ++k2) {
        const int r = lane + 32 * k2, n = n0 + r;
        qs[r] = n < g.N ? p.q_scale[((size_t)b * g.N + n) * g.Hh + h] : 0u;
      }
      if (g.rope_on)
        tile_rowrec<kTcTile>(g, win, n0, lane, sm + TcApplyMxSmem::ROWREC + s * kTcTile * kRecBytes);
      __syncwarp();
      if (lane == 0) mbar_arrive(&qfull[s]);
      ++issued;
      if (iw.first) {
        if (!combined) {
          pdl_wait();
          combined = true;
        }
        if (!mbar_wait_warp(sfree, (uint32_t)((seg & 1) ^ 1), abort_flag)) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(zfull, 512 + 16);
          bulk_load(sm + TcApplyMxSmem::Z, p.z + (size_t)bh * 128, 512, zfull);
          bulk_load(sm + TcApplyMxSmem::SCL, p.S_scale + (size_t)bh * 4, 16, zfull);
          if (seg == 0) {
            if (g.rope_on) {
              const RopeCopy rc = rope_copy_plan(g, win);
              uint32_t bytes = 0;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (i < rc.n) bytes += (uint32_t)rc.len[i] * 8u;
              mbar_arrive_expect_tx(tfull, bytes);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (i < rc.n)
                  bulk_load(tab + rc.dst[i], p.rope_tab + rc.src[i], (uint32_t)rc.len[i] * 8u, tfull);
            } else {
              mbar_arrive(tfull);
            }
          }
          mbar_arrive_expect_tx(sfull, kTileBytes);
          bulk_load(sm + TcApplyMxSmem::SIMG, p.S_img + (size_t)bh * 128 * 128, kTileBytes, sfull);
        }
        ++seg;
      }
    }
    if (*abort_flag && lane == 0) {
      for (int i2 = issued - (issued < kApQ ? issued : kApQ); i2 < issued; ++i2) {
        int dummy = 0;
        mbar_wait(&qfull[i2 % kApQ], (uint32_t)((i2 / kApQ) & 1),
                  reinterpret_cast<volatile int*>(&dummy));
      }
      int dummy = 0;
      if (seg > 0) {
        volatile int* nd = reinterpret_cast<volatile int*>(&dummy);
        mbar_wait(sfull, (uint32_t)((seg - 1) & 1), nd);
        mbar_wait(zfull, (uint32_t)((seg - 1) & 1), nd);
        mbar_wait(tfull, 0u, nd);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------ producer: g
    const uint64_t pol = policy_evict_first();
    long long it = 0;
    int issued = 0;
    ItemWalk iw(wb, we, tph, g.Hh);
    ItemWalk ahead = iw;
    for (int k = 0; k < kApPrefetch && ahead.more(); ++k) ahead.next();
    RingPos<kMxApG> rg_;
    const bool go = !iw.more() || mbar_wait_warp(tfull, 0u, abort_flag);
    for (; go && iw.more(); iw.next(), rg_.next(), ++it) {
      const int b = iw.b, h = iw.h;
      const int s = rg_.s;
      if (ahead.more()) {
        if (lane == 0) tma_prefetch_3d(&tmG, ahead.h * 128, ahead.ti * kTcTile, ahead.b);
        ahead.next();
      }
      if (!mbar_wait_warp(&gempty[s], rg_.ph ^ 1u, abort_flag)) break;
      const int n0 = iw.ti * kTcTile;
      if (lane == 0) {
        mbar_arrive_expect_tx(&gfull[s], kMxApIn);
        tma_load_3d(sm + TcApplyMxSmem::G8 + s * kMxApIn, &tmG, &gfull[s], h * 128, n0, b, pol);
      }
      uint32_t* gs = reinterpret_cast<uint32_t*>(sm + TcApplyMxSmem::GSC + s * 512);
#pragma unroll
      for (int k2 = 0; k2 < kTcTile / 32; ++k2) {
        const int r = lane + 32 * k2, n = n0 + r;
        gs[r] = n < g.N ? p.g_scale[((size_t)b * g.N + n) * g.Hh + h] : 0u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&gfull[s]);
      ++issued;
    }
    if (*abort_flag && lane == 0) {
      long long first = it - (issued < kMxApG ? issued : kMxApG);
      for (long long i2 = first; i2 < it; ++i2) {
        int dummy = 0;
        mbar_wait(&gfull[i2 % kMxApG], (uint32_t)((i2 / kMxApG) & 1),
                  reinterpret_cast<volatile int*>(&dummy));
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, 128, false, false);
      int seg = 0;
      const uint32_t simg = sbase + TcApplyMxSmem::SIMG;
      ItemWalk iw(wb, we, tph, g.Hh);
      RingPos<kApAcc> ra;
      RingPos<kApQ> rq;
      for (; iw.more(); iw.next(), ra.next(), rq.next()) {
        const bool first = iw.first, last = iw.last;
        if (first && !mbar_wait(sfull, (uint32_t)(seg & 1), abort_flag)) break;
        const int ab = ra.s;
        if (!mbar_wait(&accempty[ab], ra.ph ^ 1u, abort_flag)) break;
        const int s = rq.s;
        if (!mbar_wait(&qready[s], rq.ph, abort_flag)) break;
        tc_fence_after();
        const uint32_t qt = sbase + TcApplyMxSmem::QT + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32;
          umma_f16kind(tmem + ab * 128, sdesc_sw128(qt + koff, 16, 1024),
                       sdesc_sw128(simg + koff, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&qtfree[s]);
        umma_commit(&accfull[ab]);
        if (last) {
          umma_commit(sfree);
          ++seg;
        }
      }
      umma_commit(drain);
      int dummy = 0;
      mbar_wait(drain, 0, reinterpret_cast<volatile int*>(&dummy));
    }
  } else if (warp < kApEW0) {
    // ------------------------------ transform warps: decode q -> q_til, den
    const bool tab_ok = wb >= we || mbar_wait_warp(tfull, 0u, abort_flag);
    const int tw = warp - kApTW0;
    const int rg = tw_row(lane), j = tw_chunk(lane);
    LaneRope lr;
    lane_rope(g, j, smem_u32(tab), lr);
    uint32_t ch0, ch1;
    lane_chunks(0, kBox, tw * 4 + rg, j, ch0, ch1);
    f2_t zr[8];
    float hscale = 1.f;
    int seg = 0;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<kApQ> rq;
    RingPos<kApDen> rd;
    for (; tab_ok && iw.more(); iw.next(), rq.next(), rd.next()) {
      const int b = iw.b, h = iw.h;
      if (iw.first) {
        if (!mbar_wait_warp(zfull, (uint32_t)(seg & 1), abort_flag)) break;
#pragma unroll
        for (int i = 0; i < 8; ++i) zr[i] = f2(zs[16 * j + 2 * i], zs[16 * j + 2 * i + 1]);
        hscale = scl_s[0];
        ++seg;
      }
      const int s = rq.s;
      if (!mbar_wait_warp(&qfull[s], rq.ph, abort_flag)) break;
      if (!mbar_wait_warp(&qtfree[s], rq.ph ^ 1u, abort_flag)) break;
      const int n0 = iw.ti * kTcTile;
      const uint32_t q8 = sbase + TcApplyMxSmem::Q8 + s * kMxApIn;
      const uint32_t qt = sbase + TcApplyMxSmem::QT + s * kTileBytes;
      const uint32_t* qs = reinterpret_cast<const uint32_t*>(sm + TcApplyMxSmem::QSC + s * 512);
      float* den = den_ring + rd.s * 128;
      const uint32_t rec_s = sbase + TcApplyMxSmem::ROWREC + s * kTcTile * kRecBytes;
#pragma unroll 1
      for (int ps = 0; ps < kApPasses; ++ps) {
        uint32_t t012[kApIL], t345[kApIL], t67[kApIL];
        uint4 raw[kApIL];
        float qsc[kApIL];
        f2_t e[kApIL][8];
        int rr[kApIL];
#pragma unroll
        for (int u = 0; u < kApIL; ++u) {
          rr[u] = ps * kApRowsPerPass + u * kApTW * 4 + tw * 4 + rg;
          if (g.rope_on) lane_rope_row(lr, rec_s + rr[u] * kRecBytes, t012[u], t345[u], t67[u]);
          raw[u] = lds128(mx_chunk(q8, rr[u], j));
          qsc[u] = e8m0_value((qs[rr[u]] >> (8 * (j >> 1))) & 0xFFu);
        }
        if (g.rope_on) {
#pragma unroll
          for (int u = 0; u < kApIL; ++u) tab_load8(t012[u], t345[u], t67[u], e[u]);
        }
        float dn[kApIL];
#pragma unroll
        for (int u = 0; u < kApIL; ++u) {
          f2_t x[8];
          mx_decode16(raw[u], qsc[u], x);
          const float rstd = row_rstd(x);
          f2_t dp2 = 0ull;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            x[i] = f2_relu(x[i]);
            dp2 = f2_fma(zr[i], x[i], dp2);
          }
          uint4 o0, o1;
          rope_scale_pack<true>(g.rope_on, e[u], x, rstd, o0, o1);
          const uint32_t roff = (uint32_t)(ps * kApRowsPerPass + u * kApTW * 4) * 128u;
          sts128(qt + ch0 + roff, o0);
          sts128(qt + ch1 + roff, o1);
          const float dp = row_sum(f2_lo(dp2) + f2_hi(dp2));
          dn[u] = fmaf(dp, rstd, g.eps);
        }
        if (j == 0) {
#pragma unroll
          for (int u = 0; u < kApIL; ++u) {
            den[rr[u]] = dn[u] * hscale;
            const int n = n0 + rr[u];
            if (kDebug && p.den_out && n < g.N) p.den_out[((size_t)b * g.N + n) * g.Hh + h] = dn[u];
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&q8free[s]);
        mbar_arrive(&qready[s]);
      }
    }
  } else {
    // ------------------------- epilogue warps: gate, denominator, RMSNorm
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<kApAcc> ra;
    RingPos<kMxApG> rg_;
    RingPos<kApDen> rd;
    for (; iw.more(); iw.next(), ra.next(), rg_.next(), rd.next()) {
      const int b = iw.b, h = iw.h;
      const int n0 = iw.ti * kTcTile;
      const int ab = ra.s;
      if (!mbar_wait_warp(&accfull[ab], ra.ph, abort_flag)) break;
      tc_fence_after();
      const int gsl = rg_.s;
      if (!mbar_wait_warp(&gfull[gsl], rg_.ph, abort_flag)) break;
      const float hc = 0.5f / den_ring[rd.s * 128 + row];
      const uint32_t taddr = tmem + (uint32_t)(ab * 128) + ((uint32_t)(q4 * 32) << 16);
      const uint32_t g8 = sbase + TcApplyMxSmem::G8 + gsl * kMxApIn;
      const uint32_t gsw = reinterpret_cast<const uint32_t*>(sm + TcApplyMxSmem::GSC + gsl * 512)[row];
      const f2_t hc2 = f2(hc, hc), half2 = f2(0.5f, 0.5f);
      const int n = n0 + row;
      const bool valid = n < g.N;
      f2_t ss2 = 0ull;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float u[32];
        tmem_ld32(taddr + cb * 32, u);
        // channels 32 cb .. 32 cb + 31: chunks 2 cb, 2 cb + 1 of the row, one scale
        const float gsc = e8m0_value((gsw >> (8 * cb)) & 0xFFu);
        f2_t gx[16];
        {
          f2_t t0[8], t1[8];
          mx_decode16(lds128(mx_chunk(g8, row, 2 * cb)), gsc, t0);
          mx_decode16(lds128(mx_chunk(g8, row, 2 * cb + 1)), gsc, t1);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            gx[i] = t0[i];
            gx[8 + i] = t1[i];
          }
        }
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const f2_t hg = f2_mul(gx[e], half2);
          const f2_t t = f2(tanh_approx(f2_lo(hg)), tanh_approx(f2_hi(hg)));
          const f2_t sg = f2_fma(hc2, t, hc2);
          const f2_t x = f2_mul(sg, f2(u[2 * e], u[2 * e + 1]));
          ss2 = f2_fma(x, x, ss2);
          u[2 * e] = f2_lo(x);
          u[2 * e + 1] = f2_hi(x);
        }
        if (kDebug && p.x_out && valid) {
          float* xo = p.x_out + (((size_t)b * g.N + n) * g.Hh + h) * 128 + cb * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(xo + i) = make_float4(u[i], u[i + 1], u[i + 2], u[i + 3]);
        }
        tmem_st32(taddr + cb * 32, u);
      }
      tmem_wait_st();
      const float rstd = rsqrtf((f2_lo(ss2) + f2_hi(ss2)) * (1.f / 128.f) + kRmsEps);
      const f2_t rstd2 = f2(rstd, rstd);
      __nv_bfloat16* orow = p.out + (((size_t)b * g.N + (valid ? n : 0)) * g.Hh + h) * 128;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float x[32];
        tmem_ld32(taddr + cb * 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const f2_t y = f2_mul(f2(x[q * 8 + 2 * e], x[q * 8 + 2 * e + 1]), rstd2);
            o[e] = pack_bf16(f2_lo(y), f2_hi(y));
          }
          if (valid) {
            uint4 v4 = make_uint4(o[0], o[1], o[2], o[3]);
            asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(orow + cb * 32 + 8 * q),
                         "r"(v4.x), "r"(v4.y), "r"(v4.z), "r"(v4.w)
                         : "memory");
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&accempty[ab]);
        mbar_arrive(&gempty[gsl]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------- CUDA-core helper

// out[i] = bf16(e4m3(codes[i]) * 2^(scales[i / 32] - 127)) for n elements.
__global__ void mx_decode_kernel(const uint8_t* __restrict__ codes,
                                 const uint8_t* __restrict__ scales,
                                 __nv_bfloat16* __restrict__ out, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)codes[i], __NV_E4M3);
    const float v = __half2float(*reinterpret_cast<const __half*>(&hr)) * e8m0_value(scales[i >> 5]);
    out[i] = __float2bfloat16_rn(v);
  }
}

// ------------------------------------------------------------------ host

// [B][N][Hh][128] bytes as a 3D map (byte, token, batch) with boxes of 128
// bytes x `rows` tokens, 128-byte swizzle, zero fill past N.
inline bool make_mx_map(CUtensorMap* m, const void* ptr, const Geom& g, uint32_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)g.Hh * 128, (cuuint64_t)g.N, (cuuint64_t)g.B};
  cuuint64_t strides[2] = {(cuuint64_t)g.Hh * 128, (cuuint64_t)g.N * g.Hh * 128};
  cuuint32_t box[3] = {128, rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline size_t tc_state_mx_smem(int tab_entries) {
  return 1024 + TcStateMxSmem::TAB + (size_t)tab_entries * 8;
}
inline size_t tc_apply_mx_smem(int tab_entries) {
  return 1024 + TcApplyMxSmem::TAB + (size_t)tab_entries * 8;
}

struct MxInputs {
  const void *q, *q_scale, *k, *k_scale, *v, *v_scale, *g, *g_scale;
};

// The tensor path on MX inputs: state reduction, combine, read-out, each a
// programmatic dependent of the kernel before it.
inline gla_status run_tensor_mx(const Geom& g, const MxInputs& in, const void* beta, void* out,
                                float* S, float* z, bool write_state, float* part_S,
                                float* part_z, __half* S_img, float* S_scale, float2* rope_tab,
                                float* den_dbg, float* x_dbg, int sms, cudaStream_t stream,
                                void* const* events) {
  auto mark = [&](int i) {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream);
  };
  if (sms <= 0) return GLA_ERR_CUDA;
  if (g.H >= (1 << kPosBits) || g.W >= (1 << kPosBits) || g.T >= (1 << kPosBits))
    return GLA_ERR_UNSUPPORTED;
  if (!tc_rope_lanes_ok(g)) return GLA_ERR_UNSUPPORTED;
  const Partition spart = tc_state_partition(g, sms);
  const Partition part = tc_apply_partition(g, sms);
  const int stab = tc_table_entries(g, spart), tab = tc_table_entries(g, part);
  const size_t smem_st = tc_state_mx_smem(stab), smem_ap = tc_apply_mx_smem(tab);
  if (smem_st > kMaxSmem || smem_ap > kMaxSmem) return GLA_ERR_UNSUPPORTED;

  CUtensorMap mK, mV, mQ, mG;
  if (!make_mx_map(&mK, in.k, g, kStTile) || !make_mx_map(&mV, in.v, g, kStTile) ||
      !make_mx_map(&mQ, in.q, g, kTcTile) || !make_mx_map(&mG, in.g, g, kTcTile))
    return GLA_ERR_CUDA;

  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;

  TcStateMxParams sp = {};
  sp.g = g; sp.part = spart;
  sp.beta = static_cast<const __nv_bfloat16*>(beta);
  sp.k_scale = static_cast<const uint32_t*>(in.k_scale);
  sp.v_scale = static_cast<const uint32_t*>(in.v_scale);
  sp.part_S = part_S; sp.part_z = part_z; sp.tab_entries = stab;
  sp.rope_tab = g.rope_on ? rope_tab : nullptr;
  if (!ensure_max_smem(tc_state_mx_kernel, 0)) return GLA_ERR_CUDA;
  if (mark(0) != cudaSuccess) return GLA_ERR_CUDA;
  cudaLaunchConfig_t sc = {};
  sc.gridDim = dim3(spart.grid);
  sc.blockDim = dim3(kStThreads);
  sc.dynamicSmemBytes = smem_st;
  sc.stream = stream;
  sc.attrs = pdl;
  sc.numAttrs = 1;
  if (cudaLaunchKernelEx(&sc, tc_state_mx_kernel, mK, mV, sp) != cudaSuccess || mark(1) != cudaSuccess)
    return GLA_ERR_CUDA;

  CombineParams cp = {};
  cp.part = spart; cp.d = 128; cp.zparts = kStTW;
  cp.part_S = part_S; cp.part_z = part_z;
  cp.S_in = nullptr; cp.z_in = nullptr;
  cp.S_out = write_state ? S : nullptr;
  cp.z_out = z; cp.S_img = S_img; cp.S_scale = S_scale;
  cp.chunked = 1;
  int max_slots = 0;
  for (int bh = 0; bh < g.B * g.Hh; ++bh) {
    const int lo = part_cta_of(spart, (long long)bh * spart.tiles_per_head);
    const int hi = part_cta_of(spart, (long long)(bh + 1) * spart.tiles_per_head - 1);
    if (hi - lo + 1 > max_slots) max_slots = hi - lo + 1;
  }
  const bool bulk = max_slots <= kCombineBulkSlots;
  cudaLaunchConfig_t cc = {};
  cc.gridDim = dim3(kCombineCluster, g.B * g.Hh);
  cc.blockDim = dim3(kCombineThreads);
  cc.dynamicSmemBytes = bulk ? combine_bulk_smem(max_slots) : 0;
  cc.stream = stream;
  cc.attrs = pdl;
  cc.numAttrs = 1;
  cudaError_t ce;
  if (bulk) {
    if (!ensure_max_smem(combine_bulk_kernel, 3)) return GLA_ERR_CUDA;
    ce = cudaLaunchKernelEx(&cc, combine_bulk_kernel, cp);
  } else {
    ce = cudaLaunchKernelEx(&cc, combine_kernel, cp);
  }
  if (ce != cudaSuccess || mark(2) != cudaSuccess) return GLA_ERR_CUDA;

  TcApplyMxParams ap = {};
  ap.g = g; ap.part = part; ap.S_img = S_img; ap.S_scale = S_scale; ap.z = z;
  ap.rope_tab = rope_tab;
  ap.q_scale = static_cast<const uint32_t*>(in.q_scale);
  ap.g_scale = static_cast<const uint32_t*>(in.g_scale);
  ap.out = static_cast<__nv_bfloat16*>(out);
  ap.den_out = den_dbg; ap.x_out = x_dbg; ap.tab_entries = tab;
  const bool dbg = den_dbg != nullptr || x_dbg != nullptr;
  cudaLaunchConfig_t ac = {};
  ac.gridDim = dim3(part.grid);
  ac.blockDim = dim3(kMxApThreads);
  ac.dynamicSmemBytes = smem_ap;
  ac.stream = stream;
  ac.attrs = pdl;
  ac.numAttrs = 1;
  cudaError_t e;
  if (dbg) {
    if (!ensure_max_smem(tc_apply_mx_kernel<true>, 1)) return GLA_ERR_CUDA;
    e = cudaLaunchKernelEx(&ac, tc_apply_mx_kernel<true>, mQ, mG, ap);
  } else {
    if (!ensure_max_smem(tc_apply_mx_kernel<false>, 2)) return GLA_ERR_CUDA;
    e = cudaLaunchKernelEx(&ac, tc_apply_mx_kernel<false>, mQ, mG, ap);
  }
  if (e != cudaSuccess || mark(3) != cudaSuccess) return GLA_ERR_CUDA;
  return GLA_OK;
}

}  // namespace gla
