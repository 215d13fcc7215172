// Tensor-core path (bf16 inputs, head dim 128) for sm_100a.
//
//   tc_state_kernel  persistent split-N state reduction.  TMA streams 96-token
//                    tiles of k and v (128-byte swizzle) into a 4-stage ring;
//                    transform warps apply RMSNorm, ReLU, 3D RoPE and beta to
//                    the k tile in place (bf16) while summing z in registers;
//                    one thread issues tcgen05.mma  S += V^T (beta K_til)  with
//                    both operands MN-major, accumulating in TMEM; the
//                    transform warps drain each finished head segment to its
//                    partial slot.  The producer warps also write the call's
//                    whole RoPE table for the read-out.
//   combine_kernel   (combine.cuh) fixed-order sum of the partials, plus the
//                    swizzled fp16 image of S.
//   tc_apply_kernel  persistent read-out.  TMA streams q and g tiles, bulk
//                    copies bring S, z and its RoPE window; transform
//                    warps turn q into q_til (fp16, in place) and the
//                    denominator z.q_pls + eps; one thread issues
//                    tcgen05.mma  U = Q_til S^T  into a double-buffered TMEM
//                    accumulator; epilogue warps (one token row per thread)
//                    apply sigmoid(g) / den and the output RMSNorm, round to
//                    bf16 into the g tile, and a store warp TMA-stores it.
//
// All waits are bounded (mbar_wait): on expiry the kernel records a timeout in
// the device error word, stops issuing work, drains its copies and frees TMEM.
#pragma once

#include <atomic>

#include "combine.cuh"
#include "ptx.cuh"

namespace gla {

constexpr int kTcTile = 128;                 // tokens per read-out tile (MMA M)
constexpr uint32_t kBox = 16384;             // one TMA box: 128 rows x 128 bytes
constexpr uint32_t kTileBytes = 2 * kBox;    // 128 tokens x 128 channels, 16-bit
constexpr int kStTile = 96;                  // tokens per state tile (MMA K)
constexpr uint32_t kStBox = kStTile * 128;   // 96 rows x 128 bytes
constexpr uint32_t kStTileBytes = 2 * kStBox;
constexpr int kPosBits = 11;                 // (t, h, w) positions, < 2048 each
constexpr int kRecBytes = 20;                // per-row RoPE record (tile_rowrec)

// --------------------------------------------------------------- state kernel

constexpr int kStStages = 4;
constexpr int kStTW = 12;                    // transform warps; they also drain
                                             // finished S partials, three per
                                             // TMEM lane quarter
constexpr int kStTW0 = 2;                    // first transform warp
constexpr int kStThreads = (kStTW0 + kStTW) * 32;
static_assert(kStTW <= kMaxZPartsCombined, "combine adds at most this many z partials");
static_assert(kStTW == 12, "the S drain splits each lane quarter over three warps");
static_assert((kStTW * 4) % 8 == 0, "rows per pass keep the 8-row swizzle phase");
static_assert(kStTile % (kStTW * 4) == 0, "whole row groups per state tile");
static_assert(kStTile % 16 == 0 && kStBox % 1024 == 0, "MMA K steps and swizzle atoms");
constexpr int kStRowsPerPass = kStTW * 4;
constexpr int kStRows = kStTile / kStRowsPerPass;   // row groups per transform warp

struct TcStateSmem {
  static constexpr uint32_t K = 0;
  static constexpr uint32_t V = kStStages * kStTileBytes;
  static constexpr uint32_t ROWREC = 2 * kStStages * kStTileBytes;   // [stage][96] records
  static constexpr uint32_t BETA = ROWREC + kStStages * kStTile * kRecBytes;  // [stage][96] f32
  static constexpr uint32_t BAR = BETA + kStStages * kStTile * 4;     // barriers
  static constexpr uint32_t NBAR = 3 * kStStages + 5;
  static constexpr uint32_t MISC = BAR + NBAR * 8;                     // tmem base, abort
  static constexpr uint32_t TAB = (MISC + 16 + 15) & ~15u;              // RoPE table
};

struct TcStateParams {
  Geom g;
  Partition part;
  const __nv_bfloat16* beta;
  float* part_S;
  float* part_z;
  float2* rope_tab;   // optional: the call's whole RoPE table for the read-out
  int tab_entries;
  unsigned long long wait_ns;   // limit of every wait (kWaitLimitNs)
  long long stall_item;         // self-test only: CTA 0 withholds this item's
                                // arrival (-1: never)
};

// A CTA's items in order, advanced without divisions: head bh (batch b and
// head h), tile ti inside the head, and whether the item opens (first) or
// closes (last) one of the CTA's head segments.
struct ItemWalk {
  int tph, Hh, bh, b, h, ti, left;
  bool first, last;
  __device__ __forceinline__ ItemWalk(long long wb, long long we, int tph_, int Hh_)
      : tph(tph_), Hh(Hh_) {
    bh = (int)(wb / tph);
    ti = (int)(wb - (long long)bh * tph);
    b = bh / Hh;
    h = bh - b * Hh;
    left = (int)(we - wb);
    first = true;
    last = ti == tph - 1 || left == 1;
  }
  __device__ __forceinline__ bool more() const { return left > 0; }
  __device__ __forceinline__ void next() {
    --left;
    first = false;
    if (++ti == tph) {
      ti = 0;
      ++bh;
      if (++h == Hh) { h = 0; ++b; }
      first = true;
    }
    last = ti == tph - 1 || left == 1;
  }
};

// Slot and phase parity of a ring of N buffers.
template <int N>
struct RingPos {
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void next() {
    if (++s == N) { s = 0; ph ^= 1u; }
  }
};

// Per-tile row records.  For every row r of a tile (token n0 + r) the producer
// warp stores the byte offsets, inside the RoPE table, of the token's time (T),
// height (H) and width (W) rows as ten 16-bit words
//   T T T H H H H W W W
// so that for axes a <= b with b - a <= 1 (0 = T, 1 = H, 2 = W) the pair of
// offsets (a, b) is the 32-bit word a + b of the record: TT, TH, HH, HW, WW.
// The table is at most 22.5 KB, so 16 bits hold each offset.

template <int kRows>
__device__ __forceinline__ void tile_rowrec(const Geom& g, RopeWindow win, int n0, int lane,
                                            unsigned char* rec) {
  const uint32_t HW = g.div_HW.d, W = g.div_W.d;
  const RopeLayout L = rope_layout(g, win.Lt);
#pragma unroll
  for (int k = 0; k < kRows / 32; ++k) {
    const int r = lane + 32 * k;
    int n = n0 + r;
    if (n >= g.N) n = n0;
    const uint32_t f = fdiv((uint32_t)n, g.div_HW);
    const uint32_t rem = (uint32_t)n - f * HW;
    const uint32_t hh = fdiv(rem, g.div_W);
    const uint32_t ww = rem - hh * W;
    int tl = (int)f - win.t_lo;
    if (tl < 0) tl += g.T;
    const uint32_t offT = 8u * (uint32_t)(L.base[0] + tl * L.stride[0]);
    const uint32_t offH = 8u * (uint32_t)(L.base[1] + (int)hh * L.stride[1]);
    const uint32_t offW = 8u * (uint32_t)(L.base[2] + (int)ww * L.stride[2]);
    uint32_t* q = reinterpret_cast<uint32_t*>(rec + r * kRecBytes);
    q[0] = offT | (offT << 16);
    q[1] = offT | (offH << 16);
    q[2] = offH | (offH << 16);
    q[3] = offH | (offW << 16);
    q[4] = offW | (offW << 16);
  }
}

// Per-lane view of the RoPE table.  Lane j of a row group handles channels
// 16j .. 16j+15, i.e. rotation pairs 8j .. 8j+7 (slots 0..7); for d = 128 the
// axes hold 22, 21 and 21 pairs, so a lane's slots lie on at most two axes A
// and B, with slots 0..2 on A, slots 6..7 on B and slots 3..5 all on one of
// them (tc_rope_lanes_ok checks this on the host).  In the table, pair 8j + i
// of axis X sits at column idx = 8j + i - start + j - (start >> 3) of its row,
// so slot i of the lane is at byte offX(row) + inX + 8 i.
struct LaneRope {
  uint32_t cA, cB;       // table base + byte offset of pair 8j inside its A / B row
  int rec;               // byte offset of the lane's (A, B) word in a row record
  bool midB;             // slots 3..5 lie on axis B
};

__host__ __device__ inline int axis_of(const Geom& g, int p) {
  return p < g.pt ? 0 : (p < g.pt + g.ph ? 1 : 2);
}

// First slot of lane j on its second axis (8: the lane stays on one axis).
__host__ __device__ inline int lane_split(const Geom& g, int j) {
  const int aA = axis_of(g, 8 * j);
  for (int i = 1; i < 8; ++i)
    if (axis_of(g, 8 * j + i) != aA) return i;
  return 8;
}

// The slot grouping above holds for every lane (d = 128 only).
inline bool tc_rope_lanes_ok(const Geom& g) {
  if (g.d != 128) return false;
  for (int j = 0; j < 8; ++j) {
    const int kb = lane_split(g, j);
    if (kb != 3 && kb != 6 && kb != 8) return false;
    if (axis_of(g, 8 * j + 7) - axis_of(g, 8 * j) > 1) return false;
  }
  return true;
}

__device__ __forceinline__ void lane_rope(const Geom& g, int j, uint32_t tab_s, LaneRope& lr) {
  const int p0 = 8 * j;
  const int start[3] = {0, g.pt, g.pt + g.ph};
  const int aA = axis_of(g, p0), aB = axis_of(g, p0 + 7);
  lr.cA = tab_s + (uint32_t)(8 * (p0 - start[aA] + j - (start[aA] >> 3)));
  lr.cB = tab_s + (uint32_t)(8 * (p0 - start[aB] + j - (start[aB] >> 3)));
  lr.rec = 4 * (aA + aB);
  lr.midB = lane_split(g, j) == 3;
}

// Shared-memory addresses of the lane's slots 0..2, 3..5 and 6..7 runs for the
// row whose record starts at rec_row.
__device__ __forceinline__ void lane_rope_row(const LaneRope& lr, uint32_t rec_row,
                                              uint32_t& a012, uint32_t& a345, uint32_t& a67) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(rec_row + (uint32_t)lr.rec));
  const uint32_t aA = (v & 0xFFFFu) + lr.cA;
  const uint32_t aB = (v >> 16) + lr.cB;
  a012 = aA;
  a67 = aB;
  a345 = lr.midB ? aB : aA;
}

// Shared-memory addresses of the two 16-byte chunks a lane owns in row r of a
// 128x128 16-bit tile stored as two 128-byte-swizzled boxes.
__device__ __forceinline__ void lane_chunks(uint32_t tile, uint32_t box, int r, int j,
                                            uint32_t& a0, uint32_t& a1) {
  const uint32_t row = tile + (uint32_t)(j >> 2) * box + (uint32_t)r * 128u;
  const uint32_t c0 = (uint32_t)((2 * j) & 7);
  a0 = row + (((c0) ^ (uint32_t)(r & 7)) << 4);
  a1 = row + (((c0 + 1) ^ (uint32_t)(r & 7)) << 4);
}

// The lane's 16 elements of a row as 8 fp32 pairs (channels 2i, 2i+1).
__device__ __forceinline__ void unpack8(uint4 a, uint4 b, f2_t (&x)[8]) {
  x[0] = f2_bf(a.x); x[1] = f2_bf(a.y); x[2] = f2_bf(a.z); x[3] = f2_bf(a.w);
  x[4] = f2_bf(b.x); x[5] = f2_bf(b.y); x[6] = f2_bf(b.z); x[7] = f2_bf(b.w);
}

// Lane layout of the transform warps: a warp holds 4 rows x 8 lanes.  Lane
// bits 0-1 pick the chunk pair inside a 64-channel box, bit 3 the box (so
// j = chunk-pair index 0..7), bits 2 and 4 the row.  Each group of 8
// consecutive lanes -- the unit in which the hardware serves 16-byte shared
// accesses -- then touches 8 different 16-byte bank groups of the swizzled
// tile, and the 8 lanes of a row are closed under xor 1, 2, 8.
__device__ __forceinline__ int tw_row(int lane) { return ((lane >> 2) & 1) | (((lane >> 4) & 1) << 1); }
__device__ __forceinline__ int tw_chunk(int lane) { return (lane & 3) | (((lane >> 3) & 1) << 2); }

__device__ __forceinline__ float row_sum(float s) {
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  s += __shfl_xor_sync(0xffffffffu, s, 8);
  return s;
}

// 1/RMS of a row whose 128 elements are spread over the 8 lanes of a group.
__device__ __forceinline__ float row_rstd(const f2_t (&x)[8]) {
  f2_t ss = 0ull;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = f2_fma(x[i], x[i], ss);
  return rsqrtf(row_sum(f2_lo(ss) + f2_hi(ss)) * (1.f / 128.f) + kRmsEps);
}

__device__ __forceinline__ f2_t f2_relu(f2_t x) {
  return f2(fmaxf(f2_lo(x), 0.f), fmaxf(f2_hi(x), 0.f));
}

// (cos, sin) of pair I of the lane: one shared load at an immediate offset.
#define GLA_TAB_LOAD(I, base, out)                                              \
  asm volatile("ld.shared.b64 %0, [%1+%2];" : "=l"(out) : "r"(base), "n"(8 * (I)))

// The lane's 8 (cos, sin) entries of one row (see LaneRope).
__device__ __forceinline__ void tab_load8(uint32_t a012, uint32_t a345, uint32_t a67,
                                          f2_t (&e)[8]) {
  GLA_TAB_LOAD(0, a012, e[0]);
  GLA_TAB_LOAD(1, a012, e[1]);
  GLA_TAB_LOAD(2, a012, e[2]);
  GLA_TAB_LOAD(3, a345, e[3]);
  GLA_TAB_LOAD(4, a345, e[4]);
  GLA_TAB_LOAD(5, a345, e[5]);
  GLA_TAB_LOAD(6, a67, e[6]);
  GLA_TAB_LOAD(7, a67, e[7]);
}

// Rotate the lane's 8 ReLU'd pairs r (still unnormalised) by the entries e,
// scaled by `scl`: y = scl * RoPE(r), packed to bf16 (kHalf = false) or fp16.
// Without RoPE the entries are ignored.
template <bool kHalf>
__device__ __forceinline__ void rope_scale_pack(bool rope_on, const f2_t (&e)[8],
                                                const f2_t (&r)[8], float scl, uint4& o0,
                                                uint4& o1) {
  uint32_t w[8];
  const f2_t scl2 = f2(scl, scl);
  if (rope_on) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float r0 = f2_lo(r[i]), r1 = f2_hi(r[i]);
      const f2_t cs = f2_mul(e[i], scl2);
      const float c = f2_lo(cs), sn = f2_hi(cs);
      const float y0 = fmaf(-r1, sn, r0 * c);
      const float y1 = fmaf(r1, c, r0 * sn);
      w[i] = kHalf ? pack_f16(y0, y1) : pack_bf16(y0, y1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const f2_t y = f2_mul(r[i], scl2);
      w[i] = kHalf ? pack_f16(f2_lo(y), f2_hi(y)) : pack_bf16(f2_lo(y), f2_hi(y));
    }
  }
  o0 = make_uint4(w[0], w[1], w[2], w[3]);
  o1 = make_uint4(w[4], w[5], w[6], w[7]);
}

__global__ void __launch_bounds__(kStThreads, 1)
    tc_state_kernel(const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, TcStateParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + TcStateSmem::BAR);
  uint64_t* full = bars;
  uint64_t* kready = bars + kStStages;
  uint64_t* empty = bars + 2 * kStStages;
  uint64_t* accfull = bars + 3 * kStStages;
  uint64_t* accempty = accfull + 2;
  uint64_t* drain = accempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + TcStateSmem::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + TcStateSmem::MISC + 4);
  float2* tab = reinterpret_cast<float2*>(sm + TcStateSmem::TAB);

  const Geom& g = p.g;
  const Partition& part = p.part;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long wb = part_begin(part, c), we = part_begin(part, c + 1);
  const RopeWindow win = rope_window(g, part, wb, we - 1);
  const int tph = part.tiles_per_head;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStStages; ++s) {
      mbar_init(&full[s], 2);     // TMA bytes + the producer's beta / metadata arrival
      mbar_init(&kready[s], kStTW);
      mbar_init(&empty[s], 1);
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
    // All lanes fetch beta and compute the tile's row metadata; lane 0 issues
    // the copies.
    {
      // Launched as a programmatic dependent of whatever precedes it on the
      // stream: the prologue above overlapped that kernel's tail, but the
      // inputs may be its outputs, so wait for it before the first load.
      pdl_wait();
      const uint64_t pol = policy_evict_first();
      const uint64_t pol_beta = policy_evict_last();
      long long it = 0;
      int issued = 0;
      ItemWalk iw(wb, we, tph, g.Hh);
      RingPos<kStStages> rp;
      // beta of the item about to be issued, fetched one item ahead so that
      // its global-load latency overlaps the wait for a free stage.
      uint16_t braw[kStTile / 32];
      auto fetch_beta = [&](const ItemWalk& w) {
#pragma unroll
        for (int k2 = 0; k2 < kStTile / 32; ++k2) {
          const int n = w.ti * kStTile + lane + 32 * k2;
          braw[k2] = n < g.N ? ld_u16_policy(p.beta + ((size_t)w.b * g.N + n) * g.Hh + w.h, pol_beta)
                             : (uint16_t)0;
        }
      };
      if (iw.more()) fetch_beta(iw);
      for (; iw.more(); iw.next(), rp.next(), ++it) {
        const int s = rp.s;
        if (!mbar_wait_warp_for(&empty[s], rp.ph ^ 1u, abort_flag, p.wait_ns)) break;
        const int b = iw.b, h = iw.h;
        const int n0 = iw.ti * kStTile;
        // Lane 0 starts the tile copies first; then the warp stores beta,
        // prefetches the next item's, computes the row metadata and arrives
        // once more.
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], 2 * kStTileBytes);
          unsigned char* kt = sm + TcStateSmem::K + s * kStTileBytes;
          unsigned char* vt = sm + TcStateSmem::V + s * kStTileBytes;
          tma_load_3d(kt, &tmK, &full[s], h * 128, n0, b, pol);
          tma_load_3d(kt + kStBox, &tmK, &full[s], h * 128 + 64, n0, b, pol);
          tma_load_3d(vt, &tmV, &full[s], h * 128, n0, b, pol);
          tma_load_3d(vt + kStBox, &tmV, &full[s], h * 128 + 64, n0, b, pol);
        }
        float* bs = reinterpret_cast<float*>(sm + TcStateSmem::BETA + s * kStTile * 4);
#pragma unroll
        for (int k2 = 0; k2 < kStTile / 32; ++k2)
          bs[lane + 32 * k2] = __uint_as_float((uint32_t)braw[k2] << 16);
        {
          ItemWalk nx = iw;
          nx.next();
          if (nx.more()) fetch_beta(nx);
        }
        if (g.rope_on)
          tile_rowrec<kStTile>(g, win, n0, lane,
                               sm + TcStateSmem::ROWREC + s * kStTile * kRecBytes);
        __syncwarp();
        // (the self-test withholds one arrival so that the consumers' waits run out)
        if (lane == 0 && !(c == 0 && it == p.stall_item)) mbar_arrive(&full[s]);
        ++issued;
        // While the first tiles land: this CTA's rows of the whole-call RoPE
        // table the read-out copies.  Written after the wait above, so the
        // previous call's read-out, which read the same buffer, has finished.
        if (it == 0 && p.rope_tab != nullptr)
          rope_build_global(p.rope_tab, g, blockIdx.x, gridDim.x, lane, 32);
      }
      if (*abort_flag && lane == 0) {
        // Let every load in flight land before shared memory is released.
        long long first = it - (issued < kStStages ? issued : kStStages);
        for (long long i2 = first; i2 < it; ++i2) {
          int dummy = 0;
          mbar_wait_for(&full[i2 % kStStages], (uint32_t)((i2 / kStStages) & 1),
                        reinterpret_cast<volatile int*>(&dummy), p.wait_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, true, true);
      int seg = 0;
      ItemWalk iw(wb, we, tph, g.Hh);
      RingPos<kStStages> rp;
      for (; iw.more(); iw.next(), rp.next()) {
        const int s = rp.s;
        const uint32_t ph = rp.ph;
        const bool first = iw.first, last = iw.last;
        const int ab = seg & 1;
        if (first && !mbar_wait_for(&accempty[ab], (uint32_t)(((seg >> 1) & 1) ^ 1), abort_flag,
                                    p.wait_ns))
          break;
        if (!mbar_wait_for(&kready[s], ph, abort_flag, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t kt = sbase + TcStateSmem::K + s * kStTileBytes;
        const uint32_t vt = sbase + TcStateSmem::V + s * kStTileBytes;
#pragma unroll
        for (int kk = 0; kk < kStTile / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(vt + kk * 2048, kStBox, 1024);
          const uint64_t bd = sdesc_sw128(kt + kk * 2048, kStBox, 1024);
          umma_f16kind(tmem + ab * 128, ad, bd, idesc, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&empty[s]);
        if (last) {
          umma_commit(&accfull[ab]);
          ++seg;
        }
      }
      // Every MMA issued above has completed before TMEM is released.
      umma_commit(drain);
      int dummy = 0;
      mbar_wait_for(drain, 0, reinterpret_cast<volatile int*>(&dummy), p.wait_ns);
    }
  } else {
    // ------------------------------------------- transform warps: k -> beta k_til
    // The RoPE table is built here, while the first tiles are in flight.
    rope_build(tab, g, win, threadIdx.x - kStTW0 * 32, kStTW * 32);
    named_barrier(1, kStTW * 32);
    const int tw = warp - kStTW0;
    const int rg = tw_row(lane), j = tw_chunk(lane);
    LaneRope lr;
    lane_rope(g, j, smem_u32(tab), lr);
    // This lane's two 16-byte chunks in row (tw*4 + rg) of a tile; rows of later
    // passes add whole multiples of 8 rows, which keeps the swizzle phase.
    uint32_t ch0, ch1;
    lane_chunks(0, kStBox, tw * 4 + rg, j, ch0, ch1);
    f2_t zacc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) zacc[i] = 0ull;
    int seg = 0;
    bool ok = true;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<kStStages> rp;
    for (; iw.more() && ok; iw.next(), rp.next()) {
      const int s = rp.s;
      const uint32_t ph = rp.ph;
      const int bh = iw.bh;
      if (!mbar_wait_warp_for(&full[s], ph, abort_flag, p.wait_ns)) { ok = false; break; }
      const uint32_t kt = sbase + TcStateSmem::K + s * kStTileBytes;
      const float* bs = reinterpret_cast<const float*>(sm + TcStateSmem::BETA + s * kStTile * 4);
      const uint32_t rec_s = sbase + TcStateSmem::ROWREC + s * kStTile * kRecBytes;
      // The warp's kStRows row groups of the tile (4 rows each, kStRowsPerPass
      // apart) are processed together: all shared loads first, then each row
      // group's arithmetic and stores.
      uint32_t a0[kStRows], a1[kStRows], t012[kStRows], t345[kStRows], t67[kStRows];
      float bcur[kStRows];
      uint4 in0[kStRows], in1[kStRows];
      f2_t e[kStRows][8];
#pragma unroll
      for (int u = 0; u < kStRows; ++u) {
        const int r = u * kStRowsPerPass + tw * 4 + rg;
        a0[u] = kt + ch0 + u * kStRowsPerPass * 128;
        a1[u] = kt + ch1 + u * kStRowsPerPass * 128;
        bcur[u] = bs[r];
        if (g.rope_on) lane_rope_row(lr, rec_s + r * kRecBytes, t012[u], t345[u], t67[u]);
      }
#pragma unroll
      for (int u = 0; u < kStRows; ++u) {
        in0[u] = lds128(a0[u]);
        in1[u] = lds128(a1[u]);
      }
      if (g.rope_on) {
#pragma unroll
        for (int u = 0; u < kStRows; ++u) tab_load8(t012[u], t345[u], t67[u], e[u]);
      }
#pragma unroll
      for (int u = 0; u < kStRows; ++u) {
        f2_t x[8];
        unpack8(in0[u], in1[u], x);
        const float rstd = row_rstd(x);
        const f2_t rstd2 = f2(rstd, rstd);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          x[i] = f2_relu(x[i]);                     // ReLU before the (positive) scale
          zacc[i] = f2_fma(x[i], rstd2, zacc[i]);   // z += k_pls
        }
        uint4 o0, o1;
        rope_scale_pack<false>(g.rope_on, e[u], x, rstd * bcur[u], o0, o1);
        sts128(a0[u], o0);
        sts128(a1[u], o1);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&kready[s]);

      if (iw.last) {
        // z of this head segment: sum the warp's four row groups, then store
        // one partial per warp (the combine adds them in warp order).
        float zf[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          zf[2 * i] = f2_lo(zacc[i]);
          zf[2 * i + 1] = f2_hi(zacc[i]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {          // add the warp's four rows
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

        // All transform warps drain the finished accumulator: row a of the
        // partial S is TMEM lane a; the three warps of a lane quarter take
        // every third group of 8 columns.
        {
          const int q4 = warp & 3;
          const int third = tw >> 2;
          const int a = q4 * 32 + lane;
          const int ab = seg & 1;
          if (!mbar_wait_warp_for(&accfull[ab], (uint32_t)((seg >> 1) & 1), abort_flag, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // Chunk-major partial: columns 8cb .. 8cb+7 of row a at (cb * 128 + a) * 8,
          // so the warp's 32 rows of a chunk are 1 KB of contiguous stores.
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

// --------------------------------------------------------------- apply kernel

constexpr int kApQ = 2;                      // q ring
constexpr int kApG = 3;                      // g / out ring
constexpr int kApAcc = 2;                    // TMEM accumulators
constexpr int kApDen = kApQ + kApAcc;        // den ring
constexpr int kApTW = 8;
constexpr int kApIL = 2;                     // row groups a transform warp takes at once
constexpr int kApTW0 = 3;                    // transform warps 3..10
constexpr int kApEW0 = kApTW0 + kApTW;       // epilogue warps 11..14
constexpr int kApEW = 4;                     // one per TMEM lane quarter
constexpr int kApST = kApEW0 + kApEW;        // store warp 15
constexpr int kApThreads = (kApST + 1) * 32;
constexpr int kApPrefetch = 2;               // items ahead whose q, g tiles go to L2 early
constexpr int kApRowsPerPass = kApTW * 4 * kApIL;
constexpr int kApPasses = kTcTile / kApRowsPerPass;
static_assert(kTcTile % kApRowsPerPass == 0, "whole passes per read-out tile");
static_assert((kApTW * 4) % 8 == 0, "row groups keep the 8-row swizzle phase");

struct TcApplySmem {
  static constexpr uint32_t Q = 0;
  static constexpr uint32_t G = kApQ * kTileBytes;
  static constexpr uint32_t SIMG = G + kApG * kTileBytes;
  static constexpr uint32_t Z = SIMG + kTileBytes;         // z [128] f32
  static constexpr uint32_t SCL = Z + 512;                  // image scale [4] f32
  static constexpr uint32_t DEN = SCL + 16;                 // [kApDen][128] den*scale per tile
  static constexpr uint32_t ROWREC = DEN + kApDen * 512;    // [q slot][128] records
  static constexpr uint32_t BAR = ROWREC + kApQ * kTcTile * kRecBytes;
  static constexpr uint32_t NBAR = 3 * kApQ + 3 * kApG + 2 * kApAcc + 5;
  static constexpr uint32_t MISC = BAR + NBAR * 8;
  static constexpr uint32_t TAB = (MISC + 16 + 15) & ~15u;
};

struct TcApplyParams {
  Geom g;
  Partition part;
  const __half* S_img;         // [BH][128*128] swizzled fp16 image of S * scale
  const float* S_scale;        // [BH][4]: [0] = scale of the image
  const float* z;              // [BH][128]
  const float2* rope_tab;      // the call's whole RoPE table (rope_layout(g, g.T))
  float* den_out;              // optional
  float* x_out;                // optional
  int tab_entries;
};

template <bool kDebug>
__global__ void __launch_bounds__(kApThreads, 1)
    tc_apply_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmG,
                    const __grid_constant__ CUtensorMap tmO, TcApplyParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + TcApplySmem::BAR);
  uint64_t* qfull = bars;
  uint64_t* qready = qfull + kApQ;
  uint64_t* qempty = qready + kApQ;
  uint64_t* gfull = qempty + kApQ;
  uint64_t* gempty = gfull + kApG;
  uint64_t* ostaged = gempty + kApG;
  uint64_t* accfull = ostaged + kApG;
  uint64_t* accempty = accfull + kApAcc;
  uint64_t* sfull = accempty + kApAcc;
  uint64_t* sfree = sfull + 1;
  uint64_t* drain = sfree + 1;
  uint64_t* zfull = drain + 1;    // z and the image scale of a segment's head
  uint64_t* tfull = zfull + 1;    // the RoPE table (once)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + TcApplySmem::MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + TcApplySmem::MISC + 4);
  float* zs = reinterpret_cast<float*>(sm + TcApplySmem::Z);
  const float* scl_s = reinterpret_cast<const float*>(sm + TcApplySmem::SCL);
  float* den_ring = reinterpret_cast<float*>(sm + TcApplySmem::DEN);
  float2* tab = reinterpret_cast<float2*>(sm + TcApplySmem::TAB);

  const Geom& g = p.g;
  const Partition& part = p.part;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long wb = part_begin(part, c), we = part_begin(part, c + 1);
  const RopeWindow win = rope_window(g, part, wb, we - 1);
  const int tph = part.tiles_per_head;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kApQ; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qready[s], kApTW);
      mbar_init(&qempty[s], 1);
    }
    for (int s = 0; s < kApG; ++s) {
      mbar_init(&gfull[s], 1);
      mbar_init(&gempty[s], 1);
      mbar_init(&ostaged[s], kApEW);
    }
    for (int a = 0; a < kApAcc; ++a) {
      mbar_init(&accfull[a], 1);
      mbar_init(&accempty[a], 4);
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
  // The next kernel on the stream may start its prologue as our CTAs finish.
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sbase = smem_u32(sm);

  if (warp == 0) {
    // ------------------------------------------------- producer: S image + q
    // All lanes compute the tile's row metadata; lane 0 issues the copies.
    // The S image, z and scale come from the combine kernel, which may still
    // be running (programmatic dependent launch): the first q tiles are
    // requested before waiting for it.
    {
      const uint64_t pol = policy_evict_first();
      int seg = 0, issued = 0;
      bool combined = false;
      ItemWalk iw(wb, we, tph, g.Hh);
      ItemWalk ahead = iw;      // the item kApPrefetch ahead of iw
      ahead.next();
      for (int k = 1; k < kApPrefetch && ahead.more(); ++k) {
        if (lane == 0) {
          tma_prefetch_3d(&tmQ, ahead.h * 128, ahead.ti * kTcTile, ahead.b);
          tma_prefetch_3d(&tmQ, ahead.h * 128 + 64, ahead.ti * kTcTile, ahead.b);
        }
        ahead.next();
      }
      RingPos<kApQ> rq;
      for (; iw.more(); iw.next(), rq.next()) {
        const int bh = iw.bh, b = iw.b, h = iw.h;
        if (ahead.more()) {
          if (lane == 0) {
            tma_prefetch_3d(&tmQ, ahead.h * 128, ahead.ti * kTcTile, ahead.b);
            tma_prefetch_3d(&tmQ, ahead.h * 128 + 64, ahead.ti * kTcTile, ahead.b);
          }
          ahead.next();
        }
        const int s = rq.s;
        if (!mbar_wait_warp(&qempty[s], rq.ph ^ 1u, abort_flag)) break;
        const int n0 = iw.ti * kTcTile;
        if (g.rope_on)
          tile_rowrec<kTcTile>(g, win, n0, lane, sm + TcApplySmem::ROWREC + s * kTcTile * kRecBytes);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&qfull[s], kTileBytes);
          unsigned char* qt = sm + TcApplySmem::Q + s * kTileBytes;
          tma_load_3d(qt, &tmQ, &qfull[s], h * 128, n0, b, pol);
          tma_load_3d(qt + kBox, &tmQ, &qfull[s], h * 128 + 64, n0, b, pol);
        }
        ++issued;
        if (iw.first) {
          if (!combined) {
            pdl_wait();
            combined = true;
          }
          // Every lane waits, so the warp leaves the loop together on a timeout.
          if (!mbar_wait_warp(sfree, (uint32_t)((seg & 1) ^ 1), abort_flag)) break;
          if (lane == 0) {
            // Smallest first: z and the scale (the transform warps' only
            // dependence on the combine), the RoPE table, then the S image.
            mbar_arrive_expect_tx(zfull, 512 + 16);
            bulk_load(sm + TcApplySmem::Z, p.z + (size_t)bh * 128, 512, zfull);
            bulk_load(sm + TcApplySmem::SCL, p.S_scale + (size_t)bh * 4, 16, zfull);
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
            bulk_load(sm + TcApplySmem::SIMG, p.S_img + (size_t)bh * 128 * 128, kTileBytes, sfull);
          }
          ++seg;
        }
      }
      if (*abort_flag && lane == 0) {
        // q loads went out for items 0 .. issued-1: let the last kApQ land.
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
    }
  } else if (warp == 2) {
    // ------------------------------------------------------ producer: g
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      long long it = 0;
      int issued = 0;
      ItemWalk iw(wb, we, tph, g.Hh);
      ItemWalk ahead = iw;
      for (int k = 0; k < kApPrefetch && ahead.more(); ++k) ahead.next();
      RingPos<kApG> rg_;
      // The first g tiles are needed only after the first read-out MMA: let
      // the q tiles, z, the table and the S image go first.  tfull completes
      // once, after the q producer has issued all of them.
      const bool go = !iw.more() || mbar_wait(tfull, 0u, abort_flag);
      for (; go && iw.more(); iw.next(), rg_.next(), ++it) {
        const int b = iw.b, h = iw.h;
        const int s = rg_.s;
        if (ahead.more()) {
          tma_prefetch_3d(&tmG, ahead.h * 128, ahead.ti * kTcTile, ahead.b);
          tma_prefetch_3d(&tmG, ahead.h * 128 + 64, ahead.ti * kTcTile, ahead.b);
          ahead.next();
        }
        if (!mbar_wait(&gempty[s], rg_.ph ^ 1u, abort_flag)) break;
        const int n0 = iw.ti * kTcTile;
        mbar_arrive_expect_tx(&gfull[s], kTileBytes);
        unsigned char* gt = sm + TcApplySmem::G + s * kTileBytes;
        tma_load_3d(gt, &tmG, &gfull[s], h * 128, n0, b, pol);
        tma_load_3d(gt + kBox, &tmG, &gfull[s], h * 128 + 64, n0, b, pol);
        ++issued;
      }
      if (*abort_flag) {
        long long first = it - (issued < kApG ? issued : kApG);
        for (long long i2 = first; i2 < it; ++i2) {
          int dummy = 0;
          mbar_wait(&gfull[i2 % kApG], (uint32_t)((i2 / kApG) & 1),
                    reinterpret_cast<volatile int*>(&dummy));
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, 128, false, false);
      int seg = 0;
      const uint32_t simg = sbase + TcApplySmem::SIMG;
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
        const uint32_t qt = sbase + TcApplySmem::Q + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32;
          const uint64_t ad = sdesc_sw128(qt + koff, 16, 1024);
          const uint64_t bd = sdesc_sw128(simg + koff, 16, 1024);
          umma_f16kind(tmem + ab * 128, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&qempty[s]);
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
    // ------------------------------------ transform warps: q -> q_til, den
    // The RoPE table comes by bulk copy from the whole-call table that the
    // state kernel's producer warps write.
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
      const int n0 = iw.ti * kTcTile;
      const uint32_t qt = sbase + TcApplySmem::Q + s * kTileBytes;
      float* den = den_ring + rd.s * 128;
      const uint32_t rec_s = sbase + TcApplySmem::ROWREC + s * kTcTile * kRecBytes;
#pragma unroll 1
      for (int ps = 0; ps < kApPasses; ++ps) {
        // kApIL row groups (4 rows each, kApTW * 4 rows apart) at once: shared
        // loads of every row first, then each row group's arithmetic and stores.
        uint32_t a0[kApIL], a1[kApIL], t012[kApIL], t345[kApIL], t67[kApIL];
        uint4 in0[kApIL], in1[kApIL];
        f2_t e[kApIL][8];
#pragma unroll
        for (int u = 0; u < kApIL; ++u) {
          const int r = ps * kApRowsPerPass + u * kApTW * 4 + tw * 4 + rg;
          a0[u] = qt + ch0 + (ps * kApRowsPerPass + u * kApTW * 4) * 128;
          a1[u] = qt + ch1 + (ps * kApRowsPerPass + u * kApTW * 4) * 128;
          if (g.rope_on) lane_rope_row(lr, rec_s + r * kRecBytes, t012[u], t345[u], t67[u]);
        }
#pragma unroll
        for (int u = 0; u < kApIL; ++u) {
          in0[u] = lds128(a0[u]);
          in1[u] = lds128(a1[u]);
        }
        if (g.rope_on) {
#pragma unroll
          for (int u = 0; u < kApIL; ++u) tab_load8(t012[u], t345[u], t67[u], e[u]);
        }
        float dn[kApIL];
#pragma unroll
        for (int u = 0; u < kApIL; ++u) {
          f2_t x[8];
          unpack8(in0[u], in1[u], x);
          const float rstd = row_rstd(x);
          f2_t dp2 = 0ull;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            x[i] = f2_relu(x[i]);
            dp2 = f2_fma(zr[i], x[i], dp2);
          }
          uint4 o0, o1;
          rope_scale_pack<true>(g.rope_on, e[u], x, rstd, o0, o1);
          sts128(a0[u], o0);
          sts128(a1[u], o1);
          const float dp = row_sum(f2_lo(dp2) + f2_hi(dp2));
          dn[u] = fmaf(dp, rstd, g.eps);               // z . q_pls + eps
        }
        if (j == 0) {
#pragma unroll
          for (int u = 0; u < kApIL; ++u) {
            const int r = ps * kApRowsPerPass + u * kApTW * 4 + tw * 4 + rg;
            // The read-out sees S * scale; fold the scale into the denominator.
            den[r] = dn[u] * hscale;
            const int n = n0 + r;
            if (kDebug && p.den_out && n < g.N) p.den_out[((size_t)b * g.N + n) * g.Hh + h] = dn[u];
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&qready[s]);
    }
  } else if (warp < kApST) {
    // ------------------------- epilogue warps: gate, denominator, RMSNorm
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    ItemWalk iw(wb, we, tph, g.Hh);
    RingPos<kApAcc> ra;
    RingPos<kApG> rg_;
    RingPos<kApDen> rd;
    for (; iw.more(); iw.next(), ra.next(), rg_.next(), rd.next()) {
      const int b = iw.b, h = iw.h;
      const int n0 = iw.ti * kTcTile;
      const int ab = ra.s;
      if (!mbar_wait_warp(&accfull[ab], ra.ph, abort_flag)) break;
      tc_fence_after();
      const int gsl = rg_.s;
      if (!mbar_wait_warp(&gfull[gsl], rg_.ph, abort_flag)) break;
      // sigma(g) / den' = (0.5 tanh(g/2) + 0.5) / den' = fma(hc, tanh(g/2), hc)
      const float hc = 0.5f / den_ring[rd.s * 128 + row];
      const uint32_t taddr = tmem + (uint32_t)(ab * 128) + ((uint32_t)(q4 * 32) << 16);
      const uint32_t gt = sbase + TcApplySmem::G + gsl * kTileBytes;
      const uint32_t grow = gt + (uint32_t)row * 128u;
      const uint32_t sw = (uint32_t)(row & 7);
      const f2_t hc2 = f2(hc, hc), half2 = f2(0.5f, 0.5f);
      f2_t ss2 = 0ull;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float u[32];
        tmem_ld32(taddr + cb * 32, u);
        const uint32_t rbase = grow + (uint32_t)(cb >> 1) * kBox;
        uint4 gv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) gv[q] = lds128(rbase + ((((uint32_t)((cb & 1) * 4 + q)) ^ sw) << 4));
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t wv[4] = {gv[q].x, gv[q].y, gv[q].z, gv[q].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const f2_t hg = f2_mul(f2_bf(wv[e]), half2);
            const f2_t t = f2(tanh_approx(f2_lo(hg)), tanh_approx(f2_hi(hg)));
            const f2_t sg = f2_fma(hc2, t, hc2);   // sigmoid(g) / den'
            const f2_t x = f2_mul(sg, f2(u[q * 8 + 2 * e], u[q * 8 + 2 * e + 1]));
            ss2 = f2_fma(x, x, ss2);
            u[q * 8 + 2 * e] = f2_lo(x);
            u[q * 8 + 2 * e + 1] = f2_hi(x);
          }
        }
        if (kDebug && p.x_out && n0 + row < g.N) {
          float* xo = p.x_out + (((size_t)b * g.N + n0 + row) * g.Hh + h) * 128 + cb * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(xo + i) = make_float4(u[i], u[i + 1], u[i + 2], u[i + 3]);
        }
        tmem_st32(taddr + cb * 32, u);
      }
      tmem_wait_st();
      const float rstd = rsqrtf((f2_lo(ss2) + f2_hi(ss2)) * (1.f / 128.f) + kRmsEps);
      const f2_t rstd2 = f2(rstd, rstd);
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        float x[32];
        tmem_ld32(taddr + cb * 32, x);
        tmem_wait_ld();
        const uint32_t rbase = grow + (uint32_t)(cb >> 1) * kBox;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const f2_t y = f2_mul(f2(x[q * 8 + 2 * e], x[q * 8 + 2 * e + 1]), rstd2);
            o[e] = pack_bf16(f2_lo(y), f2_hi(y));
          }
          sts128(rbase + ((((uint32_t)((cb & 1) * 4 + q)) ^ sw) << 4), make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&accempty[ab]);
        mbar_arrive(&ostaged[gsl]);
      }
    }
  } else if (warp == kApST) {
    // ------------------------------------------------------------- store
    // Once the four epilogue warps have staged a tile's output in its g slot,
    // store it and hand the slot back to the g producer as soon as the store
    // has read it.
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      ItemWalk iw(wb, we, tph, g.Hh);
      RingPos<kApG> rg_;
      for (; iw.more(); iw.next(), rg_.next()) {
        const int gsl = rg_.s;
        if (!mbar_wait(&ostaged[gsl], rg_.ph, abort_flag)) break;
        const int n0 = iw.ti * kTcTile;
        unsigned char* gt = sm + TcApplySmem::G + gsl * kTileBytes;
        tma_store_3d(&tmO, gt, iw.h * 128, n0, iw.b, pol);
        tma_store_3d(&tmO, gt + kBox, iw.h * 128 + 64, n0, iw.b, pol);
        bulk_commit();
        bulk_wait_read_all();
        mbar_arrive(&gempty[gsl]);
      }
      bulk_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [B][N][Hh][128] bf16 activations as a 3D map (channel, token, batch) with
// boxes of 64 channels x `rows` tokens, 128-byte swizzle, zero fill past N.
inline bool make_act_map(CUtensorMap* m, const void* ptr, const Geom& g, uint32_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)g.Hh * 128, (cuuint64_t)g.N, (cuuint64_t)g.B};
  cuuint64_t strides[2] = {(cuuint64_t)g.Hh * 128 * 2, (cuuint64_t)g.N * g.Hh * 128 * 2};
  cuuint32_t box[3] = {64, rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline size_t tc_state_smem(int tab_entries) {
  return 1024 + TcStateSmem::TAB + (size_t)tab_entries * 8;
}
inline size_t tc_apply_smem(int tab_entries) {
  return 1024 + TcApplySmem::TAB + (size_t)tab_entries * 8;
}
constexpr size_t kMaxSmem = 232448;

// Raises a kernel's dynamic shared-memory limit to all that its static shared
// memory leaves of kMaxSmem, once per device (slot: which kernel), instead of
// on every call: the attribute only bounds what a launch may ask for.
template <typename K>
inline bool ensure_max_smem(K kernel, int slot) {
  static std::atomic<unsigned char> done[4][64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < 64 && done[slot][dev].load(std::memory_order_acquire)) return true;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess || fa.sharedSizeBytes > kMaxSmem)
    return false;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)(kMaxSmem - fa.sharedSizeBytes)) != cudaSuccess)
    return false;
  if (dev >= 0 && dev < 64) done[slot][dev].store(1, std::memory_order_release);
  return true;
}

// The state reduction and the read-out split the same items differently
// (96- and 128-token tiles); each CTA count is at most the SM count.
inline Partition tc_state_partition(const Geom& g, int sms) {
  return make_partition(g.B * g.Hh, g.N, kStTile, sms);
}
inline Partition tc_apply_partition(const Geom& g, int sms) {
  return make_partition(g.B * g.Hh, g.N, kTcTile, sms);
}

// Per-CTA RoPE table size of a tensor partition (max over CTAs).
inline int tc_table_entries(const Geom& g, const Partition& part) {
  if (!g.rope_on) return 1;
  int mx = 1;
  for (int c = 0; c < part.grid; ++c) {
    const RopeWindow win = rope_window(g, part, part_begin(part, c), part_begin(part, c + 1) - 1);
    const int e = rope_table_entries(g, win.Lt);
    if (e > mx) mx = e;
  }
  return mx;
}

// The tensor path: state reduction, combine, read-out, each a programmatic
// dependent of the kernel before it.  S / z: the fp32 state (block-causal: in
// and out); z is always written, S only when write_state.
inline gla_status run_tensor(const Geom& g, const void* q, const void* k, const void* v,
                             const void* beta, const void* gate, void* out, float* S,
                             float* z, bool carry, bool write_state, float* part_S,
                             float* part_z, __half* S_img, float* S_scale, float2* rope_tab,
                             float* den_dbg, float* x_dbg, int sms, cudaStream_t stream,
                             void* const* events, unsigned long long stall_limit_ns = 0) {
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
  const size_t smem_st = tc_state_smem(stab), smem_ap = tc_apply_smem(tab);
  if (smem_st > kMaxSmem || smem_ap > kMaxSmem) return GLA_ERR_UNSUPPORTED;

  CUtensorMap mK, mV, mQ, mG, mO;
  if (!make_act_map(&mK, k, g, kStTile) || !make_act_map(&mV, v, g, kStTile) ||
      !make_act_map(&mQ, q, g, kTcTile) || !make_act_map(&mG, gate, g, kTcTile) ||
      !make_act_map(&mO, out, g, kTcTile))
    return GLA_ERR_CUDA;

  TcStateParams sp = {};
  sp.g = g; sp.part = spart;
  sp.beta = static_cast<const __nv_bfloat16*>(beta);
  sp.part_S = part_S; sp.part_z = part_z; sp.tab_entries = stab;
  sp.rope_tab = g.rope_on ? rope_tab : nullptr;
  sp.wait_ns = stall_limit_ns ? stall_limit_ns : kWaitLimitNs;
  sp.stall_item = stall_limit_ns ? 0 : -1;
  if (!ensure_max_smem(tc_state_kernel, 0)) return GLA_ERR_CUDA;
  if (mark(0) != cudaSuccess) return GLA_ERR_CUDA;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t sc = {};
  sc.gridDim = dim3(spart.grid);
  sc.blockDim = dim3(kStThreads);
  sc.dynamicSmemBytes = smem_st;
  sc.stream = stream;
  sc.attrs = pdl;
  sc.numAttrs = 1;
  if (cudaLaunchKernelEx(&sc, tc_state_kernel, mK, mV, sp) != cudaSuccess || mark(1) != cudaSuccess)
    return GLA_ERR_CUDA;

  CombineParams cp = {};
  cp.part = spart; cp.d = 128; cp.zparts = kStTW;
  cp.part_S = part_S; cp.part_z = part_z;
  cp.S_in = carry ? S : nullptr;
  cp.z_in = carry ? z : nullptr;
  cp.S_out = write_state ? S : nullptr;
  cp.z_out = z; cp.S_img = S_img; cp.S_scale = S_scale;
  cp.chunked = 1;
  // Slots of the head with the most: the bulk-copy combine takes every slot
  // of a head in one round while they fit its shared memory.
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

  TcApplyParams ap = {};
  ap.g = g; ap.part = part; ap.S_img = S_img; ap.S_scale = S_scale; ap.z = z;
  ap.rope_tab = rope_tab;
  ap.den_out = den_dbg; ap.x_out = x_dbg; ap.tab_entries = tab;
  const bool dbg = den_dbg != nullptr || x_dbg != nullptr;
  cudaLaunchConfig_t ac = {};
  ac.gridDim = dim3(part.grid);
  ac.blockDim = dim3(kApThreads);
  ac.dynamicSmemBytes = smem_ap;
  ac.stream = stream;
  ac.attrs = pdl;
  ac.numAttrs = 1;
  cudaError_t e;
  if (dbg) {
    if (!ensure_max_smem(tc_apply_kernel<true>, 1)) return GLA_ERR_CUDA;
    e = cudaLaunchKernelEx(&ac, tc_apply_kernel<true>, mQ, mG, mO, ap);
  } else {
    if (!ensure_max_smem(tc_apply_kernel<false>, 2)) return GLA_ERR_CUDA;
    e = cudaLaunchKernelEx(&ac, tc_apply_kernel<false>, mQ, mG, mO, ap);
  }
  if (e != cudaSuccess || mark(3) != cudaSuccess) return GLA_ERR_CUDA;
  return GLA_OK;
}

}  // namespace gla
