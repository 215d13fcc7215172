// Shared device/host definitions of libgla: problem geometry, the split-N
// partition of the state reduction, and the per-CTA 3D-RoPE cos/sin table.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gla {

constexpr float kRmsEps = 1e-6f;     // RMSNorm epsilon of q, k and the output
constexpr int kMaxStateCtas = 512;   // upper bound of the state-kernel grid

// Library-wide device error word (bit 0: a bounded wait timed out).
__device__ unsigned int g_device_error;

enum : unsigned { kErrTimeout = 1u };

// ----------------------------------------------------------------- geometry

// Division by a runtime-invariant divisor d >= 1 for 0 <= n < 2^30:
// q = (umulhi(n, m) + n) >> l with l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994, section 4).
struct FastDiv {
  uint32_t m, l, d;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.l = 0;
  while ((1ull << f.l) < d) ++f.l;
  f.m = (uint32_t)((((1ull << 32) * ((1ull << f.l) - d)) / d) + 1);
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.m) + n) >> f.l;
}

struct Geom {
  int B, Hh, d;          // batch, heads, head dim
  int T, H, W, N;        // latent grid of this call, N = T*H*W
  int t0;                // time position of local frame 0
  int pt, ph, pw;        // rotation pairs per axis (t, h, w)
  int rope_on;           // 0: identity rotation
  float theta;           // RoPE base
  float eps;             // denominator epsilon
  FastDiv div_HW, div_W; // n -> frame, n % HW -> row
  double freq[64];       // theta^(-i/np) of global rotation pair i .. (pair i of its axis)
};

__host__ __device__ inline void rope_split(int d, int* pt, int* ph, int* pw) {
  int p = d / 2;
  int hw = p / 3;
  *pt = p - 2 * hw;
  *ph = hw;
  *pw = hw;
}

// --------------------------------------------------------------- partition
//
// The state reduction walks "items" = (head bh, tile i) in the order
// item = bh * tiles_per_head + i.  CTA c of G owns the items
// [floor(c*I/G), floor((c+1)*I/G)).  The partial of CTA c for head bh is
// stored in slot c + bh: along the item order (c, bh) never decreases in either
// component and changes in at least one at every segment boundary, so slots
// are unique and at most G + BH are used.

struct Partition {
  int BH;              // batch * heads
  int tile;            // tokens per item
  int tiles_per_head;  // ceil(N / tile)
  long long items;     // BH * tiles_per_head
  int grid;            // G
};

__host__ __device__ inline long long part_begin(const Partition& p, int c) {
  return (long long)c * p.items / p.grid;
}

// CTA owning item w: the largest c with floor(c*I/G) <= w.
__host__ __device__ inline int part_cta_of(const Partition& p, long long w) {
  return (int)(((w + 1) * (long long)p.grid - 1) / p.items);
}

inline Partition make_partition(int BH, int N, int tile, int max_grid) {
  Partition p;
  p.BH = BH;
  p.tile = tile;
  p.tiles_per_head = (N + tile - 1) / tile;
  p.items = (long long)BH * p.tiles_per_head;
  long long g = p.items < max_grid ? p.items : max_grid;
  if (g > kMaxStateCtas) g = kMaxStateCtas;
  if (g < 1) g = 1;
  p.grid = (int)g;
  return p;
}

// --------------------------------------------------------------- RoPE table
//
// Each CTA keeps cos/sin of the rotations it needs in shared memory, as float2
// (cos, sin) entries, position-major inside each axis:
//   time axis:   Lt rows (frames t_lo .. t_lo+Lt-1, wrapping modulo T when
//                the CTA's tokens cross from the end of one head's sequence to
//                the start of the next)
//   height axis: H rows;  width axis: W rows.
// Pair p (global index 0 .. d/2-1) of axis a sits at column
//   idx(p) = (p - start_a) + (p >> 3) - (start_a >> 3)
// of its row: one padding entry after every 8 global pairs, so the 8 pairs a
// tensor-path lane handles are contiguous while lanes land on different banks.
// Row strides and axis bases (rope_layout) are chosen so that the transform
// warps' lookups are free of shared-memory bank conflicts.  Angles are formed
// and reduced in double precision; cos/sin are evaluated in fp32.

struct RopeWindow {
  int t_lo;   // first local frame held
  int Lt;     // frames held (<= T)
};

struct RopeLayout {
  int start[3];    // first global pair of each axis
  int stride[3];   // entries per row
  int base[3];     // first entry of each axis
  int entries;     // table size
};

__host__ __device__ inline int rope_idx(const RopeLayout& L, int a, int p) {
  return (p - L.start[a]) + (p >> 3) - (L.start[a] >> 3);
}

__host__ __device__ inline RopeLayout rope_layout(const Geom& g, int Lt) {
  RopeLayout L;
  const int np[3] = {g.pt, g.ph, g.pw};
  L.start[0] = 0;
  L.start[1] = g.pt;
  L.start[2] = g.pt + g.ph;
  for (int a = 0; a < 3; ++a) {
    const int last = L.start[a] + np[a] - 1;
    const int width = np[a] > 0 ? (last - L.start[a]) + (last >> 3) - (L.start[a] >> 3) + 1 : 0;
    // time rows: a multiple of 16 entries; height/width rows: 8 mod 16.
    L.stride[a] = a == 0 ? (width + 15) / 16 * 16 : ((width + 7) / 16) * 16 + 8;
  }
  const int rows[3] = {Lt, g.H, g.W};
  int off = 0;
  for (int a = 0; a < 3; ++a) {
    L.base[a] = off;
    off = (off + rows[a] * L.stride[a] + 15) / 16 * 16;
  }
  L.entries = off;
  return L;
}

// Frames touched by the items [w0, w1] (inclusive) of a partition.
__host__ __device__ inline RopeWindow rope_window(const Geom& g, const Partition& p,
                                                  long long w0, long long w1) {
  const int HW = g.H * g.W;
  const int bh0 = (int)(w0 / p.tiles_per_head), bh1 = (int)(w1 / p.tiles_per_head);
  const int n0 = (int)(w0 % p.tiles_per_head) * p.tile;
  int n1 = (int)(w1 % p.tiles_per_head) * p.tile + p.tile - 1;
  if (n1 > g.N - 1) n1 = g.N - 1;
  const int f0 = n0 / HW, f1 = n1 / HW;
  RopeWindow r;
  if (bh0 == bh1 && f1 >= f0) {
    r.t_lo = f0;
    r.Lt = f1 - f0 + 1;
  } else if (bh1 == bh0 + 1 && f1 < f0) {
    r.t_lo = f0;                      // f0 .. T-1, then 0 .. f1
    r.Lt = (g.T - f0) + (f1 + 1);
  } else {
    r.t_lo = 0;
    r.Lt = g.T;
  }
  if (r.Lt > g.T) { r.t_lo = 0; r.Lt = g.T; }
  return r;
}

__host__ __device__ inline int rope_table_entries(const Geom& g, int Lt) {
  return rope_layout(g, Lt).entries;
}

// (cos, sin) of position x at frequency freq: the angle is formed and reduced
// to [-pi, pi] in double, then evaluated in fp32.
__device__ __forceinline__ float2 rope_entry(double x, double freq) {
  const double two_pi = 6.283185307179586476925286766559;
  double ang = x * freq;
  ang -= two_pi * rint(ang * (1.0 / two_pi));
  float sn, cs;
  sincosf((float)ang, &sn, &cs);
  return make_float2(cs, sn);
}

__device__ inline void rope_build(float2* tab, const Geom& g, RopeWindow win, int tid,
                                  int nthr) {
  if (!g.rope_on) return;
  // Thread tid handles rotation pair (tid mod P) of its axis at every
  // (nthr / P)-th position: one rope_entry per row.
  const RopeLayout L = rope_layout(g, win.Lt);
  const int P = g.pt + g.ph + g.pw;
  const int pr = tid % P;
  const int lane0 = tid / P, step = nthr / P;
  if (lane0 >= step) return;
  const int axis = pr < g.pt ? 0 : (pr < g.pt + g.ph ? 1 : 2);
  const int rows = axis == 0 ? win.Lt : (axis == 1 ? g.H : g.W);
  const int col = rope_idx(L, axis, pr);
  const double freq = g.freq[pr];
  for (int pos = lane0; pos < rows; pos += step) {
    double x;
    if (axis == 0) {
      int f = win.t_lo + pos;
      if (f >= g.T) f -= g.T;
      x = (double)(g.t0 + f);
    } else {
      x = (double)pos;
    }
    tab[L.base[axis] + pos * L.stride[axis] + col] = rope_entry(x, freq);
  }
}

// The whole call's table (all T frames: rope_layout(g, g.T), frame f at time
// row f) written to global memory, one table row (an axis position) per
// (row, pair) task; CTA `cta` of `ncta` takes rows cta, cta + ncta, ...
// Entries are the same rope_entry values rope_build produces.
__device__ inline void rope_build_global(float2* gtab, const Geom& g, int cta, int ncta,
                                         int tid, int nthr) {
  if (!g.rope_on) return;
  const RopeLayout L = rope_layout(g, g.T);
  const int rows_total = g.T + g.H + g.W;
  const int np_max = g.pt > g.ph ? (g.pt > g.pw ? g.pt : g.pw) : (g.ph > g.pw ? g.ph : g.pw);
  const int per = nthr / np_max;   // rows a CTA fills at once
  if (per == 0) return;
  const int i = tid % np_max, sub = tid / np_max;
  if (sub >= per) return;
  for (int r = cta + ncta * sub; r < rows_total; r += ncta * per) {
    const int axis = r < g.T ? 0 : (r < g.T + g.H ? 1 : 2);
    const int pos = axis == 0 ? r : (axis == 1 ? r - g.T : r - g.T - g.H);
    const int np = axis == 0 ? g.pt : (axis == 1 ? g.ph : g.pw);
    if (i >= np) continue;
    const double x = axis == 0 ? (double)(g.t0 + pos) : (double)pos;
    const int pr = L.start[axis] + i;
    gtab[L.base[axis] + pos * L.stride[axis] + rope_idx(L, axis, pr)] = rope_entry(x, g.freq[pr]);
  }
}

// The copies that turn the whole-call table (rope_layout(g, g.T) in global
// memory) into a CTA's windowed table (rope_layout(g, win.Lt) in shared
// memory): time rows t_lo .. T-1 and, for a window that wraps, 0 .. the rest;
// then the height and width blocks whole.  Offsets and sizes in entries; every
// one is a multiple of 8 entries (64 bytes), as bulk copies require.
struct RopeCopy {
  int n;
  int src[4], dst[4], len[4];
};

__host__ __device__ inline RopeCopy rope_copy_plan(const Geom& g, RopeWindow win) {
  const RopeLayout G = rope_layout(g, g.T), W = rope_layout(g, win.Lt);
  RopeCopy c;
  c.n = 0;
  int rows1 = g.T - win.t_lo;
  if (rows1 > win.Lt) rows1 = win.Lt;
  c.src[c.n] = G.base[0] + win.t_lo * G.stride[0];
  c.dst[c.n] = W.base[0];
  c.len[c.n++] = rows1 * G.stride[0];
  if (win.Lt > rows1) {
    c.src[c.n] = G.base[0];
    c.dst[c.n] = W.base[0] + rows1 * W.stride[0];
    c.len[c.n++] = (win.Lt - rows1) * G.stride[0];
  }
  c.src[c.n] = G.base[1]; c.dst[c.n] = W.base[1]; c.len[c.n++] = g.H * G.stride[1];
  c.src[c.n] = G.base[2]; c.dst[c.n] = W.base[2]; c.len[c.n++] = g.W * G.stride[2];
  return c;
}

// Index of the (cos, sin) entry of rotation pair `pr` (0 .. d/2-1) for a token
// at local frame f, row hh, column ww.
__device__ inline int rope_index(const Geom& g, RopeWindow win, const RopeLayout& L, int pr,
                                 int f, int hh, int ww) {
  if (pr < g.pt) {
    int tl = f - win.t_lo;
    if (tl < 0) tl += g.T;
    return L.base[0] + tl * L.stride[0] + rope_idx(L, 0, pr);
  }
  if (pr < g.pt + g.ph) return L.base[1] + hh * L.stride[1] + rope_idx(L, 1, pr);
  return L.base[2] + ww * L.stride[2] + rope_idx(L, 2, pr);
}

// ------------------------------------------------------------------ dtypes

template <typename T> __device__ inline float to_f32(T x);
template <> __device__ inline float to_f32<float>(float x) { return x; }
template <> __device__ inline float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T> __device__ inline T from_f32(float x);
template <> __device__ inline float from_f32<float>(float x) { return x; }
template <> __device__ inline __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ inline float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace gla
