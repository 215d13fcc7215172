// CUDA-core (fp32 FFMA) kernels of the operator: the path for fp32 inputs, for
// head dims other than 128, and the cross-check of the tensor-core path.
//
//   simt_state_kernel  split-N partial S = sum v (beta k_til)^T and z = sum k_pls
//   simt_apply_kernel  den, S q_til, gate and output RMSNorm per token
//
// The state partials are combined by combine_kernel (combine.cuh).
#pragma once

#include "common.cuh"

namespace gla {

constexpr int kSimtTile = 64;      // tokens per state item
constexpr int kSimtThreads = 256;

struct SimtStateParams {
  Geom g;
  Partition part;
  const void* k;
  const void* v;
  const void* beta;
  float* part_S;   // [slots][d][d]
  float* part_z;   // [slots][d]
  int tab_entries; // capacity of the shared-memory RoPE table
};

// Loads element e of a token row and computes RMSNorm + ReLU (+ RoPE) in a
// warp: lane l holds elements l + 32 m.  Returns in x_pls / x_til.
template <int D, typename Tin>
__device__ inline void row_features(const Tin* row, const Geom& g, const float2* tab,
                                    RopeWindow win, const RopeLayout& L, int f, int hh, int ww,
                                    int lane,
                                    float (&x_pls)[D / 32], float (&x_til)[D / 32],
                                    bool valid) {
  constexpr int M = D / 32;
  float x[M];
  float ss = 0.f;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    x[m] = valid ? to_f32<Tin>(row[lane + 32 * m]) : 0.f;
    ss = fmaf(x[m], x[m], ss);
  }
  ss = warp_sum(ss);
  const float rstd = rsqrtf(ss / (float)D + kRmsEps);
#pragma unroll
  for (int m = 0; m < M; ++m) x_pls[m] = fmaxf(x[m] * rstd, 0.f);
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const float other = __shfl_xor_sync(0xffffffffu, x_pls[m], 1);
    if (g.rope_on && valid) {
      const int e = lane + 32 * m;
      const float2 cs = tab[rope_index(g, win, L, e >> 1, f, hh, ww)];
      x_til[m] = (e & 1) ? fmaf(other, cs.y, x_pls[m] * cs.x)     // x0 s + x1 c
                         : fmaf(-other, cs.y, x_pls[m] * cs.x);   // x0 c - x1 s
    } else {
      x_til[m] = x_pls[m];
    }
  }
}

template <int D, typename Tin>
__global__ void __launch_bounds__(kSimtThreads) simt_state_kernel(SimtStateParams p) {
  constexpr int M = D / 32;
  constexpr int RB = D / 16;          // each thread owns an RB x RB block of S
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  float* kb = reinterpret_cast<float*>(smem_raw);          // [tile][D]
  float* vv = kb + kSimtTile * D;                          // [tile][D]
  float* zred = vv + kSimtTile * D;                        // [8][D]
  float2* tab = reinterpret_cast<float2*>(zred + 8 * D);   // RoPE table

  const Geom& g = p.g;
  const Partition& part = p.part;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tx = tid & 15, ty = tid >> 4;
  const int c = blockIdx.x;
  const long long w_begin = part_begin(part, c), w_end = part_begin(part, c + 1);
  const RopeWindow win = rope_window(g, part, w_begin, w_end - 1);
  const RopeLayout L = rope_layout(g, win.Lt);
  rope_build(tab, g, win, tid, blockDim.x);

  const Tin* kin = static_cast<const Tin*>(p.k);
  const Tin* vin = static_cast<const Tin*>(p.v);
  const Tin* bin = static_cast<const Tin*>(p.beta);
  const int HW = g.H * g.W;

  float acc[RB][RB];
  float zacc[M];
  for (long long w = w_begin; w < w_end;) {
    const int bh = (int)(w / part.tiles_per_head);
    const int b = bh / g.Hh, h = bh % g.Hh;
    long long seg_end = (long long)(bh + 1) * part.tiles_per_head;
    if (seg_end > w_end) seg_end = w_end;
#pragma unroll
    for (int i = 0; i < RB; ++i)
#pragma unroll
      for (int j = 0; j < RB; ++j) acc[i][j] = 0.f;
#pragma unroll
    for (int m = 0; m < M; ++m) zacc[m] = 0.f;

    for (; w < seg_end; ++w) {
      const int n_base = (int)(w % part.tiles_per_head) * kSimtTile;
      __syncthreads();   // previous tile's smem fully consumed (and table built)
      for (int r = warp; r < kSimtTile; r += kSimtThreads / 32) {
        const int n = n_base + r;
        const bool valid = n < g.N;
        const int f = valid ? n / HW : 0, hh = valid ? (n / g.W) % g.H : 0,
                  ww = valid ? n % g.W : 0;
        const size_t row = (((size_t)b * g.N + (valid ? n : 0)) * g.Hh + h);
        float xp[M], xt[M];
        row_features<D, Tin>(kin + row * D, g, tab, win, L, f, hh, ww, lane, xp, xt, valid);
        const float be = valid ? to_f32<Tin>(bin[row]) : 0.f;
#pragma unroll
        for (int m = 0; m < M; ++m) {
          zacc[m] += xp[m];
          kb[r * D + lane + 32 * m] = xt[m] * be;
          vv[r * D + lane + 32 * m] = valid ? to_f32<Tin>(vin[row * D + lane + 32 * m]) : 0.f;
        }
      }
      __syncthreads();
      for (int r = 0; r < kSimtTile; ++r) {
        float va[RB], kc[RB];
#pragma unroll
        for (int i = 0; i < RB; ++i) va[i] = vv[r * D + ty * RB + i];
#pragma unroll
        for (int j = 0; j < RB; ++j) kc[j] = kb[r * D + tx * RB + j];
#pragma unroll
        for (int i = 0; i < RB; ++i)
#pragma unroll
          for (int j = 0; j < RB; ++j) acc[i][j] = fmaf(va[i], kc[j], acc[i][j]);
      }
    }
    // Segment done: write the partial of (CTA c, head bh) to slot c + bh.
    const size_t slot = (size_t)c + bh;
    float* dS = p.part_S + slot * D * D;
#pragma unroll
    for (int i = 0; i < RB; ++i)
#pragma unroll
      for (int j = 0; j < RB; ++j) dS[(ty * RB + i) * D + tx * RB + j] = acc[i][j];
#pragma unroll
    for (int m = 0; m < M; ++m) zred[warp * D + lane + 32 * m] = zacc[m];
    __syncthreads();
    if (tid < D) {
      float s = 0.f;
      for (int wi = 0; wi < kSimtThreads / 32; ++wi) s += zred[wi * D + tid];
      p.part_z[slot * D + tid] = s;
    }
  }
}

struct SimtApplyParams {
  Geom g;
  const void* q;
  const void* gate;
  const float* S;      // [BH][d][d] combined state
  const float* z;      // [BH][d]
  void* out;
  float* den_out;      // optional [B][N][Hh]
  float* x_out;        // optional [B][N][Hh][d]
  int tab_entries;
};

constexpr int kSimtApplyTile = 64;

template <int D, typename Tin>
__global__ void __launch_bounds__(kSimtThreads) simt_apply_kernel(SimtApplyParams p) {
  constexpr int M = D / 32;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  float* St = reinterpret_cast<float*>(smem_raw);   // St[c][a] = S[a][c]
  float* zs = St + D * D;
  float* qrow = zs + D;                             // [8 warps][D]
  float2* tab = reinterpret_cast<float2*>(qrow + 8 * D);

  const Geom& g = p.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y, b = bh / g.Hh, h = bh % g.Hh;
  const int n_base = blockIdx.x * kSimtApplyTile;
  const int HW = g.H * g.W;

  // Window of frames for this tile (single head, contiguous tokens).
  Partition tp;
  tp.BH = 1; tp.tile = kSimtApplyTile; tp.tiles_per_head = (g.N + kSimtApplyTile - 1) / kSimtApplyTile;
  tp.items = tp.tiles_per_head; tp.grid = 1;
  const RopeWindow win = rope_window(g, tp, blockIdx.x, blockIdx.x);
  const RopeLayout L = rope_layout(g, win.Lt);
  rope_build(tab, g, win, tid, blockDim.x);

  const float* Sg = p.S + (size_t)bh * D * D;
  for (int e = tid; e < D * D; e += blockDim.x) {
    const int a = e / D, cc = e % D;
    St[cc * D + a] = Sg[e];
  }
  for (int e = tid; e < D; e += blockDim.x) zs[e] = p.z[(size_t)bh * D + e];
  __syncthreads();

  const Tin* qin = static_cast<const Tin*>(p.q);
  const Tin* gin = static_cast<const Tin*>(p.gate);
  Tin* oout = static_cast<Tin*>(p.out);
  float* qr = qrow + warp * D;
  for (int r = warp; r < kSimtApplyTile; r += kSimtThreads / 32) {
    const int n = n_base + r;
    if (n >= g.N) break;
    const int f = n / HW, hh = (n / g.W) % g.H, ww = n % g.W;
    const size_t row = (((size_t)b * g.N + n) * g.Hh + h);
    float xp[M], xt[M];
    row_features<D, Tin>(qin + row * D, g, tab, win, L, f, hh, ww, lane, xp, xt, true);
    float dsum = 0.f;
#pragma unroll
    for (int m = 0; m < M; ++m) dsum = fmaf(zs[lane + 32 * m], xp[m], dsum);
    const float den = warp_sum(dsum) + g.eps;
#pragma unroll
    for (int m = 0; m < M; ++m) qr[lane + 32 * m] = xt[m];
    __syncwarp();
    float u[M];
#pragma unroll
    for (int m = 0; m < M; ++m) u[m] = 0.f;
    for (int cc = 0; cc < D; ++cc) {
      const float qc = qr[cc];
#pragma unroll
      for (int m = 0; m < M; ++m) u[m] = fmaf(St[cc * D + lane + 32 * m], qc, u[m]);
    }
    __syncwarp();
    float x[M], ss = 0.f;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float gl = to_f32<Tin>(gin[row * D + lane + 32 * m]);
      const float sg = 1.f / (1.f + expf(-gl));
      x[m] = sg * (u[m] / den);
      ss = fmaf(x[m], x[m], ss);
    }
    ss = warp_sum(ss);
    const float rstd = rsqrtf(ss / (float)D + kRmsEps);
#pragma unroll
    for (int m = 0; m < M; ++m) oout[row * D + lane + 32 * m] = from_f32<Tin>(x[m] * rstd);
    if (p.x_out) {
#pragma unroll
      for (int m = 0; m < M; ++m) p.x_out[row * D + lane + 32 * m] = x[m];
    }
    if (p.den_out && lane == 0) p.den_out[row] = den;
  }
}

}  // namespace gla
