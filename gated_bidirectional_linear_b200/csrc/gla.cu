// libgla: host side of the C ABI declared in include/gla.h.
//
// One translation unit: the kernels live in the included .cuh files.
// Host code validates arguments, plans the split-N partition, carves the
// caller's workspace and launches the kernels on the caller's stream.
#include <math.h>

#include <mutex>
#include <stdint.h>
#include <string.h>

#include "gla.h"

#include "common.cuh"
#include "combine.cuh"
#include "simt.cuh"
#include "tc.cuh"
#include "causal.cuh"
#include "mx.cuh"
#include "gemm.cuh"
#include "anchor.cuh"

using namespace gla;

namespace gla {

// One CTA waits on an mbarrier that no thread arrives on, through the
// pipelines' bounded wait with a short limit, then returns (see
// gla_selftest_wait_timeout).
__global__ void __launch_bounds__(32) selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  mbar_wait_for(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), limit_ns);
}

}  // namespace gla

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxZParts = kStTW;   // z partials per state slot (tensor path)

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

struct WsLayout {
  size_t part_S, part_z, S, z, S_img, S_scale, rope_tab, total;
  int slots;
};

// Bytes of the whole-call RoPE table the tensor path's combine writes for the
// read-out (every frame of the call; at least one 16-byte unit).
size_t rope_tab_bytes(int d, int T, int H, int W) {
  Geom g = {};
  g.d = d; g.T = T; g.H = H; g.W = W;
  rope_split(d, &g.pt, &g.ph, &g.pw);
  const size_t e = (size_t)rope_layout(g, T).entries;
  return (e > 2 ? e : 2) * sizeof(float2);
}

// Workspace carve-up; independent of the GPU (uses the maximum grid).
WsLayout ws_layout(int BH, int d, bool own_state, int T, int H, int W) {
  WsLayout L;
  L.slots = kMaxStateCtas + BH;
  size_t off = 0;
  L.part_S = off; off = align_up(off + (size_t)L.slots * d * d * 4, kAlign);
  L.part_z = off; off = align_up(off + (size_t)L.slots * kMaxZParts * d * 4, kAlign);
  if (own_state) {
    L.S = off; off = align_up(off + (size_t)BH * d * d * 4, kAlign);
    L.z = off; off = align_up(off + (size_t)BH * d * 4, kAlign);
  } else {
    L.S = L.z = 0;
  }
  L.S_img = off;
  if (d == 128) off = align_up(off + (size_t)BH * d * d * 2, kAlign);
  L.S_scale = off;
  if (d == 128) off = align_up(off + (size_t)BH * 4 * 4, kAlign);
  L.rope_tab = off;
  if (d == 128) off = align_up(off + rope_tab_bytes(d, T, H, W), kAlign);
  L.total = off;
  return L;
}

// The helper stream (one per device, created on first use and kept for the
// process) that carries gla_forward_host's output copies, and the events that
// fork it from and join it to the caller's stream.  The mutex keeps one
// call's fork and join together when several host threads use the device.
constexpr int kHostChunks = 8;
struct HostPipe {
  std::mutex mu;
  cudaStream_t s = nullptr;
  cudaEvent_t ev[kHostChunks + 1] = {};
};

HostPipe* host_pipe() {
  static std::mutex init_mu;
  static HostPipe pipes[64];
  static bool ready[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(init_mu);
  if (!ready[dev]) {
    HostPipe& p = pipes[dev];
    if (cudaStreamCreateWithFlags(&p.s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    for (auto& e : p.ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    ready[dev] = true;
  }
  return &pipes[dev];
}

bool dims_ok(int batch, int heads, int head_dim, int T, int H, int W) {
  if (batch <= 0 || heads <= 0 || T <= 0 || H <= 0 || W <= 0) return false;
  if (head_dim != 32 && head_dim != 64 && head_dim != 128) return false;
  const long long N = (long long)T * H * W;
  const long long elems = (long long)batch * N * heads * head_dim;
  if (N > (1LL << 30) || elems > (1LL << 40)) return false;
  return true;
}

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return -1;
  if (dev >= 0 && dev < 64) cache[dev] = sms;
  return sms;
}

Geom make_geom(int batch, int heads, int head_dim, int T, int H, int W, int t0,
               float rope_theta, float eps) {
  Geom g;
  g.B = batch; g.Hh = heads; g.d = head_dim;
  g.T = T; g.H = H; g.W = W; g.N = T * H * W;
  g.t0 = t0;
  rope_split(head_dim, &g.pt, &g.ph, &g.pw);
  g.rope_on = rope_theta > 0.f ? 1 : 0;
  g.theta = rope_theta;
  g.eps = eps;
  g.div_HW = make_fastdiv((uint32_t)(H * W));
  g.div_W = make_fastdiv((uint32_t)W);
  // Rotation frequencies in double: pair i of an axis with np pairs turns at
  // theta^(-i/np) radians per position.  Kept per thread for the last
  // (theta, d), since consecutive calls nearly always repeat them.
  struct FreqCache { float theta; int d; double freq[64]; };
  static thread_local FreqCache cache = {0.f, 0, {}};
  if (!(cache.theta == rope_theta && cache.d == head_dim)) {
    const int np[3] = {g.pt, g.ph, g.pw};
    for (int pr = 0, a = 0, i = 0; pr < 64; ++pr) {
      cache.freq[pr] = 0.0;
      if (pr >= g.pt + g.ph + g.pw || !g.rope_on) continue;
      while (i >= np[a]) { i -= np[a]; ++a; }
      cache.freq[pr] = exp(-((double)i / (double)np[a]) * log((double)rope_theta));
      ++i;
    }
    cache.theta = rope_theta;
    cache.d = head_dim;
  }
  memcpy(g.freq, cache.freq, sizeof(g.freq));
  return g;
}

// Largest per-CTA RoPE table (entries) over the CTAs of a partition.
int max_table_entries(const Geom& g, const Partition& p) {
  if (!g.rope_on) return 1;
  int mx = 1;
  for (int c = 0; c < p.grid; ++c) {
    const long long w0 = part_begin(p, c), w1 = part_begin(p, c + 1) - 1;
    const RopeWindow win = rope_window(g, p, w0, w1);
    const int e = rope_table_entries(g, win.Lt);
    if (e > mx) mx = e;
  }
  return mx;
}

int tile_table_entries(const Geom& g, int tile) {
  if (!g.rope_on) return 1;
  Partition tp;
  tp.BH = 1; tp.tile = tile; tp.tiles_per_head = (g.N + tile - 1) / tile;
  tp.items = tp.tiles_per_head; tp.grid = (int)tp.items;
  return max_table_entries(g, tp);
}

struct Call {
  Geom g;
  int dtype;
  int path;          // resolved: GLA_PATH_SIMT or GLA_PATH_TENSOR
  const void *q, *k, *v, *beta, *gate;
  void* out;
  float* S;          // combined state (workspace or caller's carried state)
  float* z;
  bool carry;        // S/z hold a carried state to add to
  unsigned char* ws;
  WsLayout L;
  cudaStream_t stream;
  float *S_dbg, *z_dbg, *den_dbg, *x_dbg;
  void* const* events;   // optional [4] cudaEvent_t records around the kernels
  unsigned long long stall_limit_ns = 0;   // self-test of the abort path (0: off)
};

inline cudaError_t mark(const Call& c, int i) {
  if (!c.events || !c.events[i]) return cudaSuccess;
  return cudaEventRecord(static_cast<cudaEvent_t>(c.events[i]), c.stream);
}

// The tensor path keeps the RoPE table of each CTA in shared memory next to
// its tile rings; grids whose table does not fit use the CUDA-core path.
bool tensor_fits(const Geom& g, int sms) {
  if (g.H >= (1 << kPosBits) || g.W >= (1 << kPosBits) || g.T >= (1 << kPosBits)) return false;
  if (!tc_rope_lanes_ok(g)) return false;
  const int stab = tc_table_entries(g, tc_state_partition(g, sms));
  const int tab = tc_table_entries(g, tc_apply_partition(g, sms));
  return tc_state_smem(stab) <= kMaxSmem && tc_apply_smem(tab) <= kMaxSmem;
}

int resolve_path(int requested, int dtype, int d, const Geom* g = nullptr, int sms = 0) {
  bool tensor_ok = dtype == GLA_DTYPE_BF16 && d == 128;
  if (tensor_ok && requested == GLA_PATH_AUTO && g && sms > 0) tensor_ok = tensor_fits(*g, sms);
  if (requested == GLA_PATH_AUTO) return tensor_ok ? GLA_PATH_TENSOR : GLA_PATH_SIMT;
  if (requested == GLA_PATH_SIMT) return GLA_PATH_SIMT;
  if (requested == GLA_PATH_TENSOR) return tensor_ok ? GLA_PATH_TENSOR : -1;
  return -1;
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int D, typename Tin>
gla_status run_simt(const Call& c) {
  const Geom& g = c.g;
  const int sms = device_sm_count();
  if (sms <= 0) return GLA_ERR_CUDA;
  const Partition part = make_partition(g.B * g.Hh, g.N, kSimtTile, 2 * sms);

  SimtStateParams sp;
  sp.g = g; sp.part = part;
  sp.k = c.k; sp.v = c.v; sp.beta = c.beta;
  sp.part_S = reinterpret_cast<float*>(c.ws + c.L.part_S);
  sp.part_z = reinterpret_cast<float*>(c.ws + c.L.part_z);
  sp.tab_entries = max_table_entries(g, part);
  const size_t smem_state = (size_t)(2 * kSimtTile * D + 8 * D) * 4 + (size_t)sp.tab_entries * 8;
  if (smem_state > 200 * 1024) return GLA_ERR_UNSUPPORTED;
  if (set_smem(simt_state_kernel<D, Tin>, smem_state) != cudaSuccess) return GLA_ERR_CUDA;
  if (mark(c, 0) != cudaSuccess) return GLA_ERR_CUDA;
  simt_state_kernel<D, Tin><<<part.grid, kSimtThreads, smem_state, c.stream>>>(sp);
  if (cudaGetLastError() != cudaSuccess || mark(c, 1) != cudaSuccess) return GLA_ERR_CUDA;

  CombineParams cp = {};
  cp.part = part; cp.d = D; cp.zparts = 1;
  cp.part_S = sp.part_S; cp.part_z = sp.part_z;
  cp.S_in = c.carry ? c.S : nullptr;
  cp.z_in = c.carry ? c.z : nullptr;
  cp.S_out = c.S; cp.z_out = c.z;
  cp.S_img = nullptr; cp.S_scale = nullptr;
  cp.chunked = 0;
  dim3 cgrid(kCombineCluster, g.B * g.Hh);
  combine_kernel<<<cgrid, kCombineThreads, 0, c.stream>>>(cp);
  if (cudaGetLastError() != cudaSuccess || mark(c, 2) != cudaSuccess) return GLA_ERR_CUDA;

  SimtApplyParams ap;
  ap.g = g; ap.q = c.q; ap.gate = c.gate; ap.S = c.S; ap.z = c.z; ap.out = c.out;
  ap.den_out = c.den_dbg; ap.x_out = c.x_dbg;
  ap.tab_entries = tile_table_entries(g, kSimtApplyTile);
  const size_t smem_apply = (size_t)(D * D + D + 8 * D) * 4 + (size_t)ap.tab_entries * 8;
  if (smem_apply > 200 * 1024) return GLA_ERR_UNSUPPORTED;
  if (set_smem(simt_apply_kernel<D, Tin>, smem_apply) != cudaSuccess) return GLA_ERR_CUDA;
  dim3 agrid((g.N + kSimtApplyTile - 1) / kSimtApplyTile, g.B * g.Hh);
  simt_apply_kernel<D, Tin><<<agrid, kSimtThreads, smem_apply, c.stream>>>(ap);
  if (cudaGetLastError() != cudaSuccess || mark(c, 3) != cudaSuccess) return GLA_ERR_CUDA;
  return GLA_OK;
}

template <typename Tin>
gla_status run_simt_dtype(const Call& c) {
  switch (c.g.d) {
    case 32: return run_simt<32, Tin>(c);
    case 64: return run_simt<64, Tin>(c);
    case 128: return run_simt<128, Tin>(c);
  }
  return GLA_ERR_UNSUPPORTED;
}

gla_status run_call(Call& c) {
  gla_status st;
  if (c.path == GLA_PATH_TENSOR) {
    const bool write_state = c.carry || c.S_dbg != nullptr;
    st = run_tensor(c.g, c.q, c.k, c.v, c.beta, c.gate, c.out, c.S, c.z, c.carry, write_state,
                    reinterpret_cast<float*>(c.ws + c.L.part_S),
                    reinterpret_cast<float*>(c.ws + c.L.part_z),
                    reinterpret_cast<__half*>(c.ws + c.L.S_img),
                    reinterpret_cast<float*>(c.ws + c.L.S_scale),
                    reinterpret_cast<float2*>(c.ws + c.L.rope_tab), c.den_dbg, c.x_dbg,
                    device_sm_count(), c.stream, c.events, c.stall_limit_ns);
  } else {
    st = c.dtype == GLA_DTYPE_F32 ? run_simt_dtype<float>(c)
                                  : run_simt_dtype<__nv_bfloat16>(c);
  }
  if (st != GLA_OK) return st;
  const size_t dd = (size_t)c.g.B * c.g.Hh * c.g.d * c.g.d;
  const size_t dz = (size_t)c.g.B * c.g.Hh * c.g.d;
  if (c.S_dbg && cudaMemcpyAsync(c.S_dbg, c.S, dd * 4, cudaMemcpyDeviceToDevice, c.stream) != cudaSuccess)
    return GLA_ERR_CUDA;
  if (c.z_dbg && cudaMemcpyAsync(c.z_dbg, c.z, dz * 4, cudaMemcpyDeviceToDevice, c.stream) != cudaSuccess)
    return GLA_ERR_CUDA;
  return GLA_OK;
}

// Workspace of a causal call (tensor path): the state partials and, per
// partial slot, the state before it.
struct CausalWs {
  size_t part_S, part_z, S_start, z_start, total;
};

CausalWs causal_ws(int BH, int d) {
  CausalWs L;
  const size_t slots = (size_t)kMaxStateCtas + BH;
  size_t off = 0;
  L.part_S = off; off = align_up(off + slots * d * d * 4, kAlign);
  L.part_z = off; off = align_up(off + slots * kMaxZParts * d * 4, kAlign);
  L.S_start = off; off = align_up(off + slots * d * d * 4, kAlign);
  L.z_start = off; off = align_up(off + slots * d * 4, kAlign);
  L.total = off;
  return L;
}

bool causal_tensor_fits(const Geom& g, int sms) {
  if (g.H >= (1 << kPosBits) || g.W >= (1 << kPosBits) || g.T >= (1 << kPosBits)) return false;
  if (!tc_rope_lanes_ok(g)) return false;
  const int stab = tc_table_entries(g, tc_state_partition(g, sms));
  return tc_state_smem(stab) <= kMaxSmem && tc_causal_smem(stab) <= kMaxSmem;
}

template <int D, typename Tin>
gla_status run_simt_causal(const Geom& g, const void* q, const void* k, const void* v,
                           const void* beta, const void* gate, void* out, float* S, float* z,
                           float* den_out, float* x_out, cudaStream_t stream) {
  SimtCausalParams sp;
  sp.g = g;
  sp.q = q; sp.k = k; sp.v = v; sp.beta = beta; sp.gate = gate; sp.out = out;
  sp.S = S; sp.z = z; sp.den_out = den_out; sp.x_out = x_out;
  const size_t smem = simt_causal_smem<D>();
  if (set_smem(simt_causal_kernel<D, Tin>, smem) != cudaSuccess) return GLA_ERR_CUDA;
  simt_causal_kernel<D, Tin><<<g.B * g.Hh, kSimtCausalThreads, smem, stream>>>(sp);
  return cudaGetLastError() == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

template <typename Tin>
gla_status run_simt_causal_dim(const Geom& g, const void* q, const void* k, const void* v,
                               const void* beta, const void* gate, void* out, float* S,
                               float* z, float* den_out, float* x_out, cudaStream_t stream) {
  switch (g.d) {
    case 32: return run_simt_causal<32, Tin>(g, q, k, v, beta, gate, out, S, z, den_out, x_out, stream);
    case 64: return run_simt_causal<64, Tin>(g, q, k, v, beta, gate, out, S, z, den_out, x_out, stream);
    case 128: return run_simt_causal<128, Tin>(g, q, k, v, beta, gate, out, S, z, den_out, x_out, stream);
  }
  return GLA_ERR_UNSUPPORTED;
}

// Device bytes of one call's five inputs and its output, staged in an arena
// for the host entry points of the stateful variants.
size_t staged_inputs_bytes(int batch, int heads, int head_dim, int T, int H, int W, int dtype) {
  const size_t esz = dtype == GLA_DTYPE_F32 ? 4 : 2;
  const size_t th = (size_t)batch * T * H * W * heads;
  return 5 * align_up(th * head_dim * esz, kAlign) + align_up(th * esz, kAlign);
}

// Copies one call's host inputs into the device arena, runs `step` on them
// (the state stays in device memory) and copies the output back, all
// enqueued on `stream`.
template <typename Step>
gla_status staged_step(const void* q_h, const void* k_h, const void* v_h, const void* beta_h,
                       const void* g_h, void* out_h, int batch, int heads, int head_dim, int T,
                       int H, int W, int dtype, void* arena, size_t arena_bytes, size_t need,
                       void* stream, Step step) {
  const void* hp[6] = {q_h, k_h, v_h, beta_h, g_h, out_h};
  for (const void* p : hp)
    if (!p) return GLA_ERR_INVALID_ARG;
  if (!arena || ((uintptr_t)arena % kAlign) != 0 || arena_bytes < need) return GLA_ERR_WORKSPACE;
  const size_t esz = dtype == GLA_DTYPE_F32 ? 4 : 2;
  const size_t th = (size_t)batch * T * H * W * heads;
  const size_t big = th * head_dim * esz, small = th * esz;
  unsigned char* a = static_cast<unsigned char*>(arena);
  unsigned char* dq = a;
  unsigned char* dk = dq + align_up(big, kAlign);
  unsigned char* dv = dk + align_up(big, kAlign);
  unsigned char* dg = dv + align_up(big, kAlign);
  unsigned char* dout = dg + align_up(big, kAlign);
  unsigned char* dbeta = dout + align_up(big, kAlign);
  unsigned char* dws = dbeta + align_up(small, kAlign);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(dq, q_h, big, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dk, k_h, big, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dv, v_h, big, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dg, g_h, big, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dbeta, beta_h, small, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return GLA_ERR_CUDA;
  const gla_status st = step(dq, dk, dv, dbeta, dg, dout, dws, arena_bytes - (size_t)(dws - a));
  if (st != GLA_OK) return st;
  if (cudaMemcpyAsync(out_h, dout, big, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GLA_ERR_CUDA;
  return GLA_OK;
}

gla_status forward_common(const void* q, const void* k, const void* v, const void* beta,
                          const void* g, int batch, int heads, int head_dim, int T, int H,
                          int W, float rope_theta, float eps, int dtype, void* out,
                          void* workspace, size_t workspace_bytes, void* stream, int path,
                          float* S_out, float* z_out, float* den_out, float* x_out,
                          void* const* events = nullptr,
                          unsigned long long stall_limit_ns = 0) {
  if (!dims_ok(batch, heads, head_dim, T, H, W)) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
  if (!(eps > 0.f) || !isfinite(eps) || !isfinite(rope_theta)) return GLA_ERR_INVALID_ARG;
  const void* ptrs[6] = {q, k, v, beta, g, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return GLA_ERR_INVALID_ARG;
  if (resolve_path(path, dtype, head_dim) < 0) return GLA_ERR_UNSUPPORTED;
  const WsLayout L = ws_layout(batch * heads, head_dim, true, T, H, W);
  if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < L.total)
    return GLA_ERR_WORKSPACE;
  Call c;
  c.g = make_geom(batch, heads, head_dim, T, H, W, 0, rope_theta, eps);
  const int sms = device_sm_count();
  if (sms <= 0) return GLA_ERR_CUDA;
  c.dtype = dtype; c.path = resolve_path(path, dtype, head_dim, &c.g, sms);
  c.q = q; c.k = k; c.v = v; c.beta = beta; c.gate = g; c.out = out;
  c.ws = static_cast<unsigned char*>(workspace);
  c.L = L;
  c.S = reinterpret_cast<float*>(c.ws + L.S);
  c.z = reinterpret_cast<float*>(c.ws + L.z);
  c.carry = false;
  c.stream = static_cast<cudaStream_t>(stream);
  c.S_dbg = S_out; c.z_dbg = z_out; c.den_dbg = den_out; c.x_dbg = x_out;
  c.events = events;
  c.stall_limit_ns = stall_limit_ns;
  return run_call(c);
}

}  // namespace

extern "C" {

int gla_version(void) { return 100; }

const char* gla_status_string(int status) {
  switch (status) {
    case GLA_OK: return "GLA_OK";
    case GLA_ERR_INVALID_ARG: return "GLA_ERR_INVALID_ARG: invalid argument";
    case GLA_ERR_UNSUPPORTED: return "GLA_ERR_UNSUPPORTED: unsupported configuration";
    case GLA_ERR_WORKSPACE: return "GLA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case GLA_ERR_CUDA: return "GLA_ERR_CUDA: CUDA runtime error";
    case GLA_ERR_TIMEOUT: return "GLA_ERR_TIMEOUT: a device-side wait timed out";
  }
  return "unknown gla_status";
}

size_t gla_forward_workspace_size(int batch, int heads, int head_dim, int T, int H, int W,
                                  int dtype) {
  if (!dims_ok(batch, heads, head_dim, T, H, W)) return 0;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return 0;
  return ws_layout(batch * heads, head_dim, true, T, H, W).total;
}

size_t gla_block_causal_workspace_size(int batch, int heads, int head_dim, int T_blk, int H,
                                       int W, int dtype) {
  if (!dims_ok(batch, heads, head_dim, T_blk, H, W)) return 0;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return 0;
  return ws_layout(batch * heads, head_dim, false, T_blk, H, W).total;
}

gla_status gla_forward(const void* q, const void* k, const void* v, const void* beta,
                       const void* g, int batch, int heads, int head_dim, int T, int H, int W,
                       float rope_theta, float eps, int dtype, void* out, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return forward_common(q, k, v, beta, g, batch, heads, head_dim, T, H, W, rope_theta, eps,
                        dtype, out, workspace, workspace_bytes, stream, GLA_PATH_AUTO,
                        nullptr, nullptr, nullptr, nullptr);
}

gla_status gla_forward_ex(const void* q, const void* k, const void* v, const void* beta,
                          const void* g, int batch, int heads, int head_dim, int T, int H,
                          int W, float rope_theta, float eps, int dtype, void* out,
                          void* workspace, size_t workspace_bytes, void* stream, int path) {
  return forward_common(q, k, v, beta, g, batch, heads, head_dim, T, H, W, rope_theta, eps,
                        dtype, out, workspace, workspace_bytes, stream, path, nullptr,
                        nullptr, nullptr, nullptr);
}

gla_status gla_forward_debug(const void* q, const void* k, const void* v, const void* beta,
                             const void* g, int batch, int heads, int head_dim, int T, int H,
                             int W, float rope_theta, float eps, int dtype, void* out,
                             void* workspace, size_t workspace_bytes, void* stream, int path,
                             float* S_out, float* z_out, float* den_out, float* x_out) {
  return forward_common(q, k, v, beta, g, batch, heads, head_dim, T, H, W, rope_theta, eps,
                        dtype, out, workspace, workspace_bytes, stream, path, S_out, z_out,
                        den_out, x_out);
}

gla_status gla_forward_timed(const void* q, const void* k, const void* v, const void* beta,
                             const void* g, int batch, int heads, int head_dim, int T, int H,
                             int W, float rope_theta, float eps, int dtype, void* out,
                             void* workspace, size_t workspace_bytes, void* stream, int path,
                             void* const* events) {
  return forward_common(q, k, v, beta, g, batch, heads, head_dim, T, H, W, rope_theta, eps,
                        dtype, out, workspace, workspace_bytes, stream, path, nullptr,
                        nullptr, nullptr, nullptr, events);
}

gla_status gla_block_causal_step_ex(float* state, float* z, const void* q, const void* k,
                                    const void* v, const void* beta, const void* g,
                                    int batch, int heads, int head_dim, int T_blk, int H,
                                    int W, int t0, float rope_theta, float eps, int dtype,
                                    void* out, void* workspace, size_t workspace_bytes,
                                    void* stream, int path) {
  if (!dims_ok(batch, heads, head_dim, T_blk, H, W) || t0 < 0) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
  if (!(eps > 0.f) || !isfinite(eps) || !isfinite(rope_theta)) return GLA_ERR_INVALID_ARG;
  const void* ptrs[8] = {state, z, q, k, v, beta, g, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return GLA_ERR_INVALID_ARG;
  if (resolve_path(path, dtype, head_dim) < 0) return GLA_ERR_UNSUPPORTED;
  const WsLayout L = ws_layout(batch * heads, head_dim, false, T_blk, H, W);
  if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < L.total)
    return GLA_ERR_WORKSPACE;
  Call c;
  c.g = make_geom(batch, heads, head_dim, T_blk, H, W, t0, rope_theta, eps);
  const int sms = device_sm_count();
  if (sms <= 0) return GLA_ERR_CUDA;
  c.dtype = dtype; c.path = resolve_path(path, dtype, head_dim, &c.g, sms);
  c.q = q; c.k = k; c.v = v; c.beta = beta; c.gate = g; c.out = out;
  c.ws = static_cast<unsigned char*>(workspace);
  c.L = L;
  c.S = state; c.z = z; c.carry = true;
  c.stream = static_cast<cudaStream_t>(stream);
  c.S_dbg = c.z_dbg = c.den_dbg = c.x_dbg = nullptr;
  c.events = nullptr;
  return run_call(c);
}

gla_status gla_block_causal_step(float* state, float* z, const void* q, const void* k,
                                 const void* v, const void* beta, const void* g, int batch,
                                 int heads, int head_dim, int T_blk, int H, int W, int t0,
                                 float rope_theta, float eps, int dtype, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return gla_block_causal_step_ex(state, z, q, k, v, beta, g, batch, heads, head_dim, T_blk,
                                  H, W, t0, rope_theta, eps, dtype, out, workspace,
                                  workspace_bytes, stream, GLA_PATH_AUTO);
}

size_t gla_causal_workspace_size(int batch, int heads, int head_dim, int T, int H, int W,
                                 int dtype) {
  if (!dims_ok(batch, heads, head_dim, T, H, W)) return 0;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return 0;
  return causal_ws(batch * heads, head_dim).total;
}

gla_status gla_causal_step_timed(float* state, float* z, const void* q, const void* k,
                                 const void* v, const void* beta, const void* g, int batch,
                                 int heads, int head_dim, int T, int H, int W, int t0,
                                 float rope_theta, float eps, int dtype, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream, int path,
                                 float* den_out, float* x_out, void* const* events) {
  if (!dims_ok(batch, heads, head_dim, T, H, W) || t0 < 0) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
  if (!(eps > 0.f) || !isfinite(eps) || !isfinite(rope_theta)) return GLA_ERR_INVALID_ARG;
  const void* ptrs[8] = {state, z, q, k, v, beta, g, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return GLA_ERR_INVALID_ARG;
  if (resolve_path(path, dtype, head_dim) < 0) return GLA_ERR_UNSUPPORTED;
  const Geom geom = make_geom(batch, heads, head_dim, T, H, W, t0, rope_theta, eps);
  const int sms = device_sm_count();
  if (sms <= 0) return GLA_ERR_CUDA;
  int used = resolve_path(path, dtype, head_dim);
  if (used == GLA_PATH_TENSOR && !causal_tensor_fits(geom, sms)) {
    if (path == GLA_PATH_TENSOR) return GLA_ERR_UNSUPPORTED;
    used = GLA_PATH_SIMT;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (used == GLA_PATH_SIMT && events && events[0] &&
      cudaEventRecord(static_cast<cudaEvent_t>(events[0]), st) != cudaSuccess)
    return GLA_ERR_CUDA;
  if (used == GLA_PATH_SIMT)
    return dtype == GLA_DTYPE_F32
               ? run_simt_causal_dim<float>(geom, q, k, v, beta, g, out, state, z, den_out, x_out, st)
               : run_simt_causal_dim<__nv_bfloat16>(geom, q, k, v, beta, g, out, state, z, den_out,
                                                    x_out, st);
  const CausalWs L = causal_ws(batch * heads, head_dim);
  if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < L.total)
    return GLA_ERR_WORKSPACE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  return run_causal_tensor(geom, q, k, v, beta, g, out, state, z,
                           reinterpret_cast<float*>(ws + L.part_S),
                           reinterpret_cast<float*>(ws + L.part_z),
                           reinterpret_cast<float*>(ws + L.S_start),
                           reinterpret_cast<float*>(ws + L.z_start), den_out, x_out, sms, st,
                           events);
}

gla_status gla_causal_step_ex(float* state, float* z, const void* q, const void* k,
                              const void* v, const void* beta, const void* g, int batch,
                              int heads, int head_dim, int T, int H, int W, int t0,
                              float rope_theta, float eps, int dtype, void* out,
                              void* workspace, size_t workspace_bytes, void* stream, int path,
                              float* den_out, float* x_out) {
  return gla_causal_step_timed(state, z, q, k, v, beta, g, batch, heads, head_dim, T, H, W, t0,
                               rope_theta, eps, dtype, out, workspace, workspace_bytes, stream,
                               path, den_out, x_out, nullptr);
}

gla_status gla_causal_step(float* state, float* z, const void* q, const void* k, const void* v,
                           const void* beta, const void* g, int batch, int heads, int head_dim,
                           int T, int H, int W, int t0, float rope_theta, float eps, int dtype,
                           void* out, void* workspace, size_t workspace_bytes, void* stream) {
  return gla_causal_step_ex(state, z, q, k, v, beta, g, batch, heads, head_dim, T, H, W, t0,
                            rope_theta, eps, dtype, out, workspace, workspace_bytes, stream,
                            GLA_PATH_AUTO, nullptr, nullptr);
}

size_t gla_forward_mx_workspace_size(int batch, int heads, int head_dim, int T, int H, int W,
                                     int path) {
  if (!dims_ok(batch, heads, head_dim, T, H, W) || head_dim != 128) return 0;
  const size_t ws = ws_layout(batch * heads, head_dim, true, T, H, W).total;
  if (path != GLA_PATH_SIMT) return ws;
  // The CUDA-core path decodes q, k, v and g to bf16 first.
  const size_t n = (size_t)batch * T * H * W * heads * head_dim;
  return 4 * align_up(n * 2, kAlign) + ws;
}

gla_status gla_forward_mx_ex(const void* q, const void* q_scale, const void* k,
                             const void* k_scale, const void* v, const void* v_scale,
                             const void* beta, const void* g, const void* g_scale, int batch,
                             int heads, int head_dim, int T, int H, int W, float rope_theta,
                             float eps, void* out, void* workspace, size_t workspace_bytes,
                             void* stream, int path, float* S_out, float* z_out,
                             float* den_out, float* x_out, void* const* events) {
  if (!dims_ok(batch, heads, head_dim, T, H, W)) return GLA_ERR_INVALID_ARG;
  if (head_dim != 128) return GLA_ERR_UNSUPPORTED;
  if (!(eps > 0.f) || !isfinite(eps) || !isfinite(rope_theta)) return GLA_ERR_INVALID_ARG;
  const void* ptrs[10] = {q, q_scale, k, k_scale, v, v_scale, beta, g, g_scale, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return GLA_ERR_INVALID_ARG;
  if (path != GLA_PATH_AUTO && path != GLA_PATH_SIMT && path != GLA_PATH_TENSOR)
    return GLA_ERR_UNSUPPORTED;
  const size_t need = gla_forward_mx_workspace_size(batch, heads, head_dim, T, H, W, path);
  if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < need)
    return GLA_ERR_WORKSPACE;
  const Geom geom = make_geom(batch, heads, head_dim, T, H, W, 0, rope_theta, eps);
  const int sms = device_sm_count();
  if (sms <= 0) return GLA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (path == GLA_PATH_SIMT) {
    // Decode to bf16 (exact: E4M3 values times powers of two), then the
    // bf16 CUDA-core kernels.
    const size_t n = (size_t)batch * T * H * W * heads * head_dim;
    const void* codes[4] = {q, k, v, g};
    const void* scales[4] = {q_scale, k_scale, v_scale, g_scale};
    unsigned char* dec[4];
    for (int i = 0; i < 4; ++i) {
      dec[i] = ws + i * align_up(n * 2, kAlign);
      mx_decode_kernel<<<4 * sms, 256, 0, st>>>(static_cast<const uint8_t*>(codes[i]),
                                                static_cast<const uint8_t*>(scales[i]),
                                                reinterpret_cast<__nv_bfloat16*>(dec[i]), n);
      if (cudaGetLastError() != cudaSuccess) return GLA_ERR_CUDA;
    }
    unsigned char* rest = ws + 4 * align_up(n * 2, kAlign);
    return forward_common(dec[0], dec[1], dec[2], beta, dec[3], batch, heads, head_dim, T, H, W,
                          rope_theta, eps, GLA_DTYPE_BF16, out, rest,
                          workspace_bytes - (size_t)(rest - ws), stream, GLA_PATH_SIMT, S_out,
                          z_out, den_out, x_out, events);
  }
  const WsLayout L = ws_layout(batch * heads, head_dim, true, T, H, W);
  MxInputs in = {q, q_scale, k, k_scale, v, v_scale, g, g_scale};
  float* S = reinterpret_cast<float*>(ws + L.S);
  float* z = reinterpret_cast<float*>(ws + L.z);
  gla_status r = run_tensor_mx(geom, in, beta, out, S, z, S_out != nullptr,
                               reinterpret_cast<float*>(ws + L.part_S),
                               reinterpret_cast<float*>(ws + L.part_z),
                               reinterpret_cast<__half*>(ws + L.S_img),
                               reinterpret_cast<float*>(ws + L.S_scale),
                               reinterpret_cast<float2*>(ws + L.rope_tab), den_out, x_out, sms, st,
                               events);
  if (r == GLA_ERR_UNSUPPORTED && path == GLA_PATH_AUTO)
    return gla_forward_mx_ex(q, q_scale, k, k_scale, v, v_scale, beta, g, g_scale, batch, heads,
                             head_dim, T, H, W, rope_theta, eps, out, workspace, workspace_bytes,
                             stream, GLA_PATH_SIMT, S_out, z_out, den_out, x_out, events);
  if (r != GLA_OK) return r;
  const size_t dd = (size_t)batch * heads * head_dim * head_dim;
  const size_t dz = (size_t)batch * heads * head_dim;
  if (S_out && cudaMemcpyAsync(S_out, S, dd * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return GLA_ERR_CUDA;
  if (z_out && cudaMemcpyAsync(z_out, z, dz * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return GLA_ERR_CUDA;
  return GLA_OK;
}

gla_status gla_forward_mx(const void* q, const void* q_scale, const void* k, const void* k_scale,
                          const void* v, const void* v_scale, const void* beta, const void* g,
                          const void* g_scale, int batch, int heads, int head_dim, int T, int H,
                          int W, float rope_theta, float eps, void* out, void* workspace,
                          size_t workspace_bytes, void* stream) {
  return gla_forward_mx_ex(q, q_scale, k, k_scale, v, v_scale, beta, g, g_scale, batch, heads,
                           head_dim, T, H, W, rope_theta, eps, out, workspace, workspace_bytes,
                           stream, GLA_PATH_AUTO, nullptr, nullptr, nullptr, nullptr, nullptr);
}

gla_status gla_gemm_bf16(const void* A, const void* B, void* C, int M, int N, int K,
                         void* stream) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 8 || N % 8) return GLA_ERR_INVALID_ARG;
  if (!A || !B || !C || !aligned16(A) || !aligned16(B) || !aligned16(C)) return GLA_ERR_INVALID_ARG;
  GemmParams p = {};
  p.M = M; p.N = N; p.K = K; p.mode = kGemmPlain;
  p.C = static_cast<__nv_bfloat16*>(C);
  return run_gemm(A, B, p, device_sm_count(), static_cast<cudaStream_t>(stream));
}

gla_status gla_project_in(const void* x, const void* W_in, int tokens, int C, int heads,
                          int head_dim, void* q, void* k, void* v, void* g, void* beta,
                          void* stream) {
  if (tokens <= 0 || C <= 0 || C % 8 || heads <= 0 || head_dim <= 0) return GLA_ERR_INVALID_ARG;
  const int HD = heads * head_dim;
  if (HD % 32) return GLA_ERR_UNSUPPORTED;
  const void* ptrs[8] = {x, W_in, q, k, v, g, beta, nullptr};
  for (int i = 0; i < 7; ++i)
    if (!ptrs[i] || !aligned16(ptrs[i])) return GLA_ERR_INVALID_ARG;
  GemmParams p = {};
  p.M = tokens; p.N = 4 * HD + heads; p.K = C; p.mode = kGemmSplit;
  p.dst[0] = static_cast<__nv_bfloat16*>(q);
  p.dst[1] = static_cast<__nv_bfloat16*>(k);
  p.dst[2] = static_cast<__nv_bfloat16*>(v);
  p.dst[3] = static_cast<__nv_bfloat16*>(g);
  p.beta = static_cast<__nv_bfloat16*>(beta);
  p.HD = HD; p.heads = heads;
  return run_gemm(x, W_in, p, device_sm_count(), static_cast<cudaStream_t>(stream));
}

// Layer workspace: q, k, v, g, the operator's output (tokens x HD bf16 each),
// beta (tokens x heads bf16), then the operator's own workspace.
size_t gla_layer_workspace_size(int batch, int heads, int head_dim, int T, int H, int W) {
  const size_t op = gla_forward_workspace_size(batch, heads, head_dim, T, H, W, GLA_DTYPE_BF16);
  if (!op) return 0;
  const size_t th = (size_t)batch * T * H * W * heads;
  return 5 * align_up(th * head_dim * 2, kAlign) + align_up(th * 2, kAlign) + op;
}

gla_status gla_layer_forward(const void* x, const void* W_in, const void* W_o, int batch, int C,
                             int C_out, int heads, int head_dim, int T, int H, int W,
                             float rope_theta, float eps, void* y, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!dims_ok(batch, heads, head_dim, T, H, W) || C <= 0 || C_out <= 0) return GLA_ERR_INVALID_ARG;
  if (C % 8 || C_out % 8 || (heads * head_dim) % 32) return GLA_ERR_UNSUPPORTED;
  if (!x || !W_in || !W_o || !y || !aligned16(x) || !aligned16(W_in) || !aligned16(W_o) ||
      !aligned16(y))
    return GLA_ERR_INVALID_ARG;
  const size_t need = gla_layer_workspace_size(batch, heads, head_dim, T, H, W);
  if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < need)
    return GLA_ERR_WORKSPACE;
  const int tokens = batch * T * H * W;
  const size_t th = (size_t)tokens * heads;
  const size_t big = align_up(th * head_dim * 2, kAlign);
  unsigned char* w = static_cast<unsigned char*>(workspace);
  unsigned char *q = w, *k = q + big, *v = k + big, *g = v + big, *o = g + big, *beta = o + big;
  unsigned char* ows = beta + align_up(th * 2, kAlign);
  gla_status st = gla_project_in(x, W_in, tokens, C, heads, head_dim, q, k, v, g, beta, stream);
  if (st != GLA_OK) return st;
  st = gla_forward(q, k, v, beta, g, batch, heads, head_dim, T, H, W, rope_theta, eps,
                   GLA_DTYPE_BF16, o, ows, workspace_bytes - (size_t)(ows - w), stream);
  if (st != GLA_OK) return st;
  return gla_gemm_bf16(o, W_o, y, tokens, C_out, heads * head_dim, stream);
}

// Anchor workspace: q_til and k_til, fp16, the inputs' layout.
size_t gla_softmax_anchor_workspace_size(int batch, int heads, int head_dim, int T, int H,
                                         int W) {
  if (!dims_ok(batch, heads, head_dim, T, H, W) || head_dim != 128) return 0;
  const size_t th = (size_t)batch * T * H * W * heads;
  return 2 * align_up(th * head_dim * 2, kAlign);
}

gla_status gla_softmax_anchor_timed(const void* q, const void* k, const void* v, const void* g,
                                    int batch, int heads, int head_dim, int T, int H, int W,
                                    float rope_theta, void* out, void* workspace,
                                    size_t workspace_bytes, void* stream, void* const* events) {
  if (!dims_ok(batch, heads, head_dim, T, H, W)) return GLA_ERR_INVALID_ARG;
  if (head_dim != 128 || (long long)batch * heads > 65535) return GLA_ERR_UNSUPPORTED;
  if (!isfinite(rope_theta)) return GLA_ERR_INVALID_ARG;
  const void* ptrs[5] = {q, k, v, g, out};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return GLA_ERR_INVALID_ARG;
  const size_t need = gla_softmax_anchor_workspace_size(batch, heads, head_dim, T, H, W);
  if (!workspace || ((uintptr_t)workspace % kAlign) != 0 || workspace_bytes < need)
    return GLA_ERR_WORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return GLA_ERR_CUDA;
  const Geom geom = make_geom(batch, heads, head_dim, T, H, W, 0, rope_theta, 1e-6f);
  __half* qt = static_cast<__half*>(workspace);
  __half* kt = reinterpret_cast<__half*>(static_cast<unsigned char*>(workspace) + need / 2);
  return run_anchor(geom, q, k, v, g, out, qt, kt, sms, static_cast<cudaStream_t>(stream),
                    events);
}

gla_status gla_softmax_anchor(const void* q, const void* k, const void* v, const void* g,
                              int batch, int heads, int head_dim, int T, int H, int W,
                              float rope_theta, void* out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return gla_softmax_anchor_timed(q, k, v, g, batch, heads, head_dim, T, H, W, rope_theta, out,
                                  workspace, workspace_bytes, stream, nullptr);
}

size_t gla_forward_host_arena_size(int batch, int heads, int head_dim, int T, int H, int W,
                                   int dtype) {
  const size_t ws = gla_forward_workspace_size(batch, heads, head_dim, T, H, W, dtype);
  if (!ws) return 0;
  const size_t esz = dtype == GLA_DTYPE_F32 ? 4 : 2;
  const size_t th = (size_t)batch * T * H * W * heads;
  // beta: room for each batch group's slice to start on a 16-byte boundary.
  return 5 * align_up(th * head_dim * esz, kAlign) +
         align_up(th * esz + 16 * (kHostChunks + 1), kAlign) + ws;
}

gla_status gla_forward_host(const void* q_h, const void* k_h, const void* v_h,
                            const void* beta_h, const void* g_h, int batch, int heads,
                            int head_dim, int T, int H, int W, float rope_theta, float eps,
                            int dtype, void* out_h, void* arena, size_t arena_bytes,
                            void* stream) {
  const size_t need = gla_forward_host_arena_size(batch, heads, head_dim, T, H, W, dtype);
  if (!need) return GLA_ERR_INVALID_ARG;
  const void* hp[6] = {q_h, k_h, v_h, beta_h, g_h, out_h};
  for (const void* p : hp)
    if (!p) return GLA_ERR_INVALID_ARG;
  if (!arena || ((uintptr_t)arena % kAlign) != 0 || arena_bytes < need) return GLA_ERR_WORKSPACE;
  const size_t esz = dtype == GLA_DTYPE_F32 ? 4 : 2;
  const size_t th = (size_t)batch * T * H * W * heads;
  const size_t big = th * head_dim * esz, small = th * esz;
  unsigned char* a = static_cast<unsigned char*>(arena);
  unsigned char* dq = a;
  unsigned char* dk = dq + align_up(big, kAlign);
  unsigned char* dv = dk + align_up(big, kAlign);
  unsigned char* dg = dv + align_up(big, kAlign);
  unsigned char* dout = dg + align_up(big, kAlign);
  unsigned char* dbeta = dout + align_up(big, kAlign);
  unsigned char* dws = dbeta + align_up(small + 16 * (kHostChunks + 1), kAlign);
  const size_t ws_bytes = arena_bytes - (size_t)(dws - a);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned char* hq = static_cast<const unsigned char*>(q_h);
  const unsigned char* hk = static_cast<const unsigned char*>(k_h);
  const unsigned char* hv = static_cast<const unsigned char*>(v_h);
  const unsigned char* hg = static_cast<const unsigned char*>(g_h);
  const unsigned char* hb = static_cast<const unsigned char*>(beta_h);
  unsigned char* ho = static_cast<unsigned char*>(out_h);

  // Batch elements are independent and contiguous: with two or more, the
  // call runs per group of them, and each group's output copy goes out on a
  // helper stream while the next group's inputs come in (PCIe carries both
  // directions at once).  The helper is joined back into `stream` before
  // the call returns, so `stream` orders everything as before.
  HostPipe* pipe = batch >= 2 ? host_pipe() : nullptr;
  const int chunks = pipe ? (batch < kHostChunks ? batch : kHostChunks) : 1;
  std::unique_lock<std::mutex> lock;
  if (pipe) lock = std::unique_lock<std::mutex>(pipe->mu);
  bool forked = false;
  gla_status st = GLA_OK;
  for (int c = 0; c < chunks && st == GLA_OK; ++c) {
    const int b0 = (int)((long long)batch * c / chunks), b1 = (int)((long long)batch * (c + 1) / chunks);
    const size_t ob = big / batch * b0, nb = big / batch * (b1 - b0);
    const size_t os = small / batch * b0, ns = small / batch * (b1 - b0);
    // The group's beta slice starts on a 16-byte boundary in the arena (the
    // operator's pointers must be 16-byte aligned); slices stay disjoint.
    const size_t od = align_up(os, 16) + 16 * (size_t)c;
    if (cudaMemcpyAsync(dq + ob, hq + ob, nb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dk + ob, hk + ob, nb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dv + ob, hv + ob, nb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dg + ob, hg + ob, nb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(dbeta + od, hb + os, ns, cudaMemcpyHostToDevice, s) != cudaSuccess) {
      st = GLA_ERR_CUDA;
      break;
    }
    st = gla_forward(dq + ob, dk + ob, dv + ob, dbeta + od, dg + ob, b1 - b0, heads, head_dim,
                     T, H, W, rope_theta, eps, dtype, dout + ob, dws, ws_bytes, stream);
    if (st != GLA_OK) break;
    if (!pipe) {
      if (cudaMemcpyAsync(ho + ob, dout + ob, nb, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        st = GLA_ERR_CUDA;
      break;
    }
    if (cudaEventRecord(pipe->ev[c], s) != cudaSuccess ||
        cudaStreamWaitEvent(pipe->s, pipe->ev[c], 0) != cudaSuccess) {
      st = GLA_ERR_CUDA;
      break;
    }
    forked = true;
    if (cudaMemcpyAsync(ho + ob, dout + ob, nb, cudaMemcpyDeviceToHost, pipe->s) != cudaSuccess)
      st = GLA_ERR_CUDA;
  }
  if (forked) {
    // Join, also after an error, so that no copy of this call outlives it
    // unordered with `stream`.
    if (cudaEventRecord(pipe->ev[kHostChunks], pipe->s) != cudaSuccess ||
        cudaStreamWaitEvent(s, pipe->ev[kHostChunks], 0) != cudaSuccess)
      st = GLA_ERR_CUDA;
  }
  return st;
}

size_t gla_block_causal_host_arena_size(int batch, int heads, int head_dim, int T_blk, int H,
                                        int W, int dtype) {
  const size_t ws = gla_block_causal_workspace_size(batch, heads, head_dim, T_blk, H, W, dtype);
  if (!ws) return 0;
  return staged_inputs_bytes(batch, heads, head_dim, T_blk, H, W, dtype) + ws;
}

gla_status gla_block_causal_step_host(float* state, float* z, const void* q_h, const void* k_h,
                                      const void* v_h, const void* beta_h, const void* g_h,
                                      int batch, int heads, int head_dim, int T_blk, int H,
                                      int W, int t0, float rope_theta, float eps, int dtype,
                                      void* out_h, void* arena, size_t arena_bytes,
                                      void* stream) {
  const size_t need =
      gla_block_causal_host_arena_size(batch, heads, head_dim, T_blk, H, W, dtype);
  if (!need) return GLA_ERR_INVALID_ARG;
  return staged_step(
      q_h, k_h, v_h, beta_h, g_h, out_h, batch, heads, head_dim, T_blk, H, W, dtype, arena,
      arena_bytes, need, stream,
      [&](const void* dq, const void* dk, const void* dv, const void* db, const void* dg,
          void* dout, void* dws, size_t ws_bytes) {
        return gla_block_causal_step(state, z, dq, dk, dv, db, dg, batch, heads, head_dim,
                                     T_blk, H, W, t0, rope_theta, eps, dtype, dout, dws,
                                     ws_bytes, stream);
      });
}

size_t gla_causal_host_arena_size(int batch, int heads, int head_dim, int T, int H, int W,
                                  int dtype) {
  const size_t ws = gla_causal_workspace_size(batch, heads, head_dim, T, H, W, dtype);
  if (!ws) return 0;
  return staged_inputs_bytes(batch, heads, head_dim, T, H, W, dtype) + ws;
}

gla_status gla_causal_step_host(float* state, float* z, const void* q_h, const void* k_h,
                                const void* v_h, const void* beta_h, const void* g_h, int batch,
                                int heads, int head_dim, int T, int H, int W, int t0,
                                float rope_theta, float eps, int dtype, void* out_h,
                                void* arena, size_t arena_bytes, void* stream) {
  const size_t need = gla_causal_host_arena_size(batch, heads, head_dim, T, H, W, dtype);
  if (!need) return GLA_ERR_INVALID_ARG;
  return staged_step(
      q_h, k_h, v_h, beta_h, g_h, out_h, batch, heads, head_dim, T, H, W, dtype, arena,
      arena_bytes, need, stream,
      [&](const void* dq, const void* dk, const void* dv, const void* db, const void* dg,
          void* dout, void* dws, size_t ws_bytes) {
        return gla_causal_step(state, z, dq, dk, dv, db, dg, batch, heads, head_dim, T, H, W,
                               t0, rope_theta, eps, dtype, dout, dws, ws_bytes, stream);
      });
}

// ---------------------------------------------------------------------------
// Allocation-free entry point.  The scratch lives in a file-scope device array;
// host code only ever uses its device address, looked up once per device.

}  // extern "C"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GLA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device (0 on failure).
// The per-device cache is filled under a mutex: host threads that make their
// first call at the same time look the address up once.
unsigned char* noalloc_scratch() {
  static std::mutex mu;
  static unsigned char* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    addr[dev] = static_cast<unsigned char*>(p);
  }
  return addr[dev];
}

// Scratch layout sized for the grid this GPU actually runs (at most `grid`
// state CTAs, `zparts` z partials per slot) rather than the worst case.  The
// fp16 image of S, its scale and the whole-call RoPE table are read by the
// tensor read-out only, so the CUDA-core path reserves no room for them.
WsLayout noalloc_layout(int BH, int d, int grid, int zparts, int T, int H, int W, bool tensor) {
  WsLayout L;
  L.slots = grid + BH;
  size_t off = 0;
  L.part_S = off; off = align_up(off + (size_t)L.slots * d * d * 4, kAlign);
  L.part_z = off; off = align_up(off + (size_t)L.slots * zparts * d * 4, kAlign);
  L.S = off; off = align_up(off + (size_t)BH * d * d * 4, kAlign);
  L.z = off; off = align_up(off + (size_t)BH * d * 4, kAlign);
  L.S_img = off;
  if (tensor) off = align_up(off + (size_t)BH * d * d * 2, kAlign);
  L.S_scale = off;
  if (tensor) off = align_up(off + (size_t)BH * 4 * 4, kAlign);
  L.rope_tab = off;
  if (tensor) off = align_up(off + rope_tab_bytes(d, T, H, W), kAlign);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

gla_status gla_forward_noalloc(const void* q, const void* k, const void* v, const void* beta,
                               const void* g, int batch, int heads, int head_dim, int T, int H,
                               int W, float rope_theta, float eps, int dtype, void* out,
                               void* stream) {
  if (!dims_ok(batch, heads, head_dim, T, H, W)) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
  if (!(eps > 0.f) || !isfinite(eps) || !isfinite(rope_theta)) return GLA_ERR_INVALID_ARG;
  const void* ptrs[6] = {q, k, v, beta, g, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return GLA_ERR_INVALID_ARG;
  Call c;
  c.g = make_geom(batch, heads, head_dim, T, H, W, 0, rope_theta, eps);
  const int sms = device_sm_count();
  if (sms <= 0) return GLA_ERR_CUDA;
  c.dtype = dtype;
  c.path = resolve_path(GLA_PATH_AUTO, dtype, head_dim, &c.g, sms);
  const bool tensor = c.path == GLA_PATH_TENSOR;
  const Partition part = tensor ? tc_state_partition(c.g, sms)
                                : make_partition(batch * heads, c.g.N, kSimtTile, 2 * sms);
  const WsLayout L =
      noalloc_layout(batch * heads, head_dim, part.grid, tensor ? kStTW : 1, T, H, W, tensor);
  if (L.total > GLA_NOALLOC_SCRATCH_BYTES) return GLA_ERR_WORKSPACE;
  unsigned char* scratch = noalloc_scratch();
  if (!scratch) return GLA_ERR_CUDA;
  c.q = q; c.k = k; c.v = v; c.beta = beta; c.gate = g; c.out = out;
  c.ws = scratch;
  c.L = L;
  c.S = reinterpret_cast<float*>(c.ws + L.S);
  c.z = reinterpret_cast<float*>(c.ws + L.z);
  c.carry = false;
  c.stream = static_cast<cudaStream_t>(stream);
  c.S_dbg = c.z_dbg = c.den_dbg = c.x_dbg = nullptr;
  c.events = nullptr;
  return run_call(c);
}

gla_status gla_selftest_pipeline_stall(const void* q, const void* k, const void* v,
                                       const void* beta, const void* g, int batch, int heads,
                                       int head_dim, int T, int H, int W, float rope_theta,
                                       float eps, void* out, void* workspace,
                                       size_t workspace_bytes, unsigned int limit_us,
                                       void* stream) {
  if (limit_us < 1 || limit_us > 1000000u) return GLA_ERR_INVALID_ARG;
  return forward_common(q, k, v, beta, g, batch, heads, head_dim, T, H, W, rope_theta, eps,
                        GLA_DTYPE_BF16, out, workspace, workspace_bytes, stream, GLA_PATH_TENSOR,
                        nullptr, nullptr, nullptr, nullptr, nullptr,
                        (unsigned long long)limit_us * 1000ull);
}

gla_status gla_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000u) return GLA_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

gla_status gla_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GLA_ERR_CUDA;
  unsigned int w = 0;
  if (cudaMemcpyFromSymbol(&w, g_device_error, sizeof(w)) != cudaSuccess) return GLA_ERR_CUDA;
  if (w) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
      return GLA_ERR_CUDA;
    return GLA_ERR_TIMEOUT;
  }
  return GLA_OK;
}

gla_status gla_plan(int batch, int heads, int head_dim, int T, int H, int W, int dtype,
                    int path, int num_sms, int* grid, int* tile_tokens, int* path_used) {
  if (!dims_ok(batch, heads, head_dim, T, H, W) || num_sms <= 0) return GLA_ERR_INVALID_ARG;
  if (dtype != GLA_DTYPE_F32 && dtype != GLA_DTYPE_BF16) return GLA_ERR_INVALID_ARG;
  if (!grid || !tile_tokens || !path_used) return GLA_ERR_INVALID_ARG;
  const Geom g = make_geom(batch, heads, head_dim, T, H, W, 0, 10000.f, 1e-6f);
  const int resolved = resolve_path(path, dtype, head_dim, &g, num_sms);
  if (resolved < 0) return GLA_ERR_UNSUPPORTED;
  const int N = T * H * W;
  (void)N;
  Partition p = resolved == GLA_PATH_TENSOR
                    ? tc_state_partition(g, num_sms)
                    : make_partition(batch * heads, N, kSimtTile, 2 * num_sms);
  *grid = p.grid;
  *tile_tokens = p.tile;
  *path_used = resolved;
  return GLA_OK;
}

gla_status gla_check_rope_copy(int batch, int heads, int head_dim, int T, int H, int W,
                               int num_sms) {
  if (!dims_ok(batch, heads, head_dim, T, H, W) || num_sms <= 0) return GLA_ERR_INVALID_ARG;
  const Geom g = make_geom(batch, heads, head_dim, T, H, W, 0, 10000.f, 1e-6f);
  if (!tc_rope_lanes_ok(g)) return GLA_ERR_UNSUPPORTED;
  const Partition p = tc_apply_partition(g, num_sms);
  const RopeLayout G = rope_layout(g, g.T);
  const int smem_entries = tc_table_entries(g, p);
  const int P = g.pt + g.ph + g.pw;
  for (int c = 0; c < p.grid; ++c) {
    const RopeWindow win = rope_window(g, p, part_begin(p, c), part_begin(p, c + 1) - 1);
    const RopeLayout L = rope_layout(g, win.Lt);
    const RopeCopy rc = rope_copy_plan(g, win);
    if (rc.n < 3 || rc.n > 4 || L.entries > smem_entries) return GLA_ERR_INVALID_ARG;
    for (int i = 0; i < rc.n; ++i) {
      // Bulk copies: 16-byte aligned addresses and sizes (entries are 8 bytes;
      // the plan promises multiples of 8 entries).
      if (rc.src[i] % 8 || rc.dst[i] % 8 || rc.len[i] % 8 || rc.len[i] <= 0) return GLA_ERR_INVALID_ARG;
      if (rc.src[i] + rc.len[i] > G.entries || rc.dst[i] + rc.len[i] > L.entries)
        return GLA_ERR_INVALID_ARG;
    }
    // Every entry the read-out looks up comes from the whole-call entry of
    // the same pair at the same absolute position.
    for (int pr = 0; pr < P; ++pr) {
      const int a = pr < g.pt ? 0 : (pr < g.pt + g.ph ? 1 : 2);
      const int rows = a == 0 ? win.Lt : (a == 1 ? g.H : g.W);
      for (int pos = 0; pos < rows; ++pos) {
        const int e = L.base[a] + pos * L.stride[a] + rope_idx(L, a, pr);
        int gp = pos;
        if (a == 0) {
          gp = win.t_lo + pos;
          if (gp >= g.T) gp -= g.T;
        }
        const int ge = G.base[a] + gp * G.stride[a] + rope_idx(G, a, pr);
        int src = -1;
        for (int i = 0; i < rc.n; ++i)
          if (e >= rc.dst[i] && e < rc.dst[i] + rc.len[i]) src = rc.src[i] + (e - rc.dst[i]);
        if (src != ge) return GLA_ERR_INVALID_ARG;
      }
    }
  }
  return GLA_OK;
}

}  // extern "C"
