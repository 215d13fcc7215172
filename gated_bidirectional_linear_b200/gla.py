"""ctypes binding of libgla.so (include/gla.h).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  Tensors are torch tensors (device memory for the device entry
points, host memory for gla_forward_host); the binding passes their data
pointers, sizes and the current CUDA stream.  A missing or unloadable library
raises immediately: there is no fallback.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgla.so")

GLA_OK, GLA_ERR_INVALID_ARG, GLA_ERR_UNSUPPORTED, GLA_ERR_WORKSPACE, GLA_ERR_CUDA, \
    GLA_ERR_TIMEOUT = range(6)
GLA_DTYPE_F32, GLA_DTYPE_BF16 = 0, 1
GLA_PATH_AUTO, GLA_PATH_SIMT, GLA_PATH_TENSOR = 0, 1, 2

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_fp = ctypes.POINTER(ctypes.c_float)

_SIGS = {
    "gla_version": (_i, []),
    "gla_status_string": (ctypes.c_char_p, [_i]),
    "gla_forward_workspace_size": (_sz, [_i] * 7),
    "gla_block_causal_workspace_size": (_sz, [_i] * 7),
    "gla_forward_host_arena_size": (_sz, [_i] * 7),
    "gla_forward": (_i, [_vp] * 5 + [_i] * 6 + [_f, _f, _i, _vp, _vp, _sz, _vp]),
    "gla_forward_ex": (_i, [_vp] * 5 + [_i] * 6 + [_f, _f, _i, _vp, _vp, _sz, _vp, _i]),
    "gla_forward_debug": (_i, [_vp] * 5 + [_i] * 6 + [_f, _f, _i, _vp, _vp, _sz, _vp, _i]
                          + [_vp] * 4),
    "gla_forward_timed": (_i, [_vp] * 5 + [_i] * 6 + [_f, _f, _i, _vp, _vp, _sz, _vp, _i,
                                                        ctypes.POINTER(_vp)]),
    "gla_block_causal_step": (_i, [_vp] * 7 + [_i] * 7 + [_f, _f, _i, _vp, _vp, _sz, _vp]),
    "gla_block_causal_step_ex": (_i, [_vp] * 7 + [_i] * 7
                                 + [_f, _f, _i, _vp, _vp, _sz, _vp, _i]),
    "gla_forward_host": (_i, [_vp] * 5 + [_i] * 6 + [_f, _f, _i, _vp, _vp, _sz, _vp]),
    "gla_block_causal_host_arena_size": (_sz, [_i] * 7),
    "gla_block_causal_step_host": (_i, [_vp] * 7 + [_i] * 7 + [_f, _f, _i, _vp, _vp, _sz, _vp]),
    "gla_causal_workspace_size": (_sz, [_i] * 7),
    "gla_causal_step": (_i, [_vp] * 7 + [_i] * 7 + [_f, _f, _i, _vp, _vp, _sz, _vp]),
    "gla_causal_step_ex": (_i, [_vp] * 7 + [_i] * 7 + [_f, _f, _i, _vp, _vp, _sz, _vp, _i]
                           + [_vp] * 2),
    "gla_causal_step_timed": (_i, [_vp] * 7 + [_i] * 7 + [_f, _f, _i, _vp, _vp, _sz, _vp, _i]
                              + [_vp] * 2 + [ctypes.POINTER(_vp)]),
    "gla_causal_host_arena_size": (_sz, [_i] * 7),
    "gla_causal_step_host": (_i, [_vp] * 7 + [_i] * 7 + [_f, _f, _i, _vp, _vp, _sz, _vp]),
    "gla_forward_mx_workspace_size": (_sz, [_i] * 7),
    "gla_forward_mx": (_i, [_vp] * 9 + [_i] * 6 + [_f, _f, _vp, _vp, _sz, _vp]),
    "gla_forward_mx_ex": (_i, [_vp] * 9 + [_i] * 6 + [_f, _f, _vp, _vp, _sz, _vp, _i]
                          + [_vp] * 4 + [ctypes.POINTER(_vp)]),
    "gla_gemm_bf16": (_i, [_vp] * 3 + [_i] * 3 + [_vp]),
    "gla_project_in": (_i, [_vp] * 2 + [_i] * 4 + [_vp] * 6),
    "gla_layer_workspace_size": (_sz, [_i] * 6),
    "gla_layer_forward": (_i, [_vp] * 3 + [_i] * 8 + [_f, _f, _vp, _vp, _sz, _vp]),
    "gla_softmax_anchor_workspace_size": (_sz, [_i] * 6),
    "gla_softmax_anchor": (_i, [_vp] * 4 + [_i] * 6 + [_f, _vp, _vp, _sz, _vp]),
    "gla_softmax_anchor_timed": (_i, [_vp] * 4 + [_i] * 6 + [_f, _vp, _vp, _sz, _vp,
                                                          ctypes.POINTER(_vp)]),
    "gla_forward_noalloc": (_i, [_vp] * 5 + [_i] * 6 + [_f, _f, _i, _vp, _vp]),
    "gla_get_device_status": (_i, [_vp]),
    "gla_selftest_wait_timeout": (_i, [ctypes.c_uint, _vp]),
    "gla_selftest_pipeline_stall": (_i, [_vp] * 5 + [_i] * 6 + [_f, _f, _vp, _vp, _sz,
                                                               ctypes.c_uint, _vp]),
    "gla_plan": (_i, [_i] * 9 + [ctypes.POINTER(_i)] * 3),
    "gla_check_rope_copy": (_i, [_i] * 7),
}

_lib = None


class GlaError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def lib():
    """The loaded libgla.so (raises OSError if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"libgla.so not built ({LIB_PATH}); run "
                          "python -m gated_bidirectional_linear_b200.build")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status):
    return lib().gla_status_string(int(status)).decode()


def _check(status, what):
    if status != GLA_OK:
        raise GlaError(status, what)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return GLA_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return GLA_DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, dev=None):
    """The cudaStream_t of `stream` (default: the current stream of `dev`).
    The library launches on the current device, so a stream of another
    device than the tensors' is refused here."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif dev is not None and stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, the tensors on {dev}")
    return ctypes.c_void_p(stream.cuda_stream)


def _on(dev):
    """Make `dev` the current device for one library call: the C side looks
    up the SM count, the built-in scratch and its helper stream on the
    current device, and launches there."""
    return torch.cuda.device(dev)


def _dims(q, T, H, W):
    if q.dim() != 4:
        raise ValueError(f"q must be [B, N, heads, head_dim], got {tuple(q.shape)}")
    B, N, Hh, d = q.shape
    if N != T * H * W:
        raise ValueError(f"q has {N} tokens, grid {T}x{H}x{W} has {T * H * W}")
    return B, Hh, d


def _validate(q, k, v, beta, g, out, cuda=True, **extra):
    """The library sees raw pointers only: check here what it cannot, i.e.
    that every tensor has the layout and dtype the C ABI documents, is
    contiguous and lives on one device (a GPU for the device entry points,
    the host for gla_forward_host).  extra: name -> (tensor, shape, dtype)."""
    dev = q.device
    if cuda != (dev.type == "cuda"):
        raise ValueError(f"q is on {dev}; this entry point takes "
                         f"{'GPU' if cuda else 'host'} tensors")
    checks = {"q": (q, q.shape, q.dtype), "k": (k, q.shape, q.dtype), "v": (v, q.shape, q.dtype),
              "g": (g, q.shape, q.dtype), "beta": (beta, q.shape[:3], q.dtype),
              "out": (out, q.shape, q.dtype)}
    checks.update(extra)
    for name, (t, shape, dtype) in checks.items():
        if t is None:
            raise ValueError(f"{name} is missing")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"{name} is {t.dtype}, expected {dtype}")
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, q on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def _check_workspace(ws, dev):
    if ws.device != dev or ws.dtype != torch.uint8 or not ws.is_contiguous():
        raise ValueError(f"workspace must be a contiguous uint8 tensor on {dev}")


def gla_forward_workspace_size(batch, heads, head_dim, T, H, W, dtype):
    return lib().gla_forward_workspace_size(batch, heads, head_dim, T, H, W, dtype)


def gla_block_causal_workspace_size(batch, heads, head_dim, T_blk, H, W, dtype):
    return lib().gla_block_causal_workspace_size(batch, heads, head_dim, T_blk, H, W, dtype)


def gla_forward_host_arena_size(batch, heads, head_dim, T, H, W, dtype):
    return lib().gla_forward_host_arena_size(batch, heads, head_dim, T, H, W, dtype)


def alloc_workspace(nbytes, device="cuda"):
    """A 256-byte aligned device buffer of nbytes (torch allocations are)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def gla_forward(q, k, v, beta, g, T, H, W, rope_theta=10000.0, eps=1e-6, out=None,
                workspace=None, stream=None, path=GLA_PATH_AUTO):
    """o = RMSNorm(sigmoid(g) * S q_til / (z.q_pls + eps)) over all T*H*W tokens.

    q, k, v, g: [B, N, Hh, d]; beta: [B, N, Hh]; all on the GPU, same dtype."""
    B, Hh, d = _dims(q, T, H, W)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out)
    if workspace is None:
        workspace = alloc_workspace(gla_forward_workspace_size(B, Hh, d, T, H, W, code), q.device)
    _check_workspace(workspace, q.device)
    with _on(q.device):
        st = lib().gla_forward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), B, Hh, d, T,
                                  H, W, rope_theta, eps, code, _ptr(out), _ptr(workspace),
                                  workspace.numel(), _stream(stream, q.device), path)
    _check(st, "gla_forward")
    return out


def gla_forward_timed(q, k, v, beta, g, T, H, W, events, rope_theta=10000.0, eps=1e-6,
                      out=None, workspace=None, stream=None, path=GLA_PATH_AUTO):
    """gla_forward recording four torch.cuda.Event objects around its kernels
    (before the state reduction, after it, after the combine, after the
    read-out)."""
    B, Hh, d = _dims(q, T, H, W)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out)
    if workspace is None:
        workspace = alloc_workspace(gla_forward_workspace_size(B, Hh, d, T, H, W, code), q.device)
    _check_workspace(workspace, q.device)
    ev = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) if e is not None else None
                                 for e in events])
    with _on(q.device):
        st = lib().gla_forward_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), B, Hh, d,
                                     T, H, W, rope_theta, eps, code, _ptr(out),
                                     _ptr(workspace), workspace.numel(),
                                     _stream(stream, q.device), path, ev)
    _check(st, "gla_forward_timed")
    return out


def gla_forward_debug(q, k, v, beta, g, T, H, W, rope_theta=10000.0, eps=1e-6,
                      path=GLA_PATH_AUTO, stream=None):
    """gla_forward plus the hidden intermediates S, z, den and x (pre-norm)."""
    B, Hh, d = _dims(q, T, H, W)
    N = q.shape[1]
    code = _dtype_code(q)
    dev = q.device
    out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out)
    S = torch.empty(B, Hh, d, d, dtype=torch.float32, device=dev)
    z = torch.empty(B, Hh, d, dtype=torch.float32, device=dev)
    den = torch.empty(B, N, Hh, dtype=torch.float32, device=dev)
    x = torch.empty(B, N, Hh, d, dtype=torch.float32, device=dev)
    ws = alloc_workspace(gla_forward_workspace_size(B, Hh, d, T, H, W, code), dev)
    with _on(dev):
        st = lib().gla_forward_debug(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), B, Hh, d,
                                     T, H, W, rope_theta, eps, code, _ptr(out), _ptr(ws),
                                     ws.numel(), _stream(stream, dev), path, _ptr(S), _ptr(z),
                                     _ptr(den), _ptr(x))
    _check(st, "gla_forward_debug")
    return dict(out=out, S=S, z=z, den=den, x=x)


def gla_block_causal_step(state, z, q, k, v, beta, g, T_blk, H, W, t0, rope_theta=10000.0,
                          eps=1e-6, out=None, workspace=None, stream=None,
                          path=GLA_PATH_AUTO):
    """One block: state += block state, z += block key sum (in place), then the
    block is read out against the updated state.  state [B,Hh,d,d], z [B,Hh,d]
    fp32 on the GPU."""
    B, Hh, d = _dims(q, T_blk, H, W)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out, state=(state, (B, Hh, d, d), torch.float32),
              z=(z, (B, Hh, d), torch.float32))
    if workspace is None:
        workspace = alloc_workspace(
            gla_block_causal_workspace_size(B, Hh, d, T_blk, H, W, code), q.device)
    _check_workspace(workspace, q.device)
    with _on(q.device):
        st = lib().gla_block_causal_step_ex(_ptr(state), _ptr(z), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(beta), _ptr(g), B, Hh, d, T_blk, H, W, t0,
                                            rope_theta, eps, code, _ptr(out), _ptr(workspace),
                                            workspace.numel(), _stream(stream, q.device), path)
    _check(st, "gla_block_causal_step")
    return out


def gla_forward_host(q, k, v, beta, g, T, H, W, rope_theta=10000.0, eps=1e-6, out=None,
                     arena=None, stream=None):
    """gla_forward on host tensors (pin them for asynchronous copies): one H2D
    copy per input into the device `arena`, the operator, one D2H copy of out.
    Asynchronous on `stream`; synchronise before reading `out`."""
    B, Hh, d = _dims(q, T, H, W)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out, cuda=False)
    if arena is None:
        arena = alloc_workspace(gla_forward_host_arena_size(B, Hh, d, T, H, W, code))
    if arena.device.type != "cuda" or arena.dtype != torch.uint8 or not arena.is_contiguous():
        raise ValueError("arena must be a contiguous uint8 tensor on the GPU")
    with _on(arena.device):
        st = lib().gla_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), B, Hh, d,
                                    T, H, W, rope_theta, eps, code, _ptr(out), _ptr(arena),
                                    arena.numel(), _stream(stream, arena.device))
    _check(st, "gla_forward_host")
    return out


def gla_block_causal_host_arena_size(batch, heads, head_dim, T_blk, H, W, dtype):
    return lib().gla_block_causal_host_arena_size(batch, heads, head_dim, T_blk, H, W, dtype)


def gla_causal_host_arena_size(batch, heads, head_dim, T, H, W, dtype):
    return lib().gla_causal_host_arena_size(batch, heads, head_dim, T, H, W, dtype)


def gla_block_causal_step_host(state, z, q, k, v, beta, g, T_blk, H, W, t0, rope_theta=10000.0,
                               eps=1e-6, out=None, arena=None, stream=None):
    """One block-causal step on host tensors (pin them for asynchronous
    copies): the block's inputs go to the device `arena`, the step updates the
    device-resident state and z in place, and the block's output comes back
    into `out`.  Asynchronous on `stream`; synchronise before reading `out`."""
    return _staged("gla_block_causal_step_host", "gla_block_causal_host_arena_size", state, z,
                   q, k, v, beta, g, T_blk, H, W, t0, rope_theta, eps, out, arena, stream)


def gla_causal_step_host(state, z, q, k, v, beta, g, T, H, W, t0=0, rope_theta=10000.0,
                         eps=1e-6, out=None, arena=None, stream=None):
    """gla_causal_step on host tensors (pin them for asynchronous copies), the
    state (state, z) resident on the GPU and updated in place.  Asynchronous
    on `stream`; synchronise before reading `out`."""
    return _staged("gla_causal_step_host", "gla_causal_host_arena_size", state, z, q, k, v,
                   beta, g, T, H, W, t0, rope_theta, eps, out, arena, stream)


def _staged(entry, arena_size, state, z, q, k, v, beta, g, T, H, W, t0, rope_theta, eps, out,
            arena, stream):
    B, Hh, d = _dims(q, T, H, W)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out, cuda=False)
    dev = state.device
    if dev.type != "cuda" or z.device != dev:
        raise ValueError("state and z must be on the GPU, on one device")
    for name, t, shape in (("state", state, (B, Hh, d, d)), ("z", z, (B, Hh, d))):
        if tuple(t.shape) != shape or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 tensor of shape {shape}")
    if arena is None:
        arena = alloc_workspace(getattr(lib(), arena_size)(B, Hh, d, T, H, W, code), dev)
    if arena.device != dev or arena.dtype != torch.uint8 or not arena.is_contiguous():
        raise ValueError(f"arena must be a contiguous uint8 tensor on {dev}")
    with _on(dev):
        st = getattr(lib(), entry)(_ptr(state), _ptr(z), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                   _ptr(g), B, Hh, d, T, H, W, t0, rope_theta, eps, code,
                                   _ptr(out), _ptr(arena), arena.numel(), _stream(stream, dev))
    _check(st, entry)
    return out


def gla_causal_workspace_size(batch, heads, head_dim, T, H, W, dtype):
    return lib().gla_causal_workspace_size(batch, heads, head_dim, T, H, W, dtype)


def gla_causal_step(state, z, q, k, v, beta, g, T, H, W, t0=0, rope_theta=10000.0, eps=1e-6,
                    out=None, workspace=None, stream=None, path=GLA_PATH_AUTO, den_out=None,
                    x_out=None):
    """Token-level causal read-out of one segment of a sequence: token j sees
    the carried (state, z) plus tokens 0..j of this call; (state, z) are
    updated in place to the sums after the call.  state [B,Hh,d,d], z [B,Hh,d]
    fp32 on the GPU; den_out [B,N,Hh] / x_out [B,N,Hh,d] fp32 optional exports."""
    B, Hh, d = _dims(q, T, H, W)
    N = q.shape[1]
    code = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    extra = dict(state=(state, (B, Hh, d, d), torch.float32), z=(z, (B, Hh, d), torch.float32))
    if den_out is not None:
        extra["den_out"] = (den_out, (B, N, Hh), torch.float32)
    if x_out is not None:
        extra["x_out"] = (x_out, (B, N, Hh, d), torch.float32)
    _validate(q, k, v, beta, g, out, **extra)
    if workspace is None:
        workspace = alloc_workspace(gla_causal_workspace_size(B, Hh, d, T, H, W, code), q.device)
    _check_workspace(workspace, q.device)
    with _on(q.device):
        st = lib().gla_causal_step_ex(_ptr(state), _ptr(z), _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(beta), _ptr(g), B, Hh, d, T, H, W, t0, rope_theta,
                                      eps, code, _ptr(out), _ptr(workspace), workspace.numel(),
                                      _stream(stream, q.device), path, _ptr(den_out),
                                      _ptr(x_out))
    _check(st, "gla_causal_step")
    return out


def gla_causal_step_timed(state, z, q, k, v, beta, g, T, H, W, events, t0=0,
                          rope_theta=10000.0, eps=1e-6, out=None, workspace=None, stream=None,
                          path=GLA_PATH_AUTO):
    """gla_causal_step recording four torch.cuda.Event objects around its
    kernels (before the state partials, after them, after their prefix,
    after the causal read-out)."""
    B, Hh, d = _dims(q, T, H, W)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out, state=(state, (B, Hh, d, d), torch.float32),
              z=(z, (B, Hh, d), torch.float32))
    if workspace is None:
        workspace = alloc_workspace(gla_causal_workspace_size(B, Hh, d, T, H, W, code), q.device)
    _check_workspace(workspace, q.device)
    ev = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) if e is not None else None
                                 for e in events])
    with _on(q.device):
        st = lib().gla_causal_step_timed(_ptr(state), _ptr(z), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(beta), _ptr(g), B, Hh, d, T, H, W, t0, rope_theta,
                                         eps, code, _ptr(out), _ptr(workspace),
                                         workspace.numel(), _stream(stream, q.device), path,
                                         None, None, ev)
    _check(st, "gla_causal_step_timed")
    return out


def gla_causal_forward(q, k, v, beta, g, T, H, W, rope_theta=10000.0, eps=1e-6, out=None,
                       workspace=None, stream=None, path=GLA_PATH_AUTO):
    """The causal read-out of a whole sequence (zero state before it)."""
    B, Hh, d = _dims(q, T, H, W)
    state = torch.zeros(B, Hh, d, d, dtype=torch.float32, device=q.device)
    z = torch.zeros(B, Hh, d, dtype=torch.float32, device=q.device)
    return gla_causal_step(state, z, q, k, v, beta, g, T, H, W, 0, rope_theta, eps, out=out,
                           workspace=workspace, stream=stream, path=path)


def _bf16_matrix(t, name, dev=None):
    if t.dim() != 2 or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.device.type != "cuda":
        raise ValueError(f"{name} must be a contiguous 2-D bf16 GPU tensor")
    if dev is not None and t.device != dev:
        raise ValueError(f"{name} is on {t.device}, expected {dev}")


def gla_gemm_bf16(A, B, out=None, stream=None):
    """A [M, K] @ B[N, K]^T on the tensor cores (bf16 in and out, fp32 sums)."""
    _bf16_matrix(A, "A")
    _bf16_matrix(B, "B", A.device)
    M, K = A.shape
    N, K2 = B.shape
    if K2 != K:
        raise ValueError(f"A is {tuple(A.shape)}, B is {tuple(B.shape)}: K differs")
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=A.device)
    _bf16_matrix(out, "out", A.device)
    if tuple(out.shape) != (M, N):
        raise ValueError(f"out must be [{M}, {N}]")
    with _on(A.device):
        st = lib().gla_gemm_bf16(_ptr(A), _ptr(B), _ptr(out), M, N, K, _stream(stream, A.device))
    _check(st, "gla_gemm_bf16")
    return out


def gla_project_in(x, W_in, batch, N, heads, head_dim, stream=None):
    """x [batch*N, C] times W_in^T, split into the operator's inputs: returns
    dict(q, k, v, g [batch, N, heads, head_dim], beta [batch, N, heads])."""
    _bf16_matrix(x, "x")
    _bf16_matrix(W_in, "W_in", x.device)
    tokens, C = x.shape
    if tokens != batch * N or tuple(W_in.shape) != (4 * heads * head_dim + heads, C):
        raise ValueError("x must be [batch*N, C] and W_in [4*heads*head_dim + heads, C]")
    dev = x.device
    out = {n: torch.empty(batch, N, heads, head_dim, dtype=torch.bfloat16, device=dev)
           for n in "qkvg"}
    out["beta"] = torch.empty(batch, N, heads, dtype=torch.bfloat16, device=dev)
    with _on(dev):
        st = lib().gla_project_in(_ptr(x), _ptr(W_in), tokens, C, heads, head_dim, _ptr(out["q"]),
                                  _ptr(out["k"]), _ptr(out["v"]), _ptr(out["g"]), _ptr(out["beta"]),
                                  _stream(stream, dev))
    _check(st, "gla_project_in")
    return out


def gla_layer_forward(x, W_in, W_o, batch, heads, head_dim, T, H, W, rope_theta=10000.0,
                      eps=1e-6, out=None, workspace=None, stream=None):
    """y [batch*N, C_out] = W_o applied to the operator of the projections of
    x [batch*N, C]."""
    _bf16_matrix(x, "x")
    _bf16_matrix(W_in, "W_in", x.device)
    _bf16_matrix(W_o, "W_o", x.device)
    tokens, C = x.shape
    C_out, HD = W_o.shape
    if tokens != batch * T * H * W or HD != heads * head_dim or \
            tuple(W_in.shape) != (4 * heads * head_dim + heads, C):
        raise ValueError("shapes do not match the layer")
    dev = x.device
    if out is None:
        out = torch.empty(tokens, C_out, dtype=torch.bfloat16, device=dev)
    _bf16_matrix(out, "out", dev)
    if workspace is None:
        workspace = alloc_workspace(lib().gla_layer_workspace_size(batch, heads, head_dim, T, H, W),
                                    dev)
    _check_workspace(workspace, dev)
    with _on(dev):
        st = lib().gla_layer_forward(_ptr(x), _ptr(W_in), _ptr(W_o), batch, C, C_out, heads,
                                     head_dim, T, H, W, rope_theta, eps, _ptr(out),
                                     _ptr(workspace), workspace.numel(), _stream(stream, dev))
    _check(st, "gla_layer_forward")
    return out


def gla_softmax_anchor_workspace_size(batch, heads, head_dim, T, H, W):
    return lib().gla_softmax_anchor_workspace_size(batch, heads, head_dim, T, H, W)


def gla_softmax_anchor(q, k, v, g, T, H, W, rope_theta=10000.0, out=None, workspace=None,
                       stream=None, events=None):
    """The gated softmax anchor: o_j = sigmoid(g_j) * softmax(q_til_j . K_til^T
    / sqrt(d)) V over all T*H*W tokens, q_til / k_til the RMS-normalised and
    3D-rotated q / k.  q, k, v, g: bf16 [B, N, Hh, 128] on one GPU.  events:
    three torch.cuda.Event objects recorded before the q/k preparation, after
    it and after the attention kernel."""
    B, Hh, d = _dims(q, T, H, W)
    if out is None:
        out = torch.empty_like(q)
    shape = tuple(q.shape)
    for name, t in (("q", q), ("k", k), ("v", v), ("g", g), ("out", out)):
        if tuple(t.shape) != shape or t.dtype != torch.bfloat16 or t.device != q.device \
                or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor of shape {shape} "
                             f"on {q.device}")
    if q.device.type != "cuda":
        raise ValueError(f"q is on {q.device}; gla_softmax_anchor takes GPU tensors")
    if workspace is None:
        workspace = alloc_workspace(gla_softmax_anchor_workspace_size(B, Hh, d, T, H, W),
                                    q.device)
    _check_workspace(workspace, q.device)
    ev = None
    if events is not None:
        for e in events:        # torch creates an event's handle at its first record
            if e is not None and e.cuda_event == 0:
                e.record(torch.cuda.current_stream(q.device) if stream is None else stream)
        ev = (ctypes.c_void_p * 3)(*[ctypes.c_void_p(e.cuda_event) if e is not None else None
                                     for e in events])
    with _on(q.device):
        st = lib().gla_softmax_anchor_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), B, Hh, d, T, H, W,
                                            rope_theta, _ptr(out), _ptr(workspace),
                                            workspace.numel(), _stream(stream, q.device), ev)
    _check(st, "gla_softmax_anchor")
    return out


MX_NAMES = ("q", "q_scale", "k", "k_scale", "v", "v_scale", "beta", "g", "g_scale")


def gla_forward_mx(x, T, H, W, rope_theta=10000.0, eps=1e-6, out=None, workspace=None,
                   stream=None, path=GLA_PATH_AUTO, debug=False, events=None):
    """The operator on FP8 (OCP MX) inputs.  x: dict with uint8 codes q, k, v,
    g [B, N, Hh, 128] and uint8 E8M0 scales q_scale .. g_scale [B, N, Hh, 4]
    (one per 32 channels), and bf16 beta [B, N, Hh], all on one GPU.  Returns
    the bf16 output, or with debug=True dict(out, S, z, den, x) like
    gla_forward_debug.  events: four torch.cuda.Event objects recorded around
    the kernels (as gla_forward_timed)."""
    q = x["q"]
    if q.dim() != 4 or q.shape[-1] != 128:
        raise ValueError(f"q codes must be [B, N, heads, 128], got {tuple(q.shape)}")
    B, N, Hh, d = q.shape
    if N != T * H * W:
        raise ValueError(f"q has {N} tokens, grid {T}x{H}x{W} has {T * H * W}")
    dev = q.device
    if dev.type != "cuda":
        raise ValueError(f"q is on {dev}; this entry point takes GPU tensors")
    shapes = {"q": (B, N, Hh, d), "k": (B, N, Hh, d), "v": (B, N, Hh, d), "g": (B, N, Hh, d),
              "q_scale": (B, N, Hh, d // 32), "k_scale": (B, N, Hh, d // 32),
              "v_scale": (B, N, Hh, d // 32), "g_scale": (B, N, Hh, d // 32), "beta": (B, N, Hh)}
    for name, shape in shapes.items():
        t = x.get(name)
        want = torch.bfloat16 if name == "beta" else torch.uint8
        if t is None:
            raise ValueError(f"{name} is missing")
        if tuple(t.shape) != shape or t.dtype != want or t.device != dev or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {want} tensor of shape {shape} on {dev}")
    if out is None:
        out = torch.empty(B, N, Hh, d, dtype=torch.bfloat16, device=dev)
    if tuple(out.shape) != (B, N, Hh, d) or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor of the input shape")
    if workspace is None:
        workspace = alloc_workspace(lib().gla_forward_mx_workspace_size(B, Hh, d, T, H, W, path),
                                    dev)
    _check_workspace(workspace, dev)
    dbg = {}
    if debug:
        dbg = dict(S=torch.empty(B, Hh, d, d, dtype=torch.float32, device=dev),
                   z=torch.empty(B, Hh, d, dtype=torch.float32, device=dev),
                   den=torch.empty(B, N, Hh, dtype=torch.float32, device=dev),
                   x=torch.empty(B, N, Hh, d, dtype=torch.float32, device=dev))
    ev = None
    if events is not None:
        ev = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) if e is not None else None
                                     for e in events])
    with _on(dev):
        st = lib().gla_forward_mx_ex(*[_ptr(x[n]) for n in MX_NAMES], B, Hh, d, T, H, W,
                                     rope_theta, eps, _ptr(out), _ptr(workspace),
                                     workspace.numel(), _stream(stream, dev), path,
                                     _ptr(dbg.get("S")), _ptr(dbg.get("z")), _ptr(dbg.get("den")),
                                     _ptr(dbg.get("x")), ev)
    _check(st, "gla_forward_mx")
    return dict(out=out, **dbg) if debug else out


def gla_forward_noalloc(q, k, v, beta, g, T, H, W, rope_theta=10000.0, eps=1e-6, out=None,
                        stream=None):
    """gla_forward without a workspace argument, for callers that cannot
    allocate device memory: the scratch comes from an array built into
    libgla.so (GLA_NOALLOC_SCRATCH_BYTES).  Calls share that array, so keep
    them ordered on one stream."""
    B, Hh, d = _dims(q, T, H, W)
    code = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out)
    with _on(q.device):
        st = lib().gla_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), B, Hh, d,
                                       T, H, W, rope_theta, eps, code, _ptr(out),
                                       _stream(stream, q.device))
    _check(st, "gla_forward_noalloc")
    return out


def gla_get_device_status(stream=None):
    """Synchronise the stream and return (and clear) the device error status."""
    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with _on(dev):
        return lib().gla_get_device_status(_stream(stream, dev))


def gla_selftest_wait_timeout(limit_us, stream=None):
    """Launch the failure-detection self-test: a bounded wait that nothing
    satisfies gives up after `limit_us` microseconds and records a timeout
    (read it with gla_get_device_status)."""
    dev = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    with _on(dev):
        st = lib().gla_selftest_wait_timeout(int(limit_us), _stream(stream, dev))
    _check(st, "gla_selftest_wait_timeout")


def gla_selftest_pipeline_stall(q, k, v, beta, g, T, H, W, limit_us, rope_theta=10000.0,
                                eps=1e-6, out=None, workspace=None, stream=None):
    """Run gla_forward (tensor path) with the state kernel's waits limited to
    `limit_us` and one producer arrival withheld, so that its pipeline abort
    path runs for real; read the outcome with gla_get_device_status()."""
    B, Hh, d = _dims(q, T, H, W)
    if out is None:
        out = torch.empty_like(q)
    _validate(q, k, v, beta, g, out)
    if workspace is None:
        workspace = alloc_workspace(gla_forward_workspace_size(B, Hh, d, T, H, W,
                                                               _dtype_code(q)), q.device)
    _check_workspace(workspace, q.device)
    with _on(q.device):
        st = lib().gla_selftest_pipeline_stall(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g),
                                               B, Hh, d, T, H, W, rope_theta, eps, _ptr(out),
                                               _ptr(workspace), workspace.numel(),
                                               int(limit_us), _stream(stream, q.device))
    _check(st, "gla_selftest_pipeline_stall")
    return out


def gla_plan(batch, heads, head_dim, T, H, W, dtype, path, num_sms):
    grid, tile, used = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    st = lib().gla_plan(batch, heads, head_dim, T, H, W, dtype, path, num_sms,
                        ctypes.byref(grid), ctypes.byref(tile), ctypes.byref(used))
    _check(st, "gla_plan")
    return grid.value, tile.value, used.value


def gla_check_rope_copy(batch, heads, head_dim, T, H, W, num_sms):
    """Host-only check of the read-out's RoPE table copy plan (status code)."""
    return lib().gla_check_rope_copy(batch, heads, head_dim, T, H, W, num_sms)
