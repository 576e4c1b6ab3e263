"""ctypes binding of libgdn.so: torch tensors in, torch tensors out."""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(HERE, "libgdn.so")
_lib = None

STATUS = {
    0: "GDN_OK",
    1: "GDN_ERR_INVALID_ARG",
    2: "GDN_ERR_UNSUPPORTED",
    3: "GDN_ERR_MISALIGNED",
    4: "GDN_ERR_CUDA",
    5: "GDN_ERR_TIMEOUT",
    6: "GDN_ERR_WORKSPACE",
}

# exported symbol -> (restype, argtypes)
_vp, _i32, _i64, _f32, _sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
SIGNATURES = {
    "gdn_abi_version": (C.c_int, []),
    "gdn_status_string": (C.c_char_p, [C.c_int]),
    "gdn_last_cuda_error": (C.c_int, []),
    "gdn_last_cuda_error_string": (C.c_char_p, []),
    "gdn_conv1d_silu": (C.c_int, [_vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
                                  _vp, _vp]),
    "gdn_prefill_workspace_size": (_sz, [_i32, _i64, _i32, _i32, _i32]),
    "gdn_prefill": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32,
                              _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "gdn_prefill_status": (C.c_int, [_vp, _vp]),
    "gdn_prefill_bf16": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32,
                                   _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "gdn_check_async": (C.c_int, [_vp, _vp, _vp]),
    "gdn_layer_prefill_host_workspace_size": (_sz, [_i64, _i32, _i32, _i32, _i32]),
    "gdn_layer_prefill_host": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _f32,
                                         _i32, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp]),
    "gdn_prefill_noalloc": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
                                      _i32, _f32, _vp, _vp, _vp, _vp]),
    "gdn_decode_step": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                  _f32, _vp, _vp, _vp]),
    "gdn_decode_step_fused": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                        _i32, _i32, _f32, _i32, _vp, _vp, _vp]),
    "gdn_decode_step_bf16": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                       _i32, _f32, _vp, _vp, _vp]),
    "gdn_decode_step_fused_bf16": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                                             _i32, _i32, _i32, _f32, _i32, _vp, _vp, _vp]),
    "gdn_gated_norm": (C.c_int, [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _f32, _vp, _vp]),
    "gdn_selftest_bounded_wait": (C.c_int, [_i32, _i64, _vp, _vp]),
    "gdn_prefill_backward_workspace_size": (_sz, [_i32, _i64, _i32, _i32]),
    "gdn_prefill_backward": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
                                       _i32, _f32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _vp, _vp, _sz, _vp]),
    "gdn_gated_norm_backward_workspace_size": (_sz, [_i64, _i32, _i32, _i32]),
    "gdn_gated_norm_backward": (C.c_int, [_vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _f32, _vp, _vp, _vp,
                                          _vp, _sz, _vp]),
    "gdn_conv1d_silu_backward_workspace_size": (_sz, [_i64, _i32, _i32, _i32]),
    "gdn_conv1d_silu_backward": (C.c_int, [_vp, _vp, _vp, _i32, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
                                           _vp, _vp, _vp, _vp, _sz, _vp]),
    "gdn_prefill_backward_chunked_workspace_size": (_sz, [_i32, _i64, _i32, _i32]),
    "gdn_prefill_backward_chunked": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
                                               _i32, _f32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                               _vp, _vp, _sz, _vp]),
    "gdn_decode_step_gated": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                        _i32, _f32, _vp, _i32, _vp, _vp, _vp, _f32, _vp, _vp]),
    "gdn_prefill_gated": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _i32,
                                    _i32, _f32, _vp, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _sz, _vp]),
}


class GdnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = f"{fn} failed: {STATUS.get(status, status)}"
        if status == 4 and _lib is not None:
            msg += f" ({_lib.gdn_last_cuda_error_string().decode()})"
        super().__init__(msg)
        self.status = status


def lib_path() -> str:
    return _LIB_PATH


def lib():
    """Load libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libgdn.so not built at {_LIB_PATH}: run "
                              "`python -m gated_deltanet_recurrence_prefill_b200.build`")
        L = C.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _check(fn, status):
    if status != 0:
        raise GdnError(fn, status)


def _need(t, dtype, shape, name, device="cuda"):
    import torch
    if t is None:
        raise ValueError(f"{name} is required")
    if device == "cuda" and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device == "cpu" and t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    del torch
    return t


def conv1d_silu(qkv, conv_w, Hqk, Hv, d=128, cu_seqlens=None, conv_state_in=None,
                conv_state_out=None, out=None, stream=None):
    """Front end.  qkv [T, (2Hqk+Hv)d] bf16, conv_w [Ctot, 4] f32.
    Returns (q [T,Hqk,d], k [T,Hqk,d], v [T,Hv,d]) bf16."""
    import torch
    T = qkv.shape[0]
    ctot = (2 * Hqk + Hv) * d
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _need(qkv, torch.bfloat16, (T, ctot), "qkv")
    _need(conv_w, torch.float32, (ctot, 4), "conv_w")
    if cu_seqlens is not None:
        _need(cu_seqlens, torch.int32, (n_seq + 1,), "cu_seqlens")
    for nm, t in (("conv_state_in", conv_state_in), ("conv_state_out", conv_state_out)):
        if t is not None:
            _need(t, torch.float32, (n_seq, ctot, 3), nm)
    if out is None:
        q = torch.empty(T, Hqk, d, dtype=torch.bfloat16, device=qkv.device)
        k = torch.empty(T, Hqk, d, dtype=torch.bfloat16, device=qkv.device)
        v = torch.empty(T, Hv, d, dtype=torch.bfloat16, device=qkv.device)
    else:
        q, k, v = out
    st = lib().gdn_conv1d_silu(_ptr(qkv), _ptr(conv_w), _ptr(cu_seqlens), n_seq, T, Hqk, Hv, d,
                               _ptr(conv_state_in), _ptr(conv_state_out), _ptr(q), _ptr(k), _ptr(v),
                               _stream(stream))
    _check("gdn_conv1d_silu", st)
    return q, k, v


def _outputs(given, shapes, dev):
    """float32 output tensors of the given shapes (None: not wanted), taken from
    the caller's dict `given` where it has them (checked), else allocated."""
    import torch
    out = {}
    for name, shape in shapes.items():
        if shape is None:
            out[name] = None
        elif given is not None and given.get(name) is not None:
            _need(given[name], torch.float32, shape, name)
            out[name] = given[name]
        else:
            out[name] = torch.empty(*shape, dtype=torch.float32, device=dev)
    return out


def conv1d_silu_backward(qkv, conv_w, dq, dk, dv, Hqk, Hv, d=128, cu_seqlens=None, conv_state=None,
                         want_d_conv_state=True, workspace=None, stream=None, out=None):
    """gdn_conv1d_silu_backward: the front end's gradient given dL/dq, dL/dk
    [T, Hqk, d] and dL/dv [T, Hv, d] (float32).  Returns a dict of float32
    tensors d_qkv [T, Ctot], d_conv_w [Ctot, 4] and d_conv_state [N, Ctot, 3]
    (or None).  out: an optional dict of preallocated tensors under those names."""
    import torch
    T = qkv.shape[0]
    ctot = (2 * Hqk + Hv) * d
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _need(qkv, torch.bfloat16, (T, ctot), "qkv")
    _need(conv_w, torch.float32, (ctot, 4), "conv_w")
    _need(dq, torch.float32, (T, Hqk, d), "dq")
    _need(dk, torch.float32, (T, Hqk, d), "dk")
    _need(dv, torch.float32, (T, Hv, d), "dv")
    if cu_seqlens is not None:
        _need(cu_seqlens, torch.int32, (n_seq + 1,), "cu_seqlens")
    if conv_state is not None:
        _need(conv_state, torch.float32, (n_seq, ctot, 3), "conv_state")
    dev = qkv.device
    out = _outputs(out, dict(d_qkv=(T, ctot), d_conv_w=(ctot, 4),
                             d_conv_state=(n_seq, ctot, 3) if want_d_conv_state else None), dev)
    ws_bytes = int(lib().gdn_conv1d_silu_backward_workspace_size(T, Hqk, Hv, d))
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = lib().gdn_conv1d_silu_backward(
        _ptr(qkv), _ptr(conv_w), _ptr(cu_seqlens), n_seq, T, Hqk, Hv, d, _ptr(conv_state), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(out["d_qkv"]), _ptr(out["d_conv_w"]), _ptr(out["d_conv_state"]), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdn_conv1d_silu_backward", st)
    return out


def gated_norm_backward(o, z, norm_w, dy, eps=1e-6, workspace=None, stream=None, out=None):
    """gdn_gated_norm_backward: the gated norm's gradient given dL/dy [T, Hv, d]
    (float32).  o [T, Hv, d] float32, z [T, Hv, d] bf16, norm_w [layers, d] or
    [d] float32.  Returns a dict of float32 tensors d_o, d_z [T, Hv, d] and
    d_norm_w (shaped as norm_w).  out: an optional dict of preallocated tensors
    under those names (d_norm_w as [layers, d])."""
    import torch
    T, Hv, d = o.shape
    w2 = norm_w if norm_w.dim() == 2 else norm_w.view(1, -1)
    layers = w2.shape[0]
    _need(o, torch.float32, (T, Hv, d), "o")
    _need(z, torch.bfloat16, (T, Hv, d), "z")
    _need(w2, torch.float32, (layers, d), "norm_w")
    _need(dy, torch.float32, (T, Hv, d), "dy")
    dev = o.device
    out = _outputs(out, dict(d_o=(T, Hv, d), d_z=(T, Hv, d), d_norm_w=(layers, d)), dev)
    ws_bytes = int(lib().gdn_gated_norm_backward_workspace_size(T, Hv, d, layers))
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = lib().gdn_gated_norm_backward(
        _ptr(o), _ptr(z), _ptr(w2), _ptr(dy), T, Hv, d, layers, float(eps), _ptr(out["d_o"]), _ptr(out["d_z"]),
        _ptr(out["d_norm_w"]), _ptr(workspace),
        0 if workspace is None else workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdn_gated_norm_backward", st)
    if norm_w.dim() == 1:
        out["d_norm_w"] = out["d_norm_w"].view(-1)
    return out


def prefill_workspace_size(n_seq, T, Hqk, Hv, d=128) -> int:
    return int(lib().gdn_prefill_workspace_size(n_seq, T, Hqk, Hv, d))


def prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens=None, scale=None, initial_state=None,
            final_state=None, o=None, workspace=None, want_final_state=True, stream=None,
            o_dtype=None):
    """Chunked prefill.  Returns (o [T,Hv,d], final_state [N,Hv,d,d] f32 or None).
    o is float32 (gdn_prefill), or bf16 (gdn_prefill_bf16) when o_dtype is
    torch.bfloat16 or a bf16 `o` is passed."""
    import torch
    if o_dtype is None:
        o_dtype = o.dtype if o is not None else torch.float32
    if o_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("o must be float32 or bfloat16")
    T, Hqk, d = q.shape
    Hv = v.shape[1]
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _need(q, torch.bfloat16, (T, Hqk, d), "q")
    _need(k, torch.bfloat16, (T, Hqk, d), "k")
    _need(v, torch.bfloat16, (T, Hv, d), "v")
    _need(a, torch.float32, (T, Hv), "a")
    _need(b, torch.float32, (T, Hv), "b")
    _need(A_log, torch.float32, (Hv,), "A_log")
    _need(dt_bias, torch.float32, (Hv,), "dt_bias")
    if cu_seqlens is not None:
        _need(cu_seqlens, torch.int32, (n_seq + 1,), "cu_seqlens")
    if initial_state is not None:
        _need(initial_state, torch.float32, (n_seq, Hv, d, d), "initial_state")
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty(T, Hv, d, dtype=o_dtype, device=q.device)
    _need(o, o_dtype, (T, Hv, d), "o")
    if final_state is None and want_final_state:
        final_state = torch.empty(n_seq, Hv, d, d, dtype=torch.float32, device=q.device)
    ws_bytes = prefill_workspace_size(n_seq, T, Hqk, Hv, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    fn, name = ((lib().gdn_prefill_bf16, "gdn_prefill_bf16") if o_dtype == torch.bfloat16
                else (lib().gdn_prefill, "gdn_prefill"))
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
            _ptr(cu_seqlens), n_seq, T, Hqk, Hv, d, float(scale),
            _ptr(initial_state), _ptr(final_state), _ptr(o), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream))
    _check(name, st)
    return o, final_state


_copy_streams = {}


def layer_prefill_host(h_qkv, h_a, h_b, conv_w, A_log, dt_bias, Hqk, Hv, h_o=None, h_final_state=None,
                       conv_state_in=None, initial_state=None, conv_state_out=None, n_blocks=8, scale=None,
                       workspace=None, stream=None, copy_streams=None):
    """gdn_layer_prefill_host: front end + prefill of one sequence from pinned
    host tensors (h_qkv [T, (2Hqk+Hv)d] bf16, h_a, h_b [T, Hv] f32) to pinned
    host tensors (h_o [T, Hv, d] f32, h_final_state [Hv, d, d] f32), the copies
    overlapped with the compute over n_blocks token ranges.  conv_w, A_log,
    dt_bias, conv_state_in / _out and initial_state are device tensors.
    copy_streams: (upload, download) torch streams; by default two streams kept
    per device.  Returns (h_o, h_final_state), ready once `stream` (default: the
    current stream) reaches the point after the call."""
    import torch
    d = 128
    T = h_qkv.shape[0]
    dev = conv_w.device
    _need(h_qkv, torch.bfloat16, (T, (2 * Hqk + Hv) * d), "h_qkv", device="cpu")
    _need(h_a, torch.float32, (T, Hv), "h_a", device="cpu")
    _need(h_b, torch.float32, (T, Hv), "h_b", device="cpu")
    if h_o is None:
        h_o = torch.empty(T, Hv, d, dtype=torch.float32).pin_memory()
    if h_final_state is None:
        h_final_state = torch.empty(Hv, d, d, dtype=torch.float32).pin_memory()
    _need(h_o, torch.float32, (T, Hv, d), "h_o", device="cpu")
    _need(h_final_state, torch.float32, (Hv, d, d), "h_final_state", device="cpu")
    if scale is None:
        scale = d ** -0.5
    ws_bytes = lib().gdn_layer_prefill_host_workspace_size(T, Hqk, Hv, d, n_blocks)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    if copy_streams is None:
        key = dev.index if dev.index is not None else torch.cuda.current_device()
        if key not in _copy_streams:
            _copy_streams[key] = (torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev))
        copy_streams = _copy_streams[key]
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    st = lib().gdn_layer_prefill_host(
        _ptr(h_qkv), _ptr(h_a), _ptr(h_b), _ptr(conv_w), _ptr(A_log), _ptr(dt_bias), _ptr(conv_state_in),
        _ptr(initial_state), T, Hqk, Hv, d, float(scale), n_blocks, _ptr(h_o), _ptr(h_final_state),
        _ptr(conv_state_out), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream),
        _stream(copy_streams[0]), _stream(copy_streams[1]))
    _check("gdn_layer_prefill_host", st)
    return h_o, h_final_state


def prefill_noalloc(q, k, v, a, b, A_log, dt_bias, cu_seqlens=None, scale=None,
                    initial_state=None, final_state=None, o=None, want_final_state=True,
                    stream=None):
    """gdn_prefill_noalloc: the chunked prefill without a caller-provided
    workspace, for callers that cannot allocate device memory (the library
    uses its own fixed 64 KiB device array; see include/gdn.h).  The output
    tensors are created here only when not passed in."""
    import torch
    T, Hqk, d = q.shape
    Hv = v.shape[1]
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _need(q, torch.bfloat16, (T, Hqk, d), "q")
    _need(k, torch.bfloat16, (T, Hqk, d), "k")
    _need(v, torch.bfloat16, (T, Hv, d), "v")
    _need(a, torch.float32, (T, Hv), "a")
    _need(b, torch.float32, (T, Hv), "b")
    _need(A_log, torch.float32, (Hv,), "A_log")
    _need(dt_bias, torch.float32, (Hv,), "dt_bias")
    if cu_seqlens is not None:
        _need(cu_seqlens, torch.int32, (n_seq + 1,), "cu_seqlens")
    if initial_state is not None:
        _need(initial_state, torch.float32, (n_seq, Hv, d, d), "initial_state")
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty(T, Hv, d, dtype=torch.float32, device=q.device)
    if final_state is None and want_final_state:
        final_state = torch.empty(n_seq, Hv, d, d, dtype=torch.float32, device=q.device)
    st = lib().gdn_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log),
                                   _ptr(dt_bias), _ptr(cu_seqlens), n_seq, T, Hqk, Hv, d,
                                   float(scale), _ptr(initial_state), _ptr(final_state), _ptr(o),
                                   _stream(stream))
    _check("gdn_prefill_noalloc", st)
    return o, final_state


def prefill_status(workspace, stream=None) -> int:
    """Error word left by the last prefill on `workspace` (waits for the stream);
    workspace None: the array of gdn_prefill_noalloc on the current device."""
    return int(lib().gdn_prefill_status(_ptr(workspace), _stream(stream)))


def check_async(workspace, status_word, stream=None) -> None:
    """gdn_check_async: enqueue a copy of the workspace's error word (None: the
    array of gdn_prefill_noalloc) into `status_word`, a one-element int32 tensor
    on the device or in pinned host memory; returns without waiting."""
    import torch
    if status_word.numel() < 1 or status_word.dtype not in (torch.int32, torch.uint32):
        raise ValueError("status_word must be a one-element int32 tensor")
    if not status_word.is_cuda and not status_word.is_pinned():
        raise ValueError("status_word must be on the device or in pinned host memory")
    _check("gdn_check_async", lib().gdn_check_async(_ptr(workspace), _ptr(status_word), _stream(stream)))


def decode_step(q, k, v, a, b, A_log, dt_bias, state, n_seq, layers, scale=None, o=None,
                stream=None):
    """One decode step over U = n_seq*layers units; `state` [U,Hv,d,d] (float32,
    or bfloat16 for the bf16-state entry point) is updated in place.  Returns
    o [U,Hv,d] f32."""
    import torch
    U, Hqk, d = q.shape
    Hv = v.shape[1]
    if U != n_seq * layers:
        raise ValueError("q.shape[0] must equal n_seq * layers")
    _need(q, torch.bfloat16, (U, Hqk, d), "q")
    _need(k, torch.bfloat16, (U, Hqk, d), "k")
    _need(v, torch.bfloat16, (U, Hv, d), "v")
    _need(a, torch.float32, (U, Hv), "a")
    _need(b, torch.float32, (U, Hv), "b")
    _need(A_log, torch.float32, (layers, Hv), "A_log")
    _need(dt_bias, torch.float32, (layers, Hv), "dt_bias")
    bf16 = state.dtype == torch.bfloat16
    _need(state, torch.bfloat16 if bf16 else torch.float32, (U, Hv, d, d), "state")
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty(U, Hv, d, dtype=torch.float32, device=q.device)
    name = "gdn_decode_step_bf16" if bf16 else "gdn_decode_step"
    st = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log),
                              _ptr(dt_bias), n_seq, layers, Hqk, Hv, d, float(scale), _ptr(state),
                              _ptr(o), _stream(stream))
    _check(name, st)
    return o


def decode_step_fused(qkv, conv_w, conv_state, a, b, A_log, dt_bias, state, n_seq, layers, Hqk, Hv,
                      slot=None, scale=None, o=None, stream=None):
    """One decode step with the front end fused in, for n_seq sequences x
    `layers` layers.  qkv [n_seq*layers, Ctot] bf16, conv_w [layers, Ctot, 4],
    conv_state [n_slots*layers, Ctot, 3] float32 and state [n_slots*layers, Hv,
    d, d] (float32, or bfloat16 for the bf16-state entry point), both updated in
    place, slot [n_seq] int32 or None.  Returns o [n_seq*layers, Hv, d] f32."""
    import torch
    d = state.shape[-1]
    U = n_seq * layers
    ctot = (2 * Hqk + Hv) * d
    n_slots = state.shape[0] // layers
    _need(qkv, torch.bfloat16, (U, ctot), "qkv")
    _need(conv_w, torch.float32, (layers, ctot, 4), "conv_w")
    _need(conv_state, torch.float32, (n_slots * layers, ctot, 3), "conv_state")
    bf16 = state.dtype == torch.bfloat16
    _need(state, torch.bfloat16 if bf16 else torch.float32, (n_slots * layers, Hv, d, d), "state")
    _need(a, torch.float32, (U, Hv), "a")
    _need(b, torch.float32, (U, Hv), "b")
    _need(A_log, torch.float32, (layers, Hv), "A_log")
    _need(dt_bias, torch.float32, (layers, Hv), "dt_bias")
    if slot is not None:
        _need(slot, torch.int32, (n_seq,), "slot")
    if o is None:
        o = torch.empty(U, Hv, d, dtype=torch.float32, device=state.device)
    scale = 1.0 / d ** 0.5 if scale is None else float(scale)
    name = "gdn_decode_step_fused_bf16" if bf16 else "gdn_decode_step_fused"
    st = getattr(lib(), name)(_ptr(qkv), _ptr(conv_w), _ptr(conv_state), _ptr(a), _ptr(b),
                              _ptr(A_log), _ptr(dt_bias), _ptr(slot), n_seq, layers, Hqk, Hv,
                              d, scale, n_slots, _ptr(state), _ptr(o), _stream(stream))
    _check(name, st)
    return o


def gated_norm(o, z, norm_w, eps=1e-6, y=None, stream=None):
    """Gated output norm: y = norm_w * o / sqrt(mean_v o^2 + eps) * silu(z) per
    (token, value head).  o [T, Hv, d] float32, z [T, Hv, d] bf16, norm_w [d]
    or [layers, d] float32 (row t uses layer t % layers).  Returns y [T, Hv, d]
    bf16."""
    import torch
    T, Hv, d = o.shape
    w = norm_w if norm_w.dim() == 2 else norm_w.view(1, -1)
    layers = w.shape[0]
    _need(o, torch.float32, (T, Hv, d), "o")
    _need(z, torch.bfloat16, (T, Hv, d), "z")
    _need(w, torch.float32, (layers, d), "norm_w")
    if y is None:
        y = torch.empty(T, Hv, d, dtype=torch.bfloat16, device=o.device)
    st = lib().gdn_gated_norm(_ptr(o), _ptr(z), _ptr(w), T, Hv, d, layers, float(eps), _ptr(y),
                              _stream(stream))
    _check("gdn_gated_norm", st)
    return y


def prefill_gated(q, k, v, a, b, A_log, dt_bias, z, norm_w, eps=1e-6, cu_seqlens=None, scale=None,
                  initial_state=None, final_state=None, y=None, o=None, want_o=False,
                  workspace=None, want_final_state=True, stream=None):
    """gdn_prefill_gated: the chunked prefill with the gated output norm fused
    in.  z [T, Hv, d] bf16, norm_w [d] float32.  Returns (y [T, Hv, d] bf16,
    o [T, Hv, d] f32 or None, final_state or None); o is written only when
    passed in or want_o is set."""
    import torch
    T, Hqk, d = q.shape
    Hv = v.shape[1]
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _need(q, torch.bfloat16, (T, Hqk, d), "q")
    _need(k, torch.bfloat16, (T, Hqk, d), "k")
    _need(v, torch.bfloat16, (T, Hv, d), "v")
    _need(a, torch.float32, (T, Hv), "a")
    _need(b, torch.float32, (T, Hv), "b")
    _need(A_log, torch.float32, (Hv,), "A_log")
    _need(dt_bias, torch.float32, (Hv,), "dt_bias")
    _need(z, torch.bfloat16, (T, Hv, d), "z")
    _need(norm_w, torch.float32, (d,), "norm_w")
    if cu_seqlens is not None:
        _need(cu_seqlens, torch.int32, (n_seq + 1,), "cu_seqlens")
    if initial_state is not None:
        _need(initial_state, torch.float32, (n_seq, Hv, d, d), "initial_state")
    if scale is None:
        scale = d ** -0.5
    if y is None:
        y = torch.empty(T, Hv, d, dtype=torch.bfloat16, device=q.device)
    if o is None and want_o:
        o = torch.empty(T, Hv, d, dtype=torch.float32, device=q.device)
    if final_state is None and want_final_state:
        final_state = torch.empty(n_seq, Hv, d, d, dtype=torch.float32, device=q.device)
    ws_bytes = prefill_workspace_size(n_seq, T, Hqk, Hv, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    st = lib().gdn_prefill_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log),
                                 _ptr(dt_bias), _ptr(cu_seqlens), n_seq, T, Hqk, Hv, d, float(scale),
                                 _ptr(initial_state), _ptr(final_state), _ptr(o), _ptr(z),
                                 _ptr(norm_w), float(eps), _ptr(y), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdn_prefill_gated", st)
    return y, o, final_state


def decode_step_gated(q, k, v, a, b, A_log, dt_bias, state, n_seq, layers, z, norm_w, eps=1e-6,
                      scale=None, y=None, o=None, want_o=False, stream=None):
    """One decode step with the gated output norm fused in.  As decode_step,
    plus z [U, Hv, d] bf16 and norm_w [layers, d] f32.  Returns (y [U, Hv, d]
    bf16, o or None)."""
    import torch
    U, Hqk, d = q.shape
    Hv = v.shape[1]
    _need(q, torch.bfloat16, (U, Hqk, d), "q")
    _need(k, torch.bfloat16, (U, Hqk, d), "k")
    _need(v, torch.bfloat16, (U, Hv, d), "v")
    _need(a, torch.float32, (U, Hv), "a")
    _need(b, torch.float32, (U, Hv), "b")
    _need(A_log, torch.float32, (layers, Hv), "A_log")
    _need(dt_bias, torch.float32, (layers, Hv), "dt_bias")
    bf16 = state.dtype == torch.bfloat16
    _need(state, torch.bfloat16 if bf16 else torch.float32, (U, Hv, d, d), "state")
    _need(z, torch.bfloat16, (U, Hv, d), "z")
    _need(norm_w, torch.float32, (layers, d), "norm_w")
    if scale is None:
        scale = d ** -0.5
    if y is None:
        y = torch.empty(U, Hv, d, dtype=torch.bfloat16, device=q.device)
    if o is None and want_o:
        o = torch.empty(U, Hv, d, dtype=torch.float32, device=q.device)
    st = lib().gdn_decode_step_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log),
                                     _ptr(dt_bias), n_seq, layers, Hqk, Hv, d, float(scale),
                                     _ptr(state), 1 if bf16 else 0, _ptr(o), _ptr(z), _ptr(norm_w),
                                     float(eps), _ptr(y), _stream(stream))
    _check("gdn_decode_step_gated", st)
    return y, o


def prefill_backward(q, k, v, a, b, A_log, dt_bias, d_o, d_final_state=None, cu_seqlens=None,
                     scale=None, initial_state=None, want_d_initial=True, workspace=None, stream=None, out=None):
    """gdn_prefill_backward: gradients of a loss with dL/do = d_o [T, Hv, d] and
    dL/dS_T = d_final_state [N, Hv, d, d] (or zero).  Returns a dict of float32
    tensors dq, dk [T, Hqk, d], dv [T, Hv, d], da, db [T, Hv], dA_log,
    ddt_bias [Hv] and d_initial_state [N, Hv, d, d] (or None).  out: an optional
    dict of preallocated tensors under those names (float32, contiguous)."""
    return _backward("gdn_prefill_backward", q, k, v, a, b, A_log, dt_bias, d_o, d_final_state, cu_seqlens,
                     scale, initial_state, want_d_initial, workspace, stream, out)


def prefill_backward_chunked(q, k, v, a, b, A_log, dt_bias, d_o, d_final_state=None, cu_seqlens=None,
                             scale=None, initial_state=None, want_d_initial=True, workspace=None, stream=None,
                             out=None):
    """gdn_prefill_backward_chunked: the same gradients through the chunked
    form (two chains over 64-token chunks, the rest chunk-parallel).  Arguments
    and result as for prefill_backward."""
    return _backward("gdn_prefill_backward_chunked", q, k, v, a, b, A_log, dt_bias, d_o, d_final_state,
                     cu_seqlens, scale, initial_state, want_d_initial, workspace, stream, out)


def _backward(entry, q, k, v, a, b, A_log, dt_bias, d_o, d_final_state, cu_seqlens, scale, initial_state,
              want_d_initial, workspace, stream, given=None):
    import torch
    T, Hqk, d = q.shape
    Hv = v.shape[1]
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _need(q, torch.bfloat16, (T, Hqk, d), "q")
    _need(k, torch.bfloat16, (T, Hqk, d), "k")
    _need(v, torch.bfloat16, (T, Hv, d), "v")
    _need(a, torch.float32, (T, Hv), "a")
    _need(b, torch.float32, (T, Hv), "b")
    _need(A_log, torch.float32, (Hv,), "A_log")
    _need(dt_bias, torch.float32, (Hv,), "dt_bias")
    _need(d_o, torch.float32, (T, Hv, d), "d_o")
    if cu_seqlens is not None:
        _need(cu_seqlens, torch.int32, (n_seq + 1,), "cu_seqlens")
    if initial_state is not None:
        _need(initial_state, torch.float32, (n_seq, Hv, d, d), "initial_state")
    if d_final_state is not None:
        _need(d_final_state, torch.float32, (n_seq, Hv, d, d), "d_final_state")
    if scale is None:
        scale = d ** -0.5
    dev = q.device
    shapes = dict(dq=(T, Hqk, d), dk=(T, Hqk, d), dv=(T, Hv, d), da=(T, Hv), db=(T, Hv), dA_log=(Hv,),
                  ddt_bias=(Hv,), d_initial_state=(n_seq, Hv, d, d) if want_d_initial else None)
    out = _outputs(given, shapes, dev)
    ws_bytes = getattr(lib(), entry + "_workspace_size")(n_seq, T, Hv, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = getattr(lib(), entry)(
        _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias), _ptr(cu_seqlens), n_seq, T,
        Hqk, Hv, d, float(scale), _ptr(initial_state), _ptr(d_o), _ptr(d_final_state), _ptr(out["dq"]),
        _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["da"]), _ptr(out["db"]), _ptr(out["dA_log"]),
        _ptr(out["ddt_bias"]), _ptr(out["d_initial_state"]), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(entry, st)
    return out
