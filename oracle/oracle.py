"""ctypes wrapper of the fp64 oracle (numpy in, numpy out)."""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")


def _ptr(x):
    return None if x is None else x.ctypes.data_as(C.c_void_p)


def build(force: bool = False, path: str | None = None):
    """Compile and load the oracle library.  `path` loads another build of the
    same source (used by the tests that plant mistakes in a copy)."""
    global _lib
    if path is not None:
        return _bind(C.CDLL(path))
    _lib = _bind(C.CDLL(_build.build(force=force)))
    return _lib


def _bind(lib):
    vp, i32, i64, dbl = C.c_void_p, C.c_int32, C.c_int64, C.c_double
    lib.gdn_oracle_prefill.restype = C.c_int
    lib.gdn_oracle_prefill.argtypes = [vp, vp, vp, C.c_int, vp, vp, vp, vp, vp, i32, i64,
                                       i32, i32, i32, i32, dbl, vp, i32, i32, vp, vp, vp, C.c_int]
    lib.gdn_oracle_prefill_chunked.restype = C.c_int
    lib.gdn_oracle_prefill_chunked.argtypes = [vp, vp, vp, C.c_int, vp, vp, vp, vp, vp, i32, i64,
                                               i32, i32, i32, i32, dbl, vp, i32, i32, i32, vp, vp,
                                               C.c_int]
    lib.gdn_oracle_decode.restype = C.c_int
    lib.gdn_oracle_decode.argtypes = [vp, vp, vp, C.c_int, vp, vp, vp, vp, i32, i32, i32, i32,
                                      i32, i32, dbl, vp, vp, i64, vp, vp, C.c_int]
    lib.gdn_oracle_conv1d_silu.restype = C.c_int
    lib.gdn_oracle_conv1d_silu.argtypes = [vp, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp, vp,
                                           vp, C.c_int]
    lib.gdn_oracle_log_alpha.restype = dbl
    lib.gdn_oracle_log_alpha.argtypes = [dbl, dbl, dbl]
    lib.gdn_oracle_beta.restype = dbl
    lib.gdn_oracle_beta.argtypes = [dbl]
    lib.gdn_oracle_gated_norm.restype = C.c_int
    lib.gdn_oracle_gated_norm.argtypes = [vp, vp, vp, i64, C.c_int, C.c_int, C.c_int, dbl, vp]
    lib.gdn_oracle_prefill_f64.restype = C.c_int
    lib.gdn_oracle_prefill_f64.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                           dbl, vp, vp, vp]
    lib.gdn_oracle_prefill_backward.restype = C.c_int
    lib.gdn_oracle_prefill_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                                i32, dbl, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdn_oracle_prefill_backward_chunked.restype = C.c_int
    lib.gdn_oracle_prefill_backward_chunked.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                                        i32, i32, dbl, vp, vp, vp, i32, vp, vp, vp, vp, vp,
                                                        vp, vp, vp]
    lib.gdn_oracle_conv1d_silu_f64.restype = C.c_int
    lib.gdn_oracle_conv1d_silu_f64.argtypes = [vp, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp, vp]
    lib.gdn_oracle_conv1d_silu_backward.restype = C.c_int
    lib.gdn_oracle_conv1d_silu_backward.argtypes = [vp, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                                    vp, C.c_int]
    lib.gdn_oracle_gated_norm_backward.restype = C.c_int
    lib.gdn_oracle_gated_norm_backward.argtypes = [vp, vp, vp, i64, C.c_int, C.c_int, C.c_int, dbl, vp, vp, vp, vp]
    lib.gdn_oracle_max_threads.restype = C.c_int
    lib.gdn_oracle_max_threads.argtypes = [C.c_int]
    return lib


def _L(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        build()
    return _lib


def _qkv(x):
    """bf16 bits (uint16) pass through; anything else becomes float64."""
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), 0
    return np.ascontiguousarray(x, dtype=np.float64), 1


def _f32(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float32)


def max_threads(threads: int = 0, lib=None) -> int:
    return _L(lib).gdn_oracle_max_threads(int(threads))


def log_alpha(a, A_log, dt_bias, lib=None) -> float:
    return _L(lib).gdn_oracle_log_alpha(float(a), float(A_log), float(dt_bias))


def beta(b, lib=None) -> float:
    return _L(lib).gdn_oracle_beta(float(b))


def _prefill_common(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, heads):
    q, isf = _qkv(q)
    k, isf2 = _qkv(k)
    v, isf3 = _qkv(v)
    if not (isf == isf2 == isf3):
        raise TypeError("q, k, v must all be bf16 bits or all float")
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seq = 1 if cu is None else len(cu) - 1
    h0, h1 = (0, Hv) if heads is None else (int(heads[0]), int(heads[1]))
    return (q, k, v, isf, _f32(a), _f32(b), _f32(A_log), _f32(dt_bias), cu, n_seq, T, Hqk, Hv,
            dk, dv, _f32(initial_state), h0, h1)


def prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens=None, scale=None, initial_state=None,
            heads=None, seq_mask=None, want_o=True, want_state=True, threads=0, lib=None):
    """Sequential fp64 recurrence.  Returns (o [T, nh, dv] or None,
    final_state [N, nh, dv, dk] or None) for value heads in range `heads`."""
    (q, k, v, isf, a, b, A_log, dt_bias, cu, n_seq, T, Hqk, Hv, dk, dv, s0, h0, h1) = \
        _prefill_common(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, heads)
    scale = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    nh = h1 - h0
    o = np.zeros((T, nh, dv), np.float64) if want_o else None
    fs = np.zeros((n_seq, nh, dv, dk), np.float64) if want_state else None
    mask = None if seq_mask is None else np.ascontiguousarray(seq_mask, dtype=np.uint8)
    rc = _L(lib).gdn_oracle_prefill(_ptr(q), _ptr(k), _ptr(v), isf, _ptr(a), _ptr(b), _ptr(A_log),
                                    _ptr(dt_bias), _ptr(cu), n_seq, T, Hqk, Hv, dk, dv, scale,
                                    _ptr(s0), h0, h1, _ptr(mask), _ptr(o), _ptr(fs), int(threads))
    if rc != 0:
        raise ValueError("oracle prefill rejected its arguments")
    return o, fs


def prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens=None, scale=None,
                    initial_state=None, heads=None, chunk=64, threads=0, lib=None):
    """fp64 chunked WY/UT form; same outputs as prefill()."""
    (q, k, v, isf, a, b, A_log, dt_bias, cu, n_seq, T, Hqk, Hv, dk, dv, s0, h0, h1) = \
        _prefill_common(q, k, v, a, b, A_log, dt_bias, cu_seqlens, initial_state, heads)
    scale = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    nh = h1 - h0
    o = np.zeros((T, nh, dv), np.float64)
    fs = np.zeros((n_seq, nh, dv, dk), np.float64)
    rc = _L(lib).gdn_oracle_prefill_chunked(_ptr(q), _ptr(k), _ptr(v), isf, _ptr(a), _ptr(b),
                                            _ptr(A_log), _ptr(dt_bias), _ptr(cu), n_seq, T, Hqk,
                                            Hv, dk, dv, scale, _ptr(s0), h0, h1, int(chunk),
                                            _ptr(o), _ptr(fs), int(threads))
    if rc != 0:
        raise ValueError("oracle chunked prefill rejected its arguments")
    return o, fs


def decode(q, k, v, a, b, A_log, dt_bias, n_seq, layers, state, units=None, scale=None,
           threads=0, lib=None):
    """One step for the listed units.  `state` is float32 [len(units) or U, Hv, dv, dk]:
    when `units` is given, state[i] is the state of unit units[i].
    Returns (o [n, Hv, dv], state_out [n, Hv, dv, dk]) in float64."""
    q, isf = _qkv(q)
    k, _ = _qkv(k)
    v, _ = _qkv(v)
    Hqk, dk = q.shape[1], q.shape[2]
    Hv, dv = v.shape[1], v.shape[2]
    scale = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    state = _f32(state)
    U = n_seq * layers
    if units is None:
        sel, n = None, U
        st_full = state
    else:
        sel = np.ascontiguousarray(units, dtype=np.int64)
        n = len(sel)
        # the C side indexes state by unit: scatter the given states into a
        # sparse full-size view is too large, so remap units to 0..n-1 instead
        st_full = None
    o = np.zeros((n, Hv, dv), np.float64)
    so = np.zeros((n, Hv, dv, dk), np.float64)
    lib_ = _L(lib)
    if sel is None:
        rc = lib_.gdn_oracle_decode(_ptr(q), _ptr(k), _ptr(v), isf, _ptr(_f32(a)), _ptr(_f32(b)),
                                    _ptr(_f32(A_log)), _ptr(_f32(dt_bias)), n_seq, layers, Hqk, Hv,
                                    dk, dv, scale, _ptr(st_full), None, n, _ptr(o), _ptr(so),
                                    int(threads))
    else:
        # gather the selected units into a compact problem whose unit i has the
        # same layer as units[i]: one sequence per selected unit, all layers'
        # gate parameters kept, per-unit inputs gathered.
        rc = 0
        a32, b32 = _f32(a), _f32(b)
        for i, u in enumerate(sel):
            l = int(u % layers)
            # a one-unit problem with layers=1 and this layer's parameters
            r = lib_.gdn_oracle_decode(
                _ptr(np.ascontiguousarray(q[u:u + 1])), _ptr(np.ascontiguousarray(k[u:u + 1])),
                _ptr(np.ascontiguousarray(v[u:u + 1])), isf,
                _ptr(np.ascontiguousarray(a32[u:u + 1])), _ptr(np.ascontiguousarray(b32[u:u + 1])),
                _ptr(np.ascontiguousarray(_f32(A_log)[l:l + 1])),
                _ptr(np.ascontiguousarray(_f32(dt_bias)[l:l + 1])), 1, 1, Hqk, Hv, dk, dv, scale,
                _ptr(np.ascontiguousarray(state[i:i + 1])), None, 1,
                _ptr(o[i:i + 1]), _ptr(so[i:i + 1]), int(threads))
            rc |= r
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    return o, so


def conv1d_silu(qkv, conv_w, cu_seqlens=None, Hqk=16, Hv=48, d=128, conv_state=None,
                threads=0, lib=None):
    """Front end in fp64.  Returns (q [T,Hqk,d], k [T,Hqk,d], v [T,Hv,d], conv_state_out)."""
    x = np.ascontiguousarray(qkv, dtype=np.uint16)
    T = x.shape[0]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seq = 1 if cu is None else len(cu) - 1
    ctot = (2 * Hqk + Hv) * d
    q = np.zeros((T, Hqk, d), np.float64)
    k = np.zeros((T, Hqk, d), np.float64)
    v = np.zeros((T, Hv, d), np.float64)
    cso = np.zeros((n_seq, ctot, 3), np.float64)
    rc = _L(lib).gdn_oracle_conv1d_silu(_ptr(x), _ptr(_f32(conv_w)), _ptr(cu), n_seq, T, Hqk, Hv,
                                        d, _ptr(_f32(conv_state)), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(cso), int(threads))
    if rc != 0:
        raise ValueError("oracle conv1d_silu rejected its arguments")
    return q, k, v, cso



def gated_norm(o, z, norm_w, eps=1e-6, lib=None):
    """Gated output norm in fp64 (gdn_oracle_gated_norm in gdn_oracle.c, which
    states the formula and the reading of the pages it follows).

    o: [T, Hv, d] (any float); z: [T, Hv, d] float or bf16 bits (uint16);
    norm_w: [d] or [layers, d] (row t uses layer t % layers).
    Returns y [T, Hv, d] float64.
    """
    o = np.ascontiguousarray(o, dtype=np.float64)
    z = np.asarray(z)
    if z.dtype == np.uint16:
        z = (z.astype(np.uint32) << 16).view(np.float32)
    z = np.ascontiguousarray(z, dtype=np.float64)
    w = np.ascontiguousarray(norm_w, dtype=np.float64)
    if w.ndim == 1:
        w = w[None, :]
    T, Hv, d = o.shape
    y = np.zeros_like(o)
    rc = _L(lib).gdn_oracle_gated_norm(_ptr(o), _ptr(z), _ptr(w), T, Hv, d, w.shape[0], float(eps),
                                       _ptr(y))
    if rc != 0:
        raise ValueError("oracle gated_norm rejected its arguments")
    return y



def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _widen(x):
    """bf16 bits (uint16) -> float64 exactly; anything else -> float64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.ascontiguousarray(x, dtype=np.float64)


def prefill_f64(q, k, v, a, b, A_log, dt_bias, cu_seqlens=None, scale=None, initial_state=None,
                lib=None):
    """The sequential recurrence with every input in float64 (gdn_oracle_prefill_f64).
    Returns (o [T, Hv, dv], final_state [N, Hv, dv, dk])."""
    q, k, v = _widen(q), _widen(k), _widen(v)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seq = 1 if cu is None else len(cu) - 1
    scale = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    o = np.zeros((T, Hv, dv))
    fs = np.zeros((n_seq, Hv, dv, dk))
    rc = _L(lib).gdn_oracle_prefill_f64(_ptr(q), _ptr(k), _ptr(v), _ptr(_f64(a)), _ptr(_f64(b)),
                                        _ptr(_f64(A_log)), _ptr(_f64(dt_bias)), _ptr(cu), n_seq, T, Hqk,
                                        Hv, dk, dv, scale, _ptr(_f64(initial_state)), _ptr(o), _ptr(fs))
    if rc != 0:
        raise ValueError("oracle prefill_f64 rejected its arguments")
    return o, fs


def prefill_backward(q, k, v, a, b, A_log, dt_bias, d_o, d_final=None, cu_seqlens=None, scale=None,
                     initial_state=None, lib=None):
    """Gradient of <d_o, o> + <d_final, S_T> through the recurrence, in float64
    (gdn_oracle_prefill_backward).  Returns a dict with dq, dk [T, Hqk, dk],
    dv [T, Hv, dv], da, db [T, Hv], dA_log, ddt_bias [Hv] and d_initial
    [N, Hv, dv, dk]."""
    q, k, v = _widen(q), _widen(k), _widen(v)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seq = 1 if cu is None else len(cu) - 1
    scale = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    out = dict(dq=np.zeros((T, Hqk, dk)), dk=np.zeros((T, Hqk, dk)), dv=np.zeros((T, Hv, dv)),
               da=np.zeros((T, Hv)), db=np.zeros((T, Hv)), dA_log=np.zeros(Hv), ddt_bias=np.zeros(Hv),
               d_initial=np.zeros((n_seq, Hv, dv, dk)))
    rc = _L(lib).gdn_oracle_prefill_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(_f64(a)), _ptr(_f64(b)), _ptr(_f64(A_log)), _ptr(_f64(dt_bias)),
        _ptr(cu), n_seq, T, Hqk, Hv, dk, dv, scale, _ptr(_f64(initial_state)), _ptr(_f64(d_o)),
        _ptr(_f64(d_final)), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["da"]),
        _ptr(out["db"]), _ptr(out["dA_log"]), _ptr(out["ddt_bias"]), _ptr(out["d_initial"]))
    if rc != 0:
        raise ValueError("oracle prefill_backward rejected its arguments")
    return out


def prefill_backward_chunked(q, k, v, a, b, A_log, dt_bias, d_o, d_final=None, cu_seqlens=None, scale=None,
                             initial_state=None, C=64, lib=None):
    """The gradient of prefill_backward taken through the chunked (WY / UT) form
    with chunks of C tokens (gdn_oracle_prefill_backward_chunked).  Same
    arguments and outputs as prefill_backward."""
    q, k, v = _widen(q), _widen(k), _widen(v)
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seq = 1 if cu is None else len(cu) - 1
    scale = 1.0 / np.sqrt(dk) if scale is None else float(scale)
    out = dict(dq=np.zeros((T, Hqk, dk)), dk=np.zeros((T, Hqk, dk)), dv=np.zeros((T, Hv, dv)),
               da=np.zeros((T, Hv)), db=np.zeros((T, Hv)), dA_log=np.zeros(Hv), ddt_bias=np.zeros(Hv),
               d_initial=np.zeros((n_seq, Hv, dv, dk)))
    rc = _L(lib).gdn_oracle_prefill_backward_chunked(
        _ptr(q), _ptr(k), _ptr(v), _ptr(_f64(a)), _ptr(_f64(b)), _ptr(_f64(A_log)), _ptr(_f64(dt_bias)),
        _ptr(cu), n_seq, T, Hqk, Hv, dk, dv, scale, _ptr(_f64(initial_state)), _ptr(_f64(d_o)),
        _ptr(_f64(d_final)), int(C), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["da"]),
        _ptr(out["db"]), _ptr(out["dA_log"]), _ptr(out["ddt_bias"]), _ptr(out["d_initial"]))
    if rc != 0:
        raise ValueError("oracle prefill_backward_chunked rejected its arguments")
    return out


def _front_x64(qkv):
    """bf16 bits (uint16) or real values -> float64"""
    x = np.asarray(qkv)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.ascontiguousarray(x, dtype=np.float64)


def conv1d_silu_f64(qkv, conv_w, cu_seqlens=None, Hqk=16, Hv=48, d=128, conv_state=None, lib=None):
    """The front end with every input in float64 (gdn_oracle_conv1d_silu_f64):
    qkv [T, Ctot] (bf16 bits or values), conv_w [Ctot, 4], conv_state
    [N, Ctot, 3] or None.  Returns (q, k, v)."""
    x = _front_x64(qkv)
    T = x.shape[0]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seq = 1 if cu is None else len(cu) - 1
    q, k, v = np.zeros((T, Hqk, d)), np.zeros((T, Hqk, d)), np.zeros((T, Hv, d))
    rc = _L(lib).gdn_oracle_conv1d_silu_f64(_ptr(x), _ptr(_f64(conv_w)), _ptr(cu), n_seq, T, Hqk, Hv, d,
                                            _ptr(_f64(conv_state)), _ptr(q), _ptr(k), _ptr(v))
    if rc != 0:
        raise ValueError("oracle conv1d_silu_f64 rejected its arguments")
    return q, k, v


def conv1d_silu_backward(qkv, conv_w, dq, dk, dv, cu_seqlens=None, Hqk=16, Hv=48, d=128, conv_state=None,
                         threads=0, lib=None):
    """Gradient of the front end (gdn_oracle_conv1d_silu_backward) given dL/dq,
    dL/dk [T, Hqk, d] and dL/dv [T, Hv, d].  Returns a dict with d_qkv
    [T, Ctot], d_conv_w [Ctot, 4] and d_conv_state [N, Ctot, 3]."""
    x = _front_x64(qkv)
    T = x.shape[0]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    n_seq = 1 if cu is None else len(cu) - 1
    ctot = (2 * Hqk + Hv) * d
    out = dict(d_qkv=np.zeros((T, ctot)), d_conv_w=np.zeros((ctot, 4)), d_conv_state=np.zeros((n_seq, ctot, 3)))
    rc = _L(lib).gdn_oracle_conv1d_silu_backward(
        _ptr(x), _ptr(_f64(conv_w)), _ptr(cu), n_seq, T, Hqk, Hv, d, _ptr(_f64(conv_state)), _ptr(_f64(dq)),
        _ptr(_f64(dk)), _ptr(_f64(dv)), _ptr(out["d_qkv"]), _ptr(out["d_conv_w"]), _ptr(out["d_conv_state"]),
        int(threads))
    if rc != 0:
        raise ValueError("oracle conv1d_silu_backward rejected its arguments")
    return out


def gated_norm_backward(o, z, norm_w, dy, eps=1e-6, lib=None):
    """Gradient of gated_norm given dL/dy (gdn_oracle_gated_norm_backward).
    Arguments as for gated_norm; returns a dict with d_o, d_z [T, Hv, d] and
    d_norm_w [layers, d] (float64)."""
    o = np.ascontiguousarray(o, dtype=np.float64)
    z = np.asarray(z)
    if z.dtype == np.uint16:
        z = (z.astype(np.uint32) << 16).view(np.float32)
    z = np.ascontiguousarray(z, dtype=np.float64)
    w = np.ascontiguousarray(norm_w, dtype=np.float64)
    if w.ndim == 1:
        w = w[None, :]
    T, Hv, d = o.shape
    out = dict(d_o=np.zeros_like(o), d_z=np.zeros_like(o), d_norm_w=np.zeros_like(w))
    rc = _L(lib).gdn_oracle_gated_norm_backward(_ptr(o), _ptr(z), _ptr(w), T, Hv, d, w.shape[0], float(eps),
                                                _ptr(_f64(dy)), _ptr(out["d_o"]), _ptr(out["d_z"]),
                                                _ptr(out["d_norm_w"]))
    if rc != 0:
        raise ValueError("oracle gated_norm_backward rejected its arguments")
    return out
