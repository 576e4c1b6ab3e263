"""The C ABI on the CPU: the library exports every symbol include/gdn.h
declares, and the host-side argument checks reject bad calls before any launch
(these calls never reach CUDA)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from gated_deltanet_recurrence_prefill_b200 import build, _lib
    build.build()
    return _lib.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("gdn_conv1d_silu", "gdn_prefill", "gdn_prefill_workspace_size",
                     "gdn_decode_step", "gdn_decode_step_fused", "gdn_prefill_status", "gdn_check_async",
                     "gdn_gated_norm", "gdn_prefill_gated", "gdn_decode_step_gated",
                     "gdn_prefill_backward", "gdn_prefill_backward_workspace_size",
                     "gdn_prefill_backward_chunked", "gdn_prefill_backward_chunked_workspace_size",
                     "gdn_conv1d_silu_backward", "gdn_conv1d_silu_backward_workspace_size",
                     "gdn_gated_norm_backward", "gdn_gated_norm_backward_workspace_size",
                     "gdn_selftest_bounded_wait", "gdn_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    from gated_deltanet_recurrence_prefill_b200 import _lib
    names = declared_functions()
    for n in names:
        assert hasattr(L, n), f"{n} declared in gdn.h but not exported"
        assert n in _lib.SIGNATURES, f"{n} has no binding signature"


def test_status_strings_and_version(L):
    assert L.gdn_abi_version() == 1
    for s in range(7):
        assert L.gdn_status_string(s)
    assert L.gdn_status_string(99) == b"unknown status"


def test_workspace_size_is_positive_and_aligned(L):
    for n, T in ((1, 256), (16, 270000), (1, 0)):
        ws = L.gdn_prefill_workspace_size(n, T, 16, 48, 128)
        assert ws > 0 and ws % 256 == 0


def test_workspace_size_matches_the_documented_formula(L):
    # gdn.h: 256 + 397440 * min(n_seq * Hv, 64), rounded up to 256
    for n, Hqk, Hv in ((1, 16, 48), (2, 16, 48), (1, 4, 12), (3, 1, 1), (16, 16, 48)):
        units = min(n * Hv, 64)
        want = 256 + ((397440 * units + 255) // 256) * 256
        assert L.gdn_prefill_workspace_size(n, 1000, Hqk, Hv, 128) == want


FAKE = 0x10000     # 16-byte aligned non-null stand-in; never dereferenced: every call below fails validation


def _p(x=FAKE):
    return C.c_void_p(x)


def test_prefill_rejects_bad_arguments(L):
    ws = L.gdn_prefill_workspace_size(1, 64, 16, 48, 128)
    good = dict(q=_p(), k=_p(), v=_p(), a=_p(), b=_p(), A_log=_p(), dt=_p(), cu=None, n=1, T=64,
                Hqk=16, Hv=48, d=128, s0=None, s1=None, o=_p(), ws=_p(0x20000), wsb=ws)

    def call(**kw):
        a = dict(good, **kw)
        return L.gdn_prefill(a["q"], a["k"], a["v"], a["a"], a["b"], a["A_log"], a["dt"], a["cu"],
                             a["n"], a["T"], a["Hqk"], a["Hv"], a["d"], 0.088, a["s0"], a["s1"],
                             a["o"], a["ws"], a["wsb"], None)

    assert call(d=64) == 2                       # unsupported head width
    assert call(Hv=40) == 2                      # Hv % Hqk != 0
    assert call(Hqk=0) == 1
    assert call(T=-1) == 1
    assert call(n=2) == 1                        # several sequences need cu_seqlens
    assert call(q=None) == 1
    assert call(A_log=None) == 1
    assert call(o=_p(FAKE + 4)) == 3             # misaligned
    assert call(ws=None) == 6
    # the least workspace accepted: the 256-byte header and 4 bytes per
    # (sequence, value head), rounded up to 256 bytes
    min_ws = 256 + ((4 * 1 * 48 + 255) // 256) * 256
    assert ws >= min_ws
    assert call(wsb=min_ws - 1) == 6
    assert call(ws=_p(0x20000 + 16)) == 3        # workspace must be 256-byte aligned


def test_decode_rejects_bad_arguments(L):
    def call(d=128, Hv=48, layers=48, state=_p(), q=_p()):
        return L.gdn_decode_step(q, _p(), _p(), _p(), _p(), _p(), _p(), 4, layers, 16, Hv, d,
                                 0.088, state, _p(), None)
    assert call(d=256) == 2
    assert call(Hv=47) == 2
    assert call(layers=0) == 1
    assert call(state=None) == 1
    assert call(q=_p(FAKE + 2)) == 3
    # zero sequences: nothing to do, no launch
    assert L.gdn_decode_step(None, None, None, None, None, None, None, 0, 48, 16, 48, 128, 0.1,
                             None, None, None) == 0


def test_conv_rejects_bad_arguments(L):
    def call(d=128, T=16, conv_w=_p(), cs_in=None, cs_out=None, q=_p()):
        return L.gdn_conv1d_silu(_p(), conv_w, None, 1, T, 16, 48, d, cs_in, cs_out, q, _p(), _p(),
                                 None)
    assert call(d=64) == 2
    assert call(conv_w=None) == 1
    assert call(q=None) == 1
    assert call(cs_in=_p(0x30000), cs_out=_p(0x30000)) == 1      # in/out state must differ
    assert call(q=_p(FAKE + 8)) == 3


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from gated_deltanet_recurrence_prefill_b200 import _lib
    monkeypatch.setattr(_lib, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.lib()


def test_fused_decode_rejects_bad_arguments(L):
    def call(d=128, Hv=48, layers=48, n_seq=4, n_slots=4, slot=None, state=_p(), qkv=_p()):
        return L.gdn_decode_step_fused(qkv, _p(), _p(), _p(), _p(), _p(), _p(), slot, n_seq, layers,
                                       16, Hv, d, 0.088, n_slots, state, _p(), None)
    assert call(d=64) == 2
    assert call(Hv=47) == 2
    assert call(layers=0) == 1
    assert call(n_slots=0) == 1
    assert call(n_slots=3) == 1                  # identity slots need n_slots >= n_seq
    assert call(qkv=None) == 1
    assert call(state=_p(FAKE + 8)) == 3         # misaligned
    assert call(n_seq=0) == 0                    # nothing to do


def test_bf16_state_decode_rejects_bad_arguments(L):
    def call(d=128, Hv=48, layers=48, state=_p()):
        return L.gdn_decode_step_bf16(_p(), _p(), _p(), _p(), _p(), _p(), _p(), 4, layers, 16, Hv, d,
                                      0.088, state, _p(), None)
    assert call(d=64) == 2
    assert call(Hv=47) == 2
    assert call(layers=0) == 1
    assert call(state=None) == 1
    assert call(state=_p(FAKE + 2)) == 3


def test_gated_norm_rejects_bad_arguments(L):
    def call(o=_p(), z=_p(), w=_p(), T=8, Hv=48, d=128, layers=1, eps=1e-6, y=_p()):
        return L.gdn_gated_norm(o, z, w, T, Hv, d, layers, eps, y, None)
    assert call(d=64) == 2                        # unsupported head width
    assert call(T=-1) == 1
    assert call(Hv=0) == 1
    assert call(layers=0) == 1
    assert call(eps=-1.0) == 1
    assert call(eps=float("nan")) == 1
    assert call(z=None) == 1
    assert call(y=None) == 1
    assert call(o=_p(FAKE + 4)) == 3              # misaligned
    assert call(T=0, o=None, z=None, w=None, y=None) == 0   # nothing to do, nothing read


def test_prefill_gated_rejects_bad_arguments(L):
    ws = L.gdn_prefill_workspace_size(1, 64, 16, 48, 128)

    def call(z=_p(), w=_p(), y=_p(), o=None, eps=1e-6, d=128, wsp=_p(0x20000), wsb=ws):
        return L.gdn_prefill_gated(_p(), _p(), _p(), _p(), _p(), _p(), _p(), None, 1, 64, 16, 48, d, 0.088,
                                   None, None, o, z, w, eps, y, wsp, wsb, None)
    assert call(d=64) == 2
    assert call(z=None) == 1
    assert call(w=None) == 1
    assert call(y=None) == 1
    assert call(eps=-1.0) == 1
    assert call(y=_p(FAKE + 8)) == 3
    assert call(wsp=None) == 6
    assert call(wsb=16) == 6


def test_decode_gated_rejects_bad_arguments(L):
    def call(d=128, sb=0, z=_p(), w=_p(), y=_p(), eps=1e-6, layers=48):
        return L.gdn_decode_step_gated(_p(), _p(), _p(), _p(), _p(), _p(), _p(), 4, layers, 16, 48, d, 0.088,
                                       _p(), sb, None, z, w, eps, y, None)
    assert call(d=64) == 2
    assert call(sb=2) == 1
    assert call(z=None) == 1
    assert call(w=None) == 1
    assert call(y=None) == 1
    assert call(eps=-0.5) == 1
    assert call(layers=0) == 1
    assert call(y=_p(FAKE + 2)) == 3


def test_backward_workspace_formula(L):
    # gdn.h: checkpoints + one chunk of states per unit + dq, dk per value head + gate sums
    for n, T, Hv in ((1, 8192, 48), (16, 241567, 48), (3, 100, 6)):
        d = 128
        want = ((T // 64 + n + 1) * Hv * d * d * 4 + n * Hv * 64 * d * d * 4 + 2 * T * Hv * d * 4
                + n * Hv * 2 * 4)
        want = (want + 255) // 256 * 256
        assert L.gdn_prefill_backward_workspace_size(n, T, Hv, d) == want


def test_backward_rejects_bad_arguments(L):
    ws = L.gdn_prefill_backward_workspace_size(1, 64, 48, 128)

    def call(d=128, d_o=_p(), dq=_p(), dA=_p(), wsp=_p(0x20000), wsb=ws):
        return L.gdn_prefill_backward(_p(), _p(), _p(), _p(), _p(), _p(), _p(), None, 1, 64, 16, 48, d, 0.088,
                                      None, d_o, None, dq, _p(), _p(), _p(), _p(), dA, _p(), None, wsp, wsb, None)
    assert call(d=64) == 2
    assert call(d_o=None) == 1
    assert call(dq=None) == 1
    assert call(dA=None) == 1
    assert call(dq=_p(FAKE + 4)) == 3
    assert call(wsb=ws - 256) == 6
    assert call(wsp=_p(0x20000 + 16)) == 3


def test_chunked_backward_workspace_formula(L):
    # gdn.h: a 256-byte header (the error word); per (slot, value head) W, U',
    # T, Y, S, dS and the decays; dq, dk per value head; the chunk list and gate
    # sums, each region rounded to 256 bytes
    r = lambda x: (x + 255) // 256 * 256
    for n, T, Hv in ((1, 8192, 48), (16, 241567, 48), (3, 100, 6)):
        d = 128
        sh = (T // 64 + n + 1) * Hv
        want = (256 + r((T // 64 + n + 1) * 2 * 4) + 2 * r(sh * 64 * d * 4) + r(sh * 64 * 64 * 4)
                + 3 * r(sh * d * d * 4) + r(sh * 65 * 4) + 2 * r(T * Hv * d * 4) + r(sh * 2 * 4))
        assert L.gdn_prefill_backward_chunked_workspace_size(n, T, Hv, d) == want


def test_chunked_backward_rejects_bad_arguments(L):
    ws = L.gdn_prefill_backward_chunked_workspace_size(1, 64, 48, 128)

    def call(d=128, d_o=_p(), dq=_p(), dA=_p(), wsp=_p(0x20000), wsb=ws):
        return L.gdn_prefill_backward_chunked(_p(), _p(), _p(), _p(), _p(), _p(), _p(), None, 1, 64, 16, 48, d,
                                              0.088, None, d_o, None, dq, _p(), _p(), _p(), _p(), dA, _p(), None,
                                              wsp, wsb, None)
    assert call(d=64) == 2
    assert call(d_o=None) == 1
    assert call(dq=None) == 1
    assert call(dA=None) == 1
    assert call(dq=_p(FAKE + 4)) == 3
    assert call(wsb=ws - 256) == 6
    assert call(wsp=_p(0x20000 + 16)) == 3


def test_front_backward_workspace_formula(L):
    # gdn.h: ceil(T / 32) * Ctot * 4 floats, rounded up to 256 bytes; 0 for T = 0
    for T, Hqk, Hv in ((8192, 16, 48), (100, 2, 6), (1, 1, 1)):
        want = -(-T // 32) * (2 * Hqk + Hv) * 128 * 4 * 4
        assert L.gdn_conv1d_silu_backward_workspace_size(T, Hqk, Hv, 128) == (want + 255) // 256 * 256
    assert L.gdn_conv1d_silu_backward_workspace_size(0, 16, 48, 128) == 0


def test_front_backward_rejects_bad_arguments(L):
    ws = L.gdn_conv1d_silu_backward_workspace_size(64, 16, 48, 128)

    def call(d=128, w=_p(), dq=_p(), dw=_p(), dx=_p(), wsp=_p(0x20000), wsb=ws, n_seq=1, cu=None):
        return L.gdn_conv1d_silu_backward(_p(), w, cu, n_seq, 64, 16, 48, d, None, dq, _p(), _p(), dx, dw, None,
                                          wsp, wsb, None)
    assert call(d=64) == 2
    assert call(w=None) == 1
    assert call(dw=None) == 1
    assert call(dq=None) == 1
    assert call(dx=None) == 1
    assert call(n_seq=2) == 1          # several sequences need cu_seqlens
    assert call(dx=_p(FAKE + 4)) == 3
    assert call(wsb=ws - 256) == 6
    assert call(wsp=None) == 6
    assert call(wsp=_p(0x20000 + 16)) == 3


def test_norm_backward_workspace_formula(L):
    # gdn.h: per-tile partials ceil(T/8) * ceil(Hv/8) * 8 * d and per-chunk sums
    # layers * ceil(ceil(T/layers)/64) * d floats, each rounded to 256 bytes
    r = lambda x: (x + 255) // 256 * 256
    for T, Hv, layers in ((8192, 48, 1), (6144, 48, 48), (100, 6, 3)):
        want = r(-(-T // 8) * -(-Hv // 8) * 8 * 128 * 4) + r(layers * -(-(-(-T // layers)) // 64) * 128 * 4)
        assert L.gdn_gated_norm_backward_workspace_size(T, Hv, 128, layers) == want
    assert L.gdn_gated_norm_backward_workspace_size(0, 48, 128, 1) == 0


def test_norm_backward_rejects_bad_arguments(L):
    ws = L.gdn_gated_norm_backward_workspace_size(64, 48, 128, 1)

    def call(d=128, layers=1, eps=1e-6, o=_p(), dy=_p(), dw=_p(), wsp=_p(0x20000), wsb=ws):
        return L.gdn_gated_norm_backward(o, _p(), _p(), dy, 64, 48, d, layers, eps, _p(), _p(), dw, wsp, wsb,
                                         None)
    assert call(d=64) == 2
    assert call(layers=0) == 1
    assert call(eps=-1.0) == 1
    assert call(o=None) == 1
    assert call(dy=None) == 1
    assert call(dw=None) == 1
    assert call(o=_p(FAKE + 4)) == 3
    assert call(wsb=ws - 256) == 6
    assert call(wsp=_p(0x20000 + 16)) == 3


def test_selftest_rejects_bad_arguments(L):
    assert L.gdn_selftest_bounded_wait(2, 20000, _p(0x20000), None) == 1     # unknown wait
    assert L.gdn_selftest_bounded_wait(0, 10, _p(0x20000), None) == 1        # below 1 ms
    assert L.gdn_selftest_bounded_wait(0, 10_000_000, _p(0x20000), None) == 1   # above 2 s
    assert L.gdn_selftest_bounded_wait(0, 20000, _p(0x20000 + 16), None) == 3


def test_check_async_rejects_bad_arguments(L):
    """gdn_check_async validates its output word before enqueueing anything."""
    assert L.gdn_check_async(_p(0x20000), None, None) == 1          # no status word
    assert L.gdn_check_async(_p(0x20000), _p(0x30002), None) == 3   # not 4-byte aligned


def test_prefill_bf16_rejects_bad_arguments(L):
    """gdn_prefill_bf16 checks its arguments as gdn_prefill does (no launch)."""
    p = _p()
    ws = _p(0x40000)
    # no output
    assert L.gdn_prefill_bf16(p, p, p, p, p, p, p, None, 1, 64, 16, 48, 128, 0.088, None, None, None,
                              ws, 1 << 20, None) == 1
    # unsupported head size
    assert L.gdn_prefill_bf16(p, p, p, p, p, p, p, None, 1, 64, 16, 48, 64, 0.088, None, None, p,
                              ws, 1 << 20, None) == 2
    # misaligned output
    assert L.gdn_prefill_bf16(p, p, p, p, p, p, p, None, 1, 64, 16, 48, 128, 0.088, None, None, _p(FAKE + 2),
                              ws, 1 << 20, None) == 3


def test_layer_prefill_host_rejects_bad_arguments_on_the_host(L):
    """gdn_layer_prefill_host checks its arguments before touching CUDA."""
    p = _p()
    s0, s1, s2 = _p(0x1000), _p(0x2000), _p(0x3000)   # stand-in stream handles, never used

    def call(qkv=p, T=256, d=128, nb=2, o=p, wsb=1 << 30, su=s1, sd=s2, ws=_p(0x40000)):
        return L.gdn_layer_prefill_host(qkv, p, p, p, p, p, None, None, T, 2, 6, d, 0.088, nb, o, p, None,
                                        ws, wsb, s0, su, sd)

    assert call(d=64) == 2                  # unsupported head width
    assert call(nb=0) == 1                  # no ranges
    assert call(nb=5000) == 1               # too many ranges
    assert call(qkv=None) == 1              # no input
    assert call(o=None) == 1                # no output
    assert call(su=s0) == 1                 # copy stream equal to the compute stream
    assert call(sd=s1) == 1                 # the two copy streams equal
    assert call(o=_p(FAKE + 4)) == 3        # misaligned
    assert call(wsb=1024) == 6              # workspace too small
    assert call(ws=_p(0x40010)) == 3        # workspace not 256-byte aligned
    assert call(T=0) == 0                   # nothing to do
    # the workspace formula: a prefill workspace of one range first, then the buffers
    assert L.gdn_layer_prefill_host_workspace_size(256, 2, 6, 64, 2) == 0
    n1 = L.gdn_layer_prefill_host_workspace_size(8192, 16, 48, 128, 8)
    assert n1 > L.gdn_prefill_workspace_size(1, 1024, 16, 48, 128)
    assert n1 % 256 == 0
