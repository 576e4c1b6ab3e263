"""gdn_prefill_gated: the chunked prefill with the gated output norm fused into
its output path, against the fp64 oracle (recurrence, then gated norm).

Two checks per case:
- y against the oracle's norm of the kernel's own o (isolates the fused norm):
  per element within 2^-8 |y_ref| + 1e-6 max |y_ref| (bf16 output);
- y against the oracle's norm of the oracle's o (the whole layer tail):
  max |y - y_ref| / max |y_ref| <= 2e-2 (the recurrence's own 1e-2 on o passes
  through the per-row normalisation).
"""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err
from tests.test_gpu_prefill import KERNELS, kernel  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu


def _z_w(T, Hv, seed):
    rng = np.random.default_rng(seed)
    zb = (rng.standard_normal((T, Hv, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    w = rng.uniform(0.5, 1.5, 128).astype(np.float32)
    return zb, w


def _run(inp, zb, w, eps=1e-6, want_o=True):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    s0 = None if inp.initial_state is None else dev_f32(inp.initial_state)
    return gdn.prefill_gated(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a),
                             dev_f32(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_bf16(zb),
                             dev_f32(w), eps=eps, cu_seqlens=dev_i32(inp.cu_seqlens), scale=inp.scale,
                             initial_state=s0, want_o=want_o)


def _check_norm_of(y, o, zb, w, eps=1e-6):
    ref = __import__("oracle").gated_norm(o, zb, w, eps=eps)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-6 * np.max(np.abs(ref))
    bad = np.abs(y - ref) > bound
    assert not bad.any(), f"{bad.sum()} elements out of bound"


@pytest.mark.parametrize("Hqk,Hv", [(4, 12), (2, 6)])
def test_prefill_gated_varlen(kernel, norm_mode, orc, Hqk, Hv):
    lengths = [1, 63, 64, 0, 65, 127, 129, 200]
    inp = synth.make_prefill(lengths, seed=70, init_state=True, init_std=0.05, Hqk=Hqk, Hv=Hv)
    zb, w = _z_w(inp.T, Hv, 1)
    y, o, fs = _run(inp, zb, w)
    y, o = host(y), host(o)
    _check_norm_of(y, o, zb, w)
    o_ref, s_ref = orc.prefill(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                               cu_seqlens=inp.cu_seqlens, scale=inp.scale, initial_state=inp.initial_state)
    assert rel_err(o, o_ref) < 1e-2
    assert rel_err(host(fs), s_ref) < 1e-2
    assert rel_err(y, orc.gated_norm(o_ref, zb, w)) < 2e-2


@pytest.fixture(params=["auto", "fused"])
def norm_mode(request, monkeypatch):
    # with o requested: the two-pass composition (auto) or the fused kernel forced
    if request.param == "fused":
        monkeypatch.setenv("GDN_PREFILL_NORM", "fused")
    else:
        monkeypatch.delenv("GDN_PREFILL_NORM", raising=False)
    return request.param


def test_prefill_gated_o_matches_plain_prefill(kernel, norm_mode):
    # the fused kernel's o is the plain prefill's o, bit for bit, and y does not
    # depend on whether o is written too
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    inp = synth.make_prefill([300, 77], seed=71, init_state=True, Hqk=4, Hv=12)
    zb, w = _z_w(inp.T, 12, 2)
    y1, o1, s1 = _run(inp, zb, w, want_o=True)
    o0, s0 = gdn.prefill(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a),
                         dev_f32(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias),
                         cu_seqlens=dev_i32(inp.cu_seqlens), scale=inp.scale,
                         initial_state=dev_f32(inp.initial_state))
    assert torch.equal(o1, o0) and torch.equal(s1, s0)
    if kernel != "single":
        # without o the norm is fused: the same y up to the rounding of the two
        # norm implementations (bit for bit when the fused kernel was forced)
        y2, o2, _ = _run(inp, zb, w, want_o=False)
        assert o2 is None
        if norm_mode == "fused":
            assert torch.equal(y1, y2)
        else:
            _check_norm_of(host(y2), host(o1), zb, w)


def test_prefill_gated_eps_and_zero_gate(kernel, norm_mode):
    inp = synth.make_prefill([130], seed=72, init_state=False, Hqk=4, Hv=12)
    zb, w = _z_w(inp.T, 12, 3)
    zb[5] = 0                                      # silu(0) = 0: token 5 gives y = 0
    y, o, _ = _run(inp, zb, w, eps=0.25)
    y, o = host(y), host(o)
    assert np.all(y[5] == 0)
    _check_norm_of(y, o, zb, w, eps=0.25)


def test_prefill_gated_single_kernel_needs_o(monkeypatch):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    monkeypatch.setenv("GDN_PREFILL_KERNEL", "single")
    inp = synth.make_prefill([64], seed=73, init_state=False, Hqk=4, Hv=12)
    zb, w = _z_w(inp.T, 12, 4)
    with pytest.raises(gdn.GdnError, match="WORKSPACE"):
        _run(inp, zb, w, want_o=False)


def test_prefill_gated_8k_sampled(orc):
    # the bench configuration: T = 8192, 16 / 48 heads, one launch; sampled value heads
    # checked against the oracle (recurrence and norm, head by head)
    inp = synth.make_prefill([8192], seed=74, init_state=False)
    zb, w = _z_w(inp.T, 48, 5)
    y, _, _ = _run(inp, zb, w, want_o=False)
    y = host(y)
    for h in (0, 17, 47):
        o_ref, _ = orc.prefill(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                               scale=inp.scale, heads=(h, h + 1))
        ref = orc.gated_norm(o_ref[:, :1], zb[:, h:h + 1], w)
        assert rel_err(y[:, h:h + 1], ref) < 2e-2, h
