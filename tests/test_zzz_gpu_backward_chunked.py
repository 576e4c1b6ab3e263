"""gdn_prefill_backward_chunked against the fp64 oracle's gradient, on the
shapes of the token-by-token backward's tests, with each of its two gradient
kernels:
  * tc (the default): the per-chunk products on the tensor cores with bf16
    operands and float32 accumulation; the tolerance of the bf16 tensor-core
    prefill, max |x - x_ref| / max |x_ref| <= 1e-2 (a float32 model of the
    chunked backward with every product operand rounded to bf16 stays at
    ~5e-3 against the oracle, so 1e-2 holds with room);
  * simt (GDN_BACKWARD_GRAD=simt): float32 on the CUDA cores, <= 2e-3 as for
    the token-by-token kernel.

(Its kernels' source is also run on the CPU under emulation by
test_backward_chunked_emu; this file runs after every other GPU test.)"""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err

pytestmark = pytest.mark.gpu
TOLS = {"tc": 1e-2, "simt": 2e-3}


@pytest.fixture(params=sorted(TOLS))
def tol(request, monkeypatch):
    if request.param == "simt":
        monkeypatch.setenv("GDN_BACKWARD_GRAD", "simt")
    else:
        monkeypatch.delenv("GDN_BACKWARD_GRAD", raising=False)
    return TOLS[request.param]


def _grads_in(inp, seed):
    rng = np.random.default_rng(seed)
    N = len(inp.cu_seqlens) - 1
    d_o = rng.standard_normal((inp.q.shape[0], inp.Hv, 128)).astype(np.float32)
    d_fin = (0.1 * rng.standard_normal((N, inp.Hv, 128, 128))).astype(np.float32)
    return d_o, d_fin


def _run(inp, d_o, d_fin, with_s0=True, chunked=True):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    fn = gdn.prefill_backward_chunked if chunked else gdn.prefill_backward
    s0 = dev_f32(inp.initial_state) if (with_s0 and inp.initial_state is not None) else None
    return fn(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b),
              dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_f32(d_o),
              d_final_state=None if d_fin is None else dev_f32(d_fin), cu_seqlens=dev_i32(inp.cu_seqlens),
              scale=inp.scale, initial_state=s0)


def _compare(got, ref, tol):
    pairs = [("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("da", "da"), ("db", "db"), ("dA_log", "dA_log"),
             ("ddt_bias", "ddt_bias"), ("d_initial_state", "d_initial")]
    for gname, rname in pairs:
        if got[gname] is None:
            continue
        err = rel_err(host(got[gname]), ref[rname])
        assert err <= tol, f"{gname}: {err}"


@pytest.mark.parametrize("Hqk,Hv", [(2, 6), (4, 12)])
def test_chunked_backward_varlen(orc, tol, Hqk, Hv):
    lengths = [1, 63, 64, 0, 65, 130]
    inp = synth.make_prefill(lengths, seed=80, init_state=True, init_std=0.05, Hqk=Hqk, Hv=Hv)
    d_o, d_fin = _grads_in(inp, 1)
    ref = orc.prefill_backward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias, d_o, d_final=d_fin,
                               cu_seqlens=inp.cu_seqlens, scale=inp.scale, initial_state=inp.initial_state)
    _compare(_run(inp, d_o, d_fin), ref, tol)


def test_chunked_backward_no_state_gradients(orc, tol):
    inp = synth.make_prefill([150, 20], seed=81, init_state=False, Hqk=2, Hv=6)
    d_o, _ = _grads_in(inp, 2)
    ref = orc.prefill_backward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias, d_o,
                               cu_seqlens=inp.cu_seqlens, scale=inp.scale)
    _compare(_run(inp, d_o, None, with_s0=False), ref, tol)


def test_chunked_backward_deterministic_and_equal_to_token_by_token(tol):
    import torch
    inp = synth.make_prefill([200, 37], seed=82, init_state=True, Hqk=2, Hv=6)
    d_o, d_fin = _grads_in(inp, 3)
    g1, g2 = _run(inp, d_o, d_fin), _run(inp, d_o, d_fin)
    for name in g1:
        assert torch.equal(g1[name], g2[name]), name
    g3 = _run(inp, d_o, d_fin, chunked=False)
    for name in g1:
        x, r = host(g1[name]), host(g3[name])
        assert rel_err(x, r) <= tol, name


def test_chunked_backward_2k_full_heads_sampled(orc, tol):
    # 2048 tokens with the full 16 / 48 heads in one call; two value heads (with
    # their key heads) against the oracle on those heads alone
    inp = synth.make_prefill([2048], seed=83, init_state=True)
    d_o, d_fin = _grads_in(inp, 4)
    got = {n: (None if x is None else host(x)) for n, x in _run(inp, d_o, d_fin).items()}

    def one_head(hh):
        gk = hh // 3
        return orc.prefill_backward(inp.q[:, gk:gk + 1], inp.k[:, gk:gk + 1], inp.v[:, hh:hh + 1],
                                    inp.a[:, hh:hh + 1], inp.b[:, hh:hh + 1], inp.A_log[hh:hh + 1],
                                    inp.dt_bias[hh:hh + 1], d_o[:, hh:hh + 1], d_final=d_fin[:, hh:hh + 1],
                                    scale=inp.scale, initial_state=inp.initial_state[:, hh:hh + 1])

    for h in (0, 31):
        gk = h // 3
        ref = one_head(h)
        for gname, rname in (("dv", "dv"), ("da", "da"), ("db", "db"), ("d_initial_state", "d_initial")):
            assert rel_err(got[gname][:, h:h + 1], ref[rname]) <= tol, (h, gname)
        for gname in ("dA_log", "ddt_bias"):
            assert rel_err(got[gname][h:h + 1], ref[gname]) <= tol, (h, gname)
        # dq, dk of key head gk sum its three value heads
        refs = [ref if hh == h else one_head(hh) for hh in range(3 * gk, 3 * gk + 3)]
        assert rel_err(got["dq"][:, gk:gk + 1], sum(r["dq"] for r in refs)) <= tol, h
        assert rel_err(got["dk"][:, gk:gk + 1], sum(r["dk"] for r in refs)) <= tol, h


def test_chunked_backward_strong_decay(orc, tol):
    """Strong in-chunk decay on some heads (log alpha down to ~-40 per token):
    kappa and gamma underflow inside a chunk, the transitions between chunks are
    nearly zero; the gradients still match the oracle's."""
    inp = synth.make_prefill([300, 77], seed=84, init_state=True, init_std=0.05, Hqk=2, Hv=6)
    inp.A_log[:3] = np.float32(np.log(16.0))
    inp.a[:, :3] = 3.0
    d_o, d_fin = _grads_in(inp, 5)
    ref = orc.prefill_backward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias, d_o, d_final=d_fin,
                               cu_seqlens=inp.cu_seqlens, scale=inp.scale, initial_state=inp.initial_state)
    _compare(_run(inp, d_o, d_fin), ref, tol)
