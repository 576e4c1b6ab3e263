"""gdn_prefill_backward against the fp64 oracle's reverse-mode gradient (itself
pinned by finite differences of the forward).  The kernel computes in float32,
one token at a time; every gradient is compared with max |x - x_ref| / max
|x_ref| <= 2e-3 (float32 rounding accumulated over a few hundred steps)."""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _grads_in(inp, seed):
    rng = np.random.default_rng(seed)
    d_o = rng.standard_normal((inp.T, inp.Hv, 128)).astype(np.float32)
    d_fin = (0.1 * rng.standard_normal((inp.N, inp.Hv, 128, 128))).astype(np.float32)
    return d_o, d_fin


def _run(inp, d_o, d_fin, with_s0=True):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    s0 = dev_f32(inp.initial_state) if (with_s0 and inp.initial_state is not None) else None
    return gdn.prefill_backward(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a),
                                dev_f32(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias), dev_f32(d_o),
                                d_final_state=None if d_fin is None else dev_f32(d_fin),
                                cu_seqlens=dev_i32(inp.cu_seqlens), scale=inp.scale, initial_state=s0)


def _oracle(orc, inp, d_o, d_fin, with_s0=True):
    return orc.prefill_backward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias, d_o,
                                d_final=d_fin, cu_seqlens=inp.cu_seqlens, scale=inp.scale,
                                initial_state=inp.initial_state if with_s0 else None)


def _compare(got, ref):
    pairs = [("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("da", "da"), ("db", "db"), ("dA_log", "dA_log"),
             ("ddt_bias", "ddt_bias"), ("d_initial_state", "d_initial")]
    for gname, rname in pairs:
        if got[gname] is None:
            continue
        err = rel_err(host(got[gname]), ref[rname])
        assert err <= TOL, f"{gname}: {err}"


@pytest.mark.parametrize("Hqk,Hv", [(2, 6), (4, 12)])
def test_backward_varlen(orc, Hqk, Hv):
    lengths = [1, 63, 64, 0, 65, 130]
    inp = synth.make_prefill(lengths, seed=80, init_state=True, init_std=0.05, Hqk=Hqk, Hv=Hv)
    d_o, d_fin = _grads_in(inp, 1)
    _compare(_run(inp, d_o, d_fin), _oracle(orc, inp, d_o, d_fin))


def test_backward_no_state_gradients(orc):
    # no initial state, no dL/dS_T: only the outputs' gradient flows
    inp = synth.make_prefill([150, 20], seed=81, init_state=False, Hqk=2, Hv=6)
    d_o, _ = _grads_in(inp, 2)
    _compare(_run(inp, d_o, None, with_s0=False), _oracle(orc, inp, d_o, None, with_s0=False))


def test_backward_deterministic():
    import torch
    inp = synth.make_prefill([200], seed=82, init_state=True, Hqk=2, Hv=6)
    d_o, d_fin = _grads_in(inp, 3)
    g1, g2 = _run(inp, d_o, d_fin), _run(inp, d_o, d_fin)
    for name in g1:
        assert torch.equal(g1[name], g2[name]), name


def test_backward_2k_sampled_head(orc):
    # one sequence of 2048 tokens with the full 16 / 48 heads in one launch; two value
    # heads (with their key heads) checked against the oracle run on those heads alone
    inp = synth.make_prefill([2048], seed=83, init_state=True)
    d_o, d_fin = _grads_in(inp, 4)
    got = _run(inp, d_o, d_fin)
    for h in (0, 31):
        gk = h // 3
        ref = orc.prefill_backward(inp.q[:, gk:gk + 1], inp.k[:, gk:gk + 1], inp.v[:, h:h + 1], inp.a[:, h:h + 1],
                                   inp.b[:, h:h + 1], inp.A_log[h:h + 1], inp.dt_bias[h:h + 1], d_o[:, h:h + 1],
                                   d_final=d_fin[:, h:h + 1], scale=inp.scale,
                                   initial_state=inp.initial_state[:, h:h + 1])
        assert rel_err(host(got["dv"][:, h:h + 1]), ref["dv"]) <= TOL
        assert rel_err(host(got["da"][:, h:h + 1]), ref["da"]) <= TOL
        assert rel_err(host(got["db"][:, h:h + 1]), ref["db"]) <= TOL
        assert rel_err(host(got["d_initial_state"][:, h:h + 1]), ref["d_initial"]) <= TOL
        # dq, dk of key head gk sum three value heads: compare the sum of the oracle's three
        dq = np.zeros_like(ref["dq"])
        dk = np.zeros_like(ref["dk"])
        for hh in range(3 * gk, 3 * gk + 3):
            rr = ref if hh == h else orc.prefill_backward(
                inp.q[:, gk:gk + 1], inp.k[:, gk:gk + 1], inp.v[:, hh:hh + 1], inp.a[:, hh:hh + 1],
                inp.b[:, hh:hh + 1], inp.A_log[hh:hh + 1], inp.dt_bias[hh:hh + 1], d_o[:, hh:hh + 1],
                d_final=d_fin[:, hh:hh + 1], scale=inp.scale, initial_state=inp.initial_state[:, hh:hh + 1])
            dq += rr["dq"]
            dk += rr["dk"]
        assert rel_err(host(got["dq"][:, gk:gk + 1]), dq) <= TOL
        assert rel_err(host(got["dk"][:, gk:gk + 1]), dk) <= TOL
