"""Decode step on the GPU against the fp64 oracle (tolerance 1e-4, global
max-normalised, for o and the updated state)."""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, host, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _run(inp, state_dev):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    return gdn.decode_step(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a),
                           dev_f32(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias), state_dev,
                           inp.n_seq, inp.layers, scale=inp.scale)


def test_decode_small_all_units(orc):
    inp = synth.make_decode(3, 4, seed=40)
    st = inp.full_state()
    st_dev = dev_f32(st)
    o = _run(inp, st_dev)
    o_ref, s_ref = orc.decode(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                              inp.n_seq, inp.layers, st)
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(st_dev), s_ref) <= TOL


def test_decode_other_head_counts(orc):
    inp = synth.make_decode(2, 2, seed=41, Hqk=4, Hv=8)
    st = inp.full_state()
    st_dev = dev_f32(st)
    o = _run(inp, st_dev)
    o_ref, s_ref = orc.decode(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                              inp.n_seq, inp.layers, st)
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(st_dev), s_ref) <= TOL


def test_decode_is_deterministic_and_in_place():
    import torch
    inp = synth.make_decode(2, 3, seed=42)
    st = inp.full_state()
    a_dev, b_dev = dev_f32(st), dev_f32(st)
    o1 = _run(inp, a_dev)
    o2 = _run(inp, b_dev)
    assert torch.equal(o1, o2) and torch.equal(a_dev, b_dev)
    assert not torch.equal(a_dev, dev_f32(st))      # the state moved


@pytest.mark.slow
def test_decode_full_size_sampled_units(orc):
    """128 sequences x 48 layers (19.3 GB of float32 state), one launch as the
    benchmark times it; 12 units spread over the range are checked against the
    oracle."""
    import torch
    from concurrent.futures import ThreadPoolExecutor
    inp = synth.workload(4)
    st_dev = torch.empty(inp.U, inp.Hv, inp.d, inp.d, dtype=torch.float32, device="cuda")
    upb = inp.units_per_block
    with ThreadPoolExecutor(8) as ex:
        for blk, s in enumerate(ex.map(inp.state_block, range(inp.n_state_blocks()))):
            st_dev[blk * upb: blk * upb + len(s)].copy_(torch.from_numpy(s))
    o = _run(inp, st_dev)
    rng = np.random.default_rng(0)
    units = sorted({0, 1, inp.layers - 1, inp.U - 1, *rng.integers(0, inp.U, 8).tolist()})
    s0 = inp.state_of_units(units)
    o_ref, s_ref = orc.decode(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                              inp.n_seq, inp.layers, s0, units=units)
    idx = torch.tensor(units, device="cuda")
    assert rel_err(host(o[idx]), o_ref) <= TOL
    assert rel_err(host(st_dev[idx]), s_ref) <= TOL


def _bf16_state_check(got, ref):
    """Each stored element within one bf16 rounding of the exact value."""
    got = np.asarray(got, np.float64)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.max(np.abs(ref))
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} state elements beyond one bf16 ulp"


@pytest.mark.parametrize("Hqk,Hv", [(16, 48), (4, 8)])
def test_decode_bf16_state(orc, Hqk, Hv):
    """bf16-state variant: the oracle starts from the same (bf16) state values;
    o within 1e-4, every stored state element within one bf16 rounding."""
    import torch
    inp = synth.make_decode(2, 3, seed=43, Hqk=Hqk, Hv=Hv)
    st16 = torch.from_numpy(inp.full_state()).cuda().to(torch.bfloat16)
    st_in = host(st16).astype(np.float32)
    o = _run(inp, st16)
    o_ref, s_ref = orc.decode(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                              inp.n_seq, inp.layers, st_in)
    assert rel_err(host(o), o_ref) <= TOL
    _bf16_state_check(host(st16), s_ref)
