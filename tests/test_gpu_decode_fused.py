"""Decode step with the front end fused in, on the GPU, against the fp64 oracle
composed of its front end (one token per sequence, the carried convolution
history as the initial history) and its decode step.  Tolerance 1e-4 (global
max-normalised) for o and the states, as for the plain decode step: the
kernel keeps q, k and v in float32.  The convolution history is rewritten with
exact copies of its inputs, so it must match bit for bit."""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _oracle(orc, inp, qkv, a, b, conv_state, state):
    """One fused step for all units; returns (o [U,Hv,d], state, conv_state)
    with the slots' entries updated (float64 copies of the inputs)."""
    L, n_seq, Hqk, Hv, d = inp.layers, inp.n_seq, inp.Hqk, inp.Hv, inp.d
    U = n_seq * L
    q = np.zeros((U, Hqk, d)); k = np.zeros((U, Hqk, d)); v = np.zeros((U, Hv, d))
    cs_new = conv_state.astype(np.float64).copy()
    cu = np.arange(n_seq + 1, dtype=np.int32)
    for l in range(L):
        units = np.arange(n_seq) * L + l
        rows = inp.slot.astype(np.int64) * L + l
        ql, kl, vl, cso = orc.conv1d_silu(qkv[units], inp.conv_w[l], cu, Hqk, Hv, d,
                                          conv_state=conv_state[rows])
        q[units], k[units], v[units] = ql, kl, vl
        cs_new[rows] = cso
    st_units = state[(inp.slot.astype(np.int64)[:, None] * L + np.arange(L)[None, :]).reshape(-1)]
    o, so = orc.decode(q, k, v, a, b, inp.A_log, inp.dt_bias, n_seq, L, st_units, scale=inp.scale)
    st_new = state.astype(np.float64).copy()
    st_new[(inp.slot.astype(np.int64)[:, None] * L + np.arange(L)[None, :]).reshape(-1)] = so
    return o, st_new, cs_new


def _gpu(inp, qkv, a, b, cs_dev, st_dev, slot=True):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    return gdn.decode_step_fused(dev_bf16(qkv), dev_f32(inp.conv_w), cs_dev, dev_f32(a), dev_f32(b),
                                 dev_f32(inp.A_log), dev_f32(inp.dt_bias), st_dev, inp.n_seq,
                                 inp.layers, inp.Hqk, inp.Hv, slot=dev_i32(inp.slot) if slot else None,
                                 scale=inp.scale)


@pytest.mark.parametrize("Hqk,Hv", [(16, 48), (4, 8), (2, 2)])
def test_fused_decode_matches_oracle(orc, Hqk, Hv):
    inp = synth.make_decode_fused(3, 2, 5, 70, Hqk=Hqk, Hv=Hv)
    cs_dev, st_dev = dev_f32(inp.conv_state), dev_f32(inp.state)
    o = _gpu(inp, inp.qkv, inp.a, inp.b, cs_dev, st_dev)
    o_ref, st_ref, cs_ref = _oracle(orc, inp, inp.qkv, inp.a, inp.b, inp.conv_state, inp.state)
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(st_dev), st_ref) <= TOL
    np.testing.assert_array_equal(host(cs_dev), cs_ref)


def test_fused_decode_two_steps_carry_the_history(orc):
    """Two steps in a row: the second reads the convolution history and the
    state the first one left."""
    inp = synth.make_decode_fused(2, 3, 4, 71, Hqk=4, Hv=12)
    nxt = synth.make_decode_fused(2, 3, 4, 72, Hqk=4, Hv=12)       # the next token's inputs
    cs_dev, st_dev = dev_f32(inp.conv_state), dev_f32(inp.state)
    _gpu(inp, inp.qkv, inp.a, inp.b, cs_dev, st_dev)
    o2 = _gpu(inp, nxt.qkv, nxt.a, nxt.b, cs_dev, st_dev)
    _, st1, cs1 = _oracle(orc, inp, inp.qkv, inp.a, inp.b, inp.conv_state, inp.state)
    o_ref, st2, cs2 = _oracle(orc, inp, nxt.qkv, nxt.a, nxt.b, cs1.astype(np.float32),
                              st1.astype(np.float32))
    assert rel_err(host(o2), o_ref) <= TOL
    assert rel_err(host(st_dev), st2) <= TOL
    np.testing.assert_array_equal(host(cs_dev), cs2)


def test_fused_decode_leaves_other_slots_alone():
    import torch
    inp = synth.make_decode_fused(3, 2, 8, 73, Hqk=2, Hv=6)
    cs_dev, st_dev = dev_f32(inp.conv_state), dev_f32(inp.state)
    _gpu(inp, inp.qkv, inp.a, inp.b, cs_dev, st_dev)
    L = inp.layers
    untouched = sorted(set(range(inp.n_slots)) - set(int(s) for s in inp.slot))
    rows = [s * L + l for s in untouched for l in range(L)]
    idx = torch.tensor(rows, device="cuda")
    assert torch.equal(st_dev[idx], dev_f32(inp.state)[idx])
    assert torch.equal(cs_dev[idx], dev_f32(inp.conv_state)[idx])


def test_fused_decode_identity_slots_and_determinism():
    """slot = NULL means sequence n in slot n; the result is bitwise repeatable."""
    import torch
    inp = synth.make_decode_fused(3, 2, 3, 74, Hqk=4, Hv=8)
    inp.slot = np.arange(3, dtype=np.int32)
    runs = []
    for use_slot in (True, False):
        cs_dev, st_dev = dev_f32(inp.conv_state), dev_f32(inp.state)
        o = _gpu(inp, inp.qkv, inp.a, inp.b, cs_dev, st_dev, slot=use_slot)
        runs.append((o, st_dev, cs_dev))
    for x, y in zip(runs[0], runs[1]):
        assert torch.equal(x, y)


def test_fused_decode_bf16_state(orc):
    """bf16-state variant of the fused step: o within 1e-4 of the oracle started
    from the same bf16 state values, every stored state element within one bf16
    rounding, the convolution history bit for bit."""
    import torch
    inp = synth.make_decode_fused(3, 2, 4, 75, Hqk=4, Hv=12)
    st16 = torch.from_numpy(inp.state).cuda().to(torch.bfloat16)
    st_in = host(st16).astype(np.float32)
    cs_dev = dev_f32(inp.conv_state)
    import gated_deltanet_recurrence_prefill_b200 as gdn
    o = gdn.decode_step_fused(dev_bf16(inp.qkv), dev_f32(inp.conv_w), cs_dev, dev_f32(inp.a),
                              dev_f32(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias), st16,
                              inp.n_seq, inp.layers, inp.Hqk, inp.Hv, slot=dev_i32(inp.slot),
                              scale=inp.scale)
    o_ref, st_ref, cs_ref = _oracle(orc, inp, inp.qkv, inp.a, inp.b, inp.conv_state, st_in)
    assert rel_err(host(o), o_ref) <= TOL
    got = host(st16)
    bound = 2.0 ** -8 * np.abs(st_ref) + 1e-5 * np.max(np.abs(st_ref))
    assert not (np.abs(got - st_ref) > bound).any()
    np.testing.assert_array_equal(host(cs_dev), cs_ref)
