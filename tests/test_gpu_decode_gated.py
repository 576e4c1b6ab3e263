"""gdn_decode_step_gated: a decode step with the gated output norm fused in,
against the fp64 oracle (decode step, then gated norm with each unit's layer
weight).  y is bf16: each element within 2^-8 |y_ref| + 1e-6 max |y_ref| of the
oracle's norm of the kernel's own o; the state and o as for the plain step."""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, host, rel_err

pytestmark = pytest.mark.gpu


def _zw(U, Hv, layers, seed):
    rng = np.random.default_rng(seed)
    zb = (rng.standard_normal((U, Hv, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    w = rng.uniform(0.5, 1.5, (layers, 128)).astype(np.float32)
    return zb, w


def _norm_ref(orc, o, zb, w):
    layers = w.shape[0]
    ref = np.empty_like(o)
    for l in range(layers):
        ref[l::layers] = orc.gated_norm(o[l::layers], zb[l::layers], w[l])
    return ref


def _bound_ok(y, ref):
    bound = 2.0 ** -8 * np.abs(ref) + 1e-6 * np.max(np.abs(ref))
    return not (np.abs(y - ref) > bound).any()


@pytest.mark.parametrize("bf16_state", [False, True])
def test_decode_gated_matches_oracle(orc, bf16_state):
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    inp = synth.make_decode(3, 4, seed=45)
    st = inp.full_state()
    st_dev = dev_f32(st)
    if bf16_state:
        st_dev = st_dev.to(torch.bfloat16)
        st = host(st_dev)                          # the oracle starts from the same rounded values
    zb, w = _zw(inp.U, 48, inp.layers, 7)
    y, o = gdn.decode_step_gated(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a),
                                 dev_f32(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias), st_dev,
                                 inp.n_seq, inp.layers, dev_bf16(zb), dev_f32(w), scale=inp.scale,
                                 want_o=True)
    y, o = host(y), host(o)
    o_ref, s_ref = orc.decode(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                              inp.n_seq, inp.layers, st)
    assert rel_err(o, o_ref) <= 1e-4
    assert _bound_ok(y, _norm_ref(orc, o, zb, w))
    assert rel_err(y, _norm_ref(orc, o_ref, zb, w)) <= 1e-2


def test_decode_gated_without_o_and_same_state_as_plain_step():
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    inp = synth.make_decode(2, 3, seed=46, Hqk=4, Hv=8)
    st = inp.full_state()
    s1, s2 = dev_f32(st), dev_f32(st)
    zb, w = _zw(inp.U, 8, inp.layers, 8)
    args = (dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b),
            dev_f32(inp.A_log), dev_f32(inp.dt_bias))
    y, o = gdn.decode_step_gated(*args, s1, inp.n_seq, inp.layers, dev_bf16(zb), dev_f32(w), scale=inp.scale)
    o2 = gdn.decode_step(*args, s2, inp.n_seq, inp.layers, scale=inp.scale)
    assert o is None
    assert torch.equal(s1, s2)                     # the state update is the plain step's
    import oracle
    ref = np.empty((inp.U, 8, 128))
    on = host(o2)
    for l in range(inp.layers):
        ref[l::inp.layers] = oracle.gated_norm(on[l::inp.layers], zb[l::inp.layers], w[l])
    assert _bound_ok(host(y), ref)
