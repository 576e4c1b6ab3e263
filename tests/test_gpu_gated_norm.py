"""Gated output norm (gdn_gated_norm) against the fp64 oracle.

y is bf16 (round to nearest even), so each element may differ from the fp64
value by half a bf16 ulp (2^-9 relative) plus the float32 arithmetic before the
rounding; the bound used is 2^-8 |y_ref| + 1e-6 max |y_ref| per element.
"""
import numpy as np
import pytest

import oracle
from tests.helpers import dev_bf16, dev_f32, host

pytestmark = pytest.mark.gpu

TOL_REL = 2.0 ** -8


def _inputs(T, Hv, d=128, layers=1, seed=0, o_scale=1.0, z_scale=2.0):
    rng = np.random.default_rng(seed)
    # per-row magnitudes spanning several decades, so that the norm matters
    mag = np.exp(rng.uniform(-4, 4, (T, Hv, 1)))
    o = (o_scale * mag * rng.standard_normal((T, Hv, d))).astype(np.float32)
    z32 = (z_scale * rng.standard_normal((T, Hv, d))).astype(np.float32)
    zb = (z32.view(np.uint32) >> 16).astype(np.uint16)          # bf16 bits (truncation is fine for inputs)
    w = rng.uniform(0.5, 1.5, (layers, d)).astype(np.float32)
    return o, zb, w


def _check(y_dev, o, zb, w, eps=1e-6):
    y = host(y_dev)
    T, Hv, d = o.shape
    layers = w.shape[0]
    ref = np.empty((T, Hv, d))
    for l in range(layers):
        ref[l::layers] = oracle.gated_norm(o[l::layers], zb[l::layers], w[l], eps=eps)
    bound = TOL_REL * np.abs(ref) + 1e-6 * np.max(np.abs(ref))
    bad = np.abs(y - ref) > bound
    assert not bad.any(), f"{bad.sum()} elements out of bound; worst {np.max(np.abs(y - ref) - bound)}"


@pytest.mark.parametrize("T,Hv", [(1, 48), (37, 12), (200, 48)])
def test_gated_norm_matches_oracle(T, Hv):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    o, zb, w = _inputs(T, Hv, seed=T)
    y = gdn.gated_norm(dev_f32(o), dev_bf16(zb), dev_f32(w[0]))
    _check(y, o, zb, w)


def test_gated_norm_per_layer_weights():
    # decode batch layout: rows are units s * layers + l
    import gated_deltanet_recurrence_prefill_b200 as gdn
    layers = 5
    o, zb, w = _inputs(4 * layers, 48, layers=layers, seed=11)
    y = gdn.gated_norm(dev_f32(o), dev_bf16(zb), dev_f32(w))
    _check(y, o, zb, w)


def test_gated_norm_edge_values():
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T, Hv, d = 6, 4, 128
    o, zb, w = _inputs(T, Hv, seed=5)
    o[0, 0] = 0.0                                  # zero row -> zero output
    o[1, 1] *= 1e-20                               # far below eps: shrunk, not blown up
    o[2, 2] *= 1e15                                # large row: normalised
    z32 = (zb.astype(np.uint32) << 16).view(np.float32)
    z32[3, 0] = 80.0                               # silu(z) ~ z
    z32[3, 1] = -80.0                              # silu(z) ~ -0
    z32[4, 2] = 0.0
    zb = (z32.view(np.uint32) >> 16).astype(np.uint16)
    y = gdn.gated_norm(dev_f32(o), dev_bf16(zb), dev_f32(w[0]))
    assert torch.isfinite(y.float()).all()
    assert (y[0, 0].float() == 0).all()
    assert (y[4, 2].float() == 0).all()
    _check(y, o, zb, w)
    # eps as given
    y2 = gdn.gated_norm(dev_f32(o), dev_bf16(zb), dev_f32(w[0]), eps=0.5)
    _check(y2, o, zb, w, eps=0.5)


def test_gated_norm_empty_and_deterministic():
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    e = gdn.gated_norm(torch.empty(0, 48, 128, device="cuda"), torch.empty(0, 48, 128, dtype=torch.bfloat16,
                                                                           device="cuda"),
                       torch.ones(128, device="cuda"))
    assert e.shape == (0, 48, 128)
    o, zb, w = _inputs(64, 48, seed=9)
    a = gdn.gated_norm(dev_f32(o), dev_bf16(zb), dev_f32(w[0]))
    b = gdn.gated_norm(dev_f32(o), dev_bf16(zb), dev_f32(w[0]))
    assert torch.equal(a, b)


def test_gated_norm_full_size_sampled_rows():
    # T = 8192 tokens x 48 heads in one launch; rows checked one by one on a sample
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T, Hv = 8192, 48
    o, zb, w = _inputs(T, Hv, seed=21)
    y = host(gdn.gated_norm(dev_f32(o), dev_bf16(zb), dev_f32(w[0])))
    rng = np.random.default_rng(1)
    rows = rng.choice(T * Hv, 512, replace=False)
    rows = np.concatenate([rows, [0, T * Hv - 1]])
    t, h = rows // Hv, rows % Hv
    ref = oracle.gated_norm(o[t, h][:, None], zb[t, h][:, None], w[0])[:, 0]
    got = y[t, h]
    bound = TOL_REL * np.abs(ref) + 1e-6 * np.max(np.abs(ref))
    assert np.all(np.abs(got - ref) <= bound)


def test_prefill_then_gated_norm_matches_oracle():
    # the layer's tail: recurrence, then the gated norm of its output
    import gated_deltanet_recurrence_prefill_b200 as gdn
    import synth
    from tests.helpers import dev_i32
    inp = synth.make_prefill([130, 64, 1], 31, init_state=True, Hqk=4, Hv=12)
    o_ref, _ = oracle.prefill(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                              cu_seqlens=inp.cu_seqlens, scale=inp.scale,
                              initial_state=inp.initial_state)
    o, _ = gdn.prefill(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a),
                       dev_f32(inp.b), dev_f32(inp.A_log), dev_f32(inp.dt_bias),
                       cu_seqlens=dev_i32(inp.cu_seqlens), scale=inp.scale,
                       initial_state=dev_f32(inp.initial_state))
    rng = np.random.default_rng(3)
    T = o_ref.shape[0]
    zb = (rng.standard_normal((T, 12, 128)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    w = rng.uniform(0.5, 1.5, 128).astype(np.float32)
    y = host(gdn.gated_norm(o, dev_bf16(zb), dev_f32(w)))
    ref = oracle.gated_norm(o_ref, zb, w)
    # the recurrence's own error (within 1e-2 of max |o|) passes through the norm
    err = np.max(np.abs(y - ref)) / np.max(np.abs(ref))
    assert err < 2e-2, err
