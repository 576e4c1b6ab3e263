"""Front end (conv1d + SiLU + L2) on the GPU against the fp64 oracle.

The kernel computes in float32 and rounds each output to bf16 (nearest even),
so every output may differ from the exact value by at most one bf16 ulp
(2^-8 relative) plus float32 noise: |y - y_ref| <= 2^-8 |y_ref| + 1e-5 max|y_ref|.
"""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host

pytestmark = pytest.mark.gpu


def _check(got, ref):
    got = np.asarray(got, np.float64)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.max(np.abs(ref))
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} outputs outside one bf16 ulp; worst {np.max(np.abs(got - ref))}"


def _run(fe, cs_in=None, with_state_out=False, Hqk=16, Hv=48):
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    n = len(fe.cu_seqlens) - 1
    cs_out = None
    if with_state_out:
        cs_out = torch.full((n, (2 * Hqk + Hv) * 128, 3), -7.0, device="cuda")
    q, k, v = gdn.conv1d_silu(dev_bf16(fe.qkv), dev_f32(fe.conv_w), Hqk, Hv,
                              cu_seqlens=dev_i32(fe.cu_seqlens),
                              conv_state_in=None if cs_in is None else dev_f32(cs_in),
                              conv_state_out=cs_out)
    return q, k, v, cs_out


@pytest.mark.parametrize("use_state", [False, True])
def test_frontend_varlen_edges(orc, use_state):
    lengths = [1, 2, 3, 0, 31, 32, 33, 100, 0, 5]
    fe = synth.make_frontend(lengths, seed=50, conv_state=use_state, Hqk=2, Hv=4)
    q, k, v, cs = _run(fe, fe.conv_state, True, Hqk=2, Hv=4)
    rq, rk, rv, rcs = orc.conv1d_silu(fe.qkv, fe.conv_w, fe.cu_seqlens, 2, 4, 128, fe.conv_state)
    _check(host(q), rq)
    _check(host(k), rk)
    _check(host(v), rv)
    np.testing.assert_array_equal(host(cs), rcs)       # exact copies of inputs


def test_frontend_full_size(orc):
    """T = 8192, 16 key heads, 48 value heads: the front end of the 8K workload."""
    fe = synth.workload(1)
    q, k, v, _ = _run(fe)
    rq, rk, rv, _ = orc.conv1d_silu(fe.qkv, fe.conv_w, fe.cu_seqlens, 16, 48, 128)
    _check(host(q), rq)
    _check(host(k), rk)
    _check(host(v), rv)
    nrm = np.linalg.norm(host(q), axis=-1)
    assert np.all(np.abs(nrm - 1) < 1e-2)
