"""gdn_prefill_bf16 (the output o stored as bf16) against the fp64 oracle, for
each prefill kernel, at the prefill's tolerance: max|x - x_ref| / max|x_ref| <=
1e-2 for o and for the (float32) final state.  Rounding o to bf16 adds at most
2^-9 of each element, so the float32-o bound holds with room.  The bf16 o must
also be the float32 o of gdn_prefill rounded to nearest even: both variants
run the same arithmetic and differ only in the store."""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-2

KERNELS = {"pc2": {"GDN_PREFILL_KERNEL": "pc", "GDN_PREFILL_PRODUCERS": "2"},
           "pc1": {"GDN_PREFILL_KERNEL": "pc", "GDN_PREFILL_PRODUCERS": "1"},
           "single": {"GDN_PREFILL_KERNEL": "single"}}


@pytest.fixture(params=sorted(KERNELS))
def kernel(request, monkeypatch):
    monkeypatch.delenv("GDN_PREFILL_PRODUCERS", raising=False)
    for k, v in KERNELS[request.param].items():
        monkeypatch.setenv(k, v)
    return request.param


def _dev(inp):
    return [dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b),
            dev_f32(inp.A_log), dev_f32(inp.dt_bias)]


def _bf16_round(x):
    """float32 -> bf16 (nearest even) -> float64, in numpy."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("lengths", [[256], [130, 1, 0, 257], [64, 65, 200]])
def test_prefill_bf16_output_matches_oracle(kernel, orc, lengths):
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    inp = synth.make_prefill(lengths, seed=100 + len(lengths), init_state=True)
    d = _dev(inp)
    cu = dev_i32(inp.cu_seqlens)
    s0 = dev_f32(inp.initial_state)
    o16, s = gdn.prefill(*d, cu_seqlens=cu, scale=inp.scale, initial_state=s0, o_dtype=torch.bfloat16)
    assert o16.dtype == torch.bfloat16
    o_ref, s_ref = orc.prefill(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                               cu_seqlens=inp.cu_seqlens, scale=inp.scale, initial_state=inp.initial_state)
    assert rel_err(host(o16), o_ref) <= TOL
    assert rel_err(host(s), s_ref) <= TOL
    # the same arithmetic as the float32-o call, rounded once at the store
    o32, s32 = gdn.prefill(*d, cu_seqlens=cu, scale=inp.scale, initial_state=s0)
    assert np.array_equal(host(o16), _bf16_round(o32.cpu().numpy()))
    assert torch.equal(s, s32)


def test_prefill_bf16_output_strong_decay(kernel, orc):
    """Strong in-chunk decay (the same gates as the float32-o strong-decay case)."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    inp = synth.make_prefill([300, 77], seed=61, init_state=True, Hqk=2, Hv=6)
    inp.A_log[:3] = np.float32(np.log(16.0))
    inp.a[:, :3] = 3.0
    d = _dev(inp)
    o16, s = gdn.prefill(*d, cu_seqlens=dev_i32(inp.cu_seqlens), scale=inp.scale,
                         initial_state=dev_f32(inp.initial_state), o_dtype=torch.bfloat16)
    o_ref, s_ref = orc.prefill(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                               cu_seqlens=inp.cu_seqlens, scale=inp.scale, initial_state=inp.initial_state)
    assert rel_err(host(o16), o_ref) <= TOL
    assert rel_err(host(s), s_ref) <= TOL
