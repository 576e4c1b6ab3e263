"""gdn_conv1d_silu_backward against the fp64 oracle's gradient of the front end
(itself pinned by central finite differences).  Float32 arithmetic:
max |x - x_ref| / max |x_ref| <= 1e-4 per tensor.

(Its kernels' source is also run on the CPU under emulation by
test_front_backward_emu; this file runs after every other GPU test.)"""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _check(orc, fe, seed, with_cs, with_cu=True):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T = fe.qkv.shape[0]
    rng = np.random.default_rng(seed)
    dq = rng.standard_normal((T, fe.Hqk, 128)).astype(np.float32)
    dk = rng.standard_normal((T, fe.Hqk, 128)).astype(np.float32)
    dv = rng.standard_normal((T, fe.Hv, 128)).astype(np.float32)
    got = gdn.conv1d_silu_backward(dev_bf16(fe.qkv), dev_f32(fe.conv_w), dev_f32(dq), dev_f32(dk), dev_f32(dv),
                                   fe.Hqk, fe.Hv, cu_seqlens=dev_i32(fe.cu_seqlens) if with_cu else None,
                                   conv_state=dev_f32(fe.conv_state) if with_cs else None)
    ref = orc.conv1d_silu_backward(fe.qkv, fe.conv_w, dq, dk, dv, fe.cu_seqlens if with_cu else None, fe.Hqk,
                                   fe.Hv, 128, fe.conv_state if with_cs else None)
    for name in ("d_qkv", "d_conv_w", "d_conv_state"):
        assert rel_err(host(got[name]), ref[name]) <= TOL, name


def test_front_backward_varlen_with_history(orc):
    fe = synth.make_frontend([40, 1, 0, 2, 33, 31, 200], 95, conv_state=True, Hqk=2, Hv=6)
    _check(orc, fe, 1, with_cs=True)


def test_front_backward_one_sequence_no_history(orc):
    fe = synth.make_frontend([300], 96, Hqk=2, Hv=6)
    _check(orc, fe, 2, with_cs=False, with_cu=False)


def test_front_backward_full_heads(orc):
    fe = synth.make_frontend([512], 97, conv_state=True)
    _check(orc, fe, 3, with_cs=True)


def test_front_backward_deterministic():
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    fe = synth.make_frontend([100, 60], 98, conv_state=True, Hqk=2, Hv=6)
    T = fe.qkv.shape[0]
    rng = np.random.default_rng(4)
    g = [dev_f32(rng.standard_normal((T, h, 128)).astype(np.float32)) for h in (2, 2, 6)]
    args = (dev_bf16(fe.qkv), dev_f32(fe.conv_w), *g, 2, 6)
    kw = dict(cu_seqlens=dev_i32(fe.cu_seqlens), conv_state=dev_f32(fe.conv_state))
    a, b = gdn.conv1d_silu_backward(*args, **kw), gdn.conv1d_silu_backward(*args, **kw)
    for name in a:
        assert torch.equal(a[name], b[name]), name
