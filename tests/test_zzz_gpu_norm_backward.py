"""gdn_gated_norm_backward against the fp64 oracle's gradient of the gated
norm (pinned by finite differences).  Float32 arithmetic: max |x - x_ref| /
max |x_ref| <= 1e-4 per tensor.

(Its kernels' source is also run on the CPU under emulation by
test_norm_backward_emu; this file runs after every other GPU test.)"""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, host, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.mark.parametrize("T,Hv,layers", [(300, 48, 1), (96, 12, 48), (37, 6, 3)])
def test_norm_backward(orc, T, Hv, layers):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    rng = np.random.default_rng(T + Hv + layers)
    o = rng.standard_normal((T, Hv, 128)).astype(np.float32)
    z = synth.f32_to_bf16_bits(rng.standard_normal((T, Hv, 128)).astype(np.float32))
    w = (1.0 + 0.1 * rng.standard_normal((layers, 128))).astype(np.float32)
    dy = rng.standard_normal((T, Hv, 128)).astype(np.float32)
    got = gdn.gated_norm_backward(dev_f32(o), dev_bf16(z), dev_f32(w), dev_f32(dy))
    ref = orc.gated_norm_backward(o, z, w, dy)
    for name in ("d_o", "d_z", "d_norm_w"):
        assert rel_err(host(got[name]), ref[name]) <= TOL, name


def test_norm_backward_deterministic():
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    rng = np.random.default_rng(5)
    args = (dev_f32(rng.standard_normal((200, 48, 128)).astype(np.float32)),
            dev_bf16(synth.f32_to_bf16_bits(rng.standard_normal((200, 48, 128)).astype(np.float32))),
            dev_f32(np.ones((1, 128), np.float32)), dev_f32(rng.standard_normal((200, 48, 128)).astype(np.float32)))
    a, b = gdn.gated_norm_backward(*args), gdn.gated_norm_backward(*args)
    for name in a:
        assert torch.equal(a[name], b[name]), name
