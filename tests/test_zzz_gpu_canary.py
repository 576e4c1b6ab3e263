"""Canary-guarded outputs: every entry point writes into the middle of a larger
buffer whose margins (1024 elements each side) hold a NaN bit pattern; after
the call the margins must be bitwise untouched (no write outside the output)
and no element of the output may still hold the pattern (every element
written).  With compute-sanitizer unavailable, this is the check for stray
writes; determinism and parity tests cover the rest.  Inputs are the small
varlen cases of the parity tests (ragged chunks, one-token and empty
sequences).
"""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32

pytestmark = pytest.mark.gpu
GUARD = 1024
F32_PATTERN = 0x7FC0BEEF       # a NaN
BF16_PATTERN = 0x7FBE          # a NaN


class Guarded:
    """A tensor of `shape` and `dtype` (float32 or bfloat16) inside a buffer
    with patterned margins."""

    def __init__(self, shape, dtype, init=None):
        import torch
        self.n = int(np.prod(shape))
        itype, pat = (torch.int32, F32_PATTERN) if dtype == torch.float32 else (torch.int16, BF16_PATTERN)
        self.pattern = pat
        self.raw = torch.full((self.n + 2 * GUARD,), pat, dtype=itype, device="cuda")
        self.t = self.raw[GUARD:GUARD + self.n].view(dtype).view(*shape)
        if init is not None:
            self.t.copy_(init)

    def check(self, name, full=True):
        import torch
        torch.cuda.synchronize()
        h = self.raw.cpu().numpy()
        pat = h.dtype.type(self.pattern)
        assert np.all(h[:GUARD] == pat) and np.all(h[GUARD + self.n:] == pat), f"{name}: write outside the output"
        if full:
            assert not np.any(h[GUARD:GUARD + self.n] == pat), f"{name}: output element left unwritten"


def _f32(shape, init=None):
    import torch
    return Guarded(shape, torch.float32, init)


def _bf16(shape):
    import torch
    return Guarded(shape, torch.bfloat16)


LENGTHS = [1, 63, 64, 0, 65, 130]


def test_front_end_outputs_guarded():
    import gated_deltanet_recurrence_prefill_b200 as gdn
    fe = synth.make_frontend(LENGTHS, 60, conv_state=True, Hqk=2, Hv=6)
    T, N, ctot = fe.qkv.shape[0], len(LENGTHS), fe.qkv.shape[1]
    q, k, v, cso = _bf16((T, 2, 128)), _bf16((T, 2, 128)), _bf16((T, 6, 128)), _f32((N, ctot, 3))
    gdn.conv1d_silu(dev_bf16(fe.qkv), dev_f32(fe.conv_w), 2, 6, cu_seqlens=dev_i32(fe.cu_seqlens),
                    conv_state_in=dev_f32(fe.conv_state), conv_state_out=cso.t, out=(q.t, k.t, v.t))
    for name, g in (("q", q), ("k", k), ("v", v), ("conv_state_out", cso)):
        g.check(name)


def test_prefill_outputs_guarded():
    import gated_deltanet_recurrence_prefill_b200 as gdn
    inp = synth.make_prefill(LENGTHS, 61, init_state=True, Hqk=2, Hv=6)
    T, N = inp.q.shape[0], len(LENGTHS)
    o, fs = _f32((T, 6, 128)), _f32((N, 6, 128, 128))
    gdn.prefill(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b),
                dev_f32(inp.A_log), dev_f32(inp.dt_bias), cu_seqlens=dev_i32(inp.cu_seqlens), scale=inp.scale,
                initial_state=dev_f32(inp.initial_state), final_state=fs.t, o=o.t)
    o.check("o")
    fs.check("final_state")


def test_decode_state_and_output_guarded():
    import gated_deltanet_recurrence_prefill_b200 as gdn
    d = synth.make_decode(2, 3, 62, Hqk=2, Hv=6)
    U = 6
    st = _f32((U, 6, 128, 128), init=dev_f32(d.state_of_units(np.arange(U))))
    o = _f32((U, 6, 128))
    gdn.decode_step(dev_bf16(d.q), dev_bf16(d.k), dev_bf16(d.v), dev_f32(d.a), dev_f32(d.b), dev_f32(d.A_log),
                    dev_f32(d.dt_bias), st.t, 2, 3, scale=d.scale, o=o.t)
    st.check("state (in place)")
    o.check("o")


def test_gated_norm_output_guarded():
    import gated_deltanet_recurrence_prefill_b200 as gdn
    rng = np.random.default_rng(63)
    o = rng.standard_normal((37, 6, 128)).astype(np.float32)
    z = synth.f32_to_bf16_bits(rng.standard_normal((37, 6, 128)).astype(np.float32))
    y = _bf16((37, 6, 128))
    gdn.gated_norm(dev_f32(o), dev_bf16(z), dev_f32(np.ones((1, 128), np.float32)), y=y.t)
    y.check("y")


def _backward_outputs(T, N):
    shapes = dict(dq=(T, 2, 128), dk=(T, 2, 128), dv=(T, 6, 128), da=(T, 6), db=(T, 6), dA_log=(6,),
                  ddt_bias=(6,), d_initial_state=(N, 6, 128, 128))
    return {name: _f32(s) for name, s in shapes.items()}


@pytest.mark.parametrize("chunked", [False, True])
def test_backward_outputs_guarded(chunked):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    inp = synth.make_prefill(LENGTHS, 64, init_state=True, init_std=0.05, Hqk=2, Hv=6)
    T, N = inp.q.shape[0], len(LENGTHS)
    rng = np.random.default_rng(65)
    d_o = rng.standard_normal((T, 6, 128)).astype(np.float32)
    d_fin = (0.1 * rng.standard_normal((N, 6, 128, 128))).astype(np.float32)
    g = _backward_outputs(T, N)
    fn = gdn.prefill_backward_chunked if chunked else gdn.prefill_backward
    fn(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b), dev_f32(inp.A_log),
       dev_f32(inp.dt_bias), dev_f32(d_o), d_final_state=dev_f32(d_fin), cu_seqlens=dev_i32(inp.cu_seqlens),
       scale=inp.scale, initial_state=dev_f32(inp.initial_state), out={n: x.t for n, x in g.items()})
    for name, x in g.items():
        x.check(name)


def test_front_backward_outputs_guarded():
    import gated_deltanet_recurrence_prefill_b200 as gdn
    fe = synth.make_frontend(LENGTHS, 66, conv_state=True, Hqk=2, Hv=6)
    T, N, ctot = fe.qkv.shape[0], len(LENGTHS), fe.qkv.shape[1]
    rng = np.random.default_rng(67)
    grads = [dev_f32(rng.standard_normal((T, h, 128)).astype(np.float32)) for h in (2, 2, 6)]
    g = dict(d_qkv=_f32((T, ctot)), d_conv_w=_f32((ctot, 4)), d_conv_state=_f32((N, ctot, 3)))
    gdn.conv1d_silu_backward(dev_bf16(fe.qkv), dev_f32(fe.conv_w), *grads, 2, 6, cu_seqlens=dev_i32(fe.cu_seqlens),
                             conv_state=dev_f32(fe.conv_state), out={n: x.t for n, x in g.items()})
    for name, x in g.items():
        x.check(name)


def test_norm_backward_outputs_guarded():
    import gated_deltanet_recurrence_prefill_b200 as gdn
    rng = np.random.default_rng(68)
    T, Hv, layers = 37, 6, 3
    o = dev_f32(rng.standard_normal((T, Hv, 128)).astype(np.float32))
    z = dev_bf16(synth.f32_to_bf16_bits(rng.standard_normal((T, Hv, 128)).astype(np.float32)))
    w = dev_f32((1.0 + 0.1 * rng.standard_normal((layers, 128))).astype(np.float32))
    dy = dev_f32(rng.standard_normal((T, Hv, 128)).astype(np.float32))
    g = dict(d_o=_f32((T, Hv, 128)), d_z=_f32((T, Hv, 128)), d_norm_w=_f32((layers, 128)))
    gdn.gated_norm_backward(o, z, w, dy, out={n: x.t for n, x in g.items()})
    for name, x in g.items():
        x.check(name)
