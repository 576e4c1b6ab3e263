"""gdn_layer_prefill_host: the front end and the prefill of one sequence from
pinned host buffers to pinned host buffers, the copies overlapped with the
compute over token ranges.  Checked against the fp64 oracle (front end, then
recurrence) at the prefill's tolerance, max |x - x_ref| / max |x_ref| <= 1e-2,
and against the two device calls on the whole sequence: the first range's first
chunk is the same computation on the same inputs (bit for bit), the later ranges continue the
state in float32 across a range boundary (within the tolerance), and the conv
history out is the last three inputs of each channel, exactly."""
import numpy as np
import pytest

import synth
from tests.helpers import dev_f32, host, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-2
HQK, HV = 2, 6


def _host_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("T,n_blocks", [(1000, 4), (256, 1), (130, 8), (640, 3)])
def test_layer_prefill_host_matches_oracle_and_device_path(orc, T, n_blocks):
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    fe = synth.make_frontend([T], seed=300 + T, conv_state=True, init_state=True, Hqk=HQK, Hv=HV)
    g = fe.gates
    h_qkv = _host_bf16(fe.qkv)
    h_a = torch.from_numpy(np.ascontiguousarray(g.a)).pin_memory()
    h_b = torch.from_numpy(np.ascontiguousarray(g.b)).pin_memory()
    d_w, cs_in, s0 = dev_f32(fe.conv_w), dev_f32(fe.conv_state), dev_f32(g.initial_state)
    A_log, dt_bias = dev_f32(g.A_log), dev_f32(g.dt_bias)
    cs_out = torch.full_like(cs_in, -7.0)
    h_o, h_fs = gdn.layer_prefill_host(h_qkv, h_a, h_b, d_w, A_log, dt_bias, HQK, HV, conv_state_in=cs_in,
                                       initial_state=s0, conv_state_out=cs_out, n_blocks=n_blocks)
    torch.cuda.synchronize()
    # the two device calls on the whole sequence
    cs_ref = torch.full_like(cs_in, -7.0)
    q, k, v = gdn.conv1d_silu(h_qkv.cuda(), d_w, HQK, HV, conv_state_in=cs_in, conv_state_out=cs_ref)
    o, fs = gdn.prefill(q, k, v, dev_f32(g.a), dev_f32(g.b), A_log, dt_bias, initial_state=s0)
    torch.cuda.synchronize()
    # the first chunk lies in the first range: the same computation on the same inputs
    assert torch.equal(h_o[:64], o[:64].cpu())
    assert rel_err(h_o.numpy(), host(o)) <= TOL
    assert rel_err(h_fs.numpy(), host(fs)[0]) <= TOL
    assert torch.equal(cs_out, cs_ref)
    # the oracle: front end, then the recurrence
    rq, rk, rv, _ = orc.conv1d_silu(fe.qkv, fe.conv_w, None, HQK, HV, 128, fe.conv_state)
    o_ref, s_ref = orc.prefill(rq, rk, rv, g.a, g.b, g.A_log, g.dt_bias, scale=g.scale,
                               initial_state=g.initial_state)
    assert rel_err(h_o.numpy(), o_ref) <= TOL
    assert rel_err(h_fs.numpy(), s_ref[0]) <= TOL


def test_layer_prefill_host_rejects_bad_arguments():
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    L = gdn.lib()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    cur = torch.cuda.current_stream()
    nbytes = L.gdn_layer_prefill_host_workspace_size(256, HQK, HV, 128, 2)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    P = gdn._lib._ptr(ws)
    S = gdn._lib._stream

    def call(qkv=P, T=256, d=128, nb=2, wsb=nbytes, su=None):
        return L.gdn_layer_prefill_host(qkv, P, P, P, P, P, None, None, T, HQK, HV, d, 0.088, nb, P, P, None, P,
                                        wsb, S(cur), S(s1) if su is None else su, S(s2))

    assert call(d=64) == 2                       # unsupported head width
    assert call(nb=0) == 1                       # no ranges
    assert call(qkv=None) == 1
    assert call(su=S(cur)) == 1                  # the copy streams must differ from the compute stream
    assert call(wsb=nbytes - 256) == 6           # workspace too small
    assert call(T=0) == 0                        # nothing to do
    assert L.gdn_layer_prefill_host_workspace_size(256, HQK, HV, 64, 2) == 0


def test_layer_prefill_host_without_history_or_state(orc):
    """No conv history in or out and no initial state: zero history, zero state."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    T = 700
    fe = synth.make_frontend([T], seed=331, conv_state=False, init_state=False, Hqk=HQK, Hv=HV)
    g = fe.gates
    h_qkv = _host_bf16(fe.qkv)
    h_a = torch.from_numpy(np.ascontiguousarray(g.a)).pin_memory()
    h_b = torch.from_numpy(np.ascontiguousarray(g.b)).pin_memory()
    h_o, h_fs = gdn.layer_prefill_host(h_qkv, h_a, h_b, dev_f32(fe.conv_w), dev_f32(g.A_log), dev_f32(g.dt_bias),
                                       HQK, HV, n_blocks=3)
    torch.cuda.synchronize()
    rq, rk, rv, _ = orc.conv1d_silu(fe.qkv, fe.conv_w, None, HQK, HV, 128, None)
    o_ref, s_ref = orc.prefill(rq, rk, rv, g.a, g.b, g.A_log, g.dt_bias, scale=g.scale)
    assert rel_err(h_o.numpy(), o_ref) <= TOL
    assert rel_err(h_fs.numpy(), s_ref[0]) <= TOL
