"""Chunked prefill on the GPU against the fp64 oracle.

Tolerance: max|x - x_ref| / max|x_ref| <= 1e-2 for o and for the final state
(bf16 tensor-core products with float32 accumulation and a float32 state).
Sizes span several chunks and ragged tails; the full-size workloads are checked
on sampled heads / sequences, which the oracle computes one by one.
"""
import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-2

# the prefill kernels gdn_prefill can run: the producer / consumer kernel with
# two or one producer CTAs per (sequence, value head), and the single-CTA kernel
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
    return dict(q=dev_bf16(inp.q), k=dev_bf16(inp.k), v=dev_bf16(inp.v), a=dev_f32(inp.a),
                b=dev_f32(inp.b), A_log=dev_f32(inp.A_log), dt_bias=dev_f32(inp.dt_bias),
                cu_seqlens=dev_i32(inp.cu_seqlens))


def _run(inp, d=None, **kw):
    import gated_deltanet_recurrence_prefill_b200 as gdn
    d = d or _dev(inp)
    s0 = None if inp.initial_state is None else dev_f32(inp.initial_state)
    return gdn.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                       cu_seqlens=d["cu_seqlens"], scale=inp.scale, initial_state=s0, **kw)


def _oracle(orc, inp, heads=None, seq_mask=None):
    return orc.prefill(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                       cu_seqlens=inp.cu_seqlens, scale=inp.scale,
                       initial_state=inp.initial_state, heads=heads, seq_mask=seq_mask)


def test_prefill_t256(kernel, orc):
    """T = 256, one sequence, zero initial state (the 256-token workload)."""
    inp = synth.workload(0)
    o, s = _run(inp)
    o_ref, s_ref = _oracle(orc, inp)
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(s), s_ref) <= TOL


@pytest.mark.parametrize("Hqk,Hv", [(16, 48), (4, 12), (2, 2)])
def test_prefill_varlen_edges(kernel, orc, Hqk, Hv):
    """Lengths 0, 1, 63, 64, 65, 127, 129 and 200 packed together, non-zero
    per-sequence initial states."""
    lengths = [1, 63, 64, 0, 65, 127, 129, 200]
    inp = synth.make_prefill(lengths, seed=60, init_state=True, init_std=0.05, Hqk=Hqk, Hv=Hv)
    o, s = _run(inp)
    o_ref, s_ref = _oracle(orc, inp)
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(s), s_ref) <= TOL
    # the empty sequence returns its initial state unchanged
    np.testing.assert_array_equal(host(s)[3], inp.initial_state[3].astype(np.float64))


def test_prefill_strong_decay(kernel, orc):
    """A_log = ln 16 and a = +3 on some heads: the log-decay summed over a chunk
    falls far below -87 (e^G underflows float32); nothing may overflow."""
    inp = synth.make_prefill([300, 77], seed=61, init_state=True, Hqk=2, Hv=6)
    inp.A_log[:3] = np.float32(np.log(16.0))
    inp.a[:, :3] = 3.0
    o, s = _run(inp)
    o_ref, s_ref = _oracle(orc, inp)
    assert np.isfinite(host(o)).all() and np.isfinite(host(s)).all()
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(s), s_ref) <= TOL


def test_prefill_in_place_state_and_null_final(kernel, orc):
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    inp = synth.make_prefill([130, 5], seed=62, init_state=True, Hqk=2, Hv=4)
    d = _dev(inp)
    st = dev_f32(inp.initial_state)
    o, s = gdn.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                       cu_seqlens=d["cu_seqlens"], initial_state=st, final_state=st)
    assert s.data_ptr() == st.data_ptr()
    o_ref, s_ref = _oracle(orc, inp)
    assert rel_err(host(st), s_ref) <= TOL
    o2, s2 = gdn.prefill(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                         cu_seqlens=d["cu_seqlens"], initial_state=dev_f32(inp.initial_state),
                         want_final_state=False)
    assert s2 is None and torch.equal(o, o2)


def test_prefill_deterministic(kernel):
    import torch
    inp = synth.make_prefill([500, 37], seed=63, init_state=True, Hqk=4, Hv=12)
    d = _dev(inp)
    o1, s1 = _run(inp, d)
    o2, s2 = _run(inp, d)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_varlen_equals_separate_calls(kernel):
    """Packing never mixes sequences: each sequence's outputs equal a call on
    that sequence alone, bit for bit."""
    import torch
    lengths = [70, 200, 1, 64]
    inp = synth.make_prefill(lengths, seed=64, init_state=True, Hqk=4, Hv=12)
    o, s = _run(inp)
    cu = inp.cu_seqlens
    for n in range(len(lengths)):
        lo, hi = int(cu[n]), int(cu[n + 1])
        one = synth.PrefillInputs(inp.q[lo:hi], inp.k[lo:hi], inp.v[lo:hi], inp.a[lo:hi],
                                  inp.b[lo:hi], inp.A_log, inp.dt_bias,
                                  np.array([0, hi - lo], np.int32), inp.initial_state[n:n + 1],
                                  inp.scale, inp.Hqk, inp.Hv, inp.d)
        o1, s1 = _run(one)
        assert torch.equal(o[lo:hi], o1)
        assert torch.equal(s[n], s1[0])


def test_split_prefill_equals_whole(kernel):
    """prefill(T1) then prefill(T2, initial = final of the first) equals
    prefill(T1 + T2) when T1 is a whole number of chunks.  The kernel carries
    the state as Gamma * S~ with a running scale and rounds a bf16 copy of it
    each chunk, so the two runs round at different points: they agree within
    the parity bound (a wrong state hand-off would be off by O(1)), and the
    first part, computed identically, agrees bit for bit."""
    import torch
    inp = synth.make_prefill([384], seed=65, init_state=True, Hqk=4, Hv=12)
    o, s = _run(inp)
    T1 = 192
    first = synth.PrefillInputs(inp.q[:T1], inp.k[:T1], inp.v[:T1], inp.a[:T1], inp.b[:T1],
                                inp.A_log, inp.dt_bias, np.array([0, T1], np.int32),
                                inp.initial_state, inp.scale, inp.Hqk, inp.Hv, inp.d)
    o1, s1 = _run(first)
    second = synth.PrefillInputs(inp.q[T1:], inp.k[T1:], inp.v[T1:], inp.a[T1:], inp.b[T1:],
                                 inp.A_log, inp.dt_bias, np.array([0, 384 - T1], np.int32),
                                 host(s1).astype(np.float32), inp.scale, inp.Hqk, inp.Hv, inp.d)
    o2, s2 = _run(second)
    assert rel_err(host(torch.cat([o1, o2])), host(o)) <= TOL
    assert rel_err(host(s2), host(s)) <= TOL
    # the first part is the same computation on the same inputs: bit for bit
    assert torch.equal(o1, o[:T1])


def test_prefill_one_token_equals_decode_step(kernel):
    """A one-token prefill per unit is one decode step."""
    import gated_deltanet_recurrence_prefill_b200 as gdn
    dec = synth.make_decode(4, 1, seed=66, Hqk=4, Hv=12)
    st = dec.full_state()
    st_dev = dev_f32(st)
    o_dec = gdn.decode_step(dev_bf16(dec.q), dev_bf16(dec.k), dev_bf16(dec.v), dev_f32(dec.a),
                            dev_f32(dec.b), dev_f32(dec.A_log), dev_f32(dec.dt_bias), st_dev,
                            dec.n_seq, dec.layers)
    pre = synth.PrefillInputs(dec.q, dec.k, dec.v, dec.a, dec.b, dec.A_log[0], dec.dt_bias[0],
                              np.arange(dec.U + 1, dtype=np.int32), st, dec.scale, dec.Hqk,
                              dec.Hv, dec.d)
    o_pre, s_pre = _run(pre)
    assert rel_err(host(o_pre), host(o_dec)) <= TOL
    assert rel_err(host(s_pre), host(st_dev)) <= TOL


def test_frontend_then_prefill_8k(orc):
    """T = 8192 through the front end and the prefill (the 8K workload),
    against the oracle's fp64 front end feeding its fp64 recurrence."""
    import gated_deltanet_recurrence_prefill_b200 as gdn
    fe = synth.workload(1)
    g = fe.gates
    q, k, v = gdn.conv1d_silu(dev_bf16(fe.qkv), dev_f32(fe.conv_w), 16, 48)
    o, s = gdn.prefill(q, k, v, dev_f32(g.a), dev_f32(g.b), dev_f32(g.A_log),
                       dev_f32(g.dt_bias), scale=g.scale)
    rq, rk, rv, _ = orc.conv1d_silu(fe.qkv, fe.conv_w, None, 16, 48, 128)
    o_ref, s_ref = orc.prefill(rq, rk, rv, g.a, g.b, g.A_log, g.dt_bias, scale=g.scale)
    assert rel_err(host(o), o_ref) <= TOL
    assert rel_err(host(s), s_ref) <= TOL


@pytest.mark.slow
def test_prefill_262k_sampled_heads(orc):
    """T = 262144, one sequence, S0 ~ N(0, 0.02^2): the full launch, checked on
    three value heads (key heads 0, 8 and 15) over the whole sequence."""
    inp = synth.workload(2)
    o, s = _run(inp)
    for h in (0, 25, 47):
        o_ref, s_ref = _oracle(orc, inp, heads=(h, h + 1))
        assert rel_err(host(o[:, h:h + 1]), o_ref) <= TOL, f"o head {h}"
        assert rel_err(host(s[:, h:h + 1]), s_ref) <= TOL, f"state head {h}"


@pytest.mark.slow
def test_prefill_varlen_16_sequences_sampled(orc):
    """16 sequences of lengths U[1024, 32768] (~270K tokens), per-sequence S0:
    the full launch, checked on 4 sequences x 2 value heads."""
    inp = synth.workload(3)
    o, s = _run(inp)
    mask = np.zeros(inp.N, np.uint8)
    picks = [0, 5, 10, 15]
    mask[picks] = 1
    cu = inp.cu_seqlens
    for h in (7, 40):
        o_ref, s_ref = _oracle(orc, inp, heads=(h, h + 1), seq_mask=mask)
        for n in picks:
            lo, hi = int(cu[n]), int(cu[n + 1])
            assert rel_err(host(o[lo:hi, h:h + 1]), o_ref[lo:hi]) <= TOL, f"o seq {n} head {h}"
            assert rel_err(host(s[n, h]), s_ref[n, 0]) <= TOL, f"state seq {n} head {h}"
