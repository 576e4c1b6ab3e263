"""gdn_prefill_noalloc: the prefill for callers that cannot allocate device
memory (a framework that owns all device memory through its own arena, a plugin
handed only tensor pointers, a loop where cudaMalloc is not allowed).  Its
outputs are checked against the fp64 oracle, as every prefill path is, on two
calls in a row (the fixed array keeps the previous call's contents), and the
call must leave the device's free memory unchanged.

This file is collected last on purpose: the entry point shares one fixed device
array across all calls, and a run that stops at the first failure has then
already run every other test.  It passes alone in a fresh process too.
"""
import ctypes as C

import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err

TOL = 1e-2
GDN_ERR_TIMEOUT = 5


def _dev(inp):
    return [dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b),
            dev_f32(inp.A_log), dev_f32(inp.dt_bias)]


@pytest.mark.gpu
def test_noalloc_matches_oracle_on_two_calls_in_a_row(orc):
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    cases = [
        synth.make_prefill([130, 1, 0, 257], seed=91, init_state=True),
        synth.make_prefill([64, 500], seed=92, init_state=True, Hqk=4, Hv=12),
    ]
    for inp in cases:
        d = _dev(inp)
        cu = dev_i32(inp.cu_seqlens)
        s0 = dev_f32(inp.initial_state)
        o = torch.empty(inp.v.shape[0], inp.v.shape[1], 128, dtype=torch.float32, device="cuda")
        s = torch.empty_like(s0)
        # warm-up call (library load, the one-time address look-up), then the
        # measured call must not change the device's free memory
        gdn.prefill_noalloc(*d, cu_seqlens=cu, scale=inp.scale, initial_state=s0, o=o, final_state=s)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        gdn.prefill_noalloc(*d, cu_seqlens=cu, scale=inp.scale, initial_state=s0, o=o, final_state=s)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0
        assert gdn.prefill_status(None) == 0
        o_ref, s_ref = orc.prefill(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                                   cu_seqlens=inp.cu_seqlens, scale=inp.scale,
                                   initial_state=inp.initial_state)
        assert rel_err(host(o), o_ref) <= TOL
        assert rel_err(host(s), s_ref) <= TOL
        assert np.isfinite(host(o)).all()


@pytest.mark.gpu
def test_noalloc_timeout_is_reported_and_cleared():
    """A bounded wait that runs out in the library-owned array is visible through
    gdn_prefill_status(NULL) and gdn_check_async(NULL), and the next
    gdn_prefill_noalloc call clears it."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    assert gdn.lib().gdn_selftest_bounded_wait(0, 20000, None, None) == 0
    word = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    gdn.check_async(None, word)
    assert gdn.prefill_status(None) == GDN_ERR_TIMEOUT
    assert int(word.cpu()[0]) != 0
    inp = synth.make_prefill([100], seed=94, init_state=True, Hqk=4, Hv=12)
    gdn.prefill_noalloc(*_dev(inp), cu_seqlens=dev_i32(inp.cu_seqlens), scale=inp.scale,
                        initial_state=dev_f32(inp.initial_state))
    assert gdn.prefill_status(None) == 0


def test_noalloc_rejects_sizes_beyond_its_array():
    """n_seq * Hv above 16320 does not fit the fixed array: refused on the host."""
    from gated_deltanet_recurrence_prefill_b200 import build, _lib
    build.build()
    L = _lib.lib()
    p = C.c_void_p(0x10000)
    n_seq = 341                              # 341 * 48 > 16320
    st = L.gdn_prefill_noalloc(p, p, p, p, p, p, p, p, n_seq, 1000, 16, 48, 128, 0.088, None,
                               None, p, None)
    assert st == 6                           # GDN_ERR_WORKSPACE
