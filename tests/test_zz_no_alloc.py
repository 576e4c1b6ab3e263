"""gdn_prefill_noalloc: the prefill for callers that cannot allocate device
memory (a framework that owns all device memory through its own arena, a plugin
handed only tensor pointers, a loop where cudaMalloc is not allowed).  It must
give the same results as gdn_prefill with a caller-provided workspace.

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


def _dev(inp):
    return [dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b),
            dev_f32(inp.A_log), dev_f32(inp.dt_bias)]


@pytest.mark.gpu
def test_noalloc_matches_prefill_on_two_calls_in_a_row():
    import gated_deltanet_recurrence_prefill_b200 as gdn
    cases = [
        synth.make_prefill([130, 1, 0, 257], seed=91, init_state=True),
        synth.make_prefill([64, 500], seed=92, init_state=True, Hqk=4, Hv=12),
    ]
    for inp in cases:
        d = _dev(inp)
        cu = dev_i32(inp.cu_seqlens)
        s0 = dev_f32(inp.initial_state)
        o_ref, s_ref = gdn.prefill(*d, cu_seqlens=cu, scale=inp.scale, initial_state=s0)
        o, s = gdn.prefill_noalloc(*d, cu_seqlens=cu, scale=inp.scale, initial_state=s0)
        assert rel_err(host(o), host(o_ref)) <= TOL
        assert rel_err(host(s), host(s_ref)) <= TOL
        assert np.isfinite(host(o)).all()


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
