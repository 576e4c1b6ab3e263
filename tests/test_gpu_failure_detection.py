"""Failure detection: every wait of the producer / consumer prefill is bounded.
The library's self-test runs the same bounded waits (a global counter no thread
raises; an mbarrier phase that never completes) with a short limit: the wait
gives up, the error word is set exactly as the prefill sets it, and
gdn_prefill_status reports GDN_ERR_TIMEOUT.  Nothing faults or hangs, and the
context stays usable for the next call."""
import time

import numpy as np
import pytest

import synth
from tests.helpers import dev_bf16, dev_f32, dev_i32, host, rel_err

pytestmark = pytest.mark.gpu
GDN_ERR_TIMEOUT = 5


@pytest.mark.parametrize("which", [0, 1], ids=["global_counter", "mbarrier"])
def test_bounded_wait_gives_up_and_reports(which, orc):
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    from gated_deltanet_recurrence_prefill_b200._lib import _ptr
    ws = torch.zeros(gdn.prefill_workspace_size(1, 200, 4, 12, 128), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert gdn.lib().gdn_selftest_bounded_wait(which, 20000, _ptr(ws), None) == 0
    status = gdn.prefill_status(ws)
    elapsed = time.perf_counter() - t0
    assert status == GDN_ERR_TIMEOUT
    assert 0.015 <= elapsed < 5.0, elapsed
    # the same workspace and context serve a normal prefill right after
    inp = synth.make_prefill([200], seed=90, init_state=True, Hqk=4, Hv=12)
    o, s = gdn.prefill(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b),
                       dev_f32(inp.A_log), dev_f32(inp.dt_bias), cu_seqlens=dev_i32(inp.cu_seqlens),
                       scale=inp.scale, initial_state=dev_f32(inp.initial_state), workspace=ws)
    assert gdn.prefill_status(ws) == 0
    o_ref, s_ref = orc.prefill(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                               cu_seqlens=inp.cu_seqlens, scale=inp.scale, initial_state=inp.initial_state)
    assert rel_err(host(o), o_ref) <= 1e-2


@pytest.mark.parametrize("where", ["device", "pinned"])
def test_check_async_reads_the_error_word_without_waiting(where):
    """gdn_check_async enqueues the error-word read behind the kernel and returns
    at once; after an ordinary synchronisation the word shows the timeout, and a
    later successful prefill on the same workspace clears it."""
    import torch
    import gated_deltanet_recurrence_prefill_b200 as gdn
    from gated_deltanet_recurrence_prefill_b200._lib import _ptr
    ws = torch.zeros(gdn.prefill_workspace_size(1, 200, 4, 12, 128), dtype=torch.uint8, device="cuda")
    word = (torch.full((1,), -1, dtype=torch.int32, device="cuda") if where == "device"
            else torch.full((1,), -1, dtype=torch.int32).pin_memory())
    assert gdn.lib().gdn_selftest_bounded_wait(1, 20000, _ptr(ws), None) == 0
    t0 = time.perf_counter()
    gdn.check_async(ws, word)
    enqueue_s = time.perf_counter() - t0
    assert enqueue_s < 0.015, enqueue_s            # returned before the 20 ms wait ran out
    torch.cuda.synchronize()
    assert int(word.cpu()[0]) != 0
    inp = synth.make_prefill([200], seed=93, init_state=True, Hqk=4, Hv=12)
    gdn.prefill(dev_bf16(inp.q), dev_bf16(inp.k), dev_bf16(inp.v), dev_f32(inp.a), dev_f32(inp.b),
                dev_f32(inp.A_log), dev_f32(inp.dt_bias), cu_seqlens=dev_i32(inp.cu_seqlens),
                scale=inp.scale, initial_state=dev_f32(inp.initial_state), workspace=ws)
    gdn.check_async(ws, word)
    torch.cuda.synchronize()
    assert int(word.cpu()[0]) == 0
