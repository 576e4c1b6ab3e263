"""The chunked backward's kernels (backward_chunked.cuh) run on the CPU under a
thread-per-CUDA-thread emulation (tests/emu/bwc_emu.cpp, built with
AddressSanitizer), against the fp64 oracle's gradient.

This checks the kernels' own source -- index arithmetic, shared-memory
layout, barrier phases, the chunk list over packed sequences -- without a GPU:
an out-of-bounds access aborts the emulator, and shared memory and the
workspace start as NaN, so a value read before it is written reaches the
result.  The emulation computes in float32 as the kernels do; the bound is
max |x - x_ref| / max |x_ref| <= 1e-4 (float32 rounding through chunk-sized
sums, with no bf16 rounding anywhere on this path).
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "emu", "bwc_emu.cpp")
HDR = os.path.join(ROOT, "gated_deltanet_recurrence_prefill_b200", "csrc", "backward_chunked.cuh")
TOL = 1e-4


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("bwc") / "bwc_emu")
    subprocess.run(["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address", "-fno-omit-frame-pointer", "-pthread",
                    "-o", exe, SRC], check=True)
    return exe


def _rel(x, r):
    return float(np.max(np.abs(x - r)) / max(float(np.max(np.abs(r))), 1e-30))


def _run(emu, tmp, inp, d_o, d_fin, with_s0, with_cu):
    N, Hqk, Hv = len(inp.cu_seqlens) - 1, inp.q.shape[1], inp.v.shape[1]
    T = inp.q.shape[0]
    d = str(tmp)
    with open(os.path.join(d, "meta.txt"), "w") as f:
        f.write(f"{N} {T} {Hqk} {Hv} {inp.scale!r} {int(with_cu)} {int(with_s0)} {int(d_fin is not None)} 1\n")
    files = {"q": inp.q, "k": inp.k, "v": inp.v, "a": inp.a, "b": inp.b, "A_log": inp.A_log,
             "dt_bias": inp.dt_bias, "do": d_o}
    if with_cu:
        files["cu"] = inp.cu_seqlens.astype(np.int32)
    if with_s0:
        files["s0"] = inp.initial_state.astype(np.float32)
    if d_fin is not None:
        files["fin"] = d_fin.astype(np.float32)
    for name, x in files.items():
        np.ascontiguousarray(x).tofile(os.path.join(d, name + ".bin"))
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=0")
    p = subprocess.run([emu, d], capture_output=True, text=True, env=env, timeout=900)
    assert p.returncode == 0, p.stderr[-3000:]
    shp = {"dq": (T, Hqk, 128), "dk": (T, Hqk, 128), "dv": (T, Hv, 128), "da": (T, Hv), "db": (T, Hv),
           "dA_log": (Hv,), "ddt_bias": (Hv,), "dinit": (N, Hv, 128, 128)}
    return {n: np.fromfile(os.path.join(d, n + ".out"), dtype=np.float32).reshape(s) for n, s in shp.items()}


def _check(orc, got, inp, d_o, d_fin, with_s0, with_cu):
    ref = orc.prefill_backward(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias, d_o, d_final=d_fin,
                               cu_seqlens=inp.cu_seqlens if with_cu else None, scale=inp.scale,
                               initial_state=inp.initial_state if with_s0 else None)
    pairs = [("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("da", "da"), ("db", "db"), ("dA_log", "dA_log"),
             ("ddt_bias", "ddt_bias"), ("dinit", "d_initial")]
    for g, r in pairs:
        assert np.all(np.isfinite(got[g])), g
        err = _rel(got[g], ref[r])
        assert err <= TOL, f"{g}: {err}"


def _grads(inp, seed, fin=True):
    rng = np.random.default_rng(seed)
    T, Hv = inp.q.shape[0], inp.v.shape[1]
    N = len(inp.cu_seqlens) - 1
    d_o = rng.standard_normal((T, Hv, 128)).astype(np.float32)
    d_fin = (0.1 * rng.standard_normal((N, Hv, 128, 128))).astype(np.float32) if fin else None
    return d_o, d_fin


def test_emulated_chunked_backward_varlen(orc, emu, tmp_path):
    # several chunks, ragged tails, a one-token and an empty sequence, two value
    # heads per key head
    inp = synth.make_prefill([130, 1, 0, 64, 70], seed=90, init_state=True, init_std=0.05, Hqk=1, Hv=2)
    d_o, d_fin = _grads(inp, 1)
    got = _run(emu, tmp_path, inp, d_o, d_fin, with_s0=True, with_cu=True)
    _check(orc, got, inp, d_o, d_fin, with_s0=True, with_cu=True)


def test_emulated_chunked_backward_one_sequence_no_states(orc, emu, tmp_path):
    # no cu_seqlens, no initial state, no dL/dS_T; three value heads per key head
    inp = synth.make_prefill([100], seed=91, init_state=False, Hqk=1, Hv=3)
    d_o, _ = _grads(inp, 2, fin=False)
    got = _run(emu, tmp_path, inp, d_o, None, with_s0=False, with_cu=False)
    _check(orc, got, inp, d_o, None, with_s0=False, with_cu=False)


def test_emulated_chunked_backward_two_key_heads(orc, emu, tmp_path):
    # two key heads of two value heads each: the key-head mapping and the sum of
    # dq, dk over each key head's value heads
    inp = synth.make_prefill([70, 5], seed=92, init_state=True, init_std=0.05, Hqk=2, Hv=4)
    d_o, d_fin = _grads(inp, 3)
    got = _run(emu, tmp_path, inp, d_o, d_fin, with_s0=True, with_cu=True)
    _check(orc, got, inp, d_o, d_fin, with_s0=True, with_cu=True)


def test_emulated_chunked_backward_strong_decay(orc, emu, tmp_path):
    # one head decays by ~e^-48 per token, so gam = e^G underflows to zero inside
    # a chunk; the other is almost undecayed
    inp = synth.make_prefill([100, 30], seed=93, init_state=True, init_std=0.05, Hqk=1, Hv=2)
    inp.A_log[0] = np.float32(np.log(16.0))
    inp.a[:, 0] = 3.0
    inp.A_log[1] = np.float32(np.log(1.0))
    inp.dt_bias[1] = np.float32(-9.0)
    d_o, d_fin = _grads(inp, 4)
    got = _run(emu, tmp_path, inp, d_o, d_fin, with_s0=True, with_cu=True)
    _check(orc, got, inp, d_o, d_fin, with_s0=True, with_cu=True)
