"""The front end's gradient kernels (conv1d_silu_backward.cuh) run on the CPU
under the thread-per-CUDA-thread emulation (tests/emu/fbw_emu.cpp, built with
AddressSanitizer), against the fp64 oracle's gradient.  Outputs and the
workspace start as NaN, so anything left unwritten or read before it is
written shows.  Float32 arithmetic as in the kernels: max |x - x_ref| /
max |x_ref| <= 1e-4 per tensor.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "emu", "fbw_emu.cpp")
TOL = 1e-4


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("fbw") / "fbw_emu")
    subprocess.run(["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address", "-fno-omit-frame-pointer", "-pthread",
                    "-o", exe, SRC], check=True)
    return exe


def _rel(x, r):
    return float(np.max(np.abs(x - r)) / max(float(np.max(np.abs(r))), 1e-30))


def _case(emu, tmp, orc, lengths, seed, Hqk, Hv, with_cs, with_cu=True, want_dcs=True):
    fe = synth.make_frontend(lengths, seed, conv_state=with_cs, Hqk=Hqk, Hv=Hv)
    T = fe.qkv.shape[0]
    N = len(lengths)
    rng = np.random.default_rng(seed + 7)
    dq = rng.standard_normal((T, Hqk, 128)).astype(np.float32)
    dk = rng.standard_normal((T, Hqk, 128)).astype(np.float32)
    dv = rng.standard_normal((T, Hv, 128)).astype(np.float32)
    d = str(tmp)
    with open(os.path.join(d, "meta.txt"), "w") as f:
        f.write(f"{N} {T} {Hqk} {Hv} {int(with_cu)} {int(with_cs)} {int(want_dcs)}\n")
    files = {"qkv": fe.qkv, "w": fe.conv_w, "dq": dq, "dk": dk, "dv": dv}
    if with_cu:
        files["cu"] = fe.cu_seqlens.astype(np.int32)
    if with_cs:
        files["cs"] = fe.conv_state.astype(np.float32)
    for name, x in files.items():
        np.ascontiguousarray(x).tofile(os.path.join(d, name + ".bin"))
    p = subprocess.run([emu, d], capture_output=True, text=True, env=dict(os.environ, ASAN_OPTIONS="detect_leaks=0"),
                       timeout=900)
    assert p.returncode == 0, p.stderr[-3000:]
    ctot = (2 * Hqk + Hv) * 128
    got = {"d_qkv": np.fromfile(os.path.join(d, "dx.out"), np.float32).reshape(T, ctot),
           "d_conv_w": np.fromfile(os.path.join(d, "dw.out"), np.float32).reshape(ctot, 4)}
    if want_dcs:
        got["d_conv_state"] = np.fromfile(os.path.join(d, "dcs.out"), np.float32).reshape(N, ctot, 3)
    ref = orc.conv1d_silu_backward(fe.qkv, fe.conv_w, dq, dk, dv, fe.cu_seqlens if with_cu else None, Hqk, Hv, 128,
                                   fe.conv_state if with_cs else None)
    for name, x in got.items():
        assert np.all(np.isfinite(x)), name
        err = _rel(x, ref[name])
        assert err <= TOL, f"{name}: {err}"


def test_emulated_front_backward_varlen_with_history(orc, emu, tmp_path):
    # sequences starting inside a tile, across tile edges, of one token and empty
    _case(emu, tmp_path, orc, [40, 1, 0, 2, 33, 31], seed=95, Hqk=1, Hv=2, with_cs=True)


def test_emulated_front_backward_one_sequence_no_history(orc, emu, tmp_path):
    _case(emu, tmp_path, orc, [70], seed=96, Hqk=1, Hv=1, with_cs=False, with_cu=False)


def test_emulated_front_backward_without_history_output(orc, emu, tmp_path):
    _case(emu, tmp_path, orc, [5, 64], seed=97, Hqk=2, Hv=2, with_cs=True, want_dcs=False)
