"""The gated norm's gradient kernels (gated_norm_backward.cuh) run on the CPU
under the thread-per-CUDA-thread emulation (tests/emu/nbw_emu.cpp, built with
AddressSanitizer), against the fp64 oracle (pinned by finite differences).
Outputs and workspace start as NaN.  Float32 arithmetic: max |x - x_ref| /
max |x_ref| <= 1e-4 per tensor."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "emu", "nbw_emu.cpp")
TOL = 1e-4


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("g++ not available")
    exe = str(tmp_path_factory.mktemp("nbw") / "nbw_emu")
    subprocess.run(["g++", "-std=c++20", "-O1", "-g", "-fsanitize=address", "-fno-omit-frame-pointer", "-pthread",
                    "-o", exe, SRC], check=True)
    return exe


def _rel(x, r):
    return float(np.max(np.abs(x - r)) / max(float(np.max(np.abs(r))), 1e-30))


@pytest.mark.parametrize("T,Hv,layers", [(19, 12, 1), (21, 6, 3), (5, 4, 8)])
def test_emulated_norm_backward(orc, emu, tmp_path, T, Hv, layers):
    # one layer with a ragged head group (12 heads); several layers, T not a
    # multiple of the 8-token tile; more layers than tokens
    rng = np.random.default_rng(T * 100 + Hv + layers)
    o = rng.standard_normal((T, Hv, 128)).astype(np.float32)
    z = synth.f32_to_bf16_bits(rng.standard_normal((T, Hv, 128)).astype(np.float32))
    w = (1.0 + 0.1 * rng.standard_normal((layers, 128))).astype(np.float32)
    dy = rng.standard_normal((T, Hv, 128)).astype(np.float32)
    d = str(tmp_path)
    with open(os.path.join(d, "meta.txt"), "w") as f:
        f.write(f"{T} {Hv} {layers} 1e-6\n")
    for name, x in (("o", o), ("z", z), ("w", w), ("dy", dy)):
        np.ascontiguousarray(x).tofile(os.path.join(d, name + ".bin"))
    p = subprocess.run([emu, d], capture_output=True, text=True, env=dict(os.environ, ASAN_OPTIONS="detect_leaks=0"),
                       timeout=600)
    assert p.returncode == 0, p.stderr[-3000:]
    got = {"d_o": np.fromfile(os.path.join(d, "d_o.out"), np.float32).reshape(T, Hv, 128),
           "d_z": np.fromfile(os.path.join(d, "d_z.out"), np.float32).reshape(T, Hv, 128),
           "d_norm_w": np.fromfile(os.path.join(d, "d_w.out"), np.float32).reshape(layers, 128)}
    ref = orc.gated_norm_backward(o, z, w, dy, eps=1e-6)
    for name, x in got.items():
        assert np.all(np.isfinite(x)), name
        if name == "d_norm_w" and layers > T:
            assert np.all(x[T:] == 0.0)
        assert _rel(x, ref[name]) <= TOL, name
