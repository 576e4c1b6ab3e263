"""Pins for the fp64 oracle: checks against facts that do not come from the
oracle itself (CPU only).

- The unrolled-product form of the recurrence, evaluated with explicit matrix
  products (brute force on tiny inputs).
- Invariants of the delta rule: retrieval (alpha = beta = 1, unit key:
  S_t k_t = v_t), no write (beta = 0), pure decay, orthonormal keys, alpha = 0,
  superposition, and the ungated rule of the Qwen3.8-27B architecture page
  (2kiu.com), section 2.2, when alpha = 1.
- Closed forms of the gates.
- The chunked WY/UT algebra against the recurrence.
- The front end against a library convolution and special tap patterns.
"""
import math

import numpy as np
import pytest


def _gates(a, b, A_log, dt_bias):
    """alpha, beta for per-token a, b [T, Hv] and per-head A_log, dt_bias [Hv]."""
    x = a + dt_bias[None, :]
    sp = np.where(x > 0, x + np.log1p(np.exp(-np.abs(x))), np.log1p(np.exp(np.minimum(x, 0))))
    alpha = np.exp(-np.exp(A_log)[None, :] * sp)
    beta = 1.0 / (1.0 + np.exp(-b))
    return alpha, beta


def _brute(q, k, v, alpha, beta, S0, scale):
    """Unrolled product form for one head: S_t = S0 P_1..P_t + sum_j beta_j v_j k_j^T
    P_{j+1}..P_t with P_s = alpha_s (I - beta_s k_s k_s^T).  Returns (o [T, dv], S_T)."""
    T, dk = k.shape
    I = np.eye(dk)
    P = [alpha[s] * (I - beta[s] * np.outer(k[s], k[s])) for s in range(T)]
    outs = []
    S_t = S0
    for t in range(T):
        S_t = S0 @ _chain(P, 0, t + 1)
        for j in range(t + 1):
            S_t = S_t + beta[j] * np.outer(v[j], k[j]) @ _chain(P, j + 1, t + 1)
        outs.append(scale * S_t @ q[t])
    return np.array(outs), S_t


def _chain(P, lo, hi):
    out = np.eye(P[0].shape[0])
    for s in range(lo, hi):
        out = out @ P[s]
    return out


def _rand_case(rng, T, Hqk, Hv, dk, dv, unit_keys=False):
    q = rng.standard_normal((T, Hqk, dk))
    k = rng.standard_normal((T, Hqk, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, Hv, dv))
    a = rng.standard_normal((T, Hv)).astype(np.float32)
    b = rng.standard_normal((T, Hv)).astype(np.float32)
    A_log = np.log(rng.uniform(1, 16, Hv)).astype(np.float32)
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(0.1), Hv))
    dt_bias = np.log(np.expm1(dt)).astype(np.float32)
    return q, k, v, a, b, A_log, dt_bias


def test_brute_force_unrolled_product(orc):
    """Every prefix output and the final state equal the explicit product form;
    value head h reads key head h // 3 (6 value heads over 2 key heads)."""
    rng = np.random.default_rng(11)
    T, Hqk, Hv, dk, dv = 9, 2, 6, 5, 4
    q, k, v, a, b, A_log, dt_bias = _rand_case(rng, T, Hqk, Hv, dk, dv)
    S0 = (0.3 * rng.standard_normal((1, Hv, dv, dk))).astype(np.float32)
    scale = 0.37
    o, fs = orc.prefill(q, k, v, a, b, A_log, dt_bias, scale=scale, initial_state=S0)
    alpha, beta = _gates(a.astype(np.float64), b.astype(np.float64),
                         A_log.astype(np.float64), dt_bias.astype(np.float64))
    for h in range(Hv):
        g = h // 3
        ob, Sb = _brute(q[:, g], k[:, g], v[:, h], alpha[:, h], beta[:, h],
                        S0[0, h].astype(np.float64), scale)
        np.testing.assert_allclose(o[:, h], ob, rtol=0, atol=1e-12)
        np.testing.assert_allclose(fs[0, h], Sb, rtol=0, atol=1e-12)


def test_retrieval_invariant(orc):
    """alpha = beta = 1 and unit keys: after writing v_t under k_t, reading with
    q_t = k_t returns v_t exactly (up to fp64 rounding)."""
    rng = np.random.default_rng(3)
    T, dk, dv = 40, 16, 8
    k = rng.standard_normal((T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, 1, dv))
    a = np.full((T, 1), -np.inf, np.float32)          # softplus(-inf) = 0 -> alpha = 1
    b = np.full((T, 1), np.inf, np.float32)           # sigmoid(inf) = 1
    S0 = rng.standard_normal((1, 1, dv, dk)).astype(np.float32)
    o, fs = orc.prefill(k, k, v, a, b, np.zeros(1, np.float32), np.zeros(1, np.float32),
                        scale=1.0, initial_state=S0)
    np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(fs[0, 0] @ k[-1, 0], v[-1, 0], rtol=0, atol=1e-13)


def test_no_write_keeps_state(orc):
    """beta = 0, alpha = 1: the state is unchanged and o_t = scale S0 q_t."""
    rng = np.random.default_rng(4)
    T, dk, dv = 17, 8, 6
    q = rng.standard_normal((T, 1, dk))
    k = rng.standard_normal((T, 1, dk))
    v = rng.standard_normal((T, 1, dv))
    a = np.full((T, 1), -np.inf, np.float32)
    b = np.full((T, 1), -np.inf, np.float32)
    S0 = rng.standard_normal((1, 1, dv, dk)).astype(np.float32)
    o, fs = orc.prefill(q, k, v, a, b, np.zeros(1, np.float32), np.zeros(1, np.float32),
                        scale=0.5, initial_state=S0)
    np.testing.assert_array_equal(fs[0, 0], S0[0, 0].astype(np.float64))
    np.testing.assert_allclose(o[:, 0], 0.5 * q[:, 0] @ S0[0, 0].astype(np.float64).T,
                               rtol=0, atol=1e-13)


def test_pure_decay(orc):
    """beta = 0 and a + dt_bias = 0, A_log = 0: alpha = exp(-ln 2) = 1/2 per token,
    so S_T = 2^-T S0."""
    rng = np.random.default_rng(5)
    T, dk, dv = 13, 4, 3
    q = rng.standard_normal((T, 1, dk))
    k = rng.standard_normal((T, 1, dk))
    v = rng.standard_normal((T, 1, dv))
    a = np.zeros((T, 1), np.float32)
    b = np.full((T, 1), -np.inf, np.float32)
    S0 = rng.standard_normal((1, 1, dv, dk)).astype(np.float32)
    _, fs = orc.prefill(q, k, v, a, b, np.zeros(1, np.float32), np.zeros(1, np.float32),
                        initial_state=S0)
    np.testing.assert_allclose(fs[0, 0], S0[0, 0] * 2.0 ** -T, rtol=1e-14, atol=0)


def test_orthonormal_keys_write_columns(orc):
    """alpha = beta = 1, zero S0, keys e_1..e_d: column t of S_T is v_t (the
    textbook associative-memory write)."""
    rng = np.random.default_rng(6)
    d = 8
    k = np.eye(d)[:, None, :]
    v = rng.standard_normal((d, 1, d))
    a = np.full((d, 1), -np.inf, np.float32)
    b = np.full((d, 1), np.inf, np.float32)
    _, fs = orc.prefill(k, k, v, a, b, np.zeros(1, np.float32), np.zeros(1, np.float32))
    np.testing.assert_allclose(fs[0, 0], v[:, 0].T, rtol=0, atol=1e-15)


def test_alpha_zero_forgets(orc):
    """alpha = 0 (a = +inf): S_t = beta_t v_t k_t^T, whatever came before."""
    rng = np.random.default_rng(7)
    T, dk, dv = 6, 5, 4
    q = rng.standard_normal((T, 1, dk))
    k = rng.standard_normal((T, 1, dk))
    v = rng.standard_normal((T, 1, dv))
    a = np.full((T, 1), np.inf, np.float32)
    b = rng.standard_normal((T, 1)).astype(np.float32)
    S0 = rng.standard_normal((1, 1, dv, dk)).astype(np.float32)
    o, fs = orc.prefill(q, k, v, a, b, np.zeros(1, np.float32), np.zeros(1, np.float32),
                        scale=1.0, initial_state=S0)
    be = 1.0 / (1.0 + np.exp(-b[:, 0].astype(np.float64)))
    np.testing.assert_allclose(fs[0, 0], be[-1] * np.outer(v[-1, 0], k[-1, 0]), atol=1e-14)
    for t in range(T):
        np.testing.assert_allclose(o[t, 0], be[t] * v[t, 0] * (k[t, 0] @ q[t, 0]), atol=1e-13)


def test_superposition(orc):
    """For fixed keys and gates the map (S0, V) -> (o, S_T) is linear:
    f(S1 + S2, V1 + V2) = f(S1, V1) + f(S2, V2)."""
    rng = np.random.default_rng(8)
    T, dk, dv = 11, 6, 5
    q, k, v1, a, b, A_log, dt_bias = _rand_case(rng, T, 1, 1, dk, dv)
    v2 = rng.standard_normal(v1.shape)
    # halves of float32 draws, so that the sum of two states is exact in float32
    S1 = (0.5 * rng.standard_normal((1, 1, dv, dk))).astype(np.float32)
    S2 = (0.5 * rng.standard_normal((1, 1, dv, dk))).astype(np.float32)
    S12 = S1.astype(np.float64) + S2.astype(np.float64)
    o1, f1 = orc.prefill(q, k, v1, a, b, A_log, dt_bias, initial_state=S1)
    o2, f2 = orc.prefill(q, k, v2, a, b, A_log, dt_bias, initial_state=S2)
    # S1 + S2 rounds in float32 by at most 1e-7 relative: compare at that level
    o12, f12 = orc.prefill(q, k, v1 + v2, a, b, A_log, dt_bias,
                           initial_state=(S1 + S2).astype(np.float32))
    assert np.max(np.abs((S1 + S2).astype(np.float64) - S12)) < 1e-6
    np.testing.assert_allclose(o12, o1 + o2, rtol=0, atol=1e-6)
    np.testing.assert_allclose(f12, f1 + f2, rtol=0, atol=1e-6)
    # exact version: zero states, values only
    z = np.zeros_like(S1)
    oa, fa = orc.prefill(q, k, v1, a, b, A_log, dt_bias, initial_state=z)
    ob, fb = orc.prefill(q, k, v2, a, b, A_log, dt_bias, initial_state=z)
    oab, fab = orc.prefill(q, k, v1 + v2, a, b, A_log, dt_bias, initial_state=z)
    np.testing.assert_allclose(oab, oa + ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(fab, fa + fb, rtol=0, atol=1e-12)
    # and states only, with zero values: S -> f(S) is linear (scaling by 2 is exact)
    z_v = np.zeros_like(v1)
    os1, fs1 = orc.prefill(q, k, z_v, a, b, A_log, dt_bias, initial_state=S1)
    os2, fs2 = orc.prefill(q, k, z_v, a, b, A_log, dt_bias, initial_state=2 * S1)
    np.testing.assert_allclose(os2, 2 * os1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(fs2, 2 * fs1, rtol=0, atol=1e-14)


def test_ungated_rule_of_the_page(orc):
    """alpha = 1: S_t = S_{t-1}(I - beta k k^T) + beta v k^T, evaluated as written
    (matrix form) on the page."""
    rng = np.random.default_rng(9)
    T, dk, dv = 10, 6, 6
    q, k, v, _, b, _, _ = _rand_case(rng, T, 1, 1, dk, dv)
    a = np.full((T, 1), -np.inf, np.float32)
    S0 = rng.standard_normal((1, 1, dv, dk)).astype(np.float32)
    o, fs = orc.prefill(q, k, v, a, b, np.zeros(1, np.float32), np.zeros(1, np.float32),
                        scale=1.0, initial_state=S0)
    S = S0[0, 0].astype(np.float64)
    be = 1.0 / (1.0 + np.exp(-b[:, 0].astype(np.float64)))
    for t in range(T):
        kt = k[t, 0]
        S = S @ (np.eye(dk) - be[t] * np.outer(kt, kt)) + be[t] * np.outer(v[t, 0], kt)
        np.testing.assert_allclose(o[t, 0], S @ q[t, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(fs[0, 0], S, rtol=0, atol=1e-12)


def test_gate_closed_forms(orc):
    # a + dt_bias = 0 -> softplus = ln 2; A_log = 0 -> rate 1
    assert orc.log_alpha(0.0, 0.0, 0.0) == pytest.approx(-math.log(2.0), abs=1e-16)
    assert orc.log_alpha(1.0, 0.0, -1.0) == pytest.approx(-math.log(2.0), abs=1e-16)
    # A_log = ln 16 -> rate 16
    assert orc.log_alpha(0.0, math.log(16.0), 0.0) == pytest.approx(-16 * math.log(2.0), rel=1e-15)
    # large arguments: softplus(x) -> x, softplus(-x) -> e^{-x}
    assert orc.log_alpha(60.0, 0.0, 0.0) == pytest.approx(-60.0, rel=1e-15)
    assert orc.log_alpha(-60.0, 0.0, 0.0) == pytest.approx(-math.exp(-60.0), rel=1e-12)
    # dt_bias = ln(expm1(dt)) is the inverse of softplus: log_alpha = -exp(A_log) dt at a = 0
    for dt in (1e-3, 0.02, 0.1):
        assert orc.log_alpha(0.0, 0.5, math.log(math.expm1(dt))) == pytest.approx(
            -math.exp(0.5) * dt, rel=1e-12)
    assert orc.beta(0.0) == 0.5
    assert orc.beta(40.0) == pytest.approx(1.0, abs=1e-16)
    assert orc.beta(-40.0) == pytest.approx(math.exp(-40.0), rel=1e-12)


@pytest.mark.parametrize("C", [1, 2, 16, 64, 128])
def test_chunked_equals_recurrent(orc, C):
    """The chunked WY/UT algebra reproduces the recurrence, with ragged chunks,
    several packed sequences (one empty, one of length 1), non-zero S0 and
    decay strong enough that the in-chunk log-decay falls far below -87."""
    rng = np.random.default_rng(100 + C)
    lengths = [70, 0, 1, 133, 64]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T, Hqk, Hv, dk, dv = int(cu[-1]), 2, 6, 16, 12
    q, k, v, a, b, A_log, dt_bias = _rand_case(rng, T, Hqk, Hv, dk, dv, unit_keys=True)
    A_log[:2] = np.float32(math.log(16.0))       # strong decay heads
    a[:, :2] = 3.0
    S0 = rng.standard_normal((len(lengths), Hv, dv, dk)).astype(np.float32)
    o_r, s_r = orc.prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens=cu, initial_state=S0)
    o_c, s_c = orc.prefill_chunked(q, k, v, a, b, A_log, dt_bias, cu_seqlens=cu,
                                   initial_state=S0, chunk=C)
    np.testing.assert_allclose(o_c, o_r, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s_c, s_r, rtol=0, atol=1e-12)
    # the empty sequence keeps its initial state
    np.testing.assert_array_equal(s_r[1], S0[1].astype(np.float64))


def test_varlen_equals_separate_calls(orc):
    rng = np.random.default_rng(12)
    lengths = [5, 9, 3]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v, a, b, A_log, dt_bias = _rand_case(rng, T, 1, 3, 4, 4)
    S0 = rng.standard_normal((3, 3, 4, 4)).astype(np.float32)
    o, fs = orc.prefill(q, k, v, a, b, A_log, dt_bias, cu_seqlens=cu, initial_state=S0)
    for n in range(3):
        s, e = cu[n], cu[n + 1]
        o1, f1 = orc.prefill(q[s:e], k[s:e], v[s:e], a[s:e], b[s:e], A_log, dt_bias,
                             initial_state=S0[n:n + 1])
        np.testing.assert_array_equal(o[s:e], o1)
        np.testing.assert_array_equal(fs[n], f1[0])


def test_head_subset_and_decode_step(orc):
    """A one-token prefill equals one decode step, per unit and layer."""
    import synth
    inp = synth.make_decode(3, 2, seed=21, Hqk=2, Hv=6, d=8)
    st = inp.full_state()
    o_d, s_d = orc.decode(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                          inp.n_seq, inp.layers, st)
    for u in range(inp.U):
        l = u % inp.layers
        o_p, s_p = orc.prefill(inp.q[u:u + 1], inp.k[u:u + 1], inp.v[u:u + 1], inp.a[u:u + 1],
                               inp.b[u:u + 1], inp.A_log[l], inp.dt_bias[l],
                               initial_state=st[u:u + 1])
        np.testing.assert_array_equal(o_d[u], o_p[0])
        np.testing.assert_array_equal(s_d[u], s_p[0])
    # the unit-list path gives the same numbers
    sel = [4, 1]
    o_s, s_s = orc.decode(inp.q, inp.k, inp.v, inp.a, inp.b, inp.A_log, inp.dt_bias,
                          inp.n_seq, inp.layers, st[sel], units=sel)
    np.testing.assert_array_equal(o_s, o_d[sel])
    np.testing.assert_array_equal(s_s, s_d[sel])


# ---- front end ------------------------------------------------------------------

def _fe_case(rng, T, Hqk=1, Hv=2, d=8):
    import synth
    ctot = (2 * Hqk + Hv) * d
    x = synth.f32_to_bf16_bits(rng.standard_normal((T, ctot)).astype(np.float32))
    return x, ctot


def _silu(y):
    return y / (1.0 + np.exp(-y))


def test_conv_identity_tap(orc):
    """w = e_3 (current token only): y = SiLU(x); q, k then have unit norm."""
    import synth
    rng = np.random.default_rng(31)
    Hqk, Hv, d, T = 1, 2, 8, 7
    x, ctot = _fe_case(rng, T, Hqk, Hv, d)
    w = np.zeros((ctot, 4), np.float32)
    w[:, 3] = 1.0
    q, k, v, _ = orc.conv1d_silu(x, w, None, Hqk, Hv, d)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    y = _silu(xf)
    np.testing.assert_allclose(v.reshape(T, -1), y[:, 2 * Hqk * d:], rtol=0, atol=1e-15)
    yq = y[:, :d]
    np.testing.assert_allclose(q[:, 0], yq / np.sqrt((yq ** 2).sum(1, keepdims=True) + 1e-6),
                               rtol=0, atol=1e-15)
    nrm = np.linalg.norm(k[:, 0], axis=-1)
    assert np.all(np.abs(nrm - 1.0) < 1e-4)


def test_conv_oldest_tap_shifts(orc):
    """w = e_0: y[t] = SiLU(x[t-3]), zero history before the start."""
    import synth
    rng = np.random.default_rng(32)
    Hqk, Hv, d, T = 1, 1, 8, 9
    x, ctot = _fe_case(rng, T, Hqk, Hv, d)
    w = np.zeros((ctot, 4), np.float32)
    w[:, 0] = 1.0
    _, _, v, _ = orc.conv1d_silu(x, w, None, Hqk, Hv, d)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)[:, 2 * d:]
    exp = np.zeros_like(xf)
    exp[3:] = _silu(xf[:-3])
    np.testing.assert_allclose(v[:, 0], exp, rtol=0, atol=1e-15)


def test_conv_matches_library_conv1d(orc):
    """General weights and several packed sequences against
    torch.nn.functional.conv1d (depthwise, left padding 3), per sequence."""
    torch = pytest.importorskip("torch")
    import synth
    rng = np.random.default_rng(33)
    Hqk, Hv, d = 2, 3, 8
    lengths = [5, 1, 0, 12]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    x, ctot = _fe_case(rng, T, Hqk, Hv, d)
    w = (0.5 * rng.standard_normal((ctot, 4))).astype(np.float32)
    q, k, v, _ = orc.conv1d_silu(x, w, cu, Hqk, Hv, d)
    xf = torch.from_numpy(synth.bf16_bits_to_f32(x).astype(np.float64))
    wt = torch.from_numpy(w.astype(np.float64)).view(ctot, 1, 4)
    for n in range(len(lengths)):
        s, e = int(cu[n]), int(cu[n + 1])
        if e == s:
            continue
        seg = xf[s:e].T.unsqueeze(0)                                    # [1, C, L]
        y = torch.nn.functional.conv1d(seg, wt, padding=3, groups=ctot)[0, :, : e - s].T
        y = torch.nn.functional.silu(y).numpy()
        for hh in range(2 * Hqk + Hv):
            blk = y[:, hh * d:(hh + 1) * d]
            if hh < 2 * Hqk:
                blk = blk / np.sqrt((blk ** 2).sum(1, keepdims=True) + 1e-6)
            got = q[s:e, hh] if hh < Hqk else (k[s:e, hh - Hqk] if hh < 2 * Hqk
                                              else v[s:e, hh - 2 * Hqk])
            np.testing.assert_allclose(got, blk, rtol=0, atol=1e-13)


def test_conv_state_carries_history(orc):
    """Running a sequence in two parts, passing the conv state, equals one run."""
    rng = np.random.default_rng(34)
    Hqk, Hv, d, T = 1, 1, 8, 11
    x, ctot = _fe_case(rng, T, Hqk, Hv, d)
    w = (0.5 * rng.standard_normal((ctot, 4))).astype(np.float32)
    q, k, v, cs = orc.conv1d_silu(x, w, None, Hqk, Hv, d)
    for cut in (1, 2, 3, 7):
        q1, k1, v1, cs1 = orc.conv1d_silu(x[:cut], w, None, Hqk, Hv, d)
        q2, k2, v2, cs2 = orc.conv1d_silu(x[cut:], w, None, Hqk, Hv, d,
                                          conv_state=cs1.astype(np.float32))
        np.testing.assert_array_equal(np.concatenate([v1, v2]), v)
        np.testing.assert_array_equal(np.concatenate([q1, q2]), q)
        np.testing.assert_array_equal(cs2, cs)


# ---- gated output norm -------------------------------------------------------

def _gn_inputs(T=5, Hv=3, d=16, seed=3):
    rng = np.random.default_rng(seed)
    o = rng.standard_normal((T, Hv, d))
    z = rng.standard_normal((T, Hv, d))
    w = rng.uniform(0.5, 1.5, d)
    return o, z, w


def test_gated_norm_silu_closed_forms(orc):
    # with o a constant row and w = 1, eps = 0 the norm is exactly 1 per channel, so y is silu(z):
    # silu(0) = 0, silu(1) = 1 / (1 + 1/e), silu(-1) = -1 / (1 + e), silu(2) = 2 / (1 + e^-2)
    o = np.full((1, 1, 4), 3.0)
    z = np.array([[[0.0, 1.0, -1.0, 2.0]]])
    y = orc.gated_norm(o, z, np.ones(4), eps=0.0)
    e = np.e
    want = [0.0, 1.0 / (1.0 + 1.0 / e), -1.0 / (1.0 + e), 2.0 / (1.0 + e ** -2)]
    assert np.allclose(y[0, 0], want, rtol=0, atol=1e-15)


def test_gated_norm_unit_rms(orc):
    # constant gate c per row, w = 1, eps = 0: the mean square of y over d_v is silu(c)^2
    o, _, _ = _gn_inputs(T=7, Hv=4, d=32)
    c = 1.0
    z = np.full_like(o, c)
    y = orc.gated_norm(o, z, np.ones(32), eps=0.0)
    s = c / (1.0 + np.exp(-c))
    assert np.allclose(np.mean(y * y, axis=-1), s * s, rtol=1e-13)


def test_gated_norm_scale_invariance_and_eps(orc):
    o, z, w = _gn_inputs()
    y = orc.gated_norm(o, z, w, eps=0.0)
    assert np.allclose(orc.gated_norm(37.5 * o, z, w, eps=0.0), y, rtol=1e-13, atol=0)
    assert np.allclose(orc.gated_norm(-o, z, w, eps=0.0), -y, rtol=1e-13, atol=0)
    # eps only matters against the row's mean square: a tiny row is shrunk, not blown up
    tiny = 1e-6 * o
    yt = orc.gated_norm(tiny, z, w, eps=1e-6)
    ms = np.mean(tiny * tiny, axis=-1, keepdims=True)
    assert np.allclose(yt, y * np.sqrt(ms / (ms + 1e-6)), rtol=1e-12)
    # o = 0 gives 0
    assert np.all(orc.gated_norm(np.zeros_like(o), z, w) == 0.0)


def test_gated_norm_heads_and_tokens_independent(orc):
    # the norm runs over d_v within one (token, head): changing another head or token
    # changes nothing else; the weight scales channel v alone
    o, z, w = _gn_inputs(T=4, Hv=3, d=8)
    y = orc.gated_norm(o, z, w)
    o2 = o.copy()
    o2[1, 2] *= 5.0
    o2[3, 0] += 1.0
    y2 = orc.gated_norm(o2, z, w)
    mask = np.ones(y.shape[:2], bool)
    mask[1, 2] = mask[3, 0] = False
    assert np.array_equal(y[mask], y2[mask])
    w2 = w.copy()
    w2[5] *= 3.0
    y3 = orc.gated_norm(o, z, w2)
    assert np.allclose(y3[..., 5], 3.0 * y[..., 5], rtol=1e-14)
    assert np.array_equal(np.delete(y3, 5, axis=-1), np.delete(y, 5, axis=-1))


def test_gated_norm_bf16_gate_bits(orc):
    # z given as bf16 bit patterns is widened exactly
    o, z, w = _gn_inputs()
    zb = (z.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    zw = (zb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(orc.gated_norm(o, zb, w), orc.gated_norm(o, zw, w))


def test_gated_norm_layer_of_each_row(orc):
    # rows are units s * layers + l: row t takes the weight of layer t % layers.  With the same
    # o and z in every row and w[l] = (l + 1), row t is (t % layers + 1) times row 0.
    layers, T = 3, 7
    o1, z1, _ = _gn_inputs(T=1, Hv=2, d=8)
    o = np.repeat(o1, T, axis=0)
    z = np.repeat(z1, T, axis=0)
    w = np.array([[l + 1.0] * 8 for l in range(layers)])
    y = orc.gated_norm(o, z, w)
    for t in range(T):
        assert np.allclose(y[t], (t % layers + 1) * y[0], rtol=1e-14, atol=0)


# ---- the backward pass: gradients pinned by central finite differences ----------

def _bw_case(seed=0, lengths=(5, 3), Hqk=1, Hv=2, d=4):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    q = rng.standard_normal((T, Hqk, d)) / np.sqrt(d)
    k = rng.standard_normal((T, Hqk, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    return dict(q=q, k=k, v=rng.standard_normal((T, Hv, d)), a=rng.standard_normal((T, Hv)),
                b=rng.standard_normal((T, Hv)), A_log=np.log(rng.uniform(1, 4, Hv)),
                dt_bias=rng.uniform(-3, 0, Hv), cu_seqlens=cu,
                initial_state=0.3 * rng.standard_normal((len(lengths), Hv, d, d))), \
        rng.standard_normal((T, Hv, d)), rng.standard_normal((len(lengths), Hv, d, d))


def test_prefill_f64_equals_prefill(orc):
    # float-representable gates: the all-double forward is the forward
    inp, _, _ = _bw_case(1)
    f32 = {n: inp[n].astype(np.float32) for n in ("a", "b", "A_log", "dt_bias", "initial_state")}
    o1, s1 = orc.prefill_f64(inp["q"], inp["k"], inp["v"], f32["a"], f32["b"], f32["A_log"], f32["dt_bias"],
                             cu_seqlens=inp["cu_seqlens"], initial_state=f32["initial_state"])
    o2, s2 = orc.prefill(inp["q"], inp["k"], inp["v"], f32["a"], f32["b"], f32["A_log"], f32["dt_bias"],
                         cu_seqlens=inp["cu_seqlens"], initial_state=f32["initial_state"])
    assert np.allclose(o1, o2, rtol=0, atol=1e-14) and np.allclose(s1, s2, rtol=0, atol=1e-14)


def test_backward_matches_finite_differences(orc):
    for seed in (0, 3):
        _backward_vs_finite_differences(orc, seed)


def _backward_vs_finite_differences(orc, seed):
    inp, d_o, d_fin = _bw_case(seed)

    def loss(**over):
        x = dict(inp, **over)
        o, s = orc.prefill_f64(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                               cu_seqlens=x["cu_seqlens"], initial_state=x["initial_state"])
        return float(np.sum(d_o * o) + np.sum(d_fin * s))

    g = orc.prefill_backward(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["A_log"], inp["dt_bias"],
                             d_o, d_final=d_fin, cu_seqlens=inp["cu_seqlens"],
                             initial_state=inp["initial_state"])
    names = {"q": "dq", "k": "dk", "v": "dv", "a": "da", "b": "db", "A_log": "dA_log",
             "dt_bias": "ddt_bias", "initial_state": "d_initial"}
    h = 1e-6
    for name, gname in names.items():
        base = inp[name]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            xp, xm = base.copy(), base.copy()
            xp[idx] += h
            xm[idx] -= h
            fd[idx] = (loss(**{name: xp}) - loss(**{name: xm})) / (2 * h)
        scale_ = max(1.0, np.max(np.abs(fd)))
        assert np.max(np.abs(g[gname] - fd)) <= 2e-7 * scale_, name


def test_backward_of_a_sum_over_heads(orc):
    # dq and dk collect every value head of the key group: with two key heads of two
    # value heads each, the gradient equals the sum of the per-head gradients taken alone
    inp, d_o, d_fin = _bw_case(5, lengths=(6,), Hqk=2, Hv=4)
    g = orc.prefill_backward(**{n: inp[n] for n in ("q", "k", "v", "a", "b", "A_log", "dt_bias")},
                             d_o=d_o, d_final=d_fin, cu_seqlens=inp["cu_seqlens"], initial_state=inp["initial_state"])
    for gk in range(2):
        acc_q = np.zeros_like(g["dq"][:, gk])
        acc_k = np.zeros_like(g["dk"][:, gk])
        for h in (2 * gk, 2 * gk + 1):
            sub = dict(q=inp["q"][:, gk:gk + 1], k=inp["k"][:, gk:gk + 1], v=inp["v"][:, h:h + 1],
                       a=inp["a"][:, h:h + 1], b=inp["b"][:, h:h + 1], A_log=inp["A_log"][h:h + 1],
                       dt_bias=inp["dt_bias"][h:h + 1])
            gh = orc.prefill_backward(**sub, d_o=d_o[:, h:h + 1], d_final=d_fin[:, h:h + 1],
                                      cu_seqlens=inp["cu_seqlens"], initial_state=inp["initial_state"][:, h:h + 1])
            acc_q += gh["dq"][:, 0]
            acc_k += gh["dk"][:, 0]
        assert np.allclose(g["dq"][:, gk], acc_q, rtol=1e-13, atol=1e-15)
        assert np.allclose(g["dk"][:, gk], acc_k, rtol=1e-13, atol=1e-15)


def test_chunked_backward_equals_sequential_backward(orc):
    # the chunked (WY) gradient is the same function as the token-by-token one: for
    # any chunk length, with chunks that span several tokens, a ragged tail and a
    # one-token sequence
    inp, d_o, d_fin = _bw_case(7, lengths=(37, 5, 1), Hqk=2, Hv=4, d=6)
    args = {n: inp[n] for n in ("q", "k", "v", "a", "b", "A_log", "dt_bias")}
    ref = orc.prefill_backward(**args, d_o=d_o, d_final=d_fin, cu_seqlens=inp["cu_seqlens"],
                               initial_state=inp["initial_state"])
    for C in (1, 2, 3, 8, 16, 64, 128):
        got = orc.prefill_backward_chunked(**args, d_o=d_o, d_final=d_fin, cu_seqlens=inp["cu_seqlens"],
                                           initial_state=inp["initial_state"], C=C)
        for name, x in ref.items():
            s = max(1.0, np.max(np.abs(x)))
            assert np.max(np.abs(got[name] - x)) <= 1e-11 * s, (C, name)


def test_chunked_backward_without_initial_or_final_state(orc):
    inp, d_o, _ = _bw_case(8, lengths=(20,), Hqk=1, Hv=1, d=4)
    args = {n: inp[n] for n in ("q", "k", "v", "a", "b", "A_log", "dt_bias")}
    ref = orc.prefill_backward(**args, d_o=d_o, cu_seqlens=inp["cu_seqlens"])
    got = orc.prefill_backward_chunked(**args, d_o=d_o, cu_seqlens=inp["cu_seqlens"], C=8)
    for name, x in ref.items():
        assert np.max(np.abs(got[name] - x)) <= 1e-11 * max(1.0, np.max(np.abs(x))), name


# ---- the front end's backward: pinned by central finite differences ---------------------

def _front_case(seed, lengths=(5, 2), Hqk=1, Hv=1, d=4):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    ctot = (2 * Hqk + Hv) * d
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    bits = lambda x: (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return dict(qkv=bits(rng.standard_normal((T, ctot))), conv_w=(0.5 * rng.standard_normal((ctot, 4))).astype(np.float32),
                conv_state=rng.standard_normal((len(lengths), ctot, 3)).astype(np.float32), cu=cu,
                Hqk=Hqk, Hv=Hv, d=d)


def test_front_f64_equals_front_end(orc):
    c = _front_case(11)
    q1, k1, v1 = orc.conv1d_silu_f64(c["qkv"], c["conv_w"], c["cu"], c["Hqk"], c["Hv"], c["d"], c["conv_state"])
    q2, k2, v2, _ = orc.conv1d_silu(c["qkv"], c["conv_w"], c["cu"], c["Hqk"], c["Hv"], c["d"], c["conv_state"])
    for x, y in ((q1, q2), (k1, k2), (v1, v2)):
        assert np.max(np.abs(x - y)) <= 1e-14


def test_front_backward_matches_finite_differences(orc):
    for seed in (12, 13):
        c = _front_case(seed)
        rng = np.random.default_rng(seed + 100)
        T, Hqk, Hv, d = c["qkv"].shape[0], c["Hqk"], c["Hv"], c["d"]
        gq, gk, gv = rng.standard_normal((T, Hqk, d)), rng.standard_normal((T, Hqk, d)), rng.standard_normal((T, Hv, d))
        x0 = (c["qkv"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        w0, s0 = c["conv_w"].astype(np.float64), c["conv_state"].astype(np.float64)

        def loss(x, w, s):
            q, k, v = orc.conv1d_silu_f64(x, w, c["cu"], Hqk, Hv, d, s)
            return float(np.sum(gq * q) + np.sum(gk * k) + np.sum(gv * v))

        g = orc.conv1d_silu_backward(x0, w0, gq, gk, gv, c["cu"], Hqk, Hv, d, s0)
        h = 1e-6
        for name, base, gname in (("x", x0, "d_qkv"), ("w", w0, "d_conv_w"), ("s", s0, "d_conv_state")):
            fd = np.zeros_like(base)
            for idx in np.ndindex(base.shape):
                p_, m_ = base.copy(), base.copy()
                p_[idx] += h
                m_[idx] -= h
                args_p = dict(x=x0, w=w0, s=s0)
                args_m = dict(x=x0, w=w0, s=s0)
                args_p[name], args_m[name] = p_, m_
                fd[idx] = (loss(**args_p) - loss(**args_m)) / (2 * h)
            assert np.max(np.abs(g[gname] - fd)) <= 2e-7 * max(1.0, np.max(np.abs(fd))), (seed, gname)


def test_front_backward_without_history_and_one_sequence(orc):
    # no conv_state: the history is zero; the gradient with respect to it is the
    # one taken at an explicit zero history
    c = _front_case(14, lengths=(6,))
    rng = np.random.default_rng(114)
    T = c["qkv"].shape[0]
    gq, gk, gv = rng.standard_normal((T, 1, 4)), rng.standard_normal((T, 1, 4)), rng.standard_normal((T, 1, 4))
    g = orc.conv1d_silu_backward(c["qkv"], c["conv_w"], gq, gk, gv, None, 1, 1, 4, None)
    x0 = (c["qkv"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    w0 = c["conv_w"].astype(np.float64)
    h = 1e-6
    base = orc.conv1d_silu_f64(x0, w0, None, 1, 1, 4, None)
    fd = np.zeros_like(x0)
    for idx in np.ndindex(x0.shape):
        p_ = x0.copy()
        p_[idx] += h
        m_ = x0.copy()
        m_[idx] -= h
        lp = sum(float(np.sum(gg * o)) for gg, o in zip((gq, gk, gv), orc.conv1d_silu_f64(p_, w0, None, 1, 1, 4, None)))
        lm = sum(float(np.sum(gg * o)) for gg, o in zip((gq, gk, gv), orc.conv1d_silu_f64(m_, w0, None, 1, 1, 4, None)))
        fd[idx] = (lp - lm) / (2 * h)
    assert base[0].shape == (T, 1, 4)
    assert np.max(np.abs(g["d_qkv"] - fd)) <= 2e-7 * max(1.0, np.max(np.abs(fd)))
    g0 = orc.conv1d_silu_backward(c["qkv"], c["conv_w"], gq, gk, gv, None, 1, 1, 4, np.zeros((1, 12, 3)))
    assert np.array_equal(g["d_conv_state"], g0["d_conv_state"])
    assert np.array_equal(g["d_qkv"], g0["d_qkv"])


def test_gated_norm_backward_matches_finite_differences(orc):
    # two layers, so that the weight gradient's rows collect the right tokens
    rng = np.random.default_rng(21)
    T, Hv, d, layers = 5, 2, 6, 2
    o = rng.standard_normal((T, Hv, d))
    z = rng.standard_normal((T, Hv, d))
    w = rng.standard_normal((layers, d))
    dy = rng.standard_normal((T, Hv, d))
    g = orc.gated_norm_backward(o, z, w, dy, eps=1e-3)
    h = 1e-6
    for name, base, gname in (("o", o, "d_o"), ("z", z, "d_z"), ("w", w, "d_norm_w")):
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            xp, xm = base.copy(), base.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = dict(o=o, z=z, norm_w=w)
            args_m = dict(o=o, z=z, norm_w=w)
            key = {"o": "o", "z": "z", "w": "norm_w"}[name]
            args_p[key], args_m[key] = xp, xm
            fd[idx] = (np.sum(dy * orc.gated_norm(eps=1e-3, **args_p))
                       - np.sum(dy * orc.gated_norm(eps=1e-3, **args_m))) / (2 * h)
        assert np.max(np.abs(g[gname] - fd)) <= 2e-7 * max(1.0, np.max(np.abs(fd))), gname
