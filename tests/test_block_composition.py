"""Two chunks of the chunked form composed into one block, as a consumer that
takes 2C-token blocks would receive them (W, U', Qh, O' of the second chunk
rewritten against the block's start state), reproduce the recurrence.

With M = W2 K1^T and N = Qh2 K1^T the block's rows are
    W  = [W1; gC1 W2 - M diag(kap1) W1],   U' = [U1'; U2' - M diag(kap1) U1'],
    Qh = [Qh1; gC1 Qh2 - N diag(kap1) W1], O' = [O1'; O2' + N diag(kap1) U1'],
and U = U' - W S^T, o = scale (O' + Qh S^T), S_end = gC1 gC2 S + U^T diag(kap) K
with kap taken to the block end.  Checked in float64 against the oracle.
"""
import numpy as np
import pytest


def _chunk(q, k, v, la, be):
    G = np.cumsum(la)
    gam, kap = np.exp(G), np.exp(G[-1] - G)
    Gm = np.tril(np.exp(G[:, None] - G[None, :]))
    L = len(la)
    A = np.tril(be[:, None] * Gm * (k @ k.T), -1)
    Tm = np.linalg.inv(np.eye(L) + A)
    W = Tm @ ((be * gam)[:, None] * k)
    Up = Tm @ (be[:, None] * v)
    P = np.tril(Gm * (q @ k.T))
    return dict(k=k, W=W, Up=Up, Qh=gam[:, None] * q - P @ W, Op=P @ Up, kap=kap, gC=gam[-1])


@pytest.mark.parametrize("seed", [0, 1])
def test_two_chunks_composed_into_one_block(orc, seed):
    rng = np.random.default_rng(seed)
    d, C = 16, 8
    T = 2 * C
    q = rng.standard_normal((T, 1, d)) / np.sqrt(d)
    k = rng.standard_normal((T, 1, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, 1, d))
    a = rng.standard_normal((T, 1)).astype(np.float32)
    b = rng.standard_normal((T, 1)).astype(np.float32)
    A_log, dt_bias = np.array([0.3], np.float32), np.array([-1.0], np.float32)
    S0 = rng.standard_normal((1, 1, d, d))
    scale = 0.7
    o_ref, s_ref = orc.prefill_f64(q, k, v, a, b, A_log, dt_bias, scale=scale, initial_state=S0)
    la = np.array([orc.log_alpha(float(a[t, 0]), float(A_log[0]), float(dt_bias[0])) for t in range(T)])
    be = np.array([orc.beta(float(b[t, 0])) for t in range(T)])
    c1 = _chunk(q[:C, 0], k[:C, 0], v[:C, 0], la[:C], be[:C])
    c2 = _chunk(q[C:, 0], k[C:, 0], v[C:, 0], la[C:], be[C:])
    M, N = c2["W"] @ c1["k"].T, c2["Qh"] @ c1["k"].T
    kW, kU = c1["kap"][:, None] * c1["W"], c1["kap"][:, None] * c1["Up"]
    W = np.vstack([c1["W"], c1["gC"] * c2["W"] - M @ kW])
    Up = np.vstack([c1["Up"], c2["Up"] - M @ kU])
    Qh = np.vstack([c1["Qh"], c1["gC"] * c2["Qh"] - N @ kW])
    Op = np.vstack([c1["Op"], c2["Op"] + N @ kU])
    S = S0[0, 0]
    U = Up - W @ S.T
    o = scale * (Op + Qh @ S.T)
    kap = np.concatenate([c1["kap"] * c2["gC"], c2["kap"]])
    S_end = c1["gC"] * c2["gC"] * S + U.T @ (kap[:, None] * np.vstack([c1["k"], c2["k"]]))
    assert np.max(np.abs(o - o_ref[:, 0])) <= 1e-12
    assert np.max(np.abs(S_end - s_ref[0, 0])) <= 1e-12
