"""Pins for oracle.recurrence: closed forms, brute force, special cases, and the pages' replay invariant."""

import itertools
import math

import numpy as np
import pytest

from oracle import recurrence as rc

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ----------------------------------------------------------------------------- Mamba-2

def test_mamba2_scalar_closed_form():
    """P = N = 1, constant inputs: s_t = a^t s0 + dt x b (1 - a^t) / (1 - a) (geometric series)."""
    A, D, dt, x, b, c, s0 = -2.0, 0.7, 0.05, 1.3, 0.4, -0.9, 0.25
    a = math.exp(dt * A)
    S = np.array([[[[s0]]]])
    recs = []
    for t in range(1, 21):
        inp = {"x": np.array([[[x]]]), "B": np.array([[[b]]]), "C": np.array([[[c]]]), "dt": np.array([[dt]])}
        S, y = rc.mamba2_step(S, inp["x"], inp["B"], inp["C"], inp["dt"], [A], [D], [0])
        recs.append(inp)
        s_t = a ** t * s0 + dt * x * b * (1 - a ** t) / (1 - a)
        y_t = s_t * c + D * x
        assert S[0, 0, 0, 0] == pytest.approx(s_t, rel=1e-13)
        assert y[0, 0, 0] == pytest.approx(y_t, rel=1e-13)
        y_rep = rc.mamba2_replay_output(np.array([[[[s0]]]]), recs, inp["C"], [A], [D], [0])
        assert y_rep[0, 0, 0] == pytest.approx(y_t, rel=1e-12)
        S_fold = rc.mamba2_fold(np.array([[[[s0]]]]), recs, [A], [0])
        assert S_fold[0, 0, 0, 0] == pytest.approx(s_t, rel=1e-12)


def _mamba2_bruteforce(S0, toks, A, D, H, G):
    """Definition written index by index in plain Python: S[h][p][n], group g = h // (H/G)."""
    P, N = len(S0[0]), len(S0[0][0])
    S = [[[S0[h][p][n] for n in range(N)] for p in range(P)] for h in range(H)]
    ys = []
    for tok in toks:
        y = [[0.0] * P for _ in range(H)]
        for h in range(H):
            g = h // (H // G)
            dA = math.exp(tok["dt"][h] * A[h])
            for p in range(P):
                for n in range(N):
                    S[h][p][n] = dA * S[h][p][n] + tok["dt"][h] * tok["x"][h][p] * tok["B"][g][n]
                y[h][p] = sum(S[h][p][n] * tok["C"][g][n] for n in range(N)) + D[h] * tok["x"][h][p]
        ys.append(y)
    return S, ys


@pytest.mark.parametrize("H,G", [(2, 1), (4, 2)])
def test_mamba2_bruteforce_tiny(H, G):
    rng = np.random.default_rng(7)
    P, N, steps = 4, 8, 12
    A = -np.exp(rng.uniform(0, np.log(16), H))
    D = rng.standard_normal(H)
    S0 = rng.standard_normal((H, P, N)) * 0.1
    toks = [{"x": rng.standard_normal((H, P)), "B": rng.standard_normal((G, N)),
             "C": rng.standard_normal((G, N)), "dt": rng.uniform(1e-3, 0.1, H)} for _ in range(steps)]
    S_bf, ys_bf = _mamba2_bruteforce(S0.tolist(), [{k: v.tolist() for k, v in t.items()} for t in toks],
                                     A.tolist(), D.tolist(), H, G)
    hg = [h // (H // G) for h in range(H)]
    S = S0
    for t, tok in enumerate(toks):
        S, y = rc.mamba2_step(S, tok["x"], tok["B"], tok["C"], tok["dt"], A, D, hg)
        np.testing.assert_allclose(y, np.array(ys_bf[t]), rtol=1e-12, atol=1e-13)
        y_rep = rc.mamba2_replay_output(S0, toks[: t + 1], tok["C"], A, D, hg)
        np.testing.assert_allclose(y_rep, y, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, np.array(S_bf), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(rc.mamba2_fold(S0, toks, A, hg), S, rtol=1e-12, atol=1e-14)


def test_mamba2_special_cases():
    rng = np.random.default_rng(3)
    H, P, N = 2, 3, 5
    A = np.array([-1.0, -4.0])
    S0 = rng.standard_normal((H, P, N))
    tok = {"x": rng.standard_normal((H, P)), "B": rng.standard_normal((1, N)), "C": np.zeros((1, N)),
           "dt": np.array([0.05, 0.01])}
    # C = 0 and D = 0 give y = 0
    _, y = rc.mamba2_step(S0, tok["x"], tok["B"], tok["C"], tok["dt"], A, np.zeros(H), [0, 0])
    assert np.all(y == 0)
    # linearity of y in (S0, x) for fixed B, C, dt
    tok["C"] = rng.standard_normal((1, N))
    D = rng.standard_normal(H)
    S1 = rng.standard_normal((H, P, N))
    x1 = rng.standard_normal((H, P))
    f = lambda S, x: rc.mamba2_step(S, x, tok["B"], tok["C"], tok["dt"], A, D, [0, 0])[1]
    np.testing.assert_allclose(f(2.0 * S0 + S1, 2.0 * tok["x"] + x1), 2.0 * f(S0, tok["x"]) + f(S1, x1),
                               rtol=1e-12, atol=1e-12)
    # dt -> 0 leaves the state unchanged: y = S0 C + D x
    _, y0 = rc.mamba2_step(S0, tok["x"], tok["B"], tok["C"], np.zeros(H), A, D, [0, 0])
    np.testing.assert_allclose(y0, S0 @ tok["C"][0] + D[:, None] * tok["x"], rtol=1e-13)


# ----------------------------------------------------------------------------- Gated DeltaNet

def _gdn_bruteforce(S0, toks, q_scale):
    """S_t = alpha S (I - beta k k^T) + beta v k^T with the matrices formed element by element."""
    dv, dk = len(S0), len(S0[0])
    S = [row[:] for row in S0]
    ys = []
    for tok in toks:
        k, v, a, b, q = tok["k"], tok["v"], tok["alpha"], tok["beta"], tok["q"]
        M = [[(1.0 if i == j else 0.0) - b * k[i] * k[j] for j in range(dk)] for i in range(dk)]
        S = [[a * sum(S[r][m] * M[m][c] for m in range(dk)) + b * v[r] * k[c] for c in range(dk)] for r in range(dv)]
        ys.append([q_scale * sum(S[r][c] * q[c] for c in range(dk)) for r in range(dv)])
    return S, ys


def test_gdn_bruteforce_rectangular():
    """d_v != d_k so that a transposed operand cannot pass."""
    rng = np.random.default_rng(11)
    dv, dk, steps, qs = 3, 5, 9, 0.7
    S0 = rng.standard_normal((dv, dk))
    toks = []
    for _ in range(steps):
        k = rng.standard_normal(dk)
        q = rng.standard_normal(dk)
        toks.append({"q": q / np.linalg.norm(q), "k": k / np.linalg.norm(k), "v": rng.standard_normal(dv),
                     "alpha": rng.uniform(0.8, 1.0), "beta": rng.uniform(0.0, 1.0)})
    S_bf, ys_bf = _gdn_bruteforce(S0.tolist(), [{k: (v.tolist() if isinstance(v, np.ndarray) else v)
                                                  for k, v in t.items()} for t in toks], qs)
    S = S0[None]
    for t, tok in enumerate(toks):
        arr = {k: np.asarray(v)[None] for k, v in tok.items()}
        S, y = rc.gdn_step(S, arr["q"], arr["k"], arr["v"], arr["alpha"], arr["beta"], qs)
        np.testing.assert_allclose(y[0], ys_bf[t], rtol=1e-12, atol=1e-13)
        recs = [{k: np.asarray(v)[None] for k, v in tt.items()} for tt in toks[: t + 1]]
        y_rep = rc.gdn_replay_output(S0[None], recs, arr["q"], qs)
        np.testing.assert_allclose(y_rep, y, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S[0], np.array(S_bf), rtol=1e-12, atol=1e-13)
    recs = [{k: np.asarray(v)[None] for k, v in tt.items()} for tt in toks]
    np.testing.assert_allclose(rc.gdn_fold(S0[None], recs)[0], S[0], rtol=1e-12, atol=1e-13)


def test_gdn_delta_rule_exact_write():
    """alpha = beta = 1 and a unit key: S_t k = v_t (the delta rule overwrites the value at k)."""
    rng = np.random.default_rng(5)
    dv, dk = 6, 8
    S = rng.standard_normal((1, dv, dk))
    for _ in range(5):
        k = rng.standard_normal(dk)
        k /= np.linalg.norm(k)
        v = rng.standard_normal(dv)
        S, y = rc.gdn_step(S, k[None], k[None], v[None], np.ones(1), np.ones(1))
        np.testing.assert_allclose(y[0], v, rtol=1e-12, atol=1e-12)


def test_gdn_orthonormal_keys_and_pure_decay():
    rng = np.random.default_rng(9)
    dv, dk, m = 4, 8, 5
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys, vals = Q[:, :m].T, rng.standard_normal((m, dv))
    S0 = rng.standard_normal((1, dv, dk))
    recs = [{"k": keys[i][None], "v": vals[i][None], "alpha": np.ones(1), "beta": np.ones(1)} for i in range(m)]
    S = rc.gdn_fold(S0, recs)
    for i in range(m):                               # every written key reads back its value
        np.testing.assert_allclose(S[0] @ keys[i], vals[i], rtol=1e-12, atol=1e-12)
    q_perp = Q[:, m]                                  # orthogonal to every key: reads the old state
    np.testing.assert_allclose(S[0] @ q_perp, S0[0] @ q_perp, rtol=1e-12, atol=1e-12)
    # beta = 0: the state only decays, y = (prod alpha) S0 q
    alphas = rng.uniform(0.5, 1.0, 7)
    recs = [{"k": keys[0][None], "v": vals[0][None], "alpha": np.array([a]), "beta": np.zeros(1)} for a in alphas]
    y = rc.gdn_replay_output(S0, recs, q_perp[None])
    np.testing.assert_allclose(y[0], np.prod(alphas) * (S0[0] @ q_perp), rtol=1e-12)


# ----------------------------------------------------------------------------- the pages' invariant at workload shapes

def test_replay_equals_stepwise_mamba2_workload_shape():
    from synth import MAMBA2_TINY, mamba2_params, mamba2_step_inputs
    wl = MAMBA2_TINY.replace(batch=2, init="normal")
    p = mamba2_params(wl)
    hg = [0] * wl.nheads
    rng = np.random.default_rng(0)
    S0 = rng.standard_normal((2, wl.nheads, wl.headdim, wl.dstate)) * 0.05
    S = S0.copy()
    recs = []
    for t in range(wl.window):
        tok = mamba2_step_inputs(wl, t)
        recs.append(tok)
        S, y = rc.mamba2_step(S, tok["x"], tok["B"], tok["C"], tok["dt"], p["A"], p["D"], hg)
        y_rep = rc.mamba2_replay_output(S0, recs, tok["C"], p["A"], p["D"], hg)
        assert np.linalg.norm(y_rep - y) <= 1e-12 * np.linalg.norm(y)
    assert np.linalg.norm(rc.mamba2_fold(S0, recs, p["A"], hg) - S) <= 1e-12 * np.linalg.norm(S)


def test_replay_equals_stepwise_gdn_workload_shape():
    from synth import GDN_B256, gdn_initial_state, gdn_step_inputs
    wl = GDN_B256.replace(batch=2, nheads=3)
    S0 = gdn_initial_state(wl).astype(np.float64)
    S = S0.copy()
    recs = []
    for t in range(wl.window):
        tok = gdn_step_inputs(wl, t)
        recs.append(tok)
        S, y = rc.gdn_step(S, tok["q"], tok["k"], tok["v"], tok["alpha"], tok["beta"])
        y_rep = rc.gdn_replay_output(S0, recs, tok["q"])
        assert np.linalg.norm(y_rep - y) <= 1e-12 * np.linalg.norm(y)
    assert np.linalg.norm(rc.gdn_fold(S0, recs) - S) <= 1e-12 * np.linalg.norm(S)


@pytest.mark.parametrize("m,decay", [(1, 0.05), (5, 0.05), (16, 0.05), (16, 3.0)])
def test_gdn_fold_rank_m_form(m, decay):
    """The chunked form the GPU fold uses equals folding the records one by one: with a_r = prod_{j<=r} alpha_j,
    b_r = prod_{r<j<m} alpha_j, L_ri = beta_r (prod_{i<j<=r} alpha_j) k_i.k_r (i < r) and T = (I + L)^-1,
    each row s becomes a_{m-1} s + sum_r b_r u_r k_r with u = T rt, rt_r = beta_r (v_r[row] - a_r s.k_r).
    Written out here in float64 with numpy's inverse; decay 3.0 spreads alpha down to ~0.05 (products far
    below one), and m = 1 leaves L empty."""
    from synth import GDN_B256, gdn_initial_state, gdn_step_inputs
    wl = GDN_B256.replace(batch=2, nheads=3, decay_scale=decay)
    S0 = gdn_initial_state(wl).astype(np.float64)
    recs = [gdn_step_inputs(wl, t) for t in range(m)]
    want = rc.gdn_fold(S0, recs)
    K = np.stack([np.asarray(r["k"], np.float64) for r in recs], axis=-2)        # [B, H, m, dk]
    V = np.stack([np.asarray(r["v"], np.float64) for r in recs], axis=-1)        # [B, H, dv, m]
    al = np.stack([np.asarray(r["alpha"], np.float64) for r in recs], axis=-1)   # [B, H, m]
    be = np.stack([np.asarray(r["beta"], np.float64) for r in recs], axis=-1)
    got = np.empty_like(want)
    for b in range(wl.batch):
        for h in range(wl.nheads):
            k, v, a_, bt = K[b, h], V[b, h], al[b, h], be[b, h]
            a = np.cumprod(a_)
            bsuf = np.array([np.prod(a_[r + 1:]) for r in range(m)])
            L = np.zeros((m, m))
            for r in range(m):
                for i in range(r):
                    L[r, i] = bt[r] * np.prod(a_[i + 1:r + 1]) * (k[i] @ k[r])
            T = np.linalg.inv(np.eye(m) + L)
            Z = S0[b, h] @ k.T                                  # [dv, m]
            rt = bt[None, :] * (v - a[None, :] * Z)
            U = rt @ T.T
            got[b, h] = a[-1] * S0[b, h] + (U * bsuf[None, :]) @ k
    assert np.linalg.norm(got - want) <= 1e-12 * np.linalg.norm(want)
