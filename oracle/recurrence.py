"""Step-by-step recurrences, replay formulas and folds in float64 (oracle; test infrastructure only).

Mamba-2 (Dao & Gu 2024, selective SSM with a scalar decay per head), for one
sequence and head h reading group g(h), with S in R^{P x N}:

    dA_t = exp(dt_t * A_h)
    S_t  = dA_t * S_{t-1} + dt_t * x_t B_t^T
    y_t  = S_t C_t + D_h * x_t

Gated DeltaNet (Yang et al. 2024, gated delta rule), with S in R^{d_v x d_k}:

    S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
    y_t = q_scale * S_t q_t

Conventional decoding applies these one token at a time, reading and writing S
every step ("Hybrid-model decoding has a new bottleneck", Interpretation,
second paragraph; "SSM decoding stops writing state every step",
Interpretation, first paragraph).

ReplaySSM keeps a checkpoint S_0 and the inputs of the k tokens since it, and
computes y_k from them without forming S_k ("SSM decoding stops writing state
every step", Interpretation, second paragraph: a non-flush step appends its
inputs and computes the output from the checkpoint and the buffer).  Unrolling
the recurrences gives the replay formulas below.  The pages state that these
outputs equal conventional decoding up to floating-point differences ("NVIDIA
and Dao AI Lab speed up hybrid-model decoding", third paragraph); the tests
check exactly that.

Shapes: leading dimensions are free (batch, selected heads).  Mamba-2 B and C
arrive per group and are expanded to heads with ``head_group``, a list giving
each head's group.
"""

from __future__ import annotations

import numpy as np

f64 = np.float64


def _per_head(a_grouped: np.ndarray, head_group) -> np.ndarray:
    """[..., G, N] -> [..., H, N] using head h's group index head_group[h]."""
    return np.take(np.asarray(a_grouped, f64), np.asarray(head_group), axis=-2)


# --------------------------------------------------------------------------- Mamba-2

def mamba2_step(S, x, B, C, dt, A, D, head_group):
    """One conventional Mamba-2 decode step.

    S [..., H, P, N]; x [..., H, P]; B, C [..., G, N]; dt [..., H] (post-activation);
    A, D [H].  Returns (S_t, y_t) with y_t [..., H, P].
    """
    S = np.asarray(S, f64)
    x = np.asarray(x, f64)
    dt = np.asarray(dt, f64)
    Bh = _per_head(B, head_group)
    Ch = _per_head(C, head_group)
    dA = np.exp(dt * np.asarray(A, f64))
    S_new = dA[..., None, None] * S + (dt[..., None] * x)[..., :, None] * Bh[..., None, :]
    y = np.einsum("...pn,...n->...p", S_new, Ch) + np.asarray(D, f64)[:, None] * x
    return S_new, y


def mamba2_replay_output(S0, records, C, A, D, head_group):
    """y_k from the checkpoint and the buffered records, without forming S_k.

    records: list of k dicts {x [..., H, P], B [..., G, N], dt [..., H]} in token
    order; the last one is the current token.  C [..., G, N] is the current
    token's C.  Formula (unrolled Mamba-2 recurrence):

        y_k = (prod_{j<=k} dA_j) S0 C_k
              + sum_{i<=k} (prod_{i<j<=k} dA_j) dt_i (B_i . C_k) x_i + D x_k
    """
    A = np.asarray(A, f64)
    Ch = _per_head(C, head_group)
    k = len(records)
    dA = [np.exp(np.asarray(r["dt"], f64) * A) for r in records]
    total = np.ones_like(dA[0])
    for d in dA:
        total = total * d
    y = total[..., None] * np.einsum("...pn,...n->...p", np.asarray(S0, f64), Ch)
    for i in range(k):
        w = np.ones_like(dA[0])
        for j in range(i + 1, k):
            w = w * dA[j]
        g = np.sum(_per_head(records[i]["B"], head_group) * Ch, axis=-1)
        y = y + (w * np.asarray(records[i]["dt"], f64) * g)[..., None] * np.asarray(records[i]["x"], f64)
    return y + np.asarray(D, f64)[:, None] * np.asarray(records[-1]["x"], f64)


def mamba2_fold(S0, records, A, head_group):
    """New checkpoint after the buffered records (the state the recurrence reaches):

        S_k = (prod_j dA_j) S0 + sum_i (prod_{j>i} dA_j) dt_i x_i B_i^T
    """
    A = np.asarray(A, f64)
    k = len(records)
    dA = [np.exp(np.asarray(r["dt"], f64) * A) for r in records]
    total = np.ones_like(dA[0])
    for d in dA:
        total = total * d
    S = total[..., None, None] * np.asarray(S0, f64)
    for i in range(k):
        w = np.ones_like(dA[0])
        for j in range(i + 1, k):
            w = w * dA[j]
        Bh = _per_head(records[i]["B"], head_group)
        xi = np.asarray(records[i]["x"], f64)
        S = S + (w * np.asarray(records[i]["dt"], f64))[..., None, None] * xi[..., :, None] * Bh[..., None, :]
    return S


def mamba2_output(S, C, x, D, head_group):
    """y = S C + D x for a state that already includes the current token."""
    Ch = _per_head(C, head_group)
    return np.einsum("...pn,...n->...p", np.asarray(S, f64), Ch) + np.asarray(D, f64)[:, None] * np.asarray(x, f64)


# --------------------------------------------------------------------------- Gated DeltaNet

def gdn_step(S, q, k, v, alpha, beta, q_scale=1.0):
    """One conventional gated-delta-rule step.

    S [..., H, dv, dk]; q, k [..., H, dk]; v [..., H, dv]; alpha, beta [..., H].
    S_t = alpha S (I - beta k k^T) + beta v k^T ;  y = q_scale S_t q.
    """
    S = np.asarray(S, f64)
    k = np.asarray(k, f64)
    v = np.asarray(v, f64)
    a = np.asarray(alpha, f64)[..., None, None]
    b = np.asarray(beta, f64)[..., None, None]
    Sk = np.einsum("...ij,...j->...i", S, k)                      # S k
    S_new = a * (S - b * Sk[..., :, None] * k[..., None, :]) + b * v[..., :, None] * k[..., None, :]
    y = q_scale * np.einsum("...ij,...j->...i", S_new, np.asarray(q, f64))
    return S_new, y


def gdn_replay_output(S0, records, q, q_scale=1.0):
    """y_k from the checkpoint and the buffered records by walking q back.

    records: list of k dicts {k, v, alpha, beta} in token order (last = current).
    Each buffered token contributes the factor alpha_i (I - beta_i k_i k_i^T) on
    the right of S and the term beta_i v_i k_i^T.  Walking q back from the
    newest record to the oldest:

        u <- q;  r <- 0
        for i = k .. 1:  c_i = k_i . u ;  r += beta_i c_i v_i ;  u <- alpha_i (u - beta_i c_i k_i)
        y = q_scale (S0 u + r)

    so the checkpoint enters through a single matrix-vector product.
    """
    u = np.asarray(q, f64).copy()
    r = None
    for rec in reversed(records):
        kk = np.asarray(rec["k"], f64)
        b = np.asarray(rec["beta"], f64)[..., None]
        a = np.asarray(rec["alpha"], f64)[..., None]
        c = np.sum(kk * u, axis=-1, keepdims=True)
        term = b * c * np.asarray(rec["v"], f64)
        r = term if r is None else r + term
        u = a * (u - b * c * kk)
    out = np.einsum("...ij,...j->...i", np.asarray(S0, f64), u)
    if r is not None:
        out = out + r
    return q_scale * out


def gdn_fold(S0, records):
    """New checkpoint after the buffered records: the recurrence applied to each in order."""
    S = np.asarray(S0, f64)
    for rec in records:
        S, _ = gdn_step(S, np.zeros_like(np.asarray(rec["k"], f64)), rec["k"], rec["v"], rec["alpha"], rec["beta"])
    return S


def gdn_output(S, q, q_scale=1.0):
    return q_scale * np.einsum("...ij,...j->...i", np.asarray(S, f64), np.asarray(q, f64))
