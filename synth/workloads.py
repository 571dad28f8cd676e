"""Seeded synthetic inputs for the ReplaySSM decode path.

This module is the one piece shared by the CPU oracle and the GPU path.  It
draws layer parameters, initial checkpoints and per-token inputs with the
distributions stated for each workload, rounds each tensor to its storage
dtype and returns float32 numpy arrays whose values are exactly representable
in that dtype.  It contains none of the method's arithmetic: no recurrence, no
replay, no fold, no quantiser.

Every tensor comes from its own PCG64 stream keyed by (workload seed, stream
id, index), so any step, draft round or sequence can be regenerated on its own
(the full-size parity tests regenerate only the sampled sequences).

Distributions (per workload family):

* Mamba-2: x ~ N(0,1); B, C ~ N(0, 1/N); dt = clamp(softplus(z + dt_bias_h),
  1e-3, 0.1) with z ~ N(0,1) and dt_bias_h = softplus^-1(exp(U(ln 1e-3, ln 0.1)))
  (log-uniform time-step bias, the usual Mamba-2 initialisation); A_h =
  -exp(U(0, ln 16)) (times decay_scale, 1 unless a case asks for faster decay);
  D_h ~ N(0,1).  Initial checkpoint zero (tiny workload) or
  N(0, 0.05^2).
* Gated DeltaNet: q, k = z/||z|| per head with z ~ N(0, I), normalised in fp32
  and then rounded; v ~ N(0,1); beta = sigmoid(N(0,1)); alpha =
  exp(-softplus(N(0,1)) * decay_scale) with decay_scale 0.05 (alpha mostly in
  (0.9, 1)).  Initial checkpoint N(0, 1/d_k).  Optionally the state gets row
  and column structure: v channel i of head h scaled by exp(value_spread *
  N(0,1)) and key dimension j of q and k by exp(key_spread * N(0,1)) before the
  normalisation, both fixed per layer (drawn once, from the parameter stream).
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np

__all__ = [
    "Mamba2Workload", "GDNWorkload",
    "MAMBA2_TINY", "MAMBA2_120B", "GDN_B256", "SPEC_MAMBA2_B512", "GDN_LOWPREC",
    "round_to_dtype", "mamba2_params", "mamba2_initial_state", "mamba2_step_inputs",
    "mamba2_draft_inputs", "gdn_initial_state", "gdn_step_inputs", "gdn_draft_inputs",
    "accepted_lengths", "group_of_head",
]

# stream ids: one independent PCG64 stream per tensor kind
_S_PARAMS, _S_INIT, _S_X, _S_B, _S_C, _S_DT, _S_Q, _S_K, _S_V, _S_ALPHA, _S_BETA, _S_ACC = range(12)
_S_DRAFT_OFFSET = 100  # draft-round streams live above the step streams


@dataclass(frozen=True)
class Mamba2Workload:
    name: str
    batch: int
    nheads: int
    headdim: int      # P
    dstate: int       # N
    ngroups: int      # G; head h reads group h // (nheads // ngroups)
    window: int       # L
    steps: int
    in_dtype: str     # "f32" or "bf16": storage dtype of x, B, C, dt
    init: str         # "zero" or "normal"
    seed: int
    init_std: float = 0.05
    decay_scale: float = 1.0   # multiplies A_h (faster-decaying heads for the decay-aware skipping cases)

    kind = "mamba2"

    def replace(self, **kw) -> "Mamba2Workload":
        return dataclasses.replace(self, **kw)

    @property
    def state_bytes(self) -> int:
        return self.batch * self.nheads * self.headdim * self.dstate * 4


@dataclass(frozen=True)
class GDNWorkload:
    name: str
    batch: int
    nheads: int
    dk: int
    dv: int
    window: int
    steps: int
    in_dtype: str     # storage dtype of q, k, v ("bf16" or "f32"); alpha, beta are fp32
    seed: int
    decay_scale: float = 0.05
    q_scale: float = 1.0
    value_spread: float = 0.0  # sigma of a log-normal scale per (head, value channel); 0 = none
    key_spread: float = 0.0    # sigma of a log-normal scale per (head, key dimension) of q and k; 0 = none

    kind = "gdn"

    def replace(self, **kw) -> "GDNWorkload":
        return dataclasses.replace(self, **kw)

    @property
    def state_bytes(self) -> int:
        return self.batch * self.nheads * self.dv * self.dk * 4


# The five workloads of the study: tiny Mamba-2 (parity at every step),
# a Mamba-2 layer shaped like a 120B-class hybrid (4 MiB fp32 state per
# sequence), a Gated DeltaNet layer, speculative verify/commit on the Mamba-2
# shape at batch 512, and separate-precision GDN decode.
MAMBA2_TINY = Mamba2Workload("mamba2_tiny", batch=4, nheads=8, headdim=64, dstate=128, ngroups=1,
                             window=16, steps=64, in_dtype="f32", init="zero", seed=1)
MAMBA2_120B = Mamba2Workload("mamba2_b256", batch=256, nheads=128, headdim=64, dstate=128, ngroups=8,
                             window=16, steps=1024, in_dtype="bf16", init="normal", seed=2)
GDN_B256 = GDNWorkload("gdn_b256", batch=256, nheads=32, dk=128, dv=128, window=16, steps=1024,
                       in_dtype="bf16", seed=3)
SPEC_MAMBA2_B512 = MAMBA2_120B.replace(name="spec_mamba2_b512", batch=512, steps=256, seed=4)
GDN_LOWPREC = GDN_B256.replace(name="gdn_lowprec", steps=4096, seed=5)


def _rng(seed: int, stream: int, index: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, index])))


def round_to_dtype(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to ``dtype`` (round-to-nearest-even) and return them as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    if dtype == "f32":
        return a
    if dtype == "bf16":
        bits = a.view(np.uint32)
        lsb = (bits >> np.uint32(16)) & np.uint32(1)
        out = (bits + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
        return out.view(np.float32)
    if dtype == "f16":
        return a.astype(np.float16).astype(np.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


def group_of_head(h: int, nheads: int, ngroups: int) -> int:
    return h // (nheads // ngroups)


def _softplus(z: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, z)


def mamba2_params(wl: Mamba2Workload) -> dict:
    """Per-head layer parameters: A_h < 0 and D_h (fp32), plus the dt bias used by the generator."""
    r = _rng(wl.seed, _S_PARAMS, 0)
    A = -np.exp(r.uniform(0.0, np.log(16.0), wl.nheads)) * wl.decay_scale
    D = r.standard_normal(wl.nheads)
    dt0 = np.exp(r.uniform(np.log(1e-3), np.log(0.1), wl.nheads))
    dt_bias = dt0 + np.log(-np.expm1(-dt0))  # inverse softplus
    return {"A": A.astype(np.float32), "D": D.astype(np.float32), "dt_bias": dt_bias.astype(np.float32)}


def mamba2_initial_state(wl: Mamba2Workload, seqs=None) -> np.ndarray:
    """Initial fp32 checkpoint [len(seqs)][H][P][N]; each sequence has its own stream."""
    seqs = range(wl.batch) if seqs is None else seqs
    shape = (wl.nheads, wl.headdim, wl.dstate)
    out = np.zeros((len(seqs),) + shape, np.float32)
    if wl.init == "zero":
        return out
    for i, b in enumerate(seqs):
        out[i] = _rng(wl.seed, _S_INIT, b).standard_normal(shape, dtype=np.float32) * np.float32(wl.init_std)
    return out


def _mamba2_tokens(wl: Mamba2Workload, stream_base: int, index: int, lead: tuple) -> dict:
    p = mamba2_params(wl)
    x = _rng(wl.seed, stream_base + _S_X, index).standard_normal(lead + (wl.nheads, wl.headdim), dtype=np.float32)
    sd = np.float32(1.0 / np.sqrt(wl.dstate))
    B = _rng(wl.seed, stream_base + _S_B, index).standard_normal(lead + (wl.ngroups, wl.dstate), dtype=np.float32) * sd
    C = _rng(wl.seed, stream_base + _S_C, index).standard_normal(lead + (wl.ngroups, wl.dstate), dtype=np.float32) * sd
    z = _rng(wl.seed, stream_base + _S_DT, index).standard_normal(lead + (wl.nheads,))
    dt = np.clip(_softplus(z + p["dt_bias"].astype(np.float64)), 1e-3, 0.1).astype(np.float32)
    d = wl.in_dtype
    return {"x": round_to_dtype(x, d), "B": round_to_dtype(B, d), "C": round_to_dtype(C, d),
            "dt": round_to_dtype(dt, d)}


def mamba2_step_inputs(wl: Mamba2Workload, step: int) -> dict:
    """One decode token for every sequence: x [Bt][H][P], B, C [Bt][G][N], dt [Bt][H] (post-softplus)."""
    return _mamba2_tokens(wl, 0, step, (wl.batch,))


def mamba2_draft_inputs(wl: Mamba2Workload, rnd: int, T: int) -> dict:
    """T draft tokens per sequence for verify round ``rnd``: leading dims [Bt][T]."""
    return _mamba2_tokens(wl, _S_DRAFT_OFFSET, rnd, (wl.batch, T))


def gdn_initial_state(wl: GDNWorkload, seqs=None) -> np.ndarray:
    """Initial fp32 checkpoint [len(seqs)][H][d_v][d_k], entries N(0, 1/d_k)."""
    seqs = range(wl.batch) if seqs is None else seqs
    shape = (wl.nheads, wl.dv, wl.dk)
    out = np.zeros((len(seqs),) + shape, np.float32)
    sd = np.float32(1.0 / np.sqrt(wl.dk))
    for i, b in enumerate(seqs):
        out[i] = _rng(wl.seed, _S_INIT, b).standard_normal(shape, dtype=np.float32) * sd
    return out


def _unit_rows(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.float32)
    n = np.sqrt(np.sum(z * z, axis=-1, keepdims=True, dtype=np.float32))
    return z / n


def gdn_structure(wl: GDNWorkload):
    """Per-layer scales (value channels [H][d_v], key dimensions [H][d_k]) of a structured GDN workload, or
    None where the spread is 0."""
    r = _rng(wl.seed, _S_PARAMS, 1)
    vs = r.standard_normal((wl.nheads, wl.dv))
    ks = r.standard_normal((wl.nheads, wl.dk))
    v_scale = np.exp(wl.value_spread * vs).astype(np.float32) if wl.value_spread else None
    k_scale = np.exp(wl.key_spread * ks).astype(np.float32) if wl.key_spread else None
    return v_scale, k_scale


def _gdn_tokens(wl: GDNWorkload, stream_base: int, index: int, lead: tuple) -> dict:
    hd = lead + (wl.nheads,)
    v_scale, k_scale = gdn_structure(wl)
    zq = _rng(wl.seed, stream_base + _S_Q, index).standard_normal(hd + (wl.dk,), dtype=np.float32)
    zk = _rng(wl.seed, stream_base + _S_K, index).standard_normal(hd + (wl.dk,), dtype=np.float32)
    if k_scale is not None:
        zq, zk = zq * k_scale, zk * k_scale
    q = _unit_rows(zq)
    k = _unit_rows(zk)
    v = _rng(wl.seed, stream_base + _S_V, index).standard_normal(hd + (wl.dv,), dtype=np.float32)
    if v_scale is not None:
        v = v * v_scale
    zb = _rng(wl.seed, stream_base + _S_BETA, index).standard_normal(hd)
    za = _rng(wl.seed, stream_base + _S_ALPHA, index).standard_normal(hd)
    beta = (1.0 / (1.0 + np.exp(-zb))).astype(np.float32)
    alpha = np.exp(-_softplus(za) * wl.decay_scale).astype(np.float32)
    d = wl.in_dtype
    return {"q": round_to_dtype(q, d), "k": round_to_dtype(k, d), "v": round_to_dtype(v, d),
            "alpha": alpha, "beta": beta}


def gdn_step_inputs(wl: GDNWorkload, step: int) -> dict:
    """One decode token per sequence: q, k [Bt][H][d_k], v [Bt][H][d_v], alpha, beta [Bt][H]."""
    return _gdn_tokens(wl, 0, step, (wl.batch,))


def gdn_draft_inputs(wl: GDNWorkload, rnd: int, T: int) -> dict:
    return _gdn_tokens(wl, _S_DRAFT_OFFSET, rnd, (wl.batch, T))


def accepted_lengths(wl, rnd: int, T: int) -> np.ndarray:
    """Accepted draft count per sequence for verify round ``rnd``, uniform on 0..T (int32 [Bt])."""
    return _rng(wl.seed, _S_ACC, rnd * 64 + T).integers(0, T + 1, wl.batch).astype(np.int32)
