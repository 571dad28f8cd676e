"""ReplaySSM decode for B200: Python binding of the C-ABI library in include/rssm.h.

Every call is marshalled straight to ``lib/librssm.so``; PyTorch provides the
device memory (the context's arena, outputs) and the current CUDA stream.

    from hybrid_model_ssm_gdn_b200 import ReplaySSM
    layer = ReplaySSM("mamba2", batch=256, nheads=128, headdim=64, ngroups=8, window=16,
                      A=A, D=D, in_dtype=torch.bfloat16)
    layer.load_checkpoint(S0)            # fp32 [Bt][H][P][N]
    y = layer.mamba2_step(x, B, C, dt)   # fp32 [Bt][H][P]
"""

from __future__ import annotations

import ctypes as C

import torch

from . import abi
from .abi import RSSMError

__all__ = ["ReplaySSM", "RSSMError", "conv_mamba2_step", "conv_gdn_step", "snap_verify", "snap_commit", "sched_probe",
           "make_config", "abi"]

_DT = {torch.float32: abi.F32, torch.bfloat16: abi.BF16}
_HP = {"f32": abi.HP_F32, "f16sr": abi.HP_F16_SR, "f8sr": abi.HP_F8_SR}
_READ = {"same": abi.READ_SAME, "nvfp4": abi.READ_NVFP4, "shared_nvfp4": abi.READ_SHARED_NVFP4,
         "nvfp4d": abi.READ_NVFP4D}


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t, dtype, name, need=None):
    """``t`` after checking that it is a contiguous CUDA tensor of ``dtype`` with at least ``need`` elements
    (what the kernels read or write through it; a smaller buffer would be overrun on the device)."""
    if t is None:
        return None
    if need is not None and t.numel() < need:
        raise ValueError(f"{name}: needs at least {need} elements, got {t.numel()} (shape {tuple(t.shape)})")
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA tensor of {dtype}, got {t.dtype} on {t.device}")
    return t


def make_config(kind, batch, nheads, headdim, dstate=128, ngroups=1, window=16, max_draft=0,
                in_dtype=torch.bfloat16, hp="f32", read="same", seed=0, q_scale=1.0, A=None, D=None,
                skip_tau=0.0) -> abi.Config:
    return abi.Config(kind={"mamba2": abi.MAMBA2, "gdn": abi.GDN}[kind], batch=batch, nheads=nheads,
                      headdim=headdim, dstate=dstate, ngroups=ngroups, window=window, max_draft=max_draft,
                      in_dtype=_DT[in_dtype], hp=_HP[hp], read=_READ[read], seed=seed, q_scale=q_scale,
                      A=None if A is None else A.data_ptr(), D=None if D is None else D.data_ptr(),
                      skip_tau=skip_tau)


class ReplaySSM:
    """One SSM layer's decode state (checkpoint, read copy, input ring, bookkeeping) on the current GPU."""

    def __init__(self, kind, batch, nheads, headdim, dstate=128, ngroups=1, window=16, max_draft=0,
                 in_dtype=torch.bfloat16, hp="f32", read="same", seed=0, q_scale=1.0, A=None, D=None,
                 device=None, skip_tau=0.0):
        self.lib = abi.load()
        self.kind, self.batch, self.nheads, self.headdim = kind, batch, nheads, headdim
        self.ngroups, self.window, self.max_draft, self.in_dtype = ngroups, window, max_draft, in_dtype
        self.device = torch.device(device or "cuda")
        if kind == "mamba2":
            # the kernels read nheads floats from each through raw pointers: check before any device copy
            for name, t in (("A", A), ("D", D)):
                if t is None or t.numel() < nheads:
                    raise ValueError(f"{name}: needs at least {nheads} elements (one per head), got "
                                     f"{None if t is None else t.numel()}")
            self.A = _dev(A.to(self.device, torch.float32).contiguous(), torch.float32, "A", nheads)
            self.D = _dev(D.to(self.device, torch.float32).contiguous(), torch.float32, "D", nheads)
        else:
            self.A = self.D = None
        self.cfg = make_config(kind, batch, nheads, headdim, dstate, ngroups, window, max_draft, in_dtype, hp, read,
                               seed, q_scale, self.A, self.D, skip_tau)
        nbytes = C.c_size_t()
        abi.check(self.lib.rssm_arena_bytes(C.byref(self.cfg), C.byref(nbytes)), "rssm_arena_bytes")
        self.arena_bytes = nbytes.value
        self.arena = torch.empty(self.arena_bytes, dtype=torch.uint8, device=self.device)
        h = C.c_void_p()
        abi.check(self.lib.rssm_create(C.byref(self.cfg), _ptr(self.arena), self.arena_bytes, C.byref(h)),
                  "rssm_create")
        self.handle = h
        self.rows = headdim
        self.dstate = dstate

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            self.lib.rssm_destroy(h)
            self.handle = None

    # ------------------------------------------------------------------ calls
    def load_checkpoint(self, S):
        S = _dev(S, torch.float32, "S", self.batch * self.nheads * self.rows * self.dstate)
        abi.check(self.lib.rssm_load_checkpoint(self.handle, _ptr(S), _stream()), "rssm_load_checkpoint")

    def _out(self, y, lead):
        if y is None:
            y = torch.empty(*lead, self.nheads, self.rows, dtype=torch.float32, device=self.device)
        n = self.nheads * self.rows
        for s in lead:
            n *= s
        return _dev(y, torch.float32, "y", n)

    def _need(self, name, lead):
        """Elements of token input ``name`` with leading dims ``lead`` ([Bt] or [Bt][T])."""
        n = 1
        for s in lead:
            n *= s
        H, R, N, G = self.nheads, self.rows, self.dstate, self.ngroups
        per = {"x": H * R, "B": G * N, "C": G * N, "dt": H, "q": H * N, "k": H * N, "v": H * R,
               "alpha": H, "beta": H}[name]
        return n * per

    def mamba2_step(self, x, B, C_, dt, y=None):
        d = self.in_dtype
        lead = (self.batch,)
        args = [_dev(x, d, "x", self._need("x", lead)), _dev(B, d, "B", self._need("B", lead)),
                _dev(C_, d, "C", self._need("C", lead)), _dev(dt, d, "dt", self._need("dt", lead))]
        y = self._out(y, lead)
        abi.check(self.lib.rssm_mamba2_step(self.handle, *map(_ptr, args), _ptr(y), _stream()), "rssm_mamba2_step")
        return y

    def gdn_step(self, q, k, v, alpha, beta, y=None):
        d = self.in_dtype
        lead = (self.batch,)
        args = [_dev(q, d, "q", self._need("q", lead)), _dev(k, d, "k", self._need("k", lead)),
                _dev(v, d, "v", self._need("v", lead)), _dev(alpha, torch.float32, "alpha", self._need("alpha", lead)),
                _dev(beta, torch.float32, "beta", self._need("beta", lead))]
        y = self._out(y, lead)
        abi.check(self.lib.rssm_gdn_step(self.handle, *map(_ptr, args), _ptr(y), _stream()), "rssm_gdn_step")
        return y

    def verify(self, T, y=None, **tok):
        d = self.in_dtype
        f32 = {"alpha", "beta"}
        t = {k: _dev(v, torch.float32 if k in f32 else d, k, self._need(k, (self.batch, T))) for k, v in tok.items()}
        toks = abi.Tokens(**{k: v.data_ptr() for k, v in t.items()})
        y = self._out(y, (self.batch, T))
        abi.check(self.lib.rssm_verify(self.handle, T, C.byref(toks), _ptr(y), _stream()), "rssm_verify")
        return y

    def commit(self, accepted):
        a = _dev(accepted, torch.int32, "accepted", self.batch)
        abi.check(self.lib.rssm_commit(self.handle, _ptr(a), _stream()), "rssm_commit")

    def flush(self, mask=None):
        m = _dev(mask, torch.uint8, "mask", self.batch)
        abi.check(self.lib.rssm_flush(self.handle, _ptr(m), _stream()), "rssm_flush")

    # ------------------------------------------------------------------ inspection
    def export(self, state=True, ring=True):
        """Return {"S": fp32 checkpoint, "meta": int32 [Bt][4], ring views...} (device tensors)."""
        dev, Bt, H, L, R = self.device, self.batch, self.nheads, self.window, self.rows
        out = {"meta": torch.empty(Bt, 4, dtype=torch.int32, device=dev)}
        if state:
            out["S"] = torch.empty(Bt, H, R, 128, dtype=torch.float32, device=dev)
        raw = None
        if ring:
            nb = C.c_size_t()
            abi.check(self.lib.rssm_ring_bytes(C.byref(self.cfg), C.byref(nb)), "rssm_ring_bytes")
            raw = torch.empty(nb.value, dtype=torch.uint8, device=dev)
        abi.check(self.lib.rssm_export(self.handle, _ptr(out.get("S")), _ptr(raw), _ptr(out["meta"]), _stream()),
                  "rssm_export")
        if raw is not None:
            esz = 2 if self.in_dtype == torch.bfloat16 else 4
            parts = ([("x", (Bt, H, L, R), esz), ("B", (Bt, self.ngroups, L, 128), esz), ("dt", (Bt, H, L), 4)]
                     if self.kind == "mamba2" else
                     [("k", (Bt, H, L, 128), esz), ("v", (Bt, H, L, R), esz), ("alpha", (Bt, H, L), 4),
                      ("beta", (Bt, H, L), 4)])
            off = 0
            for name, shape, sz in parts:
                n = 1
                for s in shape:
                    n *= s
                dt = self.in_dtype if sz == esz and name not in ("dt", "alpha", "beta") else torch.float32
                out["ring_" + name] = raw[off:off + n * sz].view(dt).view(shape)
                off += n * sz
        return out

    def export_read_copy(self):
        dev, Bt, H, R = self.device, self.batch, self.nheads, self.rows
        codes = torch.empty(Bt, H, R, 64, dtype=torch.uint8, device=dev)
        scales = torch.empty(Bt, H, R, 8, dtype=torch.uint8, device=dev)
        g = torch.empty(Bt, H, (R + 63) // 64, dtype=torch.float32, device=dev)
        abi.check(self.lib.rssm_export_read_copy(self.handle, _ptr(codes), _ptr(scales), _ptr(g), _stream()),
                  "rssm_export_read_copy")
        return {"packed": codes, "scales": scales, "g": g}

    def export_column_scales(self):
        """Column-group scales of the two-axis read copy: uint8 E4M3 [Bt][H][ceil(rows/16)][128]."""
        cs = torch.empty(self.batch, self.nheads, (self.rows + 15) // 16, 128, dtype=torch.uint8, device=self.device)
        abi.check(self.lib.rssm_export_column_scales(self.handle, _ptr(cs), _stream()), "rssm_export_column_scales")
        return cs

    def export_skip(self):
        """Decay-aware skip flags uint8 [Bt][H] (1 = the next call skips that head's checkpoint read)."""
        flags = torch.empty(self.batch, self.nheads, dtype=torch.uint8, device=self.device)
        abi.check(self.lib.rssm_export_skip(self.handle, _ptr(flags), _stream()), "rssm_export_skip")
        return flags

    def get_error(self):
        """(code, seq) of the sticky device error word; synchronises the current stream."""
        code, seq = C.c_int(), C.c_int()
        st = self.lib.rssm_get_error(self.handle, C.byref(code), C.byref(seq), _stream())
        if st not in (0, 6):
            abi.check(st, "rssm_get_error")
        return code.value, seq.value


# ---------------------------------------------------------------------- comparison kernels

def conv_mamba2_step(cfg, S, x, B, C_, dt, y):
    lib = abi.load()
    abi.check(lib.rssm_conv_mamba2_step(C.byref(cfg), *map(_ptr, (S, x, B, C_, dt, y)), _stream()),
              "rssm_conv_mamba2_step")
    return y


def conv_gdn_step(cfg, S, q, k, v, alpha, beta, y):
    lib = abi.load()
    abi.check(lib.rssm_conv_gdn_step(C.byref(cfg), *map(_ptr, (S, q, k, v, alpha, beta, y)), _stream()),
              "rssm_conv_gdn_step")
    return y


def snap_verify(cfg, snaps, cur, T, y, **tok):
    lib = abi.load()
    toks = abi.Tokens(**{k: v.data_ptr() for k, v in tok.items()})
    abi.check(lib.rssm_snap_verify(C.byref(cfg), _ptr(snaps), _ptr(cur), T, C.byref(toks), _ptr(y), _stream()),
              "rssm_snap_verify")
    return y


def sched_probe(units, blocks):
    """Run the unit-scheduler self-test (no caller device memory): -> (units drawn per block, units not drawn
    exactly once)."""
    lib = abi.load()
    per_block = (C.c_int * blocks)()
    bad = C.c_int(-1)
    abi.check(lib.rssm_sched_probe(units, blocks, C.cast(per_block, C.c_void_p), C.cast(C.pointer(bad), C.c_void_p),
                                   _stream()), "rssm_sched_probe")
    return list(per_block), bad.value


def snap_commit(cfg, cur, accepted):
    lib = abi.load()
    abi.check(lib.rssm_snap_commit(C.byref(cfg), _ptr(cur), _ptr(accepted), _stream()), "rssm_snap_commit")
