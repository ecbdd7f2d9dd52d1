"""fp64 CPU oracle for Native Sparse Attention (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  It shares
no code with the CUDA library and never imports it.

The arithmetic lives in ``nsa_oracle.c`` (plain double-precision loops, one
function per step of the method, each citing the page passage it follows).
This module only converts arrays to contiguous float64 / int32 and calls it.

Layouts follow the C file: q/o [B,T,Hq,D], k/v [B,T,Hkv,D],
kc/vc [B,Nc,Hkv,D], gates [B,T,Hq,3] (cmp, sel, swa), lse [B,T,Hq],
score [B,T,Hkv,Nc], idx [B,T,Hkv,topk].
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import math
import os

import numpy as np

from . import build as _build

BR_CMP, BR_SEL, BR_SWA = 1, 2, 4
BR_ALL = BR_CMP | BR_SEL | BR_SWA

KV_KEEP, KV_F32, KV_BF16 = 0, 1, 2


class _CCfg(C.Structure):
    _fields_ = [("B", C.c_int), ("T", C.c_int), ("Hq", C.c_int),
                ("Hkv", C.c_int), ("D", C.c_int), ("cmp_block", C.c_int),
                ("cmp_stride", C.c_int), ("sel_block", C.c_int),
                ("topk", C.c_int), ("window", C.c_int),
                ("scale", C.c_double), ("kv_round", C.c_int),
                ("branch_mask", C.c_int), ("o_round", C.c_int)]


@dataclasses.dataclass
class Cfg:
    """Problem description for the oracle (independent of the CUDA ABI)."""
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int = 64
    cmp_block: int = 64
    cmp_stride: int = 64
    sel_block: int = 64
    topk: int = 16
    window: int = 512
    scale: float | None = None
    kv_round: int = KV_KEEP
    branch_mask: int = BR_ALL
    o_round: int = KV_KEEP  # precision of the stored branch outputs the gate gradient reads

    def c(self) -> _CCfg:
        s = self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)
        return _CCfg(self.B, self.T, self.Hq, self.Hkv, self.D, self.cmp_block,
                     self.cmp_stride, self.sel_block, self.topk, self.window,
                     float(s), self.kv_round, self.branch_mask, self.o_round)

    @property
    def Nc(self) -> int:
        if self.T < self.cmp_block:
            return 0
        return (self.T - self.cmp_block) // self.cmp_stride + 1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


_lib = None


def _load():
    global _lib
    if _lib is None:
        # NSA_ORACLE_LIB lets the mutation test load a deliberately broken
        # build of the oracle to show that the pins catch it.
        path = os.environ.get("NSA_ORACLE_LIB") or _build.build()
        _lib = C.CDLL(path)
        _lib.orc_round_bf16.restype = C.c_double
        _lib.orc_round_bf16.argtypes = [C.c_double]
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def round_bf16(x: float) -> float:
    """Nearest bfloat16 value of x, ties to even (the oracle's own rounding)."""
    return _load().orc_round_bf16(float(x))


def compress(cfg: Cfg, k, v):
    """Mean-pooled compressed keys and values: kc, vc [B, Nc, Hkv, D]."""
    lib = _load()
    k, v = _f64(k), _f64(v)
    kc = np.zeros((cfg.B, cfg.Nc, cfg.Hkv, cfg.D))
    vc = np.zeros_like(kc)
    cc = cfg.c()
    lib.orc_compress(C.byref(cc), _p(k), _p(v), _p(kc), _p(vc))
    return kc, vc


def cmp_attn_scores(cfg: Cfg, q, kc, vc):
    """Compression branch: (o_cmp, lse_cmp, score) for every row."""
    lib = _load()
    q, kc, vc = _f64(q), _f64(kc), _f64(vc)
    o = np.zeros((cfg.B, cfg.T, cfg.Hq, cfg.D))
    lse = np.zeros((cfg.B, cfg.T, cfg.Hq))
    score = np.zeros((cfg.B, cfg.T, cfg.Hkv, max(cfg.Nc, 1)))[..., :cfg.Nc].copy()
    cc = cfg.c()
    lib.orc_cmp_attn_scores(C.byref(cc), _p(q), _p(kc), _p(vc), _p(o), _p(lse),
                            _p(score))
    return o, lse, score


def sel_block_scores(cfg: Cfg, score):
    """Importance of every selection block [B, T, Hkv, Nb] from the
    compressed-block scores [B, T, Hkv, Nc] (the ranking top-k uses)."""
    lib = _load()
    score = _f64(score)
    nb = -(-cfg.T // cfg.sel_block)
    out = np.zeros((cfg.B, cfg.T, cfg.Hkv, nb))
    cc = cfg.c()
    lib.orc_sel_scores(C.byref(cc), _p(score), _p(out))
    return out


def select_topk(cfg: Cfg, score):
    """Per-(token, KV group) block indices [B, T, Hkv, topk], -1 padded."""
    lib = _load()
    score = _f64(score)
    idx = np.zeros((cfg.B, cfg.T, cfg.Hkv, cfg.topk), dtype=np.int32)
    cc = cfg.c()
    lib.orc_select_topk(C.byref(cc), _p(score), _p(idx))
    return idx


def sel_attn_fwd(cfg: Cfg, q, k, v, idx):
    """Selection branch over the given block indices: (o_sel, lse_sel)."""
    lib = _load()
    q, k, v, idx = _f64(q), _f64(k), _f64(v), _i32(idx)
    o = np.zeros((cfg.B, cfg.T, cfg.Hq, cfg.D))
    lse = np.zeros((cfg.B, cfg.T, cfg.Hq))
    cc = cfg.c()
    lib.orc_sel_attn_fwd(C.byref(cc), _p(q), _p(k), _p(v), _p(idx), _p(o), _p(lse))
    return o, lse


def swa_fwd(cfg: Cfg, q, k, v):
    """Sliding-window branch: (o_swa, lse_swa)."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    o = np.zeros((cfg.B, cfg.T, cfg.Hq, cfg.D))
    lse = np.zeros((cfg.B, cfg.T, cfg.Hq))
    cc = cfg.c()
    lib.orc_swa_fwd(C.byref(cc), _p(q), _p(k), _p(v), _p(o), _p(lse))
    return o, lse


def gate_combine(cfg: Cfg, gates, o_cmp, o_sel, o_swa):
    """out = sum over enabled branches of gate * branch output."""
    lib = _load()
    gates, o_cmp, o_sel, o_swa = _f64(gates), _f64(o_cmp), _f64(o_sel), _f64(o_swa)
    out = np.zeros((cfg.B, cfg.T, cfg.Hq, cfg.D))
    cc = cfg.c()
    lib.orc_gate_combine(C.byref(cc), _p(gates), _p(o_cmp), _p(o_sel), _p(o_swa),
                         _p(out))
    return out


def forward(cfg: Cfg, q, k, v, gates) -> dict:
    """Whole NSA forward; returns every intermediate tensor by name."""
    lib = _load()
    q, k, v, gates = _f64(q), _f64(k), _f64(v), _f64(gates)
    B, T, Hq, Hkv, D, Nc = cfg.B, cfg.T, cfg.Hq, cfg.Hkv, cfg.D, cfg.Nc
    r = {
        "kc": np.zeros((B, Nc, Hkv, D)), "vc": np.zeros((B, Nc, Hkv, D)),
        "o_cmp": np.zeros((B, T, Hq, D)), "lse_cmp": np.zeros((B, T, Hq)),
        "score": np.zeros((B, T, Hkv, Nc)),
        "idx": np.zeros((B, T, Hkv, cfg.topk), dtype=np.int32),
        "o_sel": np.zeros((B, T, Hq, D)), "lse_sel": np.zeros((B, T, Hq)),
        "o_swa": np.zeros((B, T, Hq, D)), "lse_swa": np.zeros((B, T, Hq)),
        "out": np.zeros((B, T, Hq, D)),
    }
    cc = cfg.c()
    lib.orc_forward(C.byref(cc), _p(q), _p(k), _p(v), _p(gates), _p(r["kc"]),
                    _p(r["vc"]), _p(r["o_cmp"]), _p(r["lse_cmp"]), _p(r["score"]),
                    _p(r["idx"]), _p(r["o_sel"]), _p(r["lse_sel"]), _p(r["o_swa"]),
                    _p(r["lse_swa"]), _p(r["out"]))
    return r


def forward_rows(cfg: Cfg, q, k, v, gates, rows, kc=None, vc=None) -> dict:
    """Forward for a sample of tokens.  rows: int array [n, 2] of (b, t).

    Every output is packed per sampled token (leading dim n).  kc/vc are
    computed with `compress` unless given (they must be the oracle's own).
    """
    lib = _load()
    q, k, v, gates = _f64(q), _f64(k), _f64(v), _f64(gates)
    if kc is None or vc is None:
        kc, vc = compress(cfg, k, v)
    kc, vc = _f64(kc), _f64(vc)
    rows = _i32(np.asarray(rows).reshape(-1, 2))
    n = rows.shape[0]
    Hq, Hkv, D, Nc = cfg.Hq, cfg.Hkv, cfg.D, cfg.Nc
    r = {
        "o_cmp": np.zeros((n, Hq, D)), "lse_cmp": np.zeros((n, Hq)),
        "score": np.zeros((n, Hkv, Nc)),
        "idx": np.zeros((n, Hkv, cfg.topk), dtype=np.int32),
        "o_sel": np.zeros((n, Hq, D)), "lse_sel": np.zeros((n, Hq)),
        "o_swa": np.zeros((n, Hq, D)), "lse_swa": np.zeros((n, Hq)),
        "out": np.zeros((n, Hq, D)),
    }
    cc = cfg.c()
    lib.orc_forward_rows(C.byref(cc), _p(q), _p(k), _p(v), _p(gates), _p(kc),
                         _p(vc), C.c_int(n), _p(rows), _p(r["o_cmp"]),
                         _p(r["lse_cmp"]), _p(r["score"]), _p(r["idx"]),
                         _p(r["o_sel"]), _p(r["lse_sel"]), _p(r["o_swa"]),
                         _p(r["lse_swa"]), _p(r["out"]))
    return r


def sel_attn_bwd(cfg: Cfg, q, k, v, idx, dO_sel):
    """Selection-branch gradients (dq, dk, dv) for a fixed selection."""
    lib = _load()
    q, k, v, idx, dO = _f64(q), _f64(k), _f64(v), _i32(idx), _f64(dO_sel)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    cc = cfg.c()
    lib.orc_sel_attn_bwd(C.byref(cc), _p(q), _p(k), _p(v), _p(idx), _p(dO),
                         _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def swa_bwd(cfg: Cfg, q, k, v, dO_swa):
    """Window-branch gradients (dq, dk, dv)."""
    lib = _load()
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO_swa)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    cc = cfg.c()
    lib.orc_swa_bwd(C.byref(cc), _p(q), _p(k), _p(v), _p(dO), _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def cmp_bwd(cfg: Cfg, q, kc, vc, dO_cmp):
    """Compression-branch gradients (dq, dk, dv), dk/dv on the raw rows."""
    lib = _load()
    q, kc, vc, dO = _f64(q), _f64(kc), _f64(vc), _f64(dO_cmp)
    dq = np.zeros_like(q)
    dk = np.zeros((cfg.B, cfg.T, cfg.Hkv, cfg.D))
    dv = np.zeros_like(dk)
    cc = cfg.c()
    lib.orc_cmp_bwd(C.byref(cc), _p(q), _p(kc), _p(vc), _p(dO), _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def cmp_bwd_kc(cfg: Cfg, q, kc, vc, dO_cmp):
    """Compression-branch gradients stopped at the compressed tensors:
    (dq, dkc, dvc), dkc/dvc [B, Nc, Hkv, D]."""
    lib = _load()
    q, kc, vc, dO = _f64(q), _f64(kc), _f64(vc), _f64(dO_cmp)
    dq, dkc, dvc = np.zeros_like(q), np.zeros_like(kc), np.zeros_like(vc)
    cc = cfg.c()
    lib.orc_cmp_bwd_kc(C.byref(cc), _p(q), _p(kc), _p(vc), _p(dO), _p(dq), _p(dkc), _p(dvc))
    return dq, dkc, dvc


def gate_combine_bwd(cfg: Cfg, gates, dout, o_cmp, o_sel, o_swa):
    """(dgates, dO_cmp, dO_sel, dO_swa) of the gated combination."""
    lib = _load()
    gates, dout = _f64(gates), _f64(dout)
    o_cmp, o_sel, o_swa = _f64(o_cmp), _f64(o_sel), _f64(o_swa)
    dg = np.zeros_like(gates)
    d1, d2, d3 = np.zeros_like(dout), np.zeros_like(dout), np.zeros_like(dout)
    cc = cfg.c()
    lib.orc_gate_combine_bwd(C.byref(cc), _p(gates), _p(dout), _p(o_cmp), _p(o_sel),
                             _p(o_swa), _p(dg), _p(d1), _p(d2), _p(d3))
    return dg, d1, d2, d3


def backward(cfg: Cfg, q, k, v, gates, dout):
    """Full NSA backward: (dq, dk, dv, dgates), selection held constant."""
    lib = _load()
    q, k, v, gates, dout = _f64(q), _f64(k), _f64(v), _f64(gates), _f64(dout)
    dq, dk, dv, dg = (np.zeros_like(q), np.zeros_like(k), np.zeros_like(v),
                      np.zeros_like(gates))
    cc = cfg.c()
    lib.orc_backward(C.byref(cc), _p(q), _p(k), _p(v), _p(gates), _p(dout),
                     _p(dq), _p(dk), _p(dv), _p(dg))
    return dq, dk, dv, dg


def decode(cfg: Cfg, q_last, kcache, vcache, kc, vc, gates_last, with_score=False):
    """One query per sequence at position T-1 (cfg.T = cache length).

    q_last [B, Hq, D], caches [B, T, Hkv, D], kc/vc [B, Nc, Hkv, D],
    gates_last [B, Hq, 3].  Returns (out [B, Hq, D], idx [B, Hkv, topk]),
    plus the block scores [B, Hkv, Nc] when with_score=True.
    """
    lib = _load()
    q_last, kcache, vcache = _f64(q_last), _f64(kcache), _f64(vcache)
    kc, vc, gates_last = _f64(kc), _f64(vc), _f64(gates_last)
    out = np.zeros((cfg.B, cfg.Hq, cfg.D))
    idx = np.zeros((cfg.B, cfg.Hkv, cfg.topk), dtype=np.int32)
    score = np.zeros((cfg.B, cfg.Hkv, max(cfg.Nc, 1)))
    cc = cfg.c()
    lib.orc_decode(C.byref(cc), _p(q_last), _p(kcache), _p(vcache), _p(kc), _p(vc),
                   _p(gates_last), _p(out), _p(idx), _p(score))
    if with_score:
        return out, idx, score[..., :cfg.Nc]
    return out, idx


def backward_dq_rows(cfg: Cfg, q, k, v, gates, dout, rows, kc=None, vc=None):
    """dq [n, Hq, D] of the full backward for a sample of (b, t) tokens."""
    lib = _load()
    q, k, v, gates, dout = _f64(q), _f64(k), _f64(v), _f64(gates), _f64(dout)
    if kc is None or vc is None:
        kc, vc = compress(cfg, k, v)
    kc, vc = _f64(kc), _f64(vc)
    rows = _i32(np.asarray(rows).reshape(-1, 2))
    dq = np.zeros((rows.shape[0], cfg.Hq, cfg.D))
    cc = cfg.c()
    lib.orc_backward_dq_rows(C.byref(cc), _p(q), _p(k), _p(v), _p(gates), _p(dout), _p(kc),
                             _p(vc), C.c_int(rows.shape[0]), _p(rows), _p(dq))
    return dq


def moba_fwd(cfg: Cfg, q, k, v):
    """MoBA block attention (cfg.cmp_block = cfg.cmp_stride = cfg.sel_block =
    the MoBA block size, cfg.topk = k): (o [B,T,Hq,D], lse [B,T,Hq],
    idx [B,T,Hkv,k] MoBA block indices)."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    o = np.zeros((cfg.B, cfg.T, cfg.Hq, cfg.D))
    lse = np.zeros((cfg.B, cfg.T, cfg.Hq))
    idx = np.zeros((cfg.B, cfg.T, cfg.Hkv, cfg.topk), dtype=np.int32)
    cc = cfg.c()
    lib.orc_moba_fwd(C.byref(cc), _p(q), _p(k), _p(v), _p(idx), _p(o), _p(lse))
    return o, lse, idx


def compress_mlp(cfg: Cfg, k, v, wk, wv):
    """Parametric compression: one linear layer over each block's l rows
    flattened in token order, wk, wv [l D, D] (reading R17)."""
    lib = _load()
    k, v, wk, wv = _f64(k), _f64(v), _f64(wk), _f64(wv)
    kc = np.zeros((cfg.B, cfg.Nc, cfg.Hkv, cfg.D))
    vc = np.zeros_like(kc)
    cc = cfg.c()
    lib.orc_compress_mlp(C.byref(cc), _p(k), _p(v), _p(wk), _p(wv), _p(kc), _p(vc))
    return kc, vc


def compress_mlp_bwd(cfg: Cfg, k, v, wk, wv, dkc, dvc):
    """(dk, dv, dwk, dwv) of compress_mlp for upstream dkc, dvc."""
    lib = _load()
    k, v, wk, wv, dkc, dvc = (_f64(x) for x in (k, v, wk, wv, dkc, dvc))
    dk, dv = np.zeros_like(k), np.zeros_like(v)
    dwk, dwv = np.zeros_like(wk), np.zeros_like(wv)
    cc = cfg.c()
    lib.orc_compress_mlp_bwd(C.byref(cc), _p(k), _p(v), _p(wk), _p(wv), _p(dkc), _p(dvc),
                             _p(dk), _p(dv), _p(dwk), _p(dwv))
    return dk, dv, dwk, dwv
