"""Shared helpers for the GPU parity tests: oracle configs, comparisons.

Tolerances (from the method's stated targets, applied on the same
bf16-rounded inputs):
  fp32 path  : 1e-4 max-abs on every floating-point output
  bf16 path  : 2e-2 max-abs on every floating-point output
  block idx  : bit-exact, except rows where the oracle's k-th and (k+1)-th
               candidate scores differ by less than 1e-5 (relative); such a
               row must still hold a valid selection.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
from sparse_attention_nsa_b200 import inputs as W

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
LSE_TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-3}
NEAR_TIE = 1e-5


def ocfg(w: W.Workload, **kw) -> orc.Cfg:
    """Oracle config for a workload; compressed keys/values and the branch
    outputs the gate gradient reads are stored in the path's dtype, exactly
    as the library stores them (readings R13 and R15)."""
    c = orc.Cfg(B=w.B, T=w.T, Hq=w.Hq, Hkv=w.Hkv, D=w.D, cmp_block=w.cmp_block,
                cmp_stride=w.cmp_stride, sel_block=w.sel_block, topk=w.topk,
                window=w.window, scale=w.scale,
                kv_round=orc.KV_BF16 if w.dtype == torch.bfloat16 else orc.KV_F32,
                branch_mask=w.branch_mask,
                o_round=orc.KV_BF16 if w.dtype == torch.bfloat16 else orc.KV_F32)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy() if t.dtype != torch.int32 \
        else t.detach().cpu().numpy()


def max_abs(a, b) -> float:
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    d = np.where(both_inf, 0.0, np.abs(a - b))
    return float(np.nanmax(d)) if d.size else 0.0


def assert_close(got, want, tol, what=""):
    err = max_abs(got, want)
    assert np.all(np.isfinite(got) == np.isfinite(want)), f"{what}: finiteness differs"
    assert err <= tol, f"{what}: max-abs error {err:.3e} > {tol:.1e}"
    return err


def candidate_ranking(score_row: np.ndarray, cur: int) -> list[int]:
    return sorted(range(1, cur), key=lambda j: (-score_row[j], j))


def idx_mismatch_rows(gpu_idx, orc_idx, orc_score, t_of_row, topk, l, band=None):
    """Compare selections row by row.  Returns the boolean mask of rows that
    differ; asserts that every differing row is a near-tie of the oracle's
    scores and that the GPU's selection is a valid one for that row.  band:
    optional per-row relative near-tie width (default NEAR_TIE), for paths
    whose scores may move by a known bound."""
    g = gpu_idx.reshape(-1, topk)
    o = orc_idx.reshape(-1, topk)
    s = orc_score.reshape(g.shape[0], -1)
    t = np.asarray(t_of_row).reshape(-1)
    bw = np.full(g.shape[0], NEAR_TIE) if band is None else np.asarray(band).reshape(-1)
    diff = np.any(g != o, axis=1)
    for r in np.nonzero(diff)[0]:
        tie = float(bw[r])
        cur = int(t[r]) // l
        assert cur + 1 > topk, f"row {r}: all-causal selection differs"
        gs = set(int(x) for x in g[r] if x >= 0)
        assert len(gs) == topk and 0 in gs and cur in gs, f"row {r}: invalid selection {g[r]}"
        assert list(g[r]) == sorted(g[r]), f"row {r}: not ascending"
        rank = candidate_ranking(s[r], cur)
        kth, nxt = s[r][rank[topk - 3]], s[r][rank[topk - 2]]
        assert abs(kth - nxt) <= tie * max(abs(kth), 1e-30), \
            f"row {r}: selections differ without a near-tie ({kth} vs {nxt})"
        # every GPU pick must score within the near-tie band of the k-th score
        for j in gs - {0, cur}:
            assert s[r][j] >= kth - tie * abs(kth) * 2, f"row {r}: block {j} not a top pick"
    return diff


def stored(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """x as the library stores it in `dtype` (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype).double().numpy()


def oracle_backward_given_idx(c: orc.Cfg, w: W.Workload, inp: dict, dout, idx) -> tuple:
    """The oracle's whole backward (dq, dk, dv, dgates) for a GIVEN selection
    idx [B, T, Hkv, topk], composed from its branch functions exactly as
    orc_backward composes them (the pins check that composition): the
    selection is a constant of the backward, so a valid selection that
    differs from the oracle's own only at near-ties has one correct
    gradient, and this is it.  The branch outputs the gate gradient reads
    are rounded to the path's dtype (reading R15)."""
    q, k, v, gates = inp["q"], inp["k"], inp["v"], inp["gates"]
    kc, vc = orc.compress(c, k, v)
    o_cmp, _, _ = orc.cmp_attn_scores(c, q, kc, vc)
    o_sel, _ = orc.sel_attn_fwd(c, q, k, v, idx)
    o_swa, _ = orc.swa_fwd(c, q, k, v)
    dg, d1, d2, d3 = orc.gate_combine_bwd(c, gates, dout, stored(o_cmp, w.dtype),
                                          stored(o_sel, w.dtype), stored(o_swa, w.dtype))
    dq = np.zeros((w.B, w.T, w.Hq, w.D))
    dk = np.zeros((w.B, w.T, w.Hkv, w.D))
    dv = np.zeros_like(dk)
    parts = []
    if w.branch_mask & W.BR_CMP:
        parts.append(orc.cmp_bwd(c, q, kc, vc, d1))
    if w.branch_mask & W.BR_SEL:
        parts.append(orc.sel_attn_bwd(c, q, k, v, idx, d2))
    if w.branch_mask & W.BR_SWA:
        parts.append(orc.swa_bwd(c, q, k, v, d3))
    for a, b_, c_ in parts:
        dq += a
        dk += b_
        dv += c_
    return dq, dk, dv, dg


def assert_dgates_close(got, want, dout, o_branches, w: W.Workload, tol, what="dgates"):
    """dgates[..., i] = dout . o_i is a 64-term dot product of the upstream
    gradient with the forward's branch output.  The oracle reads its own
    outputs rounded to the path dtype (reading R15), but the forward's own
    arithmetic (P rounded to bf16 before P.V, 2^-9 relative) moves each
    o_i,d before that rounding, and one rounding step of o_i,d (2^-9
    relative for bf16) moves the product by up to 2^-9 |dout_d o_i,d|.
    Bound per element: the dtype tolerance plus 2^-8 sum_d |dout_d o_i,d|
    (two such steps); 2^-23 instead of 2^-8 for an fp32 path."""
    do = np.asarray(dout, dtype=np.float64)
    err = np.abs(np.asarray(got) - np.asarray(want))
    rel = 2.0 ** -8 if w.dtype == torch.bfloat16 else 2.0 ** -23
    for i, o in enumerate(o_branches):
        if not w.branch_mask & (1 << i):
            assert np.all(np.asarray(got)[..., i] == 0), f"{what}[{i}]: disabled branch not 0"
            continue
        bound = tol + rel * np.abs(do * o).sum(-1)
        assert np.all(err[..., i] <= bound), \
            f"{what}[{i}]: exceeds bound by {float((err[..., i] - bound).max()):.3e}"
