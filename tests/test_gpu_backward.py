"""GPU parity of the backward: every branch's two-pass backward, the gate
backward and the whole nsa_backward against the fp64 oracle.

Small cases are compared element by element.  One 340M-shape
sequence (T=8192) is compared element by element; the B=8 training shape on
sampled dq rows (dq is local to its row) and on an identity that holds
exactly at any size: the value gradients of a KV group sum to the gated
upstream gradient summed over every row that has at least one key in the
branch.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import sparse_attention_nsa_b200 as nsa
from sparse_attention_nsa_b200 import inputs as W

from helpers import (TOL, assert_close, assert_dgates_close, idx_mismatch_rows, ocfg,
                     oracle_backward_given_idx, to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def small(name, **kw):
    base = dict(name=name, B=1, T=256, Hq=16, Hkv=4, D=64, cmp_block=64, cmp_stride=64,
                sel_block=64, topk=4, window=96, dtype=torch.bfloat16, qk_norm=True)
    base.update(kw)
    return W.Workload(**base)


BWD = [
    W.TINY_F32,
    small("bwd_gqa4_t700_bf16", T=700, topk=5, window=150),
    small("bwd_mqa_t600_bf16", T=600, Hkv=1, topk=4, window=100, qk_norm=False),
    small("bwd_gqa2_t500_f32", T=500, Hq=4, Hkv=2, topk=3, window=90, dtype=torch.float32,
          qk_norm=False, qkv_std=0.5),
    small("bwd_l32_t300_bf16", T=300, Hq=4, Hkv=4, cmp_block=32, cmp_stride=32, sel_block=32,
          topk=3, window=40),
    small("bwd_b2_ragged_t333_bf16", B=2, T=333, topk=3, window=70),
    small("bwd_l128_t700_bf16", T=700, Hq=8, Hkv=2, cmp_block=128, cmp_stride=128,
          sel_block=128, topk=3, window=200),
    small("bwd_pruned_mqa_t500_bf16", T=500, Hkv=1, topk=4, window=64,
          branch_mask=W.BR_SEL | W.BR_SWA, cmp_gate_zero=True, qk_norm=False),
    # general geometry: overlapping compressed blocks (stride < block), and
    # compression blocks of another size than the selection block
    small("bwd_geo_l32_d16_s64_t700_bf16", T=700, cmp_block=32, cmp_stride=16, topk=5,
          window=150),
    small("bwd_geo_l128_d64_s64_mqa_t900_bf16", T=900, Hkv=1, cmp_block=128, cmp_stride=64,
          topk=4, window=100, qk_norm=False),
    small("bwd_geo_l16_d8_s32_t300_f32", T=300, Hq=4, Hkv=2, cmp_block=16, cmp_stride=8,
          sel_block=32, topk=4, window=50, dtype=torch.float32, qk_norm=False, qkv_std=0.5),
]


def dout_for(w, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((w.B, w.T, w.Hq, w.D), generator=g).to(w.dtype)


def zeros_grads(w):
    f = torch.float32
    return (torch.zeros((w.B, w.T, w.Hq, w.D), dtype=f, device=DEV),
            torch.zeros((w.B, w.T, w.Hkv, w.D), dtype=f, device=DEV),
            torch.zeros((w.B, w.T, w.Hkv, w.D), dtype=f, device=DEV))


def bwd_ws(p):
    return torch.empty(nsa.nsa_backward_workspace_size(p), dtype=torch.uint8, device=DEV)


@pytest.mark.parametrize("w", BWD[:7], ids=lambda w: w.name)
def test_sel_attn_bwd_two_pass(cuda_lib, w):
    inp = W.make_inputs(w, seed=31)
    c = ocfg(w)
    r = orc.forward(c, inp["q"], inp["k"], inp["v"], inp["gates"])
    g = torch.Generator().manual_seed(32)
    dO = torch.randn((w.B, w.T, w.Hq, w.D), generator=g)
    want = orc.sel_attn_bwd(c, inp["q"], inp["k"], inp["v"], r["idx"], dO)
    p = nsa.params_for(w)
    d = {k_: v_.to(DEV) for k_, v_ in inp.items()}
    idx = torch.from_numpy(r["idx"]).to(DEV)
    o = torch.empty((w.B, w.T, w.Hq, w.D), dtype=w.dtype, device=DEV)
    lse = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=DEV)
    nsa.nsa_sel_attn_fwd(p, d["q"], d["k"], d["v"], idx, o, lse)
    dq, dk, dv = zeros_grads(w)
    ws = bwd_ws(p)
    nsa.nsa_sel_attn_bwd(p, d["q"], d["k"], d["v"], idx, o, lse, dO.to(DEV), dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    for got, ref, name in zip((dq, dk, dv), want, ("dq", "dk", "dv")):
        assert_close(to_np(got), ref, TOL[w.dtype], name)
    # gradients accumulate: a second call doubles them
    nsa.nsa_sel_attn_bwd(p, d["q"], d["k"], d["v"], idx, o, lse, dO.to(DEV), dq, dk, dv, ws)
    assert_close(to_np(dk), 2 * want[1], 2 * TOL[w.dtype], "dk twice")


@pytest.mark.parametrize("w", [BWD[1], BWD[2], BWD[5], BWD[7],
                               small("bwd_atomic_gqa4_t2100_k6_bf16", T=2100, topk=6)],
                         ids=lambda w: w.name)
def test_sel_attn_bwd_single_pass_atomic(cuda_lib, w):
    """The single-pass variant (dK / dV by atomics from the query-stationary
    pass) against the oracle, like the two-pass backward; union block counts
    odd and even occur across the tiles of these cases."""
    inp = W.make_inputs(w, seed=31)
    c = ocfg(w)
    r = orc.forward(c, inp["q"], inp["k"], inp["v"], inp["gates"])
    g = torch.Generator().manual_seed(32)
    dO = torch.randn((w.B, w.T, w.Hq, w.D), generator=g)
    want = orc.sel_attn_bwd(c, inp["q"], inp["k"], inp["v"], r["idx"], dO)
    p = nsa.params_for(w)
    d = {k_: v_.to(DEV) for k_, v_ in inp.items()}
    idx = torch.from_numpy(r["idx"]).to(DEV)
    o = torch.empty((w.B, w.T, w.Hq, w.D), dtype=w.dtype, device=DEV)
    lse = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=DEV)
    nsa.nsa_sel_attn_fwd(p, d["q"], d["k"], d["v"], idx, o, lse)
    dq, dk, dv = zeros_grads(w)
    nsa.nsa_sel_attn_bwd_atomic(p, d["q"], d["k"], d["v"], idx, o, lse, dO.to(DEV), dq, dk, dv,
                                bwd_ws(p))
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    for got, ref, name in zip((dq, dk, dv), want, ("dq", "dk", "dv")):
        assert_close(to_np(got), ref, TOL[w.dtype], name)


@pytest.mark.parametrize("w", BWD[:7], ids=lambda w: w.name)
def test_swa_bwd(cuda_lib, w):
    inp = W.make_inputs(w, seed=33)
    c = ocfg(w)
    g = torch.Generator().manual_seed(34)
    dO = torch.randn((w.B, w.T, w.Hq, w.D), generator=g)
    want = orc.swa_bwd(c, inp["q"], inp["k"], inp["v"], dO)
    p = nsa.params_for(w)
    d = {k_: v_.to(DEV) for k_, v_ in inp.items()}
    o = torch.empty((w.B, w.T, w.Hq, w.D), dtype=w.dtype, device=DEV)
    lse = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=DEV)
    nsa.nsa_swa_fwd(p, d["q"], d["k"], d["v"], o, lse)
    dq, dk, dv = zeros_grads(w)
    nsa.nsa_swa_bwd(p, d["q"], d["k"], d["v"], o, lse, dO.to(DEV), dq, dk, dv, bwd_ws(p))
    for got, ref, name in zip((dq, dk, dv), want, ("dq", "dk", "dv")):
        assert_close(to_np(got), ref, TOL[w.dtype], name)


@pytest.mark.parametrize("w", BWD[:7] + BWD[8:] + [small("bwd_short_T40", T=40)],
                         ids=lambda w: w.name)
def test_cmp_bwd(cuda_lib, w):
    inp = W.make_inputs(w, seed=35)
    c = ocfg(w)
    okc, ovc = orc.compress(c, inp["k"], inp["v"])
    g = torch.Generator().manual_seed(36)
    dO = torch.randn((w.B, w.T, w.Hq, w.D), generator=g)
    want = orc.cmp_bwd(c, inp["q"], okc, ovc, dO)
    p = nsa.params_for(w)
    d = {k_: v_.to(DEV) for k_, v_ in inp.items()}
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=DEV)
    vc = torch.empty_like(kc)
    nsa.nsa_compress(p, d["k"], d["v"], kc, vc)
    o = torch.empty((w.B, w.T, w.Hq, w.D), dtype=w.dtype, device=DEV)
    lse = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=DEV)
    score = torch.empty((w.B, w.T, w.Hkv, w.Nc), dtype=torch.float32, device=DEV)
    nsa.nsa_cmp_attn_scores(p, d["q"], kc, vc, o, lse, score)
    dq, dk, dv = zeros_grads(w)
    nsa.nsa_cmp_bwd(p, d["q"], kc, vc, o, lse, dO.to(DEV), dq, dk, dv, bwd_ws(p))
    for got, ref, name in zip((dq, dk, dv), want, ("dq", "dk", "dv")):
        assert_close(to_np(got), ref, TOL[w.dtype], name)


@pytest.mark.parametrize("mask", [7, 6, 4, 1])
def test_gate_combine_bwd(cuda_lib, mask):
    w = small("gate_bwd", T=300, branch_mask=mask)
    g = torch.Generator().manual_seed(37)
    shape = (w.B, w.T, w.Hq, w.D)
    br = [torch.randn(shape, generator=g).to(w.dtype) for _ in range(3)]
    gates = torch.rand((w.B, w.T, w.Hq, 3), generator=g)
    dout = torch.randn(shape, generator=g).to(w.dtype)
    want = orc.gate_combine_bwd(ocfg(w), gates, dout, *br)
    p = nsa.params_for(w)
    dg = torch.empty((w.B, w.T, w.Hq, 3), dtype=torch.float32, device=DEV)
    dOs = [torch.full(shape, 7.0, dtype=torch.float32, device=DEV) for _ in range(3)]
    args = [b.to(DEV) if mask & (1 << i) else None for i, b in enumerate(br)]
    nsa.nsa_gate_combine_bwd(p, gates.to(DEV), dout.to(DEV), *args, dg, *dOs)
    assert_close(to_np(dg), want[0], 1e-3, "dgates")
    for i in range(3):
        if mask & (1 << i):
            assert_close(to_np(dOs[i]), want[1 + i], 1e-6, f"dO_{i}")


def gpu_fwd_bwd(w, inp, dout):
    p = nsa.params_for(w)
    d = {k_: v_.to(DEV) for k_, v_ in inp.items()}
    out, saved = nsa.forward(p, d["q"], d["k"], d["v"], d["gates"], keep=True)
    grads = nsa.backward(p, d["q"], d["k"], d["v"], d["gates"], dout.to(DEV), saved)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    return saved, grads


@pytest.mark.parametrize("w", BWD, ids=lambda w: w.name)
def test_backward_small(cuda_lib, w):
    inp = W.make_inputs(w, seed=38)
    dout = dout_for(w, 39)
    c = ocfg(w)
    saved, (dq, dk, dv, dg) = gpu_fwd_bwd(w, inp, dout)
    r = orc.forward(c, inp["q"], inp["k"], inp["v"], inp["gates"])
    if w.branch_mask & W.BR_SEL:
        np.testing.assert_array_equal(to_np(saved["idx"]), r["idx"])
    want = orc.backward(c, inp["q"], inp["k"], inp["v"], inp["gates"], dout)
    tol = TOL[w.dtype]
    for got, ref, name in zip((dq, dk, dv), want[:3], ("dq", "dk", "dv")):
        assert_close(to_np(got), ref, tol, name)
    # dgates = dout . o_i reads the forward's stored branch outputs; the
    # oracle reads its own outputs rounded the same way (reading R15)
    assert_dgates_close(to_np(dg), want[3], dout.double().numpy(),
                        (r["o_cmp"], r["o_sel"], r["o_swa"]), w, tol)


def test_backward_training_shape_sampled(cuda_lib):
    """B=8 training shape: dq on sampled rows.  Every sampled (row, group)
    whose selection differs from the oracle's must be a near-tie with a
    valid selection (its dq is then a different correct answer and is
    excluded; at most 2 % of the sampled rows)."""
    w = W.TRAIN_340M
    inp = W.make_inputs(w, seed=0, with_dout=True)
    saved, (dq, dk, dv, dg) = gpu_fwd_bwd(w, inp, inp["dout"])
    c = ocfg(w)
    rng = np.random.default_rng(40)
    ts = sorted(set([0, 63, 64, 511, 512, 1023, 1024, 4095, w.T - 1] +
                    list(rng.integers(0, w.T, 40))))
    rows = np.array([[int(rng.integers(0, w.B)), t] for t in ts])
    fr = orc.forward_rows(c, inp["q"], inp["k"], inp["v"], inp["gates"], rows)
    gi = to_np(saved["idx"])[rows[:, 0], rows[:, 1]]
    diff = idx_mismatch_rows(gi, fr["idx"], fr["score"], np.repeat(rows[:, 1], w.Hkv),
                             w.topk, w.sel_block).reshape(len(rows), w.Hkv)
    same = ~diff.any(axis=1)
    assert (~same).sum() <= max(1, int(0.02 * len(rows))), f"{(~same).sum()} near-tie rows"
    rows = rows[same]
    want = orc.backward_dq_rows(c, inp["q"], inp["k"], inp["v"], inp["gates"], inp["dout"], rows)
    assert_close(to_np(dq)[rows[:, 0], rows[:, 1]], want, TOL[w.dtype], "dq rows")
    # sum over keys of dv is the gated upstream gradient of every row with keys
    gates = inp["gates"].double()
    t = torch.arange(w.T)
    has_cmp = (t + 1 >= w.cmp_block).double()[None, :, None]
    gsum = gates[..., 0] * has_cmp + gates[..., 1] + gates[..., 2]
    want_dv = (gsum[..., None] * inp["dout"].double()).reshape(w.B, w.T, w.Hkv, w.G, w.D)
    want_dv = want_dv.sum(dim=(1, 3)).numpy()
    assert_close(to_np(dv).sum(axis=1), want_dv, 5e-2 * max(1.0, np.abs(want_dv).max()) / 10,
                 "sum dv")


def test_backward_t8192_elementwise(cuda_lib):
    """One 340M-shape sequence (T=8192, GQA-4, bf16): dq, dk, dv and dgates
    element by element against the oracle's whole backward.  The GPU's
    selection must equal the oracle's except at validated near-ties; the
    oracle's backward is then taken on the GPU's (valid) selection, which
    the backward holds constant, so nothing is excluded."""
    w = W.TRAIN_340M.replace(name="bwd_340m_b1_t8192", B=1)
    inp = W.make_inputs(w, seed=3, with_dout=True)
    saved, (dq, dk, dv, dg) = gpu_fwd_bwd(w, inp, inp["dout"])
    c = ocfg(w)
    r = orc.forward(c, inp["q"], inp["k"], inp["v"], inp["gates"])
    gi = to_np(saved["idx"])
    t_of_row = np.broadcast_to(np.arange(w.T)[None, :, None], gi.shape[:3])
    diff = idx_mismatch_rows(gi, r["idx"], r["score"], t_of_row, w.topk, w.sel_block)
    assert diff.sum() <= 0.01 * diff.size, f"{diff.sum()} near-tie (token, group) rows"
    want = oracle_backward_given_idx(c, w, inp, inp["dout"], gi)
    tol = TOL[w.dtype]
    for got, ref, name in zip((dq, dk, dv), want, ("dq", "dk", "dv")):
        assert_close(to_np(got), ref, tol, name)
    o_sel, _ = orc.sel_attn_fwd(c, inp["q"], inp["k"], inp["v"], gi)
    assert_dgates_close(to_np(dg), want[3], inp["dout"].double().numpy(),
                        (r["o_cmp"], o_sel, r["o_swa"]), w, tol)
