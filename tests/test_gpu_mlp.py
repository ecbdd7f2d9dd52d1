"""GPU parity of the parametric compressor (nsa_compress_mlp / _bwd) and of
the whole path on it (nsa_forward_mlp / nsa_backward_mlp) against the fp64
oracle (reading R17: one linear layer over each block's l rows flattened in
token order, weights [l*D, D] shared by every block and group).

Bounds, from the arithmetic:
  kc, vc   the library sums in fp32 and rounds once to bf16, the oracle sums
           in fp64 and rounds once: |got - ref| <= 2^-8 |ref| + the fp32
           sum's error (n 2^-24 sum|terms|), with slack (assert_rounded_sum);
           entries that differ at all stay rare (<= 1 %).
  compressor backward on given dkc, dvc: every product is exact in fp32
           except the upstream gradient's second bf16 piece (2^-9 of 2^-9
           of it); fp32 accumulation over n terms adds n 2^-24 at worst.
           Bound: 2^-13 times the same sums taken over absolute values
           (the oracle's own backward on |inputs|).
  lse_cmp  the dtype's bound plus the largest logit change the kc rounding
           bound allows (scale sum_e |q_e| bnd_e over the row's blocks).
  top-k    rows may pick differently only where the oracle's k-th and next
           scores are within the gap those logit changes can close.
  whole backward: dq, dk, dv, dgates as the mean-pool path; dW and the
           compressor's share of dk, dv carry the compression branch's
           dkc, dvc error (the bf16 tolerance, per element) through the
           layer: tolerance times the layer's backward on all-ones upstream
           and absolute inputs.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import sparse_attention_nsa_b200 as nsa
from sparse_attention_nsa_b200 import inputs as W

from helpers import (LSE_TOL, NEAR_TIE, TOL, assert_close, assert_dgates_close,
                     idx_mismatch_rows, ocfg, stored, to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def case(name, **kw):
    base = dict(name=name, B=1, T=1000, Hq=16, Hkv=4, D=64, cmp_block=32, cmp_stride=16,
                sel_block=64, topk=4, window=96, dtype=torch.bfloat16, qk_norm=True)
    base.update(kw)
    return W.Workload(**base)


CASES = [
    # the original NSA geometry: blocks of 32 every 16 tokens
    case("mlp_l32_d16_gqa4_t1000_bf16"),
    case("mlp_l64_d64_b2_t700_bf16", B=2, T=700, cmp_block=64, cmp_stride=64, topk=3,
         window=130),
    case("mlp_l16_d8_mqa_t777_bf16", T=777, Hkv=1, cmp_block=16, cmp_stride=8, topk=5,
         window=64, qk_norm=False),
    case("mlp_l8_d4_gqa2_t300_bf16", T=300, Hq=4, Hkv=2, cmp_block=8, cmp_stride=4,
         sel_block=32, topk=3, window=40),
    # odd block length: the last dW row pair is half empty
    case("mlp_l33_d7_gqa4_t400_bf16", T=400, cmp_block=33, cmp_stride=7, topk=3, window=50),
    # more than 128 compressed blocks per sequence, B > 1
    case("mlp_l32_d16_b2_gqa4_t3000_bf16", B=2, T=3000, topk=6, window=200),
]
NC0 = case("mlp_below_block_t20_bf16", T=20, cmp_block=32, cmp_stride=16, window=8)
# enough output tiles that the forward and the dA kernel run one CTA per tile
# (the cases above split the token offsets of a tile over several CTAs)
WIDE = case("mlp_mha64_t2400_bf16", T=2400, Hq=64, Hkv=64, window=64, qk_norm=False)


def dev(inp):
    return {k: v.to(DEV) for k, v in inp.items()}


def weights(w, seed=5):
    wk, wv = W.make_mlp_weights(w, seed)
    return wk, wv


def oracle_kc(w, inp, wk, wv):
    return orc.compress_mlp(ocfg(w), inp["k"], inp["v"], wk, wv)


def assert_rounded_sum(got, ref, absref, what):
    """got = bf16(fp32 sum), ref = bf16(exact sum).  The fp32 sum is off by
    at most n 2^-24 sum|terms| (n <= 2^11 products here: 2^-13), and each
    rounding moves a value by at most half a bf16 step (2^-9 relative):
    |got - ref| <= 2^-8 |ref| + 2^-12 sum|terms| (a step of slack on both).
    Entries that differ at all must stay rare (<= 1 %): only sums within the
    fp32 noise of a rounding midpoint may round the other way."""
    diff = np.abs(got - ref)
    bound = 2.0 ** -7 * np.abs(ref) + 2.0 ** -12 * absref
    assert np.all(diff <= bound), \
        f"{what}: exceeds bound by {float((diff - bound).max()):.3e}"
    frac = float((diff > 0).mean()) if diff.size else 0.0
    assert frac <= 0.01, f"{what}: {frac:.3%} of entries differ"


def abs_kc(w, inp, wk, wv):
    """sum|terms| of every compressed entry: the layer on absolute values."""
    return orc.compress_mlp(ocfg(w, kv_round=orc.KV_KEEP), np.abs(to_np(inp["k"])),
                            np.abs(to_np(inp["v"])), np.abs(to_np(wk)), np.abs(to_np(wv)))


@pytest.mark.parametrize("w", CASES + [NC0, WIDE], ids=lambda w: w.name)
def test_compress_mlp(cuda_lib, w):
    inp = W.make_inputs(w, seed=61)
    wk, wv = weights(w)
    p = nsa.params_for(w)
    d = dev(inp)
    kc = torch.full((w.B, w.Nc, w.Hkv, w.D), 7.0, dtype=w.dtype, device=DEV)
    vc = torch.full_like(kc, 7.0)
    nsa.nsa_compress_mlp(p, d["k"], d["v"], wk.to(DEV), wv.to(DEV), kc, vc)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    okc, ovc = oracle_kc(w, inp, wk, wv)
    akc, avc = abs_kc(w, inp, wk, wv)
    assert_rounded_sum(to_np(kc), okc, akc, "kc")
    assert_rounded_sum(to_np(vc), ovc, avc, "vc")


def test_compress_mlp_mean_weights_is_nsa_compress(cuda_lib):
    """Mean weights (1/32, a power of two) make the layer the mean pool:
    every product is exact, so the result is nsa_compress's (exact sum
    rounded once) up to the fp32 accumulation."""
    w = CASES[0]
    inp = W.make_inputs(w, seed=62)
    p = nsa.params_for(w)
    d = dev(inp)
    eye = torch.eye(w.D) / w.cmp_block
    wm = eye.repeat(w.cmp_block, 1).to(w.dtype).to(DEV)
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=DEV)
    vc, kc2, vc2 = torch.empty_like(kc), torch.empty_like(kc), torch.empty_like(kc)
    nsa.nsa_compress_mlp(p, d["k"], d["v"], wm, wm, kc, vc)
    nsa.nsa_compress(p, d["k"], d["v"], kc2, vc2)
    torch.cuda.synchronize()
    wm_cpu = wm.cpu()
    akc, avc = abs_kc(w, inp, wm_cpu, wm_cpu)
    assert_rounded_sum(to_np(kc), to_np(kc2), akc, "kc")
    assert_rounded_sum(to_np(vc), to_np(vc2), avc, "vc")


def upstream(w, seed):
    g = np.random.default_rng(seed)
    shape = (w.B, w.Nc, w.Hkv, w.D)
    return g.standard_normal(shape).astype(np.float32), g.standard_normal(shape).astype(np.float32)


@pytest.mark.parametrize("w", CASES + [NC0, WIDE], ids=lambda w: w.name)
def test_compress_mlp_bwd(cuda_lib, w):
    inp = W.make_inputs(w, seed=63)
    wk, wv = weights(w)
    gk, gv = upstream(w, 64)
    c = ocfg(w)
    want = orc.compress_mlp_bwd(c, inp["k"], inp["v"], wk, wv, gk, gv)
    absb = orc.compress_mlp_bwd(c, np.abs(to_np(inp["k"])), np.abs(to_np(inp["v"])),
                                np.abs(to_np(wk)), np.abs(to_np(wv)), np.abs(gk), np.abs(gv))
    p = nsa.params_for(w)
    d = dev(inp)
    f = torch.float32
    # dk, dv are added to: start from a known value
    dk = torch.full((w.B, w.T, w.Hkv, w.D), 0.5, dtype=f, device=DEV)
    dv = torch.full_like(dk, -0.25)
    dwk = torch.full((w.cmp_block * w.D, w.D), 9.0, dtype=f, device=DEV)
    dwv = torch.full_like(dwk, 9.0)
    ws = torch.empty(max(nsa.nsa_compress_mlp_bwd_workspace_size(p), 1), dtype=torch.uint8,
                     device=DEV)
    nsa.nsa_compress_mlp_bwd(p, d["k"], d["v"], wk.to(DEV), wv.to(DEV),
                             torch.from_numpy(gk).to(DEV), torch.from_numpy(gv).to(DEV),
                             dk, dv, dwk, dwv, ws)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    got = (to_np(dk) - 0.5, to_np(dv) + 0.25, to_np(dwk), to_np(dwv))
    for name, g_, r_, a_ in zip(("dk", "dv", "dwk", "dwv"), got, want, absb):
        bound = 2.0 ** -13 * a_ + 1e-6
        err = np.abs(g_ - r_)
        assert np.all(err <= bound), \
            f"{name}: exceeds bound by {float((err - bound).max()):.3e}"


def compare_mlp_forward(w, inp, wk, wv, out, saved):
    """The library's forward on the parametric compressor against the
    oracle's forward on the oracle's own compressed keys (forward_rows with
    kc, vc given, every row)."""
    c = ocfg(w)
    tol, ltol = TOL[w.dtype], LSE_TOL[w.dtype]
    okc, ovc = oracle_kc(w, inp, wk, wv)
    if w.Nc > 0:
        akc, avc = abs_kc(w, inp, wk, wv)
        assert_rounded_sum(to_np(saved["kc"]), okc, akc, "kc")
        assert_rounded_sum(to_np(saved["vc"]), ovc, avc, "vc")
    rows = np.array([[b, t] for b in range(w.B) for t in range(w.T)])
    r = orc.forward_rows(c, inp["q"], inp["k"], inp["v"], inp["gates"], rows, kc=okc, vc=ovc)
    r = {k_: v_.reshape((w.B, w.T) + v_.shape[1:]) for k_, v_ in r.items()}
    assert_close(to_np(saved["o_cmp"]), r["o_cmp"], tol, "o_cmp")
    # The library's kc may differ from the oracle's by the rounding bound
    # above, which moves logit (t, h, j) by at most scale sum_e |q_e| bnd_je;
    # lse moves by at most the largest such change (it is 1-Lipschitz in the
    # max norm of the logits): the lse bound is the dtype's plus that.
    if w.Nc > 0:
        bnd = 2.0 ** -7 * np.abs(okc) + 2.0 ** -12 * abs_kc(w, inp, wk, wv)[0]
        qa = np.abs(to_np(inp["q"])).reshape(w.B, w.T, w.Hkv, w.G, w.D)
        shift = w.scale * np.einsum("btgxe,bjge->btgxj", qa, bnd).max(-1).reshape(w.B, w.T, w.Hq)
    else:
        shift = np.zeros((w.B, w.T, w.Hq))
    lerr = np.abs(to_np(saved["lse_cmp"]) - r["lse_cmp"])
    lerr = np.where(np.isinf(r["lse_cmp"]) & (to_np(saved["lse_cmp"]) == r["lse_cmp"]), 0.0, lerr)
    assert np.all(lerr <= ltol + shift), \
        f"lse_cmp: exceeds bound by {float((lerr - ltol - shift).max()):.3e}"
    gi = to_np(saved["idx"])
    t_rows = np.broadcast_to(np.arange(w.T)[None, :, None], gi.shape[:3])
    ssel = orc.sel_block_scores(c, r["score"])
    # each head's probabilities move by at most a factor e^(+-2 shift), so a
    # group's block scores by e^(+-2 max shift) and two of them can swap order
    # only within a relative gap of 1 - e^(-4 max shift)
    dmax = shift.reshape(w.B, w.T, w.Hkv, w.G).max(-1)
    band = NEAR_TIE + (1.0 - np.exp(-4.0 * dmax))
    diff = idx_mismatch_rows(gi, r["idx"], ssel, t_rows, w.topk, w.sel_block, band=band)
    bad = diff.reshape(gi.shape[:3]).any(-1)
    assert bad.mean() < 0.01
    keep = ~bad
    assert_close(to_np(saved["o_sel"])[keep], r["o_sel"][keep], tol, "o_sel")
    assert_close(to_np(saved["o_swa"]), r["o_swa"], tol, "o_swa")
    assert_close(to_np(out)[keep], r["out"][keep], tol, "out")
    return r


@pytest.mark.parametrize("w", CASES[:5] + [NC0], ids=lambda w: w.name)
def test_forward_mlp(cuda_lib, w):
    inp = W.make_inputs(w, seed=65)
    wk, wv = weights(w)
    p = nsa.params_for(w)
    d = dev(inp)
    out, saved = nsa.forward_mlp(p, d["q"], d["k"], d["v"], wk.to(DEV), wv.to(DEV), d["gates"],
                                 keep=True)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    compare_mlp_forward(w, inp, wk, wv, out, saved)


def oracle_backward_mlp(w, inp, wk, wv, dout, idx):
    """The oracle's backward on the parametric compressor for a given
    selection, composed from its branch functions as orc_backward composes
    them, with the compression branch stopped at kc, vc and carried through
    the layer (cmp_bwd_kc, then compress_mlp_bwd)."""
    c = ocfg(w)
    q, k, v, gates = inp["q"], inp["k"], inp["v"], inp["gates"]
    okc, ovc = oracle_kc(w, inp, wk, wv)
    o_cmp, _, _ = orc.cmp_attn_scores(c, q, okc, ovc)
    o_sel, _ = orc.sel_attn_fwd(c, q, k, v, idx)
    o_swa, _ = orc.swa_fwd(c, q, k, v)
    dg, d1, d2, d3 = orc.gate_combine_bwd(c, gates, dout, stored(o_cmp, w.dtype),
                                          stored(o_sel, w.dtype), stored(o_swa, w.dtype))
    dq_c, dkc, dvc = orc.cmp_bwd_kc(c, q, okc, ovc, d1)
    dk_c, dv_c, dwk, dwv = orc.compress_mlp_bwd(c, k, v, wk, wv, dkc, dvc)
    dq_s, dk_s, dv_s = orc.sel_attn_bwd(c, q, k, v, idx, d2)
    dq_w, dk_w, dv_w = orc.swa_bwd(c, q, k, v, d3)
    return (dq_c + dq_s + dq_w, dk_c + dk_s + dk_w, dv_c + dv_s + dv_w, dwk, dwv, dg,
            (o_cmp, o_sel, o_swa))


@pytest.mark.parametrize("w", CASES[:5] + [NC0], ids=lambda w: w.name)
def test_backward_mlp(cuda_lib, w):
    inp = W.make_inputs(w, seed=66)
    wk, wv = weights(w)
    g = torch.Generator().manual_seed(67)
    dout = torch.randn((w.B, w.T, w.Hq, w.D), generator=g).to(w.dtype)
    p = nsa.params_for(w)
    d = dev(inp)
    wkd, wvd = wk.to(DEV), wv.to(DEV)
    out, saved = nsa.forward_mlp(p, d["q"], d["k"], d["v"], wkd, wvd, d["gates"], keep=True)
    dq, dk, dv, dwk, dwv, dg = nsa.backward_mlp(p, d["q"], d["k"], d["v"], wkd, wvd, d["gates"],
                                                dout.to(DEV), saved)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    compare_mlp_forward(w, inp, wk, wv, out, saved)
    # the selection is a constant of the backward: the library's (checked
    # valid above) gives the one correct gradient
    idx = to_np(saved["idx"])
    want = oracle_backward_mlp(w, inp, wk, wv, dout, idx)
    tol = TOL[w.dtype]
    c = ocfg(w)
    ones = np.ones((w.B, w.Nc, w.Hkv, w.D))
    prop = orc.compress_mlp_bwd(c, np.abs(to_np(inp["k"])), np.abs(to_np(inp["v"])),
                                np.abs(to_np(wk)), np.abs(to_np(wv)), ones, ones)
    assert_close(to_np(dq), want[0], tol, "dq")
    for name, got, ref, a_ in (("dk", dk, want[1], prop[0]), ("dv", dv, want[2], prop[1]),
                               ("dwk", dwk, want[3], prop[2]), ("dwv", dwv, want[4], prop[3])):
        bound = tol + tol * a_
        err = np.abs(to_np(got) - ref)
        print(f"{w.name} {name}: max err {err.max():.3e}, max |ref| {np.abs(ref).max():.3e}, "
              f"min slack {float((bound - err).min()):.3e}")
        assert np.all(err <= bound), \
            f"{name}: exceeds bound by {float((err - bound).max()):.3e}"
    assert_dgates_close(to_np(dg), want[5], dout.double().numpy(), want[6], w, tol)


def test_backward_mlp_without_compression_branch_zeroes_weight_grads(cuda_lib):
    """Top-k passes no gradient: with the compression branch off the layer's
    weights get exactly zero, and dk, dv equal nsa_backward's."""
    w = case("mlp_pruned_t600_bf16", T=600, branch_mask=W.BR_SEL | W.BR_SWA,
             cmp_gate_zero=True)
    inp = W.make_inputs(w, seed=68)
    wk, wv = weights(w)
    g = torch.Generator().manual_seed(69)
    dout = torch.randn((w.B, w.T, w.Hq, w.D), generator=g).to(w.dtype).to(DEV)
    p = nsa.params_for(w)
    d = dev(inp)
    wkd, wvd = wk.to(DEV), wv.to(DEV)
    out, saved = nsa.forward_mlp(p, d["q"], d["k"], d["v"], wkd, wvd, d["gates"], keep=True)
    dq, dk, dv, dwk, dwv, dg = nsa.backward_mlp(p, d["q"], d["k"], d["v"], wkd, wvd, d["gates"],
                                                dout, saved)
    ref = nsa.backward(p, d["q"], d["k"], d["v"], d["gates"], dout, saved)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dwk) == 0 and torch.count_nonzero(dwv) == 0
    for a, b in zip((dq, dk, dv, dg), ref):
        assert torch.equal(a, b)


def test_forward_mlp_chunked_queries_equal_the_full_forward_tail(cuda_lib):
    """Queries as the last Tq positions (chunked prefill) see the same
    compressed keys (the layer runs over all T keys), so their outputs are
    the full forward's last Tq rows, bit for bit."""
    w = CASES[0]
    inp = W.make_inputs(w, seed=70)
    wk, wv = (t.to(DEV) for t in weights(w))
    d = dev(inp)
    p = nsa.params_for(w)
    full = nsa.forward_mlp(p, d["q"], d["k"], d["v"], wk, wv, d["gates"])
    tq = w.T - 300
    pc = nsa.params_for(w, Tq=tq)
    part = nsa.forward_mlp(pc, d["q"][:, w.T - tq:].contiguous(), d["k"], d["v"], wk, wv,
                           d["gates"][:, w.T - tq:].contiguous())
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    assert torch.equal(part, full[:, w.T - tq:])
