"""GPU parity: every libnsa entry point against the fp64 oracle.

Inputs are the seeded synthetic workloads (sparse_attention_nsa_b200.inputs);
the GPU path is called through the C ABI (ctypes binding) and the oracle sees
the same bf16-rounded values.  Small cases are compared element by element;
the full-size workloads are compared on sampled tokens the oracle computes
one by one.  Tolerances are in tests/helpers.py.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import sparse_attention_nsa_b200 as nsa
from sparse_attention_nsa_b200 import inputs as W

from helpers import (LSE_TOL, TOL, assert_close, idx_mismatch_rows, ocfg, to_np)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def dev(inp):
    return {k: v.to(DEV) for k, v in inp.items()}


def small(name, **kw):
    base = dict(name=name, B=1, T=256, Hq=16, Hkv=4, D=64, cmp_block=64, cmp_stride=64,
                sel_block=64, topk=4, window=96, dtype=torch.bfloat16, qk_norm=True)
    base.update(kw)
    return W.Workload(**base)


SMALL = [
    W.TINY_F32,
    small("gqa4_t1000_ragged_bf16", T=1000, topk=5, window=200),
    small("gqa4_t700_b2_bf16", B=2, T=700, topk=4, window=130),
    small("mqa_t777_bf16", T=777, Hq=16, Hkv=1, topk=6, window=64, qk_norm=False),
    small("gqa2_t640_f32", T=640, Hq=4, Hkv=2, topk=3, window=100, dtype=torch.float32,
          qk_norm=False, qkv_std=0.5),
    small("mha_t300_l32_bf16", T=300, Hq=4, Hkv=4, cmp_block=32, cmp_stride=32,
          sel_block=32, topk=3, window=40),
    small("pruned_mqa_t900_bf16", T=900, Hq=16, Hkv=1, topk=5, window=128,
          branch_mask=W.BR_SEL | W.BR_SWA, cmp_gate_zero=True, qk_norm=False),
    small("swa_only_t500_bf16", T=500, branch_mask=W.BR_SWA),
    small("cmp_only_t500_bf16", T=500, branch_mask=W.BR_CMP),
    small("window_ge_T_t200_bf16", T=200, window=4096, topk=2),
    small("short_T_below_block_bf16", T=40, window=16),
    small("single_token_f32", T=1, Hq=4, Hkv=1, dtype=torch.float32, window=8),
]


def gpu_forward(w, inp, Tq=None):
    p = nsa.params_for(w, Tq=Tq)
    d = dev(inp)
    if Tq is not None:
        d["q"] = d["q"][:, w.T - Tq:].contiguous()
        d["gates"] = d["gates"][:, w.T - Tq:].contiguous()
    out, saved = nsa.forward(p, d["q"], d["k"], d["v"], d["gates"], keep=True)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    return out, saved


def compare_forward(w, r, out, saved, t0=0):
    """Compare GPU tensors (rows t0..) with oracle results r (all rows)."""
    tol, ltol = TOL[w.dtype], LSE_TOL[w.dtype]
    sl = slice(t0, None)
    m = w.branch_mask
    if m & (W.BR_CMP | W.BR_SEL) and w.Nc > 0:
        if w.dtype == torch.bfloat16:
            np.testing.assert_array_equal(to_np(saved["kc"]), r["kc"])
            np.testing.assert_array_equal(to_np(saved["vc"]), r["vc"])
        else:
            assert_close(to_np(saved["kc"]), r["kc"], 1e-6, "kc")
            assert_close(to_np(saved["vc"]), r["vc"], 1e-6, "vc")
        assert_close(to_np(saved["score"]), r["score"][:, sl], 2e-5, "score")
    if m & W.BR_CMP:
        assert_close(to_np(saved["o_cmp"]), r["o_cmp"][:, sl], tol, "o_cmp")
        assert_close(to_np(saved["lse_cmp"]), r["lse_cmp"][:, sl], ltol, "lse_cmp")
    bad = np.zeros(to_np(out).shape[:2], dtype=bool)
    if m & W.BR_SEL:
        gi = to_np(saved["idx"])
        t_rows = np.broadcast_to((np.arange(gi.shape[1]) + t0)[None, :, None],
                                 gi.shape[:3])
        ssel = orc.sel_block_scores(ocfg(w), r["score"])  # ranking the top-k uses
        diff = idx_mismatch_rows(gi, r["idx"][:, sl], ssel[:, sl], t_rows, w.topk,
                                 w.sel_block)
        bad = diff.reshape(gi.shape[:3]).any(-1)
        assert bad.mean() < 0.01
        keep = ~bad
        assert_close(to_np(saved["o_sel"])[keep], r["o_sel"][:, sl][keep], tol, "o_sel")
        assert_close(to_np(saved["lse_sel"])[keep], r["lse_sel"][:, sl][keep], ltol, "lse_sel")
    if m & W.BR_SWA:
        assert_close(to_np(saved["o_swa"]), r["o_swa"][:, sl], tol, "o_swa")
        assert_close(to_np(saved["lse_swa"]), r["lse_swa"][:, sl], ltol, "lse_swa")
    assert_close(to_np(out)[~bad], r["out"][:, sl][~bad], tol, "out")


# ------------------------------------------------------------------ per entry point
@pytest.mark.parametrize("w", SMALL[:6], ids=lambda w: w.name)
def test_compress(cuda_lib, w):
    inp = W.make_inputs(w, seed=1)
    p = nsa.params_for(w)
    d = dev(inp)
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=DEV)
    vc = torch.empty_like(kc)
    nsa.nsa_compress(p, d["k"], d["v"], kc, vc)
    okc, ovc = orc.compress(ocfg(w), inp["k"], inp["v"])
    if w.dtype == torch.bfloat16:  # exact mean rounded once: bit-exact
        np.testing.assert_array_equal(to_np(kc), okc)
        np.testing.assert_array_equal(to_np(vc), ovc)
    else:
        assert_close(to_np(kc), okc, 1e-6, "kc")
        assert_close(to_np(vc), ovc, 1e-6, "vc")


@pytest.mark.parametrize("w", SMALL[:6] + [SMALL[10]], ids=lambda w: w.name)
def test_cmp_attn_scores(cuda_lib, w):
    inp = W.make_inputs(w, seed=2)
    c = ocfg(w)
    okc, ovc = orc.compress(c, inp["k"], inp["v"])
    o, lse, score = orc.cmp_attn_scores(c, inp["q"], okc, ovc)
    p = nsa.params_for(w)
    d = dev(inp)
    kc = torch.from_numpy(okc).to(w.dtype).to(DEV)  # exact: okc holds dtype values
    vc = torch.from_numpy(ovc).to(w.dtype).to(DEV)
    go = torch.empty((w.B, w.T, w.Hq, w.D), dtype=w.dtype, device=DEV)
    gl = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=DEV)
    gs = torch.empty((w.B, w.T, w.Hkv, w.Nc), dtype=torch.float32, device=DEV)
    nsa.nsa_cmp_attn_scores(p, d["q"], kc, vc, go, gl, gs)
    assert_close(to_np(go), o, TOL[w.dtype], "o_cmp")
    assert_close(to_np(gl), lse, LSE_TOL[w.dtype], "lse_cmp")
    assert_close(to_np(gs), score, 2e-5, "score")
    # scores-only call (pruned compression branch) gives the same scores
    gs2 = torch.empty_like(gs)
    nsa.nsa_cmp_attn_scores(p, d["q"], kc, vc, None, None, gs2)
    assert torch.equal(gs, gs2)


def test_topk_exact_ties(cuda_lib):
    w = small("topk_ties", T=2048, Hkv=4, topk=16)
    c = ocfg(w)
    g = np.random.default_rng(3)
    score = (np.round(g.random((w.B, w.T, w.Hkv, w.Nc)) * 8) / 8).astype(np.float32)
    want = orc.select_topk(c, score.astype(np.float64))
    idx = torch.empty((w.B, w.T, w.Hkv, w.topk), dtype=torch.int32, device=DEV)
    nsa.nsa_select_topk(nsa.params_for(w), torch.from_numpy(score).to(DEV), idx)
    np.testing.assert_array_equal(to_np(idx), want)


@pytest.mark.parametrize("w", [small("topk_gqa", T=3000, topk=16),
                               small("topk_mqa_k8", T=2500, Hkv=1, topk=8),
                               small("topk_l32", T=999, cmp_block=32, cmp_stride=32,
                                     sel_block=32, topk=7)], ids=lambda w: w.name)
def test_topk_on_oracle_scores(cuda_lib, w):
    c = ocfg(w)
    g = np.random.default_rng(4)
    score = g.random((w.B, w.T, w.Hkv, w.Nc)).astype(np.float32).astype(np.float64)
    want = orc.select_topk(c, score)
    idx = torch.empty((w.B, w.T, w.Hkv, w.topk), dtype=torch.int32, device=DEV)
    nsa.nsa_select_topk(nsa.params_for(w), torch.from_numpy(score).float().to(DEV), idx)
    np.testing.assert_array_equal(to_np(idx), want)  # same fp32 values: exact


@pytest.mark.parametrize("w", SMALL[:7], ids=lambda w: w.name)
def test_sel_attn_fwd_on_oracle_idx(cuda_lib, w):
    inp = W.make_inputs(w, seed=5)
    c = ocfg(w)
    r = orc.forward(c, inp["q"], inp["k"], inp["v"], inp["gates"])
    d = dev(inp)
    o = torch.empty((w.B, w.T, w.Hq, w.D), dtype=w.dtype, device=DEV)
    lse = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=DEV)
    nsa.nsa_sel_attn_fwd(nsa.params_for(w), d["q"], d["k"], d["v"],
                         torch.from_numpy(r["idx"]).to(DEV), o, lse)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    assert_close(to_np(o), r["o_sel"], TOL[w.dtype], "o_sel")
    assert_close(to_np(lse), r["lse_sel"], LSE_TOL[w.dtype], "lse_sel")


@pytest.mark.parametrize("window", [1, 37, 64, 200, 5000])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_swa_fwd(cuda_lib, window, dtype):
    w = small("swa", T=611, Hq=8, Hkv=2, window=window, dtype=dtype)
    inp = W.make_inputs(w, seed=6)
    o_ref, lse_ref = orc.swa_fwd(ocfg(w), inp["q"], inp["k"], inp["v"])
    d = dev(inp)
    o = torch.empty((w.B, w.T, w.Hq, w.D), dtype=dtype, device=DEV)
    lse = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=DEV)
    nsa.nsa_swa_fwd(nsa.params_for(w), d["q"], d["k"], d["v"], o, lse)
    assert_close(to_np(o), o_ref, TOL[dtype], "o_swa")
    assert_close(to_np(lse), lse_ref, LSE_TOL[dtype], "lse_swa")


@pytest.mark.parametrize("mask", [7, 6, 4, 1, 3])
def test_gate_combine(cuda_lib, mask):
    w = small("combine", T=300, branch_mask=mask)
    g = torch.Generator().manual_seed(7)
    shape = (w.B, w.T, w.Hq, w.D)
    br = [torch.randn(shape, generator=g).to(w.dtype) for _ in range(3)]
    gates = torch.rand((w.B, w.T, w.Hq, 3), generator=g)
    want = orc.gate_combine(ocfg(w), gates, *br)
    out = torch.empty(shape, dtype=w.dtype, device=DEV)
    args = [b.to(DEV) if mask & (1 << i) else None for i, b in enumerate(br)]
    nsa.nsa_gate_combine(nsa.params_for(w), gates.to(DEV), *args, out)
    assert_close(to_np(out), want, TOL[w.dtype], "out")


# ------------------------------------------------------------------ whole forward
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_small(cuda_lib, w):
    inp = W.make_inputs(w, seed=8)
    r = orc.forward(ocfg(w), inp["q"], inp["k"], inp["v"], inp["gates"])
    out, saved = gpu_forward(w, inp)
    compare_forward(w, r, out, saved)


@pytest.mark.parametrize("onehot", [(1, 0, 0), (0, 1, 0), (0, 0, 1)])
def test_forward_onehot_gates_isolate_branches(cuda_lib, onehot):
    w = small("onehot", T=500, topk=5)
    inp = W.make_inputs(w, seed=9)
    inp["gates"] = torch.tensor(onehot, dtype=torch.float32).expand(w.B, w.T, w.Hq, 3).contiguous()
    out, saved = gpu_forward(w, inp)
    which = ["o_cmp", "o_sel", "o_swa"][onehot.index(1)]
    assert torch.equal(out, saved[which])


def test_forward_chunked_queries(cuda_lib):
    """Queries that are the last Tq positions of a longer key sequence."""
    w = small("chunked", T=900, topk=5, window=150)
    inp = W.make_inputs(w, seed=10)
    r = orc.forward(ocfg(w), inp["q"], inp["k"], inp["v"], inp["gates"])
    Tq = 333
    out, saved = gpu_forward(w, inp, Tq=Tq)
    compare_forward(w, r, out, saved, t0=w.T - Tq)


def test_dense_degeneration_short_context(cuda_lib):
    """T <= topk * block: the selection branch is dense causal attention."""
    w = small("dense", T=1024, topk=16, window=512, Hq=16, Hkv=4)
    inp = W.make_inputs(w, seed=11)
    out, saved = gpu_forward(w, inp)
    idx = to_np(saved["idx"])
    t = np.arange(w.T)
    for s in range(w.topk):
        want = np.where(s <= t // 64, s, -1)
        assert np.all(idx[0, :, :, s] == want[:, None])


def test_bad_block_index_is_reported_not_read(cuda_lib):
    w = small("badidx", T=256, topk=4)
    inp = dev(W.make_inputs(w, seed=12))
    idx = torch.full((w.B, w.T, w.Hkv, w.topk), -1, dtype=torch.int32, device=DEV)
    idx[..., 0] = 0
    idx[0, 100, 0, 1] = 3          # not causal for t = 100 (block 1)
    idx[0, 200, 1, 1] = 1 << 30    # far out of range
    o = torch.empty((w.B, w.T, w.Hq, w.D), dtype=w.dtype, device=DEV)
    nsa.nsa_sel_attn_fwd(nsa.params_for(w), inp["q"], inp["k"], inp["v"], idx, o, None)
    assert nsa.nsa_last_device_error() == 5  # NSA_ERR_DEVICE_CHECK
    assert nsa.nsa_last_device_error() == 0  # cleared by the read


# ------------------------------------------------------------------ decode
def gpu_decode(w, inp):
    pk = nsa.params_for(w)
    d = dev(inp)
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=DEV)
    vc = torch.empty_like(kc)
    nsa.nsa_compress(pk, d["k_cache"], d["v_cache"], kc, vc)
    p = nsa.params_for(w, Tq=1)
    out = torch.empty((w.B, 1, w.Hq, w.D), dtype=w.dtype, device=DEV)
    idx = torch.empty((w.B, 1, w.Hkv, w.topk), dtype=torch.int32, device=DEV)
    nsa.nsa_decode(p, d["q"].unsqueeze(1), d["k_cache"], d["v_cache"], kc, vc,
                   d["gates"].unsqueeze(1), out, idx, nsa.alloc_workspace(p))
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    return out[:, 0], idx[:, 0]


def check_decode(w, inp, seqs):
    out, idx = gpu_decode(w, inp)
    ws = w.replace(B=len(seqs))
    c = ocfg(ws)
    kcache, vcache = inp["k_cache"][seqs], inp["v_cache"][seqs]
    okc, ovc = orc.compress(c, kcache, vcache)
    o_ref, i_ref, s_ref = orc.decode(c, inp["q"][seqs], kcache, vcache, okc, ovc,
                                     inp["gates"][seqs], with_score=True)
    if w.branch_mask & W.BR_SEL:  # idx_out is written when selection runs
        if (w.cmp_block, w.cmp_stride) != (w.sel_block, w.sel_block):
            # the selection-block importances the top-k ranks (query at T-1)
            full = np.zeros((len(seqs), w.T, w.Hkv, w.Nc))
            full[:, w.T - 1] = s_ref
            s_ref = orc.sel_block_scores(c, full)[:, w.T - 1]
        diff = idx_mismatch_rows(to_np(idx)[seqs], i_ref, s_ref,
                                 np.full(len(seqs) * w.Hkv, w.T - 1), w.topk, w.sel_block)
        keep = ~diff.reshape(len(seqs), w.Hkv).any(-1)
    else:
        keep = np.ones(len(seqs), dtype=bool)
    assert_close(to_np(out)[seqs][keep], o_ref[keep], TOL[w.dtype], "decode out")


@pytest.mark.parametrize("w", [
    W.DECODE_32K.replace(name="decode_small", B=3, T=1500),
    W.DECODE_32K.replace(name="decode_gqa_ragged", B=5, T=2049, Hq=16, Hkv=4),
    W.DECODE_32K.replace(name="decode_short", B=2, T=70),
    # 625 compressed blocks: ten K1 chunks and the 32-slot-per-lane top-k
    W.DECODE_32K.replace(name="decode_long_nc625", B=2, T=40000),
    W.DECODE_32K.replace(name="decode_pruned_w100_k4", B=4, T=5000, topk=4, window=100,
                         branch_mask=W.BR_SEL | W.BR_SWA, cmp_gate_zero=True),
    W.DECODE_32K.replace(name="decode_swa_only_gqa8", B=3, T=3333, Hq=16, Hkv=2, window=200,
                         branch_mask=W.BR_SWA),
    W.DECODE_32K.replace(name="decode_cmp_sel_mha", B=2, T=1999, Hq=4, Hkv=4, topk=6,
                         branch_mask=W.BR_CMP | W.BR_SEL),
], ids=lambda w: w.name)
def test_decode_small(cuda_lib, w):
    inp = W.make_decode_inputs(w, seed=13)
    check_decode(w, inp, list(range(w.B)))


# ------------------------------------------------------------------ general geometry
# Compression block l and stride d other than the selection block l' (the
# pages give block size and stride as parameters): overlapping compressed
# blocks, and a selection block's importance summed over the compressed
# blocks that overlap it (reading R14).
GEOM = [
    small("geo_l32_d16_s64_gqa4_t900_bf16", T=900, cmp_block=32, cmp_stride=16, topk=5,
          window=150),
    small("geo_l64_d32_s64_gqa4_t1000_bf16", T=1000, cmp_block=64, cmp_stride=32, topk=5,
          window=200),
    small("geo_l128_d64_s64_mqa_t1300_bf16", T=1300, Hkv=1, cmp_block=128, cmp_stride=64,
          topk=6, window=100, qk_norm=False),
    small("geo_l16_d8_s32_gqa2_t300_f32", T=300, Hq=4, Hkv=2, cmp_block=16, cmp_stride=8,
          sel_block=32, topk=4, window=50, dtype=torch.float32, qk_norm=False, qkv_std=0.5),
    # block-major selection (Nb >= 8 top-k) with stride < block
    small("geo_l64_d32_s64_gqa4_t4200_k4_bf16", T=4200, cmp_block=64, cmp_stride=32, topk=4,
          window=128),
]


@pytest.mark.parametrize("w", GEOM, ids=lambda w: w.name)
def test_compress_general_geometry(cuda_lib, w):
    inp = W.make_inputs(w, seed=41)
    d = dev(inp)
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device=DEV)
    vc = torch.empty_like(kc)
    nsa.nsa_compress(nsa.params_for(w), d["k"], d["v"], kc, vc)
    okc, ovc = orc.compress(ocfg(w), inp["k"], inp["v"])
    if w.dtype == torch.bfloat16:
        np.testing.assert_array_equal(to_np(kc), okc)
        np.testing.assert_array_equal(to_np(vc), ovc)
    else:
        assert_close(to_np(kc), okc, 1e-6, "kc")
        assert_close(to_np(vc), ovc, 1e-6, "vc")


@pytest.mark.parametrize("w", GEOM, ids=lambda w: w.name)
def test_forward_general_geometry(cuda_lib, w):
    inp = W.make_inputs(w, seed=42)
    r = orc.forward(ocfg(w), inp["q"], inp["k"], inp["v"], inp["gates"])
    out, saved = gpu_forward(w, inp)
    compare_forward(w, r, out, saved)


def test_topk_general_geometry_on_oracle_scores(cuda_lib):
    """The top-k's score remap alone, on scores drawn in fp32: the GPU sums
    the overlapping compressed blocks in fp32, so only near-ties may differ."""
    w = small("geo_topk_l32_d16", T=2000, cmp_block=32, cmp_stride=16, topk=8)
    c = ocfg(w)
    g = np.random.default_rng(43)
    score = g.random((w.B, w.T, w.Hkv, w.Nc)).astype(np.float32).astype(np.float64)
    want = orc.select_topk(c, score)
    idx = torch.empty((w.B, w.T, w.Hkv, w.topk), dtype=torch.int32, device=DEV)
    nsa.nsa_select_topk(nsa.params_for(w), torch.from_numpy(score).float().to(DEV), idx)
    t_rows = np.broadcast_to(np.arange(w.T)[None, :, None], (w.B, w.T, w.Hkv))
    diff = idx_mismatch_rows(to_np(idx), want, orc.sel_block_scores(c, score), t_rows, w.topk,
                             w.sel_block)
    assert diff.mean() < 0.01


@pytest.mark.parametrize("w", [
    W.DECODE_32K.replace(name="decode_geo_l32_d16", B=3, T=2500, cmp_block=32, cmp_stride=16),
    W.DECODE_32K.replace(name="decode_geo_l128_d64_gqa4", B=2, T=3001, Hq=16, Hkv=4,
                         cmp_block=128, cmp_stride=64),
], ids=lambda w: w.name)
def test_decode_general_geometry(cuda_lib, w):
    inp = W.make_decode_inputs(w, seed=44)
    check_decode(w, inp, list(range(w.B)))


# ------------------------------------------------------------------ full size, sampled
def sample_rows(w, n, seed):
    g = np.random.default_rng(seed)
    special = [0, 1, w.sel_block - 1, w.sel_block, w.window - 1, w.window,
               w.topk * w.sel_block, w.T // 2, w.T - 2, w.T - 1]
    ts = sorted(set([t for t in special if t < w.T] + list(g.integers(0, w.T, n))))
    return np.array([[int(g.integers(0, w.B)), t] for t in ts])


@pytest.mark.parametrize("w", [W.NSA_340M, W.PRUNED_32K, W.NSA_1P3B,
                               # 625 selection blocks: the 32-slot-per-lane top-k
                               W.NSA_340M.replace(name="gqa4_t40000_nb625", T=40000),
                               # the limits: 1024 blocks per sequence, top-k 64 (the
                               # block-major path's 6-bit slot numbers), 32 heads a group
                               W.NSA_340M.replace(name="gqa4_t65536_nb1024", T=65536),
                               W.PRUNED_32K.replace(name="mqa_t32768_k64", topk=64),
                               W.NSA_340M.replace(name="mqa_g32_t8192", Hq=32, Hkv=1)],
                         ids=lambda w: w.name)
def test_forward_full_size_sampled(cuda_lib, w):
    inp = W.make_inputs(w, seed=0)
    out, saved = gpu_forward(w, inp)
    rows = sample_rows(w, 24, seed=14)
    c = ocfg(w)
    r = orc.forward_rows(c, inp["q"], inp["k"], inp["v"], inp["gates"], rows)
    b, t = rows[:, 0], rows[:, 1]
    tol, ltol = TOL[w.dtype], LSE_TOL[w.dtype]
    gi = to_np(saved["idx"])[b, t]
    diff = idx_mismatch_rows(gi, r["idx"], r["score"], np.repeat(t, w.Hkv), w.topk, w.sel_block)
    bad = diff.reshape(len(rows), w.Hkv)
    head_bad = np.repeat(bad, w.G, axis=1)
    assert_close(to_np(saved["score"])[b, t], r["score"], 2e-5, "score")
    if w.branch_mask & W.BR_CMP:
        assert_close(to_np(saved["o_cmp"])[b, t], r["o_cmp"], tol, "o_cmp")
    assert_close(to_np(saved["o_sel"])[b, t][~head_bad], r["o_sel"][~head_bad], tol, "o_sel")
    assert_close(to_np(saved["lse_sel"])[b, t][~head_bad], r["lse_sel"][~head_bad], ltol, "lse_sel")
    assert_close(to_np(saved["o_swa"])[b, t], r["o_swa"], tol, "o_swa")
    assert_close(to_np(out)[b, t][~head_bad], r["out"][~head_bad], tol, "out")


def test_decode_full_size_sampled(cuda_lib):
    w = W.DECODE_32K
    inp = W.make_decode_inputs(w, seed=0)
    check_decode(w, inp, [0, 17, 42, 63])


@pytest.mark.parametrize("w", [small("host_fwd_gqa4_t1000", T=1000, topk=5, window=200),
                               small("host_fwd_bm_t4200_k4", T=4200, topk=4, window=150)],
                         ids=lambda w: w.name)
def test_forward_host_buffers_match_device_forward(cuda_lib, w):
    """nsa_forward_host (pinned host tensors in and out) gives the device
    forward's output bit for bit."""
    inp = W.make_inputs(w, seed=33)
    p = nsa.params_for(w)
    d = {n: inp[n].to(DEV) for n in ("q", "k", "v", "gates")}
    out_d = torch.empty_like(d["q"])
    nsa.nsa_forward(p, d["q"], d["k"], d["v"], d["gates"], out_d, None, nsa.alloc_workspace(p))
    h = {n: inp[n].contiguous().pin_memory() for n in ("q", "k", "v", "gates")}
    out_h = torch.full(tuple(out_d.shape), float("nan"), dtype=out_d.dtype).pin_memory()
    ws = torch.empty(nsa.nsa_forward_host_workspace_size(p), dtype=torch.uint8, device=DEV)
    nsa.nsa_forward_host(p, h["q"], h["k"], h["v"], h["gates"], out_h, ws)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    assert torch.equal(out_h, out_d.cpu())
