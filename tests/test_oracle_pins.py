"""Pins for the fp64 oracle, checked against things other than itself.

CPU only.  Each test ties one oracle function to a closed form, a library
routine (torch's scaled_dot_product_attention / avg_pool1d / bf16 cast, in
float64 on the CPU), a hand-derived fixture, brute force, or central finite
differences.  Together they are chosen so that a dropped term, a wrong sign,
a wrong index or a swapped operand in the oracle fails at least one test.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers
def rand(shape, seed, std=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * std


def sdpa(q, k, v, mask, scale):
    """Library attention in float64: q [B,T,Hq,D], k/v [B,S,Hkv,D],
    mask broadcastable to [B,Hq,T,S] (True = attend).  Returns (o, lse)."""
    G = q.shape[2] // k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    m = torch.as_tensor(mask)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    logits = torch.einsum("bhtd,bhsd->bhts", qt, kt) * scale
    lse = torch.logsumexp(logits.masked_fill(~m, -math.inf), dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.permute(0, 2, 1).numpy()


def causal(T, S=None):
    S = T if S is None else S
    return torch.ones(T, S, dtype=torch.bool).tril()


def cfg_small(**kw):
    base = dict(B=2, T=64, Hq=4, Hkv=2, D=8, cmp_block=8, cmp_stride=8,
                sel_block=8, topk=3, window=12)
    base.update(kw)
    return orc.Cfg(**base)


def qkv(c, seed=0, std=1.0):
    return (rand((c.B, c.T, c.Hq, c.D), seed, std),
            rand((c.B, c.T, c.Hkv, c.D), seed + 1, std),
            rand((c.B, c.T, c.Hkv, c.D), seed + 2, std))


# ---------------------------------------------------------------- rounding
def test_round_bf16_matches_torch_cast():
    x = torch.randn(20000, dtype=torch.float32) * 3
    # exact ties between two bf16 neighbours must go to the even one
    ties = torch.tensor([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8), 2 + 2**-7,
                         0.5 + 2**-9, 1.5 + 2**-8], dtype=torch.float32)
    x = torch.cat([x, ties])
    want = x.to(torch.bfloat16).double().numpy()
    got = np.array([orc.round_bf16(float(a)) for a in x.double().numpy()])
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------------- compression
def test_compress_closed_form_ramp_and_constant():
    c = orc.Cfg(B=1, T=12, Hq=1, Hkv=1, D=3, cmp_block=4, cmp_stride=4,
                sel_block=4, topk=2, window=4)
    t = np.arange(12, dtype=np.float64)
    k = np.stack([t, 2 * t, np.repeat([7.0, -1.0, 3.0], 4)], -1).reshape(1, 12, 1, 3)
    kc, vc = orc.compress(c, k, -k)
    # mean of a ramp over [4j, 4j+4) is 4j + 1.5; a constant stays constant
    np.testing.assert_allclose(kc[0, :, 0, 0], [1.5, 5.5, 9.5], rtol=0, atol=1e-15)
    np.testing.assert_allclose(kc[0, :, 0, 1], [3.0, 11.0, 19.0], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(kc[0, :, 0, 2], [7.0, -1.0, 3.0])
    np.testing.assert_array_equal(vc, -kc)


@pytest.mark.parametrize("l,d", [(8, 8), (4, 4), (8, 4), (5, 3)])
def test_compress_matches_avg_pool(l, d):
    c = orc.Cfg(B=2, T=40, Hq=2, Hkv=2, D=5, cmp_block=l, cmp_stride=d,
                sel_block=l, topk=2, window=4)
    k = rand((2, 40, 2, 5), 3)
    v = rand((2, 40, 2, 5), 4)
    kc, vc = orc.compress(c, k, v)
    for src, got in ((k, kc), (v, vc)):
        x = torch.from_numpy(src).permute(0, 2, 3, 1).reshape(-1, 1, 40)
        want = F.avg_pool1d(x, kernel_size=l, stride=d)
        want = want.reshape(2, 2, 5, -1).permute(0, 3, 1, 2).numpy()
        assert got.shape == want.shape
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


def test_compress_rounds_to_storage_precision():
    c = cfg_small(kv_round=orc.KV_BF16)
    _, k, v = qkv(c, 11)
    kc, _ = orc.compress(c, k, v)
    c0 = cfg_small()
    kc0, _ = orc.compress(c0, k, v)
    want = torch.from_numpy(kc0).float().to(torch.bfloat16).double().numpy()
    # bf16(float32(x)) can double-round; it agrees except at exact fp32 ties
    assert np.mean(kc == want) > 0.999
    assert np.all(np.abs(kc - kc0) <= np.abs(kc0) * 2**-8 + 1e-300)


# ---------------------------------------------------------------- cmp branch
def test_cmp_block1_is_full_causal_attention():
    """Compression with block = stride = 1 is ordinary causal attention."""
    c = cfg_small(cmp_block=1, cmp_stride=1)
    q, k, v = qkv(c, 21)
    kc, vc = orc.compress(c, k, v)
    np.testing.assert_array_equal(kc, k)
    o, lse, score = orc.cmp_attn_scores(c, q, kc, vc)
    o_ref, lse_ref = sdpa(q, k, v, causal(c.T), 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_cmp_visibility_and_scores():
    """Block j is visible at t iff j*d + l - 1 <= t; scores are the group's
    summed softmax probabilities (library softmax on a masked logit matrix)."""
    c = cfg_small(cmp_block=8, cmp_stride=4)  # overlapping blocks
    q, k, v = qkv(c, 31)
    kc, vc = orc.compress(c, k, v)
    o, lse, score = orc.cmp_attn_scores(c, q, kc, vc)
    Nc = c.Nc
    t = np.arange(c.T)[:, None]
    j = np.arange(Nc)[None, :]
    vis = torch.from_numpy(j * c.cmp_stride + c.cmp_block - 1 <= t)
    rows = vis.any(-1)
    o_ref, lse_ref = sdpa(q[:, rows.numpy()], kc, vc, vis[rows], 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o[:, rows.numpy()], o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse[:, rows.numpy()], lse_ref, atol=1e-12, rtol=0)
    # no visible block: zero output, -inf lse, zero score
    assert np.all(o[:, ~rows.numpy()] == 0)
    assert np.all(np.isneginf(lse[:, ~rows.numpy()]))
    assert np.all(score[:, ~rows.numpy()] == 0)
    # scores via torch.softmax over masked logits, summed over group heads
    qt = torch.from_numpy(q)
    kg = torch.from_numpy(kc).repeat_interleave(c.G, dim=2)
    lg = torch.einsum("bthd,bjhd->bthj", qt, kg) / math.sqrt(c.D)
    p = torch.softmax(lg.masked_fill(~vis[None, :, None, :], -math.inf), -1)
    p = torch.nan_to_num(p, nan=0.0)
    want = p.reshape(c.B, c.T, c.Hkv, c.G, Nc).sum(3).numpy()
    np.testing.assert_allclose(score, want, atol=1e-12, rtol=0)
    # each visible row's probabilities sum to 1 -> group score sums to G
    np.testing.assert_allclose(score[:, rows.numpy()].sum(-1), c.G, atol=1e-12)


# ---------------------------------------------------------------- top-k
def _golden_topk():
    cases = []
    with open(os.path.join(GOLDEN, "topk_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, sc, exp = (p.strip() for p in line.split("|"))
            t, l, n = (int(x) for x in head.split())
            cases.append((t, l, n, [float(x) for x in sc.split()],
                          [int(x) for x in exp.split()]))
    return cases


@pytest.mark.parametrize("case", _golden_topk())
def test_topk_golden(case):
    t, l, n, scores, expected = case
    T = len(scores) * l
    c = orc.Cfg(B=1, T=T, Hq=1, Hkv=1, D=1, cmp_block=l, cmp_stride=l,
                sel_block=l, topk=n, window=1)
    assert c.Nc == len(scores)
    score = np.zeros((1, T, 1, c.Nc))
    score[0, t, 0] = scores
    idx = orc.select_topk(c, score)
    assert idx[0, t, 0].tolist() == expected


def test_topk_brute_force():
    c = cfg_small(T=256, sel_block=8, cmp_block=8, cmp_stride=8, topk=6, Hkv=3)
    g = np.random.default_rng(5)
    # quantised scores so that ties really occur
    score = np.round(g.random((c.B, c.T, c.Hkv, c.Nc)) * 20) / 20
    idx = orc.select_topk(c, score)
    for b in range(c.B):
        for t in range(c.T):
            for h in range(c.Hkv):
                cur = t // c.sel_block
                if cur + 1 <= c.topk:
                    want = list(range(cur + 1)) + [-1] * (c.topk - cur - 1)
                else:
                    cands = sorted(range(1, cur), key=lambda j: (-score[b, t, h, j], j))
                    want = sorted([0, cur] + cands[:c.topk - 2])
                assert idx[b, t, h].tolist() == want


# Compression and selection with different block geometry (compressed
# blocks of l tokens every d tokens, selection blocks of l' tokens): a
# selection block's importance is the sum over the compressed blocks whose
# tokens overlap it.
@pytest.mark.parametrize("l,d,ls", [(4, 2, 8), (8, 8, 16), (6, 4, 8), (4, 2, 4)])
def test_topk_general_geometry_brute_force(l, d, ls):
    """Overlap written as a token-set intersection, ranking as in the
    equal-geometry brute force."""
    c = cfg_small(T=96, cmp_block=l, cmp_stride=d, sel_block=ls, topk=4, Hkv=2)
    g = np.random.default_rng(7)
    score = np.round(g.random((c.B, c.T, c.Hkv, c.Nc)) * 20) / 20  # ties occur
    idx = orc.select_topk(c, score)
    cmp_tokens = [set(range(i * d, i * d + l)) for i in range(c.Nc)]
    for b in range(c.B):
        for t in range(c.T):
            for h in range(c.Hkv):
                cur = t // ls
                if cur + 1 <= c.topk:
                    want = list(range(cur + 1)) + [-1] * (c.topk - cur - 1)
                else:
                    sel = [sum(score[b, t, h, i] for i in range(c.Nc)
                               if cmp_tokens[i] & set(range(j * ls, (j + 1) * ls)))
                           for j in range(cur + 1)]
                    cands = sorted(range(1, cur), key=lambda j: (-sel[j], j))
                    want = sorted([0, cur] + cands[:c.topk - 2])
                assert idx[b, t, h].tolist() == want, (b, t, h)


@pytest.mark.parametrize("l,d,ls", [(4, 2, 8), (8, 8, 8), (6, 4, 8), (32, 16, 64)])
def test_sel_block_scores_are_token_overlap_sums(l, d, ls):
    """The exported selection-block importances equal the token-set
    intersection sums (for l = d = l' the compressed scores themselves,
    and 0 for a selection block with no complete compressed block)."""
    c = cfg_small(T=130, cmp_block=l, cmp_stride=d, sel_block=ls, topk=4, Hkv=2)
    g = np.random.default_rng(9)
    score = g.random((c.B, c.T, c.Hkv, c.Nc))
    got = orc.sel_block_scores(c, score)
    nb = -(-c.T // ls)
    assert got.shape == (c.B, c.T, c.Hkv, nb)
    cmp_tokens = [set(range(i * d, i * d + l)) for i in range(c.Nc)]
    for j in range(nb):
        over = [i for i in range(c.Nc) if cmp_tokens[i] & set(range(j * ls, (j + 1) * ls))]
        want = score[..., over].sum(-1) if over else np.zeros(score.shape[:3])
        np.testing.assert_allclose(got[..., j], want, rtol=1e-15, atol=0)
    if l == d == ls:
        np.testing.assert_array_equal(got[..., :c.Nc], score)


def test_topk_general_geometry_hand_cases():
    """Hand-derived: with l = 4, d = 2 a compressed block i covers tokens
    [2i, 2i + 4), so for selection blocks of 4 tokens block j collects the
    compressed blocks 2j - 1, 2j and 2j + 1; a lone importance on an odd
    compressed block 2m + 1 lifts selection blocks m and m + 1 alike (the
    tie goes to m).  With l = d = 4 and selection blocks of 8 tokens, block j
    collects compressed blocks 2j and 2j + 1."""
    c = cfg_small(B=1, T=64, Hkv=1, Hq=1, cmp_block=4, cmp_stride=2, sel_block=4, topk=3)
    t = 63  # cur = 15: candidates 1 .. 14, one winner besides 0 and 15
    score = np.zeros((1, c.T, 1, c.Nc))
    score[0, t, 0, 2 * 6 + 1] = 1.0  # blocks 6 and 7 tie: 6 wins
    assert orc.select_topk(c, score)[0, t, 0].tolist() == [0, 6, 15]
    score[0, t, 0, 2 * 7] = 0.5      # block 7 alone gets 1.5 (13 and 14)
    assert orc.select_topk(c, score)[0, t, 0].tolist() == [0, 7, 15]
    c2 = cfg_small(B=1, T=64, Hkv=1, Hq=1, cmp_block=4, cmp_stride=4, sel_block=8, topk=3)
    t = 63  # cur = 7
    score = np.zeros((1, c2.T, 1, c2.Nc))
    score[0, t, 0, 2 * 3] = 0.6       # selection block 3: 0.6 + 0.0
    score[0, t, 0, 2 * 5 + 1] = 0.4   # block 5: 0.0 + 0.4 + the next one
    score[0, t, 0, 2 * 5] = 0.3       #          = 0.7 > 0.6
    assert orc.select_topk(c2, score)[0, t, 0].tolist() == [0, 5, 7]


def test_forward_general_geometry_selection_and_compression():
    """With every selection block selected the selection branch is dense
    causal attention whatever the scores; with l = d = 1 the compression
    branch is dense causal attention (selection blocks of 4 tokens)."""
    c = cfg_small(T=48, Hq=4, Hkv=2, cmp_block=1, cmp_stride=1, sel_block=4, topk=12,
                  branch_mask=orc.BR_ALL)
    q, k, v = qkv(c, 61)
    r = orc.forward(c, q, k, v, rand((c.B, c.T, c.Hq, 3), 62))
    o_ref, lse_ref = sdpa(q, k, v, causal(c.T), 1 / math.sqrt(c.D))
    np.testing.assert_allclose(r["o_sel"], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["o_cmp"], o_ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- sel branch
def test_sel_covering_every_block_is_full_causal_attention():
    c = cfg_small(T=64, sel_block=8, topk=8)  # 8 blocks, all selected
    q, k, v = qkv(c, 41)
    score = rand((c.B, c.T, c.Hkv, c.Nc), 42)
    idx = orc.select_topk(c, score)
    assert np.all(idx[:, -1] == np.arange(8))
    o, lse = orc.sel_attn_fwd(c, q, k, v, idx)
    o_ref, lse_ref = sdpa(q, k, v, causal(c.T), 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_sel_equals_block_masked_attention():
    """Gathered-list attention equals dense attention under the block mask
    built from the same indices (a different formulation of the branch)."""
    c = cfg_small(T=96, Hq=6, Hkv=2, sel_block=8, topk=4)
    q, k, v = qkv(c, 51)
    score = rand((c.B, c.T, c.Hkv, c.Nc), 52)
    idx = orc.select_topk(c, score)
    o, lse = orc.sel_attn_fwd(c, q, k, v, idx)
    mask = torch.zeros(c.B, c.Hq, c.T, c.T, dtype=torch.bool)
    blk = torch.arange(c.T) // c.sel_block
    for b in range(c.B):
        for t in range(c.T):
            for h in range(c.Hq):
                chosen = [j for j in idx[b, t, h // c.G] if j >= 0]
                mask[b, h, t] = torch.isin(blk, torch.tensor(chosen)) & (torch.arange(c.T) <= t)
    o_ref, lse_ref = sdpa(q, k, v, mask, 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- swa branch
def test_swa_window_at_least_T_is_full_causal_attention():
    c = cfg_small(window=64)
    q, k, v = qkv(c, 61)
    o, lse = orc.swa_fwd(c, q, k, v)
    o_ref, lse_ref = sdpa(q, k, v, causal(c.T), 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("w", [1, 5, 12])
def test_swa_equals_band_masked_attention(w):
    c = cfg_small(window=w)
    q, k, v = qkv(c, 62)
    o, lse = orc.swa_fwd(c, q, k, v)
    t = torch.arange(c.T)
    band = (t[None, :] <= t[:, None]) & (t[None, :] >= t[:, None] - w + 1)
    o_ref, lse_ref = sdpa(q, k, v, band, 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)
    if w == 1:  # one key: the output is that key's value row
        np.testing.assert_allclose(o, np.repeat(v, c.G, axis=2), atol=1e-15)


def test_attention_two_key_closed_form():
    """q.k = (0, ln 3) with scale 1 gives p = (1/4, 3/4)."""
    c = orc.Cfg(B=1, T=2, Hq=1, Hkv=1, D=2, cmp_block=1, cmp_stride=1,
                sel_block=1, topk=2, window=2, scale=1.0)
    q = np.array([[[[1.0, 0.0]], [[math.log(3), 1.0]]]])
    k = np.array([[[[0.0, 5.0]], [[1.0, 0.0]]]])
    v = np.array([[[[4.0, -8.0]], [[8.0, 4.0]]]])
    o, lse = orc.swa_fwd(c, q, k, v)
    # row 1: logits (5, ln3) -> weights e^5, 3 ; row 0 sees only key 0
    np.testing.assert_allclose(o[0, 0, 0], [4.0, -8.0])
    w0, w1 = math.exp(5.0), 3.0
    np.testing.assert_allclose(o[0, 1, 0], (w0 * np.array([4.0, -8.0]) + w1 * np.array([8.0, 4.0])) / (w0 + w1))
    np.testing.assert_allclose(lse[0, 1, 0], math.log(w0 + w1))
    q2 = np.array([[[[1.0, 0.0]], [[1.0, math.log(3) / 5.0]]]])
    o2, _ = orc.swa_fwd(c, q2, k, v)
    # logits (ln3, 1) for row 1 with k0=(0,5): ln3 ; k1=(1,0): 1
    p0 = 3.0 / (3.0 + math.e)
    np.testing.assert_allclose(o2[0, 1, 0], p0 * np.array([4.0, -8.0]) + (1 - p0) * np.array([8.0, 4.0]))


# ---------------------------------------------------------------- gates / full
@pytest.mark.parametrize("onehot", [(1, 0, 0), (0, 1, 0), (0, 0, 1)])
def test_onehot_gates_isolate_each_branch(onehot):
    c = cfg_small()
    q, k, v = qkv(c, 71)
    gates = np.broadcast_to(np.array(onehot, dtype=np.float64), (c.B, c.T, c.Hq, 3)).copy()
    r = orc.forward(c, q, k, v, gates)
    which = ["o_cmp", "o_sel", "o_swa"][onehot.index(1)]
    np.testing.assert_array_equal(r["out"], r[which])
    # the branch tensors themselves come from the separate entry points
    kc, vc = orc.compress(c, k, v)
    np.testing.assert_array_equal(r["kc"], kc)
    o_c, l_c, sc = orc.cmp_attn_scores(c, q, kc, vc)
    np.testing.assert_array_equal(r["o_cmp"], o_c)
    np.testing.assert_array_equal(r["score"], sc)
    idx = orc.select_topk(c, sc)
    np.testing.assert_array_equal(r["idx"], idx)
    o_s, _ = orc.sel_attn_fwd(c, q, k, v, idx)
    np.testing.assert_array_equal(r["o_sel"], o_s)
    o_w, _ = orc.swa_fwd(c, q, k, v)
    np.testing.assert_array_equal(r["o_swa"], o_w)


def test_gate_combine_is_linear_and_respects_branch_mask():
    c = cfg_small(branch_mask=orc.BR_SEL | orc.BR_SWA)
    q, k, v = qkv(c, 72)
    gates = np.random.default_rng(3).random((c.B, c.T, c.Hq, 3))
    r = orc.forward(c, q, k, v, gates)
    want = gates[..., 1:2] * r["o_sel"] + gates[..., 2:3] * r["o_swa"]
    np.testing.assert_allclose(r["out"], want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("mask", [7, 6, 5, 3, 4, 1])
def test_gate_combine_bwd_is_autograd_of_the_masked_sum(mask):
    """The combination's backward against torch autograd of
    out = sum over the kept branches of gate_i * o_i: a pruned branch gets
    neither a gate gradient nor an output gradient ("Sparsity is Cool",
    Key claims: unused branches are dropped)."""
    c = cfg_small(branch_mask=mask)
    rng = np.random.default_rng(40 + mask)
    shp = (c.B, c.T, c.Hq, c.D)
    gates = rng.random((c.B, c.T, c.Hq, 3))
    o3 = [rng.standard_normal(shp) for _ in range(3)]
    dout = rng.standard_normal(shp)
    gt = torch.from_numpy(gates).requires_grad_()
    ot = [torch.from_numpy(o).requires_grad_() for o in o3]
    bits = (orc.BR_CMP, orc.BR_SEL, orc.BR_SWA)
    out = sum(gt[..., i:i + 1] * ot[i] for i in range(3) if mask & bits[i])
    (out * torch.from_numpy(dout)).sum().backward()
    dg, *dO = orc.gate_combine_bwd(c, gates, dout, *o3)
    np.testing.assert_allclose(dg, gt.grad.numpy(), rtol=1e-13, atol=1e-13)
    for i in range(3):
        want = ot[i].grad.numpy() if ot[i].grad is not None else np.zeros(shp)
        np.testing.assert_allclose(dO[i], want, rtol=0, atol=1e-15)


def test_dense_degeneration_at_short_context():
    """With block 64, top-k 16 and window 512, a 1024-token sequence selects
    every causal block, so the selection branch is dense causal attention,
    and the window branch is dense for t < 512 ("Sparsity is Cool", Key
    claims: at <= 1.5k tokens NSA degenerates to dense attention)."""
    c = orc.Cfg(B=1, T=1024, Hq=2, Hkv=1, D=8)
    q, k, v = qkv(c, 81, std=0.5)
    gates = np.full((1, c.T, c.Hq, 3), 0.5)
    r = orc.forward(c, q, k, v, gates)
    o_ref, lse_ref = sdpa(q, k, v, causal(c.T), 1 / math.sqrt(c.D))
    np.testing.assert_allclose(r["o_sel"], o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["o_swa"][:, :512], o_ref[:, :512], rtol=0, atol=1e-12)
    assert not np.allclose(r["o_swa"][:, 600:], o_ref[:, 600:], atol=1e-6)


def test_group_head_permutation_equivariance():
    c = cfg_small(Hq=4, Hkv=2)
    q, k, v = qkv(c, 91)
    gates = np.random.default_rng(9).random((c.B, c.T, c.Hq, 3))
    perm = [1, 0, 3, 2]  # swap heads inside each KV group
    r = orc.forward(c, q, k, v, gates)
    rp = orc.forward(c, q[:, :, perm], k, v, gates[:, :, perm])
    np.testing.assert_array_equal(rp["idx"], r["idx"])
    np.testing.assert_allclose(rp["out"], r["out"][:, :, perm], atol=1e-14)


def test_forward_rows_matches_forward():
    c = cfg_small(T=64)
    q, k, v = qkv(c, 95)
    gates = np.random.default_rng(4).random((c.B, c.T, c.Hq, 3))
    r = orc.forward(c, q, k, v, gates)
    rows = np.array([[0, 0], [1, 63], [0, 17], [1, 40]])
    s = orc.forward_rows(c, q, k, v, gates, rows)
    for i, (b, t) in enumerate(rows):
        for key in ("out", "o_cmp", "o_sel", "o_swa", "idx", "score", "lse_sel"):
            np.testing.assert_array_equal(s[key][i], r[key][b, t])


@pytest.mark.parametrize("geom", [dict(), dict(cmp_block=4, cmp_stride=2, sel_block=8, T=50)],
                         ids=["equal_blocks", "overlapping_cmp_blocks"])
def test_decode_is_last_row_of_forward(geom):
    c = cfg_small(**{"B": 3, "T": 48, **geom})
    q, k, v = qkv(c, 97)
    gates = np.random.default_rng(8).random((c.B, c.T, c.Hq, 3))
    r = orc.forward(c, q, k, v, gates)
    out, idx = orc.decode(c, q[:, -1], k, v, r["kc"], r["vc"], gates[:, -1])
    np.testing.assert_array_equal(out, r["out"][:, -1])
    np.testing.assert_array_equal(idx, r["idx"][:, -1])


def test_decode_dense_when_everything_is_selected():
    c = cfg_small(B=2, T=32, sel_block=8, topk=4, window=32)
    q, k, v = qkv(c, 98)
    gates = np.zeros((c.B, c.T, c.Hq, 3))
    gates[..., 1] = 1.0
    kc, vc = orc.compress(c, k, v)
    out, _ = orc.decode(c, q[:, -1], k, v, kc, vc, gates[:, -1])
    o_ref, _ = sdpa(q, k, v, causal(c.T), 1 / math.sqrt(c.D))
    np.testing.assert_allclose(out, o_ref[:, -1], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- gradients
def _loss(c, q, k, v, gates, dout):
    r = orc.forward(c, q, k, v, gates)
    return float(np.sum(r["out"] * dout)), r["idx"]


@pytest.mark.parametrize("shape", [
    dict(B=1, T=14, Hq=2, Hkv=1, D=4, cmp_block=2, cmp_stride=2, sel_block=2,
         topk=3, window=4),
    dict(B=2, T=12, Hq=4, Hkv=2, D=3, cmp_block=3, cmp_stride=3, sel_block=3,
         topk=2, window=5),
    # overlapping compressed blocks (a token in two of them), selection blocks
    # of another size: the pooling backward spreads over both blocks
    dict(B=1, T=16, Hq=2, Hkv=1, D=3, cmp_block=4, cmp_stride=2, sel_block=4,
         topk=2, window=5),
])
def test_backward_matches_central_differences(shape):
    c = orc.Cfg(**shape)
    q, k, v = qkv(c, 101, std=0.7)
    g = np.random.default_rng(102)
    gates = g.random((c.B, c.T, c.Hq, 3))
    dout = g.standard_normal((c.B, c.T, c.Hq, c.D))
    dq, dk, dv, dg = orc.backward(c, q, k, v, gates, dout)
    _, idx0 = _loss(c, q, k, v, gates, dout)
    eps = 1e-6
    checked = skipped = 0
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("g", gates, dg)):
        for i in range(x.size):
            args = {"q": q, "k": k, "v": v, "g": gates}
            xp, xm = x.copy(), x.copy()
            xp.flat[i] += eps
            xm.flat[i] -= eps
            args[name] = xp
            lp, ip = _loss(c, args["q"], args["k"], args["v"], args["g"], dout)
            args[name] = xm
            lm, im = _loss(c, args["q"], args["k"], args["v"], args["g"], dout)
            if not (np.array_equal(ip, idx0) and np.array_equal(im, idx0)):
                skipped += 1  # the perturbation moved the discrete selection
                continue
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad.flat[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, grad.flat[i])
            checked += 1
    assert checked > 0.95 * (checked + skipped)


def test_branch_backwards_sum_to_full_backward():
    c = cfg_small(T=32)
    q, k, v = qkv(c, 111)
    g = np.random.default_rng(112)
    gates = g.random((c.B, c.T, c.Hq, 3))
    dout = g.standard_normal((c.B, c.T, c.Hq, c.D))
    r = orc.forward(c, q, k, v, gates)
    dg, d1, d2, d3 = orc.gate_combine_bwd(c, gates, dout, r["o_cmp"], r["o_sel"], r["o_swa"])
    np.testing.assert_allclose(dg[..., 1], np.sum(dout * r["o_sel"], -1), atol=1e-14)
    np.testing.assert_allclose(d2, gates[..., 1:2] * dout, atol=1e-15)
    a = orc.cmp_bwd(c, q, r["kc"], r["vc"], d1)
    b = orc.sel_attn_bwd(c, q, k, v, r["idx"], d2)
    w = orc.swa_bwd(c, q, k, v, d3)
    dq, dk, dv, dgf = orc.backward(c, q, k, v, gates, dout)
    np.testing.assert_allclose(a[0] + b[0] + w[0], dq, atol=1e-13)
    np.testing.assert_allclose(a[1] + b[1] + w[1], dk, atol=1e-13)
    np.testing.assert_allclose(a[2] + b[2] + w[2], dv, atol=1e-13)
    np.testing.assert_allclose(dg, dgf, atol=1e-14)


def test_sel_backward_matches_autograd_of_masked_attention():
    """dq/dk/dv of the selection branch equal torch autograd (float64) of
    dense attention under the block mask of the same indices."""
    c = cfg_small(T=40, Hq=4, Hkv=2, sel_block=4, topk=3, D=6)
    q, k, v = qkv(c, 121)
    idx = orc.select_topk(c, rand((c.B, c.T, c.Hkv, c.Nc), 122))
    dO = rand((c.B, c.T, c.Hq, c.D), 123)
    dq, dk, dv = orc.sel_attn_bwd(c, q, k, v, idx, dO)
    blk = torch.arange(c.T) // c.sel_block
    mask = torch.zeros(c.B, c.Hq, c.T, c.T, dtype=torch.bool)
    for b in range(c.B):
        for t in range(c.T):
            for h in range(c.Hq):
                chosen = torch.tensor([j for j in idx[b, t, h // c.G] if j >= 0])
                mask[b, h, t] = torch.isin(blk, chosen) & (torch.arange(c.T) <= t)
    qt = torch.from_numpy(q).requires_grad_()
    kt = torch.from_numpy(k).requires_grad_()
    vt = torch.from_numpy(v).requires_grad_()
    o = F.scaled_dot_product_attention(
        qt.permute(0, 2, 1, 3), kt.repeat_interleave(c.G, 2).permute(0, 2, 1, 3),
        vt.repeat_interleave(c.G, 2).permute(0, 2, 1, 3), attn_mask=mask,
        scale=1 / math.sqrt(c.D)).permute(0, 2, 1, 3)
    (o * torch.from_numpy(dO)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-12)


def test_backward_dq_rows_match_full_backward():
    c = cfg_small(T=40)
    q, k, v = qkv(c, 131)
    g = np.random.default_rng(132)
    gates = g.random((c.B, c.T, c.Hq, 3))
    dout = g.standard_normal((c.B, c.T, c.Hq, c.D))
    dq, _, _, _ = orc.backward(c, q, k, v, gates, dout)
    rows = np.array([[0, 0], [1, 39], [0, 8], [1, 23], [0, 31]])
    got = orc.backward_dq_rows(c, q, k, v, gates, dout, rows)
    for i, (b, t) in enumerate(rows):
        np.testing.assert_allclose(got[i], dq[b, t], rtol=0, atol=1e-13)


@pytest.mark.parametrize("mode", [orc.KV_BF16, orc.KV_F32])
def test_backward_gate_gradient_reads_stored_outputs(mode):
    """Reading R15: with the branch outputs stored in a lower precision, the
    gate gradient is dout . o_i of the STORED o_i (rounded here by torch's
    own cast, independent of the oracle's rounding), while dq, dk and dv
    keep using the exact outputs."""
    c = cfg_small(T=40)
    q, k, v = qkv(c, 141)
    g = np.random.default_rng(142)
    gates = g.random((c.B, c.T, c.Hq, 3))
    dout = g.standard_normal((c.B, c.T, c.Hq, c.D))
    r = orc.forward(c, q, k, v, gates)
    exact = orc.backward(c, q, k, v, gates, dout)
    c.o_round = mode
    stored = orc.backward(c, q, k, v, gates, dout)
    to = torch.bfloat16 if mode == orc.KV_BF16 else torch.float32
    for i, name in enumerate(("o_cmp", "o_sel", "o_swa")):
        o_st = torch.from_numpy(r[name]).to(to).double().numpy()
        np.testing.assert_allclose(stored[3][..., i], np.sum(dout * o_st, -1), rtol=0,
                                   atol=1e-13)
        if mode == orc.KV_BF16:  # the rounding must actually move dgates
            assert np.abs(stored[3][..., i] - exact[3][..., i]).max() > 1e-6
    for a, b in zip(stored[:3], exact[:3]):
        np.testing.assert_array_equal(a, b)


def test_backward_composed_on_own_selection_equals_backward():
    """The GPU tests' composition of the oracle's branch backwards on a given
    selection reproduces orc_backward exactly when given the oracle's own
    selection (with the stored-output rounding of reading R15)."""
    import torch as _t

    from helpers import oracle_backward_given_idx
    from sparse_attention_nsa_b200 import inputs as W
    w = W.Workload("compose_check", B=2, T=40, Hq=4, Hkv=2, D=8, cmp_block=8, cmp_stride=8,
                   sel_block=8, topk=3, window=12, dtype=_t.bfloat16)
    inp = {n: x.double().numpy() for n, x in W.make_inputs(w, seed=151, with_dout=True).items()}
    c = orc.Cfg(B=w.B, T=w.T, Hq=w.Hq, Hkv=w.Hkv, D=w.D, cmp_block=8, cmp_stride=8,
                sel_block=8, topk=3, window=12, kv_round=orc.KV_BF16, o_round=orc.KV_BF16)
    r = orc.forward(c, inp["q"], inp["k"], inp["v"], inp["gates"])
    got = oracle_backward_given_idx(c, w, inp, inp["dout"], r["idx"])
    want = orc.backward(c, inp["q"], inp["k"], inp["v"], inp["gates"], inp["dout"])
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- MoBA
def moba_cfg(**kw):
    base = dict(B=2, T=48, Hq=4, Hkv=2, D=8, cmp_block=8, cmp_stride=8, sel_block=8,
                topk=3, window=1)
    base.update(kw)
    return orc.Cfg(**base)


def test_moba_with_every_block_selected_is_full_causal_attention():
    """k >= the number of blocks: every causal block is read, so MoBA is
    dense causal attention (library SDPA)."""
    c = moba_cfg(topk=6)
    q, k, v = qkv(c, 161)
    o, lse, idx = orc.moba_fwd(c, q, k, v)
    o_ref, lse_ref = sdpa(q, k, v, causal(c.T), 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_moba_dense_below_k_blocks():
    """The pages' short-context claim in miniature: with block L and top-3,
    a sequence of 3 L tokens is dense attention (1.5k tokens at L = 512)."""
    c = moba_cfg(T=24, topk=3)
    q, k, v = qkv(c, 162)
    o, _, idx = orc.moba_fwd(c, q, k, v)
    o_ref, _ = sdpa(q, k, v, causal(c.T), 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    assert np.all(idx[:, 23, :, :].tolist() == np.array([0, 1, 2]))


def test_moba_equals_block_masked_attention():
    """Given its selection, MoBA is SDPA under the block mask of the
    selected blocks (and causal)."""
    c = moba_cfg(T=64, topk=3)
    q, k, v = qkv(c, 163)
    o, lse, idx = orc.moba_fwd(c, q, k, v)
    blk = torch.arange(c.T) // c.sel_block
    mask = torch.zeros(c.B, c.Hq, c.T, c.T, dtype=torch.bool)
    for b in range(c.B):
        for t in range(c.T):
            for h in range(c.Hq):
                chosen = torch.tensor([j for j in idx[b, t, h // c.G] if j >= 0])
                mask[b, h, t] = torch.isin(blk, chosen) & (torch.arange(c.T) <= t)
    o_ref, lse_ref = sdpa(q, k, v, mask, 1 / math.sqrt(c.D))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)
    # the query's own block is always selected, the rest are complete past blocks
    for b in range(c.B):
        for t in range(c.T):
            cur = t // c.sel_block
            for g in range(c.Hkv):
                sel = [j for j in idx[b, t, g] if j >= 0]
                assert cur in sel and all(j <= cur for j in sel)
                assert sel == sorted(sel) and len(sel) == min(cur + 1, c.topk)


def test_moba_gate_hand_cases():
    """Hand-built gates: keys constant inside each block (so the block mean
    is that constant) along one axis, queries along the same axis; head
    gates are summed over the KV group.  Block 5 is the query's own."""
    c = moba_cfg(B=1, T=48, Hq=2, Hkv=1, topk=3)
    t = 47  # cur = 5: blocks 0..4 compete for two places
    k = np.zeros((1, c.T, 1, c.D))
    v = np.zeros_like(k)
    a = [0.1, 0.9, 0.4, 0.9, 0.2, 0.0]   # block j's key value on axis 0
    b_ = [0.0, 0.0, 0.5, 0.0, 0.8, 0.0]  # ... on axis 1
    for j in range(6):
        k[0, j * 8:(j + 1) * 8, 0, 0] = a[j]
        k[0, j * 8:(j + 1) * 8, 0, 1] = b_[j]
    q = np.zeros((1, c.T, 2, c.D))
    q[0, t, 0, 0] = 1.0  # head 0 reads axis 0: gates a
    _, _, idx = orc.moba_fwd(c, q, k, v)
    assert idx[0, t, 0].tolist() == [1, 3, 5]  # 0.9 and 0.9 tie: both taken
    q[0, t, 1, 1] = 1.0  # head 1 adds axis 1: sums 0.1, 0.9, 0.9, 0.9, 1.0
    _, _, idx = orc.moba_fwd(c, q, k, v)
    assert idx[0, t, 0].tolist() == [1, 4, 5]  # 1.0 first, then the lowest of three 0.9


# ---------------------------------------------------------------- parametric compression
def unfold_blocks(x, l, d):
    """[B, T, H, D] -> [B, Nc, H, l*D]: each block's l rows flattened in
    token order (torch's unfold; independent of the oracle)."""
    t = torch.from_numpy(x)
    u = t.unfold(1, l, d)                 # [B, Nc, H, D, l]
    return u.permute(0, 1, 2, 4, 3).reshape(u.shape[0], u.shape[1], u.shape[2], -1)


@pytest.mark.parametrize("l,d", [(8, 8), (8, 4), (4, 2), (6, 3)])
def test_compress_mlp_is_unfold_matmul(l, d):
    """One linear layer over the flattened block (reading R17) equals torch
    unfold + matmul."""
    c = cfg_small(T=40, cmp_block=l, cmp_stride=d, D=8)
    _, k, v = qkv(c, 171)
    g = np.random.default_rng(172)
    wk, wv = g.standard_normal((l * c.D, c.D)), g.standard_normal((l * c.D, c.D))
    kc, vc = orc.compress_mlp(c, k, v, wk, wv)
    want_k = (unfold_blocks(k, l, d) @ torch.from_numpy(wk)).numpy()
    want_v = (unfold_blocks(v, l, d) @ torch.from_numpy(wv)).numpy()
    np.testing.assert_allclose(kc, want_k, rtol=0, atol=1e-12)
    np.testing.assert_allclose(vc, want_v, rtol=0, atol=1e-12)


def test_compress_mlp_with_mean_weights_is_mean_pooling():
    """W[i D + e, n] = (e == n) / l makes the layer mean-pooling (the pages'
    replacement of the MLP is its special case): torch avg_pool1d."""
    c = cfg_small(T=40, cmp_block=8, cmp_stride=4, D=8)
    _, k, v = qkv(c, 173)
    w = np.tile(np.eye(c.D) / c.cmp_block, (c.cmp_block, 1))
    kc, vc = orc.compress_mlp(c, k, v, w, w)
    pool = F.avg_pool1d(torch.from_numpy(k).permute(0, 2, 3, 1).reshape(-1, 1, c.T),
                        c.cmp_block, c.cmp_stride)
    want = pool.reshape(c.B, c.Hkv, c.D, -1).permute(0, 3, 1, 2).numpy()
    np.testing.assert_allclose(kc, want, rtol=0, atol=1e-14)


@pytest.mark.parametrize("l,d", [(4, 4), (4, 2)])
def test_compress_mlp_backward_matches_autograd_and_differences(l, d):
    c = cfg_small(B=1, T=14, Hkv=2, Hq=2, cmp_block=l, cmp_stride=d, D=3)
    _, k, v = qkv(c, 174)
    g = np.random.default_rng(175)
    wk, wv = g.standard_normal((l * c.D, c.D)), g.standard_normal((l * c.D, c.D))
    gk, gv = g.standard_normal((c.B, c.Nc, c.Hkv, c.D)), g.standard_normal((c.B, c.Nc, c.Hkv, c.D))
    dk, dv, dwk, dwv = orc.compress_mlp_bwd(c, k, v, wk, wv, gk, gv)
    tk, tv = torch.from_numpy(k).requires_grad_(), torch.from_numpy(v).requires_grad_()
    twk, twv = torch.from_numpy(wk).requires_grad_(), torch.from_numpy(wv).requires_grad_()
    uk = tk.unfold(1, l, d).permute(0, 1, 2, 4, 3).reshape(c.B, c.Nc, c.Hkv, -1)
    uv = tv.unfold(1, l, d).permute(0, 1, 2, 4, 3).reshape(c.B, c.Nc, c.Hkv, -1)
    loss = ((uk @ twk) * torch.from_numpy(gk)).sum() + ((uv @ twv) * torch.from_numpy(gv)).sum()
    loss.backward()
    for got, t in ((dk, tk), (dv, tv), (dwk, twk), (dwv, twv)):
        np.testing.assert_allclose(got, t.grad.numpy(), rtol=0, atol=1e-12)
    # and central differences of the oracle's own forward, on a few entries
    def lossf(kk, vv, wkk, wvv):
        a, b = orc.compress_mlp(c, kk, vv, wkk, wvv)
        return float((a * gk).sum() + (b * gv).sum())
    eps = 1e-6
    for arr, grad in ((k, dk), (wk, dwk), (wv, dwv)):
        for i in (0, arr.size // 2, arr.size - 1):
            xp, xm = arr.copy(), arr.copy()
            xp.flat[i] += eps
            xm.flat[i] -= eps
            args_p = [xp if a is arr else a for a in (k, v, wk, wv)]
            args_m = [xm if a is arr else a for a in (k, v, wk, wv)]
            fd = (lossf(*args_p) - lossf(*args_m)) / (2 * eps)
            assert abs(fd - grad.flat[i]) <= 1e-7 * max(1.0, abs(fd))


@pytest.mark.parametrize("l,d", [(4, 4), (4, 2)])
def test_cmp_bwd_kc_matches_central_differences(l, d):
    """dkc, dvc, dq of the compression branch against central differences of
    sum(dO . o_cmp) computed by the oracle's forward."""
    c = cfg_small(B=1, T=20, Hq=4, Hkv=2, D=4, cmp_block=l, cmp_stride=d)
    q, k, v = qkv(c, 176)
    kc, vc = orc.compress(c, k, v)
    g = np.random.default_rng(177)
    kc, vc = kc + 0.3 * g.standard_normal(kc.shape), vc + 0.3 * g.standard_normal(vc.shape)
    dO = g.standard_normal((c.B, c.T, c.Hq, c.D))
    dq, dkc, dvc = orc.cmp_bwd_kc(c, q, kc, vc, dO)

    def lossf(qq, a, b):
        o, _, _ = orc.cmp_attn_scores(c, qq, a, b)
        return float((o * dO).sum())
    eps = 1e-6
    for which, grad in ((0, dq), (1, dkc), (2, dvc)):
        base = (q, kc, vc)[which]
        for i in range(0, base.size, max(1, base.size // 9)):
            xp, xm = base.copy(), base.copy()
            xp.flat[i] += eps
            xm.flat[i] -= eps
            ap = [xp if j == which else (q, kc, vc)[j] for j in range(3)]
            am = [xm if j == which else (q, kc, vc)[j] for j in range(3)]
            fd = (lossf(*ap) - lossf(*am)) / (2 * eps)
            assert abs(fd - grad.flat[i]) <= 1e-7 * max(1.0, abs(fd)), (which, i)


def test_cmp_bwd_kc_through_mean_weights_is_cmp_bwd():
    """Stopping at kc / vc and going on through the linear layer with mean
    weights gives the mean-pool branch gradient on the raw rows."""
    c = cfg_small(B=2, T=48, cmp_block=8, cmp_stride=4, D=8)
    q, k, v = qkv(c, 178)
    kc, vc = orc.compress(c, k, v)
    dO = rand((c.B, c.T, c.Hq, c.D), 179)
    dq_ref, dk_ref, dv_ref = orc.cmp_bwd(c, q, kc, vc, dO)
    dq, dkc, dvc = orc.cmp_bwd_kc(c, q, kc, vc, dO)
    w = np.tile(np.eye(c.D) / c.cmp_block, (c.cmp_block, 1))
    dk, dv, _, _ = orc.compress_mlp_bwd(c, k, v, w, w, dkc, dvc)
    np.testing.assert_allclose(dq, dq_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk, dk_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv, dv_ref, rtol=0, atol=1e-13)
