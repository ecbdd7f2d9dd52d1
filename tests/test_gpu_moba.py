"""GPU parity of MoBA block attention (nsa_moba_forward / _backward) against
the fp64 oracle's MoBA (reading R16: gate = q . mean-pooled block key,
summed over the KV group's query heads; own block always read).

The chosen blocks must equal the oracle's except where the oracle's gates
of the last winner and the first loser differ by less than 1e-5 relative
(a near-tie the fp32 gate may resolve either way); such a row must still
hold a valid selection, and its outputs are then a different correct
answer and are left out (at most 1 % of the rows).
"""
import numpy as np
import pytest
import torch

import oracle as orc
import sparse_attention_nsa_b200 as nsa
from sparse_attention_nsa_b200 import inputs as W

from helpers import LSE_TOL, TOL, assert_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def moba_case(name, T, L, k, Hq=16, Hkv=4, B=1, dtype=torch.bfloat16, qk_norm=True, std=1.0):
    return dict(w=W.Workload(name, B=B, T=T, Hq=Hq, Hkv=Hkv, D=64, cmp_block=L, cmp_stride=L,
                             sel_block=L, topk=k, window=1, dtype=dtype, qk_norm=qk_norm,
                             qkv_std=std), L=L, k=k)


CASES = [
    moba_case("moba_gqa4_t2048_L512_k3_bf16", 2048, 512, 3),
    moba_case("moba_mqa_t3000_L256_k4_bf16", 3000, 256, 4, Hkv=1, qk_norm=False),
    moba_case("moba_gqa2_t700_L128_k3_f32", 700, 128, 3, Hq=4, Hkv=2, dtype=torch.float32,
              qk_norm=False, std=0.5),
    moba_case("moba_b2_gqa4_t1300_L64_k5_bf16", 1300, 64, 5, B=2),
    # block-major selection path (64-key blocks >= 8 x top-k)
    moba_case("moba_gqa4_t4096_L128_k2_bf16", 4096, 128, 2),
    # the pages' dense regime: 3 blocks of 512 at top-3 is full attention
    moba_case("moba_dense_t1536_L512_k3_bf16", 1536, 512, 3),
]


def ocfg_moba(w, L, k):
    return orc.Cfg(B=w.B, T=w.T, Hq=w.Hq, Hkv=w.Hkv, D=w.D, cmp_block=L, cmp_stride=L,
                   sel_block=L, topk=k, window=1, scale=w.scale,
                   kv_round=orc.KV_BF16 if w.dtype == torch.bfloat16 else orc.KV_F32)


def gates_of(c, q, k):
    """The oracle-side gates [B, T, Hkv, nblocks] (fp64, from the oracle's
    own pooled keys), for the near-tie rule only."""
    kc, _ = orc.compress(c, k, k)
    qd = q.double().numpy().reshape(c.B, c.T, c.Hkv, c.G, c.D).sum(3)
    return np.einsum("btgd,bjgd->btgj", qd, kc)


def check_selection(gi, oi, gates, L, k):
    """Rows whose selection differs must be valid near-ties; returns the
    mask of differing (b, t, g) rows."""
    diff = np.any(gi != oi, axis=-1)
    for b, t, g in zip(*np.nonzero(diff)):
        cur = t // L
        sel = [int(j) for j in gi[b, t, g] if j >= 0]
        assert cur + 1 > k, f"row {(b, t, g)}: all-causal selection differs"
        assert sel == sorted(set(sel)) and cur in sel and len(sel) == k, (b, t, g, sel)
        assert all(0 <= j <= cur for j in sel)
        ranked = sorted(range(cur), key=lambda j: (-gates[b, t, g, j], j))
        kth, nxt = gates[b, t, g, ranked[k - 2]], gates[b, t, g, ranked[k - 1]]
        assert abs(kth - nxt) <= 1e-5 * max(abs(kth), 1e-30), (b, t, g, kth, nxt)
    return diff


def run_gpu(w, L, k, inp):
    p = nsa.make_moba_params(w.B, w.T, w.Hq, w.Hkv, block=L, topk=k, dtype=w.dtype)
    d = {n: inp[n].to(DEV) for n in ("q", "k", "v")}
    out = torch.empty_like(d["q"])
    lse = torch.empty((w.B, w.T, w.Hq), dtype=torch.float32, device=DEV)
    idx = torch.empty((w.B, w.T, w.Hkv, k), dtype=torch.int32, device=DEV)
    nsa.nsa_moba_forward(p, d["q"], d["k"], d["v"], out, lse, idx)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    return p, d, out, lse, idx


@pytest.mark.parametrize("case", CASES, ids=lambda c: c["w"].name)
def test_moba_forward(cuda_lib, case):
    w, L, k = case["w"], case["L"], case["k"]
    inp = W.make_inputs(w, seed=51)
    c = ocfg_moba(w, L, k)
    o_ref, lse_ref, i_ref = orc.moba_fwd(c, inp["q"], inp["k"], inp["v"])
    _, _, out, lse, idx = run_gpu(w, L, k, inp)
    diff = check_selection(to_np(idx), i_ref, gates_of(c, inp["q"], inp["k"]), L, k)
    assert diff.mean() < 0.01
    keep = ~np.repeat(diff, w.G, axis=2)  # [B, T, Hq]
    assert_close(to_np(out)[keep], o_ref[keep], TOL[w.dtype], "out")
    assert_close(to_np(lse)[keep], lse_ref[keep], LSE_TOL[w.dtype], "lse")


def test_moba_dense_regime_is_full_attention(cuda_lib):
    """Block 512, top-3, 1536 tokens: every causal block is read, as the
    pages state for MoBA at short context; the output equals the oracle's
    window branch with a window covering the sequence (dense attention)."""
    case = CASES[-1]
    w, L, k = case["w"], case["L"], case["k"]
    inp = W.make_inputs(w, seed=52)
    _, _, out, _, idx = run_gpu(w, L, k, inp)
    t = np.arange(w.T)
    want = np.where(np.arange(k)[None, :] <= (t // L)[:, None], np.arange(k)[None, :], -1)
    assert np.all(to_np(idx)[0] == want[:, None, :])
    c = orc.Cfg(B=w.B, T=w.T, Hq=w.Hq, Hkv=w.Hkv, D=w.D, window=w.T, scale=w.scale)
    o_dense, _ = orc.swa_fwd(c, inp["q"], inp["k"], inp["v"])
    assert_close(to_np(out), o_dense, TOL[w.dtype], "dense")


@pytest.mark.parametrize("case", CASES[:4], ids=lambda c: c["w"].name)
def test_moba_backward(cuda_lib, case):
    """Gradients with the forward's selection held fixed: the oracle's
    selection-branch backward over the same MoBA blocks."""
    w, L, k = case["w"], case["L"], case["k"]
    inp = W.make_inputs(w, seed=53)
    p, d, out, lse, idx = run_gpu(w, L, k, inp)
    g = torch.Generator().manual_seed(54)
    dout = torch.randn((w.B, w.T, w.Hq, w.D), generator=g)
    dq = torch.empty((w.B, w.T, w.Hq, w.D), dtype=torch.float32, device=DEV)
    dk = torch.empty((w.B, w.T, w.Hkv, w.D), dtype=torch.float32, device=DEV)
    dv = torch.empty_like(dk)
    nsa.nsa_moba_backward(p, d["q"], d["k"], d["v"], idx, out, lse, dout.to(DEV), dq, dk, dv)
    torch.cuda.synchronize()
    assert nsa.nsa_last_device_error() == 0
    c = ocfg_moba(w, L, k)
    want = orc.sel_attn_bwd(c, inp["q"], inp["k"], inp["v"], to_np(idx), dout)
    for got, ref, name in zip((dq, dk, dv), want, ("dq", "dk", "dv")):
        assert_close(to_np(got), ref, TOL[w.dtype], name)
