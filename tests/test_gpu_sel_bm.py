"""GPU parity of the block-major selection forward (nsa_sel_attn_fwd_ws).

The block-major path inverts the iteration of the selection branch: a
reverse map lists, per key block, the queries that selected it; each
(query, head, block) pair gets its own softmax over the block and the
partials are merged by their log-sum-exps.  Its outputs are compared with
the fp64 oracle's selection branch on the same bf16-rounded inputs, element
by element, for tile shapes G = 1, 2, 4, 8, 16 (128/G queries per tile),
ragged lists and unit tails, sparse and padded index rows, and queries that
are the last Tq positions of a longer sequence.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import sparse_attention_nsa_b200 as nsa
from sparse_attention_nsa_b200 import inputs as W

from helpers import LSE_TOL, TOL, assert_close, ocfg, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda"


def small(name, **kw):
    base = dict(name=name, B=1, T=256, Hq=16, Hkv=4, D=64, cmp_block=64, cmp_stride=64,
                sel_block=64, topk=4, window=96, dtype=torch.bfloat16, qk_norm=True)
    base.update(kw)
    return W.Workload(**base)


CASES = [
    small("g4_t1000_k5", T=1000, topk=5),
    small("g4_b2_t700", B=2, T=700, topk=4),
    small("g16_mqa_t777_k6", T=777, Hq=16, Hkv=1, topk=6, qk_norm=False),
    small("g1_mha_t1300_k6", T=1300, Hq=4, Hkv=4, topk=6),
    small("g8_t900_k7", T=900, Hq=16, Hkv=2, topk=7),
    small("g2_b3_t555_k3", B=3, T=555, Hq=4, Hkv=2, topk=3),
    small("g4_t3000_k16", T=3000, topk=16),
]


def run_ws(w, q, k, v, idx, Tq=None, want_o=True, want_lse=True):
    p = nsa.params_for(w, Tq=Tq)
    tq = w.T if Tq is None else Tq
    o = torch.empty((w.B, tq, w.Hq, w.D), dtype=w.dtype, device=DEV) if want_o else None
    lse = torch.empty((w.B, tq, w.Hq), dtype=torch.float32, device=DEV) if want_lse else None
    ws = torch.empty(nsa.nsa_sel_workspace_size(p), dtype=torch.uint8, device=DEV)
    nsa.nsa_sel_attn_fwd_ws(p, q, k, v, idx, o, lse, ws)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_sel_bm_on_oracle_idx(cuda_lib, w):
    inp = W.make_inputs(w, seed=21)
    c = ocfg(w)
    r = orc.forward(c, inp["q"], inp["k"], inp["v"], inp["gates"])
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = run_ws(w, q, k, v, torch.from_numpy(r["idx"]).to(DEV))
    assert nsa.nsa_last_device_error() == 0
    assert_close(to_np(o), r["o_sel"], TOL[w.dtype], "o_sel")
    assert_close(to_np(lse), r["lse_sel"], LSE_TOL[w.dtype], "lse_sel")


def random_idx(w, rng, p_empty=0.05):
    """Ascending, -1-padded causal selections of random size 0..topk."""
    idx = np.full((w.B, w.T, w.Hkv, w.topk), -1, dtype=np.int32)
    for b in range(w.B):
        for t in range(w.T):
            cur = t // w.sel_block
            for g in range(w.Hkv):
                if rng.random() < p_empty:
                    continue
                n = int(rng.integers(1, min(w.topk, cur + 1) + 1))
                pick = np.sort(rng.choice(cur + 1, size=n, replace=False))
                idx[b, t, g, :n] = pick
    return idx


@pytest.mark.parametrize("w", [small("sparse_g4_t1100", T=1100, topk=6),
                               small("sparse_g16_t900", T=900, Hq=16, Hkv=1, topk=5)],
                         ids=lambda w: w.name)
def test_sel_bm_sparse_padded_rows(cuda_lib, w):
    """Rows with fewer than topk blocks, rows with none (o = 0, lse = -inf),
    rows whose only block is their own."""
    inp = W.make_inputs(w, seed=22)
    rng = np.random.default_rng(23)
    idx = random_idx(w, rng)
    idx[0, 70, 0, :] = -1
    idx[0, 70, 0, 0] = 1                 # only its own block
    idx[0, w.T - 1, :, :] = -1           # no block at all
    o_ref, lse_ref = orc.sel_attn_fwd(ocfg(w), inp["q"], inp["k"], inp["v"], idx)
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = run_ws(w, q, k, v, torch.from_numpy(idx).to(DEV))
    assert nsa.nsa_last_device_error() == 0
    assert_close(to_np(o), o_ref, TOL[w.dtype], "o_sel")
    assert_close(to_np(lse), lse_ref, LSE_TOL[w.dtype], "lse_sel")
    assert np.all(to_np(o)[0, w.T - 1] == 0.0)
    assert np.all(np.isneginf(to_np(lse)[0, w.T - 1]))


def test_sel_bm_chunked_queries(cuda_lib):
    """Queries that are the last Tq positions of a longer key sequence."""
    w = small("chunked_g4_t1200", T=1200, topk=5)
    inp = W.make_inputs(w, seed=24)
    r = orc.forward(ocfg(w), inp["q"], inp["k"], inp["v"], inp["gates"])
    Tq = 333
    t0 = w.T - Tq
    q = inp["q"][:, t0:].contiguous().to(DEV)
    k, v = inp["k"].to(DEV), inp["v"].to(DEV)
    idx = torch.from_numpy(np.ascontiguousarray(r["idx"][:, t0:])).to(DEV)
    o, lse = run_ws(w, q, k, v, idx, Tq=Tq)
    assert nsa.nsa_last_device_error() == 0
    assert_close(to_np(o), r["o_sel"][:, t0:], TOL[w.dtype], "o_sel")
    assert_close(to_np(lse), r["lse_sel"][:, t0:], LSE_TOL[w.dtype], "lse_sel")


def test_sel_bm_optional_outputs(cuda_lib):
    """o_sel or lse_sel may be omitted; what is written is unchanged."""
    w = small("optional_g4_t600", T=600, topk=4)
    inp = W.make_inputs(w, seed=25)
    r = orc.forward(ocfg(w), inp["q"], inp["k"], inp["v"], inp["gates"])
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    idx = torch.from_numpy(r["idx"]).to(DEV)
    o_full, lse_full = run_ws(w, q, k, v, idx)
    o_only, _ = run_ws(w, q, k, v, idx, want_lse=False)
    _, lse_only = run_ws(w, q, k, v, idx, want_o=False)
    assert torch.equal(o_full, o_only)
    assert torch.equal(lse_full, lse_only)


def test_sel_bm_bad_index_is_reported(cuda_lib):
    w = small("badidx_bm", T=256, topk=4)
    inp = {n: t.to(DEV) for n, t in W.make_inputs(w, seed=26).items()}
    idx = torch.full((w.B, w.T, w.Hkv, w.topk), -1, dtype=torch.int32, device=DEV)
    idx[..., 0] = 0
    idx[0, 100, 0, 1] = 3          # not causal for t = 100 (block 1)
    idx[0, 200, 1, 1] = 1 << 30    # far out of range
    idx[0, 150, 2, 1] = 0          # repeats the previous entry
    run_ws(w, inp["q"], inp["k"], inp["v"], idx)
    assert nsa.nsa_last_device_error() == 5  # NSA_ERR_DEVICE_CHECK
    assert nsa.nsa_last_device_error() == 0


def test_sel_bm_workspace_checks(cuda_lib):
    w = small("ws_g4", T=300)
    p = nsa.params_for(w)
    need = nsa.nsa_sel_workspace_size(p)
    assert need > 0
    inp = {n: t.to(DEV) for n, t in W.make_inputs(w, seed=27).items()}
    idx = torch.zeros((w.B, w.T, w.Hkv, w.topk), dtype=torch.int32, device=DEV)
    o = torch.empty((w.B, w.T, w.Hq, w.D), dtype=w.dtype, device=DEV)
    short = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(nsa.NsaError) as e:
        nsa.nsa_sel_attn_fwd_ws(p, inp["q"], inp["k"], inp["v"], idx, o, None, short)
    assert e.value.status == 6  # NSA_ERR_WORKSPACE
    f32 = nsa.params_for(w.replace(dtype=torch.float32))
    with pytest.raises(nsa.NsaError) as e:
        nsa.nsa_sel_workspace_size(f32)
    assert e.value.status == 2  # NSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("w", [small("fwd_bm_g4_t4200_k4", T=4200, topk=4, window=150),
                               small("fwd_bm_pruned_g16_t4300_k4", T=4300, Hq=16, Hkv=1, topk=4,
                                     window=128, branch_mask=W.BR_SEL | W.BR_SWA,
                                     cmp_gate_zero=True, qk_norm=False)],
                         ids=lambda w: w.name)
def test_forward_takes_block_major_path(cuda_lib, w):
    """nsa_forward with Nb >= 8 topk runs the selection block-major (the merge
    applies the gates); the whole forward still matches the oracle."""
    from test_gpu_parity import compare_forward, gpu_forward
    assert -(-w.T // w.sel_block) >= 16 * w.topk  # Nb
    inp = W.make_inputs(w, seed=28)
    r = orc.forward(ocfg(w), inp["q"], inp["k"], inp["v"], inp["gates"])
    out, saved = gpu_forward(w, inp)
    assert nsa.nsa_last_device_error() == 0
    compare_forward(w, r, out, saved)


def test_sel_bm_partial_range_is_reported(cuda_lib):
    """Per-block partials are held in fp16: values beyond its range are
    reported through the device error word instead of stored as inf."""
    w = small("range_g4_t300", T=300, topk=4)
    inp = {n: t.to(DEV) for n, t in W.make_inputs(w, seed=29).items()}
    idx = torch.full((w.B, w.T, w.Hkv, w.topk), -1, dtype=torch.int32, device=DEV)
    idx[..., 0] = 0
    v = torch.full_like(inp["v"], 1.0e5)
    run_ws(w, inp["q"], inp["k"], v, idx)
    assert nsa.nsa_last_device_error() == 5  # NSA_ERR_DEVICE_CHECK
    v = torch.full_like(inp["v"], 6.0e4)  # in range: the output is that constant
    o, _ = run_ws(w, inp["q"], inp["k"], v, idx)
    assert nsa.nsa_last_device_error() == 0
    assert torch.all(o.float() == torch.tensor(6.0e4).bfloat16().float())


def test_kernel_event_hook_times_the_kernel(cuda_lib):
    """Events handed to nsa_set_kernel_events bracket the block-major kernel
    of the next call on its stream; the hook is off again afterwards."""
    w = small("events_g4_t900", T=900, topk=4)
    inp = W.make_inputs(w, seed=30)
    r = orc.forward(ocfg(w), inp["q"], inp["k"], inp["v"], inp["gates"])
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    idx = torch.from_numpy(r["idx"]).to(DEV)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    b.record()
    nsa.nsa_set_kernel_events(a, b)
    try:
        o, _ = run_ws(w, q, k, v, idx)
    finally:
        nsa.nsa_set_kernel_events(None, None)
    torch.cuda.synchronize()
    assert 0.0 < a.elapsed_time(b) < 1000.0
    assert_close(to_np(o), r["o_sel"], TOL[w.dtype], "o_sel")


@pytest.mark.parametrize("w", [
    # 576 (sequence, group) pairs: the units are dealt by size, two groups per
    # scanning thread
    small("dealt_b9_mha64_t200_k3", B=9, T=200, Hq=64, Hkv=64, topk=3),
    # 1040 pairs, beyond the groups whose units are dealt by size: round-robin slots
    small("roundrobin_b260_g2_t130_k2", B=260, T=130, Hq=8, Hkv=4, topk=2, window=64),
], ids=lambda w: w.name)
def test_sel_bm_many_groups(cuda_lib, w):
    inp = W.make_inputs(w, seed=31)
    rng = np.random.default_rng(32)
    idx = random_idx(w, rng)
    o_ref, lse_ref = orc.sel_attn_fwd(ocfg(w), inp["q"], inp["k"], inp["v"], idx)
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = run_ws(w, q, k, v, torch.from_numpy(idx).to(DEV))
    assert nsa.nsa_last_device_error() == 0
    assert_close(to_np(o), o_ref, TOL[w.dtype], "o_sel")
    assert_close(to_np(lse), lse_ref, LSE_TOL[w.dtype], "lse_sel")
