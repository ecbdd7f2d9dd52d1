"""nsa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin that its host framework hands only input and output
buffers, a runtime serving from a fixed pool with no allocation hook) cannot
provide nsa_decode's workspace; the variant uses the library's fixed device
scratch instead.  This file is collected last on purpose, so that a run that
stops at the first failure has already run every other test.  It must pass
both alone in a fresh process and after the rest of the suite.

Every compared call runs right after a no-alloc call of a LARGER problem on
other inputs, so that stale partials, logits or indices left in the shared
scratch would change the result if the decode ever read scratch it had not
written in the same call.
"""
import ctypes as C

import pytest
import torch

import sparse_attention_nsa_b200 as nsa
from sparse_attention_nsa_b200 import inputs as W

from helpers import TOL

pytestmark = pytest.mark.gpu

# the problem whose leftovers fill the scratch before each compared call
POISON = W.DECODE_32K.replace(name="noalloc_poison_mqa_b16_t8192", B=16, T=8192)


def _decode_inputs(w, seed):
    inp = W.make_decode_inputs(w, seed=seed)
    d = {k: v.cuda() for k, v in inp.items()}
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device="cuda")
    vc = torch.empty_like(kc)
    nsa.nsa_compress(nsa.params_for(w), d["k_cache"], d["v_cache"], kc, vc)
    return d["q"].unsqueeze(1).contiguous(), d["k_cache"], d["v_cache"], kc, vc, \
        d["gates"].unsqueeze(1).contiguous()


def _poison_scratch():
    q, kcache, vcache, kc, vc, gates = _decode_inputs(POISON, seed=99)
    p = nsa.params_for(POISON, Tq=1)
    out = torch.empty_like(q)
    idx = torch.empty((POISON.B, 1, POISON.Hkv, POISON.topk), dtype=torch.int32, device="cuda")
    nsa.nsa_decode_noalloc(p, q, kcache, vcache, kc, vc, gates, out, idx)


CASES = [
    # bf16, block 64: the three streaming decode kernels
    (W.DECODE_32K.replace(name="noalloc_mqa_b16_t8192", B=16, T=8192), True),
    (W.DECODE_32K.replace(name="noalloc_gqa4_b5_t3000", B=5, T=3000, Hq=16, Hkv=4), True),
    # fewer causal blocks than top-k: selection slots of -1 (stale slot
    # partials must get no weight)
    (W.DECODE_32K.replace(name="noalloc_short_mqa_b8_t700", B=8, T=700), True),
    # fp32, block 32: the prefill kernels with Tq = 1 on the carved layout
    (W.TINY_F32.replace(name="noalloc_tiny_f32_b3_t256", B=3), True),
    # no idx_out: the index slot is carved from the scratch as well
    (W.TINY_F32.replace(name="noalloc_tiny_f32_b3_t256_noidx", B=3), False),
    (W.DECODE_32K.replace(name="noalloc_gqa4_b5_t3000_noidx", B=5, T=3000, Hq=16, Hkv=4), False),
]


@pytest.mark.parametrize("w,with_idx", CASES, ids=lambda x: x.name if hasattr(x, "name") else "")
def test_noalloc_decode_matches_workspace_decode(cuda_lib, w, with_idx):
    q, kcache, vcache, kc, vc, gates = _decode_inputs(w, seed=21)
    p = nsa.params_for(w, Tq=1)
    ref = torch.empty_like(q)
    ref_idx = torch.empty((w.B, 1, w.Hkv, w.topk), dtype=torch.int32, device="cuda")
    nsa.nsa_decode(p, q, kcache, vcache, kc, vc, gates, ref, ref_idx, nsa.alloc_workspace(p))
    for call in range(2):  # the shared scratch keeps the previous call's contents
        _poison_scratch()
        out = torch.full_like(q, float("nan"))
        idx = torch.full_like(ref_idx, -7) if with_idx else None
        nsa.nsa_decode_noalloc(p, q, kcache, vcache, kc, vc, gates, out, idx)
        torch.cuda.synchronize()
        assert nsa.nsa_last_device_error() == 0
        if with_idx:
            assert torch.equal(idx, ref_idx), f"call {call}: indices differ"
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= TOL[w.dtype], f"call {call}: max-abs {err:.3e}"


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_lib):
    assert nsa.nsa_decode_noalloc_max_scratch() == 16 << 20
    # 4096 sequences x 16 heads: the per-block partials alone exceed 16 MiB
    p = nsa.make_params(4096, 32768, 16, 1, Tq=1)
    ptr = C.c_void_p(1 << 20)  # never dereferenced: rejected before launch
    st = nsa.load().nsa_decode_noalloc(C.byref(p), ptr, ptr, ptr, ptr, ptr, ptr, ptr, None, None)
    assert st == 7  # NSA_ERR_SCRATCH_TOO_SMALL
    assert nsa.nsa_status_string(7) == "NSA_ERR_SCRATCH_TOO_SMALL"
