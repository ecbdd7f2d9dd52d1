"""nsa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin that its host framework hands only input and output
buffers, a runtime serving from a fixed pool with no allocation hook) cannot
provide nsa_decode's workspace; the variant uses the library's fixed device
scratch instead.  This file is collected last on purpose, so that a run that
stops at the first failure has already run every other test.  It must pass
both alone in a fresh process and after the rest of the suite.
"""
import ctypes as C

import pytest
import torch

import sparse_attention_nsa_b200 as nsa
from sparse_attention_nsa_b200 import inputs as W

from helpers import TOL

pytestmark = pytest.mark.gpu


def _decode_inputs(w):
    inp = W.make_decode_inputs(w, seed=21)
    d = {k: v.cuda() for k, v in inp.items()}
    kc = torch.empty((w.B, w.Nc, w.Hkv, w.D), dtype=w.dtype, device="cuda")
    vc = torch.empty_like(kc)
    nsa.nsa_compress(nsa.params_for(w), d["k_cache"], d["v_cache"], kc, vc)
    return d["q"].unsqueeze(1).contiguous(), d["k_cache"], d["v_cache"], kc, vc, \
        d["gates"].unsqueeze(1).contiguous()


@pytest.mark.parametrize("w", [
    W.DECODE_32K.replace(name="noalloc_mqa_b16_t8192", B=16, T=8192),
    W.DECODE_32K.replace(name="noalloc_gqa4_b5_t3000", B=5, T=3000, Hq=16, Hkv=4),
], ids=lambda w: w.name)
def test_noalloc_decode_matches_workspace_decode(cuda_lib, w):
    q, kcache, vcache, kc, vc, gates = _decode_inputs(w)
    p = nsa.params_for(w, Tq=1)
    ref = torch.empty_like(q)
    ref_idx = torch.empty((w.B, 1, w.Hkv, w.topk), dtype=torch.int32, device="cuda")
    nsa.nsa_decode(p, q, kcache, vcache, kc, vc, gates, ref, ref_idx, nsa.alloc_workspace(p))
    for call in range(2):  # the shared scratch keeps the previous call's contents
        out = torch.full_like(q, float("nan"))
        idx = torch.full_like(ref_idx, -7)
        nsa.nsa_decode_noalloc(p, q, kcache, vcache, kc, vc, gates, out, idx)
        torch.cuda.synchronize()
        assert nsa.nsa_last_device_error() == 0
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
