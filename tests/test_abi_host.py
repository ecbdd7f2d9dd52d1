"""Host-side checks of the C-ABI library (CPU only, no kernel launches).

The library must load, export every symbol include/nsa.h declares, and
reject bad parameter blocks before launching anything.
"""
import ctypes as C
import os
import re

import pytest

import sparse_attention_nsa_b200 as nsa
from sparse_attention_nsa_b200 import abi
from sparse_attention_nsa_b200 import inputs as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(nsa_[a-z0-9_]+)\s*\(", text))
    return names


def test_header_and_binding_agree():
    assert declared_symbols() == set(abi.EXPORTS)


def test_library_loads_and_exports_every_declared_symbol():
    lib = nsa.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert isinstance(C.CDLL(abi.LIB_PATH).nsa_forward, C._CFuncPtr)


def test_status_strings():
    for code, name in abi.STATUS.items():
        assert nsa.nsa_status_string(code) == name


@pytest.mark.parametrize("w", list(W.WORKLOADS.values()), ids=lambda w: w.name)
def test_workload_params_are_accepted(w):
    p = nsa.params_for(w, Tq=1 if "decode" in w.name else None)
    assert nsa.nsa_check_params(p) == 0
    assert nsa.nsa_workspace_size(p) > 0


BAD = [
    (dict(B=0), 1), (dict(T=0), 1), (dict(Tq=5000), 1), (dict(Hkv=3), 1),
    (dict(topk=1), 1), (dict(window=0), 1), (dict(dtype=7), 1), (dict(branch_mask=0), 1),
    (dict(branch_mask=9), 1), (dict(scale=float("nan")), 1), (dict(scale=-0.125), 1), (dict(scale=0.0), 1),
    (dict(scale=float("inf")), 1),
    (dict(D=128), 2), (dict(cmp_stride=2), 2), (dict(sel_block=2), 2),
    (dict(Hq=24, Hkv=4), 2), (dict(topk=65), 2), (dict(T=200000), 2),
    # T + l' - 1 past INT_MAX: the block count must not wrap to a negative number
    (dict(T=2**31 - 1, cmp_block=2**31 - 1, cmp_stride=1, sel_block=2), 2),
    # B T >= 2^31 key rows (32-bit tensor-map coordinates), geometry otherwise valid
    (dict(B=2**15, T=2**16, cmp_block=2**16, sel_block=2**10), 2),
]


@pytest.mark.parametrize("change", [dict(cmp_stride=32), dict(sel_block=32),
                                    dict(cmp_block=128, cmp_stride=64, sel_block=64),
                                    dict(cmp_block=32, cmp_stride=16, sel_block=64),
                                    dict(cmp_block=16, cmp_stride=8, sel_block=32)])
def test_general_block_geometry_accepted(change):
    """Compression block and stride other than the selection block run
    (reading R14: a selection block's importance is summed over the
    compressed blocks that overlap it)."""
    p = nsa.make_params(1, 4096, 16, 4)
    for k, v in change.items():
        setattr(p, k, v)
    assert nsa.nsa_check_params(p) == 0
    assert nsa.nsa_workspace_size(p) > 0
    assert nsa.nsa_backward_workspace_size(p) > 0


@pytest.mark.parametrize("change,code", BAD)
def test_bad_params_rejected(change, code):
    base = dict(B=1, T=4096, Hq=16, Hkv=4)
    kw = {k: change.pop(k) for k in list(change) if k in base}
    base.update(kw)
    p = nsa.make_params(**base)
    for k, v in change.items():
        setattr(p, k, v)
    assert nsa.nsa_check_params(p) == code
    n = C.c_size_t(0)
    assert nsa.load().nsa_workspace_size(C.byref(p), C.byref(n)) == code


def test_null_pointers_rejected_before_launch():
    lib = nsa.load()
    p = nsa.make_params(1, 256, 4, 1, cmp_block=32, topk=4, window=64, dtype=nsa.NSA_F32)
    assert lib.nsa_compress(C.byref(p), None, None, None, None, None) == 1
    assert lib.nsa_swa_fwd(C.byref(p), None, None, None, None, None, None) == 1
    assert lib.nsa_forward(C.byref(p), None, None, None, None, None, None, None, 0, None) == 1
    assert lib.nsa_sel_attn_fwd(C.byref(p), C.c_void_p(16), C.c_void_p(32), C.c_void_p(48),
                                C.c_void_p(64), C.c_void_p(8), None, None) == 1  # misaligned o
    p.Tq = 2
    assert lib.nsa_decode(C.byref(p), *([C.c_void_p(256)] * 7), None, None, 0, None) == 1


def test_forward_without_workspace_is_rejected():
    lib = nsa.load()
    p = nsa.make_params(1, 256, 4, 1, cmp_block=32, topk=4, window=64, dtype=nsa.NSA_F32)
    ptr = C.c_void_p(4096)
    assert lib.nsa_forward(C.byref(p), ptr, ptr, ptr, ptr, ptr, None, None, 0, None) == 6


def test_kernel_event_hook_arguments():
    """The profiling hook takes both events or neither; it touches no device."""
    lib = nsa.load()
    assert lib.nsa_set_kernel_events(C.c_void_p(64), None) == 1  # NSA_ERR_INVALID_ARG
    assert lib.nsa_set_kernel_events(None, C.c_void_p(64)) == 1
    assert lib.nsa_set_kernel_events(None, None) == 0


def test_forward_host_workspace_and_argument_checks():
    """The host-buffer forward needs nsa_forward's workspace plus device room
    for q, k, v, gates and out; NULL host pointers and a missing workspace
    are rejected before anything is enqueued."""
    p = nsa.make_params(2, 1000, 16, 4, topk=5, window=200)
    fwd = nsa.nsa_workspace_size(p)
    need = nsa.nsa_forward_host_workspace_size(p)
    al = lambda n: (n + 255) // 256 * 256
    tens = 2 * al(2 * 1000 * 16 * 64 * 2) + 2 * al(2 * 1000 * 4 * 64 * 2) + al(2 * 1000 * 16 * 3 * 4)
    assert need == tens + al(fwd)
    lib = nsa.load()
    host = C.c_void_p(4096)  # never dereferenced: the checks come first
    assert lib.nsa_forward_host(C.byref(p), None, host, host, host, host, host, need, None) == 1
    assert lib.nsa_forward_host(C.byref(p), host, host, host, host, None, host, need, None) == 1
    assert lib.nsa_forward_host(C.byref(p), host, host, host, host, host, None, need, None) == 6
    assert lib.nsa_forward_host(C.byref(p), host, host, host, host, host, host, need - 1,
                                None) == 6  # NSA_ERR_WORKSPACE
    bad = nsa.make_params(2, 1000, 16, 4, scale=-1.0)
    assert lib.nsa_forward_host(C.byref(bad), host, host, host, host, host, host, need,
                                None) == 1


def test_parametric_compression_checks_before_launch():
    """The parametric compressor runs bf16 only (NSA_ERR_UNSUPPORTED for
    fp32), rejects NULL or misaligned pointers, a missing workspace and a
    missing saved-tensor block before anything is enqueued, and sizes its
    workspaces as the mean-pool path's plus its own."""
    lib = nsa.load()
    ptr = C.c_void_p(4096)  # aligned, never dereferenced: the checks come first
    f32 = nsa.make_params(1, 1000, 16, 4, cmp_block=32, cmp_stride=16, dtype=nsa.NSA_F32)
    assert lib.nsa_compress_mlp(C.byref(f32), *([ptr] * 6), ptr, 1 << 30, None) == 2
    assert lib.nsa_forward_mlp(C.byref(f32), *([ptr] * 7), None, ptr, 1 << 30, None) == 2
    p = nsa.make_params(1, 1000, 16, 4, cmp_block=32, cmp_stride=16)
    assert lib.nsa_compress_mlp(C.byref(p), None, ptr, ptr, ptr, ptr, ptr, ptr, 1 << 30,
                                None) == 1
    assert lib.nsa_compress_mlp(C.byref(p), ptr, ptr, C.c_void_p(4100), ptr, ptr, ptr, ptr,
                                1 << 30, None) == 1  # misaligned wk
    fws = nsa.nsa_compress_mlp_workspace_size(p)
    assert fws > 0  # 61 blocks x 4 groups: the token offsets are split over CTAs
    assert lib.nsa_compress_mlp(C.byref(p), *([ptr] * 6), None, 0, None) == 6
    assert lib.nsa_compress_mlp(C.byref(p), *([ptr] * 6), ptr, fws - 1, None) == 6
    assert nsa.nsa_forward_mlp_workspace_size(p) >= nsa.nsa_workspace_size(p) + fws
    bws = nsa.nsa_compress_mlp_bwd_workspace_size(p)
    nq = 1 * p.Nc * 4
    assert bws >= 2 * nq * 32 * 64 * 4  # the per-block row gradients, fp32
    assert nsa.nsa_backward_mlp_workspace_size(p) == nsa.nsa_backward_workspace_size(p) + bws
    args = [ptr] * 4 + [ptr] * 6
    assert lib.nsa_compress_mlp_bwd(C.byref(p), *args, None, 0, None) == 6
    # nsa_backward_mlp: q k v wk wv gates dout saved dq dk dv dwk dwv dgates
    assert lib.nsa_backward_mlp(C.byref(p), *([ptr] * 7), None, *([ptr] * 6), ptr,
                                1 << 30, None) == 1  # no saved tensors
    # enough output tiles: one CTA per tile, no partial sums
    wide = nsa.make_params(1, 2400, 64, 64, cmp_block=32, cmp_stride=16, window=64)
    assert nsa.nsa_compress_mlp_workspace_size(wide) == 0


MOBA_CASES = [
    (dict(), 0),                                  # block 512, top-3 at T 8192
    (dict(block=64, topk=16), 0),                 # 128 blocks of 64
    (dict(block=0), 1), (dict(topk=0), 1), (dict(Hkv=3), 1), (dict(scale=float("nan")), 1),
    (dict(block=100), 2),                         # not a multiple of 64
    (dict(block=64, topk=1), 2),                  # one 64-key block: below the kernels' two
    (dict(block=64, T=16384), 2),                 # 256 MoBA blocks > 128
    (dict(topk=9), 2),                            # 9 x 8 = 72 selection blocks > 64
    (dict(T=131072, block=1024), 2),              # 2048 64-key blocks > 1024
    (dict(block=256, topk=2**30 + 4), 2),         # k L / 64 wraps to 16 in 32 bits
    (dict(D=128), 2),
]


@pytest.mark.parametrize("change,code", MOBA_CASES)
def test_moba_params_checked_before_launch(change, code):
    """MoBA's limits (MoBA blocks of a multiple of 64 tokens, at most 128 of
    them, k L / 64 <= 64 selection blocks) and the shared parameter checks,
    all answered by the workspace query without a device."""
    base = dict(B=1, T=8192, Hq=16, Hkv=4, block=512, topk=3)
    base.update({k: v for k, v in change.items() if k in base})
    p = nsa.make_moba_params(**base)
    for k, v in change.items():
        if k not in base:
            setattr(p, k, v)
    n = C.c_size_t(0)
    assert nsa.load().nsa_moba_workspace_size(C.byref(p), C.byref(n)) == code
    if code == 0:
        assert n.value > 0


def test_moba_pointer_and_workspace_checks():
    """Every case fails a check before anything is enqueued (the pointers
    are never dereferenced)."""
    lib = nsa.load()
    p = nsa.make_moba_params(1, 8192, 16, 4)
    need = nsa.nsa_moba_workspace_size(p)
    ptr = C.c_void_p(4096)  # aligned, never dereferenced: the checks come first
    assert lib.nsa_moba_forward(C.byref(p), None, ptr, ptr, ptr, None, None, ptr, need,
                                None) == 1
    assert lib.nsa_moba_forward(C.byref(p), ptr, ptr, ptr, ptr, C.c_void_p(4100), None, ptr,
                                need, None) == 1  # misaligned lse
    assert lib.nsa_moba_forward(C.byref(p), ptr, ptr, ptr, ptr, None, None, ptr, 0,
                                None) == 6  # NSA_ERR_WORKSPACE
    assert lib.nsa_moba_forward(C.byref(p), ptr, ptr, ptr, ptr, None, None, None, need,
                                None) == 6
    assert lib.nsa_moba_backward(C.byref(p), *([ptr] * 6), None, *([ptr] * 3), ptr, need,
                                 None) == 1  # no dout
    assert lib.nsa_moba_backward(C.byref(p), *([ptr] * 10), None, 0, None) == 6


def test_binding_checks_tensors_before_calling_the_library():
    """The binding's marshalling refuses host tensors where the library
    wants device pointers (and the reverse for the host-buffer forward),
    non-contiguous tensors, wrong dtypes and wrong shapes, before any call
    into the library."""
    import torch
    p = nsa.make_params(1, 256, 4, 1, cmp_block=32, topk=4, window=64, dtype=nsa.NSA_F32)
    q = torch.zeros(1, 256, 4, 64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        nsa.nsa_swa_fwd(p, q, q[:, :, :1], q[:, :, :1], q, torch.zeros(1, 256, 4))
    with pytest.raises(ValueError, match="required"):
        abi._ptr(None, name="q")
    assert abi._ptr(None, name="lse", nullable=True) is None
    with pytest.raises(TypeError):
        abi._ptr([0.0], name="q")
    s = abi._shapes(p)
    with pytest.raises(ValueError, match="contiguous"):
        abi._host_ptr(torch.zeros(1, 4, 256, 64).transpose(1, 2), s["q"], torch.float32, "q")
    with pytest.raises(ValueError, match="float32"):
        abi._host_ptr(torch.zeros(s["q"], dtype=torch.float64), s["q"], torch.float32, "q")
    with pytest.raises(ValueError, match="shape"):
        abi._host_ptr(torch.zeros(1, 255, 4, 64), s["q"], torch.float32, "q")
    assert abi._host_ptr(q, s["q"], torch.float32, "q").value == q.data_ptr()
