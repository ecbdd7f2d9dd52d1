"""ctypes binding of libnsa (include/nsa.h), one function per C entry point.

Argument marshalling only: every function checks that its torch tensors
live on the current CUDA device with the dtype, shape and contiguity the C
ABI documents, passes their device pointers and the current CUDA stream to
the library, and raises NsaError on a non-OK status.  All arithmetic runs in
libnsa's CUDA kernels; there is no fallback path.  PyTorch only provides
device memory and streams.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnsa.so")

NSA_F32, NSA_BF16 = 0, 1
NSA_BRANCH_CMP, NSA_BRANCH_SEL, NSA_BRANCH_SWA = 1, 2, 4
NSA_BRANCH_ALL = 7

STATUS = {0: "NSA_OK", 1: "NSA_ERR_INVALID_ARG", 2: "NSA_ERR_UNSUPPORTED",
          3: "NSA_ERR_CUDA", 4: "NSA_ERR_TIMEOUT", 5: "NSA_ERR_DEVICE_CHECK",
          6: "NSA_ERR_WORKSPACE", 7: "NSA_ERR_SCRATCH_TOO_SMALL"}

# every symbol include/nsa.h declares
EXPORTS = ("nsa_status_string", "nsa_check_params", "nsa_workspace_size",
           "nsa_last_device_error", "nsa_compress", "nsa_cmp_attn_scores",
           "nsa_select_topk", "nsa_sel_attn_fwd", "nsa_swa_fwd", "nsa_gate_combine",
           "nsa_forward", "nsa_decode", "nsa_backward_workspace_size",
           "nsa_gate_combine_bwd", "nsa_sel_attn_bwd", "nsa_swa_bwd", "nsa_cmp_bwd",
           "nsa_backward", "nsa_decode_noalloc", "nsa_decode_noalloc_max_scratch",
           "nsa_sel_workspace_size", "nsa_sel_attn_fwd_ws", "nsa_set_kernel_events",
           "nsa_forward_host_workspace_size", "nsa_forward_host",
           "nsa_moba_workspace_size", "nsa_moba_forward", "nsa_moba_backward",
           "nsa_sel_attn_bwd_atomic", "nsa_compress_mlp_workspace_size", "nsa_compress_mlp",
           "nsa_compress_mlp_bwd_workspace_size", "nsa_compress_mlp_bwd",
           "nsa_forward_mlp_workspace_size", "nsa_forward_mlp", "nsa_backward_mlp_workspace_size",
           "nsa_backward_mlp")


class NsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class Params(C.Structure):
    """Mirror of nsa_params."""
    _fields_ = [("B", C.c_int), ("T", C.c_int), ("Tq", C.c_int), ("Hq", C.c_int),
                ("Hkv", C.c_int), ("D", C.c_int), ("cmp_block", C.c_int),
                ("cmp_stride", C.c_int), ("sel_block", C.c_int), ("topk", C.c_int),
                ("window", C.c_int), ("scale", C.c_float), ("dtype", C.c_int),
                ("branch_mask", C.c_int)]

    @property
    def Nc(self) -> int:
        if self.T < self.cmp_block:
            return 0
        return (self.T - self.cmp_block) // self.cmp_stride + 1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == NSA_BF16 else torch.float32


class Saved(C.Structure):
    """Mirror of nsa_saved (device pointers, 0 = put it in the workspace)."""
    _fields_ = [("kc", C.c_void_p), ("vc", C.c_void_p), ("o_cmp", C.c_void_p),
                ("lse_cmp", C.c_void_p), ("score", C.c_void_p), ("idx", C.c_void_p),
                ("o_sel", C.c_void_p), ("lse_sel", C.c_void_p), ("o_swa", C.c_void_p),
                ("lse_swa", C.c_void_p)]


_lib = None


def load():
    """Load libnsa.so; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_attention_nsa_b200.build`")
        lib = C.CDLL(LIB_PATH)
        vp, P = C.c_void_p, C.POINTER(Params)
        sig = {
            "nsa_status_string": ([C.c_int], C.c_char_p),
            "nsa_check_params": ([P], C.c_int),
            "nsa_workspace_size": ([P, C.POINTER(C.c_size_t)], C.c_int),
            "nsa_last_device_error": ([vp], C.c_int),
            "nsa_compress": ([P, vp, vp, vp, vp, vp], C.c_int),
            "nsa_cmp_attn_scores": ([P, vp, vp, vp, vp, vp, vp, vp], C.c_int),
            "nsa_select_topk": ([P, vp, vp, vp], C.c_int),
            "nsa_sel_attn_fwd": ([P, vp, vp, vp, vp, vp, vp, vp], C.c_int),
            "nsa_swa_fwd": ([P, vp, vp, vp, vp, vp, vp], C.c_int),
            "nsa_gate_combine": ([P, vp, vp, vp, vp, vp, vp], C.c_int),
            "nsa_forward": ([P, vp, vp, vp, vp, vp, C.POINTER(Saved), vp, C.c_size_t, vp],
                            C.c_int),
            "nsa_decode": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp, C.c_size_t, vp], C.c_int),
            "nsa_forward_host_workspace_size": ([P, C.POINTER(C.c_size_t)], C.c_int),
            "nsa_forward_host": ([P, vp, vp, vp, vp, vp, vp, C.c_size_t, vp], C.c_int),
            "nsa_decode_noalloc": ([P, vp, vp, vp, vp, vp, vp, vp, vp, vp], C.c_int),
            "nsa_backward_workspace_size": ([P, C.POINTER(C.c_size_t)], C.c_int),
            "nsa_gate_combine_bwd": ([P] + [vp] * 10, C.c_int),
            "nsa_sel_attn_bwd": ([P] + [vp] * 11 + [C.c_size_t, vp], C.c_int),
            "nsa_sel_attn_bwd_atomic": ([P] + [vp] * 11 + [C.c_size_t, vp], C.c_int),
            "nsa_swa_bwd": ([P] + [vp] * 10 + [C.c_size_t, vp], C.c_int),
            "nsa_cmp_bwd": ([P] + [vp] * 10 + [C.c_size_t, vp], C.c_int),
            "nsa_backward": ([P, vp, vp, vp, vp, vp, C.POINTER(Saved), vp, vp, vp, vp, vp,
                              C.c_size_t, vp], C.c_int),
            "nsa_decode_noalloc_max_scratch": ([], C.c_size_t),
            "nsa_sel_workspace_size": ([P, C.POINTER(C.c_size_t)], C.c_int),
            "nsa_sel_attn_fwd_ws": ([P, vp, vp, vp, vp, vp, vp, vp, C.c_size_t, vp], C.c_int),
            "nsa_set_kernel_events": ([vp, vp], C.c_int),
            "nsa_moba_workspace_size": ([C.POINTER(MobaParams), C.POINTER(C.c_size_t)],
                                        C.c_int),
            "nsa_moba_forward": ([C.POINTER(MobaParams)] + [vp] * 7 + [C.c_size_t, vp],
                                 C.c_int),
            "nsa_moba_backward": ([C.POINTER(MobaParams)] + [vp] * 11 + [C.c_size_t, vp],
                                  C.c_int),
            "nsa_compress_mlp_workspace_size": ([P, C.POINTER(C.c_size_t)], C.c_int),
            "nsa_compress_mlp": ([P] + [vp] * 7 + [C.c_size_t, vp], C.c_int),
            "nsa_forward_mlp_workspace_size": ([P, C.POINTER(C.c_size_t)], C.c_int),
            "nsa_compress_mlp_bwd_workspace_size": ([P, C.POINTER(C.c_size_t)], C.c_int),
            "nsa_compress_mlp_bwd": ([P] + [vp] * 11 + [C.c_size_t, vp], C.c_int),
            "nsa_forward_mlp": ([P, vp, vp, vp, vp, vp, vp, vp, C.POINTER(Saved), vp,
                                 C.c_size_t, vp], C.c_int),
            "nsa_backward_mlp_workspace_size": ([P, C.POINTER(C.c_size_t)], C.c_int),
            "nsa_backward_mlp": ([P, vp, vp, vp, vp, vp, vp, vp, C.POINTER(Saved)] + [vp] * 7
                                 + [C.c_size_t, vp], C.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
    return _lib


class MobaParams(C.Structure):
    """Mirror of nsa_moba_params."""
    _fields_ = [("B", C.c_int), ("T", C.c_int), ("Tq", C.c_int), ("Hq", C.c_int),
                ("Hkv", C.c_int), ("D", C.c_int), ("block", C.c_int), ("topk", C.c_int),
                ("scale", C.c_float), ("dtype", C.c_int)]


def make_moba_params(B, T, Hq, Hkv, D=64, *, Tq=None, block=512, topk=3, scale=None,
                     dtype=NSA_BF16) -> MobaParams:
    if isinstance(dtype, torch.dtype):
        dtype = NSA_BF16 if dtype == torch.bfloat16 else NSA_F32
    return MobaParams(B, T, T if Tq is None else Tq, Hq, Hkv, D, block, topk,
                      float(D ** -0.5 if scale is None else scale), dtype)


def make_params(B, T, Hq, Hkv, D=64, *, Tq=None, cmp_block=64, cmp_stride=None,
                sel_block=None, topk=16, window=512, scale=None, dtype=NSA_BF16,
                branch_mask=NSA_BRANCH_ALL) -> Params:
    if isinstance(dtype, torch.dtype):
        dtype = NSA_BF16 if dtype == torch.bfloat16 else NSA_F32
    return Params(B, T, T if Tq is None else Tq, Hq, Hkv, D, cmp_block,
                  cmp_block if cmp_stride is None else cmp_stride,
                  cmp_block if sel_block is None else sel_block, topk, window,
                  float(D ** -0.5 if scale is None else scale), dtype, branch_mask)


def params_for(w, Tq=None) -> Params:
    """Params of a sparse_attention_nsa_b200.inputs.Workload."""
    return make_params(w.B, w.T, w.Hq, w.Hkv, w.D, Tq=Tq, cmp_block=w.cmp_block,
                       cmp_stride=w.cmp_stride, sel_block=w.sel_block, topk=w.topk,
                       window=w.window, scale=w.scale, dtype=w.dtype,
                       branch_mask=w.branch_mask)


# ------------------------------------------------------------------ helpers
def _stream(stream):
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


def _ptr(t, shape=None, dtype=None, name="tensor", nullable=False):
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return C.c_void_p(t.data_ptr())


def _check(st: int, where: str):
    if st != 0:
        raise NsaError(st, where)


def _shapes(p: Params):
    B, T, Tq, Hq, Hkv, D = p.B, p.T, p.Tq, p.Hq, p.Hkv, p.D
    return {"q": (B, Tq, Hq, D), "k": (B, T, Hkv, D), "kc": (B, p.Nc, Hkv, D),
            "o": (B, Tq, Hq, D), "lse": (B, Tq, Hq), "score": (B, Tq, Hkv, p.Nc),
            "idx": (B, Tq, Hkv, p.topk), "gates": (B, Tq, Hq, 3)}


# ------------------------------------------------------------------ entry points
def nsa_status_string(status: int) -> str:
    return load().nsa_status_string(status).decode()


def nsa_check_params(p: Params) -> int:
    return load().nsa_check_params(C.byref(p))


def nsa_workspace_size(p: Params) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_workspace_size(C.byref(p), C.byref(n)), "nsa_workspace_size")
    return n.value


def nsa_last_device_error(stream=None) -> int:
    return load().nsa_last_device_error(_stream(stream))


def nsa_compress(p: Params, k, v, kc, vc, stream=None):
    s, dt = _shapes(p), p.torch_dtype
    _check(load().nsa_compress(C.byref(p), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
                               _ptr(kc, s["kc"], dt, "kc"), _ptr(vc, s["kc"], dt, "vc"),
                               _stream(stream)), "nsa_compress")


def nsa_cmp_attn_scores(p: Params, q, kc, vc, o_cmp, lse_cmp, score, stream=None):
    s, dt = _shapes(p), p.torch_dtype
    _check(load().nsa_cmp_attn_scores(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(kc, s["kc"], dt, "kc"),
        _ptr(vc, s["kc"], dt, "vc"), _ptr(o_cmp, s["o"], dt, "o_cmp", True),
        _ptr(lse_cmp, s["lse"], torch.float32, "lse_cmp", True),
        _ptr(score, s["score"], torch.float32, "score"), _stream(stream)),
        "nsa_cmp_attn_scores")


def nsa_select_topk(p: Params, score, idx, stream=None):
    s = _shapes(p)
    _check(load().nsa_select_topk(C.byref(p), _ptr(score, s["score"], torch.float32, "score"),
                                  _ptr(idx, s["idx"], torch.int32, "idx"), _stream(stream)),
           "nsa_select_topk")


def nsa_sel_attn_fwd(p: Params, q, k, v, idx, o_sel, lse_sel, stream=None):
    s, dt = _shapes(p), p.torch_dtype
    _check(load().nsa_sel_attn_fwd(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"),
        _ptr(v, s["k"], dt, "v"), _ptr(idx, s["idx"], torch.int32, "idx"),
        _ptr(o_sel, s["o"], dt, "o_sel"), _ptr(lse_sel, s["lse"], torch.float32, "lse_sel", True),
        _stream(stream)), "nsa_sel_attn_fwd")


def nsa_set_kernel_events(start=None, stop=None):
    """Record torch.cuda.Event pair (start, stop) around the block-major
    selection kernel of later calls; None, None turns it off."""
    ptr = lambda e: None if e is None else C.c_void_p(e.cuda_event)
    _check(load().nsa_set_kernel_events(ptr(start), ptr(stop)), "nsa_set_kernel_events")


def nsa_sel_workspace_size(p: Params) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_sel_workspace_size(C.byref(p), C.byref(n)), "nsa_sel_workspace_size")
    return n.value


def nsa_sel_attn_fwd_ws(p: Params, q, k, v, idx, o_sel, lse_sel, workspace, stream=None):
    s, dt = _shapes(p), p.torch_dtype
    _check(load().nsa_sel_attn_fwd_ws(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"),
        _ptr(v, s["k"], dt, "v"), _ptr(idx, s["idx"], torch.int32, "idx"),
        _ptr(o_sel, s["o"], dt, "o_sel", True),
        _ptr(lse_sel, s["lse"], torch.float32, "lse_sel", True),
        _ptr(workspace, None, torch.uint8, "workspace"), C.c_size_t(workspace.numel()),
        _stream(stream)), "nsa_sel_attn_fwd_ws")


def nsa_swa_fwd(p: Params, q, k, v, o_swa, lse_swa, stream=None):
    s, dt = _shapes(p), p.torch_dtype
    _check(load().nsa_swa_fwd(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"),
        _ptr(v, s["k"], dt, "v"), _ptr(o_swa, s["o"], dt, "o_swa"),
        _ptr(lse_swa, s["lse"], torch.float32, "lse_swa", True), _stream(stream)),
        "nsa_swa_fwd")


def nsa_gate_combine(p: Params, gates, o_cmp, o_sel, o_swa, out, stream=None):
    s, dt = _shapes(p), p.torch_dtype
    m = p.branch_mask
    _check(load().nsa_gate_combine(
        C.byref(p), _ptr(gates, s["gates"], torch.float32, "gates"),
        _ptr(o_cmp, s["o"], dt, "o_cmp", not m & 1), _ptr(o_sel, s["o"], dt, "o_sel", not m & 2),
        _ptr(o_swa, s["o"], dt, "o_swa", not m & 4), _ptr(out, s["o"], dt, "out"),
        _stream(stream)), "nsa_gate_combine")


def nsa_forward(p: Params, q, k, v, gates, out, saved: dict | None = None,
                workspace=None, stream=None):
    """saved: optional dict of tensors named like nsa_saved's fields."""
    s, dt = _shapes(p), p.torch_dtype
    sv = Saved()
    if saved:
        want = {"kc": (s["kc"], dt), "vc": (s["kc"], dt), "o_cmp": (s["o"], dt),
                "lse_cmp": (s["lse"], torch.float32), "score": (s["score"], torch.float32),
                "idx": (s["idx"], torch.int32), "o_sel": (s["o"], dt),
                "lse_sel": (s["lse"], torch.float32), "o_swa": (s["o"], dt),
                "lse_swa": (s["lse"], torch.float32)}
        for name, t in saved.items():
            shp, tdt = want[name]
            setattr(sv, name, _ptr(t, shp, tdt, name).value)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size()
    _check(load().nsa_forward(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(gates, s["gates"], torch.float32, "gates"), _ptr(out, s["o"], dt, "out"),
        C.byref(sv), ws_ptr, ws_bytes, _stream(stream)), "nsa_forward")


def _host_ptr(t, shape, dtype, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return C.c_void_p(t.data_ptr())


def nsa_forward_host_workspace_size(p: Params) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_forward_host_workspace_size(C.byref(p), C.byref(n)),
           "nsa_forward_host_workspace_size")
    return n.value


def nsa_forward_host(p: Params, q, k, v, gates, out, workspace, stream=None):
    """nsa_forward on host (CPU, ideally pinned) tensors: the library copies
    them in, runs the forward and copies out back, all enqueued on the
    stream; out is valid once the stream has been synchronised."""
    s, dt = _shapes(p), p.torch_dtype
    _check(load().nsa_forward_host(
        C.byref(p), _host_ptr(q, s["q"], dt, "q"), _host_ptr(k, s["k"], dt, "k"),
        _host_ptr(v, s["k"], dt, "v"), _host_ptr(gates, s["gates"], torch.float32, "gates"),
        _host_ptr(out, s["o"], dt, "out"), _ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "nsa_forward_host")


def nsa_decode(p: Params, q, k_cache, v_cache, kc_cache, vc_cache, gates, out,
               idx_out=None, workspace=None, stream=None):
    s, dt = _shapes(p), p.torch_dtype
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size()
    _check(load().nsa_decode(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k_cache, s["k"], dt, "k_cache"),
        _ptr(v_cache, s["k"], dt, "v_cache"), _ptr(kc_cache, s["kc"], dt, "kc_cache", p.Nc == 0),
        _ptr(vc_cache, s["kc"], dt, "vc_cache", p.Nc == 0),
        _ptr(gates, s["gates"], torch.float32, "gates"), _ptr(out, s["o"], dt, "out"),
        _ptr(idx_out, s["idx"], torch.int32, "idx_out", True), ws_ptr, ws_bytes,
        _stream(stream)), "nsa_decode")


# ------------------------------------------------------------------ backward
def nsa_backward_workspace_size(p: Params) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_backward_workspace_size(C.byref(p), C.byref(n)),
           "nsa_backward_workspace_size")
    return n.value


def _ws(workspace):
    if workspace is None:
        return None, 0
    return _ptr(workspace, name="workspace"), workspace.numel() * workspace.element_size()


def nsa_gate_combine_bwd(p: Params, gates, dout, o_cmp, o_sel, o_swa, dgates,
                         dO_cmp=None, dO_sel=None, dO_swa=None, stream=None):
    s, dt, f = _shapes(p), p.torch_dtype, torch.float32
    m = p.branch_mask
    _check(load().nsa_gate_combine_bwd(
        C.byref(p), _ptr(gates, s["gates"], f, "gates"), _ptr(dout, s["o"], dt, "dout"),
        _ptr(o_cmp, s["o"], dt, "o_cmp", not m & 1), _ptr(o_sel, s["o"], dt, "o_sel", not m & 2),
        _ptr(o_swa, s["o"], dt, "o_swa", not m & 4), _ptr(dgates, s["gates"], f, "dgates"),
        _ptr(dO_cmp, s["o"], f, "dO_cmp", True), _ptr(dO_sel, s["o"], f, "dO_sel", True),
        _ptr(dO_swa, s["o"], f, "dO_swa", True), _stream(stream)), "nsa_gate_combine_bwd")


def nsa_sel_attn_bwd(p: Params, q, k, v, idx, o_sel, lse_sel, dO_sel, dq, dk, dv,
                     workspace, stream=None):
    s, dt, f = _shapes(p), p.torch_dtype, torch.float32
    wp, wb = _ws(workspace)
    _check(load().nsa_sel_attn_bwd(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(idx, s["idx"], torch.int32, "idx"), _ptr(o_sel, s["o"], dt, "o_sel"),
        _ptr(lse_sel, s["lse"], f, "lse_sel"), _ptr(dO_sel, s["o"], f, "dO_sel"),
        _ptr(dq, s["q"], f, "dq"), _ptr(dk, s["k"], f, "dk"), _ptr(dv, s["k"], f, "dv"),
        wp, wb, _stream(stream)), "nsa_sel_attn_bwd")


def nsa_sel_attn_bwd_atomic(p: Params, q, k, v, idx, o_sel, lse_sel, dO_sel, dq, dk, dv,
                            workspace, stream=None):
    """Single-pass selection backward (dK / dV by atomics); arguments as
    nsa_sel_attn_bwd."""
    s, dt, f = _shapes(p), p.torch_dtype, torch.float32
    wp, wb = _ws(workspace)
    _check(load().nsa_sel_attn_bwd_atomic(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(idx, s["idx"], torch.int32, "idx"), _ptr(o_sel, s["o"], dt, "o_sel"),
        _ptr(lse_sel, s["lse"], f, "lse_sel"), _ptr(dO_sel, s["o"], f, "dO_sel"),
        _ptr(dq, s["q"], f, "dq"), _ptr(dk, s["k"], f, "dk"), _ptr(dv, s["k"], f, "dv"),
        wp, wb, _stream(stream)), "nsa_sel_attn_bwd_atomic")


def nsa_swa_bwd(p: Params, q, k, v, o_swa, lse_swa, dO_swa, dq, dk, dv, workspace,
                stream=None):
    s, dt, f = _shapes(p), p.torch_dtype, torch.float32
    wp, wb = _ws(workspace)
    _check(load().nsa_swa_bwd(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(o_swa, s["o"], dt, "o_swa"), _ptr(lse_swa, s["lse"], f, "lse_swa"),
        _ptr(dO_swa, s["o"], f, "dO_swa"), _ptr(dq, s["q"], f, "dq"), _ptr(dk, s["k"], f, "dk"),
        _ptr(dv, s["k"], f, "dv"), wp, wb, _stream(stream)), "nsa_swa_bwd")


def nsa_cmp_bwd(p: Params, q, kc, vc, o_cmp, lse_cmp, dO_cmp, dq, dk, dv, workspace,
                stream=None):
    s, dt, f = _shapes(p), p.torch_dtype, torch.float32
    wp, wb = _ws(workspace)
    _check(load().nsa_cmp_bwd(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(kc, s["kc"], dt, "kc", p.Nc == 0),
        _ptr(vc, s["kc"], dt, "vc", p.Nc == 0), _ptr(o_cmp, s["o"], dt, "o_cmp"),
        _ptr(lse_cmp, s["lse"], f, "lse_cmp"), _ptr(dO_cmp, s["o"], f, "dO_cmp"),
        _ptr(dq, s["q"], f, "dq"), _ptr(dk, s["k"], f, "dk"), _ptr(dv, s["k"], f, "dv"),
        wp, wb, _stream(stream)), "nsa_cmp_bwd")


def nsa_backward(p: Params, q, k, v, gates, dout, saved: dict, dq, dk, dv, dgates,
                 workspace, stream=None):
    """saved: the forward's tensors by nsa_saved field name (see nsa.h)."""
    s, dt, f = _shapes(p), p.torch_dtype, torch.float32
    sv = Saved()
    for name, t in saved.items():
        if t is not None and t.numel() > 0:
            setattr(sv, name, _ptr(t, name=name).value)
    wp, wb = _ws(workspace)
    _check(load().nsa_backward(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(gates, s["gates"], f, "gates"), _ptr(dout, s["o"], dt, "dout"), C.byref(sv),
        _ptr(dq, s["q"], f, "dq"), _ptr(dk, s["k"], f, "dk"), _ptr(dv, s["k"], f, "dv"),
        _ptr(dgates, s["gates"], f, "dgates"), wp, wb, _stream(stream)), "nsa_backward")


def backward(p: Params, q, k, v, gates, dout, saved: dict, workspace=None, stream=None):
    """Allocate fp32 gradients with torch and run nsa_backward."""
    s, dev = _shapes(p), q.device
    dq = torch.empty(s["q"], dtype=torch.float32, device=dev)
    dk = torch.empty(s["k"], dtype=torch.float32, device=dev)
    dv = torch.empty(s["k"], dtype=torch.float32, device=dev)
    dg = torch.empty(s["gates"], dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(max(nsa_backward_workspace_size(p), 1), dtype=torch.uint8,
                                device=dev)
    nsa_backward(p, q, k, v, gates, dout, saved, dq, dk, dv, dg, workspace, stream)
    return dq, dk, dv, dg


def nsa_decode_noalloc(p: Params, q, k_cache, v_cache, kc_cache, vc_cache, gates, out,
                       idx_out=None, stream=None):
    """nsa_decode without a workspace: the library's fixed device scratch is
    used instead (for callers that cannot allocate; see include/nsa.h)."""
    s, dt = _shapes(p), p.torch_dtype
    _check(load().nsa_decode_noalloc(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k_cache, s["k"], dt, "k_cache"),
        _ptr(v_cache, s["k"], dt, "v_cache"), _ptr(kc_cache, s["kc"], dt, "kc_cache", p.Nc == 0),
        _ptr(vc_cache, s["kc"], dt, "vc_cache", p.Nc == 0),
        _ptr(gates, s["gates"], torch.float32, "gates"), _ptr(out, s["o"], dt, "out"),
        _ptr(idx_out, s["idx"], torch.int32, "idx_out", True), _stream(stream)),
        "nsa_decode_noalloc")


def nsa_decode_noalloc_max_scratch() -> int:
    return int(load().nsa_decode_noalloc_max_scratch())


# ------------------------------------------------------------------ conveniences
def alloc_workspace(p: Params, device=None) -> torch.Tensor:
    n = nsa_workspace_size(p)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device or "cuda")


def alloc_saved(p: Params, dev) -> dict:
    s, dt = _shapes(p), p.torch_dtype
    saved = {"kc": torch.empty(s["kc"], dtype=dt, device=dev),
             "vc": torch.empty(s["kc"], dtype=dt, device=dev),
             "o_cmp": torch.zeros(s["o"], dtype=dt, device=dev),
             "lse_cmp": torch.zeros(s["lse"], dtype=torch.float32, device=dev),
             "score": torch.zeros(s["score"], dtype=torch.float32, device=dev),
             "idx": torch.zeros(s["idx"], dtype=torch.int32, device=dev),
             "o_sel": torch.zeros(s["o"], dtype=dt, device=dev),
             "lse_sel": torch.zeros(s["lse"], dtype=torch.float32, device=dev),
             "o_swa": torch.zeros(s["o"], dtype=dt, device=dev),
             "lse_swa": torch.zeros(s["lse"], dtype=torch.float32, device=dev)}
    return {k_: t for k_, t in saved.items() if t.numel() > 0}


def forward(p: Params, q, k, v, gates, keep: bool = False, workspace=None, stream=None):
    """Allocate outputs with torch and run nsa_forward.

    Returns out, or (out, saved-dict) with every intermediate when keep=True.
    """
    dev = q.device
    out = torch.empty(_shapes(p)["o"], dtype=p.torch_dtype, device=dev)
    saved = alloc_saved(p, dev) if keep else None
    if workspace is None:
        workspace = alloc_workspace(p, dev)
    nsa_forward(p, q, k, v, gates, out, saved, workspace, stream)
    return (out, saved) if keep else out


def forward_mlp(p: Params, q, k, v, wk, wv, gates, keep: bool = False, workspace=None,
                stream=None):
    """forward() with the parametric compressor (nsa_forward_mlp)."""
    dev = q.device
    out = torch.empty(_shapes(p)["o"], dtype=p.torch_dtype, device=dev)
    saved = alloc_saved(p, dev) if keep else None
    if workspace is None:
        workspace = torch.empty(max(nsa_forward_mlp_workspace_size(p), 1), dtype=torch.uint8,
                                device=dev)
    nsa_forward_mlp(p, q, k, v, wk, wv, gates, out, saved, workspace, stream)
    return (out, saved) if keep else out


def backward_mlp(p: Params, q, k, v, wk, wv, gates, dout, saved: dict, workspace=None,
                 stream=None):
    """Allocate fp32 gradients with torch and run nsa_backward_mlp:
    (dq, dk, dv, dwk, dwv, dgates)."""
    s, dev = _shapes(p), q.device
    f = torch.float32
    dq = torch.empty(s["q"], dtype=f, device=dev)
    dk = torch.empty(s["k"], dtype=f, device=dev)
    dv = torch.empty(s["k"], dtype=f, device=dev)
    dwk = torch.empty(_w_shape(p), dtype=f, device=dev)
    dwv = torch.empty(_w_shape(p), dtype=f, device=dev)
    dg = torch.empty(s["gates"], dtype=f, device=dev)
    if workspace is None:
        workspace = torch.empty(max(nsa_backward_mlp_workspace_size(p), 1), dtype=torch.uint8,
                                device=dev)
    nsa_backward_mlp(p, q, k, v, wk, wv, gates, dout, saved, dq, dk, dv, dwk, dwv, dg,
                     workspace, stream)
    return dq, dk, dv, dwk, dwv, dg


# ------------------------------------------------------------------ MoBA
def nsa_moba_workspace_size(p: MobaParams) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_moba_workspace_size(C.byref(p), C.byref(n)), "nsa_moba_workspace_size")
    return n.value


def _moba_shapes(p: MobaParams) -> dict:
    return {"q": (p.B, p.Tq, p.Hq, p.D), "k": (p.B, p.T, p.Hkv, p.D),
            "lse": (p.B, p.Tq, p.Hq), "idx": (p.B, p.Tq, p.Hkv, p.topk)}


def nsa_moba_forward(p: MobaParams, q, k, v, out, lse=None, idx=None, workspace=None,
                     stream=None):
    s = _moba_shapes(p)
    dt = torch.bfloat16 if p.dtype == NSA_BF16 else torch.float32
    if workspace is None:
        workspace = torch.empty(max(nsa_moba_workspace_size(p), 1), dtype=torch.uint8,
                                device=q.device)
    _check(load().nsa_moba_forward(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(out, s["q"], dt, "out"), _ptr(lse, s["lse"], torch.float32, "lse", True),
        _ptr(idx, s["idx"], torch.int32, "idx", True), _ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "nsa_moba_forward")


def nsa_moba_backward(p: MobaParams, q, k, v, idx, out, lse, dout, dq, dk, dv, workspace=None,
                      stream=None):
    s = _moba_shapes(p)
    dt = torch.bfloat16 if p.dtype == NSA_BF16 else torch.float32
    f = torch.float32
    if workspace is None:
        workspace = torch.empty(max(nsa_moba_workspace_size(p), 1), dtype=torch.uint8,
                                device=q.device)
    _check(load().nsa_moba_backward(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(idx, s["idx"], torch.int32, "idx"), _ptr(out, s["q"], dt, "out"),
        _ptr(lse, s["lse"], f, "lse"), _ptr(dout, s["q"], f, "dout"), _ptr(dq, s["q"], f, "dq"),
        _ptr(dk, s["k"], f, "dk"), _ptr(dv, s["k"], f, "dv"), _ptr(workspace, name="workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "nsa_moba_backward")


# ------------------------------------------------------------------ parametric compression
def _w_shape(p: Params):
    return (p.cmp_block * p.D, p.D)


def nsa_compress_mlp_workspace_size(p: Params) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_compress_mlp_workspace_size(C.byref(p), C.byref(n)),
           "nsa_compress_mlp_workspace_size")
    return n.value


def nsa_compress_mlp(p: Params, k, v, wk, wv, kc, vc, workspace=None, stream=None):
    """workspace: None allocates nsa_compress_mlp_workspace_size(p) bytes."""
    s, dt = _shapes(p), p.torch_dtype
    if workspace is None:
        n = nsa_compress_mlp_workspace_size(p)
        workspace = torch.empty(n, dtype=torch.uint8, device=k.device) if n else None
    wp, wb = _ws(workspace)
    _check(load().nsa_compress_mlp(
        C.byref(p), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(wk, _w_shape(p), dt, "wk"), _ptr(wv, _w_shape(p), dt, "wv"),
        _ptr(kc, s["kc"], dt, "kc", p.Nc == 0), _ptr(vc, s["kc"], dt, "vc", p.Nc == 0),
        wp, wb, _stream(stream)), "nsa_compress_mlp")


def nsa_compress_mlp_bwd_workspace_size(p: Params) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_compress_mlp_bwd_workspace_size(C.byref(p), C.byref(n)),
           "nsa_compress_mlp_bwd_workspace_size")
    return n.value


def nsa_compress_mlp_bwd(p: Params, k, v, wk, wv, dkc, dvc, dk, dv, dwk, dwv, workspace,
                         stream=None):
    s, dt, f = _shapes(p), p.torch_dtype, torch.float32
    wp, wb = _ws(workspace)
    _check(load().nsa_compress_mlp_bwd(
        C.byref(p), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(wk, _w_shape(p), dt, "wk"), _ptr(wv, _w_shape(p), dt, "wv"),
        _ptr(dkc, s["kc"], f, "dkc", p.Nc == 0), _ptr(dvc, s["kc"], f, "dvc", p.Nc == 0),
        _ptr(dk, s["k"], f, "dk"), _ptr(dv, s["k"], f, "dv"),
        _ptr(dwk, _w_shape(p), f, "dwk"), _ptr(dwv, _w_shape(p), f, "dwv"), wp, wb,
        _stream(stream)), "nsa_compress_mlp_bwd")


def _saved_struct(p: Params, saved: dict | None) -> "Saved":
    s, dt = _shapes(p), p.torch_dtype
    sv = Saved()
    if saved:
        want = {"kc": (s["kc"], dt), "vc": (s["kc"], dt), "o_cmp": (s["o"], dt),
                "lse_cmp": (s["lse"], torch.float32), "score": (s["score"], torch.float32),
                "idx": (s["idx"], torch.int32), "o_sel": (s["o"], dt),
                "lse_sel": (s["lse"], torch.float32), "o_swa": (s["o"], dt),
                "lse_swa": (s["lse"], torch.float32)}
        for name, t in saved.items():
            if t is None or t.numel() == 0:
                continue
            shp, tdt = want[name]
            setattr(sv, name, _ptr(t, shp, tdt, name).value)
    return sv


def nsa_forward_mlp_workspace_size(p: Params) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_forward_mlp_workspace_size(C.byref(p), C.byref(n)),
           "nsa_forward_mlp_workspace_size")
    return n.value


def nsa_forward_mlp(p: Params, q, k, v, wk, wv, gates, out, saved: dict | None = None,
                    workspace=None, stream=None):
    """nsa_forward with the parametric compressor (weights wk, wv [l D, D])."""
    s, dt = _shapes(p), p.torch_dtype
    sv = _saved_struct(p, saved)
    wp, wb = _ws(workspace)
    _check(load().nsa_forward_mlp(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(wk, _w_shape(p), dt, "wk"), _ptr(wv, _w_shape(p), dt, "wv"),
        _ptr(gates, s["gates"], torch.float32, "gates"), _ptr(out, s["o"], dt, "out"),
        C.byref(sv), wp, wb, _stream(stream)), "nsa_forward_mlp")


def nsa_backward_mlp_workspace_size(p: Params) -> int:
    n = C.c_size_t(0)
    _check(load().nsa_backward_mlp_workspace_size(C.byref(p), C.byref(n)),
           "nsa_backward_mlp_workspace_size")
    return n.value


def nsa_backward_mlp(p: Params, q, k, v, wk, wv, gates, dout, saved: dict, dq, dk, dv, dwk,
                     dwv, dgates, workspace, stream=None):
    s, dt, f = _shapes(p), p.torch_dtype, torch.float32
    sv = Saved()
    for name, t in saved.items():
        if t is not None and t.numel() > 0:
            setattr(sv, name, _ptr(t, name=name).value)
    wp, wb = _ws(workspace)
    _check(load().nsa_backward_mlp(
        C.byref(p), _ptr(q, s["q"], dt, "q"), _ptr(k, s["k"], dt, "k"), _ptr(v, s["k"], dt, "v"),
        _ptr(wk, _w_shape(p), dt, "wk"), _ptr(wv, _w_shape(p), dt, "wv"),
        _ptr(gates, s["gates"], f, "gates"), _ptr(dout, s["o"], dt, "dout"), C.byref(sv),
        _ptr(dq, s["q"], f, "dq"), _ptr(dk, s["k"], f, "dk"), _ptr(dv, s["k"], f, "dv"),
        _ptr(dwk, _w_shape(p), f, "dwk"), _ptr(dwv, _w_shape(p), f, "dwv"),
        _ptr(dgates, s["gates"], f, "dgates"), wp, wb, _stream(stream)), "nsa_backward_mlp")
