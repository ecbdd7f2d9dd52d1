"""Seeded synthetic workloads for the NSA hot path.

This module describes problem shapes and draws input tensors.  It holds
none of the method's arithmetic, so both the CUDA library's tests/bench and
the fp64 oracle can take their inputs from it.

The shapes follow the pages' training setups ("Sparsity is Cool:
Reverse-Engineering MoBA and NSA", Method: 340M and 1.3B transformer++
models with QK-Norm, 8192-token sequences, GQA-4 / MQA, NSA with block 64,
top-k 16, window 512, mean-pool compression).  The pages' datasets
(SlimPajama, PG-19, GovReport) are not available; seeded Gaussian tensors of
the same shapes stand in for the activations, as described per workload.

All tensors are drawn on the CPU from ``torch.Generator().manual_seed(seed)``
in a fixed order, then rounded once to the workload dtype, so every consumer
sees identical values.
"""
from __future__ import annotations

import dataclasses
import math

import torch

BR_CMP, BR_SEL, BR_SWA = 1, 2, 4
BR_ALL = BR_CMP | BR_SEL | BR_SWA


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int
    cmp_block: int
    cmp_stride: int
    sel_block: int
    topk: int
    window: int
    dtype: torch.dtype
    branch_mask: int = BR_ALL
    qk_norm: bool = False       # unit-RMS q/k rows (QK-Norm)
    qkv_std: float = 1.0        # scale of the N(0,1) draws
    gate_dist: str = "sigmoid"  # "sigmoid": sigmoid(N(0,1)); "uniform": U(0,1)
    cmp_gate_zero: bool = False  # compression gate fixed at 0 (pruned branch)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def Nc(self) -> int:
        if self.T < self.cmp_block:
            return 0
        return (self.T - self.cmp_block) // self.cmp_stride + 1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the study, named by what they are.
TINY_F32 = Workload("tiny_mqa_t256_f32", B=1, T=256, Hq=4, Hkv=1, D=64,
                    cmp_block=32, cmp_stride=32, sel_block=32, topk=4, window=64,
                    dtype=torch.float32, qkv_std=1.0 / 8.0, gate_dist="uniform")
NSA_340M = Workload("nsa_340m_gqa4_t8192_bf16", B=1, T=8192, Hq=16, Hkv=4, D=64,
                    cmp_block=64, cmp_stride=64, sel_block=64, topk=16, window=512,
                    dtype=torch.bfloat16, qk_norm=True)
NSA_1P3B = Workload("nsa_1p3b_gqa4_b4_t8192_bf16", B=4, T=8192, Hq=32, Hkv=8, D=64,
                    cmp_block=64, cmp_stride=64, sel_block=64, topk=16, window=512,
                    dtype=torch.bfloat16, qk_norm=True)
PRUNED_32K = Workload("nsa_pruned_mqa_t32768_bf16", B=1, T=32768, Hq=16, Hkv=1, D=64,
                      cmp_block=64, cmp_stride=64, sel_block=64, topk=16, window=512,
                      dtype=torch.bfloat16, branch_mask=BR_SEL | BR_SWA,
                      cmp_gate_zero=True)
DECODE_32K = Workload("nsa_decode_mqa_b64_cache32768_bf16", B=64, T=32768, Hq=16,
                      Hkv=1, D=64, cmp_block=64, cmp_stride=64, sel_block=64,
                      topk=16, window=512, dtype=torch.bfloat16)
TRAIN_340M = Workload("nsa_train_340m_gqa4_b8_t8192_bf16", B=8, T=8192, Hq=16, Hkv=4,
                      D=64, cmp_block=64, cmp_stride=64, sel_block=64, topk=16,
                      window=512, dtype=torch.bfloat16, qk_norm=True)

WORKLOADS = {w.name: w for w in (TINY_F32, NSA_340M, NSA_1P3B, PRUNED_32K,
                                 DECODE_32K, TRAIN_340M)}


def _unit_rms(x: torch.Tensor) -> torch.Tensor:
    # input preparation only: rescale each head row to unit RMS, as a
    # QK-Norm layer would leave it before attention
    return x / x.pow(2).mean(dim=-1, keepdim=True).sqrt()


def make_inputs(w: Workload, seed: int = 0, with_dout: bool = False) -> dict:
    """Draw q, k, v, gates (and dout) for a prefill workload, on the CPU.

    q [B,T,Hq,D], k/v [B,T,Hkv,D] in w.dtype; gates [B,T,Hq,3] float32 in
    branch order (cmp, sel, swa); dout [B,T,Hq,D] in w.dtype.
    """
    g = torch.Generator().manual_seed(seed)
    B, T, Hq, Hkv, D = w.B, w.T, w.Hq, w.Hkv, w.D
    q = torch.randn((B, T, Hq, D), generator=g, dtype=torch.float32)
    k = torch.randn((B, T, Hkv, D), generator=g, dtype=torch.float32)
    v = torch.randn((B, T, Hkv, D), generator=g, dtype=torch.float32)
    if w.qk_norm:
        q, k = _unit_rms(q), _unit_rms(k)
    q, k, v = q * w.qkv_std, k * w.qkv_std, v * w.qkv_std
    if w.gate_dist == "uniform":
        gates = torch.rand((B, T, Hq, 3), generator=g, dtype=torch.float32)
    else:
        gates = torch.sigmoid(torch.randn((B, T, Hq, 3), generator=g,
                                          dtype=torch.float32))
    if w.cmp_gate_zero:
        gates[..., 0] = 0.0
    out = {"q": q.to(w.dtype), "k": k.to(w.dtype), "v": v.to(w.dtype),
           "gates": gates.contiguous()}
    if with_dout:
        out["dout"] = torch.randn((B, T, Hq, D), generator=g,
                                  dtype=torch.float32).to(w.dtype)
    return out


def make_mlp_weights(w: Workload, seed: int = 0) -> tuple:
    """Draw the parametric compressor's weights wk, wv [cmp_block * D, D] in
    w.dtype: Gaussian with variance 1 / (cmp_block * D), the usual fan-in
    initialisation of a linear layer (the pages train theirs; no trained
    weights exist here)."""
    g = torch.Generator().manual_seed(seed)
    fan_in = w.cmp_block * w.D
    std = 1.0 / math.sqrt(fan_in)
    wk = torch.randn((fan_in, w.D), generator=g, dtype=torch.float32) * std
    wv = torch.randn((fan_in, w.D), generator=g, dtype=torch.float32) * std
    return wk.to(w.dtype), wv.to(w.dtype)


def make_decode_inputs(w: Workload, seed: int = 0) -> dict:
    """Draw one decode step: the query of position T-1 of each sequence and
    caches of T keys/values that already hold that position.

    q [B,Hq,D], k_cache/v_cache [B,T,Hkv,D] in w.dtype, gates [B,Hq,3] fp32.
    The compressed cache is not drawn: it is the mean-pool of k_cache/v_cache
    and is produced by the library's own compression call.
    """
    g = torch.Generator().manual_seed(seed)
    B, T, Hq, Hkv, D = w.B, w.T, w.Hq, w.Hkv, w.D
    q = torch.randn((B, Hq, D), generator=g, dtype=torch.float32)
    kc = torch.randn((B, T, Hkv, D), generator=g, dtype=torch.float32)
    vc = torch.randn((B, T, Hkv, D), generator=g, dtype=torch.float32)
    if w.qk_norm:
        q, kc = _unit_rms(q), _unit_rms(kc)
    gates = torch.sigmoid(torch.randn((B, Hq, 3), generator=g, dtype=torch.float32))
    if w.cmp_gate_zero:
        gates[..., 0] = 0.0
    return {"q": (q * w.qkv_std).to(w.dtype), "k_cache": (kc * w.qkv_std).to(w.dtype),
            "v_cache": (vc * w.qkv_std).to(w.dtype), "gates": gates.contiguous()}
