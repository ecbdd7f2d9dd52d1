"""B200-native Native Sparse Attention (NSA).

The compute path is libnsa.so (C ABI in include/nsa.h): hand-written sm_100a
CUDA kernels for mean-pool compression, the compression branch with block
scores, per-KV-group top-k selection, selection and sliding-window
attention, the gated combination, the whole forward and decode, the
backward of every branch, the parametric (linear-layer) compressor with its
gradient, and MoBA block attention on the selection kernels.  This package is its thin ctypes binding (``abi``) plus seeded
synthetic workloads (``inputs``).  Build the library with ``python -m sparse_attention_nsa_b200.build``.
"""
from .abi import (EXPORTS, backward, nsa_backward, nsa_backward_workspace_size,
                  nsa_cmp_bwd, nsa_gate_combine_bwd, nsa_sel_attn_bwd, nsa_sel_attn_bwd_atomic,
                  nsa_swa_bwd, NSA_BF16, NSA_BRANCH_ALL, NSA_BRANCH_CMP, NSA_BRANCH_SEL,
                  NSA_BRANCH_SWA, NSA_F32, NsaError, Params, Saved, alloc_workspace,
                  forward, load, make_params, nsa_check_params, nsa_cmp_attn_scores,
                  nsa_forward_host, nsa_forward_host_workspace_size,
                  nsa_compress, nsa_decode, nsa_decode_noalloc,
                  nsa_decode_noalloc_max_scratch, nsa_forward, nsa_gate_combine,
                  nsa_last_device_error, nsa_sel_attn_fwd, nsa_sel_attn_fwd_ws,
                  nsa_sel_workspace_size, nsa_select_topk, nsa_set_kernel_events,
                  nsa_status_string, nsa_swa_fwd, nsa_workspace_size, params_for,
                  MobaParams, make_moba_params, nsa_moba_backward, nsa_moba_forward,
                  nsa_moba_workspace_size, nsa_backward_mlp, nsa_backward_mlp_workspace_size,
                  nsa_compress_mlp, nsa_compress_mlp_bwd, nsa_compress_mlp_bwd_workspace_size,
                  nsa_forward_mlp, forward_mlp, backward_mlp, alloc_saved,
                  nsa_compress_mlp_workspace_size, nsa_forward_mlp_workspace_size)

__all__ = [n for n in dir() if not n.startswith("_")]
