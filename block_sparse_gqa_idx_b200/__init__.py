"""MiniMax Sparse Attention (MSA) forward path for B200 (sm_100a).

The compute lives in ``libmsa_b200.so`` (hand-written CUDA behind the C ABI
of ``include/msa.h``); this package is its thin Python binding:

* ``index_topk``      Index Branch, Eq. 6-7 (fused scores, block max, Top-k)
* ``sparse_attn_fwd`` Main Branch, Eq. 8 (KV-outer sparse attention + merge)
* ``forward``         both, for one prefill sequence
* ``forward_varlen``  both, for a packed batch of sequences of any lengths
* ``project``         the Q, K, V and index projections upstream of the path
* ``sparse_attn_bwd`` the backward of the Main Branch (dQ, dK, dV)
* ``sparse_decode``   one decode step for a batch of sequences
* ``paged_decode_fp8`` the same step on a paged FP8 (E4M3) KV cache

``inputs`` holds the seeded synthetic workload generators.  The binding is
loaded on first use of one of the names above and raises if the CUDA library
has not been built (``python -m block_sparse_gqa_idx_b200.build``).
"""
_CAPI = ("index_topk", "sparse_attn_fwd", "forward", "sparse_decode", "device_status",
         "version", "MSAError", "dims", "decode_dims", "index_topk_workspace_size",
         "sparse_attn_fwd_workspace_size", "sparse_decode_workspace_size", "EXPORTS", "LIB_PATH",
         "profile_enable", "profile_read", "sparse_decode_noalloc", "selftest_bounded_wait",
         "index_lse", "index_lse_workspace_size", "paged_dims", "paged_decode_fp8",
         "paged_decode_fp8_workspace_size", "quantize_fp8_rows", "index_topk_varlen",
         "sparse_attn_fwd_varlen", "forward_varlen", "varlen_dims", "project",
         "varlen_workspace_size", "sparse_attn_bwd",
         "sparse_attn_bwd_workspace_size")

__all__ = list(_CAPI) + ["inputs"]


def __getattr__(name):
    if name in _CAPI:
        from . import _capi

        return getattr(_capi, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
