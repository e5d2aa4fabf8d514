"""ctypes binding of ``include/msa.h`` (libmsa_b200.so).

Argument marshalling only: every step of the MSA path runs in the CUDA
library.  Tensors are torch CUDA tensors (PyTorch provides device memory and
streams); the binding checks dtype, shape, device and contiguity, allocates
outputs/workspaces with torch when the caller does not pass them, and passes
raw pointers plus the current CUDA stream.  If the library is missing this
module raises at import: there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa_b200.so")


class MSAError(RuntimeError):
    def __init__(self, what: str, status: int, text: str):
        super().__init__(f"{what}: {text} (status {status})")
        self.status = status


class msa_dims(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("H_q", ctypes.c_int32), ("H_kv", ctypes.c_int32),
                ("d_h", ctypes.c_int32), ("d_idx", ctypes.c_int32), ("B_k", ctypes.c_int32),
                ("k", ctypes.c_int32), ("attn_scale", ctypes.c_float),
                ("idx_scale", ctypes.c_float)]


class msa_decode_dims(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int32), ("L_max", ctypes.c_int64), ("H_q", ctypes.c_int32),
                ("H_kv", ctypes.c_int32), ("d_h", ctypes.c_int32), ("d_idx", ctypes.c_int32),
                ("B_k", ctypes.c_int32), ("k", ctypes.c_int32), ("attn_scale", ctypes.c_float),
                ("idx_scale", ctypes.c_float)]


class msa_paged_dims(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int32), ("max_pages", ctypes.c_int32), ("n_pages", ctypes.c_int64),
                ("H_q", ctypes.c_int32), ("H_kv", ctypes.c_int32), ("d_h", ctypes.c_int32),
                ("d_idx", ctypes.c_int32), ("B_k", ctypes.c_int32), ("k", ctypes.c_int32),
                ("attn_scale", ctypes.c_float), ("idx_scale", ctypes.c_float)]


class msa_varlen_dims(ctypes.Structure):
    _fields_ = [("n_seqs", ctypes.c_int32), ("N", ctypes.c_int64), ("H_q", ctypes.c_int32),
                ("H_kv", ctypes.c_int32), ("d_h", ctypes.c_int32), ("d_idx", ctypes.c_int32),
                ("B_k", ctypes.c_int32), ("k", ctypes.c_int32), ("attn_scale", ctypes.c_float),
                ("idx_scale", ctypes.c_float)]


class msa_proj_dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d_model", ctypes.c_int32), ("H_q", ctypes.c_int32),
                ("H_kv", ctypes.c_int32), ("d_h", ctypes.c_int32), ("d_idx", ctypes.c_int32)]


class msa_kernel_time(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int32),
                ("total_ms", ctypes.c_double)]


# every symbol include/msa.h declares
EXPORTS = ("msa_index_topk_workspace", "msa_index_topk", "msa_sparse_attn_fwd_workspace",
           "msa_sparse_attn_fwd", "msa_sparse_decode_workspace", "msa_sparse_decode",
           "msa_get_device_status", "msa_profile_enable", "msa_profile_read",
           "msa_status_string", "msa_version", "msa_sparse_decode_noalloc", "msa_last_error",
           "msa_selftest_bounded_wait", "msa_index_lse_workspace", "msa_index_lse",
           "msa_paged_decode_fp8_workspace", "msa_paged_decode_fp8", "msa_quantize_fp8_rows",
           "msa_index_topk_varlen_workspace", "msa_index_topk_varlen",
           "msa_sparse_attn_fwd_varlen_workspace", "msa_sparse_attn_fwd_varlen",
           "msa_project_workspace", "msa_project", "msa_sparse_attn_bwd_workspace",
           "msa_sparse_attn_bwd")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build the CUDA library first "
            "(python -m block_sparse_gqa_idx_b200.build); there is no fallback path")
    lib = ctypes.CDLL(LIB_PATH)
    P, Z, I32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    D, DD = ctypes.POINTER(msa_dims), ctypes.POINTER(msa_decode_dims)
    lib.msa_index_topk_workspace.argtypes = [D]
    lib.msa_index_topk_workspace.restype = Z
    lib.msa_index_topk.argtypes = [D, P, P, P, P, P, Z, P]
    lib.msa_index_topk.restype = I32
    lib.msa_sparse_attn_fwd_workspace.argtypes = [D]
    lib.msa_sparse_attn_fwd_workspace.restype = Z
    lib.msa_sparse_attn_fwd.argtypes = [D, P, P, P, P, P, P, P, Z, P]
    lib.msa_sparse_attn_fwd.restype = I32
    lib.msa_sparse_decode_workspace.argtypes = [DD]
    lib.msa_sparse_decode_workspace.restype = Z
    lib.msa_sparse_decode.argtypes = [DD] + [P] * 12 + [Z, P]
    lib.msa_sparse_decode.restype = I32
    lib.msa_sparse_decode_noalloc.argtypes = [DD] + [P] * 11 + [P]
    lib.msa_sparse_decode_noalloc.restype = I32
    lib.msa_get_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32),
                                          ctypes.POINTER(ctypes.c_int32)]
    lib.msa_get_device_status.restype = I32
    lib.msa_index_lse_workspace.argtypes = [D]
    lib.msa_index_lse_workspace.restype = Z
    lib.msa_index_lse.argtypes = [D, P, P, P, P, P, Z, P]
    lib.msa_index_lse.restype = I32
    PD = ctypes.POINTER(msa_paged_dims)
    lib.msa_paged_decode_fp8_workspace.argtypes = [PD]
    lib.msa_paged_decode_fp8_workspace.restype = Z
    lib.msa_paged_decode_fp8.argtypes = [PD] + [P] * 15 + [P, Z, P]
    lib.msa_paged_decode_fp8.restype = I32
    lib.msa_quantize_fp8_rows.argtypes = [P, ctypes.c_int64, I32, P, P, P]
    lib.msa_quantize_fp8_rows.restype = I32
    VD, CU = ctypes.POINTER(msa_varlen_dims), ctypes.POINTER(ctypes.c_int64)
    lib.msa_index_topk_varlen_workspace.argtypes = [VD, CU]
    lib.msa_index_topk_varlen_workspace.restype = Z
    lib.msa_index_topk_varlen.argtypes = [VD, CU, P, P, P, P, P, Z, P]
    lib.msa_index_topk_varlen.restype = I32
    lib.msa_sparse_attn_fwd_varlen_workspace.argtypes = [VD, CU]
    lib.msa_sparse_attn_fwd_varlen_workspace.restype = Z
    lib.msa_sparse_attn_fwd_varlen.argtypes = [VD, CU, P, P, P, P, P, P, P, Z, P]
    lib.msa_sparse_attn_fwd_varlen.restype = I32
    lib.msa_sparse_attn_bwd_workspace.argtypes = [D]
    lib.msa_sparse_attn_bwd_workspace.restype = Z
    lib.msa_sparse_attn_bwd.argtypes = [D] + [P] * 11 + [Z, P]
    lib.msa_sparse_attn_bwd.restype = I32
    PJ = ctypes.POINTER(msa_proj_dims)
    lib.msa_project_workspace.argtypes = [PJ]
    lib.msa_project_workspace.restype = Z
    lib.msa_project.argtypes = [PJ] + [P] * 12 + [Z, P]
    lib.msa_project.restype = I32
    lib.msa_selftest_bounded_wait.argtypes = [P, P]
    lib.msa_selftest_bounded_wait.restype = I32
    lib.msa_profile_enable.argtypes = [ctypes.c_int32]
    lib.msa_profile_enable.restype = I32
    lib.msa_profile_read.argtypes = [ctypes.POINTER(msa_kernel_time), ctypes.c_int32]
    lib.msa_profile_read.restype = ctypes.c_int32
    lib.msa_status_string.argtypes = [I32]
    lib.msa_status_string.restype = ctypes.c_char_p
    lib.msa_last_error.argtypes = []
    lib.msa_last_error.restype = ctypes.c_char_p
    lib.msa_version.argtypes = []
    lib.msa_version.restype = ctypes.c_char_p
    return lib


LIB = _load()


def version() -> str:
    return LIB.msa_version().decode()


def _raise(what: str, st: int) -> None:
    if st != 0:
        text = LIB.msa_status_string(st).decode()
        if st == 4:
            text += ": " + LIB.msa_last_error().decode()
        raise MSAError(what, st, text)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _want(t: torch.Tensor, name: str, dtype, shape) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def dims(N, H_q, H_kv, d_h, d_idx, B_k, k, attn_scale=0.0, idx_scale=0.0) -> msa_dims:
    return msa_dims(int(N), int(H_q), int(H_kv), int(d_h), int(d_idx), int(B_k), int(k),
                    float(attn_scale), float(idx_scale))


def decode_dims(S, L_max, H_q, H_kv, d_h, d_idx, B_k, k, attn_scale=0.0,
                idx_scale=0.0) -> msa_decode_dims:
    return msa_decode_dims(int(S), int(L_max), int(H_q), int(H_kv), int(d_h), int(d_idx),
                           int(B_k), int(k), float(attn_scale), float(idx_scale))


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is None:
        return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    if ws.dtype != torch.uint8 or not ws.is_cuda or ws.numel() < nbytes:
        raise ValueError(f"workspace must be a CUDA uint8 tensor of >= {nbytes} bytes")
    return ws


def index_topk_workspace_size(d: msa_dims) -> int:
    return int(LIB.msa_index_topk_workspace(ctypes.byref(d)))


def sparse_attn_fwd_workspace_size(d: msa_dims) -> int:
    return int(LIB.msa_sparse_attn_fwd_workspace(ctypes.byref(d)))


def sparse_decode_workspace_size(d: msa_decode_dims) -> int:
    return int(LIB.msa_sparse_decode_workspace(ctypes.byref(d)))


def index_topk(q_idx: torch.Tensor, k_idx: torch.Tensor, B_k: int, k: int,
               idx_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None, score_out: Optional[torch.Tensor] = None,
               idx_scale: float = 0.0) -> torch.Tensor:
    """Eq. 6-7: q_idx [N,H_kv,d_idx] bf16, k_idx [N,d_idx] bf16 -> idx [N,H_kv,k] int32.
    If ``score_out`` ([N,H_kv,k] fp32) is given, it receives each selected
    block's Eq. 6 score (scale ``idx_scale``, 0 -> 1/sqrt(d_idx)), -inf in -1 slots."""
    N, H_kv, d_idx = q_idx.shape
    _want(q_idx, "q_idx", torch.bfloat16, (N, H_kv, d_idx))
    _want(k_idx, "k_idx", torch.bfloat16, (N, d_idx))
    if idx_out is None:
        idx_out = torch.empty((N, H_kv, k), dtype=torch.int32, device=q_idx.device)
    _want(idx_out, "idx_out", torch.int32, (N, H_kv, k))
    if score_out is not None:
        _want(score_out, "score_out", torch.float32, (N, H_kv, k))
    d = dims(N, H_kv, H_kv, 64, d_idx, B_k, k, idx_scale=idx_scale)
    ws = _workspace(index_topk_workspace_size(d), q_idx.device, workspace)
    _raise("msa_index_topk", LIB.msa_index_topk(ctypes.byref(d), _ptr(q_idx), _ptr(k_idx),
                                                _ptr(idx_out), _ptr(score_out), _ptr(ws),
                                                ws.numel(), _stream(stream)))
    return idx_out


def index_lse_workspace_size(d: msa_dims) -> int:
    return int(LIB.msa_index_lse_workspace(ctypes.byref(d)))


def index_lse(q_idx: torch.Tensor, k_idx: torch.Tensor, idx: torch.Tensor, B_k: int,
              lse_idx: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    """KL-loss fusion: LSE_idx [N,H_kv] fp32 = log of the sum of exp(S^idx)
    over each row's selected tokens j <= i (Eq. 9's Index Branch normaliser).
    q_idx [N,H_kv,d_idx] bf16, k_idx [N,d_idx] bf16, idx [N,H_kv,k] int32."""
    N, H_kv, d_idx = q_idx.shape
    k = idx.shape[2]
    _want(q_idx, "q_idx", torch.bfloat16, (N, H_kv, d_idx))
    _want(k_idx, "k_idx", torch.bfloat16, (N, d_idx))
    _want(idx, "idx", torch.int32, (N, H_kv, k))
    if lse_idx is None:
        lse_idx = torch.empty((N, H_kv), dtype=torch.float32, device=q_idx.device)
    _want(lse_idx, "lse_idx", torch.float32, (N, H_kv))
    d = dims(N, H_kv, H_kv, 64, d_idx, B_k, k)
    ws = _workspace(index_lse_workspace_size(d), q_idx.device, workspace)
    _raise("msa_index_lse", LIB.msa_index_lse(ctypes.byref(d), _ptr(q_idx), _ptr(k_idx),
                                              _ptr(idx), _ptr(lse_idx), _ptr(ws), ws.numel(),
                                              _stream(stream)))
    return lse_idx


def sparse_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
                    B_k: int, attn_scale: float = 0.0, o: Optional[torch.Tensor] = None,
                    lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                    workspace: Optional[torch.Tensor] = None, stream=None
                    ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Eq. 8: q [N,H_q,d_h], k/v [N,H_kv,d_h] bf16, idx [N,H_kv,kk] int32 ->
    o [N,H_q,d_h] bf16 and lse [N,H_q] fp32."""
    N, H_q, d_h = q.shape
    H_kv = k.shape[1]
    kk = idx.shape[2]
    _want(q, "q", torch.bfloat16, (N, H_q, d_h))
    _want(k, "k", torch.bfloat16, (N, H_kv, d_h))
    _want(v, "v", torch.bfloat16, (N, H_kv, d_h))
    _want(idx, "idx", torch.int32, (N, H_kv, kk))
    if o is None:
        o = torch.empty((N, H_q, d_h), dtype=torch.bfloat16, device=q.device)
    _want(o, "o", torch.bfloat16, (N, H_q, d_h))
    if lse is None and want_lse:
        lse = torch.empty((N, H_q), dtype=torch.float32, device=q.device)
    if lse is not None:
        _want(lse, "lse", torch.float32, (N, H_q))
    d = dims(N, H_q, H_kv, d_h, 64, B_k, kk, attn_scale)
    ws = _workspace(sparse_attn_fwd_workspace_size(d), q.device, workspace)
    _raise("msa_sparse_attn_fwd",
           LIB.msa_sparse_attn_fwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o),
                                   _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return o, lse


def sparse_attn_bwd_workspace_size(d: msa_dims) -> int:
    return int(LIB.msa_sparse_attn_bwd_workspace(ctypes.byref(d)))


def sparse_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
                    o: torch.Tensor, lse: torch.Tensor, d_o: torch.Tensor, B_k: int,
                    attn_scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Backward of Eq. 8 with the selection fixed: (dq, dk, dv) bf16 from the
    forward's o [N,H_q,d_h], lse [N,H_q] and d_o [N,H_q,d_h]."""
    N, H_q, d_h = q.shape
    H_kv = k.shape[1]
    kk = idx.shape[2]
    for t, name, dt, sh in ((q, "q", torch.bfloat16, (N, H_q, d_h)),
                            (k, "k", torch.bfloat16, (N, H_kv, d_h)),
                            (v, "v", torch.bfloat16, (N, H_kv, d_h)),
                            (idx, "idx", torch.int32, (N, H_kv, kk)),
                            (o, "o", torch.bfloat16, (N, H_q, d_h)),
                            (lse, "lse", torch.float32, (N, H_q)),
                            (d_o, "d_o", torch.bfloat16, (N, H_q, d_h))):
        _want(t, name, dt, sh)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    d = dims(N, H_q, H_kv, d_h, 64, B_k, kk, attn_scale)
    ws = _workspace(int(LIB.msa_sparse_attn_bwd_workspace(ctypes.byref(d))), q.device, workspace)
    _raise("msa_sparse_attn_bwd",
           LIB.msa_sparse_attn_bwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o),
                                   _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                   ws.numel(), _stream(stream)))
    return dq, dk, dv


def forward(q, k, v, q_idx, k_idx, B_k: int, kk: int, attn_scale: float = 0.0, stream=None,
            workspace: Optional[torch.Tensor] = None):
    """Whole MSA forward (Eq. 6-8): returns (o, lse, idx)."""
    idx = index_topk(q_idx, k_idx, B_k, kk, workspace=workspace, stream=stream)
    o, lse = sparse_attn_fwd(q, k, v, idx, B_k, attn_scale, workspace=workspace, stream=stream)
    return o, lse, idx


def project(x: torch.Tensor, w_q: torch.Tensor, w_k: torch.Tensor, w_v: torch.Tensor,
            w_qidx: torch.Tensor, w_kidx: torch.Tensor, H_q: int, H_kv: int,
            workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """The projections upstream of the path: x [T,d_model] bf16 and the five
    weights [d_model, out] bf16 -> q [T,H_q,d_h], k, v [T,H_kv,d_h], q_idx
    [T,H_kv,d_idx], k_idx [T,d_idx] (x W for each; the index branch's
    stopgrad(x) is x forward)."""
    T, d_model = x.shape
    d_h = w_q.shape[1] // H_q
    d_idx = w_kidx.shape[1]
    _want(x, "x", torch.bfloat16, (T, d_model))
    _want(w_q, "w_q", torch.bfloat16, (d_model, H_q * d_h))
    _want(w_k, "w_k", torch.bfloat16, (d_model, H_kv * d_h))
    _want(w_v, "w_v", torch.bfloat16, (d_model, H_kv * d_h))
    _want(w_qidx, "w_qidx", torch.bfloat16, (d_model, H_kv * d_idx))
    _want(w_kidx, "w_kidx", torch.bfloat16, (d_model, d_idx))
    dev = x.device
    out = {"q": torch.empty((T, H_q, d_h), dtype=torch.bfloat16, device=dev),
           "k": torch.empty((T, H_kv, d_h), dtype=torch.bfloat16, device=dev),
           "v": torch.empty((T, H_kv, d_h), dtype=torch.bfloat16, device=dev),
           "q_idx": torch.empty((T, H_kv, d_idx), dtype=torch.bfloat16, device=dev),
           "k_idx": torch.empty((T, d_idx), dtype=torch.bfloat16, device=dev)}
    d = msa_proj_dims(int(T), int(d_model), int(H_q), int(H_kv), int(d_h), int(d_idx))
    ws = _workspace(int(LIB.msa_project_workspace(ctypes.byref(d))), dev, workspace)
    _raise("msa_project",
           LIB.msa_project(ctypes.byref(d), _ptr(x), _ptr(w_q), _ptr(w_k), _ptr(w_v), _ptr(w_qidx),
                           _ptr(w_kidx), _ptr(out["q"]), _ptr(out["k"]), _ptr(out["v"]),
                           _ptr(out["q_idx"]), _ptr(out["k_idx"]), _ptr(ws), ws.numel(),
                           _stream(stream)))
    return out


def _cu(cu_seqlens, N: int):
    """cu_seqlens (a list, numpy array or CPU tensor of n + 1 ints) as a host
    int64 array for the C ABI, with the count of sequences."""
    vals = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist")
                             else cu_seqlens)]
    if len(vals) < 2 or vals[0] != 0 or vals[-1] != N:
        raise ValueError(f"cu_seqlens must run from 0 to N={N}")
    return (ctypes.c_int64 * len(vals))(*vals), len(vals) - 1


def varlen_dims(n_seqs, N, H_q, H_kv, d_h, d_idx, B_k, k, attn_scale=0.0,
                idx_scale=0.0) -> msa_varlen_dims:
    return msa_varlen_dims(int(n_seqs), int(N), int(H_q), int(H_kv), int(d_h), int(d_idx),
                           int(B_k), int(k), float(attn_scale), float(idx_scale))


def varlen_workspace_size(cu_seqlens, N, H_q, H_kv, d_h, d_idx, B_k, k) -> int:
    """Bytes of one workspace that serves both packed-batch calls."""
    cu, n = _cu(cu_seqlens, N)
    d = varlen_dims(n, N, H_q, H_kv, d_h, d_idx, B_k, k)
    return max(int(LIB.msa_index_topk_varlen_workspace(ctypes.byref(d), cu)),
               int(LIB.msa_sparse_attn_fwd_varlen_workspace(ctypes.byref(d), cu)))


def index_topk_varlen(q_idx: torch.Tensor, k_idx: torch.Tensor, cu_seqlens, B_k: int, k: int,
                      idx_out: Optional[torch.Tensor] = None,
                      score_out: Optional[torch.Tensor] = None, idx_scale: float = 0.0,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Eq. 6-7 per sequence of a packed batch: q_idx [N,H_kv,d_idx], k_idx
    [N,d_idx] bf16, sequence s = tokens cu_seqlens[s] .. cu_seqlens[s+1]-1 ->
    idx [N,H_kv,k] int32 with block indices local to each token's sequence."""
    N, H_kv, d_idx = q_idx.shape
    _want(q_idx, "q_idx", torch.bfloat16, (N, H_kv, d_idx))
    _want(k_idx, "k_idx", torch.bfloat16, (N, d_idx))
    if idx_out is None:
        idx_out = torch.empty((N, H_kv, k), dtype=torch.int32, device=q_idx.device)
    _want(idx_out, "idx_out", torch.int32, (N, H_kv, k))
    if score_out is not None:
        _want(score_out, "score_out", torch.float32, (N, H_kv, k))
    cu, n = _cu(cu_seqlens, N)
    d = varlen_dims(n, N, H_kv, H_kv, 64, d_idx, B_k, k, idx_scale=idx_scale)
    ws = _workspace(int(LIB.msa_index_topk_varlen_workspace(ctypes.byref(d), cu)), q_idx.device,
                    workspace)
    _raise("msa_index_topk_varlen",
           LIB.msa_index_topk_varlen(ctypes.byref(d), cu, _ptr(q_idx), _ptr(k_idx), _ptr(idx_out),
                                     _ptr(score_out), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out


def sparse_attn_fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                           idx: torch.Tensor, cu_seqlens, B_k: int, attn_scale: float = 0.0,
                           o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                           want_lse: bool = True, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Eq. 8 per sequence of a packed batch (idx local to each sequence):
    o [N,H_q,d_h] bf16 and lse [N,H_q] fp32."""
    N, H_q, d_h = q.shape
    H_kv = k.shape[1]
    kk = idx.shape[2]
    _want(q, "q", torch.bfloat16, (N, H_q, d_h))
    _want(k, "k", torch.bfloat16, (N, H_kv, d_h))
    _want(v, "v", torch.bfloat16, (N, H_kv, d_h))
    _want(idx, "idx", torch.int32, (N, H_kv, kk))
    if o is None:
        o = torch.empty((N, H_q, d_h), dtype=torch.bfloat16, device=q.device)
    _want(o, "o", torch.bfloat16, (N, H_q, d_h))
    if lse is None and want_lse:
        lse = torch.empty((N, H_q), dtype=torch.float32, device=q.device)
    if lse is not None:
        _want(lse, "lse", torch.float32, (N, H_q))
    cu, n = _cu(cu_seqlens, N)
    d = varlen_dims(n, N, H_q, H_kv, d_h, 64, B_k, kk, attn_scale)
    ws = _workspace(int(LIB.msa_sparse_attn_fwd_varlen_workspace(ctypes.byref(d), cu)), q.device,
                    workspace)
    _raise("msa_sparse_attn_fwd_varlen",
           LIB.msa_sparse_attn_fwd_varlen(ctypes.byref(d), cu, _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(idx), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                                          _stream(stream)))
    return o, lse


def forward_varlen(q, k, v, q_idx, k_idx, cu_seqlens, B_k: int, kk: int, attn_scale: float = 0.0,
                   stream=None):
    """Whole MSA forward (Eq. 6-8) of a packed batch of sequences: (o, lse, idx)."""
    idx = index_topk_varlen(q_idx, k_idx, cu_seqlens, B_k, kk, stream=stream)
    o, lse = sparse_attn_fwd_varlen(q, k, v, idx, cu_seqlens, B_k, attn_scale, stream=stream)
    return o, lse, idx


def sparse_decode(q, q_idx, k_new, v_new, k_idx_new, k_cache, v_cache, k_idx_cache,
                  seq_len, B_k: int, kk: int, attn_scale: float = 0.0,
                  o: Optional[torch.Tensor] = None, idx_out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, stream=None):
    """One decode step (append + Eq. 6-8 for the new token of each sequence).
    Returns (o [S,H_q,d_h] bf16, idx_out or None); seq_len is incremented."""
    S, H_q, d_h = q.shape
    H_kv, d_idx = q_idx.shape[1], q_idx.shape[2]
    L_max = k_cache.shape[1]
    _want(q, "q", torch.bfloat16, (S, H_q, d_h))
    _want(q_idx, "q_idx", torch.bfloat16, (S, H_kv, d_idx))
    _want(k_new, "k_new", torch.bfloat16, (S, H_kv, d_h))
    _want(v_new, "v_new", torch.bfloat16, (S, H_kv, d_h))
    _want(k_idx_new, "k_idx_new", torch.bfloat16, (S, d_idx))
    _want(k_cache, "k_cache", torch.bfloat16, (S, L_max, H_kv, d_h))
    _want(v_cache, "v_cache", torch.bfloat16, (S, L_max, H_kv, d_h))
    _want(k_idx_cache, "k_idx_cache", torch.bfloat16, (S, L_max, d_idx))
    _want(seq_len, "seq_len", torch.int32, (S,))
    if o is None:
        o = torch.empty((S, H_q, d_h), dtype=torch.bfloat16, device=q.device)
    _want(o, "o", torch.bfloat16, (S, H_q, d_h))
    if idx_out is not None:
        _want(idx_out, "idx_out", torch.int32, (S, H_kv, kk))
    d = decode_dims(S, L_max, H_q, H_kv, d_h, d_idx, B_k, kk, attn_scale)
    ws = _workspace(sparse_decode_workspace_size(d), q.device, workspace)
    _raise("msa_sparse_decode",
           LIB.msa_sparse_decode(ctypes.byref(d), _ptr(q), _ptr(q_idx), _ptr(k_new), _ptr(v_new),
                                 _ptr(k_idx_new), _ptr(k_cache), _ptr(v_cache), _ptr(k_idx_cache),
                                 _ptr(seq_len), _ptr(o), _ptr(idx_out), _ptr(ws), ws.numel(),
                                 _stream(stream)))
    return o, idx_out


def profile_enable(on: bool) -> None:
    """Start (clearing earlier records) or stop per-kernel event timing."""
    LIB.msa_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """{kernel name: (launches, total milliseconds)} recorded since enable."""
    buf = (msa_kernel_time * 64)()
    n = LIB.msa_profile_read(buf, 64)
    if n < 0:
        raise MSAError("msa_profile_read", 4, "CUDA error")
    return {buf[j].name.decode(): (int(buf[j].launches), float(buf[j].total_ms))
            for j in range(min(n, 64))}


def sparse_decode_noalloc(q, q_idx, k_new, v_new, k_idx_new, k_cache, v_cache, k_idx_cache,
                          seq_len, B_k: int, kk: int, attn_scale: float = 0.0,
                          o: Optional[torch.Tensor] = None,
                          idx_out: Optional[torch.Tensor] = None, stream=None):
    """sparse_decode without a workspace: the library's fixed scratch array is
    used (for callers that cannot allocate device memory while serving).  Pass
    ``o`` to avoid the one output allocation this binding would otherwise make."""
    S, H_q, d_h = q.shape
    H_kv, d_idx = q_idx.shape[1], q_idx.shape[2]
    L_max = k_cache.shape[1]
    _want(q, "q", torch.bfloat16, (S, H_q, d_h))
    _want(q_idx, "q_idx", torch.bfloat16, (S, H_kv, d_idx))
    _want(k_new, "k_new", torch.bfloat16, (S, H_kv, d_h))
    _want(v_new, "v_new", torch.bfloat16, (S, H_kv, d_h))
    _want(k_idx_new, "k_idx_new", torch.bfloat16, (S, d_idx))
    _want(k_cache, "k_cache", torch.bfloat16, (S, L_max, H_kv, d_h))
    _want(v_cache, "v_cache", torch.bfloat16, (S, L_max, H_kv, d_h))
    _want(k_idx_cache, "k_idx_cache", torch.bfloat16, (S, L_max, d_idx))
    _want(seq_len, "seq_len", torch.int32, (S,))
    if o is None:
        o = torch.empty((S, H_q, d_h), dtype=torch.bfloat16, device=q.device)
    _want(o, "o", torch.bfloat16, (S, H_q, d_h))
    if idx_out is not None:
        _want(idx_out, "idx_out", torch.int32, (S, H_kv, kk))
    d = decode_dims(S, L_max, H_q, H_kv, d_h, d_idx, B_k, kk, attn_scale)
    _raise("msa_sparse_decode_noalloc",
           LIB.msa_sparse_decode_noalloc(ctypes.byref(d), _ptr(q), _ptr(q_idx), _ptr(k_new),
                                         _ptr(v_new), _ptr(k_idx_new), _ptr(k_cache),
                                         _ptr(v_cache), _ptr(k_idx_cache), _ptr(seq_len),
                                         _ptr(o), _ptr(idx_out), _stream(stream)))
    return o, idx_out


def selftest_bounded_wait(workspace: torch.Tensor, stream=None) -> None:
    """Launch the library's bounded-wait self-test (times out after about 2 s
    and records MSA_DEV_TIMEOUT, where 99, in the workspace's status word)."""
    _raise("msa_selftest_bounded_wait",
           LIB.msa_selftest_bounded_wait(_ptr(workspace), _stream(stream)))


def device_status(workspace: torch.Tensor, stream=None) -> Tuple[int, int]:
    """(code, where) of the workspace's device status word; syncs the stream."""
    code, where = ctypes.c_int32(0), ctypes.c_int32(0)
    LIB.msa_get_device_status(_ptr(workspace), _stream(stream), ctypes.byref(code),
                              ctypes.byref(where))
    return int(code.value), int(where.value)


def paged_dims(S, max_pages, n_pages, H_q, H_kv, d_h, d_idx, B_k, k, attn_scale=0.0,
               idx_scale=0.0) -> msa_paged_dims:
    return msa_paged_dims(int(S), int(max_pages), int(n_pages), int(H_q), int(H_kv), int(d_h),
                          int(d_idx), int(B_k), int(k), float(attn_scale), float(idx_scale))


def paged_decode_fp8_workspace_size(d: msa_paged_dims) -> int:
    return int(LIB.msa_paged_decode_fp8_workspace(ctypes.byref(d)))


def paged_decode_fp8(q, q_idx, k_new, v_new, k_idx_new, k_pages, k_scale, v_pages, v_scale,
                     kidx_pages, kidx_scale, page_table, seq_len, B_k: int, kk: int,
                     attn_scale: float = 0.0, o: Optional[torch.Tensor] = None,
                     idx_out: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None):
    """One decode step on a paged FP8 (E4M3) cache: the new tokens are
    quantized into their pages, then Eq. 6-8 run on the dequantized cache.
    k_pages/v_pages [P,B_k,H_kv,d_h] uint8, k_scale/v_scale [P,B_k,H_kv] fp32,
    kidx_pages [P,B_k,d_idx] uint8, kidx_scale [P,B_k] fp32, page_table
    [S,max_pages] int32.  Returns (o [S,H_q,d_h] bf16, idx_out or None)."""
    S, H_q, d_h = q.shape
    H_kv, d_idx = q_idx.shape[1], q_idx.shape[2]
    P = k_pages.shape[0]
    max_pages = page_table.shape[1]
    _want(q, "q", torch.bfloat16, (S, H_q, d_h))
    _want(q_idx, "q_idx", torch.bfloat16, (S, H_kv, d_idx))
    _want(k_new, "k_new", torch.bfloat16, (S, H_kv, d_h))
    _want(v_new, "v_new", torch.bfloat16, (S, H_kv, d_h))
    _want(k_idx_new, "k_idx_new", torch.bfloat16, (S, d_idx))
    _want(k_pages, "k_pages", torch.uint8, (P, B_k, H_kv, d_h))
    _want(v_pages, "v_pages", torch.uint8, (P, B_k, H_kv, d_h))
    _want(k_scale, "k_scale", torch.float32, (P, B_k, H_kv))
    _want(v_scale, "v_scale", torch.float32, (P, B_k, H_kv))
    _want(kidx_pages, "kidx_pages", torch.uint8, (P, B_k, d_idx))
    _want(kidx_scale, "kidx_scale", torch.float32, (P, B_k))
    _want(page_table, "page_table", torch.int32, (S, max_pages))
    _want(seq_len, "seq_len", torch.int32, (S,))
    if o is None:
        o = torch.empty((S, H_q, d_h), dtype=torch.bfloat16, device=q.device)
    _want(o, "o", torch.bfloat16, (S, H_q, d_h))
    if idx_out is not None:
        _want(idx_out, "idx_out", torch.int32, (S, H_kv, kk))
    d = paged_dims(S, max_pages, P, H_q, H_kv, d_h, d_idx, B_k, kk, attn_scale)
    ws = _workspace(paged_decode_fp8_workspace_size(d), q.device, workspace)
    _raise("msa_paged_decode_fp8",
           LIB.msa_paged_decode_fp8(ctypes.byref(d), _ptr(q), _ptr(q_idx), _ptr(k_new),
                                    _ptr(v_new), _ptr(k_idx_new), _ptr(k_pages), _ptr(k_scale),
                                    _ptr(v_pages), _ptr(v_scale), _ptr(kidx_pages),
                                    _ptr(kidx_scale), _ptr(page_table), _ptr(seq_len), _ptr(o),
                                    _ptr(idx_out), _ptr(ws), ws.numel(), _stream(stream)))
    return o, idx_out


def quantize_fp8_rows(x: torch.Tensor, codes: Optional[torch.Tensor] = None,
                      scales: Optional[torch.Tensor] = None, stream=None):
    """bf16 rows [..., dim] -> (E4M3 codes [..., dim] uint8, scales [...] fp32)
    with the FP8 decode's append rule (scale = amax / 448 per row)."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor")
    dim = x.shape[-1]
    rows = x.numel() // dim
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _want(codes, "codes", torch.uint8, tuple(x.shape))
    _want(scales, "scales", torch.float32, tuple(x.shape[:-1]))
    _raise("msa_quantize_fp8_rows",
           LIB.msa_quantize_fp8_rows(_ptr(x), rows, dim, _ptr(codes), _ptr(scales),
                                     _stream(stream)))
    return codes, scales

