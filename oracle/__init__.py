"""CPU oracle of the MSA forward pass -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product path (the CUDA library and its binding)
never loads it, and this package never loads the CUDA library.

The arithmetic lives in ``msa_oracle.c`` (plain C, fp64 sums, OpenMP threads
over rows), compiled here with gcc on first use.  Each function cites the
equation of the MSA pages it follows (xllm-io review, "核心公式" section:
Eq. 1, 4, 6, 7, 8, 12; chlience notes, section 5.1.1).  Arrays of bf16 values
are numpy ``uint16`` bit patterns.

Pins (tests/test_oracle_pins.py): planted block maxima with a hand-derived
selection, brute-force subset enumeration, numpy stable argsort, rescale
invariance, dense equivalence with torch's scaled_dot_product_attention,
block-diagonal causal attention for k = 1, softmax weights summing to one,
the LSE split/merge identity and the Eq. 12 closed form (28.4x at 1M).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_HDR = os.path.join(_HERE, "msa_oracle.h")
# MSA_ORACLE_SANITIZE=1 selects a copy built with AddressSanitizer and
# UndefinedBehaviorSanitizer (the process must preload libasan and libubsan),
# to check the oracle's own memory accesses and arithmetic.
_SANITIZE = os.environ.get("MSA_ORACLE_SANITIZE") == "1"
_LIB = os.path.join(_HERE, "liboracle_san.so" if _SANITIZE else "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile msa_oracle.c into liboracle.so (gcc, -O2, no fast-math), or the
    sanitized copy (-O1 with -fsanitize=address,undefined) when selected."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".{os.getpid()}.tmp"
        opt = (["-O1", "-g", "-fsanitize=address,undefined", "-fno-omit-frame-pointer"]
               if _SANITIZE else ["-O2"])
        cmd = ["gcc", "-std=c11", *opt, "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I64, I32, D = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.oracle_max_threads.restype = I32
            lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_value.restype = D
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_quantize_rows.argtypes = [P, I64, I32, P, P]
            lib.oracle_paged_decode_fp8.argtypes = (
                [P] * 5 + [P] * 6 + [P, I32, P] + [I32] * 6 + [D, D] + [P, I64] + [P] * 5
                + [P] * 5)
            lib.oracle_block_scores.argtypes = [P, P, I64, I32, I32, I64, P]
            lib.oracle_index_topk.argtypes = [P, P, I64, I32, I32, I32, I32, P, I64, P, P, P, I32]
            lib.oracle_sparse_attn.argtypes = [P, P, P, P, I64, I32, I32, I32, I32, I32, D, P, I64,
                                               P, P, I32]
            lib.oracle_dense_attn.argtypes = [P, P, P, I64, I32, I32, I32, D, P, I64, P, P, I32]
            lib.oracle_sparse_attn_bwd.argtypes = [P, P, P, P, P, I64, I32, I32, I32, I32, I32, D,
                                                   P, P, P, I32]
            lib.oracle_sparse_attn_bwd.restype = I32
            lib.oracle_index_lse.argtypes = [P, P, P, I64, I32, I32, I32, I32, D, P, I64, P, I32]
            lib.oracle_flops.argtypes = [D] * 7 + [P, P, P]
            for f in ("oracle_block_scores", "oracle_index_topk", "oracle_sparse_attn",
                      "oracle_dense_attn", "oracle_index_lse"):
                getattr(lib, f).restype = I32
            lib.oracle_flops.restype = None
            _lib = lib
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def block_scores(q_idx_row: np.ndarray, k_idx: np.ndarray, B_k: int, i: int) -> np.ndarray:
    """Eq. 6: M[b] for b = 0..i//B_k of one index-query row (float64)."""
    q = _c(q_idx_row, np.uint16).reshape(-1)
    kk = _c(k_idx, np.uint16)
    out = np.empty(i // B_k + 1, dtype=np.float64)
    _check(_load().oracle_block_scores(_p(q), _p(kk), kk.shape[0], q.size, B_k, i, _p(out)),
           "block_scores")
    return out


def index_topk(q_idx: np.ndarray, k_idx: np.ndarray, B_k: int, k: int,
               rows: Optional[np.ndarray] = None, threads: int = 0
               ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Eq. 6-7 for ``rows`` (default: all).  q_idx [N,H_kv,d_idx], k_idx [N,d_idx].

    Returns idx [n,H_kv,k] int32 (ascending, -1 padded), cut and next [n,H_kv]
    float64 (tie-band bounds).
    """
    kk = _c(k_idx, np.uint16)
    N, d_idx = kk.shape
    H_kv = q_idx.shape[1]
    rows = np.arange(N, dtype=np.int64) if rows is None else _c(rows, np.int64)
    qr = _c(np.asarray(q_idx)[rows], np.uint16)
    idx = np.empty((rows.size, H_kv, k), dtype=np.int32)
    cut = np.empty((rows.size, H_kv), dtype=np.float64)
    nxt = np.empty((rows.size, H_kv), dtype=np.float64)
    _check(_load().oracle_index_topk(_p(qr), _p(kk), N, H_kv, d_idx, B_k, k, _p(rows), rows.size,
                                     _p(idx), _p(cut), _p(nxt), threads), "index_topk")
    return idx, cut, nxt


def index_topk_rows(q_idx_rows: np.ndarray, k_idx: np.ndarray, N: int, B_k: int, k: int,
                    rows: np.ndarray, threads: int = 0
                    ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """As ``index_topk`` but with the index queries of the rows given directly
    (q_idx_rows [n,H_kv,d_idx]) and the first N rows of k_idx as the keys."""
    kk = _c(k_idx, np.uint16)
    d_idx = kk.shape[1]
    rows = _c(rows, np.int64)
    qr = _c(q_idx_rows, np.uint16)
    H_kv = qr.shape[1]
    idx = np.empty((rows.size, H_kv, k), dtype=np.int32)
    cut = np.empty((rows.size, H_kv), dtype=np.float64)
    nxt = np.empty((rows.size, H_kv), dtype=np.float64)
    _check(_load().oracle_index_topk(_p(qr), _p(kk), N, H_kv, d_idx, B_k, k, _p(rows), rows.size,
                                     _p(idx), _p(cut), _p(nxt), threads), "index_topk")
    return idx, cut, nxt


def sparse_attn(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, idx_rows: np.ndarray,
                B_k: int, rows: np.ndarray, N: Optional[int] = None,
                scale: Optional[float] = None, threads: int = 0
                ) -> Tuple[np.ndarray, np.ndarray]:
    """Eq. 8 for the listed rows.  q_rows [n,H_q,d_h] (the rows' queries),
    k/v [>=N,H_kv,d_h], idx_rows [n,H_kv,kk].  Returns O [n,H_q,d_h] and
    LSE [n,H_q] (float64, natural log)."""
    qr = _c(q_rows, np.uint16)
    kk_ = _c(k, np.uint16)
    vv = _c(v, np.uint16)
    ir = _c(idx_rows, np.int32)
    rows = _c(rows, np.int64)
    n, H_q, d_h = qr.shape
    H_kv = kk_.shape[1]
    N = kk_.shape[0] if N is None else N
    scale = 1.0 / np.sqrt(d_h) if scale is None else scale
    o = np.empty((n, H_q, d_h), dtype=np.float64)
    lse = np.empty((n, H_q), dtype=np.float64)
    _check(_load().oracle_sparse_attn(_p(qr), _p(kk_), _p(vv), _p(ir), N, H_q, H_kv, d_h, B_k,
                                      ir.shape[2], float(scale), _p(rows), n, _p(o), _p(lse),
                                      threads), "sparse_attn")
    return o, lse


def sparse_attn_bwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, idx: np.ndarray,
                    d_o: np.ndarray, B_k: int, scale: Optional[float] = None,
                    threads: int = 0) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients of Eq. 8 with the selection fixed, all rows of one sequence:
    q, d_o [N,H_q,d_h], k/v [N,H_kv,d_h] (bf16 bits), idx [N,H_kv,kk] ->
    dQ [N,H_q,d_h], dK, dV [N,H_kv,d_h] (float64)."""
    qq, kk_, vv, gg = (_c(a, np.uint16) for a in (q, k, v, d_o))
    ir = _c(idx, np.int32)
    N, H_q, d_h = qq.shape
    H_kv = kk_.shape[1]
    scale = 1.0 / np.sqrt(d_h) if scale is None else scale
    dq = np.empty((N, H_q, d_h), dtype=np.float64)
    dk = np.empty((N, H_kv, d_h), dtype=np.float64)
    dv = np.empty((N, H_kv, d_h), dtype=np.float64)
    _check(_load().oracle_sparse_attn_bwd(_p(qq), _p(kk_), _p(vv), _p(ir), _p(gg), N, H_q, H_kv,
                                          d_h, B_k, ir.shape[2], float(scale), _p(dq), _p(dk),
                                          _p(dv), threads), "sparse_attn_bwd")
    return dq, dk, dv


def index_lse(q_idx_rows: np.ndarray, k_idx: np.ndarray, idx_rows: np.ndarray, B_k: int,
              rows: np.ndarray, N: Optional[int] = None, scale: Optional[float] = None,
              threads: int = 0) -> np.ndarray:
    """Eq. 9's Index Branch normaliser (the LSE_idx of the KL loss fusion) for
    the listed rows: log of the sum of exp(S^idx) over the selected tokens
    j <= i.  q_idx_rows [n,H_kv,d_idx], k_idx [>=N,d_idx], idx_rows [n,H_kv,kk].
    Returns [n,H_kv] float64 (-inf for an empty token set)."""
    qr = _c(q_idx_rows, np.uint16)
    kr = _c(k_idx, np.uint16)
    ir = _c(idx_rows, np.int32)
    rows = _c(rows, np.int64)
    n, H_kv, d_idx = qr.shape
    N = kr.shape[0] if N is None else N
    scale = 1.0 / np.sqrt(d_idx) if scale is None else scale
    out = np.empty((n, H_kv), dtype=np.float64)
    _check(_load().oracle_index_lse(_p(qr), _p(kr), _p(ir), N, H_kv, d_idx, B_k, ir.shape[2],
                                    float(scale), _p(rows), n, _p(out), threads), "index_lse")
    return out


def dense_attn(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, rows: np.ndarray,
               N: Optional[int] = None, scale: Optional[float] = None, threads: int = 0
               ) -> Tuple[np.ndarray, np.ndarray]:
    """Eq. 1 dense causal GQA for the listed rows (same layouts as sparse_attn)."""
    qr = _c(q_rows, np.uint16)
    kk_ = _c(k, np.uint16)
    vv = _c(v, np.uint16)
    rows = _c(rows, np.int64)
    n, H_q, d_h = qr.shape
    H_kv = kk_.shape[1]
    N = kk_.shape[0] if N is None else N
    scale = 1.0 / np.sqrt(d_h) if scale is None else scale
    o = np.empty((n, H_q, d_h), dtype=np.float64)
    lse = np.empty((n, H_q), dtype=np.float64)
    _check(_load().oracle_dense_attn(_p(qr), _p(kk_), _p(vv), N, H_q, H_kv, d_h, float(scale),
                                     _p(rows), n, _p(o), _p(lse), threads), "dense_attn")
    return o, lse


def forward(inp: dict, B_k: int, k: int, rows: Optional[np.ndarray] = None,
            idx_rows: Optional[np.ndarray] = None, threads: int = 0) -> dict:
    """Whole forward pass (Eq. 6-8) for ``rows``: selection, then attention.

    If ``idx_rows`` is given it replaces the oracle's own selection in the
    attention step (so a selection made elsewhere can be checked on its own).
    """
    N = inp["k_idx"].shape[0]
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    idx, cut, nxt = index_topk(inp["q_idx"], inp["k_idx"], B_k, k, rows, threads)
    use = idx if idx_rows is None else idx_rows
    o, lse = sparse_attn(inp["q"][rows], inp["k"], inp["v"], use, B_k, rows, N=N,
                         threads=threads)
    return {"idx": idx, "cut": cut, "next": nxt, "o": o, "lse": lse, "rows": rows}


def project(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """One projection of Algorithm 1, lines 1-2 (xllm-io review): x W in fp64
    from the exactly widened bf16 operands.  x [T, d_model], w [d_model, n]
    (bf16 bits) -> [T, n] float64.  The index projections take stopgrad(x),
    which is x itself in a forward pass."""
    xf = (np.ascontiguousarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    wf = (np.ascontiguousarray(w, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    return xf.astype(np.float64) @ wf.astype(np.float64)


def forward_varlen(inp: dict, cu_seqlens, B_k: int, k: int, rows: Optional[np.ndarray] = None,
                   idx_rows: Optional[np.ndarray] = None, threads: int = 0) -> dict:
    """Eq. 6-8 for a batch of sequences packed along the token axis: sequence
    s is tokens cu_seqlens[s] .. cu_seqlens[s+1]-1 of every input, and each
    sequence is its own prefill (``forward`` on its slice; block indices in
    ``idx`` are local to the sequence).  Returns the fields of ``forward`` for
    ``rows`` (global token indices, default all) plus each row's sequence.
    ``idx_rows`` (one selection per row, local block indices) replaces the
    oracle's own selection in the attention step, as in ``forward``."""
    cu = [int(x) for x in cu_seqlens]
    N = cu[-1]
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    n = rows.size
    H_kv, H_q, d_h = inp["q_idx"].shape[1], inp["q"].shape[1], inp["q"].shape[2]
    out = {"idx": np.empty((n, H_kv, k), np.int32), "cut": np.empty((n, H_kv)),
           "next": np.empty((n, H_kv)), "o": np.empty((n, H_q, d_h)), "lse": np.empty((n, H_q)),
           "rows": rows, "seq": np.searchsorted(np.asarray(cu[1:]), rows, side="right")}
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        pick = np.nonzero((rows >= a) & (rows < b))[0]
        if pick.size == 0:
            continue
        sub = {key: inp[key][a:b] for key in ("q", "k", "v", "q_idx", "k_idx")}
        r = forward(sub, B_k, k, rows[pick] - a,
                    idx_rows=None if idx_rows is None else idx_rows[pick], threads=threads)
        for key in ("idx", "cut", "next", "o", "lse"):
            out[key][pick] = r[key]
    return out


def decode_reference(state: dict, step_in: dict, B_k: int, k: int, seqs=None,
                     idx_rows: Optional[np.ndarray] = None, threads: int = 0) -> dict:
    """One decode step for the listed sequences, on host copies of the caches.

    Appends the new rows at position L_s (the query attends to itself, Eq. 1's
    i <= t), then runs Eq. 6-8 for the single query at i = L_s (new length
    L_s + 1).  The caches in ``state`` are not modified.
    """
    S = state["seq_len"].shape[0]
    seqs = range(S) if seqs is None else seqs
    outs = {"idx": [], "cut": [], "next": [], "o": [], "lse": []}
    for n, s in enumerate(seqs):
        L = int(state["seq_len"][s])
        kc = state["k_cache"][s, : L + 1].copy()
        vc = state["v_cache"][s, : L + 1].copy()
        kic = state["k_idx_cache"][s, : L + 1].copy()
        kc[L] = step_in["k_new"][s]
        vc[L] = step_in["v_new"][s]
        kic[L] = step_in["k_idx_new"][s]
        row = np.array([L], dtype=np.int64)
        idx, cut, nxt = index_topk_rows(step_in["q_idx"][s][None], kic, L + 1, B_k, k, row,
                                        threads)
        use = idx if idx_rows is None else idx_rows[n][None]
        o, lse = sparse_attn(step_in["q"][s][None], kc, vc, use, B_k, row, N=L + 1,
                             threads=threads)
        for key, val in (("idx", idx), ("cut", cut), ("next", nxt), ("o", o), ("lse", lse)):
            outs[key].append(val[0])
    return {key: np.stack(val) for key, val in outs.items()}


def flops(N: float, H_q: int, H_kv: int, d_h: int, d_idx: int, B_k: int, k: int) -> dict:
    """Eq. 12: F_GQA, F_MSA index term, F_MSA main term (FLOPs)."""
    g, fi, fm = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    _load().oracle_flops(float(N), H_q, H_kv, d_h, d_idx, B_k, k, ctypes.byref(g),
                         ctypes.byref(fi), ctypes.byref(fm))
    return {"gqa": g.value, "index": fi.value, "main": fm.value,
            "msa": fi.value + fm.value, "ratio": g.value / (fi.value + fm.value)}


# ------------------------------------------------- FP8 (E4M3) paged decode --
def e4m3_values() -> np.ndarray:
    """Value of every E4M3 code 0..255 (float64; NaN for the two NaN codes)."""
    lib = _load()
    return np.array([lib.oracle_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 values -> E4M3 codes (nearest, ties to the even code, saturated)."""
    lib = _load()
    flat = np.asarray(x, dtype=np.float32).reshape(-1)
    return np.array([lib.oracle_e4m3_encode(float(v)) for v in flat],
                    dtype=np.uint8).reshape(np.shape(x))


def quantize_rows(x_bf16: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """bf16 rows [..., dim] -> (E4M3 codes [..., dim] uint8, scales [...] float32),
    scale = amax / 448 per row (1 for an all-zero row)."""
    x = _c(x_bf16, np.uint16)
    dim = x.shape[-1]
    rows = x.size // dim
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty(x.shape[:-1], dtype=np.float32)
    _check(_load().oracle_quantize_rows(_p(x), rows, dim, _p(codes), _p(scales)),
           "quantize_rows")
    return codes, scales


def paged_decode_fp8(pages: dict, step_in: dict, seq_len: np.ndarray, B_k: int, k: int,
                     seqs=None, attn_scale: Optional[float] = None,
                     idx_scale: Optional[float] = None) -> dict:
    """One decode step on an FP8 paged cache for the listed sequences.

    pages: k_pages/v_pages [P,B_k,H_kv,d_h] uint8, k_scale/v_scale [P,B_k,H_kv]
    float32, kidx_pages [P,B_k,d_idx] uint8, kidx_scale [P,B_k] float32,
    page_table [S,max_pages] int32.  step_in: q [S,H_q,d_h], q_idx
    [S,H_kv,d_idx], k_new/v_new [S,H_kv,d_h], k_idx_new [S,d_idx] (bf16).
    Returns idx, cut, next, o, lse and the new token's quantized rows
    (new_k, new_v [n,H_kv,d_h], new_kv_scale [n,2,H_kv], new_kidx [n,d_idx],
    new_kidx_scale [n])."""
    S, H_q, d_h = step_in["q"].shape
    H_kv, d_idx = step_in["q_idx"].shape[1], step_in["q_idx"].shape[2]
    seqs = np.arange(S, dtype=np.int64) if seqs is None else np.asarray(seqs, dtype=np.int64)
    n = seqs.size
    pt = _c(pages["page_table"], np.int32)
    a = {key: _c(step_in[key], np.uint16) for key in ("q", "q_idx", "k_new", "v_new",
                                                        "k_idx_new")}
    pg = {key: _c(pages[key], np.uint8) for key in ("k_pages", "v_pages", "kidx_pages")}
    sc = {key: _c(pages[key], np.float32) for key in ("k_scale", "v_scale", "kidx_scale")}
    out = {"idx": np.empty((n, H_kv, k), np.int32), "cut": np.empty((n, H_kv)),
           "next": np.empty((n, H_kv)), "o": np.empty((n, H_q, d_h)), "lse": np.empty((n, H_q)),
           "new_k": np.empty((n, H_kv, d_h), np.uint8), "new_v": np.empty((n, H_kv, d_h), np.uint8),
           "new_kv_scale": np.empty((n, 2, H_kv), np.float32),
           "new_kidx": np.empty((n, d_idx), np.uint8), "new_kidx_scale": np.empty(n, np.float32)}
    sl = _c(seq_len, np.int32)
    rc = _load().oracle_paged_decode_fp8(
        _p(a["q"]), _p(a["q_idx"]), _p(a["k_new"]), _p(a["v_new"]), _p(a["k_idx_new"]),
        _p(pg["k_pages"]), _p(sc["k_scale"]), _p(pg["v_pages"]), _p(sc["v_scale"]),
        _p(pg["kidx_pages"]), _p(sc["kidx_scale"]), _p(pt), pt.shape[1], _p(sl),
        H_q, H_kv, d_h, d_idx, B_k, k,
        1.0 / np.sqrt(d_h) if attn_scale is None else attn_scale,
        1.0 / np.sqrt(d_idx) if idx_scale is None else idx_scale,
        _p(seqs), n, _p(out["idx"]), _p(out["cut"]), _p(out["next"]), _p(out["o"]),
        _p(out["lse"]), _p(out["new_k"]), _p(out["new_v"]), _p(out["new_kv_scale"]),
        _p(out["new_kidx"]), _p(out["new_kidx_scale"]))
    _check(rc, "paged_decode_fp8")
    return out
