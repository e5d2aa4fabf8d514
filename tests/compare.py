"""Comparators for the CUDA path against the oracle.

Top-k (Eq. 7): sets must be identical, except where the oracle's last kept
non-local score ("cut") and best left-out score ("next") lie within a
relative band of each other; there, a different set is accepted when it is a
valid selection and every block in the symmetric difference has an oracle
score inside the band around the cut.  The band is 1e-3 relative to
max(|cut|, |next|) with an absolute floor of 1e-5.

Attention (Eq. 8): max-abs <= 2e-2 and mean-abs <= 2e-3 (bf16 inputs, fp32
accumulation), LSE within 1e-3 absolute.
"""
from __future__ import annotations

import numpy as np

import oracle

TIE_REL = 1e-3
TIE_ABS = 1e-5
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def _band(a: float, b: float) -> float:
    return max(TIE_REL * max(abs(a), abs(b)), TIE_ABS)


def valid_selection(sel: np.ndarray, i: int, B_k: int, k: int) -> bool:
    """Structural validity of one selection row (Eq. 7 + local block rule)."""
    b_i = i // B_k
    sel = [int(x) for x in sel]
    n = sum(1 for x in sel if x >= 0)
    # entries first (ascending, unique, all visible), then -1 padding only
    if any(x < 0 for x in sel[:n]) or any(x != -1 for x in sel[n:]):
        return False
    vals = sel[:n]
    if vals != sorted(set(vals)) or b_i not in vals or vals[-1] > b_i:
        return False
    return n == min(k, b_i + 1)


def check_topk(gpu_idx: np.ndarray, ref_idx: np.ndarray, cut: np.ndarray, nxt: np.ndarray,
               rows: np.ndarray, B_k: int, k: int, q_idx_rows=None, k_idx=None,
               max_report: int = 5):
    """Returns (n_exact, n_band, failures).  gpu_idx/ref_idx: [n, H_kv, k]."""
    n, H_kv, _ = ref_idx.shape
    exact = band = 0
    failures = []
    for t in range(n):
        i = int(rows[t])
        for r in range(H_kv):
            g = gpu_idx[t, r]
            o = ref_idx[t, r]
            if np.array_equal(g, o):
                exact += 1
                continue
            why = None
            if not valid_selection(g, i, B_k, k):
                why = "invalid selection"
            elif np.isnan(cut[t, r]) or np.isnan(nxt[t, r]):
                why = "differs where no tie is possible"
            elif abs(cut[t, r] - nxt[t, r]) >= _band(cut[t, r], nxt[t, r]):
                why = "differs outside the tie band"
            elif q_idx_rows is None or k_idx is None:
                why = "differs inside the band, scores unavailable"
            else:
                M = oracle.block_scores(q_idx_rows[t, r], k_idx, B_k, i)
                c = cut[t, r]
                diff = set(int(x) for x in g if x >= 0) ^ set(int(x) for x in o if x >= 0)
                if any(abs(M[b] - c) >= _band(M[b], c) for b in diff):
                    why = "swapped block outside the tie band"
            if why is None:
                band += 1
            else:
                failures.append((i, r, why, g.tolist(), o.tolist()))
    return exact, band, failures[:max_report] if failures else []


def attn_errors(o_gpu: np.ndarray, o_ref: np.ndarray):
    d = np.abs(o_gpu.astype(np.float64) - o_ref)
    return float(d.max()), float(d.mean())


def assert_attn_close(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    mx, mean = attn_errors(o_gpu, o_ref)
    assert mx <= O_MAX_ABS and mean <= O_MEAN_ABS, \
        f"{what}: max-abs {mx:.3e} (<= {O_MAX_ABS}), mean-abs {mean:.3e} (<= {O_MEAN_ABS})"
    if lse_gpu is not None and lse_ref is not None:
        e = float(np.abs(lse_gpu.astype(np.float64) - lse_ref).max())
        assert e <= LSE_ABS, f"{what}: LSE max-abs {e:.3e} (<= {LSE_ABS})"
