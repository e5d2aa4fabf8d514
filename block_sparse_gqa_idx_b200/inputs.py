"""Seeded synthetic inputs for the MSA forward pass.

This module only draws numbers: it holds none of the method's arithmetic and
is shared by the CUDA path's tests and benchmark and by the CPU oracle's
tests, so both sides always see the same bytes.  Arrays are numpy ``uint16``
holding bfloat16 bit patterns (round-to-nearest-even from float32).

Workload shapes follow the pages' setting (B_k = 128, k = 16, G = H_q/H_kv
adjacent query heads per KV head; xllm-io review, "实验设置" table; chlience
notes, 5.1) at the sizes listed in ``CONFIGS``.  The planted structure is:

* ``iid``: every tensor i.i.d. N(0, 1).  Q, K and V are drawn in blocks of
  2^24 values, each block from its own child stream of the tensor's seed
  (so they can be drawn in parallel).
* ``sink_ar1``: Q, K, V i.i.d. N(0, 1).  Q_idx (each group) and K_idx follow
  an AR(1) process along the sequence, x_0 = e_0, x_i = rho x_{i-1} +
  sqrt(1 - rho^2) e_i (rho = 0.9, N(0,1) marginals), for locality.  A seeded
  unit vector u is added, times ``sink_strength``, to every index query, and
  2*sqrt(d_idx)*u to every index key of block 0: block-0 scores gain
  +2*strength on average, against a spread of 2 from the queries' own
  component along u, so the strength sets how many rows pick the sink.
* ``sink_ar1_retrieval``: ``sink_ar1`` plus, per group, 8 "retrieval" blocks
  drawn from [1, B-2]; each gets a unit vector v, one random token of the
  block gets K_idx += 2*sqrt(d_idx)*v, and a random 1/8 of the later queries
  get Q_idx += 2*v.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

SEED_BASE = 0x4D5341  # "MSA"
_CHUNK = 1 << 24


@dataclasses.dataclass(frozen=True)
class MSAConfig:
    name: str
    N: int
    H_q: int
    H_kv: int
    d_h: int
    d_idx: int
    B_k: int
    k: int
    structure: str = "iid"
    sink_strength: float = 1.0
    seed_index: int = 0

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def B(self) -> int:
        return (self.N + self.B_k - 1) // self.B_k

    @property
    def seed(self) -> int:
        return SEED_BASE + self.seed_index

    def with_N(self, N: int) -> "MSAConfig":
        return dataclasses.replace(self, N=N, name=f"{self.name}@N={N}")


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    S: int
    L0: int
    steps: int
    H_q: int
    H_kv: int
    d_h: int
    d_idx: int
    B_k: int
    k: int
    sink_strength: float = 1.0
    seed_index: int = 3

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def L_max(self) -> int:
        return self.L0 + self.steps

    @property
    def seed(self) -> int:
        return SEED_BASE + self.seed_index


@dataclasses.dataclass(frozen=True)
class VarlenConfig:
    """A packed batch of prefill sequences: n_seqs lengths drawn by
    ``varlen_lengths`` (log-uniform in [len_lo, len_hi], summing to N), each
    sequence with ``prefill_inputs``' recipe for ``structure``."""
    name: str
    n_seqs: int
    N: int
    len_lo: int
    len_hi: int
    H_q: int
    H_kv: int
    d_h: int
    d_idx: int
    B_k: int
    k: int
    structure: str = "sink_ar1"
    seed_index: int = 0

    @property
    def seed(self) -> int:
        return SEED_BASE + self.seed_index

    @property
    def prefill(self) -> "MSAConfig":
        """The per-sequence heads and recipe (N = 0: each sequence sets its own)."""
        return MSAConfig(self.name, 0, self.H_q, self.H_kv, self.d_h, self.d_idx, self.B_k,
                         self.k, self.structure, 1.0, self.seed_index)

    def lengths(self) -> np.ndarray:
        return varlen_lengths(self.n_seqs, self.N, self.len_lo, self.len_hi, self.seed)


CONFIGS: Dict[str, object] = {
    # tiny prefill: the oracle finishes in seconds
    "tiny": MSAConfig("tiny", N=2048, H_q=8, H_kv=2, d_h=64, d_idx=32, B_k=64, k=4,
                      structure="iid", seed_index=0),
    # prefill at the pages' sparsity, 32K context
    "32k": MSAConfig("32k", N=32768, H_q=32, H_kv=4, d_h=128, d_idx=64, B_k=128, k=16,
                     structure="sink_ar1", seed_index=1),
    # long-context prefill, 128K, sink + retrieval blocks
    "128k": MSAConfig("128k", N=131072, H_q=32, H_kv=4, d_h=128, d_idx=64, B_k=128, k=16,
                      structure="sink_ar1_retrieval", seed_index=2),
    # decode: 64 sequences of 131072 cached tokens, 256 appended steps
    "decode": DecodeConfig("decode", S=64, L0=131072, steps=1152, H_q=32, H_kv=4, d_h=128,
                           d_idx=64, B_k=128, k=16, seed_index=3),
    # the decode step at 8 sequences (2.3 GB of caches): a case small enough
    # for counter captures of the decode kernels
    "decode8": DecodeConfig("decode8", S=8, L0=131072, steps=256, H_q=32, H_kv=4, d_h=128,
                            d_idx=64, B_k=128, k=16, seed_index=5),
    # the decode workload on a paged FP8 (E4M3) cache (decode_fp8_state)
    "decode_fp8": DecodeConfig("decode_fp8", S=64, L0=131072, steps=1152, H_q=32, H_kv=4,
                               d_h=128, d_idx=64, B_k=128, k=16, seed_index=6),
    # the FP8 decode at 8 sequences (1.2 GB of pages): the case its kernels
    # are profiled on
    "decode_fp8_s8": DecodeConfig("decode_fp8_s8", S=8, L0=131072, steps=256, H_q=32, H_kv=4,
                                  d_h=128, d_idx=64, B_k=128, k=16, seed_index=7),
    # a packed batch of 32 prefill sequences, 131072 tokens in all, lengths
    # log-uniform in [512, 16384], pages' heads
    "varlen": VarlenConfig("varlen", n_seqs=32, N=131072, len_lo=512, len_hi=16384, H_q=32,
                           H_kv=4, d_h=128, d_idx=64, B_k=128, k=16, structure="sink_ar1",
                           seed_index=8),
    # 1M-token prefill with a strong sink (block 0 picked by >= 90% of rows)
    "1m": MSAConfig("1m", N=1048576, H_q=32, H_kv=4, d_h=128, d_idx=64, B_k=128, k=16,
                    structure="sink_ar1", sink_strength=3.0, seed_index=4),
}


def varlen_lengths(n_seqs: int, total: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """A seeded mix of n_seqs sequence lengths, log-uniform in [lo, hi] and
    rescaled to sum to ``total`` (the last one takes the rounding)."""
    r = np.random.default_rng(np.random.SeedSequence(seed + 901))
    x = np.exp(r.uniform(np.log(lo), np.log(hi), n_seqs))
    L = np.maximum(1, np.floor(x * total / x.sum())).astype(np.int64)
    L[-1] += total - L.sum()
    return L


def varlen_inputs(cfg: MSAConfig, lengths, seed: Optional[int] = None):
    """A packed batch: sequence s is ``prefill_inputs`` of cfg's heads and
    structure at N = lengths[s] (its own seed), the sequences concatenated
    along the token axis.  Returns (inputs, cu_seqlens int64 [n+1])."""
    lengths = [int(x) for x in lengths]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    base = cfg.seed if seed is None else seed
    parts = []
    for s, n in enumerate(lengths):
        if n == 0:
            continue
        sub = MSAConfig(f"{cfg.name}/{s}", n, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.B_k, cfg.k,
                        cfg.structure, cfg.sink_strength, cfg.seed_index)
        parts.append(prefill_inputs(sub, seed=base + 7919 * (s + 1)))
    out = {}
    for key, shape in (("q", (cfg.H_q, cfg.d_h)), ("k", (cfg.H_kv, cfg.d_h)),
                       ("v", (cfg.H_kv, cfg.d_h)), ("q_idx", (cfg.H_kv, cfg.d_idx)),
                       ("k_idx", (cfg.d_idx,))):
        out[key] = (np.concatenate([p[key] for p in parts]) if parts
                    else np.zeros((0,) + shape, np.uint16))
    return out, cu


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (finite input)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + r) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    out = np.empty(int(np.prod(shape)), dtype=np.uint16)
    for s in range(0, out.size, _CHUNK):
        e = min(out.size, s + _CHUNK)
        out[s:e] = bf16_bits(rng.standard_normal(e - s, dtype=np.float32))
    return out.reshape(shape)


def _normal_bf16_blocks(seq: np.random.SeedSequence, shape) -> np.ndarray:
    """i.i.d. N(0,1) as bf16 bits, drawn in blocks of _CHUNK elements, block j
    from its own stream seq.spawn(...)[j], so the blocks are drawn in
    parallel threads and the values do not depend on the thread count."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    starts = list(range(0, n, _CHUNK))
    seqs = seq.spawn(len(starts))

    def fill(j):
        s = starts[j]
        e = min(n, s + _CHUNK)
        out[s:e] = bf16_bits(np.random.default_rng(seqs[j]).standard_normal(e - s, dtype=np.float32))

    with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(len(starts))))
    return out.reshape(shape)


def _ar1(rng: np.random.Generator, n: int, c: int, rho: float) -> np.ndarray:
    """AR(1) along axis 0 with N(0,1) marginals: [n, c] float32."""
    from scipy.signal import lfilter

    out = np.empty((n, c), dtype=np.float32)
    a = math.sqrt(1.0 - rho * rho)
    step = max(1, _CHUNK // max(n, 1))
    for c0 in range(0, c, step):
        c1 = min(c, c0 + step)
        e = rng.standard_normal((n, c1 - c0))
        e[0, :] /= a  # so that x_0 = e_0 after the filter's a*e_0
        out[:, c0:c1] = lfilter([a], [1.0, -rho], e, axis=0).astype(np.float32)
    return out


def _unit(rng: np.random.Generator, d: int) -> np.ndarray:
    v = rng.standard_normal(d)
    return (v / np.linalg.norm(v)).astype(np.float32)


def prefill_inputs(cfg: MSAConfig, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """q [N,H_q,d_h], k/v [N,H_kv,d_h], q_idx [N,H_kv,d_idx], k_idx [N,d_idx] (bf16 bits)."""
    from concurrent.futures import ThreadPoolExecutor

    ss = np.random.SeedSequence(cfg.seed if seed is None else seed)
    s_q, s_k, s_v, s_qi, s_ki, s_s = ss.spawn(6)
    r_qi, r_ki, r_s = (np.random.default_rng(s) for s in (s_qi, s_ki, s_s))
    N, H_q, H_kv, d_h, d_idx = cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx
    if cfg.structure not in ("iid", "sink_ar1", "sink_ar1_retrieval"):
        raise ValueError(f"unknown structure {cfg.structure!r}")
    iid = cfg.structure == "iid"
    # the tensors draw from independent streams: generate them concurrently
    # (Q, K and V block by block, each block from its own stream)
    jobs = {
        "q": lambda: _normal_bf16_blocks(s_q, (N, H_q, d_h)),
        "k": lambda: _normal_bf16_blocks(s_k, (N, H_kv, d_h)),
        "v": lambda: _normal_bf16_blocks(s_v, (N, H_kv, d_h)),
        "qi": (lambda: _normal_bf16(r_qi, (N, H_kv, d_idx))) if iid
        else (lambda: _ar1(r_qi, N, H_kv * d_idx, 0.9).reshape(N, H_kv, d_idx)),
        "ki": (lambda: _normal_bf16(r_ki, (N, d_idx))) if iid
        else (lambda: _ar1(r_ki, N, d_idx, 0.9)),
    }
    with ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        futs = {name: ex.submit(fn) for name, fn in jobs.items()}
        res = {name: f.result() for name, f in futs.items()}
    out = {"q": res["q"], "k": res["k"], "v": res["v"]}
    if iid:
        out["q_idx"] = res["qi"]
        out["k_idx"] = res["ki"]
        return out
    qi, ki = res["qi"], res["ki"]
    u = _unit(r_s, d_idx)
    qi += cfg.sink_strength * u[None, None, :]
    ki[: min(N, cfg.B_k)] += (2.0 * math.sqrt(d_idx)) * u[None, :]
    if cfg.structure == "sink_ar1_retrieval":
        B = cfg.B
        if B >= 4:
            for r in range(H_kv):
                blocks = r_s.choice(np.arange(1, B - 1), size=min(8, B - 2), replace=False)
                for b in blocks:
                    v = _unit(r_s, d_idx)
                    j = int(b) * cfg.B_k + int(r_s.integers(0, cfg.B_k))
                    ki[j] += 2.0 * math.sqrt(d_idx) * v
                    later = np.arange((int(b) + 1) * cfg.B_k, N)
                    if later.size:
                        pick = later[r_s.random(later.size) < 0.125]
                        qi[pick, r, :] += 2.0 * v[None, :]
    out["q_idx"] = bf16_bits(qi)
    out["k_idx"] = bf16_bits(ki)
    return out


def decode_state(cfg: DecodeConfig, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Initial caches for the decode workload.

    k_cache/v_cache [S, L_max, H_kv, d_h], k_idx_cache [S, L_max, d_idx] with the
    first L0 rows filled (i.i.d. N(0,1), sink on block 0 of every sequence) and
    the rest zero; seq_len [S] int32 = L0; sink [S, d_idx] float32 (u per sequence).
    Every sequence has its own seeded streams, so sequences are generated in
    parallel threads.
    """
    from concurrent.futures import ThreadPoolExecutor

    ss = np.random.SeedSequence(cfg.seed if seed is None else seed)
    r_s = np.random.default_rng(ss.spawn(1)[0])
    per_seq = ss.spawn(1 + cfg.S)[1:]
    S, L0, Lm, H_kv, d_h, d_idx = cfg.S, cfg.L0, cfg.L_max, cfg.H_kv, cfg.d_h, cfg.d_idx
    k_cache = np.zeros((S, Lm, H_kv, d_h), dtype=np.uint16)
    v_cache = np.zeros((S, Lm, H_kv, d_h), dtype=np.uint16)
    k_idx_cache = np.zeros((S, Lm, d_idx), dtype=np.uint16)
    sink = np.stack([_unit(r_s, d_idx) for _ in range(S)])
    nb = min(L0, cfg.B_k)
    shift = 2.0 * math.sqrt(d_idx) * cfg.sink_strength

    def fill(s):
        r_k, r_v, r_ki = (np.random.default_rng(x) for x in per_seq[s].spawn(3))
        k_cache[s, :L0] = _normal_bf16(r_k, (L0, H_kv, d_h))
        v_cache[s, :L0] = _normal_bf16(r_v, (L0, H_kv, d_h))
        ki = r_ki.standard_normal((L0, d_idx), dtype=np.float32)
        ki[:nb] += shift * sink[s][None, :]
        k_idx_cache[s, :L0] = bf16_bits(ki)

    import os

    with ThreadPoolExecutor(max_workers=min(S, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(S)))
    return {"k_cache": k_cache, "v_cache": v_cache, "k_idx_cache": k_idx_cache,
            "seq_len": np.full(S, L0, dtype=np.int32), "sink": sink}


def decode_step_inputs(cfg: DecodeConfig, step: int, sink: np.ndarray,
                       seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """New rows of one decode step: q [S,H_q,d_h], q_idx [S,H_kv,d_idx] (+ sink u),
    k_new/v_new [S,H_kv,d_h], k_idx_new [S,d_idx]; i.i.d. N(0,1)."""
    base = cfg.seed if seed is None else seed
    ss = np.random.SeedSequence([base, 1 + step])
    r_q, r_qi, r_k, r_v, r_ki = (np.random.default_rng(s) for s in ss.spawn(5))
    S, H_q, H_kv, d_h, d_idx = cfg.S, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx
    qi = r_qi.standard_normal((S, H_kv, d_idx), dtype=np.float32) + sink[:, None, :]
    return {
        "q": _normal_bf16(r_q, (S, H_q, d_h)),
        "q_idx": bf16_bits(qi),
        "k_new": _normal_bf16(r_k, (S, H_kv, d_h)),
        "v_new": _normal_bf16(r_v, (S, H_kv, d_h)),
        "k_idx_new": _normal_bf16(r_ki, (S, d_idx)),
    }


def decode_fp8_state(cfg: DecodeConfig, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """A paged FP8 (E4M3) decode cache drawn directly as codes and scales.

    Pages hold B_k tokens; page_table [S, n_blocks] is a seeded random
    permutation of the n_pages = S * n_blocks pages (n_blocks = L_max / B_k,
    rounded up), so every sequence's blocks are scattered over the pool.
    Codes are uniform over the E4M3 bit patterns whose exponent field is at
    most 9 (magnitude below 8, no NaN) with a random sign; scales are uniform
    in [0.05, 0.15).  Sink: the index keys of every sequence's block 0 carry
    the exponent-6 code 0x30 (value 0.5) with the sign of the sequence's unit
    vector u, and scale 0.6, so index queries drawn around u score block 0
    high.  Only the first L0 tokens are meaningful; seq_len = L0.
    Returns k_pages/v_pages [P,B_k,H_kv,d_h] uint8, k_scale/v_scale
    [P,B_k,H_kv] float32, kidx_pages [P,B_k,d_idx] uint8, kidx_scale [P,B_k]
    float32, page_table [S,n_blocks] int32, seq_len [S] int32, sink [S,d_idx].
    """
    import os
    from concurrent.futures import ThreadPoolExecutor

    ss = np.random.SeedSequence((cfg.seed if seed is None else seed) + 77)
    s_pt, s_k, s_v, s_ki, s_sc, s_sink = ss.spawn(6)
    S, B_k, H_kv, d_h, d_idx = cfg.S, cfg.B_k, cfg.H_kv, cfg.d_h, cfg.d_idx
    n_blocks = (cfg.L_max + B_k - 1) // B_k
    P = S * n_blocks
    page_table = np.random.default_rng(s_pt).permutation(P).astype(np.int32).reshape(S, n_blocks)

    def codes(seq, shape):
        n = int(np.prod(shape))
        out = np.empty(n, dtype=np.uint8)
        starts = list(range(0, n, _CHUNK))
        kids = seq.spawn(len(starts))

        def fill(j):
            a, b = starts[j], min(n, starts[j] + _CHUNK)
            r = np.random.default_rng(kids[j])
            out[a:b] = (r.integers(0, 0x50, b - a, dtype=np.uint8)
                        | (r.integers(0, 2, b - a, dtype=np.uint8) << 7))

        with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(len(starts))))
        return out.reshape(shape)

    r_sc = np.random.default_rng(s_sc)
    out = {
        "k_pages": codes(s_k, (P, B_k, H_kv, d_h)),
        "v_pages": codes(s_v, (P, B_k, H_kv, d_h)),
        "kidx_pages": codes(s_ki, (P, B_k, d_idx)),
        "k_scale": r_sc.uniform(0.05, 0.15, (P, B_k, H_kv)).astype(np.float32),
        "v_scale": r_sc.uniform(0.05, 0.15, (P, B_k, H_kv)).astype(np.float32),
        "kidx_scale": r_sc.uniform(0.05, 0.15, (P, B_k)).astype(np.float32),
        "page_table": page_table,
        "seq_len": np.full(S, cfg.L0, dtype=np.int32),
    }
    r_sink = np.random.default_rng(s_sink)
    sink = np.stack([_unit(r_sink, d_idx) for _ in range(S)])
    sign = (sink < 0).astype(np.uint8) << 7
    for s_ in range(S):
        pg = page_table[s_, 0]
        out["kidx_pages"][pg] = (0x30 | sign[s_])[None, :]
        out["kidx_scale"][pg] = np.float32(0.6)
    out["sink"] = sink
    return out


def zipf_indices(N: int, H_kv: int, B_k: int, k: int, p_sink: float = 0.9,
                 alpha: float = 1.1, seed: int = SEED_BASE + 5,
                 rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Synthetic block selections shaped like a sink-skewed index branch.

    Per (row i, group r): the local block b_i; block 0 with probability p_sink
    (when b_i > 0); the remaining slots drawn without replacement from
    {1..b_i-1} with P(b) proportional to (b_i - b)^-alpha.  Ascending, -1
    padded.  Returns int32 [len(rows), H_kv, k] (rows default: all N).
    """
    rng = np.random.default_rng(seed)
    rows = np.arange(N) if rows is None else np.asarray(rows)
    out = np.full((rows.size, H_kv, k), -1, dtype=np.int32)
    for t, i in enumerate(rows):
        b_i = int(i) // B_k
        for r in range(H_kv):
            sel = [b_i]
            if b_i > 0 and k > 1 and rng.random() < p_sink:
                sel.append(0)
            cand = np.arange(1, b_i)
            need = min(k - len(sel), cand.size)
            if need > 0:
                w = (b_i - cand).astype(np.float64) ** (-alpha)
                pick = rng.choice(cand, size=need, replace=False, p=w / w.sum())
                sel.extend(int(x) for x in pick)
            sel.sort()
            out[t, r, : len(sel)] = sel
    return out
