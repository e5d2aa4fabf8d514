"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

None of these tests compare the oracle with a retyped copy of itself: each
expected value comes from a hand-built case (tests/golden), a closed form,
brute-force enumeration, a library routine (numpy argsort, torch's
scaled_dot_product_attention) or an invariant of the definitions.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_idx_b200 import inputs
from tests import compare

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(x) -> np.ndarray:
    return inputs.bf16_bits(np.asarray(x, dtype=np.float32))


def _f32(bits) -> np.ndarray:
    return inputs.bf16_to_f32(bits)


def _rand_case(seed, N, H_q, H_kv, d_h, d_idx):
    rng = np.random.default_rng(seed)
    return {
        "q": _bits(rng.standard_normal((N, H_q, d_h))),
        "k": _bits(rng.standard_normal((N, H_kv, d_h))),
        "v": _bits(rng.standard_normal((N, H_kv, d_h))),
        "q_idx": _bits(rng.standard_normal((N, H_kv, d_idx))),
        "k_idx": _bits(rng.standard_normal((N, d_idx))),
    }


# ---------------------------------------------------------------- Eq. 6-7 --

def _load_planted():
    xs = ys = None
    rows = []
    with open(os.path.join(GOLDEN, "planted_selection.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "x":
                xs = [float(t) for t in tok[1:]]
            elif tok[0] == "y":
                ys = [float(t) for t in tok[1:]]
            else:
                rows.append([int(t) for t in tok])
    return np.array(xs), np.array(ys), np.array(rows)


def test_planted_selection_matches_hand_derivation():
    xs, ys, table = _load_planted()
    N, B_k, k, H_kv = 24, 4, 3, 2
    k_idx = _bits(np.stack([xs, ys], axis=1))
    q_idx = _bits(np.tile(np.array([[1.0, 0.0], [0.0, 1.0]]), (N, 1, 1)))
    idx, _, _ = oracle.index_topk(q_idx, k_idx, B_k, k)
    for i, r, *expect in table:
        assert idx[i, r].tolist() == expect, (i, r)
    # Eq. 6's scale: the max-pooled score of block b is (its max value)/sqrt(d_idx)
    M = oracle.block_scores(q_idx[23, 0], k_idx, B_k, 23)
    np.testing.assert_allclose(M, np.array([5, 2, 7, 1, 5, 3]) / math.sqrt(2), rtol=1e-15)
    # a negated index query reverses the ranking (ties still go to the lower block)
    idx_neg, _, _ = oracle.index_topk(_bits(-_f32(q_idx)), k_idx, B_k, k, rows=np.array([20]))
    # group 0 with -x: block minima -> scores -min(x): b0=0, b1=1, b2=0, b3=3, b4=1
    assert idx_neg[0, 0].tolist() == [1, 3, 5]


def test_causal_rule_inside_block_scores():
    """Eq. 6: tokens after i do not enter M; a future spike must be invisible."""
    N, B_k, d = 16, 8, 2
    k_idx = np.zeros((N, d), dtype=np.float32)
    k_idx[:, 0] = 0.5
    k_idx[13, 0] = 100.0  # future for i = 10, visible for i = 14
    q = _bits([1.0, 0.0])
    kb = _bits(k_idx)
    s = 1 / math.sqrt(d)
    assert oracle.block_scores(q, kb, B_k, 10)[1] == pytest.approx(0.5 * s, rel=1e-15)
    assert oracle.block_scores(q, kb, B_k, 14)[1] == pytest.approx(100.0 * s, rel=1e-15)


def test_block_scores_against_numpy_library_path():
    """Independent library computation (numpy matmul + masked max) of Eq. 6."""
    inp = _rand_case(1, 200, 4, 2, 16, 8)
    qf, kf = _f32(inp["q_idx"]).astype(np.float64), _f32(inp["k_idx"]).astype(np.float64)
    B_k = 16
    for i in (0, 15, 16, 77, 199):
        for r in range(2):
            S = (kf[: i + 1] @ qf[i, r]) / math.sqrt(8)
            ref = np.array([S[b * B_k: min((b + 1) * B_k, i + 1)].max()
                            for b in range(i // B_k + 1)])
            got = oracle.block_scores(inp["q_idx"][i, r], inp["k_idx"], B_k, i)
            np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def _brute_force(M32: np.ndarray, b_i: int, k: int):
    """Enumerate every candidate set; return the unique one where each kept
    non-local block precedes each dropped visible block in the order
    (score desc, block asc)."""
    others = list(range(b_i))
    size = min(k - 1, len(others))
    found = []
    for sub in itertools.combinations(others, size):
        dropped = [b for b in others if b not in sub]
        ok = all((M32[a] > M32[d]) or (M32[a] == M32[d] and a < d)
                 for a in sub for d in dropped)
        if ok:
            found.append(sorted(list(sub) + [b_i]))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(12))
def test_selection_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    B_k = int(rng.choice([4, 8]))
    N = int(rng.integers(1, 12 * B_k + 1))
    k = int(rng.integers(1, 6))
    d_idx = int(rng.choice([2, 4, 8]))
    inp = _rand_case(seed, N, 2, 2, 4, d_idx)
    if seed % 3 == 0:  # coarse values force exact ties
        inp["q_idx"] = _bits(np.round(_f32(inp["q_idx"])))
        inp["k_idx"] = _bits(np.round(_f32(inp["k_idx"])))
    idx, _, _ = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, k)
    for i in range(N):
        for r in range(2):
            M32 = oracle.block_scores(inp["q_idx"][i, r], inp["k_idx"], B_k, i).astype(np.float32)
            expect = _brute_force(M32, i // B_k, k)
            expect += [-1] * (k - len(expect))
            assert idx[i, r].tolist() == expect, (seed, i, r)


@pytest.mark.parametrize("seed", range(4))
def test_selection_numpy_stable_argsort(seed):
    """Library pin: stable argsort with the local block forced to +inf."""
    cfg = inputs.CONFIGS["tiny"]
    inp = _rand_case(seed, 700, 4, 2, 8, 16)
    B_k, k = 32, 5
    rows = np.array([0, 31, 32, 100, 255, 256, 511, 699])
    idx, _, _ = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, k, rows=rows)
    del cfg
    for t, i in enumerate(rows):
        for r in range(2):
            b_i = i // B_k
            M32 = oracle.block_scores(inp["q_idx"][i, r], inp["k_idx"], B_k, i).astype(np.float32)
            key = M32.astype(np.float64)
            key[b_i] = np.inf
            order = np.argsort(-key, kind="stable")[: min(k, b_i + 1)]
            expect = sorted(order.tolist()) + [-1] * (k - min(k, b_i + 1))
            assert idx[t, r].tolist() == expect


def test_selection_invariances():
    inp = _rand_case(7, 1000, 4, 2, 8, 16)
    B_k, k = 32, 6
    idx, _, _ = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, k)
    # order preservation (xllm-io review 4.1; chlience 5.4): a positive
    # rescale of the index queries (x2 is exact in bf16) keeps every set
    idx2, _, _ = oracle.index_topk(_bits(2 * _f32(inp["q_idx"])), inp["k_idx"], B_k, k)
    assert np.array_equal(idx, idx2)
    # the local block is always selected (Eq. 7 note; chlience 5.1.1)
    for i in range(1000):
        assert (idx[i] == i // B_k).any(axis=1).all()
    # k >= number of blocks: every visible block is selected
    B = (1000 + B_k - 1) // B_k
    idx_all, _, _ = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, B)
    for i in (0, 31, 32, 500, 999):
        for r in range(2):
            assert idx_all[i, r].tolist() == list(range(i // B_k + 1)) + [-1] * (B - i // B_k - 1)


def test_tie_band_outputs():
    xs, ys, _ = _load_planted()
    k_idx = _bits(np.stack([xs, ys], axis=1))
    q_idx = _bits(np.tile(np.array([[1.0, 0.0], [0.0, 1.0]]), (24, 1, 1)))
    _, cut, nxt = oracle.index_topk(q_idx, k_idx, 4, 3, rows=np.array([20, 4]))
    # row 20 group 0: kept b2 (7), b0 (5); best left out b4 (5): an exact tie
    assert cut[0, 0] == pytest.approx(5 / math.sqrt(2)) and nxt[0, 0] == cut[0, 0]
    # row 4: a single non-local candidate, kept; nothing left out
    assert math.isnan(nxt[1, 0]) and cut[1, 0] == pytest.approx(5 / math.sqrt(2))


def test_comparator_catches_planted_mistake():
    """A wrong block planted into a copy of the oracle's answer must fail."""
    inp = _rand_case(3, 512, 4, 2, 8, 16)
    B_k, k = 32, 4
    idx, cut, nxt = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, k)
    rows = np.arange(512)
    ok = compare.check_topk(idx, idx, cut, nxt, rows, B_k, k)
    assert ok[2] == [] and ok[0] == 512 * 2
    bad = idx.copy()
    i = 400
    sel = set(bad[i, 0].tolist())
    swap = next(b for b in range(i // B_k) if b not in sel)
    victim = next(b for b in bad[i, 0] if b != i // B_k)
    bad[i, 0] = sorted((sel - {victim}) | {swap})
    res = compare.check_topk(bad, idx, cut, nxt, rows, B_k, k,
                             q_idx_rows=inp["q_idx"], k_idx=inp["k_idx"])
    assert len(res[2]) == 1 and res[2][0][0] == i
    # a dropped local block is invalid whatever the scores
    bad2 = idx.copy()
    bad2[300, 1] = [0, 1, 2, 3]
    assert not compare.valid_selection(bad2[300, 1], 300, B_k, k)


# ------------------------------------------------------------------ Eq. 8 --

def _sdpa(q, k, v, mask=None, causal=False):
    qt = torch.from_numpy(_f32(q).astype(np.float64)).permute(1, 0, 2)[None]
    kt = torch.from_numpy(_f32(k).astype(np.float64)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(_f32(v).astype(np.float64)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=mask, is_causal=causal, enable_gqa=True)
    return o[0].permute(1, 0, 2).numpy()


def test_dense_equivalence_with_library_sdpa():
    """k*B_k >= N: every visible block is selected, so Eq. 8 = Eq. 1 = SDPA."""
    N, H_q, H_kv, d_h, B_k = 300, 8, 2, 16, 32
    inp = _rand_case(11, N, H_q, H_kv, d_h, 8)
    B = (N + B_k - 1) // B_k
    rows = np.arange(N)
    idx, _, _ = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, B)
    o_sp, lse_sp = oracle.sparse_attn(inp["q"], inp["k"], inp["v"], idx, B_k, rows)
    o_de, lse_de = oracle.dense_attn(inp["q"], inp["k"], inp["v"], rows)
    ref = _sdpa(inp["q"], inp["k"], inp["v"], causal=True)
    np.testing.assert_allclose(o_sp, ref, atol=1e-10)
    np.testing.assert_allclose(o_de, ref, atol=1e-10)
    np.testing.assert_allclose(lse_sp, lse_de, atol=1e-12)


def test_local_only_is_block_causal_attention():
    """k = 1: only the local block -> SDPA with a block-diagonal causal mask."""
    N, H_q, H_kv, d_h, B_k = 200, 4, 2, 8, 16
    inp = _rand_case(12, N, H_q, H_kv, d_h, 8)
    rows = np.arange(N)
    idx, _, _ = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, 1)
    assert (idx[:, :, 0] == (rows // B_k)[:, None]).all()
    o, _ = oracle.sparse_attn(inp["q"], inp["k"], inp["v"], idx, B_k, rows)
    i = rows[:, None]
    j = rows[None, :]
    mask = torch.from_numpy((j <= i) & (j // B_k == i // B_k))
    np.testing.assert_allclose(o, _sdpa(inp["q"], inp["k"], inp["v"], mask=mask), atol=1e-10)


def test_weights_sum_to_one_and_lse_identity():
    """Eq. 8: sum_j exp(s_j - LSE) over the selected tokens is 1."""
    N, H_q, H_kv, d_h, B_k, k = 500, 8, 2, 32, 32, 4
    inp = _rand_case(13, N, H_q, H_kv, d_h, 16)
    rows = np.array([0, 33, 250, 499])
    idx, _, _ = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, k, rows=rows)
    _, lse = oracle.sparse_attn(inp["q"][rows], inp["k"], inp["v"], idx, B_k, rows, N=N)
    qf = _f32(inp["q"]).astype(np.float64)
    kf = _f32(inp["k"]).astype(np.float64)
    for t, i in enumerate(rows):
        for h in range(H_q):
            r = h // (H_q // H_kv)
            toks = [j for b in idx[t, r] if b >= 0
                    for j in range(b * B_k, min((b + 1) * B_k, N)) if j <= i]
            s = kf[toks, r] @ qf[i, h] / math.sqrt(d_h)
            assert np.exp(s - lse[t, h]).sum() == pytest.approx(1.0, abs=1e-12)


def test_split_merge_identity():
    """The two-phase forward's merge (xllm-io review 4.2, chlience 5.4): the
    LSE-weighted merge of partial results over disjoint block subsets equals
    attention over their union."""
    N, H_q, H_kv, d_h, B_k, k = 640, 4, 2, 16, 32, 6
    inp = _rand_case(14, N, H_q, H_kv, d_h, 8)
    rows = np.array([300, 639])
    idx, _, _ = oracle.index_topk(inp["q_idx"], inp["k_idx"], B_k, k, rows=rows)
    o, lse = oracle.sparse_attn(inp["q"][rows], inp["k"], inp["v"], idx, B_k, rows, N=N)
    rng = np.random.default_rng(0)
    part = rng.random(idx.shape) < 0.5
    a = np.where(part, idx, -1)
    b = np.where(~part, idx, -1)
    # make sure each row/group has something in both halves
    a[..., 0] = idx[..., 0]
    b[..., 0] = -1
    b[..., -1] = idx[..., -1]
    a[..., -1] = -1
    oa, la = oracle.sparse_attn(inp["q"][rows], inp["k"], inp["v"], a, B_k, rows, N=N)
    ob, lb = oracle.sparse_attn(inp["q"][rows], inp["k"], inp["v"], b, B_k, rows, N=N)
    m = np.maximum(la, lb)
    wa, wb = np.exp(la - m), np.exp(lb - m)
    merged = (wa[..., None] * oa + wb[..., None] * ob) / (wa + wb)[..., None]
    np.testing.assert_allclose(merged, o, atol=1e-12)
    np.testing.assert_allclose(m + np.log(wa + wb), lse, atol=1e-12)


# ----------------------------------------------------------------- Eq. 12 --

def test_eq12_reproduces_printed_ratio():
    with open(os.path.join(GOLDEN, "eq12_flop_ratio.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            N, H_q, H_kv, d_h, d_idx, B_k, k, printed = line.split()
            f12 = oracle.flops(float(N), int(H_q), int(H_kv), int(d_h), int(d_idx), int(B_k),
                               int(k))
            assert round(f12["ratio"], 1) == float(printed)
    # closed form at the 32K..1M prefill shapes (H_q=32, d_idx=64): 8192 N / (256 N + 2^25)
    for N, expect in ((32768, 6.4), (131072, 16.0), (1048576, 28.444444444444443)):
        f12 = oracle.flops(N, 32, 4, 128, 64, 128, 16)
        assert f12["ratio"] == pytest.approx(expect, rel=1e-12)


# ----------------------------------------------------------------- decode --

def test_decode_equals_last_prefill_row():
    """A decode step (append, then attend from the new token) is the last row
    of a prefill over the extended sequence (Eq. 1: i <= t)."""
    cfg = inputs.DecodeConfig("mini", S=2, L0=300, steps=2, H_q=4, H_kv=2, d_h=16, d_idx=8,
                              B_k=32, k=3)
    st = inputs.decode_state(cfg)
    step = inputs.decode_step_inputs(cfg, 0, st["sink"])
    dec = oracle.decode_reference(st, step, cfg.B_k, cfg.k)
    for s in range(2):
        L = 300
        full = {
            "q": np.concatenate([np.zeros((L, 4, 16), np.uint16), step["q"][s][None]]),
            "k": np.concatenate([st["k_cache"][s, :L], step["k_new"][s][None]]),
            "v": np.concatenate([st["v_cache"][s, :L], step["v_new"][s][None]]),
            "q_idx": np.concatenate([np.zeros((L, 2, 8), np.uint16), step["q_idx"][s][None]]),
            "k_idx": np.concatenate([st["k_idx_cache"][s, :L], step["k_idx_new"][s][None]]),
        }
        ref = oracle.forward(full, cfg.B_k, cfg.k, rows=np.array([L]))
        assert dec["idx"][s].tolist() == ref["idx"][0].tolist()
        np.testing.assert_allclose(dec["o"][s], ref["o"][0], atol=0)


# ------------------------------------------ KL-loss fusion: LSE_idx (Eq. 9) --

def test_index_lse_worked_example():
    """Hand-worked Eq. 9 normaliser: q = (1, 0), keys (0,0), (1,0), (2,0),
    (5,0) in one block of 4, query at i = 2, scale 1: the causal set is
    tokens 0..2 with scores 0, 1, 2, so LSE_idx = log(1 + e + e^2); token 3
    (score 5) must not count."""
    q = inputs.bf16_bits(np.array([[[1, 0]]], dtype=np.float32))
    k = inputs.bf16_bits(np.array([[0, 0], [1, 0], [2, 0], [5, 0]], dtype=np.float32))
    got = oracle.index_lse(q, k, np.array([[[0]]], np.int32), B_k=4, rows=np.array([2]),
                           scale=1.0)
    assert got[0, 0] == pytest.approx(math.log(1 + math.e + math.e ** 2), rel=1e-15)


def test_index_lse_equal_keys_closed_form():
    """Every selected key equal to one vector c: each token scores s = <q, c> *
    scale, so LSE_idx = s + log(number of selected tokens j <= i), with -1
    slots skipped, the query's own block cut at j = i and a ragged last block."""
    rng = np.random.default_rng(5)
    N, H_kv, d_idx, B_k, k = 300, 2, 8, 64, 3  # blocks 0..4, the last holds 44 tokens
    c = rng.standard_normal(d_idx).astype(np.float32)
    k_idx = np.tile(inputs.bf16_bits(c), (N, 1))
    q = inputs.bf16_bits(rng.standard_normal((4, H_kv, d_idx)).astype(np.float32))
    rows = np.array([5, 130, 299, 263])
    idx = np.array([[[0, -1, -1], [0, -1, -1]],
                    [[0, 2, -1], [1, 2, -1]],
                    [[0, 3, 4], [4, -1, -1]],
                    [[1, 4, -1], [2, 3, 4]]], np.int32)
    got = oracle.index_lse(q, k_idx, idx, B_k, rows, N=N)
    cw = k_idx[0].astype(np.uint32) << 16
    cf = cw.view(np.float32).astype(np.float64)
    for t, i in enumerate(rows):
        for r in range(H_kv):
            qf = (q[t, r].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            s = float(qf @ cf) / math.sqrt(d_idx)
            n = 0
            for b in idx[t, r]:
                if b >= 0:
                    n += max(0, min(b * B_k + B_k, N, i + 1) - b * B_k)
            assert got[t, r] == pytest.approx(s + math.log(n), abs=1e-12)


def test_index_lse_empty_set_and_bounds():
    """No selected token gives -inf; otherwise max S <= LSE_idx <= max S + log n."""
    cfg = inputs.CONFIGS["tiny"]
    inp = inputs.prefill_inputs(cfg)
    rows = np.array([0, 63, 64, 700, 2047])
    sel = oracle.index_topk(inp["q_idx"], inp["k_idx"], cfg.B_k, cfg.k, rows=rows)[0]
    got = oracle.index_lse(inp["q_idx"][rows], inp["k_idx"], sel, cfg.B_k, rows)
    empty = np.full_like(sel, -1)
    assert np.isneginf(oracle.index_lse(inp["q_idx"][rows], inp["k_idx"], empty, cfg.B_k,
                                        rows)).all()
    qf = (inp["q_idx"][rows].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    kf = (inp["k_idx"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for t, i in enumerate(rows):
        for r in range(cfg.H_kv):
            toks = [j for b in sel[t, r] if b >= 0
                    for j in range(b * cfg.B_k, min(b * cfg.B_k + cfg.B_k, cfg.N)) if j <= i]
            s = kf[toks] @ qf[t, r] / math.sqrt(cfg.d_idx)
            assert s.max() - 1e-12 <= got[t, r] <= s.max() + math.log(len(toks)) + 1e-12


def test_index_lse_is_a_one_head_attention_lse():
    """Eq. 9's index distribution is an attention over the selected tokens with
    Q = q_idx and K = K_idx, so its normaliser equals the LSE the (separately
    written) Eq. 8 routine returns for one head of dimension d_idx."""
    cfg = inputs.CONFIGS["tiny"]
    inp = inputs.prefill_inputs(cfg)
    rows = np.array([1, 100, 600, 1500, 2047])
    sel = oracle.index_topk(inp["q_idx"], inp["k_idx"], cfg.B_k, cfg.k, rows=rows)[0]
    got = oracle.index_lse(inp["q_idx"][rows], inp["k_idx"], sel, cfg.B_k, rows)
    kv = inp["k_idx"][:, None, :]
    for r in range(cfg.H_kv):
        _, lse = oracle.sparse_attn(inp["q_idx"][rows][:, r:r + 1, :], kv, kv,
                                    sel[:, r:r + 1, :], cfg.B_k, rows,
                                    scale=1.0 / math.sqrt(cfg.d_idx))
        np.testing.assert_allclose(got[:, r], lse[:, 0], rtol=0, atol=1e-12)
