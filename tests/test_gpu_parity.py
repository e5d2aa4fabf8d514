"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Top-k sets must match exactly except inside the stated tie band; attention
outputs are compared from the GPU-chosen selection fed to both sides
(max-abs <= 2e-2, mean-abs <= 2e-3, LSE within 1e-3).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_idx_b200 import inputs
from tests import compare
from tests.gpu_util import bf16_to_f64, dev_inputs, prefill_inputs_cached, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_gqa_idx_b200 as m

    return m


def _cfg(name, **kw):
    import dataclasses

    return dataclasses.replace(inputs.CONFIGS[name], **kw)


# Outputs are poisoned before every call (NaN for O, LSE and block scores, -7
# for the selection), so a row the kernels never write fails the comparison.
SENTINEL = -7


def _index(msa, dev, cfg, scores=False):
    N = dev["q_idx"].shape[0]
    idx = torch.full((N, cfg.H_kv, cfg.k), SENTINEL, dtype=torch.int32, device="cuda")
    sc = (torch.full((N, cfg.H_kv, cfg.k), float("nan"), dtype=torch.float32, device="cuda")
          if scores else None)
    msa.index_topk(dev["q_idx"], dev["k_idx"], cfg.B_k, cfg.k, idx_out=idx, score_out=sc)
    torch.cuda.synchronize()
    return (idx, sc) if scores else idx


def _attn(msa, dev, idx_dev, B_k):
    N, H_q, d_h = dev["q"].shape
    o = torch.full((N, H_q, d_h), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((N, H_q), float("nan"), dtype=torch.float32, device="cuda")
    msa.sparse_attn_fwd(dev["q"], dev["k"], dev["v"], idx_dev, B_k, o=o, lse=lse)
    torch.cuda.synchronize()
    return o, lse


def structured_rows(cfg, gidx=None, extra=(), per_group=16):
    """Every row of blocks 0, 1, B/2 and B-1, plus (given the selection) the
    first and the last `per_group` queries of each group that selected block
    0 -- the hot list that the tile schedule splits the most."""
    B_k, N, B = cfg.B_k, cfg.N, cfg.B
    parts = [np.arange(b * B_k, min((b + 1) * B_k, N)) for b in sorted({0, 1, B // 2, B - 1})
             if b * B_k < N]
    if gidx is not None:
        for r in range(cfg.H_kv):
            hot = np.nonzero((gidx[:, r, :] == 0).any(axis=1))[0]
            parts += [hot[:per_group], hot[-per_group:]]
    parts.append(np.asarray(extra, dtype=np.int64))
    return np.unique(np.concatenate(parts).astype(np.int64))


def _check_scores(sc, gidx, inp, cfg, rows):
    """score_out of the sampled rows against the oracle's block scores, within
    the tie band's 1e-3 relative tolerance; -inf in the -1 slots."""
    for i in rows:
        for r in range(cfg.H_kv):
            M = oracle.block_scores(inp["q_idx"][i, r], inp["k_idx"], cfg.B_k, int(i))
            for s_ in range(cfg.k):
                b = int(gidx[i, r, s_])
                got = float(sc[i, r, s_])
                if b < 0:
                    assert got == -np.inf, (i, r, s_, got)
                else:
                    assert abs(got - M[b]) <= compare._band(got, M[b]), (i, r, s_, b, got, M[b])


def _check_index(msa, cfg, rows=None, seed=None, score_rows=None):
    inp = prefill_inputs_cached(cfg, seed)
    dev = dev_inputs(inp)
    idx, sc = _index(msa, dev, cfg, scores=True)
    gidx = idx.cpu().numpy()
    rows = np.arange(cfg.N) if rows is None else np.asarray(rows)
    ref, cut, nxt = oracle.index_topk(inp["q_idx"], inp["k_idx"], cfg.B_k, cfg.k, rows=rows)
    exact, band, fails = compare.check_topk(gidx[rows], ref, cut, nxt, rows, cfg.B_k, cfg.k,
                                            q_idx_rows=inp["q_idx"][rows], k_idx=inp["k_idx"])
    assert not fails, f"{cfg.name}: {len(fails)} mismatching rows, e.g. {fails[:3]}"
    assert exact + band == rows.size * cfg.H_kv
    _check_scores(sc.cpu().numpy(), gidx, inp, cfg, rows if score_rows is None else score_rows)
    return inp, dev, gidx, exact, band


def test_index_topk_tiny_all_rows(msa):
    cfg = inputs.CONFIGS["tiny"]
    _, _, _, exact, band = _check_index(msa, cfg)
    assert band <= 2  # i.i.d. N(0,1) scores: ties in fp32 are essentially absent


def test_index_topk_32k_full(msa):
    """The 32K workload at its full length: every row of blocks 0, 1, B/2,
    B-1, the ends of each group's block-0 list and random rows."""
    cfg = inputs.CONFIGS["32k"]
    inp = prefill_inputs_cached(cfg)
    gidx = _index(msa, dev_inputs(inp), cfg).cpu().numpy()
    rng = np.random.default_rng(4)
    rows = structured_rows(cfg, gidx, extra=rng.integers(0, cfg.N, 64))
    _check_index(msa, cfg, rows=rows, score_rows=rows[::8])


@pytest.mark.parametrize("N,H_kv,d_idx,B_k,k", [
    (1000, 2, 32, 64, 5),     # ragged tail, B_k=64 (two blocks per key tile)
    (3001, 4, 128, 128, 32),  # largest k, d_idx=128 (two swizzle chunks)
    (777, 8, 64, 128, 3),     # H_kv=8 (16 queries per M-tile)
    (200, 1, 64, 128, 4),     # H_kv=1 (128 queries per M-tile)
    (130, 4, 64, 128, 16),    # fewer visible blocks than k everywhere
    (2048, 4, 64, 64, 1),     # k = 1: local block only
])
def test_index_topk_edge_shapes(msa, N, H_kv, d_idx, B_k, k):
    cfg = inputs.MSAConfig("edge", N=N, H_q=H_kv * 2, H_kv=H_kv, d_h=64, d_idx=d_idx, B_k=B_k,
                           k=k, structure="iid", seed_index=17)
    _check_index(msa, cfg)


def test_index_topk_exact_ties_go_to_lower_blocks(msa):
    """Every block's K_idx rows identical: all block maxima tie exactly (the
    same bf16 products in the same order), so Eq. 7's ties-to-the-lower-index
    rule fixes each row's selection bit-exactly: its own block and blocks
    0 .. k-2 (or every visible block when there are fewer)."""
    N, H_kv, d_idx, B_k, k = 4096, 4, 64, 128, 6
    rng = np.random.default_rng(11)
    q_idx = inputs.bf16_bits(rng.standard_normal((N, H_kv, d_idx), dtype=np.float32))
    block = inputs.bf16_bits(rng.standard_normal((B_k, d_idx), dtype=np.float32))
    k_idx = np.tile(block, (N // B_k, 1))
    idx = msa.index_topk(to_dev(q_idx), to_dev(k_idx), B_k, k)
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    for i in range(N):
        b_i = i // B_k
        want = sorted(set(range(min(k - 1, b_i))) | {b_i})
        want = want + [-1] * (k - len(want))
        assert (got[i] == np.array(want)[None, :]).all(), (i, got[i].tolist(), want)
    ref = oracle.index_topk(q_idx, k_idx, B_k, k, rows=np.arange(0, N, 37))[0]
    assert (ref == got[np.arange(0, N, 37)]).all()


def test_index_topk_128k_sampled(msa):
    """Full 128K workload (same launch as the benchmark): every row of blocks
    0, 1, B/2, B-1, the ends of each group's block-0 list and random rows."""
    cfg = inputs.CONFIGS["128k"]
    inp = prefill_inputs_cached(cfg)
    gidx = _index(msa, dev_inputs(inp), cfg).cpu().numpy()
    rng = np.random.default_rng(0)
    rows = structured_rows(cfg, gidx, extra=np.concatenate([
        rng.integers(0, cfg.N, 48), [4095, cfg.N // 2, cfg.N - 129]]))
    _check_index(msa, cfg, rows=rows, score_rows=rows[::16])


def _check_attn(msa, inp, dev, idx_dev, cfg, rows, what):
    o, lse = _attn(msa, dev, idx_dev, cfg.B_k)
    rows = np.asarray(rows)
    idx_rows = idx_dev.cpu().numpy()[rows]
    ro, rlse = oracle.sparse_attn(inp["q"][rows], inp["k"], inp["v"], idx_rows, cfg.B_k, rows,
                                  N=cfg.N)
    go = bf16_to_f64(o)[rows]
    gl = lse.cpu().numpy().astype(np.float64)[rows]
    compare.assert_attn_close(go, ro, gl, rlse, what=what)


def test_attention_tiny_all_rows(msa):
    cfg = inputs.CONFIGS["tiny"]
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = _index(msa, dev, cfg)
    _check_attn(msa, inp, dev, idx, cfg, np.arange(cfg.N), "tiny")


def test_attention_32k_full(msa):
    """The 32K workload at its full length: every row of blocks 0, 1, B/2,
    B-1, the ends of each group's block-0 list and random rows."""
    cfg = inputs.CONFIGS["32k"]
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = _index(msa, dev, cfg)
    rng = np.random.default_rng(1)
    rows = structured_rows(cfg, idx.cpu().numpy(), extra=rng.integers(0, cfg.N, 400))
    _check_attn(msa, inp, dev, idx, cfg, rows, "32k")


@pytest.mark.parametrize("N,H_q,H_kv,d_h,B_k,k", [
    (1000, 16, 2, 64, 64, 5),    # G = 8, ragged tail
    (700, 8, 2, 128, 128, 3),    # G = 4 (8-head boxes, half used), d_h = 128
    (513, 64, 4, 128, 128, 4),   # G = 16 (pages' 64/4 heads)
    (300, 16, 2, 128, 64, 8),    # k * B_k >= N: every visible block selected
    (600, 8, 8, 64, 64, 4),      # G = 1, d_h = 64: 64 outputs per (query, group)
    (600, 8, 4, 64, 64, 4),      # G = 2, d_h = 64: 128 outputs per (query, group)
    (640, 8, 8, 128, 128, 3),    # G = 1, d_h = 128
])
def test_attention_edge_shapes(msa, N, H_q, H_kv, d_h, B_k, k):
    cfg = inputs.MSAConfig("edge", N=N, H_q=H_q, H_kv=H_kv, d_h=d_h, d_idx=64, B_k=B_k, k=k,
                           structure="iid", seed_index=23)
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = _index(msa, dev, cfg)
    _check_attn(msa, inp, dev, idx, cfg, np.arange(N), f"edge {N},{H_q},{H_kv},{d_h},{B_k},{k}")


def test_attention_dense_equivalence(msa):
    """k*B_k >= N: the GPU result equals the dense causal GQA oracle (Eq. 1)."""
    N, H_q, H_kv, d_h, B_k = 640, 16, 2, 128, 128
    cfg = inputs.MSAConfig("dense", N=N, H_q=H_q, H_kv=H_kv, d_h=d_h, d_idx=64, B_k=B_k, k=5,
                           seed_index=29)
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = _index(msa, dev, cfg)
    o, lse = _attn(msa, dev, idx, B_k)
    rows = np.arange(N)
    ro, rlse = oracle.dense_attn(inp["q"], inp["k"], inp["v"], rows)
    compare.assert_attn_close(bf16_to_f64(o), ro, lse.cpu().numpy(), rlse, what="dense")


def test_attention_synthetic_sink_zipf_selection(msa):
    """Sink-skewed selections (block 0 in ~90% of rows, Zipf(1.1) by recency):
    hot-block splitting and tiles mixing local and non-local rows."""
    cfg = _cfg("32k", N=6144)
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    sel = inputs.zipf_indices(cfg.N, cfg.H_kv, cfg.B_k, cfg.k)
    idx = torch.from_numpy(sel).cuda()
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([rng.integers(0, cfg.N, 300), np.arange(cfg.N - 64, cfg.N)]))
    _check_attn(msa, inp, dev, idx, cfg, rows, "zipf")


def test_attention_empty_and_future_entries(msa):
    """-1 slots are skipped; a block after the query's own contributes nothing
    (causal rule); an all-empty row gives o = 0, lse = -inf."""
    cfg = inputs.MSAConfig("odd", N=512, H_q=16, H_kv=2, d_h=64, d_idx=64, B_k=64, k=4,
                           seed_index=31)
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = np.full((cfg.N, cfg.H_kv, cfg.k), -1, dtype=np.int32)
    B = cfg.B
    for i in range(cfg.N):
        b_i = i // cfg.B_k
        row = [b_i] + ([0] if b_i >= 2 else []) + ([b_i + 2] if b_i + 2 < B else [])
        idx[i, 0, : len(row)] = row  # group 1 stays empty
    o, lse = _attn(msa, dev, torch.from_numpy(idx).cuda(), cfg.B_k)
    rows = np.arange(cfg.N)
    ro, rlse = oracle.sparse_attn(inp["q"], inp["k"], inp["v"], idx, cfg.B_k, rows)
    go = bf16_to_f64(o)
    G = cfg.G
    compare.assert_attn_close(go[:, :G], ro[:, :G], lse.cpu().numpy()[:, :G], rlse[:, :G],
                              what="group 0")
    assert (go[:, G:] == 0).all() and np.isneginf(lse.cpu().numpy()[:, G:]).all()


def test_attention_128k_sampled(msa):
    """Full 128K workload: every row of blocks 0, 1, B/2, B-1, the ends of
    each group's block-0 list and random rows."""
    cfg = inputs.CONFIGS["128k"]
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = _index(msa, dev, cfg)
    rng = np.random.default_rng(3)
    rows = structured_rows(cfg, idx.cpu().numpy(), extra=rng.integers(0, cfg.N, 96))
    _check_attn(msa, inp, dev, idx, cfg, rows, "128k")


def test_attention_key_set_beyond_shared_histogram(msa):
    """H_kv * B = 50000 (group, block) keys: more than a per-CTA shared-memory
    histogram of the inverse index holds, so the global-atomic inverse index
    runs.  Selection: the local block and k-1 earlier blocks at a per-row
    random stride (strictly decreasing, so distinct), ascending, -1 padded."""
    N, H_kv, d_h, B_k, k = 400000, 8, 64, 64, 8
    assert H_kv * ((N + B_k - 1) // B_k) * 4 > 192 * 1024
    rng = np.random.default_rng(41)
    inp = {t: inputs.bf16_bits(rng.standard_normal((N, H_kv, d_h), dtype=np.float32))
           for t in ("q", "k", "v")}
    b_i = (np.arange(N) // B_k)[:, None, None]
    stride = rng.integers(1, 14, size=(N, H_kv, 1))
    offset = rng.integers(0, 6, size=(N, H_kv, 1))
    j = np.arange(k)[None, None, :]
    blk = np.where(j == 0, b_i, b_i - j * stride - offset)
    blk = np.where(blk < 0, np.iinfo(np.int32).max, blk)
    idx = np.sort(blk, axis=2)
    idx = np.where(idx == np.iinfo(np.int32).max, -1, idx).astype(np.int32)
    cfg = inputs.MSAConfig("wide", N=N, H_q=H_kv, H_kv=H_kv, d_h=d_h, d_idx=64, B_k=B_k, k=k,
                           seed_index=41)
    dev = dev_inputs(inp)
    rows = np.unique(np.concatenate([rng.integers(0, N, 64), [0, 63, 64, N - 1]]))
    _check_attn(msa, inp, dev, torch.from_numpy(idx).cuda(), cfg, rows, "wide key set")


def test_bounded_wait_times_out_reports_and_context_survives(msa):
    """Failure detection without a fault: a wait that nothing completes gives
    up after its limit, the status word says so, and the next call works."""
    import time

    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    msa.selftest_bounded_wait(ws)
    code, where = msa.device_status(ws)
    elapsed = time.time() - t0
    assert (code, where) == (1, 99)
    assert 1.0 < elapsed < 20.0
    cfg = inputs.CONFIGS["tiny"]
    _check_index(msa, cfg, rows=np.arange(0, cfg.N, 97))


def _check_index_lse(msa, cfg, dev, inp, idx_dev, rows, what):
    """LSE_idx (Eq. 9's Index Branch normaliser) on the GPU against the oracle
    for the listed rows, from the same selection."""
    lse_idx = torch.full((dev["q_idx"].shape[0], cfg.H_kv), float("nan"), dtype=torch.float32,
                         device="cuda")
    msa.index_lse(dev["q_idx"], dev["k_idx"], idx_dev, cfg.B_k, lse_idx=lse_idx)
    torch.cuda.synchronize()
    rows = np.asarray(rows)
    sel = idx_dev.cpu().numpy()[rows]
    ref = oracle.index_lse(inp["q_idx"][rows], inp["k_idx"], sel, cfg.B_k, rows, N=cfg.N)
    got = lse_idx.cpu().numpy().astype(np.float64)[rows]
    assert (np.isneginf(got) == np.isneginf(ref)).all(), what
    fin = np.isfinite(ref)
    np.testing.assert_allclose(got[fin], ref[fin], rtol=1e-5, atol=1e-4, err_msg=what)


def test_index_lse_tiny_all_rows(msa):
    cfg = inputs.CONFIGS["tiny"]
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = _index(msa, dev, cfg)
    _check_index_lse(msa, cfg, dev, inp, idx, np.arange(cfg.N), "tiny")


def test_index_lse_32k_recipe_and_128k_sampled(msa):
    for cfg, n_rand in ((_cfg("32k", N=8192), 200), (inputs.CONFIGS["128k"], 96)):
        inp = prefill_inputs_cached(cfg)
        dev = dev_inputs(inp)
        idx = _index(msa, dev, cfg)
        rng = np.random.default_rng(7)
        rows = np.unique(np.concatenate([rng.integers(0, cfg.N, n_rand),
                                         [0, 1, 127, 128, cfg.N - 1]]))
        _check_index_lse(msa, cfg, dev, inp, idx, rows, cfg.name)


@pytest.mark.parametrize("N,H_kv,d_idx,B_k,k", [
    (1000, 2, 32, 64, 5),     # ragged tail, B_k = 64
    (3001, 4, 128, 128, 32),  # largest k, d_idx = 128
    (300, 4, 64, 128, 8),     # k above the visible blocks: -1 padding everywhere
])
def test_index_lse_edge_shapes_and_empty_rows(msa, N, H_kv, d_idx, B_k, k):
    cfg = inputs.MSAConfig("lse", N=N, H_q=H_kv * 2, H_kv=H_kv, d_h=64, d_idx=d_idx, B_k=B_k,
                           k=k, structure="iid", seed_index=43)
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = _index(msa, dev, cfg)
    idx[5, 0, :] = -1       # a row with no token: -inf
    idx[N - 1, H_kv - 1, 1:] = -1
    _check_index_lse(msa, cfg, dev, inp, idx, np.arange(N), "edge")


def test_device_status_reports_bad_index(msa):
    cfg = inputs.MSAConfig("bad", N=256, H_q=16, H_kv=2, d_h=64, d_idx=64, B_k=64, k=2,
                           seed_index=37)
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = np.zeros((cfg.N, cfg.H_kv, cfg.k), dtype=np.int32)
    idx[:, :, 1] = -1
    idx[5, 1, 1] = 99  # outside [-1, B)
    d = msa.dims(cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, 64, cfg.B_k, cfg.k)
    ws = torch.empty(msa.sparse_attn_fwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    msa.sparse_attn_fwd(dev["q"], dev["k"], dev["v"], torch.from_numpy(idx).cuda(), cfg.B_k,
                        workspace=ws)
    code, where = msa.device_status(ws)
    assert code == 2
    # a clean call on the same workspace clears the word
    idx[5, 1, 1] = -1
    msa.sparse_attn_fwd(dev["q"], dev["k"], dev["v"], torch.from_numpy(idx).cuda(), cfg.B_k,
                        workspace=ws)
    assert msa.device_status(ws)[0] == 0


# ------------------------------------------------------------------ decode --

def _decode_run(msa, cfg, steps, check_seqs, seed=None):
    st = inputs.decode_state(cfg, seed)
    dev = {k: to_dev(st[k]) for k in ("k_cache", "v_cache", "k_idx_cache")}
    seq_len = torch.from_numpy(st["seq_len"]).cuda()
    for step in range(steps):
        si = inputs.decode_step_inputs(cfg, step, st["sink"], seed)
        d = {k: to_dev(v) for k, v in si.items()}
        idx_out = torch.full((cfg.S, cfg.H_kv, cfg.k), SENTINEL, dtype=torch.int32,
                             device="cuda")
        o = torch.full((cfg.S, cfg.H_q, cfg.d_h), float("nan"), dtype=torch.bfloat16,
                       device="cuda")
        o, _ = msa.sparse_decode(d["q"], d["q_idx"], d["k_new"], d["v_new"], d["k_idx_new"],
                                 dev["k_cache"], dev["v_cache"], dev["k_idx_cache"], seq_len,
                                 cfg.B_k, cfg.k, o=o, idx_out=idx_out)
        torch.cuda.synchronize()
        gidx = idx_out.cpu().numpy()
        ref = oracle.decode_reference(st, si, cfg.B_k, cfg.k, seqs=check_seqs,
                                      idx_rows=gidx[check_seqs])
        rows = np.array([int(st["seq_len"][s]) for s in check_seqs])
        q_idx_rows = si["q_idx"][check_seqs]
        kic = [st["k_idx_cache"][s] for s in check_seqs]
        for n, s in enumerate(check_seqs):
            kk = kic[n].copy()
            kk[rows[n]] = si["k_idx_new"][s]
            ex, band, fails = compare.check_topk(gidx[[s]], ref["idx"][[n]], ref["cut"][[n]],
                                                 ref["next"][[n]], rows[[n]], cfg.B_k, cfg.k,
                                                 q_idx_rows=q_idx_rows[[n]], k_idx=kk)
            assert not fails, (step, s, fails)
        compare.assert_attn_close(bf16_to_f64(o)[check_seqs], ref["o"], what=f"decode step {step}")
        # host mirror of the append so the next step's oracle sees the same caches
        for s in range(cfg.S):
            L = int(st["seq_len"][s])
            st["k_cache"][s, L] = si["k_new"][s]
            st["v_cache"][s, L] = si["v_new"][s]
            st["k_idx_cache"][s, L] = si["k_idx_new"][s]
            st["seq_len"][s] = L + 1
        assert (seq_len.cpu().numpy() == st["seq_len"]).all()


def test_decode_small_crosses_block_boundary(msa):
    # L0 = 255 -> the first step's token closes block 1, the second opens block 2
    cfg = inputs.DecodeConfig("dsmall", S=5, L0=255, steps=3, H_q=32, H_kv=4, d_h=128, d_idx=64,
                              B_k=128, k=4, seed_index=41)
    _decode_run(msa, cfg, 3, list(range(5)))


def test_decode_small_shapes(msa):
    cfg = inputs.DecodeConfig("dshape", S=3, L0=1000, steps=2, H_q=16, H_kv=2, d_h=64, d_idx=32,
                              B_k=64, k=6, seed_index=43)
    _decode_run(msa, cfg, 2, [0, 1, 2])


def test_decode_empty_cache(msa):
    cfg = inputs.DecodeConfig("dempty", S=2, L0=0, steps=2, H_q=32, H_kv=4, d_h=128, d_idx=64,
                              B_k=128, k=16, seed_index=47)
    _decode_run(msa, cfg, 2, [0, 1])


def test_decode_cache_full_is_reported(msa):
    cfg = inputs.DecodeConfig("dfull", S=2, L0=64, steps=0, H_q=16, H_kv=2, d_h=64, d_idx=64,
                              B_k=64, k=2, seed_index=53)
    st = inputs.decode_state(cfg)
    dev = {k: to_dev(st[k]) for k in ("k_cache", "v_cache", "k_idx_cache")}
    seq_len = torch.tensor([64, 10], dtype=torch.int32, device="cuda")  # seq 0 is full
    si = inputs.decode_step_inputs(cfg, 0, st["sink"])
    d = {k: to_dev(v) for k, v in si.items()}
    dd = msa.decode_dims(cfg.S, cfg.L_max, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.B_k, cfg.k)
    ws = torch.empty(msa.sparse_decode_workspace_size(dd), dtype=torch.uint8, device="cuda")
    msa.sparse_decode(d["q"], d["q_idx"], d["k_new"], d["v_new"], d["k_idx_new"],
                      dev["k_cache"], dev["v_cache"], dev["k_idx_cache"], seq_len, cfg.B_k, cfg.k,
                      workspace=ws)
    assert msa.device_status(ws)[0] == 3
    assert seq_len.cpu().tolist() == [64, 11]


def test_decode_full_size_sampled(msa):
    """The 64 x 131072-token decode workload, two steps; four sequences checked."""
    cfg = inputs.CONFIGS["decode"]
    _decode_run(msa, cfg, 2, [0, 17, 42, 63])


def test_forward_1m_sampled(msa):
    """The 1M-token sink-skewed workload through the whole forward (index +
    attention in 8 query chunks of 131072); structured and sampled rows
    checked against the oracle."""
    cfg = inputs.CONFIGS["1m"]
    inp = prefill_inputs_cached(cfg)
    dev = dev_inputs(inp)
    idx = _index(msa, dev, cfg)
    o, lse = _attn(msa, dev, idx, cfg.B_k)
    del dev
    rng = np.random.default_rng(5)
    all_idx = idx.cpu().numpy()
    # every row of blocks 0, 1, B/2, B-1 and the ends of each group's block-0
    # list (chunks of 131072 queries: rows around a chunk boundary too)
    rows = structured_rows(cfg, all_idx, extra=np.concatenate([
        rng.integers(0, cfg.N, 20), [8191, 8192, 131071, 131072, cfg.N // 2 + 5]]))
    gidx = all_idx[rows]
    ref, cut, nxt = oracle.index_topk(inp["q_idx"], inp["k_idx"], cfg.B_k, cfg.k, rows=rows)
    exact, band, fails = compare.check_topk(gidx, ref, cut, nxt, rows, cfg.B_k, cfg.k,
                                            q_idx_rows=inp["q_idx"][rows], k_idx=inp["k_idx"])
    assert not fails, fails
    # the workload's defining property: block 0 chosen by >= 90% of (row, group)
    late = rows >= cfg.B_k
    assert (ref[late] == 0).any(axis=2).mean() >= 0.9
    ro, rlse = oracle.sparse_attn(inp["q"][rows], inp["k"], inp["v"], gidx, cfg.B_k, rows,
                                  N=cfg.N)
    compare.assert_attn_close(bf16_to_f64(o)[rows], ro, lse.cpu().numpy()[rows], rlse, what="1m")
