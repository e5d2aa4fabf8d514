"""GPU parity of the packed-batch (variable-length) prefill against the
oracle: each sequence's selection exactly (ties within the band), its block
scores, and the attention outputs from the GPU's selection fed to both
sides; outputs poisoned before every call."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_idx_b200 import inputs
from tests import compare
from tests.gpu_util import bf16_to_f64, dev_inputs

pytestmark = pytest.mark.gpu
SENTINEL = -7


@pytest.fixture(scope="module")
def msa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_gqa_idx_b200 as m

    return m


def _run(msa, dev, cu, cfg):
    N = int(cu[-1])
    idx = torch.full((N, cfg.H_kv, cfg.k), SENTINEL, dtype=torch.int32, device="cuda")
    sc = torch.full((N, cfg.H_kv, cfg.k), float("nan"), dtype=torch.float32, device="cuda")
    msa.index_topk_varlen(dev["q_idx"], dev["k_idx"], cu, cfg.B_k, cfg.k, idx_out=idx,
                          score_out=sc)
    o = torch.full((N, cfg.H_q, cfg.d_h), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((N, cfg.H_q), float("nan"), dtype=torch.float32, device="cuda")
    msa.sparse_attn_fwd_varlen(dev["q"], dev["k"], dev["v"], idx, cu, cfg.B_k, o=o, lse=lse)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy(), o, lse


def _check(msa, cfg, lengths, rows=None, score_every=1):
    inp, cu = inputs.varlen_inputs(cfg, lengths)
    dev = dev_inputs(inp)
    gidx, gsc, o, lse = _run(msa, dev, cu, cfg)
    N = int(cu[-1])
    rows = np.arange(N) if rows is None else np.unique(np.asarray(rows, dtype=np.int64))
    ref = oracle.forward_varlen(inp, cu, cfg.B_k, cfg.k, rows=rows, idx_rows=gidx[rows])
    seq = ref["seq"]
    for s in np.unique(seq):
        a, b = int(cu[s]), int(cu[s + 1])
        pick = np.nonzero(seq == s)[0]
        loc = rows[pick] - a
        exact, band, fails = compare.check_topk(
            gidx[rows[pick]], ref["idx"][pick], ref["cut"][pick], ref["next"][pick], loc,
            cfg.B_k, cfg.k, q_idx_rows=inp["q_idx"][rows[pick]], k_idx=inp["k_idx"][a:b])
        assert not fails, (s, fails[:3])
        for t in pick[::score_every]:
            i = int(rows[t])
            for r in range(cfg.H_kv):
                M = oracle.block_scores(inp["q_idx"][i, r], inp["k_idx"][a:b], cfg.B_k, i - a)
                for s_ in range(cfg.k):
                    bb = int(gidx[i, r, s_])
                    got = float(gsc[i, r, s_])
                    if bb < 0:
                        assert got == -np.inf, (i, r, s_, got)
                    else:
                        assert abs(got - M[bb]) <= compare._band(got, M[bb]), (i, r, s_, got)
    go = bf16_to_f64(o)[rows]
    gl = lse.cpu().numpy().astype(np.float64)[rows]
    compare.assert_attn_close(go, ref["o"], gl, ref["lse"], what=f"varlen {cfg.name}")
    return inp, cu, gidx, o, lse


@pytest.mark.parametrize("lengths,H_q,H_kv,d_h,d_idx,B_k,k", [
    ([300, 1, 0, 129, 64, 1000, 65], 8, 2, 64, 32, 64, 4),
    ([5000, 128, 1, 2999, 777, 256], 32, 4, 128, 64, 128, 16),
    ([700, 33, 2048, 5], 16, 8, 128, 64, 128, 5),   # H_kv = 8: 16 queries per M-tile
    ([450, 129, 1300], 8, 1, 64, 128, 128, 6),       # H_kv = 1: 128 queries per M-tile
    ([0, 640, 0, 1], 16, 2, 64, 64, 64, 32),         # empty sequences, largest k
])
def test_varlen_forward_all_rows(msa, lengths, H_q, H_kv, d_h, d_idx, B_k, k):
    cfg = inputs.MSAConfig("vl", 0, H_q, H_kv, d_h, d_idx, B_k, k, "sink_ar1", seed_index=41)
    _check(msa, cfg, lengths)


def test_varlen_128k_mix_sampled(msa):
    """The bench's packed workload (32 sequences, 131072 tokens, pages'
    heads): the first, last and block-boundary rows of every sequence."""
    cfg = inputs.CONFIGS["varlen"]
    lengths = cfg.lengths()
    cu = np.concatenate([[0], np.cumsum(lengths)])
    rows = []
    for s in range(len(lengths)):
        a, b = int(cu[s]), int(cu[s + 1])
        for x in (a, a + 1, a + cfg.B_k - 1, a + cfg.B_k, (a + b) // 2, b - 2, b - 1):
            if a <= x < b:
                rows.append(x)
    _check(msa, cfg.prefill, lengths, rows=rows, score_every=4)


def test_varlen_one_sequence_matches_the_single_sequence_path(msa):
    """One sequence through the packed entry points gives bit-for-bit the
    single-sequence kernels' selection and outputs (same kernels, same tiles)."""
    cfg = inputs.MSAConfig("vl1", 3001, 32, 4, 128, 64, 128, 16, "sink_ar1", seed_index=43)
    inp = inputs.prefill_inputs(cfg)
    dev = dev_inputs(inp)
    gidx, _, o, lse = _run(msa, dev, np.array([0, cfg.N]), cfg)
    idx2 = msa.index_topk(dev["q_idx"], dev["k_idx"], cfg.B_k, cfg.k)
    o2, lse2 = msa.sparse_attn_fwd(dev["q"], dev["k"], dev["v"], idx2, cfg.B_k)
    torch.cuda.synchronize()
    assert np.array_equal(gidx, idx2.cpu().numpy())
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_varlen_bad_block_is_reported(msa):
    """A selection entry past the batch's global block count is skipped and
    recorded as MSA_DEV_BAD_INDEX."""
    cfg = inputs.MSAConfig("vlbad", 0, 8, 2, 64, 32, 64, 4, "iid", seed_index=47)
    inp, cu = inputs.varlen_inputs(cfg, [200, 300])
    dev = dev_inputs(inp)
    idx = msa.index_topk_varlen(dev["q_idx"], dev["k_idx"], cu, cfg.B_k, cfg.k)
    idx[250, 1, 0] = 1000
    d = msa.varlen_dims(2, int(cu[-1]), cfg.H_q, cfg.H_kv, cfg.d_h, 64, cfg.B_k, cfg.k)
    import ctypes
    from block_sparse_gqa_idx_b200 import _capi

    cuc = (ctypes.c_int64 * 3)(*[int(x) for x in cu])
    ws = torch.zeros(_capi.LIB.msa_sparse_attn_fwd_varlen_workspace(ctypes.byref(d), cuc),
                     dtype=torch.uint8, device="cuda")
    msa.sparse_attn_fwd_varlen(dev["q"], dev["k"], dev["v"], idx, cu, cfg.B_k, workspace=ws)
    code, where = msa.device_status(ws)
    assert code == 2 and where == 40
