"""GPU parity of the paged FP8 (E4M3) decode against the oracle: the append's
quantization bit for bit, the selection (exact, ties within the band), the
outputs within the attention tolerance, and a bad page reported, not read."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_idx_b200 import inputs
from tests import compare
from tests.gpu_util import bf16_to_f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_gqa_idx_b200 as m

    return m


def test_quantize_fp8_rows_matches_oracle(msa):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((300, 128)).astype(np.float32) * rng.uniform(0.01, 50, (300, 1))
    x[7] = 0.0
    x[11, 5] = 1e4  # one large value: the rest of the row rounds to small codes
    bits = inputs.bf16_bits(x.astype(np.float32))
    codes, scales = msa.quantize_fp8_rows(to_dev(bits))
    torch.cuda.synchronize()
    want_c, want_s = oracle.quantize_rows(bits)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    assert np.array_equal(scales.cpu().numpy(), want_s)


def _dev_pages(st):
    keys = ("k_pages", "v_pages", "kidx_pages", "k_scale", "v_scale", "kidx_scale", "page_table")
    return {k: torch.from_numpy(np.ascontiguousarray(st[k])).cuda() for k in keys}


def _run(msa, cfg, st, steps, seqs, q_idx_pow2=None):
    """`steps` decode steps on the GPU and on the oracle (which carries the
    oracle's own quantized appends forward), comparing the listed sequences.
    q_idx_pow2: per index head, a power of two the index queries are
    multiplied by (exact in bf16) before both sides see them."""
    dev = _dev_pages(st)
    seq_len = torch.from_numpy(st["seq_len"].copy()).cuda()
    host = {k: st[k].copy() for k in ("k_pages", "v_pages", "kidx_pages", "k_scale", "v_scale",
                                      "kidx_scale", "page_table")}
    L = st["seq_len"].copy()
    for step in range(steps):
        si = inputs.decode_step_inputs(cfg, step, st["sink"])
        if q_idx_pow2 is not None:
            f = np.asarray(q_idx_pow2, dtype=np.float32)[None, :, None]
            qf = (si["q_idx"].astype(np.uint32) << 16).view(np.float32) * f
            si["q_idx"] = inputs.bf16_bits(qf)
        d = {k: to_dev(v) for k, v in si.items()}
        o = torch.full((cfg.S, cfg.H_q, cfg.d_h), float("nan"), dtype=torch.bfloat16,
                       device="cuda")
        idx = torch.full((cfg.S, cfg.H_kv, cfg.k), -7, dtype=torch.int32, device="cuda")
        msa.paged_decode_fp8(d["q"], d["q_idx"], d["k_new"], d["v_new"], d["k_idx_new"],
                             dev["k_pages"], dev["k_scale"], dev["v_pages"], dev["v_scale"],
                             dev["kidx_pages"], dev["kidx_scale"], dev["page_table"], seq_len,
                             cfg.B_k, cfg.k, o=o, idx_out=idx)
        torch.cuda.synchronize()
        ref = oracle.paged_decode_fp8(host, si, L, cfg.B_k, cfg.k, seqs=seqs)
        gidx = idx.cpu().numpy()[seqs]
        rows = L[seqs].astype(np.int64)  # the query position of each compared sequence
        exact, band, fails = compare.check_topk(gidx, ref["idx"], ref["cut"], ref["next"], rows,
                                                cfg.B_k, cfg.k)
        assert not fails, (step, fails)
        same = (gidx == ref["idx"]).all(axis=(1, 2))
        go = bf16_to_f64(o)[seqs]
        assert np.isfinite(go).all()
        compare.assert_attn_close(go[same], ref["o"][same], what=f"fp8 step {step}")
        # the append, bit for bit: the GPU pages at the new token's slot
        for n, s_ in enumerate(seqs):
            pg = int(st["page_table"][s_, L[s_] // cfg.B_k])
            sl = int(L[s_] % cfg.B_k)
            assert np.array_equal(dev["k_pages"][pg, sl].cpu().numpy(), ref["new_k"][n])
            assert np.array_equal(dev["v_pages"][pg, sl].cpu().numpy(), ref["new_v"][n])
            assert np.array_equal(dev["kidx_pages"][pg, sl].cpu().numpy(), ref["new_kidx"][n])
            assert np.array_equal(dev["k_scale"][pg, sl].cpu().numpy(), ref["new_kv_scale"][n, 0])
            assert np.array_equal(dev["v_scale"][pg, sl].cpu().numpy(), ref["new_kv_scale"][n, 1])
            assert dev["kidx_scale"][pg, sl].item() == ref["new_kidx_scale"][n]
            # the oracle carries its own quantized rows into the next step
            host["k_pages"][pg, sl] = ref["new_k"][n]
            host["v_pages"][pg, sl] = ref["new_v"][n]
            host["kidx_pages"][pg, sl] = ref["new_kidx"][n]
            host["k_scale"][pg, sl] = ref["new_kv_scale"][n, 0]
            host["v_scale"][pg, sl] = ref["new_kv_scale"][n, 1]
            host["kidx_scale"][pg, sl] = ref["new_kidx_scale"][n]
        L = L + 1
        assert seq_len.cpu().numpy().tolist() == L.tolist()
    return exact, band


@pytest.mark.parametrize("L0,B_k,d_h,d_idx,k", [
    (1000, 128, 128, 64, 8),   # the new token inside block 7
    (1279, 128, 128, 64, 8),   # the second step starts a new page
    (700, 64, 64, 128, 5),     # B_k = 64, d_h = 64, d_idx = 128
    (300, 128, 128, 64, 16),   # fewer visible blocks than k
    (900, 64, 128, 64, 8),     # B_k = 64 with d_h = 128
    (900, 128, 64, 64, 8),     # B_k = 128 with d_h = 64
])
def test_paged_fp8_decode_small(msa, L0, B_k, d_h, d_idx, k):
    cfg = inputs.DecodeConfig("fp8", S=5, L0=L0, steps=3, H_q=32, H_kv=4, d_h=d_h, d_idx=d_idx,
                              B_k=B_k, k=k, seed_index=63)
    st = inputs.decode_fp8_state(cfg)
    _run(msa, cfg, st, 3, np.arange(cfg.S))


def test_paged_fp8_decode_full_size_sampled(msa):
    """The 64 x 131072-token workload on its FP8 paged cache, two steps;
    three sequences checked against the oracle."""
    cfg = inputs.CONFIGS["decode_fp8"]
    st = inputs.decode_fp8_state(cfg)
    _run(msa, cfg, st, 2, np.array([0, 31, 63]))


def test_paged_fp8_decode_index_query_magnitudes(msa):
    """Index queries from 2^-24 to 2^24 times the recipe's (beyond f16's
    range at both ends): the selection and outputs still match the oracle."""
    cfg = inputs.DecodeConfig("fp8mag", S=4, L0=2000, steps=2, H_q=32, H_kv=4, d_h=128,
                              d_idx=64, B_k=128, k=8, seed_index=68)
    st = inputs.decode_fp8_state(cfg)
    _run(msa, cfg, st, 2, np.arange(cfg.S), q_idx_pow2=[2.0 ** 24, 2.0 ** -24, 1.0, 2.0 ** 10])


def test_paged_fp8_bad_page_is_reported(msa):
    """A page-table entry outside the pool is skipped by every kernel and
    recorded as MSA_DEV_BAD_INDEX (no access outside the pool)."""
    cfg = inputs.DecodeConfig("fp8bad", S=2, L0=500, steps=1, H_q=16, H_kv=2, d_h=64,
                              d_idx=64, B_k=64, k=4, seed_index=67)
    st = inputs.decode_fp8_state(cfg)
    st["page_table"][1, 2] = st["k_pages"].shape[0] + 5  # past the pool
    dev = _dev_pages(st)
    si = {k: to_dev(v) for k, v in inputs.decode_step_inputs(cfg, 0, st["sink"]).items()}
    seq_len = torch.from_numpy(st["seq_len"].copy()).cuda()
    d = msa.paged_dims(cfg.S, st["page_table"].shape[1], st["k_pages"].shape[0], cfg.H_q,
                       cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.B_k, cfg.k)
    ws = torch.zeros(msa.paged_decode_fp8_workspace_size(d), dtype=torch.uint8, device="cuda")
    msa.paged_decode_fp8(si["q"], si["q_idx"], si["k_new"], si["v_new"], si["k_idx_new"],
                         dev["k_pages"], dev["k_scale"], dev["v_pages"], dev["v_scale"],
                         dev["kidx_pages"], dev["kidx_scale"], dev["page_table"], seq_len,
                         cfg.B_k, cfg.k, workspace=ws)
    code, where = msa.device_status(ws)
    assert code == 2 and where == 88  # MSA_DEV_BAD_INDEX from the page lookup
