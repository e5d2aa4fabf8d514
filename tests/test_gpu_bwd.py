"""GPU parity of the backward of Eq. 8 (selection fixed) against the
oracle's fp64 gradients, fed the GPU forward's selection: every element of
dQ, dK and dV.  The bar follows from the arithmetic: P and dS enter the
tensor cores as bf16 (2^-9 relative), D and the outputs are bf16 roundings
of fp32 sums, so each gradient is compared with a max-abs error of 2% and
a mean-abs error of 1% of its own mean magnitude."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_idx_b200 import inputs
from tests.gpu_util import bf16_to_f64, dev_inputs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_gqa_idx_b200 as m

    return m


def _check_grad(got, want, what):
    scale = float(np.abs(want).mean())
    err = np.abs(got - want)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    assert err.max() <= 2e-2 * max(float(np.abs(want).max()), 1e-6), \
        f"{what}: max-abs {err.max():.3e} vs max {np.abs(want).max():.3e}"
    assert err.mean() <= 1e-2 * max(scale, 1e-9), \
        f"{what}: mean-abs {err.mean():.3e} vs mean {scale:.3e}"


def _run(msa, cfg, seed=5):
    inp = inputs.prefill_inputs(cfg)
    dev = dev_inputs(inp)
    idx = msa.index_topk(dev["q_idx"], dev["k_idx"], cfg.B_k, cfg.k)
    o, lse = msa.sparse_attn_fwd(dev["q"], dev["k"], dev["v"], idx, cfg.B_k)
    rng = np.random.default_rng(seed)
    d_o = inputs.bf16_bits(rng.standard_normal((cfg.N, cfg.H_q, cfg.d_h)).astype(np.float32))
    dq = torch.full_like(dev["q"], float("nan"))
    dq, dk, dv = msa.sparse_attn_bwd(dev["q"], dev["k"], dev["v"], idx, o, lse, to_dev(d_o),
                                     cfg.B_k)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.sparse_attn_bwd(inp["q"], inp["k"], inp["v"], idx.cpu().numpy(), d_o,
                                        cfg.B_k)
    _check_grad(bf16_to_f64(dq), rq, f"{cfg.name} dQ")
    _check_grad(bf16_to_f64(dk), rk, f"{cfg.name} dK")
    _check_grad(bf16_to_f64(dv), rv, f"{cfg.name} dV")
    return idx.cpu().numpy(), bf16_to_f64(dk)


@pytest.mark.parametrize("N,H_q,H_kv,d_h,B_k,k", [
    (1000, 16, 2, 64, 64, 5),    # G = 8, ragged tail
    (700, 8, 2, 128, 128, 3),    # G = 4: 32 queries per tile
    (513, 64, 4, 128, 128, 4),   # G = 16: 8 queries per tile
    (600, 8, 8, 64, 64, 4),      # G = 1: 128 queries per tile
    (3001, 32, 4, 128, 128, 16), # the pages' heads, several hundred tiles
])
def test_backward_matches_oracle(msa, N, H_q, H_kv, d_h, B_k, k):
    cfg = inputs.MSAConfig("bwd", N=N, H_q=H_q, H_kv=H_kv, d_h=d_h, d_idx=64, B_k=B_k, k=k,
                           structure="sink_ar1", seed_index=53)
    _run(msa, cfg)


def test_backward_unselected_keys_get_zero_gradients(msa):
    """With k = 1 every query selects only its own block: a key's gradient
    comes only from its own block's queries, and the padding rows of the
    last block (past N) are never written."""
    cfg = inputs.MSAConfig("bwd1", N=777, H_q=16, H_kv=2, d_h=64, d_idx=64, B_k=64, k=1,
                           structure="iid", seed_index=59)
    idx, dk = _run(msa, cfg)
    assert (idx[:, :, 0] == (np.arange(cfg.N) // cfg.B_k)[:, None]).all()
    assert np.isfinite(dk).all()
