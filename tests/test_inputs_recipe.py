"""The seeded synthetic inputs have the structure the documentation states
(CPU only): bf16 rounding, AR(1) index keys, the sink bias on block 0, the
planted retrieval tokens, determinism per seed."""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import pytest
import torch

from block_sparse_gqa_idx_b200 import inputs


def _f32(bits):
    return inputs.bf16_to_f32(bits).astype(np.float64)


def test_bf16_rounding_is_round_to_nearest_even():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-3, 4, 100000),
                        # exact halfway cases between two bf16 values: ties go to even
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)])
    ours = inputs.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (ours == ref).all()


def _small(name, **kw):
    return dataclasses.replace(inputs.CONFIGS[name], **kw)


def test_index_keys_are_ar1_with_unit_marginals():
    cfg = _small("32k", N=16384)
    inp = inputs.prefill_inputs(cfg)
    k = _f32(inp["k_idx"])[cfg.B_k:]  # block 0 carries the sink shift
    k = k - k.mean(axis=0)
    lag1 = (k[1:] * k[:-1]).sum(axis=0) / (k * k).sum(axis=0)
    assert abs(lag1.mean() - 0.9) < 0.01
    assert abs(k.std(axis=0).mean() - 1.0) < 0.05


@pytest.mark.parametrize("name,bias", [("32k", 2.0), ("1m", 6.0)])
def test_sink_gives_block0_the_stated_score_bias(name, bias):
    """q_idx += s*u and K_idx[block 0] += 2*sqrt(d_idx)*u: block 0's expected
    index score exceeds the others' by 2*s (s = 1 at 32K, 3 for the 1M recipe)."""
    cfg = _small(name, N=8192)
    inp = inputs.prefill_inputs(cfg)
    q = _f32(inp["q_idx"])[::7]  # a sample of rows, every group
    k = _f32(inp["k_idx"])
    scores = np.einsum("nrd,jd->nrj", q, k) / math.sqrt(cfg.d_idx)
    gap = scores[:, :, :cfg.B_k].mean() - scores[:, :, cfg.B_k:].mean()
    assert abs(gap - bias) < 0.15 * bias


def test_retrieval_tokens_are_planted_once_per_block():
    """The 128K recipe plants, per group, one token of 8 blocks with
    K_idx += 2*sqrt(d_idx)*v (|v| = 1): those rows stand out in norm."""
    cfg = _small("128k", N=16384)
    inp = inputs.prefill_inputs(cfg)
    k = _f32(inp["k_idx"])
    norms = np.linalg.norm(k, axis=1)
    # an ordinary row has norm ~ sqrt(d_idx) = 8; a planted one ~ sqrt(64 + 256) = 17.9
    planted = np.nonzero(norms[cfg.B_k:] > 14.0)[0] + cfg.B_k
    assert planted.size == 8 * cfg.H_kv
    blocks = planted // cfg.B_k
    assert blocks.min() >= 1 and blocks.max() <= cfg.B - 2


def test_generation_is_deterministic_per_seed():
    cfg = _small("32k", N=4096)
    a = inputs.prefill_inputs(cfg)
    b = inputs.prefill_inputs(cfg)
    c = inputs.prefill_inputs(cfg, seed=cfg.seed + 1000)
    for name in a:
        assert (a[name] == b[name]).all(), name
    assert not (a["q"] == c["q"]).all()
