"""GPU parity of the projections (five cuBLAS GEMMs behind msa_project)
against the oracle's fp64 x W: every output element within bf16 rounding of
the exact product plus an fp32-accumulation allowance."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_idx_b200 import inputs
from tests.gpu_util import bf16_to_f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_gqa_idx_b200 as m

    return m


@pytest.mark.parametrize("T,d_model,H_q,H_kv,d_h,d_idx", [
    (3000, 512, 32, 4, 128, 64),   # the pages' heads, a ragged token count
    (77, 1024, 16, 2, 64, 128),
])
def test_project_matches_oracle(msa, T, d_model, H_q, H_kv, d_h, d_idx):
    rng = np.random.default_rng(T + d_model)
    x = inputs.bf16_bits(rng.standard_normal((T, d_model)).astype(np.float32))
    ws = {name: inputs.bf16_bits((rng.standard_normal((d_model, n)) / np.sqrt(d_model))
                                 .astype(np.float32))
          for name, n in (("w_q", H_q * d_h), ("w_k", H_kv * d_h), ("w_v", H_kv * d_h),
                          ("w_qidx", H_kv * d_idx), ("w_kidx", d_idx))}
    dev = {k: to_dev(v) for k, v in ws.items()}
    out = msa.project(to_dev(x), dev["w_q"], dev["w_k"], dev["w_v"], dev["w_qidx"],
                      dev["w_kidx"], H_q, H_kv)
    torch.cuda.synchronize()
    xf = inputs.bf16_to_f32(x).astype(np.float64)
    for name, key in (("w_q", "q"), ("w_k", "k"), ("w_v", "v"), ("w_qidx", "q_idx"),
                      ("w_kidx", "k_idx")):
        ref = oracle.project(x, ws[name])
        got = bf16_to_f64(out[key]).reshape(T, -1)
        # |x| |w| bounds the fp32 accumulation error (d_model terms, 2^-23 each)
        mag = np.abs(xf) @ np.abs(inputs.bf16_to_f32(ws[name]).astype(np.float64))
        tol = 2.0 ** -8 * np.abs(ref) + d_model * 2.0 ** -23 * mag + 1e-30
        assert (np.abs(got - ref) <= tol).all(), (key, float(np.abs(got - ref).max()))
