"""The product path has no CPU fallback: host (CPU) tensors are refused by
every entry point before anything is launched, and a missing CUDA library is
an import error, not a silent substitute."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import block_sparse_gqa_idx_b200 as msa  # noqa: E402

N, H_q, H_kv, d_h, d_idx, B_k, k = 256, 8, 2, 64, 32, 64, 4


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_prefill_entry_points_refuse_host_tensors():
    q, kv = _bf16(N, H_q, d_h), _bf16(N, H_kv, d_h)
    q_idx, k_idx = _bf16(N, H_kv, d_idx), _bf16(N, d_idx)
    idx = torch.zeros((N, H_kv, k), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        msa.index_topk(q_idx, k_idx, B_k, k)
    with pytest.raises(ValueError, match="CUDA"):
        msa.sparse_attn_fwd(q, kv, kv, idx, B_k)
    with pytest.raises(ValueError, match="CUDA"):
        msa.forward(q, kv, kv, q_idx, k_idx, B_k, k)
    with pytest.raises(ValueError, match="CUDA"):
        msa.forward_varlen(q, kv, kv, q_idx, k_idx, [0, 100, N], B_k, k)
    with pytest.raises(ValueError, match="CUDA"):
        msa.sparse_attn_bwd(q, kv, kv, idx, q, torch.zeros((N, H_q)), q, B_k)


def test_projection_and_decode_refuse_host_tensors():
    d_model = 64
    x = _bf16(N, d_model)
    w = [_bf16(d_model, H_q * d_h), _bf16(d_model, H_kv * d_h), _bf16(d_model, H_kv * d_h),
         _bf16(d_model, H_kv * d_idx), _bf16(d_model, d_idx)]
    with pytest.raises(ValueError, match="CUDA"):
        msa.project(x, *w, H_q=H_q, H_kv=H_kv)
    S, L_max = 2, 512
    with pytest.raises(ValueError, match="CUDA"):
        msa.sparse_decode(_bf16(S, H_q, d_h), _bf16(S, H_kv, d_idx), _bf16(S, H_kv, d_h),
                          _bf16(S, H_kv, d_h), _bf16(S, d_idx), _bf16(S, L_max, H_kv, d_h),
                          _bf16(S, L_max, H_kv, d_h), _bf16(S, L_max, d_idx),
                          torch.zeros(S, dtype=torch.int32), B_k, k)


def test_missing_library_is_an_import_error():
    code = (
        "import os\n"
        "real = os.path.exists\n"
        "os.path.exists = lambda p: False if str(p).endswith('libmsa_b200.so') else real(p)\n"
        "import block_sparse_gqa_idx_b200 as msa\n"
        "try:\n"
        "    msa.index_topk\n"
        "except ImportError as e:\n"
        "    print('IMPORT_ERROR', 'no fallback path' in str(e))\n"
    )
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "IMPORT_ERROR True" in r.stdout
