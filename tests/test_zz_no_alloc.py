"""The decode entry point that allocates nothing (msa_sparse_decode_noalloc).

It serves callers that cannot hand the library device memory during a decode
step (a plain-C host program without a device allocator, or a serving loop
whose memory is fully reserved up front); it uses the library's fixed scratch
array instead of a workspace.  Here it is called through the C ABI and checked
against the workspace-taking entry point, msa_sparse_decode, on the same
inputs, for two consecutive steps (the scratch keeps the previous call's
contents, so the second step also checks that nothing stale leaks through).

This file is collected last, so a run that stops at the first failure has
already run every other test; it also passes alone in a fresh process.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from block_sparse_gqa_idx_b200 import inputs
from tests import compare
from tests.gpu_util import bf16_to_f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def capi():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_gqa_idx_b200 import _capi

    return _capi


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_decode_matches_workspace_entry_point(capi):
    cfg = inputs.DecodeConfig("noalloc", S=6, L0=3000, steps=2, H_q=32, H_kv=4, d_h=128,
                              d_idx=64, B_k=128, k=16, seed_index=59)
    st = inputs.decode_state(cfg)
    # two identical copies of the caches: one per entry point
    caches = [{k: to_dev(st[k]) for k in ("k_cache", "v_cache", "k_idx_cache")} for _ in range(2)]
    lens = [torch.from_numpy(st["seq_len"].copy()).cuda() for _ in range(2)]
    d = capi.decode_dims(cfg.S, cfg.L_max, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.B_k, cfg.k)
    ws = torch.empty(capi.sparse_decode_workspace_size(d), dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for step in range(2):
        si = {k: to_dev(v) for k, v in inputs.decode_step_inputs(cfg, step, st["sink"]).items()}
        outs = []
        for which in range(2):
            c = caches[which]
            o = torch.full((cfg.S, cfg.H_q, cfg.d_h), float("nan"), dtype=torch.bfloat16,
                           device="cuda")
            idx = torch.full((cfg.S, cfg.H_kv, cfg.k), -7, dtype=torch.int32, device="cuda")
            args = [_ptr(si["q"]), _ptr(si["q_idx"]), _ptr(si["k_new"]), _ptr(si["v_new"]),
                    _ptr(si["k_idx_new"]), _ptr(c["k_cache"]), _ptr(c["v_cache"]),
                    _ptr(c["k_idx_cache"]), _ptr(lens[which]), _ptr(o), _ptr(idx)]
            if which == 0:
                rc = capi.LIB.msa_sparse_decode(ctypes.byref(d), *args, _ptr(ws), ws.numel(),
                                                stream)
            else:
                rc = capi.LIB.msa_sparse_decode_noalloc(ctypes.byref(d), *args, stream)
            assert rc == 0, (which, rc)
            outs.append((o, idx))
        torch.cuda.synchronize()
        (o_ref, i_ref), (o_na, i_na) = outs
        assert torch.equal(i_ref, i_na), f"step {step}: selections differ"
        compare.assert_attn_close(bf16_to_f64(o_na), bf16_to_f64(o_ref), what=f"step {step}")
        assert torch.equal(lens[0], lens[1])
    assert lens[1].cpu().tolist() == [cfg.L0 + 2] * cfg.S


def test_noalloc_rejects_problems_beyond_the_fixed_scratch(capi):
    # 512 sequences x 32 slots of fp32 partials need far more than the fixed array
    d = capi.decode_dims(512, 1 << 20, 64, 4, 128, 64, 128, 32)
    assert capi.sparse_decode_workspace_size(d) > (64 << 20)
    fake = ctypes.c_void_p(1 << 20)
    rc = capi.LIB.msa_sparse_decode_noalloc(ctypes.byref(d), *([fake] * 11), None)
    assert rc == 3  # MSA_ERR_WORKSPACE_TOO_SMALL, nothing launched
