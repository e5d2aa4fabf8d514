"""Pins of the oracle's backward pass (gradients of Eq. 8 with the selection
fixed) against torch's autograd of its scaled-dot-product attention in fp64
with the selection as a boolean mask (a library routine), and the dense
special case: every visible block selected equals causal GQA attention."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from block_sparse_gqa_idx_b200 import inputs


def _f64(bits):
    return torch.from_numpy(inputs.bf16_to_f32(bits).astype(np.float64))


def _torch_grads(q, k, v, d_o, mask, G):
    """mask [N, H_kv, N] (query, group, key) -> torch's dQ, dK, dV (fp64)."""
    qt, kt, vt = (_f64(a).requires_grad_(True) for a in (q, k, v))
    # [heads, N, d] with each group's K/V repeated over its G heads
    Q = qt.permute(1, 0, 2)
    Kx = kt.permute(1, 0, 2).repeat_interleave(G, dim=0)
    Vx = vt.permute(1, 0, 2).repeat_interleave(G, dim=0)
    M = torch.from_numpy(mask).permute(1, 0, 2).repeat_interleave(G, dim=0)
    O = torch.nn.functional.scaled_dot_product_attention(Q, Kx, Vx, attn_mask=M)
    O.backward(_f64(d_o).permute(1, 0, 2))
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


def _mask_of(idx, N, B_k):
    H_kv = idx.shape[1]
    m = np.zeros((N, H_kv, N), dtype=bool)
    for i in range(N):
        for r in range(H_kv):
            for b in idx[i, r]:
                if b >= 0:
                    m[i, r, b * B_k:min((b + 1) * B_k, i + 1)] = True
    return m


def _inputs(N, H_q, H_kv, d_h, seed):
    rng = np.random.default_rng(seed)
    f = lambda *sh: inputs.bf16_bits(rng.standard_normal(sh).astype(np.float32))  # noqa: E731
    return f(N, H_q, d_h), f(N, H_kv, d_h), f(N, H_kv, d_h), f(N, H_q, d_h)


def test_backward_matches_torch_autograd_on_a_sparse_selection():
    N, H_q, H_kv, d_h, d_idx, B_k, k = 200, 8, 2, 16, 16, 16, 3
    q, kk, v, d_o = _inputs(N, H_q, H_kv, d_h, 1)
    rng = np.random.default_rng(2)
    qi = inputs.bf16_bits(rng.standard_normal((N, H_kv, d_idx)).astype(np.float32))
    ki = inputs.bf16_bits(rng.standard_normal((N, d_idx)).astype(np.float32))
    idx = oracle.index_topk(qi, ki, B_k, k)[0]
    dq, dk, dv = oracle.sparse_attn_bwd(q, kk, v, idx, d_o, B_k)
    tq, tk, tv = _torch_grads(q, kk, v, d_o, _mask_of(idx, N, B_k), H_q // H_kv)
    for got, want in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.abs(got - want).max() <= 1e-10 * max(1.0, np.abs(want).max())


def test_every_block_selected_gives_causal_gqa_gradients():
    N, H_q, H_kv, d_h, B_k = 96, 4, 1, 8, 16
    q, kk, v, d_o = _inputs(N, H_q, H_kv, d_h, 3)
    B = N // B_k
    idx = np.full((N, H_kv, B), -1, np.int32)
    for i in range(N):
        idx[i, :, : i // B_k + 1] = np.arange(i // B_k + 1)
    dq, dk, dv = oracle.sparse_attn_bwd(q, kk, v, idx, d_o, B_k)
    causal = np.tril(np.ones((N, N), dtype=bool))[:, None, :].repeat(H_kv, axis=1)
    tq, tk, tv = _torch_grads(q, kk, v, d_o, causal, H_q // H_kv)
    for got, want in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.abs(got - want).max() <= 1e-10 * max(1.0, np.abs(want).max())


def test_gradients_of_unselected_keys_are_zero():
    N, H_q, H_kv, d_h, B_k = 128, 4, 2, 8, 16
    q, kk, v, d_o = _inputs(N, H_q, H_kv, d_h, 4)
    idx = np.stack([np.full((H_kv,), i // B_k) for i in range(N)])[:, :, None].astype(np.int32)
    idx[:, 1, 0] = -1  # group 1 selects nothing: its K/V and its queries get no gradient
    idx[idx[:, 0, 0] >= 0, 0, 0] = np.minimum(idx[:, 0, 0], 2)[idx[:, 0, 0] >= 0]
    dq, dk, dv = oracle.sparse_attn_bwd(q, kk, v, idx, d_o, B_k)
    assert (dk[:, 1] == 0).all() and (dv[:, 1] == 0).all() and (dq[:, 2:] == 0).all()
    assert (dk[3 * B_k:, 0] == 0).all() and (dv[3 * B_k:, 0] == 0).all()
