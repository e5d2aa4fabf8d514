"""Pins of the oracle's packed-batch forward (several sequences along the
token axis), against facts that do not come from the oracle itself: a
sequence's first token can only attend to itself (closed form), and no
sequence sees another's tokens (changing one sequence changes no other)."""
from __future__ import annotations

import numpy as np

import oracle
from block_sparse_gqa_idx_b200 import inputs

CFG = inputs.MSAConfig("vl", 0, 8, 2, 64, 32, 64, 4, "sink_ar1", seed_index=31)
LENGTHS = [300, 1, 0, 129, 64, 200]


def test_first_token_of_each_sequence_attends_to_itself_only():
    inp, cu = inputs.varlen_inputs(CFG, LENGTHS)
    first = np.array([cu[s] for s in range(len(LENGTHS)) if LENGTHS[s] > 0])
    r = oracle.forward_varlen(inp, cu, CFG.B_k, CFG.k, rows=first)
    G = CFG.H_q // CFG.H_kv
    v = inputs.bf16_to_f32(inp["v"][first]).astype(np.float64)
    q = inputs.bf16_to_f32(inp["q"][first]).astype(np.float64)
    kk = inputs.bf16_to_f32(inp["k"][first]).astype(np.float64)
    for t in range(first.size):
        for r_ in range(CFG.H_kv):
            assert r["idx"][t, r_].tolist() == [0] + [-1] * (CFG.k - 1)
        for h in range(CFG.H_q):
            # one visible token: softmax weight 1, O = v, LSE = the one logit
            assert np.array_equal(r["o"][t, h], v[t, h // G])
            logit = float(q[t, h] @ kk[t, h // G]) / np.sqrt(CFG.d_h)
            assert abs(r["lse"][t, h] - logit) <= 1e-12 * max(1.0, abs(logit))


def test_sequences_do_not_see_each_other():
    inp, cu = inputs.varlen_inputs(CFG, LENGTHS)
    base = oracle.forward_varlen(inp, cu, CFG.B_k, CFG.k)
    # redraw every input of sequence 0: the other sequences' results stay
    rng = np.random.default_rng(5)
    other = {key: val.copy() for key, val in inp.items()}
    a, b = int(cu[0]), int(cu[1])
    for key in other:
        other[key][a:b] = inputs.bf16_bits(
            rng.standard_normal(other[key][a:b].shape).astype(np.float32) * 3)
    again = oracle.forward_varlen(other, cu, CFG.B_k, CFG.k)
    rest = np.arange(b, int(cu[-1]))
    for key in ("idx", "o", "lse"):
        assert np.array_equal(base[key][rest], again[key][rest]), key
    assert not np.array_equal(base["o"][a:b], again["o"][a:b])


def test_one_sequence_equals_the_single_sequence_forward():
    inp, cu = inputs.varlen_inputs(CFG, [777])
    a = oracle.forward_varlen(inp, cu, CFG.B_k, CFG.k)
    b = oracle.forward(inp, CFG.B_k, CFG.k)
    for key in ("idx", "o", "lse"):
        assert np.array_equal(a[key], b[key]), key


def test_varlen_lengths_recipe():
    L = inputs.varlen_lengths(32, 131072, 512, 16384, seed=3)
    assert L.sum() == 131072 and L.size == 32 and (L >= 1).all()
    assert np.array_equal(L, inputs.varlen_lengths(32, 131072, 512, 16384, seed=3))
