"""Pins of the oracle's FP8 (E4M3) paged decode, checked against things
outside it: torch's float8_e4m3fn for the code values and the rounding, the
closed form of per-row scaling, and the bf16 decode oracle (itself pinned in
test_oracle_pins.py) on caches that E4M3 represents exactly."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_gqa_idx_b200 import inputs


def test_e4m3_values_match_torch():
    v = oracle.e4m3_values()
    t = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(v), np.isnan(t)) and np.isnan(v).sum() == 2
    fin = ~np.isnan(v)
    assert np.array_equal(v[fin], t[fin])
    assert v[0x7E] == 448.0 and v[0x01] == 2.0 ** -9 and v[0x08] == 2.0 ** -6


def test_e4m3_encode_rounds_to_nearest_even_and_saturates():
    rng = np.random.default_rng(0)
    vals = oracle.e4m3_values()[:0x7F]  # the non-negative finite values, ascending
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)  # exact ties
    x = np.concatenate([rng.standard_normal(4000).astype(np.float32) * np.float32(s)
                        for s in (1e-3, 0.05, 1.0, 30.0, 300.0)] + [mids, -mids])
    x = np.clip(x, -448, 448).astype(np.float32)
    got = oracle.e4m3_encode(x)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)
    # ties go to the even code: the midpoint between codes c and c+1
    for c in range(0, 0x7E):
        assert oracle.e4m3_encode(np.float32(mids[c])) == (c if c % 2 == 0 else c + 1)
    # saturation, signed zero, NaN
    sat = oracle.e4m3_encode(np.array([449.0, 500.0, 1e30, -1e30], dtype=np.float32))
    assert sat.tolist() == [0x7E, 0x7E, 0x7E, 0xFE]
    assert oracle.e4m3_encode(np.float32(-0.0)) == 0x80
    assert oracle.e4m3_encode(np.float32(np.nan)) == 0x7F


def test_quantize_rows_scale_and_error_bound():
    rng = np.random.default_rng(1)
    x = inputs.bf16_bits(rng.standard_normal((64, 128)).astype(np.float32) * 3)
    x[5] = 0  # an all-zero row: scale 1, codes 0
    codes, scales = oracle.quantize_rows(x)
    xf = inputs.bf16_to_f32(x)
    amax = np.abs(xf).max(axis=1)
    want = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(scales, want)
    assert (codes[5] == 0).all()
    deq = oracle.e4m3_values()[codes] * scales[:, None]
    # each code is within half a step of E4M3 (3 mantissa bits) of x / scale
    y = xf / scales[:, None]
    err = np.abs(deq / scales[:, None] - y)
    assert (err <= np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) + 1e-12).all()
    # the row maximum lands exactly on +-448
    assert (np.abs(oracle.e4m3_values()[codes[np.arange(64) != 5].max(axis=1) & 0x7F]) > 0).all()
    for t in range(64):
        if t != 5:
            assert 0x7E in (codes[t] & 0x7F)


def _exact_fp8_state(S, L0, L_max, H_kv, d_h, d_idx, B_k, seed, min_abs=0.0):
    """An FP8 paged cache with scale 1 everywhere (values = E4M3 values, exact
    in bf16), its bf16 twin in the contiguous decode layout, and a random
    page table."""
    rng = np.random.default_rng(seed)
    vals = oracle.e4m3_values()
    finite = np.array([c for c in range(256) if not np.isnan(vals[c])
                       and min_abs <= abs(vals[c]) <= 8], dtype=np.uint8)
    n_blocks = (L_max + B_k - 1) // B_k
    P = S * n_blocks
    perm = rng.permutation(P).astype(np.int32)
    page_table = perm.reshape(S, n_blocks)
    pages = {
        "k_pages": rng.choice(finite, size=(P, B_k, H_kv, d_h)).astype(np.uint8),
        "v_pages": rng.choice(finite, size=(P, B_k, H_kv, d_h)).astype(np.uint8),
        "kidx_pages": rng.choice(finite, size=(P, B_k, d_idx)).astype(np.uint8),
        "k_scale": np.ones((P, B_k, H_kv), np.float32),
        "v_scale": np.ones((P, B_k, H_kv), np.float32),
        "kidx_scale": np.ones((P, B_k), np.float32),
        "page_table": page_table,
    }

    def contiguous(key):
        arr = pages[key][page_table.reshape(-1)]  # [S * n_blocks, B_k, ...]
        arr = arr.reshape((S, n_blocks * B_k) + arr.shape[2:])[:, :L_max]
        return inputs.bf16_bits(vals[arr].astype(np.float32))

    state = {"k_cache": contiguous("k_pages"), "v_cache": contiguous("v_pages"),
             "k_idx_cache": contiguous("kidx_pages"),
             "seq_len": np.full(S, L0, dtype=np.int32)}
    return pages, state


def _exact_new_rows(rng, S, H_q, H_kv, d_h, d_idx):
    """New rows whose per-row maximum is 448, so quantization is exact."""
    vals = oracle.e4m3_values()
    ok = vals[[c for c in range(0x7F) if vals[c] <= 8]]

    def draw(shape):
        x = rng.choice(ok, size=shape) * rng.choice([-1.0, 1.0], size=shape)
        x[..., 0] = 448.0
        return inputs.bf16_bits(x.astype(np.float32))

    return {"q": inputs.bf16_bits(rng.standard_normal((S, H_q, d_h)).astype(np.float32)),
            "q_idx": inputs.bf16_bits(rng.standard_normal((S, H_kv, d_idx)).astype(np.float32)),
            "k_new": draw((S, H_kv, d_h)), "v_new": draw((S, H_kv, d_h)),
            "k_idx_new": draw((S, d_idx))}


@pytest.mark.parametrize("L0", [700, 1023, 1024, 1500])
def test_paged_fp8_decode_equals_bf16_decode_on_exact_caches(L0):
    """With scale 1 and E4M3 values exactly representable in bf16, the FP8
    paged step must reproduce the (pinned) bf16 decode oracle bit for bit,
    whatever the page order."""
    S, H_q, H_kv, d_h, d_idx, B_k, k = 3, 8, 2, 64, 32, 128, 4
    pages, state = _exact_fp8_state(S, L0, 1536, H_kv, d_h, d_idx, B_k, seed=L0)
    si = _exact_new_rows(np.random.default_rng(L0 + 1), S, H_q, H_kv, d_h, d_idx)
    got = oracle.paged_decode_fp8(pages, si, state["seq_len"], B_k, k)
    ref = oracle.decode_reference(state, si, B_k, k)
    assert np.array_equal(got["idx"], ref["idx"])
    assert np.array_equal(got["o"], ref["o"]) and np.array_equal(got["lse"], ref["lse"])
    # the new token's rows quantize exactly (scale 1)
    assert (got["new_kv_scale"] == 1.0).all() and (got["new_kidx_scale"] == 1.0).all()
    vals = oracle.e4m3_values()
    assert np.array_equal(inputs.bf16_bits(vals[got["new_k"]].astype(np.float32)), si["k_new"])


def test_paged_fp8_decode_page_order_and_scales():
    """Renumbering the physical pages changes nothing; scaling a token's codes
    by a power of two in its scale changes nothing either."""
    S, H_q, H_kv, d_h, d_idx, B_k, k = 2, 16, 2, 64, 64, 64, 5
    # codes of magnitude >= 2^-5: every one has an exact half
    pages, state = _exact_fp8_state(S, 900, 1024, H_kv, d_h, d_idx, B_k, seed=7,
                                    min_abs=2.0 ** -5)
    si = _exact_new_rows(np.random.default_rng(8), S, H_q, H_kv, d_h, d_idx)
    base = oracle.paged_decode_fp8(pages, si, state["seq_len"], B_k, k)
    P = pages["k_pages"].shape[0]
    rng = np.random.default_rng(9)
    new_of_old = rng.permutation(P)
    moved = dict(pages)
    for key in ("k_pages", "v_pages", "kidx_pages", "k_scale", "v_scale", "kidx_scale"):
        arr = np.empty_like(pages[key])
        arr[new_of_old] = pages[key]
        moved[key] = arr
    moved["page_table"] = new_of_old[pages["page_table"]].astype(np.int32)
    again = oracle.paged_decode_fp8(moved, si, state["seq_len"], B_k, k)
    for key in ("idx", "o", "lse"):
        assert np.array_equal(base[key], again[key]), key
    # halve every code's value and double its scale: exactly the same values
    vals = oracle.e4m3_values()
    half = {}
    for c in range(256):
        if np.isnan(vals[c]) or abs(vals[c]) < 2.0 ** -5:
            continue
        hit = np.nonzero(vals == vals[c] / 2)[0]
        half[c] = int(hit[0])
    sc = dict(pages)
    for key, skey in (("k_pages", "k_scale"), ("v_pages", "v_scale"), ("kidx_pages", "kidx_scale")):
        sc[key] = np.vectorize(lambda c: half[int(c)])(pages[key]).astype(np.uint8)
        sc[skey] = pages[skey] * np.float32(2.0)
    assert not np.array_equal(sc["k_pages"], pages["k_pages"])
    scaled = oracle.paged_decode_fp8(sc, si, state["seq_len"], B_k, k)
    for key in ("idx", "o", "lse"):
        assert np.array_equal(base[key], scaled[key]), key
