"""Host-side logic of bench.py that needs no GPU: the DRAM-traffic figure is
tied to the code of the kernel it was captured on, and goes away when that
code changes (but not when only comments or code elsewhere in the file do)."""
from __future__ import annotations

import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_gqa_idx_b200", "csrc", "sparse_attn.cu")


def test_traffic_figures_match_the_current_kernels():
    for name in bench.NCU_TRAFFIC:
        traffic, where = bench.ncu_traffic(name, 131072)
        assert traffic is not None and traffic > 0 and "ncu capture" in where, name


def test_kernel_hash_ignores_comments_and_other_code():
    text = open(SRC, encoding="utf-8").read()
    h = bench.kernel_code_hash(text, "attn_phase1_kernel")
    line = "const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;"
    i = text.index("attn_phase1_kernel(")
    j = text.index(line, i)  # a line inside the kernel
    commented = text[:j] + line + "  // warp and lane" + text[j + len(line):]
    assert commented != text
    assert bench.kernel_code_hash(commented, "attn_phase1_kernel") == h
    elsewhere = text + "\n__global__ void unrelated_kernel() {}\n"
    assert bench.kernel_code_hash(elsewhere, "attn_phase1_kernel") == h


def test_kernel_hash_sees_a_code_change_inside_the_kernel():
    text = open(SRC, encoding="utf-8").read()
    h = bench.kernel_code_hash(text, "attn_phase1_kernel")
    i = text.index("attn_phase1_kernel(")
    j = text.index("const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;", i)
    changed = text[:j] + "const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;" + \
        text[j + len("const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;"):]
    assert bench.kernel_code_hash(changed, "attn_phase1_kernel") != h
