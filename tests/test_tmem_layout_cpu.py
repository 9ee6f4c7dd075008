"""The TMEM page order and the page-aligned task split (no GPU).

Weights of the ops whose pages pass through tensor memory are stored so that
one tcgen05.cp.128x256b per 4 KB block (no swizzle, leading offset 2048 B,
stride offset 128 B) hands every worker warp its two page rows, each as 32
consecutive columns of its own lane quarter, vectors in the order the
shared-memory path reads them.  layout_check.cpp checks the permutation
(mk_internal.h, tmem_page_src) against that copy's lane/column mapping; the
planner must then start every such task on a 16-page-row boundary.
"""
import os
import subprocess

import numpy as np
import pytest

from persistent_decode_megakernel_02_b200 import workloads as wl

mk = pytest.importorskip("persistent_decode_megakernel_02_b200.mk")

HERE = os.path.dirname(os.path.abspath(__file__))
QKV, ATTN, OPROJ, GATEUP, DOWN, LMHEAD = range(6)


def test_tmem_page_order_matches_the_copy_lane_mapping(tmp_path):
    exe = str(tmp_path / "layout_check")
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-I/usr/local/cuda/include",
                           os.path.join(HERE, "layout_check.cpp"), "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout


@pytest.mark.parametrize("shape", [wl.LLAMA_1B, wl.LLAMA_8B], ids=["1b", "8b"])
def test_tasks_of_tmem_ops_start_on_page_boundaries(shape):
    cfg = mk.make_config(shape, 560, 1)
    pl = mk.plan(cfg, 148)
    K = {QKV: shape.hidden, OPROJ: shape.n_q_heads * shape.head_dim, GATEUP: shape.hidden,
         DOWN: shape.ffn, LMHEAD: shape.hidden}
    for t in pl["tasks"]:
        kind, begin = int(t[0]), int(t[4])
        if kind == ATTN or K[kind] % 2048 or K[kind] // 2048 not in (1, 2, 4):
            continue
        rows = begin * (16 if kind == GATEUP else 8)          # first row of the task
        assert (rows * (K[kind] // 2048)) % 16 == 0, (kind, begin)
    # the flag that keeps every page in shared memory lifts the constraint:
    # the q/k/v split then uses single 8-row tiles again
    pl2 = mk.plan(mk.make_config(shape, 560, 1, flags=mk.MK_FLAG_NO_TMEM_RING), 148)
    begins = [int(t[4]) for t in pl2["tasks"] if t[0] == QKV and t[1] == 0]
    if shape is wl.LLAMA_1B:
        assert any(b % 2 for b in begins)
