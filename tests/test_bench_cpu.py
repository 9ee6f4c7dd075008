"""Host-side checks of the bench's roofline arithmetic (no GPU)."""
import json
import os

import torch

import bench
from persistent_decode_megakernel_02_b200 import workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))


def test_bandwidth_bound_matches_the_pages_worked_example():
    g = json.load(open(os.path.join(HERE, "golden", "bandwidth_bound_a100.json")))
    assert abs(bench.bandwidth_bound_ms(g["bytes_per_step"], g["bandwidth_gbs"]) - g["bound_ms"]) < 1e-12


def test_step_weight_bytes_counts_each_generated_tensor_once():
    # independent count: the bytes of the tensors the generator makes for a
    # small shape, minus the embedding table but plus one embedding row
    shape = wl.ModelShape("s", 3, 64, 4, 2, 16, 96, 50, False, 1e4)
    w = wl.make_weights(shape, seed=1, device="cpu")
    total = sum(t.numel() * 2 for k in ("attn_norm", "mlp_norm", "wq", "wk", "wv", "wo", "wg", "wu", "wd")
                for t in getattr(w, k))
    total += w.final_norm.numel() * 2 + w.lm_head.numel() * 2 + shape.hidden * 2
    assert bench.step_weight_bytes(shape) == total


def test_one_b_shape_step_bytes():
    assert bench.step_weight_bytes(wl.LLAMA_1B) == 2_471_632_896
    # K and V, 8 heads x 64 dims bf16, 16 layers: 32 KiB per attended position
    assert bench.step_kv_bytes(wl.LLAMA_1B, [1]) == 32768
