"""Host-side checks of the bench's roofline arithmetic (no GPU)."""
import json
import os

import numpy as np
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


def _clock_rows(path, rows):
    # nvidia-smi csv,noheader,nounits: index, clocks.sm, clocks.max.sm,
    # power.draw, reasons.active, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    with open(path, "w") as f:
        for r in rows:
            f.write(", ".join(str(x) for x in r) + "\n")


def test_clock_summary_takes_the_loaded_samples_and_their_reasons(tmp_path):
    p = str(tmp_path / "c.csv")
    idle = [(0, 1980, 1965, 150.0, "0x0", "Not Active", "Not Active", "Not Active", "Not Active")] * 4
    busy = [(0, 1965, 1965, 900.0, "0x4", "Not Active", "Not Active", "Not Active", "Active")] * 5
    _clock_rows(p, idle + busy + ["garbage line"])
    c = bench.ClockSampler(0, p)
    c.proc = object()            # as if nvidia-smi had run
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 9
    assert os.path.exists(p)     # a caller's file is kept


def test_clock_summary_flags_thermal_slowdown_and_missing_samples(tmp_path):
    p = str(tmp_path / "c.csv")
    rows = [(0, 1500, 1965, 950.0, "0x20", "Not Active", "Active", "Not Active", "Not Active")] * 3
    _clock_rows(p, rows)
    c = bench.ClockSampler(0, p)
    c.proc = object()
    assert c.summary()["reasons"] == ["hw_thermal_slowdown"]
    empty = bench.ClockSampler(0)    # temporary file, nothing sampled
    assert empty.summary()["reasons"] == ["unsampled"]
    assert not os.path.exists(empty.path)
    t = bench.ClockSampler(0)
    _clock_rows(t.path, rows)
    t.proc = object()
    assert t.summary()["sm_mhz"] == 1500.0
    assert not os.path.exists(t.path)   # its own temporary file is removed


def test_oracle_baseline_times_full_steps_pinned_to_one_core():
    # the CPU baseline and the reference arm time whole oracle decode steps
    # (every layer and LM-head row), on one pinned core, and restore the mask
    import os
    shape = wl.TINY
    w = wl.make_weights(shape, seed=3, device="cpu")
    runner = bench.OracleRunner(shape, w.numpy_bits(), 32, 0)
    before = os.sched_getaffinity(0)
    with bench.PinnedCore() as pin:
        assert os.sched_getaffinity(0) == {pin.core}
        times = bench.run_oracle_steps(runner, [5, 6, 7, 8, 9], list(range(5)), 2, 10, 0.0)
    assert os.sched_getaffinity(0) == before
    # budget 0: the minimum of 3 timed steps after the 2 warm-up ones
    assert len(times) == 3 and all(t > 0 for t in times)
    # the runner's cache advanced through every step: position 4 was written
    assert any(np.any(k[:, 4] != 0) for k in runner.kc)


def test_profiled_traffic_is_keyed_to_the_profiled_kernel_sources(tmp_path, monkeypatch):
    import json
    import bench
    csrc = tmp_path / "persistent_decode_megakernel_02_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in set(bench.STEP_KERNEL_SOURCES) | set(bench.ROWS_KERNEL_SOURCES):
        (csrc / name).write_text(f"// {name}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    entries = [{"workload": "llama1b", "sources": list(bench.STEP_KERNEL_SOURCES),
                "kernel_digest": bench.kernel_digest(bench.STEP_KERNEL_SOURCES),
                "dram_bytes_read_per_launch": 1000, "dram_bytes_write_per_launch": 24},
               {"workload": "batched16", "sources": list(bench.ROWS_KERNEL_SOURCES),
                "kernel_digest": bench.kernel_digest(bench.ROWS_KERNEL_SOURCES),
                "dram_bytes_read_per_launch": 7, "dram_bytes_write_per_launch": 1}]
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"entries": entries}))
    assert bench.profiled_traffic("llama1b") == 1024
    assert bench.profiled_traffic("batched16") == 8
    assert bench.profiled_traffic("longctx") is None          # no capture for it
    # a change to the batched kernel's sources voids its record only
    (csrc / "mk_rows.cu").write_text("// changed\n")
    assert bench.profiled_traffic("batched16") is None
    assert bench.profiled_traffic("llama1b") == 1024
    # and a change to a shared header voids both
    (csrc / "mk_ptx.cuh").write_text("// changed\n")
    assert bench.profiled_traffic("llama1b") is None


def test_reference_arm_of_a_batched_workload_times_the_oracle(capsys):
    # the reference arm of a batched workload reports the kernel arm's metric
    # and config, and its oracle steps visit every sequence at its own
    # staggered position (steps j, j + B, ... belong to sequence j)
    import argparse
    wk = wl.Workload("tiny4", wl.TINY, 4, 0, 8, 2112, prefill_len=2048, staggered=True)
    args = argparse.Namespace(ref_budget_s=0.0)
    seen = []
    real = bench.OracleRunner.step_ms

    def spy(self, token, pos):
        seen.append(int(pos))
        return real(self, token, pos)

    bench.OracleRunner.step_ms = spy
    try:
        bench.main_reference(args, 1, 0, wk, 3, 5)
    finally:
        bench.OracleRunner.step_ms = real
    rec = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    starts, _, metric, config = bench.batched_workload(wk, 3, 5, 1)
    assert rec["impl"] == "reference" and rec["metric"] == metric and rec["config"] == config
    assert rec["unit"] == "ms/token" and rec["value"] > 0 and rec["steps"] == 3
    assert seen == [int(starts[j % 4]) + j // 4 for j in range(6)]
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["e2e"]["h2d_bytes_per_step"] == 0
