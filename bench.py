"""Decode-step benchmark of the persistent megakernel (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama1b]
                    [--impl mk|reference] [--no-cpu-baseline]

A step is one decode step (the whole hot path: every layer's fused
RMSNorm->QKV->RoPE->KV append, split-K attention + merge, O-proj+residual,
RMSNorm->gate/up->SiLU*up, down+residual, then final norm->LM head->argmax)
for one sequence, run as one persistent-kernel launch through the C ABI.
Warm-up steps feed the synthetic prompt at positions 0..W-1; the K timed
steps continue autoregressively on the device (each step reads the token
the previous step wrote) at positions W..W+K-1.  Weights (2.47 GB for the
1B shape) exceed the 126 MB L2, so no flush is needed between steps.

`value` is device time per token (CUDA events over the K launches on the
launching stream, max over ranks); `e2e` is the same through host buffers:
per step the token and position are copied from pinned host memory, the
step launched, and the next token copied back and waited for.  `generate`
times the same K steps as ONE launch (mk_generate: the kernel runs the
steps back to back, each step's argmax feeding the next on the device).

Multi-GPU: every rank runs an independent replica (the single-sequence step
does not shard without a per-layer exchange); `value` is then the max rank
time divided by all ranks' tokens.

--impl reference times the oracle (the plain fp64 CPU definition in
oracle/) on the host, single-threaded and pinned to one core: W untimed and
then K timed FULL decode steps of the same shape, weights and positions
(every layer, every LM-head row), stopping early once --ref-budget-s has
passed (the line's `steps` is then the number actually timed).  The CPU
baseline leg of the default arm times full oracle steps the same way for
about --cpu-sample-s seconds (at least 3 steps).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from persistent_decode_megakernel_02_b200 import workloads as wl  # noqa: E402

METRIC = "decode ms/token @bs1 (Llama-3.2-1B shape); achieved HBM GB/s vs roofline"
UNIT = "ms/token"


# ---------------------------------------------------------------------------
# algorithmic bytes (the roofline numerator)
# ---------------------------------------------------------------------------
def step_weight_bytes(shape: wl.ModelShape) -> int:
    """bf16 bytes one decode step must read: every weight matrix once, every
    RMSNorm gain once, one embedding row (the LM head is read in full)."""
    H, F, V, L = shape.hidden, shape.ffn, shape.vocab, shape.layers
    QD, KD = shape.n_q_heads * shape.head_dim, shape.n_kv_heads * shape.head_dim
    mats = L * ((QD + 2 * KD) * H + H * QD + 3 * F * H) + V * H
    norms = (2 * L + 1) * H
    return 2 * (mats + norms + H)


def step_kv_bytes(shape: wl.ModelShape, contexts) -> int:
    """bf16 K and V bytes attention reads: C positions per sequence per layer."""
    per_pos = 2 * shape.n_kv_heads * shape.head_dim * 2 * shape.layers
    return int(per_pos * int(np.sum(contexts)))


def bandwidth_bound_ms(bytes_per_step: float, gbs: float) -> float:
    """Time to stream `bytes_per_step` at `gbs` GB/s (1 GB = 1e9 B)."""
    return bytes_per_step / (gbs * 1e9) * 1e3


STEP_KERNEL_SOURCES = ("mk_kernel.cu", "mk_internal.h", "mk_ptx.cuh")
ROWS_KERNEL_SOURCES = ("mk_rows.cu", "mk_rows.h", "mk_internal.h", "mk_ptx.cuh")


def kernel_digest(sources=STEP_KERNEL_SOURCES) -> str:
    """Hash of the sources a kernel is compiled from."""
    import hashlib
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "persistent_decode_megakernel_02_b200", "csrc", name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()


def step_kernel_digest() -> str:
    """Hash of the sources the batch-1 step kernel is compiled from."""
    return kernel_digest(STEP_KERNEL_SOURCES)


def profiled_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu capture of the kernel
    that runs `workload` (profiles/traffic.json, one record per workload),
    only while that kernel's sources are the ones profiled (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    for e in t.get("entries", []):
        if e.get("workload") != workload:
            continue
        try:
            if e.get("kernel_digest") != kernel_digest(tuple(e.get("sources", STEP_KERNEL_SOURCES))):
                return None
        except OSError:
            return None
        return int(e["dram_bytes_read_per_launch"]) + int(e["dram_bytes_write_per_launch"])
    return None


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, path: str | None = None):
        """`path`: where the raw samples go (CSV); a temporary file if None."""
        self.dev = device_index
        self.proc = None
        self.tmp = path is None
        if path is None:
            fd, path = tempfile.mkstemp(prefix=f"mk_clocks_{device_index}_", suffix=".csv")
            os.close(fd)
        self.path = path

    def __enter__(self):
        try:
            d = os.path.dirname(self.path)
            if d:
                os.makedirs(d, exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        lines = []
        if os.path.exists(self.path):
            with open(self.path) as f:
                lines = f.readlines()
            if self.tmp:
                os.remove(self.path)
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        rows = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        pw = np.array([r[2] for r in rows])
        load = [r for r in rows if r[2] >= np.median(pw)] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in load:
            for n, v in zip(names, r[3][1:5]):
                if v.lower() in ("active", "1", "yes"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median([r[0] for r in load])),
                "sm_max_mhz": float(max(r[1] for r in rows)),
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------
class OracleRunner:
    """The oracle (the plain fp64 C decode step in oracle/) on the full model
    of `shape`, same weights, one sequence.  Every timed step is one whole
    decode step: every layer and every LM-head row.  The KV cache starts
    from the same seeded prefix the GPU side uses (zeros beyond it)."""

    def __init__(self, shape: wl.ModelShape, bits: dict, max_seq: int, prefill: int):
        import oracle
        cfg = dict(layers=shape.layers, hidden=shape.hidden, n_q_heads=shape.n_q_heads,
                   n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, ffn=shape.ffn,
                   vocab=shape.vocab, max_seq=max_seq, rope_theta=shape.rope_theta,
                   rms_eps=shape.rms_eps)
        self.model = oracle.OracleModel(cfg, bits)
        self.kc, self.vc = self.model.new_cache()
        if prefill:
            k, v = wl.make_kv(shape, 1, max_seq, device="cpu", prefill_len=prefill)
            for l in range(shape.layers):
                self.kc[l][...] = wl.cache_bits(k[l][0])
                self.vc[l][...] = wl.cache_bits(v[l][0])
        self.next = 0

    def step_ms(self, token: int, pos: int) -> float:
        t0 = time.perf_counter()
        out = self.model.decode_step(self.kc, self.vc, int(token), int(pos))
        dt = (time.perf_counter() - t0) * 1e3
        self.next = out["next"]
        return dt


class PinnedCore:
    """Pin the calling thread to one core for the duration (the oracle is
    single-threaded C called from this thread); restores the old mask."""

    def __enter__(self):
        self.old = None
        self.core = None
        try:
            self.old = os.sched_getaffinity(0)
            self.core = min(self.old)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            pass
        return self

    def __exit__(self, *a):
        if self.old is not None:
            try:
                os.sched_setaffinity(0, self.old)
            except OSError:
                pass


def host_cores() -> int:
    return os.cpu_count() or 1


def run_oracle_steps(runner: OracleRunner, tokens, positions, n_warm: int, n_max: int,
                     budget_s: float, min_steps: int = 3):
    """n_warm untimed full steps, then full steps until n_max steps or the
    time budget (at least min_steps).  Returns the per-step times (ms)."""
    for i in range(n_warm):
        runner.step_ms(tokens[i], positions[i])
    times = []
    t_end = time.perf_counter() + budget_s
    i = n_warm
    while len(times) < n_max and (len(times) < min_steps or time.perf_counter() < t_end):
        times.append(runner.step_ms(tokens[i % len(tokens)], positions[i % len(positions)]))
        i += 1
    return times


def batched_workload(wk, W: int, K: int, world: int):
    """Start positions, KV capacity, metric and config of a batched workload
    (the same for the kernel's arm and the reference arm)."""
    shape, B = wk.shape, wk.batch
    starts = wl.make_start_positions(B, seed=7)
    max_seq = max(wk.max_seq, int(starts.max()) + W + K + 1)
    metric = (f"decode ms/token @bs{B} ({shape.name}, staggered positions); achieved HBM GB/s vs roofline")
    config = {"workload": f"{wk.name}: {shape.name} L{shape.layers} H{shape.hidden} {shape.n_q_heads}/"
                          f"{shape.n_kv_heads} heads d{shape.head_dim} F{shape.ffn} V{shape.vocab}, {B} sequences "
                          f"starting at positions uniform in [32, 2048] (KV prefix N(0,1))",
              "batch": B, "start_positions": [int(x) for x in starts],
              "l2": "weights exceed L2 (no flush needed)", "parallelism": f"replicas x{world}"}
    return starts, max_seq, metric, config


def single_workload(wk, W: int, K: int, world: int):
    """First position, KV capacity and config of a batch-1 workload."""
    shape = wk.shape
    prefill = wk.prefill_len
    start = prefill if prefill else 0
    max_seq = max(wk.max_seq, start + W + K + 1)
    config = {"workload": f"{wk.name}: {shape.name} L{shape.layers} H{shape.hidden} "
                          f"{shape.n_q_heads}/{shape.n_kv_heads} heads d{shape.head_dim} "
                          f"F{shape.ffn} V{shape.vocab}" + (f", KV prefilled to {prefill}" if prefill else ""),
              "batch": 1, "positions": [start + W, start + W + K - 1],
              "l2": "weights exceed L2 (no flush needed)", "parallelism": f"replicas x{world}"}
    return start, max_seq, config


def main_reference(args, world, rank, wk, W, K):
    """--impl reference: the oracle as it stands, full decode steps on one
    pinned host core, for the same workload, metric and unit as the kernel's
    arm; rank 0 alone (the other ranks exit at once).  A batched workload's
    tokens are independent sequences, so its sample cycles through them:
    oracle step j decodes one token of sequence j mod B at that sequence's
    own position, and ms per oracle step is ms per token."""
    if rank != 0:
        return
    import torch
    shape = wk.shape
    w_host = wl.make_weights(shape, seed=1234, device="cuda" if torch.cuda.is_available() else "cpu")
    bits = w_host.numpy_bits()
    del w_host
    n_all = W + K
    prompt = wl.make_prompt(shape.vocab, n_all, seed=42)
    if wk.batch > 1:
        B = wk.batch
        starts, max_seq, metric, config = batched_workload(wk, W, K, world)
        positions = np.array([int(starts[j % B]) + j // B for j in range(n_all)])
        where = lambda n: f"step j decoding one token of sequence j mod {B} at its own position"
    else:
        start, max_seq, config = single_workload(wk, W, K, world)
        metric = METRIC
        positions = np.arange(start, start + n_all)
        where = lambda n: f"positions {start + W}..{start + W + n - 1}"
    runner = OracleRunner(shape, bits, max_seq, wk.prefill_len)
    with PinnedCore() as pin:
        t_run = time.perf_counter()
        times = run_oracle_steps(runner, prompt, positions, W, K, args.ref_budget_s)
        t_run = time.perf_counter() - t_run
    n = len(times)
    ms = float(np.mean(times))
    sample = (f"{n} full oracle decode steps (every layer, every LM-head row; fp64 C, "
              f"single thread pinned to core {pin.core} of {host_cores()}) after {W} untimed "
              f"ones, {where(n)}"
              + ("" if n == K else f"; {K} requested, capped by the {args.ref_budget_s:.0f} s budget"))
    out = {"impl": "reference", "metric": metric, "value": ms, "unit": UNIT, "n_gpus": world,
           "steps": n, "warmup": W, "ms_per_step": ms, "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config,
           "cpu_baseline": {"value": ms, "unit": UNIT, "cores": 1, "kind": "oracle",
                            "sample": sample, "pinned_core": pin.core, "host_cores": host_cores(),
                            "wall_s": round(t_run, 2)},
           "e2e": {"value": ms, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main_batched(args, world, rank, local, wk, W, K):
    """Batched decode (the batched tensor-core step): wk.batch independent
    sequences at start positions uniform in [32, 2048] over KV prefixes of
    seeded N(0,1) values; every step decodes one token of every sequence at
    its own position, each step's argmax feeding the next on the device."""
    import torch
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from persistent_decode_megakernel_02_b200 import mk
    shape, B = wk.shape, wk.batch
    starts, max_seq, metric, config = batched_workload(wk, W, K, world)
    weights = wl.make_weights(shape, seed=1234, device=dev)
    kc, vc = wl.make_kv(shape, B, max_seq, device=dev, prefill_len=wk.prefill_len)
    ctx = mk.Context(weights, kc, vc, max_seq, B)
    stream = torch.cuda.Stream(device=dev)
    pos = torch.tensor([[int(starts[b]) + i for b in range(B)] for i in range(W + K)], dtype=torch.int32,
                       device=dev)
    toks = torch.zeros(2, B, dtype=torch.int32, device=dev)
    toks[0] = torch.from_numpy(wl.make_prompt(shape.vocab, B, seed=42)).to(dev)

    def one(i):
        ctx.decode_step(toks[i % 2], pos[i], toks[(i + 1) % 2], None, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(W):
            one(i)
        stream.synchronize()
        st = ctx.sync(stream)
        if st != 0:
            raise mk.MkError(st, "warm-up")
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with ClockSampler(torch.cuda.current_device()) as clk:
            e0.record(stream)
            for i in range(W, W + K):
                one(i)
            e1.record(stream)
            stream.synchronize()
        st = ctx.sync(stream)
        if st != 0:
            raise mk.MkError(st, "timed steps")
        dev_ms = e0.elapsed_time(e1)
    dev_ms = max_over_ranks(dev_ms, world, dev)
    step_ms = dev_ms / K
    value = step_ms / (B * world)
    # roofline: every weight once per step (whatever the batch) plus every
    # sequence's K/V of its C positions
    contexts = np.array([[int(starts[b]) + i + 1 for b in range(B)] for i in range(W, W + K)])
    alg_bytes = step_weight_bytes(shape) + step_kv_bytes(shape, contexts) / K
    peaks = measured_peaks()
    achieved = alg_bytes / (step_ms * 1e-3) / 1e9
    flops = 2.0 * B * (step_weight_bytes(shape) / 2)   # one multiply-add per weight per row
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": profiled_traffic(wk.name),
                "peak_source": peaks["source"], "bytes_per_launch": int(alg_bytes),
                "bound_ms": round(bandwidth_bound_ms(alg_bytes, peaks["hbm_gbs"]), 4),
                "tensor_tflops": round(flops / (step_ms * 1e-3) / 1e12, 2)}
    # end to end: tokens and positions from pinned host memory, next tokens back
    e2e = None
    if not args.no_e2e:
        n = min(args.e2e_steps, K)
        h_tok = torch.zeros(B, dtype=torch.int32).pin_memory()
        h_pos = torch.zeros(B, dtype=torch.int32).pin_memory()
        h_next = torch.zeros(B, dtype=torch.int32).pin_memory()
        d_tok = torch.zeros(B, dtype=torch.int32, device=dev)
        d_pos = torch.zeros(B, dtype=torch.int32, device=dev)
        d_next = torch.zeros(B, dtype=torch.int32, device=dev)
        h_tok.copy_(toks[(W + K) % 2].cpu())
        with torch.cuda.stream(stream):
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for i in range(n):
                h_pos.copy_(torch.from_numpy((starts + W + K + i).astype(np.int32)))
                d_tok.copy_(h_tok, non_blocking=True)
                d_pos.copy_(h_pos, non_blocking=True)
                ctx.decode_step(d_tok, d_pos, d_next, None, stream=stream)
                h_next.copy_(d_next, non_blocking=True)
                stream.synchronize()
                h_tok.copy_(h_next)
            f1.record(stream)
            stream.synchronize()
            st = ctx.sync(stream)
            if st != 0:
                raise mk.MkError(st, "e2e steps")
            e2e_ms = f0.elapsed_time(f1)
        e2e_ms = max_over_ranks(e2e_ms, world, dev)
        e2e = {"value": round(e2e_ms / (n * B * world), 5), "unit": UNIT, "h2d_bytes_per_step": 8 * B,
               "d2h_bytes_per_step": 4 * B, "steps": n}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        runner = OracleRunner(shape, weights.numpy_bits(), max_seq, wk.prefill_len)
        ptoks = toks[0].cpu().numpy()
        with PinnedCore() as pin:
            times = run_oracle_steps(runner, ptoks, [int(starts[0]) + i for i in range(len(ptoks))], 0, K,
                                     args.cpu_sample_s)
        cpu = {"value": round(float(np.mean(times)), 3), "unit": UNIT, "cores": 1, "kind": "oracle",
               "pinned_core": pin.core, "host_cores": host_cores(),
               "sample": f"{len(times)} full oracle decode steps of one sequence (one token each; fp64 C, "
                         f"single thread pinned to core {pin.core} of {host_cores()}) from position {int(starts[0])}"}
    if rank == 0:
        out = {"metric": metric, "value": round(value, 5), "unit": UNIT, "n_gpus": world, "steps": K,
               "warmup": W, "ms_per_step": round(step_ms, 5), "higher_is_better": False, "scaling": "weak",
               "vs_baseline": None, "dtype": "bf16 weights/KV, tcgen05 bf16 (high + low) x bf16, fp32 accumulate",
               "data": "synthetic", "config": config, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
               "gpu_launches": K, "clocks": clk.summary(), "tokens_per_s": round(B * world / (step_ms * 1e-3), 1),
               "achieved_gbs": round(achieved, 1)}
        print(json.dumps(out), flush=True)
    ctx.close()
    if world > 1:
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------------------
def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512)
    ap.add_argument("--warmup", type=int, default=39)
    ap.add_argument("--workload", default="llama1b",
                    choices=["llama1b", "llama8b", "longctx", "tiny", "batched4", "batched8", "batched16"])
    ap.add_argument("--impl", default="mk", choices=["mk", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-generate", action="store_true",
                    help="skip the one-launch generation measurement")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prompt-in-one-launch measurement")
    ap.add_argument("--e2e-steps", type=int, default=64)
    ap.add_argument("--cpu-sample-s", type=float, default=8.0,
                    help="CPU baseline: time full oracle steps for about this long (at least 3)")
    ap.add_argument("--ref-budget-s", type=float, default=180.0,
                    help="--impl reference: stop timing oracle steps after this long")
    ap.add_argument("--flags", type=int, default=0, help="mk_config.flags")
    ap.add_argument("--attn-chunks", type=int, default=0)
    ap.add_argument("--clocks-csv", default=None,
                    help="keep the raw nvidia-smi clock samples of the timed region in this CSV "
                         "('{rank}' is replaced by the rank); default: a temporary file")
    return ap.parse_args()


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value: device times are taken as the max over
    ranks (all ranks call this the same number of times, in the same order)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_token(max_rank_ms: float, steps: int, world: int) -> float:
    """Whole-job time per token: every rank decodes `steps` tokens of its own
    replica in the slowest rank's time."""
    return max_rank_ms / (steps * world)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    W = max(3, args.warmup)
    K = max(1, args.steps)
    wk = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        return main_reference(args, world, rank, wk, W, K)
    if wk.batch > 1:
        return main_batched(args, world, rank, local, wk, W, K)
    shape = wk.shape
    prefill = wk.prefill_len
    start, max_seq, config = single_workload(wk, W, K, world)

    import torch
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from persistent_decode_megakernel_02_b200 import mk

    weights = wl.make_weights(shape, seed=1234, device=dev)
    kc, vc = wl.make_kv(shape, 1, max_seq, device=dev, prefill_len=prefill)
    ctx = mk.Context(weights, kc, vc, max_seq, 1, flags=args.flags, attn_chunks=args.attn_chunks)
    inf = ctx.info()
    config["attention_items"] = {"q_heads_per_item": inf.attn_heads, "chunks": inf.attn_chunks}
    stream = torch.cuda.Stream(device=dev)
    prompt = torch.from_numpy(wl.make_prompt(shape.vocab, W, seed=42)).to(dev)
    toks = torch.zeros(W + K + 1, dtype=torch.int32, device=dev)
    toks[:W] = prompt
    pos = torch.arange(start, start + W + K + 1, dtype=torch.int32, device=dev)
    logits = torch.empty(1, shape.vocab, dtype=torch.float32, device=dev)
    dummy_next = torch.zeros(1, dtype=torch.int32, device=dev)

    def one(i, next_slot):
        ctx.decode_step(toks[i:i + 1], pos[i:i + 1], next_slot, logits, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(W):           # prompt, teacher-forced
            one(i, dummy_next if i < W - 1 else toks[W:W + 1])
        stream.synchronize()
        st = ctx.sync(stream)
        if st != 0:
            raise mk.MkError(st, "warm-up")
        if world > 1:
            torch.distributed.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        clk_path = None
        if args.clocks_csv:
            clk_path = args.clocks_csv.replace("{rank}", str(rank))
        with ClockSampler(torch.cuda.current_device(), clk_path) as clk:
            e0.record(stream)
            for i in range(W, W + K):
                one(i, toks[i + 1:i + 2])
            e1.record(stream)
            stream.synchronize()
        st = ctx.sync(stream)
        if st != 0:
            raise mk.MkError(st, "timed steps")
        dev_ms = e0.elapsed_time(e1)
    dev_ms = max_over_ranks(dev_ms, world, dev)
    per_launch_ms = dev_ms / K
    value = job_ms_per_token(dev_ms, K, world)

    # ---- roofline of the kernel (the only kernel in the step)
    contexts = np.arange(start + W, start + W + K) + 1
    wbytes = step_weight_bytes(shape)
    kvbytes = step_kv_bytes(shape, contexts) / K
    alg_bytes = wbytes + kvbytes
    peaks = measured_peaks()
    achieved = alg_bytes / (per_launch_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": profiled_traffic(args.workload),
                "peak_source": peaks["source"], "bytes_per_launch": int(alg_bytes),
                "bound_ms": round(bandwidth_bound_ms(alg_bytes, peaks["hbm_gbs"]), 4)}

    # ---- end to end through host buffers
    e2e = None
    if not args.no_e2e:
        h_tok = torch.zeros(1, dtype=torch.int32).pin_memory()
        h_pos = torch.zeros(1, dtype=torch.int32).pin_memory()
        h_next = torch.zeros(1, dtype=torch.int32).pin_memory()
        d_tok = torch.zeros(1, dtype=torch.int32, device=dev)
        d_pos = torch.zeros(1, dtype=torch.int32, device=dev)
        d_next = torch.zeros(1, dtype=torch.int32, device=dev)
        n = min(args.e2e_steps, K)
        h_tok[0] = int(toks[W].item())
        p0 = start + W
        with torch.cuda.stream(stream):
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for i in range(n):
                h_pos[0] = p0 + i
                d_tok.copy_(h_tok, non_blocking=True)
                d_pos.copy_(h_pos, non_blocking=True)
                ctx.decode_step(d_tok, d_pos, d_next, logits, stream=stream)
                h_next.copy_(d_next, non_blocking=True)
                stream.synchronize()
                h_tok[0] = h_next[0]
            f1.record(stream)
            stream.synchronize()
            st = ctx.sync(stream)
            if st != 0:
                raise mk.MkError(st, "e2e steps")
            e2e_ms = f0.elapsed_time(f1)
        e2e_ms = max_over_ranks(e2e_ms, world, dev)
        e2e = {"value": round(job_ms_per_token(e2e_ms, n, world), 5), "unit": UNIT, "h2d_bytes_per_step": 8,
               "d2h_bytes_per_step": 4, "steps": n}

    # ---- the same K steps as one launch (mk_generate: each step's argmax
    # feeds the next on the device; same positions, free-running tokens)
    gen = None
    if not args.no_generate:
        g_out = torch.zeros(K, 1, dtype=torch.int32, device=dev)
        g_next = torch.zeros(1, dtype=torch.int32, device=dev)
        with torch.cuda.stream(stream):
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            g0 = torch.cuda.Event(enable_timing=True)
            g1 = torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            ctx.generate(toks[W:W + 1], pos[W:W + 1], K, g_out, g_next, stream=stream)
            g1.record(stream)
            stream.synchronize()
            st = ctx.sync(stream)
            if st != 0:
                raise mk.MkError(st, "generate")
            gen_ms = g0.elapsed_time(g1)
        gen_ms = max_over_ranks(gen_ms, world, dev)
        gen = {"value": round(job_ms_per_token(gen_ms, K, world), 5), "unit": UNIT, "steps": K, "launches": 1,
               "api": "mk_generate"}

    # ---- the prompt in one launch (mk_prefill on the batched tensor-core
    # step: 16 tokens per kernel step, one weight read per 16 tokens) against
    # the same prompt fed one token per launch through the batch-1 step
    pre = None
    if not args.no_prefill and wk.prompt_len > 1 and shape.hidden % 128 == 0:
        n = wk.prompt_len
        kc2, vc2 = wl.make_kv(shape, 1, max_seq, device=dev)
        ctx2 = mk.Context(weights, kc2, vc2, max_seq, 1, flags=mk.MK_FLAG_ROWS)
        ptok = torch.from_numpy(wl.make_prompt(shape.vocab, n, seed=42)).to(dev)
        pnext = torch.zeros(1, dtype=torch.int32, device=dev)
        with torch.cuda.stream(stream):
            for _ in range(2):
                ctx2.prefill(ptok, pnext, slot=0, start_pos=0, stream=stream)
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            p0 = torch.cuda.Event(enable_timing=True)
            p1 = torch.cuda.Event(enable_timing=True)
            reps = 5
            p0.record(stream)
            for _ in range(reps):
                ctx2.prefill(ptok, pnext, slot=0, start_pos=0, stream=stream)
            p1.record(stream)
            stream.synchronize()
            st = ctx2.sync(stream)
            if st != 0:
                raise mk.MkError(st, "prefill")
            pf_ms = p0.elapsed_time(p1) / reps
            # the same prompt one token per launch (batch-1 step, positions 0..n-1)
            q0 = torch.cuda.Event(enable_timing=True)
            q1 = torch.cuda.Event(enable_timing=True)
            ppos = torch.arange(0, n, dtype=torch.int32, device=dev)
            q0.record(stream)
            for i in range(n):
                ctx.decode_step(ptok[i:i + 1], ppos[i:i + 1], dummy_next, None, stream=stream)
            q1.record(stream)
            stream.synchronize()
            st = ctx.sync(stream)
            if st != 0:
                raise mk.MkError(st, "prompt token by token")
            tt_ms = q0.elapsed_time(q1)
        pf_ms = max_over_ranks(pf_ms, world, dev)
        tt_ms = max_over_ranks(tt_ms, world, dev)
        pre = {"tokens": n, "ms": round(pf_ms, 4), "launches": 1, "api": "mk_prefill",
               "ms_token_by_token": round(tt_ms, 4), "speedup": round(tt_ms / pf_ms, 2)}
        ctx2.close()
        del kc2, vc2

    # ---- CPU baseline: full oracle steps on one pinned core (rank 0, N=1)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        bits = weights.numpy_bits()
        runner = OracleRunner(shape, bits, max_seq, prefill)
        ptoks = toks.cpu().numpy()
        positions = pos.cpu().numpy()
        with PinnedCore() as pin:
            times = run_oracle_steps(runner, ptoks[W:W + K], positions[W:W + K], 0, K,
                                     args.cpu_sample_s)
        n = len(times)
        cpu = {"value": round(float(np.mean(times)), 3), "unit": UNIT, "cores": 1,
               "kind": "oracle", "pinned_core": pin.core, "host_cores": host_cores(),
               "sample": f"{n} full oracle decode steps (every layer, every LM-head row; fp64 C, "
                         f"single thread pinned to core {pin.core} of {host_cores()}) on the timed "
                         f"steps' tokens at positions {start + W}..{start + W + n - 1}; the oracle's "
                         f"cache holds the seeded prefix only (attention cost depends on C alone)"}

    if rank == 0:
        out = {"metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world,
               "steps": K, "warmup": W, "ms_per_step": round(per_launch_ms, 5),
               "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
               "dtype": "bf16 weights/KV, fp32 accumulate", "data": "synthetic",
               "config": config, "roofline": roofline, "cpu_baseline": cpu,
               "e2e": e2e, "generate": gen, "prefill": pre, "gpu_launches": K, "clocks": clk.summary(),
               "achieved_gbs": round(achieved, 1)}
        print(json.dumps(out), flush=True)
    ctx.close()
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
