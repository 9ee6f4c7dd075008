"""Per-task scheduling overhead from the kernel's globaltimer trace.

The MPK blog translation ("显著提升小LLM的性能，所有kernel集成一个巨大kernel！",
the paragraph on task-transition cost) puts the price of moving from one task
to the next inside a persistent kernel at 1-2 us, against a kernel launch.
This module measures that price for this kernel from the per-task records
`mk_get_trace` returns (MK_FLAG_TRACE) and the static graph `mk_get_graph`
returns.

A task could start once (a) the event it depends on has fired -- the last of
the tasks that trigger that event has posted its completion -- and (b) the
previous task in its SM's queue has ended.  Its scheduling overhead is the
time from that moment to the moment the workers actually started it:

    overhead = t_start - max(fire(dep), end(previous task on the same SM))

`fire(e)` is the largest `t_end` among the tasks whose triggering event is e
(`t_end` is stamped once the workers have posted the completion).  A task
with no dependency (the first layer's QKV) or at the head of its queue drops
the missing term; a task with neither has no defined overhead (NaN).

In the default wait mode `t_start` is the moment every input word the task
reads carried this step's tag, so the overhead includes the data's round
trip; an attention task needs only its own heads' q/k/v words, not the whole
QKV op, so its overhead can be negative.  With MK_FLAG_EVENT_WAIT `t_start`
is the moment the scheduler warp saw the event counter reach its threshold
and released the task to the workers.

Host-side analysis only (numpy); nothing here runs on the decode path.
"""
from __future__ import annotations

import numpy as np

OP_NAMES = ("qkv", "attn", "oproj", "gateup", "down", "lmhead")


def task_overheads(trace: np.ndarray, tasks: np.ndarray, queue: np.ndarray,
                   qoff: np.ndarray) -> dict:
    """Decode one step's trace.

    trace: structured array (fields t_start, t_end, ...) indexed by task id,
    as `Context.trace()` returns it; tasks: int32 [n][8] (kind, layer, dep,
    trig, begin, end, sm, slot); queue: task ids grouped by SM in execution
    order; qoff: [num_sms + 1] offsets into queue.

    Returns per-task arrays (float64 ns, indexed by task id): `fire_dep`,
    `prev_end`, `ready` (= max of the two that exist), `overhead`
    (= t_start - ready), plus `kind`.
    """
    n = tasks.shape[0]
    t_start = trace["t_start"].astype(np.float64)
    t_end = trace["t_end"].astype(np.float64)
    trig = tasks[:, 3]
    dep = tasks[:, 2]
    # fire time of every event: the last posted completion among its triggers
    n_ev = int(trig.max()) + 1 if n else 0
    fire = np.full(n_ev, -np.inf)
    np.maximum.at(fire, trig, t_end)
    fire_dep = np.where(dep >= 0, fire[np.clip(dep, 0, max(n_ev - 1, 0))], np.nan)
    prev_end = np.full(n, np.nan)
    for sm in range(len(qoff) - 1):
        q = queue[qoff[sm]:qoff[sm + 1]]
        if len(q) > 1:
            prev_end[q[1:]] = t_end[q[:-1]]
    ready = np.fmax(fire_dep, prev_end)   # NaN only where both are missing
    return {"kind": tasks[:, 0].copy(), "fire_dep": fire_dep, "prev_end": prev_end,
            "ready": ready, "overhead": t_start - ready}


def summarize(overhead: np.ndarray, kind: np.ndarray) -> dict:
    """Median, p90, max (us) and count of the defined overheads, overall and
    per op kind."""
    def stats(v):
        v = v[~np.isnan(v)] / 1e3
        if v.size == 0:
            return {"n": 0}
        return {"n": int(v.size), "median_us": float(np.median(v)),
                "p90_us": float(np.percentile(v, 90)), "max_us": float(v.max()),
                "mean_us": float(v.mean())}
    out = {"all": stats(overhead)}
    for k, name in enumerate(OP_NAMES):
        sel = kind == k
        if np.any(sel):
            out[name] = stats(overhead[sel])
    return out


def critical_path(trace: np.ndarray, tasks: np.ndarray, layers=None) -> dict:
    """How each op extends the step: for the ops in graph order (layer by
    layer, then the LM head), `inc` = last t_done of the op - last t_done of
    the op before it, split into `to_ready` (until the op's last task was
    ready: its inputs fresh) and the rest; averaged per op kind over
    `layers` (default: all but the first and last two).  Values in us."""
    kind, layer = tasks[:, 0], tasks[:, 1]
    done = trace["t_done"].astype(np.float64)
    ready = trace["t_ready"].astype(np.float64)
    L = int(layer[kind != 5].max()) + 1 if np.any(kind != 5) else 0
    if layers is None:
        layers = range(1, max(L - 2, 1))
    rows = {}
    prev = None
    for l in range(L + 1):
        for k in range(6):
            sel = (kind == k) & (layer == l)
            if not np.any(sel):
                continue
            last = done[sel].max()
            if prev is not None and (l in layers or k == 5):
                rows.setdefault(OP_NAMES[k], []).append(((last - prev), (ready[sel].max() - prev)))
            prev = last
    out = {}
    for name, v in rows.items():
        a = np.asarray(v) / 1e3
        out[name] = {"inc_us": float(a[:, 0].mean()), "to_ready_us": float(a[:, 1].mean()), "n": len(v)}
    return out


def transitions(trace: np.ndarray, tasks: np.ndarray) -> dict:
    """Per-SM task transitions: for consecutive tasks a, b on one SM (in
    start order), medians (us) per kind of b of `tail` = t_end(a) - t_done(a)
    (end barrier and completion post), `to_ready` = t_ready(b) - t_end(a)
    (dispatch, prologue and the input round trip, waits included) and
    `compute` = t_done(b) - t_input(b)."""
    sm = tasks[:, 6]
    f = {k: trace[k].astype(np.float64) for k in ("t_ready", "t_start", "t_input", "t_done", "t_end")}
    rows = {}
    for s in np.unique(sm):
        idx = np.where(sm == s)[0]
        idx = idx[np.argsort(f["t_start"][idx], kind="stable")]
        for a, b in zip(idx[:-1], idx[1:]):
            rows.setdefault(OP_NAMES[tasks[b, 0]], []).append(
                (f["t_end"][a] - f["t_done"][a], f["t_ready"][b] - f["t_end"][a], f["t_done"][b] - f["t_input"][b]))
    out = {}
    for name, v in rows.items():
        med = np.median(np.asarray(v), axis=0) / 1e3
        out[name] = {"tail_us": float(med[0]), "to_ready_us": float(med[1]), "compute_us": float(med[2]),
                     "n": len(v)}
    return out


def _measure(workload: str, flags: int, steps: int, warmup: int, traced: bool):
    """Run `warmup` + `steps` decode steps of `workload` (batch 1, synthetic
    weights) with mk_config.flags = flags; return (ms per step over the timed
    steps, [per-step overhead dicts] if traced)."""
    import torch
    from . import mk, workloads as wl
    wk = wl.WORKLOADS[workload]
    shape = wk.shape
    start = wk.prefill_len
    max_seq = max(wk.max_seq, start + warmup + steps + 1)
    w = wl.make_weights(shape, seed=1234, device="cuda")
    kc, vc = wl.make_kv(shape, 1, max_seq, device="cuda", prefill_len=start)
    ctx = mk.Context(w, kc, vc, max_seq, 1, flags=flags)
    g = ctx.graph()
    toks = torch.from_numpy(wl.make_prompt(shape.vocab, warmup + steps, seed=42)).cuda()
    pos = torch.arange(start, start + warmup + steps, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(1, dtype=torch.int32, device="cuda")
    per_step = []
    for i in range(warmup):
        ctx.decode_step(toks[i:i + 1], pos[i:i + 1], nxt)
    if ctx.sync() != 0:
        raise RuntimeError("warm-up failed")
    if traced:
        for i in range(warmup, warmup + steps):
            ctx.decode_step(toks[i:i + 1], pos[i:i + 1], nxt)
            if ctx.sync() != 0:
                raise RuntimeError("traced step failed")
            tr = ctx.trace()
            d = task_overheads(tr, g["tasks"], g["queue"], g["qoff"])
            d["critical_path"] = critical_path(tr, g["tasks"])
            d["transitions"] = transitions(tr, g["tasks"])
            per_step.append(d)
        ms = None
    else:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for i in range(warmup, warmup + steps):
            ctx.decode_step(toks[i:i + 1], pos[i:i + 1], nxt)
        e1.record()
        torch.cuda.synchronize()
        if ctx.sync() != 0:
            raise RuntimeError("timed steps failed")
        ms = e0.elapsed_time(e1) / steps
    ctx.close()
    return ms, per_step


def main(argv=None):
    """python -m persistent_decode_megakernel_02_b200.trace [--workload llama1b]
    [--steps N] [--warmup W]: per-task scheduling overhead in both wait modes
    (one JSON line per mode), how each op extends the step (critical_path),
    the per-SM task transitions, and the cost of trace mode (device time per
    step with and without MK_FLAG_TRACE)."""
    import argparse
    import json
    from . import mk
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama1b")
    ap.add_argument("--steps", type=int, default=8)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args(argv)
    for name, mode in (("tagged", 0), ("event", mk.MK_FLAG_EVENT_WAIT)):
        base_ms, _ = _measure(a.workload, mode, 64, a.warmup, False)
        tr_ms, _ = _measure(a.workload, mode | mk.MK_FLAG_TRACE, 64, a.warmup, False)
        _, steps = _measure(a.workload, mode | mk.MK_FLAG_TRACE, a.steps, a.warmup, True)
        ov = np.concatenate([s["overhead"] for s in steps])
        kind = np.concatenate([s["kind"] for s in steps])
        def mean_of(key):
            names = steps[0][key].keys()
            return {n: {f: round(float(np.mean([s[key][n][f] for s in steps])), 3)
                        for f in steps[0][key][n] if f != "n"} for n in names}
        out = {"workload": a.workload, "wait_mode": name, "traced_steps": a.steps,
               "ms_per_step": round(base_ms, 5), "ms_per_step_traced": round(tr_ms, 5),
               "overhead": summarize(ov, kind), "critical_path": mean_of("critical_path"),
               "transitions": mean_of("transitions")}
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
