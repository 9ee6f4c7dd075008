"""Host-side checks of the C-ABI library and its task-graph builder (no GPU).

The library is loaded and every function include/mk.h declares must be
exported; mk_plan builds the static task graph on the host, which is checked
for coverage, event thresholds, dependency order, load balance, and by a
simulator that runs the per-SM queues in random interleavings with event
counters the way the persistent kernel does.
"""
import ctypes

import numpy as np
import pytest

from persistent_decode_megakernel_02_b200 import workloads as wl

mk = pytest.importorskip("persistent_decode_megakernel_02_b200.mk")

QKV, ATTN, OPROJ, GATEUP, DOWN, LMHEAD = range(6)
SMS = 148


def test_library_exports_every_declared_function():
    names = mk.header_functions()
    assert "mk_create" in names and "mk_decode_step" in names and "mk_destroy" in names
    lib = ctypes.CDLL(mk.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in mk.h but not exported"


def test_status_strings():
    assert mk.status_string(0) == "ok"
    for s in range(1, 6):
        assert mk.status_string(s) != "unknown status"
    assert mk.status_string(99) == "unknown status"


def test_device_admission():
    # mk_create and the no-allocation entry point run this check on the
    # current device: B200 (compute capability 10.0, cooperative launches,
    # 227 KB = 232448 bytes of opt-in shared memory per block) is accepted;
    # the library's arch-specific sm_100a code runs on no other device
    for batched in (False, True):
        assert mk.device_supported(10, 0, True, 232448, batched) == 0
        for major, minor in ((10, 1), (10, 3), (11, 0), (12, 0), (12, 1), (9, 0), (8, 0)):
            assert mk.device_supported(major, minor, True, 232448, batched) == mk.MK_ERR_INVALID
        assert mk.device_supported(10, 0, False, 232448, batched) == mk.MK_ERR_INVALID
        assert mk.device_supported(10, 0, True, 200 * 1024, batched) == mk.MK_ERR_INVALID


def _tiles(shape):
    d, H, F, V = shape.head_dim, shape.hidden, shape.ffn, shape.vocab
    # q/k/v tiles 8 rows, gate/up tiles 8 gate + 8 up rows, the others 8 rows
    return {QKV: (shape.n_q_heads + 2 * shape.n_kv_heads) * d // 8,
            OPROJ: H // 8, GATEUP: F // 8, DOWN: H // 8, LMHEAD: (V + 7) // 8}


CASES = [("tiny", wl.TINY, 64), ("1b", wl.LLAMA_1B, 560), ("8b", wl.LLAMA_8B, 560),
         ("longctx", wl.LLAMA_1B, 16640)]


@pytest.fixture(scope="module", params=CASES, ids=[c[0] for c in CASES])
def planned(request):
    name, shape, S = request.param
    cfg = mk.make_config(shape, S, 1)
    return shape, cfg, mk.plan(cfg, SMS)


def test_every_row_and_item_covered_once(planned):
    shape, cfg, pl = planned
    tasks = pl["tasks"]
    tiles = _tiles(shape)
    nc = pl["info"].attn_chunks
    for layer in range(shape.layers + 1):
        for kind in (QKV, ATTN, OPROJ, GATEUP, DOWN, LMHEAD):
            sel = tasks[(tasks[:, 0] == kind) & (tasks[:, 1] == layer)]
            if (kind == LMHEAD) != (layer == shape.layers):
                assert len(sel) == 0
                continue
            ha = pl["info"].attn_heads
            n = shape.n_q_heads // ha * nc if kind == ATTN else tiles[kind]
            cover = np.zeros(n, np.int32)
            for t in sel:
                cover[t[4]:t[5]] += 1
            assert np.all(cover == 1), (kind, layer)
            # slots number the op's tasks 0..T-1
            assert sorted(sel[:, 7].tolist()) == list(range(len(sel)))


def test_thresholds_equal_triggering_tasks_and_deps_form_a_chain(planned):
    shape, cfg, pl = planned
    tasks, thr = pl["tasks"], pl["thresholds"]
    E = len(thr)
    assert E == 5 * shape.layers + 1
    counts = np.bincount(tasks[:, 3], minlength=E)
    assert np.array_equal(counts, thr.astype(np.int64))
    for t in tasks:
        # each op waits on the event of the op right before it (none for the first)
        assert t[2] == t[3] - 1
    # one op per event: all tasks triggering an event share kind and layer
    for e in range(E):
        sel = tasks[tasks[:, 3] == e]
        assert len(set(map(tuple, sel[:, :2].tolist()))) == 1


def test_queues_partition_tasks_in_op_order(planned):
    shape, cfg, pl = planned
    tasks, queue, qoff = pl["tasks"], pl["queue"], pl["qoff"]
    assert qoff[0] == 0 and qoff[-1] == len(tasks)
    assert sorted(queue.tolist()) == list(range(len(tasks)))
    for sm in range(SMS):
        q = queue[qoff[sm]:qoff[sm + 1]]
        assert np.all(tasks[q, 6] == sm)
        assert np.all(np.diff(tasks[q, 3]) >= 0)     # events (= op order) never go back
        assert np.all(np.diff(q) > 0)


def test_weight_bytes_balanced_and_complete(planned):
    shape, cfg, pl = planned
    tasks, nbytes = pl["tasks"], pl["bytes"]
    gemv = tasks[:, 0] != ATTN
    H, F, V = shape.hidden, shape.ffn, shape.vocab
    QD, KD = shape.n_q_heads * shape.head_dim, shape.n_kv_heads * shape.head_dim
    matrices = 2 * (shape.layers * ((QD + 2 * KD) * H + H * QD + 3 * F * H) + V * H)
    assert int(nbytes[gemv].sum()) == matrices
    if shape.layers >= 16:
        per_sm = np.bincount(tasks[:, 6], weights=nbytes.astype(np.float64), minlength=SMS)
        assert per_sm.max() / per_sm.mean() < 1.02


def _simulate(tasks, queue, qoff, thr, steps, rng):
    """Run the per-SM queues in random interleavings; returns event counts."""
    ev = np.zeros(len(thr), np.int64)
    for ep in range(1, steps + 1):
        pos = [int(qoff[s]) for s in range(SMS)]
        live = [s for s in range(SMS) if pos[s] < qoff[s + 1]]
        while live:
            progressed = False
            for s in rng.permutation(live):
                t = tasks[queue[pos[s]]]
                if t[2] < 0 or ev[t[2]] >= thr[t[2]] * ep:
                    ev[t[3]] += 1
                    pos[s] += 1
                    progressed = True
            live = [s for s in live if pos[s] < qoff[s + 1]]
            assert progressed, "schedule deadlocked"
    return ev


def test_schedule_runs_to_completion_with_exact_event_counts(planned):
    shape, cfg, pl = planned
    if shape.layers > 16:
        pytest.skip("covered by the smaller shapes")
    rng = np.random.default_rng(0)
    ev = _simulate(pl["tasks"], pl["queue"], pl["qoff"], pl["thresholds"], 2, rng)
    assert np.array_equal(ev, 2 * pl["thresholds"].astype(np.int64))


@pytest.mark.parametrize("bad", [
    dict(head_dim=96), dict(n_q_heads=12, n_kv_heads=4), dict(hidden=2044),
    dict(ffn=20000), dict(max_batch=99), dict(vocab=0), dict(max_seq=0), dict(hidden=8192),
])
def test_plan_rejects_unsupported_shapes(bad):
    base = dict(layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=768,
                vocab=4096, tied=True, rope_theta=1e4)
    run = {k: bad[k] for k in ("max_seq", "max_batch") if k in bad}
    base.update({k: v for k, v in bad.items() if k not in run})
    shape = wl.ModelShape("bad", **base)
    cfg = mk.make_config(shape, bad.get("max_seq", 64), bad.get("max_batch", 1))
    with pytest.raises(mk.MkError) as ei:
        mk.plan(cfg, SMS)
    assert ei.value.status == mk.MK_ERR_INVALID


def test_default_attention_chunks():
    # one task per (sequence, q head, chunk): as many chunks as fill the SMs
    # (148 // 32 q heads = 4), but no more than a full cache needs at 1024
    # positions per chunk
    def info(shape, S, **kw):
        return mk.plan(mk.make_config(shape, S, **kw), SMS)["info"]
    assert (info(wl.LLAMA_1B, 560).attn_chunks, info(wl.LLAMA_1B, 560).attn_heads) == (1, 1)
    assert (info(wl.TINY, 64).attn_chunks, info(wl.TINY, 64).attn_heads) == (1, 1)
    assert (info(wl.TINY, 4096).attn_chunks, info(wl.TINY, 4096).attn_heads) == (4, 1)
    assert info(wl.TINY, 64, attn_chunks=7).attn_chunks == 7
    assert info(wl.LLAMA_1B, 4096).attn_heads == 1           # 4 chunks per q head reach 1024 positions
    # a 16k cache needs 17 chunks, the SMs give 4 per q head: one task per
    # (sequence, KV head, chunk) instead, its 4 q heads together, and
    # 148 // 8 = 18 chunks, capped at the 17 a full cache needs
    i = info(wl.LLAMA_1B, 16640)
    assert (i.attn_heads, i.attn_chunks) == (4, 17)
    i = info(wl.LLAMA_1B, 16640, flags=mk.MK_FLAG_ATTN_Q_ITEMS)
    assert (i.attn_heads, i.attn_chunks) == (1, 4)
    i = info(wl.LLAMA_1B, 560, flags=mk.MK_FLAG_ATTN_KV_ITEMS)
    assert (i.attn_heads, i.attn_chunks) == (4, 1)
    # 8B shape: G = 4 at head_dim 128 (4 x 128 <= 512); 16k: 17 chunks fit
    # the stage only up to 8192 // (4 * 130) = 15
    i = info(wl.LLAMA_8B, 16640)
    assert (i.attn_heads, i.attn_chunks) == (4, 15)
    # a group of 8 q heads of 128 dims is split in halves of 4
    g8 = wl.ModelShape("g8", 2, 1024, 16, 2, 128, 2048, 4096, True, 1e4)
    assert info(g8, 64, flags=mk.MK_FLAG_ATTN_KV_ITEMS).attn_heads == 4
    g8s = wl.ModelShape("g8s", 2, 512, 8, 1, 64, 2048, 4096, True, 1e4)
    assert info(g8s, 64, flags=mk.MK_FLAG_ATTN_KV_ITEMS).attn_heads == 8
    # no grouping without shared KV heads
    mha = wl.ModelShape("mha", 2, 256, 4, 4, 64, 768, 4096, True, 1e4)
    assert info(mha, 16640, flags=mk.MK_FLAG_ATTN_KV_ITEMS).attn_heads == 1
    with pytest.raises(mk.MkError):
        info(wl.TINY, 64, flags=mk.MK_FLAG_ATTN_KV_ITEMS | mk.MK_FLAG_ATTN_Q_ITEMS)


@pytest.mark.parametrize("flags", [0, mk.MK_FLAG_ATTN_KV_ITEMS])
@pytest.mark.parametrize("sms,chunks", [(5, 7), (16, 8), (SMS, 0)])
def test_attention_merger_runs_after_its_chunks(sms, chunks, flags):
    """With one item per q head, chunk 0's task of every head merges the
    partials and waits for the other chunks' tagged outputs: on every queue
    it must come after each other chunk of its head, and the whole graph must
    run to completion when tasks wait on exactly their inputs.  KV-head items
    merge the same way, chunk 0's item of every (sequence, KV head)."""
    shape = wl.TINY
    cfg = mk.make_config(shape, 256, 1, attn_chunks=chunks, flags=flags)
    pl = mk.plan(cfg, sms)
    tasks, queue, qoff = pl["tasks"], pl["queue"], pl["qoff"]
    NC = pl["info"].attn_chunks
    for s in range(sms):
        q = list(queue[qoff[s]:qoff[s + 1]])
        for k, i in enumerate(q):
            t = tasks[i]
            if t[0] == ATTN and t[4] % NC == 0:
                later = tasks[q[k + 1:]]
                assert not np.any((later[:, 0] == ATTN) & (later[:, 1] == t[1]) &
                                  (later[:, 4] // NC == t[4] // NC))
    # run the queues with data dependencies: a task needs every task of the
    # op before it, except that attention chunks need only the QKV op and
    # chunk 0 additionally needs the other chunks of its head
    rng = np.random.default_rng(1)
    done = np.zeros(len(tasks), bool)
    by_event = {e: np.where(tasks[:, 3] == e)[0] for e in np.unique(tasks[:, 3])}
    pos = [int(qoff[s]) for s in range(sms)]

    def runnable(i):
        t = tasks[i]
        if t[2] >= 0 and not done[by_event[t[2]]].all():
            return False
        if t[0] == ATTN and t[4] % NC == 0:
            mates = by_event[t[3]]
            mates = mates[(tasks[mates, 4] // NC == t[4] // NC) & (mates != i)]
            return bool(done[mates].all())
        return True

    while any(pos[s] < qoff[s + 1] for s in range(sms)):
        progressed = False
        for s in rng.permutation(sms):
            if pos[s] < qoff[s + 1] and runnable(queue[pos[s]]):
                done[queue[pos[s]]] = True
                pos[s] += 1
                progressed = True
        assert progressed, "tasks wait on each other in a cycle"
    assert done.all()


def test_plan_refuses_partials_that_overflow_the_merge_stage():
    # chunk 0's task stages every chunk's (o[d], m, l) of its q head in 8192
    # floats of shared memory: 124 chunks x 66 fit, 125 do not
    base = dict(layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=768,
                vocab=4096, tied=True, rope_theta=1e4)
    shape = wl.ModelShape("chunks", **base)
    assert mk.plan(mk.make_config(shape, 64, 1, attn_chunks=124), SMS)["info"].attn_chunks == 124
    with pytest.raises(mk.MkError) as ei:
        mk.plan(mk.make_config(shape, 64, 1, attn_chunks=125), SMS)
    assert ei.value.status == mk.MK_ERR_INVALID
    # an item of 2 q heads (MK_FLAG_ATTN_KV_ITEMS, G = 2) stages both heads'
    # partials: 62 chunks x 2 x 66 fit, 63 do not
    kv = mk.MK_FLAG_ATTN_KV_ITEMS
    assert mk.plan(mk.make_config(shape, 64, 1, attn_chunks=62, flags=kv), SMS)["info"].attn_chunks == 62
    with pytest.raises(mk.MkError):
        mk.plan(mk.make_config(shape, 64, 1, attn_chunks=63, flags=kv), SMS)
    # chosen by default for a long cache, KV-head items give way to q-head
    # items when the given chunk count would not fit with them
    i = mk.plan(mk.make_config(shape, 126008, 1, attn_chunks=124), SMS)["info"]
    assert (i.attn_heads, i.attn_chunks) == (1, 124)
    i = mk.plan(mk.make_config(shape, 126008, 1, attn_chunks=62), SMS)["info"]
    assert (i.attn_heads, i.attn_chunks) == (2, 62)
