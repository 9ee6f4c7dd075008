"""Host-side checks of the batched step's task graph (mk_rows_graph.cpp,
built by mk_plan for a context with max_batch > 1 or MK_FLAG_ROWS; no GPU).

The unit of a matrix op there is a page of 128 weight rows x 128 reduction
columns (one tensor-core contraction); each op's pages are cut into one
contiguous range per SM of equal size +-1, attention items are one per
(row, KV head, chunk) for all 16 rows a kernel step can hold, and chunk 0's
item of a (row, KV head) merges the other chunks' partials.  Checked here:
coverage, event thresholds and the dependency chain (a step's embedding
waits for the previous step's LM head), queue order, and runs of the queues
in random interleavings with the data waits the kernel makes.
"""
import numpy as np
import pytest

from persistent_decode_megakernel_02_b200 import workloads as wl

mk = pytest.importorskip("persistent_decode_megakernel_02_b200.mk")

EMBED, QKV, ATTN, OPROJ, GATEUP, DOWN, LMHEAD = range(7)
ROWS, TILE, SLAB, PAGE_BYTES = 16, 128, 128, 128 * 128 * 2
SMS = 148


def _geometry(shape):
    """(tiles, slabs) of every matrix op: 128-row tiles, 128-column slabs."""
    H, F, V = shape.hidden, shape.ffn, shape.vocab
    QD, KD = shape.n_q_heads * shape.head_dim, shape.n_kv_heads * shape.head_dim
    return {QKV: ((QD + 2 * KD) // TILE, H // SLAB), OPROJ: (H // TILE, QD // SLAB),
            GATEUP: (2 * F // TILE, H // SLAB), DOWN: (H // TILE, F // SLAB),
            LMHEAD: ((V + TILE - 1) // TILE, H // SLAB)}


CASES = [("tiny_b4", wl.TINY, 2112, 4, 0, SMS), ("1b_b16", wl.LLAMA_1B, 2112, 16, 0, SMS),
         ("8b_b16", wl.LLAMA_8B, 2112, 16, 0, SMS),
         ("1b_prefill", wl.LLAMA_1B, 560, 1, mk.MK_FLAG_ROWS, SMS),
         ("tiny_long_5sms", wl.TINY, 9000, 8, 0, 5)]


@pytest.fixture(scope="module", params=CASES, ids=[c[0] for c in CASES])
def planned(request):
    name, shape, S, B, flags, sms = request.param
    cfg = mk.make_config(shape, S, B, flags=flags)
    return shape, S, sms, mk.plan(cfg, sms)


def test_rows_plan_info(planned):
    shape, S, sms, pl = planned
    info = pl["info"]
    assert info.page_bytes == PAGE_BYTES and info.num_pages == 5
    assert info.num_events == 2 + 5 * shape.layers
    # chunks of 4096 positions; items score all q heads of a KV head
    assert info.attn_chunks == (S + 4095) // 4096
    assert info.attn_heads == shape.n_q_heads // shape.n_kv_heads


def test_every_page_and_item_covered_once(planned):
    shape, S, sms, pl = planned
    tasks, nbytes = pl["tasks"], pl["bytes"]
    geo = _geometry(shape)
    NC = pl["info"].attn_chunks
    for layer in range(shape.layers + 1):
        for kind in (EMBED, QKV, ATTN, OPROJ, GATEUP, DOWN, LMHEAD):
            sel = tasks[(tasks[:, 0] == kind) & (tasks[:, 1] == layer)]
            expected_here = (layer == shape.layers) if kind == LMHEAD else \
                (layer == 0) if kind == EMBED else (layer < shape.layers)
            if not expected_here:
                assert len(sel) == 0, (kind, layer)
                continue
            if kind == EMBED:
                n = shape.hidden // TILE
            elif kind == ATTN:
                n = ROWS * shape.n_kv_heads * NC
            else:
                n = geo[kind][0] * geo[kind][1]
            cover = np.zeros(n, np.int32)
            for t in sel:
                cover[t[4]:t[5]] += 1
            assert np.all(cover == 1), (kind, layer)
            assert sorted(sel[:, 7].tolist()) == list(range(len(sel)))
            if kind in (EMBED, ATTN):
                assert np.all(sel[:, 5] - sel[:, 4] == 1)
                continue
            # a matrix op: min(pages, SMs) tasks on distinct SMs, page ranges
            # consecutive in slot order and of equal size +-1
            T = min(n, sms)
            assert len(sel) == T and len(set(sel[:, 6].tolist())) == T
            by_slot = sel[np.argsort(sel[:, 7])]
            assert by_slot[0, 4] == 0 and by_slot[-1, 5] == n
            assert np.array_equal(by_slot[1:, 4], by_slot[:-1, 5])
            sizes = by_slot[:, 5] - by_slot[:, 4]
            assert sizes.max() - sizes.min() <= 1 and sizes.min() == n // T
            ids = np.where((tasks[:, 0] == kind) & (tasks[:, 1] == layer))[0]
            assert np.array_equal(nbytes[ids], (tasks[ids, 5] - tasks[ids, 4]).astype(np.int64) * PAGE_BYTES)


def test_thresholds_and_dependency_chain(planned):
    shape, S, sms, pl = planned
    tasks, thr = pl["tasks"], pl["thresholds"]
    E = len(thr)
    e_lm = E - 1
    assert np.array_equal(np.bincount(tasks[:, 3], minlength=E), thr.astype(np.int64))
    for e in range(E):
        sel = tasks[tasks[:, 3] == e]
        assert len(set(map(tuple, sel[:, :2].tolist()))) == 1
    emb = tasks[tasks[:, 0] == EMBED]
    assert np.all(emb[:, 3] == 0) and np.all(emb[:, 2] == e_lm)
    rest = tasks[tasks[:, 0] != EMBED]
    assert np.all(rest[:, 2] == rest[:, 3] - 1)
    # event order = op order: embed, then QKV..DOWN per layer, then the LM head
    first = {int(t[3]): (int(t[0]), int(t[1])) for t in tasks}
    assert first[0] == (EMBED, 0) and first[e_lm] == (LMHEAD, shape.layers)
    for layer in range(shape.layers):
        for k, kind in enumerate((QKV, ATTN, OPROJ, GATEUP, DOWN)):
            assert first[1 + 5 * layer + k] == (kind, layer)


def test_queues_partition_tasks_in_op_order(planned):
    shape, S, sms, pl = planned
    tasks, queue, qoff = pl["tasks"], pl["queue"], pl["qoff"]
    assert qoff[0] == 0 and qoff[-1] == len(tasks)
    assert sorted(queue.tolist()) == list(range(len(tasks)))
    assert pl["info"].max_queue == int(np.diff(qoff).max())
    for sm in range(sms):
        q = queue[qoff[sm]:qoff[sm + 1]]
        assert np.all(tasks[q, 6] == sm)
        assert np.all(np.diff(tasks[q, 3]) >= 0)
        assert np.all(np.diff(q) > 0)


def test_merging_item_comes_after_its_chunks_on_every_queue(planned):
    shape, S, sms, pl = planned
    tasks, queue, qoff = pl["tasks"], pl["queue"], pl["qoff"]
    NC = pl["info"].attn_chunks
    for sm in range(sms):
        q = list(queue[qoff[sm]:qoff[sm + 1]])
        for k, i in enumerate(q):
            t = tasks[i]
            if t[0] == ATTN and t[4] % NC == 0:
                later = tasks[q[k + 1:]]
                assert not np.any((later[:, 0] == ATTN) & (later[:, 1] == t[1]) &
                                  (later[:, 4] // NC == t[4] // NC))


def _run(tasks, queue, qoff, thr, sms, NC, steps, rng):
    """The queues in random interleavings.  A task starts once its dependency
    event has reached threshold x epoch (the embedding: the previous epoch's
    LM head), and a merging attention item also waits for the other chunks of
    its (row, KV head).  Returns the event counts."""
    E = len(thr)
    e_lm = E - 1
    ev = np.zeros(E, np.int64)
    attn = tasks[:, 0] == ATTN
    for ep in range(1, steps + 1):
        pos = [int(qoff[s]) for s in range(sms)]
        done = np.zeros(len(tasks), bool)

        def ready(i):
            t = tasks[i]
            need = thr[t[2]] * (ep - 1 if t[2] == e_lm and t[0] == EMBED else ep)
            if ev[t[2]] < need:
                return False
            if t[0] == ATTN and t[4] % NC == 0:
                mates = attn & (tasks[:, 1] == t[1]) & (tasks[:, 4] // NC == t[4] // NC)
                mates[i] = False
                return bool(done[mates].all())
            return True

        while any(pos[s] < qoff[s + 1] for s in range(sms)):
            progressed = False
            for s in rng.permutation(sms):
                if pos[s] < qoff[s + 1] and ready(queue[pos[s]]):
                    i = queue[pos[s]]
                    done[i] = True
                    ev[tasks[i, 3]] += 1
                    pos[s] += 1
                    progressed = True
            assert progressed, "schedule deadlocked"
    return ev


def test_schedule_runs_to_completion_with_exact_event_counts(planned):
    shape, S, sms, pl = planned
    if shape.layers > 16:
        pytest.skip("covered by the smaller shapes")
    rng = np.random.default_rng(3)
    ev = _run(pl["tasks"], pl["queue"], pl["qoff"], pl["thresholds"], sms, pl["info"].attn_chunks, 2, rng)
    assert np.array_equal(ev, 2 * pl["thresholds"].astype(np.int64))


@pytest.mark.parametrize("bad", [
    dict(n_q_heads=16, n_kv_heads=2),                  # group of 8 q heads
    dict(hidden=320, ffn=768),                         # hidden not a multiple of 128
    dict(ffn=800),                                     # ffn not a multiple of 128
    dict(flags=mk.MK_FLAG_EVENT_WAIT),                 # always gated on counters already
    dict(max_batch=17),
])
def test_rows_plan_rejects_unsupported_shapes(bad):
    base = dict(layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=768,
                vocab=4096, tied=True, rope_theta=1e4)
    run = {k: bad[k] for k in ("flags", "max_batch") if k in bad}
    base.update({k: v for k, v in bad.items() if k not in run})
    shape = wl.ModelShape("bad", **base)
    cfg = mk.make_config(shape, 64, run.get("max_batch", 4), flags=run.get("flags", 0))
    with pytest.raises(mk.MkError) as ei:
        mk.plan(cfg, SMS)
    assert ei.value.status == mk.MK_ERR_INVALID


def test_explicit_chunk_count():
    pl = mk.plan(mk.make_config(wl.TINY, 2112, 4, attn_chunks=3), SMS)
    assert pl["info"].attn_chunks == 3
    tasks = pl["tasks"]
    items = tasks[(tasks[:, 0] == ATTN) & (tasks[:, 1] == 0)]
    assert len(items) == ROWS * wl.TINY.n_kv_heads * 3
