"""GPU parity: the persistent kernel, called through the C ABI, against the
fp64 CPU oracle on the same seeded bits, teacher-forced.

Bar (per step): max|dlogit| <= 1e-2 * max|logit_oracle| + 1e-3; the GPU's
next token is the oracle's argmax or within that tolerance of it; the
residual stream after the last layer within 5e-3 relative L2; event
counters equal threshold * steps exactly.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from persistent_decode_megakernel_02_b200 import workloads as wl
from harness import Pair, logit_tol, rel_l2, token_ok

pytestmark = pytest.mark.gpu


def _check_step(pair, step, g_tok, g_log, ref):
    d = np.abs(g_log - ref["logits"]).max()
    assert d <= logit_tol(ref["logits"]), f"step {step}: max|dlogit| {d:.3e}"
    assert token_ok(g_tok, ref["logits"]), f"step {step}: token {g_tok} vs {ref['next']}"


def _check_hidden(pair, ref):
    h = pair.ctx.read_buffer(pair.mk.MK_BUF_HIDDEN, pair.shape.hidden).astype(np.float64)
    assert rel_l2(h, ref["hidden"]) <= 5e-3


def _check_events(pair, steps):
    counts, thr = pair.ctx.event_counts()
    assert np.array_equal(counts.astype(np.uint64), (thr.astype(np.uint64) * steps) % (1 << 32))


# 0: tasks wait on their tagged inputs; 4 (MK_FLAG_EVENT_WAIT): a scheduler
# warp gates every task on its dependency's event counter first
WAIT_MODES = [0, 4]


@pytest.mark.parametrize("flags", WAIT_MODES)
def test_tiny_teacher_forced_prompt_and_decode(flags):
    shape = wl.TINY
    pair = Pair(shape, max_seq=64, flags=flags)
    prompt = wl.make_prompt(shape.vocab, 16, seed=42)
    n = 0
    for step, pos, g_tok, g_log, ref in pair.teacher_forced(prompt, 32):
        _check_step(pair, step, g_tok, g_log, ref)
        n += 1
    assert n == 48
    _check_hidden(pair, ref)
    _check_events(pair, n)
    # KV entries written by the kernel match the oracle's (bf16 values)
    for l in range(shape.layers):
        kg = pair.k_gpu[l][0, :, :n].float().cpu().numpy()
        kr = torch.from_numpy(pair.k_ref[l][:, :n].view(np.int16)).view(torch.bfloat16).float().numpy()
        assert np.abs(kg - kr).max() <= 2e-2 * np.abs(kr).max()


@pytest.mark.parametrize("flags", WAIT_MODES)
def test_tiny_random_gains_untied_head_and_intermediates(flags):
    shape = wl.ModelShape("tiny-untied", 2, 256, 4, 2, 64, 768, 4096, False, 1e4)
    pair = Pair(shape, max_seq=40, gains="random", std=0.05, flags=flags)
    toks = wl.make_prompt(shape.vocab, 20, seed=9)
    for pos, t in enumerate(toks):
        g_tok, g_log = pair.gpu_step(int(t), pos)
        ref = pair.ref_step(int(t), pos, intermediates=True)
        _check_step(pair, pos, g_tok, g_log, ref)
    mk = pair.mk
    for buf, key in ((mk.MK_BUF_Q, "q"), (mk.MK_BUF_ATTN, "attn"), (mk.MK_BUF_ACT, "act")):
        got = pair.ctx.read_buffer(buf, ref[key].size).astype(np.float64)
        if key == "q":   # the kernel keeps q before RoPE; rotate it per head like the oracle
            d = shape.head_dim
            got = np.concatenate([orc.rope(got[h * d:(h + 1) * d], pos, shape.rope_theta)
                                  for h in range(shape.n_q_heads)])
        assert rel_l2(got, ref[key]) <= 5e-3, key
    _check_hidden(pair, ref)


# Split-K attention with many ACTIVE chunks: a step uses ceil(C / 1024)
# chunks (at most attn_chunks), so each case prefills a random cache long
# enough that every configured chunk holds positions and chunk 0's task merges
# all of them.  124 chunks is the most the merge stage holds at head_dim 64
# (124 * 66 <= 8192 floats), 63 at head_dim 128.
TINY_D128 = wl.ModelShape("tiny-d128", 2, 256, 2, 1, 128, 768, 4096, True, 1e4)


@pytest.mark.parametrize("head_dim,chunks,prefix", [(64, 13, 13000), (64, 40, 40000),
                                                    (64, 124, 126000), (128, 63, 64000)])
def test_many_active_attention_chunks_merged(head_dim, chunks, prefix):
    shape = wl.TINY if head_dim == 64 else TINY_D128
    S = prefix + 8
    pair = Pair(shape, max_seq=S, prefill_len=prefix, attn_chunks=chunks)
    assert pair.ctx.info().attn_chunks == chunks
    assert -(-(prefix + 1) // 1024) >= chunks      # every chunk is active
    toks = wl.make_prompt(shape.vocab, 3, seed=11)
    for i, t in enumerate(toks):
        pos = prefix + i
        g_tok, g_log = pair.gpu_step(int(t), pos)
        ref = pair.ref_step(int(t), pos, intermediates=True)
        _check_step(pair, pos, g_tok, g_log, ref)
        got = pair.ctx.read_buffer(pair.mk.MK_BUF_ATTN, ref["attn"].size).astype(np.float64)
        assert rel_l2(got, ref["attn"]) <= 5e-3
    _check_hidden(pair, ref)


# Attention items of one KV head's q heads together (MK_FLAG_ATTN_KV_ITEMS):
# many merged chunks (chunk 0's item stages every head's partials: 62
# chunks x 2 heads x 66 floats at head_dim 64, 31 x 2 x 130 at 128).
KV = 32


@pytest.mark.parametrize("head_dim,chunks,prefix", [(64, 13, 13000), (64, 62, 63000), (128, 31, 32000)])
def test_kv_head_items_many_chunks_merged(head_dim, chunks, prefix):
    shape = wl.TINY if head_dim == 64 else TINY_D128
    S = prefix + 8
    pair = Pair(shape, max_seq=S, prefill_len=prefix, attn_chunks=chunks, flags=KV)
    assert (pair.ctx.info().attn_chunks, pair.ctx.info().attn_heads) == (chunks, 2)
    toks = wl.make_prompt(shape.vocab, 2, seed=17)
    for i, t in enumerate(toks):
        pos = prefix + i
        g_tok, g_log = pair.gpu_step(int(t), pos)
        ref = pair.ref_step(int(t), pos, intermediates=True)
        _check_step(pair, pos, g_tok, g_log, ref)
        got = pair.ctx.read_buffer(pair.mk.MK_BUF_ATTN, ref["attn"].size).astype(np.float64)
        assert rel_l2(got, ref["attn"]) <= 5e-3
    _check_hidden(pair, ref)


# Group sizes and head dims of the KV-head items: G = 4 and 8 at head_dim
# 64 (4 and 8 heads per item), G = 4 at 128 (4 heads), and G = 8 at 128,
# split into two items of 4 heads per KV head (only the first appends the
# new key).  A prefix of 2600 positions (3 merged chunks), then decode.
G4_D64 = wl.ModelShape("g4-d64", 2, 256, 8, 2, 64, 768, 4096, True, 1e4)
G8_D64 = wl.ModelShape("g8-d64", 2, 512, 8, 1, 64, 768, 4096, False, 1e4)
G4_D128 = wl.ModelShape("g4-d128", 2, 512, 4, 1, 128, 768, 4096, True, 1e4)
G8_D128 = wl.ModelShape("g8-d128", 2, 1024, 8, 1, 128, 768, 4096, True, 1e4)


@pytest.mark.parametrize("shape,heads", [(G4_D64, 4), (G8_D64, 8), (G4_D128, 4), (G8_D128, 4)],
                         ids=["g4-d64", "g8-d64", "g4-d128", "g8-d128"])
@pytest.mark.parametrize("flags", [KV, KV | 4])
def test_kv_head_items_group_sizes(shape, heads, flags):
    S = 2624
    pair = Pair(shape, max_seq=S, prefill_len=2600, attn_chunks=3, flags=flags)
    assert pair.ctx.info().attn_heads == heads
    toks = wl.make_prompt(shape.vocab, 3, seed=19)
    for i, t in enumerate(toks):
        pos = 2600 + i
        g_tok, g_log = pair.gpu_step(int(t), pos)
        ref = pair.ref_step(int(t), pos, intermediates=True)
        _check_step(pair, pos, g_tok, g_log, ref)
        got = pair.ctx.read_buffer(pair.mk.MK_BUF_ATTN, ref["attn"].size).astype(np.float64)
        assert rel_l2(got, ref["attn"]) <= 5e-3
    _check_hidden(pair, ref)
    # short contexts (one chunk, positions 0..): the same items, no merge
    short = Pair(shape, max_seq=48, flags=flags)
    for step, pos, g_tok, g_log, ref in short.teacher_forced(wl.make_prompt(shape.vocab, 20, seed=3), 20):
        _check_step(short, step, g_tok, g_log, ref)
    _check_events(short, 40)


@pytest.mark.parametrize("chunks", [1, 3, 64])
def test_short_contexts_with_more_chunks_than_positions(chunks):
    # contexts of at most 40 positions use one active chunk whatever the
    # configured count; the other chunks' items find no positions and must
    # write nothing (and their empty partials must not reach a merge)
    shape = wl.TINY
    pair = Pair(shape, max_seq=96, attn_chunks=chunks)
    toks = wl.make_prompt(shape.vocab, 40, seed=11)
    for pos, t in enumerate(toks):
        g_tok, g_log = pair.gpu_step(int(t), pos)
        ref = pair.ref_step(int(t), pos)
        _check_step(pair, pos, g_tok, g_log, ref)


@pytest.mark.parametrize("chunks", [3, 5])
def test_long_prefix_split_into_chunks_and_merged(chunks):
    # 2600+ positions: ceil(C / 1024) = 3 active chunks per q head, merged by
    # chunk 0's task (with 5 chunks, two are empty)
    shape = wl.TINY
    S = 2624
    pair = Pair(shape, max_seq=S, prefill_len=2600, attn_chunks=chunks)
    toks = wl.make_prompt(shape.vocab, 4, seed=13)
    for i, t in enumerate(toks):
        pos = 2600 + i
        g_tok, g_log = pair.gpu_step(int(t), pos)
        ref = pair.ref_step(int(t), pos, intermediates=True)
        _check_step(pair, pos, g_tok, g_log, ref)
    got = pair.ctx.read_buffer(pair.mk.MK_BUF_ATTN, ref["attn"].size).astype(np.float64)
    assert rel_l2(got, ref["attn"]) <= 5e-3


def test_edge_positions_tokens_and_null_logits():
    shape = wl.TINY
    S = 24
    pair = Pair(shape, max_seq=S, prefill_len=S)     # full random prefix
    # last legal position attends to every slot; extreme token ids
    for pos, t in ((S - 1, shape.vocab - 1), (0, 0), (5, 1)):
        g_tok, g_log = pair.gpu_step(t, pos)
        ref = pair.ref_step(t, pos)
        _check_step(pair, pos, g_tok, g_log, ref)
    g_tok, _ = pair.gpu_step(7, 6, want_logits=False)
    ref = pair.ref_step(7, 6)
    assert token_ok(g_tok, ref["logits"])


def test_invalid_inputs_reported_then_reset():
    shape = wl.TINY
    pair = Pair(shape, max_seq=16)
    mk = pair.mk
    # host-side checks: synchronous MK_ERR_INVALID, nothing launched
    assert pair.ctx.decode_step_status(pair.tok, pair.pos, pair.nxt, batch=0) == mk.MK_ERR_INVALID
    assert pair.ctx.decode_step_status(pair.tok, pair.pos, pair.nxt, batch=2) == mk.MK_ERR_INVALID
    # device-side checks: bad position, then bad token
    for tok, pos in ((1, 16), (shape.vocab, 0), (-1, 0)):
        pair.tok.fill_(tok)
        pair.pos.fill_(pos)
        pair.ctx.decode_step(pair.tok, pair.pos, pair.nxt, pair.logits)
        assert pair.ctx.sync() == mk.MK_ERR_INVALID
        assert pair.ctx.decode_step_status(pair.tok, pair.pos, pair.nxt) == mk.MK_ERR_STATE
        pair.ctx.reset()
    g_tok, g_log = pair.gpu_step(3, 0)
    ref = pair.ref_step(3, 0)
    _check_step(pair, 0, g_tok, g_log, ref)
    _check_events(pair, 1)


def test_event_that_never_fires_times_out_and_context_recovers():
    shape = wl.TINY
    # counter-gated scheduling: the scheduler's wait on event 3 never ends
    pair = Pair(shape, max_seq=16, timeout_ns=50_000_000, flags=4)   # 50 ms bound per wait
    mk = pair.mk
    g_tok, _ = pair.gpu_step(1, 0)
    _, thr = pair.ctx.event_counts()
    pair.ctx.debug_set_threshold(3, int(thr[3]) + 1)          # one trigger short, forever
    pair.tok.fill_(2)
    pair.pos.fill_(1)
    pair.ctx.decode_step(pair.tok, pair.pos, pair.nxt, pair.logits)
    assert pair.ctx.sync() == mk.MK_ERR_TIMEOUT
    info = pair.ctx.info()
    assert info.err_code == mk.MK_ERR_TIMEOUT
    pair.ctx.reset()
    # the oracle replays both positions; the GPU restarts from position 0
    pair.ref_step(1, 0)
    g_tok, g_log = pair.gpu_step(2, 1)
    ref = pair.ref_step(2, 1)
    _check_step(pair, 1, g_tok, g_log, ref)


def test_withheld_outputs_time_out_and_context_recovers():
    shape = wl.TINY
    # tagged-input waits: the gate/up tasks of layer 0 (event 3) store stale
    # tags, the down projection's poll of its input never succeeds
    pair = Pair(shape, max_seq=16, timeout_ns=50_000_000)
    mk = pair.mk
    pair.gpu_step(1, 0)
    pair.ctx.debug_withhold_event(3)
    pair.tok.fill_(2)
    pair.pos.fill_(1)
    pair.ctx.decode_step(pair.tok, pair.pos, pair.nxt, pair.logits)
    assert pair.ctx.sync() == mk.MK_ERR_TIMEOUT
    assert pair.ctx.info().err_code == mk.MK_ERR_TIMEOUT
    pair.ctx.reset()
    pair.ref_step(1, 0)
    g_tok, g_log = pair.gpu_step(2, 1)
    ref = pair.ref_step(2, 1)
    _check_step(pair, 1, g_tok, g_log, ref)
    g_tok, g_log = pair.gpu_step(3, 2)
    ref = pair.ref_step(3, 2)
    _check_step(pair, 2, g_tok, g_log, ref)


@pytest.mark.parametrize("flags", WAIT_MODES)
def test_trace_records_respect_dependencies(flags):
    shape = wl.TINY
    pair = Pair(shape, max_seq=32, flags=1 | flags)
    for pos, t in enumerate([5, 6, 7]):
        pair.gpu_step(t, pos)
    tr = pair.ctx.trace()
    g = pair.ctx.graph()
    tasks = g["tasks"]
    assert np.all(tr["t_start"] >= tr["t_ready"]) and np.all(tr["t_input"] >= tr["t_start"])
    assert np.all(tr["t_done"] >= tr["t_input"]) and np.all(tr["t_end"] >= tr["t_done"])
    fire = {}
    for e in np.unique(tasks[:, 3]):
        fire[e] = tr["t_end"][tasks[:, 3] == e].max()
    for i, t in enumerate(tasks):
        # an attention task waiting on its inputs needs only its own KV
        # head's q/k/v, not the whole QKV op (the event's other tasks)
        if t[2] >= 0 and (flags or t[0] != 1):
            # a task becomes ready only after every task of its dependency
            # signalled (t_end is stamped just after the signal; allow 5 us)
            assert int(tr["t_ready"][i]) + 5000 >= int(fire[t[2]])


@pytest.mark.slow
def test_llama1b_shape_prompt_of_39_then_decode():
    # the benchmark's workload from its first position: a 39-token prompt
    # teacher-forced, then decode steps at positions 39..43
    shape = wl.LLAMA_1B
    pair = Pair(shape, max_seq=560)
    prompt = wl.make_prompt(shape.vocab, 39, seed=42)
    n = 0
    for step, pos, g_tok, g_log, ref in pair.teacher_forced(prompt, 5):
        _check_step(pair, step, g_tok, g_log, ref)
        n += 1
    assert n == 44 and pos == 43
    _check_hidden(pair, ref)
    _check_events(pair, n)


@pytest.mark.slow
def test_llama1b_shape_at_the_end_of_the_benchmark_range():
    # positions 540..545 (the bench's 512 decode steps end at 550) over a
    # seeded random prefix of 540 positions
    shape = wl.LLAMA_1B
    pair = Pair(shape, max_seq=560, prefill_len=540)
    prompt = wl.make_prompt(shape.vocab, 1, seed=8)
    n = 0
    for step, pos, g_tok, g_log, ref in pair.teacher_forced(prompt, 5, start_pos=540):
        _check_step(pair, pos, g_tok, g_log, ref)
        n += 1
    assert n == 6
    _check_hidden(pair, ref)


@pytest.mark.slow
@pytest.mark.parametrize("flags,heads,chunks", [(0, 4, 17), (64, 1, 4)], ids=["kv-items", "q-items"])
def test_llama1b_long_context_prefilled(flags, heads, chunks):
    # the default at 16k: one item per (KV head, chunk) for its 4 q heads,
    # 17 chunks; MK_FLAG_ATTN_Q_ITEMS: one per (q head, chunk), 4 chunks
    shape = wl.LLAMA_1B
    S = 16640
    pair = Pair(shape, max_seq=S, prefill_len=16384, flags=flags)
    assert (pair.ctx.info().attn_heads, pair.ctx.info().attn_chunks) == (heads, chunks)
    prompt = wl.make_prompt(shape.vocab, 1, seed=5)
    for step, pos, g_tok, g_log, ref in pair.teacher_forced(prompt, 1, start_pos=16384):
        _check_step(pair, step, g_tok, g_log, ref)
    _check_hidden(pair, ref)


@pytest.mark.slow
def test_llama8b_shape_teacher_forced():
    shape = wl.LLAMA_8B
    pair = Pair(shape, max_seq=560)
    prompt = wl.make_prompt(shape.vocab, 1, seed=42)
    for step, pos, g_tok, g_log, ref in pair.teacher_forced(prompt, 1):
        _check_step(pair, step, g_tok, g_log, ref)
    _check_hidden(pair, ref)
