"""GPU parity of the batched step (tcgen05 tensor cores) against the oracle.

A context with max_batch > 1 (or MK_FLAG_ROWS) runs every step on the
batched kernel: up to 16 rows per kernel step, every matrix op a contraction
of the weights with the rows on the tensor cores.

* decode batches of 4, 8 and 16 sequences at staggered positions (start
  positions uniform in [32, 2048], KV prefixes of seeded N(0,1) values, the
  batched workload's recipe): every sequence's logits against the oracle's
  step on that sequence, teacher-forced, at the stated tolerance; and 4
  sequences at 4500..9000 positions, whose attention items are merged;
* a prompt in one launch (mk_prefill, 16 tokens per kernel step, causal
  attention within the prompt): the KV entries it writes and the last
  token's logits against the oracle fed the same prompt token by token;
* a batch of one row and the Llama-3.2-1B shape.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from persistent_decode_megakernel_02_b200 import workloads as wl
from harness import logit_tol, token_ok, rel_l2

pytestmark = pytest.mark.gpu


class Batch:
    """A model on the GPU (batched context) and per-sequence oracle caches
    holding the same bits."""

    def __init__(self, shape, max_batch, max_seq, prefill_len=0, seed=1234, gains="ones", flags=0):
        from persistent_decode_megakernel_02_b200 import mk
        self.mk = mk
        self.shape = shape
        self.B = max_batch
        self.w = wl.make_weights(shape, seed=seed, device="cuda", gains=gains)
        self.k, self.v = wl.make_kv(shape, max_batch, max_seq, device="cuda", prefill_len=prefill_len)
        cfg = dict(layers=shape.layers, hidden=shape.hidden, n_q_heads=shape.n_q_heads,
                   n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, ffn=shape.ffn,
                   vocab=shape.vocab, max_seq=max_seq, rope_theta=shape.rope_theta,
                   rms_eps=shape.rms_eps)
        self.oracle = orc.OracleModel(cfg, self.w.numpy_bits())
        self.kr = [[wl.cache_bits(k[b]).copy() for k in self.k] for b in range(max_batch)]
        self.vr = [[wl.cache_bits(v[b]).copy() for v in self.v] for b in range(max_batch)]
        self.ctx = mk.Context(self.w, self.k, self.v, max_seq, max_batch, flags=flags)

    def gpu_step(self, tokens, positions):
        n = len(tokens)
        tok = torch.tensor(tokens, dtype=torch.int32, device="cuda")
        pos = torch.tensor(positions, dtype=torch.int32, device="cuda")
        nxt = torch.zeros(n, dtype=torch.int32, device="cuda")
        logits = torch.zeros(n, self.shape.vocab, dtype=torch.float32, device="cuda")
        self.ctx.decode_step(tok, pos, nxt, logits)
        st = self.ctx.sync()
        if st != 0:
            raise self.mk.MkError(st, "batched step")
        return nxt.cpu().numpy(), logits.double().cpu().numpy()

    def ref_step(self, b, token, pos):
        return self.oracle.decode_step(self.kr[b], self.vr[b], int(token), int(pos))


def _check(g_log, g_tok, ref, what):
    d = np.abs(g_log - ref["logits"]).max()
    assert d <= logit_tol(ref["logits"]), f"{what}: max|dlogit| {d:.3e} > {logit_tol(ref['logits']):.3e}"
    assert token_ok(int(g_tok), ref["logits"]), what


@pytest.mark.parametrize("B", [4, 8, 16])
def test_batched_decode_staggered_positions(B):
    shape = wl.TINY
    S = 2048 + 8
    starts = wl.make_start_positions(B, seed=B)
    bt = Batch(shape, B, S, prefill_len=2048)
    toks = [int(t) for t in wl.make_prompt(shape.vocab, B, seed=3)]
    for step in range(3):
        pos = [int(starts[b]) + step for b in range(B)]
        g_tok, g_log = bt.gpu_step(toks, pos)
        refs = [bt.ref_step(b, toks[b], pos[b]) for b in range(B)]
        for b in range(B):
            _check(g_log[b], g_tok[b], refs[b], f"step {step} seq {b} pos {pos[b]}")
        toks = [r["next"] for r in refs]          # teacher-forced: the oracle's tokens
    # the KV entries the batched step wrote (the step's positions of every sequence)
    for b in range(B):
        for l in range(shape.layers):
            p0 = int(starts[b])
            kg = bt.k[l][b, :, p0:p0 + 3].float().cpu().numpy()
            kr = torch.from_numpy(bt.kr[b][l][:, p0:p0 + 3].view(np.int16)).view(torch.bfloat16).float().numpy()
            assert np.abs(kg - kr).max() <= 2e-2 * np.abs(kr).max()


def test_batched_decode_long_contexts_merged_chunks():
    # a row's positions split into chunks of at least 4096 (one item each,
    # chunk 0's item merges): start positions in [4500, 9000] give 2 or 3
    # chunks per row, merged in every layer
    shape = wl.TINY
    B = 4
    S = 9000 + 8
    starts = wl.make_start_positions(B, seed=21, lo=4500, hi=9000)
    bt = Batch(shape, B, S, prefill_len=9000)
    assert bt.ctx.info().attn_chunks == 3
    toks = [int(t) for t in wl.make_prompt(shape.vocab, B, seed=8)]
    for step in range(2):
        pos = [int(starts[b]) + step for b in range(B)]
        g_tok, g_log = bt.gpu_step(toks, pos)
        refs = [bt.ref_step(b, toks[b], pos[b]) for b in range(B)]
        for b in range(B):
            _check(g_log[b], g_tok[b], refs[b], f"step {step} seq {b} pos {pos[b]}")
        toks = [r["next"] for r in refs]


def test_batch_smaller_than_the_context_and_random_gains():
    # 5 sequences on a 16-slot context, short contexts (one attention chunk)
    shape = wl.ModelShape("tiny-untied", 2, 256, 4, 2, 64, 768, 4096, False, 1e4)
    bt = Batch(shape, 16, 64, gains="random")
    toks = [11, 22, 33, 44, 55]
    for step in range(4):
        g_tok, g_log = bt.gpu_step(toks, [step] * 5)
        refs = [bt.ref_step(b, toks[b], step) for b in range(5)]
        for b in range(5):
            _check(g_log[b], g_tok[b], refs[b], f"step {step} seq {b}")
        toks = [r["next"] for r in refs]
    h = bt.ctx.read_buffer(bt.mk.MK_BUF_HIDDEN, 5 * shape.hidden).reshape(5, shape.hidden)
    # the oracle's last hidden state of sequence 4
    assert rel_l2(h[4].astype(np.float64), refs[4]["hidden"]) <= 5e-3


@pytest.mark.parametrize("n", [1, 16, 17, 39])
def test_prompt_in_one_launch_matches_token_by_token(n):
    from persistent_decode_megakernel_02_b200 import mk
    shape = wl.TINY
    S = 64
    bt = Batch(shape, 2, S, flags=mk.MK_FLAG_ROWS)
    prompt = [int(t) for t in wl.make_prompt(shape.vocab, n, seed=n)]
    slot, start = 1, 3
    # the oracle: positions 0..2 of slot 1 hold what three earlier decode
    # steps wrote; then the prompt token by token
    for i, t in enumerate([5, 6, 7]):
        ref = bt.ref_step(slot, t, i)
    tok = torch.tensor([5, 6, 7], dtype=torch.int32, device="cuda")
    nxt = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt.ctx.prefill(tok, nxt, slot=slot, start_pos=0)
    assert bt.ctx.sync() == 0
    for i, t in enumerate(prompt):
        ref = bt.ref_step(slot, t, start + i)
    tok = torch.tensor(prompt, dtype=torch.int32, device="cuda")
    logits = torch.zeros(shape.vocab, dtype=torch.float32, device="cuda")
    bt.ctx.prefill(tok, nxt, logits=logits, slot=slot, start_pos=start)
    assert bt.ctx.sync() == 0
    _check(logits.double().cpu().numpy(), int(nxt.item()), ref, f"prompt of {n}")
    # every KV entry the prompt wrote, both layers
    for l in range(shape.layers):
        for cache, refc in ((bt.k, bt.kr), (bt.v, bt.vr)):
            g = cache[l][slot, :, :start + n].float().cpu().numpy()
            r = torch.from_numpy(refc[slot][l][:, :start + n].view(np.int16)).view(torch.bfloat16).float().numpy()
            assert np.abs(g - r).max() <= 2e-2 * np.abs(r).max() + 1e-3
    # slot 0 was not touched
    assert float(bt.k[0][0].abs().max()) == 0.0


def test_prompt_then_batched_decode():
    # a prompt in one launch, then decode steps of that sequence and another
    from persistent_decode_megakernel_02_b200 import mk
    shape = wl.TINY
    bt = Batch(shape, 2, 64)
    prompt = [int(t) for t in wl.make_prompt(shape.vocab, 20, seed=1)]
    for i, t in enumerate(prompt):
        ref0 = bt.ref_step(0, t, i)
    tok = torch.tensor(prompt, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt.ctx.prefill(tok, nxt, slot=0, start_pos=0)
    assert bt.ctx.sync() == 0
    assert token_ok(int(nxt.item()), ref0["logits"])
    toks = [ref0["next"], 99]
    for step in range(3):
        pos = [20 + step, step]
        g_tok, g_log = bt.gpu_step(toks, pos)
        refs = [bt.ref_step(0, toks[0], pos[0]), bt.ref_step(1, toks[1], pos[1])]
        for b in range(2):
            _check(g_log[b], g_tok[b], refs[b], f"step {step} seq {b}")
        toks = [r["next"] for r in refs]


def test_batched_context_refusals_and_device_checks():
    from persistent_decode_megakernel_02_b200 import mk
    shape = wl.TINY
    bt = Batch(shape, 4, 32)
    c = bt.ctx
    tok = torch.zeros(4, dtype=torch.int32, device="cuda")
    pos = torch.zeros(4, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = torch.zeros(8, 1, dtype=torch.int32, device="cuda")
    with pytest.raises(mk.MkError):
        c.generate(tok[:1], pos[:1], 4, out, nxt[:1])           # one launch per generation: batch-1 contexts only
    with pytest.raises(mk.MkError):
        c.prefill(tok, nxt, slot=4)                              # slot beyond max_batch
    with pytest.raises(mk.MkError):
        c.prefill(tok, nxt, slot=0, start_pos=30)                # past max_seq
    # a position past max_seq inside a batch: detected on the device
    pos[2] = 32
    c.decode_step(tok, pos, nxt)
    assert c.sync() == mk.MK_ERR_INVALID
    c.reset()
    pos[2] = 0
    g_tok, g_log = bt.gpu_step([1, 2, 3, 4], [0, 0, 0, 0])
    for b in range(4):
        _check(g_log[b], g_tok[b], bt.ref_step(b, b + 1, 0), f"after reset seq {b}")
    counts, thr = c.event_counts()
    assert np.array_equal(counts.astype(np.uint64), thr.astype(np.uint64))


@pytest.mark.slow
def test_llama1b_shape_batch_of_16():
    shape = wl.LLAMA_1B
    B = 16
    S = 2048 + 8
    starts = wl.make_start_positions(B, seed=11)
    bt = Batch(shape, B, S, prefill_len=2048)
    toks = [int(t) for t in wl.make_prompt(shape.vocab, B, seed=5)]
    pos = [int(p) for p in starts]
    g_tok, g_log = bt.gpu_step(toks, pos)
    for b in range(B):
        ref = bt.ref_step(b, toks[b], pos[b])
        _check(g_log[b], g_tok[b], ref, f"seq {b} pos {pos[b]}")
