"""GPU: once-per-generation launch (mk_generate) -- n greedy steps in one
kernel launch, each step's argmax feeding the next step's embedding.

Checks: the tokens equal those of n single-step launches fed back by the
host (same arithmetic, so identical); each generated token is an argmax of
the oracle's logits for the same token sequence (within the logit
tolerance); the KV slots the launch writes match the step-by-step path; an
eos stops the launch (later slots untouched); a run past max_seq is
refused on the device.
"""
import numpy as np
import pytest
import torch

from persistent_decode_megakernel_02_b200 import workloads as wl
from harness import Pair, token_ok

pytestmark = pytest.mark.gpu


def _prefill(pair, prompt):
    """Feed the prompt through single steps on both sides; returns the
    position after it and the GPU's argmax of the last prompt token."""
    tok = None
    for pos, t in enumerate(prompt):
        tok, _ = pair.gpu_step(int(t), pos)
        pair.ref_step(int(t), pos)
    return len(prompt), tok


def _generate(pair, first_tok, pos, n, eos=-1):
    mk = pair.mk
    out = torch.full((n, 1), -7, dtype=torch.int32, device="cuda")
    pair.tok.fill_(int(first_tok))
    pair.pos.fill_(int(pos))
    pair.ctx.generate(pair.tok, pair.pos, n, out, pair.nxt, eos=eos)
    st = pair.ctx.sync()
    if st != 0:
        raise mk.MkError(st, "generate")
    return out[:, 0].cpu().numpy(), int(pair.nxt.item())


# 32: MK_FLAG_ATTN_KV_ITEMS (the attention items of the long-cache kernel)
@pytest.mark.parametrize("flags", [0, 4, 32])
def test_generate_equals_step_by_step_and_oracle(flags):
    shape = wl.TINY
    n = 24
    prompt = wl.make_prompt(shape.vocab, 8, seed=21)
    a = Pair(shape, max_seq=64, flags=flags)
    b = Pair(shape, max_seq=64, flags=flags)
    pos0, first = _prefill(a, prompt)
    _prefill(b, prompt)
    gen, last = _generate(a, first, pos0, n)
    # step by step, host feeding back the argmax
    steps = []
    t = first
    for i in range(n):
        t, _ = b.gpu_step(t, pos0 + i, want_logits=False)
        steps.append(t)
    assert gen.tolist() == steps
    assert last == steps[-1]
    # KV slots written by the generation equal the step-by-step ones
    for l in range(shape.layers):
        assert torch.equal(a.k_gpu[l][0, :, :pos0 + n], b.k_gpu[l][0, :, :pos0 + n])
        assert torch.equal(a.v_gpu[l][0, :, :pos0 + n], b.v_gpu[l][0, :, :pos0 + n])
    # every generated token is an argmax of the oracle's logits for the
    # same token sequence
    t = first
    for i in range(n):
        ref = a.ref_step(t, pos0 + i)
        assert token_ok(int(gen[i]), ref["logits"]), f"step {i}"
        t = int(gen[i])
    counts, thr = a.ctx.event_counts()
    steps_run = len(prompt) + n
    assert np.array_equal(counts.astype(np.uint64), (thr.astype(np.uint64) * steps_run) % (1 << 32))


def test_generate_stops_at_eos_and_leaves_later_slots():
    shape = wl.TINY
    prompt = wl.make_prompt(shape.vocab, 5, seed=3)
    a = Pair(shape, max_seq=64)
    pos0, first = _prefill(a, prompt)
    gen, _ = _generate(a, first, pos0, 12)
    # eos := the token first produced at step k (the latest step with a new
    # token; greedy runs on random weights soon repeat themselves)
    new = [i for i in range(12) if gen[i] not in gen[:i]]
    k = new[-1]
    eos = int(gen[k])
    b = Pair(shape, max_seq=64)
    _prefill(b, prompt)
    before_k = b.k_gpu[0].clone()
    gen_b, last = _generate(b, first, pos0, 12, eos=eos)
    assert gen_b[:k + 1].tolist() == gen[:k + 1].tolist()
    assert last == eos
    # steps after the stop were not run: their outputs and KV slots are untouched
    assert np.all(gen_b[k + 1:] == -7)
    slot = pos0 + k + 1   # the first step that would have followed
    assert torch.equal(b.k_gpu[0][0, :, slot:], before_k[0, :, slot:])
    # the context goes on with single steps afterwards
    t, _ = b.gpu_step(eos, pos0 + k + 1)
    assert 0 <= t < shape.vocab


def test_generate_past_max_seq_is_refused_on_device():
    shape = wl.TINY
    a = Pair(shape, max_seq=16)
    mk = a.mk
    out = torch.zeros((8, 1), dtype=torch.int32, device="cuda")
    a.tok.fill_(3)
    a.pos.fill_(10)                       # 10 + 8 > 16
    a.ctx.generate(a.tok, a.pos, 8, out, a.nxt)
    assert a.ctx.sync() == mk.MK_ERR_INVALID
    a.ctx.reset()
    a.tok.fill_(3)
    a.pos.fill_(8)                        # 8 + 8 = 16: fits
    a.ctx.generate(a.tok, a.pos, 8, out, a.nxt)
    assert a.ctx.sync() == 0


@pytest.mark.slow
def test_llama1b_generate_equals_step_by_step():
    shape = wl.LLAMA_1B
    n = 16
    prompt = wl.make_prompt(shape.vocab, 4, seed=42)
    a = Pair(shape, max_seq=64)
    b = Pair(shape, max_seq=64)
    pos0, first = _prefill(a, prompt)
    _prefill(b, prompt)
    gen, _ = _generate(a, first, pos0, n)
    t = first
    steps = []
    for i in range(n):
        t, _ = b.gpu_step(t, pos0 + i, want_logits=False)
        steps.append(t)
    assert gen.tolist() == steps


@pytest.mark.parametrize("flags", [0, 4])
def test_prompt_and_generation_in_one_launch(flags):
    """The prompt (teacher-forced) and the generation in ONE launch equal the
    same sequence of single-step launches; every generated token is an
    argmax of the oracle's logits."""
    shape = wl.TINY
    n_prompt, n_gen = 11, 13
    n = n_prompt + n_gen - 1            # the last prompt step yields the first generated token
    prompt = wl.make_prompt(shape.vocab, n_prompt, seed=77)
    a = Pair(shape, max_seq=64, flags=flags)
    b = Pair(shape, max_seq=64, flags=flags)
    out = torch.full((n, 1), -7, dtype=torch.int32, device="cuda")
    toks = torch.from_numpy(prompt.astype(np.int32)).cuda().view(n_prompt, 1)
    a.pos.fill_(0)
    a.ctx.generate(toks, a.pos, n, out, a.nxt)
    assert a.ctx.sync() == 0
    gen = out[:, 0].cpu().numpy()
    # single steps: the prompt, then the argmax fed back
    ref_argmax = []
    t = int(prompt[0])
    for s in range(n):
        g, _ = b.gpu_step(t, s, want_logits=False)
        ref_argmax.append(g)
        t = int(prompt[s + 1]) if s + 1 < n_prompt else g
    assert gen.tolist() == ref_argmax
    for l in range(shape.layers):
        assert torch.equal(a.k_gpu[l][0, :, :n], b.k_gpu[l][0, :, :n])
    # the oracle, fed the prompt and then the GPU's tokens
    t = int(prompt[0])
    for s in range(n):
        ref = a.ref_step(t, s)
        if s >= n_prompt - 1:
            assert token_ok(int(gen[s]), ref["logits"]), f"step {s}"
        t = int(prompt[s + 1]) if s + 1 < n_prompt else int(gen[s])


def test_prompt_token_out_of_range_is_refused():
    shape = wl.TINY
    a = Pair(shape, max_seq=32)
    mk = a.mk
    toks = torch.tensor([[1], [2], [shape.vocab]], dtype=torch.int32, device="cuda")
    out = torch.zeros((6, 1), dtype=torch.int32, device="cuda")
    a.pos.fill_(0)
    a.ctx.generate(toks, a.pos, 6, out, a.nxt)
    assert a.ctx.sync() == mk.MK_ERR_INVALID
    a.ctx.reset()
