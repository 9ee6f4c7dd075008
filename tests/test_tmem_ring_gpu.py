"""The tensor-memory weight ring on the GPU.

Ops whose rows are 2048 columns wide (and 4096 / 8192 as 2048-column
segments) stream their weight pages through tensor memory: the shared-memory
page is copied on into a TMEM slot as soon as it lands and the workers read
it back from there.  A small model with hidden = ffn = 2048 takes that path in
every GEMV op; its steps must match the oracle teacher-forced, and the
logits must equal, bit for bit, those of the same model run with every page
in shared memory (MK_FLAG_NO_TMEM_RING): both paths add the same products in
the same order.
"""
import numpy as np
import pytest
import torch

from persistent_decode_megakernel_02_b200 import workloads as wl
from harness import Pair, logit_tol, token_ok, rel_l2

pytestmark = pytest.mark.gpu

MID = wl.ModelShape("mid-2048", 2, 2048, 32, 8, 64, 2048, 8192, True, 5e5)
MID_SEG = wl.ModelShape("mid-seg", 2, 2048, 16, 4, 128, 8192, 6144, False, 5e5)


@pytest.mark.parametrize("flags", [0, 4])
@pytest.mark.parametrize("shape", [MID, MID_SEG], ids=["k2048", "down-k8192"])
def test_tmem_ring_matches_oracle_and_shared_memory_path(shape, flags):
    from persistent_decode_megakernel_02_b200 import mk
    pair = Pair(shape, max_seq=64, flags=flags, gains="random")
    ref_pair = Pair(shape, max_seq=64, flags=flags | mk.MK_FLAG_NO_TMEM_RING, gains="random")
    prompt = [int(t) for t in wl.make_prompt(shape.vocab, 5, seed=4)]
    fed = list(prompt)
    for step, pos, g_tok, g_log, ref in pair.teacher_forced(prompt, 4):
        d = np.abs(g_log - ref["logits"]).max()
        assert d <= logit_tol(ref["logits"]), f"step {step}: {d:.3e}"
        assert token_ok(g_tok, ref["logits"])
        # the same token through the shared-memory-only context
        _, s_log = ref_pair.gpu_step(fed[step], pos)
        assert np.array_equal(g_log, s_log), f"step {step}: TMEM and shared-memory paths differ"
        if step >= len(prompt) - 1:      # from the last prompt token on, the oracle's argmax is fed
            fed.append(ref["next"])
    h = pair.ctx.read_buffer(mk.MK_BUF_HIDDEN, shape.hidden).astype(np.float64)
    assert rel_l2(h, ref["hidden"]) <= 5e-3
    counts, thr = pair.ctx.event_counts()
    assert np.array_equal(counts.astype(np.uint64), thr.astype(np.uint64) * 9)


def test_tmem_ring_in_one_launch_generation():
    # many steps in one launch keep the TMEM slots cycling across steps
    from persistent_decode_megakernel_02_b200 import mk
    shape = MID
    pair = Pair(shape, max_seq=64)
    single = Pair(shape, max_seq=64, flags=mk.MK_FLAG_NO_TMEM_RING)
    n = 24
    tok = torch.tensor([7], dtype=torch.int32, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_a = torch.zeros(n, 1, dtype=torch.int32, device="cuda")
    out_b = torch.zeros(n, 1, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(1, dtype=torch.int32, device="cuda")
    pair.ctx.generate(tok, pos, n, out_a, nxt)
    assert pair.ctx.sync() == 0
    single.ctx.generate(tok, pos, n, out_b, nxt)
    assert single.ctx.sync() == 0
    assert torch.equal(out_a, out_b)
    assert torch.equal(pair.k_gpu[0], single.k_gpu[0]) and torch.equal(pair.v_gpu[1], single.v_gpu[1])
