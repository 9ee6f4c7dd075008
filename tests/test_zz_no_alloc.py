"""mk_decode_step_static -- the decode step for callers that cannot allocate
device memory where they decode (an arena that owns all device memory, an
allocation-free serving loop).  It keeps its scratch in a fixed device array
inside the library instead of allocating, and takes weights in the kernel's
packed layout.

This file is collected last on purpose (so a run that stops at the first
failure has already run every other test).  It checks, through the C ABI,
that two consecutive calls give the same result as the context-based
mk_decode_step on the same inputs, within the logit tolerance the parity
tests use, and that a shape too large for the fixed scratch is refused.
"""
import numpy as np
import pytest
import torch

from persistent_decode_megakernel_02_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _pack(weights):
    """q/k/v and gate/up in the packed tile order documented in mk.h."""
    s = weights.shape
    H, d, F = s.hidden, s.head_dim, s.ffn
    qkv, gu = [], []
    for l in range(s.layers):
        qkv.append(torch.cat([weights.wq[l], weights.wk[l], weights.wv[l]]).contiguous())
        gu.append(torch.stack([weights.wg[l].view(F // 8, 8, H), weights.wu[l].view(F // 8, 8, H)],
                              dim=1).reshape(2 * F, H).contiguous())
    return {"embed": weights.embed, "lm_head": weights.lm_head, "final_norm": weights.final_norm,
            "attn_norm": weights.attn_norm, "mlp_norm": weights.mlp_norm, "qkv": qkv,
            "wo": weights.wo, "gu": gu, "wd": weights.wd}


def test_static_step_matches_context_step_twice():
    from persistent_decode_megakernel_02_b200 import mk
    shape = wl.TINY
    S = 48
    w = wl.make_weights(shape, seed=99, device="cuda")
    packed = _pack(w)
    k_ctx, v_ctx = wl.make_kv(shape, 1, S, device="cuda")
    k_st, v_st = wl.make_kv(shape, 1, S, device="cuda")
    ctx = mk.Context(w, k_ctx, v_ctx, S, 1)
    cfg = mk.make_config(shape, S, 1)
    tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    nxt_a = torch.zeros(1, dtype=torch.int32, device="cuda")
    nxt_b = torch.zeros(1, dtype=torch.int32, device="cuda")
    log_a = torch.zeros(1, shape.vocab, dtype=torch.float32, device="cuda")
    log_b = torch.zeros(1, shape.vocab, dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for p_, t_ in ((0, 17), (1, 4093)):
        tok.fill_(t_)
        pos.fill_(p_)
        ctx.decode_step(tok, pos, nxt_a, log_a)
        assert ctx.sync() == 0
        st = mk.decode_step_static(cfg, packed, k_st, v_st, tok, pos, nxt_b, log_b, status)
        assert st == 0, mk.status_string(st)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        a = log_a[0].double().cpu().numpy()
        b = log_b[0].double().cpu().numpy()
        tol = 1e-2 * np.abs(a).max() + 1e-3
        assert np.abs(a - b).max() <= tol
        assert int(nxt_a.item()) == int(nxt_b.item())
    # the KV entries both paths wrote agree
    for l in range(shape.layers):
        assert torch.allclose(k_ctx[l][:, :, :2].float(), k_st[l][:, :, :2].float(), rtol=1e-2, atol=1e-3)
    ctx.close()


def test_static_step_refuses_shapes_beyond_the_fixed_scratch():
    from persistent_decode_megakernel_02_b200 import mk
    shape = wl.TINY
    w = wl.make_weights(shape, seed=5, device="cuda")
    packed = _pack(w)
    k, v = wl.make_kv(shape, 1, 8, device="cuda")
    big = mk.make_config(shape, 1 << 20, 1)     # RoPE table alone would exceed the scratch
    tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    nxt = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert mk.decode_step_static(big, packed, k, v, tok, pos, nxt) == mk.MK_ERR_INVALID
