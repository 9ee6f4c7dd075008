"""mk_decode_step_static -- the decode step for callers that cannot allocate
device memory where they decode (an arena that owns all device memory, an
allocation-free serving loop).  It keeps its scratch in a fixed device array
inside the library instead of allocating, and takes weights in the kernel's
packed layout.

This file is collected last on purpose (so a run that stops at the first
failure has already run every other test).  It checks, through the C ABI,
that consecutive calls give the same logits, bit for bit, as the
context-based mk_decode_step on the same inputs (same kernel, same task
graph), also when calls alternate between shapes and weight sets; that on
the Llama-3.2-1B shape it matches the oracle within the logit tolerance of
the parity tests; and that a shape too large for the fixed scratch is
refused.
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


def _io(vocab):
    z = lambda: torch.zeros(1, dtype=torch.int32, device="cuda")
    return {"tok": z(), "pos": z(), "nxt_a": z(), "nxt_b": z(),
            "log_a": torch.zeros(1, vocab, dtype=torch.float32, device="cuda"),
            "log_b": torch.zeros(1, vocab, dtype=torch.float32, device="cuda"),
            "status": torch.full((1,), -1, dtype=torch.int32, device="cuda")}


def _both(mk, ctx, cfg, packed, k_st, v_st, io, tok, pos):
    """One step through the context and one through the no-allocation entry
    point on the same inputs; both run the same kernel on the same task graph,
    so the logits agree bit for bit."""
    io["tok"].fill_(tok)
    io["pos"].fill_(pos)
    ctx.decode_step(io["tok"], io["pos"], io["nxt_a"], io["log_a"])
    assert ctx.sync() == 0
    io["status"].fill_(-1)
    st = mk.decode_step_static(cfg, packed, k_st, v_st, io["tok"], io["pos"], io["nxt_b"],
                               io["log_b"], io["status"])
    assert st == 0, mk.status_string(st)
    torch.cuda.synchronize()
    assert int(io["status"].item()) == 0
    assert torch.equal(io["log_a"], io["log_b"])
    assert int(io["nxt_a"].item()) == int(io["nxt_b"].item())
    return int(io["nxt_b"].item()), io["log_b"][0].double().cpu().numpy()


@pytest.mark.parametrize("flags", [0, 32], ids=["q-items", "kv-items"])
def test_static_step_matches_context_step_twice(flags):
    from persistent_decode_megakernel_02_b200 import mk
    shape = wl.TINY
    S = 48
    w = wl.make_weights(shape, seed=99, device="cuda")
    packed = _pack(w)
    k_ctx, v_ctx = wl.make_kv(shape, 1, S, device="cuda")
    k_st, v_st = wl.make_kv(shape, 1, S, device="cuda")
    ctx = mk.Context(w, k_ctx, v_ctx, S, 1, flags=flags)
    cfg = mk.make_config(shape, S, 1, flags=flags)
    assert ctx.info().attn_heads == (2 if flags else 1)
    io = _io(shape.vocab)
    for p_, t_ in ((0, 17), (1, 4093)):
        _both(mk, ctx, cfg, packed, k_st, v_st, io, t_, p_)
    # the KV entries both paths wrote are identical
    for l in range(shape.layers):
        assert torch.equal(k_ctx[l], k_st[l]) and torch.equal(v_ctx[l], v_st[l])
    ctx.close()


def test_static_step_alternating_shapes_and_weights():
    # every change of shape re-uploads the task and RoPE tables, every change
    # of weight or KV pointers the layer table: alternate both and compare
    # each call with a context built for the same model
    from persistent_decode_megakernel_02_b200 import mk
    untied = wl.ModelShape("tiny-untied", 2, 256, 4, 2, 64, 768, 4096, False, 1e4)
    models = []
    # model 3: model 0's sizes with the attention items of one KV head's q
    # heads together (MK_FLAG_ATTN_KV_ITEMS): the same config sizes, another
    # task graph and scratch layout
    for shape, S, seed, flags in ((wl.TINY, 48, 1, 0), (untied, 40, 2, 0), (wl.TINY, 48, 3, 0),
                                  (wl.TINY, 48, 4, 32)):
        w = wl.make_weights(shape, seed=seed, device="cuda")
        kc, vc = wl.make_kv(shape, 1, S, device="cuda")
        ks, vs = wl.make_kv(shape, 1, S, device="cuda")
        models.append(dict(shape=shape, packed=_pack(w), ctx=mk.Context(w, kc, vc, S, 1, flags=flags),
                           cfg=mk.make_config(shape, S, 1, flags=flags), k=ks, v=vs, pos=0,
                           io=_io(shape.vocab)))
    for i, m in enumerate([0, 1, 0, 3, 2, 1, 3, 2, 0, 3]):
        M = models[m]
        _both(mk, M["ctx"], M["cfg"], M["packed"], M["k"], M["v"], M["io"], 100 + 7 * i, M["pos"])
        M["pos"] += 1
    for M in models:
        M["ctx"].close()


@pytest.mark.slow
def test_static_step_on_the_llama1b_shape_against_the_oracle():
    # the 1B shape needs about 3.2 MiB of the fixed scratch at max_seq 560
    import oracle as orc
    from persistent_decode_megakernel_02_b200 import mk
    shape = wl.LLAMA_1B
    S = 560
    w = wl.make_weights(shape, seed=1234, device="cuda")
    packed = _pack(w)
    k_ctx, v_ctx = wl.make_kv(shape, 1, S, device="cuda")
    k_st, v_st = wl.make_kv(shape, 1, S, device="cuda")
    ctx = mk.Context(w, k_ctx, v_ctx, S, 1)
    cfg = mk.make_config(shape, S, 1)
    io = _io(shape.vocab)
    ocfg = dict(layers=shape.layers, hidden=shape.hidden, n_q_heads=shape.n_q_heads,
                n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, ffn=shape.ffn,
                vocab=shape.vocab, max_seq=S, rope_theta=shape.rope_theta, rms_eps=shape.rms_eps)
    model = orc.OracleModel(ocfg, w.numpy_bits())
    kr, vr = model.new_cache()
    tok = 12345
    for pos in range(2):
        g_tok, g_log = _both(mk, ctx, cfg, packed, k_st, v_st, io, tok, pos)
        ref = model.decode_step(kr, vr, tok, pos)
        tol = 1e-2 * np.abs(ref["logits"]).max() + 1e-3
        assert np.abs(g_log - ref["logits"]).max() <= tol
        top = int(np.argmax(ref["logits"]))
        assert g_tok == top or ref["logits"][top] - ref["logits"][g_tok] <= tol
        tok = ref["next"]
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
