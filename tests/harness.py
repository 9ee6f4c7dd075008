"""Shared setup for the GPU parity tests: build a model on the GPU from the
seeded generators, give the oracle host copies of the same bits, and run the
two side by side teacher-forced (the oracle's token is fed to both)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
from persistent_decode_megakernel_02_b200 import workloads as wl


def logit_tol(ref: np.ndarray) -> float:
    """max|dlogit| <= 1e-2 * max|logit| + 1e-3 (the stated acceptance bound)."""
    return 1e-2 * float(np.abs(ref).max()) + 1e-3


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def token_ok(gpu_tok: int, ref_logits: np.ndarray) -> bool:
    """The GPU's argmax is accepted if it is the oracle's, or if its oracle
    logit is within the logit tolerance of the oracle maximum (several
    tokens can be correct when logits nearly tie)."""
    top = int(np.argmax(ref_logits))
    if gpu_tok == top:
        return True
    if not 0 <= gpu_tok < ref_logits.size:
        return False
    return ref_logits[top] - ref_logits[gpu_tok] <= logit_tol(ref_logits)


class Pair:
    """A model instantiated on both sides with identical bits."""

    def __init__(self, shape: wl.ModelShape, max_seq: int, seed: int = 1234,
                 gains: str = "ones", tied=None, prefill_len: int = 0, std: float = 0.02,
                 flags: int = 0, attn_chunks: int = 0, timeout_ns: int = 0):
        from persistent_decode_megakernel_02_b200 import mk
        self.mk = mk
        self.shape = shape
        self.max_seq = max_seq
        self.w_gpu = wl.make_weights(shape, seed=seed, device="cuda", gains=gains, tied=tied,
                                     std=std)
        self.k_gpu, self.v_gpu = wl.make_kv(shape, 1, max_seq, device="cuda",
                                            prefill_len=prefill_len)
        bits = self.w_gpu.numpy_bits()
        cfg = dict(layers=shape.layers, hidden=shape.hidden, n_q_heads=shape.n_q_heads,
                   n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, ffn=shape.ffn,
                   vocab=shape.vocab, max_seq=max_seq, rope_theta=shape.rope_theta,
                   rms_eps=shape.rms_eps)
        self.oracle = orc.OracleModel(cfg, bits)
        # oracle's own cache for sequence 0 (starts from the same prefill)
        self.k_ref = [wl.cache_bits(k[0]) .copy() for k in self.k_gpu]
        self.v_ref = [wl.cache_bits(v[0]).copy() for v in self.v_gpu]
        self.ctx = mk.Context(self.w_gpu, self.k_gpu, self.v_gpu, max_seq, 1, flags=flags,
                              attn_chunks=attn_chunks, timeout_ns=timeout_ns)
        self.tok = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.pos = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.nxt = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.logits = torch.zeros(1, shape.vocab, dtype=torch.float32, device="cuda")

    def gpu_step(self, token: int, pos: int, want_logits: bool = True):
        self.tok.fill_(int(token))
        self.pos.fill_(int(pos))
        self.ctx.decode_step(self.tok, self.pos, self.nxt, self.logits if want_logits else None)
        st = self.ctx.sync()
        if st != 0:
            raise self.mk.MkError(st, "device step")
        return int(self.nxt.item()), self.logits[0].double().cpu().numpy()

    def ref_step(self, token: int, pos: int, intermediates: bool = False) -> dict:
        return self.oracle.decode_step(self.k_ref, self.v_ref, int(token), int(pos),
                                       want_intermediates=intermediates)

    def teacher_forced(self, prompt, n_decode: int, start_pos: int = 0, check_every: int = 1):
        """Feed the prompt then the oracle's own argmax for n_decode steps.
        Yields (step, pos, gpu_tok, gpu_logits, ref) per step."""
        feed = [int(t) for t in prompt]
        pos = start_pos
        step = 0
        while feed:
            t = feed.pop(0)
            g_tok, g_log = self.gpu_step(t, pos)
            ref = self.ref_step(t, pos)
            yield step, pos, g_tok, g_log, ref
            if not feed and n_decode > 0:
                feed.append(ref["next"])
                n_decode -= 1
            pos += 1
            step += 1
