"""Named model shapes and the seeded synthetic inputs that both the CUDA path
and the oracle consume.

This module holds no arithmetic of the decode step: it only draws random
numbers and lays them out.  Recipe (the reference pages publish no weights,
prompts or datasets, so these stand in for them):

* weights: i.i.d. N(0, 0.02) drawn in fp32 and rounded to bf16 (round to
  nearest even); RMSNorm gains 1.0 unless ``gains="random"`` (then
  1 + N(0, 0.1), used to check that gains are applied).
* prompt tokens: uniform in [0, vocab).
* prefilled KV prefix (long-context and batched workloads): i.i.d. N(0, 1)
  rounded to bf16.
* batched start positions: uniform in [32, 2048].

Generation runs on the requested torch device with a seeded torch generator
(on a GPU host the weights are drawn on the GPU, which is fast, and copied
to host memory for the oracle).  The same (seed, device type) always gives
the same bits.
"""
from __future__ import annotations

from dataclasses import dataclass, field, asdict

import numpy as np
import torch


@dataclass(frozen=True)
class ModelShape:
    name: str
    layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    tied: bool
    rope_theta: float
    rms_eps: float = 1e-5

    def as_dict(self) -> dict:
        return asdict(self)

    def weight_bytes(self) -> int:
        """bf16 bytes of every weight matrix and gain vector (the embedding
        table is counted once when tied)."""
        H, F, V = self.hidden, self.ffn, self.vocab
        QD, KD = self.n_q_heads * self.head_dim, self.n_kv_heads * self.head_dim
        per_layer = (QD + 2 * KD) * H + H * QD + 2 * F * H + H * F + 2 * H
        emb = V * H * (1 if self.tied else 2)
        return 2 * (self.layers * per_layer + emb + H)


TINY = ModelShape("tiny", 2, 256, 4, 2, 64, 768, 4096, True, 1e4)
LLAMA_1B = ModelShape("llama-3.2-1b-shape", 16, 2048, 32, 8, 64, 8192, 128256, True, 5e5)
LLAMA_8B = ModelShape("llama-3-8b-shape", 32, 4096, 32, 8, 128, 14336, 128256, False, 5e5)

SHAPES = {s.name: s for s in (TINY, LLAMA_1B, LLAMA_8B)}


@dataclass(frozen=True)
class Workload:
    """A decode workload: a model shape, a batch, a prompt and step count."""
    name: str
    shape: ModelShape
    batch: int
    prompt_len: int          # tokens fed teacher-forced before decoding
    decode_steps: int
    max_seq: int             # KV capacity per sequence
    prefill_len: int = 0     # positions 0..prefill_len-1 prefilled with N(0,1)
    staggered: bool = False  # batched: per-sequence start positions in [32, 2048]


WORKLOADS = {
    "tiny": Workload("tiny", TINY, 1, 16, 32, 64),
    "llama1b": Workload("llama1b", LLAMA_1B, 1, 39, 512, 560),
    "llama8b": Workload("llama8b", LLAMA_8B, 1, 39, 512, 560),
    "longctx": Workload("longctx", LLAMA_1B, 1, 0, 256, 16640, prefill_len=16384),
    "batched4": Workload("batched4", LLAMA_1B, 4, 0, 128, 2048 + 136, prefill_len=2048, staggered=True),
    "batched8": Workload("batched8", LLAMA_1B, 8, 0, 128, 2048 + 136, prefill_len=2048, staggered=True),
    "batched16": Workload("batched16", LLAMA_1B, 16, 0, 128, 2048 + 136, prefill_len=2048, staggered=True),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal_bf16(shape, std: float, g: torch.Generator, device) -> torch.Tensor:
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


@dataclass
class ModelWeights:
    """bf16 weights of one model, as torch tensors on one device."""
    shape: ModelShape
    embed: torch.Tensor
    lm_head: torch.Tensor
    final_norm: torch.Tensor
    attn_norm: list = field(default_factory=list)
    mlp_norm: list = field(default_factory=list)
    wq: list = field(default_factory=list)
    wk: list = field(default_factory=list)
    wv: list = field(default_factory=list)
    wo: list = field(default_factory=list)
    wg: list = field(default_factory=list)
    wu: list = field(default_factory=list)
    wd: list = field(default_factory=list)

    def to(self, device) -> "ModelWeights":
        mv = lambda t: t.to(device)
        emb = mv(self.embed)
        lm = emb if self.lm_head is self.embed else mv(self.lm_head)
        return ModelWeights(self.shape, emb, lm, mv(self.final_norm),
                            *[[mv(t) for t in getattr(self, k)] for k in
                              ("attn_norm", "mlp_norm", "wq", "wk", "wv", "wo", "wg", "wu", "wd")])

    def numpy_bits(self) -> dict:
        """uint16 bf16 bit patterns (host) in the oracle's dict layout."""
        def b(t):
            return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        d = {"embed": b(self.embed), "final_norm": b(self.final_norm)}
        d["lm_head"] = d["embed"] if self.lm_head is self.embed else b(self.lm_head)
        for k in ("attn_norm", "mlp_norm", "wq", "wk", "wv", "wo", "wg", "wu", "wd"):
            d[k] = [b(t) for t in getattr(self, k)]
        return d


def make_weights(shape: ModelShape, seed: int = 1234, device="cpu",
                 gains: str = "ones", tied: bool | None = None,
                 std: float = 0.02) -> ModelWeights:
    """Draw every weight of `shape` in a fixed order from one generator."""
    tied = shape.tied if tied is None else tied
    g = _gen(device, seed)
    H, F, V = shape.hidden, shape.ffn, shape.vocab
    QD, KD = shape.n_q_heads * shape.head_dim, shape.n_kv_heads * shape.head_dim

    def gain():
        if gains == "ones":
            return torch.ones(H, device=device, dtype=torch.bfloat16)
        t = torch.randn(H, generator=g, device=device, dtype=torch.float32)
        return (1.0 + 0.1 * t).to(torch.bfloat16)

    embed = _normal_bf16((V, H), std, g, device)
    lm = embed if tied else _normal_bf16((V, H), std, g, device)
    w = ModelWeights(shape, embed, lm, gain())
    for _ in range(shape.layers):
        w.attn_norm.append(gain())
        w.mlp_norm.append(gain())
        w.wq.append(_normal_bf16((QD, H), std, g, device))
        w.wk.append(_normal_bf16((KD, H), std, g, device))
        w.wv.append(_normal_bf16((KD, H), std, g, device))
        w.wo.append(_normal_bf16((H, QD), std, g, device))
        w.wg.append(_normal_bf16((F, H), std, g, device))
        w.wu.append(_normal_bf16((F, H), std, g, device))
        w.wd.append(_normal_bf16((H, F), std, g, device))
    return w


def make_kv(shape: ModelShape, max_batch: int, max_seq: int, device="cpu",
            prefill_len: int = 0, seed: int = 77) -> tuple[list, list]:
    """Per-layer bf16 caches [max_batch][nkv][max_seq][d]; positions
    0..prefill_len-1 of every sequence hold N(0,1) values, the rest zeros."""
    g = _gen(device, seed)
    shp = (max_batch, shape.n_kv_heads, max_seq, shape.head_dim)
    ks, vs = [], []
    for _ in range(shape.layers):
        k = torch.zeros(shp, device=device, dtype=torch.bfloat16)
        v = torch.zeros(shp, device=device, dtype=torch.bfloat16)
        if prefill_len:
            k[:, :, :prefill_len].copy_(_normal_bf16(
                (max_batch, shape.n_kv_heads, prefill_len, shape.head_dim), 1.0, g, device))
            v[:, :, :prefill_len].copy_(_normal_bf16(
                (max_batch, shape.n_kv_heads, prefill_len, shape.head_dim), 1.0, g, device))
        ks.append(k)
        vs.append(v)
    return ks, vs


def make_prompt(vocab: int, n: int, seed: int = 42) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def make_start_positions(batch: int, seed: int = 7, lo: int = 32, hi: int = 2048) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=batch, dtype=np.int64).astype(np.int32)


def cache_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 view (host copy) of a bf16 tensor."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
