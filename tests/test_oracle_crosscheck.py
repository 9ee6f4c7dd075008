"""CPU cross-checks of the oracle by independent formulations.

- The split-K merge the kernel uses for long contexts (per chunk c of
  positions a partial (m_c = max s, l_c = sum exp(s - m_c), o_c = sum
  exp(s - m_c) v); merged o = sum exp(m_c - M) o_c / sum exp(m_c - M) l_c
  with M = max m_c) equals the oracle's unsplit attention for every chunk
  count, ragged and empty chunks included.
- A whole decode step restated with library operations in fp64 -- RoPE as
  a complex rotation of the pairs (x_i, x_{i+d/2}), GQA by repeating each
  KV head over its q heads, torch softmax and SiLU -- equals the oracle's
  step on the tiny shape with random gains and an untied head, position by
  position, KV cache writes included.  This is a restatement with library
  routines, not a pin by itself; it catches composition slips (a gain
  applied at the wrong norm, a residual in the wrong place, a head mapping
  or cache slot off by one) that the per-function pins cannot see.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from persistent_decode_megakernel_02_b200 import workloads as wl


def _bits(a) -> np.ndarray:
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _widen(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---- split-K merge -----------------------------------------------------------

def _partials(q, K, V, lo, hi):
    """(o, m, l) of positions [lo, hi) for one q head, fp64."""
    d = q.size
    if hi <= lo:
        return np.zeros(d), -np.inf, 0.0
    s = K[lo:hi] @ q / np.sqrt(d)
    m = s.max()
    e = np.exp(s - m)
    return e @ V[lo:hi], m, e.sum()


def _merge(parts):
    M = max(m for _, m, _ in parts)
    num = sum(np.exp(m - M) * o for o, m, _ in parts if m != -np.inf)
    den = sum(np.exp(m - M) * l for _, m, l in parts if m != -np.inf)
    return num / den


@pytest.mark.parametrize("nchunks", [1, 2, 3, 5, 7])
def test_split_k_merge_equals_unsplit_attention(nchunks):
    rng = np.random.default_rng(100 + nchunks)
    nq, nkv, d, S, C = 4, 2, 64, 40, 37
    q = rng.standard_normal((nq, d))
    kc = _bits(rng.standard_normal((nkv, S, d)))
    vc = _bits(rng.standard_normal((nkv, S, d)))
    ref = orc.attention(q, kc, vc, C)
    K, V = _widen(kc), _widen(vc)
    # ragged chunks: ceil(C / nchunks) positions each, the last ones short or
    # empty (as the kernel splits a context)
    Lc = -(-C // nchunks)
    for h in range(nq):
        g = h // (nq // nkv)
        parts = [_partials(q[h], K[g], V[g], min(c * Lc, C), min((c + 1) * Lc, C))
                 for c in range(nchunks)]
        got = _merge(parts)
        assert np.allclose(got, ref[h], rtol=1e-12, atol=1e-12)


def test_split_k_merge_with_empty_chunks_and_one_position():
    rng = np.random.default_rng(7)
    d = 64
    q = rng.standard_normal((1, d))
    kc = _bits(rng.standard_normal((1, 8, d)))
    vc = _bits(rng.standard_normal((1, 8, d)))
    K, V = _widen(kc), _widen(vc)
    # C = 1: one position in chunk 0, the other chunks empty -> o = v_0
    parts = [_partials(q[0], K[0], V[0], 0, 1)] + [_partials(q[0], K[0], V[0], 1, 1)] * 3
    assert np.allclose(_merge(parts), V[0, 0], rtol=0, atol=1e-15)
    assert np.allclose(orc.attention(q, kc, vc, 1)[0], V[0, 0], rtol=0, atol=1e-15)


# ---- whole step, restated with library operations ----------------------------

def _rope_complex(x: torch.Tensor, pos: int, theta: float) -> torch.Tensor:
    """x [..., d]: pairs (x_i, x_{i+d/2}) rotated by pos * theta^(-2i/d)."""
    d = x.shape[-1]
    h = d // 2
    z = torch.complex(x[..., :h], x[..., h:])
    i = torch.arange(h, dtype=torch.float64)
    ang = pos * theta ** (-2.0 * i / d)
    z = z * torch.polar(torch.ones_like(ang), ang)
    return torch.cat([z.real, z.imag], dim=-1)


class _TorchModel:
    def __init__(self, shape, bits, max_seq):
        self.s = shape
        f = lambda a: torch.from_numpy(_widen(a))
        H, d = shape.hidden, shape.head_dim
        self.E = f(bits["embed"]).reshape(shape.vocab, H)
        self.lm = f(bits["lm_head"]).reshape(shape.vocab, H)
        self.gf = f(bits["final_norm"])
        self.layers = []
        for l in range(shape.layers):
            self.layers.append(dict(
                g1=f(bits["attn_norm"][l]), g2=f(bits["mlp_norm"][l]),
                wq=f(bits["wq"][l]).reshape(-1, H), wk=f(bits["wk"][l]).reshape(-1, H),
                wv=f(bits["wv"][l]).reshape(-1, H), wo=f(bits["wo"][l]).reshape(H, -1),
                wg=f(bits["wg"][l]).reshape(-1, H), wu=f(bits["wu"][l]).reshape(-1, H),
                wd=f(bits["wd"][l]).reshape(H, -1)))
        z = lambda: torch.zeros(shape.n_kv_heads, max_seq, d, dtype=torch.float64)
        self.K = [z() for _ in range(shape.layers)]
        self.V = [z() for _ in range(shape.layers)]

    def _norm(self, x, g):
        return x * torch.rsqrt(torch.mean(x * x) + self.s.rms_eps) * g

    def step(self, tok, pos):
        s = self.s
        nq, nkv, d = s.n_q_heads, s.n_kv_heads, s.head_dim
        x = self.E[tok].clone()
        for l, w in enumerate(self.layers):
            xn = self._norm(x, w["g1"])
            q = _rope_complex((w["wq"] @ xn).reshape(nq, d), pos, s.rope_theta)
            k = _rope_complex((w["wk"] @ xn).reshape(nkv, d), pos, s.rope_theta)
            v = (w["wv"] @ xn).reshape(nkv, d)
            self.K[l][:, pos] = k.to(torch.bfloat16).to(torch.float64)
            self.V[l][:, pos] = v.to(torch.bfloat16).to(torch.float64)
            Kg = self.K[l][:, :pos + 1].repeat_interleave(nq // nkv, dim=0)   # [nq, C, d]
            Vg = self.V[l][:, :pos + 1].repeat_interleave(nq // nkv, dim=0)
            p = torch.softmax(torch.einsum("hd,hcd->hc", q, Kg) / d ** 0.5, dim=-1)
            o = torch.einsum("hc,hcd->hd", p, Vg).reshape(-1)
            x = x + w["wo"] @ o
            hn = self._norm(x, w["g2"])
            x = x + w["wd"] @ (torch.nn.functional.silu(w["wg"] @ hn) * (w["wu"] @ hn))
        logits = self.lm @ self._norm(x, self.gf)
        return logits.numpy(), x.numpy()


def test_torch_fp64_forward_matches_oracle_step_by_step():
    shape = wl.TINY
    S = 20
    w = wl.make_weights(shape, seed=31, device="cpu", gains="random", tied=False)
    bits = w.numpy_bits()
    cfg = dict(layers=shape.layers, hidden=shape.hidden, n_q_heads=shape.n_q_heads,
               n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim, ffn=shape.ffn,
               vocab=shape.vocab, max_seq=S, rope_theta=shape.rope_theta,
               rms_eps=shape.rms_eps)
    model = orc.OracleModel(cfg, bits)
    kc, vc = model.new_cache()
    tm = _TorchModel(shape, bits, S)
    toks = wl.make_prompt(shape.vocab, 12, seed=8)
    for pos, t in enumerate(toks):
        out = model.decode_step(kc, vc, int(t), pos)
        logits, hidden = tm.step(int(t), pos)
        # both sides round the same fp64 k, v to bf16; the caches agree bit for bit
        for l in range(shape.layers):
            assert np.array_equal(_widen(kc[l][:, :pos + 1]), tm.K[l][:, :pos + 1].numpy())
            assert np.array_equal(_widen(vc[l][:, :pos + 1]), tm.V[l][:, :pos + 1].numpy())
        scale = np.abs(logits).max()
        assert np.max(np.abs(out["logits"] - logits)) <= 1e-9 * scale, pos
        assert np.allclose(out["hidden"], hidden, rtol=1e-9, atol=1e-12)
        assert out["next"] == int(np.argmax(logits))
