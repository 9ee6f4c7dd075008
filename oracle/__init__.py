"""ctypes wrapper of the C oracle (mk_oracle.c).

TEST INFRASTRUCTURE ONLY: the plain fp64 CPU definition of the decode step
that the CUDA library is checked against.  Only tests/, the smoke check in
__graft_entry__ and the CPU-baseline leg of bench.py may import this module.
It imports nothing from the CUDA package and shares no code with it.

Arrays are numpy: weights and KV caches as uint16 bf16 bit patterns,
activations as float64.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mk_oracle.c")
_LIB = os.path.join(_HERE, "libmk_oracle.so")


def build(force: bool = False) -> str:
    """Compile mk_oracle.c into libmk_oracle.so next to it (gcc, -O2, no
    fast-math so every sum keeps its written order)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "mk_oracle.h"))
    ):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-Wall", "-Wextra",
             "-o", _LIB, _SRC, "-lm"]
        )
    return _LIB


class _Config(C.Structure):
    _fields_ = [
        ("layers", C.c_int), ("hidden", C.c_int), ("n_q_heads", C.c_int),
        ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
        ("vocab", C.c_int), ("max_seq", C.c_int),
        ("rope_theta", C.c_double), ("rms_eps", C.c_double),
    ]


_P16 = C.POINTER(C.c_uint16)
_PP16 = C.POINTER(_P16)


class _Weights(C.Structure):
    _fields_ = [
        ("embed", _P16), ("lm_head", _P16), ("final_norm", _P16),
        ("attn_norm", _PP16), ("mlp_norm", _PP16),
        ("wq", _PP16), ("wk", _PP16), ("wv", _PP16), ("wo", _PP16),
        ("wg", _PP16), ("wu", _PP16), ("wd", _PP16),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        D = C.POINTER(C.c_double)
        _lib.orc_bf16_to_double.argtypes = [C.c_uint16]
        _lib.orc_bf16_to_double.restype = C.c_double
        _lib.orc_double_to_bf16.argtypes = [C.c_double]
        _lib.orc_double_to_bf16.restype = C.c_uint16
        _lib.orc_rmsnorm.argtypes = [D, _P16, C.c_int, C.c_double, D]
        _lib.orc_gemv.argtypes = [_P16, C.c_int, C.c_int, D, D]
        _lib.orc_rope.argtypes = [D, C.c_int, C.c_int, C.c_double]
        _lib.orc_silu.argtypes = [C.c_double]
        _lib.orc_silu.restype = C.c_double
        _lib.orc_argmax.argtypes = [D, C.c_int]
        _lib.orc_argmax.restype = C.c_int
        _lib.orc_attention.argtypes = [D, _P16, _P16, C.c_int, C.c_int, C.c_int,
                                       C.c_int, C.c_int, D]
        _lib.orc_decode_step.argtypes = [C.POINTER(_Config), C.POINTER(_Weights),
                                         _PP16, _PP16, C.c_int, C.c_int,
                                         D, D, D, D, D]
        _lib.orc_decode_step.restype = C.c_int
        _lib.orc_forward_recompute.argtypes = [C.POINTER(_Config), C.POINTER(_Weights),
                                               C.POINTER(C.c_int), C.c_int, D, D]
        _lib.orc_forward_recompute.restype = C.c_int
    return _lib


# ---- array helpers ---------------------------------------------------------

def _u16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 bf16 bits, got {a.dtype}")
    return a


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p16(a: np.ndarray):
    return a.ctypes.data_as(_P16)


def _pd(a: np.ndarray):
    return a.ctypes.data_as(C.POINTER(C.c_double))


# ---- building blocks -------------------------------------------------------

def bf16_to_double(bits: int) -> float:
    return lib().orc_bf16_to_double(int(bits))


def double_to_bf16(x: float) -> int:
    return int(lib().orc_double_to_bf16(float(x)))


def rmsnorm(x, g_bits: np.ndarray, eps: float) -> np.ndarray:
    x = _f64(x)
    g = _u16(g_bits)
    y = np.empty_like(x)
    lib().orc_rmsnorm(_pd(x), _p16(g), x.size, float(eps), _pd(y))
    return y


def gemv(W_bits: np.ndarray, x) -> np.ndarray:
    W = _u16(W_bits)
    x = _f64(x)
    N, K = W.shape
    y = np.empty(N, dtype=np.float64)
    lib().orc_gemv(_p16(W), N, K, _pd(x), _pd(y))
    return y


def rope(v, pos: int, theta: float) -> np.ndarray:
    v = _f64(v).copy()
    lib().orc_rope(_pd(v), v.size, int(pos), float(theta))
    return v


def silu(x: float) -> float:
    return lib().orc_silu(float(x))


def argmax(v) -> int:
    v = _f64(v)
    return lib().orc_argmax(_pd(v), v.size)


def attention(q, kc_bits: np.ndarray, vc_bits: np.ndarray, C_: int) -> np.ndarray:
    """q [nq][d]; kc, vc bf16 [nkv][max_seq][d]; positions 0..C_-1."""
    q = _f64(q)
    kc = _u16(kc_bits)
    vc = _u16(vc_bits)
    nq, d = q.shape
    nkv, S, d2 = kc.shape
    assert d2 == d and vc.shape == kc.shape
    out = np.empty_like(q)
    lib().orc_attention(_pd(q), _p16(kc), _p16(vc), nq, nkv, d, S, int(C_), _pd(out))
    return out


# ---- model-level -----------------------------------------------------------

@dataclass
class OracleModel:
    """Host-side view of a model for the oracle.

    cfg: dict with layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn,
    vocab, max_seq, rope_theta, rms_eps.  weights: dict of uint16 arrays
    (embed, lm_head, final_norm, and per-layer lists attn_norm, mlp_norm,
    wq, wk, wv, wo, wg, wu, wd)."""

    cfg: dict
    weights: dict

    def __post_init__(self):
        c = self.cfg
        self._c = _Config(c["layers"], c["hidden"], c["n_q_heads"], c["n_kv_heads"],
                          c["head_dim"], c["ffn"], c["vocab"], c["max_seq"],
                          float(c["rope_theta"]), float(c["rms_eps"]))
        w = self.weights
        self._keep = []

        def one(a):
            a = _u16(a)
            self._keep.append(a)
            return _p16(a)

        def many(lst):
            arr = (_P16 * len(lst))(*[one(a) for a in lst])
            self._keep.append(arr)
            return C.cast(arr, _PP16)

        self._w = _Weights(one(w["embed"]), one(w["lm_head"]), one(w["final_norm"]),
                           many(w["attn_norm"]), many(w["mlp_norm"]),
                           many(w["wq"]), many(w["wk"]), many(w["wv"]), many(w["wo"]),
                           many(w["wg"]), many(w["wu"]), many(w["wd"]))

    def new_cache(self) -> tuple[list, list]:
        """Empty bf16 caches for one sequence: per layer [nkv][max_seq][d]."""
        c = self.cfg
        shp = (c["n_kv_heads"], c["max_seq"], c["head_dim"])
        return ([np.zeros(shp, np.uint16) for _ in range(c["layers"])],
                [np.zeros(shp, np.uint16) for _ in range(c["layers"])])

    def decode_step(self, kcache: list, vcache: list, token: int, pos: int,
                    want_intermediates: bool = False) -> dict:
        """One cached step of one sequence; writes entry `pos` of the caches
        (lists of per-layer uint16 [nkv][max_seq][d] arrays, modified in place)."""
        c = self.cfg
        for a in kcache + vcache:
            assert a.dtype == np.uint16 and a.flags.c_contiguous
        kp = (_P16 * len(kcache))(*[_p16(a) for a in kcache])
        vp = (_P16 * len(vcache))(*[_p16(a) for a in vcache])
        logits = np.empty(c["vocab"], np.float64)
        hidden = np.empty(c["hidden"], np.float64)
        QD = c["n_q_heads"] * c["head_dim"]
        qb = np.empty(QD, np.float64) if want_intermediates else None
        ab = np.empty(QD, np.float64) if want_intermediates else None
        mb = np.empty(c["ffn"], np.float64) if want_intermediates else None
        nul = C.POINTER(C.c_double)()
        nxt = lib().orc_decode_step(C.byref(self._c), C.byref(self._w),
                                    C.cast(kp, _PP16), C.cast(vp, _PP16),
                                    int(token), int(pos), _pd(logits), _pd(hidden),
                                    _pd(qb) if qb is not None else nul,
                                    _pd(ab) if ab is not None else nul,
                                    _pd(mb) if mb is not None else nul)
        if nxt < 0:
            raise ValueError("oracle rejected the arguments")
        out = {"next": nxt, "logits": logits, "hidden": hidden}
        if want_intermediates:
            out.update(q=qb, attn=ab, act=mb)
        return out

    def forward_recompute(self, tokens) -> dict:
        c = self.cfg
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        logits = np.empty(c["vocab"], np.float64)
        hidden = np.empty(c["hidden"], np.float64)
        nxt = lib().orc_forward_recompute(C.byref(self._c), C.byref(self._w),
                                          t.ctypes.data_as(C.POINTER(C.c_int)), t.size,
                                          _pd(logits), _pd(hidden))
        if nxt < 0:
            raise ValueError("oracle rejected the arguments")
        return {"next": nxt, "logits": logits, "hidden": hidden}
