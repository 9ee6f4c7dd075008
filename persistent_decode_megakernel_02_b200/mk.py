"""Thin ctypes binding of libmk.so (include/mk.h).

Argument marshalling only: every step of the decode path runs in the CUDA
library.  Torch tensors are used for device memory and streams.  If the
library is missing this module raises at import time: there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "mk.h")

MK_OK, MK_ERR_INVALID, MK_ERR_CUDA, MK_ERR_TIMEOUT, MK_ERR_OOM, MK_ERR_STATE = range(6)
MK_FLAG_TRACE = 1
MK_FLAG_NO_L2_PREFETCH = 2
MK_FLAG_EVENT_WAIT = 4
MK_FLAG_NO_TMEM_RING = 8
MK_FLAG_ROWS = 16
MK_FLAG_ATTN_KV_ITEMS = 32
MK_FLAG_ATTN_Q_ITEMS = 64
MAX_BATCH = 16
MK_BUF_HIDDEN, MK_BUF_Q, MK_BUF_ATTN, MK_BUF_ACT = range(4)
OP_NAMES = ["qkv", "attn", "oproj", "gateup", "down", "lmhead"]

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m persistent_decode_megakernel_02_b200.build`")
_lib = C.CDLL(LIB_PATH)


class MkError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class Config(C.Structure):
    _fields_ = [
        ("layers", C.c_int), ("hidden", C.c_int), ("n_q_heads", C.c_int),
        ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int), ("vocab", C.c_int),
        ("max_seq", C.c_int), ("max_batch", C.c_int),
        ("rope_theta", C.c_float), ("rms_eps", C.c_float),
        ("flags", C.c_int), ("attn_chunks", C.c_int), ("timeout_ns", C.c_longlong),
        ("l2_lookahead_kb", C.c_int), ("poll_ns", C.c_int),
    ]


_VPP = C.POINTER(C.c_void_p)


class Weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("lm_head", C.c_void_p), ("final_norm", C.c_void_p),
                ("attn_norm", _VPP), ("mlp_norm", _VPP),
                ("wq", _VPP), ("wk", _VPP), ("wv", _VPP), ("wo", _VPP),
                ("wg", _VPP), ("wu", _VPP), ("wd", _VPP)]


class KV(C.Structure):
    _fields_ = [("k", _VPP), ("v", _VPP)]


class PackedWeights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("lm_head", C.c_void_p), ("final_norm", C.c_void_p),
                ("attn_norm", _VPP), ("mlp_norm", _VPP),
                ("qkv", _VPP), ("wo", _VPP), ("gu", _VPP), ("wd", _VPP)]


class Info(C.Structure):
    _fields_ = [("num_sms", C.c_int), ("num_tasks", C.c_int), ("num_events", C.c_int),
                ("num_ops", C.c_int), ("attn_chunks", C.c_int), ("max_queue", C.c_int),
                ("page_bytes", C.c_int), ("num_pages", C.c_int),
                ("steps_run", C.c_longlong), ("err_code", C.c_uint), ("err_info", C.c_uint),
                ("err_task", C.c_uint), ("attn_heads", C.c_int)]


class TraceRec(C.Structure):
    _fields_ = [("t_ready", C.c_ulonglong), ("t_start", C.c_ulonglong), ("t_input", C.c_ulonglong),
                ("t_done", C.c_ulonglong), ("t_end", C.c_ulonglong), ("t_wait", C.c_ulonglong),
                ("sm", C.c_int), ("kind", C.c_int), ("layer", C.c_int), ("trig_event", C.c_int)]


_P = C.c_void_p
_lib.mk_status_string.argtypes = [C.c_int]
_lib.mk_status_string.restype = C.c_char_p
_lib.mk_create.argtypes = [C.POINTER(Config), C.POINTER(Weights), C.POINTER(KV), C.POINTER(_P)]
_lib.mk_decode_step.argtypes = [_P, _P, _P, C.c_int, _P, _P, _P]
_lib.mk_sync.argtypes = [_P, _P]
_lib.mk_reset.argtypes = [_P]
_lib.mk_destroy.argtypes = [_P]
_lib.mk_get_info.argtypes = [_P, C.POINTER(Info)]
_lib.mk_get_event_counts.argtypes = [_P, _P, _P, C.c_int]
_lib.mk_read_buffer.argtypes = [_P, C.c_int, _P, C.c_size_t]
_lib.mk_get_trace.argtypes = [_P, _P, C.c_int]
_lib.mk_get_graph.argtypes = [_P, _P, _P, _P]
_lib.mk_get_sm_stats.argtypes = [_P, _P, C.c_int]
_lib.mk_plan.argtypes = [C.POINTER(Config), C.c_int, C.POINTER(Info), _P, _P, _P, _P, _P]
_lib.mk_device_supported.argtypes = [C.c_int, C.c_int, C.c_int, C.c_size_t, C.c_int]
_lib.mk_debug_set_threshold.argtypes = [_P, C.c_int, C.c_uint]
_lib.mk_debug_withhold_event.argtypes = [_P, C.c_int]
_lib.mk_generate.argtypes = [_P, _P, C.c_int, _P, C.c_int, C.c_int, C.c_int, _P, _P, _P]
_lib.mk_prefill.argtypes = [_P, _P, C.c_int, C.c_int, C.c_int, _P, _P, _P]
_lib.mk_decode_step_static.argtypes = [C.POINTER(Config), C.POINTER(PackedWeights), C.POINTER(KV),
                                       _P, _P, C.c_int, _P, _P, _P, _P]
for _f in ("mk_create", "mk_decode_step", "mk_sync", "mk_reset", "mk_destroy", "mk_get_info",
           "mk_get_event_counts", "mk_read_buffer", "mk_get_trace", "mk_get_graph", "mk_plan",
           "mk_get_sm_stats", "mk_decode_step_static",
           "mk_debug_set_threshold", "mk_debug_withhold_event", "mk_generate", "mk_prefill"):
    getattr(_lib, _f).restype = C.c_int


def status_string(status: int) -> str:
    return _lib.mk_status_string(int(status)).decode()


def device_supported(major: int, minor: int, cooperative_launch: bool, smem_optin_bytes: int,
                     batched: bool = False) -> int:
    """mk_device_supported: MK_OK if mk_create would accept a device with
    these properties (host-only)."""
    return _lib.mk_device_supported(int(major), int(minor), int(bool(cooperative_launch)),
                                    int(smem_optin_bytes), int(bool(batched)))


def _check(status: int, what: str):
    if status != MK_OK:
        raise MkError(status, what)


def header_functions() -> list[str]:
    """Names of the functions include/mk.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z_]+)\s*\(", text)))


def make_config(shape, max_seq: int, max_batch: int = 1, flags: int = 0,
                attn_chunks: int = 0, timeout_ns: int = 0, l2_lookahead_kb: int = 0,
                poll_ns: int = 0) -> Config:
    """`shape`: a workloads.ModelShape (or anything with the same fields)."""
    return Config(shape.layers, shape.hidden, shape.n_q_heads, shape.n_kv_heads,
                  shape.head_dim, shape.ffn, shape.vocab, int(max_seq), int(max_batch),
                  float(shape.rope_theta), float(shape.rms_eps), int(flags),
                  int(attn_chunks), int(timeout_ns), int(l2_lookahead_kb), int(poll_ns))


def plan(cfg: Config, num_sms: int) -> dict:
    """Host-only task-graph build (no GPU): tasks [n][8], queue, qoff,
    thresholds, per-task bytes."""
    info = Info()
    _check(_lib.mk_plan(C.byref(cfg), int(num_sms), C.byref(info), None, None, None, None, None),
           "mk_plan")
    n, e = info.num_tasks, info.num_events
    tasks = np.zeros((n, 8), np.int32)
    queue = np.zeros(n, np.int32)
    qoff = np.zeros(num_sms + 1, np.int32)
    thr = np.zeros(e, np.uint32)
    nbytes = np.zeros(n, np.int64)
    _check(_lib.mk_plan(C.byref(cfg), int(num_sms), C.byref(info), tasks.ctypes.data,
                        queue.ctypes.data, qoff.ctypes.data, thr.ctypes.data, nbytes.ctypes.data),
           "mk_plan")
    return {"info": info, "tasks": tasks, "queue": queue, "qoff": qoff, "thresholds": thr,
            "bytes": nbytes}


def _ptr(t) -> int:
    return int(t.data_ptr())


def decode_step_static(cfg: Config, packed: dict, kcache, vcache, tokens, positions, next_tok,
                       logits=None, status=None, stream=None, batch=None) -> int:
    """mk_decode_step_static: one step without a context and without any
    allocation.  `packed`: dict of CUDA tensors embed, lm_head, final_norm and
    per-layer lists attn_norm, mlp_norm, qkv, wo, gu, wd (qkv and gu in the
    packed tile order documented in mk.h).  Returns the status code."""
    L = len(packed["qkv"])
    keep = []

    def arr(ts):
        a = (C.c_void_p * L)(*[_ptr(t) for t in ts])
        keep.append(a)
        return C.cast(a, _VPP)

    w = PackedWeights(_ptr(packed["embed"]), _ptr(packed["lm_head"]), _ptr(packed["final_norm"]),
                      arr(packed["attn_norm"]), arr(packed["mlp_norm"]), arr(packed["qkv"]),
                      arr(packed["wo"]), arr(packed["gu"]), arr(packed["wd"]))
    kv = KV(arr(kcache), arr(vcache))
    b = int(tokens.numel()) if batch is None else int(batch)
    return _lib.mk_decode_step_static(C.byref(cfg), C.byref(w), C.byref(kv), _ptr(tokens),
                                      _ptr(positions), b,
                                      _ptr(logits) if logits is not None else None,
                                      _ptr(next_tok), _ptr(status) if status is not None else None,
                                      _stream_ptr(stream))


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) or None


class Context:
    """Owns one mk_ctx.  `weights`: workloads.ModelWeights on the GPU;
    `kcache`/`vcache`: per-layer bf16 CUDA tensors [max_batch][nkv][max_seq][d]."""

    def __init__(self, weights, kcache, vcache, max_seq: int, max_batch: int = 1,
                 flags: int = 0, attn_chunks: int = 0, timeout_ns: int = 0,
                 l2_lookahead_kb: int = 0, poll_ns: int = 0):
        shape = weights.shape
        self.cfg = make_config(shape, max_seq, max_batch, flags, attn_chunks, timeout_ns,
                               l2_lookahead_kb, poll_ns)
        L = shape.layers
        self._keep = [weights, kcache, vcache]

        def arr(ts):
            a = (C.c_void_p * L)(*[_ptr(t) for t in ts])
            self._keep.append(a)
            return C.cast(a, _VPP)

        self._w = Weights(_ptr(weights.embed), _ptr(weights.lm_head), _ptr(weights.final_norm),
                          arr(weights.attn_norm), arr(weights.mlp_norm), arr(weights.wq),
                          arr(weights.wk), arr(weights.wv), arr(weights.wo), arr(weights.wg),
                          arr(weights.wu), arr(weights.wd))
        self._kv = KV(arr(kcache), arr(vcache))
        h = C.c_void_p()
        _check(_lib.mk_create(C.byref(self.cfg), C.byref(self._w), C.byref(self._kv), C.byref(h)),
               "mk_create")
        self._h = h

    # -- stepping -------------------------------------------------------------
    def decode_step(self, tokens, positions, next_tok, logits=None, stream=None, batch=None):
        """Enqueue one step.  tokens/positions/next_tok: int32 CUDA tensors;
        logits: float32 CUDA tensor [batch][vocab] or None."""
        b = int(tokens.numel()) if batch is None else int(batch)
        st = _lib.mk_decode_step(self._h, _ptr(tokens), _ptr(positions), b,
                                 _ptr(logits) if logits is not None else None,
                                 _ptr(next_tok), _stream_ptr(stream))
        _check(st, "mk_decode_step")

    def decode_step_status(self, tokens, positions, next_tok, logits=None, stream=None,
                           batch=None) -> int:
        b = int(tokens.numel()) if batch is None else int(batch)
        return _lib.mk_decode_step(self._h, _ptr(tokens), _ptr(positions), b,
                                   _ptr(logits) if logits is not None else None,
                                   _ptr(next_tok), _stream_ptr(stream))

    def generate(self, tokens, positions, n_steps: int, tokens_out, next_tok, eos: int = -1,
                 stream=None, batch=None):
        """Enqueue a prompt plus greedy steps, `n_steps` in all, in one launch.
        tokens: int32 CUDA tensor [n_prompt][batch] (or [batch] for one
        token); positions: int32 CUDA tensor [batch] (first step's);
        tokens_out: int32 CUDA tensor [n_steps][batch]; next_tok: [batch]."""
        b = int(positions.numel()) if batch is None else int(batch)
        n_prompt = int(tokens.numel()) // b
        st = _lib.mk_generate(self._h, _ptr(tokens), n_prompt, _ptr(positions), b, int(n_steps),
                              int(eos), _ptr(tokens_out), _ptr(next_tok), _stream_ptr(stream))
        _check(st, "mk_generate")

    def prefill(self, tokens, next_tok, logits=None, slot: int = 0, start_pos: int = 0, stream=None,
                n_tokens=None):
        """Enqueue a prompt as one launch (batched contexts): tokens int32 CUDA
        tensor [n] at positions start_pos.., KV slot `slot`; next_tok int32
        [1] and logits float32 [vocab] (or None) receive the last token's."""
        n = int(tokens.numel()) if n_tokens is None else int(n_tokens)
        st = _lib.mk_prefill(self._h, _ptr(tokens), n, int(slot), int(start_pos),
                             _ptr(logits) if logits is not None else None, _ptr(next_tok),
                             _stream_ptr(stream))
        _check(st, "mk_prefill")

    def sync(self, stream=None) -> int:
        return _lib.mk_sync(self._h, _stream_ptr(stream))

    def reset(self):
        _check(_lib.mk_reset(self._h), "mk_reset")

    def close(self):
        if getattr(self, "_h", None):
            _lib.mk_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- introspection ----------------------------------------------------------
    def info(self) -> Info:
        i = Info()
        _check(_lib.mk_get_info(self._h, C.byref(i)), "mk_get_info")
        return i

    def event_counts(self) -> tuple[np.ndarray, np.ndarray]:
        n = self.info().num_events
        c = np.zeros(n, np.uint32)
        t = np.zeros(n, np.uint32)
        _check(_lib.mk_get_event_counts(self._h, c.ctypes.data, t.ctypes.data, n),
               "mk_get_event_counts")
        return c, t

    def read_buffer(self, which: int, count: int) -> np.ndarray:
        out = np.zeros(count, np.float32)
        _check(_lib.mk_read_buffer(self._h, int(which), out.ctypes.data, count), "mk_read_buffer")
        return out

    def trace(self) -> np.ndarray:
        n = self.info().num_tasks
        recs = (TraceRec * n)()
        _check(_lib.mk_get_trace(self._h, C.cast(recs, C.c_void_p), n), "mk_get_trace")
        dt = np.dtype([("t_ready", np.uint64), ("t_start", np.uint64), ("t_input", np.uint64),
                       ("t_done", np.uint64), ("t_end", np.uint64), ("t_wait", np.uint64),
                       ("sm", np.int32), ("kind", np.int32), ("layer", np.int32),
                       ("trig_event", np.int32)])
        return np.frombuffer(bytes(recs), dtype=dt).copy()

    STAT_NAMES = ["loader_empty_ns", "loader_pages", "loader_total_ns", "worker_full_ns",
                  "worker_ready_ns", "worker_sync_ns", "worker_total_ns", "sched_dep_ns",
                  "worker_prologue_ns", "worker_dot_ns", "worker_epi_ns", "worker_end_ns",
                  "worker_tasks", "worker_attn_tail_ns", "cols_first_page_ns", "cols_dot_ns"]

    def sm_stats(self) -> np.ndarray:
        """Per-SM wait accounting of the last step (trace mode): [num_sms][16]."""
        n = self.info().num_sms
        out = np.zeros((n, 16), np.uint64)
        _check(_lib.mk_get_sm_stats(self._h, out.ctypes.data, n * 16), "mk_get_sm_stats")
        return out

    def graph(self) -> dict:
        i = self.info()
        tasks = np.zeros((i.num_tasks, 8), np.int32)
        queue = np.zeros(i.num_tasks, np.int32)
        qoff = np.zeros(i.num_sms + 1, np.int32)
        _check(_lib.mk_get_graph(self._h, tasks.ctypes.data, queue.ctypes.data, qoff.ctypes.data),
               "mk_get_graph")
        return {"tasks": tasks, "queue": queue, "qoff": qoff}

    def debug_set_threshold(self, event: int, value: int):
        _check(_lib.mk_debug_set_threshold(self._h, int(event), int(value)),
               "mk_debug_set_threshold")

    def debug_withhold_event(self, event: int):
        _check(_lib.mk_debug_withhold_event(self._h, int(event)), "mk_debug_withhold_event")
