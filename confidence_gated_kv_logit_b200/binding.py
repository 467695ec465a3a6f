"""Thin ctypes binding of libconfkv.so (include/confkv.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity and passed as raw pointers together with the current CUDA stream;
every step of the decode path runs in the library's kernels. If the library
has not been built, every entry point raises instead of falling back to
anything else.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
# CONFKV_LIBRARY selects another build of the same library (e.g. the
# self-checking one); there is no non-CUDA implementation to fall back to.
LIB_PATH = os.environ.get("CONFKV_LIBRARY", os.path.join(HERE, "libconfkv.so"))

ALL_LAYERS = -1
MODE_CONF, MODE_FIXED = 0, 1
GATE_PROSE, GATE_LITERAL = 0, 1
COMPACT_HOLEFILL, COMPACT_STABLE, COMPACT_LINEAR = 0, 1, 2
SCORE_EMA, SCORE_ACCUM, SCORE_RANDOM = 0, 1, 2

STATUS = {0: "OK", 1: "ERR_ARG", 2: "ERR_CAPACITY", 3: "ERR_STATE", 4: "ERR_NONFINITE",
          5: "ERR_CUDA", 6: "ERR_OOM", 7: "ERR_DEVICE"}

EXPORTED = ["confkv_default_params", "confkv_create", "confkv_destroy", "confkv_prefill",
            "confkv_confidence", "confkv_decode_attn", "confkv_evict_compact", "confkv_query",
            "confkv_export_segment", "confkv_last_error", "confkv_last_error_detail",
            "confkv_profile_enable", "confkv_profile_read", "confkv_confidence_noalloc",
            "confkv_status_string", "confkv_version"]
KERNEL_KINDS = ["confidence", "append", "attention", "combine", "ema", "evict", "prefill", "ema_evict"]


class ConfKVError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_status_string(status)})")


class Params(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("n_low", ctypes.c_int32), ("n_high", ctypes.c_int32),
                ("tau", ctypes.c_float), ("alpha", ctypes.c_float), ("ema_decay", ctypes.c_float),
                ("protect_last", ctypes.c_int32), ("fp16_window", ctypes.c_int32),
                ("n_sink", ctypes.c_int32), ("fixed_budget", ctypes.c_int32),
                ("pyramidal", ctypes.c_int32), ("gate", ctypes.c_int32),
                ("int8_enable", ctypes.c_int32), ("compact", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("max_prefill", ctypes.c_int32),
                ("score_source", ctypes.c_int32), ("seed", ctypes.c_uint32), ("single_stream", ctypes.c_int32)]


class Stats(ctypes.Structure):
    _fields_ = [("tokens_int8", ctypes.c_int64), ("tokens_fp16", ctypes.c_int64),
                ("bytes_payload", ctypes.c_int64), ("bytes_meta", ctypes.c_int64),
                ("bytes_capacity", ctypes.c_int64), ("min_len", ctypes.c_int32),
                ("max_len", ctypes.c_int32), ("attn_tokens_int8", ctypes.c_int64),
                ("attn_tokens_fp16", ctypes.c_int64), ("evict_tokens", ctypes.c_int64),
                ("moved_rows", ctypes.c_int64), ("requant_rows", ctypes.c_int64),
                ("kernel_launches", ctypes.c_int64), ("evict_block_segments", ctypes.c_int64),
                ("moved_window_rows", ctypes.c_int64)]


class Profile(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int64 * 8), ("ms", ctypes.c_double * 8)]


_LIB = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libconfkv.so (raises if it has not been built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with confidence_gated_kv_logit_b200.build.build()")
    lib = ctypes.CDLL(path)
    P, I32, VP, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.POINTER(ctypes.c_float)
    lib.confkv_default_params.argtypes = [ctypes.POINTER(Params)]
    lib.confkv_create.argtypes = [I32, I32, I32, I32, ctypes.POINTER(Params), ctypes.POINTER(P)]
    lib.confkv_destroy.argtypes = [P]
    lib.confkv_prefill.argtypes = [P, I32, I32, ctypes.POINTER(ctypes.c_int32), I32, VP, VP, VP, VP]
    lib.confkv_confidence.argtypes = [P, VP, I32, I32, VP, VP, VP]
    lib.confkv_decode_attn.argtypes = [P, I32, VP, VP, VP, VP, VP, VP, VP]
    lib.confkv_evict_compact.argtypes = [P, I32, VP]
    lib.confkv_query.argtypes = [P, ctypes.POINTER(Stats)]
    lib.confkv_export_segment.argtypes = [P, I32, I32, I32, VP, ctypes.POINTER(ctypes.c_size_t)]
    lib.confkv_last_error.argtypes = [P, I32]
    lib.confkv_last_error_detail.argtypes = [P, ctypes.POINTER(ctypes.c_int32)]
    lib.confkv_confidence_noalloc.argtypes = [ctypes.POINTER(Params), I32, VP, I32, I32, VP, VP, VP]
    lib.confkv_profile_enable.argtypes = [P, I32]
    lib.confkv_profile_read.argtypes = [P, ctypes.POINTER(Profile), I32]
    lib.confkv_status_string.argtypes = [ctypes.c_int]
    lib.confkv_status_string.restype = ctypes.c_char_p
    lib.confkv_version.restype = ctypes.c_int32
    for name in EXPORTED:
        if name not in ("confkv_status_string", "confkv_version"):
            getattr(lib, name).restype = ctypes.c_int
    _LIB = lib
    return lib


def _status_string(st: int) -> str:
    try:
        return load_library().confkv_status_string(int(st)).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(st: int, what: str):
    if st != 0:
        raise ConfKVError(st, what)


def default_params() -> Params:
    p = Params()
    _check(load_library().confkv_default_params(ctypes.byref(p)), "confkv_default_params")
    return p


def _ptr(t, dtype, shape, name):
    import torch
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def confidence_noalloc(logits, layers: int, c_out, budget_out, stream=None, **params):
    """Confidence and per-layer budgets through confkv_confidence_noalloc: no
    handle and no device allocation inside the library (for callers that
    cannot allocate). Policy fields default as in confkv_default_params."""
    import torch
    B, V = logits.shape
    p = default_params()
    for k, v in params.items():
        if not hasattr(p, k):
            raise TypeError(f"unknown parameter {k}")
        setattr(p, k, v)
    lp = _ptr(logits, torch.float32, (B, V), "logits")
    cp = _ptr(c_out, torch.float32, (B,), "c_out")
    bp = _ptr(budget_out, torch.int32, (B, layers), "budget_out")
    _check(load_library().confkv_confidence_noalloc(ctypes.byref(p), layers, lp, B, V, cp, bp, _stream(stream)),
           "confkv_confidence_noalloc")


class ConfKV:
    """One cache handle: layers x max_batch x kv_heads segments on the current device."""

    def __init__(self, layers: int, kv_heads: int, q_heads: int, head_dim: int, **params):
        lib = load_library()
        self.L, self.Hkv, self.Hq, self.D = layers, kv_heads, q_heads, head_dim
        self.G = q_heads // kv_heads
        p = default_params()
        for k, v in params.items():
            if not hasattr(p, k):
                raise TypeError(f"unknown parameter {k}")
            setattr(p, k, v)
        self.params = p
        self.batch = 0
        self._h = ctypes.c_void_p()
        _check(lib.confkv_create(layers, kv_heads, q_heads, head_dim, ctypes.byref(p), ctypes.byref(self._h)),
               "confkv_create")

    # -- lifecycle -----------------------------------------------------------
    def close(self):
        if self._h:
            _check(load_library().confkv_destroy(self._h), "confkv_destroy")
            self._h = ctypes.c_void_p()

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    def _layers(self, layer):
        return self.L if layer == ALL_LAYERS else 1

    def _lead(self, layer):
        return (self.L, self.batch) if layer == ALL_LAYERS else (self.batch,)

    # -- the decode step -----------------------------------------------------
    def prefill(self, k, v, lens, layer: int = ALL_LAYERS, priority=None, stream=None):
        import torch
        lens = [int(x) for x in lens]
        B = len(lens)
        T = k.shape[-2]
        lead = (self.L, B) if layer == ALL_LAYERS else (B,)
        kp = _ptr(k, torch.float16, lead + (self.Hkv, T, self.D), "k")
        vp = _ptr(v, torch.float16, lead + (self.Hkv, T, self.D), "v")
        pp = _ptr(priority, torch.float32, lead + (self.Hkv, T), "priority")
        arr = (ctypes.c_int32 * B)(*lens)
        _check(load_library().confkv_prefill(self._h, layer, B, arr, T, kp, vp, pp, _stream(stream)),
               "confkv_prefill")
        self.batch = B

    def confidence(self, logits, c_out=None, budget_out=None, stream=None):
        import torch
        B, V = logits.shape
        lp = _ptr(logits, torch.float32, (B, V), "logits")
        cp = _ptr(c_out, torch.float32, (B,), "c_out")
        bp = _ptr(budget_out, torch.int32, (B, self.L), "budget_out")
        _check(load_library().confkv_confidence(self._h, lp, B, V, cp, bp, _stream(stream)), "confkv_confidence")

    def decode_attn(self, q, k_new, v_new, out, layer: int = ALL_LAYERS, prio_new=None, lse_out=None,
                    stream=None):
        import torch
        lead = self._lead(layer)
        qp = _ptr(q, torch.float16, lead + (self.Hq, self.D), "q")
        kp = _ptr(k_new, torch.float16, lead + (self.Hkv, self.D), "k_new")
        vp = _ptr(v_new, torch.float16, lead + (self.Hkv, self.D), "v_new")
        pp = _ptr(prio_new, torch.float32, lead + (self.Hkv,), "prio_new")
        op = _ptr(out, torch.float32, lead + (self.Hq, self.D), "out")
        lp = _ptr(lse_out, torch.float32, lead + (self.Hq,), "lse_out")
        _check(load_library().confkv_decode_attn(self._h, layer, qp, kp, vp, pp, op, lp, _stream(stream)),
               "confkv_decode_attn")

    def evict_compact(self, layer: int = ALL_LAYERS, stream=None):
        _check(load_library().confkv_evict_compact(self._h, layer, _stream(stream)), "confkv_evict_compact")

    # -- inspection ----------------------------------------------------------
    def query(self) -> dict:
        s = Stats()
        _check(load_library().confkv_query(self._h, ctypes.byref(s)), "confkv_query")
        return {name: getattr(s, name) for name, _ in Stats._fields_}

    def profile(self, enable: bool):
        _check(load_library().confkv_profile_enable(self._h, 1 if enable else 0), "confkv_profile_enable")

    def profile_read(self, reset: bool = True) -> dict:
        pr = Profile()
        _check(load_library().confkv_profile_read(self._h, ctypes.byref(pr), 1 if reset else 0), "confkv_profile_read")
        return {name: {"launches": int(pr.launches[i]), "ms": float(pr.ms[i])}
                for i, name in enumerate(KERNEL_KINDS)}

    def last_error(self, clear: bool = False) -> int:
        return int(load_library().confkv_last_error(self._h, 1 if clear else 0))

    def last_error_detail(self) -> tuple:
        d = (ctypes.c_int32 * 3)()
        st = int(load_library().confkv_last_error_detail(self._h, d))
        return st, int(d[0]), int(d[1]), int(d[2])

    def export_segment(self, layer: int, seq: int, kv_head: int) -> dict:
        """Raw state of one segment, as numpy arrays in physical order."""
        lib = load_library()
        n = ctypes.c_size_t(0)
        _check(lib.confkv_export_segment(self._h, layer, seq, kv_head, None, ctypes.byref(n)), "export size")
        buf = (ctypes.c_ubyte * n.value)()
        _check(lib.confkv_export_segment(self._h, layer, seq, kv_head, buf, ctypes.byref(n)), "export")
        raw = np.frombuffer(buf, dtype=np.uint8).copy()
        hdr = raw[:32].view(np.int32)
        n_cold, W, next_pos, cold_int8, D, mode = (int(x) for x in hdr[:6])
        o = 32

        def take(count, dtype, shape=None):
            nonlocal o
            nb = count * np.dtype(dtype).itemsize
            a = raw[o:o + nb].view(dtype)
            o += nb
            return a.reshape(shape) if shape else a

        out = {"n_cold": n_cold, "W": W, "next_pos": next_pos, "cold_int8": bool(cold_int8), "D": D,
               "mode": mode}
        out["pos_c"] = take(n_cold, np.int32)
        out["sc_c"] = take(n_cold, np.float32)
        out["ks"] = take(n_cold, np.float32)
        out["vs"] = take(n_cold, np.float32)
        cd = np.int8 if cold_int8 else np.float16
        out["k_c"] = take(n_cold * D, cd, (n_cold, D))
        out["v_c"] = take(n_cold * D, cd, (n_cold, D))
        out["pos_r"] = take(W, np.int32)
        out["sc_r"] = take(W, np.float32)
        out["k_r"] = take(W * D, np.float16, (W, D))
        out["v_r"] = take(W * D, np.float16, (W, D))
        return out


def logical_segment(ex: dict) -> dict:
    """Logical content of an exported segment: every token sorted by position,
    with its precision, payload rows, scales and EMA/priority."""
    D = ex["D"]
    live = ex["pos_r"] >= 0
    pos = np.concatenate([ex["pos_c"].astype(np.int64), ex["pos_r"][live].astype(np.int64)])
    n_c, n_r = ex["n_cold"], int(live.sum())
    is16 = np.concatenate([np.full(n_c, not ex["cold_int8"]), np.ones(n_r, bool)])
    k16 = np.zeros((n_c + n_r, D), np.float16)
    v16 = np.zeros((n_c + n_r, D), np.float16)
    k8 = np.zeros((n_c + n_r, D), np.int8)
    v8 = np.zeros((n_c + n_r, D), np.int8)
    ks = np.zeros(n_c + n_r, np.float32)
    vs = np.zeros(n_c + n_r, np.float32)
    if ex["cold_int8"]:
        k8[:n_c], v8[:n_c] = ex["k_c"], ex["v_c"]
        ks[:n_c], vs[:n_c] = ex["ks"], ex["vs"]
    else:
        k16[:n_c], v16[:n_c] = ex["k_c"], ex["v_c"]
    k16[n_c:], v16[n_c:] = ex["k_r"][live], ex["v_r"][live]
    sc = np.concatenate([ex["sc_c"], ex["sc_r"][live]])
    order = np.argsort(pos, kind="stable")
    return {"pos": pos[order], "is_fp16": is16[order], "k16": k16[order], "v16": v16[order],
            "k8": k8[order], "v8": v8[order], "ks": ks[order], "vs": vs[order],
            "score_src": sc[order], "next_pos": ex["next_pos"], "n_cold": n_c}
