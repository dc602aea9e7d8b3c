"""Python binding of ``libkie.so`` (declared in ``include/kie.h``).

Argument marshalling only: every step of the decode path runs in the library's CUDA
kernels. The functions keep the C names (``kie_create``, ``kie_prefill``, ...); the
``Engine`` class is a thin owner of one ``kie_engine*``. Importing this module loads the
library and raises if it is missing; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# KIE_VARIANT selects a diagnostic build of the same library ("debug": index checks on every
# kernel write and guard words around the engine's buffers; "profile": GEMV consumer timing in
# the phase trace); unset means the product build
VARIANT = os.environ.get("KIE_VARIANT", "")
if VARIANT not in ("", "debug", "profile"):
    raise ImportError(f"KIE_VARIANT={VARIANT!r}: expected unset, 'debug' or 'profile'")
LIB_PATH = os.path.join(_HERE, "libkie.so" if not VARIANT else f"libkie_{VARIANT}.so")

KIE_OK, KIE_ERR_ARG, KIE_ERR_CAPACITY, KIE_ERR_CUDA = 0, -1, -2, -3
KIE_ERR_TIMEOUT, KIE_ERR_STATE, KIE_ERR_DEVICE, KIE_ERR_UNSUPPORTED = -4, -5, -6, -7
KIE_FP16, KIE_BF16 = 0, 1
KIE_MODE_BATCH1, KIE_MODE_TICK = 1, 2

# every symbol include/kie.h declares
EXPORTS = ("kie_config_defaults", "kie_create", "kie_destroy", "kie_session_open", "kie_session_close",
           "kie_session_length", "kie_session_rewind", "kie_session_kv", "kie_prefill", "kie_decode_step",
           "kie_generate", "kie_decode_launch", "kie_sync", "kie_tick", "kie_last_error", "kie_status_string",
           "kie_flash_decode", "kie_flash_decode_scratch_bytes", "kie_trace_enable", "kie_trace_read",
           "kie_trace_events", "kie_flash_decode_noalloc", "kie_tick_launch", "kie_inject_fault",
           "kie_session_sampling", "kie_quantize_e4m3")
KIE_TOPK_MAX = 32
KIE_FAULT_NONE, KIE_FAULT_BARRIER_SHORT = 0, 1


class KieConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "ffn",
                                               "vocab")] + \
               [("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float)] + \
               [(n, ctypes.c_int32) for n in ("dtype", "max_sessions", "max_ctx", "timeout_ms", "idle_ms", "modes",
                                               "device", "weight_fp8", "b1_staging", "b1_kv_path")]


class KieWeights(ctypes.Structure):
    _fields_ = [("tok_emb", ctypes.c_void_p), ("layers", ctypes.POINTER(ctypes.c_void_p)),
                ("final_norm", ctypes.c_void_p), ("lm_head", ctypes.c_void_p)]


class KieSampling(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("top_k", ctypes.c_int32), ("seed", ctypes.c_uint64)]


class KieError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{msg} (status {status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} not built ({LIB_PATH}); run __graft_entry__.build()"
                          + (f" or build.build_kie(variant={VARIANT!r})" if VARIANT else ""))
    h = ctypes.CDLL(LIB_PATH)
    i32, vp, i64 = ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64
    P = ctypes.POINTER
    sig = {
        "kie_config_defaults": (None, [P(KieConfig)]),
        "kie_create": (i32, [P(KieConfig), P(KieWeights), P(vp)]),
        "kie_destroy": (None, [vp]),
        "kie_session_open": (i32, [vp, P(i32)]),
        "kie_session_close": (i32, [vp, i32]),
        "kie_session_length": (i32, [vp, i32, P(i32)]),
        "kie_session_rewind": (i32, [vp, i32, i32]),
        "kie_session_kv": (i32, [vp, i32, P(vp), P(vp)]),
        "kie_prefill": (i32, [vp, i32, vp, i32, P(i32)]),
        "kie_decode_step": (i32, [vp, i32, i32, P(i32), vp]),
        "kie_generate": (i32, [vp, i32, i32, i32, vp]),
        "kie_decode_launch": (i32, [vp, i32, vp, i32, vp, vp, vp]),
        "kie_sync": (i32, [vp]),
        "kie_tick": (i32, [vp, i32, vp, vp, i32, vp, vp]),
        "kie_last_error": (i32, [vp, ctypes.c_char_p, i32]),
        "kie_status_string": (ctypes.c_char_p, [i32]),
        "kie_flash_decode": (i32, [vp, vp, vp, i32, i32, i32, i32, i64, i32, vp, vp, i64, vp]),
        "kie_flash_decode_scratch_bytes": (i64, [i32, i32, i32, i32]),
        "kie_trace_enable": (i32, [vp, i32]),
        "kie_trace_read": (i32, [vp, vp, i64, P(i64)]),
        "kie_trace_events": (i32, [vp]),
        "kie_flash_decode_noalloc": (i32, [vp, vp, vp, i32, i32, i32, i32, i64, i32, vp, vp]),
        "kie_tick_launch": (i32, [vp, i32, vp, vp, i32, vp, vp, vp]),
        "kie_inject_fault": (i32, [vp, i32]),
        "kie_session_sampling": (i32, [vp, i32, P(KieSampling)]),
        "kie_quantize_e4m3": (i32, [vp, i64, i32, i32, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(h, name)
        f.restype = res
        f.argtypes = args
    return h


lib = _load()


def _ptr(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data


def config(model, max_sessions: int = 1, max_ctx: int = 4096, timeout_ms: int = 10000, idle_ms: int = 200,
           modes: int = KIE_MODE_BATCH1, device: int = 0, weight_fp8: bool = False,
           b1_staging: int = 0, b1_kv_path: int = 0) -> KieConfig:
    """A kie_config for a model shape (any object with the shape attributes of synth.ModelConfig).

    b1_staging: 0 streams the batch-1 kernel's weights through the shared-memory ring alone;
    1 also stages the first chunks after each layer's QKV rows in TMEM where the shape allows it
    (16-bit weights, d_model 2048 or 4096).
    b1_kv_path: 0 picks by max_ctx (the weight ring above 8192 positions), 1 reads the KV cache
    from L2, 2 streams it through the weight ring."""
    c = KieConfig()
    lib.kie_config_defaults(ctypes.byref(c))
    for f in ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "ffn", "vocab", "dtype"):
        setattr(c, f, getattr(model, f))
    c.rms_eps, c.rope_theta = model.rms_eps, model.rope_theta
    c.max_sessions, c.max_ctx, c.timeout_ms, c.idle_ms, c.modes, c.device = (max_sessions, max_ctx, timeout_ms,
                                                                                idle_ms, modes, device)
    c.weight_fp8 = 1 if weight_fp8 else 0
    c.b1_staging = b1_staging
    c.b1_kv_path = b1_kv_path
    return c


class Engine:
    """Owner of one kie_engine*. Methods raise KieError on a non-OK status."""

    def __init__(self, cfg: KieConfig, weights: KieWeights):
        self.h = ctypes.c_void_p()
        self.cfg = cfg
        self._check(lib.kie_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(self.h)), "kie_create")

    def _check(self, status: int, what: str):
        if status != KIE_OK:
            msg = lib.kie_status_string(status).decode()
            if self.h:
                buf = ctypes.create_string_buffer(512)
                lib.kie_last_error(self.h, buf, 512)
                msg += ": " + buf.value.decode()
            raise KieError(status, f"{what}: {msg}")

    def close(self):
        if self.h:
            lib.kie_destroy(self.h)
            self.h = ctypes.c_void_p()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def session_open(self) -> int:
        sid = ctypes.c_int32()
        self._check(lib.kie_session_open(self.h, ctypes.byref(sid)), "kie_session_open")
        return sid.value

    def session_close(self, sid: int):
        self._check(lib.kie_session_close(self.h, sid), "kie_session_close")

    def session_length(self, sid: int) -> int:
        n = ctypes.c_int32()
        self._check(lib.kie_session_length(self.h, sid, ctypes.byref(n)), "kie_session_length")
        return n.value

    def session_rewind(self, sid: int, ctx: int):
        self._check(lib.kie_session_rewind(self.h, sid, ctx), "kie_session_rewind")

    def session_sampling(self, sid: int, temperature: float = 1.0, top_k: int = 1, seed: int = 0, greedy: bool = False):
        """Temperature / top-k sampling for a session (greedy=True restores argmax decoding)."""
        if greedy:
            self._check(lib.kie_session_sampling(self.h, sid, None), "kie_session_sampling")
            return
        sp = KieSampling(float(temperature), int(top_k), int(seed) & (2 ** 64 - 1))
        self._check(lib.kie_session_sampling(self.h, sid, ctypes.byref(sp)), "kie_session_sampling")

    def session_kv(self, sid: int):
        k, v = ctypes.c_void_p(), ctypes.c_void_p()
        self._check(lib.kie_session_kv(self.h, sid, ctypes.byref(k), ctypes.byref(v)), "kie_session_kv")
        return k.value, v.value

    def prefill(self, sid: int, tokens) -> int:
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        first = ctypes.c_int32()
        self._check(lib.kie_prefill(self.h, sid, _ptr(t), t.size, ctypes.byref(first)), "kie_prefill")
        return first.value

    def decode_step(self, sid: int, token: int, logits_dev_ptr: int | None = None) -> int:
        out = ctypes.c_int32()
        self._check(lib.kie_decode_step(self.h, sid, int(token), ctypes.byref(out), logits_dev_ptr),
                    "kie_decode_step")
        return out.value

    def generate(self, sid: int, token: int, n: int, out: np.ndarray | None = None) -> np.ndarray:
        if out is None:
            out = np.empty(n, dtype=np.int32)
        self._check(lib.kie_generate(self.h, sid, int(token), n, _ptr(out)), "kie_generate")
        return out

    def decode_launch(self, sid: int, in_tok_dev_ptr: int, n: int, out_dev_ptr: int,
                      logits_dev_ptr: int | None = None, stream_ptr: int | None = None):
        self._check(lib.kie_decode_launch(self.h, sid, in_tok_dev_ptr, n, out_dev_ptr, logits_dev_ptr, stream_ptr),
                    "kie_decode_launch")

    def tick_launch(self, sids, in_tok_dev_ptr: int, steps: int, out_dev_ptr: int, logits_dev_ptr: int | None = None,
                    stream_ptr: int | None = None):
        s = np.ascontiguousarray(sids, dtype=np.int32)
        self._check(lib.kie_tick_launch(self.h, s.size, _ptr(s), in_tok_dev_ptr, steps, out_dev_ptr, logits_dev_ptr,
                                        stream_ptr), "kie_tick_launch")

    def trace_enable(self, tokens: int):
        self._check(lib.kie_trace_enable(self.h, tokens), "kie_trace_enable")

    def trace_read(self, tokens: int) -> np.ndarray:
        """Phase stamps as [cta][token][event] (uint64 ns; the last six events are ring wait totals)."""
        ev = lib.kie_trace_events(self.h)
        n = ctypes.c_int64()
        self._check(lib.kie_trace_read(self.h, None, 0, ctypes.byref(n)), "kie_trace_read")
        out = np.zeros(n.value, dtype=np.uint64)
        if n.value:
            self._check(lib.kie_trace_read(self.h, out.ctypes.data, n.value, ctypes.byref(n)), "kie_trace_read")
        return out.reshape(-1, tokens, ev)

    def inject_fault(self, fault: int):
        self._check(lib.kie_inject_fault(self.h, fault), "kie_inject_fault")

    def sync(self):
        self._check(lib.kie_sync(self.h), "kie_sync")

    def tick(self, sids, in_tokens, steps: int, logits_dev_ptr: int | None = None) -> np.ndarray:
        s = np.ascontiguousarray(sids, dtype=np.int32)
        t = np.ascontiguousarray(in_tokens, dtype=np.int32)
        out = np.empty((steps, s.size), dtype=np.int32)
        self._check(lib.kie_tick(self.h, s.size, _ptr(s), _ptr(t), steps, _ptr(out), logits_dev_ptr), "kie_tick")
        return out


def flash_decode(q_ptr, k_ptr, v_ptr, n_heads, n_kv_heads, head_dim, n_ctx, kv_stride, dtype, out_ptr,
                 scratch_ptr, scratch_bytes, stream_ptr=None) -> int:
    return lib.kie_flash_decode(q_ptr, k_ptr, v_ptr, n_heads, n_kv_heads, head_dim, n_ctx, kv_stride, dtype,
                                out_ptr, scratch_ptr, scratch_bytes, stream_ptr)


def flash_decode_noalloc(q_ptr, k_ptr, v_ptr, n_heads, n_kv_heads, head_dim, n_ctx, kv_stride, dtype, out_ptr,
                         stream_ptr=None) -> int:
    """kie_flash_decode with its scratch in the library's static device array (allocates nothing)."""
    return lib.kie_flash_decode_noalloc(q_ptr, k_ptr, v_ptr, n_heads, n_kv_heads, head_dim, n_ctx, kv_stride, dtype,
                                        out_ptr, stream_ptr)


FLASH_DECODE_NOALLOC_MAX_BYTES = 4 << 20


def quantize_e4m3(w_ptr, rows, cols, dtype, q_ptr, scale_ptr, stream_ptr=None) -> int:
    return lib.kie_quantize_e4m3(w_ptr, rows, cols, dtype, q_ptr, scale_ptr, stream_ptr)


def flash_decode_scratch_bytes(n_heads, n_kv_heads, head_dim, n_ctx) -> int:
    return int(lib.kie_flash_decode_scratch_bytes(n_heads, n_kv_heads, head_dim, n_ctx))


class DeviceWeights:
    """Seeded synthetic weights of a model shape, uploaded tensor by tensor to a CUDA device.

    Holds the torch tensors (keeping the device memory alive) and the kie_weights record.
    """

    def __init__(self, model, seed: int = 0, device: str = "cuda:0", host_copy: bool = False):
        import torch

        from . import synth
        self.tensors = {}
        self.host = {"layers": [dict() for _ in range(model.n_layers)]} if host_copy else None
        for name, layer, arr in synth.iter_tensors(model, seed):
            t = torch.from_numpy(arr.view(np.int16)).to(device)
            self.tensors[(name, layer)] = t
            if host_copy:
                if layer >= 0:
                    self.host["layers"][layer][name] = arr
                else:
                    self.host[name] = arr
        lp = [self.tensors[(n, l)].data_ptr() for l in range(model.n_layers) for n in synth.LAYER_TENSORS]
        self._layers = (ctypes.c_void_p * len(lp))(*lp)
        self.kie = KieWeights(self.tensors[("tok_emb", -1)].data_ptr(),
                              ctypes.cast(self._layers, ctypes.POINTER(ctypes.c_void_p)),
                              self.tensors[("final_norm", -1)].data_ptr(), self.tensors[("lm_head", -1)].data_ptr())

    def free(self):
        self.tensors.clear()
