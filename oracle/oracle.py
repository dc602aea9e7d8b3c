"""ctypes wrapper around the CPU oracle (``oracle.c``). Test infrastructure only.

The oracle takes plain numpy arrays: weights as uint16 storage bits (fp16 or bf16) and
token ids as int32. It never imports the engine package.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

LAYER_TENSORS = ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "w_gate", "w_up", "w_down")


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim",
                                               "ffn", "vocab", "dtype")] + \
               [("rms_eps", ctypes.c_double), ("rope_theta", ctypes.c_double)]


class _Weights(ctypes.Structure):
    _fields_ = [("tok_emb", ctypes.c_void_p), ("final_norm", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("layers", ctypes.POINTER(ctypes.c_void_p)), ("q8", ctypes.POINTER(ctypes.c_void_p)),
                ("q8_scale", ctypes.POINTER(ctypes.c_void_p)), ("q8_head", ctypes.c_void_p),
                ("q8_head_scale", ctypes.c_void_p)]


def lib():
    if not hasattr(lib, "h"):
        h = ctypes.CDLL(_build.build())
        dp, vp, i32 = ctypes.POINTER(ctypes.c_double), ctypes.c_void_p, ctypes.c_int32
        h.orc_value.restype = ctypes.c_double
        h.orc_value.argtypes = [ctypes.c_uint16, i32]
        h.orc_store.restype = ctypes.c_uint16
        h.orc_store.argtypes = [ctypes.c_double, i32]
        h.orc_rmsnorm.argtypes = [i32, vp, vp, i32, ctypes.c_double, vp]
        h.orc_matvec.argtypes = [i32, i32, vp, i32, vp, vp]
        h.orc_rope.argtypes = [i32, i32, ctypes.c_double, vp]
        h.orc_attention.argtypes = [i32, i32, vp, vp, vp, i32, vp]
        h.orc_silu.restype = ctypes.c_double
        h.orc_silu.argtypes = [ctypes.c_double]
        h.orc_argmax.restype = i32
        h.orc_argmax.argtypes = [i32, vp]
        h.orc_step.restype = i32
        h.orc_step.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(_Weights), vp, vp, i32, i32, i32, vp]
        h.orc_forward_sequence.restype = i32
        h.orc_forward_sequence.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(_Weights), i32, vp, vp]
        h.orc_num_threads.restype = i32
        h.orc_splitmix64.restype = ctypes.c_uint64
        h.orc_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        h.orc_uniform.restype = ctypes.c_double
        h.orc_uniform.argtypes = [ctypes.c_uint64, i32]
        h.orc_sample.restype = i32
        h.orc_sample.argtypes = [i32, vp, ctypes.c_double, i32, ctypes.c_double, vp]
        h.orc_e4m3_value.restype = ctypes.c_double
        h.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        h.orc_e4m3_encode.restype = ctypes.c_uint8
        h.orc_e4m3_encode.argtypes = [ctypes.c_float]
        h.orc_quantize_rows.argtypes = [i32, i32, vp, i32, vp, vp]
        h.orc_matvec_q8.argtypes = [i32, i32, vp, vp, vp, vp]
        del dp
        lib.h = h
    return lib.h


def _ptr(a: np.ndarray):
    assert a.flags.c_contiguous
    return a.ctypes.data


# ---------------------------------------------------------------- building blocks

def value(bits, dtype: int) -> np.ndarray:
    b = np.atleast_1d(np.asarray(bits, dtype=np.uint16))
    return np.array([lib().orc_value(int(x), dtype) for x in b.ravel()]).reshape(b.shape)


def store(values, dtype: int) -> np.ndarray:
    v = np.atleast_1d(np.asarray(values, dtype=np.float64))
    return np.array([lib().orc_store(float(x), dtype) for x in v.ravel()], dtype=np.uint16).reshape(v.shape)


def rmsnorm(x: np.ndarray, g_bits: np.ndarray, dtype: int, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(g_bits, dtype=np.uint16)
    out = np.empty_like(x)
    lib().orc_rmsnorm(x.size, _ptr(x), _ptr(g), dtype, eps, _ptr(out))
    return out


def matvec(W_bits: np.ndarray, dtype: int, x: np.ndarray) -> np.ndarray:
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    x = np.ascontiguousarray(x, dtype=np.float64)
    N, K = W.shape
    y = np.empty(N)
    lib().orc_matvec(N, K, _ptr(W), dtype, _ptr(x), _ptr(y))
    return y


def rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    out = np.array(v, dtype=np.float64, copy=True)
    lib().orc_rope(out.size, pos, theta, _ptr(out))
    return out


def attention(q: np.ndarray, K_bits: np.ndarray, V_bits: np.ndarray, dtype: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    V = np.ascontiguousarray(V_bits, dtype=np.uint16)
    n, D = K.shape
    out = np.empty(D)
    lib().orc_attention(D, n, _ptr(q), _ptr(K), _ptr(V), dtype, _ptr(out))
    return out


def silu(z: float) -> float:
    return lib().orc_silu(z)


def argmax(v: np.ndarray) -> int:
    v = np.ascontiguousarray(v, dtype=np.float64)
    return int(lib().orc_argmax(v.size, _ptr(v)))


def splitmix64(seed: int, n: int) -> int:
    """Output n >= 1 of the splitmix64 generator started from state `seed`."""
    return int(lib().orc_splitmix64(seed & (2 ** 64 - 1), n))


def uniform(seed: int, pos: int) -> float:
    """The sampling draw of the decode step at position `pos`."""
    return float(lib().orc_uniform(seed & (2 ** 64 - 1), pos))


def sample(logits, temperature: float, top_k: int, u: float):
    """(token, margin) of temperature / top-k sampling with draw u (token -1: bad arguments,
    -2: a candidate's logit is not finite)."""
    v = np.ascontiguousarray(logits, dtype=np.float64)
    m = np.zeros(1)
    tok = int(lib().orc_sample(v.size, _ptr(v), float(temperature), int(top_k), float(u), _ptr(m)))
    return tok, float(m[0])


def e4m3_value(codes) -> np.ndarray:
    c = np.atleast_1d(np.asarray(codes, dtype=np.uint8))
    return np.array([lib().orc_e4m3_value(int(x)) for x in c.ravel()]).reshape(c.shape)


def e4m3_encode(values) -> np.ndarray:
    """fp32 values (given as any floats, converted to fp32 first) -> E4M3 codes."""
    v = np.atleast_1d(np.asarray(values, dtype=np.float32))
    return np.array([lib().orc_e4m3_encode(float(x)) for x in v.ravel()], dtype=np.uint8).reshape(v.shape)


def quantize_rows(W_bits: np.ndarray, dtype: int):
    """Per-row E4M3 quantisation of a 16-bit matrix: (codes [N][K] uint8, scales [N] fp32)."""
    W = np.ascontiguousarray(W_bits, dtype=np.uint16)
    N, K = W.shape
    q = np.empty((N, K), dtype=np.uint8)
    sc = np.empty(N, dtype=np.float32)
    lib().orc_quantize_rows(N, K, _ptr(W), dtype, _ptr(q), _ptr(sc))
    return q, sc


def matvec_q8(Q: np.ndarray, scale: np.ndarray, x: np.ndarray) -> np.ndarray:
    Q = np.ascontiguousarray(Q, dtype=np.uint8)
    sc = np.ascontiguousarray(scale, dtype=np.float32)
    x = np.ascontiguousarray(x, dtype=np.float64)
    N, K = Q.shape
    y = np.empty(N)
    lib().orc_matvec_q8(N, K, _ptr(Q), _ptr(sc), _ptr(x), _ptr(y))
    return y


FP8_MATRICES = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")


def quantize_model(cfg, weights: dict) -> dict:
    """The FP8 form of a model's weights: every matrix of every layer and the LM head quantised
    per row ({"layers": [{name: (codes, scales)}], "lm_head": (codes, scales)})."""
    return {"layers": [{n: quantize_rows(layer[n], cfg.dtype) for n in FP8_MATRICES} for layer in weights["layers"]],
            "lm_head": quantize_rows(weights["lm_head"], cfg.dtype)}


def num_threads() -> int:
    return int(lib().orc_num_threads())


# ---------------------------------------------------------------- the model

class OracleModel:
    """One session of the oracle: weights (uint16 numpy arrays) plus its own KV cache.

    ``cfg`` is any object with the shape attributes (n_layers, d_model, n_heads,
    n_kv_heads, head_dim, ffn, vocab, dtype, rms_eps, rope_theta). ``weights`` is
    {"tok_emb", "final_norm", "lm_head", "layers": [ {name: array} per layer ]}.
    """

    def __init__(self, cfg, weights: dict, max_ctx: int, q8: dict | None = None):
        """q8 (optional): the FP8 form of the weights (quantize_model); every matrix-vector
        product then uses the E4M3 codes times their row scales."""
        self.cfg = cfg
        self.max_ctx = max_ctx
        self._c = _Config(cfg.n_layers, cfg.d_model, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn,
                          cfg.vocab, cfg.dtype, cfg.rms_eps, cfg.rope_theta)
        self._keep = []
        ptrs = []
        for layer in weights["layers"]:
            for name in LAYER_TENSORS:
                a = np.ascontiguousarray(layer[name], dtype=np.uint16)
                self._keep.append(a)
                ptrs.append(_ptr(a))
        self._layer_ptrs = (ctypes.c_void_p * len(ptrs))(*ptrs)
        emb = np.ascontiguousarray(weights["tok_emb"], dtype=np.uint16)
        fin = np.ascontiguousarray(weights["final_norm"], dtype=np.uint16)
        head = np.ascontiguousarray(weights["lm_head"], dtype=np.uint16)
        self._keep += [emb, fin, head]
        self._w = _Weights(_ptr(emb), _ptr(fin), _ptr(head),
                           ctypes.cast(self._layer_ptrs, ctypes.POINTER(ctypes.c_void_p)))
        if q8 is not None:
            qp, sp = [], []
            for layer in q8["layers"]:
                for name in LAYER_TENSORS:
                    if name in layer:
                        qa = np.ascontiguousarray(layer[name][0], dtype=np.uint8)
                        sa = np.ascontiguousarray(layer[name][1], dtype=np.float32)
                        self._keep += [qa, sa]
                        qp.append(_ptr(qa))
                        sp.append(_ptr(sa))
                    else:
                        qp.append(None)
                        sp.append(None)
            self._q8_ptrs = (ctypes.c_void_p * len(qp))(*qp)
            self._q8_sc = (ctypes.c_void_p * len(sp))(*sp)
            hq = np.ascontiguousarray(q8["lm_head"][0], dtype=np.uint8)
            hs = np.ascontiguousarray(q8["lm_head"][1], dtype=np.float32)
            self._keep += [hq, hs]
            self._w.q8 = ctypes.cast(self._q8_ptrs, ctypes.POINTER(ctypes.c_void_p))
            self._w.q8_scale = ctypes.cast(self._q8_sc, ctypes.POINTER(ctypes.c_void_p))
            self._w.q8_head = _ptr(hq)
            self._w.q8_head_scale = _ptr(hs)
        shape = (cfg.n_layers, cfg.n_kv_heads, max_ctx, cfg.head_dim)
        self.k_cache = np.zeros(shape, dtype=np.uint16)
        self.v_cache = np.zeros(shape, dtype=np.uint16)
        self.pos = 0

    def step(self, token: int, pos: int | None = None, want_logits: bool = True):
        """One decode step at ``pos`` (default: the next position). Returns the fp64 logits (or None)."""
        if pos is None:
            pos = self.pos
        logits = np.empty(self.cfg.vocab) if want_logits else None
        r = lib().orc_step(ctypes.byref(self._c), ctypes.byref(self._w), _ptr(self.k_cache), _ptr(self.v_cache),
                           self.max_ctx, pos, int(token), _ptr(logits) if want_logits else None)
        if r == -1:
            raise ValueError("oracle step: bad position or token")
        self.pos = pos + 1
        return logits

    def prefill(self, tokens) -> np.ndarray:
        """Teacher-forced steps over a prompt; returns the logits after the last prompt token."""
        logits = None
        for j, t in enumerate(tokens):
            logits = self.step(int(t), want_logits=(j == len(tokens) - 1))
        return logits

    def forward_sequence(self, tokens) -> np.ndarray:
        """Full-sequence recompute (no carried cache): logits [n][vocab]."""
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        out = np.empty((toks.size, self.cfg.vocab))
        if lib().orc_forward_sequence(ctypes.byref(self._c), ctypes.byref(self._w), toks.size, _ptr(toks),
                                      _ptr(out)) != 0:
            raise ValueError("oracle forward_sequence: bad token")
        return out
