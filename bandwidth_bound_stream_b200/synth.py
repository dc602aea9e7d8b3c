"""Seeded synthetic inputs: model shapes, weights, prompts and tick-session lengths.

Only numbers are drawn here (no forward-pass arithmetic). The engine's harness and the
oracle's harness both take the bytes produced by this module, so both sides see the
same weights and tokens. The generator itself lives in ``csrc/synth.c``
(counter-based splitmix64 with Box-Muller normals).

Recipe (one per workload, all seeded):

* every matrix and the embedding table ~ N(0, 0.02), rounded to the storage dtype;
* RMSNorm gains = 1.0 (standard initialisation; N(0, 0.02) gains would shrink the
  activations ~50x per norm);
* prompt token j of session s = word j of stream ``PROMPT_STREAM + s`` mod vocab;
* tick session s starts from a prompt of 1000 + (word s of ``LENGTH_STREAM`` mod 501)
  tokens, i.e. uniform on [1000, 1500].
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

FP16, BF16 = 0, 1
WEIGHT_STD = 0.02
PROMPT_STREAM = 0x10000000
LENGTH_STREAM = 0x20000000
# per-layer tensor order used everywhere (engine ABI, oracle, generator)
LAYER_TENSORS = ("attn_norm", "wq", "wk", "wv", "wo", "mlp_norm", "w_gate", "w_up", "w_down")
_MATRIX_IDS = {"wq": 0, "wk": 1, "wv": 2, "wo": 3, "w_gate": 4, "w_up": 5, "w_down": 6}


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    dtype: int  # 0 = fp16, 1 = bf16
    rms_eps: float = 1e-5
    rope_theta: float = 1e4

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    def shape(self, tensor: str) -> tuple:
        d, q, kv, f = self.d_model, self.q_dim, self.kv_dim, self.ffn
        return {
            "attn_norm": (d,), "mlp_norm": (d,), "final_norm": (d,),
            "wq": (q, d), "wk": (kv, d), "wv": (kv, d), "wo": (d, q),
            "w_gate": (f, d), "w_up": (f, d), "w_down": (d, f),
            "tok_emb": (self.vocab, d), "lm_head": (self.vocab, d),
        }[tensor]

    def n_params(self) -> int:
        per_layer = sum(int(np.prod(self.shape(t))) for t in LAYER_TENSORS)
        return (self.n_layers * per_layer + int(np.prod(self.shape("tok_emb")))
                + int(np.prod(self.shape("lm_head"))) + self.d_model)

    def weight_bytes_per_token(self, fp8: bool = False) -> int:
        """Bytes one decode step must stream: every weight except the embedding table, plus one
        embedding row. With fp8, the matrices and the LM head stream as one-byte E4M3 codes plus
        a 4-byte scale per row; the norm gains and the embedding row stay 16-bit."""
        if not fp8:
            return 2 * (self.n_params() - self.vocab * self.d_model + self.d_model)
        d, q, kv, f, V, L = self.d_model, self.q_dim, self.kv_dim, self.ffn, self.vocab, self.n_layers
        elems = L * (q * d + 2 * kv * d + d * q + 2 * f * d + d * f) + V * d
        rows = L * (q + 2 * kv + d + 2 * f + d) + V
        return elems + 4 * rows + 2 * (2 * L + 1) * d + 2 * d

    def kv_bytes_per_position(self) -> int:
        """K and V bytes of one context position over all layers."""
        return self.n_layers * 2 * self.kv_dim * 2


# The workloads. Shapes follow the dense Llama-style decoder of the decode path.
TINY = ModelConfig("tiny", 2, 256, 4, 4, 64, 1024, 4096, FP16, rope_theta=1e4)
DENSE_1P9B = ModelConfig("dense-1.9b", 28, 2048, 16, 8, 128, 8192, 32000, FP16, rope_theta=1e4)
DENSE_8B = ModelConfig("dense-8b", 32, 4096, 32, 8, 128, 14336, 128256, BF16, rope_theta=5e5)
TICK_10P8B = ModelConfig("dense-10.8b", 48, 4096, 32, 8, 128, 14336, 32000, BF16, rope_theta=1e4)
# Test-only shapes: two layers of the 1.9B / 8B shapes (full-width tiles), and ragged ones.
SLICE_1P9B = dataclasses.replace(DENSE_1P9B, name="slice-1.9b", n_layers=2)
SLICE_8B = dataclasses.replace(DENSE_8B, name="slice-8b", n_layers=2)
SLICE_TICK = dataclasses.replace(TICK_10P8B, name="slice-10.8b", n_layers=2)
RAGGED = ModelConfig("ragged", 3, 384, 6, 2, 64, 1216, 5003, BF16, rope_theta=1e4)
# head_dim 32, 5 query heads per kv head, odd k-step counts (d = 320, F = 576), odd vocabulary
SMALL_HEAD = ModelConfig("small-head", 2, 320, 10, 2, 32, 576, 3001, FP16, rope_theta=1e4)
# head_dim 64 with 6 query heads per kv head: the tick's tensor-core attention takes two passes
# per unit (4 heads, then 2)
GQA6 = ModelConfig("gqa6", 2, 512, 12, 2, 64, 1024, 3001, BF16, rope_theta=1e4)
# 32 kv heads of 5 query heads: a 64-position prefill chunk has 64 x 32 x 2 attention passes,
# more than the tick kernel balances per step, and more than one stream of them per SM
WIDE_KV = ModelConfig("wide-kv", 2, 256, 160, 32, 64, 512, 1031, FP16, rope_theta=1e4)
CONFIGS = {c.name: c for c in (TINY, DENSE_1P9B, DENSE_8B, TICK_10P8B, SLICE_1P9B, SLICE_8B,
                                SLICE_TICK, RAGGED, SMALL_HEAD, GQA6, WIDE_KV)}


def _lib():
    if not hasattr(_lib, "h"):
        if not os.path.exists(_LIB_PATH):
            from . import build as _build
            _build.build_synth()
        h = ctypes.CDLL(_LIB_PATH)
        u64, i64, i32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32
        h.synth_word.restype = u64
        h.synth_word.argtypes = [u64, u64, u64]
        h.synth_stream_key.restype = u64
        h.synth_stream_key.argtypes = [u64, u64]
        h.synth_splitmix64_next.restype = u64
        h.synth_splitmix64_next.argtypes = [ctypes.POINTER(u64)]
        h.synth_normal_u16.restype = None
        h.synth_normal_u16.argtypes = [u64, u64, i64, i64, ctypes.c_double, i32, ctypes.c_void_p]
        h.synth_fill_u16.restype = None
        h.synth_fill_u16.argtypes = [i64, ctypes.c_uint16, ctypes.c_void_p]
        h.synth_tokens.restype = None
        h.synth_tokens.argtypes = [u64, u64, i64, i32, ctypes.c_void_p]
        h.synth_uniform_int.restype = i32
        h.synth_uniform_int.argtypes = [u64, u64, u64, i32, i32]
        h.synth_round_f32.restype = ctypes.c_uint16
        h.synth_round_f32.argtypes = [ctypes.c_float, i32]
        _lib.h = h
    return _lib.h


def word(seed: int, stream: int, i: int) -> int:
    return int(_lib().synth_word(seed, stream, i))


def splitmix64_sequence(state: int, n: int) -> list:
    s = ctypes.c_uint64(state)
    return [int(_lib().synth_splitmix64_next(ctypes.byref(s))) for _ in range(n)]


def stream_key(seed: int, stream: int) -> int:
    return int(_lib().synth_stream_key(seed, stream))


def tensor_stream(tensor: str, layer: int = -1) -> int:
    if tensor == "tok_emb":
        return 0x100
    if tensor == "lm_head":
        return 0x101
    return 0x102 + 7 * layer + _MATRIX_IDS[tensor]


def normal_u16(seed: int, stream: int, n: int, dtype: int, offset: int = 0, std: float = WEIGHT_STD,
               out: np.ndarray | None = None) -> np.ndarray:
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.size == n and out.flags.c_contiguous
    _lib().synth_normal_u16(seed, stream, offset, n, std, dtype, out.ctypes.data)
    return out


def gain_u16(n: int, dtype: int) -> np.ndarray:
    one = 0x3C00 if dtype == FP16 else 0x3F80
    return np.full(n, one, dtype=np.uint16)


def tensor(cfg: ModelConfig, name: str, layer: int = -1, seed: int = 0) -> np.ndarray:
    """One weight tensor as uint16 storage bits, in its natural row-major shape."""
    shape = cfg.shape(name)
    n = int(np.prod(shape))
    if name in ("attn_norm", "mlp_norm", "final_norm"):
        return gain_u16(n, cfg.dtype).reshape(shape)
    return normal_u16(seed, tensor_stream(name, layer), n, cfg.dtype).reshape(shape)


def iter_tensors(cfg: ModelConfig, seed: int = 0):
    """Yield (name, layer, array) for every tensor, one at a time (bounded host memory)."""
    yield "tok_emb", -1, tensor(cfg, "tok_emb", seed=seed)
    for layer in range(cfg.n_layers):
        for name in LAYER_TENSORS:
            yield name, layer, tensor(cfg, name, layer, seed)
    yield "final_norm", -1, tensor(cfg, "final_norm", seed=seed)
    yield "lm_head", -1, tensor(cfg, "lm_head", seed=seed)


def model_weights(cfg: ModelConfig, seed: int = 0) -> dict:
    """All tensors in host memory: {"tok_emb", "final_norm", "lm_head", "layers": [dict per layer]}."""
    w = {"layers": [dict() for _ in range(cfg.n_layers)]}
    for name, layer, arr in iter_tensors(cfg, seed):
        if layer >= 0:
            w["layers"][layer][name] = arr
        else:
            w[name] = arr
    return w


def prompt(cfg: ModelConfig, n: int, session: int = 0, seed: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _lib().synth_tokens(seed, PROMPT_STREAM + session, n, cfg.vocab, out.ctypes.data)
    return out


def tick_prompt_length(session: int, seed: int = 0, lo: int = 1000, hi: int = 1500) -> int:
    return int(_lib().synth_uniform_int(seed, LENGTH_STREAM, session, lo, hi))


def round_f32(value: float, dtype: int) -> int:
    return int(_lib().synth_round_f32(value, dtype))
