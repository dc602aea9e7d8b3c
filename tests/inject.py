"""State-injected parity (test helper): the oracle continues from the engine's own KV cache.

At full size the oracle cannot afford to replay a 1,024- to 32,768-token prompt plus
hundreds of decode steps. Every decode step reads the whole KV cache, so the step at
position c is a function of (token, c, cache[0..c-1]) alone. The helper therefore copies
the engine's cache of a session into an OracleModel, runs the oracle's step at c from it,
and compares that step with the engine's: the logits (tests/parity.py tolerances), the
argmax (margin rule) and the K/V the step appends at c in every layer. The engine's own
K/V at c are then copied into the oracle as well, so each step starts from the same state
on both sides. Attention over the whole cache (every split, tile and merge of the kernels)
and every layer's arithmetic are checked at the context length the benchmark runs.
"""
from __future__ import annotations

import numpy as np

from tests.parity import compare_step

# K/V appended at a deep layer. The engine's residual stream is fp32 and the oracle's fp64;
# the tick kernel also feeds each contraction its activations as two 16-bit halves
# (hi + lo), which keep 22 significant bits for fp16 but only 16 for bf16 (per element,
# relative error up to 2^-16 ~ 1.5e-5). Over a 4,096-term dot product of N(0, 0.02) weights
# and up to 32 layers of residual accumulation, that reaches ~1e-4 absolute in the tail of
# the ~30,000 K/V values of one position (8B shape). Rounded to the storage type, the two
# sides land on the same or a neighbouring value (one step: fp16 2^-10, bf16 2^-7 relative
# to the value); near zero, where the step is tiny, the unrounded absolute difference bounds
# it instead: KV_ATOL, per storage type, with a margin of about 3x over that estimate.
# The deviation of the residual, and so of a deep layer's K/V, grows with the layers before
# it, each adding its own rounding: the absolute term scales with depth beyond 16 layers
# (kv_atol). The 48-layer bf16 tick model exceeded the flat 4e-4 by up to 4.3e-5 in one of
# three runs of the same launch (the tick kernel's k-split partial sums meet through fp32
# atomics, whose order varies from run to run).
KV_ATOL = {0: 1e-4, 1: 4e-4}


def kv_atol(dtype: int, n_layers: int) -> float:
    """The absolute term of the K/V comparison for a model of n_layers."""
    return KV_ATOL[dtype] * max(1.0, n_layers / 16.0)


def device_view(ptr: int, n: int):
    """A torch int16 tensor aliasing n elements of engine-owned device memory (read-only use)."""
    import torch

    class _Holder:
        __cuda_array_interface__ = {"shape": (n,), "typestr": "<i2", "data": (ptr, False), "version": 2}
    return torch.as_tensor(_Holder(), device="cuda")


def _views(eng, sid, model, max_ctx):
    kp, vp = eng.session_kv(sid)
    shape = (model.n_layers, model.n_kv_heads, max_ctx, model.head_dim)
    n = int(np.prod(shape))
    return device_view(kp, n).view(shape), device_view(vp, n).view(shape)


def copy_cache(eng, sid, model, max_ctx, orc, upto: int):
    """The engine's K/V of positions [0, upto) of session sid into the oracle's cache."""
    K, V = _views(eng, sid, model, max_ctx)
    orc.k_cache[:, :, :upto] = K[:, :, :upto].cpu().numpy().view(np.uint16)
    orc.v_cache[:, :, :upto] = V[:, :, :upto].cpu().numpy().view(np.uint16)


def cache_at(eng, sid, model, max_ctx, pos: int):
    """The engine's K and V of one position, [n_layers][n_kv_heads][head_dim] storage bits."""
    K, V = _views(eng, sid, model, max_ctx)
    return K[:, :, pos].cpu().numpy().view(np.uint16), V[:, :, pos].cpu().numpy().view(np.uint16)


def kv_mismatch(got_bits, want_bits, dtype, atol=None):
    """Largest |got - want| beyond one storage step at |want| plus atol (0.0 when within)."""
    from oracle import oracle as orc
    atol = KV_ATOL[dtype] if atol is None else atol
    got = orc.value(np.ravel(got_bits), dtype)
    want = orc.value(np.ravel(want_bits), dtype)
    frac = 10 if dtype == 0 else 7
    mag = np.maximum(np.abs(want), 2.0 ** -14)
    step = 2.0 ** (np.floor(np.log2(mag)) - frac)
    excess = np.abs(got - want) - (step * (1 + 1e-9) + atol)
    return float(max(0.0, excess.max()))


def check_position_kv(eng, sid, model, max_ctx, orc, pos: int, dtype: int):
    """The oracle's K/V at pos (just written by its step) against the engine's, every layer;
    then the oracle takes the engine's values at pos (same state for the next step)."""
    kg, vg = cache_at(eng, sid, model, max_ctx, pos)
    atol = kv_atol(dtype, model.n_layers)
    bad = max(kv_mismatch(kg, orc.k_cache[:, :, pos], dtype, atol), kv_mismatch(vg, orc.v_cache[:, :, pos], dtype, atol))
    assert bad == 0.0, f"K/V at position {pos} differ beyond one storage step + {atol:.3g}: excess {bad:.3g}"
    orc.k_cache[:, :, pos] = kg
    orc.v_cache[:, :, pos] = vg


def injected_decode_steps(eng, sid, model, max_ctx, orc, token: int, n_steps: int, logits_dev):
    """n_steps batch-1 decode steps with logits, each compared with the oracle's step from the
    engine's cache. Returns the step reports; the next input is the oracle's argmax."""
    reports = []
    ctx = eng.session_length(sid)
    copy_cache(eng, sid, model, max_ctx, orc, ctx)
    for _ in range(n_steps):
        out = eng.decode_step(sid, token, logits_dev.data_ptr())
        got = logits_dev.cpu().numpy()
        ref = orc.step(token, pos=ctx)
        reports.append(compare_step(got, out, ref, model.dtype))
        check_position_kv(eng, sid, model, max_ctx, orc, ctx, model.dtype)
        token = int(np.argmax(ref))
        ctx += 1
    return reports


def check_prompt_positions(eng, sid, model, max_ctx, orc, prompt, positions):
    """K/V the engine's prefill wrote at sampled prompt positions, every layer: the oracle
    recomputes the step at p from the engine's cache below p. Layer l > 0 at p depends on
    the attention of layers < l over positions 0..p, so this checks the prefill's attention
    over its whole range (every tile and chunk boundary before p)."""
    copy_cache(eng, sid, model, max_ctx, orc, max(positions) + 1)
    for p in positions:
        orc.step(int(prompt[p]), pos=p, want_logits=False)
        check_position_kv(eng, sid, model, max_ctx, orc, p, model.dtype)
