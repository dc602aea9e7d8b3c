"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a library routine, a closed form, an invariant
or an independent formulation, chosen so that a plausible slip (a dropped term, a sign,
a transposed operand, an off-by-one position, a wrong head mapping) fails.
"""
import dataclasses
import os

import numpy as np
import pytest
import scipy.special
import torch

from bandwidth_bound_stream_b200 import synth
from oracle import oracle as orc

FP16, BF16 = 0, 1
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- storage types

def test_fp16_values_match_numpy_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    got = orc.value(bits, FP16)
    want = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def test_bf16_values_match_torch_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    got = orc.value(bits, BF16)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    ok = ~np.isnan(want)
    assert np.array_equal(np.isnan(got), ~ok)
    assert np.array_equal(got[ok], want[ok])


def test_store_fp16_matches_numpy_rounding():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 1e-5, 2000), rng.normal(0, 2e4, 1000),
                        rng.normal(0, 1e-7, 1000), [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, 2.0**-24, 2.0**-25,
                                                    3 * 2.0**-26, 1 + 2.0**-11, 1 + 3 * 2.0**-11]])
    want = v.astype(np.float32).astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.store(v, FP16), want)


def test_store_bf16_matches_torch_rounding():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 1e-30, 500), [0.0, 1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8]])
    want = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.store(v, BF16), want)


# ---------------------------------------------------------------- building blocks

def test_matvec_matches_numpy_matmul_and_orientation():
    rng = np.random.default_rng(2)
    W = synth.normal_u16(5, 0x333, 37 * 131, FP16).reshape(37, 131)
    x = rng.normal(size=131)
    want = W.view(np.float16).astype(np.float64) @ x
    got = orc.matvec(W, FP16, x)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-15)
    # a transposed operand would not even have the right length
    assert got.shape == (37,)


def test_rmsnorm_closed_forms():
    g = synth.gain_u16(64, BF16)
    x = np.full(64, 3.0)
    np.testing.assert_allclose(orc.rmsnorm(x, g, BF16, 1e-5), 3.0 / np.sqrt(9.0 + 1e-5), rtol=1e-15)
    rng = np.random.default_rng(3)
    x = rng.normal(0, 7, 256)
    y = orc.rmsnorm(x, synth.gain_u16(256, FP16), FP16, 0.0)
    assert abs(np.sqrt(np.mean(y * y)) - 1.0) < 1e-14
    # the gain multiplies element-wise (fp16 0x4000 = 2.0)
    g2 = synth.gain_u16(256, FP16)
    g2[7] = 0x4000
    y2 = orc.rmsnorm(x, g2, FP16, 0.0)
    assert y2[7] == pytest.approx(2 * y[7], rel=1e-15) and np.array_equal(np.delete(y2, 7), np.delete(y, 7))


def _rope_complex(v, pos, theta):
    """Rotate-half RoPE as complex multiplication: (v_i + i v_{i+D/2}) * exp(i pos theta^(-2i/D))."""
    D = v.size
    half = D // 2
    z = v[:half] + 1j * v[half:]
    ang = pos * theta ** (-2.0 * np.arange(half) / D)
    r = z * np.exp(1j * ang)
    return np.concatenate([r.real, r.imag])


def test_rope_equals_complex_rotation():
    rng = np.random.default_rng(4)
    for D, pos, theta in [(128, 0, 1e4), (128, 1, 1e4), (128, 4095, 5e5), (64, 17, 1e4), (2, 3, 1e4)]:
        v = rng.normal(size=D)
        np.testing.assert_allclose(orc.rope(v, pos, theta), _rope_complex(v, pos, theta), rtol=0, atol=1e-12)


def test_rope_invariants():
    rng = np.random.default_rng(5)
    q, k = rng.normal(size=128), rng.normal(size=128)
    assert np.array_equal(orc.rope(q, 0, 1e4), q)
    for p in (1, 100, 32000):
        assert np.linalg.norm(orc.rope(q, p, 1e4)) == pytest.approx(np.linalg.norm(q), rel=1e-13)
    # <R_p q, R_p' k> depends only on p - p'
    a = orc.rope(q, 1000, 1e4) @ orc.rope(k, 990, 1e4)
    b = orc.rope(q, 10, 1e4) @ orc.rope(k, 0, 1e4)
    assert a == pytest.approx(b, rel=1e-9)
    # D = 2 is a plane rotation by pos radians
    c, s = np.cos(3.0), np.sin(3.0)
    np.testing.assert_allclose(orc.rope(np.array([1.0, 0.0]), 3, 1e4), [c, s], atol=1e-15)


def _kv(rng, n, D, dtype):
    K = orc.store(rng.normal(0, 1, (n, D)), dtype)
    V = orc.store(rng.normal(0, 1, (n, D)), dtype)
    return K, V


def test_attention_single_key_returns_v_exactly():
    rng = np.random.default_rng(6)
    K, V = _kv(rng, 1, 128, FP16)
    out = orc.attention(rng.normal(size=128) * 10, K, V, FP16)
    assert np.array_equal(out, orc.value(V[0], FP16))


def test_attention_matches_scipy_softmax():
    rng = np.random.default_rng(7)
    for n, D, dt in [(5, 64, FP16), (300, 128, BF16)]:
        K, V = _kv(rng, n, D, dt)
        q = rng.normal(size=D)
        Kf, Vf = orc.value(K, dt), orc.value(V, dt)
        w = scipy.special.softmax(Kf @ q / np.sqrt(D))
        assert w.sum() == pytest.approx(1.0, abs=1e-12)
        np.testing.assert_allclose(orc.attention(q, K, V, dt), w @ Vf, rtol=1e-11, atol=1e-13)


def test_attention_weights_sum_to_one():
    # with every value row equal to 1 the output is the sum of the softmax weights, whatever
    # the scores (peaked, flat or spread over many positions)
    rng = np.random.default_rng(12)
    for n, D, dt, scale in [(1, 32, FP16, 1.0), (7, 64, BF16, 30.0), (513, 128, FP16, 0.1)]:
        K, _ = _kv(rng, n, D, dt)
        ones = orc.store(np.ones((n, D)), dt)
        out = orc.attention(rng.normal(size=D) * scale, K, ones, dt)
        np.testing.assert_allclose(out, np.ones(D), rtol=0, atol=1e-13)


def test_attention_uniform_scores_average_values():
    rng = np.random.default_rng(8)
    _, V = _kv(rng, 9, 64, FP16)
    K = np.tile(orc.store(rng.normal(size=64), FP16), (9, 1))
    out = orc.attention(rng.normal(size=64), K, V, FP16)
    np.testing.assert_allclose(out, orc.value(V, FP16).mean(axis=0), rtol=1e-13, atol=1e-15)


def test_silu_and_argmax():
    for z in (-20.0, -1.0, 0.0, 0.5, 3.0, 30.0):
        assert orc.silu(z) == pytest.approx(z * scipy.special.expit(z), rel=1e-14, abs=1e-300)
    assert orc.argmax(np.array([1.0, 5.0, 2.0, 5.0])) == 1
    assert orc.argmax(np.array([-3.0, -3.0])) == 0


# ---------------------------------------------------------------- the whole step

MINI = synth.ModelConfig("mini", 2, 128, 4, 2, 32, 192, 97, FP16, rope_theta=1e4)


def _weights(cfg, seed=0):
    return synth.model_weights(cfg, seed)


def test_incremental_decode_equals_full_recompute():
    for cfg in (MINI, dataclasses.replace(MINI, dtype=BF16, n_kv_heads=4, rope_theta=5e5)):
        w = _weights(cfg)
        toks = synth.prompt(cfg, 13)
        m = orc.OracleModel(cfg, w, max_ctx=16)
        inc = np.stack([m.step(t) for t in toks])
        full = orc.OracleModel(cfg, w, max_ctx=16).forward_sequence(toks)
        np.testing.assert_allclose(inc, full, rtol=0, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv_heads():
    cfg = MINI
    w = _weights(cfg)
    mha_cfg = dataclasses.replace(cfg, n_kv_heads=cfg.n_heads)
    rep = cfg.n_heads // cfg.n_kv_heads
    w_mha = {k: v for k, v in w.items() if k != "layers"}
    w_mha["layers"] = []
    D = cfg.head_dim
    for L in w["layers"]:
        L2 = dict(L)
        for name in ("wk", "wv"):
            heads = L[name].reshape(cfg.n_kv_heads, D, cfg.d_model)
            L2[name] = np.repeat(heads, rep, axis=0).reshape(cfg.n_heads * D, cfg.d_model)
        w_mha["layers"].append(L2)
    toks = synth.prompt(cfg, 6)
    a = orc.OracleModel(cfg, w, 8)
    b = orc.OracleModel(mha_cfg, w_mha, 8)
    for t in toks:
        np.testing.assert_array_equal(a.step(t), b.step(t))


def _f(bits, dt):
    return orc.value(bits, dt)


def test_identity_blocks_reduce_to_embedding_times_head():
    """With Wo = 0 and Wd = 0 the residual stays E[tok]: logits = W_lm rmsnorm(E[tok])."""
    cfg = MINI
    w = _weights(cfg)
    for L in w["layers"]:
        L["wo"] = np.zeros_like(L["wo"])
        L["w_down"] = np.zeros_like(L["w_down"])
    m = orc.OracleModel(cfg, w, 4)
    tok = 11
    e = _f(w["tok_emb"][tok], cfg.dtype)
    h = e / np.sqrt(np.mean(e * e) + cfg.rms_eps)
    want = _f(w["lm_head"], cfg.dtype) @ h
    np.testing.assert_allclose(m.step(tok), want, rtol=1e-12, atol=1e-14)


def test_first_position_value_path_and_cache_write():
    """One layer at position 0: attention returns the stored v, so x = E + Wo v (+ MLP)."""
    cfg = dataclasses.replace(MINI, n_layers=1)
    w = _weights(cfg)
    L = w["layers"][0]
    L["w_down"] = np.zeros_like(L["w_down"])
    m = orc.OracleModel(cfg, w, 4)
    tok, pos = 5, 0
    dt, D = cfg.dtype, cfg.head_dim
    e = _f(w["tok_emb"][tok], dt)
    h = e / np.sqrt(np.mean(e * e) + cfg.rms_eps)
    k = _f(L["wk"], dt) @ h
    v = _f(L["wv"], dt) @ h
    v_st = v.astype(np.float32).astype(np.float16)
    k_st = np.concatenate([_rope_complex(k[g * D:(g + 1) * D], pos, cfg.rope_theta)
                           for g in range(cfg.n_kv_heads)]).astype(np.float32).astype(np.float16)
    o = np.concatenate([v_st[(hh * cfg.n_kv_heads // cfg.n_heads) * D:][:D].astype(np.float64)
                        for hh in range(cfg.n_heads)])
    x = e + _f(L["wo"], dt) @ o
    hf = x / np.sqrt(np.mean(x * x) + cfg.rms_eps)
    want = _f(w["lm_head"], dt) @ hf
    got = m.step(tok, pos)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-13)
    assert np.array_equal(m.k_cache[0, :, pos].ravel(), k_st.view(np.uint16))
    assert np.array_equal(m.v_cache[0, :, pos].ravel(), v_st.view(np.uint16))


def test_cache_append_at_later_position_uses_that_position():
    """Layer-0 K at position p depends on token p only: rotated by p, stored rounded."""
    cfg = MINI
    w = _weights(cfg)
    m = orc.OracleModel(cfg, w, 8)
    toks = synth.prompt(cfg, 5)
    for t in toks:
        m.step(t, want_logits=False)
    p = 4
    e = _f(w["tok_emb"][toks[p]], cfg.dtype)
    h = e / np.sqrt(np.mean(e * e) + cfg.rms_eps)
    k = _f(w["layers"][0]["wk"], cfg.dtype) @ h
    D = cfg.head_dim
    k_rot = np.concatenate([_rope_complex(k[g * D:(g + 1) * D], p, cfg.rope_theta) for g in range(cfg.n_kv_heads)])
    assert np.array_equal(m.k_cache[0, :, p].ravel(), k_rot.astype(np.float32).astype(np.float16).view(np.uint16))


def _torch_values(bits, dt):
    """Stored fp16/bf16 bits -> float64 tensor, decoded by numpy / torch (not by the oracle)."""
    if dt == FP16:
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.float16).astype(np.float64))
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(torch.float64)


def _torch_bits(values, dt):
    """float64 array -> storage bits (fp32 first, then round to nearest even), by numpy / torch."""
    f32 = np.asarray(values, dtype=np.float64).astype(np.float32)
    if dt == FP16:
        return f32.astype(np.float16).view(np.uint16)
    return torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_whole_network_matches_torch_library_formulation():
    """Every decode step of the chain against the same network written over the whole sequence
    with torch library routines: F.rms_norm, rotation as complex multiplication, causal
    scaled_dot_product_attention on kv heads repeated per query group, F.silu. Random norm gains
    and a scaled-up Wq/Wk (peaked attention) pin the wiring that the building-block pins leave
    open: which gain goes where, gate vs up, the query's rotation at later positions, the score
    scale and the kv-head map."""
    import torch.nn.functional as F
    rng = np.random.default_rng(21)
    for cfg in (MINI, dataclasses.replace(MINI, dtype=BF16, n_heads=6, n_kv_heads=2, head_dim=16, rope_theta=5e5)):
        dt, d, Hq, Hkv, D = cfg.dtype, cfg.d_model, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
        w = _weights(cfg)
        for L in w["layers"]:
            for name in ("wq", "wk"):
                L[name] = _torch_bits(8.0 * _torch_values(L[name], dt).numpy(), dt)
            for name in ("attn_norm", "mlp_norm"):
                L[name] = _torch_bits(rng.uniform(0.5, 1.5, d), dt)
        w["final_norm"] = _torch_bits(rng.uniform(0.5, 1.5, d), dt)
        toks = synth.prompt(cfg, 9)
        n = len(toks)

        store = torch.float16 if dt == FP16 else torch.bfloat16
        half = D // 2
        ang = torch.arange(n, dtype=torch.float64)[:, None] * cfg.rope_theta ** (
            -2.0 * torch.arange(half, dtype=torch.float64) / D)
        turn = torch.polar(torch.ones_like(ang), ang)[:, None, :]  # [position, 1, D/2]

        def rotate(t):  # [position, head, D]: the pair (i, i + D/2) as one complex number
            z = torch.complex(t[..., :half], t[..., half:]) * turn
            return torch.cat([z.real, z.imag], dim=-1)

        def val(bits):
            return _torch_values(bits, dt)

        x = val(w["tok_emb"])[torch.from_numpy(toks.astype(np.int64))]
        for L in w["layers"]:
            h = F.rms_norm(x, (d,), weight=val(L["attn_norm"]), eps=cfg.rms_eps)
            q = rotate((h @ val(L["wq"]).T).view(n, Hq, D))
            k = rotate((h @ val(L["wk"]).T).view(n, Hkv, D)).to(torch.float32).to(store).to(torch.float64)
            v = (h @ val(L["wv"]).T).view(n, Hkv, D).to(torch.float32).to(store).to(torch.float64)
            rep = Hq // Hkv
            o = F.scaled_dot_product_attention(q.transpose(0, 1), k.repeat_interleave(rep, 1).transpose(0, 1),
                                               v.repeat_interleave(rep, 1).transpose(0, 1), is_causal=True)
            x = x + o.transpose(0, 1).reshape(n, Hq * D) @ val(L["wo"]).T
            h = F.rms_norm(x, (d,), weight=val(L["mlp_norm"]), eps=cfg.rms_eps)
            x = x + (F.silu(h @ val(L["w_gate"]).T) * (h @ val(L["w_up"]).T)) @ val(L["w_down"]).T
        want = (F.rms_norm(x, (d,), weight=val(w["final_norm"]), eps=cfg.rms_eps) @ val(w["lm_head"]).T).numpy()

        m = orc.OracleModel(cfg, w, n)
        got = np.stack([m.step(t) for t in toks])
        assert np.abs(want).max() > 0.1  # logits of a visible size
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-10)


def test_bad_arguments_rejected():
    m = orc.OracleModel(MINI, _weights(MINI), 2)
    with pytest.raises(ValueError):
        m.step(MINI.vocab)
    with pytest.raises(ValueError):
        m.step(1, pos=2)


def test_logit_scale_of_synthetic_model():
    """N(0, 0.02) weights give logits of std ~0.02*sqrt(d) after the final unit-RMS norm."""
    cfg = synth.TINY
    m = orc.OracleModel(cfg, _weights(cfg), 4)
    lg = m.step(int(synth.prompt(cfg, 1)[0]))
    assert 0.5 * 0.02 * np.sqrt(cfg.d_model) < lg.std() < 2.0 * 0.02 * np.sqrt(cfg.d_model)


# ------------------------------------------------------------------ sampling (the variant beside argmax)

def test_splitmix64_and_draw_match_the_published_vector():
    """The oracle's own splitmix64 reproduces the published first five outputs from state
    1234567, and a step's draw is the top 24 bits of output pos + 1 over 2^24."""
    want = [int(l) for l in open(os.path.join(GOLDEN, "splitmix64_1234567.txt")) if not l.startswith("#")]
    assert [orc.splitmix64(1234567, n) for n in range(1, 6)] == want
    for pos, w in enumerate(want):
        assert orc.uniform(1234567, pos) == (w >> 40) / 2.0 ** 24


def test_sample_top1_is_argmax_for_any_temperature_and_draw():
    rng = np.random.default_rng(5)
    for _ in range(50):
        z = rng.normal(size=37)
        for T, u in ((0.1, 0.0), (1.0, 0.5), (7.0, 0.999)):
            tok, m = orc.sample(z, T, 1, u)
            assert tok == int(np.argmax(z)) and m == 1.0


def test_sample_two_candidates_closed_form():
    """Top-2 of (a, b, much smaller...): the first is chosen iff u < 1 / (1 + e^{(b - a) / T})."""
    a, b, T = 1.3, 0.4, 0.7
    z = np.array([-5.0, b, -9.0, a, -7.0])
    p_first = 1.0 / (1.0 + np.exp((b - a) / T))
    for u in np.linspace(0.0, 0.9999, 97):
        tok, m = orc.sample(z, T, 2, u)
        assert tok == (3 if u < p_first else 1)
        assert m == pytest.approx(abs(u - p_first), abs=1e-12)


def test_sample_frequencies_equal_the_tempered_top_k_softmax():
    """Draws spread evenly over [0, 1) pick each candidate with its probability, and never a
    token outside the top k: the temperature, the restriction and the order all enter."""
    rng = np.random.default_rng(9)
    z = rng.normal(size=64) * 2.0
    T, k, N = 0.7, 10, 20000
    top = np.argsort(-z, kind="stable")[:k]
    w = np.exp((z[top] - z[top[0]]) / T)
    p = w / w.sum()
    counts = np.zeros(64)
    for i in range(N):
        tok, _ = orc.sample(z, T, k, (i + 0.5) / N)
        counts[tok] += 1
    assert counts[np.setdiff1d(np.arange(64), top)].sum() == 0
    np.testing.assert_allclose(counts[top] / N, p, atol=1.5 / N)


def test_sample_order_breaks_ties_by_index():
    z = np.array([1.0, 5.0, 5.0, 0.0])
    assert orc.sample(z, 1.0, 2, 0.49)[0] == 1 and orc.sample(z, 1.0, 2, 0.51)[0] == 2
    # a draw exactly on a boundary (u * total = 1 = the first weight) goes to the next candidate:
    # the token is the first whose cumulative weight exceeds the draw
    assert orc.sample(z, 1.0, 2, 0.5) == (2, 0.0)
    # third candidate: weights 1, 1, e^-4, so it takes draws above 2 / (2 + e^-4) = 0.99093
    assert orc.sample(z, 1.0, 3, 0.995)[0] == 0 and orc.sample(z, 1.0, 3, 0.99)[0] == 2


def test_sample_rejects_bad_arguments_and_non_finite_candidates():
    z = np.array([0.5, 2.0, 1.0])
    assert orc.sample(z, 0.0, 2, 0.5)[0] == -1
    assert orc.sample(z, 1.0, 4, 0.5)[0] == -1
    assert orc.sample(z, 1.0, 2, 1.0)[0] == -1
    assert orc.sample(np.array([np.nan, 1.0, 0.0]), 1.0, 3, 0.2)[0] == -2
    assert orc.sample(np.array([np.inf, 1.0, 0.0]), 1.0, 2, 0.2)[0] == -2
    assert orc.sample(np.array([np.nan, 1.0, 0.0]), 1.0, 2, 0.2)[0] in (1, 2)  # NaN ranks below every number


# ------------------------------------------------------------------ FP8 (E4M3) weights

def test_e4m3_values_match_torch_for_every_pattern():
    want = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = orc.e4m3_value(np.arange(256))
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.array_equal(got[~np.isnan(got)], want[~np.isnan(want)])


def test_e4m3_encode_matches_torch_rounding_and_saturates():
    """Round to nearest, ties to the even code, against torch's conversion for values in range,
    including every exact midpoint between neighbouring codes (ties) and the subnormals; beyond
    the largest finite value (448) the encoding saturates (torch's conversion returns NaN past
    464, so that part is pinned by value)."""
    codes = np.arange(256, dtype=np.uint8)
    vals = orc.e4m3_value(codes)
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = (fin[:-1] + fin[1:]) / 2
    rng = np.random.default_rng(3)
    x = np.concatenate([fin, mids, rng.normal(size=5000) * 60, rng.normal(size=2000) * 0.01]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.e4m3_encode(x), want)
    assert list(orc.e4m3_encode([449.0, 463.9, 1e6, -1e6, float("inf")])) == [0x7E, 0x7E, 0x7E, 0xFE, 0x7E]
    assert orc.e4m3_encode([float("nan")])[0] == 0x7F


def test_quantize_rows_closed_forms():
    rng = np.random.default_rng(4)
    for dtype in (FP16, BF16):
        W = synth.normal_u16(77, 0x51, 24 * 96, dtype).reshape(24, 96)
        W[5] = 0  # an all-zero row
        q, s = orc.quantize_rows(W, dtype)
        w = orc.value(W, dtype)
        amax = np.abs(w).max(axis=1)
        want_s = np.where(amax > 0, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32), np.float32(1.0))
        assert np.array_equal(s, want_s)
        assert (q[5] == 0).all() and s[5] == 1.0
        deq = orc.e4m3_value(q) * s[:, None].astype(np.float64)
        # each code is the nearest to w / s: within half a code step of it (steps: 2^-9 below 2^-6)
        ratio = (w / s[:, None].astype(np.float64))
        e = np.floor(np.log2(np.maximum(np.abs(ratio), 2.0 ** -6)))
        half_step = 2.0 ** (e - 3) / 2
        assert (np.abs(orc.e4m3_value(q) - ratio) <= half_step * (1 + 1e-6) + 1e-12).all()
        # the largest element of each non-zero row encodes as +-448
        rows = np.arange(24)[amax > 0]
        top = np.abs(w[rows]).argmax(axis=1)
        assert (np.abs(orc.e4m3_value(q[rows, top])) == 448.0).all()
        assert np.isfinite(deq).all()
    del rng


def test_matvec_q8_matches_numpy():
    rng = np.random.default_rng(6)
    q = rng.integers(0, 256, size=(33, 70)).astype(np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x01  # no NaN codes
    s = rng.uniform(0.01, 2.0, 33).astype(np.float32)
    x = rng.normal(size=70)
    want = (orc.e4m3_value(q) * s[:, None].astype(np.float64)) @ x
    np.testing.assert_allclose(orc.matvec_q8(q, s, x), want, rtol=1e-13, atol=1e-13)


def test_fp8_step_equals_the_16bit_step_on_the_same_values():
    """A model whose 16-bit matrices equal value(code) * 2^k for E4M3 codes and power-of-two row
    scales 2^k (exact in fp16): the FP8 path (codes and scales) gives the same logits, bit for
    bit, at every step. A scale applied to the wrong rows, or a matrix taken from the wrong
    slot, would differ."""
    from oracle.oracle import OracleModel
    m = synth.TINY
    w = synth.model_weights(m)
    rng = np.random.default_rng(12)

    def on_grid(W):
        codes = orc.e4m3_encode(orc.value(W, m.dtype) * 50.0)
        codes[(codes & 0x7F) == 0x7F] = 0  # no NaN
        k = rng.integers(-3, 4, size=W.shape[0]).astype(np.float64)
        vals = orc.e4m3_value(codes) * np.exp2(k)[:, None] / 64.0
        return codes, (np.exp2(k) / 64.0).astype(np.float32), orc.store(vals, m.dtype)

    q8 = {"layers": [], "lm_head": None}
    w16 = {"tok_emb": w["tok_emb"], "final_norm": w["final_norm"], "layers": []}
    for layer in w["layers"]:
        ql, wl = {}, dict(layer)
        for name in orc.FP8_MATRICES:
            c, sc, bits = on_grid(layer[name])
            ql[name] = (c, sc)
            wl[name] = bits
        q8["layers"].append(ql)
        w16["layers"].append(wl)
    c, sc, bits = on_grid(w["lm_head"])
    q8["lm_head"] = (c, sc)
    w16["lm_head"] = bits
    a, b = OracleModel(m, w16, 16), OracleModel(m, w16, 16, q8=q8)
    prompt = synth.prompt(m, 6)
    for t in prompt:
        assert np.array_equal(a.step(int(t)), b.step(int(t)))
    # and the FP8 path reads the codes of every matrix: changing one matrix's codes (same 16-bit
    # weights) changes the logits (after a 6-token prompt: at position 0 the query and key
    # matrices cannot show, attention over one position returns its value)
    base = OracleModel(m, w16, 16, q8=q8).prefill(prompt)
    for where in [(0, n) for n in orc.FP8_MATRICES] + [("head", None)]:
        q = {"layers": [dict(l) for l in q8["layers"]], "lm_head": q8["lm_head"]}
        if where[0] == "head":
            c, sc = q["lm_head"]
            q["lm_head"] = (c ^ 1, sc)
        else:
            c, sc = q["layers"][0][where[1]]
            q["layers"][0][where[1]] = (c ^ 1, sc)
        assert not np.array_equal(OracleModel(m, w16, 16, q8=q).prefill(prompt), base), where
