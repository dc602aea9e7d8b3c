"""Parity of the batch-1 decode megakernel with the CPU oracle (GPU tests).

Every test runs the CUDA path through the C ABI (libkie.so via the ctypes binding) and
compares with the oracle on the same seeded inputs. Tolerances are those of
``tests/parity.py``: logits max-abs 2e-2 (fp16) / 5e-2 (bf16) at every step, token ids
exact wherever the oracle's top-1/top-2 margin exceeds 0.05 (teacher forcing keeps both
sides on the oracle's sequence).
"""
import dataclasses

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def kie():
    from bandwidth_bound_stream_b200 import build
    build.build_kie()
    from bandwidth_bound_stream_b200 import kie as k
    return k


def _setup(kie, model, max_ctx, seed=0, **kw):
    from oracle.oracle import OracleModel
    dw = kie.DeviceWeights(model, seed=seed, host_copy=True)
    eng = kie.Engine(kie.config(model, max_ctx=max_ctx, timeout_ms=5000, idle_ms=50, **kw), dw.kie)
    orc = OracleModel(model, dw.host, max_ctx)
    return dw, eng, orc


def _lockstep(kie, eng, orc, model, prompt, n_steps):
    """Prefill then n_steps teacher-forced decode steps with logits; returns the step reports."""
    from tests.parity import compare_step
    V = model.vocab
    logits = torch.empty(V, dtype=torch.float32, device="cuda")
    sid = eng.session_open()
    first = eng.prefill(sid, prompt)
    ref = orc.prefill(prompt)
    reports = [compare_step(ref, first, ref, model.dtype)]  # token only (no logits out of prefill)
    tok = int(np.argmax(ref))
    for _ in range(n_steps):
        out = eng.decode_step(sid, tok, logits.data_ptr())
        got = logits.cpu().numpy()
        ref = orc.step(tok)
        reports.append(compare_step(got, out, ref, model.dtype))
        tok = int(np.argmax(ref))
    assert eng.session_length(sid) == len(prompt) + n_steps
    return reports


# ------------------------------------------------------------------ attention op

@pytest.mark.parametrize("Hq,Hkv,D,ctx,dtype", [
    (4, 4, 64, 1, 0), (16, 8, 128, 7, 0), (16, 8, 128, 129, 0), (32, 8, 128, 1025, 1),
    (6, 2, 64, 300, 1), (16, 8, 128, 5000, 0), (16, 8, 128, 32768, 0),
])
def test_flash_decode_op_matches_oracle(kie, Hq, Hkv, D, ctx, dtype):
    from bandwidth_bound_stream_b200 import synth
    from oracle import oracle as orc
    rng = np.random.default_rng(ctx)
    q = rng.normal(0, 1, (Hq, D))
    stride = ctx + 3
    K = synth.normal_u16(ctx, 0x7001, Hkv * stride * D, dtype, std=1.0).reshape(Hkv, stride, D)
    Vv = synth.normal_u16(ctx, 0x7002, Hkv * stride * D, dtype, std=1.0).reshape(Hkv, stride, D)
    q_d = torch.tensor(q, dtype=torch.float32, device="cuda")
    k_d = torch.from_numpy(K.view(np.int16)).cuda()
    v_d = torch.from_numpy(Vv.view(np.int16)).cuda()
    out = torch.full((Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = kie.flash_decode_scratch_bytes(Hq, Hkv, D, ctx)
    scratch = torch.full((nbytes,), 0x55, dtype=torch.uint8, device="cuda")
    st = kie.flash_decode(q_d.data_ptr(), k_d.data_ptr(), v_d.data_ptr(), Hq, Hkv, D, ctx, stride, dtype,
                          out.data_ptr(), scratch.data_ptr(), nbytes)
    assert st == kie.KIE_OK
    got = out.cpu().numpy()
    # the oracle sees the query as the fp32 values the kernel reads
    qf = q.astype(np.float32).astype(np.float64)
    for h in range(Hq):
        g = h * Hkv // Hq
        want = orc.attention(qf[h], K[g, :ctx], Vv[g, :ctx], dtype)
        np.testing.assert_allclose(got[h], want, rtol=0, atol=2e-5 * max(1.0, np.abs(want).max()))


# ------------------------------------------------------------------ whole-model parity

def test_tiny_parity(kie):
    from bandwidth_bound_stream_b200 import synth
    from tests.parity import assert_reports
    m = synth.TINY
    dw, eng, orc = _setup(kie, m, 64)
    with eng:
        reps = _lockstep(kie, eng, orc, m, synth.prompt(m, 16), 32)
    assert_reports(reps, m.dtype)


def test_tiny_generate_and_launch_match_oracle_chain(kie):
    """kie_generate (doorbell, argmax fed back on the GPU) and kie_decode_launch (one stream-ordered
    launch) both follow the oracle's greedy chain while its margins exceed 0.05."""
    from bandwidth_bound_stream_b200 import synth
    from tests.parity import MARGIN, margin
    m = synth.TINY
    dw, eng, orc = _setup(kie, m, 96)
    prompt = synth.prompt(m, 16, session=3)
    n = 24
    with eng:
        sid = eng.session_open()
        first = eng.prefill(sid, prompt)
        ref = orc.prefill(prompt)
        assert first == int(np.argmax(ref)) or margin(ref) <= MARGIN
        chain, margins = [], []
        tok = first
        for _ in range(n):
            ref = orc.step(tok)
            tok = int(np.argmax(ref))
            chain.append(tok)
            margins.append(margin(ref))
        gen = eng.generate(sid, first, n)
        # compare up to the first low-margin step (after it the two chains may legitimately differ)
        k = next((i for i, mg in enumerate(margins) if mg <= MARGIN), n)
        assert list(gen[:k]) == chain[:k]
        # the stream-ordered launch from the same prefix gives the same tokens as the doorbell path
        eng.session_rewind(sid, len(prompt))
        tok_d = torch.tensor([first], dtype=torch.int32, device="cuda")
        out_d = torch.zeros(n, dtype=torch.int32, device="cuda")
        eng.decode_launch(sid, tok_d.data_ptr(), n, out_d.data_ptr())
        eng.sync()
        assert np.array_equal(out_d.cpu().numpy(), gen)


@pytest.mark.parametrize("name,prompt_len,steps,staging,kv_path", [
    ("slice-1.9b", 40, 8, 0, 1), ("slice-8b", 24, 6, 0, 1), ("ragged", 33, 10, 0, 1),
    ("slice-1.9b", 150, 8, 1, 1), ("slice-8b", 90, 6, 1, 1),
    ("tiny", 16, 12, 0, 2), ("ragged", 33, 10, 0, 2), ("slice-1.9b", 40, 8, 0, 2), ("slice-8b", 24, 6, 0, 2),
    ("slice-1.9b", 150, 8, 1, 2),
])
def test_sliced_shapes_parity(kie, name, prompt_len, steps, staging, kv_path):
    """Two-layer slices of the 1.9B (fp16, GQA 2) and 8B (bf16, GQA 4) shapes at full width, and a ragged
    shape (odd vocab, GQA 3, rows not divisible by the SM count). staging 1: the slices again with
    the weight chunks of the attention step staged in TMEM (d_model 2048 and 4096 take it).
    kv_path 2: the attention's K/V rows stream through the weight ring (one pass per two query
    heads: two passes on the 8B slice); 1: read from L2."""
    from bandwidth_bound_stream_b200 import synth
    from tests.parity import assert_reports
    m = synth.CONFIGS[name]
    dw, eng, orc = _setup(kie, m, prompt_len + steps + 4, b1_staging=staging, b1_kv_path=kv_path)
    with eng:
        reps = _lockstep(kie, eng, orc, m, synth.prompt(m, prompt_len), steps)
    assert_reports(reps, m.dtype)


def test_full_1p9b_parity_short_context(kie):
    """All 28 layers of the 1.9B shape, 64-token prompt, 4 decode steps with logits."""
    from bandwidth_bound_stream_b200 import synth
    from tests.parity import assert_reports
    m = synth.DENSE_1P9B
    dw, eng, orc = _setup(kie, m, 80)
    with eng:
        reps = _lockstep(kie, eng, orc, m, synth.prompt(m, 64), 4)
    assert_reports(reps, m.dtype)


INJECTED_STEPS = 3


def _bench_launch_layer0_check(kie, m, prompt_len, decode_n, positions, modes, prompt_checks=()):
    """One launch of the bench's configuration, then:
    * layer-0 K/V at sampled positions equal the oracle's projection of that position's token
      (they depend on that token alone);
    * the prefill's K/V of every layer at `prompt_checks` positions, recomputed by the oracle
      from the engine's cache below each (tests/inject.py);
    * INJECTED_STEPS more decode steps at the end of the launch's context, each compared with
      the oracle's full-depth step from the engine's cache: logits, argmax and the appended K/V
      of every layer. This checks the megakernel's attention (every split of every kv head and
      their merge) at the context lengths the benchmark runs."""
    from bandwidth_bound_stream_b200 import synth
    from oracle import oracle as orc
    from oracle.oracle import OracleModel
    from tests import inject
    from tests.parity import assert_reports
    max_ctx = prompt_len + decode_n + INJECTED_STEPS
    dw = kie.DeviceWeights(m, host_copy=True)
    prompt = synth.prompt(m, prompt_len)
    with kie.Engine(kie.config(m, max_ctx=max_ctx, timeout_ms=20000, idle_ms=50, modes=modes), dw.kie) as eng:
        sid = eng.session_open()
        first = eng.prefill(sid, prompt)
        tok_d = torch.tensor([first], dtype=torch.int32, device="cuda")
        out_d = torch.zeros(decode_n, dtype=torch.int32, device="cuda")
        eng.decode_launch(sid, tok_d.data_ptr(), decode_n, out_d.data_ptr())
        eng.sync()
        gen = out_d.cpu().numpy()
        assert gen.min() >= 0 and gen.max() < m.vocab
        kp, vp = eng.session_kv(sid)
        n = m.n_kv_heads * max_ctx * m.head_dim
        # copy layer 0 of the cache through a torch view of the engine's buffer
        K0 = _device_view(kp, n).cpu().numpy().view(np.uint16).reshape(m.n_kv_heads, max_ctx, m.head_dim)
        V0 = _device_view(vp, n).cpu().numpy().view(np.uint16).reshape(m.n_kv_heads, max_ctx, m.head_dim)
        o = OracleModel(m, dw.host, max_ctx)
        if prompt_checks:
            inject.check_prompt_positions(eng, sid, m, max_ctx, o, prompt, prompt_checks)
        logits = torch.empty(m.vocab, dtype=torch.float32, device="cuda")
        reps = inject.injected_decode_steps(eng, sid, m, max_ctx, o, int(gen[-1]), INJECTED_STEPS, logits)
        assert_reports(reps, m.dtype)
        assert eng.session_length(sid) == max_ctx
    seq = np.concatenate([prompt, [first], gen[:-1]])
    L0 = dw.host["layers"][0]
    D = m.head_dim
    for p in positions:
        e = orc.value(dw.host["tok_emb"][seq[p]], m.dtype)
        h = orc.rmsnorm(e, L0["attn_norm"], m.dtype, m.rms_eps)
        k = orc.matvec(L0["wk"], m.dtype, h)
        v = orc.matvec(L0["wv"], m.dtype, h)
        for g in range(m.n_kv_heads):
            kr = orc.rope(k[g * D:(g + 1) * D], p, m.rope_theta)
            want_k = orc.value(orc.store(kr, m.dtype), m.dtype)
            want_v = orc.value(orc.store(v[g * D:(g + 1) * D], m.dtype), m.dtype)
            # fp32 accumulation vs fp64: the stored 16-bit values are at most one rounding step apart
            _within_one_ulp(orc.value(K0[g, p], m.dtype), want_k, m.dtype)
            _within_one_ulp(orc.value(V0[g, p], m.dtype), want_v, m.dtype)


def _within_one_ulp(got, want, dtype):
    """|got - want| <= one unit in the last place of the storage type (fp16: 10 fraction bits,
    bf16: 7) at |want|, plus 1e-5 absolute. A value computed in fp32 and one computed in fp64 can
    round to the two neighbours of a rounding boundary. Near zero (RoPE's rotation cancels O(1)
    terms) the fp32 accumulation's absolute error, ~1e-6 for these dot products, exceeds the
    storage step. A wrong row or position differs by O(0.1)."""
    frac = 10 if dtype == 0 else 7
    mag = np.maximum(np.abs(np.asarray(want, dtype=np.float64)), 2.0 ** -14)  # fp16 subnormal spacing floor
    ulp = 2.0 ** (np.floor(np.log2(mag)) - frac)
    bad = np.abs(np.asarray(got, dtype=np.float64) - want) > ulp * (1 + 1e-9) + 1e-5
    assert not bad.any(), (np.asarray(got)[bad][:4], np.asarray(want)[bad][:4])


def test_full_1p9b_bench_launch_layer0_cache(kie):
    """The benchmark's configuration (1.9B, prompt 1024, one launch of 512 steps), prompt
    prefilled by the batch-1 kernel; then full-depth steps at contexts 1536-1538 against the
    oracle from the engine's cache (about 85 positions per attention split)."""
    from bandwidth_bound_stream_b200 import synth
    _bench_launch_layer0_check(kie, synth.DENSE_1P9B, 1024, 512, (0, 1, 777, 1023, 1024, 1300, 1535),
                               kie.KIE_MODE_BATCH1, prompt_checks=(700, 1023))


def test_full_8b_bench_launch_layer0_cache(kie):
    """The 8B (Llama-3-8B shape, bf16, theta 5e5) configuration: prompt 4096 prefilled in tick-kernel
    chunks, one launch of 256 decode steps; prefill K/V of every layer at two prompt positions and
    full-depth steps at contexts 4352-4354, against the oracle from the engine's cache."""
    from bandwidth_bound_stream_b200 import synth
    _bench_launch_layer0_check(kie, synth.DENSE_8B, 4096, 256, (0, 63, 64, 2049, 4095, 4096, 4351),
                               kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK, prompt_checks=(1500, 4095))


def test_full_1p9b_32k_bench_launch_layer0_cache(kie):
    """The long-context configuration: 1.9B, prompt 32768 prefilled in tick-kernel chunks, one
    launch of 256 decode steps (attention over a 32K cache); prefill K/V of every layer at two
    prompt positions and full-depth steps at contexts 33024-33026 (about 1,835 positions per
    attention split), against the oracle from the engine's cache."""
    from bandwidth_bound_stream_b200 import synth
    _bench_launch_layer0_check(kie, synth.DENSE_1P9B, 32768, 256, (0, 4095, 16384, 32703, 32767, 32768, 33023),
                               kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK, prompt_checks=(20000, 32767))


def _device_view(ptr, n):
    """A torch int16 tensor aliasing n elements of engine-owned device memory (read-only use)."""
    class _Holder:
        __cuda_array_interface__ = {"shape": (n,), "typestr": "<i2", "data": (ptr, False), "version": 2}
    return torch.as_tensor(_Holder(), device="cuda")


# ------------------------------------------------------------------ host-side errors and lifecycle

def test_errors_are_reported_not_fatal(kie):
    from bandwidth_bound_stream_b200 import synth
    m = synth.TINY
    dw = kie.DeviceWeights(m)
    with kie.Engine(kie.config(m, max_ctx=20, max_sessions=1, timeout_ms=5000, idle_ms=50), dw.kie) as eng:
        sid = eng.session_open()
        with pytest.raises(kie.KieError) as ei:
            eng.session_open()
        assert ei.value.status == kie.KIE_ERR_CAPACITY
        with pytest.raises(kie.KieError) as ei:
            eng.prefill(sid, np.zeros(21, dtype=np.int32))
        assert ei.value.status == kie.KIE_ERR_CAPACITY
        assert eng.session_length(sid) == 0
        with pytest.raises(kie.KieError) as ei:
            eng.decode_step(sid, m.vocab)
        assert ei.value.status == kie.KIE_ERR_ARG
        with pytest.raises(kie.KieError) as ei:
            eng.decode_step(sid + 1, 1)
        assert ei.value.status == kie.KIE_ERR_ARG
        # the engine still works afterwards
        first = eng.prefill(sid, synth.prompt(m, 8))
        assert 0 <= first < m.vocab
        with pytest.raises(kie.KieError) as ei:
            eng.generate(sid, first, 13)
        assert ei.value.status == kie.KIE_ERR_CAPACITY


def test_empty_inputs_and_a_cache_filled_to_max_ctx(kie):
    """Empty inputs are argument errors that change nothing. A session fills its cache to exactly
    max_ctx in parity with the oracle at every position, after which one more token is a capacity
    error from every entry point. A tick may end on the last position."""
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    from tests.parity import assert_reports, compare_step
    m = synth.TINY
    max_ctx = 40
    dw, eng, orc = _setup(kie, m, max_ctx, max_sessions=2, modes=kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK)
    with eng:
        # prefill 24 (tick kernel chunks), then batch-1 decode up to position max_ctx - 1
        assert_reports(_lockstep(kie, eng, orc, m, synth.prompt(m, 24), max_ctx - 24), m.dtype)
        sid = eng.session_open()
        full = 1 - sid  # the two slots are 0 and 1; the other one holds the full session
        assert eng.session_length(full) == max_ctx
        for call in (lambda: eng.decode_step(full, 1), lambda: eng.generate(full, 1, 1),
                     lambda: eng.prefill(full, [1]), lambda: eng.tick([full], [1], 1)):
            with pytest.raises(kie.KieError) as ei:
                call()
            assert ei.value.status == kie.KIE_ERR_CAPACITY
        assert eng.session_length(full) == max_ctx
        for call in (lambda: eng.prefill(sid, np.zeros(0, dtype=np.int32)), lambda: eng.generate(sid, 1, 0),
                     lambda: eng.tick([], np.zeros(0, dtype=np.int32), 1), lambda: eng.tick([sid], [1], 0)):
            with pytest.raises(kie.KieError) as ei:
                call()
            assert ei.value.status == kie.KIE_ERR_ARG
        assert eng.session_length(sid) == 0
        # a two-step tick that writes positions max_ctx - 2 and max_ctx - 1
        o2 = OracleModel(m, dw.host, max_ctx)
        p2 = synth.prompt(m, max_ctx - 2, session=3)
        first = eng.prefill(sid, p2)
        ref = o2.prefill(p2)
        reps = [compare_step(ref, first, ref, m.dtype)]
        t0 = int(np.argmax(ref))
        logits = torch.empty((2, 1, m.vocab), dtype=torch.float32, device="cuda")
        out = eng.tick([sid], [t0], 2, logits.data_ptr())
        got = logits.cpu().numpy()
        ref1 = o2.step(t0)
        reps.append(compare_step(got[0, 0], int(out[0, 0]), ref1, m.dtype))
        if int(out[0, 0]) == int(np.argmax(ref1)):  # else a low-margin step: the chains part here
            reps.append(compare_step(got[1, 0], int(out[1, 0]), o2.step(int(out[0, 0])), m.dtype))
        assert_reports(reps, m.dtype)
        assert eng.session_length(sid) == max_ctx


def _randomize_gains(dw, model, seed):
    """Norm gains from U(0.5, 1.5) and Wq, Wk scaled by 8 (peaked attention), rounded to the
    storage dtype by numpy / torch, written to the device tensors and to the host copy the
    oracle reads (before the engine is created)."""
    rng = np.random.default_rng(seed)
    for (name, layer), t in dw.tensors.items():
        if name in ("attn_norm", "mlp_norm", "final_norm"):
            f32 = rng.uniform(0.5, 1.5, model.d_model).astype(np.float32)
        elif name in ("wq", "wk"):
            old = t.cpu().numpy().view(np.uint16)
            if model.dtype == 0:
                f32 = 8.0 * old.view(np.float16).astype(np.float32)
            else:
                f32 = 8.0 * torch.from_numpy(old.view(np.int16)).view(torch.bfloat16).float().numpy()
        else:
            continue
        if model.dtype == 0:
            bits = f32.astype(np.float16).view(np.uint16)
        else:
            bits = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        t.copy_(torch.from_numpy(bits.view(np.int16)))
        if layer >= 0:
            dw.host["layers"][layer][name] = bits
        else:
            dw.host[name] = bits


def test_random_norm_gains_and_peaked_attention_parity(kie):
    """The synthetic models' gains are all 1.0, which cannot show a gain applied in the wrong
    place, and their small models attend almost uniformly, which hides a wrong score scale.
    With random gains and Wq, Wk scaled by 8: the prompt through the tick kernel's chunks
    (tensor-core scores), decode steps through the batch-1 kernel, then two-step ticks, each
    against the oracle on the same weights."""
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    from tests.parity import assert_reports, compare_step
    for i, m in enumerate((synth.TINY, synth.RAGGED)):
        max_ctx = 48
        dw = kie.DeviceWeights(m, host_copy=True)
        _randomize_gains(dw, m, 40 + i)
        orc = OracleModel(m, dw.host, max_ctx)
        cfg = kie.config(m, max_ctx=max_ctx, max_sessions=2, timeout_ms=5000, idle_ms=50,
                         modes=kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK)
        with kie.Engine(cfg, dw.kie) as eng:
            reps = _lockstep(kie, eng, orc, m, synth.prompt(m, 20), 8)
            sid = eng.session_open()
            o2 = OracleModel(m, dw.host, max_ctx)
            p2 = synth.prompt(m, 12, session=4)
            first = eng.prefill(sid, p2)
            ref = o2.prefill(p2)
            reps.append(compare_step(ref, first, ref, m.dtype))
            tok = int(np.argmax(ref))
            logits = torch.empty((2, 1, m.vocab), dtype=torch.float32, device="cuda")
            for _ in range(3):
                out = eng.tick([sid], [tok], 2, logits.data_ptr())
                got = logits.cpu().numpy()
                ref1 = o2.step(tok)
                reps.append(compare_step(got[0, 0], int(out[0, 0]), ref1, m.dtype))
                if int(out[0, 0]) != int(np.argmax(ref1)):
                    break  # a low-margin step (accepted above): the two chains part here
                ref2 = o2.step(int(out[0, 0]))
                reps.append(compare_step(got[1, 0], int(out[1, 0]), ref2, m.dtype))
                if int(out[1, 0]) != int(np.argmax(ref2)):
                    break
                tok = int(out[1, 0])
        assert_reports(reps, m.dtype)
        dw.free()


def test_resident_kernel_idles_out_and_relaunches(kie):
    """With no command the resident kernel gives up waiting after idle_ms and exits cleanly; the
    next call relaunches it and the results are unchanged."""
    import time
    from bandwidth_bound_stream_b200 import synth
    m = synth.TINY
    dw = kie.DeviceWeights(m)
    prompt = synth.prompt(m, 10)
    with kie.Engine(kie.config(m, max_ctx=64, timeout_ms=5000, idle_ms=20), dw.kie) as eng:
        sid = eng.session_open()
        first = eng.prefill(sid, prompt)
        a = eng.generate(sid, first, 5)
        time.sleep(0.3)  # well past idle_ms: the kernel has exited
        eng.session_rewind(sid, len(prompt))
        b = eng.generate(sid, first, 5)
        assert np.array_equal(a, b)


def test_tick_prefill_then_batch1_decode(kie):
    """An engine with both kernels: the prompt goes through the tick kernel's chunked prefill (its
    K/V land in the shared cache), then the batch-1 kernel decodes from that cache."""
    from bandwidth_bound_stream_b200 import synth
    from tests.parity import assert_reports
    for m, plen, steps in [(synth.TINY, 100, 12), (synth.SLICE_1P9B, 70, 6)]:
        dw, eng, orc = _setup(kie, m, plen + steps + 4, modes=kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK)
        with eng:
            reps = _lockstep(kie, eng, orc, m, synth.prompt(m, plen, session=5), steps)
        assert_reports(reps, m.dtype)
