"""FP8 (E4M3) weights in the batch-1 kernel against the oracle (GPU tests).

The quantisation decides integers (the codes), so the engine's codes and scales must equal
the oracle's bit for bit (both divide in fp32 and round to the nearest code). The forward
pass is then compared with the oracle running on the same codes and scales, at the
tolerances of tests/parity.py: the only differences left are fp32 against fp64 arithmetic.
"""
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


@pytest.mark.parametrize("dtype", [0, 1])
def test_quantize_matches_the_oracle_bit_for_bit(kie, dtype):
    from bandwidth_bound_stream_b200 import synth
    from oracle import oracle as orc
    rows, cols = 300, 1216
    W = synth.normal_u16(21 + dtype, 0x61, rows * cols, dtype, std=1.0).reshape(rows, cols)
    # rows at very different magnitudes (subnormal codes, large values), an all-zero row
    f = orc.value(W, dtype) * np.exp2(np.arange(rows) % 40 - 20.0)[:, None]
    W = orc.store(f, dtype).reshape(rows, cols)
    W[7] = 0
    w = torch.from_numpy(W.view(np.int16)).cuda()
    q = torch.zeros((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.zeros(rows, dtype=torch.float32, device="cuda")
    assert kie.quantize_e4m3(w.data_ptr(), rows, cols, dtype, q.data_ptr(), s.data_ptr()) == kie.KIE_OK
    torch.cuda.synchronize()
    want_q, want_s = orc.quantize_rows(W, dtype)
    assert np.array_equal(s.cpu().numpy(), want_s)
    assert np.array_equal(q.cpu().numpy(), want_q)


def _fp8_lockstep(kie, m, prompt_len, steps, max_extra=2):
    from bandwidth_bound_stream_b200 import synth
    from oracle import oracle as orc
    from oracle.oracle import OracleModel
    from tests.parity import assert_reports, compare_step
    dw = kie.DeviceWeights(m, host_copy=True)
    max_ctx = prompt_len + steps + max_extra
    o = OracleModel(m, dw.host, max_ctx, q8=orc.quantize_model(m, dw.host))
    prompt = synth.prompt(m, prompt_len)
    logits = torch.empty(m.vocab, dtype=torch.float32, device="cuda")
    reports = []
    with kie.Engine(kie.config(m, max_ctx=max_ctx, timeout_ms=10000, idle_ms=50, weight_fp8=True), dw.kie) as eng:
        sid = eng.session_open()
        first = eng.prefill(sid, prompt)
        ref = o.prefill(prompt)
        reports.append(compare_step(ref, first, ref, m.dtype))
        tok = int(np.argmax(ref))
        for _ in range(steps):
            out = eng.decode_step(sid, tok, logits.data_ptr())
            ref = o.step(tok)
            reports.append(compare_step(logits.cpu().numpy(), out, ref, m.dtype))
            tok = int(np.argmax(ref))
    dw.free()
    return assert_reports(reports, m.dtype)


@pytest.mark.parametrize("name,prompt_len,steps", [("tiny", 16, 16), ("ragged", 21, 8), ("slice-1.9b", 40, 8),
                                                   ("slice-8b", 24, 6)])
def test_fp8_parity(kie, name, prompt_len, steps):
    """Tiny (fp16), ragged (bf16, 3 query heads per kv head), 2-layer slices of the 1.9B and 8B
    shapes; the prompt goes through the batch-1 kernel too."""
    from bandwidth_bound_stream_b200 import synth
    _fp8_lockstep(kie, synth.CONFIGS[name], prompt_len, steps)


def test_fp8_full_1p9b_bench_launch(kie):
    """The FP8 benchmark configuration: all 28 layers, prompt 1024, one launch of 512 decode steps,
    then three steps compared with the oracle's FP8 step from the engine's cache (logits, argmax
    and the appended K/V of every layer)."""
    from bandwidth_bound_stream_b200 import synth
    from oracle import oracle as orc
    from oracle.oracle import OracleModel
    from tests import inject
    from tests.parity import assert_reports
    m = synth.DENSE_1P9B
    prompt_len, decode_n, extra = 1024, 512, 3
    max_ctx = prompt_len + decode_n + extra
    dw = kie.DeviceWeights(m, host_copy=True)
    prompt = synth.prompt(m, prompt_len)
    with kie.Engine(kie.config(m, max_ctx=max_ctx, timeout_ms=20000, idle_ms=50, weight_fp8=True), dw.kie) as eng:
        sid = eng.session_open()
        first = eng.prefill(sid, prompt)
        tok_d = torch.tensor([first], dtype=torch.int32, device="cuda")
        out_d = torch.zeros(decode_n, dtype=torch.int32, device="cuda")
        eng.decode_launch(sid, tok_d.data_ptr(), decode_n, out_d.data_ptr())
        eng.sync()
        gen = out_d.cpu().numpy()
        assert gen.min() >= 0 and gen.max() < m.vocab
        o = OracleModel(m, dw.host, max_ctx, q8=orc.quantize_model(m, dw.host))
        logits = torch.empty(m.vocab, dtype=torch.float32, device="cuda")
        reps = inject.injected_decode_steps(eng, sid, m, max_ctx, o, int(gen[-1]), extra, logits)
    assert_reports(reps, m.dtype)
    dw.free()


def test_fp8_needs_the_batch1_mode_only(kie):
    from bandwidth_bound_stream_b200 import synth
    m = synth.TINY
    dw = kie.DeviceWeights(m)
    with pytest.raises(kie.KieError) as ei:
        kie.Engine(kie.config(m, max_ctx=32, weight_fp8=True, modes=kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK), dw.kie)
    assert ei.value.status == kie.KIE_ERR_ARG
    dw.free()
