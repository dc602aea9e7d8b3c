"""Parity of the multi-session tick kernel (tcgen05 weight contractions) with the CPU oracle.

Each session of a tick is an independent decode step, so the oracle runs every sampled
session on its own. Tolerances are those of tests/parity.py. Within one tick the first
step's argmax feeds the second step on the GPU; the oracle follows its own argmax, so the
second step is compared only where the first step's tokens are the oracle's (always, when
the oracle's margin exceeds 0.05).
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


def _run_tick_parity(kie, model, n_sess, prompt_lens, checked, ticks, max_ctx, modes=None):
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    from tests.parity import MARGIN, assert_reports, compare_step, margin
    modes = kie.KIE_MODE_TICK if modes is None else modes
    dw = kie.DeviceWeights(model, host_copy=True)
    eng = kie.Engine(kie.config(model, max_sessions=n_sess, max_ctx=max_ctx, timeout_ms=20000, idle_ms=100,
                                modes=modes), dw.kie)
    V = model.vocab
    reports = []
    checked = list(checked)
    with eng:
        sids = [eng.session_open() for _ in range(n_sess)]
        prompts = [synth.prompt(model, prompt_lens[i], session=i) for i in range(n_sess)]
        firsts = [eng.prefill(sids[i], prompts[i]) for i in range(n_sess)]
        orcs = {i: OracleModel(model, dw.host, max_ctx) for i in checked}
        toks = {}
        for i in checked:
            ref = orcs[i].prefill(prompts[i])
            reports.append(compare_step(ref, firsts[i], ref, model.dtype))
            toks[i] = int(np.argmax(ref))
        inputs = np.array(firsts, dtype=np.int32)
        for i in checked:
            inputs[i] = toks[i]  # teacher-force the checked sessions with the oracle's token
        logits = torch.empty((2, n_sess, V), dtype=torch.float32, device="cuda")
        for _ in range(ticks):
            # one teacher-forced step (logits compared for every checked session) ...
            out = eng.tick(sids, inputs, 1, logits.data_ptr())
            got = logits[0].cpu().numpy()
            for i in checked:
                ref = orcs[i].step(int(inputs[i]))
                reports.append(compare_step(got[i], int(out[0, i]), ref, model.dtype))
                inputs[i] = int(np.argmax(ref))
            for i in range(n_sess):
                if i not in checked:
                    inputs[i] = out[0, i]
            # ... then a two-step tick: step 1's argmax feeds step 2 on the GPU
            out = eng.tick(sids, inputs, 2, logits.data_ptr())
            got = logits.cpu().numpy()
            for i in list(checked):
                ref1 = orcs[i].step(int(inputs[i]))
                reports.append(compare_step(got[0, i], int(out[0, i]), ref1, model.dtype))
                t1 = int(np.argmax(ref1))
                if int(out[0, i]) != t1:  # a low-margin step: the two chains part here
                    assert margin(ref1) <= MARGIN
                    checked.remove(i)
                    continue
                ref2 = orcs[i].step(t1)
                reports.append(compare_step(got[1, i], int(out[1, i]), ref2, model.dtype))
                inputs[i] = int(np.argmax(ref2))
            for i in range(n_sess):
                if i not in checked:
                    inputs[i] = out[1, i]
            assert out.min() >= 0 and out.max() < V
        for i in range(n_sess):
            assert eng.session_length(sids[i]) == prompt_lens[i] + 3 * ticks
    return assert_reports(reports, model.dtype)


def test_tick_tiny_parity(kie):
    """fp16 tiny model, 5 sessions, prompts spanning one and two prefill chunks."""
    from bandwidth_bound_stream_b200 import synth
    _run_tick_parity(kie, synth.TINY, 5, [9, 17, 33, 69, 100], checked=[0, 1, 2, 3, 4], ticks=2, max_ctx=128)


def test_tick_ragged_parity(kie):
    """bf16, odd vocabulary (row blocks padded), 3 query heads per kv head, d = 384."""
    from bandwidth_bound_stream_b200 import synth
    _run_tick_parity(kie, synth.RAGGED, 7, [5, 12, 64, 65, 3, 30, 20], checked=[0, 3, 6], ticks=2, max_ctx=96)


def test_tick_small_head_parity(kie):
    """head_dim 32 (the CUDA-core attention path, contexts spanning several K/V chunks), 5 query
    heads per kv head (two passes), odd k-step counts (single-tile atoms), fp16, odd vocabulary."""
    from bandwidth_bound_stream_b200 import synth
    _run_tick_parity(kie, synth.SMALL_HEAD, 6, [5, 40, 100, 129, 7, 250], checked=[0, 2, 3, 5], ticks=2,
                     max_ctx=280)


def test_tick_slice_10p8b_56_sessions(kie):
    """Two layers of the 10.8B tick shape at full width (bf16, GQA 4), 56 sessions; 5 sampled
    sessions are checked against the oracle."""
    from bandwidth_bound_stream_b200 import synth
    lens = [4 + (7 * i) % 61 for i in range(56)]
    _run_tick_parity(kie, synth.SLICE_TICK, 56, lens, checked=[0, 13, 27, 41, 55], ticks=1, max_ctx=80)


def test_tick_errors(kie):
    from bandwidth_bound_stream_b200 import synth
    m = synth.TINY
    dw = kie.DeviceWeights(m)
    with kie.Engine(kie.config(m, max_sessions=3, max_ctx=16, timeout_ms=5000, idle_ms=50,
                               modes=kie.KIE_MODE_TICK), dw.kie) as eng:
        a, b = eng.session_open(), eng.session_open()
        eng.prefill(a, synth.prompt(m, 4))
        eng.prefill(b, synth.prompt(m, 14))
        with pytest.raises(kie.KieError) as ei:
            eng.tick([a, a], [1, 2], 1)
        assert ei.value.status == kie.KIE_ERR_ARG
        with pytest.raises(kie.KieError) as ei:
            eng.tick([a, b], [1, 2], 3)  # b has 14 of 16 positions
        assert ei.value.status == kie.KIE_ERR_CAPACITY
        with pytest.raises(kie.KieError) as ei:
            eng.decode_step(a, 1)  # no batch-1 kernel in this engine
        assert ei.value.status == kie.KIE_ERR_UNSUPPORTED
        out = eng.tick([a, b], [1, 2], 2)
        assert out.shape == (2, 2) and eng.session_length(a) == 6


def test_tick_launch_matches_doorbell(kie):
    """The stream-ordered launch (device buffers) computes the same tick as the doorbell path
    (split-K partial sums meet through atomics in either order, so logits agree to a tight
    tolerance, not bit for bit), and both match the oracle's steps of every session."""
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    from tests.parity import assert_reports, compare_step
    m = synth.TINY
    dw = kie.DeviceWeights(m, host_copy=True)
    n = 6
    with kie.Engine(kie.config(m, max_sessions=n, max_ctx=64, timeout_ms=5000, idle_ms=50,
                               modes=kie.KIE_MODE_TICK), dw.kie) as eng:
        sids = [eng.session_open() for _ in range(n)]
        lens = [5, 9, 17, 33, 2, 40]
        firsts = np.array([eng.prefill(sids[i], synth.prompt(m, lens[i], session=i)) for i in range(n)],
                          dtype=np.int32)
        la = torch.empty((2, n, m.vocab), dtype=torch.float32, device="cuda")
        lb = torch.empty_like(la)
        out_a = eng.tick(sids, firsts, 2, la.data_ptr())
        for i in range(n):
            eng.session_rewind(sids[i], lens[i])
        tok_d = torch.tensor(firsts, device="cuda")
        out_d = torch.zeros((2, n), dtype=torch.int32, device="cuda")
        eng.tick_launch(sids, tok_d.data_ptr(), 2, out_d.data_ptr(), lb.data_ptr())
        eng.sync()
        np.testing.assert_allclose(lb.cpu().numpy(), la.cpu().numpy(), rtol=0, atol=1e-3)
        assert all(eng.session_length(sids[i]) == lens[i] + 2 for i in range(n))
        out_b = out_d.cpu().numpy()
        reports = []
        for i in range(n):
            orc = OracleModel(m, dw.host, 64)
            orc.prefill(synth.prompt(m, lens[i], session=i))
            ref1 = orc.step(int(firsts[i]))
            for out, lg in ((out_a, la), (out_b, lb)):
                reports.append(compare_step(lg[0, i].cpu().numpy(), int(out[0, i]), ref1, m.dtype))
            if int(out_a[0, i]) == int(out_b[0, i]):  # step 2's input is step 1's argmax on each path
                ref2 = orc.step(int(out_a[0, i]))
                for out, lg in ((out_a, la), (out_b, lb)):
                    reports.append(compare_step(lg[1, i].cpu().numpy(), int(out[1, i]), ref2, m.dtype))
        assert_reports(reports, m.dtype)


# ------------------------------------------------------------------ many attention tiles

def test_tick_tiny_parity_many_tiles(kie):
    """Prompts of 300-700 positions: chunked prefill crosses 5-11 chunks of 64 positions and the
    tensor-core attention of both prefill and tick walks 3-6 tiles of 128 positions (the stage
    alternation and the prefetch of tile t + 2), against the oracle end to end."""
    from bandwidth_bound_stream_b200 import synth
    _run_tick_parity(kie, synth.TINY, 4, [300, 417, 555, 700], checked=[0, 1, 2, 3], ticks=2, max_ctx=720)


def test_tick_ragged_parity_many_tiles(kie):
    """bf16, 3 query heads per kv head, prompts ending mid-tile and mid-chunk (301, 480, 650)."""
    from bandwidth_bound_stream_b200 import synth
    _run_tick_parity(kie, synth.RAGGED, 3, [301, 480, 650], checked=[0, 1, 2], ticks=2, max_ctx=670)


def test_tick_two_passes_per_unit(kie):
    """bf16, head_dim 64, 6 query heads per kv head: every unit of the tensor-core attention is
    two passes (4 heads, then 2) over the same K/V tiles; prompts end mid-tile and mid-chunk."""
    from bandwidth_bound_stream_b200 import synth
    _run_tick_parity(kie, synth.GQA6, 3, [300, 129, 517], checked=[0, 1, 2], ticks=2, max_ctx=540)


def test_tick_wide_kv_many_passes(kie):
    """32 kv heads of 5 query heads: a prefill chunk's 64 x 32 x 2 attention passes exceed the
    per-step balancing (they are dealt in turn) and fill more than one stream per SM."""
    from bandwidth_bound_stream_b200 import synth
    _run_tick_parity(kie, synth.WIDE_KV, 2, [200, 70], checked=[0, 1], ticks=2, max_ctx=220)


def _run_tick_injected(kie, model, lens, checked, ticks, prompt_checks=()):
    """Prefill every session (tick-kernel chunks), then `ticks` two-step ticks with logits. For
    each checked session the oracle continues from the engine's cache (tests/inject.py): both
    steps of every tick are compared (logits, argmax, appended K/V of every layer), and the
    prefill's K/V at `prompt_checks` positions (negative: from the end of the prompt)."""
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    from tests import inject
    from tests.parity import assert_reports, compare_step
    n = len(lens)
    max_ctx = max(lens) + 2 * ticks + 4
    dw = kie.DeviceWeights(model, host_copy=True)
    reports = []
    with kie.Engine(kie.config(model, max_sessions=n, max_ctx=max_ctx, timeout_ms=30000, idle_ms=100,
                               modes=kie.KIE_MODE_TICK), dw.kie) as eng:
        sids = [eng.session_open() for _ in range(n)]
        prompts = [synth.prompt(model, lens[i], session=i) for i in range(n)]
        toks = np.array([eng.prefill(sids[i], prompts[i]) for i in range(n)], dtype=np.int32)
        orcs = {}
        for i in checked:
            orcs[i] = OracleModel(model, dw.host, max_ctx)
            if prompt_checks:
                inject.check_prompt_positions(eng, sids[i], model, max_ctx, orcs[i], prompts[i],
                                              sorted(p % lens[i] for p in prompt_checks))
            inject.copy_cache(eng, sids[i], model, max_ctx, orcs[i], lens[i])
        logits = torch.empty((2, n, model.vocab), dtype=torch.float32, device="cuda")
        for _ in range(ticks):
            ctx = [eng.session_length(s) for s in sids]
            out = eng.tick(sids, toks, 2, logits.data_ptr())
            got = logits.cpu().numpy()
            for i in checked:
                ref1 = orcs[i].step(int(toks[i]), pos=ctx[i])
                reports.append(compare_step(got[0, i], int(out[0, i]), ref1, model.dtype))
                inject.check_position_kv(eng, sids[i], model, max_ctx, orcs[i], ctx[i], model.dtype)
                # step 2's input on the GPU was step 1's argmax: the oracle takes the same token
                ref2 = orcs[i].step(int(out[0, i]), pos=ctx[i] + 1)
                reports.append(compare_step(got[1, i], int(out[1, i]), ref2, model.dtype))
                inject.check_position_kv(eng, sids[i], model, max_ctx, orcs[i], ctx[i] + 1, model.dtype)
            assert out.min() >= 0 and out.max() < model.vocab
            toks = out[1].copy()
        for i in range(n):
            assert eng.session_length(sids[i]) == lens[i] + 2 * ticks
    dw.free()
    return assert_reports(reports, model.dtype)


def test_tick_slice_10p8b_56_sessions_bench_contexts(kie):
    """The tick workload's shape (2 of its 48 layers at full width, bf16, GQA 4) with its 56
    seeded prompt lengths in [1000, 1500]: 8-12 attention tiles per session. Five sessions are
    checked over two ticks from the engine's cache, plus their prefill K/V at three positions."""
    from bandwidth_bound_stream_b200 import synth
    lens = [synth.tick_prompt_length(s) for s in range(56)]
    _run_tick_injected(kie, synth.SLICE_TICK, lens, checked=[0, 13, 27, 41, 55], ticks=2,
                       prompt_checks=(129, 777, -1))


def test_tick_full_depth_10p8b(kie):
    """All 48 layers of the tick model (10.8B, bf16), two sessions at their seeded prompt lengths,
    one two-step tick compared with the oracle's full-depth steps from the engine's cache, and the
    prefill's K/V of every layer at the last prompt position."""
    from bandwidth_bound_stream_b200 import synth
    lens = [synth.tick_prompt_length(s) for s in range(2)]
    _run_tick_injected(kie, synth.TICK_10P8B, lens, checked=[0, 1], ticks=1, prompt_checks=(-1,))
