"""Failure paths of both kernels on the GPU, with every failure made on the host.

No test here faults, traps or hangs a GPU:
  * a grid barrier that cannot complete comes from kie_inject_fault (the host starts the
    barrier counter one arrival short), so every CTA's bounded wait runs out after
    timeout_ms and the kernel returns an error status;
  * an out-of-range token is written by the host into the device input buffer of a
    stream-ordered launch; both kernels check it before any row of the embedding table is
    read, and fail the command;
  * non-finite logits come from a NaN final-norm gain: no index wins the argmax, and the
    command fails instead of feeding an invalid token to the next step.
Each failed call must report its status, poison the engine (KIE_ERR_STATE afterwards), let
kie_destroy finish, and leave the GPU usable: a new engine afterwards decodes the same
tokens as before the failure.
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


@pytest.fixture(scope="module")
def tiny(kie):
    from bandwidth_bound_stream_b200 import synth
    return synth.TINY, kie.DeviceWeights(synth.TINY)


MODES = {"batch1": 1, "tick": 2}


def _engine(kie, m, dw, modes, timeout_ms=300):
    return kie.Engine(kie.config(m, max_sessions=2, max_ctx=64, timeout_ms=timeout_ms, idle_ms=30, modes=modes), dw.kie)


def _reference_tokens(kie, m, dw):
    """Greedy tokens of a healthy engine: 8 batch-1 steps and one 2-step tick of two sessions."""
    from bandwidth_bound_stream_b200 import synth
    with _engine(kie, m, dw, kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK) as eng:
        a, b = eng.session_open(), eng.session_open()
        fa = eng.prefill(a, synth.prompt(m, 9, session=1))
        fb = eng.prefill(b, synth.prompt(m, 12, session=2))
        gen = eng.generate(a, fa, 8)
        tick = eng.tick([a, b], [int(gen[-1]), fb], 2)
    return gen, tick


def _expect(kie, call, status):
    with pytest.raises(kie.KieError) as ei:
        call()
    assert ei.value.status == status, str(ei.value)
    return ei.value


@pytest.mark.parametrize("path", ["decode_step", "decode_launch", "tick", "tick_launch"])
def test_barrier_that_cannot_complete_times_out_and_poisons(kie, tiny, path):
    from bandwidth_bound_stream_b200 import synth
    m, dw = tiny
    before = _reference_tokens(kie, m, dw)
    eng = _engine(kie, m, dw, kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK)
    sid = eng.session_open()
    first = eng.prefill(sid, synth.prompt(m, 9, session=1))
    eng.inject_fault(kie.KIE_FAULT_BARRIER_SHORT)
    tok_d = torch.tensor([first], dtype=torch.int32, device="cuda")
    out_d = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    if path == "decode_step":
        err = _expect(kie, lambda: eng.decode_step(sid, first), kie.KIE_ERR_TIMEOUT)
    elif path == "decode_launch":
        eng.decode_launch(sid, tok_d.data_ptr(), 2, out_d.data_ptr())  # queued; the status comes at sync
        err = _expect(kie, eng.sync, kie.KIE_ERR_TIMEOUT)
    elif path == "tick":
        err = _expect(kie, lambda: eng.tick([sid], [first], 2), kie.KIE_ERR_TIMEOUT)
    else:
        eng.tick_launch([sid], tok_d.data_ptr(), 2, out_d.data_ptr())
        err = _expect(kie, eng.sync, kie.KIE_ERR_TIMEOUT)
    # whichever bounded wait runs out first names itself (a grid barrier, or the tick kernel's
    # producer waiting for the attention phase that follows it); all are timeouts
    assert "timed out" in str(err) or "no answer" in str(err)
    # poisoned: every later call except the error text and destroy
    _expect(kie, lambda: eng.decode_step(sid, first), kie.KIE_ERR_STATE)
    _expect(kie, lambda: eng.tick([sid], [first], 1), kie.KIE_ERR_STATE)
    _expect(kie, eng.session_open, kie.KIE_ERR_STATE)
    eng.close()  # kie_destroy returns once the kernel has left
    torch.cuda.synchronize()
    after = _reference_tokens(kie, m, dw)
    assert np.array_equal(before[0], after[0]) and np.array_equal(before[1], after[1])


@pytest.mark.parametrize("path", ["decode_launch", "tick_launch"])
def test_out_of_range_device_token_fails_the_command(kie, tiny, path):
    from bandwidth_bound_stream_b200 import synth
    m, dw = tiny
    eng = _engine(kie, m, dw, kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK, timeout_ms=2000)
    sid = eng.session_open()
    eng.prefill(sid, synth.prompt(m, 9, session=1))
    bad = torch.tensor([m.vocab], dtype=torch.int32, device="cuda")  # one past the last row
    out_d = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    if path == "decode_launch":
        eng.decode_launch(sid, bad.data_ptr(), 2, out_d.data_ptr())
    else:
        eng.tick_launch([sid], bad.data_ptr(), 2, out_d.data_ptr())
    err = _expect(kie, eng.sync, kie.KIE_ERR_DEVICE)
    assert "token id out of range" in str(err)
    _expect(kie, lambda: eng.decode_step(sid, 1), kie.KIE_ERR_STATE)
    eng.close()
    torch.cuda.synchronize()


def test_non_finite_logits_fail_the_command(kie):
    """A NaN final-norm gain makes every logit NaN. The argmax then has no winner; the batch-1
    kernel (one step, and a two-step generate whose second step would read that token) and the
    tick kernel (two steps) report KIE_ERR_DEVICE instead of returning or reusing an invalid id."""
    from bandwidth_bound_stream_b200 import synth
    m = synth.TINY
    dw = kie.DeviceWeights(m)
    dw.tensors[("final_norm", -1)].fill_(0x7E00)  # fp16 NaN
    for call in ("decode_step", "generate", "tick"):
        eng = _engine(kie, m, dw, kie.KIE_MODE_BATCH1 | kie.KIE_MODE_TICK, timeout_ms=2000)
        sid = eng.session_open()
        prompt = synth.prompt(m, 9, session=1)
        if call == "tick":  # the tick kernel's prefill chunk ends in its own argmax: reaching it fails too
            _expect(kie, lambda: eng.prefill(sid, prompt), kie.KIE_ERR_DEVICE)
        else:
            eng2 = _engine(kie, m, dw, kie.KIE_MODE_BATCH1)  # batch-1 prefill: its head fails the same way
            s2 = eng2.session_open()
            _expect(kie, lambda: eng2.prefill(s2, prompt), kie.KIE_ERR_DEVICE)
            eng2.close()
            if call == "decode_step":
                _expect(kie, lambda: eng.decode_step(sid, 1), kie.KIE_ERR_DEVICE)
            else:
                _expect(kie, lambda: eng.generate(sid, 1, 2), kie.KIE_ERR_DEVICE)
        _expect(kie, lambda: eng.decode_step(sid, 1), kie.KIE_ERR_STATE)
        eng.close()
    torch.cuda.synchronize()
    dw.free()
