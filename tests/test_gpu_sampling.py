"""Temperature / top-k sampling on the GPU against the oracle's sampler (GPU tests).

The oracle's sampler (orc_sample, pinned in tests/test_oracle_pins.py) defines a step's token
from its logits and (temperature, top_k, seed, position). Every GPU step is checked twice:
  * on the same logits: the oracle's sampler applied to the GPU's own fp32 logits must pick
    the GPU's token unless the draw lies within SAME_EPS of the total weight from a boundary
    between candidates (the GPU sums the weights in fp32, in its own order);
  * on the oracle's logits: the oracle's token must be the GPU's wherever the draw's distance
    to a boundary exceeds what the step's logit difference can move it. With every logit
    within delta, each weight moves by a factor within e^(+-2 delta / T) relative to the top
    one, so the normalised cumulative weights move by less than e^(2 delta / T) - 1.
Logits are held to the tolerances of tests/parity.py. Each next input is the GPU's token, so
both sides follow one sequence.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SAME_EPS = 1e-5


@pytest.fixture(scope="module")
def kie():
    from bandwidth_bound_stream_b200 import build
    build.build_kie()
    from bandwidth_bound_stream_b200 import kie as k
    return k


class Checker:
    def __init__(self, T, k, seed, dtype):
        self.T, self.k, self.seed, self.dtype = T, k, seed, dtype
        self.steps = self.strict_same = self.strict_ref = 0
        self.worst = 0.0

    def step(self, got_logits, gpu_tok, ref_logits, pos):
        from oracle import oracle as orc
        from tests.parity import LOGIT_TOL
        u = orc.uniform(self.seed, pos)
        self.steps += 1
        ref_tok, ref_margin = orc.sample(ref_logits, self.T, self.k, u)
        if got_logits is None:  # no logits out of this call: the tolerance bounds the difference
            delta = LOGIT_TOL[self.dtype]
        else:
            got = np.asarray(got_logits, dtype=np.float64)
            delta = float(np.max(np.abs(got - ref_logits)))
            self.worst = max(self.worst, delta)
            assert delta <= LOGIT_TOL[self.dtype], f"logits differ by {delta:.3g} at position {pos}"
            same_tok, same_margin = orc.sample(got, self.T, self.k, u)
            if same_margin > SAME_EPS:
                self.strict_same += 1
                assert gpu_tok == same_tok, (pos, gpu_tok, same_tok, same_margin)
        if ref_margin > np.expm1(2 * delta / self.T) + SAME_EPS:
            self.strict_ref += 1
            assert gpu_tok == ref_tok, (pos, gpu_tok, ref_tok, ref_margin, delta)
        return ref_tok

    def enough(self):
        # most steps must have been decided strictly, else the test says nothing
        assert self.strict_same >= 0.9 * (self.steps - 1) and self.strict_ref >= 0.6 * self.steps, vars(self)


@pytest.mark.parametrize("name,T,k,seed", [("tiny", 0.8, 8, 1234), ("tiny", 1.0, 32, 7), ("ragged", 0.5, 2, 99),
                                           ("ragged", 2.0, 32, 2 ** 63 + 5), ("slice-1.9b", 0.7, 20, 31337)])
def test_batch1_decode_steps_sample_like_the_oracle(kie, name, T, k, seed):
    """Prefill (its last position draws the first token), then decode steps with logits. Tiny with
    top_k 32 has fewer head rows per SM (27-28) than candidates: padding slots must never win."""
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    m = synth.CONFIGS[name]
    prompt = synth.prompt(m, 12, session=2)
    n_steps = 20
    max_ctx = len(prompt) + n_steps + 2
    dw = kie.DeviceWeights(m, host_copy=True)
    orc = OracleModel(m, dw.host, max_ctx)
    chk = Checker(T, k, seed, m.dtype)
    logits = torch.empty(m.vocab, dtype=torch.float32, device="cuda")
    with kie.Engine(kie.config(m, max_ctx=max_ctx, timeout_ms=5000, idle_ms=50), dw.kie) as eng:
        sid = eng.session_open()
        eng.session_sampling(sid, temperature=T, top_k=k, seed=seed)
        tok = eng.prefill(sid, prompt)
        chk.step(None, tok, orc.prefill(prompt), len(prompt) - 1)
        for i in range(n_steps):
            pos = len(prompt) + i
            out = eng.decode_step(sid, tok, logits.data_ptr())
            chk.step(logits.cpu().numpy(), out, orc.step(tok), pos)
            tok = out
    chk.enough()
    dw.free()


def test_decode_launch_samples_every_step_on_the_gpu(kie):
    """n sampled steps in one launch, each step's token fed back on the GPU; per-step logits out."""
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    m = synth.TINY
    T, k, seed = 0.9, 16, 4242
    prompt = synth.prompt(m, 10, session=5)
    n = 24
    dw = kie.DeviceWeights(m, host_copy=True)
    orc = OracleModel(m, dw.host, 64)
    with kie.Engine(kie.config(m, max_ctx=64, timeout_ms=5000, idle_ms=50), dw.kie) as eng:
        sid = eng.session_open()
        eng.session_sampling(sid, temperature=T, top_k=k, seed=seed)
        first = eng.prefill(sid, prompt)
        orc.prefill(prompt)
        tok_d = torch.tensor([first], dtype=torch.int32, device="cuda")
        out_d = torch.zeros(n, dtype=torch.int32, device="cuda")
        lg_d = torch.empty((n, m.vocab), dtype=torch.float32, device="cuda")
        eng.decode_launch(sid, tok_d.data_ptr(), n, out_d.data_ptr(), lg_d.data_ptr())
        eng.sync()
        out, lg = out_d.cpu().numpy(), lg_d.cpu().numpy()
    chk = Checker(T, k, seed, m.dtype)
    tok = first
    for i in range(n):
        chk.step(lg[i], int(out[i]), orc.step(tok), len(prompt) + i)
        tok = int(out[i])
    chk.enough()
    # a different seed draws a different chain (20 sampled steps at T near 1 over 16 candidates)
    with kie.Engine(kie.config(m, max_ctx=64, timeout_ms=5000, idle_ms=50), dw.kie) as eng:
        sid = eng.session_open()
        eng.session_sampling(sid, temperature=T, top_k=k, seed=seed + 1)
        eng.prefill(sid, prompt)
        other = eng.generate(sid, first, n)
    assert not np.array_equal(other, out)
    dw.free()


def test_tick_samples_each_session_with_its_own_settings(kie):
    """Three sessions in one tick: greedy, top-5 at T 0.7, top-32 at T 1.3 (the tick kernel's
    sampling over the whole vocabulary of a row); two steps, logits of both compared."""
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    from tests.parity import compare_step
    m = synth.RAGGED
    settings = [None, (0.7, 5, 11), (1.3, 32, 12)]
    lens = [9, 30, 17]
    dw = kie.DeviceWeights(m, host_copy=True)
    with kie.Engine(kie.config(m, max_sessions=3, max_ctx=48, timeout_ms=5000, idle_ms=50,
                               modes=kie.KIE_MODE_TICK), dw.kie) as eng:
        sids = [eng.session_open() for _ in range(3)]
        orcs, chks, firsts = [], [], []
        for i, sid in enumerate(sids):
            if settings[i]:
                T, k, seed = settings[i]
                eng.session_sampling(sid, temperature=T, top_k=k, seed=seed)
                chks.append(Checker(T, k, seed, m.dtype))
            else:
                chks.append(None)
            p = synth.prompt(m, lens[i], session=i)
            firsts.append(eng.prefill(sid, p))
            orcs.append(OracleModel(m, dw.host, 48))
            ref = orcs[i].prefill(p)
            if chks[i]:
                chks[i].step(None, firsts[i], ref, lens[i] - 1)
        logits = torch.empty((2, 3, m.vocab), dtype=torch.float32, device="cuda")
        toks = np.array(firsts, dtype=np.int32)
        for tick in range(3):
            out = eng.tick(sids, toks, 2, logits.data_ptr())
            got = logits.cpu().numpy()
            for i in range(3):
                pos = lens[i] + 2 * tick
                ref1 = orcs[i].step(int(toks[i]))
                ref2 = None
                if chks[i]:
                    chks[i].step(got[0, i], int(out[0, i]), ref1, pos)
                    ref2 = orcs[i].step(int(out[0, i]))
                    chks[i].step(got[1, i], int(out[1, i]), ref2, pos + 1)
                else:
                    r = compare_step(got[0, i], int(out[0, i]), ref1, m.dtype)
                    assert r.token_ok and r.max_abs <= 5e-2
                    ref2 = orcs[i].step(int(out[0, i]))
                    r = compare_step(got[1, i], int(out[1, i]), ref2, m.dtype)
                    assert r.token_ok and r.max_abs <= 5e-2
            toks = out[1].copy()
        for c in chks:
            if c:
                c.enough()
    dw.free()


def test_sampling_settings_are_checked(kie):
    from bandwidth_bound_stream_b200 import synth
    m = synth.TINY
    dw = kie.DeviceWeights(m)
    with kie.Engine(kie.config(m, max_ctx=32, timeout_ms=5000, idle_ms=50), dw.kie) as eng:
        sid = eng.session_open()
        for T, k in ((1.0, 0), (1.0, kie.KIE_TOPK_MAX + 1), (0.0, 4), (float("inf"), 4), (float("nan"), 4),
                     (-1.0, 4)):
            with pytest.raises(kie.KieError) as ei:
                eng.session_sampling(sid, temperature=T, top_k=k, seed=1)
            assert ei.value.status == kie.KIE_ERR_ARG
        eng.session_sampling(sid, temperature=0.0, top_k=1)  # greedy: the temperature is unused
        eng.session_sampling(sid, greedy=True)
        with pytest.raises(kie.KieError) as ei:
            eng.session_sampling(sid + 1, temperature=1.0, top_k=4)
        assert ei.value.status == kie.KIE_ERR_ARG
    dw.free()
