"""The batch-1 kernel's phase trace on the GPU (GPU tests): stamps in order, totals sane."""
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


@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_batch1_trace_is_ordered_and_parses(kie, name):
    from bandwidth_bound_stream_b200 import synth, trace
    m = synth.CONFIGS[name]
    n_tok = 4
    dw = kie.DeviceWeights(m)
    with kie.Engine(kie.config(m, max_ctx=64, timeout_ms=5000, idle_ms=50), dw.kie) as eng:
        sid = eng.session_open()
        first = eng.prefill(sid, synth.prompt(m, 9))
        eng.trace_enable(n_tok)
        tok_d = torch.tensor([first], dtype=torch.int32, device="cuda")
        out_d = torch.zeros(n_tok, dtype=torch.int32, device="cuda")
        eng.decode_launch(sid, tok_d.data_ptr(), n_tok, out_d.data_ptr())
        eng.sync()
        tr = eng.trace_read(n_tok)
        eng.trace_enable(0)
    dw.free()
    assert tr.shape == (tr.shape[0], n_tok, trace.batch1_events(m.n_layers))
    x = tr.astype(np.int64)
    for t in range(n_tok):
        stamps = [x[:, t, 0]]
        for l in range(m.n_layers):
            stamps += [x[:, t, 1 + 16 * l + i] for i in range(len(trace.LAYER_PHASES))]
        eh = 1 + 16 * m.n_layers
        stamps += [x[:, t, eh + k] for k in range(3)]
        s = np.stack(stamps, axis=1)
        assert (s > 0).all() and (np.diff(s, axis=1) >= 0).all(), f"token {t}: stamps out of order"
        if t + 1 < n_tok:  # the next token starts after this one's final argmax
            assert (x[:, t + 1, 0] >= x[:, t, eh + 2]).all()
        span = int(s[:, -1].max() - s[:, 0].min())
        waits = x[:, t, -1 - len(trace.RING_PHASES):]
        assert (waits >= 0).all() and (waits <= span).all()
    out = trace.batch1_phase_us(tr, m.n_layers)
    assert out["per_layer"] > 0 and out["tokens"] == n_tok - 1
    assert set(out["ring_wait"]) == set(trace.RING_PHASES)
