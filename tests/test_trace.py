"""The batch-1 phase breakdown recovers known durations from a synthetic trace (CPU)."""
import numpy as np
import pytest

from bandwidth_bound_stream_b200 import trace as tr


def _synthetic(n_cta, n_tok, L, phase_ns, pos_ns, head_ns):
    ev = tr.batch1_events(L)
    x = np.zeros((n_cta, n_tok, ev), dtype=np.int64)
    for c in range(n_cta):
        for t in range(n_tok):
            now = 1_000_000 * (t + 1) + 7 * c
            x[c, t, 0] = now
            for l in range(L):
                base = 1 + 16 * l
                for i, d in enumerate(phase_ns):
                    now += d
                    x[c, t, base + i] = now
                    if i == 2:
                        bar1_end = now
                x[c, t, base + 15] = bar1_end + pos_ns if c % 2 == 0 else 0  # odd CTAs own no unit
            eh = 1 + 16 * L
            for k, d in enumerate(head_ns):
                now += d
                x[c, t, eh + k] = now
            for k in range(len(tr.RING_PHASES)):  # ring waits: (k + 1) us per layer, head 9 us
                x[c, t, ev - 1 - len(tr.RING_PHASES) + k] = 9000 if k == 4 else (k + 1) * 1000 * L
            x[c, t, ev - 1] = 123_000
    return x


def test_phase_breakdown_recovers_known_durations():
    phase = [4200, 840, 2970, 9080, 1740, 1900, 2500, 11230, 3120, 5750]
    x = _synthetic(4, 3, 5, phase, pos_ns=4720, head_ns=(20320, 2700, 1570))
    out = tr.batch1_phase_us(x, 5)
    for name, d in zip(tr.LAYER_PHASES, phase):
        assert out[name] == pytest.approx(d / 1e3)
    assert out["attention_positions"] == pytest.approx(4.72)
    assert out["attention_publish_merge"] == pytest.approx((9080 - 4720) / 1e3)
    assert out["lm_head_rows"] == pytest.approx(20.32)
    assert out["lm_head_barrier"] == pytest.approx(2.70)
    assert out["argmax"] == pytest.approx(1.57)
    assert out["per_layer"] == pytest.approx(sum(phase) / 1e3)
    assert out["tokens"] == 2 and out["layers_averaged"] == 4
    assert out["ring_wait"] == pytest.approx({"qkv_rows": 1.0, "o_fold": 2.0, "gate_up_rows": 3.0, "down_fold": 4.0,
                                              "lm_head_rows": 9.0})
    assert out["producer_wait_per_token"] == pytest.approx(123.0)


def test_phase_breakdown_single_layer_and_shape_check():
    x = _synthetic(2, 1, 1, [10] * 10, pos_ns=3, head_ns=(5, 6, 7))
    out = tr.batch1_phase_us(x, 1)
    assert out["qkv_rows"] == pytest.approx(0.01) and out["tokens"] == 1 and "per_layer" not in out
    with pytest.raises(ValueError):
        tr.batch1_phase_us(x, 2)
