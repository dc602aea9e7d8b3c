"""The seeded input generator: published splitmix64 vector, counter form, distributions, rounding."""
import os

import numpy as np
import torch

from bandwidth_bound_stream_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_vector():
    want = [int(l) for l in open(os.path.join(GOLDEN, "splitmix64_1234567.txt")) if not l.startswith("#")]
    assert synth.splitmix64_sequence(1234567, 5) == want


def test_counter_form_equals_sequential_stream():
    for seed, stream in [(0, 0x100), (7, 0x10000003), (2**63 + 5, 1)]:
        seq = synth.splitmix64_sequence(synth.stream_key(seed, stream), 40)
        assert [synth.word(seed, stream, i) for i in range(40)] == seq


def test_normals_have_requested_moments():
    x = synth.normal_u16(0, 0x105, 1 << 20, synth.FP16).view(np.float16).astype(np.float64)
    assert abs(x.mean()) < 3 * 0.02 / np.sqrt(x.size) * 2
    assert abs(x.std() - 0.02) < 2e-4
    # Box-Muller pairs are uncorrelated
    assert abs(np.corrcoef(x[0::2], x[1::2])[0, 1]) < 5e-3
    # tails of a normal: ~0.27% beyond 3 sigma
    assert 0.002 < np.mean(np.abs(x) > 0.06) < 0.0035


def test_offsets_draw_the_same_elements():
    full = synth.normal_u16(3, 0x110, 1001, synth.BF16)
    part = synth.normal_u16(3, 0x110, 500, synth.BF16, offset=301)
    assert np.array_equal(full[301:801], part)


def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.normal(0, 0.02, 20000), rng.normal(0, 1e-6, 2000), rng.normal(0, 3e4, 2000),
                           [65519.0, 65520.0, 6.0e-8, 2.98e-8, 0.0, -0.0]]).astype(np.float32)
    want = vals.astype(np.float16).view(np.uint16)
    got = np.array([synth.round_f32(float(v), synth.FP16) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(2)
    vals = rng.normal(0, 0.02, 20000).astype(np.float32)
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([synth.round_f32(float(v), synth.BF16) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_tokens_and_tick_lengths_in_range():
    cfg = synth.TINY
    t = synth.prompt(cfg, 5000)
    assert t.min() >= 0 and t.max() < cfg.vocab
    assert len(set(t.tolist())) > 2700  # ~2888 expected distinct of 4096
    assert not np.array_equal(t[:100], synth.prompt(cfg, 100, session=1))
    lens = [synth.tick_prompt_length(s) for s in range(56)]
    assert min(lens) >= 1000 and max(lens) <= 1500 and len(set(lens)) > 30


def test_param_counts_match_the_named_shapes():
    assert synth.DENSE_1P9B.n_params() == 1_892_796_416
    assert synth.DENSE_8B.n_params() == 8_030_261_248
    assert synth.TICK_10P8B.n_params() == 10_731_524_096
    # one decode step streams all weights except the embedding table, plus one embedding row
    assert synth.DENSE_1P9B.weight_bytes_per_token() == 3_654_524_928
