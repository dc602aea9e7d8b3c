"""The roofline's numerator: algorithmic bytes of one bench launch, recounted from the shape (CPU)."""
import bench
from bandwidth_bound_stream_b200 import synth


def test_algorithmic_bytes_of_the_default_launch():
    # 1.9B shape: 28 layers, d 2048, 16 query / 8 kv heads of 128, ffn 8192, vocab 32000, 2-byte weights
    L, d, Hq, Hkv, D, F, V = 28, 2048, 16, 8, 128, 8192, 32000
    layer = (Hq * D * d + 2 * Hkv * D * d + d * Hq * D + 2 * F * d + d * F + 2 * d) * 2  # QKV, O, gate/up, down, 2 norms
    weights = L * layer + d * 2 + V * d * 2 + d * 2  # + final norm, LM head, one embedding row
    kv_pos = L * Hkv * D * 2 * 2  # K and V of one position, every layer
    prompt, n = 1024, 512
    # token t attends positions 0 .. prompt + t (its own included) and writes one position
    want = sum(weights + (prompt + t + 1) * kv_pos + kv_pos for t in range(n))
    assert bench.algorithmic_bytes(synth.DENSE_1P9B, prompt, n) == want == 1_946_366_771_200


def test_algorithmic_bytes_grow_with_context():
    m = synth.DENSE_8B
    a, b = bench.algorithmic_bytes(m, 4096, 1), bench.algorithmic_bytes(m, 4097, 1)
    assert b - a == m.kv_bytes_per_position() == 32 * 8 * 128 * 2 * 2


def test_fp8_weight_bytes():
    """E4M3 codes (one byte) for every matrix and the LM head, a 4-byte scale per row, 16-bit
    norms and embedding row."""
    L, d, Hq, Hkv, D, F, V = 28, 2048, 16, 8, 128, 8192, 32000
    elems = L * (Hq * D * d + 2 * Hkv * D * d + d * Hq * D + 3 * F * d) + V * d
    rows = L * (Hq * D + 2 * Hkv * D + d + 2 * F + d) + V
    assert synth.DENSE_1P9B.weight_bytes_per_token(fp8=True) == elems + 4 * rows + 2 * (2 * L + 1) * d + 2 * d
    assert abs(synth.DENSE_1P9B.weight_bytes_per_token(fp8=True) / synth.DENSE_1P9B.weight_bytes_per_token() - 0.5) < 0.001
