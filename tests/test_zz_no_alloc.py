"""The allocation-free attention entry point (kie_flash_decode_noalloc), called through the C ABI.

It is for callers of this library that cannot allocate device memory while they run (a
memory budget fixed at start-up, memory owned by another framework's allocator, or a loop
that cannot afford the stall of cudaMalloc/cudaFree). Its scratch is one static device array
shared by all calls, so this test makes two calls in a row, on different inputs, and checks
each against kie_flash_decode (which takes caller-allocated scratch) with the tolerance the
attention parity tests use. This file is collected last on purpose.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _case(kie, Hq, Hkv, D, ctx, dtype, seed):
    from bandwidth_bound_stream_b200 import synth
    stride = ctx + 5
    q = torch.tensor(np.random.default_rng(seed).normal(0, 1, (Hq, D)), dtype=torch.float32, device="cuda")
    K = synth.normal_u16(seed, 0x7101, Hkv * stride * D, dtype, std=1.0)
    V = synth.normal_u16(seed, 0x7102, Hkv * stride * D, dtype, std=1.0)
    _case.host = (K.reshape(Hkv, stride, D), V.reshape(Hkv, stride, D))
    k = torch.from_numpy(K.view(np.int16)).cuda()
    v = torch.from_numpy(V.view(np.int16)).cuda()
    # reference: the entry point with caller-allocated scratch
    nbytes = kie.flash_decode_scratch_bytes(Hq, Hkv, D, ctx)
    scratch = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    ref = torch.full((Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    assert kie.flash_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), Hq, Hkv, D, ctx, stride, dtype,
                            ref.data_ptr(), scratch.data_ptr(), nbytes) == kie.KIE_OK
    return q, k, v, stride, ref, _case.host


def test_noalloc_matches_flash_decode_on_two_calls_in_a_row():
    """Both entry points against each other and against the oracle's attention (a bug the two
    share would pass the first comparison, not the second)."""
    from bandwidth_bound_stream_b200 import kie
    from oracle import oracle as orc
    cases = [(16, 8, 128, 1300, 0, 1), (32, 8, 128, 777, 1, 2)]  # 1.9B-like fp16, then 8B-like bf16
    prepared = [_case(kie, *c) for c in cases]
    torch.cuda.synchronize()
    for (Hq, Hkv, D, ctx, dtype, _), (q, k, v, stride, ref, (K, V)) in zip(cases, prepared):
        out = torch.full((Hq, D), float("nan"), dtype=torch.float32, device="cuda")
        st = kie.flash_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), Hq, Hkv, D, ctx, stride, dtype,
                                      out.data_ptr())
        assert st == kie.KIE_OK
        got, want = out.cpu().numpy(), ref.cpu().numpy()
        assert np.isfinite(got).all()
        np.testing.assert_allclose(got, want, rtol=0, atol=2e-5 * max(1.0, float(np.abs(want).max())))
        qf = q.cpu().numpy().astype(np.float64)  # the fp32 query the kernels read
        for h in range(Hq):
            g = h * Hkv // Hq
            o = orc.attention(qf[h], K[g, :ctx], V[g, :ctx], dtype)
            np.testing.assert_allclose(got[h], o, rtol=0, atol=2e-5 * max(1.0, float(np.abs(o).max())))


def test_noalloc_rejects_shapes_beyond_its_array():
    from bandwidth_bound_stream_b200 import kie
    # 128 heads x 128 dims at a long context needs more scratch than the static array holds
    assert kie.flash_decode_scratch_bytes(128, 128, 128, 40000) > kie.FLASH_DECODE_NOALLOC_MAX_BYTES
    out = torch.empty(1, dtype=torch.float32, device="cuda")
    st = kie.flash_decode_noalloc(out.data_ptr(), out.data_ptr(), out.data_ptr(), 128, 128, 128, 40000, 40000, 0,
                                  out.data_ptr())
    assert st == kie.KIE_ERR_CAPACITY
