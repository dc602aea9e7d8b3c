"""Checks run under the diagnostic build of the engine (KIE_VARIANT=debug; test helper).

In that build every kernel write to global memory checks its index (an out-of-range one is
skipped and recorded as a device error) and every engine buffer lies between guard words
that the host checks after each command; it stands in for a memory checker, which this
machine does not offer. Run as a program: both kernels on the tiny and ragged models against
the oracle (batch-1 decode on both K/V paths, the tick's chunked prefill and a two-step
tick), then a guard word changed from the host must be reported. Exit status 0 when all hold.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def batch1(kie, m, kv_path):
    import numpy as np
    import torch
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    from tests.parity import assert_reports, compare_step
    dw = kie.DeviceWeights(m, host_copy=True)
    orc = OracleModel(m, dw.host, 48)
    prompt = synth.prompt(m, 20)
    logits = torch.empty(m.vocab, dtype=torch.float32, device="cuda")
    with kie.Engine(kie.config(m, max_ctx=48, timeout_ms=5000, idle_ms=50, b1_kv_path=kv_path), dw.kie) as eng:
        sid = eng.session_open()
        first = eng.prefill(sid, prompt)
        ref = orc.prefill(prompt)
        reports = [compare_step(ref, first, ref, m.dtype)]
        tok = int(np.argmax(ref))
        for _ in range(8):
            out = eng.decode_step(sid, tok, logits.data_ptr())
            ref = orc.step(tok)
            reports.append(compare_step(logits.cpu().numpy(), out, ref, m.dtype))
            tok = int(np.argmax(ref))
        eng.sync()
    dw.free()
    return assert_reports(reports, m.dtype)


def tick(kie, m):
    import numpy as np
    import torch
    from bandwidth_bound_stream_b200 import synth
    from oracle.oracle import OracleModel
    from tests.parity import assert_reports, compare_step
    dw = kie.DeviceWeights(m, host_copy=True)
    reports = []
    with kie.Engine(kie.config(m, max_sessions=2, max_ctx=160, timeout_ms=5000, idle_ms=50,
                               modes=kie.KIE_MODE_TICK), dw.kie) as eng:
        sids = [eng.session_open(), eng.session_open()]
        orcs = [OracleModel(m, dw.host, 160) for _ in sids]
        toks = []
        for i, sid in enumerate(sids):
            p = synth.prompt(m, 70 + 41 * i, session=i + 1)  # crosses a 64-position chunk
            first = eng.prefill(sid, p)
            ref = orcs[i].prefill(p)
            reports.append(compare_step(ref, first, ref, m.dtype))
            toks.append(int(np.argmax(ref)))
        lg = torch.empty((2, 2, m.vocab), dtype=torch.float32, device="cuda")
        out = eng.tick(sids, toks, 2, lg.data_ptr())
        got = lg.cpu().numpy()
        for i in range(2):
            ref1 = orcs[i].step(toks[i])
            reports.append(compare_step(got[0, i], int(out[0, i]), ref1, m.dtype))
        eng.sync()
    dw.free()
    return assert_reports(reports, m.dtype)


def guard_words_are_checked(kie, m):
    """A byte written from the host just past the K cache (into its trailing guard words) makes
    the next check report a device error."""
    import torch
    from tests.inject import device_view
    dw = kie.DeviceWeights(m)
    with kie.Engine(kie.config(m, max_sessions=2, max_ctx=16, timeout_ms=5000, idle_ms=50), dw.kie) as eng:
        a, b = eng.session_open(), eng.session_open()
        eng.prefill(b, [1, 2, 3])
        eng.sync()
        kp, _ = eng.session_kv(b)
        stride = m.n_layers * m.n_kv_heads * 16 * m.head_dim  # elements of one session's K
        device_view(kp + 2 * stride, 2).fill_(7)  # the first bytes after the last session's K (2-byte elements)
        torch.cuda.synchronize()
        try:
            eng.sync()
        except kie.KieError as e:
            assert e.status == kie.KIE_ERR_DEVICE and "guard" in str(e), str(e)
        else:
            raise AssertionError("a changed guard word went unreported")
    dw.free()


def main() -> int:
    assert os.environ.get("KIE_VARIANT") == "debug", "run with KIE_VARIANT=debug"
    from bandwidth_bound_stream_b200 import kie, synth
    assert kie.LIB_PATH.endswith("libkie_debug.so"), kie.LIB_PATH
    for name in ("tiny", "ragged"):
        m = synth.CONFIGS[name]
        for kv_path in (1, 2):
            print(f"{name} batch-1, K/V path {kv_path}: max |logit diff| {batch1(kie, m, kv_path):.2e}", flush=True)
        print(f"{name} tick: max |logit diff| {tick(kie, m):.2e}", flush=True)
    guard_words_are_checked(kie, synth.CONFIGS["tiny"])
    print("guard words: a changed word is reported", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
