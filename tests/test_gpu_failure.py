"""Failure detection without a GPU fault: a bounded device wait runs out on
a barrier nothing signals, the kernel reports JSV_ERR_TIMEOUT through the
status word, and the context stays usable for ordinary work -- for the
stand-alone self-test kernel and for the LM head itself."""
import math
import time

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    from tree_verification_jsv_b200 import build, jsv
    build.build()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    jsv.jsv_selftest_wait_timeout(status, 20_000)      # 20 ms limit
    torch.cuda.synchronize()
    assert int(status.item()) == jsv.JSV_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    # the context is still fine: an ordinary LM-head call works afterwards
    T, d, V = 8, 128, 500
    g = torch.Generator(device="cuda").manual_seed(0)
    H = (torch.randn(T, d, device="cuda", generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W = (torch.randn(V, d, device="cuda", generator=g) / math.sqrt(d)).to(torch.bfloat16)
    arg = torch.empty(T, dtype=torch.int32, device="cuda")
    ws = torch.zeros(jsv.jsv_lmhead_argmax_workspace_size(T, d, V), dtype=torch.uint8, device="cuda")
    jsv.jsv_lmhead_argmax(H, W, T, d, V, arg, None, ws)
    torch.cuda.synchronize()
    a = arg.cpu().numpy()
    assert np.all((a >= 0) & (a < V))


def test_selftest_rejects_bad_limits():
    from tree_verification_jsv_b200 import jsv
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(jsv.JsvError):
        jsv.jsv_selftest_wait_timeout(status, 0)
    with pytest.raises(jsv.JsvError):
        jsv.jsv_selftest_wait_timeout(status, 3_000_000)


def _certified_case(T, d, V, seed):
    import oracle
    from helpers import bf16
    rng = np.random.default_rng(seed)
    H = bf16(rng.standard_normal((T, d)) / math.sqrt(d))
    W = bf16(rng.standard_normal((V, d)) / math.sqrt(d))
    a, t1, t2 = oracle.lmhead_top2(H, W)
    ok, _ = oracle.certify_margin(H, W, a, t1, t2)
    assert ok.mean() > 0.8
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return dev(H), dev(W), a, ok


# T = 64 runs the single-CTA form (148 CTAs, one wave, so the first CTA always
# starts and takes the injected wait); T = 256 runs the CTA-pair form.
@pytest.mark.parametrize("T", [64, 256])
@pytest.mark.parametrize("noalloc", [False, True], ids=["workspace", "noalloc"])
def test_lmhead_timeout_is_reported_and_scratch_left_clean(T, noalloc):
    """The LM head's own timeout path: one CTA's wait gives up (a wait that
    nothing signals, injected before the CTA issues any copy), the call
    reports JSV_ERR_TIMEOUT through the status word, and the scratch it used
    -- a caller workspace or the no-alloc entry point's array -- is left
    zeroed, so the next ordinary call on it matches the oracle."""
    from tree_verification_jsv_b200 import build, jsv
    build.build()
    d, V = 256, 6000
    H, W, want, ok = _certified_case(T, d, V, seed=900 + T)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    arg = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    ws = None if noalloc else torch.zeros(jsv.jsv_lmhead_argmax_workspace_size(T, d, V), dtype=torch.uint8,
                                         device="cuda")
    t0 = time.time()
    jsv.jsv_selftest_lmhead_timeout(H, W, T, d, V, arg, None, ws, status, 20_000)
    torch.cuda.synchronize()
    assert time.time() - t0 < 30.0
    assert int(status.item()) == jsv.JSV_ERR_TIMEOUT
    if ws is not None:
        assert not ws.any().item()
    status.zero_()
    arg2 = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    if noalloc:
        jsv.jsv_lmhead_argmax_noalloc(H, W, T, d, V, arg2, None, dev_status=status)
    else:
        jsv.jsv_lmhead_argmax(H, W, T, d, V, arg2, None, ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = arg2.cpu().numpy()
    assert np.array_equal(got[ok], want[ok])
    if ws is not None:
        assert not ws.any().item()


def test_lmhead_timeout_selftest_rejects_bad_arguments():
    from tree_verification_jsv_b200 import jsv
    T, d, V = 8, 128, 500
    H = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((V, d), dtype=torch.bfloat16, device="cuda")
    arg = torch.empty(T, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for limit in (0, 3_000_000):
        with pytest.raises(jsv.JsvError):
            jsv.jsv_selftest_lmhead_timeout(H, W, T, d, V, arg, None, None, status, limit)
    with pytest.raises(jsv.JsvError):
        jsv.jsv_selftest_lmhead_timeout(H, W, T, d, V, arg, None, None, None, 10)
