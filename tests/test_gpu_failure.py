"""Failure detection without a GPU fault: a bounded device wait runs out on
a barrier nothing signals, the kernel reports JSV_ERR_TIMEOUT through the
status word, and the context stays usable for ordinary work."""
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
