"""The allocation-free LM-head entry point gives the same result as the
workspace entry point.

jsv_lmhead_argmax_noalloc serves callers that cannot allocate device memory
where they run the verify step (inside a CUDA-graph capture, in a plugin
whose host owns every allocation, or in a loop that cannot pay for
cudaMalloc's synchronisation).  Its scratch is a fixed array inside the
library, shared by every call and kept between calls, so this test runs it
twice in a row -- with a larger problem first and a smaller one second, so
stale keys from the first call would show up -- and compares both with
jsv_lmhead_argmax, which takes its scratch from the caller.

This file is collected last on purpose.  It passes alone in a fresh process
and after the rest of the suite.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from tree_verification_jsv_b200 import build, jsv
    build.build()
    return jsv.load()


def _bf16_dev(rng, shape, scale):
    from tree_verification_jsv_b200 import synth
    bits = synth.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(scale))
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _with_workspace(lib, H, W, T, d, V):
    arg = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    ml = torch.zeros(T, dtype=torch.float32, device="cuda")
    ws = torch.zeros(lib.jsv_lmhead_argmax_workspace_size(T, d, V), dtype=torch.uint8, device="cuda")
    st = lib.jsv_lmhead_argmax(H.data_ptr(), W.data_ptr(), T, d, V, arg.data_ptr(), ml.data_ptr(),
                               ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return arg, ml


def _no_alloc(lib, H, W, T, d, V):
    arg = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    ml = torch.zeros(T, dtype=torch.float32, device="cuda")
    st = lib.jsv_lmhead_argmax_noalloc(H.data_ptr(), W.data_ptr(), T, d, V, arg.data_ptr(),
                                       ml.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return arg, ml


def test_no_alloc_matches_workspace_entry_point_twice(lib):
    rng = np.random.default_rng(2024)
    cases = [(300, 512, 5003), (37, 256, 2048)]     # big first, then small: stale keys would show
    inputs = []
    for T, d, V in cases:
        H = _bf16_dev(rng, (T, d), 1 / math.sqrt(d))
        W = _bf16_dev(rng, (V, d), 1 / math.sqrt(d))
        inputs.append((H, W, T, d, V))
    refs = [_with_workspace(lib, *x) for x in inputs]
    got = [_no_alloc(lib, *x) for x in inputs]
    torch.cuda.synchronize()
    for (ra, rm), (ga, gm), (_, _, T, d, V) in zip(refs, got, inputs):
        ra, ga = ra.cpu().numpy(), ga.cpu().numpy()
        assert np.all((ga >= 0) & (ga < V))
        assert np.array_equal(ga, ra)                  # argmax: bit-exact
        assert np.allclose(gm.cpu().numpy(), rm.cpu().numpy(), rtol=1e-4, atol=1e-5)


def test_no_alloc_rejects_oversized_trees(lib):
    from tree_verification_jsv_b200 import jsv
    T = jsv.NOALLOC_MAX_NODES + 1
    st = lib.jsv_lmhead_argmax_noalloc(ctypes.c_void_p(256), ctypes.c_void_p(256), T, 64, 10,
                                       ctypes.c_void_p(256), None, None)
    assert st == jsv.JSV_ERR_UNSUPPORTED
