"""The allocation-free LM-head entry point gives the same result as the
workspace entry point and as the oracle.

jsv_lmhead_argmax_noalloc serves callers that cannot allocate device memory
where they run the verify step (inside a CUDA-graph capture, in a plugin
whose host owns every allocation, or in a loop that cannot pay for
cudaMalloc's synchronisation).  Its scratch is a fixed array inside the
library, shared by every call and kept between calls, so these tests run it
several times in a row -- larger then smaller, and smaller then larger up to
the array's node limit, so a stale key or completion counter left by one call
would show up in the next -- and compare every result with
jsv_lmhead_argmax (which takes its scratch from the caller) and, on the rows
whose choice no fp32 summation order can change, with the fp64 oracle.

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


def _bf16_pair(rng, shape, scale):
    """(host bf16 bits, device tensor) of a seeded N(0, scale^2) draw."""
    from tree_verification_jsv_b200 import synth
    bits = synth.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(scale))
    return bits, torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _oracle(Hb, Wb):
    """Oracle argmax and max logit, and the rows whose argmax is certified."""
    import oracle
    a, t1, t2 = oracle.lmhead_top2(Hb, Wb)
    ok, _ = oracle.certify_margin(Hb, Wb, a, t1, t2)
    assert ok.mean() > 0.8
    return a, t1, ok


def _with_workspace(lib, H, W, T, d, V):
    arg = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    ml = torch.zeros(T, dtype=torch.float32, device="cuda")
    ws = torch.zeros(lib.jsv_lmhead_argmax_workspace_size(T, d, V), dtype=torch.uint8, device="cuda")
    st = lib.jsv_lmhead_argmax(H.data_ptr(), W.data_ptr(), T, d, V, arg.data_ptr(), ml.data_ptr(),
                               ws.data_ptr(), ws.numel(), None, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return arg, ml


def _no_alloc(lib, H, W, T, d, V, status=None):
    arg = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    ml = torch.zeros(T, dtype=torch.float32, device="cuda")
    st = lib.jsv_lmhead_argmax_noalloc(H.data_ptr(), W.data_ptr(), T, d, V, arg.data_ptr(),
                                       ml.data_ptr(), None if status is None else status.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == 0
    return arg, ml


def _check(got, ref, orc, V):
    (ga, gm), (ra, rm), (oa, ot1, ok) = got, ref, orc
    ga, gm, ra, rm = ga.cpu().numpy(), gm.cpu().numpy(), ra.cpu().numpy(), rm.cpu().numpy()
    assert np.all((ga >= 0) & (ga < V))
    assert np.array_equal(ga, ra)                  # argmax: bit-exact against the workspace entry point
    assert np.allclose(gm, rm, rtol=1e-4, atol=1e-5)
    assert np.array_equal(ga[ok], oa[ok])          # and against the oracle on certified rows
    assert np.allclose(gm[ok], ot1[ok], rtol=1e-4, atol=1e-5)


def test_no_alloc_matches_workspace_entry_point_twice(lib):
    rng = np.random.default_rng(2024)
    cases = [(300, 512, 5003), (37, 256, 2048)]     # big first, then small: stale keys would show
    inputs, orcs = [], []
    for T, d, V in cases:
        Hb, H = _bf16_pair(rng, (T, d), 1 / math.sqrt(d))
        Wb, W = _bf16_pair(rng, (V, d), 1 / math.sqrt(d))
        inputs.append((H, W, T, d, V))
        orcs.append(_oracle(Hb, Wb))
    refs = [_with_workspace(lib, *x) for x in inputs]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = [_no_alloc(lib, *x, status=status) for x in inputs]
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for g, r, o, x in zip(got, refs, orcs, inputs):
        _check(g, r, o, x[4])


def test_no_alloc_small_then_at_the_node_limit_then_small(lib):
    """Back-to-back calls on one stream with no synchronisation between them:
    37 nodes, then JSV_NOALLOC_MAX_NODES (every key and the counter slot of
    the array in use; 32 node groups on CTA pairs), then 300 nodes.  The
    completion counter sits after each call's last key, so each call's
    counter slot is an earlier or later call's key."""
    from tree_verification_jsv_b200 import jsv
    rng = np.random.default_rng(77)
    cases = [(37, 256, 2048), (jsv.NOALLOC_MAX_NODES, 64, 520), (300, 128, 3001)]
    inputs, orcs = [], []
    for T, d, V in cases:
        Hb, H = _bf16_pair(rng, (T, d), 1 / math.sqrt(d))
        Wb, W = _bf16_pair(rng, (V, d), 1 / math.sqrt(d))
        inputs.append((H, W, T, d, V))
        orcs.append(_oracle(Hb, Wb))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = [_no_alloc(lib, *x, status=status) for x in inputs]
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    refs = [_with_workspace(lib, *x) for x in inputs]
    torch.cuda.synchronize()
    for g, r, o, x in zip(got, refs, orcs, inputs):
        _check(g, r, o, x[4])


def test_no_alloc_rejects_oversized_trees(lib):
    from tree_verification_jsv_b200 import jsv
    T = jsv.NOALLOC_MAX_NODES + 1
    st = lib.jsv_lmhead_argmax_noalloc(ctypes.c_void_p(256), ctypes.c_void_p(256), T, 64, 10,
                                       ctypes.c_void_p(256), None, None, None)
    assert st == jsv.JSV_ERR_UNSUPPORTED
