"""The verify step captured in a CUDA graph: its replay matches the oracle
(argmax, walk, compaction, attention output) on the tiny and the
Qwen3-8B-shaped 64- and 256-node workloads, and gives the same bytes as the
eager step; the end-to-end form through host buffers gives the device
step's outputs."""
import numpy as np
import pytest
import torch

from helpers import assert_step_matches_oracle, golden_workload

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "8b_64", "8b_256"])
def test_graph_replay_matches_oracle(name):
    """Capture, restore the caches the capture's warm-up step compacted, then
    replay twice on the restored caches: each replay is one whole verify
    step and must match the oracle (the second replay restores the caches
    first, so it starts from the same state)."""
    from tree_verification_jsv_b200 import build
    from tree_verification_jsv_b200.step import VerifyStep
    build.build()
    wl, tokens, gold_arg = golden_workload(name)
    k0, v0 = wl.k_cache.copy(), wl.v_cache.copy()
    st = VerifyStep(wl, tokens)
    kd, vd = st.k_cache.clone(), st.v_cache.clone()
    st.capture()                            # runs one eager step first
    for rep in range(2):
        st.k_cache.copy_(kd)
        st.v_cache.copy_(vd)
        st.status.zero_()
        st.out.zero_()
        st.argmax.fill_(-1)
        st.path.fill_(-9)
        torch.cuda.synchronize()
        st.replay()
        torch.cuda.synchronize()
        assert_step_matches_oracle(st, wl, tokens, gold_arg, k0, v0, f"{name} replay {rep}")


@pytest.mark.parametrize("name", ["tiny", "8b_64"])
def test_graph_replay_matches_eager_step(name):
    from tree_verification_jsv_b200 import build
    from tree_verification_jsv_b200.step import VerifyStep
    build.build()
    wl, tokens, _ = golden_workload(name)
    eager = VerifyStep(wl, tokens)
    eager.run()
    torch.cuda.synchronize()

    graphed = VerifyStep(wl, tokens)
    k0, v0 = graphed.k_cache.clone(), graphed.v_cache.clone()
    graphed.capture()                       # runs one eager step first
    graphed.k_cache.copy_(k0)
    graphed.v_cache.copy_(v0)
    graphed.status.zero_()
    graphed.replay()
    torch.cuda.synchronize()
    assert int(graphed.status.item()) == 0
    for name_ in ("out", "argmax", "max_logit", "path", "accept_len", "bonus", "new_len", "k_cache", "v_cache"):
        assert np.array_equal(_bits(getattr(eager, name_)), _bits(getattr(graphed, name_))), name_


@pytest.mark.parametrize("name", ["tiny", "8b_64"])
def test_host_step_matches_device_step(name):
    """run_host (inputs copied up from pinned host memory, outputs copied
    back) returns the same outputs as the device-resident step, over several
    steps in a row, and leaves the same caches."""
    from tree_verification_jsv_b200 import build
    from tree_verification_jsv_b200.step import VerifyStep
    build.build()
    wl, tokens, _ = golden_workload(name)
    dev = VerifyStep(wl, tokens)
    host = VerifyStep(wl, tokens)
    outs = []
    for _ in range(3):
        dev.run()
        got = host.run_host()
        torch.cuda.synchronize()            # the host views are filled asynchronously
        outs.append({k: v.clone() for k, v in got.items()})
    assert int(host.status.item()) == 0 and int(dev.status.item()) == 0
    for k in ("path", "accept_len", "bonus", "new_len"):
        assert np.array_equal(outs[-1][k].numpy(), getattr(dev, k).cpu().numpy()), k
    for name_ in ("out", "argmax", "k_cache", "v_cache"):
        assert np.array_equal(_bits(getattr(dev, name_)), _bits(getattr(host, name_))), name_


def _changed_tokens(wl, tokens, gold_arg):
    """Draft tokens that the oracle accepts along other paths: every other
    node's token moved off its value, and if that changes no path, node 1 of
    each request given its parent's argmax (a match at depth 1)."""
    import oracle
    walk = lambda tok: oracle.accept_batch(wl.node_offsets, wl.parent, tok, gold_arg)
    changed = np.where(np.arange(tokens.size) % 2 == 1, (tokens + 1) % wl.V, tokens).astype(np.int32)
    if walk(changed) == walk(tokens):
        for b in range(len(wl.node_offsets) - 1):
            base = int(wl.node_offsets[b])
            if int(wl.node_offsets[b + 1]) - base > 1:
                changed[base + 1] = gold_arg[base + int(wl.parent[base + 1])]
    assert walk(changed) != walk(tokens)
    return changed


@pytest.mark.parametrize("name", ["tiny", "8b_64"])
def test_host_graph_matches_oracle(name):
    """The end-to-end step from one CUDA graph (copy up, the calls, copy back)
    matches the oracle, and its input copy reads the pinned arena when the
    graph runs: draft tokens changed on the host between replays change the
    accepted paths as the oracle says, and the returned host views equal the
    device outputs."""
    from tree_verification_jsv_b200 import build
    from tree_verification_jsv_b200.step import VerifyStep
    build.build()
    wl, tokens, gold_arg = golden_workload(name)
    k0, v0 = wl.k_cache.copy(), wl.v_cache.copy()
    st = VerifyStep(wl, tokens)
    kd, vd = st.k_cache.clone(), st.v_cache.clone()
    st.capture_host()                       # runs one eager end-to-end step first
    tokens = np.asarray(tokens, dtype=np.int32)
    changed = _changed_tokens(wl, tokens, gold_arg)
    for rep, tok in enumerate((tokens, changed, tokens)):
        st.host_inputs()["tokens"].copy_(torch.from_numpy(tok))
        st.k_cache.copy_(kd)
        st.v_cache.copy_(vd)
        st.status.zero_()
        st.out.zero_()
        st.argmax.fill_(-1)
        st.path.fill_(-9)
        torch.cuda.synchronize()
        got = st.replay_host()
        torch.cuda.synchronize()
        assert_step_matches_oracle(st, wl, tok, gold_arg, k0, v0, f"{name} host replay {rep}")
        for k in ("path", "accept_len", "bonus", "new_len"):
            assert np.array_equal(got[k].numpy(), getattr(st, k).cpu().numpy()), (rep, k)
