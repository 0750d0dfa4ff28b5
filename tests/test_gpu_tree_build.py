"""GPU parity of the accum_logp tree construction with its oracle: parent,
tokens, depth and fp32 scores bit-exact, node counts equal."""
import numpy as np
import pytest
import torch

import oracle
from tree_verification_jsv_b200 import jsv, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_jsv_b200 import build
    build.build()
    jsv.load()


def _run(logp, toks, root, budget):
    B, D, k = logp.shape
    dev = lambda a, dt: torch.as_tensor(np.ascontiguousarray(a, dtype=dt)).cuda()
    par = torch.empty((B, budget), dtype=torch.int32, device="cuda")
    tok = torch.empty_like(par)
    dep = torch.empty_like(par)
    sc = torch.empty((B, budget), dtype=torch.float32, device="cuda")
    nn = torch.empty(B, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    jsv.jsv_accum_logp_tree(dev(logp, np.float32), dev(toks, np.int32), dev(root, np.int32), B, D, k, budget,
                            par, tok, dep, sc, nn, status)
    torch.cuda.synchronize()
    return (par.cpu().numpy(), tok.cpu().numpy(), dep.cpu().numpy(), sc.cpu().numpy(), nn.cpu().numpy(),
            int(status.item()))


def _check(logp, toks, root, budget):
    par, tok, dep, sc, nn, st = _run(logp, toks, root, budget)
    assert st == 0
    for b in range(logp.shape[0]):
        ref = oracle.accum_logp_tree(logp[b], toks[b], root[b], budget)
        n = len(ref["parent"])
        assert nn[b] == n
        assert np.array_equal(par[b, :n], ref["parent"])
        assert np.array_equal(tok[b, :n], ref["tokens"])
        assert np.array_equal(dep[b, :n], ref["depth"])
        assert np.array_equal(sc[b, :n].view(np.uint32), ref["score"].view(np.uint32))
        assert np.all(par[b, n:] == -1) and np.all(dep[b, n:] == -1)


@pytest.mark.parametrize("B,D,k,budget", [(1, 8, 4, 64), (1, 16, 8, 256), (4, 16, 8, 512), (16, 12, 4, 128),
                                          (3, 20, 7, 128), (2, 32, 32, 512), (5, 3, 2, 100)])
def test_matches_oracle(B, D, k, budget):
    logp, toks, root = synth.draft_topk(7 + D * k + budget, B, D, k, 151936)
    _check(logp, toks, root, budget)


def test_exact_ties_and_degenerate_shapes():
    rng = np.random.default_rng(3)
    B, D, k = 6, 6, 5
    u = np.round(rng.random((B, D, k)) * 3) + 1          # few distinct values: many ties
    p = np.sort(u / u.sum(axis=2, keepdims=True), axis=2)[:, :, ::-1]
    logp = np.log(p).astype(np.float32)
    toks = rng.integers(0, 50, (B, D, k)).astype(np.int32)
    root = np.arange(B, dtype=np.int32)
    for budget in (1, 2, 7, 31, 100, 512):
        _check(logp, toks, root, budget)
    # depth 0: the root alone
    _check(np.zeros((2, 0, 3), np.float32), np.zeros((2, 0, 3), np.int32), np.array([4, 5], np.int32), 16)


def test_unsorted_logprobs_are_reported():
    logp, toks, root = synth.draft_topk(1, 2, 4, 3, 100)
    logp = logp.copy()
    logp[1, 2] = logp[1, 2][::-1]                         # request 1: row not sorted
    par, tok, dep, sc, nn, st = _run(logp, toks, root, 20)
    assert st == jsv.JSV_ERR_DEVICE_INPUT
    assert nn[1] == 1 and par[1, 0] == -1 and tok[1, 0] == root[1]
    ref = oracle.accum_logp_tree(logp[0], toks[0], root[0], 20)
    assert np.array_equal(par[0, :len(ref["parent"])], ref["parent"])
