"""GPU parity of the whole verify step against the oracle, on every named
workload at full size, through the C ABI.

Bit-exact: argmax (certified goldens), accepted path, accept length, bonus,
new lengths and the ENTIRE K and V cache buffers after compaction.
Attention: within the tolerance in ``helpers.attention_close`` on all rows
(small workloads) or on a seeded sample of rows the oracle computes one by
one (large workloads).
"""
import numpy as np
import pytest
import torch

from helpers import assert_step_matches_oracle, golden_workload

pytestmark = pytest.mark.gpu

WORKLOADS = ["tiny", "8b_64", "8b_256", "ragged16", "30b_512x4"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_jsv_b200 import build, jsv
    build.build()
    jsv.load()


@pytest.mark.parametrize("name", WORKLOADS)
def test_verify_step_matches_oracle(name):
    from tree_verification_jsv_b200.step import VerifyStep
    wl, tokens, gold_arg = golden_workload(name)
    k0, v0 = wl.k_cache.copy(), wl.v_cache.copy()
    st = VerifyStep(wl, tokens)
    st.run()
    torch.cuda.synchronize()
    assert_step_matches_oracle(st, wl, tokens, gold_arg, k0, v0, name)
