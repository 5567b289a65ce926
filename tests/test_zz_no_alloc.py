"""The allocation-free attention backward (lh_attn_bwd_static).

Some callers hold only their inputs and outputs and cannot allocate device
memory; lh_attn_bwd_static serves them by keeping its scratch (the row term D)
in a fixed array inside the library.  This file is collected after the stage
and whole-layer tests so that a run stopping at the first failure has run
them before it; it passes alone in a fresh process and after the rest of the
suite.
"""
import ctypes

import pytest
import torch

from long_context_hierarchical_b200.synth import make_inputs
from tests.helpers import assert_close, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,BH,S", [("bf16", 6, 1000), ("f32", 2, 300)])
def test_static_scratch_matches_workspace_entry_point(dtype, BH, S):
    from long_context_hierarchical_b200 import lh
    Q, K, V, dO = make_inputs(1, BH, S, 64, dtype, seed=11, device="cuda")
    O, lse = lh.attn_fwd(Q, K, V)
    ref = lh.attn_bwd(Q, K, V, O, lse, dO, None)  # caller-provided workspace
    torch.cuda.synchronize()
    dt = Q.dtype
    for _ in range(2):  # two calls in a row share the library's scratch
        got = lh.attn_bwd_static(Q, K, V, O, lse, dO)
        torch.cuda.synchronize()
        for g, r, name in zip(got, ref, ("dQ", "dK", "dV")):
            assert_close(np64(g), np64(r), dt, name)


def test_static_scratch_rejects_oversized_problems():
    from long_context_hierarchical_b200 import lh
    p = ctypes.c_void_p(1 << 20)
    st = lh.LIB.lh_attn_bwd_static(2048, 1024, 64, lh.LH_BF16, p, p, p, p, p, p, p, p, p, None)
    assert st == lh.LH_ERR_WORKSPACE
    assert b"LH_ATTN_BWD_STATIC_MAX_ROWS" in lh.LIB.lh_last_error()
