"""Calls from host threads other than the one that first used the library.

Launch attributes (the opt-in to more than 48 KB of shared memory of the
attention kernels) belong to the current device's context, so the library
applies them on every launch rather than once per process: a kernel
launched first from a second thread, or from two threads at once with
distinct buffers, must run and give the bytes a single-threaded call gives.
"""
import threading

import numpy as np
import pytest
import torch

from long_context_hierarchical_b200.synth import make_inputs

pytestmark = pytest.mark.gpu


def _run_in_thread(fn):
    out, err = {}, []

    def body():
        try:
            torch.cuda.set_device(0)
            out["value"] = fn()
            torch.cuda.synchronize()
        except BaseException as e:  # noqa: BLE001 - reported to the main thread
            err.append(e)

    t = threading.Thread(target=body)
    t.start()
    t.join(timeout=600)
    assert not t.is_alive(), "worker thread did not finish"
    if err:
        raise err[0]
    return out["value"]


def test_layer_from_a_second_thread_matches_the_main_thread():
    from long_context_hierarchical_b200 import lh
    B, H, N, p, L, k = 1, 4, 4096, 4, 3, 64
    Q, K, V, dO = (x.cuda() for x in make_inputs(B, H, N, 64, "bf16", seed=2))
    pl = lh.plan(B, H, N, 64, p, L, k, "bf16")

    def layer():
        with torch.cuda.stream(torch.cuda.Stream()):
            O, ctx = lh.forward(pl, Q, K, V)
            lh.set_deterministic(True)
            try:
                g = lh.backward(pl, dO, ctx)
            finally:
                lh.set_deterministic(False)
            torch.cuda.current_stream().synchronize()
        return O, g

    O2, g2 = _run_in_thread(layer)     # the worker thread runs first
    O1, g1 = layer()
    torch.cuda.synchronize()
    assert torch.equal(O1, O2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    lh.device_status()


def test_two_threads_at_once_with_distinct_buffers():
    from long_context_hierarchical_b200 import lh
    S, BH = 2304, 4
    g = np.random.default_rng(5)
    inputs = [[torch.from_numpy(g.standard_normal((BH, S, 64))).to("cuda", torch.bfloat16)
               for _ in range(3)] for _ in range(2)]
    ref = [lh.attn_fwd(*x) for x in inputs]
    torch.cuda.synchronize()
    results = [None, None]
    errors = []
    barrier = threading.Barrier(2)

    def worker(i):
        try:
            torch.cuda.set_device(0)
            barrier.wait(timeout=60)
            with torch.cuda.stream(torch.cuda.Stream()):
                for _ in range(3):
                    results[i] = lh.attn_fwd(*inputs[i])
                torch.cuda.current_stream().synchronize()
        except BaseException as e:  # noqa: BLE001 - reported to the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=600)
    assert not any(t.is_alive() for t in threads)
    assert not errors, errors
    for (o, l), (ro, rl) in zip(results, ref):
        assert torch.equal(o, ro) and torch.equal(l, rl)
    lh.device_status()
