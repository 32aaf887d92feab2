"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every spin-wait in the library's kernels is bounded by 1 s of wall-clock
time, after which the kernel records a bit in a device error word and
returns.  fca_selftest_wait_timeout runs that same wait on a barrier phase
that nothing completes; the host must get the word back, and the context
must stay usable for the next decode.
"""
import time

import numpy as np
import pytest

import fca_workloads
import oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_that_runs_out_returns_a_status():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import shared_prefix_kv_fca_b200 as fca
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    word = fca.fca_selftest_wait_timeout()
    dt = time.perf_counter() - t0
    assert word & 1, f"the wait did not report a timeout (word {word:#x})"
    assert 0.9 < dt < 60.0, f"the wait took {dt:.2f} s"

    # the context is still usable: a decode right after matches the oracle
    w = fca_workloads.make("tiny")
    q, k, v, bt, sl = w.torch_inputs("cuda")
    with fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D) as plan:
        out = torch.empty_like(q)
        lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device="cuda")
        fca.fca_decode(q, k, v, plan, out, lse, w.scale)
        assert fca.fca_check_device_status(plan) == 0
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    o = out.float().cpu().numpy().astype(np.float64)
    assert np.abs(o - o_ref).max() <= 1e-2
    assert np.abs(lse.cpu().numpy().astype(np.float64) - l_ref).max() <= 1e-3
