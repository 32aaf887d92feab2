"""fca_paged_decode_static: the flat paged decode that allocates nothing.

Its work list and partials live in the library's fixed device array instead
of a plan's workspace.  The GPU tests call it twice in a row through the C
ABI and compare each result with fca_flat_decode (the existing entry point
running the same kernels from a plan) on the same inputs, within twice the
oracle tolerance (each side is within the oracle tolerance of the exact
result), and with the oracle itself.  The file is named to be
collected last, so it also runs after every other test has used the device.
"""
import ctypes

import numpy as np
import pytest

import fca_workloads
import oracle

TOL_MAX, TOL_MEAN, TOL_LSE = 1e-2, 1e-3, 1e-3


def _torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _flat(w, q, k, v, bt, sl):
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    plan = fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D, flat=True)
    out = torch.empty_like(q)
    lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device="cuda")
    fca.fca_flat_decode(q, k, v, plan, out, lse, w.scale)
    assert fca.fca_check_device_status(plan) == 0
    plan.close()
    return out, lse


def _static(w, q, k, v, bt, sl, status):
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    out = torch.empty_like(q)
    lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device="cuda")
    fca.fca_paged_decode_static(q, k, v, bt, sl, w.num_blocks, out, lse, w.scale, dev_status=status)
    return out, lse


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check_pair(o, l, o_ref, l_ref, tol_scale, what):
    err = np.abs(_f64(o) - _f64(o_ref))
    assert np.isfinite(_f64(o)).all(), f"{what}: non-finite output"
    assert err.max() <= tol_scale * TOL_MAX, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= tol_scale * TOL_MEAN, f"{what}: mean-abs {err.mean():.3e}"
    le = np.abs(_f64(l) - _f64(l_ref)).max()
    assert le <= tol_scale * TOL_LSE, f"{what}: lse {le:.3e}"


def _two_calls_match_flat(w, check_oracle):
    torch = _torch()
    q, k, v, bt, sl = w.torch_inputs("cuda")
    o_flat, l_flat = _flat(w, q, k, v, bt, sl)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1 = _static(w, q, k, v, bt, sl, status)
    o2, l2 = _static(w, q, k, v, bt, sl, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_pair(o1, l1, o_flat, l_flat, 2.0, f"{w.name} first call vs fca_flat_decode")
    _check_pair(o2, l2, o_flat, l_flat, 2.0, f"{w.name} second call vs fca_flat_decode")
    # the same work list is rebuilt each call: the two calls agree bit for bit
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    if check_oracle:
        o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
        err = np.abs(_f64(o2) - o_ref)
        assert err.max() <= TOL_MAX and err.mean() <= TOL_MEAN, f"{w.name} vs oracle: {err.max():.3e}"
        assert np.abs(_f64(l2) - l_ref).max() <= TOL_LSE


# ----------------------------------------------------------- host only (CPU)

def test_static_entry_rejects_bad_arguments_without_a_device():
    import shared_prefix_kv_fca_b200 as fca
    lib = fca.load_library()
    p = 1 << 20          # a 16-byte aligned stand-in; rejected before any use
    args = dict(q=p, k=p, v=p, bt=p, mb=8, sl=p, R=4, nb=64, hq=8, hkv=2, d=128, out=p, lse=p)

    def call(**kw):
        a = dict(args, **kw)
        return lib.fca_paged_decode_static(a["q"], a["k"], a["v"], a["bt"], a["mb"], a["sl"], a["R"], a["nb"],
                                           a["hq"], a["hkv"], a["d"], a["out"], a["lse"], ctypes.c_float(0.1),
                                           None, None)
    assert call(q=None) == 1
    assert call(out=p + 8) == 1          # misaligned
    assert call(hq=6, hkv=4) == 1        # not a multiple
    assert call(R=-1) == 1
    assert call(d=96) == 3
    assert call(hq=64, hkv=2) == 3       # 32 query heads per KV head
    assert call(R=0) == 0                # nothing to do
    # 8192 requests x 32 heads x (128 + 1) floats of partials is past the 64 MiB array
    assert call(R=8192, hq=32, hkv=8) == 7
    assert fca.fca_status_string(7).startswith("problem larger than")


# ------------------------------------------------------------------- on a GPU

@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(6))
def test_static_matches_flat_decode_small(seed):
    w = fca_workloads.random_small(seed, Hq=8, Hkv=2, D=128, max_requests=16, poison_padding=True)
    _two_calls_match_flat(w, check_oracle=True)


@pytest.mark.gpu
def test_static_matches_flat_decode_wide_gqa():
    w = fca_workloads.random_small(31, Hq=16, Hkv=1, D=128, max_requests=16, poison_padding=True)
    _two_calls_match_flat(w, check_oracle=True)


@pytest.mark.gpu
def test_static_matches_flat_decode_head_dim_64():
    _two_calls_match_flat(fca_workloads.make("tiny"), check_oracle=True)


@pytest.mark.gpu
def test_static_matches_flat_decode_full_size():
    _two_calls_match_flat(fca_workloads.make("llama8b"), check_oracle=True)


@pytest.mark.gpu
def test_static_allocates_no_device_memory():
    torch = _torch()
    w = fca_workloads.make("llama8b")
    q, k, v, bt, sl = w.torch_inputs("cuda")
    out = torch.empty_like(q)
    lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    import shared_prefix_kv_fca_b200 as fca
    fca.fca_paged_decode_static(q, k, v, bt, sl, w.num_blocks, out, lse, w.scale, dev_status=status)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    reserved0 = torch.cuda.memory_reserved()
    for _ in range(2):
        fca.fca_paged_decode_static(q, k, v, bt, sl, w.num_blocks, out, lse, w.scale, dev_status=status)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_reserved() == reserved0
    assert int(status.item()) == 0


@pytest.mark.gpu
def test_static_flags_bad_requests_and_skips_them():
    torch = _torch()
    w = fca_workloads.random_small(3, Hq=8, Hkv=2, D=128, max_requests=16)
    assert w.R >= 3
    q, k, v, bt, sl = w.torch_inputs("cuda")
    o_flat, l_flat = _flat(w, q, k, v, bt, sl)
    bad_len = sl.clone()
    bad_len[0] = bt.shape[1] * 16 + 1            # longer than its table row
    bad_len[1] = 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, l = _static(w, q, k, v, bt, bad_len, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 8
    assert torch.all(o[:2] == 0) and torch.all(torch.isneginf(l[:2]))
    _check_pair(o[2:], l[2:], o_flat[2:], l_flat[2:], 2.0, "requests after the skipped ones")

    bad_id = bt.clone()
    bad_id[2, 0] = w.num_blocks                  # one past the last physical block
    status.zero_()
    o, l = _static(w, q, k, v, bad_id, sl, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 16
    assert torch.all(o[2] == 0) and torch.all(torch.isneginf(l[2]))
    keep = [r for r in range(w.R) if r != 2]
    _check_pair(o[keep], l[keep], o_flat[keep], l_flat[keep], 2.0, "requests other than the bad one")
