"""The Python binding's argument checks, without a GPU.

The C ABI takes raw pointers and cannot see a tensor's size, so the binding
checks every tensor's dtype, layout and shape against the plan before it
passes a pointer on: a cache with fewer blocks than the plan's num_blocks, or
q/out/lse of another batch, would have the kernels read or write past the
buffers.  Here CPU tensors stand in for CUDA ones and a stand-in library
records the calls, so that the checks are exercised on the shapes the GPU
tests and the bench use, and on wrong ones.
"""
import types

import pytest
import torch

import shared_prefix_kv_fca_b200 as fca

R, HQ, HKV, D, NB, MB = 5, 8, 2, 64, 40, 6


class FakeLib:
    """Every entry point succeeds and is recorded; fca_plan hands out a handle."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append(name)
            if name == "fca_plan":
                args[10]._obj.value = 1234   # the byref'd output handle
            return 0
        return call


PLANS = []


@pytest.fixture
def lib(monkeypatch):
    fake = FakeLib()
    monkeypatch.setattr(fca, "load_library", lambda: fake)
    monkeypatch.setattr(torch.Tensor, "is_cuda", property(lambda self: True))
    yield fake
    # the stand-in handles must never reach the real library's destroy
    for plan in PLANS:
        plan.handle = None
    PLANS.clear()


def tensors():
    bf = torch.bfloat16
    return types.SimpleNamespace(
        q=torch.zeros(R, HQ, D, dtype=bf), out=torch.zeros(R, HQ, D, dtype=bf),
        k=torch.zeros(NB, 16, HKV, D, dtype=bf), v=torch.zeros(NB, 16, HKV, D, dtype=bf),
        lse=torch.zeros(R, HQ, dtype=torch.float32),
        bt=torch.zeros(R, MB, dtype=torch.int32), sl=torch.ones(R, dtype=torch.int32))


def make_plan(t, flat=False):
    plan = fca.fca_plan(t.bt, t.sl, NB, HQ, HKV, D, flat=flat, stream=0)
    PLANS.append(plan)
    return plan


def test_valid_calls_pass_through(lib):
    t = tensors()
    plan = make_plan(t)
    fca.fca_decode(t.q, t.k, t.v, plan, t.out, t.lse, 0.125, stream=0)
    fca.fca_decode(t.q, t.k, t.v, plan, t.out, None, 0.125, stream=0)
    fca.fca_prefix_pass(t.q, t.k, t.v, plan, 0.125, stream=0)
    fca.fca_suffix_pass(t.q, t.k, t.v, plan, 0.125, stream=0)
    fca.fca_merge_pass(plan, t.out, t.lse, stream=0)
    plan.update(t.bt, t.sl, stream=0)
    # a cache pool with spare blocks past the plan's num_blocks is fine
    big = torch.zeros(NB + 7, 16, HKV, D, dtype=torch.bfloat16)
    fca.fca_decode(t.q, big, big, plan, t.out, t.lse, 0.125, stream=0)
    fca.fca_paged_decode_static(t.q, t.k, t.v, t.bt, t.sl, NB, t.out, t.lse, 0.125,
                                dev_status=torch.zeros(1, dtype=torch.int32), stream=0)
    assert lib.calls.count("fca_decode") == 3 and "fca_paged_decode_static" in lib.calls


@pytest.mark.parametrize("what", ["q_rows", "q_heads", "q_dim", "out", "lse", "lse_dtype", "k_blocks", "k_heads",
                                  "v_dim", "k_block_size", "k_dtype", "q_layout"])
def test_decode_rejects_tensors_that_do_not_fit_the_plan(lib, what):
    t = tensors()
    plan = make_plan(t)
    bf = torch.bfloat16
    bad = {
        "q_rows": dict(q=torch.zeros(R + 1, HQ, D, dtype=bf)),
        "q_heads": dict(q=torch.zeros(R, HQ // 2, D, dtype=bf)),
        "q_dim": dict(q=torch.zeros(R, HQ, 2 * D, dtype=bf)),
        "out": dict(out=torch.zeros(R - 1, HQ, D, dtype=bf)),
        "lse": dict(lse=torch.zeros(R, HQ + 1)),
        "lse_dtype": dict(lse=torch.zeros(R, HQ, dtype=torch.float64)),
        "k_blocks": dict(k=torch.zeros(NB - 1, 16, HKV, D, dtype=bf)),
        "k_heads": dict(k=torch.zeros(NB, 16, HKV + 1, D, dtype=bf)),
        "v_dim": dict(v=torch.zeros(NB, 16, HKV, D // 2, dtype=bf)),
        "k_block_size": dict(k=torch.zeros(NB * 2, 8, HKV, D, dtype=bf)),
        "k_dtype": dict(k=torch.zeros(NB, 16, HKV, D, dtype=torch.float16)),
        "q_layout": dict(q=torch.zeros(R, D, HQ, dtype=bf).transpose(1, 2)),
    }[what]
    a = dict(q=t.q, k=t.k, v=t.v, out=t.out, lse=t.lse, **{})
    a.update(bad)
    before = list(lib.calls)
    with pytest.raises(ValueError):
        fca.fca_decode(a["q"], a["k"], a["v"], plan, a["out"], a["lse"], 0.125, stream=0)
    assert lib.calls == before          # nothing reached the library


def test_passes_and_merge_check_their_tensors(lib):
    t = tensors()
    plan = make_plan(t)
    short = torch.zeros(NB - 3, 16, HKV, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fca.fca_prefix_pass(t.q, short, t.v, plan, 0.125, stream=0)
    with pytest.raises(ValueError):
        fca.fca_suffix_pass(t.q[:-1], t.k, t.v, plan, 0.125, stream=0)
    with pytest.raises(ValueError):
        fca.fca_merge_pass(plan, t.out[:, :4], t.lse, stream=0)
    with pytest.raises(ValueError):
        fca.fca_merge_pass(plan, t.out, t.lse[:-1], stream=0)
    assert "fca_prefix_pass" not in lib.calls and "fca_merge_pass" not in lib.calls


def test_tables_must_agree_with_each_other(lib):
    t = tensors()
    with pytest.raises(ValueError):
        fca.fca_plan(t.bt, t.sl[:-1], NB, HQ, HKV, D, stream=0)
    with pytest.raises(ValueError):
        fca.fca_plan(t.bt.reshape(-1), t.sl, NB, HQ, HKV, D, stream=0)
    with pytest.raises(ValueError):
        fca.fca_plan(t.bt.to(torch.int64), t.sl, NB, HQ, HKV, D, stream=0)
    plan = make_plan(t)
    with pytest.raises(ValueError):
        plan.update(t.bt, t.sl[:-1], stream=0)
    # a request fewer in both is the library's to refuse (it knows the plan's size)
    plan.update(t.bt[:-1], t.sl[:-1], stream=0)
    assert lib.calls.count("fca_plan_update") == 1
    # the module-level call of the C name is the same call
    fca.fca_plan_update(plan, t.bt, t.sl, stream=0)
    with pytest.raises(ValueError):
        fca.fca_plan_update(plan, t.bt, t.sl.to(torch.int64), stream=0)
    assert lib.calls.count("fca_plan_update") == 2


def test_static_decode_checks_its_tensors(lib):
    t = tensors()
    st = torch.zeros(1, dtype=torch.int32)
    for kw in (dict(bt=t.bt[:-1], sl=t.sl[:-1]), dict(k=torch.zeros(NB - 1, 16, HKV, D, dtype=torch.bfloat16)),
               dict(out=torch.zeros(R, HQ, D + 8, dtype=torch.bfloat16)), dict(lse=torch.zeros(R + 2, HQ)),
               dict(status=torch.zeros(1, dtype=torch.float32))):
        a = dict(q=t.q, k=t.k, v=t.v, bt=t.bt, sl=t.sl, out=t.out, lse=t.lse, status=st)
        a.update(kw)
        with pytest.raises(ValueError):
            fca.fca_paged_decode_static(a["q"], a["k"], a["v"], a["bt"], a["sl"], NB, a["out"], a["lse"], 0.125,
                                        dev_status=a["status"], stream=0)
    assert "fca_paged_decode_static" not in lib.calls


class OnDevice:
    """A CPU tensor that reports itself as living on CUDA device `idx`."""

    def __init__(self, t, idx):
        self._t = t
        self.device = torch.device("cuda", idx)

    def __getattr__(self, name):
        return getattr(self._t, name)


def test_buffers_on_another_device_are_refused(lib):
    # a pointer on another device would be dereferenced on the device the call
    # runs on: refused before anything reaches the library
    t = tensors()
    on = lambda x, i: OnDevice(x, i)          # noqa: E731
    with pytest.raises(ValueError, match="one device"):
        fca.fca_plan(on(t.bt, 0), on(t.sl, 1), NB, HQ, HKV, D, stream=0)
    assert lib.calls == []
    with pytest.raises(ValueError, match="one device"):
        fca.fca_paged_decode_static(on(t.q, 0), on(t.k, 0), on(t.v, 0), on(t.bt, 0), on(t.sl, 0), NB,
                                    on(t.out, 1), on(t.lse, 0), 0.125, stream=0)
    with pytest.raises(ValueError, match="one device"):
        fca.fca_paged_decode_static(on(t.q, 0), on(t.k, 0), on(t.v, 0), on(t.bt, 0), on(t.sl, 0), NB,
                                    on(t.out, 0), on(t.lse, 0), 0.125,
                                    dev_status=on(torch.zeros(1, dtype=torch.int32), 2), stream=0)
    assert lib.calls == []
    plan = make_plan(t)
    plan.device = 0
    q1, k1, v1, out1, lse1 = (on(x, 1) for x in (t.q, t.k, t.v, t.out, t.lse))
    with pytest.raises(ValueError, match="plan belongs to cuda:0"):
        fca.fca_decode(q1, k1, v1, plan, out1, lse1, 0.125, stream=0)
    with pytest.raises(ValueError, match="plan belongs to cuda:0"):
        fca.fca_prefix_pass(q1, k1, v1, plan, 0.125, stream=0)
    with pytest.raises(ValueError, match="plan belongs to cuda:0"):
        fca.fca_merge_pass(plan, out1, lse1, stream=0)
    with pytest.raises(ValueError, match="plan belongs to cuda:0"):
        plan.update(on(t.bt, 1), on(t.sl, 1), stream=0)
    with pytest.raises(ValueError, match="one device"):
        fca.fca_decode(on(t.q, 0), on(t.k, 0), on(t.v, 1), plan, on(t.out, 0), on(t.lse, 0), 0.125, stream=0)
    assert lib.calls == ["fca_plan"]
    # all on the plan's device: passes through
    fca.fca_decode(*(on(x, 0) for x in (t.q, t.k, t.v)), plan, on(t.out, 0), on(t.lse, 0), 0.125, stream=0)
    assert lib.calls == ["fca_plan", "fca_decode"]
