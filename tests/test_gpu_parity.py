"""CUDA path vs the CPU oracle, through the C ABI.

Plans must match the oracle planner bit for bit.  Attention outputs (bf16
inputs, fp32 accumulation, bf16 output) must be within max-abs 1e-2 and
mean-abs 1e-3 of the oracle's fp64 result, and the LSE within 1e-3
(absolute, natural log).  Every test compares every output with the oracle,
the full-size configurations included (the fp64 oracle takes seconds on the
host's cores for the largest of them); those also compare FCA with the flat
paged decode kernel, as an extra check.
"""
import math

import numpy as np
import pytest

import fca_workloads
import oracle

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE = 1e-2, 1e-3, 1e-3


def _torch():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def run(w, flat=False, lse=True, **opts):
    """Plan + decode through the binding; returns (out f64 [R,Hq,D], lse f64, plan export, stats).
    Every shared prefix is used (min_saved_blocks 0) unless the caller says
    otherwise, so that the small random forests exercise the grouped pass."""
    torch = _torch()
    opts.setdefault("min_saved_blocks", 0)
    import shared_prefix_kv_fca_b200 as fca
    q, k, v, bt, sl = w.torch_inputs("cuda")
    plan = fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D, flat=flat, **opts)
    out = torch.empty_like(q)
    l = torch.empty(w.R, w.Hq, dtype=torch.float32, device="cuda") if lse else None
    (fca.fca_flat_decode if flat else fca.fca_decode)(q, k, v, plan, out, l, w.scale)
    assert fca.fca_check_device_status(plan) == 0
    exp = plan.export()
    st = plan.stats()
    plan.close()
    o = out.float().cpu().numpy().astype(np.float64)
    return o, (l.cpu().numpy().astype(np.float64) if lse else None), exp, st


def assert_close(o, l, o_ref, l_ref, what=""):
    err = np.abs(o - o_ref)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert err.max() <= TOL_MAX, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= TOL_MEAN, f"{what}: mean-abs {err.mean():.3e}"
    if l is not None:
        le = np.abs(l - l_ref).max()
        assert le <= TOL_LSE, f"{what}: lse err {le:.3e}"


def assert_all_vs_oracle(w, o, l, what, block_tables=None, seq_lens=None):
    """Every (request, query head) of o / l against the fp64 oracle."""
    bt = w.block_tables if block_tables is None else block_tables
    sl = w.seq_lens if seq_lens is None else seq_lens
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, bt, sl, w.scale)
    assert_close(o, l, o_ref, l_ref, what)
    return o_ref, l_ref


def assert_plan_equal(exp, ref):
    for key in ("a", "b", "parent", "member_off", "n_members", "members", "suffix_start"):
        np.testing.assert_array_equal(exp[key], ref[key], err_msg=key)


# --------------------------------------------------------------- planner

@pytest.mark.parametrize("seed", range(30))
def test_plan_bit_exact_random_forests(seed):
    w = fca_workloads.random_small(seed, max_requests=24)
    _, _, exp, st = run(w)
    assert_plan_equal(exp, oracle.plan(w.block_tables, w.seq_lens, w.block_size))
    assert st["unique_kv_tokens"] == oracle.unique_kv_tokens(w.block_tables, w.seq_lens,
                                                               w.block_size, w.num_blocks)


@pytest.mark.parametrize("mgs,msb,msv", [(3, 1, 0), (2, 2, 0), (4, 3, 0), (2, 5, 0), (2, 1, 5), (2, 1, 32),
                                         (3, 2, 12), (2, 1, 1000)])
def test_plan_options(mgs, msb, msv):
    for seed in range(12):
        w = fca_workloads.random_small(seed, max_requests=24)
        _, _, exp, _ = run(w, min_group_size=mgs, min_shared_blocks=msb, min_saved_blocks=msv)
        assert_plan_equal(exp, oracle.plan(w.block_tables, w.seq_lens, w.block_size, mgs, msb, msv))


def test_default_plan_folds_groups_too_small_to_pay():
    # the default plan (min_saved_blocks 32) on pairs of requests sharing short
    # prompts: the groups that save fewer than 32 block reads are folded, the
    # plan still matches the oracle bit for bit, and decode matches attention
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    w = fca_workloads.make("pairs", prompts=24)
    q, k, v, bt, sl = w.torch_inputs("cuda")
    with fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D) as plan:
        exp = plan.export()
        out = torch.empty_like(q)
        lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device="cuda")
        fca.fca_decode(q, k, v, plan, out, lse, w.scale)
        assert fca.fca_check_device_status(plan) == 0
    ref = oracle.plan(w.block_tables, w.seq_lens, 16, min_saved_blocks=32)
    assert_plan_equal(exp, ref)
    assert len(ref["a"]) < len(oracle.plan(w.block_tables, w.seq_lens, 16)["a"])
    o = out.float().cpu().numpy().astype(np.float64)
    assert_all_vs_oracle(w, o, lse.cpu().numpy().astype(np.float64), "pairs default plan")


def inconsistent_workload():
    """Tables whose block ids do not identify prefixes: block 11 sits under two
    different parents, block 20 at two logical positions."""
    w = fca_workloads.random_small(2, Hq=4, Hkv=2, D=64)
    B = 16
    bt = np.array([[10, 11, 12, 13, 30],
                   [10, 11, 12, 14, 31],
                   [15, 11, 12, 13, 32],
                   [15, 11, 12, 13, 33],
                   [20, 21, 22, 34, 0],
                   [23, 20, 21, 35, 0],
                   [10, 11, 16, 36, 37]], np.int32)
    sl = np.array([5 * B - 3, 5 * B, 4 * B + 1, 4 * B + 9, 3 * B + 2, 4 * B, 5 * B - 1], np.int32)
    nb = 40
    k = fca_workloads.normal_bf16((nb, B, w.Hkv, w.D), 5, 1)
    v = fca_workloads.normal_bf16((nb, B, w.Hkv, w.D), 5, 2)
    q = fca_workloads.normal_bf16((bt.shape[0], w.Hq, w.D), 5, 0)
    return fca_workloads.Workload("inconsistent", q, k, v, bt, sl, w.Hq, w.Hkv, w.D, B, 5)


def test_plan_fallback_for_tables_without_prefix_identity():
    w = inconsistent_workload()
    o, l, exp, _ = run(w)
    ref = oracle.plan(w.block_tables, w.seq_lens, w.block_size)
    assert_plan_equal(exp, ref)
    assert len(ref["a"]) >= 3
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, l, o_ref, l_ref, "fallback plan decode")


def test_plan_named_configs_bit_exact():
    for name in ("tiny", "llama8b", "forest", "longctx"):
        w = fca_workloads.make(name)
        torch = _torch()
        import shared_prefix_kv_fca_b200 as fca
        bt = torch.from_numpy(w.block_tables).cuda()
        sl = torch.from_numpy(w.seq_lens).cuda()
        with fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D) as plan:
            exp = plan.export()
            st = plan.stats()
        assert_plan_equal(exp, oracle.plan(w.block_tables, w.seq_lens, 16))
        assert st["unique_kv_tokens"] == oracle.unique_kv_tokens(w.block_tables, w.seq_lens, 16,
                                                                   w.num_blocks)


# --------------------------------------------------------------- attention, all outputs

@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("flat", [False, True])
def test_decode_matches_oracle_random(seed, flat):
    Hq, Hkv, D = [(4, 2, 64), (8, 2, 128), (4, 4, 128), (16, 2, 64), (6, 2, 128), (8, 1, 128)][seed % 6]
    w = fca_workloads.random_small(seed, Hq=Hq, Hkv=Hkv, D=D, max_requests=20,
                                   poison_padding=seed % 2 == 1)
    o, l, _, _ = run(w, flat=flat)
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, l, o_ref, l_ref, f"seed {seed} flat={flat}")


@pytest.mark.parametrize("shape", [(16, 1, 128), (32, 2, 64), (16, 1, 64), (12, 1, 128)])
@pytest.mark.parametrize("flat", [False, True])
def test_decode_wide_gqa(shape, flat):
    # 9 to 16 query heads per KV head: the per-request pass's second column
    # tile, and group tiles of 16 rows per member
    Hq, Hkv, D = shape
    for seed in (21, 22, 23):
        w = fca_workloads.random_small(seed, Hq=Hq, Hkv=Hkv, D=D, max_requests=20, poison_padding=True)
        o, l, _, _ = run(w, flat=flat)
        o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
        assert_close(o, l, o_ref, l_ref, f"gqa {shape} seed {seed} flat={flat}")


def test_decode_one_group_of_many_members():
    # one prompt shared by 40 requests x 16 query heads = 640 stacked rows:
    # five 128-row tiles of one group
    rng = np.random.default_rng(9)
    reqs = [[("p", 300), (None, int(rng.integers(1, 40)))] for _ in range(40)]
    w = fca_workloads.fill("wide", reqs, Hq=16, Hkv=1, D=128, seed=9, rng=rng, poison_padding=True)
    o, l, exp, st = run(w)
    assert len(exp["a"]) == 1 and st["prefix_items"] >= 5
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, l, o_ref, l_ref, "one wide group")


@pytest.mark.parametrize("shape", [(8, 2, 128), (6, 2, 64)])
def test_decode_deep_chain(shape):
    # request j shares blocks 0..j with every request after it: one nested
    # group per block, so the last requests sit under 30-40 groups (chains
    # longer than a warp's 32 lanes take the merge's sequential walk)
    Hq, Hkv, D = shape
    rng = np.random.default_rng(31)
    n = 42
    reqs = [[(f"k{d}", 16) for d in range(j + 1)] + [(None, int(rng.integers(0, 24)))] for j in range(n)]
    w = fca_workloads.fill("deep", reqs, Hq=Hq, Hkv=Hkv, D=D, seed=31, rng=rng, poison_padding=True)
    o, l, exp, _ = run(w)
    ref = oracle.plan(w.block_tables, w.seq_lens, w.block_size)
    assert_plan_equal(exp, ref)
    assert len(ref["a"]) >= 36
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, l, o_ref, l_ref, f"deep chain {shape}")


@pytest.mark.parametrize("split", [64, 128, 256])
def test_decode_small_splits(split):
    # many split chunks per group and per request, ragged tails
    for seed in (3, 7):
        w = fca_workloads.random_small(seed, Hq=8, Hkv=2, D=128, max_requests=16)
        o, l, _, _ = run(w, split_tokens=split)
        o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens,
                                              w.scale)
        assert_close(o, l, o_ref, l_ref, f"split {split}")


def test_tiny_config_all_outputs():
    w = fca_workloads.make("tiny", poison_padding=True)
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    for flat in (False, True):
        o, l, _, _ = run(w, flat=flat)
        assert_close(o, l, o_ref, l_ref, f"tiny flat={flat}")


def test_one_plan_serves_several_layers():
    # the plan depends only on the block tables and lengths: every layer of a
    # model reuses it with that layer's q and caches
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    w = fca_workloads.random_small(5, Hq=8, Hkv=2, D=128, max_requests=16)
    bt = torch.from_numpy(w.block_tables).cuda()
    sl = torch.from_numpy(w.seq_lens).cuda()
    with fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D) as plan:
        for layer in range(3):
            q = fca_workloads.normal_bf16(w.q.shape, 200 + layer, 0)
            k = fca_workloads.normal_bf16(w.k_cache.shape, 200 + layer, 1)
            v = fca_workloads.normal_bf16(w.v_cache.shape, 200 + layer, 2)
            lw = fca_workloads.Workload(f"layer{layer}", q, k, v, w.block_tables, w.seq_lens, w.Hq, w.Hkv,
                                        w.D, w.block_size, 200 + layer)
            qd, kd, vd, _, _ = lw.torch_inputs("cuda")
            out = torch.empty_like(qd)
            lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device="cuda")
            fca.fca_decode(qd, kd, vd, plan, out, lse, w.scale)
            assert fca.fca_check_device_status(plan) == 0
            o_ref, l_ref = oracle.paged_attention(q, k, v, w.block_tables, w.seq_lens, w.scale)
            assert_close(out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                         o_ref, l_ref, f"layer {layer}")


def test_lse_optional():
    w = fca_workloads.random_small(4, D=64)
    o, l, _, _ = run(w, lse=False)
    o_ref, _ = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, None, o_ref, None, "no lse")


def growing_keys_workload(seed=0):
    """One 16-request group over a 1024-token prompt whose key norms grow
    with the logical position, so the running maximum keeps rising from stage
    to stage (exercises the grouped pass's rescaling of its accumulator)."""
    rng = np.random.default_rng(seed)
    reqs = [[("p", 1024), (None, int(rng.integers(1, 200)))] for _ in range(16)]
    w = fca_workloads.fill("growing", reqs, Hq=16, Hkv=2, D=128, seed=seed, rng=rng)
    k = (w.k_cache.astype(np.uint32) << 16).view(np.float32).copy()
    done = np.zeros(w.num_blocks, bool)
    for r in range(w.R):
        nblk = (int(w.seq_lens[r]) + 15) // 16
        for j in range(nblk):
            b = w.block_tables[r, j]
            if not done[b]:
                k[b] *= 0.25 * (1 + j)
                done[b] = True
    u = k.view(np.uint32)
    w.k_cache = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    # the softmax ends up peaked on single tokens; keep |o| < 2, where half a
    # bf16 ulp of the output (3.9e-3) stays inside the 1e-2 bound
    v = (w.v_cache.astype(np.uint32) << 16).view(np.float32) * 0.4
    u = v.view(np.uint32)
    w.v_cache = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return w


@pytest.mark.parametrize("split", [0, 256])
def test_prefix_rescale_path(split):
    w = growing_keys_workload()
    o, l, exp, _ = run(w, split_tokens=split)
    assert len(exp["a"]) == 1
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, l, o_ref, l_ref, f"growing keys split {split}")


def test_many_items_per_cta():
    # far more grouped-pass items than SMs: every CTA walks several items
    for seed in (1, 2):
        w = fca_workloads.make("llama8b", seed=seed, prompts=8)
        o, l, _, st = run(w, split_tokens=64)
        assert st["prefix_items"] > 4 * 148
        assert_all_vs_oracle(w, o, l, "many items")


# --------------------------------------------------------------- full-size configurations

@pytest.mark.parametrize("name", ["llama8b", "longctx", "forest", "mixed"])
def test_full_size_configs(name):
    w = fca_workloads.make(name)
    o, l, exp, st = run(w, min_saved_blocks=32)      # the default plan, as the bench runs it
    o0, l0, _, _ = run(w)                            # every shared prefix kept
    of, lf, _, _ = run(w, flat=True)
    # every output of the three against the oracle
    o_ref, l_ref = assert_all_vs_oracle(w, o, l, f"{name} fca")
    assert_close(o0, l0, o_ref, l_ref, f"{name} fca, every group kept")
    assert_close(of, lf, o_ref, l_ref, f"{name} flat")
    # and FCA against the flat (standard) attention kernel.  Both are within
    # the oracle tolerance of the exact result, so they are within twice that
    # of each other (one bf16 ulp is already 1.56e-2 for |o| in [2, 4)).
    err = np.abs(o - of)
    assert np.isfinite(o).all() and np.isfinite(of).all()
    assert err.max() <= 2 * TOL_MAX, f"{name} fca vs flat: max-abs {err.max():.3e}"
    assert err.mean() <= 2 * TOL_MEAN, f"{name} fca vs flat: mean-abs {err.mean():.3e}"
    assert np.abs(l - lf).max() <= 2 * TOL_LSE
    assert st["unique_kv_bytes"] == oracle.unique_kv_tokens(
        w.block_tables, w.seq_lens, 16, w.num_blocks) * w.Hkv * w.D * 4


# --------------------------------------------------------------- errors

def test_error_paths_return_status():
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    w = fca_workloads.random_small(1, D=64)
    bt = torch.from_numpy(w.block_tables).cuda()
    sl = torch.from_numpy(w.seq_lens).cuda()
    bad = w.block_tables.copy()
    bad[0, 0] = w.num_blocks + 5
    with pytest.raises(fca.FcaError) as e:
        fca.fca_plan(torch.from_numpy(bad).cuda(), sl, w.num_blocks, w.Hq, w.Hkv, w.D)
    assert e.value.status == 2
    bad = w.block_tables.copy()
    bad[0, 0] = -1
    with pytest.raises(fca.FcaError) as e:
        fca.fca_plan(torch.from_numpy(bad).cuda(), sl, w.num_blocks, w.Hq, w.Hkv, w.D)
    assert e.value.status == 2
    for L in (0, w.max_blocks * 16 + 1):
        s2 = w.seq_lens.copy()
        s2[-1] = L
        with pytest.raises(fca.FcaError) as e:
            fca.fca_plan(bt, torch.from_numpy(s2).cuda(), w.num_blocks, w.Hq, w.Hkv, w.D)
        assert e.value.status == 1
    with pytest.raises(fca.FcaError) as e:
        fca.fca_plan(bt, sl, w.num_blocks, 6, 4, w.D)
    assert e.value.status == 1
    with pytest.raises(fca.FcaError) as e:
        fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, 96)
    assert e.value.status == 3
    # a flat decode needs a flat plan
    q, k, v, _, _ = w.torch_inputs("cuda")
    with fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D) as plan:
        with pytest.raises(fca.FcaError):
            fca.fca_flat_decode(q, k, v, plan, torch.empty_like(q))
        # the scale must be positive and finite
        for bad_scale in (0.0, -0.125, float("inf"), float("nan")):
            with pytest.raises(fca.FcaError) as e:
                fca.fca_decode(q, k, v, plan, torch.empty_like(q), None, bad_scale)
            assert e.value.status == 1
        # the good plan still works after the failed calls
        out = torch.empty_like(q)
        fca.fca_decode(q, k, v, plan, out)
        assert fca.fca_check_device_status(plan) == 0


# --------------------------------------------------------------- limits and degenerate shapes

def test_plan_and_decode_at_the_request_limit():
    # 16384 requests (the planner's limit): 1024 prompts of 2-3 blocks x 16
    # samples with 1..20 own tokens; head_dim 64, one KV head
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    rng = np.random.default_rng(77)
    reqs = []
    for p in range(1024):
        plen = int(rng.integers(32, 49))
        for _ in range(16):
            reqs.append([(f"p{p}", plen), (None, int(rng.integers(1, 21)))])
    w = fca_workloads.fill("limit", reqs, Hq=4, Hkv=1, D=64, seed=77, rng=rng)
    assert w.R == 16384
    o, l, exp, st = run(w)
    assert_plan_equal(exp, oracle.plan(w.block_tables, w.seq_lens, 16))
    assert st["num_groups"] == 1024
    assert_all_vs_oracle(w, o, l, "request limit")
    # one request more is refused, without touching the device state
    bt = torch.from_numpy(np.concatenate([w.block_tables, w.block_tables[:1]])).cuda()
    sl = torch.from_numpy(np.concatenate([w.seq_lens, w.seq_lens[:1]])).cuda()
    with pytest.raises(fca.FcaError) as e:
        fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D)
    assert e.value.status == 3


def test_fallback_planner_limit():
    # tables whose block ids do not identify prefixes take the all-pairs
    # planner, which handles up to 4096 requests; past that the plan is refused
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    base = inconsistent_workload()
    for R, ok in ((4096, True), (4100, False)):
        reps = (R + base.R - 1) // base.R
        bt = np.tile(base.block_tables, (reps, 1))[:R]
        sl = np.tile(base.seq_lens, reps)[:R]
        if ok:
            w = fca_workloads.Workload("fallback_limit", fca_workloads.normal_bf16((R, base.Hq, base.D), 8, 0),
                                       base.k_cache, base.v_cache, bt, sl, base.Hq, base.Hkv, base.D, 16, 8)
            o, l, exp, _ = run(w)
            assert_plan_equal(exp, oracle.plan(bt, sl, 16))
            assert_all_vs_oracle(w, o, l, "fallback at its limit")
        else:
            with pytest.raises(fca.FcaError) as e:
                fca.fca_plan(torch.from_numpy(bt).cuda(), torch.from_numpy(sl).cuda(), base.num_blocks, base.Hq,
                             base.Hkv, base.D)
            assert e.value.status == 3


@pytest.mark.parametrize("case", ["single_request", "identical_full_tables", "one_token", "full_table"])
def test_degenerate_batches(case):
    rng = np.random.default_rng(11)
    if case == "single_request":
        reqs = [[(None, 77)]]
    elif case == "identical_full_tables":
        # every token of every request is shared: no own tokens at all
        reqs = [[("p", 96)] for _ in range(6)]
    elif case == "one_token":
        reqs = [[(None, 1)] for _ in range(5)] + [[("p", 16), (None, 1)] for _ in range(3)]
    else:
        # sequences that end exactly on a block boundary, one at max_blocks * 16
        reqs = [[("p", 64), (None, 64)] for _ in range(4)] + [[("p", 64), (None, 128)]]
    w = fca_workloads.fill(case, reqs, Hq=8, Hkv=2, D=128, seed=11, rng=rng, poison_padding=True)
    o, l, exp, _ = run(w)
    assert_plan_equal(exp, oracle.plan(w.block_tables, w.seq_lens, 16))
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, l, o_ref, l_ref, case)
    if case == "identical_full_tables":
        assert list(exp["suffix_start"]) == [6] * 6


@pytest.mark.parametrize("cover", [True, False])
def test_parent_folded_into_child_items(cover):
    # 16 query heads per KV head: a 16-member system-prompt group is 256 rows
    # (two tiles) and each of its two 8-member prompt groups one tile, so the
    # root's blocks can be streamed inside its children's items; with one
    # member that has no prompt of its own the root keeps its own items
    rng = np.random.default_rng(41)
    reqs = []
    for p in range(2):
        for _ in range(8):
            reqs.append([("sys", 64), (f"p{p}", 80), (None, int(rng.integers(1, 40)))])
    if not cover:
        reqs.append([("sys", 64), (None, 30)])
    w = fca_workloads.fill("fold_in", reqs, Hq=16, Hkv=1, D=128, seed=41, rng=rng, poison_padding=True)
    o, l, exp, st = run(w)
    ref = oracle.plan(w.block_tables, w.seq_lens, 16)
    assert_plan_equal(exp, ref)
    assert len(ref["a"]) == 3
    # folded: only the two prompt groups have items (one tile each, one chunk);
    # kept: the root adds its own tiles (17 members x 16 rows = three tiles)
    if cover:
        assert st["prefix_items"] == 2
    else:
        assert st["prefix_items"] >= 5
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, l, o_ref, l_ref, f"fold-in cover={cover}")


# --------------------------------------------------------------- plan update

def pooled(w, extra_blocks, max_blocks, seed):
    """w with its K/V cache inside a pool of extra_blocks more blocks (their
    K/V drawn fresh, free for later tokens) and its tables widened to
    max_blocks columns, as an engine with a block pool keeps a batch."""
    shape = (extra_blocks, w.block_size, w.Hkv, w.D)
    kc = np.concatenate([w.k_cache, fca_workloads.normal_bf16(shape, seed, 11)])
    vc = np.concatenate([w.v_cache, fca_workloads.normal_bf16(shape, seed, 12)])
    bt = np.zeros((w.R, max_blocks), np.int32)
    bt[:, :w.max_blocks] = w.block_tables
    return fca_workloads.Workload(w.name, w.q, kc, vc, bt, w.seq_lens.copy(), w.Hq, w.Hkv, w.D,
                                  w.block_size, w.seed)


def grown(w, extra, first_free, seed):
    """The batch w after request r has extra[r] more tokens: they go first into
    r's last block (always private: a shared prompt's partial tail is a private
    copy) and then into new blocks taken in turn from first_free on.  Same pool,
    same table width, new queries."""
    B = w.block_size
    sl = (w.seq_lens.astype(np.int64) + np.asarray(extra, np.int64)).astype(np.int32)
    bt = w.block_tables.copy()
    nxt = first_free
    for r in range(w.R):
        for j in range((int(w.seq_lens[r]) + B - 1) // B, (int(sl[r]) + B - 1) // B):
            bt[r, j] = nxt
            nxt += 1
    assert nxt <= w.num_blocks and bt.shape[1] * B >= sl.max()
    q = fca_workloads.normal_bf16(w.q.shape, seed, 13)
    return fca_workloads.Workload(w.name + "+", q, w.k_cache, w.v_cache, bt, sl, w.Hq, w.Hkv, w.D, B, w.seed)


def decode_with(plan, w, flat=False):
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    q, k, v, _, _ = w.torch_inputs("cuda")
    out = torch.empty_like(q)
    lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device="cuda")
    (fca.fca_flat_decode if flat else fca.fca_decode)(q, k, v, plan, out, lse, w.scale)
    assert fca.fca_check_device_status(plan) == 0
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check_all(plan, w, what, flat=False):
    o, l = decode_with(plan, w, flat)
    o_ref, l_ref = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    assert_close(o, l, o_ref, l_ref, what)


def growth_steps(w0, seed, n_steps=4, most=80):
    """w0 in a pool with room for n_steps steps of 1..most tokens a request,
    and the batch after each step."""
    rng = np.random.default_rng(500 + seed)
    steps = [rng.integers(1, most + 1, size=w0.R) for _ in range(n_steps)]
    B = w0.block_size
    final = w0.seq_lens.astype(np.int64) + np.sum(steps, axis=0)
    need = int(((final + B - 1) // B - (w0.seq_lens.astype(np.int64) + B - 1) // B).sum())
    base = pooled(w0, need, int(((final + B - 1) // B).max()), seed)
    out, cur = [], base
    for ex in steps:
        # each step's new blocks follow the ones taken before
        used = int(((cur.seq_lens.astype(np.int64) + B - 1) // B).sum()
                   - ((w0.seq_lens.astype(np.int64) + B - 1) // B).sum())
        cur = grown(cur, ex, w0.num_blocks + used, seed + len(out))
        out.append(cur)
    return base, out


@pytest.mark.parametrize("seed", range(10))
@pytest.mark.parametrize("split", [0, 64])
def test_plan_update_follows_growing_requests(seed, split):
    # one plan kept over four decode steps: after each step every request has
    # grown by 1-80 tokens (some into new blocks); the updated plan decodes like
    # attention over the new tables and holds the forest the oracle finds in
    # them.  A split of 64 tokens makes the own-pass work outgrow the plan's
    # first allocation.
    import shared_prefix_kv_fca_b200 as fca
    w0 = fca_workloads.random_small(seed, max_requests=24)
    base, steps = growth_steps(w0, seed)
    bt, sl = base.torch_inputs("cuda")[3:]
    ref = oracle.plan(base.block_tables, base.seq_lens, 16)
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D, min_saved_blocks=0,
                      split_tokens=split) as plan:
        assert_plan_equal(plan.export(), ref)
        check_all(plan, base, f"seed {seed} step 0")
        for s, cur in enumerate(steps):
            bt2, sl2 = cur.torch_inputs("cuda")[3:]
            plan.update(bt2, sl2)
            exp = plan.export()
            assert_plan_equal(exp, oracle.plan(cur.block_tables, cur.seq_lens, 16))
            assert_plan_equal(exp, ref)
            st = plan.stats()
            assert st["unique_kv_tokens"] == oracle.unique_kv_tokens(cur.block_tables, cur.seq_lens, 16,
                                                                       cur.num_blocks)
            check_all(plan, cur, f"seed {seed} step {s + 1}")


@pytest.mark.parametrize("seed", range(4))
def test_plan_update_flat(seed):
    import shared_prefix_kv_fca_b200 as fca
    w0 = fca_workloads.random_small(seed, max_requests=24)
    base, steps = growth_steps(w0, seed, n_steps=2)
    bt, sl = base.torch_inputs("cuda")[3:]
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D, flat=True) as plan:
        check_all(plan, base, f"flat seed {seed} step 0", flat=True)
        for s, cur in enumerate(steps):
            bt2, sl2 = cur.torch_inputs("cuda")[3:]
            plan.update(bt2, sl2)
            assert plan.stats()["num_groups"] == 0
            check_all(plan, cur, f"flat seed {seed} step {s + 1}", flat=True)


def test_plan_update_refusals_leave_the_plan_usable():
    # tables that no longer fit the plan's forest are refused with a status,
    # and the plan still decodes the batch it was built or last updated for
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    for seed in range(40):
        w0 = fca_workloads.random_small(seed, max_requests=24)
        ref = oracle.plan(w0.block_tables, w0.seq_lens, 16)
        if w0.R >= 2 and ref["suffix_start"].max() > 1:
            break
    base, (nxt,) = growth_steps(w0, seed, n_steps=1)
    r = int(np.argmax(ref["suffix_start"]))
    ss = int(ref["suffix_start"][r])
    B = 16

    def attempt(bt_np, sl_np):
        bt_t = torch.from_numpy(np.ascontiguousarray(bt_np, np.int32)).cuda()
        sl_t = torch.from_numpy(np.ascontiguousarray(sl_np, np.int32)).cuda()
        with pytest.raises(fca.FcaError) as ei:
            plan.update(bt_t, sl_t)
        return ei.value.status

    bt, sl = base.torch_inputs("cuda")[3:]
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D, min_saved_blocks=0) as plan:
        bad = nxt.block_tables.copy()
        bad[r, ss - 1] = base.num_blocks - 1          # a shared entry replaced
        assert attempt(bad, nxt.seq_lens) == 1
        short = nxt.seq_lens.copy()
        short[r] = ss * B - 1                        # the request no longer covers its groups
        assert attempt(nxt.block_tables, short) == 1
        assert attempt(nxt.block_tables[:-1], nxt.seq_lens[:-1]) == 1    # a request fewer
        wide = np.zeros((nxt.R, nxt.max_blocks + 1), np.int32)
        wide[:, :-1] = nxt.block_tables
        assert attempt(wide, nxt.seq_lens) == 1                          # another table width
        oob = nxt.block_tables.copy()
        last = (int(nxt.seq_lens[r]) + B - 1) // B - 1
        oob[r, last] = base.num_blocks                # a used entry outside the pool
        assert attempt(oob, nxt.seq_lens) == 2
        too_long = nxt.seq_lens.copy()
        too_long[r] = nxt.max_blocks * B + 1
        assert attempt(nxt.block_tables, too_long) == 1
        assert_plan_equal(plan.export(), ref)
        check_all(plan, base, "after refused updates")
        bt2, sl2 = nxt.torch_inputs("cuda")[3:]
        plan.update(bt2, sl2)
        check_all(plan, nxt, "after the good update")


def test_plan_update_full_size_one_token_steps():
    # the decode loop on the llama8b workload: every request gains one token a
    # step for 20 steps (some cross into new blocks); one plan, updated each step
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    w0 = fca_workloads.make("llama8b")
    B = 16
    n_steps = 20
    final = w0.seq_lens.astype(np.int64) + n_steps
    need = int(((final + B - 1) // B - (w0.seq_lens.astype(np.int64) + B - 1) // B).sum())
    base = pooled(w0, need, int(((final + B - 1) // B).max()), 0)
    q, k, v, bt, sl = base.torch_inputs("cuda")
    cur = base
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D) as plan:
        ref = plan.export()
        taken = 0
        for s in range(n_steps):
            nb_before = (cur.seq_lens.astype(np.int64) + B - 1) // B
            cur = grown(cur, np.ones(w0.R, np.int64), w0.num_blocks + taken, s)
            taken += int(((cur.seq_lens.astype(np.int64) + B - 1) // B - nb_before).sum())
            bt2, sl2 = cur.torch_inputs("cuda")[3:]
            plan.update(bt2, sl2)
        assert_plan_equal(plan.export(), ref)
        assert_plan_equal(ref, oracle.plan(cur.block_tables, cur.seq_lens, 16, min_saved_blocks=32))
        o, l = decode_with(plan, cur)
    assert_all_vs_oracle(cur, o, l, "llama8b after 20 updates")


# ---- plans with asynchronous updates (FCA_PLAN_ASYNC_UPDATE): the same
# growth, checked and applied on the device without a host synchronisation


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("split", [0, 64])
def test_plan_update_async_follows_growing_requests(seed, split):
    import shared_prefix_kv_fca_b200 as fca
    w0 = fca_workloads.random_small(seed, max_requests=24)
    base, steps = growth_steps(w0, seed)
    bt, sl = base.torch_inputs("cuda")[3:]
    ref = oracle.plan(base.block_tables, base.seq_lens, 16)
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D, min_saved_blocks=0,
                      split_tokens=split, async_update=True) as plan:
        assert_plan_equal(plan.export(), ref)
        check_all(plan, base, f"async seed {seed} step 0")
        for s, cur in enumerate(steps):
            bt2, sl2 = cur.torch_inputs("cuda")[3:]
            plan.update(bt2, sl2)
            check_all(plan, cur, f"async seed {seed} step {s + 1}")
            assert_plan_equal(plan.export(), ref)


@pytest.mark.parametrize("seed", range(3))
def test_plan_update_async_flat(seed):
    import shared_prefix_kv_fca_b200 as fca
    w0 = fca_workloads.random_small(seed, max_requests=24)
    base, steps = growth_steps(w0, seed, n_steps=2)
    bt, sl = base.torch_inputs("cuda")[3:]
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D, flat=True, async_update=True) as plan:
        check_all(plan, base, f"async flat seed {seed} step 0", flat=True)
        for s, cur in enumerate(steps):
            bt2, sl2 = cur.torch_inputs("cuda")[3:]
            plan.update(bt2, sl2)
            check_all(plan, cur, f"async flat seed {seed} step {s + 1}", flat=True)


def test_plan_update_async_refusal_is_recorded_and_leaves_the_plan():
    # a refused asynchronous update returns at once; the plan's device status
    # records it (bit 32) and the plan still decodes the batch it last had
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    for seed in range(40):
        w0 = fca_workloads.random_small(seed, max_requests=24)
        ref = oracle.plan(w0.block_tables, w0.seq_lens, 16)
        if w0.R >= 2 and ref["suffix_start"].max() > 1:
            break
    base, (nxt,) = growth_steps(w0, seed, n_steps=1)
    r = int(np.argmax(ref["suffix_start"]))
    ss = int(ref["suffix_start"][r])
    bt, sl = base.torch_inputs("cuda")[3:]
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D, min_saved_blocks=0,
                      async_update=True) as plan:
        replaced = nxt.block_tables.copy()
        replaced[r, ss - 1] = base.num_blocks - 1    # a shared entry replaced
        short = nxt.seq_lens.copy()
        short[r] = ss * 16 - 1                       # the request no longer covers its groups
        for bad_bt, bad_sl in ((replaced, nxt.seq_lens), (nxt.block_tables, short)):
            bt_t = torch.from_numpy(np.ascontiguousarray(bad_bt, np.int32)).cuda()
            sl_t = torch.from_numpy(np.ascontiguousarray(bad_sl, np.int32)).cuda()
            plan.update(bt_t, sl_t)              # queued, no status yet
            with pytest.raises(fca.FcaError) as ei:
                fca.fca_check_device_status(plan)
            assert "0x20" in str(ei.value)
            check_all(plan, base, "after a refused asynchronous update")
        bt2, sl2 = nxt.torch_inputs("cuda")[3:]
        plan.update(bt2, sl2)
        check_all(plan, nxt, "after the good asynchronous update")


def test_plan_update_async_full_size_one_token_steps():
    # the llama8b decode loop with an asynchronous plan: 20 one-token steps
    # queued back to back, one check at the end
    import shared_prefix_kv_fca_b200 as fca
    w0 = fca_workloads.make("llama8b")
    B = 16
    n_steps = 20
    final = w0.seq_lens.astype(np.int64) + n_steps
    need = int(((final + B - 1) // B - (w0.seq_lens.astype(np.int64) + B - 1) // B).sum())
    base = pooled(w0, need, int(((final + B - 1) // B).max()), 0)
    q, k, v, bt, sl = base.torch_inputs("cuda")
    cur = base
    keep = []
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D, async_update=True) as plan:
        taken = 0
        for s in range(n_steps):
            nb_before = (cur.seq_lens.astype(np.int64) + B - 1) // B
            cur = grown(cur, np.ones(w0.R, np.int64), w0.num_blocks + taken, s)
            taken += int(((cur.seq_lens.astype(np.int64) + B - 1) // B - nb_before).sum())
            bt2, sl2 = cur.torch_inputs("cuda")[3:]
            keep.append((bt2, sl2))
            plan.update(bt2, sl2)
        o, l = decode_with(plan, cur)
    assert_all_vs_oracle(cur, o, l, "llama8b after 20 asynchronous updates")


def test_update_and_decode_replayed_as_a_cuda_graph():
    # one decode step of a kept plan (asynchronous update + decode, the
    # launch dependencies between the three decode kernels included) captured
    # once as a CUDA graph; each replay, after the next step's queries and
    # tables are copied into the captured buffers, decodes that step like
    # attention over them
    torch = _torch()
    import shared_prefix_kv_fca_b200 as fca
    w0 = fca_workloads.random_small(5, max_requests=24)
    base, steps = growth_steps(w0, 5, n_steps=3)
    q, k, v, bt, sl = base.torch_inputs("cuda")
    bt_d, sl_d = bt.clone(), sl.clone()
    out = torch.empty_like(q)
    lse = torch.empty(base.R, base.Hq, dtype=torch.float32, device="cuda")
    with fca.fca_plan(bt, sl, base.num_blocks, w0.Hq, w0.Hkv, w0.D, min_saved_blocks=0,
                      async_update=True) as plan:
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):   # one eager step first (the kernels' attributes)
            plan.update(bt_d, sl_d, cap)
            fca.fca_decode(q, k, v, plan, out, lse, base.scale, cap)
        cap.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            plan.update(bt_d, sl_d, cap)
            fca.fca_decode(q, k, v, plan, out, lse, base.scale, cap)
        for s, cur in enumerate(steps):
            q2, _, _, bt2, sl2 = cur.torch_inputs("cuda")   # (same caches, new queries)
            q.copy_(q2)
            bt_d.copy_(bt2)
            sl_d.copy_(sl2)
            g.replay()
            torch.cuda.synchronize()
            assert fca.fca_check_device_status(plan) == 0
            o_ref, l_ref = oracle.paged_attention(cur.q, cur.k_cache, cur.v_cache, cur.block_tables,
                                                  cur.seq_lens, cur.scale)
            assert_close(out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                         o_ref, l_ref, f"graph replay step {s + 1}")
        del g
