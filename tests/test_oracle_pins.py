"""Pins of the CPU oracle against things other than itself.

Every function of the oracle is checked here against what the pages or the
mathematics fix: an independent brute force written directly from the
definition (numpy, no max-subtraction, no paging helper), closed forms, the
log-sum-exp merge identity ("ZoRRo Inference & Forest Cascade Attention",
"Core Mechanism" step 3; "Move the Query, Not the Cache", "Metodologia" item
4), worked examples printed on the pages (``tests/golden``), and, for the
planner, all-pairs longest common prefixes computed by brute force.
"""
import json
import math
import os

import numpy as np
import pytest

import fca_workloads
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def direct_softmax_attention(q, K, V, scale):
    """Attention straight from the definition: weights exp(s)/sum exp(s)."""
    s = scale * (K @ q)
    w = np.exp(s)
    z = w.sum()
    return (w[:, None] * V).sum(0) / z, math.log(z)


# ---------------------------------------------------------------- attention

@pytest.mark.parametrize("n", [1, 2, 7, 40])
def test_attend_matches_direct_definition(n):
    rng = np.random.default_rng(n)
    D = 16
    q, K, V = rng.normal(size=D), rng.normal(size=(n, D)), rng.normal(size=(n, D))
    o, lse = oracle.attend(q, K, V, 0.25)
    o_ref, lse_ref = direct_softmax_attention(q, K, V, 0.25)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    assert abs(lse - lse_ref) < 1e-12


def test_attend_closed_forms():
    rng = np.random.default_rng(7)
    D = 8
    q = rng.normal(size=D)
    # one key: its value comes back exactly, lse is its score
    k, v = rng.normal(size=(1, D)), rng.normal(size=(1, D))
    o, lse = oracle.attend(q, k, v, 0.5)
    np.testing.assert_allclose(o, v[0], rtol=0, atol=1e-15)
    assert abs(lse - 0.5 * float(q @ k[0])) < 1e-14
    # n identical keys: the mean of the values, lse = s + ln n
    n = 13
    K = np.repeat(k, n, 0)
    V = rng.normal(size=(n, D))
    o, lse = oracle.attend(q, K, V, 0.5)
    np.testing.assert_allclose(o, V.mean(0), rtol=0, atol=1e-14)
    assert abs(lse - (0.5 * float(q @ k[0]) + math.log(n))) < 1e-13
    # q = 0: the mean of the values, lse = ln L
    K = rng.normal(size=(n, D))
    o, lse = oracle.attend(np.zeros(D), K, V, 0.5)
    np.testing.assert_allclose(o, V.mean(0), rtol=0, atol=1e-14)
    assert abs(lse - math.log(n)) < 1e-13
    # empty key set: the identity of the merge
    o, lse = oracle.attend(q, np.zeros((0, D)), np.zeros((0, D)), 0.5)
    assert lse == -math.inf and not o.any()


def test_attend_is_shift_invariant_in_large_scores():
    # large logits must not overflow: exp is taken after subtracting the max
    D = 4
    q = np.full(D, 30.0)
    K = np.array([[30.0] * D, [29.0] * D])
    V = np.array([[1.0] * D, [3.0] * D])
    o, lse = oracle.attend(q, K, V, 1.0)
    s = np.array([3600.0, 3480.0])
    w = np.exp(s - s.max())
    np.testing.assert_allclose(o, (w[:, None] * V).sum(0) / w.sum(), atol=1e-12)
    assert abs(lse - (3600.0 + math.log(w.sum()))) < 1e-9


# -------------------------------------------------------------------- merge

@pytest.mark.parametrize("seed", range(6))
def test_merge_of_any_split_equals_attention_over_union(seed):
    rng = np.random.default_rng(100 + seed)
    D, n = 12, int(rng.integers(2, 60))
    q, K, V = rng.normal(size=D), rng.normal(size=(n, D)) * 2, rng.normal(size=(n, D))
    o_all, lse_all = oracle.attend(q, K, V, 0.3)
    labels = rng.integers(0, int(rng.integers(1, 6)), size=n)
    parts_o, parts_l = [], []
    for lab in range(labels.max() + 2):          # the last label is always empty
        idx = np.flatnonzero(labels == lab)
        o, l = oracle.attend(q, K[idx], V[idx], 0.3)
        parts_o.append(o)
        parts_l.append(l)
    o_m, lse_m = oracle.merge(np.array(parts_o), np.array(parts_l))
    np.testing.assert_allclose(o_m, o_all, rtol=0, atol=1e-12)
    assert abs(lse_m - lse_all) < 1e-12


def test_merge_identity_and_degenerate_cases():
    o = np.array([[1.0, 2.0]])
    m, l = oracle.merge(o, np.array([0.7]))
    np.testing.assert_allclose(m, o[0], atol=0)
    assert l == 0.7
    m, l = oracle.merge(np.array([[1.0, 2.0], [5.0, 6.0]]), np.array([0.7, -math.inf]))
    np.testing.assert_allclose(m, [1.0, 2.0], atol=0)
    assert l == 0.7
    m, l = oracle.merge(np.zeros((1, 2)), np.array([-math.inf]))
    assert l == -math.inf and not m.any()
    # two equal-weight partials average
    m, l = oracle.merge(np.array([[1.0, 0.0], [3.0, 2.0]]), np.array([1.0, 1.0]))
    np.testing.assert_allclose(m, [2.0, 1.0], atol=1e-15)
    assert abs(l - (1.0 + math.log(2.0))) < 1e-15


# ----------------------------------------------------------- paged attention

def brute_paged(w, r, h):
    """Rebuild request r's sequence token by token from its table; direct softmax."""
    G = w.Hq // w.Hkv
    kv = h // G
    L = int(w.seq_lens[r])
    toks = np.arange(L)
    blocks = w.block_tables[r, toks // w.block_size]
    K = bf16_to_f64(w.k_cache[blocks, toks % w.block_size, kv, :])
    V = bf16_to_f64(w.v_cache[blocks, toks % w.block_size, kv, :])
    q = bf16_to_f64(w.q[r, h])
    s = w.scale * (K @ q)
    m = s.max()
    e = np.exp(s - m)   # shift only for range; the result is the plain definition
    return (e[:, None] * V).sum(0) / e.sum(), m + math.log(e.sum())


@pytest.mark.parametrize("seed", range(8))
def test_paged_attention_matches_brute_force(seed):
    w = fca_workloads.random_small(seed, Hq=6, Hkv=2, D=32)
    out, lse = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens,
                                      w.scale)
    for r in range(w.R):
        for h in range(w.Hq):
            o_ref, l_ref = brute_paged(w, r, h)
            np.testing.assert_allclose(out[r, h], o_ref, rtol=0, atol=1e-12)
            assert abs(lse[r, h] - l_ref) < 1e-12


def test_paged_attention_head_mapping_and_pairs():
    # KV head 1 is all-constant: query heads G..2G-1 must see it, heads 0..G-1 must not.
    w = fca_workloads.random_small(3, Hq=4, Hkv=2, D=16)
    v = w.v_cache.copy()
    v[:, :, 1, :] = 0x3F80          # bf16 1.0
    pairs = np.array([[r, h] for r in range(w.R) for h in range(w.Hq)], np.int32)
    out, _ = oracle.paged_attention(w.q, w.k_cache, v, w.block_tables, w.seq_lens, w.scale,
                                    pairs=pairs)
    out = out.reshape(w.R, w.Hq, -1)
    np.testing.assert_allclose(out[:, 2:], 1.0, atol=1e-14)
    assert np.abs(out[:, :2] - 1.0).max() > 0.1
    full, _ = oracle.paged_attention(w.q, w.k_cache, v, w.block_tables, w.seq_lens, w.scale)
    np.testing.assert_array_equal(full, out)


def test_paged_attention_never_reads_padding():
    clean = fca_workloads.random_small(5, D=32)
    dirty = fca_workloads.random_small(5, D=32, poison_padding=True)
    np.testing.assert_array_equal(clean.block_tables, dirty.block_tables)
    assert (dirty.k_cache == 0x7FC0).any()
    o1, l1 = oracle.paged_attention(clean.q, clean.k_cache, clean.v_cache, clean.block_tables,
                                    clean.seq_lens, clean.scale)
    o2, l2 = oracle.paged_attention(dirty.q, dirty.k_cache, dirty.v_cache, dirty.block_tables,
                                    dirty.seq_lens, dirty.scale)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_paged_attention_rejects_bad_input():
    w = fca_workloads.random_small(1, D=16)
    bt = w.block_tables.copy()
    bt[0, 0] = w.num_blocks
    with pytest.raises(RuntimeError):
        oracle.paged_attention(w.q, w.k_cache, w.v_cache, bt, w.seq_lens, w.scale)
    sl = w.seq_lens.copy()
    sl[0] = 0
    with pytest.raises(RuntimeError):
        oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, sl, w.scale)


# ------------------------------------------------------------------ planner

def full_lcp_matrix(bt, seq_lens, B):
    R = bt.shape[0]
    nf = seq_lens // B
    lcp = np.zeros((R, R), np.int64)
    for r in range(R):
        for s in range(R):
            n = min(nf[r], nf[s])
            k = 0
            while k < n and bt[r, k] == bt[s, k]:
                k += 1
            lcp[r, s] = k
    return lcp


def check_plan_against_lcp(p, bt, seq_lens, B, min_group_size=2):
    """The forest must be exactly the distinct member sets of the all-pairs LCP."""
    R = bt.shape[0]
    nf = seq_lens // B
    lcp = full_lcp_matrix(bt, seq_lens, B)
    ng = len(p["a"])
    members = [set(p["members"][p["member_off"][g]:p["member_off"][g] + p["n_members"][g]])
               for g in range(ng)]
    # expected: every (set, depth range) where {s : lcp(r, s) >= d} has >= mgs members
    expected = {}
    for r in range(R):
        for d in range(1, nf[r] + 1):
            S = frozenset(np.flatnonzero(lcp[r] >= d).tolist()) | {r}
            if len(S) >= min_group_size:
                lo, hi = expected.get(S, (d, d))
                expected[S] = (min(lo, d), max(hi, d))
    got = {}
    for g in range(ng):
        S = frozenset(int(x) for x in members[g])
        assert S not in got, "duplicate member set"
        got[S] = (int(p["a"][g]) + 1, int(p["b"][g]))
    assert got == expected
    # canonical order, members ascending, parents
    keys = [(int(p["a"][g]), min(members[g])) for g in range(ng)]
    assert keys == sorted(keys)
    for g in range(ng):
        seg = p["members"][p["member_off"][g]:p["member_off"][g] + p["n_members"][g]]
        assert list(seg) == sorted(seg)
        par = int(p["parent"][g])
        if par < 0:
            assert p["a"][g] == 0
        else:
            assert members[g] < members[par] and p["b"][par] == p["a"][g]
    # suffix start = b of the deepest group containing r, and groups tile [0, b)
    for r in range(R):
        mine = sorted((int(p["a"][g]), int(p["b"][g])) for g in range(ng) if r in members[g])
        edge = 0
        for a, b in mine:
            assert a == edge
            edge = b
        assert p["suffix_start"][r] == edge
    # siblings are disjoint
    for g in range(ng):
        for h in range(g + 1, ng):
            if p["parent"][g] == p["parent"][h]:
                assert not (members[g] & members[h])


@pytest.mark.parametrize("seed", range(40))
def test_plan_matches_all_pairs_lcp(seed):
    w = fca_workloads.random_small(seed, max_requests=14)
    p = oracle.plan(w.block_tables, w.seq_lens, w.block_size)
    check_plan_against_lcp(p, w.block_tables, w.seq_lens, w.block_size)


@pytest.mark.parametrize("mgs", [3, 4])
def test_plan_min_group_size(mgs):
    for seed in range(15):
        w = fca_workloads.random_small(seed, max_requests=14)
        p = oracle.plan(w.block_tables, w.seq_lens, w.block_size, min_group_size=mgs)
        check_plan_against_lcp(p, w.block_tables, w.seq_lens, w.block_size, min_group_size=mgs)


def test_plan_min_shared_blocks_folds_short_groups():
    B = 16
    # r0..r3 share block 0 only at the top ([0,1)); r0,r1 then share [1,6); r2,r3 share [1,2)
    bt = np.array([[1, 2, 3, 4, 5, 6, 40],
                   [1, 2, 3, 4, 5, 6, 41],
                   [1, 7, 42, 0, 0, 0, 0],
                   [1, 7, 43, 0, 0, 0, 0]], np.int32)
    sl = np.array([7 * B, 7 * B, 3 * B, 3 * B], np.int32)
    p = oracle.plan(bt, sl, B)
    assert list(zip(p["a"], p["b"], p["n_members"])) == [(0, 1, 4), (1, 6, 2), (1, 2, 2)]
    assert list(p["parent"]) == [-1, 0, 0]
    p = oracle.plan(bt, sl, B, min_shared_blocks=2)
    # the 1-block root is folded into the groups below it; the [1,2) child,
    # now [0,2), is long enough to stay
    assert list(zip(p["a"], p["b"], p["n_members"])) == [(0, 6, 2), (0, 2, 2)]
    assert list(p["members"]) == [0, 1, 2, 3]
    assert list(p["parent"]) == [-1, -1]
    assert list(p["suffix_start"]) == [6, 6, 2, 2]
    p = oracle.plan(bt, sl, B, min_shared_blocks=3)
    assert list(zip(p["a"], p["b"], p["n_members"])) == [(0, 6, 2)]
    assert list(p["suffix_start"]) == [6, 6, 0, 0]


def test_plan_min_saved_blocks_hand_example():
    # three groups: r0,r1 share 3 blocks (saves 1 x 3 block reads), r2..r5
    # share 10 (3 x 10 = 30), r6..r9 share 12 (3 x 12 = 36)
    B = 16
    rows, lens = [], []
    nxt = 1000
    for members, shared, base in ((2, 3, 100), (4, 10, 200), (4, 12, 300)):
        for _ in range(members):
            rows.append([base + j for j in range(shared)] + [nxt])
            lens.append((shared + 1) * B)
            nxt += 1
    mb = max(len(x) for x in rows)
    bt = np.array([x + [0] * (mb - len(x)) for x in rows], np.int32)
    sl = np.array(lens, np.int32)
    for T, kept in ((0, [2, 4, 4]), (3, [2, 4, 4]), (4, [4, 4]), (30, [4, 4]), (31, [4]), (36, [4]), (37, [])):
        p = oracle.plan(bt, sl, B, min_saved_blocks=T)
        assert list(p["n_members"]) == kept, (T, p["n_members"])
        saved = [(int(n) - 1) * (int(b) - int(a)) for n, a, b in zip(p["n_members"], p["a"], p["b"])]
        assert all(x >= T for x in saved)
        # members of a folded group read their whole table in their own pass
        ss = np.zeros(len(rows), np.int32)
        for g in range(len(p["a"])):
            for m in p["members"][p["member_off"][g]:p["member_off"][g] + p["n_members"][g]]:
                ss[m] = p["b"][g]
        assert list(p["suffix_start"]) == list(ss)


@pytest.mark.parametrize("T", [2, 5, 12, 40])
def test_plan_min_saved_blocks_properties(T):
    """Against the unfolded forest (pinned by the all-pairs LCP test): kept
    groups are unfolded groups whose interval starts at the end of their
    nearest kept ancestor; a group is kept exactly when (members - 1) x that
    interval's length reaches T; suffix starts follow the kept groups."""
    for seed in range(20):
        w = fca_workloads.random_small(seed, max_requests=16)
        full = oracle.plan(w.block_tables, w.seq_lens, w.block_size)
        fold = oracle.plan(w.block_tables, w.seq_lens, w.block_size, min_saved_blocks=T)
        def sets(p):
            return [frozenset(int(x) for x in p["members"][p["member_off"][g]:p["member_off"][g] + p["n_members"][g]])
                    for g in range(len(p["a"]))]
        fs, ks = sets(full), sets(fold)
        kept_b = {(S, int(b)): int(a) for S, a, b in zip(ks, fold["a"], fold["b"])}
        # walk the unfolded forest root first (canonical order lists parents first)
        kept_end = {}
        for g in range(len(fs)):
            par = int(full["parent"][g])
            start = 0
            q = par
            while q >= 0 and q not in kept_end:
                q = int(full["parent"][q])
            if q >= 0:
                start = kept_end[q]
            length = int(full["b"][g]) - start
            keep = (len(fs[g]) - 1) * length >= T and length >= 1
            assert ((fs[g], int(full["b"][g])) in kept_b) == keep, (seed, g)
            if keep:
                assert kept_b[(fs[g], int(full["b"][g]))] == start
                kept_end[g] = int(full["b"][g])
        assert len(ks) == len(kept_end)
        for r in range(w.R):
            deepest = max([int(b) for S, b in zip(ks, fold["b"]) if r in S], default=0)
            assert fold["suffix_start"][r] == deepest


def test_plan_partial_blocks_and_identical_tables():
    B = 16
    bt = np.array([[3, 4, 5], [3, 4, 5], [3, 4, 6], [3, 9, 9]], np.int32)
    # r0, r1 identical tables but r1 ends inside block 2; r2 shares two full blocks
    sl = np.array([48, 40, 33, 16], np.int32)
    p = oracle.plan(bt, sl, B)
    check_plan_against_lcp(p, bt, sl, B)
    assert list(zip(p["a"], p["b"], p["n_members"])) == [(0, 1, 4), (1, 2, 3)]
    assert list(p["suffix_start"]) == [2, 2, 2, 1]
    # a block is never shared past a request's last full block
    sl2 = np.array([48, 48, 48, 16], np.int32)
    p2 = oracle.plan(bt, sl2, B)
    assert list(zip(p2["a"], p2["b"], p2["n_members"])) == [(0, 1, 4), (1, 2, 3), (2, 3, 2)]


def test_plan_no_sharing_and_single_request():
    B = 16
    bt = np.arange(12, dtype=np.int32).reshape(4, 3)
    p = oracle.plan(bt, np.full(4, 48, np.int32), B)
    assert len(p["a"]) == 0 and not p["suffix_start"].any()
    p = oracle.plan(bt[:1], np.array([48], np.int32), B)
    assert len(p["a"]) == 0


def test_plan_radix_example_golden():
    with open(os.path.join(GOLDEN, "radix_three_requests.json")) as f:
        g = json.load(f)
    p = oracle.plan(np.array(g["block_tables"], np.int32), np.array(g["seq_lens"], np.int32),
                    g["block_size"])
    for key, val in g["expected"].items():
        assert list(p[key]) == val, key


def test_plan_known_structure_of_named_configs():
    w = fca_workloads.make("tiny")
    p = oracle.plan(w.block_tables, w.seq_lens, 16)
    assert list(zip(p["a"], p["b"], p["n_members"])) == [(0, 8, 8)]
    w = fca_workloads.make("llama8b")
    p = oracle.plan(w.block_tables, w.seq_lens, 16)
    assert len(p["a"]) == 16 and set(p["n_members"]) == {16}
    assert set(p["a"]) == {0} and set(p["b"]) == {128}
    w = fca_workloads.make("forest")
    p = oracle.plan(w.block_tables, w.seq_lens, 16)
    assert (p["a"][0], p["b"][0], p["n_members"][0], p["parent"][0]) == (0, 64, 512, -1)
    assert len(p["a"]) == 33
    assert set(p["a"][1:]) == {64} and set(p["b"][1:]) == {192}
    assert set(p["n_members"][1:]) == {16} and set(p["parent"][1:]) == {0}


# ---------------------------------------------------------- byte accounting

def test_unique_kv_tokens_hand_count():
    with open(os.path.join(GOLDEN, "radix_three_requests.json")) as f:
        g = json.load(f)
    bt = np.array(g["block_tables"], np.int32)
    sl = np.array(g["seq_lens"], np.int32)
    # 3 shared full blocks + own tokens 5, 12 and 16 + 11
    assert oracle.unique_kv_tokens(bt, sl, 16, 10) == 48 + 5 + 12 + 16 + 11


def test_unique_kv_tokens_shared_partial_block_counts_its_longest_use():
    # physical block 5 is the partly filled second block of requests 0 and 1
    # (4 and 10 valid tokens) and the full first block of request 2; block 3
    # holds 2 tokens of request 2.  Each physical slot is read once, so block 5
    # counts 16 tokens (its longest use), not 4 + 10 + 16.
    bt = np.array([[7, 5], [7, 5], [5, 3]], np.int32)
    sl = np.array([20, 26, 18], np.int32)
    assert oracle.unique_kv_tokens(bt, sl, 16, 8) == 16 + 16 + 2
    # without request 2, block 5's longest use is request 1's 10 tokens
    assert oracle.unique_kv_tokens(bt[:2], sl[:2], 16, 8) == 16 + 10
    # one request alone: every slot it reads
    assert oracle.unique_kv_tokens(bt[:1], sl[:1], 16, 8) == 20


@pytest.mark.parametrize("seed", range(8))
def test_unique_kv_tokens_is_the_number_of_distinct_slots(seed):
    # brute force: the set of (physical block, slot) pairs any request reads
    w = fca_workloads.random_small(seed, max_requests=24)
    slots = set()
    for r in range(w.R):
        for t in range(int(w.seq_lens[r])):
            slots.add((int(w.block_tables[r, t // 16]), t % 16))
    assert oracle.unique_kv_tokens(w.block_tables, w.seq_lens, 16, w.num_blocks) == len(slots)


def test_kv_bytes_per_token_worked_example():
    with open(os.path.join(GOLDEN, "kv_bytes_llama3_8b.json")) as f:
        g = json.load(f)
    # one request, one layer, 1 token per block slot: bytes = tokens * Hkv * D * 2 * 2
    bt = np.arange(4, dtype=np.int32).reshape(1, 4)
    tokens = oracle.unique_kv_tokens(bt, np.array([64], np.int32), 16, 4)
    per_token_layer = g["kv_heads"] * g["head_dim"] * 2 * g["bytes_per_element"]
    assert tokens == 64
    assert per_token_layer * g["layers"] == g["page_bytes_per_token_kib"] * 1024
    total_kib = g["page_context_tokens"] * per_token_layer * g["layers"] / 1024
    assert total_kib == 12.8e6


def test_oracle_attention_independent_of_thread_count():
    # the CPU baseline times the oracle on all cores and on one; each
    # (request, head) is computed alone, so the results are bit-identical
    w = fca_workloads.random_small(3, max_requests=12)
    before = oracle.set_threads(1)
    try:
        o1, l1 = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    finally:
        oracle.set_threads(before)
    on, ln = oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    np.testing.assert_array_equal(o1, on)
    np.testing.assert_array_equal(l1, ln)
