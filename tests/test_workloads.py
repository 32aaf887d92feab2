"""The seeded input generator shared by the oracle and the CUDA path.

It holds none of the method's arithmetic, but every parity test trusts it to
lay out shared prompts the way a paged cache does: requests whose leading
prompt segments agree hold the same K/V for those tokens, full blocks of a
shared prompt are one physical block, a prompt's partial tail is a private
copy, own tokens are private, and the same seed gives the same arrays.
"""
import itertools

import numpy as np
import pytest

import fca_workloads

B = fca_workloads.BLOCK_SIZE


def random_requests(rng, n):
    reqs = []
    for _ in range(n):
        segs, key = [], "r%d" % rng.integers(0, 2)
        for _ in range(int(rng.integers(0, 4))):
            key = key + ".%d" % rng.integers(0, 2)
            segs.append((key, 1 + fca_workloads.hash_key(key) % 45))
        own = int(rng.integers(0, 30))
        if own or not segs:
            segs.append((None, max(own, 1)))
        reqs.append(segs)
    return reqs


def gathered(cache, bt, r, L):
    t = np.arange(L)
    return cache[bt[r, t // B], t % B]


def common_prefix_tokens(a, b):
    n = 0
    for (ka, la), (kb, lb) in zip(a, b):
        if ka is None or kb is None or ka != kb:
            break
        n += la
    return n


@pytest.mark.parametrize("seed", range(12))
def test_shared_prompts_are_shared(seed):
    rng = np.random.default_rng(900 + seed)
    reqs = random_requests(rng, int(rng.integers(2, 14)))
    w = fca_workloads.fill("gen", reqs, Hq=4, Hkv=2, D=64, seed=seed, rng=rng)
    assert w.R == len(reqs)
    assert list(w.seq_lens) == [sum(n for _, n in segs) for segs in reqs]
    owners = {}
    for r in range(w.R):
        for j in range((int(w.seq_lens[r]) + B - 1) // B):
            owners.setdefault(int(w.block_tables[r, j]), set()).add(r)
    for a, b in itertools.combinations(range(w.R), 2):
        n = common_prefix_tokens(reqs[a], reqs[b])
        # same K/V for every shared prompt token, full blocks or partial tail
        np.testing.assert_array_equal(gathered(w.k_cache, w.block_tables, a, n),
                                      gathered(w.k_cache, w.block_tables, b, n))
        np.testing.assert_array_equal(gathered(w.v_cache, w.block_tables, a, n),
                                      gathered(w.v_cache, w.block_tables, b, n))
        # its full blocks are the same physical blocks
        full = n // B
        np.testing.assert_array_equal(w.block_tables[a, :full], w.block_tables[b, :full])
        # past the shared prompt the two requests hold no block in common
        la = (int(w.seq_lens[a]) + B - 1) // B
        lb = (int(w.seq_lens[b]) + B - 1) // B
        assert not set(w.block_tables[a, full:la].tolist()) & set(w.block_tables[b, full:lb].tolist())
    # every physical block is referenced (the pool holds exactly the blocks in use)
    assert set(owners) == set(range(w.num_blocks))


def test_same_seed_same_arrays():
    def make():
        rng = np.random.default_rng(5)
        return fca_workloads.fill("gen", random_requests(rng, 9), Hq=8, Hkv=2, D=128, seed=5, rng=rng)
    a, b = make(), make()
    for name in ("q", "k_cache", "v_cache", "block_tables", "seq_lens"):
        np.testing.assert_array_equal(getattr(a, name), getattr(b, name), err_msg=name)


def test_poisoned_padding_is_only_where_no_request_reads():
    rng = np.random.default_rng(3)
    reqs = [[("p", 40), (None, 5)], [("p", 40), (None, 17)], [(None, 3)]]
    w = fca_workloads.fill("gen", reqs, Hq=4, Hkv=1, D=64, seed=3, rng=rng, poison_padding=True)
    nan_bits = 0x7FC0
    for r in range(w.R):
        L = int(w.seq_lens[r])
        assert not (gathered(w.k_cache, w.block_tables, r, L) == nan_bits).any()
    assert (w.k_cache == nan_bits).any()      # padding exists and is poisoned
