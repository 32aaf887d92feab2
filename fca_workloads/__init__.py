"""Seeded synthetic decode workloads for FCA (inputs only, no method arithmetic).

Both sides of every parity check consume what this module produces: the CUDA
path through the product binding, the oracle directly.  It holds no attention
or grouping arithmetic; it only lays out paged KV caches and fills them.

Layout ("PagedAttention vs. RadixAttention", section "How PagedAttention
Works"): K and V caches are bf16 ``[num_blocks, block_size, kv_heads,
head_dim]``; each request has a row of ``block_tables`` (int32) mapping its
logical blocks to physical ones and a ``seq_len``.  Requests that share a
prompt reference the same physical blocks for every FULL block of it (step 4,
block sharing); a prompt that ends inside a block leaves that block private
to each request, holding a copy of the prompt's tail tokens (copy-on-write),
followed by the request's own tokens.  Physical ids are a seeded random
permutation of a pool holding exactly the referenced blocks.  Table entries
past ``ceil(seq_len / block_size)`` are padding: valid-looking ids of other
blocks that no kernel may read.

Values are ~N(0, 1) (Box-Muller over a counter-based generator, ``gen.c``)
rounded to bf16, drawn per physical cache slot (K: stream 1, V: stream 2,
Q: stream 0).

Named configurations (one layer's decode step each):

* ``tiny``       R=8 from 1 prompt; 4/1/64 heads; prompt 128 tokens; own
                 tokens U{1..32}.
* ``llama8b``    R=256 = 16 prompts x 16 samples; 32/8/128; prompt 2048;
                 own U{1..1024}.
* ``longctx``    R=64 = 4 x 16; 32/8/128; prompt 32768; own U{1..8192};
                 K x3 (before bf16 rounding) on a seeded uniform 1% of the
                 valid token slots, all heads and dims of each.
* ``forest``     R=512 share a 1024-token system prompt; under it 32 prompts
                 of 2048 tokens with 16 samples each; 64/8/128; own U{0..512}.
* ``mixed``      R=1024; group sizes truncated Zipf(s=1.2) on {1..64} drawn
                 until they sum to 1024 (last one cut); prompt lengths
                 log-uniform in [128, 16384] tokens, integer, not block
                 aligned; own U{1..2048}; 32/8/128.
* ``pairs``      R=1024 = 512 pairs of requests, each pair on its own prompt
                 of U{16..256} tokens; own U{256..1024}; 32/8/128.  Not one of
                 the task's configurations: the low-sharing case that the
                 planner's automatic folding of small groups is for.
"""
from __future__ import annotations

import ctypes
import bisect
import dataclasses
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libfcagen.so")
_lib = None

BLOCK_SIZE = 16

CONFIGS = {
    "tiny": dict(Hq=4, Hkv=1, D=64),
    "llama8b": dict(Hq=32, Hkv=8, D=128),
    "longctx": dict(Hq=32, Hkv=8, D=128),
    "forest": dict(Hq=64, Hkv=8, D=128),
    "mixed": dict(Hq=32, Hkv=8, D=128),
    "pairs": dict(Hq=32, Hkv=8, D=128),
}


def build(force: bool = False) -> str:
    """Compile the value generator (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.fca_gen_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p,
                                            ctypes.c_int64]
        lib.fca_gen_normal_bf16.restype = None
        _lib = lib
    return _lib


def normal_bf16(shape, seed: int, stream: int, row_factor: Optional[np.ndarray] = None,
                row_len: int = 1) -> np.ndarray:
    """uint16 bf16 bit patterns of seeded ~N(0,1) values (optionally scaled per row)."""
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16)
    rf = None
    if row_factor is not None:
        row_factor = np.ascontiguousarray(row_factor, dtype=np.float32)
        rf = row_factor.ctypes.data
    _load().fca_gen_normal_bf16(out.ctypes.data, n, 0, seed, stream, rf, row_len)
    return out.reshape(shape)


@dataclasses.dataclass
class Workload:
    name: str
    q: np.ndarray              # uint16 bf16 bits [R, Hq, D]
    k_cache: np.ndarray        # uint16 bf16 bits [num_blocks, B, Hkv, D]
    v_cache: np.ndarray
    block_tables: np.ndarray   # int32 [R, max_blocks]
    seq_lens: np.ndarray       # int32 [R]
    Hq: int
    Hkv: int
    D: int
    block_size: int
    seed: int
    description: str = ""

    @property
    def R(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def torch_inputs(self, device="cpu"):
        """(q, k_cache, v_cache, block_tables, seq_lens) as torch tensors."""
        import torch

        def bf(a):
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return (bf(self.q), bf(self.k_cache), bf(self.v_cache),
                torch.from_numpy(self.block_tables).to(device),
                torch.from_numpy(self.seq_lens).to(device))


def layout(requests, rng: np.random.Generator, block_size: int = BLOCK_SIZE,
           pad_to: Optional[int] = None):
    """Physical layout of requests given as token segments.

    ``requests[r]`` is a list of ``(key, n_tokens)``; ``key`` names a shared
    prompt segment (requests whose leading keys agree share those tokens) and
    ``None`` marks the request's own tokens.  Shared keys must come first, and
    a key names its whole path (the same key never follows two different
    paths).
    Returns (block_tables, seq_lens, num_blocks, copies) where ``copies`` is a
    list of (dst_block, dst_slot, src_block, src_slot): prompt tokens that sit
    in more than one physical block (a block that holds the end of one prompt
    segment and the start of the next, or a private block that holds a
    prompt's partial tail) take the content of the token's first copy, as
    copy-on-write leaves them.  A source slot is never a destination.
    """
    key_to_id = {}
    first_slot = {}     # (segment key, offset in the segment) -> (block, slot) of its first copy
    copies = []
    tables, lens = [], []
    next_id = 0
    for segs in requests:
        L = int(sum(n for _, n in segs))
        if L < 1:
            raise ValueError("every request needs at least one token")
        starts, path, shared = [], [], 0
        for key, n in segs:
            if key is None:
                break
            starts.append(shared)
            path.append(key)
            shared += int(n)
        row = []
        for j in range((L + block_size - 1) // block_size):
            lo, end = j * block_size, (j + 1) * block_size
            if end <= shared:
                keys = tuple(k for k, s in zip(path, starts) if s < end)
                bid = key_to_id.get((keys, j))
                new = bid is None
                if new:
                    bid = key_to_id[(keys, j)] = next_id
                    next_id += 1
            else:
                bid = next_id
                next_id += 1
                new = True
            hi = min(end, shared)
            if new and lo < hi:
                seg_lo = bisect.bisect_right(starts, lo) - 1
                seg_hi = bisect.bisect_right(starts, hi - 1) - 1
                # only a block that spans a segment boundary, or holds a
                # prompt's tail next to private tokens, can hold prompt tokens
                # that another physical block also holds
                if seg_lo != seg_hi or end > shared:
                    for t in range(lo, hi):
                        sg = bisect.bisect_right(starts, t) - 1
                        ck = (path[sg], t - starts[sg])
                        src = first_slot.get(ck)
                        if src is None:
                            first_slot[ck] = (bid, t - lo)
                        else:
                            copies.append((bid, t - lo, src[0], src[1]))
            row.append(bid)
        tables.append(row)
        lens.append(L)
    num_blocks = next_id
    perm = rng.permutation(num_blocks).astype(np.int32)
    mb = max(len(t) for t in tables)
    if pad_to is not None:
        mb = max(mb, pad_to)
    bt = rng.integers(0, num_blocks, size=(len(tables), mb), dtype=np.int32)  # padding
    for r, row in enumerate(tables):
        bt[r, :len(row)] = perm[np.asarray(row, dtype=np.int64)]
    copies = [(int(perm[d]), so, int(perm[sb]), ss) for d, so, sb, ss in copies]
    return bt, np.asarray(lens, np.int32), num_blocks, copies


def fill(name: str, requests, Hq: int, Hkv: int, D: int, seed: int,
         rng: np.random.Generator, block_size: int = BLOCK_SIZE, k_boost_frac: float = 0.0,
         k_boost: float = 3.0, poison_padding: bool = False, description: str = "") -> Workload:
    """Lay out ``requests`` and draw Q, K and V."""
    bt, sl, nb, copies = layout(requests, rng, block_size)
    R = len(requests)
    slots = nb * block_size
    row_factor = None
    if k_boost_frac > 0:
        valid = np.zeros(slots, bool)
        for r in range(R):
            L = int(sl[r])
            nblk = (L + block_size - 1) // block_size
            ids = bt[r, :nblk].astype(np.int64)
            pos = (ids[:, None] * block_size + np.arange(block_size)[None, :]).reshape(-1)[:L]
            valid[pos] = True
        cand = np.flatnonzero(valid)
        pick = rng.choice(cand, size=int(round(k_boost_frac * cand.size)), replace=False)
        row_factor = np.ones(slots, np.float32)
        row_factor[pick] = k_boost
    kv_shape = (nb, block_size, Hkv, D)
    k = normal_bf16(kv_shape, seed, 1, row_factor, Hkv * D)
    v = normal_bf16(kv_shape, seed, 2)
    if copies:
        c = np.asarray(copies, np.int64)
        k[c[:, 0], c[:, 1]] = k[c[:, 2], c[:, 3]]
        v[c[:, 0], c[:, 1]] = v[c[:, 2], c[:, 3]]
    if poison_padding:
        # slots past every referencing request's length hold NaN: never read
        used = np.zeros(slots, bool)
        for r in range(R):
            L = int(sl[r])
            nblk = (L + block_size - 1) // block_size
            ids = bt[r, :nblk].astype(np.int64)
            pos = (ids[:, None] * block_size + np.arange(block_size)[None, :]).reshape(-1)[:L]
            used[pos] = True
        bad = ~used.reshape(nb, block_size)
        k[bad] = 0x7FC0
        v[bad] = 0x7FC0
    q = normal_bf16((R, Hq, D), seed, 0)
    return Workload(name, q, k, v, bt, sl, Hq, Hkv, D, block_size, seed, description)


def _zipf_truncated(rng, s: float, kmax: int, total: int):
    k = np.arange(1, kmax + 1)
    p = k ** (-s)
    p /= p.sum()
    sizes, acc = [], 0
    while acc < total:
        g = int(rng.choice(k, p=p))
        g = min(g, total - acc)
        sizes.append(g)
        acc += g
    return sizes


def make(name: str, seed: int = 0, poison_padding: bool = False,
         prompts: Optional[int] = None) -> Workload:
    """One of the named configurations (see module docstring).  ``prompts``
    shrinks ``llama8b`` / ``longctx`` / ``forest`` to that many prompts (same
    per-prompt structure), for profiling captures that must stay small."""
    rng = np.random.default_rng(seed)
    c = CONFIGS[name]
    reqs = []
    desc = ""
    if name == "tiny":
        for _ in range(8):
            reqs.append([("p0", 128), (None, int(rng.integers(1, 33)))])
        desc = "8 requests from 1 prompt of 128 tokens, own tokens U{1..32}"
        return fill(name, reqs, seed=seed, rng=rng, poison_padding=poison_padding,
                    description=desc, **c)
    if name == "llama8b":
        for p in range(prompts or 16):
            for _ in range(16):
                reqs.append([(f"p{p}", 2048), (None, int(rng.integers(1, 1025)))])
        desc = "16 prompts x 16 samples, prompt 2048 tokens, own U{1..1024}"
        return fill(name, reqs, seed=seed, rng=rng, poison_padding=poison_padding,
                    description=desc, **c)
    if name == "longctx":
        for p in range(prompts or 4):
            for _ in range(16):
                reqs.append([(f"p{p}", 32768), (None, int(rng.integers(1, 8193)))])
        desc = "4 prompts x 16 samples, prompt 32768 tokens, own U{1..8192}, K x3 on 1% of slots"
        return fill(name, reqs, seed=seed, rng=rng, k_boost_frac=0.01,
                    poison_padding=poison_padding, description=desc, **c)
    if name == "forest":
        for p in range(prompts or 32):
            for _ in range(16):
                reqs.append([("sys", 1024), (f"p{p}", 2048), (None, int(rng.integers(0, 513)))])
        desc = "512 requests: 1024-token system prompt, 32 prompts x 2048 tokens x 16 samples, own U{0..512}"
        return fill(name, reqs, seed=seed, rng=rng, poison_padding=poison_padding,
                    description=desc, **c)
    if name == "mixed":
        sizes = _zipf_truncated(rng, 1.2, 64, 1024)
        lo, hi = math.log(128), math.log(16384)
        for gi, gsz in enumerate(sizes):
            plen = int(round(math.exp(rng.uniform(lo, hi))))
            key = f"p{gi}" if gsz > 1 else None
            for _ in range(gsz):
                reqs.append([(key, plen), (None, int(rng.integers(1, 2049)))])
        desc = (f"1024 requests in {len(sizes)} groups (Zipf 1.2 on 1..64), prompts "
                "log-U[128,16384] tokens, own U{1..2048}")
        return fill(name, reqs, seed=seed, rng=rng, poison_padding=poison_padding,
                    description=desc, **c)
    if name == "pairs":
        # the case sharing barely pays for: many pairs of requests on short prompts
        for p in range(prompts or 512):
            plen = int(rng.integers(16, 257))
            for _ in range(2):
                reqs.append([(f"p{p}", plen), (None, int(rng.integers(256, 1025)))])
        desc = "512 pairs of requests, prompts U{16..256} tokens, own U{256..1024}"
        return fill(name, reqs, seed=seed, rng=rng, poison_padding=poison_padding,
                    description=desc, **c)
    raise KeyError(name)


def random_small(seed: int, Hq: int = 4, Hkv: int = 2, D: int = 64, max_requests: int = 12,
                 poison_padding: bool = False) -> Workload:
    """A small random forest: nested prompt segments, singletons, partial blocks,
    empty own-token tails.  Sized for the oracle to finish in well under a second."""
    rng = np.random.default_rng(1000 + seed)
    R = int(rng.integers(1, max_requests + 1))
    reqs = []
    n_roots = int(rng.integers(1, 4))
    for r in range(R):
        segs = []
        root = int(rng.integers(0, n_roots))
        depth = int(rng.integers(0, 4))
        key = f"r{root}"
        for d in range(depth):
            key = key + f".{int(rng.integers(0, 2))}"
            # segment lengths depend only on the key, so equal keys agree
            seg_len = 1 + (hash_key(key) % 53)
            segs.append((key, seg_len))
        own = int(rng.integers(0, 40))
        if own == 0 and not segs:
            own = 1
        if own:
            segs.append((None, own))
        reqs.append(segs)
    return fill(f"random{seed}", reqs, Hq=Hq, Hkv=Hkv, D=D, seed=seed, rng=rng,
                poison_padding=poison_padding, description="random small forest")


def hash_key(key: str) -> int:
    """Deterministic small hash of a segment key (stable across processes)."""
    h = 2166136261
    for ch in key.encode():
        h = ((h ^ ch) * 16777619) & 0xFFFFFFFF
    return h
