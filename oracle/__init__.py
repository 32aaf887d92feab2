"""CPU oracle for Forest Cascade Attention (FCA) decode.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
library never does, and this package imports nothing from it.

The arithmetic lives in ``fca_oracle.c`` (plain C, fp64, OpenMP over
(request, head) pairs); this module only builds and loads it and marshals
numpy arrays.  What each entry point computes, and which passage of the pages
defines it, is stated in the C file's header:

* :func:`paged_attention` -- standard softmax attention over every cached token
  of a request ("ZoRRo Inference & Forest Cascade Attention", "Overview": FCA
  is mathematically equivalent to standard attention).
* :func:`attend`, :func:`merge` -- attention over an explicit key set and the
  log-sum-exp weighted reduction of partials ("Core Mechanism" step 3).
* :func:`plan` -- group discovery by a naive trie over full-block prefixes
  ("Core Mechanism" step 1).
* :func:`unique_kv_tokens` -- every referenced physical block counted once.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fca_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        lib.oracle_attend.argtypes = [f64p, f64p, f64p, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_double, f64p, f64p]
        lib.oracle_attend.restype = ctypes.c_int
        lib.oracle_merge.argtypes = [f64p, f64p, ctypes.c_int32, ctypes.c_int32, f64p, f64p]
        lib.oracle_merge.restype = ctypes.c_int
        lib.oracle_paged_attention.argtypes = [
            u16p, u16p, u16p, i32p, ctypes.c_int32, i32p, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int64, f64p, f64p]
        lib.oracle_paged_attention.restype = ctypes.c_int
        lib.oracle_plan.argtypes = [
            i32p, ctypes.c_int32, ctypes.c_int32, i32p, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_int32, ctypes.c_int32, i32p, i32p, i32p, i32p, i32p, i32p, i32p, i32p,
            ctypes.c_int32, ctypes.c_int64]
        lib.oracle_plan.restype = ctypes.c_int
        lib.oracle_unique_kv_tokens.argtypes = [i32p, ctypes.c_int32, ctypes.c_int32, i32p,
                                                ctypes.c_int32, ctypes.c_int64]
        lib.oracle_unique_kv_tokens.restype = ctypes.c_int64
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def set_threads(n: int) -> int:
    """Threads of paged_attention's parallel loop (for timing; the result does
    not depend on it); n <= 0 leaves it.  Returns the count in force before."""
    return int(_load().oracle_set_threads(int(n)))


def _bits(a) -> np.ndarray:
    """bf16 tensor / uint16 array -> C-contiguous uint16 bit patterns."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns as uint16")
    return np.ascontiguousarray(a)


def attend(q, keys, vals, scale: float):
    """fp64 attention of one query over an explicit key set; returns (o, lse)."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    keys = np.ascontiguousarray(keys, dtype=np.float64).reshape(-1, q.shape[0])
    vals = np.ascontiguousarray(vals, dtype=np.float64).reshape(-1, q.shape[0])
    o = np.zeros(q.shape[0], np.float64)
    lse = np.zeros(1, np.float64)
    rc = _load().oracle_attend(q, keys, vals, keys.shape[0], q.shape[0], float(scale), o, lse)
    if rc:
        raise RuntimeError(f"oracle_attend failed ({rc})")
    return o, float(lse[0])


def merge(o_parts, lse_parts):
    """LSE-weighted reduction of partial results; returns (o, lse)."""
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64).reshape(-1)
    n = lse_parts.shape[0]
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64).reshape(n, -1) if n else \
        np.zeros((0, np.asarray(o_parts).shape[-1]), np.float64)
    D = o_parts.shape[1]
    o = np.zeros(D, np.float64)
    lse = np.zeros(1, np.float64)
    rc = _load().oracle_merge(np.ascontiguousarray(o_parts.reshape(-1) if n else np.zeros(1)),
                              lse_parts if n else np.zeros(1), n, D, o, lse)
    if rc:
        raise RuntimeError(f"oracle_merge failed ({rc})")
    return o, float(lse[0])


def paged_attention(q, k_cache, v_cache, block_tables, seq_lens, scale: float, pairs=None):
    """Standard paged decode attention in fp64.

    q: bf16 [R, Hq, D]; k_cache / v_cache: bf16 [num_blocks, B, Hkv, D];
    block_tables: int32 [R, max_blocks]; seq_lens: int32 [R].
    pairs: optional int array [n, 2] of (request, q_head); default all pairs.
    Returns (out [n, D] or [R, Hq, D], lse [n] or [R, Hq]) as float64.
    """
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    R, Hq, D = qb.shape
    nb, B, Hkv, D2 = kb.shape
    assert D2 == D and vb.shape == kb.shape
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    if pairs is None:
        n, pptr = R * Hq, None
    else:
        pairs = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
        n, pptr = pairs.shape[0], pairs.ctypes.data
    out = np.zeros((n, D), np.float64)
    lse = np.zeros(n, np.float64)
    rc = _load().oracle_paged_attention(qb.reshape(-1), kb.reshape(-1), vb.reshape(-1),
                                        bt.reshape(-1), bt.shape[1], sl, R, Hq, Hkv, D, B, nb,
                                        float(scale), pptr, n, out, lse)
    if rc:
        raise RuntimeError(f"oracle_paged_attention failed ({rc})")
    if pairs is None:
        return out.reshape(R, Hq, D), lse.reshape(R, Hq)
    return out, lse


def plan(block_tables, seq_lens, block_size: int, min_group_size: int = 2,
         min_shared_blocks: int = 1, min_saved_blocks: int = 0) -> dict:
    """Canonical FCA plan from the naive trie.

    min_saved_blocks: a group is kept only if (members - 1) x its length in
    blocks reaches this (0 keeps every shared prefix; the CUDA planner's
    default is 32).

    Returns dict with int32 arrays: a, b, parent, member_off, n_members (one
    entry per group, canonical order), members (concatenated, ascending per
    group) and suffix_start [R] (blocks).
    """
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    R, mb = bt.shape
    cap_g = max(R, 1)
    cap_m = int(np.sum(sl // block_size)) + R
    ng = np.zeros(1, np.int32)
    a = np.zeros(cap_g, np.int32)
    b = np.zeros(cap_g, np.int32)
    parent = np.zeros(cap_g, np.int32)
    moff = np.zeros(cap_g, np.int32)
    nm = np.zeros(cap_g, np.int32)
    members = np.zeros(max(cap_m, 1), np.int32)
    ss = np.zeros(R, np.int32)
    rc = _load().oracle_plan(bt.reshape(-1), R, mb, sl, block_size, min_group_size,
                             min_shared_blocks, min_saved_blocks, ng, a, b, parent, moff, nm,
                             members, ss,
                             cap_g, members.shape[0])
    if rc:
        raise RuntimeError(f"oracle_plan failed ({rc})")
    g = int(ng[0])
    tot = int(nm[:g].sum())
    return {"a": a[:g].copy(), "b": b[:g].copy(), "parent": parent[:g].copy(),
            "member_off": moff[:g].copy(), "n_members": nm[:g].copy(),
            "members": members[:tot].copy(), "suffix_start": ss}


def unique_kv_tokens(block_tables, seq_lens, block_size: int, num_blocks: int) -> int:
    """Tokens of KV that must be read at least once (each physical block once)."""
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    v = _load().oracle_unique_kv_tokens(bt.reshape(-1), bt.shape[0], bt.shape[1], sl,
                                        block_size, num_blocks)
    if v < 0:
        raise RuntimeError(f"oracle_unique_kv_tokens failed ({v})")
    return int(v)
