"""Forest Cascade Attention (FCA) decode on B200 -- Python binding.

A thin ctypes layer over ``libfca_b200.so`` (C ABI in ``include/fca.h``):
the functions below carry the C names and only marshal arguments (torch CUDA
tensors -> device pointers, CUDA streams -> handles).  Every step of the
decode runs in the library's CUDA kernels; there is no Python or CPU
fallback, and using any of these calls without the built library raises.

    plan = fca_plan(block_tables, seq_lens, num_blocks, Hq, Hkv, D)
    fca_decode(q, k_cache, v_cache, plan, out, lse, scale)
    fca_plan_destroy(plan)

The method ("ZoRRo Inference & Forest Cascade Attention", "Core Mechanism"):
group discovery over the requests' block tables, one grouped pass per group
over its shared prefix blocks, one pass per request over its own blocks, and
a log-sum-exp weighted merge; equal to standard attention.
"""
from __future__ import annotations

import contextlib
import ctypes
import math
import os
from typing import Optional

__all__ = [
    "FcaError", "Plan", "fca_plan", "fca_decode", "fca_flat_decode", "fca_plan_get_stats",
    "fca_plan_export", "fca_plan_member_count", "fca_plan_destroy", "fca_check_device_status",
    "fca_status_string", "fca_version", "fca_plan_opts_default", "library_path", "load_library",
    "fca_prefix_pass", "fca_suffix_pass", "fca_merge_pass", "fca_last_cuda_error",
    "FCA_PLAN_FLAT", "FCA_PLAN_ASYNC_UPDATE", "STATUS", "fca_paged_decode_static", "FCA_STATIC_SCRATCH_BYTES",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfca_b200.so")
_lib = None

FCA_PLAN_FLAT = 1
FCA_PLAN_ASYNC_UPDATE = 2
STATUS = {0: "FCA_OK", 1: "FCA_ERR_INVALID_ARG", 2: "FCA_ERR_BAD_BLOCK_ID", 3: "FCA_ERR_UNSUPPORTED",
          4: "FCA_ERR_CUDA", 5: "FCA_ERR_OOM", 6: "FCA_ERR_DEVICE_FLAG", 7: "FCA_ERR_TOO_LARGE"}
FCA_STATIC_SCRATCH_BYTES = 64 << 20


class FcaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)} ({fca_status_string(status)})"
        if status == 4:
            msg += f": {load_library().fca_last_cuda_error().decode()}"
        super().__init__(msg)


class fca_plan_opts(ctypes.Structure):
    _fields_ = [("min_group_size", ctypes.c_int32), ("min_shared_blocks", ctypes.c_int32),
                ("split_tokens", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("min_saved_blocks", ctypes.c_int32)]


class fca_plan_stats(ctypes.Structure):
    _fields_ = [("num_requests", ctypes.c_int32), ("num_groups", ctypes.c_int32),
                ("max_depth", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("split_tokens", ctypes.c_int32), ("prefix_split_tokens", ctypes.c_int32),
                ("prefix_items", ctypes.c_int32),
                ("suffix_items", ctypes.c_int32), ("num_partials", ctypes.c_int64),
                ("unique_kv_tokens", ctypes.c_int64), ("unique_kv_bytes", ctypes.c_int64),
                ("flat_kv_bytes", ctypes.c_int64), ("fca_kv_bytes", ctypes.c_int64),
                ("prefix_kv_bytes", ctypes.c_int64), ("suffix_kv_bytes", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_int64)]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libfca_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m shared_prefix_kv_fca_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.fca_plan_opts_default.argtypes = [ctypes.POINTER(fca_plan_opts)]
    lib.fca_plan_opts_default.restype = None
    lib.fca_plan.argtypes = [vp, i32, vp, i32, i32, i32, i32, i32, i32, ctypes.POINTER(fca_plan_opts),
                             ctypes.POINTER(vp), vp]
    lib.fca_plan.restype = ctypes.c_int
    lib.fca_decode.argtypes = [vp, vp, vp, vp, vp, vp, f32, vp]
    lib.fca_decode.restype = ctypes.c_int
    lib.fca_flat_decode.argtypes = [vp, vp, vp, vp, vp, vp, f32, vp]
    lib.fca_flat_decode.restype = ctypes.c_int
    lib.fca_prefix_pass.argtypes = [vp, vp, vp, vp, f32, vp]
    lib.fca_prefix_pass.restype = ctypes.c_int
    lib.fca_suffix_pass.argtypes = [vp, vp, vp, vp, f32, vp]
    lib.fca_suffix_pass.restype = ctypes.c_int
    lib.fca_merge_pass.argtypes = [vp, vp, vp, vp]
    lib.fca_merge_pass.restype = ctypes.c_int
    lib.fca_plan_get_stats.argtypes = [vp, ctypes.POINTER(fca_plan_stats)]
    lib.fca_plan_get_stats.restype = ctypes.c_int
    lib.fca_plan_export.argtypes = [vp, i32p, i32p, i32p, i32p, i32p, i32p, i32p]
    lib.fca_plan_export.restype = ctypes.c_int
    lib.fca_plan_member_count.argtypes = [vp, ctypes.POINTER(ctypes.c_int64)]
    lib.fca_plan_member_count.restype = ctypes.c_int
    lib.fca_plan_update.argtypes = [vp, vp, i32, vp, i32, vp]
    lib.fca_selftest_wait_timeout.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    lib.fca_selftest_wait_timeout.restype = ctypes.c_int
    lib.fca_plan_update.restype = ctypes.c_int
    lib.fca_plan_destroy.argtypes = [vp]
    lib.fca_plan_destroy.restype = ctypes.c_int
    lib.fca_check_device_status.argtypes = [vp, vp, i32p]
    lib.fca_check_device_status.restype = ctypes.c_int
    lib.fca_paged_decode_static.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, vp, vp, f32,
                                            vp, vp]
    lib.fca_paged_decode_static.restype = ctypes.c_int
    lib.fca_status_string.argtypes = [ctypes.c_int]
    lib.fca_status_string.restype = ctypes.c_char_p
    lib.fca_version.argtypes = []
    lib.fca_version.restype = ctypes.c_char_p
    lib.fca_last_cuda_error.argtypes = []
    lib.fca_last_cuda_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream_handle(stream, device: Optional[int] = None) -> Optional[int]:
    """The cudaStream_t of `stream`; None means torch's current stream of
    `device` (of the current device when that is None too)."""
    if stream is None:
        import torch
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _one_device(*named) -> int:
    """Index of the CUDA device that every given (name, tensor) pair is on.

    The C entry points take raw pointers and run on one device (the plan's,
    or the current one); a buffer on another device would be dereferenced
    there, which is a fault, not an error code.  So a mismatch is refused
    here, before anything reaches the library."""
    idx, first = None, None
    for name, t in named:
        if t is None:
            continue
        i = t.device.index
        if idx is None:
            idx, first = i, name
        elif i != idx:
            raise ValueError(f"{name} is on cuda:{i} but {first} is on cuda:{idx}: "
                             "every buffer of a call must be on one device")
    return idx


def _on_device(idx: Optional[int]):
    """Context that makes CUDA device `idx` current for the call (no change
    when no tensor named a device)."""
    if idx is None:
        return contextlib.nullcontext()
    import torch
    return torch.cuda.device(idx)


def _check_tables(block_tables, seq_lens) -> None:
    for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens")):
        if not t.is_cuda or str(t.dtype) != "torch.int32" or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
    if block_tables.dim() != 2 or tuple(seq_lens.shape) != (block_tables.shape[0],):
        raise ValueError("block_tables must be [R, max_blocks] and seq_lens [R]")


def _check_bf16(t, name: str, shape=None) -> None:
    if not t.is_cuda or str(t.dtype) != "torch.bfloat16" or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")


def _check_caches(k_cache, v_cache, num_blocks: int, Hkv: int, D: int) -> None:
    """The kernels read num_blocks x 16 x Hkv x D elements of each cache."""
    for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _check_bf16(t, name)
        if t.dim() != 4 or tuple(t.shape[1:]) != (16, Hkv, D) or t.shape[0] < num_blocks:
            raise ValueError(f"{name} must be [>= {num_blocks}, 16, {Hkv}, {D}], not {tuple(t.shape)}")


def _check_lse(lse, R: int, Hq: int) -> None:
    if lse is None:
        return
    if not lse.is_cuda or str(lse.dtype) != "torch.float32" or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 CUDA tensor")
    if tuple(lse.shape) != (R, Hq):
        raise ValueError(f"lse must have shape {(R, Hq)}, not {tuple(lse.shape)}")


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise FcaError(rc, where)


def fca_status_string(status: int) -> str:
    return load_library().fca_status_string(int(status)).decode()


def fca_version() -> str:
    return load_library().fca_version().decode()


def fca_last_cuda_error() -> str:
    return load_library().fca_last_cuda_error().decode()


def fca_plan_opts_default() -> fca_plan_opts:
    o = fca_plan_opts()
    load_library().fca_plan_opts_default(ctypes.byref(o))
    return o


def fca_plan(block_tables, seq_lens, num_blocks: int, num_q_heads: int, num_kv_heads: int,
             head_dim: int, block_size: int = 16, min_group_size: int = 2,
             min_shared_blocks: int = 1, split_tokens: int = 0, flat: bool = False,
             stream=None, min_saved_blocks: int = 32, async_update: bool = False) -> "Plan":
    """Group discovery + work lists.  block_tables int32 [R, max_blocks] and
    seq_lens int32 [R] are CUDA tensors.  min_saved_blocks: groups whose
    sharing saves fewer block reads ((members - 1) x length in blocks) are
    folded (0 keeps every shared prefix).  async_update: FCA_PLAN_ASYNC_UPDATE
    (Plan.update queues its work without synchronising the host; a refused
    update shows in fca_check_device_status)."""
    lib = load_library()
    _check_tables(block_tables, seq_lens)
    dev = _one_device(("block_tables", block_tables), ("seq_lens", seq_lens))
    R, mb = block_tables.shape
    o = fca_plan_opts(min_group_size, min_shared_blocks, split_tokens,
                      (FCA_PLAN_FLAT if flat else 0) | (FCA_PLAN_ASYNC_UPDATE if async_update else 0),
                      min_saved_blocks)
    handle = ctypes.c_void_p()
    with _on_device(dev):       # the plan belongs to the device current when it is built
        rc = lib.fca_plan(_ptr(block_tables), mb, _ptr(seq_lens), R, block_size, num_blocks, num_q_heads,
                          num_kv_heads, head_dim, ctypes.byref(o), ctypes.byref(handle),
                          _stream_handle(stream, dev))
    _check(rc, "fca_plan")
    return Plan(handle, R, num_q_heads, num_kv_heads, head_dim, flat, num_blocks, dev)


def _decode(fn_name: str, q, k_cache, v_cache, plan: "Plan", out, lse, scale, stream) -> None:
    lib = load_library()
    if scale is None:
        scale = 1.0 / math.sqrt(plan.head_dim)
    qshape = (plan.num_requests, plan.num_q_heads, plan.head_dim)
    _check_bf16(q, "q", qshape)
    _check_bf16(out, "out", qshape)
    _check_caches(k_cache, v_cache, plan.num_blocks, plan.num_kv_heads, plan.head_dim)
    _check_lse(lse, plan.num_requests, plan.num_q_heads)
    _plan_device(plan, ("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out), ("lse", lse))
    rc = getattr(lib, fn_name)(_ptr(q), _ptr(k_cache), _ptr(v_cache), plan.handle, _ptr(out),
                               _ptr(lse), float(scale), _stream_handle(stream, plan.device))
    _check(rc, fn_name)


def _plan_device(plan: "Plan", *named) -> None:
    """Every buffer of a call that takes a plan must be on the plan's device
    (the library makes that device current for the call)."""
    idx = _one_device(*named)
    if idx is not None and plan.device is not None and idx != plan.device:
        name = next(n for n, t in named if t is not None)
        raise ValueError(f"{name} is on cuda:{idx} but the plan belongs to cuda:{plan.device}")


def fca_decode(q, k_cache, v_cache, plan: "Plan", out, lse=None, scale=None, stream=None) -> None:
    """Grouped prefix pass + per-request pass + LSE merge into out (and lse)."""
    _decode("fca_decode", q, k_cache, v_cache, plan, out, lse, scale, stream)


def fca_flat_decode(q, k_cache, v_cache, plan: "Plan", out, lse=None, scale=None,
                    stream=None) -> None:
    """Flat (non-cascaded) paged decode; plan must be built with flat=True."""
    _decode("fca_flat_decode", q, k_cache, v_cache, plan, out, lse, scale, stream)


def fca_paged_decode_static(q, k_cache, v_cache, block_tables, seq_lens, num_blocks: int, out, lse=None,
                            scale=None, dev_status=None, stream=None) -> None:
    """Flat paged decode that allocates nothing (no plan; work list and
    partials in the library's fixed 64 MiB device array).  q/out bf16
    [R, Hq, D]; caches bf16 [num_blocks, 16, Hkv, D]; block_tables int32
    [R, max_blocks] and seq_lens int32 [R] CUDA tensors; dev_status an int32
    CUDA tensor of one element (zeroed by the caller) or None.  Calls on one
    device must be ordered: they share the array."""
    lib = load_library()
    _check_bf16(q, "q")
    if q.dim() != 3:
        raise ValueError(f"q must be [R, Hq, D], not {tuple(q.shape)}")
    R, Hq, D = q.shape
    _check_bf16(out, "out", q.shape)
    if k_cache.dim() != 4:
        raise ValueError(f"k_cache must be [num_blocks, 16, Hkv, D], not {tuple(k_cache.shape)}")
    Hkv = k_cache.shape[2]
    _check_caches(k_cache, v_cache, num_blocks, Hkv, D)
    _check_tables(block_tables, seq_lens)
    if block_tables.shape[0] != R:
        raise ValueError(f"block_tables must have {R} rows (one per request of q)")
    _check_lse(lse, R, Hq)
    if dev_status is not None and (not dev_status.is_cuda or str(dev_status.dtype) != "torch.int32"
                                   or dev_status.numel() < 1):
        raise ValueError("dev_status must be an int32 CUDA tensor of at least one element")
    dev = _one_device(("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("block_tables", block_tables),
                      ("seq_lens", seq_lens), ("out", out), ("lse", lse), ("dev_status", dev_status))
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    with _on_device(dev):       # the call runs on (and finds its array on) the current device
        rc = lib.fca_paged_decode_static(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                         block_tables.shape[1], _ptr(seq_lens), R, num_blocks, Hq, Hkv, D,
                                         _ptr(out), _ptr(lse), float(scale), _ptr(dev_status),
                                         _stream_handle(stream, dev))
    _check(rc, "fca_paged_decode_static")


def _check_pass_inputs(q, k_cache, v_cache, plan: "Plan") -> None:
    _check_bf16(q, "q", (plan.num_requests, plan.num_q_heads, plan.head_dim))
    _check_caches(k_cache, v_cache, plan.num_blocks, plan.num_kv_heads, plan.head_dim)
    _plan_device(plan, ("q", q), ("k_cache", k_cache), ("v_cache", v_cache))


def fca_prefix_pass(q, k_cache, v_cache, plan: "Plan", scale=None, stream=None) -> None:
    """Grouped pass over shared prefix blocks only (writes the plan's partials)."""
    scale = 1.0 / math.sqrt(plan.head_dim) if scale is None else scale
    _check_pass_inputs(q, k_cache, v_cache, plan)
    _check(load_library().fca_prefix_pass(_ptr(q), _ptr(k_cache), _ptr(v_cache), plan.handle,
                                          float(scale), _stream_handle(stream, plan.device)), "fca_prefix_pass")


def fca_suffix_pass(q, k_cache, v_cache, plan: "Plan", scale=None, stream=None) -> None:
    """Per-request pass over own blocks only (writes the plan's partials)."""
    scale = 1.0 / math.sqrt(plan.head_dim) if scale is None else scale
    _check_pass_inputs(q, k_cache, v_cache, plan)
    _check(load_library().fca_suffix_pass(_ptr(q), _ptr(k_cache), _ptr(v_cache), plan.handle,
                                          float(scale), _stream_handle(stream, plan.device)), "fca_suffix_pass")


def fca_merge_pass(plan: "Plan", out, lse=None, stream=None) -> None:
    """Log-sum-exp merge of the plan's partials into out (and lse)."""
    _check_bf16(out, "out", (plan.num_requests, plan.num_q_heads, plan.head_dim))
    _check_lse(lse, plan.num_requests, plan.num_q_heads)
    _plan_device(plan, ("out", out), ("lse", lse))
    _check(load_library().fca_merge_pass(plan.handle, _ptr(out), _ptr(lse), _stream_handle(stream, plan.device)),
           "fca_merge_pass")


def fca_plan_get_stats(plan: "Plan") -> dict:
    st = fca_plan_stats()
    _check(load_library().fca_plan_get_stats(plan.handle, ctypes.byref(st)), "fca_plan_get_stats")
    return {name: getattr(st, name) for name, _ in fca_plan_stats._fields_}


def fca_plan_member_count(plan: "Plan") -> int:
    n = ctypes.c_int64()
    _check(load_library().fca_plan_member_count(plan.handle, ctypes.byref(n)),
           "fca_plan_member_count")
    return int(n.value)


def fca_plan_export(plan: "Plan") -> dict:
    """Canonical forest as numpy int32 arrays (synchronises the device)."""
    import numpy as np
    st = fca_plan_get_stats(plan)
    ng, R = st["num_groups"], st["num_requests"]
    nm = fca_plan_member_count(plan)
    arr = {k: np.zeros(max(ng, 1), np.int32) for k in ("a", "b", "parent", "member_off", "n_members")}
    arr["members"] = np.zeros(max(nm, 1), np.int32)
    arr["suffix_start"] = np.zeros(R, np.int32)

    def p(a):
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    rc = load_library().fca_plan_export(plan.handle, p(arr["a"]), p(arr["b"]), p(arr["parent"]),
                                        p(arr["member_off"]), p(arr["n_members"]),
                                        p(arr["members"]), p(arr["suffix_start"]))
    _check(rc, "fca_plan_export")
    for k in ("a", "b", "parent", "member_off", "n_members"):
        arr[k] = arr[k][:ng]
    arr["members"] = arr["members"][:nm]
    return arr


def fca_check_device_status(plan: "Plan", stream=None) -> int:
    """Raw device error word (0 = fine); raises FcaError when it is set."""
    code = ctypes.c_int32()
    rc = load_library().fca_check_device_status(plan.handle, _stream_handle(stream, plan.device),
                                                ctypes.byref(code))
    if rc not in (0, 6):
        _check(rc, "fca_check_device_status")
    if rc == 6:
        raise FcaError(rc, f"fca_check_device_status (word {code.value:#x})")
    return int(code.value)


def fca_plan_update(plan: "Plan", block_tables, seq_lens, stream=None) -> None:
    """The plan for the next decode step of the same batch: new lengths and
    grown tables over the plan's forest (the C call of the same name)."""
    _check_tables(block_tables, seq_lens)
    _plan_device(plan, ("block_tables", block_tables), ("seq_lens", seq_lens))
    R, mb = block_tables.shape
    _check(load_library().fca_plan_update(plan.handle, _ptr(block_tables), mb, _ptr(seq_lens), R,
                                          _stream_handle(stream, plan.device)), "fca_plan_update")


def fca_selftest_wait_timeout(stream=None) -> int:
    """Run the kernel whose bounded wait is made to run out; return the device
    error word it recorded (bit 1: the wait gave up after its 1 s bound)."""
    word = ctypes.c_int32()
    _check(load_library().fca_selftest_wait_timeout(_stream_handle(stream), ctypes.byref(word)),
           "fca_selftest_wait_timeout")
    return int(word.value)


def fca_plan_destroy(plan: "Plan") -> None:
    plan.close()


class Plan:
    """Owner of an fca_plan_t handle."""

    def __init__(self, handle: ctypes.c_void_p, R: int, Hq: int, Hkv: int, D: int, flat: bool,
                 num_blocks: int, device: Optional[int] = None):
        self.handle = handle
        self.num_requests, self.num_q_heads, self.num_kv_heads, self.head_dim = R, Hq, Hkv, D
        self.flat = flat
        self.num_blocks = num_blocks
        self.device = device        # CUDA device index the plan belongs to

    def stats(self) -> dict:
        """Sizes and byte counts (fca_plan_get_stats): of the plan as built or
        last updated synchronously; an asynchronously updated plan keeps the
        figures of the plan as built."""
        return fca_plan_get_stats(self)

    def update(self, block_tables, seq_lens, stream=None) -> None:
        """Next decode step of the same batch (fca_plan_update): new lengths
        and grown tables over this plan's forest."""
        fca_plan_update(self, block_tables, seq_lens, stream)

    def export(self) -> dict:
        return fca_plan_export(self)

    def close(self) -> None:
        if self.handle is not None and self.handle.value:
            _check(load_library().fca_plan_destroy(self.handle), "fca_plan_destroy")
        self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
