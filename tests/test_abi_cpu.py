"""The C-ABI library loads and exports everything include/fca.h declares.

No GPU needed: only calls that return before touching the device are made
(status strings, version, default options, argument checks).
"""
import ctypes
import os
import re
import shutil
import subprocess

import pytest

import shared_prefix_kv_fca_b200 as fca
from shared_prefix_kv_fca_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "fca.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(fca_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    fbuild.build()
    return fca.load_library()


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    for n in ["fca_plan", "fca_decode", "fca_flat_decode", "fca_plan_get_stats", "fca_plan_export",
              "fca_plan_member_count", "fca_plan_destroy", "fca_check_device_status",
              "fca_status_string", "fca_version", "fca_plan_opts_default", "fca_plan_update"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", fca.library_path()]).decode()
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_library_is_built_for_sm100a_only():
    assert fbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_host_only_calls(lib):
    assert fca.fca_version().startswith("fca_b200")
    assert fca.fca_status_string(0) == "ok"
    assert fca.fca_status_string(2) == "block id out of range"
    o = fca.fca_plan_opts_default()
    assert (o.min_group_size, o.min_shared_blocks, o.split_tokens, o.flags, o.min_saved_blocks) == (2, 1, 0, 0, 32)


def test_argument_checks_return_status_without_a_device(lib):
    h = ctypes.c_void_p()
    opts = fca.fca_plan_opts_default()
    fake = ctypes.c_void_p(16)  # never dereferenced: every call below fails its host checks
    # no output handle
    assert lib.fca_plan(fake, 4, fake, 2, 16, 8, 4, 1, 64, ctypes.byref(opts), None, None) == 1
    # null tables
    assert lib.fca_plan(None, 4, fake, 2, 16, 8, 4, 1, 64, ctypes.byref(opts), ctypes.byref(h), None) == 1
    # Hq not a multiple of Hkv
    assert lib.fca_plan(fake, 4, fake, 2, 16, 8, 6, 4, 64, ctypes.byref(opts), ctypes.byref(h), None) == 1
    # head_dim / block_size not built
    assert lib.fca_plan(fake, 4, fake, 2, 16, 8, 4, 1, 96, ctypes.byref(opts), ctypes.byref(h), None) == 3
    assert lib.fca_plan(fake, 4, fake, 2, 32, 8, 4, 1, 64, ctypes.byref(opts), ctypes.byref(h), None) == 3
    # GQA ratio above the built maximum
    assert lib.fca_plan(fake, 4, fake, 2, 16, 8, 32, 1, 64, ctypes.byref(opts), ctypes.byref(h), None) == 3
    # bad options
    bad = fca.fca_plan_opts(1, 1, 0, 0)
    assert lib.fca_plan(fake, 4, fake, 2, 16, 8, 4, 1, 64, ctypes.byref(bad), ctypes.byref(h), None) == 1
    bad = fca.fca_plan_opts(2, 1, 100, 0)
    assert lib.fca_plan(fake, 4, fake, 2, 16, 8, 4, 1, 64, ctypes.byref(bad), ctypes.byref(h), None) == 1
    assert h.value is None
    # decode without a plan, flat decode without a plan
    assert lib.fca_decode(fake, fake, fake, None, fake, None, 0.1, None) == 1
    assert lib.fca_flat_decode(fake, fake, fake, None, fake, None, 0.1, None) == 1
    assert lib.fca_plan_destroy(None) == 0
    # the wait self-test without somewhere to put the word
    assert lib.fca_selftest_wait_timeout(None, None) == 1
    # update without a plan, or without tables
    assert lib.fca_plan_update(None, fake, 4, fake, 2, None) == 1
    assert lib.fca_plan_update(fake, None, 4, fake, 2, None) == 1
    assert lib.fca_plan_update(fake, fake, 4, None, 2, None) == 1


def test_selftest_binding_without_a_device(lib):
    # the binding's whole path up to the first CUDA call, which fails here
    # (no device); on a GPU machine the gpu-marked test runs the kernel itself
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present: tests/test_zy_failure_detection.py covers the call")
    with pytest.raises(fca.FcaError) as ei:
        fca.fca_selftest_wait_timeout(stream=0)
    assert ei.value.status == 4


def test_binding_has_every_entry_point_under_its_c_name():
    # the Python layer is a thin binding: one function per C entry point, same name
    missing = [n for n in declared_functions() if not callable(getattr(fca, n, None))]
    assert not missing, missing


def test_header_is_plain_c(tmp_path):
    # the public header compiles on its own as pedantic C99 and as C++
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    header = os.path.join(ROOT, "include", "fca.h")
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                           "-x", "c", header])
    gxx = shutil.which("g++")
    if gxx is not None:
        subprocess.check_call([gxx, "-std=c++11", "-Wall", "-Werror", "-fsyntax-only", "-x", "c++", header])


def test_c_client_links_and_runs(tmp_path, lib):
    # a C99 program linked against the library calls it through the header alone
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(fca.library_path())
    exe = str(tmp_path / "abi_c_client")
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Werror", "-I" + os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "abi_c_client.c"), "-L" + libdir, "-lfca_b200",
                           "-Wl,-rpath," + libdir, "-o", exe])
    out = subprocess.check_output([exe]).decode().strip()
    version, msg, s_plan, s_dim, no_plan, s_upd, s_self, s_destroy, mgs, msv, word = out.split("|")
    assert version == fca.fca_version()
    assert msg == "block id out of range"
    assert (s_plan, s_dim, no_plan, s_upd, s_self, s_destroy) == ("1", "3", "1", "1", "1", "0")
    assert (mgs, msv, word) == ("2", "32", "-1")


def test_binding_constants_match_the_header():
    # the plan flags the binding passes on are the header's values
    src = open(os.path.join(ROOT, "include", "fca.h")).read()
    defines = dict(re.findall(r"^#define\s+(FCA_\w+)\s+\(?([0-9xa-fA-F]+)[uUlL]*", src, flags=re.M))
    assert int(defines["FCA_PLAN_FLAT"], 0) == fca.FCA_PLAN_FLAT
    assert int(defines["FCA_PLAN_ASYNC_UPDATE"], 0) == fca.FCA_PLAN_ASYNC_UPDATE
    assert fca.FCA_PLAN_FLAT & fca.FCA_PLAN_ASYNC_UPDATE == 0
