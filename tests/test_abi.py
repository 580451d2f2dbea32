"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/attn.h declares, and rejects invalid arguments
before touching the device."""
import ctypes
import os
import re

import pytest

from attention_attn_fwd_10_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared, "no declarations parsed"
    assert sorted(_abi.EXPORTED) == declared
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in _abi.STATUS_NAMES.items():
        assert _abi.status_string(code).startswith(name)
    assert lib.attn_abi_version() == 4


def _fwd(lib, **kw):
    a = dict(q=16, k=32, v=48, o=64, lse=80, B=1, H_q=2, H_kv=2, S_q=8, S_k=8, D=64, causal=0, scale=0.125)
    a.update(kw)
    return lib.attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H_q"], a["H_kv"], a["S_q"],
                        a["S_k"], a["D"], a["causal"], a["scale"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(S_q=0), 1), (dict(S_k=-3), 1), (dict(H_q=3, H_kv=2), 1),
    (dict(causal=2), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1),
    (dict(D=96), 2), (dict(D=256), 2), (dict(q=0), 1), (dict(lse=0), 1), (dict(q=17), 3), (dict(o=8), 3),
])
def test_fwd_rejects_bad_arguments(lib, kw, code):
    assert _fwd(lib, **kw) == code


def test_fwd_options_validation(lib):
    opt = _abi.FwdOptions()
    lib.attn_fwd_default_options(ctypes.byref(opt))
    assert opt.rescale_threshold == 8.0 and opt.poly_exp_every == 8 and opt.rescale_count is None
    assert opt.persistent == 1
    for field, bad in (("rescale_threshold", -1.0), ("rescale_threshold", 17.0), ("poly_exp_every", 3)):
        o = _abi.FwdOptions(opt.rescale_threshold, opt.poly_exp_every, None)
        setattr(o, field, bad)
        r = lib.attn_fwd_ex(16, 32, 48, 64, 80, 1, 2, 2, 8, 8, 64, 0, 0.125, ctypes.byref(o), None)
        assert r == 1


def test_bwd_workspace_size(lib):
    B, H, S, D = 2, 16, 8192, 128
    n = lib.attn_bwd_workspace_size(B, H, S, D)
    assert n >= B * S * H * D * 4 + B * H * S * 4
    assert n % 256 == 0
    assert lib.attn_bwd_workspace_size(0, H, S, D) == 0
    assert lib.attn_bwd_workspace_size(B, H, S, 96) == 0


def test_bwd_rejects_bad_arguments(lib):
    p = [16] * 10
    assert lib.attn_bwd(*p, 1, 3, 2, 8, 8, 64, 0, 0.125, None) == 1
    assert lib.attn_bwd(*p, 1, 2, 2, 8, 8, 80, 0, 0.125, None) == 2
    p0 = list(p)
    p0[9] = 0
    assert lib.attn_bwd(*p0, 1, 2, 2, 8, 8, 64, 0, 0.125, None) == 1


def test_exp2_eval_rejects_bad_arguments(lib):
    assert lib.attn_exp2_poly_eval(None, None, -1, None) == 1
    assert lib.attn_exp2_poly_eval(None, None, 0, None) == 0


def test_read_probe_rejects_bad_arguments(lib):
    sink = ctypes.c_void_p(0x1000)
    assert lib.attn_read_probe(ctypes.c_void_p(0x1000), -16, sink, None) == 1   # negative size
    assert lib.attn_read_probe(ctypes.c_void_p(0x1000), 24, sink, None) == 1    # not a multiple of 16
    assert lib.attn_read_probe(ctypes.c_void_p(0x1008), 32, sink, None) == 1    # x not 16-byte aligned
    assert lib.attn_read_probe(ctypes.c_void_p(0x1000), 32, ctypes.c_void_p(0x1004), None) == 1  # sink
    assert lib.attn_read_probe(None, 32, sink, None) == 1
    assert lib.attn_read_probe(None, 0, None, None) == 0                        # nothing to read


def test_fwd_split_count(lib):
    # enough CTAs already: no split
    assert lib.attn_fwd_split_count(2, 16, 16, 8192, 8192, 1) == 1
    # one query row per head, long context: split, never more ranges than key blocks or 128
    n = lib.attn_fwd_split_count(1, 32, 8, 1, 32768, 1)
    assert 1 < n <= 128
    # packing the 4 heads of a kv group into one CTA leaves fewer CTAs: at least as many ranges
    assert lib.attn_fwd_split_count(1, 32, 8, 1, 32768, 1) >= lib.attn_fwd_split_count(1, 32, 32, 1, 32768, 1)
    assert lib.attn_fwd_split_count(1, 1, 1, 1, 128, 0) == 1  # a single key block cannot be split
    assert lib.attn_fwd_split_count(1, 1, 1, 1, 1 << 20, 0) == 128
    for S_k in (129, 1000, 4096, 70000):
        n = lib.attn_fwd_split_count(1, 4, 2, 3, S_k, 0)
        assert 1 <= n <= (S_k + 127) // 128
    assert lib.attn_fwd_split_count(0, 4, 4, 3, 100, 0) == 1
    assert lib.attn_fwd_split_count(1, 4, 3, 3, 100, 0) == 1  # H_q not a multiple of H_kv


def test_fwd_split_workspace_size(lib):
    B, H, S, D, n = 2, 8, 5, 128, 7
    size = lib.attn_fwd_split_workspace_size(B, H, S, D, n)
    assert size >= n * B * H * S * (D + 1) * 4
    assert size % 256 == 0
    assert lib.attn_fwd_split_workspace_size(B, H, S, D, 1) == 0
    assert lib.attn_fwd_split_workspace_size(B, H, S, 96, n) == 0
    assert lib.attn_fwd_split_workspace_size(B, H, S, D, 129) == 0


def test_fwd_split_rejects_bad_arguments(lib):
    p = [16] * 5
    # n_splits out of range
    assert lib.attn_fwd_split(*p, 16, 1, 2, 2, 8, 4096, 64, 0, 0.125, -1, None) == 1
    assert lib.attn_fwd_split(*p, 16, 1, 2, 2, 8, 4096, 64, 0, 0.125, 129, None) == 1
    # more than one key range needs a workspace
    assert lib.attn_fwd_split(*p, None, 1, 2, 2, 8, 4096, 64, 0, 0.125, 4, None) == 1
    # sizes are checked as for attn_fwd
    assert lib.attn_fwd_split(*p, 16, 1, 3, 2, 8, 4096, 64, 0, 0.125, 4, None) == 1
    assert lib.attn_fwd_split(*p, 16, 1, 2, 2, 8, 4096, 80, 0, 0.125, 4, None) == 2


def test_fwd_qk8_rejects_bad_arguments(lib):
    p = [16] * 5
    assert lib.attn_fwd_qk8(*p, 1, 2, 2, 8, 8, 64, 0, 0.125, None, None) == 2   # head dim 64: unsupported
    assert lib.attn_fwd_qk8(*p, 1, 3, 2, 8, 8, 128, 0, 0.125, None, None) == 1  # H_q % H_kv != 0
    assert lib.attn_fwd_qk8(16, 32, 48, None, 80, 1, 2, 2, 8, 8, 128, 0, 0.125, None, None) == 1


def test_header_is_c99_and_links(lib, tmp_path):
    """include/attn.h compiles as C99, every declared entry point resolves at link
    time, and a C program can call the host-only entry points."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    exe = tmp_path / "abi_consumer"
    lib_dir = os.path.join(ROOT, "attention_attn_fwd_10_b200")
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-pedantic-errors", "-Wno-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_consumer.c"),
           "-L", lib_dir, "-lattn", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert "abi 4" in run.stdout


def test_timeline_only_in_the_timeline_build(lib):
    """include/attn_timeline.h declares the timeline read-out; the default library
    carries no timeline, the -DATTN_TIMELINE build exports it."""
    text = open(os.path.join(ROOT, "include", "attn_timeline.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    assert sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text))) == ["attn_timeline_read"]
    assert not hasattr(lib, "attn_timeline_read")
    tl = ctypes.CDLL(build.build(timeline=True))
    assert hasattr(tl, "attn_timeline_read")
