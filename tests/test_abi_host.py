"""CPU-only checks of the C ABI: the shared library builds and loads, exports
every function include/moe_dispatch.h declares, sizes its buffers as
documented, and rejects bad arguments on the host before touching a device.
No compute call is made (the rejected calls return before any CUDA call)."""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_dispatch.h")


@pytest.fixture(scope="module")
def L():
    from combine_moe_dispatch_03_b200 import build
    build.build()
    from combine_moe_dispatch_03_b200._lib import lib
    return lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    from combine_moe_dispatch_03_b200._lib import LIB_PATH, SIGNATURES
    names = declared_functions()
    assert len(names) >= 9
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(names) == set(SIGNATURES), "binding and header disagree"
    for n in names:
        getattr(L, n)


def test_strings(L):
    assert L.moe_strerror(0) == b"ok"
    assert b"invalid" in L.moe_strerror(-1)
    assert b"cover" in L.moe_status_bit_name(8)
    assert b"sm_100a" in L.moe_version()


def test_worst_case_rows(L):
    assert L.moe_worst_case_rows(8192, 8, 256, 128) == 8192 * 8 + 256 * 127
    assert L.moe_worst_case_rows(4096, 2, 8, 16) == 8312
    assert L.moe_worst_case_rows(64, 2, 8, 8) == 184
    assert L.moe_worst_case_rows(10, 0, 8, 8) == -1
    assert L.moe_worst_case_rows(10, 2, 8, 0) == -1


def test_workspace_bytes(L):
    for T, K, E, R in [(64, 2, 8, 2), (8192, 8, 256, 8), (16384, 8, 128, 8), (4096, 2, 8, 1),
                       (0, 2, 8, 2), (1, 1, 1, 1)]:
        n = L.moe_layout_workspace_bytes(T, K, E, R)
        assert n >= 64 + 4 * E and n % 256 == 0
        assert n < 64 + 4 * E * max(T, 1) + 4 * R * max(T, 1) + 4 * E + 4096
    assert L.moe_layout_workspace_bytes(64, 2, 7, 2) == 0       # E % R
    assert L.moe_layout_workspace_bytes(63, 2, 8, 2) == 0       # T % R
    assert L.moe_layout_workspace_bytes(64, 33, 8, 2) == 0      # K > 32
    assert L.moe_layout_workspace_bytes(64, 2, 1025, 1) == 0    # E > 1024
    assert L.moe_layout_workspace_bytes(64, 2, 128, 128) == 0   # R > 64


# Fake, aligned, never-dereferenced addresses: every call below must fail a
# host check before it reaches the CUDA runtime.
A16 = 0x10000


@pytest.mark.parametrize("kw,expect", [
    (dict(H=60), -1),                  # H % 8
    (dict(xp=A16 + 2), -1),            # misaligned row buffer
    (dict(x=A16 + 8), -1),             # misaligned x
    (dict(topk=A16 + 4), -1),          # misaligned topk (int64)
    (dict(N=127), -1),                 # N_cap < A
    (dict(K=0), -1),
    (dict(K=33), -1),
    (dict(E=0), -1),
    (dict(E=1025), -1),
    (dict(T=-1), -1),
    (dict(ws=0), -1),                  # null workspace
    (dict(status=0), -1),              # null status
])
def test_permute_host_checks(L, kw, expect):
    a = dict(x=A16, topk=A16, T=64, K=2, E=8, H=64, off=A16, ws=A16, N=128, xp=A16, r2f=A16,
             f2r=A16, status=A16)
    a.update(kw)
    rc = L.moe_permute(a["x"], a["topk"], a["T"], a["K"], a["E"], a["H"], a["off"], a["ws"], 1,
                       a["N"], a["xp"], a["r2f"], a["f2r"], a["status"], None)
    assert rc == expect


@pytest.mark.parametrize("kw", [dict(R=3), dict(T=63), dict(align=0), dict(R=0), dict(R=65),
                                dict(cnt=0), dict(ws=A16 + 8)])
def test_layout_host_checks(L, kw):
    a = dict(topk=A16, T=64, K=2, E=8, R=2, align=4, cnt=A16, ws=A16)
    a.update(kw)
    rc = L.moe_dispatch_layout(a["topk"], a["T"], a["K"], a["E"], a["R"], a["align"], A16,
                               a["cnt"], A16, A16, A16, A16, a["ws"], A16, None)
    assert rc == -1


@pytest.mark.parametrize("kw", [
    dict(H=60), dict(xp=A16 + 2), dict(x=A16 + 8), dict(topk=A16 + 4), dict(N=127),
    dict(K=0), dict(K=33), dict(E=1025), dict(T=-1), dict(ws=0), dict(status=0),   # permute's
    dict(R=3), dict(T=63), dict(align=0), dict(R=0), dict(R=65), dict(cnt=0),      # layout's
    dict(ws=A16 + 8), dict(itr=0), dict(f2r=0), dict(r2f=A16 + 2),
])
def test_dispatch_host_checks(L, kw):
    """moe_dispatch runs every check of the layout and of the permute before
    it enqueues anything."""
    a = dict(x=A16, topk=A16, T=64, K=2, E=8, R=2, H=64, align=4, cnt=A16, itr=A16, ws=A16,
             N=128, xp=A16, r2f=A16, f2r=A16, status=A16)
    a.update(kw)
    rc = L.moe_dispatch(a["x"], a["topk"], a["T"], a["K"], a["E"], a["R"], a["H"], a["align"],
                        A16, a["cnt"], A16, A16, a["itr"], A16, a["ws"], 1, a["N"], a["xp"],
                        a["r2f"], a["f2r"], a["status"], None)
    assert rc == -1


@pytest.mark.parametrize("kw", [dict(wd=2), dict(H=12), dict(out=A16 + 4), dict(w=A16 + 2),
                                dict(f2r=0), dict(validate=1, r2f=0)])
def test_combine_host_checks(L, kw):
    a = dict(rows=A16, N=256, r2f=A16, f2r=A16, w=A16, wd=0, T=64, K=2, H=64, validate=0,
             out=A16)
    a.update(kw)
    rc = L.moe_combine_weighted(a["rows"], a["N"], a["r2f"], a["f2r"], a["w"], a["wd"], a["T"],
                                a["K"], a["H"], a["validate"], a["out"], A16, None)
    assert rc == -1


@pytest.mark.parametrize("kw", [dict(w=0), dict(E=0), dict(gw=A16 + 2), dict(zero_pad=1, r2f=0),
                                dict(g=A16 + 8)])
def test_combine_backward_host_checks(L, kw):
    a = dict(g=A16, rows=A16, N=256, r2f=A16, f2r=A16, w=A16, T=64, K=2, H=64, off=A16, E=8,
             zero_pad=1, gr=A16, gw=A16)
    a.update(kw)
    rc = L.moe_combine_backward(a["g"], a["rows"], a["N"], a["r2f"], a["f2r"], a["w"], 0, a["T"],
                                a["K"], a["H"], a["off"], a["E"], a["zero_pad"], a["gr"], a["gw"],
                                A16, None)
    assert rc == -1


@pytest.mark.parametrize("kw", [dict(n=0), dict(n=1025), dict(modulo=0), dict(rows=-1),
                                dict(counts=0), dict(labels=0), dict(labels=A16 + 4),
                                dict(counts=A16 + 2), dict(status=0)])
def test_segment_labels_host_checks(L, kw):
    a = dict(counts=A16, n=32, modulo=8, rows=100, labels=A16, status=A16)
    a.update(kw)
    rc = L.moe_segment_labels(a["counts"], a["n"], a["modulo"], a["rows"], a["labels"],
                              a["status"], None)
    assert rc == -1


@pytest.mark.parametrize("kw", [dict(R=0), dict(R=3), dict(rank=4), dict(rank=-1), dict(H=60),
                                dict(table=0), dict(table=A16 + 4), dict(base=0),
                                dict(ws=A16 + 8), dict(cap=-1), dict(own=0),
                                dict(claims=A16 + 4), dict(claims=A16, T=1 << 22, K=16)])
def test_permute_to_ranks_host_checks(L, kw):
    a = dict(x=A16, topk=A16, T=64, K=2, E=8, R=4, H=64, base=A16, ws=A16, table=A16, claims=None,
             cap=256, rank=0, own=A16, f2r=A16)
    a.update(kw)
    rc = L.moe_permute_to_ranks(a["x"], a["topk"], a["T"], a["K"], a["E"], a["R"], a["H"],
                                a["base"], a["ws"], a["table"], a["claims"], a["cap"], a["rank"],
                                a["own"], a["own"], 1, a["f2r"], A16, None)
    assert rc == -1


@pytest.mark.parametrize("kw", [dict(R=3), dict(R=65), dict(rows=0), dict(rows=A16 + 4),
                                dict(wd=2), dict(out=A16 + 8), dict(topk=0), dict(H=12),
                                dict(claims=A16, rank=4), dict(claims=A16, rank=-1),
                                dict(claims=A16 + 4), dict(claims=A16, T=1 << 22, K=16)])
def test_combine_from_ranks_host_checks(L, kw):
    a = dict(rows=A16, claims=None, R=4, rank=0, N=256, f2r=A16, topk=A16, E=8, w=A16, wd=0, T=64,
             K=2, H=64, out=A16)
    a.update(kw)
    rc = L.moe_combine_from_ranks(a["rows"], a["claims"], a["R"], a["rank"], a["N"], a["f2r"],
                                  a["topk"], a["E"], a["w"], a["wd"], a["T"], a["K"], a["H"],
                                  a["out"], A16, None)
    assert rc == -1


def test_expert_scale_host_checks(L):
    assert L.moe_expert_scale(A16, 256, A16, A16, 8, 64, A16, A16, A16, None) == -1  # aliasing
    assert L.moe_expert_scale(A16, 256, A16, A16, 0, 64, A16, A16 + 16, A16, None) == -1
    assert L.moe_expert_scale(A16, 256, A16, A16, 8, 63, A16, A16 + 16, A16, None) == -1


def test_binding_fails_loudly_without_library(tmp_path):
    """With the shared library absent the binding raises; nothing falls back."""
    code = (
        "import combine_moe_dispatch_03_b200._lib as L\n"
        f"L.LIB_PATH = {str(tmp_path / 'missing.so')!r}\n"
        "try:\n    L.lib()\nexcept RuntimeError as e:\n    print('RAISED', 'no CPU or Python fallback' in str(e))\n"
    )
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT)
    assert "RAISED True" in out.stdout, out.stderr


def test_product_never_imports_the_oracle():
    """The package, its binding and the benchmark's product path do not name
    the oracle (only tests, the smoke check and the CPU-baseline leg may)."""
    pkg = os.path.join(ROOT, "combine_moe_dispatch_03_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "moe_oracle" not in text, f


def test_abi_usable_from_plain_c(tmp_path):
    """A C program compiled against include/moe_dispatch.h and linked to the
    library makes host-only calls (sizes, strings, argument checks) and
    gets the documented answers: the boundary is a C ABI, not a Python one."""
    import shutil
    from combine_moe_dispatch_03_b200 import build
    build.build()
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    lib_dir = os.path.dirname(build.LIB_PATH)
    exe = str(tmp_path / "abi_from_c")
    src = os.path.join(ROOT, "tests", "c", "abi_from_c.c")
    subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", cuda_inc, src, "-o", exe, "-L", lib_dir, "-lmoe_dispatch",
                    "-Wl,-rpath," + lib_dir], check=True, capture_output=True, text=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert "C ABI checks passed" in out.stdout
