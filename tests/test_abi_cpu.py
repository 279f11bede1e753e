"""Host-side checks of the C ABI (CPU only, no compute call): the library
builds and loads without a GPU, exports every symbol the header declares, and
rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "adafuse.h")


@pytest.fixture(scope="module")
def L():
    from adapter_merge_b200 import build
    build.build()
    import adapter_merge_b200 as am
    return am.lib()


def declared_functions():
    with open(HEADER) as f:
        src = f.read()
    return sorted(set(re.findall(r"ADAFUSE_API\s+[\w\s\*]+?\b(adafuse_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("adafuse_pregate", "adafuse_merge", "adafuse_apply", "adafuse_plan_create",
                 "adafuse_plan_destroy", "adafuse_plan_status", "adafuse_strerror"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    import adapter_merge_b200 as am
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) == set(am.EXPORTS)


def test_only_the_abi_is_exported(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", L._name], capture_output=True, text=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {s for s in syms if s.startswith("adafuse_")}
    assert ours == set(declared_functions())


def test_strerror_and_version(L):
    assert L.adafuse_version() == 100
    for code in range(0, 7):
        assert isinstance(L.adafuse_strerror(code), bytes)
    assert L.adafuse_strerror(99) == b"unknown error"


def test_argument_errors_need_no_device(L):
    import adapter_merge_b200 as am
    P = ctypes.c_void_p
    # pregate: null pointers, bad sizes, unsupported E/k, unknown flags
    assert L.adafuse_pregate(None, 1, 8, 8, None, None, 4, 2, 0, None, None, None) == am.ERR_INVALID_ARG
    fake = P(256)
    assert L.adafuse_pregate(fake, 0, 8, 8, fake, None, 4, 2, 0, fake, fake, None) == am.ERR_INVALID_ARG
    assert L.adafuse_pregate(fake, 1, 8, 4, fake, None, 4, 2, 0, fake, fake, None) == am.ERR_INVALID_ARG
    assert L.adafuse_pregate(fake, 1, 8, 8, fake, None, 33, 2, 0, fake, fake, None) == am.ERR_UNSUPPORTED
    assert L.adafuse_pregate(fake, 1, 8, 8, fake, None, 4, 5, 0, fake, fake, None) == am.ERR_UNSUPPORTED
    assert L.adafuse_pregate(fake, 1, 8, 8, fake, None, 4, 0, 0, fake, fake, None) == am.ERR_UNSUPPORTED
    assert L.adafuse_pregate(fake, 1, 8, 8, fake, None, 4, 2, 1 << 7, fake, fake, None) == am.ERR_INVALID_ARG
    # segments
    assert L.adafuse_segments(None, 4, 2, 4, fake, fake, fake, None, None) == am.ERR_INVALID_ARG
    assert L.adafuse_segments(fake, 4, 2, 40, fake, fake, fake, None, None) == am.ERR_UNSUPPORTED
    # plan: null, bad E / r, unaligned pointers, bad dims
    h = P()
    assert L.adafuse_plan_create(ctypes.byref(h), None, 1, 4, 8, 0) == am.ERR_INVALID_ARG
    lin = am.Linear(4096, 8192, 16384, 32768, 16, 16, 8 * 16, 16 * 8)
    arr = (am.Linear * 1)(lin)
    assert L.adafuse_plan_create(ctypes.byref(h), arr, 1, 0, 8, 0) == am.ERR_UNSUPPORTED
    assert L.adafuse_plan_create(ctypes.byref(h), arr, 1, 4, 12, 0) == am.ERR_UNSUPPORTED
    assert L.adafuse_plan_create(ctypes.byref(h), arr, 1, 4, 8, 3) == am.ERR_INVALID_ARG
    assert L.adafuse_plan_create(ctypes.byref(h), arr, 1, 4, 8, (1 << 31) | 2) == am.ERR_INVALID_ARG
    assert L.adafuse_plan_create(ctypes.byref(h), arr, 1, 4, 8, am.PLAN_Y_F32 | 4) == am.ERR_INVALID_ARG
    bad = (am.Linear * 1)(am.Linear(4096 + 2, 8192, 16384, 32768, 16, 16, 128, 128))
    assert L.adafuse_plan_create(ctypes.byref(h), bad, 1, 4, 8, 0) == am.ERR_UNSUPPORTED
    bad = (am.Linear * 1)(am.Linear(4096, 8192, 16384, 32768, 12, 16, 128, 128))
    assert L.adafuse_plan_create(ctypes.byref(h), bad, 1, 4, 8, 0) == am.ERR_UNSUPPORTED
    bad = (am.Linear * 1)(am.Linear(4096, 8192, 16384, 32768, 16, 16, 64, 128))
    assert L.adafuse_plan_create(ctypes.byref(h), bad, 1, 4, 8, 0) == am.ERR_INVALID_ARG
    # entry points on a null plan
    assert L.adafuse_merge(None, fake, fake, 2, None) == am.ERR_INVALID_ARG
    assert L.adafuse_switch(None, fake, fake, fake, fake, 2, None) == am.ERR_INVALID_ARG
    assert L.adafuse_merge_per_linear(None, fake, fake, 2, None) == am.ERR_INVALID_ARG
    assert L.adafuse_apply(None, fake, fake, 4, fake, fake, 2, fake, 1 << 20, None) == am.ERR_INVALID_ARG
    assert L.adafuse_apply_workspace_bytes(None, 4, 2) == 0
    v = ctypes.c_int32(0)
    assert L.adafuse_plan_status(None, None, ctypes.byref(v)) == am.ERR_INVALID_ARG
    # rounding: null buffers, negative n, misaligned or overlapping buffers (no launch)
    assert L.adafuse_round_bf16(None, fake, 4, None) == am.ERR_INVALID_ARG
    assert L.adafuse_round_bf16(fake, None, 4, None) == am.ERR_INVALID_ARG
    assert L.adafuse_round_bf16(fake, fake, -1, None) == am.ERR_INVALID_ARG
    assert L.adafuse_round_bf16(P(258), P(4096), 4, None) == am.ERR_INVALID_ARG
    assert L.adafuse_round_bf16(P(256), P(4097), 4, None) == am.ERR_INVALID_ARG
    assert L.adafuse_round_bf16(P(256), P(256 + 14), 4, None) == am.ERR_INVALID_ARG
    assert L.adafuse_round_bf16(P(256 + 6), P(256), 4, None) == am.ERR_INVALID_ARG
    assert L.adafuse_round_bf16(None, None, 0, None) == am.OK
    assert L.adafuse_plan_last_launches(None) == 0
    L.adafuse_plan_destroy(None)


def test_binding_has_no_fallback(tmp_path, monkeypatch):
    """Without the shared library the binding raises instead of computing."""
    import adapter_merge_b200 as am
    monkeypatch.setattr(am, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(am, "_lib", None)
    with pytest.raises(RuntimeError):
        am.lib()


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "adafuse.h"

int main(void)
{
    adafuse_plan* plan = NULL;
    adafuse_linear lin;
    memset(&lin, 0, sizeof lin);
    if (adafuse_version() != 100) return 1;
    if (strcmp(adafuse_strerror(99), "unknown error") != 0) return 2;
    if (adafuse_pregate(NULL, 1, 8, 8, NULL, NULL, 4, 2, 0, NULL, NULL, NULL) != ADAFUSE_ERR_INVALID_ARG) return 3;
    if (adafuse_plan_create(&plan, NULL, 1, 4, 8, 0) != ADAFUSE_ERR_INVALID_ARG) return 4;
    if (adafuse_merge(NULL, NULL, NULL, 2, NULL) != ADAFUSE_ERR_INVALID_ARG) return 5;
    if (adafuse_apply_workspace_bytes(NULL, 4, 2) != 0) return 6;
    adafuse_plan_destroy(NULL);
    printf("ok %s\n", adafuse_strerror(ADAFUSE_ERR_UNSUPPORTED));
    return 0;
}
"""


def test_plain_c_client_builds_and_links(L, tmp_path):
    """The header is a C ABI: a C11 program (no CUDA headers, -pedantic
    -Werror) includes it, links the library and makes the calls that need no
    device."""
    import subprocess
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(L._name)
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                           "-L", libdir, "-l:" + os.path.basename(L._name), "-Wl,-rpath," + libdir])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("ok ")


def test_product_is_independent_of_the_oracle():
    """The library, its binding and its build never name, import or link the
    oracle, and the oracle never includes the library's sources: the two
    share only the seeded input generators."""
    pkg = os.path.join(ROOT, "adapter_merge_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                with open(os.path.join(dirpath, f), errors="replace") as fh:
                    text = fh.read()
                assert "oracle" not in text.lower(), os.path.join(dirpath, f)
    with open(os.path.join(ROOT, "include", "adafuse.h")) as fh:
        assert "oracle" not in fh.read().lower()
    odir = os.path.join(ROOT, "oracle")
    for f in os.listdir(odir):
        if f.endswith((".py", ".c", ".h")):
            with open(os.path.join(odir, f)) as fh:
                text = fh.read()
            assert not re.search(r"^\s*(import|from)\s+adapter_merge_b200", text, re.M), f
            assert not re.search(r"^\s*#\s*include\s*[<\"][^>\"]*(adafuse|csrc|ptx)", text, re.M), f
            assert "libadafuse" not in text, f


def test_input_generators_import_neither_side():
    """synth/ (seeded inputs for both sides) imports neither the library nor
    the oracle."""
    sdir = os.path.join(ROOT, "synth")
    for f in os.listdir(sdir):
        if f.endswith(".py"):
            with open(os.path.join(sdir, f)) as fh:
                text = fh.read()
            assert not re.search(r"^\s*(import|from)\s+(oracle|adapter_merge_b200)\b", text, re.M), f
