"""The C ABI library loads without a GPU and exports everything the header
declares; the header is plain C and every entry point links from a C program;
host-side argument checks reject bad calls before touching CUDA."""
import ctypes as C
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "surelock.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set(re.findall(r"\b(sl_[a-z0-9_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from token_locking_b200 import _abi
    if not os.path.exists(_abi.LIB_PATH):
        from token_locking_b200 import build
        build.build()
    return _abi.lib()


def test_every_declared_symbol_is_exported(lib):
    from token_locking_b200 import _abi
    declared = _declared()
    assert len(declared) >= 25
    for name in sorted(declared):
        assert hasattr(lib, name), f"{name} declared in include/surelock.h but not exported"
        assert name in _abi.SIGNATURES, f"{name} has no ctypes signature"
    assert set(_abi.SIGNATURES) == declared


def test_version_and_error_strings(lib):
    assert b"sm_100a" in lib.sl_version()
    assert isinstance(lib.sl_last_error(), bytes)


def test_host_side_argument_checks(lib):
    from token_locking_b200 import _abi as A
    out = C.c_void_p()
    assert lib.sl_model_create(None, None, C.byref(out)) == A.SL_ERR_INVALID
    cfg = A.Config(2, 64, 4, 15, 256, 512, 511, 1e-5, 1e4, A.SL_F32)   # 4 * 15 != 64
    w = A.Weights()
    assert lib.sl_model_create(C.byref(cfg), C.byref(w), C.byref(out)) == A.SL_ERR_INVALID
    assert b"head_dim" in lib.sl_last_error()
    cfg = A.Config(2, 64, 4, 16, 256, 512, 512, 1e-5, 1e4, A.SL_F32)   # mask id out of range
    assert lib.sl_model_create(C.byref(cfg), C.byref(w), C.byref(out)) == A.SL_ERR_INVALID
    assert lib.sl_active_create(0, 10, C.byref(out)) == A.SL_ERR_INVALID
    assert lib.sl_active_create(1, 0, C.byref(out)) == A.SL_ERR_INVALID
    assert lib.sl_active_create(A.SL_MAX_BATCH + 1, 8, C.byref(out)) == A.SL_ERR_INVALID
    assert lib.sl_kv_cache_create(None, 1, 8, C.byref(out)) == A.SL_ERR_INVALID
    p = A.LockParams(0.01, -1.0, 1, -1)
    assert lib.sl_kl_lock(None, 512, 0, 0, None, None, None, None, None, C.byref(p),
                          None, None, None, None, None, None) == A.SL_ERR_INVALID
    assert lib.sl_unmask_topk(None, None, None, 0, 1, 1, None, None, None) == A.SL_ERR_INVALID
    assert lib.sl_compact_active(None, None, None, None, 0, None) == A.SL_ERR_INVALID
    assert lib.sl_step(None, None, None, None, None, None) == A.SL_ERR_INVALID
    assert lib.sl_sampler_step(None, None) == A.SL_ERR_INVALID
    # GEMM: K must be a multiple of 64; a bad epilogue code is rejected
    assert lib.sl_gemm_bf16(0, 16, 8, 100, 16, None, 128, 16, 128, None, 128, 1, 0, None) == A.SL_ERR_INVALID
    assert lib.sl_gemm_bf16(9, 16, 8, 128, 16, None, 128, 16, 128, None, 128, 1, 0, None) == A.SL_ERR_INVALID
    assert lib.sl_gemm_bf16(0, 16, 8, 128, 16, None, 128, 16, 128, None, 128, 1, 3, None) == A.SL_ERR_INVALID
    assert lib.sl_model_set_attention(None, 16, 1) == A.SL_ERR_INVALID
    assert lib.sl_model_set_ablation(None, A.ABLATE_NO_KV_CACHE) == A.SL_ERR_INVALID
    # output pitch: fp32 rows need ldo % 4 == 0, bf16 rows ldo % 8 == 0, ldo >= N
    assert lib.sl_gemm_bf16(1, 16, 8, 128, 16, None, 128, 16, 130, None, 128, 1, 0, None) == A.SL_ERR_INVALID
    assert lib.sl_gemm_bf16(0, 16, 8, 128, 16, None, 128, 16, 132, None, 128, 1, 0, None) == A.SL_ERR_INVALID
    assert lib.sl_gemm_bf16(0, 16, 8, 128, 16, None, 128, 16, 64, None, 128, 1, 0, None) == A.SL_ERR_INVALID


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not on PATH")
def test_header_is_plain_c_and_links(tmp_path):
    """include/surelock.h compiles as strict C99 (no C++ in the boundary), and a
    C program that takes the address of every declared entry point links
    against libsurelock.so and runs a host-side check through it."""
    from token_locking_b200 import _abi
    from token_locking_b200 import build
    build.build()
    names = sorted(_declared())
    src = tmp_path / "use_abi.c"
    src.write_text(
        '#include "surelock.h"\n#include <string.h>\n'
        "typedef void (*fnp)(void);\n"
        "static const fnp entry_points[] = {\n"
        + "".join(f"  (fnp){n},\n" for n in names)
        + "};\n"
        "int main(void) {\n"
        "  sl_lock_params lp = {0.05f, -1.0f, 1, -1, 0};\n"
        "  (void)lp;\n"
        "  if (sizeof(entry_points) / sizeof(entry_points[0]) != %d) return 2;\n" % len(names)
        + "  if (!strstr(sl_version(), \"sm_100a\")) return 3;\n"
        "  return sl_model_set_ablation(NULL, SL_ABLATE_NO_KV_CACHE) == SL_ERR_INVALID ? 0 : 4;\n"
        "}\n")
    exe = str(tmp_path / "use_abi")
    libdir = os.path.dirname(_abi.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I" + os.path.join(ROOT, "include"), str(src), "-L" + libdir, "-lsurelock",
           "-Wl,-rpath," + libdir, "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not on PATH")
def test_struct_layouts_match_the_header(tmp_path):
    """Every struct the binding passes through the boundary has the header's
    size and field offsets (a field added to the header but not to the
    binding, or in another order, shifts what the library reads)."""
    from token_locking_b200 import _abi as A
    pairs = [("sl_config", A.Config), ("sl_layer_weights", A.LayerWeights),
             ("sl_weights", A.Weights), ("sl_lock_params", A.LockParams),
             ("sl_sampler_params", A.SamplerParams), ("sl_sampler_state", A.SamplerState),
             ("sl_timing", A.Timing)]
    lines = []
    for cname, py in pairs:
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    src = tmp_path / "layout.c"
    src.write_text('#include "surelock.h"\n#include <stddef.h>\n#include <stdio.h>\n'
                   "int main(void) {\n" + "\n".join(lines) + "\n  return 0;\n}\n")
    exe = str(tmp_path / "layout")
    r = subprocess.run(["gcc", "-std=c99", "-I" + os.path.join(ROOT, "include"), str(src),
                        "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-4000:]
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0
    got = {}
    for line in r.stdout.splitlines():
        *key, val = line.split()
        got[tuple(key)] = int(val)
    for cname, py in pairs:
        assert got[(cname, "size")] == C.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)
