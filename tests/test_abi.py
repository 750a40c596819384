"""The C-ABI library loads and exports every entry point include/gptq.h
declares; host-side argument validation answers before anything is launched
(no GPU needed for any call made here)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptq.h")


@pytest.fixture(scope="module")
def pkg():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "gptq_b200_build", os.path.join(ROOT, "post_weight_quantization_gptq_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import post_weight_quantization_gptq_b200 as p
    return p


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z_]+)\s*\(", text)))


def test_header_declares_the_four_stages():
    names = _declared()
    for n in ("gptq_hessian_accumulate", "gptq_prepare_hinv", "gptq_quantize_layer", "gptq_pack",
              "gptq_workspace_size", "gptq_sync_status", "gptq_status_string", "gptq_version"):
        assert n in names


def test_library_exports_every_declared_symbol(pkg):
    lib = ctypes.CDLL(pkg.library_path())
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", pkg.library_path()],
                         capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (gptq_[a-z_]+)\b", out))
    assert set(_declared()) <= exported


def test_library_is_built_for_sm_100a(pkg):
    out = subprocess.run(["cuobjdump", "--list-elf", pkg.library_path()],
                         capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    assert "sm_100a" in out.stdout


def test_status_strings_and_version(pkg):
    assert pkg.gptq_version() >= 100
    assert pkg.gptq_status_string(0) == "ok"
    assert "positive definite" in pkg.gptq_status_string(3)
    assert pkg.gptq_status_string(99) == "unknown status"


def test_workspace_size_and_config_validation(pkg):
    cfg = pkg.GPTQConfig(bits=4, group_size=128)
    b = pkg.gptq_workspace_size(cfg, 4096, 4096)
    assert b >= 4096 * 128 * 4 and b % 256 == 0
    # the full layout of the column walk: eight deferred blocks of errors,
    # their lo parts, and U's lo parts (d_col^2 floats) for the pre-split update
    assert b == 2 * 4096 * 128 * 8 * 4 + 4096 * 4096 * 4
    errs = (300 * 128 * 8 * 4 + 255) // 256 * 256
    assert pkg.gptq_workspace_size(cfg, 300, 1536) == 2 * errs + 1536 * 1536 * 4
    # fewer blocks than eight: as many as the layer has
    assert pkg.gptq_workspace_size(cfg, 64, 256) == 2 * 64 * 128 * 2 * 4 + 256 * 256 * 4
    for bad in (dict(bits=5), dict(group_size=0), dict(group_size=-2), dict(damp=-1.0)):
        kw = dict(bits=4, group_size=128, damp=0.01)
        kw.update(bad)
        with pytest.raises(pkg.GPTQError) as e:
            pkg.gptq_workspace_size(pkg.GPTQConfig(**kw), 64, 256)
        assert e.value.status == 1
    for unsup in (dict(group_size=48), dict(group_size=192), dict(block_size=64),
                  dict(group_size=4), dict(group_size=1)):
        kw = dict(bits=4, group_size=128)
        kw.update(unsup)
        with pytest.raises(pkg.GPTQError) as e:
            pkg.gptq_workspace_size(pkg.GPTQConfig(**kw), 64, 1024)
        assert e.value.status == 2
    # group sizes the column walk supports
    for g in (8, 16, 32, 64, 128, 256, 1024, -1, 5000):
        pkg.gptq_workspace_size(pkg.GPTQConfig(bits=4, group_size=g), 8, 4096)
    # a group as wide as the row is one group per row, whatever its size
    pkg.gptq_workspace_size(pkg.GPTQConfig(bits=4, group_size=4), 8, 4)


def test_invalid_arguments_are_rejected_on_the_host(pkg):
    lib = ctypes.CDLL(pkg.library_path())
    lib.gptq_hessian_accumulate.restype = ctypes.c_int
    lib.gptq_pack.restype = ctypes.c_int
    P, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.gptq_hessian_accumulate.argtypes = [P, i64, i64, i64, P, i64, P, P, ctypes.c_size_t, P]
    lib.gptq_pack.argtypes = [P, i64, i64, ctypes.c_int32, P, P]
    fake = ctypes.c_void_p(1 << 20)
    # d = 0, H NULL, ldx not a multiple of 8, misaligned X: all rejected before any launch
    assert lib.gptq_hessian_accumulate(fake, 16, 0, 16, fake, 16, None, None, 0, None) == 1
    assert lib.gptq_hessian_accumulate(fake, 16, 16, 16, None, 16, None, None, 0, None) == 1
    assert lib.gptq_hessian_accumulate(fake, 16, 12, 12, fake, 12, None, None, 0, None) == 1
    assert lib.gptq_hessian_accumulate(ctypes.c_void_p((1 << 20) + 2), 16, 16, 16, fake, 16,
                                       None, None, 0, None) == 1
    # n == 0 is a no-op that succeeds
    assert lib.gptq_hessian_accumulate(fake, 0, 16, 16, fake, 16, None, None, 0, None) == 0
    assert lib.gptq_pack(fake, 4, 8, 5, fake, None) == 1
    assert lib.gptq_pack(None, 4, 8, 4, fake, None) == 1


def test_host_streaming_hessian_validation(pkg):
    lib = ctypes.CDLL(pkg.library_path())
    P, i64 = ctypes.c_void_p, ctypes.c_int64
    f = lib.gptq_hessian_accumulate_host
    f.restype = ctypes.c_int
    f.argtypes = [P, i64, i64, i64, P, i64, P, P, ctypes.c_size_t, P]
    lib.gptq_hessian_staging_size.restype = ctypes.c_size_t
    lib.gptq_hessian_staging_size.argtypes = [i64, i64]
    fake = ctypes.c_void_p(1 << 20)
    # two slots of 64-token rows, rows padded to a multiple of 8 channels
    assert lib.gptq_hessian_staging_size(4096, 16384) == 2 * 16384 * 4096 * 2
    assert lib.gptq_hessian_staging_size(12, 1) == 2 * 64 * 16 * 2
    assert lib.gptq_hessian_staging_size(0, 64) == 0
    need = lib.gptq_hessian_staging_size(16, 64)
    # bad sizes / pointers -> invalid argument; missing, misaligned or small staging -> workspace
    assert f(fake, 16, 0, 16, fake, 16, None, fake, need, None) == 1
    assert f(None, 16, 16, 16, fake, 16, None, fake, need, None) == 1
    assert f(fake, 16, 16, 8, fake, 16, None, fake, need, None) == 1
    assert f(fake, 16, 16, 16, None, 16, None, fake, need, None) == 1
    assert f(fake, 16, 16, 16, fake, 16, None, None, need, None) == 6
    assert f(fake, 16, 16, 16, fake, 16, None, ctypes.c_void_p((1 << 20) + 16), need, None) == 6
    assert f(fake, 16, 16, 16, fake, 16, None, fake, need - 1, None) == 6
    assert f(fake, 0, 16, 16, fake, 16, None, fake, need, None) == 0


def test_dequant_matmul_validation(pkg):
    lib = ctypes.CDLL(pkg.library_path())
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    f = lib.gptq_dequant_matmul
    f.restype = ctypes.c_int
    f.argtypes = [P, i64, i64, i64, P, P, P, P, i64, i32, i32, P, i64, P, ctypes.c_size_t, P]
    lib.gptq_dequant_matmul_workspace_size.restype = ctypes.c_size_t
    lib.gptq_dequant_matmul_workspace_size.argtypes = [i64, i64]
    assert lib.gptq_dequant_matmul_workspace_size(1, 256) == 1024
    assert lib.gptq_dequant_matmul_workspace_size(20, 256) == 8 * 256 * 4  # 8 tokens per launch
    assert lib.gptq_dequant_matmul_workspace_size(0, 256) == 0
    a = ctypes.c_void_p(1 << 20)
    ok = dict(X=a, n=1, k=256, ldx=256, pk=a, sc=a, ze=a, perm=None, n_out=64, bits=4, g=128,
              Y=a, ldy=64, ws=a, wsb=1024)

    def call(**kw):
        v = dict(ok)
        v.update(kw)
        return f(v["X"], v["n"], v["k"], v["ldx"], v["pk"], v["sc"], v["ze"], v["perm"],
                 v["n_out"], v["bits"], v["g"], v["Y"], v["ldy"], v["ws"], v["wsb"], None)

    assert call(n=0) == 0                                   # no tokens: nothing to do
    assert call(X=None) == 1 and call(Y=None) == 1 and call(pk=None) == 1
    assert call(k=0) == 1 and call(n_out=0) == 1 and call(ldx=100) == 1 and call(ldy=10) == 1
    assert call(bits=5) == 1 and call(g=0) == 1 and call(g=-3) == 1
    assert call(pk=ctypes.c_void_p((1 << 20) + 2)) == 1     # misaligned words
    assert call(bits=3) == 2                                # 3-bit codes straddle words
    assert call(k=252) == 2                                 # not whole 4-bit words
    assert call(g=12) == 2                                  # a word would span two groups
    assert call(ws=None) == 6 and call(wsb=1023) == 6       # workspace missing / too small
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == 6    # workspace misaligned


def test_wait_probe_arguments_are_checked_on_the_host(pkg):
    """The timeout test hook takes kernel kinds 1 and 2 and limits in
    1 .. 10^9 ns; anything else is refused before any state changes."""
    for kernel, ns in ((0, 1000), (3, 1000), (1, 0), (2, -5), (1, 2_000_000_000)):
        with pytest.raises(pkg.GPTQError) as e:
            pkg.gptq_debug_arm_wait_probe(kernel, ns)
        assert e.value.status == 1


def _entry(lib, name, argtypes, restype=ctypes.c_int):
    f = getattr(lib, name)
    f.restype = restype
    f.argtypes = argtypes
    return f


def _caller(f, order, ok):
    def call(**kw):
        v = dict(ok)
        v.update(kw)
        return f(*(v[k] for k in order))
    return call


def test_prepare_hinv_validation(pkg):
    """Sizes, pointers, alignment, the column walk's width limit, the config
    and the workspace are checked before anything is launched."""
    lib = ctypes.CDLL(pkg.library_path())
    P, i64 = ctypes.c_void_p, ctypes.c_int64
    f = _entry(lib, "gptq_prepare_hinv",
               [P, i64, i64, ctypes.POINTER(pkg.GPTQConfig), P, P, P, P, P, ctypes.c_size_t, P])
    cfg = pkg.GPTQConfig(bits=4, group_size=128)
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 24)
    order = ("H", "d", "ldh", "cfg", "U", "perm", "dead", "st", "ws", "wsb", "stream")
    ok = dict(H=a, d=256, ldh=256, cfg=ctypes.byref(cfg), U=b, perm=a, dead=a, st=None, ws=a,
              wsb=pkg.gptq_workspace_size(cfg, 1, 256), stream=None)
    call = _caller(f, order, ok)
    assert call(d=0) == 1 and call(d=-4) == 1 and call(ldh=252) == 1
    assert call(H=None) == 1 and call(U=None) == 1 and call(perm=None) == 1
    assert call(dead=None) == 1
    assert call(U=a) == 1                                       # H is consumed: U apart from it
    assert call(d=254) == 2 and call(ldh=258) == 2              # rows of whole 16-byte units
    assert call(H=ctypes.c_void_p((1 << 20) + 4)) == 2          # tiles need 16-byte aligned bases
    assert call(U=ctypes.c_void_p((1 << 24) + 8)) == 2
    assert call(d=57348, ldh=57348) == 2                        # wider than the column walk takes
    assert call(cfg=None) == 1
    assert call(cfg=ctypes.byref(pkg.GPTQConfig(bits=5))) == 1
    assert call(cfg=ctypes.byref(pkg.GPTQConfig(damp=float("nan")))) == 1
    assert call(cfg=ctypes.byref(pkg.GPTQConfig(group_size=48))) == 2
    assert call(ws=None) == 6 and call(wsb=16) == 6
    assert call(ws=ctypes.c_void_p((1 << 20) + 128)) == 6       # workspace 256-byte aligned


def test_quantize_layer_validation(pkg):
    lib = ctypes.CDLL(pkg.library_path())
    P, i64 = ctypes.c_void_p, ctypes.c_int64
    f = _entry(lib, "gptq_quantize_layer",
               [P, i64, i64, i64, P, P, P, ctypes.POINTER(pkg.GPTQConfig), P, P, P, P, P,
                ctypes.c_size_t, P])
    cfg = pkg.GPTQConfig(bits=4, group_size=128)
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 24)
    order = ("W", "r", "d", "ldw", "U", "perm", "dead", "cfg", "codes", "scales", "zeros", "st",
             "ws", "wsb", "stream")
    ok = dict(W=a, r=64, d=256, ldw=256, U=b, perm=a, dead=a, cfg=ctypes.byref(cfg), codes=a,
              scales=a, zeros=a, st=None, ws=a, wsb=pkg.gptq_workspace_size(cfg, 64, 256),
              stream=None)
    call = _caller(f, order, ok)
    assert call(r=0) == 1 and call(d=0) == 1 and call(ldw=255) == 1
    for name in ("W", "U", "perm", "dead", "codes", "scales", "zeros"):
        assert call(**{name: None}) == 1, name
    assert call(d=57348, ldw=57348) == 2                        # a row of W must fit on chip
    assert call(d=250, ldw=256) == 2                            # d_col a multiple of 4
    assert call(U=ctypes.c_void_p((1 << 24) + 4)) == 2          # U's blocks move by TMA
    assert call(cfg=None) == 1
    assert call(cfg=ctypes.byref(pkg.GPTQConfig(bits=1))) == 1
    assert call(cfg=ctypes.byref(pkg.GPTQConfig(block_size=64))) == 2
    # the workspace must hold at least one block of errors: d_row * 128 floats
    assert call(ws=None) == 6 and call(wsb=64 * 512 - 1) == 6
    assert call(ws=ctypes.c_void_p((1 << 20) + 64)) == 6


def test_quantize_layer_noalloc_validation(pkg):
    """The checks that precede any CUDA call: config, sizes, and a layer whose
    errors would not fit the fixed 16 MiB scratch."""
    lib = ctypes.CDLL(pkg.library_path())
    P, i64 = ctypes.c_void_p, ctypes.c_int64
    f = _entry(lib, "gptq_quantize_layer_noalloc",
               [P, i64, i64, i64, P, P, P, ctypes.POINTER(pkg.GPTQConfig), P, P, P, P, P])
    assert _entry(lib, "gptq_noalloc_scratch_bytes", [], ctypes.c_size_t)() == 16 << 20
    cfg = pkg.GPTQConfig(bits=4, group_size=128)
    a = ctypes.c_void_p(1 << 20)
    order = ("W", "r", "d", "ldw", "U", "perm", "dead", "cfg", "codes", "scales", "zeros", "st",
             "stream")
    ok = dict(W=a, r=64, d=256, ldw=256, U=a, perm=a, dead=a, cfg=ctypes.byref(cfg), codes=a,
              scales=a, zeros=a, st=None, stream=None)
    call = _caller(f, order, ok)
    assert call(cfg=None) == 1 and call(r=0) == 1 and call(d=0) == 1
    assert call(cfg=ctypes.byref(pkg.GPTQConfig(bits=7))) == 1
    assert call(cfg=ctypes.byref(pkg.GPTQConfig(group_size=96))) == 2
    assert call(r=32769, d=128, ldw=128) == 6                   # 32769 * 512 bytes > 16 MiB


def test_dequant_gemm_validation(pkg):
    lib = ctypes.CDLL(pkg.library_path())
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    f = _entry(lib, "gptq_dequant_gemm",
               [P, i64, i64, i64, P, P, P, P, i64, i32, i32, P, i64, P, P, ctypes.c_size_t, P])
    ws_size = _entry(lib, "gptq_dequant_gemm_workspace_size", [i64, i64], ctypes.c_size_t)
    assert ws_size(3, 256) == (3 * 256 * 2 + 255) // 256 * 256  # the tokens as bf16
    assert ws_size(0, 256) == 0 and ws_size(4, 0) == 0
    a = ctypes.c_void_p(1 << 20)
    order = ("X", "n", "k", "ldx", "pk", "sc", "ze", "perm", "n_out", "bits", "g", "Y", "ldy", "st",
             "ws", "wsb", "stream")
    ok = dict(X=a, n=16, k=256, ldx=256, pk=a, sc=a, ze=a, perm=a, n_out=256, bits=4, g=128, Y=a,
              ldy=256, st=None, ws=a, wsb=ws_size(16, 256), stream=None)
    call = _caller(f, order, ok)
    assert call(n=0) == 0                                       # no tokens: nothing to do
    for name in ("X", "pk", "sc", "ze", "Y"):
        assert call(**{name: None}) == 1, name
    assert call(n=-1) == 1 and call(n=(1 << 24) + 1) == 1
    assert call(k=0) == 1 and call(n_out=0) == 1 and call(ldx=128) == 1 and call(ldy=100) == 1
    assert call(bits=6) == 1 and call(g=0) == 1 and call(g=-2) == 1
    assert call(pk=ctypes.c_void_p((1 << 20) + 4)) == 1         # packed rows by 16-byte TMA boxes
    assert call(bits=3) == 2                                    # 3-bit codes straddle words
    assert call(k=224, ldx=256) == 2                            # whole 64-code stages
    assert call(g=12) == 2                                      # an 8-code chunk across groups
    # the act-order gather needs the workspace
    assert call(ws=None) == 6 and call(wsb=16 * 256 * 2 - 1) == 6
    assert call(ws=ctypes.c_void_p((1 << 20) + 32)) == 6


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "gptq.h"

int main(void) {
    gptq_config cfg;
    size_t bytes = 0;
    memset(&cfg, 0, sizeof cfg);
    cfg.bits = 4; cfg.group_size = 128; cfg.block_size = 128; cfg.damp = 0.01f;
    if (gptq_workspace_size(&cfg, 4096, 4096, &bytes) != GPTQ_OK) return 1;
    cfg.bits = 5;
    if (gptq_workspace_size(&cfg, 4096, 4096, &bytes) != GPTQ_ERR_INVALID_ARG) return 2;
    /* host-side rejection before any launch: a NULL H */
    if (gptq_hessian_accumulate((const uint16_t *)0x100000, 16, 16, 16, NULL, 16, NULL, NULL, 0,
                                (cudaStream_t)0) != GPTQ_ERR_INVALID_ARG) return 3;
    printf("%d %zu %s\n", gptq_version(), bytes, gptq_status_string(GPTQ_ERR_NOT_PD));
    return 0;
}
"""


def test_a_plain_c_program_compiles_links_and_calls_the_library(pkg, tmp_path):
    """The header is C (not only C++): a C99 program includes it, links
    against the shared library and calls the entry points that need no GPU."""
    import shutil
    if shutil.which("gcc") is None:
        pytest.skip("gcc unavailable")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(pkg.library_path())
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", cuda_inc, str(src), "-L", libdir, "-lgptq_b200",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    ver, nbytes, text = out.stdout.split(" ", 2)
    assert int(ver) == pkg.gptq_version()
    assert int(nbytes) == pkg.gptq_workspace_size(pkg.GPTQConfig(bits=4, group_size=128), 4096, 4096)
    assert "positive definite" in text
