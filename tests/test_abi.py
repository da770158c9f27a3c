"""The C ABI without a GPU: the library loads, exports every symbol that
include/moe.h declares, serves a plain C99 program, and rejects bad arguments
on the host (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

from sparse_moe_layer_gemm_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        from sparse_moe_layer_gemm_b200.build import build
        build()
    return B.load_library()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_and_binding_agree():
    assert header_functions() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in header_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_status_strings(lib):
    for s in range(7):
        assert B.status_string(s) not in ("", "unknown status")
    assert B.status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(hidden=4096, num_experts=288, top_k=8, intermediate=1280)
    base.update(kw)
    return B.make_config(**base)


def test_config_check_accepts_the_layer(lib):
    assert B.moe_config_check(_cfg()) == B.MOE_OK
    assert B.moe_config_check(_cfg(hidden=256, num_experts=16, top_k=4, intermediate=64,
                                   act_dtype=B.MOE_F32, weight_dtype=B.MOE_F32)) == B.MOE_OK
    assert B.moe_config_check(_cfg(swiglu_limit=7.0, swiglu_limit_shared=16.0)) == B.MOE_OK


@pytest.mark.parametrize("kw,want", [
    (dict(hidden=0), B.MOE_ERR_INVALID_ARG),
    (dict(num_experts=-1), B.MOE_ERR_INVALID_ARG),
    (dict(top_k=0), B.MOE_ERR_INVALID_ARG),
    (dict(top_k=300), B.MOE_ERR_INVALID_ARG),          # k > E
    (dict(intermediate=0), B.MOE_ERR_INVALID_ARG),
    (dict(act_dtype=7), B.MOE_ERR_INVALID_ARG),
    (dict(weight_dtype=-1), B.MOE_ERR_INVALID_ARG),
    (dict(swiglu_limit=-1.0), B.MOE_ERR_INVALID_ARG),
    (dict(routed_scaling_factor=float("nan")), B.MOE_ERR_INVALID_ARG),
    (dict(hidden=4000), B.MOE_ERR_UNSUPPORTED),          # not a multiple of 128
    (dict(num_experts=2048), B.MOE_ERR_UNSUPPORTED),
    (dict(top_k=33, num_experts=64), B.MOE_ERR_UNSUPPORTED),
    (dict(shared_intermediate=2560), B.MOE_ERR_UNSUPPORTED),
])
def test_config_check_rejects(lib, kw, want):
    assert B.moe_config_check(_cfg(**kw)) == want


def test_null_arguments_rejected_without_cuda(lib):
    assert lib.moe_config_check(None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_create(None, None) == B.MOE_ERR_INVALID_ARG
    n = ctypes.c_size_t()
    assert lib.moe_workspace_size(None, 64, ctypes.byref(n)) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_workspace_size_host(None, 64, ctypes.byref(n)) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_forward(None, None, 64, None, None, 0, None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host(None, None, 64, None, None, 0, None) == B.MOE_ERR_INVALID_ARG
    assert (lib.moe_forward_host_async(None, None, 64, None, None, 0, None) ==
            B.MOE_ERR_INVALID_ARG)
    assert lib.moe_forward_host_join(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_load_weights(*([None] * 10)) == B.MOE_ERR_INVALID_ARG
    v = ctypes.c_int()
    assert lib.moe_get_device_error(None, ctypes.byref(v)) == B.MOE_ERR_INVALID_ARG
    lib.moe_destroy(None)


def test_oneshot_rejects_bad_config_before_cuda(lib):
    r = lib.moe_forward_oneshot(*([None] * 9), 64, 4000, 288, 8, 1280, 3.0, 0.0, 0.0,
                                B.MOE_BF16, B.MOE_BF16, None, None)
    assert r == B.MOE_ERR_UNSUPPORTED
    r = lib.moe_forward_oneshot(*([None] * 9), 64, 4096, 288, 0, 1280, 3.0, 0.0, 0.0,
                                B.MOE_BF16, B.MOE_BF16, None, None)
    assert r == B.MOE_ERR_INVALID_ARG


def test_wait_self_check_rejects_bad_limits_without_cuda(lib):
    from sparse_moe_layer_gemm_b200 import binding as B
    assert B.moe_check_wait_timeout(0)[0] == B.MOE_ERR_INVALID_ARG
    assert B.moe_check_wait_timeout(20_000_000)[0] == B.MOE_ERR_INVALID_ARG


def test_fp8_weights_host_checks(lib):
    assert B.moe_config_check(_cfg(weight_dtype=B.MOE_FP8_E4M3)) == B.MOE_OK
    assert B.moe_config_check(_cfg(act_dtype=B.MOE_FP8_E4M3)) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_load_weights_fp8(*([None] * 16)) == B.MOE_ERR_INVALID_ARG
    # the one-shot list has no scales
    r = lib.moe_forward_oneshot(*([None] * 9), 64, 4096, 288, 8, 1280, 3.0, 0.0, 0.0,
                                B.MOE_BF16, B.MOE_FP8_E4M3, None, None)
    assert r == B.MOE_ERR_UNSUPPORTED
    # decode: n = 0 is a no-op, n % 4 != 0 and NULL pointers are rejected
    assert lib.moe_decode_e4m3(None, 0, None, None) == B.MOE_OK
    assert lib.moe_decode_e4m3(None, 8, None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_decode_e4m3(ctypes.c_void_p(256), 6, ctypes.c_void_p(512), None) == \
        B.MOE_ERR_INVALID_ARG


def test_dense_host_checks(lib):
    ok = B.make_dense_config(4096, 11264)
    assert B.moe_dense_config_check(ok) == B.MOE_OK
    assert B.moe_dense_config_check(B.make_dense_config(256, 320, act_dtype=B.MOE_F32,
                                                        weight_dtype=B.MOE_F32)) == B.MOE_OK
    for cfg, want in ((B.make_dense_config(0, 64), B.MOE_ERR_INVALID_ARG),
                      (B.make_dense_config(256, 0), B.MOE_ERR_INVALID_ARG),
                      (B.make_dense_config(256, 64, swiglu_limit=-1.0), B.MOE_ERR_INVALID_ARG),
                      (B.make_dense_config(256, 64, act_dtype=B.MOE_FP8_E4M3), B.MOE_ERR_INVALID_ARG),
                      (B.make_dense_config(200, 64), B.MOE_ERR_UNSUPPORTED),
                      (B.make_dense_config(256, 40000), B.MOE_ERR_UNSUPPORTED),
                      (B.make_dense_config(256, 64, weight_dtype=B.MOE_FP8_E4M3),
                       B.MOE_ERR_UNSUPPORTED)):
        assert B.moe_dense_config_check(cfg) == want
    assert lib.moe_dense_config_check(None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_dense_create(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_dense_load_weights(None, None, None, None, None) == B.MOE_ERR_INVALID_ARG
    n = ctypes.c_size_t()
    assert lib.moe_dense_workspace_size(None, 8, ctypes.byref(n)) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_dense_forward(None, None, 8, None, None, 0, None) == B.MOE_ERR_INVALID_ARG
    v = ctypes.c_int()
    assert lib.moe_dense_get_device_error(None, ctypes.byref(v)) == B.MOE_ERR_INVALID_ARG
    lib.moe_dense_destroy(None)


def test_a_plain_c_program_builds_and_calls_the_library(lib, tmp_path):
    """The boundary is C: a C99 program that includes only include/moe.h
    compiles warning-free, links against libmoe.so and calls host-only entry
    points (no CUDA call is made)."""
    src = tmp_path / "use_moe.c"
    src.write_text(
        '#include <string.h>\n'
        '#include "moe.h"\n'
        'int main(void) {\n'
        '  moe_config_t c;\n'
        '  memset(&c, 0, sizeof c);\n'
        '  c.hidden = 4096; c.num_experts = 288; c.top_k = 8;\n'
        '  c.intermediate = 1280; c.shared_intermediate = 1280;\n'
        '  c.norm_expert_weight = 1; c.routed_scaling_factor = 3.0f;\n'
        '  c.use_router_bias = 1; c.act_dtype = MOE_BF16; c.weight_dtype = MOE_BF16;\n'
        '  if (moe_config_check(&c) != MOE_OK) return 1;\n'
        '  c.top_k = 289;\n'
        '  if (moe_config_check(&c) != MOE_ERR_INVALID_ARG) return 2;\n'
        '  if (moe_config_check(0) != MOE_ERR_INVALID_ARG) return 3;\n'
        '  if (strcmp(moe_status_string(MOE_OK), "ok") != 0) return 4;\n'
        '  return 0;\n'
        '}\n')
    exe = tmp_path / "use_moe"
    libdir = os.path.dirname(B.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I" + os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L" + libdir, "-lmoe", "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
