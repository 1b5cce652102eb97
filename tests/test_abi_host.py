"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

The library must load, export every function include/coda.h declares, and
reject bad arguments with the documented status codes before touching CUDA
(the pointers below are fake and are never dereferenced).
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from gemm_epilogue_transformer_02_b200 import binding
from gemm_epilogue_transformer_02_b200.build import build

OK, NULL, SHAPE, ALIGN, WS, DEVICE = 0, 1, 2, 3, 4, 5


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def declared_functions():
    text = open(binding.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(coda_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 20
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (coda_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n), n
    # the binding declares a signature for every exported call
    assert set(names) == set(binding._SIGS), set(names) ^ set(binding._SIGS)


def test_status_strings_and_constants(lib):
    for code in range(9):
        s = lib.coda_status_string(code).decode()
        assert s.startswith(binding.STATUS_NAMES[code])
    assert lib.coda_status_string(99).decode() == "CODA_ERR_UNKNOWN"
    assert lib.coda_version() >= 1
    assert lib.coda_partial_tile_width() == 128
    assert lib.coda_partial_cols(2048) == 16
    assert lib.coda_partial_cols(512) == 4
    assert lib.coda_partial_cols(520) == 5
    assert lib.coda_partial_cols(0) == -1
    assert lib.coda_lmhead_ce_workspace_size(8192, 128256) >= 2 * 501 * 8192 * 4 + 8192 * 4
    assert lib.coda_gemm_rowscale_bwd_workspace_size(8192, 2048) >= 8192 * 2048 * 2
    assert lib.coda_rms_reduce_bwd_workspace_size(8192, 2048) >= 256 * 2048 * 4
    assert lib.coda_set_wait_limit_ns(0) == SHAPE
    assert lib.coda_set_wait_limit_ns(1_000_000_000) == OK


A = ctypes.c_void_p(0x10000)
B = ctypes.c_void_p(0x20000)
C = ctypes.c_void_p(0x30000)
D = ctypes.c_void_p(0x40000)
MIS = ctypes.c_void_p(0x30008)  # 8-byte aligned only


# The pointers below are fake: these tests run only where no kernel can launch,
# so that a validation that ever stopped rejecting them could not reach a GPU.
no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers: CPU-only check")


@no_gpu_only
def test_argument_errors_are_reported_before_any_launch(lib):
    f = lib.coda_gemm_rowscale
    assert f(None, B, None, C, 256, 512, 512, None) == NULL
    assert f(A, B, None, None, 256, 512, 512, None) == NULL
    assert f(A, B, None, C, -1, 512, 512, None) == SHAPE
    assert f(A, B, None, C, 256, 500, 512, None) == SHAPE   # N not a multiple of 8
    assert f(A, B, None, C, 256, 512, 0, None) == SHAPE
    assert f(A, B, None, MIS, 256, 512, 512, None) == ALIGN
    assert f(A, B, MIS, C, 256, 512, 512, None) == ALIGN
    assert f(A, B, None, C, 0, 512, 512, None) == OK           # M == 0 is a no-op

    g = lib.coda_gemm_res_partialrms
    assert g(A, B, None, None, None, None, None, 16, 64, 64, None) == NULL   # no output
    assert g(A, B, None, None, None, C, None, 16, 64, 64, None) == NULL      # hg needs gamma
    assert g(A, B, C, D, C, MIS, None, 16, 64, 64, None) == ALIGN

    assert lib.coda_rms_reduce(A, 16, 0, 64, 1e-6, B, None) == SHAPE
    assert lib.coda_rms_reduce(A, 16, 1, 64, -1.0, B, None) == SHAPE

    h = lib.coda_lmhead_ce
    assert h(A, B, C, None, D, D, None, None, 0, 16, 64, 64, None) == WS
    assert h(A, B, C, None, D, D, None, A, 16, 16, 64, 64, None) == WS
    assert h(A, B, None, None, D, D, None, A, 1 << 20, 16, 64, 64, None) == NULL

    k = lib.coda_gemm_rowscale_bwd
    assert k(A, B, C, D, A, B, C, None, 0, 16, 64, 64, None) == WS
    assert lib.coda_rms_reduce_bwd(A, B, C, D, A, B, C, None, 0, 16, 1, 64, None) == WS
    assert lib.coda_gemm_res_partialrms_bwd(A, B, C, None, None, 16, 64, 64, None) == NULL
    assert lib.coda_gemm_swiglu(A, B, None, C, MIS, 16, 64, 64, None) == ALIGN
    assert lib.coda_unfused_add(A, B, C, 12, None) == SHAPE
    assert lib.coda_unfused_rmsnorm(A, B, 1e-6, None, None, 16, 64, None) == NULL
    assert lib.coda_selftest_bounded_wait(0, A, None) == SHAPE

    q = lib.coda_fp8_quantize
    assert q(A, 16, 12, 0, B, C, D, None) == SHAPE        # cols not a multiple of 8
    assert q(A, 6, 16, 1, B, C, D, None) == SHAPE         # transposed: rows not a multiple of 4
    assert q(A, 16, 16, 0, None, C, D, None) == NULL
    assert q(A, 16, 16, 0, MIS, C, D, None) == ALIGN
    assert lib.coda_fp8_scale_from_amax(None, B, None) == NULL
    p8 = lib.coda_gemm_res_partialrms_fp8
    assert p8(A, B, C, D, None, A, B, None, C, D, A, 16, 64, 24, None) == SHAPE   # K not a multiple of 16
    assert p8(A, B, C, D, None, A, B, None, C, D, A, 16, 72, 64, None) == SHAPE   # N not a multiple of 16
    assert p8(A, B, C, D, None, None, B, None, C, D, A, 16, 64, 64, None) == NULL  # gamma
    assert p8(A, B, C, D, None, A, B, None, MIS, D, A, 16, 64, 64, None) == ALIGN
    assert p8(A, B, C, D, None, A, B, None, C, D, A, 0, 64, 64, None) == OK       # empty batch
    hb = lib.coda_rmsnorm_block_host
    assert hb(A, None, B, C, D, 1e-6, A, B, 1 << 30, 256, 64, 64, 64, 100, None) == SHAPE   # chunk not 256-aligned
    assert hb(None, None, B, C, D, 1e-6, A, B, 1 << 30, 256, 64, 64, 64, 256, None) == NULL
    assert hb(A, None, B, C, D, 1e-6, A, B, 16, 256, 64, 64, 64, 256, None) == WS
    r8 = lib.coda_gemm_rowscale_partial_fp8
    assert r8(A, B, C, D, A, 1, 64, 1e-6, None, B, 16, 64, 40, None) == SHAPE     # K
    assert r8(A, B, C, D, A, 0, 64, 1e-6, None, B, 16, 64, 64, None) == SHAPE     # T
    assert r8(A, B, C, D, A, 1, 64, 1e-6, None, None, 16, 64, 64, None) == NULL   # out


@no_gpu_only
def test_argument_errors_of_the_remaining_calls(lib):
    rp = lib.coda_gemm_rowscale_partial  # (A, W, partial, T, N_norm, eps, r_out, out, M, N, K, stream)
    assert rp(A, B, C, 0, 64, 1e-6, None, D, 16, 64, 64, None) == SHAPE        # T
    assert rp(A, B, C, 1, 0, 1e-6, None, D, 16, 64, 64, None) == SHAPE         # N_norm
    assert rp(A, B, None, 1, 64, 1e-6, None, D, 16, 64, 64, None) == NULL      # partial
    assert rp(A, B, C, 1, 64, 1e-6, MIS, D, 16, 64, 64, None) == ALIGN         # r_out
    assert rp(A, B, C, 1, 64, 1e-6, None, D, 0, 64, 64, None) == OK            # empty batch

    blk = lib.coda_rmsnorm_block  # (x, res, W1, W2, gamma, eps, h, hg, partial, r, out, ws, bytes, M, K, N, N2, s)
    assert blk(A, None, B, C, D, -1.0, A, B, C, D, A, B, 1 << 20, 16, 64, 64, 64, None) == SHAPE
    assert blk(A, None, B, C, D, 1e-6, None, B, C, D, A, B, 1 << 20, 16, 64, 64, 64, None) == NULL
    assert blk(A, MIS, B, C, D, 1e-6, A, B, C, D, A, B, 1 << 20, 16, 64, 64, 64, None) == ALIGN
    assert blk(A, None, B, C, D, 1e-6, A, B, C, D, A, B, 0, 16, 64, 64, 64, None) == WS

    rope = lib.coda_gemm_qkv_rope  # (x, W, positions, out, M, N, K, head_dim, rope_cols, theta, stream)
    assert rope(A, B, C, D, 16, 384, 64, 96, 192, 5e5, None) == SHAPE     # head_dim 64 or 128 only
    assert rope(A, B, C, D, 16, 328, 64, 64, 192, 5e5, None) == SHAPE     # N not whole heads
    assert rope(A, B, C, D, 16, 384, 64, 64, 100, 5e5, None) == SHAPE     # rope_cols not whole heads
    assert rope(A, B, C, D, 16, 384, 64, 64, 448, 5e5, None) == SHAPE     # rope_cols > N
    assert rope(A, B, C, D, 16, 384, 64, 64, 192, 1.0, None) == SHAPE     # theta
    assert rope(A, B, None, D, 16, 384, 64, 64, 192, 5e5, None) == NULL   # positions
    assert rope(A, B, C, MIS, 16, 384, 64, 64, 192, 5e5, None) == ALIGN
    assert rope(A, B, C, D, 0, 384, 64, 64, 192, 5e5, None) == OK

    ls = lib.coda_loss_stats  # (loss, M, stats_out, stream)
    assert ls(A, 0, B, None) == SHAPE
    assert ls(A, 1 << 24, B, None) == SHAPE      # the count must stay exact in fp32
    assert ls(None, 16, B, None) == NULL
    assert ls(A, 16, MIS, None) == ALIGN
    gf = lib.coda_ce_global_finish  # (stats, M, mean_out, d_loss_out, stream)
    assert gf(A, -1, B, C, None) == SHAPE
    assert gf(A, 16, None, None, None) == NULL
    assert gf(None, 16, B, C, None) == NULL
    assert gf(A, 16, B, MIS, None) == ALIGN

    sb = lib.coda_gemm_swiglu_bwd  # (d_out, W_down, gateup, d_gateup, M, F, N, stream)
    assert sb(A, B, C, D, 16, 60, 64, None) == SHAPE                     # F not a multiple of 8
    assert sb(A, B, None, D, 16, 64, 64, None) == NULL
    assert sb(A, B, MIS, D, 16, 64, 64, None) == ALIGN
    assert sb(A, B, C, D, 0, 64, 64, None) == OK

    cb = lib.coda_lmhead_ce_bwd  # (H, W, labels, lse, d_loss, r, dH, dW, ws, bytes, M, V, K, stream)
    assert cb(A, B, C, D, None, None, A, B, C, 1 << 30, 16, 60, 64, None) == SHAPE   # V
    assert cb(A, B, C, None, None, None, A, B, C, 1 << 30, 16, 64, 64, None) == NULL  # lse
    assert cb(A, B, C, D, MIS, None, A, B, C, 1 << 30, 16, 64, 64, None) == ALIGN     # d_loss
    assert cb(A, B, C, D, None, None, A, B, C, 0, 16, 64, 64, None) == WS
    assert lib.coda_lmhead_ce_bwd_workspace_size(8192, 128256) > 0

    na = lib.coda_rms_reduce_bwd_noalloc  # (pdr, r, d_hg, h, gamma, dh, dgamma, M, T, N, stream)
    assert na(A, B, C, D, A, B, C, 16, 0, 64, None) == SHAPE
    assert na(A, B, C, D, None, B, C, 16, 1, 64, None) == NULL
    assert na(A, B, C, D, A, B, C, 32768, 8, 2048, None) == WS   # ceil(M / 32) * N above the static 2^20 floats

    g8 = lib.coda_gemm_fp8  # (A8, sa, Wt8, sw, out, M, N, K, stream)
    assert g8(A, B, C, D, A, 16, 64, 24, None) == SHAPE   # K not a multiple of 16
    assert g8(A, None, C, D, A, 16, 64, 64, None) == NULL  # sa
    assert g8(A, B, C, D, MIS, 16, 64, 64, None) == ALIGN
    u8 = lib.coda_unfused_rmsnorm_fp8  # (h, gamma, eps, s_y, y8, amax, r, M, N, stream)
    assert u8(A, B, 1e-6, C, D, A, None, 16, 24, None) == SHAPE   # N not a multiple of 16
    assert u8(A, B, 1e-6, None, D, A, None, 16, 64, None) == NULL  # s_y
    assert u8(A, B, 1e-6, C, D, A, MIS, 16, 64, None) == ALIGN     # r_out

    # MXFP8: the scale layouts' sizes, and the calls' argument checks
    assert lib.coda_mx_sf_bytes(300, 1024, 0) == 8 * 3 * 512      # A: k-blocks x row blocks x 512-byte atoms
    assert lib.coda_mx_sf_bytes(300, 1152, 0) == 9 * 3 * 512
    assert lib.coda_mx_sf_bytes(300, 256, 1) == 2 * 2 * 4096      # B: k-blocks x 256-row tiles
    assert lib.coda_mx_sf_bytes(1, 128, 1) == 4096
    assert lib.coda_mx_sf_bytes(16, 96, 0) == -1            # cols not a multiple of 128
    assert lib.coda_mx_sf_bytes(-1, 128, 0) == -1
    assert lib.coda_mx_sf_bytes(16, 128, 2) == -1           # no such operand
    mq = lib.coda_mx_quantize  # (src, rows, cols, operand, q, sf, stream)
    assert mq(A, 16, 192, 0, B, C, None) == SHAPE
    assert mq(A, 16, 128, 2, B, C, None) == SHAPE
    assert mq(A, 16, 128, 1, None, C, None) == NULL
    assert mq(A, 16, 128, 0, B, MIS, None) == ALIGN
    assert mq(A, 0, 128, 0, B, C, None) == OK
    pm = lib.coda_gemm_res_partialrms_mx  # (x8, sx, Wt8, sw, res, gamma, h, hq, hsf, partial, M, N, K, s)
    assert pm(A, B, C, D, None, A, None, B, C, D, 16, 192, 64, None) == SHAPE  # N not a multiple of 128
    assert pm(A, B, C, D, None, A, None, B, C, D, 16, 256, 40, None) == SHAPE  # K not a multiple of 16
    assert pm(A, B, C, D, None, A, None, B, None, D, 16, 256, 64, None) == NULL  # scales
    assert pm(A, B, C, D, None, None, None, B, C, D, 16, 256, 64, None) == NULL  # gamma
    assert pm(A, B, C, D, None, A, None, B, MIS, D, 16, 256, 64, None) == ALIGN
    assert pm(A, B, C, D, None, A, None, B, C, D, 0, 256, 64, None) == OK
    rm = lib.coda_gemm_rowscale_partial_mx  # (Aq, Asf, Wq, Wsf, partial, T, N_norm, eps, r, out, M, N, K, s)
    assert rm(A, B, C, D, None, 0, 0, 0.0, None, A, 16, 256, 192, None) == SHAPE   # K
    assert rm(A, B, C, D, None, 0, 0, 0.0, None, A, 16, 200, 256, None) == SHAPE   # N
    assert rm(A, B, C, D, A, 0, 64, 1e-6, None, A, 16, 256, 256, None) == SHAPE    # T with partials
    assert rm(A, B, C, None, None, 0, 0, 0.0, None, A, 16, 256, 256, None) == NULL
    assert rm(A, B, C, D, None, 0, 0, 0.0, None, MIS, 16, 256, 256, None) == ALIGN
    assert rm(A, B, C, D, None, 0, 0, 0.0, None, A, 0, 256, 256, None) == OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_arguments_without_a_gpu_report_device_error(lib):
    assert lib.coda_gemm_rowscale(A, B, None, C, 256, 512, 512, None) == DEVICE
    assert lib.coda_rms_reduce(A, 16, 1, 64, 1e-6, B, None) == DEVICE
    assert lib.coda_fp8_quantize(A, 16, 16, 1, B, C, D, None) == DEVICE
    assert lib.coda_gemm_rowscale_partial_fp8(A, B, C, D, A, 1, 64, 1e-6, None, B, 16, 64, 64, None) == DEVICE
    assert lib.coda_mx_quantize(A, 16, 128, 1, B, C, None) == DEVICE
    assert lib.coda_gemm_rowscale_partial_mx(A, B, C, D, None, 0, 0, 0.0, None, A, 16, 256, 256, None) == DEVICE


def test_binding_refuses_cpu_tensors(lib):
    x = torch.zeros(8, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.gemm_rowscale(x, x)


def test_build_flags_target_sm100a():
    src = open(os.path.join(os.path.dirname(binding.LIB_PATH), "build.py")).read()
    assert "arch=compute_100a,code=sm_100a" in src


def test_product_never_touches_the_oracle():
    """The library package neither imports nor reads anything under oracle/:
    the oracle is test infrastructure, and there is no CPU fallback."""
    pkg = os.path.dirname(binding.LIB_PATH)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                # (the seeded input generator, shared with the tests, may name it in prose)
                assert not re.search(r"(from|import)\s+oracle\b|[\'\"]oracle[/\'\"]|coda_oracle", text), \
                    os.path.join(dirpath, f)


def test_binding_fails_loudly_without_the_library(tmp_path):
    """A missing libcoda.so is an error, never a silent fallback."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("binding_missing", binding.__file__)
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    m.LIB_PATH = str(tmp_path / "libcoda.so")
    with pytest.raises(RuntimeError, match="not found"):
        m.load_library()


@no_gpu_only
def test_abi_from_plain_c(tmp_path):
    """The header compiles as C99 and the library links and answers from C."""
    src = os.path.join(os.path.dirname(__file__), "c", "abi_from_c.c")
    inc = os.path.dirname(binding.HEADER_PATH)
    libdir = os.path.dirname(binding.LIB_PATH)
    exe = str(tmp_path / "abi_from_c")
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", inc, src, "-o", exe,
                         "-L", libdir, "-l:libcoda.so", "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "abi_from_c ok" in run.stdout
