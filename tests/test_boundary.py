"""C-ABI boundary checks that need no GPU: the library loads, exports every
function the header declares, sizes its workspace, and rejects bad arguments
before it touches the device."""
import ctypes
import os
import re

import pytest

import chunked_kl_loss_tcgen05_b200 as fk
from chunked_kl_loss_tcgen05_b200 import FcklProblem
from chunked_kl_loss_tcgen05_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fckl.h")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    return fk.load()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fckl_[a-z_]+)\s*\(", src)))


def test_header_declares_the_expected_api():
    assert _declared_functions() == sorted(fk.exported_symbols)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fk.lib_path())
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    for code in range(8):
        s = fk.fckl_status_string(code)
        assert s.startswith("FCKL_")
    assert fk.fckl_status_string(0) == "FCKL_OK"
    assert fk.fckl_status_string(99) == "FCKL_ERR_UNKNOWN"


def test_workspace_and_chunk_rules():
    p1 = FcklProblem(8192, 3072, 128256, 100, 1.0, 0)
    assert fk.fckl_resolved_chunk(p1) == 4096          # 1 GiB of bf16 dlogits
    p3 = FcklProblem(131072, 2880, 201088, 100, 1.0, 0)
    assert fk.fckl_resolved_chunk(p3) == 2560
    p0 = FcklProblem(256, 256, 4096, 16, 1.0, 64)
    assert fk.fckl_resolved_chunk(p0) == 64
    assert fk.fckl_resolved_chunk(FcklProblem(100, 256, 4096, 16, 1.0, 0)) == 100
    assert fk.fckl_resolved_chunk(FcklProblem(100, 256, 4096, 16, 1.0, 4096)) == 100
    # workspace holds the chunk's bf16 dlogits block and is linear in N beyond it
    w = fk.fckl_workspace_bytes(p1)
    assert w >= 4096 * 128256 * 2
    a = fk.fckl_workspace_bytes(FcklProblem(32768, 4096, 128256, 100, 1.0, 1024))
    b = fk.fckl_workspace_bytes(FcklProblem(65536, 4096, 128256, 100, 1.0, 1024))
    assert b - a == 32768 * 8    # only the per-row loss and the compacted row list grow
    # an explicit chunk bounds the dlogits block: one chunk of bf16 dlogits
    assert 1024 * 128256 * 2 <= a < 1024 * 128256 * 2 + 48 * 2**20
    # the automatic chunk also picks the grouping (>= 4096 rows per dW GEMM):
    # two 2560-row chunks at the gpt-oss vocabulary; the same explicit chunk
    # keeps one chunk of dlogits
    Vp3 = (201088 + 63) // 64 * 64
    auto3 = fk.fckl_workspace_bytes(p3)
    expl3 = fk.fckl_workspace_bytes(FcklProblem(131072, 2880, 201088, 100, 1.0, 2560))
    assert auto3 - expl3 >= 2560 * Vp3 * 2 and expl3 < 2 * 2560 * Vp3 * 2
    assert fk.fckl_workspace_bytes(FcklProblem(131072, 2880, 201088, 100, 1.0, 0,
                                               dw_rows=1)) == expl3
    # dw_rows = 4096 groups four 1024-row chunks into one dW GEMM
    g = fk.fckl_workspace_bytes(FcklProblem(32768, 4096, 128256, 100, 1.0, 1024, dw_rows=4096))
    assert g - a >= 3 * 1024 * 128256 * 2 + 3 * 1024 * 4096 * 2


def test_bench_restates_the_chunk_rule():
    """bench.py's oracle arm labels its workload with the library's chunk
    without loading the library; its restatement must agree with it."""
    import dataclasses

    import bench
    import synth
    cases = list(synth.CONFIGS.values())
    for N, V, chunk in [(100, 4096, 0), (5000, 1000, 0), (70000, 301, 0), (300, 700, 100),
                        (64, 512, 4096), (1, 64, 0), (1000000, 262144, 0)]:
        cases.append(dataclasses.replace(synth.CONFIGS[0], N=N, V=V, chunk=chunk))
    for cfg in cases:
        want = fk.fckl_resolved_chunk(FcklProblem(cfg.N, cfg.H, cfg.V, cfg.K, cfg.T, cfg.chunk))
        assert bench.library_chunk(cfg) == want, cfg


def test_workspace_follows_an_explicit_chunk():
    """Live workspace is O(chunk * V): at the gpt-oss shape (V = 201,088) a
    256-row chunk needs its 256 x V bf16 dlogits block plus small per-chunk
    buffers and 8 bytes per row (row loss, compacted row list)."""
    N, H, V, K = 131072, 2880, 201088, 100
    Vp = (V + 63) // 64 * 64
    small = fk.fckl_workspace_bytes(FcklProblem(N, H, V, K, 1.0, 256))
    # per-chunk buffers: 14 bytes per row and vocab tile of 256 (partials,
    # tile starts), 12 per hidden unit (two staged hidden rows, one fp32 dH
    # row), about 36 per teacher entry
    NT = (V + 255) // 256
    per_chunk = 256 * (14 * NT + 12 * H + 36 * K + 64)
    assert 256 * Vp * 2 + N * 8 <= small < 256 * Vp * 2 + N * 8 + per_chunk + 2**20
    big = fk.fckl_workspace_bytes(FcklProblem(N, H, V, K, 1.0, 2048))
    assert big - small >= (2048 - 256) * Vp * 2
    # linear in the chunk beyond the per-row arrays
    mid = fk.fckl_workspace_bytes(FcklProblem(N, H, V, K, 1.0, 1024))
    assert abs((big - mid) - (mid - small) * 1024 / 768) < 2**20
    assert fk.fckl_workspace_bytes(FcklProblem(N, H, V, K, 1.0, 256, dw_rows=-1)) == 0


@pytest.mark.parametrize("bad", [
    dict(N=0), dict(H=0), dict(V=0), dict(K=0), dict(T=0.0), dict(T=-1.0),
    dict(T=float("nan")), dict(T=float("inf")), dict(chunk=-1), dict(teacher=2), dict(teacher=-1),
    dict(dw_rows=-1)])
def test_invalid_problem_rejected(bad):
    kw = dict(N=64, H=64, V=512, K=8, T=1.0, chunk=0)
    kw.update(bad)
    p = FcklProblem(**kw)
    assert fk.fckl_workspace_bytes(p) == 0
    assert fk.fckl_resolved_chunk(p) == -1
    fake = 1 << 20
    st = fk.fckl_fwd_bwd(p, fake, fake, fake, fake, None, fake, None, fake, fake, fake, 1 << 40, None)
    assert st == fk.FCKL_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(K=257), dict(H=60), dict(K=600, V=512)])
def test_unsupported_problem_rejected(bad):
    kw = dict(N=64, H=64, V=512, K=8, T=1.0, chunk=0)
    kw.update(bad)
    p = FcklProblem(**kw)
    fake = 1 << 20
    st = fk.fckl_fwd_bwd(p, fake, fake, fake, fake, None, fake, None, fake, fake, fake, 1 << 40, None)
    assert st == fk.FCKL_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected():
    p = FcklProblem(64, 64, 512, 8, 1.0, 0)
    ws = fk.fckl_workspace_bytes(p)
    f = 1 << 20
    args = [f, f, f, f, None, f, None, f, f, f, ws]
    for i in (0, 1, 2, 3, 5, 7, 8):
        a = list(args)
        a[i] = None
        assert fk.fckl_fwd_bwd(p, *a, None) == fk.FCKL_ERR_INVALID_ARG, i
    a = list(args)
    a[0] = f + 8  # hidden must be 16-byte aligned for TMA
    assert fk.fckl_fwd_bwd(p, *a, None) == fk.FCKL_ERR_INVALID_ARG
    # forward-only does not need gradient buffers
    st = fk.fckl_fwd(p, f, f, f, f, None, f, None, None, ws, None)
    assert st == fk.FCKL_ERR_WORKSPACE


def test_small_workspace_rejected():
    p = FcklProblem(64, 64, 512, 8, 1.0, 0)
    ws = fk.fckl_workspace_bytes(p)
    f = 1 << 20
    assert fk.fckl_fwd_bwd(p, f, f, f, f, None, f, None, f, f, f, ws - 1, None) == fk.FCKL_ERR_WORKSPACE
    assert fk.fckl_fwd(p, f, f, f, f, None, f, None, f + 16, ws, None) == fk.FCKL_ERR_WORKSPACE


def test_no_gpu_fails_loudly():
    """With every argument valid and no usable sm_100 device the call refuses;
    there is no host fallback."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    p = FcklProblem(64, 64, 512, 8, 1.0, 0)
    ws = fk.fckl_workspace_bytes(p)
    f = 1 << 20
    st = fk.fckl_fwd_bwd(p, f, f, f, f, None, f, None, f, f, f, ws, None)
    assert st in (fk.FCKL_ERR_UNSUPPORTED, fk.FCKL_ERR_CUDA)


def test_noalloc_rejects_oversized_problem():
    """The allocation-free forward refuses, before touching the device, a chunk
    whose scratch would not fit in the library's static array."""
    prob = FcklProblem(8192, 4096, 1_000_000, 100, 1.0, 4096)  # ~165 MB of forward scratch
    f = 1 << 20
    assert fk.fckl_fwd_noalloc(prob, f, f, f, f, None, f, None, None, None) == fk.FCKL_ERR_WORKSPACE
    bad = FcklProblem(64, 60, 512, 8, 1.0, 0)  # H % 8 != 0
    assert fk.fckl_fwd_noalloc(bad, f, f, f, f, None, f, None, None, None) == fk.FCKL_ERR_UNSUPPORTED


def test_host_input_entry_point_checks():
    """The host-input call sizes its workspace as the device-input layout plus
    device copies of the inputs, and rejects missing host buffers and a short
    workspace before it touches the device."""
    p = FcklProblem(300, 64, 700, 9, 1.0, 100)
    base = fk.fckl_workspace_bytes(p)
    host = fk.fckl_host_workspace_bytes(p)
    assert host >= base + 300 * 64 * 2 + 2 * 300 * 9 * 4 + 300 + 4
    assert host < base + 300 * 64 * 2 + 2 * 300 * 9 * 4 + 300 + 4 + 5 * 256
    assert fk.fckl_host_workspace_bytes(FcklProblem(300, 64, 700, 0, 1.0, 0)) == 0
    f = 1 << 20
    args = [f, f, f, f, None, f, f, f, f, host]
    for i in (0, 2, 3, 5):
        a = list(args)
        a[i] = None
        assert fk.fckl_fwd_bwd_host(p, *a, None) == fk.FCKL_ERR_INVALID_ARG, i
    a = list(args)
    a[9] = host - 1
    assert fk.fckl_fwd_bwd_host(p, *a, None) == fk.FCKL_ERR_WORKSPACE
    bad = FcklProblem(300, 60, 700, 9, 1.0, 100)
    assert fk.fckl_fwd_bwd_host(bad, *args, None) == fk.FCKL_ERR_UNSUPPORTED
