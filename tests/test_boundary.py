"""Host-only checks of the C-ABI boundary (no GPU needed).

The library must load without a GPU, export every function that
include/moe_b200.h declares, answer workspace queries, and reject bad
arguments on the host with the documented status before touching the device.
"""
import ctypes
import os
import re

import pytest

import mixture_experts_routed_sigmoid_b200 as moe
from mixture_experts_routed_sigmoid_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")

OK, INVALID, UNSUPPORTED, WS_SMALL = 0, 1, 2, 3
FAKE = 0x10000  # non-null, 256-byte aligned host value; never dereferenced on rejection


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[^;(]*?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for required in ("moe_route_topk", "moe_expert_map", "moe_matmul_id", "moe_ffn_forward",
                     "moe_last_error", "moe_check_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(moe.SIGNATURES), "binding and header disagree"
    for name in names:
        assert hasattr(lib, name), name


def test_version(lib):
    assert b"sm_100a" in lib.moe_version()


def test_workspace_queries(lib):
    R = 4096 * 8
    ws_map = lib.moe_expert_map_workspace(4096, 8, 256)
    ws_mm = lib.moe_matmul_id_workspace(4096, 1536, 4096, 8, 256, 0)
    ws_ffn = lib.moe_ffn_workspace(4096, 4096, 1536, 8, 256, 0)
    assert 0 < ws_map < ws_mm < ws_ffn
    # ffn workspace holds the activation (R * inter f32 at most), y_slots
    # (R * hidden f32) and fp16 W_down copies for min(E, R / 512) experts
    fixed = 2 * R * 1536 * 2 + R * 4096 * 4 + min(256, R // 512) * 4096 * 1536 * 2
    assert fixed <= ws_ffn < fixed + 64 * 1024 * 1024
    # no copies below 512 routed rows, nor on the streaming path
    small = lib.moe_ffn_workspace(63, 4096, 1536, 8, 256, 0)
    assert small < 2 * 504 * 1536 * 2 + 504 * 4096 * 4 + 64 * 1024 * 1024
    assert lib.moe_ffn_workspace(4096, 4096, 1536, 0, 256, 0) == 0  # top_k rejected
    assert lib.moe_expert_map_workspace(4, 2, 2000) == 0           # too many experts


def test_router_workspace_follows_the_k_split(lib):
    """The router projection splits K into ranges when few 256-column output
    tiles would leave SMs idle (enough tiles for 148 SMs, >= 4 k-blocks per
    range, <= 8 ranges); the workspace holds a status word and, when split,
    the ranges' partial slabs [ranges, m, E] f32."""
    def expect(m, hidden, E, ranges):
        extra = 0 if ranges == 1 else -(-(4 * ranges * m * E) // 256) * 256
        assert lib.moe_router_workspace(m, hidden, E) == 256 + extra
    expect(4096, 4096, 256, 4)    # 32 tiles
    expect(300, 2048, 128, 8)     # 3 tiles, capped at 8 ranges
    expect(1, 512, 8, 2)          # 8 k-blocks: 2 ranges of at least 4
    expect(130, 136, 1000, 1)     # 3 k-blocks: no split
    expect(64, 1024, 512, 4)      # 2 tiles, 16 k-blocks
    expect(20000, 4096, 256, 1)   # 157 tiles: no split


def _route(lib, m=4, E=8, k=2, logits=FAKE, ids=FAKE, w=FAKE):
    return lib.moe_route_topk(logits, None, m, E, k, ids, w, None, None)


def test_route_validation(lib):
    assert _route(lib, m=0) == OK                     # empty call launches nothing
    assert _route(lib, m=-1) == INVALID
    assert _route(lib, E=0) == UNSUPPORTED
    assert _route(lib, E=1025) == UNSUPPORTED
    assert _route(lib, k=0) == UNSUPPORTED
    assert _route(lib, k=9, E=8) == UNSUPPORTED        # top_k > n_experts
    assert _route(lib, k=33, E=64) == UNSUPPORTED      # top_k > 32
    assert _route(lib, m=(1 << 22) + 1, k=4) == UNSUPPORTED  # m*top_k > 2^24
    assert _route(lib, logits=None) == INVALID
    assert b"logits" in lib.moe_last_error()
    assert _route(lib, ids=FAKE + 2) == INVALID        # misaligned


def _mm(lib, m=300, n=32, k=64, top_k=2, E=8, layout=0, x=FAKE, W=FAKE, y=FAKE, ws=FAKE,
        ws_bytes=1 << 40):
    return lib.moe_matmul_id(x, FAKE, W, y, m, n, k, top_k, E, layout, ws, ws_bytes, None)


def test_matmul_id_validation(lib):
    assert _mm(lib, m=0) == OK
    assert _mm(lib, k=37) == UNSUPPORTED               # 16-byte rows needed (k % 8)
    assert _mm(lib, k=0) == UNSUPPORTED
    assert _mm(lib, n=0) == UNSUPPORTED
    assert _mm(lib, layout=2) == INVALID
    assert _mm(lib, x=FAKE + 8) == INVALID             # x not 16-byte aligned
    assert _mm(lib, W=None) == INVALID
    assert _mm(lib, ws=FAKE + 16) == INVALID           # workspace not 256-byte aligned
    need = lib.moe_matmul_id_workspace(300, 32, 64, 2, 8, 0)
    assert _mm(lib, ws_bytes=need - 1) == WS_SMALL
    assert b"workspace" in lib.moe_last_error()


def _mms(lib, stride, m=300, n=32, k=64, top_k=2, E=8):
    return lib.moe_matmul_id_strided(FAKE, FAKE, FAKE, stride, FAKE, m, n, k, top_k, E, 0, FAKE,
                                     1 << 40, None)


def test_matmul_id_strided_validation(lib):
    dense = 32 * 64 * 2
    assert _mms(lib, dense, m=0) == OK
    assert _mms(lib, 0) == INVALID                     # a stride is required
    assert _mms(lib, dense - 16) == INVALID            # experts would overlap
    assert b"n*k*2" in lib.moe_last_error()
    assert _mms(lib, dense + 8) == UNSUPPORTED         # TMA strides are 16-byte multiples
    assert _mms(lib, 1 << 40) == UNSUPPORTED
    assert _mms(lib, dense + 16, k=37) == UNSUPPORTED  # same k rule as moe_matmul_id


def _ffn(lib, m=64, hidden=64, inter=32, top_k=2, E=4, layout=0, ws_bytes=1 << 40, W_down=FAKE):
    return lib.moe_ffn_forward(FAKE, FAKE, FAKE, FAKE, FAKE, W_down, FAKE, m, hidden, inter, top_k,
                               E, layout, FAKE, ws_bytes, None)


def test_ffn_validation(lib):
    assert _ffn(lib, m=0) == OK
    assert _ffn(lib, hidden=60) == UNSUPPORTED
    assert _ffn(lib, inter=12) == UNSUPPORTED
    assert _ffn(lib, top_k=5, E=4) == UNSUPPORTED
    assert _ffn(lib, layout=-1) == INVALID
    assert _ffn(lib, W_down=None) == INVALID
    need = lib.moe_ffn_workspace(64, 64, 32, 2, 4, 0)
    assert _ffn(lib, ws_bytes=need - 1) == WS_SMALL


def _ffn_sh(lib, m=64, hidden=64, inter=32, inter_sh=48, top_k=2, E=4, ws_bytes=1 << 40,
            w_sh=FAKE, W_sh_down=FAKE):
    return lib.moe_ffn_forward_shared(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, w_sh, FAKE, FAKE,
                                      W_sh_down, FAKE, m, hidden, inter, inter_sh, top_k, E, FAKE,
                                      ws_bytes, None)


def test_ffn_shared_validation(lib):
    assert _ffn_sh(lib, m=0) == OK
    assert _ffn_sh(lib, inter_sh=12) == UNSUPPORTED
    assert _ffn_sh(lib, hidden=60) == UNSUPPORTED
    assert _ffn_sh(lib, w_sh=None) == INVALID
    assert _ffn_sh(lib, W_sh_down=FAKE + 8) == INVALID
    need = lib.moe_ffn_shared_workspace(64, 64, 32, 48, 2, 4)
    routed = lib.moe_ffn_workspace(64, 64, 32, 2, 4, 0)
    # the shared part adds at least its activation (2 * m * inter_sh bf16) and rows (m * hidden f32)
    assert need >= routed + 2 * 64 * 48 * 2 + 64 * 64 * 4
    assert _ffn_sh(lib, ws_bytes=need - 1) == WS_SMALL
    assert lib.moe_ffn_shared_workspace(64, 64, 32, 0, 2, 4) == 0


def test_ffn_slots_validation(lib):
    f = lib.moe_ffn_slots
    need = lib.moe_ffn_workspace(64, 64, 32, 2, 4, 0)
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 32, 2, 4, 0, FAKE, need, None) == OK
    assert f(FAKE, FAKE, FAKE, FAKE, None, FAKE, 64, 64, 32, 2, 4, 0, FAKE, need, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, 60, 32, 2, 4, 0, FAKE, need, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, 64, 32, 2, 4, 0, FAKE, need - 1, None) == WS_SMALL


def test_expert_map_validation(lib):
    f = lib.moe_expert_map
    assert f(FAKE, 0, 2, 8, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None) == OK
    assert f(None, 4, 2, 8, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == INVALID
    assert f(FAKE, 4, 2, 8, FAKE, FAKE, FAKE, FAKE, FAKE, 8, None) == WS_SMALL


def test_selftest_validation(lib):
    assert lib.moe_selftest_wait_timeout(None, 1000, None) == INVALID
    assert lib.moe_selftest_wait_timeout(FAKE, 0, None) == INVALID
    assert lib.moe_selftest_wait_timeout(FAKE, 10 ** 10, None) == INVALID


def test_python_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        moe.moe_route_topk(torch.zeros((2, 4)), None, 2)
    with pytest.raises(TypeError):
        moe.moe_route_topk(torch.zeros((2, 4), dtype=torch.float64), None, 2)


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """include/moe_b200.h from plain C11 (-Wall -Werror), linked against the
    library; the program makes host-side calls only."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = os.path.join(ROOT, "tests", "c", "abi_check.c")
    libdir = os.path.dirname(moe.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror",
                           "-I", os.path.join(ROOT, "include"), src, "-o", exe,
                           "-L", libdir, "-l:libmoe_b200.so", "-Wl,-rpath," + libdir])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert "abi ok" in out.stdout
