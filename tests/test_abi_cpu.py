"""libwq.so on a machine without a GPU: it loads, exports every declared entry
point, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]


def declared_functions():
    text = (ROOT / "include" / "wq.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(wq_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("wq_pack_kmajor", "wq_unpack_kmajor", "wq_gemv", "wq_gemm", "wq_status_string",
              "wq_abi_version", "wq_device_status"):
        assert n in names


def test_every_declared_symbol_is_exported(libwq):
    L = libwq.lib()
    for n in declared_functions():
        assert hasattr(L, n), f"{n} declared in include/wq.h but not exported"


def test_version_and_strings(libwq):
    L = libwq.lib()
    assert L.wq_abi_version() == 3
    for s in range(10):
        assert L.wq_status_string(s) and L.wq_status_string(s) != b"unknown status"
    assert L.wq_checked_build() in (0, 1)
    assert L.wq_status_string(99) == b"unknown status"


P = 0x10000  # a 16-byte aligned fake device address: never dereferenced on the host path


def gemv(L, fn="wq_gemv", x=P, wq=P, wlo=None, s=P, z=P, y=P, M=1, K=512, N=256, bits=4, G=128,
         flags=0, ws=None, ws_bytes=0, bias=None):
    if fn == "wq_gemm":
        return L.wq_gemm(x, wq, wlo, s, z, bias, y, M, K, N, bits, G, flags, ws,
                         ctypes.c_size_t(ws_bytes), None)
    return getattr(L, fn)(x, wq, wlo, s, z, bias, y, M, K, N, bits, G, flags, None)


@pytest.mark.parametrize("fn", ["wq_gemv", "wq_gemm"])
def test_product_argument_checks(libwq, fn):
    L = libwq.lib()
    INV, UNS, ALI, CUDA = 1, 2, 3, 6
    assert gemv(L, fn, bits=5) == UNS
    assert gemv(L, fn, bits=0) == UNS
    assert gemv(L, fn, M=0) == INV
    assert gemv(L, fn, K=0) == INV
    assert gemv(L, fn, N=0) == INV
    assert gemv(L, fn, K=500, G=-1) == INV                # K not a multiple of 8 (4-bit)
    assert gemv(L, fn, G=100) == INV                      # does not divide K
    assert gemv(L, fn, G=0) == INV
    assert gemv(L, fn, bits=3, K=512, G=128) == INV       # 3-bit needs w_lo
    assert gemv(L, fn, bits=4, wlo=P) == INV              # w_lo only for 3-bit
    assert gemv(L, fn, bits=3, K=528, wlo=P, G=-1) == INV  # 3-bit needs K % 32 == 0
    assert gemv(L, fn, x=None) == INV
    assert gemv(L, fn, y=None) == INV
    assert gemv(L, fn, N=252) == ALI                      # N % 8
    assert gemv(L, fn, x=P + 8) == ALI
    assert gemv(L, fn, wq=P + 4) == ALI
    assert gemv(L, fn, bias=P + 1) == ALI                 # bias: 2-byte aligned fp16 / bf16
    assert gemv(L, fn, flags=8) == INV                    # unknown flag bit
    assert gemv(L, fn, flags=0x80000000 | 4) == INV
    # valid arguments: the host checks pass and the call reaches CUDA, which has no device here
    import torch
    if not torch.cuda.is_available():
        assert gemv(L, fn) == CUDA
        assert gemv(L, fn, bits=3, wlo=P, K=512, G=128) == CUDA
        assert gemv(L, fn, flags=4) == CUDA               # WQ_FLAG_BF16
        assert gemv(L, fn, flags=1 | 4) == CUDA
        assert gemv(L, fn, flags=2 | 4) == CUDA


def test_flag_values_match_the_header(libwq):
    text = (ROOT / "include" / "wq.h").read_text()
    vals = dict(re.findall(r"#define (WQ_FLAG_\w+) (\d+)u", text))
    assert vals == {"WQ_FLAG_PDL": str(libwq.WQ_FLAG_PDL),
                    "WQ_FLAG_PDL_INPUTS_READY": str(libwq.WQ_FLAG_PDL_INPUTS_READY),
                    "WQ_FLAG_BF16": str(libwq.WQ_FLAG_BF16)}


def test_gemv_specific_limits(libwq):
    L = libwq.lib()
    assert gemv(L, "wq_gemv", M=17) == 1
    assert gemv(L, "wq_gemv", bits=4, G=16, K=512) == 2   # group not a multiple of 4*eps
    assert gemv(L, "wq_gemv", bits=1, G=64, K=512) == 2
    assert gemv(L, "wq_gemm", ws=P + 8, ws_bytes=1 << 20) == 3  # workspace alignment
    assert gemv(L, "wq_gemm", bits=8, K=516, G=-1) == 3   # x rows of 516 values are not 16-byte multiples
    import torch
    if not torch.cuda.is_available():
        # any K that is a multiple of eps (and of 8) and any group that divides K and is a
        # multiple of eps pass the host checks and reach CUDA, which has no device here
        assert gemv(L, "wq_gemm", K=544, G=-1) == 6       # a ragged 64-deep block
        assert gemv(L, "wq_gemm", K=4160, N=264, M=48, G=-1) == 6
        assert gemv(L, "wq_gemm", K=576, G=96) == 6       # groups straddle 64-deep blocks
        assert gemv(L, "wq_gemm", bits=3, wlo=P, K=96 * 32, G=96) == 6
        assert gemv(L, "wq_gemm", bits=8, K=520, G=40) == 6


def test_gemm_workspace_size(libwq):
    """The size query follows the tile plan: 128-column x (<= 256)-token tiles,
    K split over 8, 4 or 2 CTAs while the grid fits the SMs once (148 SMs are
    assumed without a device) and each CTA keeps two 64-deep k blocks; one
    128 x 32 fp32 slice per CTA and 32-token chunk."""
    import torch
    L = libwq.lib()
    size = lambda *a: int(L.wq_gemm_workspace_size(*a))
    slice_bytes = 128 * 32 * 4
    if not torch.cuda.is_available():
        assert size(1, 4096, 4096, 4, 128) == 32 * 4 * 1 * slice_bytes       # 32 tiles x CS 4
        assert size(512, 4096, 4096, 4, 128) == 64 * 2 * 8 * slice_bytes     # 64 tiles x CS 2
        assert size(16, 1024, 1024, 4, 128) == 8 * 8 * 1 * slice_bytes       # KB 16: CS 8
    assert size(512, 4096, 16384, 4, 128) == 0   # 256 tiles: no split
    assert size(1, 128, 4096, 4, 128) == 0       # two k blocks: no split
    assert size(0, 4096, 4096, 4, 128) == 0      # invalid arguments
    assert size(1, 4096, 4096, 5, 128) == 0
    assert size(1, 4000, 4096, 4, 128) == 0      # the group does not divide K
    assert size(1, 4092, 4096, 4, -1) == 0       # K not a multiple of 8
    assert size(1, 4096, 4096, 4, 12) == 0       # group not a multiple of eps


def test_pack_argument_checks(libwq):
    L = libwq.lib()
    assert L.wq_pack_kmajor(P, 12, 4, 4, P, None, None, None) == 1   # K % 8
    assert L.wq_pack_kmajor(P, 32, 4, 6, P, None, None, None) == 2
    assert L.wq_pack_kmajor(P, 32, 4, 3, P, None, None, None) == 1   # 3-bit needs w_lo
    assert L.wq_pack_kmajor(None, 32, 4, 4, P, None, None, None) == 1
    assert L.wq_pack_kmajor(P, 32, 4, 4, P + 2, None, None, None) == 3
    assert L.wq_unpack_kmajor(P, P, 32, 4, 4, P, None) == 1          # w_lo with 4-bit


def test_matmul_route(libwq):
    """wq_matmul's crossover: wq_gemv for M <= 8, or M <= 16 with 4- or 8-bit
    words or M * K < 65536, when the group size is one wq_gemv takes; wq_gemm
    otherwise."""
    L = libwq.lib()
    route = lambda *a: int(L.wq_matmul_uses_gemv(*a))
    assert route(1, 4096, 4096, 4, 128) == 1
    assert route(8, 8192, 8192, 4, 128) == 1
    assert route(12, 4096, 4096, 4, 128) == 1
    assert route(12, 8192, 4096, 4, 128) == 1      # 4-bit: up to 16 tokens
    assert route(16, 4096, 4096, 8, 128) == 1
    assert route(12, 8192, 4096, 2, 128) == 0      # 2-bit: 12 x 8192 >= 65536
    assert route(16, 4096, 4096, 3, 128) == 0      # 3-bit: 16 x 4096 = 65536
    assert route(16, 2048, 4096, 1, 128) == 1      # 1-bit: 16 x 2048 < 65536
    assert route(17, 512, 256, 4, 128) == 0
    assert route(1, 4096, 4096, 4, 16) == 0        # group 16 is wq_gemm's only
    assert route(1, 4096, 4096, 4, -1) == 1
    assert route(1, 4096, 4096, 5, 128) == 0
    assert int(L.wq_matmul_workspace_size(1, 4096, 4096, 4, 128)) == 0
    assert int(L.wq_matmul_workspace_size(512, 4096, 2048, 4, 128)) == \
        int(L.wq_gemm_workspace_size(512, 4096, 2048, 4, 128))
    # argument checks pass through: M = 0 is rejected before anything runs
    assert L.wq_matmul(P, P, None, P, P, None, P, 0, 512, 256, 4, 128, 0, None, ctypes.c_size_t(0), None) == 1


def test_selftest_argument_checks(libwq):
    """The failure-path self-test rejects limits outside 1 us .. 1 s before any launch."""
    L = libwq.lib()
    assert L.wq_selftest_wait_timeout(0, None) == 1
    assert L.wq_selftest_wait_timeout(999, None) == 1
    assert L.wq_selftest_wait_timeout(2_000_000_000, None) == 1
    import torch
    if not torch.cuda.is_available():
        assert L.wq_selftest_wait_timeout(1_000_000, None) == 6   # reaches CUDA: no device here


def test_mse_search_argument_checks(libwq):
    """wq_mse_search rejects bad shapes, bit widths, candidate counts, norms and
    pointers on the host, before any launch."""
    L = libwq.lib()
    f = ctypes.c_float

    def call(w=P, rows=4, cols=64, G=16, bits=4, sym=0, steps=20, grid=100, norm=2.4, pat=0,
             out=P, ws=None, ws_bytes=0):
        return L.wq_mse_search(w, rows, cols, G, bits, sym, steps, grid, f(norm), pat, out, out, out, out, ws,
                               ctypes.c_size_t(ws_bytes), None)
    assert call(bits=0) == 2 and call(bits=9) == 2
    assert call(rows=0) == 1 and call(cols=0) == 1 and call(G=0) == 1
    assert call(cols=60, G=16) == 1                     # cols % group_size
    assert call(sym=2) == 1
    assert call(steps=0) == 1 and call(steps=33) == 1   # 1..32 candidates
    assert call(grid=0) == 1 and call(pat=-1) == 1
    assert call(norm=0.0) == 1 and call(norm=float("nan")) == 1 and call(norm=float("inf")) == 1
    assert call(w=None) == 1 and call(out=None) == 1
    assert call(pat=5) == 1                             # patience needs a 4-byte workspace
    assert call(w=P + 2) == 3
    import torch
    if not torch.cuda.is_available():
        assert call() == 6                              # valid: reaches CUDA, which has no device here
        assert call(pat=5, ws=P, ws_bytes=4) == 6


def test_gptq_argument_checks(libwq):
    """wq_gptq_quantize rejects bad shapes, bit widths, block sizes, damping,
    pointers and short workspaces on the host, before any launch."""
    L = libwq.lib()
    f = ctypes.c_float
    need = L.wq_gptq_workspace_size(16, 256)
    assert need >= 4 * (256 * 256 + 2 * 256 * 16)
    assert L.wq_gptq_workspace_size(0, 256) == 0 and L.wq_gptq_workspace_size(16, 65537) == 0

    def call(W=P, H=P, s=P, z=P, rows=16, cols=256, G=128, bits=8, bs=128, damp=0.01, Q=P, codes=P,
             losses=P, ws=P, ws_bytes=None):
        return L.wq_gptq_quantize(W, H, s, z, rows, cols, G, bits, bs, f(damp), Q, codes, losses, ws,
                                  ctypes.c_size_t(need if ws_bytes is None else ws_bytes), None)
    assert call(bits=0) == 2 and call(bits=9) == 2
    assert call(rows=0) == 1 and call(cols=0) == 1 and call(cols=65537) == 1 and call(G=0) == 1
    assert call(bs=0) == 1 and call(bs=129) == 1
    assert call(damp=-0.1) == 1 and call(damp=float("nan")) == 1 and call(damp=float("inf")) == 1
    assert call(W=None) == 1 and call(H=None) == 1 and call(s=None) == 1 and call(losses=None) == 1
    assert call(ws=None) == 1 and call(ws_bytes=need - 1) == 1
    assert call(W=P + 2) == 3 and call(ws=P + 16) == 3                # floats 4-byte, workspace 256-byte
    import torch
    if not torch.cuda.is_available():
        assert call() == 6                                 # valid: reaches CUDA, which has no device here
        assert call(Q=None, codes=None) == 6               # both outputs are optional


def test_gemv_plan_argument_checks(libwq):
    """wq_gemv_plan_*: null handles and bad shapes are refused before any CUDA call."""
    L = libwq.lib()
    P = ctypes.c_void_p(64)  # any non-null, aligned address: never dereferenced here
    h = ctypes.c_void_p()
    assert L.wq_gemv_plan_create(P, None, P, P, None, 1, 512, 256, 4, 128, 0, None) == 1     # no handle slot
    assert L.wq_gemv_plan_create(None, None, P, P, None, 1, 512, 256, 4, 128, 0, ctypes.byref(h)) == 1
    assert h.value is None                                                                  # cleared on error
    assert L.wq_gemv_plan_create(P, None, P, P, None, 17, 512, 256, 4, 128, 0, ctypes.byref(h)) == 1  # M > 16
    assert L.wq_gemv_plan_create(P, None, P, P, None, 1, 512, 260, 4, 128, 0, ctypes.byref(h)) == 3   # N % 8
    assert L.wq_gemv_plan_create(P, None, P, P, None, 1, 512, 256, 5, 128, 0, ctypes.byref(h)) == 2   # bits
    assert L.wq_gemv_plan_create(P, None, P, P, None, 1, 512, 256, 4, 16, 0, ctypes.byref(h)) == 2    # G = 16
    assert L.wq_gemv_plan_run(None, P, P, None) == 1
    L.wq_gemv_plan_destroy(None)  # allowed
