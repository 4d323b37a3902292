"""CPU-only checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching a GPU."""

import ctypes
import os
import re

import pytest

from w4a8_quantized_moe_token_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a8.h")

EINVAL, EALIGN, ENOSPACE, EUNSUPPORTED = -1, -2, -3, -5


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a(?:8|16)_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        from w4a8_quantized_moe_token_b200 import build
        build.build()
    return B.lib()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.exported_symbols())


def test_version_and_status_strings(lib):
    assert lib.w4a8_version() == 100
    assert lib.w4a8_status_string(0) == b"ok"
    assert lib.w4a8_status_string(ENOSPACE).startswith(b"buffer")


def test_packed_bytes_accounting(lib):
    # 256-byte header + one 8704-byte block per (matrix, 128-row tile, 128-wide group)
    assert lib.w4a8_packed_bytes(1, 256, 512, 0) == 256 + 2 * 4 * 8704
    assert lib.w4a8_packed_bytes(8, 2048, 2048, 1) == 256 + 8 * 16 * 16 * 8704
    assert lib.w4a8_packed_bytes(1, 100, 200, 0) == 256 + 1 * 1 * 2 * 8704
    assert lib.w4a8_packed_bytes(1, 3, 128, 1) == 0  # odd N for gate|up
    # the symmetric scheme flag keeps the format (and size); unknown flags are refused
    assert lib.w4a8_packed_bytes(8, 2048, 2048, 1 | 0x100) == lib.w4a8_packed_bytes(8, 2048, 2048, 1)
    assert lib.w4a8_packed_bytes(1, 256, 512, 0x200) == lib.w4a8_packed_bytes(1, 256, 512, 0)
    assert lib.w4a8_packed_bytes(1, 256, 512, 0x300) == 0  # two scheme flags
    assert lib.w4a8_packed_bytes(1, 256, 512, 0x1000) == 0  # unknown flag
    # group sizes: group 64 blocks carry two scale / zero-point pairs per row (9216 bytes),
    # group 256 pads K to 256 and repeats its pair in both planes (8704 bytes)
    assert lib.w4a8_packed_bytes(1, 256, 512, 0x400) == 256 + 2 * 4 * 9216
    assert lib.w4a8_packed_bytes(1, 256, 512, 0x800) == 256 + 2 * 4 * 8704
    assert lib.w4a8_packed_bytes(1, 128, 300, 0x800) == 256 + 4 * 8704  # K 300 -> 512
    assert lib.w4a8_packed_bytes(1, 128, 300, 0x400) == 256 + 3 * 9216  # K 300 -> 384
    assert lib.w4a8_packed_bytes(1, 256, 512, 0x400 | 0x800) == 0  # two group sizes
    assert lib.w4a8_packed_bytes(1, 256, 512, 0x200 | 0x400) == 0  # percentile range needs group 128
    assert lib.w4a8_packed_bytes(1, 256, 512, 0x100 | 0x800) == 256 + 2 * 4 * 8704  # symmetric, group 256
    assert lib.w4a8_packed_bytes(0, 128, 128, 0) == 0
    # per weight: 0.5 byte of codes + 4 bytes per 128-group of scale and zero point
    blk = 8704
    assert blk == 128 * 128 // 2 + 128 * 4


def test_host_validation_without_gpu(lib):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)  # aligned, never dereferenced: validation fails first
    assert lib.w4a8_quant_act(None, 4, 128, None, None, None) == EINVAL
    assert lib.w4a8_quant_act(fake, -1, 128, fake, fake, None) == EINVAL
    assert lib.w4a8_quant_act(vp((1 << 20) + 2), 4, 128, fake, fake, None) == EALIGN
    assert lib.w4a8_quant_act(fake, 0, 128, fake, fake, None) == 0  # nothing to do
    assert lib.w4a8_pack_weights(fake, 1, 256, 512, 0, fake, 100, None, None, None, None) == ENOSPACE
    assert lib.w4a8_pack_weights(fake, 1, 256, 512, 7, fake, 1 << 30, None, None, None, None) == EINVAL
    assert lib.w4a8_route_topk(fake, 4, 2000, 2, fake, fake, None) == EUNSUPPORTED
    assert lib.w4a8_route_topk(fake, 4, 8, 9, fake, fake, None) == EINVAL
    ws_small = 16
    assert lib.w4a8_moe_forward(fake, fake, 8, 256, 128, fake, 4, fake, fake, 2, fake, fake, ws_small, None) == ENOSPACE
    assert lib.w4a8_moe_forward(fake, vp((1 << 20) + 16), 8, 256, 128, fake, 4, fake, fake, 2, fake, fake, 1 << 40,
                                None) == EALIGN
    assert lib.w4a8_moe_forward(fake, fake, 2048, 256, 128, fake, 4, fake, fake, 2, fake, fake, 1 << 40,
                                None) == EUNSUPPORTED
    assert lib.w4a8_moe_forward(fake, fake, 8, 256, 128, fake, 4, fake, fake, 9, fake, fake, 1 << 40, None) == EINVAL
    assert lib.w4a8_gemm(fake, fake, 4, fake, 256, 512, fake, None, fake, 8, None) == ENOSPACE
    assert lib.w4a8_last_device_error(None, None) == EINVAL
    # INT8 KV cache
    assert lib.w4a8_kv_quant(fake, 4, 8, 100, fake, fake, None) == EUNSUPPORTED  # D % 16
    assert lib.w4a8_kv_quant(fake, 4, 2000, 128, fake, fake, None) == EUNSUPPORTED  # too many heads
    assert lib.w4a8_kv_quant(fake, 4, 0, 128, fake, fake, None) == EINVAL
    assert lib.w4a8_kv_quant(fake, 0, 8, 128, None, None, None) == 0  # nothing to do
    assert lib.w4a8_kv_quant(vp((1 << 20) + 8), 4, 8, 128, fake, fake, None) == EALIGN
    assert lib.w4a8_kv_dequant(fake, 4, 8, 128, None, fake, None) == EINVAL
    assert lib.w4a8_kv_calibrate(fake, 4, 8, 128, None, None) == EINVAL
    assert lib.w4a8_kv_calibrate(fake, 4, 8, 128, vp((1 << 20) + 2), None) == EALIGN


def test_moe_workspace_regions(lib):
    T, E, k, H, F = 64, 64, 6, 4096, 1408
    R = lib.w4a8_moe_rows_capacity(T, E, k)
    assert R % 16 == 0 and R >= T * k and R <= T * k + 15 * E + 16
    total = lib.w4a8_moe_workspace_bytes(T, E, k, H, F)
    regions = []
    for what in range(12):
        off, nb = B.w4a8_debug_region(T, E, k, H, F, what)
        assert off % 256 == 0 and off + nb <= total
        regions.append((off, nb))
    # the documented sizes
    assert regions[B.DUMP["counts"]][1] == 4 * E
    assert regions[B.DUMP["act1"]][1] == (4096 // 128) * R * 128
    assert regions[B.DUMP["h"]][1] == R * 1408 * 2  # bf16
    assert regions[B.DUMP["act2"]][1] == (1408 // 128) * R * 128
    assert regions[B.DUMP["y2"]][1] == R * H * 4
    s = sorted(r for r in regions if r[1] > 4)
    for (o1, n1), (o2, _) in zip(s, s[1:]):
        assert o1 + n1 <= o2  # no overlap
    assert lib.w4a8_moe_host_workspace_bytes(T, E, k, H, F) >= total + 2 * T * H * 2
    assert lib.w4a8_moe_workspace_bytes(T, E, 40, H, F) == 0  # k > 32
    assert lib.w4a8_moe_rows_capacity(0, 8, 2) == 0


def test_gemm_workspace(lib):
    assert lib.w4a8_gemm_workspace_bytes(16, 256, 512) >= 4 * 16 * 128
    assert lib.w4a8_gemm_workspace_bytes(0, 256, 512) > 0
    assert lib.w4a8_gemm_workspace_bytes(-1, 256, 512) == 0


def test_debug_inject_validates_its_arguments(lib):
    assert lib.w4a8_debug_inject(0x80, 0) == EINVAL  # unknown flag
    assert lib.w4a8_debug_inject(0, -1) == EINVAL  # negative wait limit
    assert lib.w4a8_debug_inject(1, 1000) == 0
    assert lib.w4a8_debug_inject(0, 0) == 0  # back to normal operation


def test_logits_host_forward_validates_on_the_host(lib):
    # invalid shapes and a missing workspace are refused before any CUDA call
    assert lib.w4a8_moe_forward_logits_host(None, None, 0, 256, 128, None, 4, None, 2, None, None, 0, None) == EINVAL
    assert lib.w4a8_moe_forward_logits_host(None, None, 8, 256, 128, None, 4, None, 2, None, None, 0, None) == EINVAL


def test_w4a16_workspaces_and_validation(lib):
    T, E, k, H, F = 64, 64, 6, 4096, 1408
    R = lib.w4a8_moe_rows_capacity(T, E, k)
    total = lib.w4a16_moe_workspace_bytes(T, E, k, H, F)
    regions = {}
    for what in range(12):
        off, nb = B.w4a8_debug_region(T, E, k, H, F, what | B.W4A8_DUMP_W4A16)
        assert off % 256 == 0 and off + nb <= total
        regions[what] = (off, nb)
    # bf16 token rows: 256 bytes per row and K group; no INT8 scales, no fp32 h
    assert regions[B.DUMP["act1"]][1] == (4096 // 128) * R * 256
    assert regions[B.DUMP["act2"]][1] == 11 * R * 256  # Fp = 1408 -> 11 groups
    assert regions[B.DUMP["s1"]][1] == regions[B.DUMP["h"]][1] == regions[B.DUMP["s2"]][1] == 0
    assert regions[B.DUMP["y2"]][1] == R * H * 4
    assert lib.w4a16_moe_workspace_bytes(T, E, 40, H, F) == 0  # k > 32
    assert lib.w4a16_gemm_workspace_bytes(16, 256, 512) >= 4 * 16 * 256
    assert lib.w4a16_gemm_workspace_bytes(-1, 256, 512) == 0
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    assert lib.w4a16_gemm(fake, 4, fake, 256, 512, fake, fake, 8, None) == ENOSPACE
    assert lib.w4a16_gemm(fake, 4, vp((1 << 20) + 16), 256, 512, fake, fake, 1 << 40, None) == EALIGN
    assert lib.w4a16_moe_forward(fake, fake, 8, 256, 128, fake, 4, fake, fake, 2, fake, fake, 16, None) == ENOSPACE
    assert lib.w4a16_moe_forward(fake, fake, 8, 256, 128, fake, 4, fake, fake, 9, fake, fake, 1 << 40, None) == EINVAL


def test_group_size_entry_points_validate(lib):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    assert lib.w4a8_gemm_workspace_bytes_g(16, 256, 300, 256) >= 4 * 16 * 128  # K 300 -> 4 planes
    assert lib.w4a8_gemm_workspace_bytes_g(16, 256, 300, 96) == 0  # not a group size
    assert lib.w4a8_gemm_g(fake, fake, 4, fake, 256, 512, 32, fake, None, fake, 1 << 40, None) == EINVAL
    assert lib.w4a8_moe_workspace_bytes_g(64, 8, 2, 300, 200, 256) > lib.w4a8_moe_workspace_bytes(64, 8, 2, 300, 200)
    assert lib.w4a8_moe_workspace_bytes_g(64, 8, 2, 300, 200, 128) == lib.w4a8_moe_workspace_bytes(64, 8, 2, 300, 200)
    assert lib.w4a8_moe_forward_g(fake, fake, 8, 256, 128, 100, fake, 4, fake, fake, 2, fake, fake, 1 << 40,
                                  None) == EINVAL
    # dump regions of a group-256 workspace: rows padded to whole groups (H 300 -> 512)
    R = lib.w4a8_moe_rows_capacity(64, 8, 2)
    _, nb = B.w4a8_debug_region(64, 8, 2, 300, 200, B.DUMP["act1"] | B.DUMP_GROUP[256])
    assert nb == 4 * R * 128
