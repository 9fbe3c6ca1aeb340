"""The C ABI library: it loads, exports every entry point include/calibq.h
declares, and rejects bad arguments on the host before launching anything.
No GPU is needed for this file."""

import ctypes
import os
import re

import pytest

import oracle
from decode_attention_cq_b200 import calibq as cq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(cq_\w+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(cq.LIB_PATH):
        from decode_attention_cq_b200 import build_lib
        build_lib.build()
    return cq.load()


def test_exports_every_declared_entry_point(lib):
    declared = _declared()
    assert {"cq_quantize_kv", "cq_decode_attn", "cq_dequant"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(cq.ENTRY_POINTS) == declared


def test_version_and_status_strings(lib):
    assert cq.cq_version() == 10000
    for s in range(5):
        assert cq.status_string(s).startswith("CQ_")
    assert "unknown" in cq.status_string(99)


@pytest.mark.parametrize("layout,bits,n", [(0, 1, 3328), (0, 2, 5), (0, 8, 8192), (1, 1, 3328),
                                           (1, 1, 9), (2, 1, 3328), (2, 1, 8192), (2, 1, 1),
                                           (1, 2, 3329), (2, 2, 3329), (1, 4, 7), (2, 4, 65),
                                           (1, 8, 1), (2, 8, 33)])
def test_codes_bytes_match_the_documented_layouts(lib, layout, bits, n):
    B, H = 3, 2
    assert cq.cq_codes_bytes(layout, B, H, n, 128, bits) == B * H * oracle.codes_nbytes(layout, n, 128, bits)


def test_size_queries_validate(lib):
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_codes_bytes(1, 1, 1, 16, 64, 2)  # octet layouts need d = 128
    assert e.value.status == cq.CQ_ERR_UNSUPPORTED
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_codes_bytes(0, 1, 1, 16, 64, 1)
    assert e.value.status == cq.CQ_ERR_UNSUPPORTED
    for bad in ((0, 0, 1, 16, 128, 1), (0, 1, 1, 0, 128, 1), (0, 1, 1, 16, 128, 3), (5, 1, 1, 16, 128, 1)):
        with pytest.raises(cq.CalibqError) as e:
            cq.cq_codes_bytes(*bad)
        assert e.value.status == cq.CQ_ERR_INVALID_ARG
    assert cq.cq_decode_attn_workspace_size(1, 2, 4, 32, 8, 8192, 128, 1) == 0
    assert cq.cq_decode_attn_workspace_size(0, 0, 4, 32, 8, 1000, 128, 2) > 4 * 32 * 1000 * 4
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_decode_attn_workspace_size(1, 0, 4, 32, 8, 100, 128, 1)  # mixed layouts
    assert e.value.status == cq.CQ_ERR_UNSUPPORTED
    with pytest.raises(cq.CalibqError) as e:
        cq.cq_decode_attn_workspace_size(0, 0, 4, 30, 8, 100, 128, 1)  # Hq % Hkv != 0
    assert e.value.status == cq.CQ_ERR_INVALID_ARG
    assert cq.cq_quantize_kv_workspace_size(64, 8, 8192, 128) > 0


def test_decode_kernel_name_follows_the_documented_choice(lib):
    K, V, C = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V, cq.LAYOUT_CANONICAL
    assert cq.cq_decode_kernel_name(C, C, 2, 8, 2, 1000, 128, 3) is None  # bits
    assert cq.cq_decode_kernel_name(K, V, 2, 8, 2, 1000, 64, 1) is None  # d
    assert cq.cq_decode_kernel_name(K, V, 2, 12, 2, 1000, 128, 1) is None  # G = 6
    assert cq.cq_decode_kernel_name(K, C, 2, 8, 2, 1000, 128, 1) is None  # mixed layouts
    assert cq.cq_decode_kernel_name(C, C, 2, 12, 2, 1000, 128, 4) == "k_scores + k_softmax_v + k_merge"
    for bits in (2, 4, 8):
        assert cq.cq_decode_kernel_name(K, V, 2, 8, 2, 32768, 128, bits) == "k_decode_ring"
        assert cq.cq_decode_kernel_name(K, V, 2, 8, 2, 32769, 128, bits) is None
    assert cq.cq_decode_kernel_name(K, V, 64, 32, 8, 8192, 128, 1) in ("k_decode_row", "k_decode_mma")
    assert cq.cq_decode_kernel_name(K, V, 64, 32, 8, 8193, 128, 1) == "k_decode_mma"
    assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 32768, 128, 1) == "k_decode_mma"
    assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 32769, 128, 1) == "k_decode_octet"
    assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 65537, 128, 1) is None


def test_set_decode_kernel_forces_and_releases(lib):
    K, V = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V
    assert lib.cq_set_decode_kernel(7) == cq.CQ_ERR_INVALID_ARG
    try:
        cq.cq_set_decode_kernel(cq.KERNEL_ROW)
        assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 1000, 128, 1) == "k_decode_row"
        assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 8193, 128, 1) == "k_decode_mma"  # row takes n <= 8192
        cq.cq_set_decode_kernel(cq.KERNEL_CLUSTER)
        assert cq.cq_decode_kernel_name(K, V, 64, 32, 8, 8192, 128, 1) == "k_decode_mma"
        assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 32769, 128, 1) == "k_decode_octet"
        cq.cq_set_decode_kernel(cq.KERNEL_TCGEN05)
        assert cq.cq_decode_kernel_name(K, V, 64, 32, 8, 1000, 128, 1) == "k_decode_octet"
        cq.cq_set_decode_kernel(cq.KERNEL_PIPE)
        assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 1000, 128, 1) == "k_decode_tc"
        assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 8193, 128, 1) == "k_decode_mma"  # pipe takes n <= 8192
        cq.cq_set_decode_kernel(cq.KERNEL_AUTO)
        assert cq.cq_decode_kernel_name(K, V, 1, 8, 2, 32768, 128, 1) == "k_decode_mma"
        assert cq.cq_decode_kernel_name(K, V, 64, 32, 8, 8192, 128, 1) in ("k_decode_row", "k_decode_mma")
    finally:
        cq.cq_set_decode_kernel(cq.KERNEL_ENV)


def test_decode_launch_count(lib):
    K, V, C = cq.LAYOUT_OCTET_K, cq.LAYOUT_OCTET_V, cq.LAYOUT_CANONICAL
    assert cq.cq_decode_launch_count(C, C, 2, 8, 2, 1000, 128, 2) == 3  # scores, softmax-V, merge
    assert cq.cq_decode_launch_count(C, C, 2, 8, 2, 1000, 128, 2, 16) == 0  # mixed calls take octet layouts
    assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 2) == 1
    assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 2, 16) == 2  # ring kernel, then the text merge
    assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 64, 1) == 0  # unsupported d
    assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 1, -1) == 0
    try:
        cq.cq_set_decode_kernel(cq.KERNEL_ROW)
        assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 1, 16) == 1  # text in the same launch
        cq.cq_set_decode_kernel(cq.KERNEL_PIPE)
        assert cq.cq_decode_launch_count(K, V, 64, 32, 8, 8192, 128, 1) == 1  # one persistent launch
        cq.cq_set_decode_kernel(cq.KERNEL_AUTO)
        mixed_auto = cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 1, 16)
        cq.cq_set_decode_kernel(cq.KERNEL_PIPE)
        assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 1, 16) == mixed_auto  # mixed: as AUTO
        cq.cq_set_decode_kernel(cq.KERNEL_CLUSTER)
        assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 1) == 1
        assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 1000, 128, 1, 16) == 2
        assert cq.cq_decode_launch_count(K, V, 2, 8, 2, 40000, 128, 1, 16) == 0  # mixed: n <= 32768
    finally:
        cq.cq_set_decode_kernel(cq.KERNEL_ENV)


def test_null_pointers_rejected_before_any_cuda_call(lib):
    st = lib.cq_quantize_kv(None, 0, 1, 1, 16, 128, 1, 0, None, None, None, None, 0, None)
    assert st == cq.CQ_ERR_INVALID_ARG
    cal = cq.cq_calib(1, 0.8, 0.9)
    st = lib.cq_decode_attn(None, 0, None, None, None, 1, None, None, None, 2, 1, 4, 1, 16, 128, 1,
                            0.0, cal, None, None, 0, None)
    assert st == cq.CQ_ERR_INVALID_ARG
    st = lib.cq_dequant(None, None, None, 0, 0, 1, 1, 16, 128, 1, None, None)
    assert st == cq.CQ_ERR_INVALID_ARG
    # bad enums and shapes are caught before pointers are looked at
    assert lib.cq_quantize_kv(None, 7, 1, 1, 16, 128, 1, 0, None, None, None, None, 0, None) == cq.CQ_ERR_INVALID_ARG
    assert lib.cq_quantize_kv(None, 0, 1, 1, 16, 96, 1, 0, None, None, None, None, 0, None) == cq.CQ_ERR_UNSUPPORTED
    bad_cal = cq.cq_calib(1, float("nan"), 0.9)
    st = lib.cq_decode_attn(None, 0, None, None, None, 1, None, None, None, 2, 1, 4, 1, 16, 128, 1,
                            0.0, bad_cal, None, None, 0, None)
    assert st == cq.CQ_ERR_INVALID_ARG


def test_host_pointer_is_rejected(lib):
    buf = (ctypes.c_uint8 * 4096)()
    addr = (ctypes.addressof(buf) + 15) & ~15
    st = lib.cq_dequant(addr, addr, addr, 0, 0, 1, 1, 4, 128, 1, addr, None)
    assert st in (cq.CQ_ERR_INVALID_ARG, cq.CQ_ERR_CUDA)


def test_noalloc_refuses_oversized_scratch_before_pointers(lib):
    """cq_quantize_kv_noalloc decides its scratch limit from the sizes alone:
    only the two-launch path (n > 16384) uses the fixed 4 MiB array."""
    C = cq.LAYOUT_CANONICAL
    f = lib.cq_quantize_kv_noalloc
    assert f(None, 0, 1, 4097, 16385, 128, 1, C, None, None, None, None) == cq.CQ_ERR_UNSUPPORTED
    assert f(None, 0, 1, 4096, 16385, 128, 1, C, None, None, None, None) == cq.CQ_ERR_INVALID_ARG
    assert f(None, 0, 1, 4097, 1, 128, 1, C, None, None, None, None) == cq.CQ_ERR_INVALID_ARG  # fill path: no limit
