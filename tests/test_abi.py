"""The C-ABI library loads, exports every symbol the header declares, and its
host-side logic (sizes, argument checks, status strings) behaves as stated.
No compute call here needs a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sta.h")
PROBE_HEADER = os.path.join(ROOT, "include", "sta_probe.h")


@pytest.fixture(scope="module")
def sta():
    import runpy

    runpy.run_path(os.path.join(ROOT, "block_sparse_attention_28_b200", "build.py"), run_name="sta_build")["build"]()
    import block_sparse_attention_28_b200 as mod

    return mod


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sta_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("sta_reorder", "sta_build_mask", "sta_build_mask_workspace", "sta_attn_fwd",
                 "sta_get_device_error", "sta_status_string", "sta_num_tiles", "sta_tiled_len"):
        assert want in names


def test_library_exports_every_declared_symbol(sta):
    lib = ctypes.CDLL(sta.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_checked_build_exports_the_same_boundary_and_says_so(sta):
    """libsta_debug.so (device-side bounds checks compiled in) carries every
    symbol of the header; sta_debug_build tells the two builds apart."""
    checked = ctypes.CDLL(os.path.join(os.path.dirname(sta.LIB_PATH), "libsta_debug.so"))
    for name in declared_functions():
        assert hasattr(checked, name), name
    product = ctypes.CDLL(os.path.join(os.path.dirname(sta.LIB_PATH), "libsta.so"))
    checked.sta_debug_build.restype = ctypes.c_int32
    product.sta_debug_build.restype = ctypes.c_int32
    assert checked.sta_debug_build() == 1 and product.sta_debug_build() == 0
    assert sta.sta_debug_build() == (1 if sta.CHECKED else 0)


def test_probe_library_exports_its_symbols_and_the_product_header_has_none(sta):
    from block_sparse_attention_28_b200 import probe

    names = declared_functions(PROBE_HEADER)
    assert names == ["sta_probe_get_device_error", "sta_probe_mma_rate", "sta_probe_tma_stream"]
    lib = ctypes.CDLL(probe.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name
    # the measurement probes are not part of the product boundary
    assert not [n for n in declared_functions() if "probe" in n or n.startswith("sta_selftest_") and
                n != "sta_selftest_wait_timeout"]


def test_tile_counts(sta):
    assert sta.sta_num_tiles(sta.grid(21, 45, 80)) == 1260
    assert sta.sta_tiled_len(sta.grid(21, 45, 80)) == 80640
    assert sta.sta_num_tiles(sta.grid(33, 45, 80)) == 1980
    assert sta.sta_num_tiles(sta.grid(21, 30, 52)) == 588
    assert sta.sta_num_tiles(sta.grid(0, 4, 4)) == -1


def test_workspace_size(sta):
    g = sta.grid(21, 45, 80)
    ws = sta.sta_build_mask_workspace(1, 40, 128, g)
    R = 40 * 1260
    ws_min = sta.sta_build_mask_workspace_min(1, 40, 128, g)
    assert ws_min >= 2 * R * 128 * 4 + R * 40 * 4 + R * 4
    # plus the low tf32 parts of the pooled Q and K and the row buffer of the
    # tensor-core layout
    assert ws >= ws_min + 2 * R * 128 * 4 + R * 1260 * 4
    assert ws % 256 == 0 and ws_min % 256 == 0
    assert sta.sta_build_mask_workspace(1, 40, 96, g) == 0


def test_argument_checks_return_before_any_launch(sta):
    g = sta.grid(4, 16, 16)
    lib = sta._lib
    # unsupported head dim, bad batch, null pointers, misaligned pointers
    assert lib.sta_reorder(16, 32, 1, 2, 96, g, 0, None) == sta.STA_ERR_UNSUPPORTED
    assert lib.sta_reorder(16, 32, 0, 2, 64, g, 0, None) == sta.STA_ERR_INVALID_ARG
    assert lib.sta_reorder(None, 32, 1, 2, 64, g, 0, None) == sta.STA_ERR_INVALID_ARG
    assert lib.sta_reorder(17, 32, 1, 2, 64, g, 0, None) == sta.STA_ERR_INVALID_ARG
    assert lib.sta_attn_fwd(None, 16, 16, 16, None, 16, 16, 1, 2, 64, g, 0.0, None) == sta.STA_ERR_INVALID_ARG
    assert lib.sta_attn_fwd(16, 16, 16, 16, None, 16, 16, 1, 2, 64, g, -1.0, None) == sta.STA_ERR_INVALID_ARG
    p = sta.mask_params(0.9, 2, True)
    assert lib.sta_build_mask(16, 16, 1, 2, 64, g, ctypes.byref(p), 16, 16, 16, None, None, None, 0,
                              None) == sta.STA_ERR_WORKSPACE
    bad = sta.mask_params(0.9, 2, True, group_lo=(1, 2), windows=16)
    assert lib.sta_build_mask(16, 16, 1, 2, 64, g, ctypes.byref(bad), 16, 16, 16, None, None, 256, 1 << 30,
                              None) == sta.STA_ERR_INVALID_ARG
    too_big = sta.grid(1 << 12, 1 << 10, 1 << 10)
    assert lib.sta_reorder(16, 32, 1, 2, 64, too_big, 0, None) != sta.STA_OK


def test_paired_attention_needs_its_pairs(sta):
    """sta_attn_fwd_paired / _raster_paired refuse a NULL or misaligned pair
    array before anything runs."""
    lib = ctypes.CDLL(sta.LIB_PATH)
    g = sta.grid(2, 16, 16)
    for fn in (lib.sta_attn_fwd_paired, lib.sta_attn_fwd_raster_paired):
        fn.argtypes = sta._lib.sta_attn_fwd_paired.argtypes
        assert fn(16, 16, 16, 16, None, 16, 16, None, 1, 1, 64, g, 0.0, None) == sta.STA_ERR_INVALID_ARG
        assert fn(16, 16, 16, 16, None, 16, 16, 18, 1, 1, 64, g, 0.0, None) == sta.STA_ERR_INVALID_ARG


def test_csr_validation_checks_its_arguments_on_the_host(sta):
    lib = ctypes.CDLL(sta.LIB_PATH)
    lib.sta_validate_csr.argtypes = sta._lib.sta_validate_csr.argtypes
    g = sta.grid(2, 16, 16)
    assert lib.sta_validate_csr(None, 16, 8, 1, 1, g, None) == sta.STA_ERR_INVALID_ARG
    assert lib.sta_validate_csr(16, None, 8, 1, 1, g, None) == sta.STA_ERR_INVALID_ARG
    assert lib.sta_validate_csr(16, 16, -1, 1, 1, g, None) == sta.STA_ERR_INVALID_ARG
    assert lib.sta_validate_csr(16, 16, 8, 0, 1, g, None) == sta.STA_ERR_INVALID_ARG
    assert lib.sta_validate_csr(16, 16, 8, 1, 1, sta.grid(0, 16, 16), None) == sta.STA_ERR_INVALID_ARG


def test_status_strings(sta):
    for s in range(8):
        assert sta.sta_status_string(s) != "unknown status"
    assert "out of range" in sta.sta_status_string(sta.STA_ERR_BAD_MASK)
    assert "checked build" in sta.sta_status_string(sta.STA_ERR_BOUNDS)


def test_selftest_limit_is_checked_on_the_host(sta):
    assert sta._lib.sta_selftest_wait_timeout(10, None) == sta.STA_ERR_INVALID_ARG
    assert sta._lib.sta_selftest_wait_timeout(3_000_000_000, None) == sta.STA_ERR_INVALID_ARG


def test_mma_rate_arguments_are_checked_on_the_host(sta):
    from block_sparse_attention_28_b200 import probe

    buf = ctypes.c_int64(0)
    for n, iters in ((96, 10), (64, 0), (128, (1 << 20) + 1)):
        assert probe._lib.sta_probe_mma_rate(n, 0, iters, ctypes.byref(buf), None) == sta.STA_ERR_INVALID_ARG
    assert probe._lib.sta_probe_mma_rate(64, 0, 10, None, None) == sta.STA_ERR_INVALID_ARG


def test_binding_mirrors_the_noalloc_array_size(sta):
    m = re.search(r"#define\s+STA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", open(HEADER).read())
    assert m, "STA_NOALLOC_SCRATCH_BYTES not found in the header"
    assert sta.STA_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
