"""Python binding of libsta (block-sparse attention over 3D tile masks, B200).

Argument marshalling only: every step of the path runs in the CUDA kernels
of libsta.so (built in-tree by `build.py`). The C entry points keep their
names: sta_reorder, sta_build_mask, sta_attn_fwd, ... Tensors are passed as
torch tensors (device pointers are taken from them) and calls go on torch's
current CUDA stream unless a stream is given. If the library is missing the
import fails: there is no fallback path.

With STA_CHECKED=1 in the environment the checked build libsta_debug.so
(same kernels, compiled with -DSTA_DEBUG=1: run-time indices and addresses
are bounds-checked on the device and reported as STA_ERR_BOUNDS) is loaded
instead of libsta.so.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
CHECKED = os.environ.get("STA_CHECKED", "0") == "1"
LIB_PATH = os.path.join(_HERE, "libsta_debug.so" if CHECKED else "libsta.so")

STA_OK = 0
STA_ERR_INVALID_ARG = 1
STA_ERR_UNSUPPORTED = 2
STA_ERR_WORKSPACE = 3
STA_ERR_CUDA = 4
STA_ERR_TIMEOUT = 5
STA_ERR_BAD_MASK = 6
STA_ERR_BOUNDS = 7
MAX_GROUPS = 8


class StaError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {sta_status_string(status)} (status {status})")


class Grid(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32)]


class MaskParams(ctypes.Structure):
    _fields_ = [
        ("top_p", ctypes.c_float),
        ("k_min", ctypes.c_int32),
        ("use_scores", ctypes.c_int32),
        ("sm_scale", ctypes.c_float),
        ("num_groups", ctypes.c_int32),
        ("group_lo", ctypes.c_int32 * MAX_GROUPS),
        ("windows", ctypes.c_void_p),
        ("head_topk_floor", ctypes.c_int32),
        ("block_scores", ctypes.c_void_p),
        ("query_pairs", ctypes.c_void_p),
    ]


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python block_sparse_attention_28_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i32, _i64, _sz, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float

_lib.sta_num_tiles.argtypes = [Grid]
_lib.sta_num_tiles.restype = _i64
_lib.sta_tiled_len.argtypes = [Grid]
_lib.sta_tiled_len.restype = _i64
_lib.sta_reorder.argtypes = [_vp, _vp, _i32, _i32, _i32, Grid, _i32, _vp]
_lib.sta_reorder.restype = ctypes.c_int
_lib.sta_build_mask_workspace.argtypes = [_i32, _i32, _i32, Grid]
_lib.sta_build_mask_workspace.restype = _sz
_lib.sta_build_mask_workspace_min.argtypes = [_i32, _i32, _i32, Grid]
_lib.sta_build_mask_workspace_min.restype = _sz
_lib.sta_build_mask_pooled_offsets.argtypes = [_i32, _i32, _i32, Grid, _sz, ctypes.POINTER(_sz)]
_lib.sta_build_mask_pooled_offsets.restype = ctypes.c_int
_lib.sta_build_mask.argtypes = [_vp, _vp, _i32, _i32, _i32, Grid, ctypes.POINTER(MaskParams), _vp, _vp,
                                _vp, _vp, _vp, _vp, _sz, _vp]
_lib.sta_build_mask.restype = ctypes.c_int
_lib.sta_build_mask_noalloc.argtypes = [_vp, _vp, _i32, _i32, _i32, Grid, ctypes.POINTER(MaskParams), _vp,
                                        _vp, _vp, _vp, _vp, _vp]
_lib.sta_build_mask_noalloc.restype = ctypes.c_int
_lib.sta_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, Grid, _f32, _vp]
_lib.sta_attn_fwd.restype = ctypes.c_int
_lib.sta_build_mask_raster.argtypes = _lib.sta_build_mask.argtypes
_lib.sta_build_mask_raster.restype = ctypes.c_int
_lib.sta_attn_fwd_raster.argtypes = _lib.sta_attn_fwd.argtypes
_lib.sta_attn_fwd_raster.restype = ctypes.c_int
_lib.sta_attn_fwd_paired.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, Grid, _f32, _vp]
_lib.sta_attn_fwd_paired.restype = ctypes.c_int
_lib.sta_attn_fwd_raster_paired.argtypes = _lib.sta_attn_fwd_paired.argtypes
_lib.sta_attn_fwd_raster_paired.restype = ctypes.c_int
_lib.sta_rectified_workspace.argtypes = [_i32, _i32, _i32, Grid]
_lib.sta_rectified_workspace.restype = _sz
_lib.sta_attn_fwd_rectified.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i32, _i32, _i32, Grid,
                                        _f32, _vp]
_lib.sta_attn_fwd_rectified.restype = ctypes.c_int
_lib.sta_attn_fwd_block_mass.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, Grid,
                                         _f32, _vp]
_lib.sta_attn_fwd_block_mass.restype = ctypes.c_int
_lib.sta_search_windows.argtypes = [_vp, _i32, _i32, Grid, _i32, ctypes.POINTER(ctypes.c_int32), _f32, _f32,
                                    _vp, _vp, _vp]
_lib.sta_search_windows.restype = ctypes.c_int
_lib.sta_set_wait_limit.argtypes = [_i64]
_lib.sta_set_wait_limit.restype = ctypes.c_int
_lib.sta_get_wait_limit.argtypes = []
_lib.sta_get_wait_limit.restype = _i64
_lib.sta_selftest_wait_timeout.argtypes = [_i64, _vp]
_lib.sta_selftest_wait_timeout.restype = ctypes.c_int
_lib.sta_get_device_error.argtypes = [_vp]
_lib.sta_get_device_error.restype = ctypes.c_int
_lib.sta_validate_csr.argtypes = [_vp, _vp, _i64, _i32, _i32, Grid, _vp]
_lib.sta_validate_csr.restype = ctypes.c_int
_lib.sta_debug_build.argtypes = []
_lib.sta_debug_build.restype = _i32
_lib.sta_status_string.argtypes = [ctypes.c_int]
_lib.sta_status_string.restype = ctypes.c_char_p


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status, what):
    if status != STA_OK:
        raise StaError(status, what)


def grid(T, H, W):
    return Grid(int(T), int(H), int(W))


def sta_validate_csr(row_ptr, col_idx, B, heads, g, col_capacity=None, stream=None):
    """Checks a caller's CSR on the device (result in sta_get_device_error);
    col_capacity defaults to col_idx.numel()."""
    cap = col_idx.numel() if col_capacity is None else int(col_capacity)
    _check(_lib.sta_validate_csr(_ptr(row_ptr), _ptr(col_idx), cap, B, heads, g, _stream(stream)),
           "sta_validate_csr")


def sta_debug_build():
    return int(_lib.sta_debug_build())


def sta_status_string(status):
    return _lib.sta_status_string(int(status)).decode()


def sta_num_tiles(g):
    return int(_lib.sta_num_tiles(g))


def sta_tiled_len(g):
    return int(_lib.sta_tiled_len(g))


def sta_reorder(src, dst, B, heads, d, g, inverse=False, stream=None):
    _check(_lib.sta_reorder(_ptr(src), _ptr(dst), B, heads, d, g, 1 if inverse else 0, _stream(stream)),
           "sta_reorder")


def sta_build_mask_workspace(B, heads, d, g):
    return int(_lib.sta_build_mask_workspace(B, heads, d, g))


def sta_build_mask_workspace_min(B, heads, d, g):
    return int(_lib.sta_build_mask_workspace_min(B, heads, d, g))


def mask_params(top_p=0.0, k_min=0, use_scores=False, sm_scale=0.0, group_lo=(0,), windows=None,
                head_floor=False, block_scores=None, query_pairs=None):
    """MaskParams; `windows` is a device int32 tensor [heads, G, 4] or None;
    `head_floor` turns on the per-head top-k floor of the selection;
    `block_scores` (device fp32 [B, heads, Nt, Nt]) replaces the pooled scores;
    `query_pairs` (device int32 [B*heads, 2*ceil(Nt/2)]) receives the
    overlap pairing of the query tiles for sta_attn_fwd_paired."""
    p = MaskParams()
    p.query_pairs = _ptr(query_pairs)
    p.head_topk_floor = 1 if head_floor else 0
    p.block_scores = _ptr(block_scores)
    p.top_p = float(top_p)
    p.k_min = int(k_min)
    p.use_scores = 1 if use_scores else 0
    p.sm_scale = float(sm_scale)
    p.num_groups = len(group_lo)
    for i, v in enumerate(group_lo):
        p.group_lo[i] = int(v)
    p.windows = _ptr(windows)
    # the struct holds raw device pointers: keep the tensors alive with it
    p._keep = (windows, block_scores, query_pairs)
    return p


def sta_build_mask_pooled_offsets(B, heads, d, g, ws_bytes):
    """(qbar, kbar, qlo, klo) byte offsets of the pooled means in a mask-build
    workspace of ws_bytes; qlo / klo are 0 when the means are not split."""
    out = (_sz * 4)()
    _check(_lib.sta_build_mask_pooled_offsets(B, heads, d, g, int(ws_bytes), out), "sta_build_mask_pooled_offsets")
    return tuple(int(x) for x in out)


def sta_build_mask(q_tiled, k_tiled, B, heads, d, g, params, row_ptr, col_idx, nnz_dev,
                   block_mask=None, block_probs=None, workspace=None, ws_bytes=0, stream=None):
    _check(_lib.sta_build_mask(_ptr(q_tiled), _ptr(k_tiled), B, heads, d, g, ctypes.byref(params),
                               _ptr(row_ptr), _ptr(col_idx), _ptr(nnz_dev), _ptr(block_mask),
                               _ptr(block_probs), _ptr(workspace), int(ws_bytes), _stream(stream)),
           "sta_build_mask")


# bytes of the static device array behind sta_build_mask_noalloc (the
# header's STA_NOALLOC_SCRATCH_BYTES)
STA_NOALLOC_SCRATCH_BYTES = 32 << 20


def sta_build_mask_noalloc(q_tiled, k_tiled, B, heads, d, g, params, row_ptr, col_idx, nnz_dev,
                           block_mask=None, block_probs=None, stream=None):
    """sta_build_mask without a workspace argument, for callers that cannot
    allocate device memory: the library's static 32 MiB device array serves as
    the workspace, so the results are those of sta_build_mask with a workspace
    of that size (see include/sta.h for the size limit and sharing rules)."""
    _check(_lib.sta_build_mask_noalloc(_ptr(q_tiled), _ptr(k_tiled), B, heads, d, g, ctypes.byref(params),
                                       _ptr(row_ptr), _ptr(col_idx), _ptr(nnz_dev), _ptr(block_mask),
                                       _ptr(block_probs), _stream(stream)),
           "sta_build_mask_noalloc")


def sta_attn_fwd(q, k, v, o, lse, row_ptr, col_idx, B, heads, d, g, sm_scale=0.0, stream=None):
    _check(_lib.sta_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(row_ptr), _ptr(col_idx),
                             B, heads, d, g, float(sm_scale), _stream(stream)),
           "sta_attn_fwd")


def sta_attn_fwd_paired(q, k, v, o, lse, row_ptr, col_idx, query_pairs, B, heads, d, g, sm_scale=0.0,
                        stream=None):
    """sta_attn_fwd with the caller's pairing of query tiles."""
    _check(_lib.sta_attn_fwd_paired(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(row_ptr), _ptr(col_idx),
                                    _ptr(query_pairs), B, heads, d, g, float(sm_scale), _stream(stream)),
           "sta_attn_fwd_paired")


def sta_attn_fwd_raster_paired(q, k, v, o, lse, row_ptr, col_idx, query_pairs, B, heads, d, g, sm_scale=0.0,
                               stream=None):
    """sta_attn_fwd_raster with the caller's pairing of query tiles."""
    _check(_lib.sta_attn_fwd_raster_paired(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(row_ptr),
                                           _ptr(col_idx), _ptr(query_pairs), B, heads, d, g, float(sm_scale),
                                           _stream(stream)),
           "sta_attn_fwd_raster_paired")


def sta_build_mask_raster(q, k, B, heads, d, g, params, row_ptr, col_idx, nnz_dev, block_mask=None,
                          block_probs=None, workspace=None, ws_bytes=0, stream=None):
    """sta_build_mask on raster [B, L, heads, d] Q and K."""
    _check(_lib.sta_build_mask_raster(_ptr(q), _ptr(k), B, heads, d, g, ctypes.byref(params), _ptr(row_ptr),
                                      _ptr(col_idx), _ptr(nnz_dev), _ptr(block_mask), _ptr(block_probs),
                                      _ptr(workspace), int(ws_bytes), _stream(stream)),
           "sta_build_mask_raster")


def sta_attn_fwd_raster(q, k, v, o, lse, row_ptr, col_idx, B, heads, d, g, sm_scale=0.0, stream=None):
    """sta_attn_fwd on raster [B, L, heads, d] Q, K, V and O (LSE tiled-indexed)."""
    _check(_lib.sta_attn_fwd_raster(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(row_ptr),
                                    _ptr(col_idx), B, heads, d, g, float(sm_scale), _stream(stream)),
           "sta_attn_fwd_raster")


def sta_rectified_workspace(B, heads, d, g):
    return int(_lib.sta_rectified_workspace(B, heads, d, g))


def sta_attn_fwd_rectified(q, k, v, o, lse, row_ptr, col_idx, workspace, ws_bytes, B, heads, d, g,
                           sm_scale=0.0, stream=None):
    """Rectified attention: unlisted tiles enter as pooled keys / values."""
    _check(_lib.sta_attn_fwd_rectified(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(row_ptr),
                                       _ptr(col_idx), _ptr(workspace), int(ws_bytes), B, heads, d, g,
                                       float(sm_scale), _stream(stream)),
           "sta_attn_fwd_rectified")


def sta_attn_fwd_block_mass(q, k, v, o, lse, row_ptr, col_idx, lse_cached, block_mass, B, heads, d, g,
                            sm_scale=0.0, stream=None):
    _check(_lib.sta_attn_fwd_block_mass(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(row_ptr),
                                        _ptr(col_idx), _ptr(lse_cached), _ptr(block_mass), B, heads, d, g,
                                        float(sm_scale), _stream(stream)),
           "sta_attn_fwd_block_mass")


def sta_search_windows(block_mass, B, heads, g, group_lo, tau, lam, windows, stats=None, stream=None):
    lo = (ctypes.c_int32 * len(group_lo))(*[int(v) for v in group_lo])
    _check(_lib.sta_search_windows(_ptr(block_mass), B, heads, g, len(group_lo), lo, float(tau), float(lam),
                                   _ptr(windows), _ptr(stats), _stream(stream)),
           "sta_search_windows")


def sta_set_wait_limit(limit_cycles):
    _check(_lib.sta_set_wait_limit(int(limit_cycles)), "sta_set_wait_limit")


def sta_get_wait_limit():
    return int(_lib.sta_get_wait_limit())


def sta_selftest_wait_timeout(limit_cycles=2000000, stream=None):
    _check(_lib.sta_selftest_wait_timeout(int(limit_cycles), _stream(stream)), "sta_selftest_wait_timeout")


def sta_get_device_error(stream=None):
    return int(_lib.sta_get_device_error(_stream(stream)))


# ------------------------------------------------------------ allocation helpers
class MaskBuffers:
    """Device buffers for one sta_build_mask call (torch allocations)."""

    def __init__(self, B, heads, d, g, device="cuda", with_mask=False, with_probs=False):
        nt = sta_num_tiles(g)
        R = B * heads * nt
        self.row_ptr = torch.empty(R + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(max(1, R * nt), dtype=torch.int32, device=device)
        self.nnz = torch.zeros(1, dtype=torch.int64, device=device)
        self.block_mask = torch.empty((B, heads, nt, nt), dtype=torch.uint8, device=device) if with_mask else None
        self.block_probs = torch.empty((B, heads, nt, nt), dtype=torch.float32, device=device) if with_probs else None
        self.ws_bytes = sta_build_mask_workspace(B, heads, d, g)
        self.workspace = torch.empty(max(1, self.ws_bytes), dtype=torch.uint8, device=device)


def build_mask(q_tiled, k_tiled, B, heads, d, g, params, bufs, stream=None, raster=False):
    fn = sta_build_mask_raster if raster else sta_build_mask
    fn(q_tiled, k_tiled, B, heads, d, g, params, bufs.row_ptr, bufs.col_idx, bufs.nnz,
       bufs.block_mask, bufs.block_probs, bufs.workspace, bufs.ws_bytes, stream)
    return bufs
