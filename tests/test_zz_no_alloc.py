"""sta_build_mask_noalloc: the mask build for callers that cannot allocate.

Some callers cannot call cudaMalloc or lend a workspace, because a host
framework or a fixed arena owns every device allocation of the process. For
them the library keeps a static 32 MiB device array as the workspace of the
mask build. These tests call that entry point through the C ABI and check
that, on two calls in a row (the array keeps the previous call's contents),
its outputs equal those of sta_build_mask with a caller-owned workspace of
the array's size, bit for bit. This file is collected last
and builds its own inputs, so it runs the same alone in a fresh process.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sta():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import block_sparse_attention_28_b200 as mod

    return mod


def _inputs(sta, T, H, W, heads, d, B, seed):
    g = sta.grid(T, H, W)
    lpad = sta.sta_tiled_len(g)
    gen = torch.Generator(device="cuda").manual_seed(seed)
    raster = [(torch.randn(B, T * H * W, heads, d, generator=gen, device="cuda") * 3).to(torch.bfloat16)
              for _ in range(2)]
    tiled = []
    for x in raster:
        t = torch.empty(B, heads, lpad, d, dtype=torch.bfloat16, device="cuda")
        sta.sta_reorder(x, t, B, heads, d, g)
        tiled.append(t)
    rng = np.random.default_rng(seed)
    win = torch.from_numpy(rng.integers(-1, 3, size=(heads, 3, 4)).astype(np.int32)).cuda()
    return g, tiled[0], tiled[1], win


def _outputs(sta, B, heads, g):
    nt = sta.sta_num_tiles(g)
    R = B * heads * nt
    return dict(
        row_ptr=torch.full((R + 1,), -7, dtype=torch.int32, device="cuda"),
        col_idx=torch.full((R * nt,), -7, dtype=torch.int32, device="cuda"),
        nnz=torch.full((1,), -7, dtype=torch.int64, device="cuda"),
        mask=torch.full((B, heads, nt, nt), 7, dtype=torch.uint8, device="cuda"),
        probs=torch.full((B, heads, nt, nt), float("nan"), dtype=torch.float32, device="cuda"),
    )


def _same(a, b):
    n = int(a["nnz"].item())
    assert n == int(b["nnz"].item())
    assert torch.equal(a["row_ptr"], b["row_ptr"])
    assert torch.equal(a["col_idx"][:n], b["col_idx"][:n])
    assert torch.equal(a["mask"], b["mask"])
    assert torch.equal(a["probs"].view(torch.int32), b["probs"].view(torch.int32))


def test_noalloc_matches_workspace_path_on_two_calls(sta):
    # two different problems in a row: the second call finds the first one's
    # data in the shared array and must not depend on it
    cases = [dict(T=3, H=19, W=37, heads=3, d=128, B=2, seed=1, top_p=0.7, k_min=3, scores=True),
             dict(T=4, H=16, W=24, heads=2, d=64, B=1, seed=2, top_p=0.9, k_min=1, scores=True)]
    for c in cases:
        g, qt, kt, win = _inputs(sta, c["T"], c["H"], c["W"], c["heads"], c["d"], c["B"], c["seed"])
        params = sta.mask_params(c["top_p"], c["k_min"], c["scores"], 0.0, (0, 1, 3), win)
        ref = _outputs(sta, c["B"], c["heads"], g)
        # the call is sta_build_mask on a workspace the size of the static
        # array (the tensor-core layout when the full workspace fits in it)
        ws_bytes = sta.STA_NOALLOC_SCRATCH_BYTES
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        sta.sta_build_mask(qt, kt, c["B"], c["heads"], c["d"], g, params, ref["row_ptr"], ref["col_idx"],
                           ref["nnz"], ref["mask"], ref["probs"], ws, ws_bytes)
        got = _outputs(sta, c["B"], c["heads"], g)
        sta.sta_build_mask_noalloc(qt, kt, c["B"], c["heads"], c["d"], g, params, got["row_ptr"],
                                   got["col_idx"], got["nnz"], got["mask"], got["probs"])
        torch.cuda.synchronize()
        assert sta.sta_get_device_error() == sta.STA_OK
        _same(ref, got)


def test_noalloc_rejects_sizes_beyond_the_array(sta):
    # 40 heads of the 21x45x80 layer need ~60 MB of workspace: refused up
    # front, before any launch. Every device pointer is NULL, so were the size
    # check to regress the call would stop at the argument checks
    # (STA_ERR_INVALID_ARG) instead of launching.
    g = sta.grid(21, 45, 80)
    assert sta.sta_build_mask_workspace_min(1, 40, 128, g) > (32 << 20)
    params = sta.mask_params(0.95, 8, True)
    status = sta._lib.sta_build_mask_noalloc(None, None, 1, 40, 128, g, sta.ctypes.byref(params), None, None,
                                             None, None, None, None)
    assert status == sta.STA_ERR_WORKSPACE
    # 40 heads of the 21x30x52 layer fit
    assert sta.sta_build_mask_workspace_min(1, 40, 128, sta.grid(21, 30, 52)) <= (32 << 20)
