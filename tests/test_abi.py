"""C-ABI boundary checks that need no GPU: the library builds, loads and
exports every function include/km.h declares; workspace sizing is linear in
N and K*D (never N*K); invalid shapes are rejected before any launch."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

import means_clustering_flashassign_b200 as km

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "km.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(km_[a-z_]+)\s*\(", src)))


def test_library_loads_and_exports_header_symbols():
    L = km.library()
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), f"{n} declared in km.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", km.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (km_\w+)", out))
    assert set(names) == exported, (set(names) ^ exported)
    assert set(km.EXPORTS) == set(names)
    assert L.km_version() == 1


def test_status_strings():
    L = km.library()
    for code in range(7):
        assert L.km_status_string(code) != b"unknown status"
    assert L.km_status_string(6) == b"injected fault"
    assert L.km_status_string(99) == b"unknown status"
    assert km.STATUS[6] == "KM_ERR_INJECTED"


@pytest.mark.parametrize("spec", ["launch", "launch:3", "h2d:2", "alloc", "bogus", "launch:0", ""])
def test_fault_spec_does_not_change_host_side_refusals(monkeypatch, spec):
    """KM_FAULT only acts on device work: argument checks still come first,
    so an invalid call is refused with its own code whatever the spec."""
    monkeypatch.setenv("KM_FAULT", spec)
    L = km.library()
    assert L.km_fit(None, None, 1, 100, 64, 10, 1, 3, None, None, None, None, None, 0, None) == 1
    assert L.km_workspace_size(km.OP_FIT, 1, 100, 12, 10, km.BF16, 0) == 0


@pytest.mark.parametrize("op", [km.OP_ASSIGN, km.OP_UPDATE, km.OP_FIT])
def test_workspace_is_linear_not_nk(op):
    # doubling N at fixed K grows the workspace by at most ~2x; doubling K at
    # fixed N grows it by O(K*D), not by N*K
    a = km.workspace_size(op, 1, 1 << 20, 128, 1024, km.BF16)
    b = km.workspace_size(op, 1, 1 << 21, 128, 1024, km.BF16)
    c = km.workspace_size(op, 1, 1 << 20, 128, 4096, km.BF16)
    assert b < 2.2 * a
    assert c - a < 64 * (4096 - 1024) * 128 + (1 << 22)
    # an N x K fp32 score matrix would be 4 GiB here
    assert a < (1 << 20) * 1024 * 4 / 50


def test_workspace_host_stream_scales_with_chunk():
    w1 = km.workspace_size(km.OP_FIT_HOST, 1, 1 << 28, 128, 4096, km.BF16, 1 << 20)
    w2 = km.workspace_size(km.OP_FIT_HOST, 1, 1 << 28, 128, 4096, km.BF16, 1 << 21)
    # two chunk buffers of chunk_rows * D * 2 bytes dominate the growth
    assert abs((w2 - w1) - 2 * (1 << 20) * 128 * 2) < 0.5 * 2 * (1 << 20) * 128 * 2


@pytest.mark.parametrize("args", [
    (km.OP_FIT, 1, 100, 128, 200, km.BF16),   # K > N
    (km.OP_FIT, 1, 1000, 12, 10, km.BF16),    # D not a multiple of 8
    (km.OP_FIT, 1, 1000, 512, 10, km.BF16),   # D too large
    (km.OP_FIT, 1, 1000, 128, 10, km.F32),    # f32 D too large
    (km.OP_FIT, 0, 1000, 64, 10, km.BF16),    # B < 1
    (km.OP_FIT, 1, 1000, 64, 0, km.BF16),     # K < 1
    (7, 1, 1000, 64, 10, km.BF16),            # unknown op
    (km.OP_FIT, 1, 1000, 64, 10, 5),          # unknown dtype
])
def test_invalid_shapes_rejected(args):
    L = km.library()
    assert L.km_workspace_size(*args, 0) == 0
    assert L.km_last_error()


def test_calls_without_gpu_fail_cleanly():
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    L = km.library()
    ws = (ctypes.c_uint8 * 4096)()
    st = L.km_selftest_timeout(ctypes.cast(ws, ctypes.c_void_p), 4096, 1000, None)
    assert st == 3  # KM_ERR_CUDA: no device
    assert b"cuda" in L.km_last_error().lower() or b"device" in L.km_last_error().lower()


def test_null_arguments_rejected_before_device_use():
    L = km.library()
    assert L.km_assign(None, None, 1, 100, 64, 10, 1, None, None, None, None, 0, None) == 1
    assert L.km_update(None, None, 1, 100, 64, 10, 1, None, None, None, 0, None) == 1
    assert L.km_fit(None, None, 1, 100, 64, 10, 1, 3, None, None, None, None, None, 0, None) == 1
    assert L.km_argsort(None, 100, 10, None, None, None, 0, None) == 1


def test_plan_describes_the_chosen_tiling():
    # CTA pairs with 256-wide centroid tiles at D=128; two point buffers and
    # four centroid stages for K > BN; one CTA per point tile with a 4 x 3
    # ring when one tile covers K and that ring fits, else pairs
    p = km.plan(km.OP_FIT, 1, 1 << 20, 128, 1024, km.BF16)
    assert (p["pair"], p["BN"], p["XB"], p["CS"], p["Kp"], p["sort_passes"]) == (1, 256, 2, 4, 1024, 1)
    assert p["smem"] <= 232448
    q = km.plan(km.OP_FIT, 512, 4096, 64, 256, km.BF16)
    assert (q["pair"], q["BN"], q["XB"], q["CS"], q["Kp"]) == (0, 256, 4, 3, 256)
    q2 = km.plan(km.OP_FIT, 1, 100000, 128, 200, km.BF16)
    assert (q2["pair"], q2["BN"], q2["Kp"]) == (1, 256, 256)
    r = km.plan(km.OP_FIT, 1, 16384, 32, 64, km.F32)
    assert (r["pair"], r["BN"]) == (0, 64)  # pairs need 128-wide tiles
    assert km.plan(km.OP_FIT, 1, 1 << 22, 128, 16384, km.BF16)["sort_passes"] == 2
    # the update's form: the fused one-CTA-per-instance kernel for batched
    # problems (N <= 8192, K <= 1024), else the sort chain
    assert q["update_form"] == 1 and p["update_form"] == 0 and r["update_form"] == 0
    assert km.plan(km.OP_UPDATE, 2, 8192, 256, 1024, km.BF16)["update_form"] == 1
    assert km.plan(km.OP_UPDATE, 2, 8193, 64, 256, km.BF16)["update_form"] == 0
    assert km.plan(km.OP_UPDATE, 2, 4096, 64, 1025, km.BF16)["update_form"] == 0
    assert km.plan(km.OP_UPDATE, 1, 4096, 64, 256, km.BF16)["update_form"] == 0


@pytest.mark.parametrize("N,block", [(16384, 2048), (147 * 4096, 2048), (147 * 4096 + 1, 4096), (1 << 20, 4096),
                                     (296 * 4096, 4096), (296 * 4096 + 1, 2048), (1 << 22, 2048)])
def test_sort_block_fills_one_wave(N, block):
    # 4096-key scatter blocks only when they fill the 148 SMs with one to two
    # resident blocks each; 2048-key blocks (4 per SM) otherwise
    assert km.plan(km.OP_FIT, 1, N, 128, 1024, km.BF16)["sort_block"] == block


@pytest.mark.parametrize("tile,ok", [("0,256,2,2", True), ("1,128,3,3", True), ("1,64,2,2", False),
                                     ("0,256,8,4", False), ("0,256,9,2", False), ("junk", False)])
def test_tiling_override_is_validated(monkeypatch, tile, ok):
    monkeypatch.setenv("KM_ASSIGN_TILE", tile)
    if ok:
        p = km.plan(km.OP_FIT, 1, 1 << 20, 128, 1024, km.BF16)
        assert f'{p["pair"]},{p["BN"]},{p["XB"]},{p["CS"]}' == tile
    else:
        with pytest.raises(km.KMError):
            km.plan(km.OP_FIT, 1, 1 << 20, 128, 1024, km.BF16)


def test_baseline_workspaces():
    assert km.library().km_ablation_workspace_size(0, 1 << 20, 128, 1024, km.BF16, 1 << 18) >= (1 << 18) * 1024 * 4
    assert km.library().km_ablation_workspace_size(1, 1 << 20, 128, 1024, km.BF16, 0) >= 1024 * 128 * 4
    assert km.library().km_ablation_workspace_size(0, 1 << 20, 128, 1024, km.BF16, 0) == 0  # chunk_rows must be >= 1
