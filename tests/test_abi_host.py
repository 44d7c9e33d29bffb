"""CPU checks of the C-ABI library: it loads, exports every function that
include/tra.h declares, validates arguments, and its host-side plan logic
(tile shape, padding, r_cap, mask layout) matches independent computations.
No CUDA compute call is made here."""
import ctypes
import math
import os
import re

import pytest

import oracle
import sparse_attention_video_tra_b200 as tra
from sparse_attention_video_tra_b200 import build as trabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tra.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    trabuild.build()
    yield


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^TRA_API\s+[\w\s\*]+?\b(tra_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"tra_plan_create", "tra_plan_destroy", "tra_plan_query", "tra_permute", "tra_entropy",
            "tra_radius_and_mask", "tra_attention", "tra_calibrate_topk", "tra_calibrate_fit",
            "tra_plan_status", "tra_status_string"} <= names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(tra.library_path())
    for name in declared_functions():
        assert hasattr(lib, name), name
    # and the binding loads it
    assert tra.load_library() is not None


def test_status_strings():
    for s in range(7):
        assert isinstance(tra.tra_status_string(s), str) and tra.tra_status_string(s)


@pytest.mark.parametrize("args,status", [
    ((0, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 8), 1),        # T < 1
    ((4, 8, 8, 0, 64, 1.0, 0.0, 0.7, 2, 8), 1),        # heads < 1
    ((4, 8, 8, 2, 64, 1.0, 0.0, 0.0, 2, 8), 1),        # gamma <= 0
    ((4, 8, 8, 2, 64, 1.0, 0.0, 1.5, 2, 8), 1),        # gamma > 1
    ((4, 8, 8, 2, 64, 1.0, 0.0, 0.7, -1, 8), 1),       # Rt < 0
    ((4, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 0), 1),        # Bmin < 1
    ((4, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 257), 1),      # Bmin > N
    ((4, 8, 8, 2, 64, float("nan"), 0.0, 0.7, 2, 8), 1),
    ((4, 8, 8, 2, 96, 1.0, 0.0, 0.7, 2, 8), 2),        # d not 64/128
    ((40, 8, 8, 2, 64, 1.0, 0.0, 0.7, 35, 8), 2),      # Rt' > 31
    ((4, 8, 2000, 2, 64, 1.0, 0.0, 0.7, 2, 8), 2),     # > 32 tile columns for every tile width
    ((10, 8, 8, 2, 64, 1.0, 0.0, 0.01, 9, 8), 2),      # r_cap beyond 2^20
])
def test_plan_create_rejects(args, status):
    with pytest.raises(tra.TraError) as e:
        tra.tra_plan_create(*args)
    assert e.value.status == status


def test_natural_layout_flag():
    """TRA_FLAG_NATURAL: q/k/v/out/entropies hold N rows per head in natural
    token order; unknown flag bits are still rejected."""
    p = tra.Plan(4, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 8, flags=tra.TRA_FLAG_NATURAL)
    assert p.natural and p.io_rows == p.info.N == 256
    q = tra.Plan(4, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 8)
    assert not q.natural and q.io_rows == q.info.N_pad
    assert p.info == q.info                      # same geometry and mask layout
    with pytest.raises(tra.TraError):
        tra.tra_plan_create(4, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 8, flags=1 << 21)   # no such flag


@pytest.mark.parametrize("grid,gamma,Rt", [((21, 45, 80), 0.8, 6), ((4, 8, 8), 0.7, 2), ((3, 7, 9), 0.5, 1),
                                           ((132, 45, 80), 0.7, 16), ((2, 256, 256), 0.9, 1)])
def test_disk_flag_r_cap_matches_oracle(grid, gamma, Rt):
    """TRA_FLAG_DISK: r_cap is the smallest r whose farthest-frame disk reaches
    the opposite frame corner, as the oracle's metric-1 definition."""
    T, H, W = grid
    p = tra.Plan(T, H, W, 1, 128, 1.0, 0.0, gamma, Rt, 8, flags=tra.TRA_FLAG_DISK)
    assert p.info.r_cap == oracle.r_cap(T, H, W, gamma, Rt, oracle.DISK)
    q = tra.Plan(T, H, W, 1, 128, 1.0, 0.0, gamma, Rt, 8)
    assert p.info.r_cap >= q.info.r_cap


def test_plan_create_rejects_bad_flags():
    with pytest.raises(tra.TraError) as e:
        tra.tra_plan_create(4, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 8, flags=1 << 3)
    assert e.value.status == 1
    with pytest.raises(tra.TraError) as e:
        tra.tra_plan_create(4, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 8, flags=tra.tra_flag_tile_w(5))
    assert e.value.status == 1


def least_padding_tile(H, W):
    best = None
    for tw in (4, 8, 16, 32):
        th = 128 // tw
        nTh, nTw = -(-H // th), -(-W // tw)
        if nTw > 32 or nTh > 64:
            continue
        # least padding; a tie goes to the tile whose long side runs along
        # the frame's short side (the taller tile when H <= W)
        key = (nTh * nTw, tw if H <= W else -tw)
        if best is None or key < best[0]:
            best = (key, th, tw)
    return best[1], best[2]


@pytest.mark.parametrize("grid", [(4, 8, 8), (21, 30, 52), (21, 45, 80), (33, 45, 80), (132, 45, 80),
                                  (3, 7, 9), (5, 17, 23), (2, 1, 1), (1, 100, 3)])
@pytest.mark.parametrize("gamma,Rt", [(0.7, 2), (0.8, 6), (0.7, 16), (1.0, 0)])
def test_plan_geometry(grid, gamma, Rt):
    T, H, W = grid
    p = tra.Plan(T, H, W, 3, 128, 1.0, 0.0, gamma, Rt, 1)
    i = p.info
    th, tw = least_padding_tile(H, W)
    assert (i.tile_h, i.tile_w) == (th, tw) and th * tw == 128
    assert i.n_tiles_h == -(-H // th) and i.n_tiles_w == -(-W // tw)
    assert i.n_tiles == T * i.n_tiles_h * i.n_tiles_w and i.N_pad == 128 * i.n_tiles
    assert i.N == T * H * W
    assert i.rt_eff == min(Rt, T - 1)
    assert i.r_cap == oracle.r_cap(T, H, W, gamma, Rt)
    assert i.list_cap == (2 * i.rt_eff + 1) * i.n_tiles_h * i.n_tiles_w
    # mask layout: 256-aligned, in order, non-overlapping, inside mask_bytes
    offs = [i.off_radius, i.off_tile_count, i.off_tile_pairs, i.off_list]
    sizes = [4 * 3 * i.N_pad, 4 * 3 * i.n_tiles, 8 * 3 * i.n_tiles, 2 * 3 * i.n_tiles * i.list_cap]
    for o in offs:
        assert o % 256 == 0
    for k in range(3):
        assert offs[k] + sizes[k] <= offs[k + 1]
    assert offs[3] + sizes[3] <= i.mask_bytes
    p.close()


def test_forced_tile_width():
    p = tra.Plan(21, 45, 80, 1, 128, 1.0, 0.0, 0.8, 6, 8, flags=tra.tra_flag_tile_w(8))
    assert (p.info.tile_h, p.info.tile_w) == (16, 8)


def test_workload_tiles_match_the_documented_choice():
    # least padding first; on a tie the tile's long side runs along the
    # frame's short side.  tiny: (1,16,8) padded x2 (ties with (1,8,16));
    # Wan-480p: (1,32,4) x1.067; 720p: (1,16,8) x1.067 (ties with (1,8,16))
    assert tra.Plan(4, 8, 8, 2, 64, 1.0, 0.0, 0.7, 2, 8).info.tile_w == 8
    wan480 = tra.Plan(21, 30, 52, 12, 128, 1.0, 0.0, 0.8, 6, 8).info
    assert (wan480.tile_h, wan480.tile_w) == (32, 4)
    assert math.isclose(wan480.N_pad / wan480.N, 1664 / 1560)
    wan720 = tra.Plan(21, 45, 80, 40, 128, 1.0, 0.0, 0.8, 6, 8).info
    assert (wan720.tile_h, wan720.tile_w) == (16, 8) and wan720.N_pad == 21 * 3840
    # a portrait frame with the same tie takes the wider tile
    portrait = tra.Plan(2, 80, 45, 1, 128, 1.0, 0.0, 0.8, 1, 8).info
    assert (portrait.tile_h, portrait.tile_w) == (8, 16) and portrait.N_pad == 2 * 3840


def test_qsort_needs_at_most_four_tile_rows():
    # (1,16,8) tiles at 45x80: 3 tile rows, accepted, with a uint16 group section
    p = tra.Plan(21, 45, 80, 2, 128, 1.0, 0.0, 0.8, 6, 8, flags=tra.TRA_FLAG_QSORT)
    i = p.info
    assert i.off_group % 256 == 0 and i.off_group >= i.off_list + 2 * i.heads * i.n_tiles * i.list_cap
    assert i.mask_bytes >= i.off_group + 2 * i.heads * i.n_tiles * 128
    assert tra.Plan(21, 45, 80, 2, 128, 1.0, 0.0, 0.8, 6, 8).info.off_group == 0
    # (1,32,4) tiles at 30x52: one tile row, accepted (the groups are the tiles)
    tra.Plan(21, 30, 52, 2, 128, 1.0, 0.0, 0.8, 6, 8, flags=tra.TRA_FLAG_QSORT).close()
    # 200 rows: 13 tile rows of 16, rejected
    with pytest.raises(tra.TraError) as e:
        tra.tra_plan_create(2, 200, 200, 2, 128, 1.0, 0.0, 0.8, 1, 8, flags=tra.TRA_FLAG_QSORT)
    assert e.value.status == 2
