"""Plain fp64 CPU oracle for the Token Radius Attention hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the product package.
It shares no code with the CUDA path.  The arithmetic lives in
``tra_oracle.c`` (compiled with gcc, fp64, OpenMP over queries); this module
only compiles it and marshals numpy arrays.

Every function works on the natural (frame-major) token order
n = (t*H + h)*W + w of the "Token Radius Attention" blog post, sections 5.1
and 9.1, with per-head arrays laid out [heads][N][...].

Parity status of each function (what pins it) is listed in the repository's
design notes; every function here is pinned by a CPU test.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tra_oracle.c")
_OUT = os.path.join(_HERE, "_build", "libtra_oracle.so")
# A prebuilt oracle library to load instead (the mutation tests point this at
# copies of tra_oracle.c with a planted mistake).
_OVERRIDE = os.environ.get("TRA_ORACLE_LIB")
_lib = None

_I64P = ctypes.POINTER(ctypes.c_int64)
_I32P = ctypes.POINTER(ctypes.c_int32)
_F32P = ctypes.POINTER(ctypes.c_float)
_F64P = ctypes.POINTER(ctypes.c_double)
_U8P = ctypes.POINTER(ctypes.c_uint8)


def compile_source(src: str, out: str) -> str:
    """gcc the oracle's C source `src` into the shared library `out`."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-std=gnu11", "-Wall", "-shared", "-fPIC", "-o", tmp, src, "-lquadmath", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile tra_oracle.c into oracle/_build/libtra_oracle.so."""
    if _OVERRIDE:
        return _OVERRIDE
    if not force and os.path.exists(_OUT) and os.path.getmtime(_OUT) >= os.path.getmtime(_SRC):
        return _OUT
    os.makedirs(os.path.dirname(_OUT), exist_ok=True)
    return compile_source(_SRC, _OUT)


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.oracle_decay_table.argtypes = [ctypes.c_double, ctypes.c_int, _F64P]
        L.oracle_halfwidth.argtypes = [ctypes.c_int64, ctypes.c_double]
        L.oracle_halfwidth.restype = ctypes.c_int64
        L.oracle_rt_eff.argtypes = [ctypes.c_int, ctypes.c_int]
        L.oracle_rt_eff.restype = ctypes.c_int
        L.oracle_r_cap.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int]
        L.oracle_r_cap.restype = ctypes.c_int64
        L.oracle_count.argtypes = [ctypes.c_int] * 3 + [ctypes.c_double, ctypes.c_int] + [ctypes.c_int] * 3 + \
            [ctypes.c_int64, ctypes.c_int]
        L.oracle_count.restype = ctypes.c_int64
        L.oracle_budget.argtypes = [ctypes.c_float, ctypes.c_double, ctypes.c_double, ctypes.c_int64, ctypes.c_int64]
        L.oracle_budget.restype = ctypes.c_int64
        L.oracle_radius.argtypes = [_F32P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_double, ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, _I64P, ctypes.c_int64, _I32P, _I64P, _I64P]
        L.oracle_token_mask.argtypes = [ctypes.c_int] * 3 + [ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                                             ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
        L.oracle_token_mask.restype = ctypes.c_int
        L.oracle_block_mask.argtypes = [_I32P] + [ctypes.c_int] * 4 + [ctypes.c_double, ctypes.c_int, ctypes.c_int] + \
            [ctypes.c_int] * 4 + [_I64P, ctypes.c_int64, _U8P]
        L.oracle_block_mask_sets.argtypes = [_I32P] + [ctypes.c_int] * 4 + [ctypes.c_double, ctypes.c_int, ctypes.c_int] + \
            [ctypes.c_int] * 2 + [_I64P, ctypes.c_int64, ctypes.c_int, _U8P]
        L.oracle_entropy.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int] + [ctypes.c_int] * 5 + \
            [ctypes.c_int] * 3 + [_I64P, ctypes.c_int64, _F64P]
        L.oracle_attention.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, _I32P] + [ctypes.c_int] * 5 + \
            [ctypes.c_double, ctypes.c_int, ctypes.c_int, _I64P, ctypes.c_int64, _F64P]
        L.oracle_topk_count.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int] + [ctypes.c_int] * 5 + \
            [ctypes.c_double, _I64P, ctypes.c_int64, _I64P]
        L.oracle_fit_log_linear.argtypes = [_F64P, _I64P, ctypes.c_int64, _F64P, _F64P, _F64P]
        L.oracle_fit_log_linear.restype = ctypes.c_int64
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _elems(x: np.ndarray):
    """(contiguous array, type flag) for the C side: 0 f32, 1 bf16 bits, 2 f64."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, 0
    if x.dtype == np.uint16:
        return x, 1
    if x.dtype == np.float64:
        return x, 2
    raise TypeError(f"oracle takes float32, float64 or bf16 bits (uint16), got {x.dtype}")


def _qlist(queries):
    if queries is None:
        return None, 0, None
    q = np.ascontiguousarray(np.asarray(queries, dtype=np.int64))
    return q, q.size, _ptr(q, _I64P)


# ----------------------------------------------------------------- scalars
def decay_table(gamma: float, rt_eff: int) -> np.ndarray:
    g = np.zeros(rt_eff + 1, dtype=np.float64)
    lib().oracle_decay_table(gamma, rt_eff, _ptr(g, _F64P))
    return g


def halfwidth(r: int, g: float) -> int:
    return int(lib().oracle_halfwidth(r, g))


def rt_eff(T: int, Rt: int) -> int:
    return int(lib().oracle_rt_eff(T, Rt))


# metric: 0 = Chebyshev square (the default reading), 1 = Euclidean disk
CHEBYSHEV, DISK = 0, 1


def r_cap(T: int, H: int, W: int, gamma: float, Rt: int, metric: int = CHEBYSHEV) -> int:
    return int(lib().oracle_r_cap(T, H, W, gamma, Rt, metric))


def count(T, H, W, gamma, Rt, t, h, w, r, metric: int = CHEBYSHEV) -> int:
    return int(lib().oracle_count(T, H, W, gamma, Rt, t, h, w, r, metric))


def budget(Hent: float, a: float, b: float, N: int, Bmin: int) -> int:
    return int(lib().oracle_budget(float(np.float32(Hent)), a, b, N, Bmin))


def token_mask(T, H, W, gamma, Rt, i, j, r_i, metric: int = CHEBYSHEV) -> bool:
    return bool(lib().oracle_token_mask(T, H, W, gamma, Rt, metric, i, j, r_i))


# ----------------------------------------------------------------- arrays
def radius(Hent, G, grid, a, b, gamma, Rt, Bmin, queries=None, metric: int = CHEBYSHEV):
    """E3+E4.  Hent: fp32 entropies (all G*N in order, or one per listed query).
    Returns (r int32, c int64, bhat int64) per row."""
    T, H, W = grid
    Hf = np.ascontiguousarray(np.asarray(Hent, dtype=np.float32).reshape(-1))
    q, nq, qp = _qlist(queries)
    rows = nq if q is not None else G * T * H * W
    assert Hf.size == rows
    r = np.zeros(rows, np.int32)
    c = np.zeros(rows, np.int64)
    bh = np.zeros(rows, np.int64)
    lib().oracle_radius(_ptr(Hf, _F32P), G, T, H, W, a, b, gamma, Rt, Bmin, metric,
                        qp, nq, _ptr(r, _I32P), _ptr(c, _I64P), _ptr(bh, _I64P))
    return r, c, bh


def block_mask(r, G, grid, gamma, Rt, qtile, ktile, qtiles=None, metric: int = CHEBYSHEV) -> np.ndarray:
    """E6.  r: int32 radii [G*N] natural order.  qtile/ktile: (th, tw) of the
    (1, th, tw) query/key tiles.  Returns uint8 [rows, nK]: 0 inactive,
    1 active, 3 active and full.  qtiles: list of g*nQ + a (None = all)."""
    T, H, W = grid
    rr = np.ascontiguousarray(np.asarray(r, dtype=np.int32).reshape(-1))
    qth, qtw = qtile
    kth, ktw = ktile
    nQ = T * (-(-H // qth)) * (-(-W // qtw))
    nK = T * (-(-H // kth)) * (-(-W // ktw))
    q, nq, qp = _qlist(qtiles)
    rows = nq if q is not None else G * nQ
    out = np.zeros((rows, nK), np.uint8)
    lib().oracle_block_mask(_ptr(rr, _I32P), G, T, H, W, gamma, Rt, metric, qth, qtw, kth, ktw,
                            qp, nq, _ptr(out, _U8P))
    return out


def query_groups(r, G, grid, tile):
    """The radius-sorted query groups of TRA_FLAG_QSORT plans (a design of this
    library, not of the pages).  Query tiles are (1, th, tw) boxes in the
    tile-major order.  A strip is one tile column of one frame: its nTh tiles,
    top to bottom, hold strip rows l = u*128 + i (row i of the tile in tile
    row u).  The strip's rows are ordered by (radius, l), pad rows (outside the
    grid, radius -1) first, and the u-th block of 128 is the group that takes
    the mask slot of the strip's tile in tile row u.

    r: int32 radii [G*N] in natural order.  Returns
      perm    uint16 [G, nQ, 128]: strip row (0 .. 128*nTh - 1) of each group slot;
      members int64 [G*nQ, 128]: the slot's query as g*N + n, -1 on pad rows."""
    T, H, W = grid
    th, tw = tile
    nTh, nTw = -(-H // th), -(-W // tw)
    tpf = nTh * nTw
    nQ = T * tpf
    N = T * H * W
    rr = np.asarray(r, dtype=np.int64).reshape(G, N)
    p = np.arange(nQ * 128)
    tile, inn = p // 128, p % 128
    t, rem = tile // tpf, tile % tpf
    h = (rem // nTw) * th + inn // tw
    w = (rem % nTw) * tw + inn % tw
    valid = (h < H) & (w < W)
    nat = np.where(valid, (t * H + h) * W + w, -1)
    perm = np.zeros((G, nQ, 128), np.uint16)
    members = np.full((G * nQ, 128), -1, np.int64)
    for g in range(G):
        rad = np.where(valid, rr[g][np.maximum(nat, 0)], -1)
        for tt in range(T):
            for c in range(nTw):
                tiles = [tt * tpf + u * nTw + c for u in range(nTh)]
                rows = np.concatenate([np.arange(a * 128, a * 128 + 128) for a in tiles])   # strip row l -> tile-major row
                order = np.argsort(rad[rows], kind="stable")        # (radius, l): stable on l
                for u, a in enumerate(tiles):
                    sl = order[128 * u:128 * (u + 1)]
                    perm[g, a] = sl
                    src = nat[rows[sl]]
                    members[g * nQ + a] = np.where(src >= 0, g * N + src, -1)
    return perm, members


def block_mask_sets(r, G, grid, gamma, Rt, ktile, members, metric: int = CHEBYSHEV) -> np.ndarray:
    """Block-mask rows of explicit query sets: members int64 [n_sets, set_size]
    (g*N + n, -1 = empty slot), one head per set.  Returns uint8 [n_sets, nK]
    with 0 / 1 / 3 as block_mask."""
    T, H, W = grid
    rr = np.ascontiguousarray(np.asarray(r, dtype=np.int32).reshape(-1))
    mem = np.ascontiguousarray(np.asarray(members, dtype=np.int64))
    n_sets, set_size = mem.shape
    kth, ktw = ktile
    nK = T * (-(-H // kth)) * (-(-W // ktw))
    out = np.zeros((n_sets, nK), np.uint8)
    lib().oracle_block_mask_sets(_ptr(rr, _I32P), G, T, H, W, gamma, Rt, metric, kth, ktw,
                                 _ptr(mem, _I64P), n_sets, set_size, _ptr(out, _U8P))
    return out


def entropy(q, k, G, grid, d, key_stride=1, ktile=(1, 1), queries=None) -> np.ndarray:
    """E1 (key_stride 1) / E2 (key_stride > 1 over (1, kth, ktw) key tiles)."""
    T, H, W = grid
    qa, tq = _elems(q)
    ka, tk = _elems(k)
    assert tq == tk
    ql, nq, qp = _qlist(queries)
    rows = nq if ql is not None else G * T * H * W
    out = np.zeros(rows, np.float64)
    lib().oracle_entropy(qa.ctypes.data, ka.ctypes.data, tq, G, T, H, W, d,
                         key_stride, ktile[0], ktile[1], qp, nq, _ptr(out, _F64P))
    return out


def attention(q, k, v, r, G, grid, d, gamma, Rt, queries=None, metric: int = CHEBYSHEV) -> np.ndarray:
    """E7: masked softmax attention, fp64 [rows, d]."""
    T, H, W = grid
    qa, tq = _elems(q)
    ka, tk = _elems(k)
    va, tv = _elems(v)
    assert tq == tk == tv
    rr = np.ascontiguousarray(np.asarray(r, dtype=np.int32).reshape(-1))
    ql, nq, qp = _qlist(queries)
    rows = nq if ql is not None else G * T * H * W
    out = np.zeros((rows, d), np.float64)
    lib().oracle_attention(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, tq, _ptr(rr, _I32P),
                           G, T, H, W, d, gamma, Rt, metric, qp, nq, _ptr(out, _F64P))
    return out


def topk_count(q, k, G, grid, d, mass, queries=None) -> np.ndarray:
    """Calibration: per query, the fewest highest-probability keys whose dense
    softmax probabilities sum to at least `mass` (exact fp64 sort)."""
    T, H, W = grid
    qa, tq = _elems(q)
    ka, tk = _elems(k)
    assert tq == tk
    ql, nq, qp = _qlist(queries)
    rows = nq if ql is not None else G * T * H * W
    out = np.zeros(rows, np.int64)
    lib().oracle_topk_count(qa.ctypes.data, ka.ctypes.data, tq, G, T, H, W, d, float(mass), qp, nq,
                            _ptr(out, _I64P))
    return out


def fit_log_linear(H, k):
    """Calibration fit: least squares of ln k = a*H + b over the rows with
    k >= 1 and a finite H.  Returns (a, b, r2, rows used); raises ValueError
    when fewer than two usable rows remain or their H are all equal."""
    Hd = np.ascontiguousarray(np.asarray(H, dtype=np.float64).reshape(-1))
    kd = np.ascontiguousarray(np.asarray(k, dtype=np.int64).reshape(-1))
    assert Hd.size == kd.size
    a, b, r2 = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    m = lib().oracle_fit_log_linear(_ptr(Hd, _F64P), _ptr(kd, _I64P), Hd.size,
                                    ctypes.byref(a), ctypes.byref(b), ctypes.byref(r2))
    if m < 0:
        raise ValueError("fewer than two usable (H, k) rows, or all H equal")
    return a.value, b.value, r2.value, int(m)


def num_threads() -> int:
    return int(lib().oracle_num_threads())
