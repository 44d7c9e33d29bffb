"""Token Radius Attention hot path on NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/tra.h`` (``libtra_b200.so``,
built in-tree by ``sparse_attention_video_tra_b200.build``).  The functions
below carry the C names and only marshal arguments; every step of the path
runs in the library's CUDA kernels.  PyTorch provides device memory and
streams.  There is no fallback: if the library is missing, every call raises.

Method: "Token Radius Attention for Efficient Video Generation" (gist.science
summary), section 2 -- entropy -> token budget (Intuition I), budget ->
temporally decayed radius (Intuition II), radius mask -> block-sparse mask,
block-sparse attention ("Le Pipeline TRA").
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

__all__ = [
    "TraError", "PlanInfo", "Plan", "library_path", "load_library",
    "tra_plan_create", "tra_plan_destroy", "tra_plan_query", "tra_permute", "tra_entropy",
    "tra_radius_and_mask", "tra_attention", "tra_calibrate_topk", "tra_calibrate_fit", "tra_plan_status",
    "tra_status_string",
    "TRA_FLAG_DEBUG_NO_WAIT", "TRA_FLAG_OUT_BF16", "TRA_FLAG_NATURAL", "TRA_FLAG_DISK", "TRA_FLAG_QSORT",
    "tra_flag_tile_w",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtra_b200.so")
_lib = None

TRA_OK = 0
TRA_FLAG_DEBUG_NO_WAIT = 1 << 16
TRA_FLAG_OUT_BF16 = 1 << 17
TRA_FLAG_NATURAL = 1 << 18
TRA_FLAG_DISK = 1 << 19
TRA_FLAG_QSORT = 1 << 20
STATUS_NAMES = {0: "TRA_OK", 1: "TRA_ERR_INVALID_ARG", 2: "TRA_ERR_UNSUPPORTED", 3: "TRA_ERR_WORKSPACE",
                4: "TRA_ERR_CUDA", 5: "TRA_ERR_TIMEOUT", 6: "TRA_ERR_DEVICE_CHECK"}


def tra_flag_tile_w(tw: int) -> int:
    return (int(tw) & 0xFF) << 8


class TraError(RuntimeError):
    def __init__(self, func: str, status: int):
        self.status = status
        super().__init__(f"{func} failed: {STATUS_NAMES.get(status, status)} ({tra_status_string(status)})")


class _Info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("T", "H", "W", "heads", "d", "N", "N_pad", "tile_h", "tile_w", "n_tiles_h", "n_tiles_w",
                 "n_tiles", "rt_eff", "r_cap", "list_cap")] + \
               [(n, ctypes.c_size_t) for n in
                ("mask_bytes", "off_radius", "off_tile_count", "off_tile_pairs", "off_list", "off_group")]


@dataclass(frozen=True)
class PlanInfo:
    T: int
    H: int
    W: int
    heads: int
    d: int
    N: int
    N_pad: int
    tile_h: int
    tile_w: int
    n_tiles_h: int
    n_tiles_w: int
    n_tiles: int
    rt_eff: int
    r_cap: int
    list_cap: int
    mask_bytes: int
    off_radius: int
    off_tile_count: int
    off_tile_pairs: int
    off_list: int
    off_group: int


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load libtra_b200.so; raise loudly if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m sparse_attention_video_tra_b200.build` (no CPU fallback exists)")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
    L.tra_plan_create.argtypes = [ctypes.POINTER(vp), i, i, i, i, i, ctypes.c_double, ctypes.c_double,
                                  ctypes.c_double, i, i, ctypes.c_uint]
    L.tra_plan_create.restype = st
    L.tra_plan_destroy.argtypes = [vp]
    L.tra_plan_destroy.restype = None
    L.tra_plan_query.argtypes = [vp, ctypes.POINTER(_Info)]
    L.tra_plan_query.restype = st
    L.tra_permute.argtypes = [vp, vp, vp, i, i, vp]
    L.tra_permute.restype = st
    L.tra_entropy.argtypes = [vp, vp, vp, vp, i, vp]
    L.tra_entropy.restype = st
    L.tra_radius_and_mask.argtypes = [vp, vp, vp, ctypes.c_size_t, vp]
    L.tra_radius_and_mask.restype = st
    L.tra_attention.argtypes = [vp, vp, vp, vp, vp, vp, vp]
    L.tra_attention.restype = st
    L.tra_calibrate_topk.argtypes = [vp, vp, vp, ctypes.c_double, i, vp, vp, vp]
    L.tra_calibrate_topk.restype = st
    L.tra_calibrate_fit.argtypes = [vp, vp, ctypes.c_longlong, ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong)]
    L.tra_calibrate_fit.restype = st
    L.tra_plan_status.argtypes = [vp]
    L.tra_plan_status.restype = st
    L.tra_status_string.argtypes = [st]
    L.tra_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(func: str, status: int):
    if status != TRA_OK:
        raise TraError(func, status)


# ------------------------------------------------------------- C-named calls
def tra_status_string(status: int) -> str:
    return load_library().tra_status_string(int(status)).decode()


def tra_plan_create(T, H, W, heads, d, a, b, gamma, Rt, Bmin, flags=0) -> int:
    h = ctypes.c_void_p()
    _check("tra_plan_create", load_library().tra_plan_create(
        ctypes.byref(h), int(T), int(H), int(W), int(heads), int(d), float(a), float(b), float(gamma),
        int(Rt), int(Bmin), int(flags)))
    return h.value


def tra_plan_destroy(plan: int) -> None:
    load_library().tra_plan_destroy(plan)


def tra_plan_query(plan: int) -> PlanInfo:
    info = _Info()
    _check("tra_plan_query", load_library().tra_plan_query(plan, ctypes.byref(info)))
    return PlanInfo(**{f: getattr(info, f) for f, _ in _Info._fields_})


def tra_permute(plan, src_ptr, dst_ptr, to_tile_major, elem_bytes=2, stream=0) -> None:
    _check("tra_permute", load_library().tra_permute(plan, src_ptr, dst_ptr, int(to_tile_major),
                                                     int(elem_bytes), stream))


def tra_entropy(plan, q_ptr, k_ptr, H_ptr, key_tile_stride=1, stream=0) -> None:
    _check("tra_entropy", load_library().tra_entropy(plan, q_ptr, k_ptr, H_ptr, int(key_tile_stride), stream))


def tra_radius_and_mask(plan, H_ptr, mask_ptr, mask_bytes, stream=0) -> None:
    _check("tra_radius_and_mask", load_library().tra_radius_and_mask(plan, H_ptr, mask_ptr, int(mask_bytes),
                                                                     stream))


def tra_attention(plan, q_ptr, k_ptr, v_ptr, mask_ptr, out_ptr, stream=0) -> None:
    _check("tra_attention", load_library().tra_attention(plan, q_ptr, k_ptr, v_ptr, mask_ptr, out_ptr, stream))


def tra_calibrate_topk(plan, q_ptr, k_ptr, mass, query_tile_stride, H_ptr, k_out_ptr, stream=0) -> None:
    _check("tra_calibrate_topk", load_library().tra_calibrate_topk(plan, q_ptr, k_ptr, float(mass),
                                                                   int(query_tile_stride), H_ptr, k_out_ptr,
                                                                   stream))


def tra_calibrate_fit(H_ptr, k_ptr, n) -> tuple[float, float, int]:
    """(a, b, rows used) of ln k = a*H + b from n host rows (fp32 H, int32 k)."""
    a, b, m = ctypes.c_double(), ctypes.c_double(), ctypes.c_longlong()
    _check("tra_calibrate_fit", load_library().tra_calibrate_fit(H_ptr, k_ptr, int(n), ctypes.byref(a),
                                                                 ctypes.byref(b), ctypes.byref(m)))
    return a.value, b.value, m.value


def tra_plan_status(plan) -> int:
    return int(load_library().tra_plan_status(plan))


# ------------------------------------------------------------- torch helpers
class Plan:
    """Owns a tra_plan handle and passes torch tensors (data pointers and the
    current CUDA stream) to the C calls.  Shape/dtype checks only."""

    def __init__(self, T, H, W, heads, d, a, b, gamma, Rt, Bmin, flags=0):
        self.handle = tra_plan_create(T, H, W, heads, d, a, b, gamma, Rt, Bmin, flags)
        self.flags = flags
        self.info = tra_plan_query(self.handle)
        self.params = dict(T=T, H=H, W=W, heads=heads, d=d, a=a, b=b, gamma=gamma, Rt=Rt, Bmin=Bmin)

    def close(self):
        if getattr(self, "handle", None):
            tra_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- buffers
    def _stream(self, stream):
        import torch
        return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream

    def _rows(self, x, rows, name, dtype=None):
        import torch
        i = self.info
        dtype = dtype or torch.bfloat16
        if x.dtype != dtype or not x.is_cuda or not x.is_contiguous() or x.numel() != i.heads * rows * i.d:
            raise ValueError(f"{name}: expected contiguous cuda {dtype} with {i.heads}*{rows}*{i.d} elements, "
                             f"got {x.dtype} {tuple(x.shape)} on {x.device}")

    @property
    def out_dtype(self):
        import torch
        return torch.bfloat16 if self.flags & TRA_FLAG_OUT_BF16 else torch.float32

    @property
    def natural(self) -> bool:
        """q, k, v, out and entropies in natural token order (TRA_FLAG_NATURAL)."""
        return bool(self.flags & TRA_FLAG_NATURAL)

    @property
    def io_rows(self) -> int:
        """Rows per head of q, k, v, out and the entropies in this plan's layout."""
        return self.info.N if self.natural else self.info.N_pad

    def new_tile_major(self, device="cuda", dtype=None):
        import torch
        i = self.info
        return torch.empty(i.heads, i.N_pad, i.d, dtype=dtype or torch.bfloat16, device=device)

    def new_input(self, device="cuda", dtype=None):
        """A q/k/v buffer in this plan's layout."""
        import torch
        i = self.info
        return torch.empty(i.heads, self.io_rows, i.d, dtype=dtype or torch.bfloat16, device=device)

    def new_out(self, device="cuda"):
        return self.new_input(device, self.out_dtype)

    def new_entropy(self, device="cuda"):
        import torch
        return torch.empty(self.info.heads, self.io_rows, dtype=torch.float32, device=device)

    def new_mask(self, device="cuda"):
        import torch
        return torch.empty(self.info.mask_bytes, dtype=torch.uint8, device=device)

    @property
    def qsort(self) -> bool:
        """Radius-sorted query groups (TRA_FLAG_QSORT)."""
        return bool(self.flags & TRA_FLAG_QSORT)

    def group_view(self, mask):
        """TRA_FLAG_QSORT: [heads, n_tiles, 128] int16 view of the uint16 strip
        row (0 .. 128*n_tiles_h - 1) of each slot of each tile's query group."""
        import torch
        i = self.info
        if not self.qsort:
            raise ValueError("the plan has no query groups (TRA_FLAG_QSORT)")
        n = i.heads * i.n_tiles * 128 * 2
        return mask[i.off_group:i.off_group + n].view(torch.int16).view(i.heads, i.n_tiles, 128)

    def mask_views(self, mask):
        """(radius [heads,N_pad] i32, tile_count [heads,n_tiles] i32,
        tile_pairs [heads,n_tiles] i64, list [heads,n_tiles,list_cap] i16)."""
        import torch
        i = self.info

        def view(off, count, dtype, shape):
            nbytes = count * torch.empty((), dtype=dtype).element_size()
            return mask[off:off + nbytes].view(dtype).view(*shape)

        return (view(i.off_radius, i.heads * i.N_pad, torch.int32, (i.heads, i.N_pad)),
                view(i.off_tile_count, i.heads * i.n_tiles, torch.int32, (i.heads, i.n_tiles)),
                view(i.off_tile_pairs, i.heads * i.n_tiles, torch.int64, (i.heads, i.n_tiles)),
                view(i.off_list, i.heads * i.n_tiles * i.list_cap, torch.int16, (i.heads, i.n_tiles, i.list_cap)))

    # -- the path
    def permute(self, src, dst, to_tile_major=True, stream=None):
        import torch
        i = self.info
        if src.dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("permute moves bf16 or fp32 rows")
        self._rows(src, i.N if to_tile_major else i.N_pad, "src", src.dtype)
        self._rows(dst, i.N_pad if to_tile_major else i.N, "dst", src.dtype)
        tra_permute(self.handle, src.data_ptr(), dst.data_ptr(), 1 if to_tile_major else 0,
                    src.element_size(), self._stream(stream))
        return dst

    def entropy(self, q, k, Hout, key_tile_stride=1, stream=None):
        import torch
        i = self.info
        self._rows(q, self.io_rows, "q")
        self._rows(k, self.io_rows, "k")
        if Hout.dtype != torch.float32 or not Hout.is_cuda or Hout.numel() != i.heads * self.io_rows:
            raise ValueError(f"Hout: expected cuda float32 [heads, {self.io_rows}]")
        tra_entropy(self.handle, q.data_ptr(), k.data_ptr(), Hout.data_ptr(), key_tile_stride, self._stream(stream))
        return Hout

    def radius_and_mask(self, Hent, mask, stream=None):
        import torch
        i = self.info
        if Hent.dtype != torch.float32 or not Hent.is_cuda or Hent.numel() != i.heads * self.io_rows:
            raise ValueError(f"Hent: expected cuda float32 [heads, {self.io_rows}]")
        tra_radius_and_mask(self.handle, Hent.data_ptr(), mask.data_ptr(), mask.numel(), self._stream(stream))
        return mask

    def attention(self, q, k, v, mask, out, stream=None):
        i = self.info
        for x, nme in ((q, "q"), (k, "k"), (v, "v")):
            self._rows(x, self.io_rows, nme)
        self._rows(out, self.io_rows, "out", self.out_dtype)
        tra_attention(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), mask.data_ptr(), out.data_ptr(),
                      self._stream(stream))
        return out

    def calibrate_topk(self, q, k, mass, query_tile_stride=1, stream=None):
        """Calibration workload: (H [heads, n_sample, 128] fp32, k [heads,
        n_sample, 128] int32) for the queries of every query_tile_stride-th
        tile; k_i = fewest top keys holding `mass` of the query's attention."""
        import torch
        i = self.info
        self._rows(q, self.io_rows, "q")
        self._rows(k, self.io_rows, "k")
        n_sample = -(-i.n_tiles // int(query_tile_stride))
        H = torch.empty(i.heads, n_sample, 128, dtype=torch.float32, device=q.device)
        K = torch.empty(i.heads, n_sample, 128, dtype=torch.int32, device=q.device)
        tra_calibrate_topk(self.handle, q.data_ptr(), k.data_ptr(), mass, query_tile_stride, H.data_ptr(),
                           K.data_ptr(), self._stream(stream))
        return H, K

    def status(self) -> int:
        return tra_plan_status(self.handle)
