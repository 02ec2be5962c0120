"""Python binding of libcalibatt.so (ctypes): argument marshalling only.

Every function here converts Python / torch arguments into the plain pointers
and sizes of the C ABI in include/calibatt.h and calls the function of the
same name; all computation happens in the library's CUDA kernels.  There is
no fallback: if the shared library is missing, importing this module raises.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libcalibatt.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_CUDA = 3
ERR_TIMEOUT = 4
ERR_OOM = 5
DTYPE_BF16 = 0
DTYPE_FP32 = 1


class CalibattError(RuntimeError):
    """A non-OK status from the library; `.status` holds the code."""

    def __init__(self, status: int, message: str):
        super().__init__(f"calibatt status {status}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("seq_len", ctypes.c_int32),
        ("heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("stride_b", ctypes.c_int64),
        ("stride_n", ctypes.c_int64),
        ("stride_h", ctypes.c_int64),
        ("dtype", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


_i32, _i64, _f32, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
_P = ctypes.POINTER

# name -> (restype, argtypes)
SIGNATURES = {
    "calibatt_status_string": (ctypes.c_char_p, [_i32]),
    "calibatt_last_error": (ctypes.c_char_p, []),
    "calibatt_abi_version": (_i32, []),
    "calibatt_csr_validate": (_i32, [_i32, _i32, _vp, _vp, _i32]),
    "calibatt_csr_to_intervals": (_i32, [_i32, _vp, _vp, _vp, _vp, _vp, _i64, _P(_i64)]),
    "calibatt_lpt_schedule": (_i32, [_i32, _vp, _i32, _vp, _vp, _P(_i64)]),
    "calibatt_dict_create": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _i64, _i32, _P(_vp)]),
    "calibatt_dict_set_layer": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp]),
    "calibatt_debug_bounded_wait": (_i32, [_vp]),
    "calibatt_dict_create_bitmap": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _P(_vp)]),
    "calibatt_dict_create_intervals": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _i64, _i32, _P(_vp)]),
    "calibatt_dict_set_anchor_geometry": (_i32, [_vp, _i32, _i32, _i32, _vp, _i32]),
    "calibatt_spatial_similarity": (_i32, [_vp, _vp, _P(Shape), _i32, _i32, _i32, _vp, _i32, _f32, _vp, _vp,
                                           ctypes.c_size_t, _vp]),
    "calibatt_repetition_flags": (_i32, [_vp, _i32, _i32, _i32, _f32, _vp, _vp, _vp]),
    "calibatt_spatial_similarity_workspace_size": (_i32, [_P(Shape), _P(ctypes.c_size_t)]),
    "calibatt_dict_info": (_i32, [_vp, _P(_i64), _P(_i64), _P(_i32)]),
    "calibatt_dict_layer_info": (_i32, [_vp, _i32, _i32, _P(_i32), _P(_i32), _P(_i64)]),
    "calibatt_dict_destroy": (_i32, [_vp]),
    "calibatt_dict_save": (_i32, [_vp, ctypes.c_char_p]),
    "calibatt_dict_load": (_i32, [ctypes.c_char_p, _i32, _P(_vp)]),
    "calibatt_block_sparse_attn": (_i32, [_vp, _vp, _vp, _vp, _P(Shape), _i32, _vp, _i32, _i32, _f32, _vp, _vp]),
    "calibatt_csr_schedule": (_i32, [_i32, _i32, _vp, _vp, _i32, _i32, _vp, _vp]),
    "calibatt_block_sparse_attn_csr": (_i32, [_vp, _vp, _vp, _vp, _P(Shape), _i32, _vp, _vp, _vp, _vp, _i32, _vp,
                                              _vp, _i32, _f32, _vp, _vp]),
    "calibatt_block_sparse_attn_host": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _P(Shape), _i32, _vp, _i32,
                                               _i32, _f32, _vp, _vp]),
    "calibatt_anchor_attn": (_i32, [_vp, _vp, _vp, _vp, _P(Shape), _i32, _i32, _i32, _i32, _vp, _i32, _vp,
                                    _i32, _f32, _vp, ctypes.c_size_t, _vp]),
    "calibatt_anchor_attn_workspace_size": (_i32, [_P(Shape), _i32, _i32, _i32, _i32, _i32,
                                                   _P(ctypes.c_size_t)]),
    "calibatt_anchor_split_plan": (_i32, [_i64, _i32, _i32, _P(_i64), _P(_i32)]),
    "calibatt_dual_path_attn": (_i32, [_vp, _vp, _vp, _vp, _P(Shape), _i32, _vp, _i32, _i32, _i32, _i32, _i32,
                                       _vp, _i32, _f32, _vp, _vp]),
    "calibatt_block_energy_workspace_size": (_i32, [_P(Shape), _P(ctypes.c_size_t)]),
    "calibatt_block_energy": (_i32, [_vp, _vp, _P(Shape), _i32, _f32, _vp, _vp, ctypes.c_size_t, _vp]),
    "calibatt_block_energy_noalloc": (_i32, [_vp, _vp, _P(Shape), _i32, _f32, _vp, _vp]),
    "calibatt_select_blocks": (_i32, [_vp, _i64, _i32, _f32, _vp, _vp, _vp]),
    "calibatt_aggregate_masks": (_i32, [_vp, _i64, _i32, _f32, _vp, _vp]),
    "calibatt_debug_exp2_fma": (_i32, [_vp, _vp, _i64, _vp]),
    "calibatt_debug_exp2_fma_quintic": (_i32, [_vp, _vp, _i64, _vp]),
    "calibatt_device_status": (_i32, [_vp, _P(_i32), _i32]),
    "calibatt_set_wait_timeout_ms": (_i32, [_i32]),
    "calibatt_device_sm_count": (_i32, [_P(_i32)]),
}


def library_path() -> str:
    return _LIB_PATH


def _load():
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"{_LIB_PATH} is missing: build it with "
            "`python -c 'import __graft_entry__ as g; g.build()'` (nvcc, sm_100a)")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def last_error() -> str:
    return LIB.calibatt_last_error().decode()


def check(status: int) -> None:
    if status != OK:
        raise CalibattError(status, last_error())


# ---------------------------------------------------------------- marshalling

def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def shape_of(t) -> Shape:
    """Shape of a [batch, N, heads, head_dim] torch tensor (last dim contiguous)."""
    import torch

    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [batch, N, heads, head_dim] tensor with contiguous head_dim")
    dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_FP32}.get(t.dtype)
    if dtype is None:
        raise ValueError(f"unsupported dtype {t.dtype}")
    b, n, h, d = t.shape
    return Shape(b, n, h, d, t.stride(0), t.stride(1), t.stride(2), dtype, 0)


def _i32_array(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


# ----------------------------------------------------------------- host utilities

def csr_validate(nq, nk, row_ptr, col_idx, require_diagonal=False) -> int:
    rp, ci = _i32_array(row_ptr), _i32_array(col_idx)
    return LIB.calibatt_csr_validate(nq, nk, _ptr(rp), _ptr(ci) if ci.size else None, int(require_diagonal))


def csr_to_intervals(nq, row_ptr, col_idx):
    rp, ci = _i32_array(row_ptr), _i32_array(col_idx)
    n = ctypes.c_int64(0)
    ptr = np.zeros(nq + 1, np.int32)
    cap = max(1, ci.size)
    start = np.zeros(cap, np.int32)
    length = np.zeros(cap, np.int32)
    check(LIB.calibatt_csr_to_intervals(nq, _ptr(rp), _ptr(ci) if ci.size else None, _ptr(ptr), _ptr(start),
                                        _ptr(length), cap, ctypes.byref(n)))
    return ptr, start[:n.value], length[:n.value]


def count_intervals(row_ptr, col_idx):
    """Contiguous key-block intervals of a layer's CSR (row_ptr [H, nq + 1],
    the heads' lists concatenated): the capacity an interval dictionary needs
    for it, as the library encodes each head (calibatt_csr_to_intervals)."""
    rp = _i32_array(row_ptr).reshape(-1, np.asarray(row_ptr).shape[-1])
    ci = _i32_array(col_idx).reshape(-1)
    nq = rp.shape[1] - 1
    total, off = 0, 0
    ptr = np.zeros(nq + 1, np.int32)
    for h in range(rp.shape[0]):
        n = int(rp[h, -1])
        head = np.ascontiguousarray(ci[off:off + n])
        cnt = ctypes.c_int64(0)
        # capacity 0: the library only counts (and reports the shortfall)
        st = LIB.calibatt_csr_to_intervals(nq, _ptr(np.ascontiguousarray(rp[h])), _ptr(head) if n else None,
                                           _ptr(ptr), None, None, 0, ctypes.byref(cnt))
        if st != OK and cnt.value == 0:
            raise CalibattError(st, last_error())
        total += cnt.value
        off += n
    return total


def lpt_schedule(cost, n_bins):
    c = np.ascontiguousarray(np.asarray(cost, dtype=np.int64))
    bin_ptr = np.zeros(n_bins + 1, np.int32)
    order = np.zeros(max(1, c.size), np.int32)
    mk = ctypes.c_int64(0)
    check(LIB.calibatt_lpt_schedule(c.size, _ptr(c), n_bins, _ptr(bin_ptr), _ptr(order), ctypes.byref(mk)))
    return bin_ptr, order[:c.size], mk.value


def csr_schedule(row_ptr, head_ids, grid):
    """Host schedule of a direct-CSR call for row_ptr [heads, nq + 1]:
    (items uint32 [len(head_ids) * nq], cta_ptr int32 [grid + 1])."""
    rp = _i32_array(row_ptr)
    heads, nq = rp.shape[0], rp.shape[1] - 1
    hid = _i32_array(head_ids)
    items = np.zeros(max(1, hid.size * nq), np.uint32)
    cta_ptr = np.zeros(grid + 1, np.int32)
    check(LIB.calibatt_csr_schedule(heads, nq, _ptr(rp), _ptr(hid) if hid.size else None, hid.size, grid,
                                    _ptr(items), _ptr(cta_ptr)))
    return items[:hid.size * nq], cta_ptr


def calibatt_debug_exp2_fma(x, y, stream=None):
    check(LIB.calibatt_debug_exp2_fma(_ptr(x), _ptr(y), x.numel(), _stream(stream)))


def calibatt_debug_exp2_fma_quintic(x, y, stream=None):
    check(LIB.calibatt_debug_exp2_fma_quintic(_ptr(x), _ptr(y), x.numel(), _stream(stream)))


def set_wait_timeout_ms(ms: int) -> None:
    check(LIB.calibatt_set_wait_timeout_ms(int(ms)))


def device_sm_count() -> int:
    n = ctypes.c_int32(0)
    check(LIB.calibatt_device_sm_count(ctypes.byref(n)))
    return n.value


def debug_bounded_wait(stream=None):
    """Launches the failure-path check of the bounded waits (see the header)."""
    check(LIB.calibatt_debug_bounded_wait(_stream(stream)))


def device_status(stream=None, clear=True) -> int:
    code = ctypes.c_int32(0)
    st = LIB.calibatt_device_status(_stream(stream), ctypes.byref(code), int(clear))
    if st not in (OK, ERR_TIMEOUT, ERR_INVALID_ARG):
        check(st)
    return code.value


# ---------------------------------------------------------------- dictionary

class MaskDictionary:
    """Owns a calibatt_dict (per (t, l, h) skip lists and repetitive flags on the GPU)."""

    def __init__(self, T, L, H, nq, nk, block, nnz_capacity=0, num_ctas=0, bitmap=False, intervals=False):
        """bitmap=True stores one bit per (query block, key block) per record
        (calibatt_dict_create_bitmap) instead of index lists; intervals=True
        stores each row's contiguous key-block intervals
        (calibatt_dict_create_intervals), nnz_capacity then counting intervals."""
        self.T, self.L, self.H, self.nq, self.nk, self.block = T, L, H, nq, nk, block
        h = ctypes.c_void_p(None)
        if bitmap:
            check(LIB.calibatt_dict_create_bitmap(T, L, H, nq, nk, block, int(num_ctas), ctypes.byref(h)))
        elif intervals:
            check(LIB.calibatt_dict_create_intervals(T, L, H, nq, nk, block, int(nnz_capacity), int(num_ctas),
                                                     ctypes.byref(h)))
        else:
            check(LIB.calibatt_dict_create(T, L, H, nq, nk, block, int(nnz_capacity), int(num_ctas),
                                           ctypes.byref(h)))
        self.handle = h

    @classmethod
    def load(cls, path, num_ctas=0):
        """A dictionary read from a file written by save() (calibatt_dict_load)."""
        h = ctypes.c_void_p(None)
        check(LIB.calibatt_dict_load(os.fsencode(path), int(num_ctas), ctypes.byref(h)))
        self = cls.__new__(cls)
        self.handle = h
        return self

    def save(self, path):
        """Writes the dictionary's records to `path` (calibatt_dict_save)."""
        check(LIB.calibatt_dict_save(self.handle, os.fsencode(path)))

    def set_layer(self, t, l, row_ptr, col_idx, repetitive=None):
        rp = _i32_array(row_ptr).reshape(-1)
        ci = _i32_array(col_idx).reshape(-1)
        rep = None if repetitive is None else np.ascontiguousarray(np.asarray(repetitive, dtype=np.uint8))
        check(LIB.calibatt_dict_set_layer(self.handle, t, l, _ptr(rp), _ptr(ci) if ci.size else None,
                                          _ptr(rep) if rep is not None else None))

    def set_anchor_geometry(self, frames, rows, cols, anchor_rows):
        """Anchor geometry of the dual path; set before the first layer so
        that calibatt_dual_path_attn runs each layer in one launch."""
        a = _i32_array(anchor_rows).reshape(-1)
        check(LIB.calibatt_dict_set_anchor_geometry(self.handle, frames, rows, cols, _ptr(a), a.size))

    def info(self):
        b, n, g = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int32(0)
        check(LIB.calibatt_dict_info(self.handle, ctypes.byref(b), ctypes.byref(n), ctypes.byref(g)))
        return {"device_bytes": b.value, "nnz": n.value, "num_ctas": g.value}

    def layer_info(self, t, l):
        s, r, tiles = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int64(0)
        check(LIB.calibatt_dict_layer_info(self.handle, t, l, ctypes.byref(s), ctypes.byref(r), ctypes.byref(tiles)))
        return {"sparse_heads": s.value, "repetitive_heads": r.value, "retained_tiles": tiles.value}

    def close(self):
        if self.handle is not None and self.handle.value:
            check(LIB.calibatt_dict_destroy(self.handle))
        self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def masks_to_layer_csr(masks, H, nq):
    """Per-head bool masks (None = repetitive head) -> (row_ptr [H, nq+1], col_idx, repetitive [H])."""
    row_ptr = np.zeros((H, nq + 1), np.int32)
    cols = []
    rep = np.zeros(H, np.uint8)
    for h in range(H):
        m = masks[h]
        if m is None:
            rep[h] = 1
            continue
        m = np.asarray(m, dtype=bool)
        row_ptr[h, 1:] = np.cumsum(m.sum(axis=1))
        cols.append(np.nonzero(m)[1].astype(np.int32))
    col_idx = np.concatenate(cols) if cols else np.zeros(0, np.int32)
    return row_ptr, col_idx, rep


# ---------------------------------------------------------------- hot path

def calibatt_block_sparse_attn(q, k, v, o, d: MaskDictionary, t=0, l=0, block=128, softmax_scale=0.0,
                               lse=None, stream=None):
    shape = shape_of(q)
    check(LIB.calibatt_block_sparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shape), block,
                                         d.handle, t, l, float(softmax_scale), _ptr(lse), _stream(stream)))


def calibatt_block_sparse_attn_host(hq, hk, hv, ho, q, k, v, o, d: MaskDictionary, t, l, block=128,
                                    softmax_scale=0.0, lse=None, stream=None):
    """Copies host hq/hk/hv into device q/k/v, runs the block-sparse attention
    into o and copies o to host ho, all enqueued on `stream` (no sync)."""
    shape = shape_of(q)
    check(LIB.calibatt_block_sparse_attn_host(_ptr(hq), _ptr(hk), _ptr(hv), _ptr(ho), _ptr(q), _ptr(k), _ptr(v),
                                              _ptr(o), ctypes.byref(shape), block, d.handle, t, l,
                                              float(softmax_scale), _ptr(lse), _stream(stream)))


def calibatt_block_sparse_attn_csr(q, k, v, o, row_ptr, col_idx, col_base, head_ids, items=None, cta_ptr=None,
                                   grid=0, block=128, softmax_scale=0.0, lse=None, stream=None):
    """Block-sparse attention from device skip lists without a dictionary:
    row_ptr int32 [heads, nq + 1], col_idx 16-bit, col_base int64 [heads] (all
    device tensors); items / cta_ptr: the device copy of csr_schedule's result
    (tensor-core path)."""
    shape = shape_of(q)
    hid = _i32_array(head_ids)
    check(LIB.calibatt_block_sparse_attn_csr(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shape), block,
                                             _ptr(row_ptr), _ptr(col_idx), _ptr(col_base),
                                             _ptr(hid) if hid.size else None, hid.size, _ptr(items), _ptr(cta_ptr),
                                             int(grid), float(softmax_scale), _ptr(lse), _stream(stream)))


def calibatt_anchor_attn(q, k, v, o, frames, rows, cols, anchor_rows, head_ids, block=128, softmax_scale=0.0,
                         workspace=None, stream=None):
    """Anchor-row attention with broadcast for head_ids; workspace (a device
    tensor of at least calibatt_anchor_attn_workspace_size bytes) lets the
    call split its last partial wave of tiles over key ranges."""
    shape = shape_of(q)
    a = _i32_array(anchor_rows)
    h = _i32_array(head_ids)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    check(LIB.calibatt_anchor_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shape), block, frames, rows,
                                   cols, _ptr(a), a.size, _ptr(h) if h.size else None, h.size,
                                   float(softmax_scale), _ptr(workspace), ws_bytes, _stream(stream)))


def calibatt_anchor_attn_workspace_size(q, frames, rows, cols, n_anchors, n_heads) -> int:
    shape = shape_of(q)
    n = ctypes.c_size_t(0)
    check(LIB.calibatt_anchor_attn_workspace_size(ctypes.byref(shape), frames, rows, cols, n_anchors, n_heads,
                                                  ctypes.byref(n)))
    return n.value


def anchor_split_plan(tiles, grid, key_blocks):
    """(first, parts): the anchor call's split of its last wave of tiles."""
    first = ctypes.c_int64(0)
    parts = ctypes.c_int32(0)
    check(LIB.calibatt_anchor_split_plan(int(tiles), int(grid), int(key_blocks), ctypes.byref(first),
                                         ctypes.byref(parts)))
    return first.value, parts.value


def calibatt_dual_path_attn(q, k, v, o, d: MaskDictionary, t, l, frames, rows, cols, anchor_rows, block=128,
                            softmax_scale=0.0, lse=None, stream=None):
    shape = shape_of(q)
    a = _i32_array(anchor_rows)
    check(LIB.calibatt_dual_path_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shape), block, d.handle, t,
                                      l, frames, rows, cols, _ptr(a), a.size, float(softmax_scale), _ptr(lse),
                                      _stream(stream)))


def calibatt_spatial_similarity_workspace_size(q) -> int:
    shape = shape_of(q)
    n = ctypes.c_size_t(0)
    check(LIB.calibatt_spatial_similarity_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def calibatt_spatial_similarity(q, k, sim, workspace, frames, rows, cols, anchor_rows, softmax_scale=0.0,
                                stream=None):
    """Spatial-repetition score of every (batch, head, frame, row) into sim
    (float32 [batch, heads, frames, rows]); workspace of at least
    calibatt_spatial_similarity_workspace_size(q) bytes."""
    shape = shape_of(q)
    a = _i32_array(anchor_rows)
    nbytes = workspace.numel() * workspace.element_size()
    check(LIB.calibatt_spatial_similarity(_ptr(q), _ptr(k), ctypes.byref(shape), frames, rows, cols, _ptr(a), a.size,
                                          float(softmax_scale), _ptr(sim), _ptr(workspace), nbytes,
                                          _stream(stream)))


def calibatt_repetition_flags(sim, threshold=0.87, mean=None, flags=None, stream=None):
    """Per-head mean over prompts and rows of sim [prompts, heads, rows...] and
    the flags mean > threshold; returns (mean, flags) device tensors."""
    import torch
    n_prompts, n_heads = int(sim.shape[0]), int(sim.shape[1])
    per_head = int(sim[0, 0].numel()) if n_heads else 1
    if mean is None:
        mean = torch.empty(n_heads, dtype=torch.float32, device=sim.device)
    if flags is None:
        flags = torch.empty(n_heads, dtype=torch.uint8, device=sim.device)
    check(LIB.calibatt_repetition_flags(_ptr(sim), n_prompts, n_heads, per_head, float(threshold), _ptr(mean),
                                        _ptr(flags), _stream(stream)))
    return mean, flags


def calibatt_block_energy_workspace_size(q) -> int:
    shape = shape_of(q)
    n = ctypes.c_size_t(0)
    check(LIB.calibatt_block_energy_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return n.value


def calibatt_block_energy(q, k, energy, workspace, block, softmax_scale=0.0, stream=None):
    shape = shape_of(q)
    nbytes = workspace.numel() * workspace.element_size()
    check(LIB.calibatt_block_energy(_ptr(q), _ptr(k), ctypes.byref(shape), block, float(softmax_scale),
                                    _ptr(energy), _ptr(workspace), nbytes, _stream(stream)))


def calibatt_block_energy_noalloc(q, k, energy, block, softmax_scale=0.0, stream=None):
    """Block energies without any device allocation (scratch built into the library)."""
    shape = shape_of(q)
    check(LIB.calibatt_block_energy_noalloc(_ptr(q), _ptr(k), ctypes.byref(shape), block, float(softmax_scale),
                                            _ptr(energy), _stream(stream)))


def calibatt_select_blocks(energy, tau, mask, count_accum=None, stream=None):
    nk = energy.shape[-1]
    n_rows = energy.numel() // nk
    check(LIB.calibatt_select_blocks(_ptr(energy), n_rows, nk, float(tau), _ptr(mask), _ptr(count_accum),
                                     _stream(stream)))


def calibatt_aggregate_masks(counts, n_prompts, rho, mask, stream=None):
    check(LIB.calibatt_aggregate_masks(_ptr(counts), counts.numel(), int(n_prompts), float(rho), _ptr(mask),
                                       _stream(stream)))
