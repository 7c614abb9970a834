"""Python binding of the C ABI with the same names (moe_router_topk, ...).

Each function takes torch tensors that already live on the handle's device
and forwards their data pointers, sizes and the current CUDA stream to
libmoe.so.  No arithmetic of the layer happens here.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import MoeShape


class MoeError(RuntimeError):
    def __init__(self, name, status):
        self.status = status
        super().__init__(f"{name} returned {_lib.STATUS_NAMES.get(status, status)}")


def _ptr(t):
    """Data pointer of a tensor for the C ABI, which takes dense row-major
    buffers in device memory: a strided view or a host tensor is refused
    here rather than read with the wrong layout."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError(f"expected a contiguous tensor, got strides {tuple(t.stride())} "
                         f"for shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"expected a CUDA tensor, got one on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


BF16, I32, F32, U8 = torch.bfloat16, torch.int32, torch.float32, torch.uint8


def _arg(h, t, dtype, name):
    """_ptr plus the checks the C ABI cannot make: the element type the
    header states for this argument (None: any, a byte buffer) and the
    handle's device (a pointer into another GPU's memory would be read as
    if it were local)."""
    if t is None:
        return None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.is_cuda and t.device.index != h.device:
        raise ValueError(f"{name}: tensor on cuda:{t.device.index}, handle on cuda:{h.device}")
    return _ptr(t)


def _stream(h, stream=None):
    """The given stream, else the current stream of the handle's device."""
    s = torch.cuda.current_stream(h.device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _call(name, *args):
    st = getattr(_lib.load(), name)(*args)
    if st != _lib.MOE_OK:
        raise MoeError(name, st)


def make_shape(T, d, f, E, k, dtype=_lib.MOE_DTYPE_BF16, renorm=False) -> MoeShape:
    return MoeShape(T, d, f, E, k, dtype, _lib.MOE_FLAG_RENORM if renorm else 0)


class Handle:
    """Owns a moe_handle_t bound to one CUDA device."""

    def __init__(self, device: int = 0):
        self.device = device
        self._h = ctypes.c_void_p()
        _call("moe_create", ctypes.byref(self._h), device)

    @property
    def ptr(self):
        return self._h

    def close(self):
        if self._h:
            _lib.load().moe_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_size(self, shape: MoeShape) -> int:
        n = ctypes.c_size_t()
        _call("moe_workspace_size", self._h, ctypes.byref(shape), ctypes.byref(n))
        return n.value

    def launch_count(self) -> int:
        v = ctypes.c_uint64()
        _call("moe_get_launch_count", self._h, ctypes.byref(v))
        return v.value

    def get_status(self) -> int:
        v = ctypes.c_int()
        _call("moe_get_status", self._h, ctypes.byref(v))
        return v.value

    def set_wait_limit(self, ns: int) -> None:
        """Time limit of the grouped GEMMs' bounded waits (default 2 s)."""
        _call("moe_set_wait_limit", self._h, int(ns))


def max_rows(shape: MoeShape) -> int:
    n = ctypes.c_int64()
    _call("moe_max_rows", ctypes.byref(shape), ctypes.byref(n))
    return n.value


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def moe_router_topk(h, shape, x, w_router, bias, route_in, topk_idx, topk_w, probs, logits, ws,
                    stream=None):
    _call("moe_router_topk", h.ptr, ctypes.byref(shape), _arg(h, x, BF16, "x"),
          _arg(h, w_router, BF16, "w_router"), _arg(h, bias, F32, "bias"),
          _arg(h, route_in, I32, "route_in"), _arg(h, topk_idx, I32, "topk_idx"),
          _arg(h, topk_w, F32, "topk_w"), _arg(h, probs, F32, "probs"),
          _arg(h, logits, F32, "logits"), _arg(h, ws, None, "ws"),
          _nbytes(ws), _stream(h, stream))


def moe_permute(h, shape, x, topk_idx, counts, offsets, row_map, x_perm, ws, stream=None):
    _call("moe_permute", h.ptr, ctypes.byref(shape), _arg(h, x, BF16, "x"),
          _arg(h, topk_idx, I32, "topk_idx"), _arg(h, counts, I32, "counts"),
          _arg(h, offsets, I32, "offsets"), _arg(h, row_map, I32, "row_map"),
          _arg(h, x_perm, BF16, "x_perm"), _arg(h, ws, None, "ws"), _nbytes(ws), _stream(h, stream))


def moe_permute_noalloc(h, shape, x, topk_idx, counts, offsets, row_map, x_perm, stream=None):
    """moe_permute for callers that cannot supply scratch memory: the library
    uses a fixed 1 MiB array of its own instead of a workspace."""
    _call("moe_permute_noalloc", h.ptr, ctypes.byref(shape), _arg(h, x, BF16, "x"),
          _arg(h, topk_idx, I32, "topk_idx"), _arg(h, counts, I32, "counts"),
          _arg(h, offsets, I32, "offsets"), _arg(h, row_map, I32, "row_map"),
          _arg(h, x_perm, BF16, "x_perm"), _stream(h, stream))


def moe_grouped_swiglu_fwd(h, shape, x_perm, offsets, w_gu, w_down, au, hbuf, o_perm, ws,
                           stream=None):
    _call("moe_grouped_swiglu_fwd", h.ptr, ctypes.byref(shape), _arg(h, x_perm, BF16, "x_perm"),
          _arg(h, offsets, I32, "offsets"), _arg(h, w_gu, BF16, "w_gu"),
          _arg(h, w_down, BF16, "w_down"), _arg(h, au, BF16, "au"), _arg(h, hbuf, BF16, "h"),
          _arg(h, o_perm, BF16, "o_perm"), _arg(h, ws, None, "ws"), _nbytes(ws), _stream(h, stream))


def moe_grouped_swiglu_recompute(h, shape, x_perm, offsets, w_gu, au, hbuf, ws, stream=None):
    _call("moe_grouped_swiglu_recompute", h.ptr, ctypes.byref(shape),
          _arg(h, x_perm, BF16, "x_perm"), _arg(h, offsets, I32, "offsets"),
          _arg(h, w_gu, BF16, "w_gu"), _arg(h, au, BF16, "au"), _arg(h, hbuf, BF16, "h"),
          _arg(h, ws, None, "ws"), _nbytes(ws), _stream(h, stream))


def moe_permute_src(h, shape, x, topk_idx, counts, offsets, row_map, row_src, x_perm, ws,
                    stream=None):
    _call("moe_permute_src", h.ptr, ctypes.byref(shape), _arg(h, x, BF16, "x"),
          _arg(h, topk_idx, I32, "topk_idx"), _arg(h, counts, I32, "counts"),
          _arg(h, offsets, I32, "offsets"), _arg(h, row_map, I32, "row_map"),
          _arg(h, row_src, I32, "row_src"), _arg(h, x_perm, BF16, "x_perm"),
          _arg(h, ws, None, "ws"), _nbytes(ws), _stream(h, stream))


def moe_grouped_swiglu_fwd_combine(h, shape, x_perm, offsets, row_map, row_src, topk_w, w_gu,
                                   w_down, au, hbuf, o_perm, shared_out, y, arrivals, stream=None):
    _call("moe_grouped_swiglu_fwd_combine", h.ptr, ctypes.byref(shape),
          _arg(h, x_perm, BF16, "x_perm"), _arg(h, offsets, I32, "offsets"),
          _arg(h, row_map, I32, "row_map"), _arg(h, row_src, I32, "row_src"),
          _arg(h, topk_w, F32, "topk_w"), _arg(h, w_gu, BF16, "w_gu"),
          _arg(h, w_down, BF16, "w_down"), _arg(h, au, BF16, "au"), _arg(h, hbuf, BF16, "h"),
          _arg(h, o_perm, BF16, "o_perm"), _arg(h, shared_out, BF16, "shared_out"),
          _arg(h, y, BF16, "y"), _arg(h, arrivals, I32, "arrivals"), _stream(h, stream))


def moe_route(h, shape, topk_idx, counts, offsets, row_map, row_src, ws, stream=None):
    _call("moe_route", h.ptr, ctypes.byref(shape), _arg(h, topk_idx, I32, "topk_idx"),
          _arg(h, counts, I32, "counts"), _arg(h, offsets, I32, "offsets"),
          _arg(h, row_map, I32, "row_map"), _arg(h, row_src, I32, "row_src"),
          _arg(h, ws, None, "ws"), _nbytes(ws), _stream(h, stream))


def moe_grouped_swiglu_fwd_gather(h, shape, x, row_src, offsets, w_gu, w_down, au, hbuf, o_perm,
                                  stream=None):
    _call("moe_grouped_swiglu_fwd_gather", h.ptr, ctypes.byref(shape), _arg(h, x, BF16, "x"),
          _arg(h, row_src, I32, "row_src"), _arg(h, offsets, I32, "offsets"),
          _arg(h, w_gu, BF16, "w_gu"), _arg(h, w_down, BF16, "w_down"), _arg(h, au, BF16, "au"),
          _arg(h, hbuf, BF16, "h"), _arg(h, o_perm, BF16, "o_perm"), _stream(h, stream))


def moe_grouped_swiglu_recompute_gather(h, shape, x, row_src, offsets, w_gu, au, hbuf,
                                        stream=None):
    _call("moe_grouped_swiglu_recompute_gather", h.ptr, ctypes.byref(shape),
          _arg(h, x, BF16, "x"), _arg(h, row_src, I32, "row_src"),
          _arg(h, offsets, I32, "offsets"), _arg(h, w_gu, BF16, "w_gu"), _arg(h, au, BF16, "au"),
          _arg(h, hbuf, BF16, "h"), _stream(h, stream))


def moe_grouped_swiglu_bwd_gather(h, shape, do_perm, x, row_src, au, hbuf, offsets, w_gu, w_down,
                                  dau, dx_perm, dw_gu, dw_down, stream=None):
    _call("moe_grouped_swiglu_bwd_gather", h.ptr, ctypes.byref(shape),
          _arg(h, do_perm, BF16, "do_perm"), _arg(h, x, BF16, "x"),
          _arg(h, row_src, I32, "row_src"), _arg(h, au, BF16, "au"), _arg(h, hbuf, BF16, "h"),
          _arg(h, offsets, I32, "offsets"), _arg(h, w_gu, BF16, "w_gu"),
          _arg(h, w_down, BF16, "w_down"), _arg(h, dau, BF16, "dau"),
          _arg(h, dx_perm, BF16, "dx_perm"), _arg(h, dw_gu, BF16, "dw_gu"),
          _arg(h, dw_down, BF16, "dw_down"), _stream(h, stream))


def moe_unpermute_combine(h, shape, o_perm, row_map, topk_w, shared_out, y, stream=None):
    _call("moe_unpermute_combine", h.ptr, ctypes.byref(shape), _arg(h, o_perm, BF16, "o_perm"),
          _arg(h, row_map, I32, "row_map"), _arg(h, topk_w, F32, "topk_w"),
          _arg(h, shared_out, BF16, "shared_out"), _arg(h, y, BF16, "y"), _stream(h, stream))


def moe_unpermute_combine_bwd(h, shape, dy, o_perm, row_map, topk_w, offsets, counts, do_perm,
                              d_topk_w, stream=None):
    _call("moe_unpermute_combine_bwd", h.ptr, ctypes.byref(shape), _arg(h, dy, BF16, "dy"),
          _arg(h, o_perm, BF16, "o_perm"), _arg(h, row_map, I32, "row_map"),
          _arg(h, topk_w, F32, "topk_w"), _arg(h, offsets, I32, "offsets"),
          _arg(h, counts, I32, "counts"), _arg(h, do_perm, BF16, "do_perm"),
          _arg(h, d_topk_w, F32, "d_topk_w"), _stream(h, stream))


def moe_grouped_swiglu_bwd(h, shape, do_perm, x_perm, au, hbuf, offsets, w_gu, w_down, dau,
                           dx_perm, dw_gu, dw_down, ws, stream=None):
    _call("moe_grouped_swiglu_bwd", h.ptr, ctypes.byref(shape), _arg(h, do_perm, BF16, "do_perm"),
          _arg(h, x_perm, BF16, "x_perm"), _arg(h, au, BF16, "au"), _arg(h, hbuf, BF16, "h"),
          _arg(h, offsets, I32, "offsets"), _arg(h, w_gu, BF16, "w_gu"),
          _arg(h, w_down, BF16, "w_down"), _arg(h, dau, BF16, "dau"),
          _arg(h, dx_perm, BF16, "dx_perm"), _arg(h, dw_gu, BF16, "dw_gu"),
          _arg(h, dw_down, BF16, "dw_down"), _arg(h, ws, None, "ws"), _nbytes(ws),
          _stream(h, stream))


def moe_permute_bwd(h, shape, dx_perm, row_map, dx_router, dx_shared, dx, stream=None):
    _call("moe_permute_bwd", h.ptr, ctypes.byref(shape), _arg(h, dx_perm, BF16, "dx_perm"),
          _arg(h, row_map, I32, "row_map"), _arg(h, dx_router, F32, "dx_router"),
          _arg(h, dx_shared, BF16, "dx_shared"), _arg(h, dx, BF16, "dx"), _stream(h, stream))


def moe_shared_expert_fwd(h, shape, x, w_gu_s, w_d_s, au_s, h_s, o_s, stream=None):
    _call("moe_shared_expert_fwd", h.ptr, ctypes.byref(shape), _arg(h, x, BF16, "x"),
          _arg(h, w_gu_s, BF16, "w_gu_s"), _arg(h, w_d_s, BF16, "w_d_s"),
          _arg(h, au_s, BF16, "au_s"), _arg(h, h_s, BF16, "h_s"), _arg(h, o_s, BF16, "o_s"),
          _stream(h, stream))


def moe_shared_expert_bwd(h, shape, dy, x, au_s, h_s, w_gu_s, w_d_s, dau_s, dx_s, dw_gu_s, dw_d_s,
                          stream=None):
    _call("moe_shared_expert_bwd", h.ptr, ctypes.byref(shape), _arg(h, dy, BF16, "dy"),
          _arg(h, x, BF16, "x"), _arg(h, au_s, BF16, "au_s"), _arg(h, h_s, BF16, "h_s"),
          _arg(h, w_gu_s, BF16, "w_gu_s"), _arg(h, w_d_s, BF16, "w_d_s"),
          _arg(h, dau_s, BF16, "dau_s"), _arg(h, dx_s, BF16, "dx_s"),
          _arg(h, dw_gu_s, BF16, "dw_gu_s"), _arg(h, dw_d_s, BF16, "dw_d_s"), _stream(h, stream))


def moe_permute_router_bwd(h, shape, dx_perm, row_map, d_topk_w, probs, topk_idx, d_probs_aux,
                           w_router, dx_shared, dx, stream=None):
    _call("moe_permute_router_bwd", h.ptr, ctypes.byref(shape), _arg(h, dx_perm, BF16, "dx_perm"),
          _arg(h, row_map, I32, "row_map"), _arg(h, d_topk_w, F32, "d_topk_w"),
          _arg(h, probs, F32, "probs"), _arg(h, topk_idx, I32, "topk_idx"),
          _arg(h, d_probs_aux, F32, "d_probs_aux"), _arg(h, w_router, BF16, "w_router"),
          _arg(h, dx_shared, BF16, "dx_shared"), _arg(h, dx, BF16, "dx"), _stream(h, stream))


def moe_router_topk_bwd(h, shape, d_topk_w, probs, topk_idx, d_probs_aux, x, w_router, dx_router,
                        dw_router, dbias, ws, stream=None):
    _call("moe_router_topk_bwd", h.ptr, ctypes.byref(shape), _arg(h, d_topk_w, F32, "d_topk_w"),
          _arg(h, probs, F32, "probs"), _arg(h, topk_idx, I32, "topk_idx"),
          _arg(h, d_probs_aux, F32, "d_probs_aux"), _arg(h, x, BF16, "x"),
          _arg(h, w_router, BF16, "w_router"), _arg(h, dx_router, F32, "dx_router"),
          _arg(h, dw_router, BF16, "dw_router"), _arg(h, dbias, F32, "dbias"),
          _arg(h, ws, None, "ws"), _nbytes(ws), _stream(h, stream))


def moe_router_load_stats(h, shape, probs, counts, accumulate, stats, ws, stream=None):
    _call("moe_router_load_stats", h.ptr, ctypes.byref(shape), _arg(h, probs, F32, "probs"),
          _arg(h, counts, I32, "counts"), 1 if accumulate else 0, _arg(h, stats, F32, "stats"),
          _arg(h, ws, None, "ws"), _nbytes(ws), _stream(h, stream))


def moe_router_aux_loss(h, shape, stats, n_tokens, alpha, loss, d_probs_aux, stream=None):
    _call("moe_router_aux_loss", h.ptr, ctypes.byref(shape), _arg(h, stats, F32, "stats"),
          int(n_tokens), ctypes.c_float(alpha), _arg(h, loss, F32, "loss"),
          _arg(h, d_probs_aux, F32, "d_probs_aux"), _stream(h, stream))


def moe_mxfp8_quantize(h, inp, axis, q, scales, stream=None):
    rows, cols = inp.shape
    _call("moe_mxfp8_quantize", h.ptr, _arg(h, inp, BF16, "in"), rows, cols, axis,
          _arg(h, q, U8, "q"), _arg(h, scales, U8, "scales"), _stream(h, stream))


def moe_mxfp8_quantize_gemm(h, inp, rows_per_group, q_row, s_row, q_col, s_col, stream=None):
    rows, cols = inp.shape
    _call("moe_mxfp8_quantize_gemm", h.ptr, _arg(h, inp, BF16, "in"), rows, cols, rows_per_group,
          _arg(h, q_row, U8, "q_row"), _arg(h, s_row, U8, "s_row"), _arg(h, q_col, U8, "q_col"),
          _arg(h, s_col, U8, "s_col"), _stream(h, stream))
