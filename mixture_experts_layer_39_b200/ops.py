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


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
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


def max_rows(shape: MoeShape) -> int:
    n = ctypes.c_int64()
    _call("moe_max_rows", ctypes.byref(shape), ctypes.byref(n))
    return n.value


def moe_router_topk(h, shape, x, w_router, bias, route_in, topk_idx, topk_w, probs, logits, ws,
                    stream=None):
    _call("moe_router_topk", h.ptr, ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias),
          _ptr(route_in), _ptr(topk_idx), _ptr(topk_w), _ptr(probs), _ptr(logits), _ptr(ws),
          ws.numel() if ws is not None else 0, _stream(stream))


def moe_permute(h, shape, x, topk_idx, counts, offsets, row_map, x_perm, ws, stream=None):
    _call("moe_permute", h.ptr, ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(counts),
          _ptr(offsets), _ptr(row_map), _ptr(x_perm), _ptr(ws), ws.numel(), _stream(stream))


def moe_permute_noalloc(h, shape, x, topk_idx, counts, offsets, row_map, x_perm, stream=None):
    """moe_permute for callers that cannot supply scratch memory: the library
    uses a fixed 1 MiB array of its own instead of a workspace."""
    _call("moe_permute_noalloc", h.ptr, ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(counts),
          _ptr(offsets), _ptr(row_map), _ptr(x_perm), _stream(stream))


def moe_grouped_swiglu_fwd(h, shape, x_perm, offsets, w_gu, w_down, au, hbuf, o_perm, ws,
                           stream=None):
    _call("moe_grouped_swiglu_fwd", h.ptr, ctypes.byref(shape), _ptr(x_perm), _ptr(offsets),
          _ptr(w_gu), _ptr(w_down), _ptr(au), _ptr(hbuf), _ptr(o_perm), _ptr(ws),
          ws.numel() if ws is not None else 0, _stream(stream))


def moe_grouped_swiglu_recompute(h, shape, x_perm, offsets, w_gu, au, hbuf, ws, stream=None):
    _call("moe_grouped_swiglu_recompute", h.ptr, ctypes.byref(shape), _ptr(x_perm), _ptr(offsets),
          _ptr(w_gu), _ptr(au), _ptr(hbuf), _ptr(ws), ws.numel() if ws is not None else 0,
          _stream(stream))


def moe_route(h, shape, topk_idx, counts, offsets, row_map, row_src, ws, stream=None):
    _call("moe_route", h.ptr, ctypes.byref(shape), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
          _ptr(row_map), _ptr(row_src), _ptr(ws), ws.numel(), _stream(stream))


def moe_grouped_swiglu_fwd_gather(h, shape, x, row_src, offsets, w_gu, w_down, au, hbuf, o_perm,
                                  stream=None):
    _call("moe_grouped_swiglu_fwd_gather", h.ptr, ctypes.byref(shape), _ptr(x), _ptr(row_src),
          _ptr(offsets), _ptr(w_gu), _ptr(w_down), _ptr(au), _ptr(hbuf), _ptr(o_perm),
          _stream(stream))


def moe_grouped_swiglu_recompute_gather(h, shape, x, row_src, offsets, w_gu, au, hbuf,
                                        stream=None):
    _call("moe_grouped_swiglu_recompute_gather", h.ptr, ctypes.byref(shape), _ptr(x),
          _ptr(row_src), _ptr(offsets), _ptr(w_gu), _ptr(au), _ptr(hbuf), _stream(stream))


def moe_grouped_swiglu_bwd_gather(h, shape, do_perm, x, row_src, au, hbuf, offsets, w_gu, w_down,
                                  dau, dx_perm, dw_gu, dw_down, stream=None):
    _call("moe_grouped_swiglu_bwd_gather", h.ptr, ctypes.byref(shape), _ptr(do_perm), _ptr(x),
          _ptr(row_src), _ptr(au), _ptr(hbuf), _ptr(offsets), _ptr(w_gu), _ptr(w_down),
          _ptr(dau), _ptr(dx_perm), _ptr(dw_gu), _ptr(dw_down), _stream(stream))


def moe_unpermute_combine(h, shape, o_perm, row_map, topk_w, shared_out, y, stream=None):
    _call("moe_unpermute_combine", h.ptr, ctypes.byref(shape), _ptr(o_perm), _ptr(row_map),
          _ptr(topk_w), _ptr(shared_out), _ptr(y), _stream(stream))


def moe_unpermute_combine_bwd(h, shape, dy, o_perm, row_map, topk_w, offsets, counts, do_perm,
                              d_topk_w, stream=None):
    _call("moe_unpermute_combine_bwd", h.ptr, ctypes.byref(shape), _ptr(dy), _ptr(o_perm),
          _ptr(row_map), _ptr(topk_w), _ptr(offsets), _ptr(counts), _ptr(do_perm),
          _ptr(d_topk_w), _stream(stream))


def moe_grouped_swiglu_bwd(h, shape, do_perm, x_perm, au, hbuf, offsets, w_gu, w_down, dau,
                           dx_perm, dw_gu, dw_down, ws, stream=None):
    _call("moe_grouped_swiglu_bwd", h.ptr, ctypes.byref(shape), _ptr(do_perm), _ptr(x_perm),
          _ptr(au), _ptr(hbuf), _ptr(offsets), _ptr(w_gu), _ptr(w_down), _ptr(dau),
          _ptr(dx_perm), _ptr(dw_gu), _ptr(dw_down), _ptr(ws),
          ws.numel() if ws is not None else 0, _stream(stream))


def moe_permute_bwd(h, shape, dx_perm, row_map, dx_router, dx_shared, dx, stream=None):
    _call("moe_permute_bwd", h.ptr, ctypes.byref(shape), _ptr(dx_perm), _ptr(row_map),
          _ptr(dx_router), _ptr(dx_shared), _ptr(dx), _stream(stream))


def moe_shared_expert_fwd(h, shape, x, w_gu_s, w_d_s, au_s, h_s, o_s, stream=None):
    _call("moe_shared_expert_fwd", h.ptr, ctypes.byref(shape), _ptr(x), _ptr(w_gu_s), _ptr(w_d_s),
          _ptr(au_s), _ptr(h_s), _ptr(o_s), _stream(stream))


def moe_shared_expert_bwd(h, shape, dy, x, au_s, h_s, w_gu_s, w_d_s, dau_s, dx_s, dw_gu_s, dw_d_s,
                          stream=None):
    _call("moe_shared_expert_bwd", h.ptr, ctypes.byref(shape), _ptr(dy), _ptr(x), _ptr(au_s),
          _ptr(h_s), _ptr(w_gu_s), _ptr(w_d_s), _ptr(dau_s), _ptr(dx_s), _ptr(dw_gu_s),
          _ptr(dw_d_s), _stream(stream))


def moe_permute_router_bwd(h, shape, dx_perm, row_map, d_topk_w, probs, topk_idx, d_probs_aux,
                           w_router, dx_shared, dx, stream=None):
    _call("moe_permute_router_bwd", h.ptr, ctypes.byref(shape), _ptr(dx_perm), _ptr(row_map),
          _ptr(d_topk_w), _ptr(probs), _ptr(topk_idx), _ptr(d_probs_aux), _ptr(w_router),
          _ptr(dx_shared), _ptr(dx), _stream(stream))


def moe_router_topk_bwd(h, shape, d_topk_w, probs, topk_idx, d_probs_aux, x, w_router, dx_router,
                        dw_router, dbias, ws, stream=None):
    _call("moe_router_topk_bwd", h.ptr, ctypes.byref(shape), _ptr(d_topk_w), _ptr(probs),
          _ptr(topk_idx), _ptr(d_probs_aux), _ptr(x), _ptr(w_router), _ptr(dx_router),
          _ptr(dw_router), _ptr(dbias), _ptr(ws), ws.numel(), _stream(stream))


def moe_router_load_stats(h, shape, probs, counts, accumulate, stats, ws, stream=None):
    _call("moe_router_load_stats", h.ptr, ctypes.byref(shape), _ptr(probs), _ptr(counts),
          1 if accumulate else 0, _ptr(stats), _ptr(ws), ws.numel(), _stream(stream))


def moe_router_aux_loss(h, shape, stats, n_tokens, alpha, loss, d_probs_aux, stream=None):
    _call("moe_router_aux_loss", h.ptr, ctypes.byref(shape), _ptr(stats), int(n_tokens),
          ctypes.c_float(alpha), _ptr(loss), _ptr(d_probs_aux), _stream(stream))


def moe_mxfp8_quantize(h, inp, axis, q, scales, stream=None):
    rows, cols = inp.shape
    _call("moe_mxfp8_quantize", h.ptr, _ptr(inp), rows, cols, axis, _ptr(q), _ptr(scales),
          _stream(stream))
