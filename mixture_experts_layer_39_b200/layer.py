"""One training step of the dropless MoE expert layer through the C ABI.

MoELayer owns the device buffers of one shape (PyTorch allocates them; the
library never does) and issues the calls of a forward and a backward pass
in order on the current stream:

  forward : moe_router_topk -> moe_permute -> moe_grouped_swiglu_fwd
            -> moe_unpermute_combine
  backward: moe_unpermute_combine_bwd -> moe_router_topk_bwd
            -> moe_grouped_swiglu_bwd -> moe_permute_router_bwd  (E <= 64)
            or, for E above 64 (router products on the tensor cores),
            moe_router_topk_bwd writes dX_router and
            moe_permute_bwd adds it.

With shared_ff > 0 a shared expert runs on every token
(moe_shared_expert_fwd / _bwd); its output joins the combine and its input
gradient the permute backward.

With fuse_combine=True (bf16) the weighted unpermute-combine runs inside
the down projection's epilogue (moe_permute_src ->
moe_grouped_swiglu_fwd_combine); y has the same bits, and a shared expert's
forward runs before the routed experts so that its output joins there.

With gather=True (bf16) no permuted copy of x is written: moe_route
produces the routing metadata and row_src, and the expert GEMMs that read
routed rows of x gather them from x itself (the *_gather entry points).

With recompute=True the forward keeps no [A | U] (H is only a transient
input to the down projection) and the backward first recomputes both
(moe_grouped_swiglu_recompute): only x_perm and O_perm live from the forward
to the backward.

With aux_alpha > 0 the forward also forms the router's load statistics and
the load-balancing loss (moe_router_load_stats -> moe_router_aux_loss) and
the backward adds the loss's gradient in the router backward.

Nothing in a step copies to the host or synchronises.
"""
from __future__ import annotations

from typing import Callable

import torch

from . import ops
from ._lib import MOE_DTYPE_BF16, MOE_DTYPE_MXFP8

BF16 = torch.bfloat16
I32 = torch.int32
F32 = torch.float32


class MoELayer:
    def __init__(self, T, d, f, E, k, device="cuda", renorm=False, keep_logits=False,
                 handle: ops.Handle | None = None, dtype: str = "bf16",
                 fuse_router_dx: bool | None = None, aux_alpha: float = 0.0,
                 aux_reduce: Callable | None = None, shared_ff: int = 0,
                 recompute: bool = False, gather: bool = False, fuse_combine: bool = False):
        """dtype: "bf16", or "mxfp8" for E4M3/E8M0 expert GEMM operands (the
        library then also aligns expert segments to 128 rows).
        fuse_router_dx: add the router's input gradient inside the permute
        backward (default, and only possible, for E <= 64); False keeps the
        separate [T, d] fp32 dX_router buffer.
        aux_alpha: weight of the load-balancing loss (0: none).  aux_reduce:
        optional callable(stats) -> n_tokens that sums the statistics over
        ranks in place and returns the global batch's token count
        (replicas.global_stats_reducer), for balancing over the global batch.
        shared_ff: hidden size of a shared expert every token passes through
        (0: none); its weights are passed to forward/backward/step as
        w_gu_s [2*shared_ff, d] and w_d_s [d, shared_ff].
        recompute: activation recompute of the expert gate/up GEMM (self.au
        and self.h then only hold values between the recompute and the end
        of the backward, and can be shared between layers)."""
        self.recompute = bool(recompute)
        self.gather = bool(gather)
        self.fuse_combine = bool(fuse_combine)
        if self.gather and dtype != "bf16":
            raise ValueError("the gather forms are bf16 only")
        if self.fuse_combine and (dtype != "bf16" or self.gather):
            raise ValueError("the fused combine is bf16 only, with a permuted copy of x")
        self._x = None  # x of the current step (gather forms read it in the GEMMs)
        self.T, self.d, self.f, self.E, self.k = T, d, f, E, k
        dev = torch.device(device)
        self.device = dev
        self.handle = handle if handle is not None else ops.Handle(dev.index or 0)
        self.dtype = dtype
        code = {"bf16": MOE_DTYPE_BF16, "mxfp8": MOE_DTYPE_MXFP8}[dtype]
        self.shape = ops.make_shape(T, d, f, E, k, code, renorm)
        M = ops.max_rows(self.shape)
        self.M_cap = M
        z = lambda *s, dt=BF16: torch.empty(*s, dtype=dt, device=dev)
        self.ws = torch.empty(self.handle.workspace_size(self.shape), dtype=torch.uint8, device=dev)
        # forward state
        self.idx, self.w = z(T, k, dt=I32), z(T, k, dt=F32)
        self.probs = z(T, E, dt=F32)
        self.logits = z(T, E, dt=F32) if keep_logits else None
        self.counts, self.offsets = z(E, dt=I32), z(E + 1, dt=I32)
        self.row_map = z(T, k, dt=I32)
        self.x_perm = None if self.gather else z(M, d)
        self.row_src = z(M, dt=I32) if (self.gather or self.fuse_combine) else None
        # per (token, 256-column tile) arrival counts of the fused combine:
        # zero here, left zero by every completed call
        self.arrivals = (torch.zeros(T, (d + 255) // 256, dtype=I32, device=dev)
                         if self.fuse_combine else None)
        self.au, self.h = z(M, 2 * f), z(M, f)
        self.o_perm, self.y = z(M, d), z(T, d)
        # backward state
        self.do_perm, self.dw = z(M, d), z(T, k, dt=F32)
        self.dau, self.dx_perm = z(M, 2 * f), z(M, d)
        self.dw_gu, self.dw_d = z(E, 2 * f, d), z(E, d, f)
        if fuse_router_dx is None:
            fuse_router_dx = E <= 64
        if fuse_router_dx and E > 64:
            raise ValueError("the fused router input gradient needs E <= 64")
        self.fuse_router_dx = fuse_router_dx
        self.dx_router = None if fuse_router_dx else z(T, d, dt=F32)
        self.dw_r = z(E, d)
        self.db = z(E, dt=F32)
        self.dx = z(T, d)
        # load-balancing loss
        self.aux_alpha = float(aux_alpha)
        self.aux_reduce = aux_reduce
        self.stats = z(2 * E, dt=F32)
        self.aux_loss = z(1, dt=F32)
        self.dprob_aux = z(E, dt=F32) if self.aux_alpha > 0 else None
        # shared expert
        self.shared_ff = int(shared_ff)
        if self.shared_ff > 0:
            fs = self.shared_ff
            self.shared_shape = ops.make_shape(T, d, fs, 1, 1, MOE_DTYPE_BF16, False)
            self.au_s, self.h_s, self.o_s = z(T, 2 * fs), z(T, fs), z(T, d)
            self.dau_s, self.dx_s = z(T, 2 * fs), z(T, d)
            self.dw_gu_s, self.dw_d_s = z(2 * fs, d), z(d, fs)
        else:
            self.o_s = self.dx_s = None

    # ------------------------------------------------------------- forward
    def router(self, x, w_r, bias=None, route=None, stream=None):
        ops.moe_router_topk(self.handle, self.shape, x, w_r, bias, route, self.idx, self.w,
                            self.probs, self.logits, self.ws, stream)

    def permute(self, x, stream=None):
        self._x = x
        if self.gather:
            ops.moe_route(self.handle, self.shape, self.idx, self.counts, self.offsets,
                          self.row_map, self.row_src, self.ws, stream)
            return
        if self.fuse_combine:
            ops.moe_permute_src(self.handle, self.shape, x, self.idx, self.counts, self.offsets,
                                self.row_map, self.row_src, self.x_perm, self.ws, stream)
            return
        ops.moe_permute(self.handle, self.shape, x, self.idx, self.counts, self.offsets,
                        self.row_map, self.x_perm, self.ws, stream)

    def experts_fwd(self, w_gu, w_d, stream=None):
        au = None if self.recompute else self.au
        if self.gather:
            ops.moe_grouped_swiglu_fwd_gather(self.handle, self.shape, self._x, self.row_src,
                                              self.offsets, w_gu, w_d, au, self.h, self.o_perm,
                                              stream)
            return
        if self.fuse_combine:  # y too (a shared expert's output must be ready)
            ops.moe_grouped_swiglu_fwd_combine(self.handle, self.shape, self.x_perm, self.offsets,
                                               self.row_map, self.row_src, self.w, w_gu, w_d, au,
                                               self.h, self.o_perm, self.o_s, self.y,
                                               self.arrivals, stream)
            return
        ops.moe_grouped_swiglu_fwd(self.handle, self.shape, self.x_perm, self.offsets, w_gu, w_d,
                                   au, self.h, self.o_perm, self.ws, stream)

    def shared_fwd(self, x, w_gu_s, w_d_s, stream=None):
        ops.moe_shared_expert_fwd(self.handle, self.shared_shape, x, w_gu_s, w_d_s, self.au_s,
                                  self.h_s, self.o_s, stream)

    def combine(self, stream=None):
        ops.moe_unpermute_combine(self.handle, self.shape, self.o_perm, self.row_map, self.w,
                                  self.o_s, self.y, stream)

    def load_stats(self, accumulate=False, stream=None):
        """[counts | sum_t probs] of this batch into self.stats (added when
        accumulate)."""
        ops.moe_router_load_stats(self.handle, self.shape, self.probs, self.counts, accumulate,
                                  self.stats, self.ws, stream)

    def balance_loss(self, stats=None, n_tokens=None, stream=None):
        """Load-balancing loss of `stats` (default self.stats) over n_tokens
        tokens (default T) into self.aux_loss, and its per-expert
        probability gradient into self.dprob_aux."""
        ops.moe_router_aux_loss(self.handle, self.shape, self.stats if stats is None else stats,
                                self.T if n_tokens is None else n_tokens, self.aux_alpha,
                                self.aux_loss, self.dprob_aux, stream)

    def _need_shared(self, w_gu_s, w_d_s):
        if self.shared_ff > 0 and (w_gu_s is None or w_d_s is None):
            raise ValueError("this layer has a shared expert: pass w_gu_s and w_d_s")

    def forward(self, x, w_r, w_gu, w_d, bias=None, route=None, stream=None, w_gu_s=None,
                w_d_s=None):
        self._need_shared(w_gu_s, w_d_s)
        self.router(x, w_r, bias, route, stream)
        self.permute(x, stream)
        if self.aux_alpha > 0:
            self.load_stats(False, stream)
            n = self.aux_reduce(self.stats) if self.aux_reduce is not None else self.T
            self.balance_loss(None, n, stream)
        if self.fuse_combine:
            if self.shared_ff > 0:
                self.shared_fwd(x, w_gu_s, w_d_s, stream)
            self.experts_fwd(w_gu, w_d, stream)  # writes y
            return self.y
        self.experts_fwd(w_gu, w_d, stream)
        if self.shared_ff > 0:
            self.shared_fwd(x, w_gu_s, w_d_s, stream)
        self.combine(stream)
        return self.y

    # ------------------------------------------------------------- backward
    def combine_bwd(self, dy, stream=None):
        ops.moe_unpermute_combine_bwd(self.handle, self.shape, dy, self.o_perm, self.row_map,
                                      self.w, self.offsets, self.counts, self.do_perm, self.dw,
                                      stream)

    def router_bwd(self, x, w_r, stream=None):
        ops.moe_router_topk_bwd(self.handle, self.shape, self.dw, self.probs, self.idx,
                                self.dprob_aux, x, w_r, self.dx_router, self.dw_r, self.db,
                                self.ws, stream)

    def experts_bwd(self, w_gu, w_d, stream=None):
        if self.gather:
            if self.recompute:
                ops.moe_grouped_swiglu_recompute_gather(self.handle, self.shape, self._x,
                                                        self.row_src, self.offsets, w_gu, self.au,
                                                        self.h, stream)
            ops.moe_grouped_swiglu_bwd_gather(self.handle, self.shape, self.do_perm, self._x,
                                              self.row_src, self.au, self.h, self.offsets, w_gu,
                                              w_d, self.dau, self.dx_perm, self.dw_gu, self.dw_d,
                                              stream)
            return
        if self.recompute:
            ops.moe_grouped_swiglu_recompute(self.handle, self.shape, self.x_perm, self.offsets,
                                             w_gu, self.au, self.h, self.ws, stream)
        ops.moe_grouped_swiglu_bwd(self.handle, self.shape, self.do_perm, self.x_perm, self.au,
                                   self.h, self.offsets, w_gu, w_d, self.dau, self.dx_perm,
                                   self.dw_gu, self.dw_d, self.ws, stream)

    def permute_bwd(self, w_r=None, stream=None):
        if self.fuse_router_dx:
            if w_r is None:
                raise ValueError("the fused permute backward needs w_r")
            ops.moe_permute_router_bwd(self.handle, self.shape, self.dx_perm, self.row_map,
                                       self.dw, self.probs, self.idx, self.dprob_aux, w_r,
                                       self.dx_s, self.dx, stream)
        else:
            ops.moe_permute_bwd(self.handle, self.shape, self.dx_perm, self.row_map,
                                self.dx_router, self.dx_s, self.dx, stream)

    def shared_bwd(self, dy, x, w_gu_s, w_d_s, stream=None):
        ops.moe_shared_expert_bwd(self.handle, self.shared_shape, dy, x, self.au_s, self.h_s,
                                  w_gu_s, w_d_s, self.dau_s, self.dx_s, self.dw_gu_s,
                                  self.dw_d_s, stream)

    def backward(self, dy, x, w_r, w_gu, w_d, stream=None, w_gu_s=None, w_d_s=None):
        self._need_shared(w_gu_s, w_d_s)
        self._x = x
        self.combine_bwd(dy, stream)
        self.router_bwd(x, w_r, stream)
        self.experts_bwd(w_gu, w_d, stream)
        if self.shared_ff > 0:
            self.shared_bwd(dy, x, w_gu_s, w_d_s, stream)
        self.permute_bwd(w_r, stream)
        return self.dx

    def step(self, x, w_r, w_gu, w_d, dy, bias=None, route=None, stream=None, w_gu_s=None,
             w_d_s=None):
        self.forward(x, w_r, w_gu, w_d, bias, route, stream, w_gu_s, w_d_s)
        self.backward(dy, x, w_r, w_gu, w_d, stream, w_gu_s, w_d_s)
