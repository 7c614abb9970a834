"""CPU oracle for the dropless MoE expert layer (router, routing metadata,
permute, SwiGLU experts, combine, and the explicit backward).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py may import this module.  The
product path (the C-ABI library and its Python binding) never calls it and
shares no code with it.

Plain NumPy, float64 arithmetic by default.  Values are rounded to bf16
(round-to-nearest-even from fp32) only where the layer's definition stores a
bf16 tensor: x_perm, AU, H, O_perm, y, dO_perm, dAU, dX_perm, dX and the
weight gradients.  `rnd=None` switches all rounding off (used for the
finite-difference checks).

Sources.  The pages describe the layer in words only; they give no formula.
  * Router: "a router network computes a distribution over experts for each
    token and picks the k highest" -- discosf.com article on Olmo-core 3,
    section 1.1 (sparse computation) and section 2.1 (how a token is sent to
    experts in one forward pass).
  * Permutation index and restore: same article, section 2.1 (the routing
    result becomes a permutation index; tokens are regrouped per expert,
    processed, and put back in their original order).
  * Rowwise permute straight into each expert's input buffer, GPU-resident
    routing metadata, grouped GEMM over all experts: Olmo-core 3
    introduction page (meetcoding.cn), section 2 "three parallelisms plus
    three routing optimisations".
  * Dropless (no token is dropped when an expert is over-subscribed):
    vibecoding.ru news item on Olmo-core 3, paragraph on grouped_gemm.
Readings taken where the pages are silent (each also listed in the design
notes): softmax over all E experts in full precision, top-k chosen on the
logit with ties to the lower expert index, slots ordered by descending
logit; gate weight = the selected probability, not renormalised unless
asked; expert FFN = SwiGLU, H = silu(x Wg^T) * (x Wu^T), O = H Wd^T, no
biases; expert segments start at multiples of 32 rows with zero pad rows;
within an expert, rows are in ascending (token, slot) order; the combine
sums in slot order and rounds once.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
SEG_ALIGN = 32


# --------------------------------------------------------------------------
# bf16 storage rounding
# --------------------------------------------------------------------------
def bf16_round(a):
    """Round to the nearest bf16 value (ties to even), going through fp32.

    bf16 keeps the top 16 bits of an IEEE fp32 word; rounding adds half an
    ulp of the kept part (0x7FFF) plus the kept LSB (ties to even) and
    truncates.  Returns float64 holding bf16-representable values.
    """
    a32 = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = a32.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(F64)


def _ident(a):
    return np.asarray(a, dtype=F64)


def _r(rnd):
    return _ident if rnd is None else rnd


# --------------------------------------------------------------------------
# Router (top-k softmax)
# --------------------------------------------------------------------------
def router_logits(x, w_r, bias=None):
    """L[t, e] = sum_i x[t, i] * W_r[e, i] (+ b[e])."""
    L = np.asarray(x, F64) @ np.asarray(w_r, F64).T
    if bias is not None:
        L = L + np.asarray(bias, F64)[None, :]
    return L


def softmax(L):
    """p[t, e] = exp(L[t, e] - max_e L[t]) / sum_e' exp(L[t, e'] - max)."""
    L = np.asarray(L, F64)
    z = np.exp(L - L.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def topk_select(L, k):
    """Indices of the k largest logits per row.

    Ties go to the lower expert index; the k slots are ordered by
    descending logit, then ascending index.  A stable sort of -L gives
    exactly that order.
    """
    L = np.asarray(L)
    return np.argsort(-L, axis=1, kind="stable")[:, :k].astype(np.int64)


def gate_weights(probs, idx, renorm=False):
    """w[t, j] = p[t, idx[t, j]]; divided by sum_j of those when renorm."""
    w = np.take_along_axis(np.asarray(probs, F64), np.asarray(idx), axis=1)
    if renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return w


def router_topk(x, w_r, k, bias=None, renorm=False, route=None):
    """Router forward.  `route` (optional [T, k] ids) replaces the top-k
    choice, as in the pages' random-routing benchmark mode; the gate
    weights still come from the router's probabilities."""
    L = router_logits(x, w_r, bias)
    p = softmax(L)
    idx = topk_select(L, k) if route is None else np.asarray(route, np.int64)
    w = gate_weights(p, idx, renorm)
    return {"logits": L, "probs": p, "idx": idx, "w": w}


# --------------------------------------------------------------------------
# Routing metadata and permute
# --------------------------------------------------------------------------
def routing_metadata(idx, E, align=SEG_ALIGN):
    """counts[e], padded offsets[E+1], row_map[T, k].

    Expert-major order; inside one expert the (t, j) entries keep their
    flat order t*k + j (a stable argsort of the flat expert ids).  Each
    expert's segment starts at a multiple of `align` rows.
    """
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    padded = (counts + align - 1) // align * align
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(padded)
    order = np.argsort(flat, kind="stable")
    pos = np.empty_like(order)
    pos[order] = np.arange(flat.size)
    first = np.zeros(E + 1, np.int64)
    first[1:] = np.cumsum(counts)
    rank = pos - first[flat]
    row_map = (offsets[flat] + rank).reshape(T, k)
    return {"counts": counts, "offsets": offsets, "row_map": row_map,
            "M_pad": int(offsets[-1])}


def permute(x, row_map, M_pad, rnd=bf16_round):
    """x_perm[row_map[t, j]] = x[t]; every other row is zero."""
    x = np.asarray(x, F64)
    T, k = row_map.shape
    x_perm = np.zeros((M_pad, x.shape[1]), F64)
    x_perm[row_map.reshape(-1)] = np.repeat(x, k, axis=0)
    return _r(rnd)(x_perm)


# --------------------------------------------------------------------------
# Expert FFN (SwiGLU), forward
# --------------------------------------------------------------------------
def silu(z):
    return z / (1.0 + np.exp(-z))


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def expert_ffn_fwd(x_perm, offsets, counts, w_gu, w_d, rnd=bf16_round,
                   expert_fn=None):
    """Per-expert loop: for the rows of expert e,
        A = X Wg[e]^T, U = X Wu[e]^T       (Wg = rows 0..f-1 of W_gu[e])
        AU = bf16([A, U])                   (saved for the backward)
        H = bf16(silu(A) * U)               (from the unrounded A, U)
        O = bf16(H W_d[e]^T)
    Pad rows stay zero.  `expert_fn(e, X) -> O` replaces the SwiGLU
    (identity-expert checks)."""
    R = _r(rnd)
    x_perm = np.asarray(x_perm, F64)
    M_pad, d = x_perm.shape
    E = len(counts)
    if expert_fn is not None:
        O = np.zeros((M_pad, d), F64)
        for e in range(E):
            r0, r1 = offsets[e], offsets[e] + counts[e]
            O[r0:r1] = R(expert_fn(e, x_perm[r0:r1]))
        return {"AU": None, "H": None, "O": O}
    f = w_gu.shape[1] // 2
    AU = np.zeros((M_pad, 2 * f), F64)
    H = np.zeros((M_pad, f), F64)
    O = np.zeros((M_pad, d), F64)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e] + counts[e]
        if r1 == r0:
            continue
        X = x_perm[r0:r1]
        Wg = np.asarray(w_gu[e, :f], F64)
        Wu = np.asarray(w_gu[e, f:], F64)
        A = X @ Wg.T
        U = X @ Wu.T
        AU[r0:r1, :f] = R(A)
        AU[r0:r1, f:] = R(U)
        H[r0:r1] = R(silu(A) * U)
        O[r0:r1] = R(H[r0:r1] @ np.asarray(w_d[e], F64).T)
    return {"AU": AU, "H": H, "O": O}


# --------------------------------------------------------------------------
# Combine (unpermute x gate weight)
# --------------------------------------------------------------------------
def combine(O, row_map, w, rnd=bf16_round, shared=None):
    """y[t] = bf16( sum_j w[t, j] * O[row_map[t, j]] + shared[t] ), summed in
    slot order, the shared expert's output (when given) last."""
    O = np.asarray(O, F64)
    w = np.asarray(w, F64)
    T, k = row_map.shape
    acc = np.zeros((T, O.shape[1]), F64)
    for j in range(k):
        acc = acc + w[:, j:j + 1] * O[row_map[:, j]]
    if shared is not None:
        acc = acc + np.asarray(shared, F64)
    return _r(rnd)(acc)


# --------------------------------------------------------------------------
# Backward
# --------------------------------------------------------------------------
def combine_bwd(dy, O, row_map, w, M_pad, rnd=bf16_round):
    """dO[row_map[t, j]] = bf16(w[t, j] * dY[t]) (pad rows zero);
    dw[t, j] = sum_i dY[t, i] * O[row_map[t, j], i]."""
    dy = np.asarray(dy, F64)
    O = np.asarray(O, F64)
    w = np.asarray(w, F64)
    T, k = row_map.shape
    dO = np.zeros((M_pad, dy.shape[1]), F64)
    dw = np.zeros((T, k), F64)
    for j in range(k):
        rows = row_map[:, j]
        dO[rows] = w[:, j:j + 1] * dy
        dw[:, j] = np.sum(dy * O[rows], axis=1)
    return {"dO": _r(rnd)(dO), "dw": dw}


def expert_ffn_bwd(dO, x_perm, AU, H, offsets, counts, w_gu, w_d,
                   rnd=bf16_round):
    """For the rows of expert e (A, U taken from the saved AU):
        dH  = dO W_d[e]                               (fp accumulate)
        s   = sigmoid(A)
        dA  = dH * U * s * (1 + A (1 - s))            d silu(A) U / dA
        dU  = dH * A * s                              = dH * silu(A)
        dAU = bf16([dA, dU])
        dW_d[e]  = bf16(dO^T H)
        dX_perm  = bf16(dAU W_gu[e])
        dW_gu[e] = bf16(dAU^T X)
    Experts with no rows get zero weight gradients."""
    R = _r(rnd)
    dO = np.asarray(dO, F64)
    x_perm = np.asarray(x_perm, F64)
    AU = np.asarray(AU, F64)
    H = np.asarray(H, F64)
    E, two_f, d = w_gu.shape
    f = two_f // 2
    M_pad = x_perm.shape[0]
    dAU = np.zeros((M_pad, 2 * f), F64)
    dX = np.zeros((M_pad, d), F64)
    dW_gu = np.zeros((E, 2 * f, d), F64)
    dW_d = np.zeros((E, d, f), F64)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e] + counts[e]
        if r1 == r0:
            continue
        dOe = dO[r0:r1]
        Wd = np.asarray(w_d[e], F64)
        dH = dOe @ Wd
        A = AU[r0:r1, :f]
        U = AU[r0:r1, f:]
        s = sigmoid(A)
        dA = dH * U * s * (1.0 + A * (1.0 - s))
        dU = dH * A * s
        dAU[r0:r1, :f] = R(dA)
        dAU[r0:r1, f:] = R(dU)
        dW_d[e] = R(dOe.T @ H[r0:r1])
        dX[r0:r1] = R(dAU[r0:r1] @ np.asarray(w_gu[e], F64))
        dW_gu[e] = R(dAU[r0:r1].T @ x_perm[r0:r1])
    return {"dAU": dAU, "dX_perm": dX, "dW_gu": dW_gu, "dW_d": dW_d}


def router_bwd(dw, probs, idx, x, w_r, renorm=False, rnd=bf16_round, dprob_aux=None):
    """Gradient through the selected probabilities (top-k itself is
    piecewise constant).
        renorm: w_j = p_j / S, S = sum_j p_j  =>  g_j = (dw_j - sum_i dw_i w_i) / S
        dp[t, idx[t, j]] = g[t, j], zero elsewhere
        dp[t, e] += dprob_aux[e]          (load-balancing loss, when given)
        dL = p * (dp - sum_e p dp)                   softmax backward
        dX_router = dL W_r     (kept unrounded; added into dX before rounding)
        dW_r = bf16(dL^T x),  db = sum_t dL
    """
    dw = np.asarray(dw, F64)
    p = np.asarray(probs, F64)
    idx = np.asarray(idx, np.int64)
    T, E = p.shape
    g = dw
    if renorm:
        psel = np.take_along_axis(p, idx, axis=1)
        S = psel.sum(axis=1, keepdims=True)
        wv = psel / S
        g = (dw - np.sum(dw * wv, axis=1, keepdims=True)) / S
    dp = np.zeros((T, E), F64)
    np.put_along_axis(dp, idx, g, axis=1)
    if dprob_aux is not None:
        dp = dp + np.asarray(dprob_aux, F64)[None, :]
    dL = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    dx_router = dL @ np.asarray(w_r, F64)
    dw_r = _r(rnd)(dL.T @ np.asarray(x, F64))
    db = dL.sum(axis=0)
    return {"dL": dL, "dx_router": dx_router, "dw_r": dw_r, "db": db}


# --------------------------------------------------------------------------
# Load balancing.  The pages say that every engineered MoE framework adds a
# load-balancing auxiliary loss (or a capacity limit) so that a few hot
# experts do not take most tokens, that its weight should start small
# (e.g. 0.001) and be tuned from the spread of expert load (discosf.com
# article on Olmo-core 3, sections 2.2 and 4.3), and that the v2 router
# balances load over the global batch (Olmo-core 3 introduction page,
# meetcoding.cn, section 4 "production-friendly details").  They give no
# formula; the reading here is the Switch-Transformer loss over the k routed
# slots, with the statistics kept as sums so that they can be added over
# micro-batches and ranks before the loss is formed.

def router_load_stats(probs, counts):
    """Per-expert statistics of one batch:
        n[e]    = counts[e]          routed (token, slot) pairs of expert e
        psum[e] = sum_t p[t, e]      router probability mass of expert e
    Returned as one float64 vector [n | psum] of length 2E."""
    p = np.asarray(probs, F64)
    return np.concatenate([np.asarray(counts, F64), p.sum(axis=0)])


def router_aux_loss(stats, n_tokens, k, alpha):
    """Load-balancing loss from (possibly summed) statistics [n | psum]:
        f_e = n[e] / (n_tokens k)      share of the routed slots
        P_e = psum[e] / n_tokens       mean router probability
        loss = alpha E sum_e f_e P_e
    f_e is piecewise constant in the router logits, so the gradient reaches
    the probabilities only:  d loss / d p[t, e] = alpha E f_e / n_tokens, the
    same for every token (returned as the per-expert vector `dprob`)."""
    stats = np.asarray(stats, F64)
    E = stats.size // 2
    n, psum = stats[:E], stats[E:]
    f = n / (n_tokens * k)
    P = psum / n_tokens
    loss = alpha * E * float(np.sum(f * P))
    dprob = alpha * E * f / n_tokens
    return loss, dprob


def permute_bwd(dX_perm, row_map, dx_router=None, rnd=bf16_round, dx_shared=None):
    """dX[t] = bf16( sum_j dX_perm[row_map[t, j]] + dX_router[t] + dX_shared[t] ),
    slot order, then the router's and the shared expert's terms (when given)."""
    dX_perm = np.asarray(dX_perm, F64)
    T, k = row_map.shape
    acc = np.zeros((T, dX_perm.shape[1]), F64)
    for j in range(k):
        acc = acc + dX_perm[row_map[:, j]]
    if dx_router is not None:
        acc = acc + np.asarray(dx_router, F64)
    if dx_shared is not None:
        acc = acc + np.asarray(dx_shared, F64)
    return _r(rnd)(acc)


# --------------------------------------------------------------------------
# Shared expert.  The pages list shared experts among the v2 router's
# features (Olmo-core 3 introduction page, meetcoding.cn, section 4,
# configuration templates) without defining them.  Reading: one more SwiGLU
# expert with its own weights W_gu_s [2 f_s, d], W_d_s [d, f_s] that every
# token passes through, its output added to the routed experts' combine with
# weight one (so its output gradient is dY itself).  It is the expert FFN
# above applied to one group holding all T tokens in token order.

def shared_expert_fwd(x, w_gu_s, w_d_s, rnd=bf16_round):
    """AU_s, H_s, O_s of the shared expert over all tokens."""
    x = np.asarray(x, F64)
    T = x.shape[0]
    return expert_ffn_fwd(x, np.array([0, T]), np.array([T]), np.asarray(w_gu_s)[None],
                          np.asarray(w_d_s)[None], rnd)


def shared_expert_bwd(dy, x, AU_s, H_s, w_gu_s, w_d_s, rnd=bf16_round):
    """dAU_s, dX_s (= bf16(dAU_s W_gu_s)), dW_gu_s, dW_d_s from dO_s = dY."""
    x = np.asarray(x, F64)
    T = x.shape[0]
    fb = expert_ffn_bwd(dy, x, AU_s, H_s, np.array([0, T]), np.array([T]),
                        np.asarray(w_gu_s)[None], np.asarray(w_d_s)[None], rnd)
    return {"dAU_s": fb["dAU"], "dX_s": fb["dX_perm"], "dW_gu_s": fb["dW_gu"][0],
            "dW_d_s": fb["dW_d"][0]}


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------
def layer_fwd(x, w_r, w_gu, w_d, k, bias=None, renorm=False, route=None,
              rnd=bf16_round, expert_fn=None, w_gu_s=None, w_d_s=None):
    E = w_r.shape[0]
    r = router_topk(x, w_r, k, bias, renorm, route)
    m = routing_metadata(r["idx"], E)
    x_perm = permute(x, m["row_map"], m["M_pad"], rnd)
    ffn = expert_ffn_fwd(x_perm, m["offsets"], m["counts"], w_gu, w_d, rnd,
                         expert_fn)
    sh = shared_expert_fwd(x, w_gu_s, w_d_s, rnd) if w_gu_s is not None else None
    y = combine(ffn["O"], m["row_map"], r["w"], rnd, None if sh is None else sh["O"])
    out = dict(r)
    out.update(m)
    out.update({"x_perm": x_perm, "AU": ffn["AU"], "H": ffn["H"],
                "O": ffn["O"], "y": y})
    if sh is not None:
        out.update({"AU_s": sh["AU"], "H_s": sh["H"], "O_s": sh["O"]})
    return out


def layer_bwd(fwd, dy, x, w_r, w_gu, w_d, renorm=False, rnd=bf16_round, w_gu_s=None,
              w_d_s=None):
    cb = combine_bwd(dy, fwd["O"], fwd["row_map"], fwd["w"], fwd["M_pad"], rnd)
    fb = expert_ffn_bwd(cb["dO"], fwd["x_perm"], fwd["AU"], fwd["H"],
                        fwd["offsets"], fwd["counts"], w_gu, w_d, rnd)
    rb = router_bwd(cb["dw"], fwd["probs"], fwd["idx"], x, w_r, renorm, rnd)
    sb = None
    if w_gu_s is not None:
        sb = shared_expert_bwd(dy, x, fwd["AU_s"], fwd["H_s"], w_gu_s, w_d_s, rnd)
    dx = permute_bwd(fb["dX_perm"], fwd["row_map"], rb["dx_router"], rnd,
                     None if sb is None else sb["dX_s"])
    out = {"dO": cb["dO"], "dw": cb["dw"], "dx": dx}
    if sb is not None:
        out.update(sb)
    out.update(fb)
    out.update({"dL": rb["dL"], "dx_router": rb["dx_router"],
                "dw_r": rb["dw_r"], "db": rb["db"]})
    return out

