"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Stage-wise: every stage's GPU output is compared with the oracle applied to
that stage's GPU inputs, so a failure names the kernel at fault.  Integer
and byte work (indices, counts, offsets, row map, the permuted copy) must
match bit-exactly; bf16 outputs must be within a normwise max relative
error of 2e-2.  Expert selection: the GPU's ids must equal the oracle's
top-k of the GPU's own fp32 logits for every token, and the oracle's fp64
top-k for every token whose k-th/(k+1)-th logit gap exceeds 1e-3.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import CONFIGS, custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from oracle import moe_ref as R
from tests import _helpers as H
from tests._helpers import TAU, assert_close, np64, topk_margin

pytestmark = pytest.mark.gpu


def _to(inp, dev):
    return {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}


def _run(cfg, inp_dev, renorm=False, fuse_router_dx=None):
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda", renorm=renorm, keep_logits=True,
                 fuse_router_dx=fuse_router_dx)
    g = inp_dev
    L.step(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["dy"], g["bias"], g["route"])
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0
    return L


def _check_full(cfg, inp, L, renorm=False):
    """Every stage against the oracle at a size the oracle finishes quickly."""
    x, w_r = np64(inp["x"]), np64(inp["w_r"])
    w_gu, w_d, dy = np64(inp["w_gu"]), np64(inp["w_d"]), np64(inp["dy"])
    bias = None if inp["bias"] is None else np64(inp["bias"])
    k, E = cfg.k, cfg.E

    # router: logits, probs, selection, gate weights
    lg = np64(L.logits)
    lo = R.router_logits(x, w_r, bias)
    assert_close("logits", lg, lo, 1e-4)
    probs = np64(L.probs)
    assert_close("probs", probs, R.softmax(lo), 1e-4)
    idx = np64(L.idx)
    if inp["route"] is None:
        np.testing.assert_array_equal(idx, R.topk_select(lg, k))
        sure = topk_margin(lo, k) > TAU
        np.testing.assert_array_equal(idx[sure], R.topk_select(lo, k)[sure])
    else:
        np.testing.assert_array_equal(idx, np64(inp["route"]))
    w = np64(L.w)
    assert_close("gate weights", w, R.gate_weights(probs, idx, renorm), 1e-6)

    # metadata + permute, bit-exact on the GPU's ids
    m = R.routing_metadata(idx, E)
    np.testing.assert_array_equal(np64(L.counts), m["counts"])
    np.testing.assert_array_equal(np64(L.offsets), m["offsets"])
    np.testing.assert_array_equal(np64(L.row_map), m["row_map"])
    Mp = m["M_pad"]
    off, cnt, rm = m["offsets"], m["counts"], m["row_map"]
    xp = np64(L.x_perm[:Mp])
    np.testing.assert_array_equal(xp, R.permute(x, rm, Mp))

    # experts forward on the GPU's x_perm
    ffn = R.expert_ffn_fwd(xp, off, cnt, w_gu, w_d)
    au, hh, oo = np64(L.au[:Mp]), np64(L.h[:Mp]), np64(L.o_perm[:Mp])
    assert_close("AU", au, ffn["AU"])
    assert_close("H", hh, ffn["H"])
    pad = np.ones(Mp, bool)
    pad[rm.reshape(-1)] = False
    for name, a in (("AU", au), ("H", hh), ("O", oo)):
        assert np.all(a[pad] == 0), f"{name} pad rows not zero"
    # down projection checked from the GPU's own H
    o_ref = np.zeros_like(oo)
    for e in range(E):
        r0, r1 = off[e], off[e] + cnt[e]
        o_ref[r0:r1] = R.bf16_round(hh[r0:r1] @ w_d[e].T)
    assert_close("O_perm", oo, o_ref)
    assert_close("O_perm (end to end)", oo, ffn["O"])

    # combine on the GPU's O and w
    y = np64(L.y)
    assert_close("y", y, R.combine(oo, rm, w))

    # combine backward
    cb = R.combine_bwd(dy, oo, rm, w, Mp)
    dO = np64(L.do_perm[:Mp])
    assert_close("dO_perm", dO, cb["dO"], 1e-2)
    assert np.all(dO[pad] == 0)
    assert_close("d gate weights", np64(L.dw), cb["dw"], 1e-4)

    # experts backward on the GPU's dO, x_perm, AU, H
    fb = R.expert_ffn_bwd(dO, xp, au, hh, off, cnt, w_gu, w_d)
    dau = np64(L.dau[:Mp])
    assert_close("dAU", dau, fb["dAU"])
    assert np.all(dau[pad] == 0)
    dxp = np64(L.dx_perm[:Mp])
    dxp_ref = np.zeros_like(dxp)
    for e in range(E):
        r0, r1 = off[e], off[e] + cnt[e]
        dxp_ref[r0:r1] = R.bf16_round(dau[r0:r1] @ w_gu[e])
    assert_close("dX_perm", dxp, dxp_ref)
    assert_close("dW_d", np64(L.dw_d), fb["dW_d"])
    dwgu_ref = np.zeros_like(fb["dW_gu"])
    for e in range(E):
        r0, r1 = off[e], off[e] + cnt[e]
        dwgu_ref[e] = R.bf16_round(dau[r0:r1].T @ xp[r0:r1])
    assert_close("dW_gu", np64(L.dw_gu), dwgu_ref)
    for e in range(E):
        if cnt[e] == 0:
            assert np.all(np64(L.dw_gu[e]) == 0) and np.all(np64(L.dw_d[e]) == 0)

    # router backward on the GPU's d(gate weights)
    rb = R.router_bwd(np64(L.dw), probs, idx, x, w_r, renorm)
    if L.dx_router is not None:
        assert_close("dX_router", np64(L.dx_router), rb["dx_router"], 1e-2)
    assert_close("dW_r", np64(L.dw_r), rb["dw_r"])
    assert_close("db", np64(L.db), rb["db"], 1e-3)

    # permute backward (with the router's input gradient added in the same
    # kernel when the layer fuses them)
    dxr = np64(L.dx_router) if L.dx_router is not None else rb["dx_router"]
    assert_close("dx", np64(L.dx), R.permute_bwd(dxp, rm, dxr))


def test_tiny_workload_every_stage(cuda_ok):
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=0, device="cpu")
    L = _run(cfg, _to(inp, "cuda"))
    _check_full(cfg, inp, L)
    # the tiny workload has no near-ties: selection is bit-exact against fp64
    x, w_r = np64(inp["x"]), np64(inp["w_r"])
    np.testing.assert_array_equal(np64(L.idx), R.topk_select(R.router_logits(x, w_r), cfg.k))


def test_tiny_workload_end_to_end(cuda_ok):
    """Whole layer against the oracle run from the inputs alone."""
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=0, device="cpu")
    L = _run(cfg, _to(inp, "cuda"))
    x, w_r, w_gu, w_d, dy = (np64(inp[n]) for n in ("x", "w_r", "w_gu", "w_d", "dy"))
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, cfg.k)
    bwd = R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d)
    assert_close("y", np64(L.y), fwd["y"])
    assert_close("dx", np64(L.dx), bwd["dx"])
    assert_close("dW_gu", np64(L.dw_gu), bwd["dW_gu"])
    assert_close("dW_d", np64(L.dw_d), bwd["dW_d"])
    assert_close("dW_r", np64(L.dw_r), bwd["dw_r"])


SMALL_CASES = [
    # T, d, f, E, k, routing
    (300, 256, 256, 4, 2, "learned"),      # ragged tails in every segment
    (257, 512, 256, 6, 3, "skewed"),       # zero-count experts, one hot expert
    (1, 256, 256, 8, 4, "learned"),        # a single token
    (700, 256, 512, 16, 1, "learned"),     # k = 1
    (130, 256, 256, 1, 1, "learned"),      # one expert: dense SwiGLU
    (520, 256, 256, 128, 4, "learned"),    # E = 128: tensor-core router
    (333, 256, 256, 64, 8, "renorm"),      # k = 8, renormalised gate weights
    (400, 512, 256, 8, 2, "bias"),         # router bias
    (384, 256, 256, 12, 3, "random"),      # caller-given ids (random routing)
    (3072, 256, 256, 8, 4, "learned"),     # long segments: 256-row CTA-pair tiles
    (2080, 512, 256, 1, 1, "learned"),     # one expert, pair tiles with a ragged tail
    (500, 768, 256, 7, 2, "renorm"),       # odd E, d not a multiple of 512
    (257, 256, 256, 13, 5, "bias"),        # second expert tile of the router partly empty
    (2048, 256, 256, 1024, 8, "learned"),  # the largest E and k
    (300, 256, 256, 4, 4, "learned"),      # k = E: every token on every expert
    (1600, 384, 640, 2, 2, "learned"),     # CTA pairs; d, f multiples of 128 but not of 256:
                                           # half-used last N tiles and wgrad M tiles
    (600, 384, 384, 8, 2, "bias"),         # single-CTA tiles, half-used last N tiles
    (700, 256, 256, 200, 6, "learned"),    # E = 200: tensor-core router, padded logits rows
    (500, 384, 128, 96, 3, "renorm"),      # E = 96, f = 128: one half-used N tile
    (1024, 256, 256, 8, 4, "learned"),     # ~512 rows per expert: several 128-row tiles
    (700, 384, 512, 4, 2, "renorm"),       # ~350 rows per expert, d an odd multiple of 128
    (1600, 256, 256, 6, 2, "skewed"),      # empty experts next to one long segment
    (300, 2304, 256, 8, 2, "learned"),     # d > 2048: router dW over two column slices
    (200, 4096, 128, 16, 4, "bias"),       # d = 4096, E = 16 (router dW: two n-tiles of experts)
    (700, 256, 256, 200, 6, "random"),     # caller-given ids with the tensor-core router's
    (500, 384, 128, 96, 3, "random"),      # padded logits rows (stride 256 and 128, not E)
    (300, 256, 256, 48, 3, "random"),      # caller-given ids on the CUDA-core router (16 < E <= 64)
    (400, 256, 256, 100, 4, "random_renorm"),  # caller-given ids, renormalised gate weights
    (300, 128, 128, 8, 2, "learned"),      # the smallest d and d_ff: one router chunk per warp
    (300, 128, 256, 100, 3, "bias"),       # d = 128 with the tensor-core router (K = 2 blocks)
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d_%s" % c)
def test_small_shapes_every_stage(cuda_ok, case):
    T, d, f, E, k, mode = case
    renorm = mode in ("renorm", "random_renorm")
    cfg = custom_config(T, d, f, E, k, random_routing=mode in ("random", "random_renorm"))
    inp = make_inputs(cfg, seed=T + E, device="cpu")
    if mode == "skewed":
        inp["bias"] = torch.tensor([4.0, -30.0, 2.0, -30.0, 0.0, -30.0][:E], dtype=torch.float32)
    if mode == "bias":
        inp["bias"] = torch.linspace(-1, 1, E, dtype=torch.float32)
    L = _run(cfg, _to(inp, "cuda"), renorm=renorm)
    _check_full(cfg, inp, L, renorm=renorm)
    if mode == "skewed":
        assert (np64(L.counts) == 0).any()


FUSION_CASES = [
    # T, d, f, E, k, mode
    (4097, 256, 256, 8, 4, "learned"),   # odd T: the last warp has one token
    (300, 768, 256, 13, 5, "renorm"),    # k > 4, renormalised gate weights
    (333, 256, 256, 64, 8, "learned"),   # the largest E of the fused path
    (130, 256, 256, 1, 1, "learned"),    # one expert
]


@pytest.mark.parametrize("case", FUSION_CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d_%s" % c)
def test_fused_router_dx_same_bits(cuda_ok, case):
    """moe_permute_router_bwd forms dL W_r inside the unpermute-reduce; it
    must give exactly the bits of moe_router_topk_bwd (dX_router written)
    followed by moe_permute_bwd on the same inputs."""
    T, d, f, E, k, mode = case
    cfg = custom_config(T, d, f, E, k)
    inp = _to(make_inputs(cfg, seed=T + k, device="cpu"), "cuda")
    renorm = mode == "renorm"
    fused = _run(cfg, inp, renorm=renorm, fuse_router_dx=True)
    split = _run(cfg, inp, renorm=renorm, fuse_router_dx=False)
    assert fused.dx_router is None and split.dx_router is not None
    Mp = int(split.offsets[-1])  # rows past the last segment are never written
    assert torch.equal(fused.dx_perm[:Mp], split.dx_perm[:Mp])
    assert torch.equal(fused.dx, split.dx)
    assert torch.equal(fused.dw_r, split.dw_r)


# ---------------------------------------------------------------- full sizes
def _seg_check(L, inp_dev, e, off, cnt, max_rows=4096):
    """Oracle on one expert's segment (rows subsampled for the row-wise
    outputs, whole segment for its weight gradients)."""
    r0, r1 = int(off[e]), int(off[e] + cnt[e])
    if r1 == r0:
        assert torch.count_nonzero(L.dw_gu[e]) == 0 and torch.count_nonzero(L.dw_d[e]) == 0
        return
    w_gu = np64(inp_dev["w_gu"][e:e + 1])
    w_d = np64(inp_dev["w_d"][e:e + 1])
    xp = np64(L.x_perm[r0:r1])
    au = np64(L.au[r0:r1])
    hh = np64(L.h[r0:r1])
    dO = np64(L.do_perm[r0:r1])
    n = r1 - r0
    o1 = np.array([0, n])
    c1 = np.array([n])
    if n <= max_rows:
        ffn = R.expert_ffn_fwd(xp, o1, c1, w_gu, w_d)
        assert_close(f"AU[{e}]", au, ffn["AU"])
        assert_close(f"H[{e}]", hh, ffn["H"])
        assert_close(f"O[{e}]", np64(L.o_perm[r0:r1]), R.bf16_round(hh @ w_d[0].T))
    fb = R.expert_ffn_bwd(dO, xp, au, hh, o1, c1, w_gu, w_d)
    if n <= max_rows:
        assert_close(f"dAU[{e}]", np64(L.dau[r0:r1]), fb["dAU"])
    dau = np64(L.dau[r0:r1])
    assert_close(f"dW_d[{e}]", np64(L.dw_d[e]), fb["dW_d"][0])
    assert_close(f"dW_gu[{e}]", np64(L.dw_gu[e]), R.bf16_round(dau.T @ xp))
    if n <= max_rows:
        assert_close(f"dX_perm[{e}]", np64(L.dx_perm[r0:r1]), R.bf16_round(dau @ w_gu[0]))


@pytest.mark.parametrize("name", ["e8", "e128", "skew", "mxfp8"])
def test_full_size_sampled(cuda_ok, name):
    """The launch configuration the benchmark times, checked on outputs the
    oracle computes one by one (sampled tokens, rows and experts) plus the
    exact routing metadata.  The mxfp8 workload's shapes run here on the
    bf16 path."""
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, seed=0, device="cuda")
    L = _run(cfg, inp)
    k, E = cfg.k, cfg.E
    log0 = len(H.LOG)
    rng = np.random.default_rng(1)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], rng.integers(0, cfg.T, 254)]))

    # selection: exact top-k of the GPU's logits everywhere; fp64 oracle on samples
    lg = np64(L.logits)
    idx = np64(L.idx)
    if inp["route"] is None:
        np.testing.assert_array_equal(idx, R.topk_select(lg, k))
        x_s = np64(inp["x"][toks])
        lo = R.router_logits(x_s, np64(inp["w_r"]), None if inp["bias"] is None else np64(inp["bias"]))
        assert_close("logits (sampled)", lg[toks], lo, 1e-4)
        sure = topk_margin(lo, k) > TAU
        np.testing.assert_array_equal(idx[toks][sure], R.topk_select(lo, k)[sure])
    else:
        np.testing.assert_array_equal(idx, np64(inp["route"]))

    # metadata: bit-exact in full
    m = R.routing_metadata(idx, E)
    np.testing.assert_array_equal(np64(L.counts), m["counts"])
    np.testing.assert_array_equal(np64(L.offsets), m["offsets"])
    rm = m["row_map"]
    np.testing.assert_array_equal(np64(L.row_map), rm)
    off, cnt = m["offsets"], m["counts"]
    # permuted copies of the sampled tokens, and zero pads
    for j in range(k):
        assert torch.equal(L.x_perm[torch.as_tensor(rm[toks, j], device="cuda")], inp["x"][toks])
    pads = [r for e in range(E) for r in range(off[e] + cnt[e], off[e + 1])]
    if pads:
        pr = torch.as_tensor(pads, device="cuda")
        assert torch.count_nonzero(L.x_perm[pr]) == 0 and torch.count_nonzero(L.do_perm[pr]) == 0

    # combine / combine-bwd / permute-bwd on sampled tokens
    w = np64(L.w)
    rows = rm[toks]
    O_rows = {int(r): np64(L.o_perm[int(r)]) for r in np.unique(rows)}
    y_ref = np.stack([R.bf16_round(sum(w[t, j] * O_rows[int(rm[t, j])] for j in range(k)))
                      for t in toks])
    assert_close("y (sampled)", np64(L.y[toks]), y_ref)
    dy_s = np64(inp["dy"][toks])
    dw_ref = np.stack([[np.dot(dy_s[i], O_rows[int(rm[t, j])]) for j in range(k)]
                       for i, t in enumerate(toks)])
    assert_close("d gate weights (sampled)", np64(L.dw[toks]), dw_ref, 1e-4)
    dxp_rows = {int(r): np64(L.dx_perm[int(r)]) for r in np.unique(rows)}
    # router backward: dL from the GPU's gate-weight gradient, sampled rows
    rb_rows = R.router_bwd(np64(L.dw[toks]), np64(L.probs[toks]), idx[toks], np64(inp["x"][toks]),
                           np64(inp["w_r"]))
    if L.dx_router is not None:
        dxr = np64(L.dx_router[toks])
        assert_close("dX_router (sampled)", dxr, rb_rows["dx_router"], 1e-2)
    else:
        dxr = rb_rows["dx_router"]
    dx_ref = np.stack([R.bf16_round(sum(dxp_rows[int(rm[t, j])] for j in range(k)) + dxr[i])
                       for i, t in enumerate(toks)])
    assert_close("dx (sampled)", np64(L.dx[toks]), dx_ref)

    # experts: the hottest, the coldest non-empty, one in the middle, empty ones
    order = np.argsort(cnt, kind="stable")
    nonempty = [e for e in order if cnt[e] > 0]
    pick = {int(nonempty[0]), int(nonempty[-1]), int(nonempty[len(nonempty) // 2])}
    pick |= {int(e) for e in order[cnt[order] == 0][:2]}
    for e in sorted(pick):
        _seg_check(L, inp, e, off, cnt)
    H.report(f"full-size {name}", log0)



def test_mxfp8_quantize_matches_oracle(cuda_ok):
    from mixture_experts_layer_39_b200 import ops
    from oracle import mxfp8_ref as M
    h = ops.Handle(0)
    g = torch.Generator().manual_seed(3)
    a = torch.randn(256, 512, generator=g) * torch.exp(torch.randn(256, 1, generator=g) * 4)
    a[3] = 0.0
    a[5, :32] = 1e-30
    a[7, 64:96] = 3e4
    a[9, 96:128] = torch.randn(32, generator=g) * 2e-39   # bf16 subnormals: scale clamp at -127
    a[:, 130] = torch.randn(256, generator=g) * 3e-39     # every column-wise block of a column
    a = a.to(torch.bfloat16)
    assert (a[9, 96:128].float().abs() < 2.0 ** -126).all() and bool(a[9, 96:128].any())
    for axis in (1, 0):
        ad = a.cuda()
        if axis == 1:
            q = torch.empty(256, 512, dtype=torch.uint8, device="cuda")
            s = torch.empty(256, 16, dtype=torch.uint8, device="cuda")
        else:
            q = torch.empty(256, 512, dtype=torch.uint8, device="cuda")
            s = torch.empty(8, 512, dtype=torch.uint8, device="cuda")
        ops.moe_mxfp8_quantize(h, ad, axis, q, s)
        torch.cuda.synchronize()
        qo, so = M.quantize_blocks(a.double().numpy(), axis)
        np.testing.assert_array_equal(s.cpu().numpy(), so)
        np.testing.assert_array_equal(q.cpu().numpy(), qo)


@pytest.mark.parametrize("rows,cols", [(64, 130), (96, 132), (32, 2)])
def test_mxfp8_quantize_columnwise_widths(cuda_ok, rows, cols):
    """Column-wise blocks where a thread takes two columns (cols % 4 == 2) and
    four (cols % 4 == 0), each column with its own magnitude, so every lane of
    a vector access has its own scale; bit-exact against the oracle."""
    from mixture_experts_layer_39_b200 import ops
    from oracle import mxfp8_ref as M
    h = ops.Handle(0)
    g = torch.Generator().manual_seed(rows + cols)
    a = torch.randn(rows, cols, generator=g) * torch.exp(torch.randn(1, cols, generator=g) * 5)
    a[:, 0] = 0.0
    if cols > 3:
        a[:32, 3] = -1e-30
        a[1, 2] = 4e5
    a = a.to(torch.bfloat16)
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows // 32, cols, dtype=torch.uint8, device="cuda")
    ops.moe_mxfp8_quantize(h, a.cuda(), 0, q, s)
    torch.cuda.synchronize()
    qo, so = M.quantize_blocks(a.double().numpy(), 0)
    np.testing.assert_array_equal(s.cpu().numpy(), so)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
