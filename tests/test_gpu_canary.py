"""Canary-filled outputs: the layer writes the rows its contract names and no
others, and reads none it did not write.

Before a training step every output buffer of the layer is filled with a NaN
canary.  Afterwards:
  - rows at and past offsets[E] of every routed-row buffer (x_perm, au, h,
    o_perm, do_perm, dau, dx_perm) still hold the canary bytes: the header
    says they are never written;
  - the pad rows of each expert segment of x_perm and do_perm are zero, and
    row_src holds T on pad rows (and past offsets[E] when moe_route wrote
    it; moe_permute_src leaves those rows alone);
  - every token-side output, the router outputs and the weight gradients
    hold no canary and are finite, and experts with no rows get exactly zero
    weight gradients;
  - the step's results still match the oracle, so no kernel read a canary
    row (a NaN read spreads into every output that depends on it).
The routing leaves several experts empty and the others ragged, so segment
ends, pad rows and the tail past offsets[E] all occur.
"""
import numpy as np
import pytest
import torch

from tests._helpers import TOL_BF16, np64, rel_err
from mixture_experts_layer_39_b200.inputs import custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from oracle import moe_ref as R

pytestmark = pytest.mark.gpu

CANARY16 = 0x7FBB            # bf16 NaN
CANARY32F = 0x7FBBBBBB       # fp32 NaN (as int32 bits)
CANARY32I = 0x7BBBBBBB       # int32: far outside every index range

ROUTED = ("x_perm", "au", "h", "o_perm", "do_perm", "dau", "dx_perm")
WRITTEN = ("idx", "w", "probs", "counts", "offsets", "row_map", "y", "dw", "dw_gu", "dw_d",
           "dw_r", "dx", "dx_router")
SKIP = ("ws", "arrivals")    # workspace; arrival counters must start at zero


def _fill(t):
    if t.dtype == torch.bfloat16:
        t.view(torch.int16).fill_(CANARY16)
    elif t.dtype == torch.float32:
        t.view(torch.int32).fill_(CANARY32F)
    elif t.dtype == torch.int32:
        t.fill_(CANARY32I)


def _canary_mask(t):
    """Elementwise: still holding the canary."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16) == CANARY16
    if t.dtype == torch.float32:
        return t.view(torch.int32) == CANARY32F
    return t == CANARY32I


def _route(T, E, k, n_active, seed):
    """k distinct experts per token drawn from n_active of the E experts, with
    a skewed (1/rank) preference, so the other experts stay empty."""
    rng = np.random.default_rng(seed)
    active = np.sort(rng.choice(E, size=n_active, replace=False))
    p = 1.0 / np.arange(1, n_active + 1)
    p /= p.sum()
    rows = [rng.choice(active, size=k, replace=False, p=p) for _ in range(T)]
    return torch.tensor(np.stack(rows), dtype=torch.int32), set(active.tolist())


CASES = [
    # (id, T, d, f, E, k, active experts or None = learned routing, layer options)
    ("bf16", 300, 256, 256, 8, 2, 5, {}),
    ("bf16_split_router_dx", 300, 256, 256, 8, 2, 5, {"fuse_router_dx": False}),
    ("gather", 300, 256, 256, 8, 2, 5, {"gather": True}),
    ("fused_combine", 300, 256, 256, 8, 2, 5, {"fuse_combine": True}),
    ("recompute", 300, 256, 256, 8, 2, 5, {"recompute": True}),
    ("mxfp8", 300, 256, 256, 8, 2, 5, {"dtype": "mxfp8"}),
    ("e96_tensor_core_router", 400, 256, 128, 96, 4, 50, {}),
    ("learned", 333, 256, 128, 8, 2, None, {}),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_canary_rows(cuda_ok, case):
    name, T, d, f, E, k, n_active, opts = case
    cfg = custom_config(T, d, f, E, k)
    inp = make_inputs(cfg, seed=11)
    active = set(range(E))
    if n_active is not None:
        inp["route"], active = _route(T, E, k, n_active, seed=12)
    g = {key: (v.to("cuda") if v is not None else None) for key, v in inp.items()}
    L = MoELayer(T, d, f, E, k, device="cuda", **opts)
    bufs = {key: v for key, v in vars(L).items()
            if isinstance(v, torch.Tensor) and key not in SKIP}
    for t in bufs.values():
        _fill(t)
    torch.cuda.synchronize()
    L.step(g["x"], g["w_r"], g["w_gu"], g["w_d"], g["dy"], g["bias"], g["route"])
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0

    counts = L.counts.cpu().numpy().astype(np.int64)
    offsets = L.offsets.cpu().numpy().astype(np.int64)
    M_pad, M_cap = int(offsets[E]), L.M_cap
    if n_active is not None:
        assert np.array_equal(counts, np.bincount(inp["route"].numpy().ravel(), minlength=E))
    assert M_pad < M_cap, "the case must leave rows past offsets[E]"

    # never written: every routed-row buffer at and past offsets[E]
    for key in ROUTED:
        t = getattr(L, key)
        if t is None:
            continue
        assert bool(_canary_mask(t[M_pad:]).all()), f"{name}: {key} written past offsets[E]"

    # pad rows of each segment: zero in x_perm and do_perm, T in row_src
    pad = np.zeros(M_cap, dtype=bool)
    for e in range(E):
        pad[offsets[e] + counts[e]:offsets[e + 1]] = True
    assert pad.any(), "the case must have pad rows"
    pad_t = torch.from_numpy(pad[:M_pad]).cuda()
    for key in ("x_perm", "do_perm"):
        t = getattr(L, key)
        if t is not None:
            assert bool((t[:M_pad][pad_t].view(torch.int16) == 0).all()), f"{name}: {key} pad rows"
    if L.row_src is not None:
        # moe_route (gather forms) writes T past offsets[E] as well;
        # moe_permute_src (fused combine) leaves those rows alone
        rs = L.row_src.cpu().numpy()
        past = (rs[M_pad:] == T) if L.gather else _canary_mask(L.row_src[M_pad:]).cpu().numpy()
        assert np.all(past), f"{name}: row_src past offsets[E]"
        assert np.all(rs[:M_pad][pad[:M_pad]] == T), f"{name}: row_src pad rows"
        real = ~pad[:M_pad]
        assert np.all((rs[:M_pad][real] >= 0) & (rs[:M_pad][real] < T))

    # fully written and finite
    for key in WRITTEN:
        t = getattr(L, key, None)
        if t is None:
            continue
        assert not bool(_canary_mask(t).any()), f"{name}: {key} not fully written"
        if t.is_floating_point():
            assert bool(torch.isfinite(t).all()), f"{name}: {key} not finite"
    for e in sorted(set(range(E)) - active):
        assert bool((L.dw_gu[e] == 0).all()) and bool((L.dw_d[e] == 0).all()), \
            f"{name}: expert {e} has no rows but a nonzero weight gradient"

    # the results still match the oracle (MXFP8 has its own emulation tests)
    if opts.get("dtype", "bf16") == "bf16":
        x, w_r, w_gu, w_d, dy = (np64(inp[n]) for n in ("x", "w_r", "w_gu", "w_d", "dy"))
        if inp["route"] is not None:
            assert np.array_equal(np64(L.idx), inp["route"].numpy())
        # the oracle takes the selection made on the device (selection parity
        # near logit ties is the parity tests' subject, not this one's)
        fwd = R.layer_fwd(x, w_r, w_gu, w_d, k, route=np64(L.idx))
        bwd = R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d)
        for key, ref in (("y", fwd["y"]), ("dx", bwd["dx"]), ("dw_gu", bwd["dW_gu"]),
                         ("dw_d", bwd["dW_d"]), ("dw_r", bwd["dw_r"])):
            err = rel_err(np64(getattr(L, key)), ref)
            assert err <= TOL_BF16, f"{name}: {key} rel err {err:.3e}"
