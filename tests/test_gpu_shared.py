"""Shared expert on the GPU (moe_shared_expert_fwd / _bwd, and its terms in
the combine and the permute backward) against the CPU oracle, each stage on
the GPU's own inputs to that stage."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import CONFIGS, custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from oracle import moe_ref as R
from tests._helpers import assert_close, np64

pytestmark = pytest.mark.gpu


def _run(cfg, inp):
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda", shared_ff=cfg.shared_ff)
    L.step(inp["x"], inp["w_r"], inp["w_gu"], inp["w_d"], inp["dy"], inp["bias"], inp["route"],
           w_gu_s=inp["w_gu_s"], w_d_s=inp["w_d_s"])
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0
    return L


CASES = [
    # T, d, f, E, k, shared_ff
    (512, 256, 512, 8, 4, 512),      # the tiny workload's shape
    (300, 256, 256, 13, 5, 256),     # ragged T (a 44-row last tile), k > 4
    (2080, 512, 256, 8, 4, 768),     # CTA-pair tiles of the shared expert, ragged tail
    (520, 256, 256, 128, 4, 256),    # E = 128: separate router dX plus the shared term
    (600, 384, 384, 8, 2, 384),      # d, d_ff multiples of 128 only: half-used last tiles
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d_fs%d" % c)
def test_shared_expert_every_stage(cuda_ok, case):
    T, d, f, E, k, fs = case
    cfg = custom_config(T, d, f, E, k, shared_ff=fs)
    inp_cpu = make_inputs(cfg, seed=T + fs, device="cpu")
    inp = {n: (v.cuda() if v is not None else None) for n, v in inp_cpu.items()}
    L = _run(cfg, inp)
    x, dy = np64(inp_cpu["x"]), np64(inp_cpu["dy"])
    w_gu_s, w_d_s = np64(inp_cpu["w_gu_s"]), np64(inp_cpu["w_d_s"])

    sh = R.shared_expert_fwd(x, w_gu_s, w_d_s)
    assert_close("AU_s", np64(L.au_s), sh["AU"])
    assert_close("H_s", np64(L.h_s), sh["H"])
    o_ref = R.bf16_round(np64(L.h_s) @ w_d_s.T)
    assert_close("O_s", np64(L.o_s), o_ref)

    Mp = int(L.offsets[-1])
    rm = np64(L.row_map)
    y_ref = R.combine(np64(L.o_perm[:Mp]), rm, np64(L.w), shared=np64(L.o_s))
    assert_close("y (routed + shared)", np64(L.y), y_ref)

    sb = R.shared_expert_bwd(dy, x, np64(L.au_s), np64(L.h_s), w_gu_s, w_d_s)
    assert_close("dAU_s", np64(L.dau_s), sb["dAU_s"])
    assert_close("dW_d_s", np64(L.dw_d_s), sb["dW_d_s"])
    dau_s = np64(L.dau_s)
    assert_close("dX_s", np64(L.dx_s), R.bf16_round(dau_s @ w_gu_s))
    assert_close("dW_gu_s", np64(L.dw_gu_s), R.bf16_round(dau_s.T @ x))

    rb = R.router_bwd(np64(L.dw), np64(L.probs), np64(L.idx), x, np64(inp_cpu["w_r"]))
    dxr = np64(L.dx_router) if L.dx_router is not None else rb["dx_router"]
    dx_ref = R.permute_bwd(np64(L.dx_perm[:Mp]), rm, dxr, dx_shared=np64(L.dx_s))
    assert_close("dx (routed + router + shared)", np64(L.dx), dx_ref)


def test_shared_expert_full_size_sampled(cuda_ok):
    """The e8 workload with a shared expert of d_ff 1024, checked on sampled
    tokens and sampled weight-gradient columns."""
    cfg = CONFIGS["e8_shared"]
    inp = make_inputs(cfg, seed=0, device="cuda")
    L = _run(cfg, inp)
    rng = np.random.default_rng(3)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], rng.integers(0, cfg.T, 126)]))
    tt = torch.as_tensor(toks, device="cuda")
    x_s, dy_s = np64(inp["x"][tt]), np64(inp["dy"][tt])
    w_gu_s, w_d_s = np64(inp["w_gu_s"]), np64(inp["w_d_s"])
    sh = R.shared_expert_fwd(x_s, w_gu_s, w_d_s)
    assert_close("AU_s (sampled)", np64(L.au_s[tt]), sh["AU"])
    assert_close("O_s (sampled)", np64(L.o_s[tt]), R.bf16_round(np64(L.h_s[tt]) @ w_d_s.T))
    sb = R.shared_expert_bwd(dy_s, x_s, np64(L.au_s[tt]), np64(L.h_s[tt]), w_gu_s, w_d_s)
    assert_close("dAU_s (sampled)", np64(L.dau_s[tt]), sb["dAU_s"])
    assert_close("dX_s (sampled)", np64(L.dx_s[tt]), R.bf16_round(np64(L.dau_s[tt]) @ w_gu_s))
    # weight gradients: all tokens, sampled output columns
    cols = torch.as_tensor(rng.choice(cfg.d, 48, replace=False), device="cuda")
    rows = torch.as_tensor(rng.choice(2 * cfg.shared_ff, 48, replace=False), device="cuda")
    # (the sampled columns are contracted on the host in float64)
    ref_gu = np64(L.dau_s[:, rows]).T @ np64(inp["x"][:, cols])
    assert_close("dW_gu_s (sampled)", np64(L.dw_gu_s[rows][:, cols]), R.bf16_round(ref_gu))
    frow = torch.as_tensor(rng.choice(cfg.shared_ff, 48, replace=False), device="cuda")
    ref_d = np64(inp["dy"][:, cols]).T @ np64(L.h_s[:, frow])
    assert_close("dW_d_s (sampled)", np64(L.dw_d_s[cols][:, frow]), R.bf16_round(ref_d))
