"""Load-balancing loss on the GPU (moe_router_load_stats, moe_router_aux_loss
and the router backward with the loss's probability gradient) against the
CPU oracle, on the GPU's own router outputs."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import CONFIGS, custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from oracle import moe_ref as R
from tests._helpers import assert_close, np64

pytestmark = pytest.mark.gpu

ALPHA = 0.01


def _run(cfg, inp, alpha=ALPHA, renorm=False, aux_reduce=None):
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda", renorm=renorm,
                 aux_alpha=alpha, aux_reduce=aux_reduce)
    L.step(inp["x"], inp["w_r"], inp["w_gu"], inp["w_d"], inp["dy"], inp["bias"], inp["route"])
    torch.cuda.synchronize()
    assert L.handle.get_status() == 0
    return L


def _check_aux(cfg, L, n_scale=1):
    """Statistics exact on counts, fp32 sums on probabilities; loss and
    gradient from the oracle on those statistics."""
    E, k, T = cfg.E, cfg.k, cfg.T
    probs, counts = np64(L.probs), np64(L.counts)
    ref = R.router_load_stats(probs, counts) * n_scale
    st = np64(L.stats)
    np.testing.assert_array_equal(st[:E], ref[:E])
    np.testing.assert_allclose(st[E:], ref[E:], rtol=2e-5, atol=1e-4)
    loss, dprob = R.router_aux_loss(st, T * n_scale, k, ALPHA)
    assert float(L.aux_loss.item()) == pytest.approx(loss, rel=1e-5)
    np.testing.assert_allclose(np64(L.dprob_aux), dprob, rtol=1e-5)
    return dprob


CASES = [
    # T, d, f, E, k, renorm
    (512, 256, 512, 8, 4, False),      # the tiny workload's shape: fused router input gradient
    (300, 256, 256, 13, 5, True),      # odd E, renormalised gate weights
    (333, 256, 256, 64, 8, False),     # largest E of the CUDA-core router backward
    (520, 256, 256, 128, 4, False),    # tensor-core router backward (E = 128)
    (300, 384, 256, 100, 4, True),     # E = 100: padded dL rows, zero-filled contraction tail
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "T%d_d%d_f%d_E%d_k%d_r%d" % c)
def test_aux_loss_and_router_backward(cuda_ok, case):
    T, d, f, E, k, renorm = case
    cfg = custom_config(T, d, f, E, k)
    inp_cpu = make_inputs(cfg, seed=E + k, device="cpu")
    inp = {n: (v.cuda() if v is not None else None) for n, v in inp_cpu.items()}
    L = _run(cfg, inp, renorm=renorm)
    dprob = _check_aux(cfg, L)

    # router backward with the loss's gradient, from the GPU's gate-weight gradient
    rb = R.router_bwd(np64(L.dw), np64(L.probs), np64(L.idx), np64(inp_cpu["x"]),
                      np64(inp_cpu["w_r"]), renorm, dprob_aux=dprob)
    assert_close("dW_r (with aux)", np64(L.dw_r), rb["dw_r"])
    assert_close("db (with aux)", np64(L.db), rb["db"], 1e-3)
    Mp = int(L.offsets[-1])
    dxr = np64(L.dx_router) if L.dx_router is not None else rb["dx_router"]
    dx_ref = R.permute_bwd(np64(L.dx_perm[:Mp]), np64(L.row_map), dxr)
    assert_close("dx (with aux)", np64(L.dx), dx_ref)

    # the loss's gradient changes the router gradient (it is not silently dropped)
    rb0 = R.router_bwd(np64(L.dw), np64(L.probs), np64(L.idx), np64(inp_cpu["x"]),
                       np64(inp_cpu["w_r"]), renorm)
    assert np.abs(rb["db"] - rb0["db"]).max() > 0

    # accumulate: a second batch's statistics add (here the same batch: exact doubling)
    before = L.stats.clone()
    L.load_stats(accumulate=True)
    torch.cuda.synchronize()
    assert torch.equal(L.stats, before * 2)


def test_global_batch_reduce_hook(cuda_ok):
    """aux_reduce sums the statistics over ranks and returns the global token
    count; a stand-in for two identical ranks doubles them.  The loss of a
    duplicated batch is the batch's own loss; the per-token gradient halves."""
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, seed=0, device="cuda")

    def two_ranks(stats):
        stats.mul_(2)
        return 2 * cfg.T

    one = _run(cfg, inp)
    two = _run(cfg, inp, aux_reduce=two_ranks)
    _check_aux(cfg, two, n_scale=2)
    assert float(two.aux_loss.item()) == pytest.approx(float(one.aux_loss.item()), rel=1e-6)
    torch.testing.assert_close(two.dprob_aux * 2, one.dprob_aux, rtol=1e-6, atol=0)


def test_aux_full_size_e8(cuda_ok):
    cfg = CONFIGS["e8"]
    inp = make_inputs(cfg, seed=0, device="cuda")
    L = _run(cfg, inp)
    _check_aux(cfg, L)
