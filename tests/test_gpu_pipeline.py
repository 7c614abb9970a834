"""HostStepper (pinned-host inputs and results, copies overlapped with the
kernels on side streams) gives exactly the results of running the same steps
one after another through MoELayer."""
import pytest
import torch

from mixture_experts_layer_39_b200.inputs import custom_config, make_inputs
from mixture_experts_layer_39_b200.layer import MoELayer
from mixture_experts_layer_39_b200.pipeline import HostStepper

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("random_routing", [False, True])
def test_host_stepper_matches_sequential_steps(cuda_ok, random_routing):
    cfg = custom_config(1024, 256, 256, 8, 2, random_routing=random_routing)
    w = make_inputs(cfg, seed=1, device="cuda")
    steps_in = [make_inputs(cfg, seed=10 + i, device="cpu") for i in range(5)]
    ref = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda")
    expect = []
    for s in steps_in:
        ref.step(s["x"].cuda(), w["w_r"], w["w_gu"], w["w_d"], s["dy"].cuda(),
                 route=None if s["route"] is None else s["route"].cuda())
        torch.cuda.synchronize()
        expect.append((ref.y.cpu().clone(), ref.dx.cpu().clone()))
    L = MoELayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, device="cuda")
    stepper = HostStepper(L, with_route=random_routing)
    plan = []
    for s in steps_in:
        st = {"x": s["x"].pin_memory(), "dy": s["dy"].pin_memory(),
              "y": torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory(),
              "dx": torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory()}
        if random_routing:
            st["route"] = s["route"].pin_memory()
        plan.append(st)
    stepper.run(plan, w["w_r"], w["w_gu"], w["w_d"])
    stepper.done_event().synchronize()
    torch.cuda.synchronize()
    for i, (st, (y, dx)) in enumerate(zip(plan, expect)):
        assert torch.equal(st["y"], y), f"step {i}: y differs"
        assert torch.equal(st["dx"], dx), f"step {i}: dx differs"
    assert L.handle.get_status() == 0
