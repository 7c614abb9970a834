"""moe_permute_noalloc: the permute for callers that cannot provide scratch
memory (no workspace and no permission to allocate) must give exactly what
moe_permute gives with a workspace, call after call, even though every call
reuses the same built-in scratch array.  The permute is integer/copy work, so
the comparison is bit-exact.  Kept in its own file, collected last."""
import pytest
import torch

from mixture_experts_layer_39_b200 import ops
from mixture_experts_layer_39_b200._lib import MOE_DTYPE_BF16

pytestmark = pytest.mark.gpu


def _ids(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.rand(T, E, generator=g).argsort(dim=1)[:, :k].to(torch.int32).cuda()


def _buffers(T, d, E, k, M):
    dev = "cuda"
    return (torch.full((E,), -7, dtype=torch.int32, device=dev),
            torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
            torch.full((T, k), -7, dtype=torch.int32, device=dev),
            torch.full((M, d), 3.0, dtype=torch.bfloat16, device=dev))


@pytest.mark.parametrize("T,d,E,k", [(512, 256, 8, 4), (1000, 256, 128, 4), (16384, 2048, 8, 4)])
def test_noalloc_matches_workspace_permute_twice(cuda_ok, T, d, E, k):
    h = ops.Handle(0)
    shape = ops.make_shape(T, d, 256, E, k, MOE_DTYPE_BF16)
    M = ops.max_rows(shape)
    ws = torch.empty(h.workspace_size(shape), dtype=torch.uint8, device="cuda")
    g = torch.Generator().manual_seed(T + E)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16).cuda()
    for call, seed in enumerate((11, 12)):           # two calls in a row, different routing
        idx = _ids(T, E, k, seed + T)
        ref = _buffers(T, d, E, k, M)
        got = _buffers(T, d, E, k, M)
        ops.moe_permute(h, shape, x, idx, *ref, ws)
        ops.moe_permute_noalloc(h, shape, x, idx, *got)
        torch.cuda.synchronize()
        assert h.get_status() == 0
        for name, a, b in zip(("counts", "offsets", "row_map"), ref[:3], got[:3]):
            assert torch.equal(a, b), f"call {call}: {name} differs"
        m_pad = int(ref[1][-1].item())
        assert torch.equal(ref[3][:m_pad], got[3][:m_pad]), f"call {call}: x_perm differs"
        assert int(got[0].sum().item()) == T * k


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_ok):
    h = ops.Handle(0)
    # (512 + 64) * 1024 int32 = 2.25 MiB > the 1 MiB built-in array
    shape = ops.make_shape(32768, 256, 256, 1024, 8, MOE_DTYPE_BF16)
    d = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    i = torch.empty(16, dtype=torch.int32, device="cuda")
    with pytest.raises(ops.MoeError) as ei:
        ops.moe_permute_noalloc(h, shape, d, i, i, i, i, d)
    assert ei.value.status == 4  # MOE_ERR_WORKSPACE, nothing launched
