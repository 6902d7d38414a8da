"""moe_dispatch_noalloc: the dispatch step for callers that cannot allocate
device memory (a process whose device memory is all handed to a fixed pool up
front, or a host runtime that passes this library only buffers it already
owns).  Its scratch is a fixed array inside the library instead of a caller
workspace.  It must give exactly what moe_dispatch gives, call after call, even
though every call reuses the same scratch array.

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import pytest
import torch

from sparse_moe_layer_noaux_b200 import abi
from sparse_moe_layer_noaux_b200.workloads import TINY, V3_DECODE, MoEShape

pytestmark = pytest.mark.gpu

RAGGED = MoEShape("ragged", T=300, hidden_size=512, n_routed_experts=32, n_group=4, topk_group=2,
                  num_experts_per_tok=4, moe_intermediate_size=256, n_shared_experts=1,
                  routed_scaling_factor=2.5, norm_topk_prob=True, seed=7)


def _tokens_and_routing(shape, seed):
    """Seeded tokens and a valid routing (k distinct experts per token)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((shape.T, shape.H), generator=g, device="cuda").to(torch.bfloat16)
    idx = torch.rand((shape.T, shape.E), generator=g, device="cuda").argsort(dim=1)[:, :shape.k]
    return x, idx.to(torch.int32).contiguous()


def _buffers(shape):
    T, k, E, H = shape.T, shape.k, shape.E, shape.H
    return (torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
            torch.zeros((T * k, H), dtype=torch.bfloat16, device="cuda"),
            torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
            torch.full((T, k), -1, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("shapes", [(RAGGED, TINY), (V3_DECODE.with_(T=512), RAGGED)],
                         ids=["ragged_then_tiny", "v3_then_ragged"])
def test_noalloc_dispatch_matches_workspace_dispatch(shapes):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    for n, shape in enumerate(shapes):  # two calls in a row, different sizes, one scratch array
        x, idx = _tokens_and_routing(shape, seed=100 + n)
        cfg = abi.MoEConfig.from_shape(shape)
        ws = torch.empty(abi.workspace_size(cfg, shape.T), dtype=torch.uint8, device="cuda")
        ref = _buffers(shape)
        abi.moe_dispatch(cfg, x, idx, *ref, ws)
        got = _buffers(shape)
        abi.moe_dispatch_noalloc(cfg, x, idx, *got)
        torch.cuda.synchronize()
        assert abi.device_status() == 0
        for a, b in zip(ref, got):  # integer and byte outputs: bit-exact
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


def test_noalloc_dispatch_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    shape = V3_DECODE.with_(T=16384 + 64)  # 2 * 514 * 256 + 256 int32 > 263168
    cfg = abi.MoEConfig.from_shape(shape)
    p = torch.empty(16, dtype=torch.int32, device="cuda")
    x = torch.empty((1, 1), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(abi.MoEError) as e:
        abi.lib()  # loaded
        rc = abi.lib().moe_dispatch_noalloc(abi.ctypes.byref(cfg), shape.T, abi._ptr(x), abi._ptr(p),
                                            abi._ptr(p), abi._ptr(x), abi._ptr(p), abi._ptr(p), None)
        abi._check("moe_dispatch_noalloc", rc)
    assert e.value.status == abi.MOE_ERR_STATIC_LIMIT
    assert "scratch" in abi.status_string(abi.MOE_ERR_STATIC_LIMIT)
