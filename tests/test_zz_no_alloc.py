"""The allocation-free router entry point (ts_moe_route_noalloc), through the C ABI.

Some callers cannot allocate device memory when they need routing -- code
running under CUDA-graph stream capture, engines that own all device memory in
their own pool, plugins handed only a stream and buffers -- so they cannot
open a handle.  ts_moe_route_noalloc takes the raw router and keeps its scratch
in the library's static device array.  Here its results are checked against
the handle-based ts_moe_route on the same router and inputs, on two calls in a
row (the static scratch keeps the previous call's contents), with the
tolerances the parity tests use (experts bit-exact, weights within 1e-5,
logits within 1e-4 of the largest)."""
import numpy as np
import pytest
import torch

from quantized_moe_routed_router_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_moe_routed_router_b200 import build
    build.build()


@pytest.mark.parametrize("cfg", [3, 4])
def test_route_noalloc_matches_route(cfg):
    from quantized_moe_routed_router_b200 import binding
    shape = synth.CONFIGS[cfg].replace(moe_inter=64, shared_inter=64 if synth.CONFIGS[cfg].shared_inter else 0,
                                       max_tokens=16)
    L = synth.make_layer(shape, 0, device="cuda")
    moe = binding.MoE(shape, [L])
    E, H, K = shape.num_experts, shape.hidden, shape.top_k
    bias_d = torch.from_numpy(L.bias).cuda() if L.bias is not None else None
    for call, M in enumerate((16, 5)):                       # two calls in a row, different inputs
        x = synth.make_x(shape, call + 1, M, device="cuda")
        idx_a = torch.full((M, K), -1, dtype=torch.int32, device="cuda")
        w_a = torch.zeros(M, K, device="cuda")
        lg_a = torch.zeros(M, E, device="cuda")
        moe.route(0, x, idx_a, w_a, lg_a)
        idx_b = torch.full((M, K), -2, dtype=torch.int32, device="cuda")
        w_b = torch.zeros(M, K, device="cuda")
        lg_b = torch.zeros(M, E, device="cuda")
        binding.route_noalloc(L.router, bias_d, None, E, H, K, shape.score, shape.bias_mode, x, idx_b, w_b, lg_b)
        torch.cuda.synchronize()
        assert torch.equal(idx_a, idx_b), f"call {call}"
        assert (w_a - w_b).abs().max().item() <= 1e-5
        assert (lg_a - lg_b).abs().max().item() <= 1e-4 * lg_a.abs().max().item()
    moe.device_status()
    moe.close()


def test_route_noalloc_refuses_oversized_scratch():
    from quantized_moe_routed_router_b200 import binding
    router = torch.zeros(256 * (16384 // 32) * 34, dtype=torch.uint8, device="cuda")   # 256 x 16384 router: > 2 MiB
    x = torch.zeros(16, 16384, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(16, 8, dtype=torch.int32, device="cuda")
    w = torch.empty(16, 8, device="cuda")
    with pytest.raises(binding.TsMoeError) as ei:
        binding.route_noalloc(router, None, None, 256, 16384, 8, 0, 0, x, idx, w)
    assert ei.value.status == 1 and "scratch" in str(ei.value)
