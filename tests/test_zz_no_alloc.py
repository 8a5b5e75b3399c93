"""The allocation-free router entry point (ts_moe_route_noalloc), through the C ABI.

Some callers cannot allocate device memory at all -- engines that give every
byte of device memory to their own pool at start-up, plugins handed only a
stream and buffers -- so they cannot open a handle (ts_moe_open allocates a
weight arena and a workspace).  ts_moe_route_noalloc takes the raw router and
keeps its scratch in the library's static device array.  Its results are
checked here against the handle-based ts_moe_route on the same router and
inputs, on two calls in a row (the static scratch keeps the previous call's
contents), with the tolerances the parity tests use (experts bit-exact, weights
within 1e-5, logits within 1e-4 of the largest).  Errors the device finds are
reported in the outputs (every idx -1, every w 0); that path is checked with a
router whose block scale is NaN and a bias holding NaN, each followed by a good
call on the same scratch."""
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


def _route_pair(shape, L, router, bias_d, x):
    from quantized_moe_routed_router_b200 import binding
    E, H, K, M = shape.num_experts, shape.hidden, shape.top_k, x.shape[0]
    idx = torch.full((M, K), 7, dtype=torch.int32, device="cuda")
    w = torch.full((M, K), 0.5, device="cuda")
    binding.route_noalloc(router, bias_d, None, E, H, K, shape.score, shape.bias_mode, x, idx, w)
    torch.cuda.synchronize()
    return idx, w


def test_route_noalloc_reports_device_errors_in_its_outputs():
    """A NaN router block scale (refused by ts_moe_open, here found on the
    device) and a NaN bias each turn every idx into -1 and every w into 0; the
    next good call on the same scratch routes normally again."""
    from quantized_moe_routed_router_b200 import binding
    shape = synth.CONFIGS[3].replace(moe_inter=64, max_tokens=16)
    L = synth.make_layer(shape, 0, device="cuda")
    moe = binding.MoE(shape, [L])
    E, K = shape.num_experts, shape.top_k
    bias_d = torch.from_numpy(L.bias).cuda()
    x = synth.make_x(shape, 1, 16, device="cuda")
    ref_idx = torch.empty(16, K, dtype=torch.int32, device="cuda")
    ref_w = torch.empty(16, K, device="cuda")
    moe.route(0, x, ref_idx, ref_w)

    bad_router = L.router.clone()
    bad_router[5, 34 * 3:34 * 3 + 2] = torch.tensor([0x00, 0x7E], dtype=torch.uint8)   # fp16 NaN scale, expert 5 block 3
    idx, w = _route_pair(shape, L, bad_router, bias_d, x)
    assert torch.all(idx == -1) and torch.all(w == 0)

    idx, w = _route_pair(shape, L, L.router, bias_d, x)              # the same scratch, good inputs again
    assert torch.equal(idx, ref_idx) and (w - ref_w).abs().max().item() <= 1e-5

    bad_bias = bias_d.clone()
    bad_bias[E - 1] = float("nan")
    idx, w = _route_pair(shape, L, L.router, bad_bias, x)
    assert torch.all(idx == -1) and torch.all(w == 0)

    idx, w = _route_pair(shape, L, L.router, bias_d, x)
    assert torch.equal(idx, ref_idx) and (w - ref_w).abs().max().item() <= 1e-5
    moe.device_status()
    moe.close()
