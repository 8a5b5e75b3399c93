"""GPU parity: the CUDA path (through the C ABI) against the FP64 oracle on
seeded inputs -- small shapes that still span several tiles, groups and a
ragged tail, every edge the kernels branch on, and the five workloads at full
size (the 24-layer stack on sampled layers)."""
import numpy as np
import pytest
import torch

from quantized_moe_routed_router_b200 import synth
from tests import parity

pytestmark = pytest.mark.gpu

S = synth.MoEShape
Q8, MX, I4 = synth.FMT_Q8_0, synth.FMT_MXFP4, synth.FMT_INT4_AFFINE

SMALL = {
    # name: shape  (cfg_id only seeds the draws)
    "q8_sel": S("q8_sel", 256, 256, 8, 2, cfg_id=101),
    "mx_odd_blocks_clamped_bias": S("mx", 96, 160, 5, 3, expert_fmt=MX, bias_mode=1, act=1, cfg_id=102),
    "q8_select_only_bias": S("q8so", 128, 192, 16, 4, bias_mode=2, cfg_id=103),
    "q8_all_norenorm_shared": S("ds", 128, 96, 16, 6, score=1, shared_inter=96, cfg_id=104),
    "k_equals_e": S("kee", 64, 128, 4, 4, cfg_id=105),
    "one_expert": S("one", 64, 64, 1, 1, cfg_id=106),
    "e256_k8": S("e256", 128, 64, 256, 8, cfg_id=107),
    "mx_large_k_window_split": S("mxk", 1088, 96, 4, 2, expert_fmt=MX, cfg_id=108),
    "q8_wide_inter": S("q8w", 64, 2080, 3, 2, cfg_id=109),
    # sigmoid scores with a selection-only correction bias (the MiniMax flow)
    "q8_sigmoid_correction_bias": S("sig", 256, 128, 16, 4, score=2, bias_mode=2, cfg_id=111),
    "mx_sigmoid_e256_k8": S("sigmx", 128, 128, 256, 8, expert_fmt=MX, score=2, bias_mode=2, cfg_id=112),
    "q8_sigmoid_no_bias": S("sig0", 64, 64, 8, 2, score=2, cfg_id=113),
    # INT4-affine experts (d * q + m per 32-block)
    "i4_sel": S("i4", 256, 160, 8, 2, expert_fmt=I4, cfg_id=114),
    "i4_odd_blocks_clamped_bias": S("i4c", 96, 224, 5, 3, expert_fmt=I4, bias_mode=1, act=1, cfg_id=115),
    "i4_sigmoid_e256_k8": S("i4sig", 128, 128, 256, 8, expert_fmt=I4, score=2, bias_mode=2, cfg_id=116),
    "i4_large_k_window_split": S("i4k", 1088, 96, 4, 2, expert_fmt=I4, cfg_id=117),
    "i4_wide_inter": S("i4w", 64, 2080, 3, 2, expert_fmt=I4, cfg_id=118),
}


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_moe_routed_router_b200 import build
    build.build()
    from oracle import oracle
    oracle.build()


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("M", [1, 3, 9, 16])
def test_small_shapes(name, M):
    shape = SMALL[name]
    rep = parity.check_shape(shape, M)
    assert rep.max_err_y <= 1e-2 * rep.rms_y


def test_small_with_xscale_and_per_expert_scale():
    from quantized_moe_routed_router_b200 import binding
    shape = S("xs", 128, 128, 8, 3, bias_mode=1, cfg_id=110)
    L = synth.make_layer(shape, 0, device="cuda")
    rng = np.random.default_rng(3)
    L.pes = rng.uniform(0.5, 1.5, 8).astype(np.float32)
    L.xscale = synth.bf16_bits_np(torch.tensor(rng.uniform(0.5, 2.0, 128), dtype=torch.float32).to(torch.bfloat16))
    moe = binding.MoE(shape, [L])
    rep = parity.check_shape(shape, 16, moe=moe, layers=[L])
    assert rep.max_err_y <= 1e-2 * rep.rms_y


def test_m0_is_a_noop_and_bad_calls_are_refused():
    from quantized_moe_routed_router_b200 import binding
    shape = SMALL["q8_sel"]
    moe = binding.MoE(shape, [synth.make_layer(shape, 0, device="cuda")])
    x = synth.make_x(shape, 0, 4, device="cuda")
    y = torch.full((4, shape.hidden), 7.0, device="cuda")
    moe.forward(0, x, None, y, M=0)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    with pytest.raises(binding.TsMoeError):
        moe.forward(1, x, None, y)                       # layer out of range
    with pytest.raises(binding.TsMoeError):
        moe.forward(0, synth.make_x(shape, 0, 17, device="cuda"), None, torch.zeros(17, 256, device="cuda"))
    with pytest.raises(binding.TsMoeError):
        moe.forward(0, x, None, None)                    # no output
    moe.device_status()


def test_deterministic_and_route_consistent():
    from quantized_moe_routed_router_b200 import binding
    shape = synth.CONFIGS[3].replace(cfg_id=111)
    L = [synth.make_layer(shape, 0, device="cuda")]
    moe = binding.MoE(shape, L)
    x = synth.make_x(shape, 0, 16, device="cuda")
    ys = []
    for _ in range(3):
        y = torch.empty(16, shape.hidden, device="cuda")
        moe.forward(0, x, None, y)
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
    idx = torch.empty(16, 4, dtype=torch.int32, device="cuda")
    w = torch.empty(16, 4, device="cuda")
    moe.route(0, x, idx, w)
    y1 = torch.empty_like(ys[0])
    moe.forward(0, x, None, y1)
    torch.cuda.synchronize()
    assert torch.equal(y1, ys[0])


def test_cuda_graph_capture_matches_eager():
    from quantized_moe_routed_router_b200 import binding
    shape = synth.CONFIGS[4].replace(cfg_id=112)
    L = [synth.make_layer(shape, 0, device="cuda")]
    moe = binding.MoE(shape, L)
    x = synth.make_x(shape, 0, 16, device="cuda")
    y_e = torch.empty(16, shape.hidden, device="cuda")
    moe.forward(0, x, None, y_e)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    y_g = torch.zeros_like(y_e)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            moe.forward(0, x, None, y_g, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y_g, y_e)
    moe.device_status()


@pytest.mark.parametrize("M", [16, 64])
def test_batch_rows_match_single_token_calls(M):
    from quantized_moe_routed_router_b200 import binding
    shape = SMALL["mx_odd_blocks_clamped_bias"].replace(max_tokens=M)
    L = [synth.make_layer(shape, 0, device="cuda")]
    moe = binding.MoE(shape, L)
    x = synth.make_x(shape, 0, M, device="cuda")
    yb = torch.empty(M, shape.hidden, device="cuda")
    moe.forward(0, x, None, yb)
    rms = yb.pow(2).mean().sqrt()
    for m in range(M):
        y1 = torch.empty(1, shape.hidden, device="cuda")
        moe.forward(0, x[m:m + 1].contiguous(), None, y1)
        assert (y1[0] - yb[m]).abs().max() <= 1e-4 * rms


# --------------------------------------------------------------------------- prefill (M > 16)
# A forward launch takes up to 64 tokens (four 16-token routing blocks) and
# reads each touched expert's weights once per 16 routes; longer calls run as
# several launches.  Experts with more than 16 routes become several entries.

@pytest.mark.parametrize("name,M", [("q8_all_norenorm_shared", 37), ("mx_odd_blocks_clamped_bias", 40),
                                    ("q8_sigmoid_correction_bias", 33), ("e256_k8", 64), ("one_expert", 17),
                                    ("k_equals_e", 64), ("i4_odd_blocks_clamped_bias", 50),
                                    ("q8_all_norenorm_shared", 100), ("one_expert", 130)])
def test_prefill_small(name, M):
    shape = SMALL[name].replace(max_tokens=M)
    rep = parity.check_shape(shape, M)
    assert rep.max_err_y <= 1e-2 * rep.rms_y


def test_prefill_launch_matches_calls_per_block():
    """A 45-token call (one launch) against calls of its 16-row blocks: the same
    experts for every token, and y within the summation-order noise (the
    launches cut the work differently); the residual epilogue is exact."""
    from quantized_moe_routed_router_b200 import binding
    shape = SMALL["q8_all_norenorm_shared"].replace(max_tokens=45)
    M, H, K = 45, shape.hidden, shape.top_k
    moe = binding.MoE(shape, [synth.make_layer(shape, 0, device="cuda")])
    x = synth.make_x(shape, 0, M, device="cuda")
    r = synth.make_x(shape, 0, M, device="cuda", tensor=synth.T_RESID)
    y_all, o_all = torch.empty(M, H, device="cuda"), r.clone()
    i_all = torch.empty(M, K, dtype=torch.int32, device="cuda")
    w_all = torch.empty(M, K, device="cuda")
    moe.forward(0, x, o_all, y_all)
    moe.route(0, x, i_all, w_all)
    rms = y_all.pow(2).mean().sqrt()
    for m0 in range(0, M, 16):
        m1 = min(M, m0 + 16)
        y_b = torch.empty(m1 - m0, H, device="cuda")
        i_b = torch.empty(m1 - m0, K, dtype=torch.int32, device="cuda")
        w_b = torch.empty(m1 - m0, K, device="cuda")
        moe.forward(0, x[m0:m1].contiguous(), None, y_b)
        moe.route(0, x[m0:m1].contiguous(), i_b, w_b)
        torch.cuda.synchronize()
        assert (y_b - y_all[m0:m1]).abs().max() <= 1e-4 * rms
        assert torch.equal(torch.sort(i_b, 1).values, torch.sort(i_all[m0:m1], 1).values)
        assert (w_b - w_all[m0:m1]).abs().max() <= 1e-6
    want = (r.float() + y_all).to(torch.bfloat16)
    assert torch.equal(o_all, want)
    moe.device_status()


def test_prefill_routes_beyond_16_per_expert():
    """64 tokens on 4 experts with top-2: every expert gets about 32 routes, so
    each is cut into entries of 16 (weights streamed once per entry)."""
    shape = S("dense4", 128, 96, 4, 2, cfg_id=119, max_tokens=64)
    rep = parity.check_shape(shape, 64)
    assert rep.max_err_y <= 1e-2 * rep.rms_y


@pytest.mark.parametrize("M,rows", [(40, [0, 7, 15, 16, 25, 31, 32, 39]), (64, [0, 13, 16, 31, 47, 48, 63]),
                                    (100, [0, 31, 63, 64, 80, 99])])
def test_prefill_gptoss_full_size_sampled(M, rows):
    """The gpt-oss-shaped MXFP4 layer at M = 40 and 64 (one launch) and 100 (64 + 36), sampled rows."""
    shape = synth.CONFIGS[3].replace(max_tokens=M)
    rep = parity.check_shape(shape, M, rows=rows)
    assert rep.max_err_y <= 1e-2 * rep.rms_y


# --------------------------------------------------------------------------- the five workloads at full size

# cfg 3 at every M of the benchmark's sweep: the router slicing, the read-back
# of the router items and the gate/up partition all switch with M
@pytest.mark.parametrize("cfg,M", [(1, 1), (2, 1), (2, 16), (3, 1), (3, 2), (3, 4), (3, 8), (3, 16), (4, 16),
                                   (8, 1), (8, 16)])
def test_workload_full_size(cfg, M):
    shape = synth.CONFIGS[cfg]
    if shape.num_layers > 1:
        shape = shape.replace(num_layers=1)          # one layer of a stack workload
    if M > shape.max_tokens:
        shape = shape.replace(max_tokens=M)
    rep = parity.check_shape(shape, M)
    assert rep.max_err_y <= 1e-2 * rep.rms_y


# dense FFN on the same kernels (E = 1, K = 1, weight 1): the deepseek2 dense lead
# layer (hidden 2048, dense width 10944, Q8_0) and a Mixtral-width dense FFN
@pytest.mark.parametrize("name,H,I,fmt", [("dense_lead_ds2", 2048, 10944, Q8), ("dense_mixtral_width", 4096, 14336, Q8),
                                          ("dense_mx", 2880, 2880, MX), ("dense_i4", 2880, 2880, I4)])
@pytest.mark.parametrize("M", [1, 16])
def test_dense_ffn(name, H, I, fmt, M):
    shape = S(name, H, I, 1, 1, expert_fmt=fmt, cfg_id=120 + H % 7 + fmt, max_tokens=16)
    rep = parity.check_shape(shape, M)
    assert rep.max_err_y <= 1e-2 * rep.rms_y


def test_workload_24_layer_stack_sampled():
    """The 24-layer gpt-oss-shaped stack in the launch configuration the
    benchmark times (one handle, all layers resident) at every M of its sweep
    (16, 8, 4, 2, 1): every layer's outputs are checked on sampled tokens
    against the oracle, three layers on the whole micro-batch."""
    from quantized_moe_routed_router_b200 import binding
    shape = synth.CONFIGS[5]
    layers = [synth.make_layer(shape, l, device="cuda") for l in range(shape.num_layers)]
    moe = binding.MoE(shape, layers)
    rng = np.random.default_rng(5)
    for M in (16, 8, 4, 2, 1):
        for l in range(shape.num_layers):
            rows = [0] if M == 1 else sorted(rng.choice(M, 2, replace=False).tolist())
            if l in (0, 11, 23):
                rows = None                              # whole micro-batch on three layers
            rep = parity.check_shape(shape, M, layer=l, rows=rows, moe=moe, layers=layers)
            assert rep.max_err_y <= 1e-2 * rep.rms_y
    moe.close()
