"""Pins the FP64 oracle to things other than itself (no GPU needed).

* block formats: exhaustive decode of every fp16 / bf16 bit pattern against
  numpy / torch, every E2M1 code against the OCP MX table, E8M0 against ldexp,
  every INT4-affine code against d * q + m and the encoder's exact round trip;
* router / top-k / weights against brute-force sorts and library softmax;
* the invariants the pages fix (softmax over the selected with per-expert
  ones; deepseek2 weights are the full softmax with no renorm so they sum to
  < 1; the bias acts only through the selection logits);
* activations against closed forms;
* the whole layer against a dense-gate-matrix numpy formulation on tiny inputs;
* hand-computed examples under tests/golden/;
* structural properties (batching and expert-relabelling invariance, zero
  down weights, the shared expert alone).
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import expit, softmax

from oracle import oracle as O
from quantized_moe_routed_router_b200 import synth
from tests import bruteforce as BF
from tests import golden_loader

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def setup_module(_):
    O.build()


# --------------------------------------------------------------------------- formats

def test_half_decode_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([O.half_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    # sign of zero too
    assert math.copysign(1.0, O.half_to_double(0x8000)) == -1.0


def test_bf16_decode_all_patterns():
    bits = np.arange(65536, dtype=np.int64)
    ref = torch.tensor(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([O.bf16_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_e2m1_all_codes_match_ocp_table():
    table = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for code in range(16):
        v = O.e2m1_to_double(code)
        mag = table[code & 7]
        assert abs(v) == mag
        if mag != 0:
            assert (v < 0) == bool(code & 8)


def test_e8m0_all_values():
    for e in range(255):
        assert O.e8m0_to_double(e) == math.ldexp(1.0, e - 127)
    assert math.isnan(O.e8m0_to_double(255))


def test_double_to_bf16_is_nearest_even():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.normal(0, 1, 3000), rng.normal(0, 1e-38, 300), rng.normal(0, 1e30, 300),
                           np.array([0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 65504.0, 3.0e38])])

    def bf(b):
        return (np.array([b], np.uint32) << 16).view(np.float32).astype(np.float64)[0]

    for v in vals:
        b = O.double_to_bf16(float(v))
        r = bf(b)
        lo, hi = bf((b - 1) & 0xFFFF), bf((b + 1) & 0xFFFF)
        err = abs(v - r)
        for n in (lo, hi):
            if np.isfinite(n) and np.sign(n) == np.sign(r):
                assert err <= abs(v - n)
                if err == abs(v - n) and err > 0:
                    assert b % 2 == 0  # tie -> even


def test_dequant_q8_0_exhaustive():
    scales = [0.03125, 1.0, 0.0001234, 6.1e-5, 3.0e-8, 1.5, -0.25, 0.0]
    rows = len(scales)
    blob = np.zeros((rows, 8, 34), np.uint8)
    qs = np.arange(-128, 128, dtype=np.int64).astype(np.int8).reshape(8, 32)
    for r, s in enumerate(scales):
        d = np.array([s], np.float16).view(np.uint16)[0]
        blob[r, :, 0] = d & 0xFF
        blob[r, :, 1] = d >> 8
        blob[r, :, 2:] = qs.view(np.uint8)
    got = O.dequant(0, blob.reshape(rows, -1), rows, 256)
    for r, s in enumerate(scales):
        d = float(np.float16(s))
        assert np.array_equal(got[r], d * np.arange(-128, 128, dtype=np.float64))


def test_dequant_mxfp4_exhaustive():
    table = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    exps = list(range(100, 151)) + [0, 1, 254]
    rows = len(exps)
    blob = np.zeros((rows, 1, 17), np.uint8)
    lo = np.arange(16) % 16
    hi = (np.arange(16) * 7 + 3) % 16
    for r, e in enumerate(exps):
        blob[r, 0, 0] = e
        blob[r, 0, 1:] = lo | (hi << 4)
    got = O.dequant(1, blob.reshape(rows, -1), rows, 32)
    for r, e in enumerate(exps):
        s = math.ldexp(1.0, e - 127)
        sign = lambda c: -1.0 if c & 8 else 1.0
        ref = np.empty(32)
        ref[0::2] = [sign(c) * table[c & 7] * s for c in lo]
        ref[1::2] = [sign(c) * table[c & 7] * s for c in hi]
        assert np.array_equal(got[r], ref)


def test_dequant_int4_affine_exhaustive():
    """Every 4-bit code in both nibble positions, under fp16 scales and offsets
    of both signs, subnormal, zero and large, against d * q + m with numpy's
    own fp16 decoding."""
    pairs = [(0.03125, 0.0), (0.03125, -0.25), (1.0, -7.5), (6.1e-5, 3.0e-8), (3.0e-8, -6.1e-5),
             (0.0, 0.5), (1.5, 1000.0), (-0.125, 0.0625), (4096.0, -65504.0)]
    rows = len(pairs)
    blob = np.zeros((rows, 1, 20), np.uint8)
    lo = np.arange(16)
    hi = (np.arange(16) * 7 + 3) % 16
    for r, (d, m) in enumerate(pairs):
        blob[r, 0, 0:2] = np.array([d], np.float16).view(np.uint8)
        blob[r, 0, 2:4] = np.array([m], np.float16).view(np.uint8)
        blob[r, 0, 4:] = lo | (hi << 4)
    got = O.dequant(synth.FMT_INT4_AFFINE, blob.reshape(rows, -1), rows, 32)
    for r, (d, m) in enumerate(pairs):
        d16, m16 = float(np.float16(d)), float(np.float16(m))
        ref = np.empty(32)
        ref[0::2] = d16 * lo + m16
        ref[1::2] = d16 * hi + m16
        assert np.array_equal(got[r], ref), r


def test_int4_affine_encoder_round_trip():
    """Blocks whose values lie on an fp16-exact grid m + d*q come back exactly
    (this ties the encoder's byte layout to the oracle's independent decoder);
    N(0, 0.02) blocks come back within half a step plus the fp16 rounding of m."""
    rng = np.random.default_rng(11)
    R, C = 6, 128
    d = np.ldexp(1.0, -rng.integers(3, 9, (R, C // 32)))
    m = -d * rng.integers(0, 40, (R, C // 32))
    q = rng.integers(0, 16, (R, C // 32, 32))
    q[:, :, 0], q[:, :, 1] = 0, 15                      # the encoder's min and max sit on the grid
    w = (m[..., None] + d[..., None] * q).reshape(R, C)
    blob = synth.encode_int4_affine(torch.tensor(w, dtype=torch.float32)).numpy()
    assert blob.shape == (R, C // 32 * synth.INT4_AFFINE_BLOCK_BYTES)
    assert np.array_equal(O.dequant(synth.FMT_INT4_AFFINE, blob, R, C), w)
    w2 = rng.normal(0, 0.02, (R, C)).astype(np.float32)
    deq = O.dequant(synth.FMT_INT4_AFFINE, synth.encode_int4_affine(torch.tensor(w2)).numpy(), R, C)
    b = w2.reshape(R, C // 32, 32).astype(np.float64)
    step = ((b.max(-1) - b.min(-1)) / 15.0)[..., None]
    err = np.abs(deq.reshape(R, C // 32, 32) - b)
    assert np.all(err <= 0.5 * step * (1 + 2e-3) + 2e-3 * np.abs(b.min(-1))[..., None] + 1e-9)


# --------------------------------------------------------------------------- router / selection

def _tiny(fmt=0, score=0, bias=0, act=0, S=0, E=4, K=2, H=64, I=64):
    return synth.MoEShape("tiny", H, I, E, K, expert_fmt=fmt, score=score, bias_mode=bias, act=act,
                          shared_inter=S, cfg_id=90 + 10 * fmt + score, max_tokens=8)


def _layer_np(shape, layer=0, xscale=False, pes=False):
    L = synth.make_layer(shape, layer).host_numpy()
    rng = np.random.default_rng(7)
    if xscale:
        L["xscale"] = synth.bf16_bits_np(torch.tensor(rng.uniform(0.5, 1.5, shape.hidden), dtype=torch.float32)
                                         .to(torch.bfloat16))
    if pes:
        L["pes"] = rng.uniform(0.5, 2.0, shape.num_experts).astype(np.float32)
    return L


def _x(shape, M, layer=0, tensor=synth.T_X):
    return synth.bf16_bits_np(synth.make_x(shape, layer, M, tensor=tensor))


def test_router_logits_match_dense_matmul():
    shape = _tiny(E=6, H=128)
    L = _layer_np(shape, xscale=True)
    x = _x(shape, 5)
    got = O.Oracle(shape, L).router_logits(x)
    X = BF.bf16_bits_to_f64(x) * BF.bf16_bits_to_f64(L["xscale"])
    ref = (X @ BF.decode_q8_0(L["router"], 6, 128).T).astype(np.float32)
    assert np.array_equal(got, ref)


def test_topk_matches_bruteforce_with_ties():
    shape = _tiny(E=16, K=5)
    orc = O.Oracle(shape, _layer_np(shape))
    rng = np.random.default_rng(3)
    logits = rng.integers(-3, 4, size=(40, 16)).astype(np.float32)   # many exact ties
    idx, _, _ = orc.select(logits)
    for m in range(40):
        assert list(idx[m]) == list(BF.topk_bruteforce(logits[m], 5))


def test_topk_two_experts_closed_form():
    shape = _tiny(E=2, K=1)
    orc = O.Oracle(shape, _layer_np(shape))
    idx, w, _ = orc.select(np.array([[0.3, 0.7], [0.7, 0.3], [0.5, 0.5]], np.float32))
    assert list(idx[:, 0]) == [1, 0, 0]
    assert np.all(w == 1.0)
    shape2 = _tiny(E=2, K=2)
    idx, w, _ = O.Oracle(shape2, _layer_np(shape2)).select(np.array([[0.25, -0.5]], np.float32))
    assert list(idx[0]) == [0, 1]
    assert abs(w[0, 0] - expit(0.75)) < 1e-15 and abs(w[0, 1] - expit(-0.75)) < 1e-15


def test_softmax_over_selected_invariants():
    shape = _tiny(E=8, K=3)
    orc = O.Oracle(shape, _layer_np(shape))
    logits = np.random.default_rng(5).normal(0, 2, (20, 8)).astype(np.float32)
    idx, w, _ = orc.select(logits)
    assert np.allclose(w.sum(1), 1.0, atol=1e-15, rtol=0)
    for m in range(20):
        assert np.allclose(w[m], softmax(logits[m, idx[m]].astype(np.float64)), atol=1e-15, rtol=0)
        assert np.all(np.diff(w[m]) <= 0)  # slot order = descending logit
    # K = E reproduces the full softmax (in slot order)
    shapeE = _tiny(E=8, K=8)
    idx, w, _ = O.Oracle(shapeE, _layer_np(shapeE)).select(logits)
    for m in range(20):
        assert np.allclose(w[m], softmax(logits[m].astype(np.float64))[idx[m]], atol=1e-15, rtol=0)


def test_per_expert_scale_multiplies_after_softmax():
    shape = _tiny(E=8, K=3)
    L = _layer_np(shape, pes=True)
    logits = np.random.default_rng(9).normal(0, 2, (10, 8)).astype(np.float32)
    idx, w, _ = O.Oracle(shape, L).select(logits)
    idx1, w1, _ = O.Oracle(shape, dict(L, pes=None)).select(logits)
    assert np.array_equal(idx, idx1)
    assert np.allclose(w, w1 * L["pes"][idx], atol=1e-15, rtol=0)
    ones = dict(L, pes=np.ones(8, np.float32))
    _, w2, _ = O.Oracle(shape, ones).select(logits)
    assert np.array_equal(w2, w1)


def test_deepseek2_all_softmax_no_renorm():
    shape = _tiny(E=16, K=6, score=1)
    orc = O.Oracle(shape, _layer_np(shape))
    logits = np.random.default_rng(11).normal(0, 1, (25, 16)).astype(np.float32)
    idx, w, _ = orc.select(logits)
    for m in range(25):
        p = softmax(logits[m].astype(np.float64))
        assert np.allclose(w[m], p[idx[m]], atol=1e-15, rtol=0)
        assert 0 < w[m].sum() < 1
        assert list(idx[m]) == list(np.argsort(-p, kind="stable")[:6])
    shapeE = _tiny(E=6, K=6, score=1)
    idx, w, _ = O.Oracle(shapeE, _layer_np(shapeE)).select(logits[:, :6])
    assert np.allclose(w.sum(1), 1.0, atol=1e-14, rtol=0)


@pytest.mark.parametrize("mode", [1, 2])
def test_bias_moves_selection_only_through_biased_logits(mode):
    shape = _tiny(E=8, K=3, bias=mode)
    L = _layer_np(shape)
    rng = np.random.default_rng(13)
    logits = rng.normal(0, 1, (30, 8)).astype(np.float32)
    b = torch.tensor(rng.normal(0, 0.5, 8), dtype=torch.float32).to(torch.bfloat16).float().numpy()
    idx, w, lsel = O.Oracle(shape, dict(L, bias=b)).select(logits)
    assert np.array_equal(lsel, (logits + b).astype(np.float32))
    for m in range(30):
        assert list(idx[m]) == list(BF.topk_bruteforce(lsel[m], 3))
        src = lsel[m] if mode == 1 else logits[m]
        assert np.allclose(w[m], softmax(src[idx[m]].astype(np.float64)), atol=1e-15, rtol=0)
    # a uniform bias changes nothing (exactly representable shift)
    u = np.full(8, 0.5, np.float32)
    idx_u, w_u, _ = O.Oracle(shape, dict(L, bias=u)).select(logits.astype(np.float32))
    idx_0, w_0, _ = O.Oracle(shape.replace(bias_mode=0), dict(L, bias=None)).select(logits)
    assert np.array_equal(idx_u, idx_0)
    assert np.allclose(w_u, w_0, atol=1e-7, rtol=0)
    # a large bias forces an expert into every token's set
    big = np.zeros(8, np.float32)
    big[5] = 1e3
    idx_b, _, _ = O.Oracle(shape, dict(L, bias=big)).select(logits)
    assert np.all(idx_b[:, 0] == 5)
    # LOGITS mode equals the unbiased path fed l + b
    if mode == 1:
        idx_f, w_f, _ = O.Oracle(shape.replace(bias_mode=0), dict(L, bias=None)).select(lsel)
        assert np.array_equal(idx_f, idx) and np.array_equal(w_f, w)


def test_sigmoid_scores_two_experts_closed_form():
    # sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4: slot order by score, weights 3/4 / (5/4) = 0.6 and 0.4
    shape = _tiny(E=2, K=2, score=2)
    idx, w, lsel = O.Oracle(shape, _layer_np(shape)).select(np.array([[0.0, math.log(3.0)]], np.float32))
    assert list(idx[0]) == [1, 0]
    assert abs(w[0, 0] - 0.6) < 1e-7 and abs(w[0, 1] - 0.4) < 1e-7
    assert abs(lsel[0, 0] - 0.5) == 0 and abs(lsel[0, 1] - 0.75) < 1e-7
    shape1 = _tiny(E=2, K=1, score=2)
    _, w1, _ = O.Oracle(shape1, _layer_np(shape1)).select(np.array([[-2.0, 1.0]], np.float32))
    assert w1[0, 0] == 1.0


def test_sigmoid_scoring_invariants():
    shape = _tiny(E=8, K=3, score=2)
    L = _layer_np(shape)
    rng = np.random.default_rng(21)
    logits = rng.normal(0, 2, (30, 8)).astype(np.float32)
    idx, w, _ = O.Oracle(shape, L).select(logits)
    # sigmoid is increasing: without a bias the set and slot order are those of the logits
    idx_soft, _, _ = O.Oracle(shape.replace(score=0), L).select(logits)
    assert np.array_equal(idx, idx_soft)
    assert np.allclose(w.sum(1), 1.0, atol=1e-15, rtol=0)
    for m in range(30):
        s = expit(logits[m, idx[m]].astype(np.float64))
        assert np.allclose(w[m], s / s.sum(), atol=1e-15, rtol=0)
    # the correction bias only moves the selection: selection on s + b, weights from s alone
    b = rng.normal(0, 0.3, 8).astype(np.float32)
    sb = shape.replace(bias_mode=2)
    idx_b, w_b, lsel_b = O.Oracle(sb, dict(L, bias=b)).select(logits)
    for m in range(30):
        key = (expit(logits[m].astype(np.float64)) + b.astype(np.float64)).astype(np.float32)
        assert np.array_equal(lsel_b[m], key)
        assert list(idx_b[m]) == list(BF.topk_bruteforce(key, 3))
        s = expit(logits[m, idx_b[m]].astype(np.float64))
        assert np.allclose(w_b[m], s / s.sum(), atol=1e-15, rtol=0)
    big = np.zeros(8, np.float32)
    big[6] = 10.0  # beyond any score difference: expert 6 is always selected first
    idx_g, _, _ = O.Oracle(sb, dict(L, bias=big)).select(logits)
    assert np.all(idx_g[:, 0] == 6)
    # K = E: all experts, weights = scores / their sum
    sE = _tiny(E=6, K=6, score=2)
    idx_e, w_e, _ = O.Oracle(sE, _layer_np(sE)).select(logits[:, :6])
    for m in range(30):
        s = expit(logits[m, :6].astype(np.float64))
        assert np.allclose(w_e[m], (s / s.sum())[idx_e[m]], atol=1e-15, rtol=0)


# --------------------------------------------------------------------------- activations

def test_activation_closed_forms():
    for g in (-3.0, -1.0, 0.0, 0.5, 2.0, 9.0):
        for u in (-8.0, -1.0, 0.0, 0.25, 3.0, 7.5):
            assert O.act(0, 1.702, 7.0, g, u) == pytest.approx(g / (1 + math.exp(-g)) * u, rel=1e-15, abs=1e-300)
            gc, uc = min(g, 7.0), max(min(u, 7.0), -7.0)
            assert O.act(1, 1.702, 7.0, g, u) == pytest.approx(gc / (1 + math.exp(-1.702 * gc)) * (uc + 1),
                                                               rel=1e-15, abs=1e-300)
    assert O.act(0, 0, 0, 0.0, 5.0) == 0.0
    assert O.act(1, 1.702, 7.0, 3.0, -1.0) == 0.0            # u = -1 zeroes the clamped unit
    assert O.act(1, 1.702, 7.0, 12.0, 2.0) == O.act(1, 1.702, 7.0, 7.0, 2.0)   # gate clamped from above only
    assert O.act(1, 1.702, 7.0, -12.0, 2.0) != O.act(1, 1.702, 7.0, -7.0, 2.0)
    assert O.act(1, 1.702, 7.0, 1.0, 100.0) == O.act(1, 1.702, 7.0, 1.0, 7.0)
    assert O.act(1, 1.702, 7.0, 1.0, -100.0) == O.act(1, 1.702, 7.0, 1.0, -7.0)


# --------------------------------------------------------------------------- whole layer

CASES = [
    dict(fmt=0, score=0, bias=0, act=0, S=0, E=4, K=2),
    dict(fmt=1, score=0, bias=1, act=1, S=0, E=4, K=2),
    dict(fmt=1, score=0, bias=2, act=1, S=0, E=5, K=3),
    dict(fmt=0, score=1, bias=0, act=0, S=96, E=6, K=3),
    dict(fmt=0, score=0, bias=0, act=0, S=0, E=4, K=4),
    dict(fmt=0, score=2, bias=2, act=0, S=0, E=8, K=3),
    dict(fmt=1, score=2, bias=0, act=1, S=0, E=6, K=2),
    dict(fmt=2, score=0, bias=0, act=0, S=0, E=4, K=2),
    dict(fmt=2, score=1, bias=0, act=0, S=96, E=6, K=3),
    dict(fmt=2, score=0, bias=1, act=1, S=0, E=5, K=3),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()))
def test_layer_matches_dense_bruteforce(case):
    shape = _tiny(**case)
    L = _layer_np(shape, xscale=True, pes=True)
    if shape.bias_mode:
        L["bias"] = torch.tensor(np.random.default_rng(2).normal(0, 0.3, shape.num_experts),
                                 dtype=torch.float32).to(torch.bfloat16).float().numpy()
    x = _x(shape, 4)
    resid = _x(shape, 4, tensor=synth.T_RESID)
    r = O.Oracle(shape, L).forward(x, resid)
    logits, idx, w, Y, OUT = BF.layer_bruteforce(shape, L, x, resid)
    assert np.array_equal(r.logits, logits)
    assert np.array_equal(r.idx, idx)
    assert np.allclose(r.w, w, rtol=0, atol=1e-14)
    scale = np.sqrt(np.mean(Y ** 2))
    assert np.max(np.abs(r.y - Y)) <= 1e-12 * scale
    assert np.max(np.abs(r.out - OUT)) <= 1e-12 * max(1.0, scale)
    # bf16 output is the round-to-nearest-even of out
    ref_bf = torch.tensor(OUT).to(torch.float32)
    exact_f32 = (ref_bf.double().numpy() == OUT)
    rb = ref_bf.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r.out_bf16[exact_f32], rb[exact_f32])


def test_layer_with_threads_equals_single_thread():
    shape = _tiny(fmt=1, bias=1, act=1)
    L = _layer_np(shape)
    x = _x(shape, 6)
    a = O.Oracle(shape, L).forward(x, nthreads=1)
    b = O.Oracle(shape, L).forward(x, nthreads=3)
    assert np.array_equal(a.y, b.y) and np.array_equal(a.idx, b.idx)


@pytest.mark.parametrize("name", ["two_expert_swiglu_sel_k2.txt", "deepseek2_all_norenorm_shared_k1.txt",
                                  "gptoss_clamped_bias_mxfp4_k2.txt", "minimax_sigmoid_correction_bias_k2.txt"])
def test_hand_computed_examples(name):
    shape, L, x, resid, expect = golden_loader.load(name)
    r = O.Oracle(shape, L).forward(x, resid)
    touched = set()
    for e in expect:
        kind = e[0]
        if kind == "logits":
            assert np.allclose(r.logits[0], [golden_loader.evaluate(v) for v in e[1:]], rtol=0, atol=0)
        elif kind == "idx":
            assert list(r.idx[0]) == [int(v) for v in e[1:]]
        elif kind == "w":
            assert np.allclose(r.w[0], [golden_loader.evaluate(v) for v in e[1:]], rtol=1e-14, atol=0)
        elif kind == "y":
            h = int(e[1])
            touched.add(h)
            assert r.y[0, h] == pytest.approx(golden_loader.evaluate(e[2]), rel=1e-14, abs=1e-300)
        elif kind == "out":
            assert r.out[0, int(e[1])] == pytest.approx(golden_loader.evaluate(e[2]), rel=1e-14)
    others = [h for h in range(shape.hidden) if h not in touched]
    assert np.all(r.y[0, others] == 0.0)


def test_batching_invariance_bit_exact():
    shape = _tiny(fmt=0, score=1, S=64, E=6, K=3)
    L = _layer_np(shape)
    x = _x(shape, 5)
    full = O.Oracle(shape, L).forward(x)
    for m in range(5):
        one = O.Oracle(shape, L).forward(x[m:m + 1])
        assert np.array_equal(one.y[0], full.y[m])
        assert np.array_equal(one.idx[0], full.idx[m])


def test_expert_relabelling_invariance():
    shape = _tiny(fmt=1, bias=1, act=1, E=6, K=2)
    L = _layer_np(shape)
    L["bias"] = np.linspace(-0.25, 0.25, 6).astype(np.float32)
    perm = np.array([3, 0, 5, 1, 4, 2])
    P = dict(L)
    E, H = shape.num_experts, shape.hidden
    P["router"] = L["router"].reshape(E, -1)[perm]
    for k in ("gate", "up", "down"):
        P[k] = L[k][perm]
    P["bias"] = L["bias"][perm]
    x = _x(shape, 4)
    a = O.Oracle(shape, L).forward(x)
    b = O.Oracle(shape, P).forward(x)
    assert np.array_equal(perm[b.idx], a.idx)
    assert np.max(np.abs(a.y - b.y)) <= 1e-13 * np.abs(a.y).max()


def test_zero_down_weights_leave_only_the_shared_expert():
    shape = _tiny(fmt=0, score=1, S=64, E=4, K=2)
    L = _layer_np(shape)
    Z = dict(L)
    z = L["down"].reshape(shape.num_experts, shape.hidden, -1).copy()
    z.reshape(shape.num_experts, shape.hidden, -1, 34)[..., 2:] = 0          # q = 0
    Z["down"] = z
    x = _x(shape, 3)
    r = O.Oracle(shape, Z).forward(x)
    X = BF.bf16_bits_to_f64(x)
    Sg = BF.decode_q8_0(L["sh_gate"], 64, shape.hidden)
    Su = BF.decode_q8_0(L["sh_up"], 64, shape.hidden)
    Sd = BF.decode_q8_0(L["sh_down"], shape.hidden, 64)
    dense = BF.act_np(0, X @ Sg.T, X @ Su.T) @ Sd.T
    assert np.max(np.abs(r.y - dense)) <= 1e-12 * np.abs(dense).max()
    # and with no shared expert the output is exactly zero
    shape0 = shape.replace(shared_inter=0)
    Z0 = {k: v for k, v in Z.items() if not k.startswith("sh_")}
    assert np.all(O.Oracle(shape0, Z0).forward(x).y == 0.0)


def test_zero_per_expert_scale_leaves_dense_shared_swiglu():
    shape = _tiny(fmt=0, score=0, S=64, E=4, K=2)
    L = _layer_np(shape)
    L["pes"] = np.zeros(4, np.float32)
    x = _x(shape, 2)
    r = O.Oracle(shape, L).forward(x)
    X = BF.bf16_bits_to_f64(x)
    dense = BF.act_np(0, X @ BF.decode_q8_0(L["sh_gate"], 64, 64).T, X @ BF.decode_q8_0(L["sh_up"], 64, 64).T) \
        @ BF.decode_q8_0(L["sh_down"], 64, 64).T
    assert np.max(np.abs(r.y - dense)) <= 1e-12 * np.abs(dense).max()


def test_forced_routing_equals_free_routing_on_its_own_choice():
    shape = _tiny(fmt=1, bias=1, act=1, E=6, K=3)
    L = _layer_np(shape)
    L["bias"] = np.zeros(6, np.float32)
    x = _x(shape, 3)
    free = O.Oracle(shape, L).forward(x)
    forced = O.Oracle(shape, L).forward(x, forced=free.idx)
    assert np.array_equal(free.y, forced.y)
    other = free.idx[:, ::-1].copy()                     # same sets, other slot order
    f2 = O.Oracle(shape, L).forward(x, forced=other)
    assert np.max(np.abs(f2.y - free.y)) <= 1e-13 * np.abs(free.y).max()
