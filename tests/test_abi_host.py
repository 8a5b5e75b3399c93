"""Host-side checks of the C-ABI library (no GPU): it loads, exports every
declared symbol, refuses bad configurations before touching CUDA, and its
work-partition arithmetic covers every unit exactly once."""
import ctypes as C
import glob
import math
import os
import re

import numpy as np
import pytest
import torch

from quantized_moe_routed_router_b200 import build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    build.build()
    from quantized_moe_routed_router_b200 import binding
    return binding


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(ts_moe_\w+)\s*\(", txt))
    return sorted(names)


def test_exports_every_declared_symbol(B):
    names = declared_functions()
    assert {"ts_moe_open", "ts_moe_route", "ts_moe_forward", "ts_moe_close", "ts_moe_last_error",
            "ts_moe_device_status"} <= set(names)
    lib = C.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def _small_layers(shape, n=None):
    n = n or shape.num_layers
    return [synth.make_layer(shape, l) for l in range(n)]


SHAPE = synth.MoEShape("t", 64, 64, 4, 2, cfg_id=77, max_tokens=4)


@pytest.mark.parametrize("over,status,frag", [
    (dict(abi_version=99), 1, "abi"),
    (dict(hidden=48), 1, "hidden"),
    (dict(moe_inter=0), 1, "moe_inter"),
    (dict(num_experts=0), 1, "num_experts"),
    (dict(num_experts=300), 1, "num_experts"),
    (dict(top_k=9), 1, "top_k"),
    (dict(top_k=5), 1, "top_k"),           # > num_experts (4)
    (dict(max_tokens=65537), 1, "max_tokens"),
    (dict(max_tokens=0), 1, "max_tokens"),
    (dict(expert_fmt=3), 1, "expert_fmt"),
    (dict(score=3), 1, "score"),
    (dict(bias_mode=7), 1, "bias_mode"),
    (dict(act=5), 1, "act"),
    (dict(act=1, act_limit=-1.0), 1, "clamped"),
    (dict(shared_inter=40), 1, "shared_inter"),
    (dict(hidden=32768), 2, "hidden"),
    (dict(weights_mem=3), 1, "weights_mem"),
])
def test_open_time_refusals(B, over, status, frag):
    st, msg = B.validate(SHAPE, _small_layers(SHAPE), **over)
    assert st == status, msg
    assert frag in msg


@pytest.mark.parametrize("mt", [16, 17, 64, 65536])
def test_max_tokens_above_one_launch_is_accepted(B, mt):
    """Calls above 16 tokens run in 16-token launches, so max_tokens may exceed 16."""
    st, msg = B.validate(SHAPE, _small_layers(SHAPE), max_tokens=mt)
    assert st == 0, msg


def test_bias_and_shared_consistency(B):
    L = _small_layers(SHAPE)
    st, msg = B.validate(SHAPE, L, bias_mode=1)
    assert st == 1 and "router_bias" in msg
    L[0].bias = np.array([0.1, np.inf, 0.0, 0.0], np.float32)
    st, msg = B.validate(SHAPE.replace(bias_mode=1), L, bias_mode=1)
    assert st == 1 and "non-finite" in msg
    L[0].bias = np.zeros(4, np.float32)
    st, msg = B.validate(SHAPE.replace(bias_mode=1), L, bias_mode=1)
    assert st == 0, msg
    # shared expert: flags and blobs must agree; MXFP4 + shared is refused as unsupported
    Ls = _small_layers(SHAPE.replace(shared_inter=64))
    st, msg = B.validate(SHAPE, Ls)
    assert st == 1 and "shared" in msg
    st, msg = B.validate(SHAPE, _small_layers(SHAPE), shared_inter=64)
    assert st == 1 and "shared" in msg
    shm = SHAPE.replace(shared_inter=64, expert_fmt=synth.FMT_MXFP4, cfg_id=78)
    st, msg = B.validate(shm, _small_layers(shm))
    assert st == 2 and "shared" in msg
    ok = SHAPE.replace(shared_inter=64)
    assert B.validate(ok, _small_layers(ok))[0] == 0
    # INT4-affine experts are accepted, but not with a shared expert (the shared expert is Q8_0)
    i4 = SHAPE.replace(expert_fmt=synth.FMT_INT4_AFFINE, cfg_id=79)
    assert B.validate(i4, _small_layers(i4))[0] == 0
    i4s = i4.replace(shared_inter=64)
    st, msg = B.validate(i4s, _small_layers(i4s))
    assert st == 2 and "shared" in msg


def test_sigmoid_scoring_takes_a_selection_only_bias(B):
    L = _small_layers(SHAPE)
    for l in L:
        l.bias = np.zeros(4, np.float32)
    sig = SHAPE.replace(score=synth.SCORE_SIGMOID_RENORM)
    st, msg = B.validate(sig.replace(bias_mode=1), L, bias_mode=1, score=2)
    assert st == 1 and "sigmoid" in msg
    assert B.validate(sig.replace(bias_mode=2), L, bias_mode=2, score=2)[0] == 0
    assert B.validate(sig, _small_layers(sig), score=2)[0] == 0


def test_open_without_gpu_fails_cleanly(B):
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(B.TsMoeError) as ei:
        B.MoE(SHAPE, _small_layers(SHAPE))
    assert ei.value.status == 4


@pytest.mark.parametrize("U,NB", [(1, 148), (7, 148), (147, 148), (148, 148), (149, 148), (1000, 148), (5040, 148),
                                  (32, 3), (100, 7), (123457, 148)])
def test_partition_covers_every_unit_once(B, U, NB):
    lib = B.lib
    starts = [lib.ts_moe_debug_range_start(U, NB, b) for b in range(NB + 1)]
    assert starts[0] == 0 and starts[-1] == U
    assert all(starts[b] <= starts[b + 1] for b in range(NB))
    sizes = [starts[b + 1] - starts[b] for b in range(NB)]
    assert max(sizes) - min(sizes) <= 1               # balanced to one unit
    for u in list(range(min(U, 400))) + [U - 1]:
        b = lib.ts_moe_debug_owner_of(U, NB, u)
        assert starts[b] <= u < starts[b + 1]


@pytest.mark.parametrize("chunks,ngroups,NB", [(8, 4, 148), (45, 96, 148), (45, 672, 148), (44, 400, 148),
                                                (448, 128, 148), (3, 5, 4), (64, 1, 148)])
def test_split_groups_use_distinct_slots(B, chunks, ngroups, NB):
    """Every CTA writes at most one partial per slot, and the last contributor of
    a group finds exactly the CTAs that worked on it (empty ranges skipped)."""
    lib = B.lib
    U = chunks * ngroups
    starts = [lib.ts_moe_debug_range_start(U, NB, b) for b in range(NB + 1)]
    used = {}
    for G in range(ngroups):
        g0, g1 = G * chunks, (G + 1) * chunks
        workers = [b for b in range(NB) if starts[b] < starts[b + 1] and starts[b] < g1 and starts[b + 1] > g0]
        bf = lib.ts_moe_debug_owner_of(U, NB, g0)
        bl = lib.ts_moe_debug_owner_of(U, NB, g1 - 1)
        found = [b for b in range(bf, bl + 1) if starts[b] != starts[b + 1]]
        assert found == workers
        if len(workers) > 1:
            for b in workers:
                s = lib.ts_moe_debug_partial_slot(U, NB, b, g0)
                assert (b, s) not in used, (b, s, G, used.get((b, s)))
                used[(b, s)] = G
                covered = min(g1, starts[b + 1]) - max(g0, starts[b])
                assert covered > 0
            assert sum(min(g1, starts[b + 1]) - max(g0, starts[b]) for b in workers) == chunks


@pytest.mark.parametrize("G,NB,chunks", [(48, 148, 45), (49, 148, 45), (37, 148, 45), (4, 148, 90), (1, 148, 45),
                                          (148, 148, 45), (12, 148, 45), (70, 148, 64), (88, 148, 45)])
def test_aligned_partition_keeps_each_cta_in_one_group(G, NB, chunks):
    from quantized_moe_routed_router_b200 import binding as B
    lib = B.lib
    starts = [lib.ts_moe_debug_aligned_start(G, NB, chunks, b) for b in range(NB + 1)]
    assert starts[0] == 0 and starts[-1] == G * chunks
    assert all(a <= b for a, b in zip(starts, starts[1:]))          # contiguous cover of every unit once
    for b in range(NB):
        if starts[b + 1] > starts[b]:
            assert starts[b] // chunks == (starts[b + 1] - 1) // chunks  # never two groups in one range
    if lib.ts_moe_debug_use_aligned(G, NB):
        sizes = [starts[b + 1] - starts[b] for b in range(NB)]
        assert max(sizes) <= 1.1 * (G * chunks / NB) + 1                # the busiest CTA within 10 %
    assert lib.ts_moe_debug_use_aligned(48, 148) == 1                   # M = 1, 4 experts x 12 groups
    assert lib.ts_moe_debug_use_aligned(88, 148) == 0                   # 1.68 CTAs per group: too uneven
    assert lib.ts_moe_debug_use_aligned(200, 148) == 0                  # more groups than CTAs


def test_group_sizes_keep_the_most_warp_slots_busy():
    from quantized_moe_routed_router_b200 import binding as B
    for tiles in (1, 8, 15, 16, 17, 30, 31, 32, 33, 88, 128, 176, 180, 192, 256, 352, 360, 1368, 1792, 97):
        gs = B.lib.ts_moe_debug_group_size(tiles)
        if tiles <= 30:
            assert gs == tiles
            continue
        assert 15 <= gs <= 30
        slots = lambda g: -(-tiles // g) * 30
        best = min(slots(g) for g in range(15, 31))
        assert slots(gs) == best                                      # fewest idle consumer-warp slots
        assert gs == max(g for g in range(15, 31) if slots(g) == best)  # ties: the larger group
    assert B.lib.ts_moe_debug_group_size(256) == 30 and B.lib.ts_moe_debug_group_size(360) == 30


def _header_constants():
    """Enum and #define values of include/ts_moe.h, parsed from the text."""
    txt = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "ts_moe.h")).read(), flags=re.S)
    vals = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(TS_\w+)\s*=\s*(\d+)", txt)}
    vals.update({m.group(1): int(m.group(2)) for m in re.finditer(r"#define\s+(TS_\w+)\s+(\d+)u?\b", txt)})
    return vals


def test_header_constants_match_the_binding_and_the_generator(B):
    h = _header_constants()
    assert h["TS_MOE_ABI_VERSION"] == B.TS_MOE_ABI_VERSION
    assert (h["TS_FMT_Q8_0"], h["TS_FMT_MXFP4"], h["TS_FMT_INT4_AFFINE"]) == \
        (synth.FMT_Q8_0, synth.FMT_MXFP4, synth.FMT_INT4_AFFINE)
    assert (h["TS_SCORE_SOFTMAX_SELECTED"], h["TS_SCORE_SOFTMAX_ALL_NORENORM"], h["TS_SCORE_SIGMOID_RENORM"]) == \
        (synth.SCORE_SOFTMAX_SELECTED, synth.SCORE_SOFTMAX_ALL_NORENORM, synth.SCORE_SIGMOID_RENORM)
    assert (h["TS_BIAS_NONE"], h["TS_BIAS_LOGITS"], h["TS_BIAS_SELECT_ONLY"]) == \
        (synth.BIAS_NONE, synth.BIAS_LOGITS, synth.BIAS_SELECT_ONLY)
    assert (h["TS_ACT_SWIGLU"], h["TS_ACT_SWIGLU_CLAMPED"]) == (synth.ACT_SWIGLU, synth.ACT_SWIGLU_CLAMPED)
    assert (h["TS_MOE_MAX_TOKENS"], h["TS_MOE_MAX_TOPK"], h["TS_MOE_MAX_EXPERTS"]) == (16, 8, 256)
    assert h["TS_MOE_MAX_LAUNCH_TOKENS"] == 64
    assert h["TS_MOE_OK"] == 0 and h["TS_MOE_EDEVICE"] == 5


def test_coresidency_rule_of_the_layer_kernel(B):
    """The layer kernel's grid barrier needs every CTA resident at once: open
    refuses when the occupancy calculator allows none per SM, or fewer than the
    launch needs (the rule ts_moe_open applies, checked without a GPU)."""
    lib = B.lib
    nb = lib.ts_moe_debug_layer_ctas(148)
    assert nb == 148 and lib.ts_moe_debug_layer_ctas(600) == 512      # one CTA per SM, at most 512
    assert lib.ts_moe_debug_coresident(1, 148, nb) == 1
    assert lib.ts_moe_debug_coresident(0, 148, nb) == 0               # does not fit on an SM at all
    assert lib.ts_moe_debug_coresident(1, 100, nb) == 0               # fewer SMs than CTAs
    assert lib.ts_moe_debug_coresident(2, 74, nb) == 1
