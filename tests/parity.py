"""GPU-vs-oracle comparison used by the GPU tests and the smoke check.

Rules (the tolerances the routed-half spec states):
* selected expert sets equal the oracle's exactly, except at a token whose
  oracle gap between the K-th and (K+1)-th selection logit is below 1e-5;
  there the GPU's set must still be a valid top-K within 1e-5 and the outputs
  are compared with the oracle's forced-routing result for the GPU's set;
* routing weights within 1e-5 absolute (FP32 softmax vs FP64);
* max |y_gpu - y_ref| <= 1e-2 * RMS(y_ref) for the FP32 routed(+shared) sum;
* the BF16 residual output: out_gpu is bit-exactly bf16_rn(resid + y_gpu) in
  FP32 (the epilogue), and |out_gpu - out_ref| <= 1e-2 * RMS(out_ref) plus half
  a BF16 ulp of out_ref (the output rounding itself, which alone exceeds
  1e-2 * RMS wherever |out| >= 4).
"""
from __future__ import annotations

import os
from dataclasses import dataclass

import numpy as np
import torch

from oracle import oracle as O
from quantized_moe_routed_router_b200 import synth

TIE_GAP = 1e-5
REL_TOL = 1e-2


@dataclass
class ParityReport:
    max_err_y: float
    rms_y: float
    max_err_out: float
    rms_out: float
    near_ties: int
    idx_equal: bool


nthreads = O.nthreads


def host_layer(L: synth.LayerBlobs) -> dict:
    return L.host_numpy()


def compare(shape, Lh: dict, x: torch.Tensor, resid_in: torch.Tensor, idx_gpu: np.ndarray, w_gpu: np.ndarray,
            y_gpu: np.ndarray, out_gpu: np.ndarray, logits_gpu: np.ndarray = None, rows=None) -> ParityReport:
    """x / resid_in: the bf16 inputs (any device); *_gpu: host copies of the GPU outputs.
    `rows` optionally restricts the check to a subset of tokens (sampled parity)."""
    xb = synth.bf16_bits_np(x)
    rb = synth.bf16_bits_np(resid_in)
    M, K = xb.shape[0], shape.top_k
    toks = np.arange(M) if rows is None else np.asarray(rows)
    orc = O.Oracle(shape, Lh)
    ref = orc.forward(xb[toks], rb[toks], nthreads=nthreads())
    if logits_gpu is not None:
        lg = logits_gpu[toks]
        scale = max(1e-30, float(np.abs(ref.logits).max()))
        assert np.max(np.abs(lg - ref.logits)) <= 1e-4 * scale, "router logits differ"
    forced = ref.idx.copy()
    ties = 0
    idx_equal = True
    for i, t in enumerate(toks):
        srt = np.sort(ref.lsel[i].astype(np.float64))[::-1]
        gap = srt[K - 1] - srt[K] if K < shape.num_experts else np.inf
        g_set, r_set = set(idx_gpu[t].tolist()), set(ref.idx[i].tolist())
        if gap < TIE_GAP:
            ties += 1
            kth = srt[K - 1]
            assert all(ref.lsel[i, e] >= kth - TIE_GAP for e in g_set), f"token {t}: GPU set not a valid top-K"
            assert len(g_set) == K
            forced[i] = idx_gpu[t]
            if g_set != r_set:
                idx_equal = False
        else:
            assert g_set == r_set, f"token {t}: GPU experts {sorted(g_set)} vs oracle {sorted(r_set)}"
            # slot order: equal wherever adjacent selection logits are separated
            sl = ref.lsel[i, ref.idx[i]].astype(np.float64)
            if np.all(np.abs(np.diff(sl)) >= TIE_GAP):
                assert list(idx_gpu[t]) == list(ref.idx[i]), f"token {t}: slot order"
    if not np.array_equal(forced, ref.idx):
        ref = orc.forward(xb[toks], rb[toks], forced=forced, nthreads=nthreads())
    # weights in GPU slot order vs oracle weights of the same experts
    for i, t in enumerate(toks):
        wr = dict(zip(ref.idx[i].tolist(), ref.w[i].tolist()))
        for k in range(K):
            assert abs(w_gpu[t, k] - wr[int(idx_gpu[t, k])]) <= 1e-5, f"token {t} slot {k}: weight"
    yg = y_gpu[toks].astype(np.float64)
    rms_y = float(np.sqrt(np.mean(ref.y ** 2)))
    err_y = float(np.max(np.abs(yg - ref.y)))
    og = out_gpu[toks].astype(np.float64)
    rms_o = float(np.sqrt(np.mean(ref.out ** 2)))
    # epilogue: out = bf16_rn(float(resid) + y) exactly
    r32 = torch.from_numpy(rb[toks].view(np.int16)).view(torch.bfloat16).float()
    want = (r32 + torch.from_numpy(y_gpu[toks].astype(np.float32))).to(torch.bfloat16).float().numpy()
    assert np.array_equal(want, out_gpu[toks].astype(np.float32)), "out != bf16(resid + y)"
    _, ex = np.frexp(np.abs(ref.out))
    half_ulp = np.ldexp(1.0, ex - 9)                  # bf16: 8 significant bits
    slack = np.abs(og - ref.out) - half_ulp
    err_o = float(np.max(np.abs(og - ref.out)))
    rep = ParityReport(err_y, rms_y, err_o, rms_o, ties, idx_equal)
    assert err_y <= REL_TOL * rms_y, f"y: max err {err_y:.3e} > 1e-2 * RMS {rms_y:.3e}"
    assert float(np.max(slack)) <= REL_TOL * rms_o, f"out: max err beyond rounding {np.max(slack):.3e}"
    return rep


def run_layer(moe, shape, layer: int, x: torch.Tensor, resid: torch.Tensor):
    """Runs route + forward on the current stream; returns host copies (idx, w, logits, y, out)."""
    M, K, E, H = x.shape[0], shape.top_k, shape.num_experts, shape.hidden
    dev = x.device
    idx = torch.full((max(M, 1), K), -1, dtype=torch.int32, device=dev)
    w = torch.zeros((max(M, 1), K), dtype=torch.float32, device=dev)
    lg = torch.zeros((max(M, 1), E), dtype=torch.float32, device=dev)
    y = torch.full((max(M, 1), H), float("nan"), dtype=torch.float32, device=dev)
    out = resid.clone()
    moe.route(layer, x, idx, w, lg)
    moe.forward(layer, x, out, y)
    moe.device_status()
    torch.cuda.synchronize()
    return (idx.cpu().numpy(), w.cpu().numpy(), lg.cpu().numpy(), y.cpu().numpy(),
            out.float().cpu().numpy())


def check_shape(shape, M: int, device="cuda", layer: int = 0, rows=None, moe=None, layers=None, gen_device=None):
    """Builds (or reuses) a handle for `shape`, runs one layer at M tokens, compares with the oracle.
    Inputs are drawn on `gen_device` (default: `device`) and copied to `device`."""
    from quantized_moe_routed_router_b200 import binding
    gen = gen_device or device
    if layers is None:
        layers = [synth.make_layer(shape, l, device=gen) for l in range(shape.num_layers)]
    own = moe is None
    if own:
        moe = binding.MoE(shape, layers)
    x = synth.make_x(shape, layer, M, device=gen).to(device)
    resid = synth.make_x(shape, layer, M, device=gen, tensor=synth.T_RESID).to(device)
    idx, w, lg, y, out = run_layer(moe, shape, layer, x, resid)
    rep = compare(shape, layers[layer].host_numpy(), x, resid, idx, w, y, out, lg, rows=rows)
    if own:
        moe.close()
    return rep
