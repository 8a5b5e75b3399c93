"""Seeded synthetic inputs for the routed MoE half (weights, router, bias, x, residual).

This module only *produces* inputs: random draws and their encoding into the
block formats the library accepts (Q8_0, MXFP4).  It holds none of the routed
half's arithmetic (no GEMV, no top-k, no activation, no combine), so the CUDA
path and the FP64 oracle can both consume what it writes without sharing code.

Block formats (the byte layouts the library's C ABI accepts):

* Q8_0, 34 bytes per 32 weights: ``{uint16 d (IEEE fp16 bits, little endian);
  int8 q[32]}``; element i of the block is ``d * q[i]``.  The pages fix only
  that Q8_0 dot products step over 32-element blocks (deepseek2 state page,
  ``build``).
* MXFP4, 17 bytes per 32 weights: ``{uint8 e (E8M0 scale 2^(e-127));
  uint8 qs[16]}``; element 2j is the low nibble of ``qs[j]``, element 2j+1 the
  high nibble; each nibble is an E2M1 code (sign bit 3, magnitudes
  0, .5, 1, 1.5, 2, 3, 4, 6).  The gpt-oss state page names MXFP4 as the
  format of its routed experts; the nibble order is this library's reading.
* INT4-affine, 20 bytes per 32 weights: ``{uint16 d; uint16 m (IEEE fp16
  bits); uint8 qs[16]}``; element 2j is the low nibble of ``qs[j]``, element
  2j+1 the high nibble; each nibble is an unsigned code q in [0, 15] and the
  weight is ``d * q + m``.  The gpt-oss state page only names the format
  (`BatchedRoutedScratch`: the batched-GEMV seam takes INT4-affine tensors
  only); block size, field types and layout are this library's reading,
  matched to the 32-element blocks of the others.

Matrices are row-major in blocks: a ``[R][C]`` matrix is R rows of C/32 blocks.
Expert tensors stack E such matrices: gate/up ``[E][I][H]``, down ``[E][H][I]``.

Encoding rules (input preparation, not the method):
* Q8_0: ``d = fp16(amax / 127)``, ``q = clamp(rint(w / d), -127, 127)``.
* MXFP4 (OCP MX v1.0 conversion): ``X = floor(log2(amax)) - 2``, ``e = X + 127``
  clamped to [0, 254]; codes are ``w / 2^X`` rounded to nearest-even on the
  E2M1 grid and saturated to +-6; an all-zero block gets e = 0.
* INT4-affine (min/max): ``m = fp16(min)``, ``d = fp16((max - min) / 15)``,
  ``q = clamp(rint((w - m) / d), 0, 15)`` with the fp16-rounded d and m
  (q = 0 when d = 0).

Seeds: every tensor draws from its own ``torch.Generator`` seeded from
(master seed, config id, layer, tensor id).  The same generator on the same
device type and torch version reproduces the same bytes.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

FMT_Q8_0 = 0
FMT_MXFP4 = 1
FMT_INT4_AFFINE = 2
SCORE_SOFTMAX_SELECTED = 0
SCORE_SOFTMAX_ALL_NORENORM = 1
SCORE_SIGMOID_RENORM = 2
BIAS_NONE = 0
BIAS_LOGITS = 1
BIAS_SELECT_ONLY = 2
ACT_SWIGLU = 0
ACT_SWIGLU_CLAMPED = 1

Q8_0_BLOCK_BYTES = 34
MXFP4_BLOCK_BYTES = 17
INT4_AFFINE_BLOCK_BYTES = 20

# tensor ids used in the per-tensor seed
T_ROUTER, T_BIAS, T_GATE, T_UP, T_DOWN, T_SH_GATE, T_SH_UP, T_SH_DOWN, T_X, T_RESID, T_PES, T_XSCALE = range(12)


def block_bytes(fmt: int) -> int:
    return {FMT_Q8_0: Q8_0_BLOCK_BYTES, FMT_MXFP4: MXFP4_BLOCK_BYTES, FMT_INT4_AFFINE: INT4_AFFINE_BLOCK_BYTES}[fmt]


def row_bytes(fmt: int, cols: int) -> int:
    assert cols % 32 == 0
    return cols // 32 * block_bytes(fmt)


@dataclass
class MoEShape:
    """One routed-MoE layer family: shapes and family flags."""

    name: str
    hidden: int
    moe_inter: int
    num_experts: int
    top_k: int
    expert_fmt: int = FMT_Q8_0
    score: int = SCORE_SOFTMAX_SELECTED
    bias_mode: int = BIAS_NONE
    act: int = ACT_SWIGLU
    act_alpha: float = 1.702
    act_limit: float = 7.0
    shared_inter: int = 0
    num_layers: int = 1
    max_tokens: int = 16
    weight_std: float = 0.02
    bias_std: float = 0.1
    cfg_id: int = 0

    def replace(self, **kw) -> "MoEShape":
        return dataclasses.replace(self, **kw)

    # algorithmic bytes of one expert's three matrices in the input format
    def expert_bytes(self) -> int:
        H, I = self.hidden, self.moe_inter
        return 2 * I * row_bytes(self.expert_fmt, H) + H * row_bytes(self.expert_fmt, I)

    def router_bytes(self) -> int:
        return self.num_experts * row_bytes(FMT_Q8_0, self.hidden)

    def shared_bytes(self) -> int:
        if not self.shared_inter:
            return 0
        H, S = self.hidden, self.shared_inter
        return 2 * S * row_bytes(FMT_Q8_0, H) + H * row_bytes(FMT_Q8_0, S)


# The five workloads (router weights are Q8_0 from N(0, 0.02) with unit x-scale).
CONFIGS = {
    1: MoEShape("tiny-q8_0", 256, 256, 8, 2, cfg_id=1, max_tokens=1),
    2: MoEShape("mixtral-shaped-q8_0", 4096, 14336, 8, 2, cfg_id=2),
    3: MoEShape("gpt-oss-20b-shaped-mxfp4", 2880, 2880, 32, 4, expert_fmt=FMT_MXFP4,
                bias_mode=BIAS_LOGITS, act=ACT_SWIGLU_CLAMPED, cfg_id=3),
    4: MoEShape("deepseek2-lite-shaped-q8_0", 2048, 1408, 64, 6,
                score=SCORE_SOFTMAX_ALL_NORENORM, shared_inter=2816, cfg_id=4),
    5: MoEShape("gpt-oss-20b-shaped-mxfp4-24-layer-stack", 2880, 2880, 32, 4, expert_fmt=FMT_MXFP4,
                bias_mode=BIAS_LOGITS, act=ACT_SWIGLU_CLAMPED, num_layers=24, cfg_id=5),
    # beyond the five: the rows that come next on the same kernels
    # the deepseek2 dense lead layer (dense SwiGLU, width 10944) as E = 1, K = 1, 24 layers (1.7 GB)
    6: MoEShape("deepseek2-dense-lead-shaped-q8_0-24-layer-stack", 2048, 10944, 1, 1, num_layers=24, cfg_id=6),
    # sigmoid scoring with a selection-only correction bias (the MiniMax flow), MiniMax-M2-like widths
    7: MoEShape("minimax-m2-shaped-q8_0-sigmoid-4-layer-stack", 3072, 1536, 256, 8, score=SCORE_SIGMOID_RENORM,
                bias_mode=BIAS_SELECT_ONLY, num_layers=4, cfg_id=7),
    # INT4-affine experts (the format the gpt-oss state page names for its batched-GEMV seam) on the
    # gpt-oss-shaped 24-layer stack: 11.9 GB of experts
    8: MoEShape("gpt-oss-20b-shaped-int4-affine-24-layer-stack", 2880, 2880, 32, 4, expert_fmt=FMT_INT4_AFFINE,
                bias_mode=BIAS_LOGITS, act=ACT_SWIGLU_CLAMPED, num_layers=24, cfg_id=8),
}


def tensor_seed(master: int, cfg_id: int, layer: int, tensor_id: int, sub: int = 0) -> int:
    s = 0x9E3779B97F4A7C15
    for v in (master, cfg_id, layer, tensor_id, sub):
        s = ((s ^ (v & 0xFFFFFFFF)) * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
        s ^= s >> 29
    return s & 0x7FFFFFFFFFFFFFFF


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn(shape, device, seed: int, std: float = 1.0) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(device, seed), device=device, dtype=torch.float32) * std


# ----------------------------------------------------------------------------- encoders

def encode_q8_0(w: torch.Tensor) -> torch.Tensor:
    """float32 [R, C] -> uint8 [R, C/32*34] Q8_0 blocks."""
    R, C = w.shape
    assert C % 32 == 0
    b = w.reshape(R, C // 32, 32)
    amax = b.abs().amax(dim=-1)
    d16 = (amax / 127.0).to(torch.float16)
    d = d16.to(torch.float32)
    safe = torch.where(d > 0, d, torch.ones_like(d))
    q = torch.where(d.unsqueeze(-1) > 0, torch.round(b / safe.unsqueeze(-1)), torch.zeros_like(b))
    q = q.clamp(-127, 127).to(torch.int8)
    out = torch.empty((R, C // 32, 34), dtype=torch.uint8, device=w.device)
    out[:, :, 0:2] = d16.contiguous().view(torch.uint8).reshape(R, C // 32, 2)
    out[:, :, 2:] = q.view(torch.uint8)
    return out.reshape(R, C // 32 * 34)


_E2M1_MIDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def encode_mxfp4(w: torch.Tensor) -> torch.Tensor:
    """float32 [R, C] -> uint8 [R, C/32*17] MXFP4 blocks (OCP MX conversion)."""
    R, C = w.shape
    assert C % 32 == 0
    b = w.reshape(R, C // 32, 32)
    amax = b.abs().amax(dim=-1)
    # floor(log2(amax)) from the float exponent (exact, no log rounding issues)
    _, ex = torch.frexp(amax)                       # amax = m * 2^ex, m in [0.5, 1)
    X = ex.to(torch.int32) - 1 - 2
    e = torch.where(amax > 0, (X + 127).clamp(0, 254), torch.zeros_like(X))
    scale = torch.ldexp(torch.ones_like(amax), (e - 127).to(torch.float32))
    v = b / scale.unsqueeze(-1)
    a = v.abs()
    mids = torch.tensor(_E2M1_MIDS, device=w.device, dtype=torch.float32)
    code = (a.unsqueeze(-1) > mids).sum(-1).to(torch.int32)          # ties rounded down so far
    tie = (a.unsqueeze(-1) == mids).any(-1)
    code = torch.where(tie & (code % 2 == 1), code + 1, code)          # ties to the even code
    code = code.clamp(0, 7)
    code = torch.where((v < 0) & (code > 0), code | 8, code)
    lo = code[..., 0::2]
    hi = code[..., 1::2]
    qs = (lo | (hi << 4)).to(torch.uint8)
    out = torch.empty((R, C // 32, 17), dtype=torch.uint8, device=w.device)
    out[:, :, 0] = e.to(torch.uint8)
    out[:, :, 1:] = qs
    return out.reshape(R, C // 32 * 17)


def encode_int4_affine(w: torch.Tensor) -> torch.Tensor:
    """float32 [R, C] -> uint8 [R, C/32*20] INT4-affine blocks (min/max encoder)."""
    R, C = w.shape
    assert C % 32 == 0
    b = w.reshape(R, C // 32, 32)
    lo, hi = b.amin(dim=-1), b.amax(dim=-1)
    m16 = lo.to(torch.float16)
    d16 = ((hi - lo) / 15.0).to(torch.float16)
    m, d = m16.to(torch.float32), d16.to(torch.float32)
    safe = torch.where(d > 0, d, torch.ones_like(d))
    q = torch.where(d.unsqueeze(-1) > 0, torch.round((b - m.unsqueeze(-1)) / safe.unsqueeze(-1)), torch.zeros_like(b))
    q = q.clamp(0, 15).to(torch.int32)
    qs = (q[..., 0::2] | (q[..., 1::2] << 4)).to(torch.uint8)
    out = torch.empty((R, C // 32, 20), dtype=torch.uint8, device=w.device)
    out[:, :, 0:2] = d16.contiguous().view(torch.uint8).reshape(R, C // 32, 2)
    out[:, :, 2:4] = m16.contiguous().view(torch.uint8).reshape(R, C // 32, 2)
    out[:, :, 4:] = qs
    return out.reshape(R, C // 32 * 20)


def encode(fmt: int, w: torch.Tensor) -> torch.Tensor:
    return {FMT_Q8_0: encode_q8_0, FMT_MXFP4: encode_mxfp4, FMT_INT4_AFFINE: encode_int4_affine}[fmt](w)


# ----------------------------------------------------------------------------- layer weights

@dataclass
class LayerBlobs:
    """One layer's inputs in the library's blob format (torch uint8 tensors on one device)."""

    router: torch.Tensor                      # [E][H/32*34] Q8_0
    gate: torch.Tensor                        # [E][I][rowbytes(H)]
    up: torch.Tensor
    down: torch.Tensor                        # [E][H][rowbytes(I)]
    bias: Optional[np.ndarray] = None         # [E] float32 (BF16-representable), host
    pes: Optional[np.ndarray] = None          # [E] float32 per-expert scale, host (None = ones)
    xscale: Optional[np.ndarray] = None       # [H] uint16 BF16 bits, host (None = ones)
    sh_gate: Optional[torch.Tensor] = None    # [S][rowbytes(H)] Q8_0
    sh_up: Optional[torch.Tensor] = None
    sh_down: Optional[torch.Tensor] = None    # [H][rowbytes(S)] Q8_0

    def to(self, device) -> "LayerBlobs":
        f = lambda t: None if t is None else t.to(device)
        return LayerBlobs(f(self.router), f(self.gate), f(self.up), f(self.down), self.bias, self.pes,
                          self.xscale, f(self.sh_gate), f(self.sh_up), f(self.sh_down))

    def host_numpy(self) -> dict:
        f = lambda t: None if t is None else t.detach().cpu().numpy()
        return dict(router=f(self.router), gate=f(self.gate), up=f(self.up), down=f(self.down),
                    bias=self.bias, pes=self.pes, xscale=self.xscale,
                    sh_gate=f(self.sh_gate), sh_up=f(self.sh_up), sh_down=f(self.sh_down))


def make_layer(shape: MoEShape, layer: int, device="cpu", master: int = 0,
               experts: Optional[list] = None) -> LayerBlobs:
    """Draw one layer: router/expert weights N(0, weight_std) encoded to the blob formats,
    router bias N(0, bias_std) rounded to BF16 (the pages narrow it to BF16 at repack)."""
    H, I, E, S = shape.hidden, shape.moe_inter, shape.num_experts, shape.shared_inter
    cid, fmt, std = shape.cfg_id, shape.expert_fmt, shape.weight_std
    router = encode_q8_0(randn((E, H), device, tensor_seed(master, cid, layer, T_ROUTER), std))
    rb_h, rb_i = row_bytes(fmt, H), row_bytes(fmt, I)
    gate = torch.empty((E, I, rb_h), dtype=torch.uint8, device=device)
    up = torch.empty((E, I, rb_h), dtype=torch.uint8, device=device)
    down = torch.empty((E, H, rb_i), dtype=torch.uint8, device=device)
    for e in range(E):
        gate[e] = encode(fmt, randn((I, H), device, tensor_seed(master, cid, layer, T_GATE, e), std))
        up[e] = encode(fmt, randn((I, H), device, tensor_seed(master, cid, layer, T_UP, e), std))
        down[e] = encode(fmt, randn((H, I), device, tensor_seed(master, cid, layer, T_DOWN, e), std))
    bias = None
    if shape.bias_mode != BIAS_NONE:
        b = randn((E,), "cpu", tensor_seed(master, cid, layer, T_BIAS), shape.bias_std)
        bias = b.to(torch.bfloat16).to(torch.float32).numpy().copy()
    sh = (None, None, None)
    if S:
        sh = (encode_q8_0(randn((S, H), device, tensor_seed(master, cid, layer, T_SH_GATE), std)),
              encode_q8_0(randn((S, H), device, tensor_seed(master, cid, layer, T_SH_UP), std)),
              encode_q8_0(randn((H, S), device, tensor_seed(master, cid, layer, T_SH_DOWN), std)))
    return LayerBlobs(router, gate, up, down, bias, None, None, *sh)


def make_x(shape: MoEShape, layer: int, M: int, device="cpu", master: int = 0, tensor=T_X,
           std: float = 1.0) -> torch.Tensor:
    """x (or the residual) for one layer: N(0, std) rounded to BF16; rows [0, M) of a
    16-row draw, so a smaller M is a prefix of the M=16 batch.  Returns torch.bfloat16 [M, H]."""
    rows = max(16, M)
    full = randn((rows, shape.hidden), device, tensor_seed(master, shape.cfg_id, layer, tensor), std)
    return full[:M].to(torch.bfloat16).contiguous()


def bf16_bits_np(t: torch.Tensor) -> np.ndarray:
    """torch bfloat16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
