"""Reads the hand-computed examples under tests/golden/ into blobs + expected values.

Each file states a tiny layer entry by entry (all other weights are zero) and
the expected logits / selection / weights / outputs as closed-form expressions
(``sig`` = logistic sigmoid, ``exp``), derived by hand in the file's comments.
"""
from __future__ import annotations

import math
import os

import numpy as np

from quantized_moe_routed_router_b200 import synth

GOLDEN_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def evaluate(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"sig": _sig, "exp": math.exp}))


def _f16_bits(v: float) -> int:
    return int(np.array([v], np.float16).view(np.uint16)[0])


def _bf16_bits(v: float) -> int:
    b = np.array([v], np.float32).view(np.uint32)[0]
    assert b & 0xFFFF == 0, "golden x/resid values must be exact in bf16"
    return int(b >> 16)


def load(name: str):
    path = os.path.join(GOLDEN_DIR, name)
    cfg = {}
    q8scale, mxscale = None, 127
    entries, xs, rs, bias, expect = [], [], [], None, []
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "cfg":
            cfg = dict(t.split("=") for t in tok[1:])
        elif tok[0] == "q8scale":
            q8scale = float(tok[1])
        elif tok[0] == "mxscale":
            mxscale = int(tok[1])
        elif tok[0] == "x":
            xs.append((int(tok[1]), float(tok[2])))
        elif tok[0] == "resid":
            rs.append((int(tok[1]), float(tok[2])))
        elif tok[0] == "bias":
            bias = np.array([float(v) for v in tok[1:]], np.float32)
        elif tok[0] == "expect":
            expect.append(tok[1:])
        else:
            entries.append((tok[0], dict(t.split("=") for t in tok[1:])))
    H, I, E, K, S = (int(cfg[k]) for k in ("H", "I", "E", "K", "S"))
    fmt = {"q8_0": synth.FMT_Q8_0, "mxfp4": synth.FMT_MXFP4}[cfg["fmt"]]
    shape = synth.MoEShape(name, H, I, E, K, expert_fmt=fmt,
                           score={"sel": 0, "all": 1, "sigmoid": 2}[cfg["score"]],
                           bias_mode={"none": 0, "logits": 1, "select_only": 2}[cfg["bias"]],
                           act={"swiglu": 0, "clamped": 1}[cfg["act"]], shared_inter=S, max_tokens=1)

    def q8_blob(rows, cols, items):
        b = np.zeros((rows, cols // 32, 34), np.uint8)
        d = _f16_bits(q8scale)
        b[:, :, 0] = d & 0xFF
        b[:, :, 1] = d >> 8
        for r, c, q in items:
            b[r, c // 32, 2 + c % 32] = np.uint8(np.int8(q).view(np.uint8))
        return b.reshape(rows, -1)

    def mx_blob(rows, cols, items):
        b = np.zeros((rows, cols // 32, 17), np.uint8)
        b[:, :, 0] = mxscale
        for r, c, code in items:
            j = 1 + (c % 32) // 2
            if c % 2 == 0:
                b[r, c // 32, j] |= code
            else:
                b[r, c // 32, j] |= code << 4
        return b.reshape(rows, -1)

    def val(d):
        return int(d["q"]) if "q" in d else int(d["code"])

    blob = q8_blob if fmt == synth.FMT_Q8_0 else mx_blob
    router = q8_blob(E, H, [(int(d["e"]), int(d["n"]), int(d["q"])) for k, d in entries if k == "router"])
    gate = np.stack([blob(I, H, [(int(d["i"]), int(d["n"]), val(d)) for k, d in entries
                                 if k == "gate" and int(d["e"]) == e]) for e in range(E)])
    up = np.stack([blob(I, H, [(int(d["i"]), int(d["n"]), val(d)) for k, d in entries
                               if k == "up" and int(d["e"]) == e]) for e in range(E)])
    down = np.stack([blob(H, I, [(int(d["h"]), int(d["i"]), val(d)) for k, d in entries
                                 if k == "down" and int(d["e"]) == e]) for e in range(E)])
    layer = dict(router=router, gate=gate, up=up, down=down, bias=bias, pes=None, xscale=None)
    if S:
        layer["sh_gate"] = q8_blob(S, H, [(int(d["i"]), int(d["n"]), int(d["q"])) for k, d in entries if k == "sh_gate"])
        layer["sh_up"] = q8_blob(S, H, [(int(d["i"]), int(d["n"]), int(d["q"])) for k, d in entries if k == "sh_up"])
        layer["sh_down"] = q8_blob(H, S, [(int(d["h"]), int(d["i"]), int(d["q"])) for k, d in entries if k == "sh_down"])
    x = np.zeros((1, H), np.uint16)
    for n, v in xs:
        x[0, n] = _bf16_bits(v)
    resid = np.zeros((1, H), np.uint16)
    for n, v in rs:
        resid[0, n] = _bf16_bits(v)
    return shape, layer, x, resid, expect
