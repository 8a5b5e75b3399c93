"""ctypes binding of the FP64 CPU oracle (``ts_moe_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.  It shares no code
with the CUDA library; the two meet only through the seeded input blobs.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ts_moe_oracle.cpp")
LIB = os.path.join(HERE, "libts_moe_oracle.so")


def nthreads() -> int:
    """Host threads the oracle runs on: the cores this process may use."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except Exception:
        return os.cpu_count() or 1


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (plain IEEE FP64, no fast-math)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
                               "-ffp-contract=off", SRC, "-o", tmp])
        os.replace(tmp, LIB)
    return LIB


class _Cfg(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("moe_inter", C.c_int32), ("num_experts", C.c_int32), ("top_k", C.c_int32),
                ("expert_fmt", C.c_int32), ("score", C.c_int32), ("bias_mode", C.c_int32), ("act", C.c_int32),
                ("act_alpha", C.c_double), ("act_limit", C.c_double), ("shared_inter", C.c_int32)]


class _Layer(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("router", "router_xscale", "router_bias", "per_expert_scale", "gate", "up",
                                           "down", "sh_gate", "sh_up", "sh_down")]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.oracle_half_to_double.restype = C.c_double
        _lib.oracle_half_to_double.argtypes = [C.c_uint16]
        _lib.oracle_bf16_to_double.restype = C.c_double
        _lib.oracle_bf16_to_double.argtypes = [C.c_uint16]
        _lib.oracle_e2m1_to_double.restype = C.c_double
        _lib.oracle_e2m1_to_double.argtypes = [C.c_int]
        _lib.oracle_e8m0_to_double.restype = C.c_double
        _lib.oracle_e8m0_to_double.argtypes = [C.c_int]
        _lib.oracle_double_to_bf16.restype = C.c_uint16
        _lib.oracle_double_to_bf16.argtypes = [C.c_double]
        _lib.oracle_act.restype = C.c_double
        _lib.oracle_act.argtypes = [C.c_int, C.c_double, C.c_double, C.c_double, C.c_double]
        _lib.oracle_dequant.argtypes = [C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p]
        _lib.oracle_select.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p,
                                       C.c_void_p, C.c_void_p, C.c_void_p]
        _lib.oracle_router_logits.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p]
        _lib.oracle_forward.restype = C.c_int
        _lib.oracle_forward.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_int,
                                        C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                        C.c_void_p]
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- scalar helpers

def half_to_double(h: int) -> float:
    return lib().oracle_half_to_double(h)


def bf16_to_double(b: int) -> float:
    return lib().oracle_bf16_to_double(b)


def e2m1_to_double(code: int) -> float:
    return lib().oracle_e2m1_to_double(code)


def e8m0_to_double(e: int) -> float:
    return lib().oracle_e8m0_to_double(e)


def double_to_bf16(v: float) -> int:
    return lib().oracle_double_to_bf16(v)


def act(kind: int, alpha: float, limit: float, g: float, u: float) -> float:
    return lib().oracle_act(kind, alpha, limit, g, u)


def dequant(fmt: int, blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    blob = _c(blob, np.uint8)
    out = np.empty((rows, cols), np.float64)
    lib().oracle_dequant(fmt, _p(blob), rows, cols, _p(out))
    return out


# --------------------------------------------------------------------------- layer-level API

@dataclass
class OracleResult:
    logits: np.ndarray   # [M][E] float32
    lsel: np.ndarray     # [M][E] float32 selection logits
    idx: np.ndarray      # [M][K] int32
    w: np.ndarray        # [M][K] float64
    y: np.ndarray        # [M][H] float64
    out: np.ndarray      # [M][H] float64
    out_bf16: np.ndarray  # [M][H] uint16


class Oracle:
    """One layer of the routed half, configured like the library (``shape`` is a synth.MoEShape)."""

    def __init__(self, shape, layer: dict):
        self.shape = shape
        self.cfg = _Cfg(shape.hidden, shape.moe_inter, shape.num_experts, shape.top_k, shape.expert_fmt, shape.score,
                        shape.bias_mode, shape.act, shape.act_alpha, shape.act_limit, shape.shared_inter)
        keep = {}
        for k, dt in (("router", np.uint8), ("xscale", np.uint16), ("bias", np.float32), ("pes", np.float32),
                      ("gate", np.uint8), ("up", np.uint8), ("down", np.uint8), ("sh_gate", np.uint8),
                      ("sh_up", np.uint8), ("sh_down", np.uint8)):
            keep[k] = _c(layer.get(k), dt)
        self._keep = keep
        self.layer = _Layer(_p(keep["router"]), _p(keep["xscale"]), _p(keep["bias"]), _p(keep["pes"]),
                            _p(keep["gate"]), _p(keep["up"]), _p(keep["down"]), _p(keep["sh_gate"]),
                            _p(keep["sh_up"]), _p(keep["sh_down"]))

    def router_logits(self, x_bits: np.ndarray) -> np.ndarray:
        x_bits = _c(x_bits, np.uint16)
        M = x_bits.shape[0]
        out = np.empty((M, self.shape.num_experts), np.float32)
        lib().oracle_router_logits(C.byref(self.cfg), C.byref(self.layer), _p(x_bits), M, _p(out))
        return out

    def select(self, logits: np.ndarray, forced: Optional[np.ndarray] = None):
        logits = _c(logits, np.float32)
        M, K, E = logits.shape[0], self.shape.top_k, self.shape.num_experts
        idx = np.empty((M, K), np.int32)
        w = np.empty((M, K), np.float64)
        lsel = np.empty((M, E), np.float32)
        forced = _c(forced, np.int32)
        lib().oracle_select(C.byref(self.cfg), _p(self._keep["bias"]), _p(self._keep["pes"]), _p(logits), M,
                            _p(forced), _p(idx), _p(w), _p(lsel))
        return idx, w, lsel

    def forward(self, x_bits: np.ndarray, resid_bits: Optional[np.ndarray] = None,
                forced: Optional[np.ndarray] = None, nthreads: int = 1) -> OracleResult:
        x_bits = _c(x_bits, np.uint16)
        resid_bits = _c(resid_bits, np.uint16)
        forced = _c(forced, np.int32)
        M, H, E, K = x_bits.shape[0], self.shape.hidden, self.shape.num_experts, self.shape.top_k
        r = OracleResult(np.empty((M, E), np.float32), np.empty((M, E), np.float32), np.empty((M, K), np.int32),
                         np.empty((M, K), np.float64), np.empty((M, H), np.float64), np.empty((M, H), np.float64),
                         np.empty((M, H), np.uint16))
        rc = lib().oracle_forward(C.byref(self.cfg), C.byref(self.layer), _p(x_bits), M, _p(resid_bits), _p(forced),
                                  nthreads, _p(r.logits), _p(r.lsel), _p(r.idx), _p(r.w), _p(r.y), _p(r.out),
                                  _p(r.out_bf16))
        assert rc == 0
        return r
