"""ctypes binding of ``libts_moe.so`` (C ABI in ``include/ts_moe.h``).

Argument marshalling only: torch tensors are passed as device pointers plus
the current CUDA stream; every step of the routed half runs in the library's
kernels.  If the library is missing this module raises on import -- there is
no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import numpy as np
import torch

from . import synth

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libts_moe.so")

TS_MOE_ABI_VERSION = 1
STATUS = {0: "OK", 1: "EINVAL", 2: "EUNSUPPORTED", 3: "ENOMEM", 4: "ECUDA", 5: "EDEVICE"}


class TsMoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Config(C.Structure):
    _fields_ = [("abi_version", C.c_uint32), ("hidden", C.c_int32), ("moe_inter", C.c_int32),
                ("num_experts", C.c_int32), ("top_k", C.c_int32), ("num_layers", C.c_int32),
                ("max_tokens", C.c_int32), ("expert_fmt", C.c_int32), ("score", C.c_int32),
                ("bias_mode", C.c_int32), ("act", C.c_int32), ("act_alpha", C.c_float), ("act_limit", C.c_float),
                ("shared_inter", C.c_int32), ("device", C.c_int32), ("weights_mem", C.c_int32)]


class LayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("router", "router_xscale", "router_bias", "per_expert_scale", "gate", "up",
                                           "down", "sh_gate", "sh_up", "sh_down")]


class Info(C.Structure):
    _fields_ = [("arena_bytes", C.c_uint64), ("workspace_bytes", C.c_uint64), ("expert_bytes", C.c_uint64),
                ("router_bytes", C.c_uint64), ("shared_bytes", C.c_uint64), ("num_ctas", C.c_int32),
                ("sm_count", C.c_int32), ("launch_tokens", C.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run quantized_moe_routed_router_b200.build.build()")
    lib = C.CDLL(LIB_PATH)
    vp, i32 = C.c_void_p, C.c_int
    lib.ts_moe_open.argtypes = [C.POINTER(Config), C.POINTER(LayerWeights), C.POINTER(vp)]
    lib.ts_moe_route.argtypes = [vp, i32, vp, i32, vp, vp, vp, vp]
    lib.ts_moe_forward.argtypes = [vp, i32, vp, i32, vp, vp, vp]
    lib.ts_moe_device_status.argtypes = [vp, vp]
    lib.ts_moe_get_info.argtypes = [vp, C.POINTER(Info)]
    lib.ts_moe_set_timing_events.argtypes = [vp, vp]
    lib.ts_moe_last_error.argtypes = [vp]
    lib.ts_moe_last_error.restype = C.c_char_p
    lib.ts_moe_close.argtypes = [vp]
    lib.ts_moe_debug_range_start.argtypes = [C.c_uint64, i32, i32]
    lib.ts_moe_debug_range_start.restype = C.c_uint64
    lib.ts_moe_debug_owner_of.argtypes = [C.c_uint64, i32, C.c_uint64]
    lib.ts_moe_debug_partial_slot.argtypes = [C.c_uint64, i32, i32, C.c_uint64]
    lib.ts_moe_debug_group_size.argtypes = [i32]
    lib.ts_moe_debug_aligned_start.argtypes = [i32, i32, i32, i32]
    lib.ts_moe_debug_aligned_start.restype = C.c_uint64
    lib.ts_moe_debug_use_aligned.argtypes = [i32, i32]
    lib.ts_moe_debug_coresident.argtypes = [i32, i32, i32]
    lib.ts_moe_debug_layer_ctas.argtypes = [i32]
    lib.ts_moe_debug_validate.argtypes = [C.POINTER(Config), C.POINTER(LayerWeights)]
    lib.ts_moe_route_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, i32, vp, vp, vp, vp]
    lib.ts_moe_debug_skew_barrier.argtypes = [vp, vp]
    for f in ("ts_moe_open", "ts_moe_route", "ts_moe_forward", "ts_moe_device_status", "ts_moe_get_info",
              "ts_moe_set_timing_events", "ts_moe_close", "ts_moe_debug_validate", "ts_moe_route_noalloc",
              "ts_moe_debug_skew_barrier"):
        getattr(lib, f).restype = C.c_int
    return lib


lib = _load()


def make_config(shape: "synth.MoEShape", device: int = 0, weights_mem: int = 0) -> Config:
    return Config(TS_MOE_ABI_VERSION, shape.hidden, shape.moe_inter, shape.num_experts, shape.top_k, shape.num_layers,
                  shape.max_tokens, shape.expert_fmt, shape.score, shape.bias_mode, shape.act, shape.act_alpha,
                  shape.act_limit, shape.shared_inter, device, weights_mem)


def _ptr(a) -> Optional[int]:
    if a is None:
        return None
    if isinstance(a, torch.Tensor):
        return a.data_ptr()
    return a.ctypes.data


def layer_struct(L: "synth.LayerBlobs", keep: list) -> LayerWeights:
    """LayerWeights for one layer; host vectors are made contiguous and kept alive in `keep`."""
    def host(a, dt):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=dt)
        keep.append(a)
        return a.ctypes.data

    def blob(t):
        if t is None:
            return None
        t = t.contiguous()
        keep.append(t)
        return t.data_ptr()

    return LayerWeights(blob(L.router), host(L.xscale, np.uint16), host(L.bias, np.float32), host(L.pes, np.float32),
                        blob(L.gate), blob(L.up), blob(L.down), blob(L.sh_gate), blob(L.sh_up), blob(L.sh_down))


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


class MoE:
    """One ts_moe handle: all layers of `shape`, repacked on `device` at construction."""

    def __init__(self, shape: "synth.MoEShape", layers: Sequence["synth.LayerBlobs"], device: int = 0):
        assert len(layers) == shape.num_layers
        on_dev = layers[0].gate.is_cuda
        self.shape = shape
        self.cfg = make_config(shape, device, 1 if on_dev else 0)
        keep: list = []
        arr = (LayerWeights * shape.num_layers)(*[layer_struct(L, keep) for L in layers])
        h = C.c_void_p()
        st = lib.ts_moe_open(C.byref(self.cfg), arr, C.byref(h))
        if st != 0:
            raise TsMoeError(st, lib.ts_moe_last_error(None).decode())
        self.h = h

    def _check(self, st: int):
        if st != 0:
            raise TsMoeError(st, lib.ts_moe_last_error(self.h).decode())

    def route(self, layer: int, x: torch.Tensor, idx: torch.Tensor, w: torch.Tensor,
              logits: Optional[torch.Tensor] = None, stream=None):
        M = x.shape[0] if x is not None else 0
        self._check(lib.ts_moe_route(self.h, layer, _ptr(x), M, _ptr(idx), _ptr(w), _ptr(logits), _stream(stream)))

    def forward(self, layer: int, x: torch.Tensor, resid: Optional[torch.Tensor] = None,
                y: Optional[torch.Tensor] = None, stream=None, M: Optional[int] = None):
        if M is None:
            M = x.shape[0]
        self._check(lib.ts_moe_forward(self.h, layer, _ptr(x), M, _ptr(resid), _ptr(y), _stream(stream)))

    def forward_ptr(self, layer: int, x_ptr: int, M: int, resid_ptr: Optional[int], y_ptr: Optional[int],
                    stream: int):
        self._check(lib.ts_moe_forward(self.h, layer, x_ptr, M, resid_ptr, y_ptr, stream))

    def device_status(self, stream=None):
        self._check(lib.ts_moe_device_status(self.h, _stream(stream)))

    def info(self) -> Info:
        i = Info()
        self._check(lib.ts_moe_get_info(self.h, C.byref(i)))
        return i

    def set_timing_events(self, events: Optional[Sequence[torch.cuda.Event]]):
        if events is None:
            self._check(lib.ts_moe_set_timing_events(self.h, None))
            return
        self._evs = list(events)
        for e in self._evs:
            if not e.cuda_event:          # torch creates the CUDA event on first record
                e.record()
        arr = (C.c_void_p * 4)(*[e.cuda_event for e in self._evs])
        self._check(lib.ts_moe_set_timing_events(self.h, arr))

    def close(self):
        if getattr(self, "h", None):
            lib.ts_moe_close(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def route_noalloc(router: torch.Tensor, bias: Optional[torch.Tensor], pes: Optional[torch.Tensor], num_experts: int,
                  hidden: int, top_k: int, score: int, bias_mode: int, x: torch.Tensor, idx: torch.Tensor,
                  w: torch.Tensor, logits: Optional[torch.Tensor] = None, stream=None):
    """Router GEMV + top-k without a handle and without any device allocation
    (scratch lives in the library's static device array).  router: device Q8_0
    blob [E][H]; bias / pes: device float32 [E] or None; x: device bf16 [M][H]."""
    M = x.shape[0]
    st = lib.ts_moe_route_noalloc(_ptr(router), _ptr(bias), _ptr(pes), num_experts, hidden, top_k, score, bias_mode,
                                  _ptr(x), M, _ptr(idx), _ptr(w), _ptr(logits), _stream(stream))
    if st != 0:
        raise TsMoeError(st, lib.ts_moe_last_error(None).decode())


def validate(shape: "synth.MoEShape", layers: Sequence["synth.LayerBlobs"], **cfg_over) -> tuple:
    """Runs the library's host-side open-time validation only (no CUDA); returns (status, message)."""
    cfg = make_config(shape)
    for k, v in cfg_over.items():
        setattr(cfg, k, v)
    keep: list = []
    arr = (LayerWeights * max(1, len(layers)))(*[layer_struct(L, keep) for L in layers])
    st = lib.ts_moe_debug_validate(C.byref(cfg), arr)
    return st, lib.ts_moe_last_error(None).decode()
