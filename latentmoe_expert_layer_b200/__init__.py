"""Python binding of the sm_100a LatentMoE layer library (liblmoe.so).

Argument marshalling only: tensors are passed to the C ABI as raw device pointers plus the current
CUDA stream.  Every step of the layer runs in the library's CUDA kernels; there is no Python or CPU
fallback, and importing this package raises if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["LatentMoE", "LmoeError", "route_noalloc", "lib", "STATUS", "BUF", "SYMBOLS", "STAGES", "library_path"]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "liblmoe.so")

if not os.path.exists(library_path):
    raise ImportError(f"{library_path} is missing: build it with `python latentmoe_expert_layer_b200/build.py`"
                      " or __graft_entry__.build()")

lib = ctypes.CDLL(library_path)

STATUS = {0: "ok", 1: "invalid argument", 2: "shape out of range", 3: "unsupported configuration",
          4: "device out of memory", 5: "CUDA error", 6: "weights not loaded",
          7: "device-side wait timed out", 8: "device-side index out of range", 9: "no suitable CUDA device"}
BUF = {"logits": 0, "counts": 1, "offsets": 2, "row_of": 3, "tok_of_row": 4, "h": 5, "z": 6, "u": 7,
       "xq": 8, "x_sf": 9, "hq": 10, "h_sf": 11, "uq": 12, "u_sf": 13, "usq": 14, "us_sf": 15, "y_s": 16,
       "act_scale": 17}
PREC = {"bf16": 0, "nvfp4": 1}
WSCALE = {"amax": 0, "mse": 1}
DTYPE = {torch.bfloat16: 0, torch.float32: 1}

# every extern "C" symbol declared in include/lmoe.h
SYMBOLS = ("lmoe_create", "lmoe_load_weights", "lmoe_forward", "lmoe_forward_host", "lmoe_get_device_status",
           "lmoe_inspect", "lmoe_profile", "lmoe_profile_read", "lmoe_route_noalloc", "lmoe_export_nvfp4",
           "lmoe_selftest_wait_timeout", "lmoe_status_string", "lmoe_destroy", "lmoe_ep_dispatch", "lmoe_ep_experts",
           "lmoe_ep_combine")
STAGES = ("router", "shared_up", "topk", "grouping", "scatter", "expert_up", "expert_down", "combine", "output")


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("d", "latent", "n_experts", "top_k", "expert_ffn", "shared_ffn",
                                             "max_tokens", "precision", "has_router_bias", "weight_scale",
                                             "ep_world", "ep_rank")]


class _Weights(ctypes.Structure):
    _fields_ = [("w_router", ctypes.c_void_p), ("b_router", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("w_up", ctypes.c_void_p), ("w1", ctypes.c_void_p), ("w2", ctypes.c_void_p),
                ("ws1", ctypes.c_void_p), ("ws2", ctypes.c_void_p), ("dtype", ctypes.c_int32)]


_vp, _i32, _i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
lib.lmoe_create.argtypes = [ctypes.POINTER(_Config), ctypes.c_int, ctypes.POINTER(_vp)]
lib.lmoe_load_weights.argtypes = [_vp, ctypes.POINTER(_Weights), _vp]
lib.lmoe_forward.argtypes = [_vp, _vp, _i32, _vp, _vp, _vp, _vp]
lib.lmoe_forward_host.argtypes = [_vp, _vp, _i32, _vp, _vp, _vp, _vp]
lib.lmoe_get_device_status.argtypes = [_vp]
lib.lmoe_inspect.argtypes = [_vp, _i32, ctypes.POINTER(_vp), ctypes.POINTER(_i64)]
lib.lmoe_profile.argtypes = [_vp, _i32]
lib.lmoe_profile_read.argtypes = [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i32), ctypes.POINTER(_i32)]
lib.lmoe_route_noalloc.argtypes = [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.lmoe_export_nvfp4.argtypes = [_vp, _i32, _i32, _vp, _vp, _vp]
lib.lmoe_selftest_wait_timeout.argtypes = [_vp, ctypes.c_uint64, _vp]
lib.lmoe_ep_dispatch.argtypes = [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.lmoe_ep_experts.argtypes = [_vp, _vp, _i32, _vp, _vp, _i32, _vp, _vp]
lib.lmoe_ep_combine.argtypes = [_vp, _vp, _i32, _vp, _vp, _vp, _vp]
lib.lmoe_status_string.argtypes = [ctypes.c_int]
lib.lmoe_status_string.restype = ctypes.c_char_p
lib.lmoe_destroy.argtypes = [_vp]
lib.lmoe_destroy.restype = None
for _f in ("lmoe_create", "lmoe_load_weights", "lmoe_forward", "lmoe_forward_host", "lmoe_get_device_status",
           "lmoe_inspect", "lmoe_profile", "lmoe_profile_read", "lmoe_route_noalloc", "lmoe_export_nvfp4",
           "lmoe_selftest_wait_timeout", "lmoe_ep_dispatch", "lmoe_ep_experts", "lmoe_ep_combine"):
    getattr(lib, _f).restype = ctypes.c_int


class LmoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)} ({code})")
        self.code = code


def _check(code: int, what: str) -> None:
    if code != 0:
        raise LmoeError(code, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


class _DevArray:
    """__cuda_array_interface__ view of a library-owned device buffer (for lmoe_inspect)."""

    def __init__(self, ptr: int, count: int, typestr: str):
        self.__cuda_array_interface__ = {"shape": (count,), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None}


_BUF_TYPES = {"logits": "<f4", "counts": "<i4", "offsets": "<i4", "row_of": "<i4", "tok_of_row": "<i4",
              "h": "<u2", "z": "<u2", "u": "<u2", "xq": "|u1", "x_sf": "|u1", "hq": "|u1", "h_sf": "|u1",
              "uq": "|u1", "u_sf": "|u1", "usq": "|u1", "us_sf": "|u1", "y_s": "<f4", "act_scale": "<f4"}


def route_noalloc(logits: torch.Tensor, top_k: int, bias: Optional[torch.Tensor] = None, stream=None):
    """Routing from precomputed logits [T, N] through lmoe_route_noalloc, which allocates no device
    memory (for callers that cannot allocate on their call path).  The outputs are allocated here by
    torch, before the call.  Returns (topk_idx, topk_gate, counts, offsets, row_of, status), where
    status is a one-element int32 device tensor holding the call's device status bits (read it after
    synchronising the stream)."""
    if not isinstance(logits, torch.Tensor) or logits.dim() != 2:
        raise ValueError("logits must be a 2-D [T, N] tensor")
    if logits.dtype != torch.float32 or not logits.is_cuda:
        raise ValueError("logits must be a float32 CUDA tensor")
    t, n = logits.shape
    dev = logits.device
    if bias is not None:
        if bias.dtype != torch.float32 or bias.device != dev or bias.numel() != n:
            raise ValueError(f"bias must be a float32 tensor of {n} elements on {dev}")
    idx = torch.empty((t, top_k), dtype=torch.int32, device=dev)
    gate = torch.empty((t, top_k), dtype=torch.float32, device=dev)
    counts = torch.empty((n,), dtype=torch.int32, device=dev)
    offsets = torch.empty((n + 1,), dtype=torch.int32, device=dev)
    row_of = torch.empty((t * top_k,), dtype=torch.int32, device=dev)
    status = torch.empty((1,), dtype=torch.int32, device=dev)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):
        _check(lib.lmoe_route_noalloc(_ptr(logits), _ptr(bias), t, n, top_k, _ptr(idx), _ptr(gate), _ptr(counts),
                                      _ptr(offsets), _ptr(row_of), _ptr(status), s.cuda_stream),
               "lmoe_route_noalloc")
    return idx, gate, counts, offsets, row_of, status


class LatentMoE:
    """One LatentMoE layer on one GPU (lmoe_create / lmoe_load_weights / lmoe_forward).

    shape: object with d, latent, n_experts, top_k, expert_ffn, shared_ffn attributes; latent = 0
        builds the standard MoE without W_down / W_up (experts work in d; bf16 only).
    max_tokens: the largest T a forward may pass (sizes the workspace).
    precision: "bf16", or "nvfp4" for block-scaled FP4 routed and shared experts.
    router_bias: a per-expert fp32 bias is added to the router logits (load_weights' b_router).
    weight_scale: NVFP4 weight block scales, "amax" or "mse" (lmoe_weight_scale).
    ep_world, ep_rank: expert parallelism; with ep_world = G >= 2 this layer is rank ep_rank of G and
        holds only experts [ep_rank * N / G, (ep_rank + 1) * N / G) (load_weights' w1 / w2 hold those);
        it runs through ep_dispatch / ep_experts / ep_combine instead of forward.
    """

    def __init__(self, shape, max_tokens: int, precision: str = "bf16", router_bias: bool = False,
                 device: int = 0, weight_scale: str = "amax", ep_world: int = 0, ep_rank: int = 0):
        cfg = _Config(shape.d, shape.latent, shape.n_experts, shape.top_k, shape.expert_ffn, shape.shared_ffn,
                      max_tokens, PREC[precision], int(router_bias), WSCALE[weight_scale], ep_world, ep_rank)
        h = _vp()
        _check(lib.lmoe_create(ctypes.byref(cfg), device, ctypes.byref(h)), "lmoe_create")
        self._h = h
        self.shape = shape
        self.max_tokens = max_tokens
        self.device = torch.device("cuda", device)
        self.ep_world = ep_world if ep_world > 1 else 0
        self.ep_rank = ep_rank if ep_world > 1 else 0

    def load_weights(self, w_router, w_down, w_up, w1, w2, ws1, ws2, b_router=None, stream=None) -> None:
        # a standard MoE (latent == 0) passes w_down = w_up = None
        ts = (w_router, w_down, w_up, w1, w2, ws1, ws2)
        dt = {t.dtype for t in ts if t is not None}
        if len(dt) != 1 or next(iter(dt)) not in DTYPE:
            raise ValueError("all weight matrices must share one dtype, bf16 or fp32")
        w = _Weights(_ptr(w_router), _ptr(b_router), _ptr(w_down), _ptr(w_up), _ptr(w1), _ptr(w2), _ptr(ws1),
                     _ptr(ws2), DTYPE[next(iter(dt))])
        _check(lib.lmoe_load_weights(self._h, ctypes.byref(w), self._stream(stream)), "lmoe_load_weights")

    def _stream(self, stream) -> int:
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return s.cuda_stream

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                gate: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
        t = x.shape[0]
        k = self.shape.top_k
        if y is None:
            y = torch.empty((t, self.shape.d), dtype=torch.bfloat16, device=self.device)
        if idx is None:
            idx = torch.empty((t, k), dtype=torch.int32, device=self.device)
        if gate is None:
            gate = torch.empty((t, k), dtype=torch.float32, device=self.device)
        _check(lib.lmoe_forward(self._h, _ptr(x), t, _ptr(y), _ptr(idx), _ptr(gate), self._stream(stream)),
               "lmoe_forward")
        return y, idx, gate

    def forward_host(self, x: torch.Tensor, y: torch.Tensor, idx: Optional[torch.Tensor] = None,
                     gate: Optional[torch.Tensor] = None, stream=None) -> None:
        """x, y, idx, gate are CPU tensors (pinned for asynchronous copies)."""
        _check(lib.lmoe_forward_host(self._h, _ptr(x), x.shape[0], _ptr(y), _ptr(idx), _ptr(gate),
                                     self._stream(stream)), "lmoe_forward_host")

    # ------------------------------------------------------------------ expert parallelism
    def ep_dispatch(self, x: torch.Tensor, stream=None) -> dict:
        """Step 1 (lmoe_ep_dispatch): routing and the send plan of this rank's tokens x [T, d].
        Returns device tensors idx, gate, send_rows (first P rows valid), send_meta, send_gate (first
        A entries valid), counts [G, 2] (pairs, assignments per destination) and tok_pairs."""
        t, s, g = x.shape[0], self.shape, self.ep_world
        gp = min(s.top_k, g)
        dev = self.device
        out = {"idx": torch.empty((t, s.top_k), dtype=torch.int32, device=dev),
               "gate": torch.empty((t, s.top_k), dtype=torch.float32, device=dev),
               "send_rows": torch.empty((t * gp, s.latent), dtype=torch.bfloat16, device=dev),
               "send_meta": torch.empty((t * s.top_k, 2), dtype=torch.int32, device=dev),
               "send_gate": torch.empty((t * s.top_k,), dtype=torch.float32, device=dev),
               "counts": torch.empty((g, 2), dtype=torch.int32, device=dev),
               "tok_pairs": torch.empty((t, gp), dtype=torch.int32, device=dev)}
        _check(lib.lmoe_ep_dispatch(self._h, _ptr(x), t, _ptr(out["idx"]), _ptr(out["gate"]), _ptr(out["send_rows"]),
                                    _ptr(out["send_meta"]), _ptr(out["send_gate"]), _ptr(out["counts"]),
                                    _ptr(out["tok_pairs"]), self._stream(stream)), "lmoe_ep_dispatch")
        return out

    def ep_experts(self, recv_rows: torch.Tensor, recv_meta: torch.Tensor, recv_gate: torch.Tensor,
                   stream=None) -> torch.Tensor:
        """Step 2 (lmoe_ep_experts): this rank's experts on the received latent rows [R, l]; recv_meta
        [A, 2] (row of recv_rows, local expert id), rows nondecreasing; recv_gate [A].  Returns the fp32
        partial sums [R, l]."""
        r, a = recv_rows.shape[0], recv_meta.shape[0]
        partial = torch.empty((r, self.shape.latent), dtype=torch.float32, device=self.device)
        _check(lib.lmoe_ep_experts(self._h, _ptr(recv_rows), r, _ptr(recv_meta) if a else None,
                                   _ptr(recv_gate) if a else None, a, _ptr(partial), self._stream(stream)),
               "lmoe_ep_experts")
        return partial

    def ep_combine(self, x: torch.Tensor, back: torch.Tensor, tok_pairs: torch.Tensor, stream=None) -> torch.Tensor:
        """Step 3 (lmoe_ep_combine): y [T, d] from this rank's tokens x, the fp32 partial sums returned
        for its pairs (send order) and tok_pairs from ep_dispatch."""
        y = torch.empty((x.shape[0], self.shape.d), dtype=torch.bfloat16, device=self.device)
        _check(lib.lmoe_ep_combine(self._h, _ptr(x), x.shape[0], _ptr(back), _ptr(tok_pairs), _ptr(y),
                                   self._stream(stream)), "lmoe_ep_combine")
        return y

    def device_status(self) -> int:
        return lib.lmoe_get_device_status(self._h)

    def selftest_wait_timeout(self, limit_ns: int, stream=None) -> None:
        """Enqueue a kernel whose bounded wait never completes (see lmoe_selftest_wait_timeout)."""
        _check(lib.lmoe_selftest_wait_timeout(self._h, int(limit_ns), self._stream(stream)),
               "lmoe_selftest_wait_timeout")

    def inspect(self, name: str) -> torch.Tensor:
        p, n = _vp(), _i64()
        _check(lib.lmoe_inspect(self._h, BUF[name], ctypes.byref(p), ctypes.byref(n)), "lmoe_inspect")
        if n.value == 0:
            return torch.empty(0)
        t = torch.as_tensor(_DevArray(p.value, n.value, _BUF_TYPES[name]), device=self.device)
        return t.clone()

    def export_nvfp4(self, which: int, index: int = 0):
        """(codes uint8 [rows, K/2], scales uint8 [rows, K/16], tensor scale float) of one quantised
        weight matrix: which 0 = W1[index], 1 = W2[index], 2 = W_s1, 3 = W_s2."""
        import numpy as np
        s = self.shape
        rows, k = {0: (s.expert_ffn, s.latent), 1: (s.latent, s.expert_ffn), 2: (s.shared_ffn, s.d),
                   3: (s.d, s.shared_ffn)}[which]
        codes = np.empty((rows, k // 2), np.uint8)
        scales = np.empty((rows, k // 16), np.uint8)
        g = np.empty(1, np.float32)
        _check(lib.lmoe_export_nvfp4(self._h, which, index, codes.ctypes.data, scales.ctypes.data, g.ctypes.data),
               "lmoe_export_nvfp4")
        return codes, scales, np.float32(g[0])

    def profile(self, enable: bool) -> None:
        """Start (clearing the record) or stop per-stage CUDA-event timing of forward calls."""
        _check(lib.lmoe_profile(self._h, int(enable)), "lmoe_profile")

    def profile_read(self):
        """(dict stage -> summed ms over the recorded calls, recorded calls, kernel launches per call)."""
        ms = (ctypes.c_double * len(STAGES))()
        n, launches = _i32(), _i32()
        _check(lib.lmoe_profile_read(self._h, ms, ctypes.byref(n), ctypes.byref(launches)), "lmoe_profile_read")
        return dict(zip(STAGES, list(ms))), n.value, launches.value

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib.lmoe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
