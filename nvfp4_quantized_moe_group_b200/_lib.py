"""ctypes binding of libnvfp4moe.so: argument marshalling only.

Every call forwards torch tensors' device pointers and the current CUDA stream to the
C ABI declared in include/nvfp4moe.h; all arithmetic runs in the library's sm_100a
kernels.  torch is used for device memory (outputs and workspaces) and streams.
Loading fails loudly when the library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libnvfp4moe.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "nvfp4moe.h")

OK, ERR_ARG, ERR_SHAPE, ERR_CUDA, ERR_WORKSPACE, ERR_NONFINITE, ERR_TIMEOUT, ERR_DEVICE = 0, -1, -2, -3, -4, -5, -6, -7
SCALES_LINEAR, SCALES_SWIZZLED = 0, 1


class NvFp4MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class Cfg(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int32), ("n_groups", ctypes.c_int32), ("topk_groups", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("routed_scale", ctypes.c_float)]

    def __repr__(self):
        return (f"Cfg(E={self.E}, n_groups={self.n_groups}, topk_groups={self.topk_groups}, "
                f"topk={self.topk}, H={self.H}, I={self.I}, routed_scale={self.routed_scale})")


class ExpertTensors(ctypes.Structure):
    _fields_ = [("gate_codes", ctypes.c_void_p), ("gate_scales", ctypes.c_void_p),
                ("up_codes", ctypes.c_void_p), ("up_scales", ctypes.c_void_p),
                ("down_codes", ctypes.c_void_p), ("down_scales", ctypes.c_void_p),
                ("g_gate", ctypes.c_float), ("g_up", ctypes.c_float), ("g_down", ctypes.c_float),
                ("g_h", ctypes.c_float)]


DEBUG_FIELDS = ("idx", "w", "g_x", "xq_codes", "xq_scales", "counts", "offsets", "perm", "hq_codes",
                "hq_scales")
STAGES = ("amax", "route", "quantize", "permute", "gather", "gateup", "down", "finalize")


class Debug(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_void_p) for n in DEBUG_FIELDS] + [("events", ctypes.POINTER(ctypes.c_void_p))]
                + [("logits", ctypes.c_void_p), ("x_norm", ctypes.c_void_p), ("xq8_codes", ctypes.c_void_p),
                   ("xq8_scales", ctypes.c_void_p), ("acc", ctypes.c_void_p), ("h_f32", ctypes.c_void_p),
                   ("wait_limit_us", ctypes.c_uint32),
                   ("inject_skip_arrive", ctypes.c_int32),
                   ("separate_gemms", ctypes.c_int32)])


class Fp8ExpertTensors(ctypes.Structure):
    _fields_ = [("gate_codes", ctypes.c_void_p), ("gate_scales", ctypes.c_void_p),
                ("up_codes", ctypes.c_void_p), ("up_scales", ctypes.c_void_p),
                ("down_codes", ctypes.c_void_p), ("down_scales", ctypes.c_void_p)]


class StageTimer:
    """CUDA events recorded around stages of a forward call (nvfp4moe_debug.events).
    ``stages``: the stage names to time (default all)."""

    def __init__(self, stages=STAGES):
        self.stages = [s for s in STAGES if s in stages]
        self.events = {}
        for name in self.stages:
            pair = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for e in pair:          # materialise the underlying cudaEvent_t
                e.record()
            self.events[name] = pair
        torch.cuda.synchronize()
        handles = []
        for name in STAGES:
            pair = self.events.get(name)
            handles += [pair[0].cuda_event, pair[1].cuda_event] if pair else [None, None]
        self.array = (ctypes.c_void_p * len(handles))(*handles)

    def stage_ms(self) -> dict:
        """Elapsed milliseconds of each timed stage of the last recorded forward (synchronises)."""
        out = {}
        for name in self.stages:
            a, b = self.events[name]
            b.synchronize()
            out[name] = a.elapsed_time(b)
        return out


_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_SIGS = {
    "nvfp4moe_cfg_default": (ctypes.c_int, [ctypes.POINTER(Cfg)]),
    "nvfp4moe_cfg_check": (ctypes.c_int, [ctypes.POINTER(Cfg)]),
    "nvfp4moe_quantize_workspace_bytes": (_SZ, [_I64, _I64]),
    "nvfp4moe_swizzled_scale_bytes": (_SZ, [_I64, _I64]),
    "nvfp4moe_quantize": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, ctypes.c_int32, _P, _P, _SZ, _P]),
    "nvfp4moe_quantize_weights_lh": (ctypes.c_int, [_P, _I64, _I64, _P, ctypes.c_int32, _P, _P, _P, _P, _SZ, _P]),
    "nvfp4moe_route_workspace_bytes": (_SZ, [ctypes.POINTER(Cfg), _I64]),
    "nvfp4moe_route": (ctypes.c_int, [ctypes.POINTER(Cfg), _P, _I64, _P, _P, _P, _P, _P, _SZ, _P]),
    "nvfp4moe_route_noalloc": (ctypes.c_int, [ctypes.POINTER(Cfg), _P, _I64, _P, _P, _P, _P, _P]),
    "nvfp4moe_experts_create": (ctypes.c_int, [ctypes.POINTER(Cfg), ctypes.POINTER(_P)]),
    "nvfp4moe_experts_set": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.POINTER(ExpertTensors), _P]),
    "nvfp4moe_experts_destroy": (None, [_P]),
    "nvfp4moe_experts_cfg": (ctypes.c_int, [_P, ctypes.POINTER(Cfg)]),
    "nvfp4moe_experts_create_local": (ctypes.c_int, [ctypes.POINTER(Cfg), ctypes.c_int32, ctypes.c_int32,
                                                     ctypes.POINTER(_P)]),
    "nvfp4moe_experts_range": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]),
    "nvfp4moe_forward_partial": (ctypes.c_int, [_P, _P, _I64, _P, _P, _P, ctypes.POINTER(Debug), _P, _SZ, _P]),
    "nvfp4moe_finalize": (ctypes.c_int, [_P, _I64, _P, _P]),
    "nvfp4moe_forward_partial_peer": (ctypes.c_int, [_P, _P, _I64, _P, _P, _P, ctypes.c_int32, _I64,
                                                     ctypes.POINTER(Debug), _P, _SZ, _P]),
    "nvfp4moe_ipc_get_handle": (ctypes.c_int, [_P, _P, ctypes.POINTER(_I64)]),
    "nvfp4moe_ipc_open": (ctypes.c_int, [_P, ctypes.POINTER(_P)]),
    "nvfp4moe_ipc_close": (ctypes.c_int, [_P]),
    "nvfp4moe_forward_workspace_bytes": (_SZ, [ctypes.POINTER(Cfg), _I64]),
    "nvfp4moe_forward": (ctypes.c_int, [_P, _P, _I64, _P, _P, _P, ctypes.POINTER(Debug), _P, _SZ, _P]),
    "nvfp4moe_forward_residual": (ctypes.c_int, [_P, _P, _I64, _P, ctypes.c_float, ctypes.c_int32, _P, _P, _P,
                                                 ctypes.POINTER(Debug), _P, _SZ, _P]),
    "nvfp4moe_quantize_fp8": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "nvfp4moe_fp8_experts_create": (ctypes.c_int, [ctypes.POINTER(Cfg), ctypes.POINTER(_P)]),
    "nvfp4moe_fp8_experts_set": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.POINTER(Fp8ExpertTensors), _P]),
    "nvfp4moe_fp8_experts_destroy": (None, [_P]),
    "nvfp4moe_forward_fp8_workspace_bytes": (_SZ, [ctypes.POINTER(Cfg), _I64]),
    "nvfp4moe_forward_fp8": (ctypes.c_int, [_P, _P, _I64, _P, _P, _P, ctypes.POINTER(Debug), _P, _SZ, _P]),
    "nvfp4moe_amax": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _SZ, _P]),
    "nvfp4moe_ep_dispatch_workspace_bytes": (_SZ, [ctypes.POINTER(Cfg), _I64]),
    "nvfp4moe_ep_dispatch": (ctypes.c_int, [ctypes.POINTER(Cfg), ctypes.c_int32, _P, _I64, _P, _P, _P, _P, _P, _P, _P,
                                            _P, _P, _P, _SZ, _P]),
    "nvfp4moe_ep_experts_workspace_bytes": (_SZ, [ctypes.POINTER(Cfg), ctypes.c_int32, _I64]),
    "nvfp4moe_ep_experts": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _P, _P, _P, _SZ, _P]),
    "nvfp4moe_ep_combine": (ctypes.c_int, [_P, _P, _I64, ctypes.c_int32, ctypes.c_int32, _P, _P]),
    "nvfp4moe_status_read": (ctypes.c_int, [_P, _P]),
    "nvfp4moe_last_device_status": (ctypes.c_int, [_P]),
    "nvfp4moe_workspace_bytes": (_SZ, [ctypes.POINTER(Cfg), _I64]),
    "nvfp4moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "nvfp4moe_last_launch_count": (ctypes.c_int32, []),
}


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m nvfp4_quantized_moe_group_b200.build` (needs nvcc 12.9)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = args
        _lib = handle
    return _lib


def declared_symbols() -> list[str]:
    """Names of the entry points include/nvfp4moe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"NVFP4MOE_API\s+[\w\s\*]+?\b(nvfp4moe_\w+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().nvfp4moe_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise NvFp4MoeError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require(*specs):
    """Raise TypeError unless every (tensor, name, dtype, shape) of ``specs`` whose tensor is
    not None is a contiguous tensor of that dtype and shape (shape None: any), and all of them
    are CUDA tensors on the first one's device, the current device.  Types and shapes are
    checked before devices.
    The library receives raw pointers, so a tensor of the wrong type or size would be read out
    of bounds rather than rejected."""
    present = [s for s in specs if s[0] is not None]
    for t, name, dtype, shape in present:
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if shape is not None and tuple(t.shape) != tuple(int(s) for s in shape):
            raise TypeError(f"{name} must have shape {tuple(int(s) for s in shape)}, got {tuple(t.shape)}")
        if not t.is_contiguous():
            raise TypeError(f"{name} must be contiguous")
    for t, name, _, _ in present:
        if not t.is_cuda or t.device != present[0][0].device:
            raise TypeError(f"{name} must be a CUDA tensor on {present[0][0].device}, got {t.device}")
    # the library launches on the current device: tensors of another one would be read
    # through addresses that device does not map
    if present and present[0][0].device.index != torch.cuda.current_device():
        raise TypeError(f"the tensors are on {present[0][0].device} but the current device is "
                        f"cuda:{torch.cuda.current_device()}: call under torch.cuda.device({present[0][0].device})")


def _rows(x, name: str, min_rows: int = 1) -> int:
    """Rows of a 2-D tensor, at least min_rows."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2 or x.shape[0] < min_rows:
        raise TypeError(f"{name} must be a 2-D tensor with at least {min_rows} rows")
    return int(x.shape[0])


def _layer_specs(cfg, x, w_router, bias, name="x") -> list:
    """x [T, H] bf16 (T >= 1), w_router [E, H] float32, bias [E] float32 or None."""
    T = _rows(x, name)
    return [(x, name, torch.bfloat16, (T, cfg.H)), (w_router, "w_router", torch.float32, (cfg.E, cfg.H)),
            (bias, "bias", torch.float32, (cfg.E,))]


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's allocator returns blocks aligned to at least 512 bytes
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def cfg_default() -> Cfg:
    c = Cfg()
    _check(lib().nvfp4moe_cfg_default(ctypes.byref(c)), "nvfp4moe_cfg_default")
    return c


def make_cfg(E, n_groups, topk_groups, topk, H, I, routed_scale=2.5) -> Cfg:
    c = Cfg(E, n_groups, topk_groups, topk, H, I, routed_scale)
    _check(lib().nvfp4moe_cfg_check(ctypes.byref(c)), "nvfp4moe_cfg_check")
    return c


def last_launch_count() -> int:
    return int(lib().nvfp4moe_last_launch_count())


def status_read(ws: torch.Tensor, stream=None) -> int:
    return int(lib().nvfp4moe_status_read(_ptr(ws), _stream(stream)))


def last_device_status(stream=None) -> int:
    """Device-side status of this thread's latest call that had a status word (waits for the
    stream); the only way to read nvfp4moe_route_noalloc's."""
    return int(lib().nvfp4moe_last_device_status(_stream(stream)))


def workspace_bytes(cfg: Cfg, T_max: int) -> int:
    """Workspace bytes of forward() for up to T_max tokens (= forward_workspace_bytes)."""
    return int(lib().nvfp4moe_workspace_bytes(ctypes.byref(cfg), T_max))


def swizzled_scale_bytes(rows: int, cols16: int) -> int:
    return int(lib().nvfp4moe_swizzled_scale_bytes(rows, cols16))


def quantize_workspace_bytes(rows: int, cols: int) -> int:
    return int(lib().nvfp4moe_quantize_workspace_bytes(rows, cols))


def quantize(x: torch.Tensor, g: torch.Tensor | None = None, swizzled: bool = False, ws=None, out=None,
             stream=None):
    """quantize_nvfp4(x) -> (codes [rows, cols/2] u8, scales u8, g [1] f32).

    ``g``: None for a dynamic global scale, else a 1-element CUDA float32 tensor.
    Scales are [rows, cols/16] (linear) or the flat swizzled array.
    """
    rows = _rows(x, "x", min_rows=0)
    cols = int(x.shape[1])
    dev = x.device
    specs = [(x, "x", torch.bfloat16, None), (g, "g", torch.float32, (1,)), (ws, "ws", torch.uint8, None)]
    if out is not None:
        specs += [(out[0], "codes", torch.uint8, (rows, cols // 2)),
                  (out[1], "scales", torch.uint8,
                   (swizzled_scale_bytes(rows, cols // 16),) if swizzled else (rows, cols // 16)),
                  (out[2], "g_out", torch.float32, (1,))]
    _require(*specs)
    if out is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
        if swizzled:
            scales = torch.empty(swizzled_scale_bytes(rows, cols // 16), dtype=torch.uint8, device=dev)
        else:
            scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
        g_out = torch.empty(1, dtype=torch.float32, device=dev)
    else:
        codes, scales, g_out = out
    if ws is None:
        ws = _workspace(quantize_workspace_bytes(rows, cols), dev)
    st = lib().nvfp4moe_quantize(_ptr(x), rows, cols, _ptr(g), _ptr(codes), _ptr(scales),
                                 SCALES_SWIZZLED if swizzled else SCALES_LINEAR, _ptr(g_out), _ptr(ws),
                                 ws.numel(), _stream(stream))
    _check(st, "nvfp4moe_quantize")
    return codes, scales, g_out


def quantize_weights_lh(w: torch.Tensor, hess_blocks: torch.Tensor, m: int = 4, ws=None, stream=None):
    """Weight quantisation with the local-Hessian block-scale search
    (nvfp4moe_quantize_weights_lh): w [rows, cols] bf16, hess_blocks [cols/16, 16, 16] float32
    -> (codes [rows, cols/2] u8, linear scales [rows, cols/16] u8, g [1] f32)."""
    rows = _rows(w, "w", min_rows=0)
    cols = int(w.shape[1])
    dev = w.device
    _require((w, "w", torch.bfloat16, None), (hess_blocks, "hess_blocks", torch.float32, (cols // 16, 16, 16)),
             (ws, "ws", torch.uint8, None))
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    g_out = torch.empty(1, dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(quantize_workspace_bytes(rows, cols), dev)
    st = lib().nvfp4moe_quantize_weights_lh(_ptr(w), rows, cols, _ptr(hess_blocks), int(m), _ptr(codes),
                                            _ptr(scales), _ptr(g_out), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "nvfp4moe_quantize_weights_lh")
    return codes, scales, g_out


def route_workspace_bytes(cfg: Cfg, T: int) -> int:
    return int(lib().nvfp4moe_route_workspace_bytes(ctypes.byref(cfg), T))


def route(cfg: Cfg, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None, ws=None,
          stream=None):
    """route(hidden, W_router) -> (idx [T, topk] int32, w [T, topk] float32)."""
    T = _rows(x, "x", min_rows=0)
    if T == 0:
        _require((x, "x", torch.bfloat16, (0, cfg.H)), (ws, "ws", torch.uint8, None))
    else:
        _require(*_layer_specs(cfg, x, w_router, bias), (ws, "ws", torch.uint8, None))
    dev = x.device
    idx = torch.empty((T, cfg.topk), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.topk), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(route_workspace_bytes(cfg, T), dev)
    st = lib().nvfp4moe_route(ctypes.byref(cfg), _ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(idx), _ptr(w),
                              _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "nvfp4moe_route")
    return idx, w


def route_noalloc(cfg: Cfg, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None,
                  stream=None):
    """route() without a workspace (nvfp4moe_route_noalloc): the router's scratch is a fixed
    device array inside the library, so T * E is limited to 1,212,416 and calls that may
    overlap on the GPU must be serialised.  -> (idx [T, topk] int32, w [T, topk] float32)."""
    T = _rows(x, "x", min_rows=0)
    if T == 0:
        _require((x, "x", torch.bfloat16, (0, cfg.H)))
    else:
        _require(*_layer_specs(cfg, x, w_router, bias))
    dev = x.device
    idx = torch.empty((T, cfg.topk), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.topk), dtype=torch.float32, device=dev)
    st = lib().nvfp4moe_route_noalloc(ctypes.byref(cfg), _ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(idx),
                                      _ptr(w), _stream(stream))
    _check(st, "nvfp4moe_route_noalloc")
    return idx, w


class Experts:
    """Library-owned NVFP4 expert weights (nvfp4moe_experts_create / _set / _destroy).  With
    ``e_count`` the handle holds only experts e_begin .. e_begin + e_count - 1 (one rank's share
    under expert parallelism, nvfp4moe_experts_create_local)."""

    def __init__(self, cfg: Cfg, e_begin: int = 0, e_count: int | None = None):
        self.cfg = cfg
        self.e_begin = int(e_begin)
        self.e_count = int(cfg.E - e_begin if e_count is None else e_count)
        h = ctypes.c_void_p()
        _check(lib().nvfp4moe_experts_create_local(ctypes.byref(cfg), self.e_begin, self.e_count, ctypes.byref(h)),
               "nvfp4moe_experts_create_local")
        self.handle = h

    def set(self, e: int, gate, up, down, g_h: float, stream=None):
        """gate/up/down: (codes, linear scales, global scale as float) from quantize()."""
        H, I = self.cfg.H, self.cfg.I
        specs = []
        for name, (codes, scales, _), rows, cols in (("gate", gate, I, H), ("up", up, I, H), ("down", down, H, I)):
            specs += [(codes, f"{name} codes", torch.uint8, (rows, cols // 2)),
                      (scales, f"{name} scales", torch.uint8, (rows, cols // 16))]
        _require(*specs)
        t = ExpertTensors(gate[0].data_ptr(), gate[1].data_ptr(), up[0].data_ptr(), up[1].data_ptr(),
                          down[0].data_ptr(), down[1].data_ptr(), float(gate[2]), float(up[2]),
                          float(down[2]), float(g_h))
        _check(lib().nvfp4moe_experts_set(self.handle, int(e), ctypes.byref(t), _stream(stream)),
               "nvfp4moe_experts_set")

    def set_from_bf16(self, e: int, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor, g_h: float,
                      stream=None):
        """Quantise BF16 gate [I, H], up [I, H], down [H, I] with nvfp4moe_quantize (dynamic
        per-tensor global scales, linear block scales) and copy them into expert e."""
        q = [quantize(w, stream=stream) for w in (gate, up, down)]
        gs = torch.cat([t[2] for t in q]).cpu().tolist()
        self.set(e, (q[0][0], q[0][1], gs[0]), (q[1][0], q[1][1], gs[1]), (q[2][0], q[2][1], gs[2]), g_h,
                 stream=stream)
        return gs

    def close(self):
        if self.handle:
            lib().nvfp4moe_experts_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def forward_workspace_bytes(cfg: Cfg, T_max: int) -> int:
    return int(lib().nvfp4moe_forward_workspace_bytes(ctypes.byref(cfg), T_max))


def _debug_tensors(cfg: Cfg, T: int, H: int, dev, x_norm: bool = False, h_f32: bool = False) -> dict:
    k, E, I = cfg.topk, cfg.E, cfg.I
    tensors = {
        "idx": torch.empty((T, k), dtype=torch.int32, device=dev),
        "w": torch.empty((T, k), dtype=torch.float32, device=dev),
        "g_x": torch.empty(1, dtype=torch.float32, device=dev),
        "xq_codes": torch.empty((T, H // 2), dtype=torch.uint8, device=dev),
        "xq_scales": torch.empty((T, H // 16), dtype=torch.uint8, device=dev),
        "counts": torch.empty(E, dtype=torch.int32, device=dev),
        "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "perm": torch.empty(T * k, dtype=torch.int32, device=dev),
        "hq_codes": torch.empty((T * k, I // 2), dtype=torch.uint8, device=dev),
        "hq_scales": torch.empty((T * k, I // 16), dtype=torch.uint8, device=dev),
        "logits": torch.empty((T, E), dtype=torch.float32, device=dev),
        "acc": torch.empty((T, H), dtype=torch.float32, device=dev),
    }
    if x_norm:
        tensors["x_norm"] = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if h_f32:
        tensors["h_f32"] = torch.empty((T * k, I), dtype=torch.float32, device=dev)
    return tensors


def forward_residual(experts: Experts, h: torch.Tensor, gamma: torch.Tensor, eps: float, step_k: int,
                     w_router: torch.Tensor, bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     ws: torch.Tensor | None = None, debug: bool = False, stream=None):
    """The layer fused with its residual-stream neighbours (nvfp4moe_forward_residual):
    h' = bf16(a h + b moe(rmsnorm(h) gamma)) for residual step ``step_k``.  ``out`` may be ``h``
    (in-place update).  Returns h' (and the intermediates, x_norm included, if debug)."""
    cfg = experts.cfg
    specs = _layer_specs(cfg, h, w_router, bias, name="h")
    T, H = h.shape
    dev = h.device
    _require(*specs, (gamma, "gamma", torch.float32, (H,)), (out, "out", torch.bfloat16, (T, H)),
             (ws, "ws", torch.uint8, None))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = _workspace(forward_workspace_bytes(cfg, T), dev)
    tensors = _debug_tensors(cfg, T, H, dev, x_norm=True) if debug else None
    dbg = Debug(**{n: t.data_ptr() for n, t in tensors.items()}) if debug else None
    st = lib().nvfp4moe_forward_residual(experts.handle, _ptr(h), T, _ptr(gamma), float(eps), int(step_k),
                                         _ptr(w_router), _ptr(bias), _ptr(out),
                                         ctypes.byref(dbg) if dbg is not None else None, _ptr(ws), ws.numel(),
                                         _stream(stream))
    _check(st, "nvfp4moe_forward_residual")
    if debug:
        return out, tensors
    return out


def forward(experts: Experts, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None,
            out: torch.Tensor | None = None, ws: torch.Tensor | None = None, debug: bool = False, stream=None,
            timer: StageTimer | None = None, wait_limit_us: int = 0, inject_skip_arrive: int = 0,
            debug_h: bool = False, separate_gemms: bool = False):
    """moe_forward(hidden, experts) -> out [T, H] bf16 (and a dict of intermediates if debug).
    ``timer``: a StageTimer whose events are recorded around each stage.  ``wait_limit_us``
    and ``inject_skip_arrive``: the failure-detection fields of nvfp4moe_debug (a bounded-wait
    limit, and the test hook that makes one front-end CTA skip a grid-barrier arrival).
    ``debug_h``: with debug, also the FP32 SwiGLU product of every pair (h_f32, [T*topk, I]).
    ``separate_gemms``: run the gate/up and down GEMMs as two launches instead of one."""
    cfg = experts.cfg
    specs = _layer_specs(cfg, x, w_router, bias)
    T, H = x.shape
    dev = x.device
    _require(*specs, (out, "out", torch.bfloat16, (T, H)), (ws, "ws", torch.uint8, None))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = _workspace(forward_workspace_bytes(cfg, T), dev)
    dbg = None
    tensors = None
    if debug:
        tensors = _debug_tensors(cfg, T, H, dev, h_f32=debug_h)
        dbg = Debug(**{n: t.data_ptr() for n, t in tensors.items()})
    if timer is not None:
        if dbg is None:
            dbg = Debug()
        dbg.events = ctypes.cast(timer.array, ctypes.POINTER(ctypes.c_void_p))
    if wait_limit_us or inject_skip_arrive or separate_gemms:
        if dbg is None:
            dbg = Debug()
        dbg.wait_limit_us = int(wait_limit_us)
        dbg.inject_skip_arrive = int(inject_skip_arrive)
        dbg.separate_gemms = int(bool(separate_gemms))
    st = lib().nvfp4moe_forward(experts.handle, _ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(out),
                                ctypes.byref(dbg) if dbg is not None else None, _ptr(ws), ws.numel(),
                                _stream(stream))
    _check(st, "nvfp4moe_forward")
    if debug:
        return out, tensors
    return out


# ------------------------------------------------------------------ FP8 W8A8 variant ----

def quantize_fp8(x: torch.Tensor, ws=None, stream=None):
    """Per-row FP8 quantisation (nvfp4moe_quantize_fp8): x [rows, cols] bf16 ->
    (codes [rows, cols] u8 E4M3, scales [rows] f32)."""
    rows = _rows(x, "x", min_rows=0)
    cols = int(x.shape[1])
    dev = x.device
    _require((x, "x", torch.bfloat16, None), (ws, "ws", torch.uint8, None))
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
    scales = torch.empty(rows, dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(quantize_workspace_bytes(rows, cols), dev)
    st = lib().nvfp4moe_quantize_fp8(_ptr(x), rows, cols, _ptr(codes), _ptr(scales), _ptr(ws), ws.numel(),
                                     _stream(stream))
    _check(st, "nvfp4moe_quantize_fp8")
    return codes, scales


class Fp8Experts:
    """Library-owned FP8 expert weights (nvfp4moe_fp8_experts_create / _set / _destroy)."""

    def __init__(self, cfg: Cfg):
        self.cfg = cfg
        h = ctypes.c_void_p()
        _check(lib().nvfp4moe_fp8_experts_create(ctypes.byref(cfg), ctypes.byref(h)),
               "nvfp4moe_fp8_experts_create")
        self.handle = h

    def set(self, e: int, gate, up, down, stream=None):
        """gate/up/down: (codes, scales) from quantize_fp8()."""
        H, I = self.cfg.H, self.cfg.I
        specs = []
        for name, (codes, scales), rows, cols in (("gate", gate, I, H), ("up", up, I, H), ("down", down, H, I)):
            specs += [(codes, f"{name} codes", torch.uint8, (rows, cols)),
                      (scales, f"{name} scales", torch.float32, (rows,))]
        _require(*specs)
        t = Fp8ExpertTensors(gate[0].data_ptr(), gate[1].data_ptr(), up[0].data_ptr(), up[1].data_ptr(),
                             down[0].data_ptr(), down[1].data_ptr())
        _check(lib().nvfp4moe_fp8_experts_set(self.handle, int(e), ctypes.byref(t), _stream(stream)),
               "nvfp4moe_fp8_experts_set")

    def set_from_bf16(self, e: int, gate: torch.Tensor, up: torch.Tensor, down: torch.Tensor, stream=None):
        """Quantise BF16 gate [I, H], up [I, H], down [H, I] per output channel and copy them in."""
        q = [quantize_fp8(w, stream=stream) for w in (gate, up, down)]
        self.set(e, q[0], q[1], q[2], stream=stream)
        return q

    def close(self):
        if self.handle:
            lib().nvfp4moe_fp8_experts_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def forward_fp8_workspace_bytes(cfg: Cfg, T_max: int) -> int:
    return int(lib().nvfp4moe_forward_fp8_workspace_bytes(ctypes.byref(cfg), T_max))


def forward_fp8(experts: Fp8Experts, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None,
                out: torch.Tensor | None = None, ws: torch.Tensor | None = None, debug: bool = False,
                stream=None):
    """The FP8 W8A8 layer (nvfp4moe_forward_fp8) -> out [T, H] bf16 (and intermediates if debug)."""
    cfg = experts.cfg
    specs = _layer_specs(cfg, x, w_router, bias)
    T, H = x.shape
    dev = x.device
    _require(*specs, (out, "out", torch.bfloat16, (T, H)), (ws, "ws", torch.uint8, None))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = _workspace(forward_fp8_workspace_bytes(cfg, T), dev)
    tensors = None
    dbg = None
    if debug:
        k, E = cfg.topk, cfg.E
        tensors = {
            "idx": torch.empty((T, k), dtype=torch.int32, device=dev),
            "w": torch.empty((T, k), dtype=torch.float32, device=dev),
            "counts": torch.empty(E, dtype=torch.int32, device=dev),
            "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "perm": torch.empty(T * k, dtype=torch.int32, device=dev),
            "logits": torch.empty((T, E), dtype=torch.float32, device=dev),
            "xq8_codes": torch.empty((T, H), dtype=torch.uint8, device=dev),
            "xq8_scales": torch.empty(T, dtype=torch.float32, device=dev),
        }
        dbg = Debug(**{n: t.data_ptr() for n, t in tensors.items()})
    st = lib().nvfp4moe_forward_fp8(experts.handle, _ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(out),
                                    ctypes.byref(dbg) if dbg is not None else None, _ptr(ws), ws.numel(),
                                    _stream(stream))
    _check(st, "nvfp4moe_forward_fp8")
    if debug:
        return out, tensors
    return out


# ------------------------------------------------------------- expert parallelism ----

def forward_partial(experts: Experts, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None = None,
                    acc_out: torch.Tensor | None = None, ws: torch.Tensor | None = None, debug: bool = False,
                    stream=None):
    """One rank's part of the layer (nvfp4moe_forward_partial): the FP32 sums [T, H] of the
    contributions of the handle's experts for all T tokens of x."""
    cfg = experts.cfg
    specs = _layer_specs(cfg, x, w_router, bias)
    T, H = x.shape
    dev = x.device
    _require(*specs, (acc_out, "acc_out", torch.float32, (T, H)), (ws, "ws", torch.uint8, None))
    if acc_out is None:
        acc_out = torch.empty((T, H), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(forward_workspace_bytes(cfg, T), dev)
    tensors = _debug_tensors(cfg, T, H, dev) if debug else None
    dbg = Debug(**{n: t.data_ptr() for n, t in tensors.items()}) if debug else None
    st = lib().nvfp4moe_forward_partial(experts.handle, _ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(acc_out),
                                        ctypes.byref(dbg) if dbg is not None else None, _ptr(ws), ws.numel(),
                                        _stream(stream))
    _check(st, "nvfp4moe_forward_partial")
    if debug:
        return acc_out, tensors
    return acc_out


def forward_partial_peer(experts: Experts, x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor | None,
                         acc_peers: torch.Tensor, rows_per_peer: int, ws: torch.Tensor | None = None, stream=None):
    """One rank's part of the layer with the cross-rank sum folded into the down GEMM
    (nvfp4moe_forward_partial_peer): token t's weighted expert rows are added into row
    t % rows_per_peer of the accumulator at acc_peers[t // rows_per_peer] (an int64 device
    tensor of device addresses, one per rank)."""
    cfg = experts.cfg
    specs = _layer_specs(cfg, x, w_router, bias)
    T, H = x.shape
    dev = x.device
    _require(*specs, (acc_peers, "acc_peers", torch.int64, (acc_peers.numel(),)), (ws, "ws", torch.uint8, None))
    if ws is None:
        ws = _workspace(forward_workspace_bytes(cfg, T), dev)
    st = lib().nvfp4moe_forward_partial_peer(experts.handle, _ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(acc_peers),
                                             acc_peers.numel(), int(rows_per_peer), None, _ptr(ws), ws.numel(),
                                             _stream(stream))
    _check(st, "nvfp4moe_forward_partial_peer")


IPC_HANDLE_BYTES = 64


def ipc_handle(t: torch.Tensor) -> tuple[bytes, int]:
    """The inter-process handle of the device allocation holding t and t's byte offset in it
    (nvfp4moe_ipc_get_handle)."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_int64()
    _check(lib().nvfp4moe_ipc_get_handle(ctypes.c_void_p(t.data_ptr()), buf, ctypes.byref(off)),
           "nvfp4moe_ipc_get_handle")
    return buf.raw, int(off.value)


def ipc_open(handle: bytes) -> int:
    """Maps another process's allocation (nvfp4moe_ipc_open); returns its device address here."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {IPC_HANDLE_BYTES} bytes, got {len(handle)}")
    ptr = ctypes.c_void_p()
    _check(lib().nvfp4moe_ipc_open(handle, ctypes.byref(ptr)), "nvfp4moe_ipc_open")
    return int(ptr.value)


def ipc_close(address: int):
    _check(lib().nvfp4moe_ipc_close(ctypes.c_void_p(address)), "nvfp4moe_ipc_close")


def finalize(acc: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """BF16 rounding of FP32 layer sums (nvfp4moe_finalize)."""
    _require((acc, "acc", torch.float32, None), (out, "out", torch.bfloat16, acc.shape))
    if out is None:
        out = torch.empty(acc.shape, dtype=torch.bfloat16, device=acc.device)
    _check(lib().nvfp4moe_finalize(_ptr(acc), acc.numel(), _ptr(out), _stream(stream)), "nvfp4moe_finalize")
    return out


# ------------------------------------------------- expert parallelism, all-to-all exchange ----

def amax(x: torch.Tensor, ws=None, stream=None) -> torch.Tensor:
    """max |x| of a BF16 tensor as its magnitude bit pattern (nvfp4moe_amax) -> int32 [1] on the
    device (below 2^15, so a maximum over int32 combines the ranks' values)."""
    rows = _rows(x, "x", min_rows=0)
    cols = int(x.shape[1])
    _require((x, "x", torch.bfloat16, None), (ws, "ws", torch.uint8, None))
    out = torch.empty(1, dtype=torch.int32, device=x.device)
    if ws is None:
        ws = _workspace(quantize_workspace_bytes(rows, cols), x.device)
    _check(lib().nvfp4moe_amax(_ptr(x), rows, cols, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "nvfp4moe_amax")
    return out


def ep_dispatch_workspace_bytes(cfg: Cfg, T: int) -> int:
    return int(lib().nvfp4moe_ep_dispatch_workspace_bytes(ctypes.byref(cfg), T))


def ep_dispatch(cfg: Cfg, n_ranks: int, x: torch.Tensor, w_router: torch.Tensor, bias, amax_bits: torch.Tensor,
                ws=None, stream=None) -> dict:
    """nvfp4moe_ep_dispatch: this rank's pairs in send order.  Returns a dict of device tensors:
    codes [P, H/2] u8, scales [P, H/16] u8, expert [P] i32 (destination-local), w [P] f32,
    pos [T*topk] i32 (send position of each pair), rank_counts [n_ranks] i32."""
    specs = _layer_specs(cfg, x, w_router, bias)
    T, H = x.shape
    dev = x.device
    _require(*specs, (amax_bits, "amax_bits", torch.int32, (1,)), (ws, "ws", torch.uint8, None))
    P = T * cfg.topk
    out = {"codes": torch.empty((P, H // 2), dtype=torch.uint8, device=dev),
           "scales": torch.empty((P, H // 16), dtype=torch.uint8, device=dev),
           "expert": torch.empty(P, dtype=torch.int32, device=dev),
           "w": torch.empty(P, dtype=torch.float32, device=dev),
           "pos": torch.empty(P, dtype=torch.int32, device=dev),
           "rank_counts": torch.empty(int(n_ranks), dtype=torch.int32, device=dev)}
    if ws is None:
        ws = _workspace(ep_dispatch_workspace_bytes(cfg, T), dev)
    st = lib().nvfp4moe_ep_dispatch(ctypes.byref(cfg), int(n_ranks), _ptr(x), T, _ptr(w_router), _ptr(bias),
                                    _ptr(amax_bits), _ptr(out["codes"]), _ptr(out["scales"]), _ptr(out["expert"]),
                                    _ptr(out["w"]), _ptr(out["pos"]), _ptr(out["rank_counts"]), _ptr(ws),
                                    ws.numel(), _stream(stream))
    _check(st, "nvfp4moe_ep_dispatch")
    return out


def ep_experts_workspace_bytes(cfg: Cfg, e_count: int, n_rows_max: int) -> int:
    return int(lib().nvfp4moe_ep_experts_workspace_bytes(ctypes.byref(cfg), int(e_count), int(n_rows_max)))


def ep_experts(experts: Experts, codes: torch.Tensor, scales: torch.Tensor, expert: torch.Tensor, w: torch.Tensor,
               amax_bits: torch.Tensor, out: torch.Tensor | None = None, ws=None, stream=None) -> torch.Tensor:
    """nvfp4moe_ep_experts: the handle's experts on received rows -> weighted FP32 rows [n, H]."""
    cfg = experts.cfg
    n = _rows(codes, "codes", min_rows=0)
    H = cfg.H
    _require((codes, "codes", torch.uint8, (n, H // 2)), (scales, "scales", torch.uint8, (n, H // 16)),
             (expert, "expert", torch.int32, (n,)), (w, "w", torch.float32, (n,)),
             (amax_bits, "amax_bits", torch.int32, (1,)), (out, "out", torch.float32, (n, H)),
             (ws, "ws", torch.uint8, None))
    dev = amax_bits.device
    if out is None:
        out = torch.empty((n, H), dtype=torch.float32, device=dev)
    if ws is None:
        ws = _workspace(ep_experts_workspace_bytes(cfg, experts.e_count, max(n, 1)), dev)
    st = lib().nvfp4moe_ep_experts(experts.handle, _ptr(codes), _ptr(scales), _ptr(expert), _ptr(w), n,
                                   _ptr(amax_bits), _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "nvfp4moe_ep_experts")
    return out


def ep_combine(rows: torch.Tensor, pos: torch.Tensor, T: int, topk: int, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """nvfp4moe_ep_combine: out [T, H] BF16, each token's topk returned rows added in slot order."""
    H = int(rows.shape[1])
    _require((rows, "rows", torch.float32, (T * topk, H)), (pos, "pos", torch.int32, (T * topk,)),
             (out, "out", torch.bfloat16, (T, H)))
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=rows.device)
    _check(lib().nvfp4moe_ep_combine(_ptr(rows), _ptr(pos), int(T), int(topk), H, _ptr(out), _stream(stream)),
           "nvfp4moe_ep_combine")
    return out
