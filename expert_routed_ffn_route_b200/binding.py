"""Thin Python binding of the C ABI in ``include/moe_b200.h`` (ctypes).

Argument marshalling only: every step of the layer runs in the CUDA library.
PyTorch provides device memory and streams. There is no fallback: if the
shared library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import _build

FMT_CODE = {"bf16": 16, "int8": 8, "int4": 4, "nvfp4": 41}
PATH_CODE = {"auto": 0, "gemv": 1, "tc": 2, "fused": 3}
N_MARKS = 6

STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported", -3: "CUDA error",
          -4: "device timeout", -5: "workspace", -6: "device check failed",
          -7: "too large for the built-in scratch"}


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} ({status})")
        self.status = status


class MoeBank(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("group", ctypes.c_int32), ("n_exp", ctypes.c_int32),
                ("reserved", ctypes.c_int32),
                ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
                ("g_gate", ctypes.c_void_p), ("g_up", ctypes.c_void_p), ("g_down", ctypes.c_void_p)]


class MoeLayer(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("f", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("path", ctypes.c_int32),
                ("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("routed", MoeBank), ("shared", MoeBank)]


_LIB = None
EXPORTS = ["moe_abi_version", "moe_status_str", "moe_validate", "moe_workspace_size",
           "moe_route", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_layer_forward",
           "moe_layer_forward_marked", "moe_device_status", "moe_launches_per_call",
           "moe_layer_forward_static", "moe_static_device_status", "moe_test_inject_hold",
           "moe_nvfp4_pack_scales", "moe_nvfp4_quantize_rows", "moe_device_wait_site"]


def load_library(build_if_missing: bool = False) -> ctypes.CDLL:
    """Load ``libmoe_b200.so`` (in-tree). Raises if it is absent."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = _build.LIB_PATH
    if not os.path.exists(path):
        if build_if_missing:
            _build.build()
        else:
            raise RuntimeError(f"CUDA library not built: {path} (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    LP = ctypes.POINTER(MoeLayer)
    sig = {
        "moe_abi_version": (I32, []),
        "moe_status_str": (ctypes.c_char_p, [I32]),
        "moe_validate": (I32, [LP]),
        "moe_workspace_size": (SZ, [LP]),
        "moe_route": (I32, [LP, P, P, P, P, SZ, P]),
        "moe_permute": (I32, [LP, P, P, P, P, P, SZ, P]),
        "moe_grouped_ffn": (I32, [LP, P, P, P, P, P, P, SZ, P]),
        "moe_combine": (I32, [LP, P, P, P, P, P, P]),
        "moe_layer_forward": (I32, [LP, P, P, P, P, P, P, P, SZ, P]),
        "moe_layer_forward_marked": (I32, [LP, P, P, P, P, P, P, P, SZ, P,
                                           ctypes.POINTER(P), I32]),
        "moe_device_status": (I32, [LP, P, SZ, ctypes.POINTER(I32), P]),
        "moe_device_wait_site": (I32, [LP, P, SZ, ctypes.POINTER(I32), P]),
        "moe_launches_per_call": (I32, [LP]),
        "moe_layer_forward_static": (I32, [LP, P, P, P]),
        "moe_static_device_status": (I32, [ctypes.POINTER(I32), P]),
        "moe_test_inject_hold": (I32, [LP, P, SZ, I32, I32, P]),
        "moe_nvfp4_pack_scales": (I32, [P, P, I32, I32, I32, P]),
        "moe_nvfp4_quantize_rows": (I32, [P, I32, I32, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


def _check(status: int, what: str):
    if status != 0:
        raise MoeError(status, what)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def bank_struct(b) -> MoeBank:
    """A bank dict (fmt, group, n_exp and device tensors w_*, s_*, g_*) -> moe_bank."""
    if b is None:
        return MoeBank(16, 128, 0, 0, None, None, None, None, None, None, None, None, None)
    return MoeBank(FMT_CODE[b["fmt"]], b["group"], b["n_exp"], 0,
                   _ptr(b["w_gate"]), _ptr(b["w_up"]), _ptr(b["w_down"]),
                   _ptr(b.get("s_gate")), _ptr(b.get("s_up")), _ptr(b.get("s_down")),
                   _ptr(b.get("g_gate")), _ptr(b.get("g_up")), _ptr(b.get("g_down")))


class DeviceLayer:
    """Device-resident inputs of one layer that do not depend on the tokens:
    router weights, optional router bias, routed and shared expert banks."""

    def __init__(self, inputs, device="cuda", path: str = "auto"):
        import torch
        cfg = inputs.cfg
        self.cfg = cfg
        self.d, self.f, self.E, self.k = cfg.d, cfg.f, cfg.E, cfg.k
        self.path = PATH_CODE[path]
        dev = torch.device(device)

        def up(a, dtype=None):
            if a is None:
                return None
            if a.dtype == np.uint16:
                return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
            if a.dtype == np.uint32:
                return torch.from_numpy(a.view(np.int32)).to(dev)
            return torch.from_numpy(a).to(dev)

        self.router_w = up(inputs.router_w)
        self.router_bias = None if inputs.router_bias is None else \
            torch.from_numpy(inputs.router_bias.astype(np.float32)).to(dev)
        self.banks = {}
        for name, bank in (("routed", inputs.routed), ("shared", inputs.shared)):
            if bank is None:
                self.banks[name] = None
                continue
            self.banks[name] = dict(fmt=bank.fmt, group=bank.group, n_exp=bank.n_exp,
                                    **{k: up(v) for k, v in bank.arrays().items()})
            if bank.fmt == "nvfp4":  # block scales into the layout the kernels read
                b = self.banks[name]
                for m, (N, K) in (("gate", (cfg.f, cfg.d)), ("up", (cfg.f, cfg.d)),
                                  ("down", (cfg.d, cfg.f))):
                    b["s_" + m] = nvfp4_pack_scales(b["s_" + m], bank.n_exp, N, K)

    @classmethod
    def from_tensors(cls, cfg, router_w, router_bias, routed: dict, shared: dict | None,
                     path="auto"):
        self = cls.__new__(cls)
        self.cfg = cfg
        self.d, self.f, self.E, self.k = cfg.d, cfg.f, cfg.E, cfg.k
        self.path = PATH_CODE[path]
        self.router_w, self.router_bias = router_w, router_bias
        self.banks = {"routed": routed, "shared": shared}
        return self

    def _bank(self, b) -> MoeBank:
        return bank_struct(b)

    def descriptor(self, T: int, path: str | None = None) -> MoeLayer:
        return MoeLayer(T, self.d, self.f, self.E, self.k,
                        self.path if path is None else PATH_CODE[path],
                        _ptr(self.router_w), _ptr(self.router_bias),
                        self._bank(self.banks["routed"]), self._bank(self.banks["shared"]))

    @property
    def has_shared(self) -> bool:
        return self.banks["shared"] is not None


def _stream(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def workspace_size(L: MoeLayer) -> int:
    n = load_library().moe_workspace_size(ctypes.byref(L))
    if n == 0:
        raise MoeError(load_library().moe_validate(ctypes.byref(L)), "moe_workspace_size")
    return n


def alloc_workspace(L: MoeLayer, device="cuda"):
    """A zeroed workspace (the status word at its start must begin at zero). The fill is
    waited for here, so the workspace may be used on any stream: a fill still queued behind
    other work while a call runs on another stream would reset the call's barrier words."""
    import torch
    ws = torch.zeros(workspace_size(L), dtype=torch.uint8, device=device)
    torch.cuda.current_stream(ws.device).synchronize()
    return ws


def route(L: MoeLayer, x, ws, stream=None):
    import torch
    idx = torch.empty((L.T, L.k), dtype=torch.int32, device=x.device)
    w = torch.empty((L.T, L.k), dtype=torch.float32, device=x.device)
    _check(load_library().moe_route(ctypes.byref(L), x.data_ptr(), idx.data_ptr(), w.data_ptr(),
                                    ws.data_ptr(), ws.numel(), _stream(stream)), "moe_route")
    return idx, w


def permute(L: MoeLayer, topk_idx, ws, stream=None):
    import torch
    dev = topk_idx.device
    offsets = torch.empty(L.E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(L.T * L.k, dtype=torch.int32, device=dev)
    inv = torch.empty(L.T * L.k, dtype=torch.int32, device=dev)
    _check(load_library().moe_permute(ctypes.byref(L), topk_idx.data_ptr(), offsets.data_ptr(),
                                      perm.data_ptr(), inv.data_ptr(), ws.data_ptr(), ws.numel(),
                                      _stream(stream)), "moe_permute")
    return offsets, perm, inv


def grouped_ffn(L: MoeLayer, x, offsets, perm, ws, has_shared=True, stream=None):
    import torch
    dev = x.device
    y_assign = torch.empty((L.T * L.k, L.d), dtype=torch.float32, device=dev)
    y_shared = torch.empty((L.T, L.d), dtype=torch.float32, device=dev) if has_shared else None
    _check(load_library().moe_grouped_ffn(ctypes.byref(L), x.data_ptr(), offsets.data_ptr(),
                                          perm.data_ptr(), y_assign.data_ptr(), _ptr(y_shared),
                                          ws.data_ptr(), ws.numel(), _stream(stream)),
           "moe_grouped_ffn")
    return y_assign, y_shared


def combine(L: MoeLayer, y_assign, y_shared, inv, topk_w, out=None, stream=None):
    import torch
    if out is None:
        out = torch.empty((L.T, L.d), dtype=torch.bfloat16, device=y_assign.device)
    _check(load_library().moe_combine(ctypes.byref(L), y_assign.data_ptr(), _ptr(y_shared),
                                      inv.data_ptr(), topk_w.data_ptr(), out.data_ptr(),
                                      _stream(stream)), "moe_combine")
    return out


def layer_forward(L: MoeLayer, x, ws, out=None, topk_idx=None, topk_w=None, offsets=None,
                  perm=None, marks=None, stream=None):
    """The fused layer call. Optional outputs are written when tensors are given."""
    import torch
    if out is None:
        out = torch.empty((L.T, L.d), dtype=torch.bfloat16, device=x.device)
    lib = load_library()
    if marks is None:
        st = lib.moe_layer_forward(ctypes.byref(L), x.data_ptr(), out.data_ptr(), _ptr(topk_idx),
                                   _ptr(topk_w), _ptr(offsets), _ptr(perm), ws.data_ptr(),
                                   ws.numel(), _stream(stream))
    else:
        arr = (ctypes.c_void_p * len(marks))(*[None if m is None else m.cuda_event for m in marks])
        st = lib.moe_layer_forward_marked(ctypes.byref(L), x.data_ptr(), out.data_ptr(),
                                          _ptr(topk_idx), _ptr(topk_w), _ptr(offsets),
                                          _ptr(perm), ws.data_ptr(), ws.numel(),
                                          _stream(stream), arr, len(marks))
    _check(st, "moe_layer_forward")
    return out


def nvfp4_pack_scales(src, n_mats: int, rows: int, K: int, stream=None):
    """Block scales of an NVFP4 bank, uint8 [n_mats][rows][K/16] on the device, rearranged
    into the layout the FP4 tensor-core kernels read (a new tensor of the same size)."""
    import torch
    src = src.contiguous()
    dst = torch.empty_like(src)
    _check(load_library().moe_nvfp4_pack_scales(src.data_ptr(), dst.data_ptr(), n_mats, rows, K,
                                                _stream(stream)), "moe_nvfp4_pack_scales")
    return dst


def nvfp4_quantize_rows(v, stream=None):
    """fp32 rows [R, K] on the device -> (E2M1 codes uint8 [R, K/2], E4M3 block-scale codes
    uint8 [R, K/16], fp32 row scales [R]) by the layer's activation quantiser."""
    import torch
    v = v.contiguous()
    R, K = v.shape
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device=v.device)
    scales = torch.empty((R, K // 16), dtype=torch.uint8, device=v.device)
    g = torch.empty(R, dtype=torch.float32, device=v.device)
    _check(load_library().moe_nvfp4_quantize_rows(v.data_ptr(), R, K, codes.data_ptr(),
                                                  scales.data_ptr(), g.data_ptr(),
                                                  _stream(stream)), "moe_nvfp4_quantize_rows")
    return codes, scales, g


def launches_per_call(L: MoeLayer) -> int:
    return load_library().moe_launches_per_call(ctypes.byref(L))


def device_status(L: MoeLayer, ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(load_library().moe_device_status(ctypes.byref(L), ws.data_ptr(), ws.numel(),
                                            ctypes.byref(code), _stream(stream)),
           "moe_device_status")
    return code.value


def device_wait_site(L: MoeLayer, ws, stream=None) -> int:
    """Site of the first device-side wait that gave up since the last read (0: none)."""
    site = ctypes.c_int32(0)
    _check(load_library().moe_device_wait_site(ctypes.byref(L), ws.data_ptr(), ws.numel(),
                                               ctypes.byref(site), _stream(stream)),
           "moe_device_wait_site")
    return site.value


def layer_forward_static(L: MoeLayer, x, out=None, stream=None):
    """The layer with the library's built-in scratch (no workspace argument): for callers
    that cannot allocate device memory. Limits and sharing rules: include/moe_b200.h."""
    import torch
    if out is None:
        out = torch.empty((L.T, L.d), dtype=torch.bfloat16, device=x.device)
    _check(load_library().moe_layer_forward_static(ctypes.byref(L), x.data_ptr(),
                                                   out.data_ptr(), _stream(stream)),
           "moe_layer_forward_static")
    return out


def static_device_status(stream=None) -> int:
    """Reads and clears the status word of the built-in scratch (moe_layer_forward_static)."""
    code = ctypes.c_int32(0)
    _check(load_library().moe_static_device_status(ctypes.byref(code), _stream(stream)),
           "moe_static_device_status")
    return code.value


def test_inject_hold(L: MoeLayer, ws, hold: bool, budget_cycles: int = 0, stream=None):
    """Sets or clears the workspace's failure-injection hold word (see the header)."""
    _check(load_library().moe_test_inject_hold(ctypes.byref(L), ws.data_ptr(), ws.numel(),
                                               int(bool(hold)), int(budget_cycles),
                                               _stream(stream)), "moe_test_inject_hold")
