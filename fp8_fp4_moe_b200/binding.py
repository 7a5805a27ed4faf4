"""Thin ctypes binding of libmoe_b200.so (argument marshalling only).

PyTorch provides device memory and streams; every step of the layer runs in
the library's CUDA kernels.  There is no fallback: if the library is missing
or cannot run, these functions raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_DIR, "libmoe_b200.so")

# return codes (include/moe_b200.h)
MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_CUDA = -3
MOE_ERR_DEVICE_TIMEOUT = -4
MOE_ERR_WORKSPACE = -5
MOE_ERR_DEBUG_BOUNDS = -6

MOE_OPT_MAX_SMS = 1
MOE_OPT_TIMEOUT_NS = 2
MOE_OPT_INJECT_FAULT = 3
MOE_OPT_PHASE_EVENTS = 5
MOE_OPT_ROUTER_TC = 4
MOE_OPT_STATIC_WEIGHTS = 6
MOE_OPT_GRAPH = 7
MOE_OPT_SWAP_ROWS = 8
MOE_OPT_PAIR_TILES = 9
MOE_OPT_FUSED = 10
MOE_OPT_DEPENDENT_LAUNCH = 11
MOE_OPT_L2_TILE_ROWS = 12
MOE_OPT_CHAIN = 13
MOE_OPT_TILE_ROWS = 14
MOE_OPT_ZERO_PAD = 15

PHASES = ["router", "topk_rank", "scan", "scatter_quant", "prepare", "linear1", "linear2", "combine"]

REGIONS = {
    "status": 0, "topk_ids": 1, "gates": 2, "counts": 3, "offsets": 4, "perm": 5, "slot_pos": 6,
    "xq": 7, "xsf": 8, "hq": 9, "hsf": 10, "y": 11, "stamps": 12,
}

EXPORTED = [
    "moe_plan", "moe_plan_set_option", "moe_plan_get_option", "moe_workspace_bytes", "moe_set_workspace", "moe_workspace_region",
    "moe_forward", "moe_debug_routing", "moe_debug_dispatch", "moe_debug_quant_x", "moe_check_status",
    "moe_plan_destroy", "moe_error_string", "moe_phase_times", "moe_prepare_weights", "moe_route_noalloc",
    "moe_update_bias", "moe_gemm_workspace_bytes", "moe_gemm_fp8_fp4",
]

_lib = None


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {error_string(code)} ({code})")


def lib() -> ctypes.CDLL:
    """Load the library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m fp8_fp4_moe_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.moe_plan.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(vp)]
    L.moe_plan.restype = i32
    L.moe_plan_set_option.argtypes = [vp, i32, ctypes.c_longlong]
    L.moe_plan_set_option.restype = i32
    L.moe_plan_get_option.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_longlong)]
    L.moe_plan_get_option.restype = i32
    L.moe_workspace_bytes.argtypes = [vp]
    L.moe_workspace_bytes.restype = sz
    L.moe_set_workspace.argtypes = [vp, vp, sz]
    L.moe_set_workspace.restype = i32
    L.moe_workspace_region.argtypes = [vp, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.moe_workspace_region.restype = i32
    L.moe_forward.argtypes = [vp] * 10
    L.moe_forward.restype = i32
    L.moe_debug_routing.argtypes = [vp] * 7
    L.moe_debug_routing.restype = i32
    L.moe_debug_dispatch.argtypes = [vp] * 7
    L.moe_debug_dispatch.restype = i32
    L.moe_debug_quant_x.argtypes = [vp] * 5
    L.moe_debug_quant_x.restype = i32
    L.moe_check_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    L.moe_check_status.restype = i32
    L.moe_route_noalloc.argtypes = [i32, i32, i32, i32] + [vp] * 6
    L.moe_route_noalloc.restype = i32
    L.moe_prepare_weights.argtypes = [vp] * 4
    L.moe_prepare_weights.restype = i32
    L.moe_phase_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float), i32]
    L.moe_phase_times.restype = i32
    L.moe_gemm_workspace_bytes.argtypes = [i32, i32, i32]
    L.moe_gemm_workspace_bytes.restype = sz
    L.moe_gemm_fp8_fp4.argtypes = [i32, i32, i32] + [vp] * 6 + [sz, vp]
    L.moe_gemm_fp8_fp4.restype = i32
    L.moe_update_bias.argtypes = [vp, vp, ctypes.c_float, vp]
    L.moe_update_bias.restype = i32
    L.moe_plan_destroy.argtypes = [vp]
    L.moe_plan_destroy.restype = None
    L.moe_error_string.argtypes = [i32]
    L.moe_error_string.restype = ctypes.c_char_p
    _lib = L
    return L


def error_string(code: int) -> str:
    try:
        return lib().moe_error_string(code).decode()
    except Exception:  # pragma: no cover - library missing
        return f"code {code}"


def _check(code: int, what: str):
    if code != MOE_OK:
        raise MoeError(code, what)


def _ptr(t: torch.Tensor, dtype, device) -> int:
    if t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"tensor on {t.device}, plan on {device}")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def gemm_fp8_fp4(A, A_scales, B, B_scales, out=None, workspace=None, stream=None):
    """Dense block-scaled GEMM through moe_gemm_fp8_fp4: out [M, N] bf16 = A . B^T with
    A E4M3 codes [M, K] (uint8) and UE8M0 scales [M, K/128], B packed E2M1 [N, K/2] and
    UE8M0 scales [N, K/32].  Returns (out, workspace); the first int32 of the workspace is
    the device status once the stream has run the call."""
    M, K = A.shape
    N = B.shape[0]
    d = A.device
    L = lib()
    need = L.moe_gemm_workspace_bytes(M, N, K)
    if need == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_gemm_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=d)
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=d)
    for t, n in ((A_scales, (M, K // 128)), (B, (N, K // 2)), (B_scales, (N, K // 32))):
        if tuple(t.shape) != n:
            raise ValueError(f"expected shape {n}, got {tuple(t.shape)}")
    _check(L.moe_gemm_fp8_fp4(M, N, K, _ptr(A, torch.uint8, d), _ptr(A_scales, torch.uint8, d),
                              _ptr(B, torch.uint8, d), _ptr(B_scales, torch.uint8, d),
                              _ptr(out, torch.bfloat16, d), _ptr(workspace, torch.uint8, d), workspace.numel(),
                              _stream_ptr(stream)), "moe_gemm_fp8_fp4")
    return out, workspace


def route_noalloc(x, W_router, bias, k: int, topk_ids=None, gates=None, stream=None):
    """Routing through moe_route_noalloc: no plan, no workspace, no device allocation
    inside the library (the outputs are the caller's; pass them to avoid any
    allocation here too).  Runs on x's device (made current for the call; `stream`, if
    given, must belong to it).  Returns (topk_ids int32 [T,k], gates fp32 [T,k])."""
    if x.dim() != 2:
        raise ValueError(f"x must be [T, H], got shape {tuple(x.shape)}")
    T, H = x.shape
    if W_router.dim() != 2 or W_router.shape[1] != H:
        raise ValueError(f"W_router must be [E, {H}], got shape {tuple(W_router.shape)}")
    E = W_router.shape[0]
    if bias.dim() != 1 or bias.numel() != E:
        raise ValueError(f"bias must be [{E}], got shape {tuple(bias.shape)}")
    d = x.device
    if d.type != "cuda":
        raise ValueError(f"x must be on a CUDA device, got {d}")
    with torch.cuda.device(d):
        if topk_ids is None:
            topk_ids = torch.empty(T, k, dtype=torch.int32, device=d)
        if gates is None:
            gates = torch.empty(T, k, dtype=torch.float32, device=d)
        for name, t in (("topk_ids", topk_ids), ("gates", gates)):
            if tuple(t.shape) != (T, k):
                raise ValueError(f"{name} must be [{T}, {k}], got shape {tuple(t.shape)}")
        if stream is None:
            stream = torch.cuda.current_stream(d)
        elif stream.device != d:
            raise ValueError(f"stream on {stream.device}, x on {d}")
        rc = lib().moe_route_noalloc(T, H, E, k, _ptr(x, torch.bfloat16, d), _ptr(W_router, torch.float32, d),
                                     _ptr(bias, torch.float32, d), _ptr(topk_ids, torch.int32, d),
                                     _ptr(gates, torch.float32, d), stream.cuda_stream)
    _check(rc, "moe_route_noalloc")
    return topk_ids, gates


class Plan:
    """One layer shape bound to one device and a torch-allocated workspace."""

    def __init__(self, T: int, H: int, I: int, E: int, k: int, shared: int, device=None):
        L = lib()
        self.T, self.H, self.I, self.E, self.k, self.shared = T, H, I, E, k, shared
        self.n = E + shared
        self.rows = T * k + shared * T
        h = ctypes.c_void_p()
        _check(L.moe_plan(T, H, I, E, k, shared, ctypes.byref(h)), "moe_plan")
        self._h = h
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        nbytes = L.moe_workspace_bytes(h)
        with torch.cuda.device(self.device):
            self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            _check(L.moe_set_workspace(h, self.workspace.data_ptr(), nbytes), "moe_set_workspace")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.moe_plan_destroy(h)
            self._h = None

    def set_option(self, key: int, value: int):
        _check(lib().moe_plan_set_option(self._h, key, value), "moe_plan_set_option")

    def get_option(self, key: int) -> int:
        """The option's value for this plan (row-tile heights resolved to what the GEMMs use)."""
        v = ctypes.c_longlong()
        _check(lib().moe_plan_get_option(self._h, key, ctypes.byref(v)), "moe_plan_get_option")
        return v.value

    def region(self, name: str) -> torch.Tensor:
        """A typed view of a workspace region (for tests and debugging)."""
        off, n = ctypes.c_size_t(), ctypes.c_size_t()
        _check(lib().moe_workspace_region(self._h, REGIONS[name], ctypes.byref(off), ctypes.byref(n)), "region")
        raw = self.workspace[off.value:off.value + n.value]
        dt = {"status": torch.int32, "topk_ids": torch.int32, "gates": torch.float32, "counts": torch.int32,
              "offsets": torch.int32, "perm": torch.int32, "slot_pos": torch.int32, "xq": torch.uint8,
              "xsf": torch.uint8, "hq": torch.uint8, "hsf": torch.uint8, "y": torch.bfloat16,
              "stamps": torch.int64}[name]
        v = raw.view(dt)
        shapes = {"topk_ids": (self.T, self.k), "gates": (self.T, self.k), "slot_pos": (self.T, self.k),
                  "xq": (self.rows, self.H), "xsf": (-1, self.H // 128, 512), "hq": (self.rows, self.I),
                  "hsf": (-1, self.I // 128, 512), "y": (self.rows, self.H), "stamps": (-1, 1024)}
        return v.view(shapes[name]) if name in shapes else v

    def forward(self, x, W_router, bias, W1, W1_scales, W2, W2_scales, out=None, stream=None):
        d = self.device
        if out is None:
            out = torch.empty(self.T, self.H, dtype=torch.bfloat16, device=d)
        rc = lib().moe_forward(self._h, _ptr(x, torch.bfloat16, d), _ptr(W_router, torch.float32, d),
                               _ptr(bias, torch.float32, d), _ptr(W1, torch.uint8, d),
                               _ptr(W1_scales, torch.uint8, d), _ptr(W2, torch.uint8, d),
                               _ptr(W2_scales, torch.uint8, d), _ptr(out, torch.bfloat16, d), _stream_ptr(stream))
        _check(rc, "moe_forward")
        return out

    def prepare_weights(self, W1_scales, W2_scales, stream=None):
        d = self.device
        _check(lib().moe_prepare_weights(self._h, _ptr(W1_scales, torch.uint8, d), _ptr(W2_scales, torch.uint8, d),
                                         _stream_ptr(stream)), "moe_prepare_weights")

    def debug_routing(self, x, W_router, bias, stream=None):
        d = self.device
        for name, t, shape in (("x", x, (self.T, self.H)), ("W_router", W_router, (self.E, self.H)),
                               ("bias", bias, (self.E,))):
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} must be {list(shape)}, got shape {tuple(t.shape)}")
        ids = torch.empty(self.T, self.k, dtype=torch.int32, device=d)
        gates = torch.empty(self.T, self.k, dtype=torch.float32, device=d)
        _check(lib().moe_debug_routing(self._h, _ptr(x, torch.bfloat16, d), _ptr(W_router, torch.float32, d),
                                       _ptr(bias, torch.float32, d), ids.data_ptr(), gates.data_ptr(),
                                       _stream_ptr(stream)), "moe_debug_routing")
        return ids, gates

    def debug_dispatch(self, topk_ids, stream=None):
        d = self.device
        counts = torch.empty(self.n, dtype=torch.int32, device=d)
        offsets = torch.empty(self.n + 1, dtype=torch.int32, device=d)
        perm = torch.empty(self.T * self.k, dtype=torch.int32, device=d)
        slot_pos = torch.empty(self.T, self.k, dtype=torch.int32, device=d)
        _check(lib().moe_debug_dispatch(self._h, _ptr(topk_ids, torch.int32, d), counts.data_ptr(),
                                        offsets.data_ptr(), perm.data_ptr(), slot_pos.data_ptr(),
                                        _stream_ptr(stream)), "moe_debug_dispatch")
        return counts, offsets, perm, slot_pos

    def debug_quant_x(self, x, stream=None):
        d = self.device
        xq = torch.empty(self.T, self.H, dtype=torch.uint8, device=d)
        xs = torch.empty(self.T, self.H // 128, dtype=torch.float32, device=d)
        _check(lib().moe_debug_quant_x(self._h, _ptr(x, torch.bfloat16, d), xq.data_ptr(), xs.data_ptr(),
                                       _stream_ptr(stream)), "moe_debug_quant_x")
        return xq, xs

    def phase_times(self):
        """Per-kernel milliseconds of the last forward run with MOE_OPT_PHASE_EVENTS = 1."""
        buf = (ctypes.c_float * len(PHASES))()
        n = lib().moe_phase_times(self._h, buf, len(PHASES))
        if n < 0:
            raise MoeError(n, "moe_phase_times")
        return dict(zip(PHASES, list(buf)[:n]))

    def update_bias(self, bias, gamma: float, stream=None):
        """bias (device fp32 [E]) += gamma * sign(mean load - load), from the last forward's counts."""
        if bias.numel() != self.E:
            raise ValueError(f"bias has {bias.numel()} entries, the plan has {self.E} routed experts")
        _check(lib().moe_update_bias(self._h, _ptr(bias, torch.float32, self.device), ctypes.c_float(gamma),
                                     _stream_ptr(stream)), "moe_update_bias")
        return bias

    def check_status(self, stream=None):
        detail = (ctypes.c_uint32 * 4)()
        code = lib().moe_check_status(self._h, _stream_ptr(stream), detail)
        return code, list(detail)
