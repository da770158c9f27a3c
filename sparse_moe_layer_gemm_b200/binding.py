"""ctypes binding of libmoe.so (include/moe.h).

Argument marshalling only: torch tensors are checked for device, dtype and
contiguity and passed as raw device pointers together with torch's current
CUDA stream.  Every step of the layer runs in the library's kernels.  If the
library is missing, :func:`load_library` raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_NOT_LOADED = 6
MOE_F32 = 0
MOE_BF16 = 1
MOE_FP8_E4M3 = 2
MOE_PATH_AUTO = 0
MOE_PATH_MULTI = 1
MOE_PATH_FUSED = 2

# every symbol include/moe.h declares
EXPORTS = (
    "moe_config_check", "moe_create", "moe_load_weights", "moe_workspace_size",
    "moe_forward", "moe_workspace_size_host", "moe_forward_host", "moe_get_device_error",
    "moe_status_string", "moe_destroy", "moe_forward_oneshot", "moe_kernel_launches",
    "moe_set_stage_timing", "moe_get_stage_times", "moe_route_static",
    "moe_check_wait_timeout", "moe_load_weights_fp8", "moe_decode_e4m3",
    "moe_dense_config_check", "moe_dense_create", "moe_dense_load_weights",
    "moe_dense_workspace_size", "moe_dense_forward", "moe_dense_get_device_error",
    "moe_dense_destroy", "moe_create_shard", "moe_set_path", "moe_forward_path",
    "moe_check_fused_timeout", "moe_load_shard_weights", "moe_forward_host_async",
    "moe_forward_host_join",
)
MOE_NUM_STAGES = 7
STAGE_NAMES = ("router", "topk", "sort", "gather", "gate_up", "down", "combine")


class moe_config_t(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int),
        ("num_experts", ctypes.c_int),
        ("top_k", ctypes.c_int),
        ("intermediate", ctypes.c_int),
        ("shared_intermediate", ctypes.c_int),
        ("norm_expert_weight", ctypes.c_int),
        ("routed_scaling_factor", ctypes.c_float),
        ("use_router_bias", ctypes.c_int),
        ("swiglu_limit", ctypes.c_float),
        ("swiglu_limit_shared", ctypes.c_float),
        ("act_dtype", ctypes.c_int),
        ("weight_dtype", ctypes.c_int),
    ]


class moe_dense_config_t(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int),
        ("intermediate", ctypes.c_int),
        ("swiglu_limit", ctypes.c_float),
        ("act_dtype", ctypes.c_int),
        ("weight_dtype", ctypes.c_int),
    ]


class moe_routing_t(ctypes.Structure):
    _fields_ = [
        ("topk_idx", ctypes.c_void_p),
        ("topk_w", ctypes.c_void_p),
        ("counts", ctypes.c_void_p),
        ("offsets", ctypes.c_void_p),
        ("perm", ctypes.c_void_p),
        ("logits", ctypes.c_void_p),
    ]


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib: Optional[ctypes.CDLL] = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads libmoe.so: `path`, else $SPARSE_MOE_LIBRARY, else the in-tree
    build of ``sparse_moe_layer_gemm_b200.build``."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    env = os.environ.get("SPARSE_MOE_LIBRARY")
    p = path or env or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libmoe.so not found at {p}: run `python -m sparse_moe_layer_gemm_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i, sz, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    lib.moe_config_check.argtypes = [ctypes.POINTER(moe_config_t)]
    lib.moe_create.argtypes = [ctypes.POINTER(moe_config_t), ctypes.POINTER(vp)]
    lib.moe_create_shard.argtypes = [ctypes.POINTER(moe_config_t), i, i, i, ctypes.POINTER(vp)]
    lib.moe_load_weights.argtypes = [vp] * 9 + [vp]
    lib.moe_load_shard_weights.argtypes = [vp] * 9 + [vp]
    lib.moe_workspace_size.argtypes = [vp, i, ctypes.POINTER(sz)]
    lib.moe_workspace_size_host.argtypes = [vp, i, ctypes.POINTER(sz)]
    lib.moe_forward.argtypes = [vp, vp, i, vp, vp, sz, vp, ctypes.POINTER(moe_routing_t)]
    lib.moe_forward_host.argtypes = [vp, vp, i, vp, vp, sz, vp]
    lib.moe_forward_host_async.argtypes = [vp, vp, i, vp, vp, sz, vp]
    lib.moe_forward_host_join.argtypes = [vp, vp]
    lib.moe_get_device_error.argtypes = [vp, ctypes.POINTER(i)]
    lib.moe_status_string.argtypes = [i]
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_destroy.argtypes = [vp]
    lib.moe_destroy.restype = None
    lib.moe_forward_oneshot.argtypes = [vp] * 9 + [i] * 5 + [f] * 3 + [i, i, vp, vp]
    lib.moe_kernel_launches.argtypes = [vp, i]
    lib.moe_set_stage_timing.argtypes = [vp, i]
    lib.moe_route_static.argtypes = [vp, i, vp, vp, i, i, i, i, i, f, vp, vp, vp]
    lib.moe_check_wait_timeout.argtypes = [i, ctypes.POINTER(i)]
    lib.moe_load_weights_fp8.argtypes = [vp] * 16
    lib.moe_decode_e4m3.argtypes = [vp, sz, vp, vp]
    lib.moe_dense_config_check.argtypes = [ctypes.POINTER(moe_dense_config_t)]
    lib.moe_dense_create.argtypes = [ctypes.POINTER(moe_dense_config_t), ctypes.POINTER(vp)]
    lib.moe_dense_load_weights.argtypes = [vp, vp, vp, vp, vp]
    lib.moe_dense_workspace_size.argtypes = [vp, i, ctypes.POINTER(sz)]
    lib.moe_dense_forward.argtypes = [vp, vp, i, vp, vp, sz, vp]
    lib.moe_dense_get_device_error.argtypes = [vp, ctypes.POINTER(i)]
    lib.moe_dense_destroy.argtypes = [vp]
    lib.moe_dense_destroy.restype = None
    lib.moe_get_stage_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float), i,
                                        ctypes.POINTER(i)]
    lib.moe_set_path.argtypes = [vp, i]
    lib.moe_check_fused_timeout.argtypes = [vp, vp, i, vp, vp, sz, i, ctypes.POINTER(i)]
    lib.moe_forward_path.argtypes = [vp, i]
    for name in EXPORTS:
        if name not in ("moe_status_string", "moe_destroy", "moe_dense_destroy"):
            getattr(lib, name).restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load_library().moe_status_string(int(status)).decode()
    except RuntimeError:
        return "libmoe.so not loaded"


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def make_config(hidden, num_experts, top_k, intermediate, shared_intermediate=None, *,
                norm_expert_weight=True, routed_scaling_factor=3.0, use_router_bias=True,
                swiglu_limit=0.0, swiglu_limit_shared=0.0, act_dtype=MOE_BF16,
                weight_dtype=MOE_BF16) -> moe_config_t:
    return moe_config_t(hidden, num_experts, top_k, intermediate,
                        intermediate if shared_intermediate is None else shared_intermediate,
                        int(bool(norm_expert_weight)), float(routed_scaling_factor),
                        int(bool(use_router_bias)), float(swiglu_limit),
                        float(swiglu_limit_shared), int(act_dtype), int(weight_dtype))


def config_from_workload(wl) -> moe_config_t:
    dt = {"f32": MOE_F32, "bf16": MOE_BF16, "fp8": MOE_FP8_E4M3}
    return make_config(wl.hidden, wl.num_experts, wl.top_k, wl.intermediate,
                       wl.shared_intermediate, routed_scaling_factor=wl.scale,
                       swiglu_limit=wl.swiglu_limit, swiglu_limit_shared=wl.swiglu_limit_shared,
                       act_dtype=dt[wl.act_dtype], weight_dtype=dt[wl.weight_dtype])


# ----------------------------------------------------------------- raw ABI
def moe_config_check(cfg: moe_config_t) -> int:
    return load_library().moe_config_check(ctypes.byref(cfg))


def moe_create(cfg: moe_config_t) -> int:
    h = ctypes.c_void_p()
    _check(load_library().moe_create(ctypes.byref(cfg), ctypes.byref(h)), "moe_create")
    return h.value


def moe_create_shard(cfg: moe_config_t, expert_first: int, expert_count: int,
                     with_shared: bool) -> int:
    h = ctypes.c_void_p()
    _check(load_library().moe_create_shard(ctypes.byref(cfg), int(expert_first), int(expert_count),
                                           int(bool(with_shared)), ctypes.byref(h)),
           "moe_create_shard")
    return h.value


def moe_destroy(handle: int) -> None:
    load_library().moe_destroy(ctypes.c_void_p(handle))


def moe_workspace_size(handle: int, T: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().moe_workspace_size(ctypes.c_void_p(handle), T, ctypes.byref(n)),
           "moe_workspace_size")
    return n.value


def moe_workspace_size_host(handle: int, T: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().moe_workspace_size_host(ctypes.c_void_p(handle), T, ctypes.byref(n)),
           "moe_workspace_size_host")
    return n.value


def _stream(stream=None) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def moe_load_weights(handle, router_w, router_bias, w_gate, w_up, w_down, sh_gate, sh_up,
                     sh_down, stream=None) -> None:
    _check(load_library().moe_load_weights(
        ctypes.c_void_p(handle), _ptr(router_w), _ptr(router_bias), _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), _ptr(sh_gate), _ptr(sh_up), _ptr(sh_down), _stream(stream)),
        "moe_load_weights")


def moe_load_shard_weights(handle, router_w, router_bias, w_gate, w_up, w_down, sh_gate, sh_up,
                           sh_down, stream=None) -> None:
    _check(load_library().moe_load_shard_weights(
        ctypes.c_void_p(handle), _ptr(router_w), _ptr(router_bias), _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), _ptr(sh_gate), _ptr(sh_up), _ptr(sh_down), _stream(stream)),
        "moe_load_shard_weights")


def moe_load_weights_fp8(handle, router_w, router_bias, w_gate, w_up, w_down, s_gate, s_up,
                         s_down, sh_gate, sh_up, sh_down, sh_s_gate, sh_s_up, sh_s_down,
                         stream=None) -> None:
    _check(load_library().moe_load_weights_fp8(
        ctypes.c_void_p(handle), _ptr(router_w), _ptr(router_bias), _ptr(w_gate), _ptr(w_up),
        _ptr(w_down), _ptr(s_gate), _ptr(s_up), _ptr(s_down), _ptr(sh_gate), _ptr(sh_up),
        _ptr(sh_down), _ptr(sh_s_gate), _ptr(sh_s_up), _ptr(sh_s_down), _stream(stream)),
        "moe_load_weights_fp8")


def moe_decode_e4m3(codes: torch.Tensor, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """E4M3FN codes (uint8, CUDA) -> bf16 through the library's converter."""
    if out is None:
        out = torch.empty(codes.shape, dtype=torch.bfloat16, device=codes.device)
    _check(load_library().moe_decode_e4m3(_ptr(codes), codes.numel(), _ptr(out),
                                          _stream(stream)), "moe_decode_e4m3")
    return out


def moe_forward(handle, x, T, out, workspace, ws_bytes, stream=None, routing=None) -> int:
    r = None if routing is None else ctypes.byref(routing)
    return load_library().moe_forward(ctypes.c_void_p(handle), x, T, out, workspace, ws_bytes,
                                      _stream(stream), r)


def moe_forward_host(handle, x_host, T, out_host, workspace, ws_bytes, stream=None) -> int:
    return load_library().moe_forward_host(ctypes.c_void_p(handle), x_host, T, out_host,
                                           workspace, ws_bytes, _stream(stream))


def moe_forward_host_async(handle, x_host, T, out_host, workspace, ws_bytes, stream=None) -> int:
    return load_library().moe_forward_host_async(ctypes.c_void_p(handle), x_host, T, out_host,
                                                 workspace, ws_bytes, _stream(stream))


def moe_forward_host_join(handle, stream=None) -> int:
    return load_library().moe_forward_host_join(ctypes.c_void_p(handle), _stream(stream))


def moe_get_device_error(handle) -> int:
    v = ctypes.c_int()
    load_library().moe_get_device_error(ctypes.c_void_p(handle), ctypes.byref(v))
    return v.value


def moe_forward_oneshot(x, router_w, router_bias, w_gate, w_up, w_down, sh_gate, sh_up, sh_down,
                        T, H, E, k, I, scale, swiglu_limit, swiglu_limit_shared, act_dtype,
                        weight_dtype, out, stream=None) -> int:
    return load_library().moe_forward_oneshot(
        _ptr(x), _ptr(router_w), _ptr(router_bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
        _ptr(sh_gate), _ptr(sh_up), _ptr(sh_down), T, H, E, k, I, scale, swiglu_limit,
        swiglu_limit_shared, act_dtype, weight_dtype, _ptr(out), _stream(stream))


def moe_kernel_launches(handle, T: int) -> int:
    return load_library().moe_kernel_launches(ctypes.c_void_p(handle), T)


def moe_set_path(handle, path: int) -> None:
    """MOE_PATH_AUTO, MOE_PATH_MULTI or MOE_PATH_FUSED (see include/moe.h)."""
    _check(load_library().moe_set_path(ctypes.c_void_p(handle), path), "moe_set_path")


def moe_forward_path(handle, T: int) -> int:
    return load_library().moe_forward_path(ctypes.c_void_p(handle), T)


def moe_check_fused_timeout(handle, x, T, out, workspace, ws_bytes, limit_us):
    """-> (status, device status word); see include/moe.h."""
    word = ctypes.c_int(-1)
    r = load_library().moe_check_fused_timeout(ctypes.c_void_p(handle), _ptr(x), T, _ptr(out),
                                               _ptr(workspace), ws_bytes, limit_us,
                                               ctypes.byref(word))
    return r, word.value


def moe_set_stage_timing(handle, capacity: int) -> None:
    _check(load_library().moe_set_stage_timing(ctypes.c_void_p(handle), capacity),
           "moe_set_stage_timing")


def moe_get_stage_times(handle):
    """-> (dict stage name -> summed ms, number of recorded forwards)."""
    ms = (ctypes.c_float * MOE_NUM_STAGES)()
    n = ctypes.c_int()
    _check(load_library().moe_get_stage_times(ctypes.c_void_p(handle), ms, MOE_NUM_STAGES,
                                              ctypes.byref(n)), "moe_get_stage_times")
    return dict(zip(STAGE_NAMES, list(ms))), n.value


def moe_route_static(x, act_dtype, router_w, router_bias, T, H, E, k, norm_expert_weight,
                     routed_scaling_factor, topk_idx, topk_w, stream=None) -> int:
    """Routing with no device allocation (see include/moe.h): for callers
    that cannot call cudaMalloc, e.g. under CUDA-graph capture."""
    return load_library().moe_route_static(
        _ptr(x), act_dtype, _ptr(router_w), _ptr(router_bias), T, H, E, k,
        int(bool(norm_expert_weight)), float(routed_scaling_factor), _ptr(topk_idx),
        _ptr(topk_w), _stream(stream))


# ----------------------------------------------------------------- layer object
_TORCH_DT = {MOE_F32: torch.float32, MOE_BF16: torch.bfloat16}


class MoeLayer:
    """One layer on the current CUDA device: owns the library handle (and its
    packed weights) and a cached device workspace."""

    def __init__(self, cfg: moe_config_t, shard: Optional[tuple] = None):
        """shard: (expert_first, expert_count, with_shared) for an expert
        shard (see moe_create_shard), else the whole layer."""
        if not torch.cuda.is_available():
            raise RuntimeError("MoeLayer needs a CUDA device")
        self.cfg = cfg
        self.shard = shard
        self.device = torch.device("cuda", torch.cuda.current_device())
        self.handle = moe_create(cfg) if shard is None else moe_create_shard(cfg, *shard)
        self._ws: Optional[torch.Tensor] = None

    @classmethod
    def from_workload(cls, wl, shard: Optional[tuple] = None) -> "MoeLayer":
        return cls(config_from_workload(wl), shard)

    @property
    def act_dtype(self) -> torch.dtype:
        return _TORCH_DT[self.cfg.act_dtype]

    def set_path(self, path: int) -> None:
        moe_set_path(self.handle, path)

    def forward_path(self, T: int) -> int:
        return moe_forward_path(self.handle, T)

    def _need(self, t: torch.Tensor, name: str, dtype: torch.dtype, shape):
        if t.device != self.device or t.dtype != dtype or not t.is_contiguous() \
                or tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: want contiguous {dtype} {tuple(shape)} on {self.device}, "
                             f"got {t.dtype} {tuple(t.shape)} on {t.device}")

    def load_weights(self, router_w, router_bias, w_gate, w_up, w_down, sh_gate, sh_up, sh_down):
        c = self.cfg
        H, E, I, Is = c.hidden, c.num_experts, c.intermediate, c.shared_intermediate
        wdt = _TORCH_DT[c.weight_dtype]
        self._need(router_w, "router_w", torch.float32, (H, E))
        if router_bias is not None:
            self._need(router_bias, "router_bias", torch.float32, (E,))
        self._need(w_gate, "w_gate", wdt, (E, H, I))
        self._need(w_up, "w_up", wdt, (E, H, I))
        self._need(w_down, "w_down", wdt, (E, I, H))
        self._need(sh_gate, "sh_gate", wdt, (H, Is))
        self._need(sh_up, "sh_up", wdt, (H, Is))
        self._need(sh_down, "sh_down", wdt, (Is, H))
        moe_load_weights(self.handle, router_w, router_bias, w_gate, w_up, w_down, sh_gate,
                         sh_up, sh_down)

    def load_shard_weights(self, router_w, router_bias, w_gate, w_up, w_down, sh_gate=None,
                           sh_up=None, sh_down=None):
        """An expert shard's own experts only: w_gate, w_up [count, H, I],
        w_down [count, I, H] (see moe_load_shard_weights)."""
        c = self.cfg
        H, E, I, Is = c.hidden, c.num_experts, c.intermediate, c.shared_intermediate
        first, count, with_shared = self.shard if self.shard is not None else (0, E, 1)
        wdt = _TORCH_DT[c.weight_dtype]
        self._need(router_w, "router_w", torch.float32, (H, E))
        if router_bias is not None:
            self._need(router_bias, "router_bias", torch.float32, (E,))
        self._need(w_gate, "w_gate", wdt, (count, H, I))
        self._need(w_up, "w_up", wdt, (count, H, I))
        self._need(w_down, "w_down", wdt, (count, I, H))
        if with_shared:
            self._need(sh_gate, "sh_gate", wdt, (H, Is))
            self._need(sh_up, "sh_up", wdt, (H, Is))
            self._need(sh_down, "sh_down", wdt, (Is, H))
        moe_load_shard_weights(self.handle, router_w, router_bias, w_gate, w_up, w_down,
                               sh_gate, sh_up, sh_down)

    def load_weights_fp8(self, router_w, router_bias, w_gate, w_up, w_down, s_gate, s_up, s_down,
                         sh_gate, sh_up, sh_down, sh_s_gate, sh_s_up, sh_s_down):
        """E4M3FN codes (uint8) in the layouts of load_weights plus their fp32
        scales per output feature."""
        c = self.cfg
        H, E, I, Is = c.hidden, c.num_experts, c.intermediate, c.shared_intermediate
        self._need(router_w, "router_w", torch.float32, (H, E))
        if router_bias is not None:
            self._need(router_bias, "router_bias", torch.float32, (E,))
        u8, f32 = torch.uint8, torch.float32
        for t, name, dt, shape in ((w_gate, "w_gate", u8, (E, H, I)), (w_up, "w_up", u8, (E, H, I)),
                                   (w_down, "w_down", u8, (E, I, H)),
                                   (s_gate, "s_gate", f32, (E, I)), (s_up, "s_up", f32, (E, I)),
                                   (s_down, "s_down", f32, (E, H)),
                                   (sh_gate, "sh_gate", u8, (H, Is)), (sh_up, "sh_up", u8, (H, Is)),
                                   (sh_down, "sh_down", u8, (Is, H)),
                                   (sh_s_gate, "sh_s_gate", f32, (Is,)),
                                   (sh_s_up, "sh_s_up", f32, (Is,)),
                                   (sh_s_down, "sh_s_down", f32, (H,))):
            self._need(t, name, dt, shape)
        moe_load_weights_fp8(self.handle, router_w, router_bias, w_gate, w_up, w_down, s_gate,
                             s_up, s_down, sh_gate, sh_up, sh_down, sh_s_gate, sh_s_up, sh_s_down)

    def load_inputs(self, inp: Dict[str, torch.Tensor]):
        if self.cfg.weight_dtype == MOE_FP8_E4M3:
            self.load_weights_fp8(inp["router_w"], inp["router_bias"], inp["w_gate"], inp["w_up"],
                                  inp["w_down"], inp["s_w_gate"], inp["s_w_up"], inp["s_w_down"],
                                  inp["sh_gate"], inp["sh_up"], inp["sh_down"], inp["s_sh_gate"],
                                  inp["s_sh_up"], inp["s_sh_down"])
            return
        self.load_weights(inp["router_w"], inp["router_bias"], inp["w_gate"], inp["w_up"],
                          inp["w_down"], inp["sh_gate"], inp["sh_up"], inp["sh_down"])

    def workspace(self, T: int, host_io: bool = False) -> torch.Tensor:
        n = (moe_workspace_size_host if host_io else moe_workspace_size)(self.handle, T)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                routing: bool = False, stream=None):
        T = x.shape[0]
        self._need(x, "x", self.act_dtype, (T, self.cfg.hidden))
        if out is None:
            out = torch.empty_like(x)
        else:
            self._need(out, "out", self.act_dtype, (T, self.cfg.hidden))
        ws = self.workspace(T)
        r = None
        rt = None
        if routing:
            k, E = self.cfg.top_k, self.cfg.num_experts
            dev = self.device
            rt = dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
                      topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
                      counts=torch.empty(E, dtype=torch.int32, device=dev),
                      offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                      perm=torch.empty(T * k, dtype=torch.int32, device=dev),
                      logits=torch.empty(T, E, dtype=torch.float32, device=dev))
            r = moe_routing_t(*(rt[n].data_ptr() for n in
                                ("topk_idx", "topk_w", "counts", "offsets", "perm", "logits")))
        _check(moe_forward(self.handle, x.data_ptr(), T, out.data_ptr(), ws.data_ptr(),
                           ws.numel(), stream, r), "moe_forward")
        return (out, rt) if routing else out

    def forward_host(self, x_host: torch.Tensor, out_host: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
        """Host tensors in and out (pinned for asynchronous copies); returns
        after the result is on the host."""
        T = x_host.shape[0]
        if x_host.device.type != "cpu" or not x_host.is_contiguous() or x_host.dtype != self.act_dtype:
            raise ValueError("x_host must be a contiguous host tensor of the layer's dtype")
        if out_host is None:
            out_host = torch.empty_like(x_host, pin_memory=x_host.is_pinned())
        ws = self.workspace(T, host_io=True)
        _check(moe_forward_host(self.handle, x_host.data_ptr(), T, out_host.data_ptr(),
                                ws.data_ptr(), ws.numel(), stream), "moe_forward_host")
        return out_host

    def forward_host_async(self, x_host: torch.Tensor, out_host: torch.Tensor, stream=None):
        """Pipelined host forward (moe_forward_host_async): returns at once;
        out_host holds the result after forward_host_join(stream) and a
        synchronisation of that stream.  Both tensors pinned; neither may be
        touched before then."""
        T = x_host.shape[0]
        for t, name in ((x_host, "x_host"), (out_host, "out_host")):
            if (t.device.type != "cpu" or not t.is_contiguous() or t.dtype != self.act_dtype
                    or not t.is_pinned() or tuple(t.shape) != (T, self.cfg.hidden)):
                raise ValueError(f"{name} must be a pinned contiguous host tensor [T, H] of "
                                 "the layer's dtype")
        n = moe_workspace_size_host(self.handle, T)
        if self._ws is None or self._ws.numel() < n:
            # a larger workspace: the calls in flight finish with the old one first
            _check(moe_forward_host_join(self.handle, stream), "moe_forward_host_join")
            torch.cuda.synchronize(self.device)
        ws = self.workspace(T, host_io=True)
        _check(moe_forward_host_async(self.handle, x_host.data_ptr(), T, out_host.data_ptr(),
                                      ws.data_ptr(), ws.numel(), stream),
               "moe_forward_host_async")

    def forward_host_join(self, stream=None):
        """`stream` waits for the output copies of every forward_host_async."""
        _check(moe_forward_host_join(self.handle, stream), "moe_forward_host_join")

    def device_error(self) -> int:
        return moe_get_device_error(self.handle)

    def close(self):
        if getattr(self, "handle", None):
            moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_check_wait_timeout(limit_us: int):
    """Runs the bounded-wait self-check (see include/moe.h); returns
    (status code, device status word)."""
    word = ctypes.c_int(-1)
    r = load_library().moe_check_wait_timeout(limit_us, ctypes.byref(word))
    return r, word.value


# ----------------------------------------------------------------- dense MLP
_DT_CODE = {"f32": MOE_F32, "bf16": MOE_BF16, "fp8": MOE_FP8_E4M3}


def make_dense_config(hidden, intermediate, swiglu_limit=0.0, act_dtype=MOE_BF16,
                      weight_dtype=MOE_BF16) -> moe_dense_config_t:
    return moe_dense_config_t(int(hidden), int(intermediate), float(swiglu_limit),
                              int(act_dtype), int(weight_dtype))


def dense_config_from_workload(wl) -> moe_dense_config_t:
    return make_dense_config(wl.hidden, wl.intermediate, wl.swiglu_limit,
                             _DT_CODE[wl.act_dtype], _DT_CODE[wl.weight_dtype])


def moe_dense_config_check(cfg: moe_dense_config_t) -> int:
    return load_library().moe_dense_config_check(ctypes.byref(cfg))


class DenseMLP:
    """The dense SwiGLU MLP layer on the current CUDA device (owns the library
    handle and a cached workspace)."""

    def __init__(self, cfg: moe_dense_config_t):
        if not torch.cuda.is_available():
            raise RuntimeError("DenseMLP needs a CUDA device")
        self.cfg = cfg
        self.device = torch.device("cuda", torch.cuda.current_device())
        h = ctypes.c_void_p()
        _check(load_library().moe_dense_create(ctypes.byref(cfg), ctypes.byref(h)),
               "moe_dense_create")
        self.handle = h.value
        self._ws: Optional[torch.Tensor] = None

    @classmethod
    def from_workload(cls, wl) -> "DenseMLP":
        return cls(dense_config_from_workload(wl))

    def load_weights(self, w_gate, w_up, w_down):
        c = self.cfg
        dt = _TORCH_DT[c.weight_dtype]
        for t, name, shape in ((w_gate, "w_gate", (c.hidden, c.intermediate)),
                               (w_up, "w_up", (c.hidden, c.intermediate)),
                               (w_down, "w_down", (c.intermediate, c.hidden))):
            if t.device != self.device or t.dtype != dt or not t.is_contiguous() \
                    or tuple(t.shape) != shape:
                raise ValueError(f"{name}: want contiguous {dt} {shape} on {self.device}")
        _check(load_library().moe_dense_load_weights(ctypes.c_void_p(self.handle), _ptr(w_gate),
                                                     _ptr(w_up), _ptr(w_down), _stream(None)),
               "moe_dense_load_weights")

    def load_inputs(self, inp: Dict[str, torch.Tensor]):
        self.load_weights(inp["w_gate"], inp["w_up"], inp["w_down"])

    def workspace(self, T: int) -> torch.Tensor:
        n = ctypes.c_size_t()
        _check(load_library().moe_dense_workspace_size(ctypes.c_void_p(self.handle), T,
                                                       ctypes.byref(n)),
               "moe_dense_workspace_size")
        if self._ws is None or self._ws.numel() < n.value:
            self._ws = torch.empty(max(n.value, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
        T = x.shape[0]
        adt = _TORCH_DT[self.cfg.act_dtype]
        if x.device != self.device or x.dtype != adt or not x.is_contiguous() \
                or tuple(x.shape) != (T, self.cfg.hidden):
            raise ValueError(f"x: want contiguous {adt} (T, {self.cfg.hidden}) on {self.device}")
        if out is None:
            out = torch.empty_like(x)
        ws = self.workspace(T)
        _check(load_library().moe_dense_forward(ctypes.c_void_p(self.handle), x.data_ptr(), T,
                                                out.data_ptr(), ws.data_ptr(), ws.numel(),
                                                _stream(stream)), "moe_dense_forward")
        return out

    def device_error(self) -> int:
        v = ctypes.c_int()
        load_library().moe_dense_get_device_error(ctypes.c_void_p(self.handle), ctypes.byref(v))
        return v.value

    def close(self):
        if getattr(self, "handle", None):
            load_library().moe_dense_destroy(ctypes.c_void_p(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
