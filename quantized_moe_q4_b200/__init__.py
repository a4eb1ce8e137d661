"""Python binding of the B200 4-bit MoE expert FFN library (libmoe_q4.so).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels (sm_100a).  PyTorch provides device memory and streams.  The function
names are the C ABI's (include/moe_q4.h).  Importing this module fails loudly
if the CUDA library has not been built; there is no fallback.

The layer is the MoE expert FFN of "A 35B Hybrid-Attention Mixture-of-Experts
Model on a 6GB 2011 GPU: Hand-Written 4-bit CUDA Inference for Fermi" (Dutch
technical summary, Methodologie 1 and 2): top-k routing, Q8_0 activations,
grouped W4A8 gate/up and down projections over Q4_0 expert weights, SwiGLU,
and the router-weighted combine.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_q4.so")

QK = 32
Q4_BYTES = 18

MOE_Q4_OK = 0
ERRORS = {
    -1: "MOE_Q4_ERR_INVALID_ARG", -2: "MOE_Q4_ERR_SHAPE", -3: "MOE_Q4_ERR_ALIGN",
    -4: "MOE_Q4_ERR_WORKSPACE", -5: "MOE_Q4_ERR_ARCH", -6: "MOE_Q4_ERR_CUDA", -7: "MOE_Q4_ERR_OVERLAP",
}
STATUS_SCALE_OVERFLOW = 0x1
STATUS_SPIN_TIMEOUT = 0x2
STATUS_NONFINITE_LOGIT = 0x4
STATUS_BAD_EXPERT_INDEX = 0x8

PATH_AUTO, PATH_GROUPED_DP4A, PATH_DECODE, PATH_TENSOR_CORE = 0, 1, 2, 3
PATH_TENSOR_CORE_N32, PATH_TENSOR_CORE_N128, PATH_TENSOR_CORE_N64 = 4, 5, 6

WS_NAMES = ["status", "logits", "topk_idx", "topk_w", "qa", "da", "cnt", "off", "tile_off",
            "chunk_cnt", "chunk_base", "sorted", "pos", "hq", "dh", "total"]

# Every extern "C" symbol of include/moe_q4.h.
EXPORTS = ["moe_q4_quantize_act", "moe_q4_route", "moe_q4_ffn_workspace_bytes", "moe_q4_ffn_forward",
           "moe_q4_ffn_host_workspace_bytes", "moe_q4_ffn_forward_host", "moe_q4_status_string",
           "moe_q4_workspace_layout", "moe_q4_ffn_forward_debug", "moe_q4_block_dots",
           "moe_q4_ffn_forward_noalloc", "moe_q4_last_cuda_error", "moe_q4_residual_rmsnorm",
           "moe_q4_stack_workspace_bytes", "moe_q4_stack_forward", "moe_q4_gemv_workspace_bytes", "moe_q4_gemv",
           "moe_q4_staging_bytes", "moe_q4_ffn_forward_streamed", "moe_q4_test_override_device",
           "moe_q4_rescale_ceiling"]


class MoeQ4Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        detail = moe_q4_status_string(code)
        if code == -6:
            detail += ": " + moe_q4_last_cuda_error()
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({detail})")


class _Layer(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("ffn", ctypes.c_int32), ("n_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("has_shared", ctypes.c_int32),
        ("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
        ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
        ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p), ("sh_down", ctypes.c_void_p),
    ]


class _Debug(ctypes.Structure):
    _fields_ = [("h_out", ctypes.c_void_p), ("path", ctypes.c_int32),
                ("ev_start", ctypes.c_void_p), ("ev_stop", ctypes.c_void_p), ("force_spin_timeout", ctypes.c_int32),
                ("block_dots_out", ctypes.c_void_p), ("block_dots_down", ctypes.c_int32),
                ("block_dots_group", ctypes.c_int32), ("block_dots_rb", ctypes.c_int32),
                ("decode_kernel_ns", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build the CUDA library first "
            "(python quantized_moe_q4_b200/build.py, or __graft_entry__.build()). There is no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    sigs = {
        "moe_q4_quantize_act": ([P, i64, i32, P, P, P, P], ctypes.c_int),
        "moe_q4_route": ([P, P, i64, P, P, P, P], ctypes.c_int),
        "moe_q4_ffn_workspace_bytes": ([P, i64], sz),
        "moe_q4_ffn_forward": ([P, P, i64, P, P, sz, P], ctypes.c_int),
        "moe_q4_ffn_host_workspace_bytes": ([P, i64], sz),
        "moe_q4_ffn_forward_host": ([P, P, i64, P, P, sz, P], ctypes.c_int),
        "moe_q4_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "moe_q4_workspace_layout": ([P, i64, P, ctypes.c_int], ctypes.c_int),
        "moe_q4_ffn_forward_debug": ([P, P, i64, P, P, sz, P, P], ctypes.c_int),
        "moe_q4_block_dots": ([P, P, i64, P, P], ctypes.c_int),
        "moe_q4_ffn_forward_noalloc": ([P, P, i64, P, P], ctypes.c_int),
        "moe_q4_last_cuda_error": ([], ctypes.c_char_p),
        "moe_q4_residual_rmsnorm": ([P, P, i64, i32, ctypes.c_float, P, P], ctypes.c_int),
        "moe_q4_stack_workspace_bytes": ([P, i64], sz),
        "moe_q4_stack_forward": ([P, i32, P, i64, ctypes.c_float, P, sz, P], ctypes.c_int),
        "moe_q4_gemv_workspace_bytes": ([i64, i32], sz),
        "moe_q4_gemv": ([P, i64, i32, P, i64, P, P, sz, P], ctypes.c_int),
        "moe_q4_staging_bytes": ([P], sz),
        "moe_q4_ffn_forward_streamed": ([P, P, i64, P, P, sz, P, sz, P], ctypes.c_int),
        "moe_q4_test_override_device": ([i32, i32, i32], ctypes.c_int),
        "moe_q4_rescale_ceiling": ([i32, i32, P, P, P], ctypes.c_int),
    }
    for name, (args, res) in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, what: str):
    if rc != MOE_Q4_OK:
        raise MoeQ4Error(rc, what)


def moe_q4_status_string(code: int) -> str:
    return _lib.moe_q4_status_string(int(code)).decode()


def moe_q4_last_cuda_error() -> str:
    return _lib.moe_q4_last_cuda_error().decode()


class Layer:
    """One MoE layer's weights on the device and its C descriptor.

    w_router [E,H] fp32, router_bias [E] fp32 or None, w_gate/w_up [E,F,H/32,18]
    uint8, w_down [E,H,F/32,18] uint8, sh_* the shared expert or None."""

    def __init__(self, hidden, ffn, n_experts, top_k, w_router, router_bias, w_gate, w_up, w_down,
                 sh_gate=None, sh_up=None, sh_down=None):
        self.hidden, self.ffn, self.n_experts, self.top_k = int(hidden), int(ffn), int(n_experts), int(top_k)
        self.tensors = dict(w_router=w_router, router_bias=router_bias, w_gate=w_gate, w_up=w_up,
                            w_down=w_down, sh_gate=sh_gate, sh_up=sh_up, sh_down=sh_down)
        for k, v in self.tensors.items():
            if v is not None and not v.is_contiguous():
                raise ValueError(f"{k} must be contiguous")
        self.has_shared = sh_gate is not None
        self.struct = _Layer(self.hidden, self.ffn, self.n_experts, self.top_k, int(self.has_shared),
                             *(None if v is None else v.data_ptr() for v in self.tensors.values()))

    @property
    def ref(self):
        return ctypes.byref(self.struct)

    @classmethod
    def from_host(cls, w, device="cuda"):
        """From an object with numpy attributes (hidden, ffn, n_experts, top_k,
        w_router, router_bias, w_gate, w_up, w_down, sh_gate, sh_up, sh_down)."""
        def dev(a):
            return None if a is None else torch.from_numpy(a).to(device).contiguous()
        return cls(w.hidden, w.ffn, w.n_experts, w.top_k, dev(w.w_router), dev(w.router_bias),
                   dev(w.w_gate), dev(w.w_up), dev(w.w_down), dev(w.sh_gate), dev(w.sh_up), dev(w.sh_down))

    @classmethod
    def from_host_pinned(cls, w, device="cuda"):
        """Router weights on the device, expert matrices in page-locked host
        memory (for moe_q4_ffn_forward_streamed)."""
        def dev(a):
            return None if a is None else torch.from_numpy(a).to(device).contiguous()

        def pinned(a):
            return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
        return cls(w.hidden, w.ffn, w.n_experts, w.top_k, dev(w.w_router), dev(w.router_bias),
                   pinned(w.w_gate), pinned(w.w_up), pinned(w.w_down), pinned(w.sh_gate), pinned(w.sh_up),
                   pinned(w.sh_down))

    def replica(self):
        """A copy of every weight tensor at new device addresses."""
        t = {k: (None if v is None else v.clone()) for k, v in self.tensors.items()}
        return Layer(self.hidden, self.ffn, self.n_experts, self.top_k, **t)


def moe_q4_quantize_act(x: torch.Tensor, q=None, d=None, status=None, stream=None):
    T, H = x.shape
    q = torch.empty((T, H), dtype=torch.int8, device=x.device) if q is None else q
    d = torch.empty((T, H // QK), dtype=torch.int16, device=x.device) if d is None else d
    _check(_lib.moe_q4_quantize_act(_p(x), T, H, _p(q), _p(d), _p(status), _stream(stream)), "moe_q4_quantize_act")
    return q, d


def moe_q4_route(layer: Layer, x: torch.Tensor, topk_idx=None, topk_w=None, logits=None, stream=None):
    T = x.shape[0]
    k, E = layer.top_k, layer.n_experts
    topk_idx = torch.empty((T, k), dtype=torch.int32, device=x.device) if topk_idx is None else topk_idx
    topk_w = torch.empty((T, k), dtype=torch.float32, device=x.device) if topk_w is None else topk_w
    logits = torch.empty((T, E), dtype=torch.float32, device=x.device) if logits is None else logits
    _check(_lib.moe_q4_route(layer.ref, _p(x), T, _p(topk_idx), _p(topk_w), _p(logits), _stream(stream)),
           "moe_q4_route")
    return topk_idx, topk_w, logits


def moe_q4_ffn_workspace_bytes(layer: Layer, T_max: int) -> int:
    return int(_lib.moe_q4_ffn_workspace_bytes(layer.ref, int(T_max)))


def moe_q4_ffn_host_workspace_bytes(layer: Layer, T_max: int) -> int:
    return int(_lib.moe_q4_ffn_host_workspace_bytes(layer.ref, int(T_max)))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned uint8 device buffer (torch's allocator aligns to 512)."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def moe_q4_ffn_forward(layer: Layer, x: torch.Tensor, y=None, workspace=None, stream=None):
    T = x.shape[0]
    y = torch.empty_like(x) if y is None else y
    if workspace is None:
        workspace = alloc_workspace(moe_q4_ffn_workspace_bytes(layer, T), x.device)
    _check(_lib.moe_q4_ffn_forward(layer.ref, _p(x), T, _p(y), _p(workspace), workspace.numel(),
                                   _stream(stream)), "moe_q4_ffn_forward")
    return y


def moe_q4_ffn_forward_debug(layer: Layer, x: torch.Tensor, y, workspace, h_out=None, path=PATH_AUTO,
                             ev_start=None, ev_stop=None, stream=None, force_spin_timeout=False,
                             block_dots=None, decode_kernel_ns=None):
    """block_dots: None or (out int32 tensor, down (bool), group, row block):
    capture the per-block integer dot products of that row block (see
    moe_q4_debug in include/moe_q4.h for the layout)."""
    T = x.shape[0]
    bd_out, bd_down, bd_group, bd_rb = (None, 0, 0, 0) if block_dots is None else block_dots
    dbg = _Debug(None if h_out is None else h_out.data_ptr(), int(path),
                 None if ev_start is None else ev_start.cuda_event,
                 None if ev_stop is None else ev_stop.cuda_event, int(bool(force_spin_timeout)),
                 None if bd_out is None else bd_out.data_ptr(), int(bool(bd_down)), int(bd_group), int(bd_rb),
                 None if decode_kernel_ns is None else decode_kernel_ns.data_ptr())
    _check(_lib.moe_q4_ffn_forward_debug(layer.ref, _p(x), T, _p(y), _p(workspace), workspace.numel(),
                                         ctypes.byref(dbg), _stream(stream)), "moe_q4_ffn_forward_debug")
    return y


def moe_q4_ffn_forward_host(layer: Layer, x_host: torch.Tensor, y_host: torch.Tensor, workspace, stream=None):
    """x_host/y_host: CPU tensors (pinned for asynchronous copies)."""
    T = x_host.shape[0]
    _check(_lib.moe_q4_ffn_forward_host(layer.ref, _p(x_host), T, _p(y_host), _p(workspace), workspace.numel(),
                                        _stream(stream)), "moe_q4_ffn_forward_host")
    return y_host


def moe_q4_workspace_layout(layer: Layer, T: int) -> dict:
    arr = (ctypes.c_size_t * len(WS_NAMES))()
    _check(_lib.moe_q4_workspace_layout(layer.ref, int(T), arr, len(WS_NAMES)), "moe_q4_workspace_layout")
    return dict(zip(WS_NAMES, list(arr)))


def workspace_views(layer: Layer, T: int, ws: torch.Tensor) -> dict:
    """Typed views of the intermediates inside a forward workspace (for tests)."""
    off = moe_q4_workspace_layout(layer, T)
    E, k, H, F = layer.n_experts, layer.top_k, layer.hidden, layer.ffn
    P = T * k
    slots = P + (T if layer.has_shared else 0)

    def v(name, dtype, shape):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return ws[off[name]:off[name] + nbytes].view(dtype).view(*shape)

    return dict(
        status=v("status", torch.int32, (4,)), logits=v("logits", torch.float32, (T, E)),
        topk_idx=v("topk_idx", torch.int32, (T, k)), topk_w=v("topk_w", torch.float32, (T, k)),
        qa=v("qa", torch.int8, (T, H)), da=v("da", torch.int16, (T, H // QK)),
        cnt=v("cnt", torch.int32, (E + 1,)), off=v("off", torch.int32, (E + 2,)),
        tile_off=v("tile_off", torch.int32, (E + 2,)), sorted=v("sorted", torch.int32, (P,)),
        pos=v("pos", torch.int32, (P,)), hq=v("hq", torch.int8, (slots, F)),
        dh=v("dh", torch.int16, (slots, F // QK)))


def moe_q4_block_dots(w_blocks: torch.Tensor, qa: torch.Tensor, out=None, stream=None):
    n = w_blocks.numel() // Q4_BYTES
    out = torch.empty(n, dtype=torch.int32, device=w_blocks.device) if out is None else out
    _check(_lib.moe_q4_block_dots(_p(w_blocks), _p(qa), n, _p(out), _stream(stream)), "moe_q4_block_dots")
    return out


def moe_q4_rescale_ceiling(int8_operands: bool, iters: int, sink: torch.Tensor, stream=None) -> int:
    """Launch the epilogue-rescale measurement kernel (include/moe_q4.h) on
    `stream`; returns the number of accumulator elements it rescales (each
    one 32 int8 multiply-adds).  sink: a device float32 tensor of >= 1."""
    n = ctypes.c_int64(0)
    _check(_lib.moe_q4_rescale_ceiling(int(bool(int8_operands)), int(iters), _p(sink), ctypes.byref(n),
                                       _stream(stream)), "moe_q4_rescale_ceiling")
    return n.value


def moe_q4_ffn_forward_noalloc(layer: Layer, x: torch.Tensor, y=None, stream=None):
    """The layer with the library's static device scratch instead of a
    caller workspace (for callers that cannot allocate device memory; see
    include/moe_q4.h).  Calls that overlap on the GPU race on the scratch."""
    T = x.shape[0]
    y = torch.empty_like(x) if y is None else y
    _check(_lib.moe_q4_ffn_forward_noalloc(layer.ref, _p(x), T, _p(y), _stream(stream)),
           "moe_q4_ffn_forward_noalloc")
    return y


# ---------------------------------------------------------------- stacks of layers

def moe_q4_residual_rmsnorm(x: torch.Tensor, y=None, eps: float = 1e-6, xn=None, stream=None):
    """x <- x + y (if y is given, in place), then returns xn = RMSNorm(x) (unit
    gain over the last dimension), written into `xn` if given."""
    T, H = x.shape
    xn = torch.empty_like(x) if xn is None else xn
    _check(_lib.moe_q4_residual_rmsnorm(_p(x), _p(y), T, H, float(eps), _p(xn), _stream(stream)),
           "moe_q4_residual_rmsnorm")
    return xn


def moe_q4_stack_workspace_bytes(layer: Layer, T_max: int) -> int:
    return int(_lib.moe_q4_stack_workspace_bytes(layer.ref, int(T_max)))


def moe_q4_stack_forward(layers, x: torch.Tensor, eps: float = 1e-6, workspace=None, stream=None):
    """x <- x + MoE_l(RMSNorm(x)) for every layer in order, in place on x."""
    T = x.shape[0]
    arr = (_Layer * len(layers))(*[l.struct for l in layers])
    if workspace is None:
        workspace = alloc_workspace(moe_q4_stack_workspace_bytes(layers[0], T), x.device)
    _check(_lib.moe_q4_stack_forward(arr, len(layers), _p(x), T, float(eps), _p(workspace), workspace.numel(),
                                     _stream(stream)), "moe_q4_stack_forward")
    return x


# ---------------------------------------------------------------- LM-head GEMV

def moe_q4_gemv_workspace_bytes(T: int, H: int) -> int:
    return int(_lib.moe_q4_gemv_workspace_bytes(int(T), int(H)))


def moe_q4_gemv(W: torch.Tensor, x: torch.Tensor, y=None, workspace=None, stream=None):
    """y [T, N] = W4A8 product of the Q4_0 matrix W [N, H/32, 18] (uint8) with
    the Q8_0 form of x [T, H] (T <= 8)."""
    T, H = x.shape
    N = W.shape[0]
    y = torch.empty((T, N), dtype=torch.float32, device=x.device) if y is None else y
    if workspace is None:
        workspace = alloc_workspace(moe_q4_gemv_workspace_bytes(T, H), x.device)
    _check(_lib.moe_q4_gemv(_p(W), N, H, _p(x), T, _p(y), _p(workspace), workspace.numel(), _stream(stream)),
           "moe_q4_gemv")
    return y


# ---------------------------------------------------------------- host-streamed experts

def moe_q4_staging_bytes(layer: Layer) -> int:
    return int(_lib.moe_q4_staging_bytes(layer.ref))


def moe_q4_ffn_forward_streamed(layer: Layer, x: torch.Tensor, y=None, workspace=None, staging=None, stream=None):
    """The layer with its expert matrices in page-locked host memory (see
    Layer.from_host_pinned): the experts the routing selects are copied into
    `staging` on the device, then the layer runs there."""
    T = x.shape[0]
    y = torch.empty_like(x) if y is None else y
    if workspace is None:
        workspace = alloc_workspace(moe_q4_ffn_workspace_bytes(layer, T), x.device)
    if staging is None:
        staging = alloc_workspace(moe_q4_staging_bytes(layer), x.device)
    _check(_lib.moe_q4_ffn_forward_streamed(layer.ref, _p(x), T, _p(y), _p(workspace), workspace.numel(),
                                            _p(staging), staging.numel(), _stream(stream)),
           "moe_q4_ffn_forward_streamed")
    return y


def moe_q4_test_override_device(enable: bool, major: int = 10, minor: int = 0) -> None:
    """Test hook: make every entry point see the current device as compute
    capability major.minor (enable=True) or query the driver again (False)."""
    _check(_lib.moe_q4_test_override_device(int(bool(enable)), int(major), int(minor)),
           "moe_q4_test_override_device")
