"""Python binding of libcoli (include/coli.h): one GLM-5.2-shaped MoE layer
forward on a B200 -- sigmoid router with correction-bias top-k, bucketing,
SwiGLU experts with packed int4 weights and Q8_0 int8 activations, weighted
combine plus the shared expert.

This module only marshals arguments: torch CUDA tensors go in as device
pointers and every step runs in the library's CUDA kernels.  There is no
fallback: if libcoli.so is missing or fails to load, every call raises.
PyTorch supplies device memory and the current stream.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcoli.so")

COLI_OK, COLI_EINVAL, COLI_ENOMEM, COLI_ECUDA, COLI_ETIMEOUT, COLI_EDEVICE = range(6)

# every symbol include/coli.h declares
EXPORTS = [
    "coli_quantize_rows_int4", "coli_quantize_act_q8", "coli_moe_route", "coli_moe_bucket",
    "coli_moe_expert_ffn", "coli_moe_layer_forward", "coli_moe_stack_forward", "coli_rmsnorm",
    "coli_moe_workspace_bytes", "coli_last_error", "coli_debug_block_partials",
    "coli_debug_phase_events", "coli_moe_layer_forward_noalloc", "coli_sync_status", "coli_debug_wait_probe",
    "coli_requantize_fp8_int4", "coli_moe_prepared_bytes", "coli_moe_prepare", "coli_quantize_rows_int8",
    "coli_debug_capture_partials",
]


class ColiError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"coli status {status}: {msg}")
        self.status = status


class MoeConfig(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("inter", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("n_shared", C.c_int32), ("shared_inter", C.c_int32),
                ("norm_topk_prob", C.c_int32), ("routed_scaling_factor", C.c_float), ("weight_bits", C.c_int32)]


class Expert(C.Structure):
    _fields_ = [("gate_q", C.c_void_p), ("gate_s", C.c_void_p), ("up_q", C.c_void_p),
                ("up_s", C.c_void_p), ("down_q", C.c_void_p), ("down_s", C.c_void_p)]


class MoeLayerC(C.Structure):
    _fields_ = [("cfg", MoeConfig), ("w_router", C.c_void_p), ("bias", C.c_void_p),
                ("experts", C.POINTER(Expert)), ("shared", C.POINTER(Expert)), ("prepared", C.c_void_p)]


_lib = None


def load(path: str | None = None):
    """Load libcoli.so (built by ``python -m int4_weight_only_sigmoid_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libcoli.so not found at {p}: build it with "
                          "`python -m int4_weight_only_sigmoid_b200.build` (no CPU fallback exists)")
    L = C.CDLL(p)
    vp, i64, i32, f32, st = C.c_void_p, C.c_int64, C.c_int32, C.c_float, C.c_int
    sig = {
        "coli_quantize_rows_int4": (st, [vp, i64, i64, vp, vp, vp]),
        "coli_quantize_act_q8": (st, [vp, i64, i64, vp, vp, vp]),
        "coli_moe_route": (st, [C.POINTER(MoeLayerC), vp, i64, vp, vp, vp, vp]),
        "coli_moe_bucket": (st, [vp, i64, i32, i32, vp, vp, vp, vp]),
        "coli_moe_expert_ffn": (st, [C.POINTER(MoeConfig), C.POINTER(Expert), vp, vp, i64, vp, vp,
                                     C.c_size_t, vp]),
        "coli_moe_layer_forward": (st, [C.POINTER(MoeLayerC), vp, i64, vp, vp, C.c_size_t, vp]),
        "coli_moe_stack_forward": (st, [C.POINTER(MoeLayerC), i32, vp, i64, f32, vp, vp,
                                        C.c_size_t, vp]),
        "coli_rmsnorm": (st, [vp, i64, i64, f32, vp, vp]),
        "coli_moe_workspace_bytes": (C.c_size_t, [C.POINTER(MoeConfig), i64]),
        "coli_last_error": (C.c_char_p, []),
        "coli_debug_block_partials": (st, [C.POINTER(Expert), i32, vp, i64, i64, i64, vp, vp]),
        "coli_debug_phase_events": (st, [vp, vp, vp]),
        "coli_moe_layer_forward_noalloc": (st, [C.POINTER(MoeLayerC), vp, i64, vp, vp]),
        "coli_sync_status": (st, [vp, vp]),
        "coli_debug_wait_probe": (st, [vp, i64, vp]),
        "coli_requantize_fp8_int4": (st, [vp, vp, i64, i64, i32, vp, vp, vp]),
        "coli_moe_prepared_bytes": (C.c_size_t, [C.POINTER(MoeConfig)]),
        "coli_quantize_rows_int8": (st, [vp, i64, i64, vp, vp, vp]),
        "coli_debug_capture_partials": (st, [vp, C.c_size_t]),
        "coli_moe_prepare": (st, [C.POINTER(MoeLayerC), vp, C.c_size_t, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def lib():
    return load()


def _check(rc: int):
    if rc != COLI_OK:
        raise ColiError(rc, lib().coli_last_error().decode(errors="replace"))


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


# ---------------------------------------------------------------------------
# data structures


def make_config(hidden, inter, n_experts, top_k, n_shared=1, shared_inter=None, norm_topk_prob=True,
                routed_scaling_factor=2.5, weight_bits=4) -> MoeConfig:
    return MoeConfig(hidden, inter, n_experts, top_k, n_shared,
                     inter if shared_inter is None else shared_inter, int(bool(norm_topk_prob)),
                     float(routed_scaling_factor), int(weight_bits))


@dataclass
class QExpert:
    """One expert's weights (torch CUDA tensors, row-major [out x in]): packed
    int4 rows of in/2 bytes, or int8 rows of `in` bytes (weight_bits 8)."""
    gate_q: object
    gate_s: object
    up_q: object
    up_s: object
    down_q: object
    down_s: object

    def cstruct(self) -> Expert:
        return Expert(*(t.data_ptr() for t in (self.gate_q, self.gate_s, self.up_q, self.up_s,
                                              self.down_q, self.down_s)))


@dataclass
class MoeLayer:
    """One MoE layer resident in HBM: router (F32), bias, experts, shared
    experts, and optionally its streaming copy (``prepare``)."""
    cfg: MoeConfig
    w_router: object
    bias: object
    experts: list
    shared: list
    prepared: object = None
    _keep: list = field(default_factory=list, repr=False)

    def cstruct(self, use_prepared: bool = True) -> MoeLayerC:
        ex = (Expert * len(self.experts))(*[e.cstruct() for e in self.experts])
        sh = (Expert * max(1, len(self.shared)))(*[e.cstruct() for e in self.shared])
        self._keep = [ex, sh]
        prep = self.prepared.data_ptr() if (use_prepared and self.prepared is not None) else None
        return MoeLayerC(self.cfg, self.w_router.data_ptr(), self.bias.data_ptr(),
                         C.cast(ex, C.POINTER(Expert)), C.cast(sh, C.POINTER(Expert)), prep)


# ---------------------------------------------------------------------------
# entry points


def quantize_rows_int4(w, q_out=None, s_out=None, stream=None):
    import torch
    rows, cols = w.shape
    q = torch.empty(rows, cols // 2, dtype=torch.uint8, device=w.device) if q_out is None else q_out
    s = torch.empty(rows, dtype=torch.float32, device=w.device) if s_out is None else s_out
    _check(lib().coli_quantize_rows_int4(_ptr(w), rows, cols, _ptr(q), _ptr(s), _stream(stream)))
    return q, s


def quantize_rows_int8(w, q_out=None, s_out=None, stream=None):
    """Per-row int8 weights: (q int8 [rows x cols], scale F32 [rows])."""
    import torch
    rows, cols = w.shape
    q = torch.empty(rows, cols, dtype=torch.int8, device=w.device) if q_out is None else q_out
    s = torch.empty(rows, dtype=torch.float32, device=w.device) if s_out is None else s_out
    _check(lib().coli_quantize_rows_int8(_ptr(w), rows, cols, _ptr(q), _ptr(s), _stream(stream)))
    return q, s


def requantize_fp8_int4(w8, block_factors, block: int = 128, stream=None):
    """FP8 e4m3 codes (uint8 [rows x cols], device) with per-tile F32
    factors -> (packed int4 [rows x cols/2] uint8, row scales [rows] F32)."""
    import torch
    rows, cols = w8.shape
    q = torch.empty(rows, cols // 2, dtype=torch.uint8, device=w8.device)
    s = torch.empty(rows, dtype=torch.float32, device=w8.device)
    _check(lib().coli_requantize_fp8_int4(_ptr(w8), _ptr(block_factors), rows, cols, int(block), _ptr(q), _ptr(s),
                                          _stream(stream)))
    return q, s


def quantize_act_q8(x, stream=None):
    import torch
    n, dim = x.shape
    q = torch.empty(n, dim, dtype=torch.int8, device=x.device)
    d = torch.empty(n, dim // 32, dtype=torch.float32, device=x.device)
    _check(lib().coli_quantize_act_q8(_ptr(x), n, dim, _ptr(q), _ptr(d), _stream(stream)))
    return q, d


def moe_route(layer: MoeLayer, x, stream=None, with_scores: bool = True):
    """(scores, idx, w); with_scores=False passes no scores buffer (the
    library keeps them on chip) and returns scores=None."""
    import torch
    T = x.shape[0]
    E, K = layer.cfg.n_experts, layer.cfg.top_k
    scores = torch.empty(T, E, dtype=torch.float32, device=x.device) if with_scores else None
    idx = torch.empty(T, K, dtype=torch.int32, device=x.device)
    w = torch.empty(T, K, dtype=torch.float32, device=x.device)
    Lc = layer.cstruct()
    _check(lib().coli_moe_route(C.byref(Lc), _ptr(x), T, _ptr(scores), _ptr(idx), _ptr(w),
                                _stream(stream)))
    return scores, idx, w


def moe_bucket(idx, n_experts: int, stream=None):
    import torch
    T, K = idx.shape
    counts = torch.empty(n_experts, dtype=torch.int32, device=idx.device)
    offsets = torch.empty(n_experts + 1, dtype=torch.int32, device=idx.device)
    perm = torch.empty(max(T * K, 4), dtype=torch.int32, device=idx.device)
    _check(lib().coli_moe_bucket(_ptr(idx) if T else None, T, K, n_experts, _ptr(counts),
                                 _ptr(offsets), _ptr(perm), _stream(stream)))
    return counts, offsets, perm[:T * K]


def prepared_bytes(cfg: MoeConfig) -> int:
    return int(lib().coli_moe_prepared_bytes(C.byref(cfg)))


def prepare(layer: MoeLayer, stream=None):
    """Make the layer's streaming copy (coli_moe_prepare) in a new device
    buffer and attach it to the layer (layer.prepared); returns the buffer."""
    import torch
    n = prepared_bytes(layer.cfg)
    if n == 0:
        raise ColiError(COLI_EINVAL, "this shape has no streaming layout")
    dev = layer.w_router.device
    buf = torch.empty(n + 256, dtype=torch.uint8, device=dev)
    off = (-buf.data_ptr()) % 256
    view = buf[off:off + n]
    Lc = layer.cstruct(use_prepared=False)
    _check(lib().coli_moe_prepare(C.byref(Lc), _ptr(view), n, _stream(stream)))
    layer.prepared = view
    layer._prep_storage = buf
    return view


def workspace_bytes(cfg: MoeConfig, max_tokens: int) -> int:
    return int(lib().coli_moe_workspace_bytes(C.byref(cfg), max_tokens))


def make_workspace(cfg: MoeConfig, max_tokens: int, device="cuda"):
    import torch
    n = workspace_bytes(cfg, max_tokens)
    if n == 0:
        raise ColiError(COLI_EINVAL, "invalid config for a workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_expert_ffn(cfg: MoeConfig, expert: QExpert, xq, xd, workspace=None, stream=None):
    import torch
    T, H = xq.shape
    y = torch.empty(T, H, dtype=torch.float32, device=xq.device)
    ws = make_workspace(cfg, T, xq.device) if workspace is None else workspace
    e = expert.cstruct()
    _check(lib().coli_moe_expert_ffn(C.byref(cfg), C.byref(e), _ptr(xq), _ptr(xd), T, _ptr(y),
                                     _ptr(ws), ws.numel(), _stream(stream)))
    return y


def moe_layer_forward(layer: MoeLayer, x, out=None, workspace=None, stream=None, cstruct=None):
    import torch
    T = x.shape[0]
    o = torch.empty_like(x) if out is None else out
    ws = make_workspace(layer.cfg, T, x.device) if workspace is None else workspace
    Lc = layer.cstruct() if cstruct is None else cstruct
    _check(lib().coli_moe_layer_forward(C.byref(Lc), _ptr(x), T, _ptr(o), _ptr(ws), ws.numel(),
                                        _stream(stream)))
    return o


def stack_cstructs(layers):
    arr = (MoeLayerC * len(layers))(*[l.cstruct() for l in layers])
    return arr


def moe_stack_forward(layers, x, eps: float = 1e-5, out=None, workspace=None, stream=None, carr=None):
    import torch
    T = x.shape[0]
    o = torch.empty_like(x) if out is None else out
    ws = make_workspace(layers[0].cfg, T, x.device) if workspace is None else workspace
    arr = stack_cstructs(layers) if carr is None else carr
    _check(lib().coli_moe_stack_forward(arr, len(layers), _ptr(x), T, float(eps), _ptr(o), _ptr(ws),
                                        ws.numel(), _stream(stream)))
    return o


def rmsnorm(x, eps: float = 1e-5, stream=None):
    import torch
    y = torch.empty_like(x)
    _check(lib().coli_rmsnorm(_ptr(x), x.shape[0], x.shape[1], float(eps), _ptr(y), _stream(stream)))
    return y


def debug_block_partials(expert: QExpert, which: int, xq, rows: int, stream=None):
    import torch
    T, dim_in = xq.shape
    out = torch.empty(T, rows, dim_in // 32, dtype=torch.int32, device=xq.device)
    e = expert.cstruct()
    _check(lib().coli_debug_block_partials(C.byref(e), which, _ptr(xq), T, dim_in, rows, _ptr(out),
                                           _stream(stream)))
    return out


def capture_partials(layer: MoeLayer, x, cstruct=None, stream=None):
    """Run one layer forward with the partials capture armed; returns
    (out, isum) with isum [T, K+S, P] int32 (coli_debug_capture_partials)."""
    import torch
    c = layer.cfg
    H, I, K, S = c.hidden, c.inter, c.top_k, c.n_shared
    P = 2 * I * (H // 32) + H * (I // 32)
    T = x.shape[0]
    buf = torch.full((T, K + S, P), -(2 ** 31), dtype=torch.int32, device=x.device)
    _check(lib().coli_debug_capture_partials(_ptr(buf), buf.numel()))
    out = moe_layer_forward(layer, x, cstruct=cstruct, stream=stream)
    return out, buf


def arm_phase_events(before_experts=None, after_gateup=None, after_down=None):
    """Arm torch.cuda.Event objects that the next layer forward on this
    thread records around its expert kernels (profiling hook)."""
    h = lambda e: None if e is None else C.c_void_p(e if isinstance(e, int) else e.cuda_event)
    _check(lib().coli_debug_phase_events(h(before_experts), h(after_gateup), h(after_down)))


def moe_layer_forward_noalloc(layer: MoeLayer, x, out=None, stream=None, cstruct=None):
    """Layer forward with the library's fixed internal scratch (no workspace,
    no device allocation by the library); see coli_moe_layer_forward_noalloc."""
    import torch
    o = torch.empty_like(x) if out is None else out
    Lc = layer.cstruct() if cstruct is None else cstruct
    _check(lib().coli_moe_layer_forward_noalloc(C.byref(Lc), _ptr(x), x.shape[0], _ptr(o), _stream(stream)))
    return o


def sync_status(workspace=None, stream=None) -> int:
    """Synchronise `stream` and return the coli_status of the device-side
    status word of `workspace` (None: the no-allocation scratch); the
    message is in coli_last_error()."""
    return lib().coli_sync_status(_ptr(workspace), _stream(stream))


def debug_wait_probe(workspace, cycles: int, stream=None):
    """Enqueue the bounded-wait test probe (records status code 30)."""
    _check(lib().coli_debug_wait_probe(_ptr(workspace), int(cycles), _stream(stream)))
