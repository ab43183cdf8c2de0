"""Seeded synthetic inputs for the MoE layer (weights, router, bias, tokens).

The generators are the only code that the oracle side and the CUDA side
share: this package holds none of the method's arithmetic.  Host numbers come
from ``synth_host.c`` (numpy arrays); device numbers from ``synth_dev.cu``
(filled into torch CUDA tensors).  Both implement the definition written at
the top of ``synth_host.c`` and give the same bits for the same element.

Workloads (the GLM-5.2 MoE shape: hidden 6144, expert inter 2048, 256 routed
experts + 1 shared, top-8, from "GLM-5.2-colibri-int4架构解析…", section
"GLM-5.2的MoE实现"):

* ``tiny``        hidden 256, inter 128, 16 experts, top-4, 1 shared, 8 tokens;
* ``mid``         hidden 512, inter 1024, 16 experts, top-4, 1 shared, 4 tokens
                  (rows that span whole 256-byte stages, as in the GLM shape);
                  x ~ N(0,1), W_r ~ N(0,0.02), bias ~ U(-0.1,0.1),
                  experts ~ N(0,0.02); norm_topk_prob, routed_scaling_factor 2.5.
* ``decode1``     GLM shape, 1 token; W_r ~ N(0,0.006), bias ~ U(-0.05,0.05),
                  experts ~ N(0,0.01), x ~ N(0,1).
* ``decode4`` / ``decode16``  GLM shape, 4 / 16 tokens, x_t = base + 0.5*N(0,1)
                  with one base ~ N(0,1) per batch (tokens share experts).
* ``prefill2048`` GLM shape, 2048 tokens, x ~ N(0,1), bias[0:32] += 0.2.
* ``stack8``      8 GLM-shaped layers (layer index 0..7 in the generator key),
                  RMSNorm (eps 1e-5) + residual between layers; 1 or 512 tokens.

"N(0, s)" always means the Irwin-Hall-12 generator of ``synth_host.c``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SRC = os.path.join(HERE, "synth_host.c")
HOST_LIB = os.path.join(HERE, "libsynth_host.so")
DEV_SRC = os.path.join(HERE, "synth_dev.cu")
DEV_LIB = os.path.join(HERE, "libsynth_dev.so")

# tensor ids in the generator key
TID_ROUTER = 1
TID_BIAS = 2
TID_X = 3
TID_X_BASE = 4
TID_FP8_CODES = 5
TID_FP8_SCALES = 6
_E_MAX = 4096
GATE, UP, DOWN = 0, 1, 2


def tid_expert(e: int, m: int) -> int:
    return 16 + 3 * e + m


def tid_shared(s: int, m: int) -> int:
    return 16 + 3 * _E_MAX + 3 * s + m


_GLM = dict(hidden=6144, inter=2048, n_experts=256, top_k=8, n_shared=1, shared_inter=2048,
            norm_topk_prob=True, routed_scaling_factor=2.5, sigma_router=0.006,
            bias_lo=-0.05, bias_hi=0.05, sigma_expert=0.01, x_kind="normal",
            bias_boost_n=0, bias_boost=0.0, n_layers=1, seed=0, weight_bits=4)

CONFIGS = {
    "tiny": dict(_GLM, hidden=256, inter=128, n_experts=16, top_k=4, shared_inter=128,
                 sigma_router=0.02, bias_lo=-0.1, bias_hi=0.1, sigma_expert=0.02, n_tok=8),
    "mid": dict(_GLM, hidden=512, inter=1024, n_experts=16, top_k=4, shared_inter=1024,
                sigma_router=0.02, bias_lo=-0.1, bias_hi=0.1, sigma_expert=0.02, n_tok=4),
    "decode1": dict(_GLM, n_tok=1),
    "decode4": dict(_GLM, n_tok=4, x_kind="base+0.5n"),
    "decode16": dict(_GLM, n_tok=16, x_kind="base+0.5n"),
    "prefill2048": dict(_GLM, n_tok=2048, bias_boost_n=32, bias_boost=0.2),
    "stack8": dict(_GLM, n_tok=1, n_layers=8, rms_eps=1e-5),
    "stack8_512": dict(_GLM, n_tok=512, n_layers=8, rms_eps=1e-5),
    "decode1_int8": dict(_GLM, n_tok=1, weight_bits=8),
}


def config(name: str, **over) -> dict:
    c = dict(CONFIGS[name])
    c.update(over)
    c["name"] = name
    return c


def _build_host(force=False):
    if force or not os.path.exists(HOST_LIB) or os.path.getmtime(HOST_LIB) < os.path.getmtime(HOST_SRC):
        tmp = HOST_LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-fopenmp", "-fPIC", "-shared", "-fvisibility=hidden", HOST_SRC,
                               "-o", tmp])
        os.replace(tmp, HOST_LIB)


def _build_dev(force=False):
    if force or not os.path.exists(DEV_LIB) or os.path.getmtime(DEV_LIB) < os.path.getmtime(DEV_SRC):
        tmp = DEV_LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
                               "-lineinfo", "-fmad=false", "-Xcompiler", "-fPIC", "-shared",
                               DEV_SRC, "-o", tmp])
        os.replace(tmp, DEV_LIB)


def build(force: bool = False) -> None:
    _build_host(force)
    _build_dev(force)


_hl = None
_dl = None


def _host():
    global _hl
    if _hl is None:
        _build_host()
        L = C.CDLL(HOST_LIB)
        u64, i64, f32, vp = C.c_uint64, C.c_int64, C.c_float, C.c_void_p
        L.synth_key.restype = u64
        L.synth_key.argtypes = [u64, C.c_uint32, C.c_uint32]
        L.synth_draw.restype = u64
        L.synth_draw.argtypes = [u64, u64]
        L.synth_normal.restype = None
        L.synth_normal.argtypes = [vp, i64, u64, u64, f32]
        L.synth_uniform.restype = None
        L.synth_uniform.argtypes = [vp, i64, u64, u64, f32, f32]
        L.synth_normal_rows.restype = None
        L.synth_normal_rows.argtypes = [vp, vp, i64, i64, u64, f32]
        _hl = L
    return _hl


def _dev():
    global _dl
    if _dl is None:
        _build_dev()
        L = C.CDLL(DEV_LIB)
        u64, i64, f32, vp = C.c_uint64, C.c_int64, C.c_float, C.c_void_p
        L.synth_dev_normal.restype = C.c_int
        L.synth_dev_normal.argtypes = [vp, i64, u64, u64, f32, vp]
        L.synth_dev_uniform.restype = C.c_int
        L.synth_dev_uniform.argtypes = [vp, i64, u64, u64, f32, f32, vp]
        L.synth_dev_add_range.restype = C.c_int
        L.synth_dev_add_range.argtypes = [vp, i64, f32, vp]
        L.synth_dev_axpy_base.restype = C.c_int
        L.synth_dev_axpy_base.argtypes = [vp, vp, i64, i64, f32, vp]
        _dl = L
    return _dl


def key(seed: int, layer: int, tid: int) -> int:
    return _host().synth_key(seed, layer, tid)


def draw(k: int, c: int) -> int:
    return _host().synth_draw(k, c)


# ---------------------------------------------------------------------------
# host (numpy)

def normal(n: int, seed: int, layer: int, tid: int, sigma: float, i0: int = 0) -> np.ndarray:
    out = np.empty(n, np.float32)
    _host().synth_normal(out.ctypes.data, n, i0, key(seed, layer, tid), sigma)
    return out


def uniform(n: int, seed: int, layer: int, tid: int, a: float, b: float, i0: int = 0) -> np.ndarray:
    out = np.empty(n, np.float32)
    _host().synth_uniform(out.ctypes.data, n, i0, key(seed, layer, tid), a, b)
    return out


def fp8_blocks(rows: int, cols: int, block: int = 128, seed: int = 0, lo: float = 1e-4, hi: float = 1e-2):
    """Synthetic FP8 weights for the FP8 -> int4 converter: e4m3 byte codes
    uniform over all 256 codes (NaN codes included) and one F32 factor per
    block x block tile, uniform in [lo, hi) (the scale range of DeepSeek-V3
    style FP8 checkpoints).  Returns (codes uint8 [rows x cols], factors
    [ceil(rows/block) x ceil(cols/block)])."""
    codes = np.floor(uniform(rows * cols, seed, 0, TID_FP8_CODES, 0.0, 256.0)).astype(np.uint8)
    nb = (-(-rows // block), -(-cols // block))
    scales = uniform(nb[0] * nb[1], seed, 0, TID_FP8_SCALES, lo, hi)
    return codes.reshape(rows, cols), scales.reshape(nb)


def normal_rows(rows, cols: int, seed: int, layer: int, tid: int, sigma: float) -> np.ndarray:
    rows = np.ascontiguousarray(rows, np.int64)
    out = np.empty((rows.size, cols), np.float32)
    _host().synth_normal_rows(out.ctypes.data, rows.ctypes.data, rows.size, cols,
                              key(seed, layer, tid), sigma)
    return out


def router_w(cfg: dict, layer: int = 0) -> np.ndarray:
    E, H = cfg["n_experts"], cfg["hidden"]
    return normal(E * H, cfg["seed"], layer, TID_ROUTER, cfg["sigma_router"]).reshape(E, H)


def bias(cfg: dict, layer: int = 0) -> np.ndarray:
    b = uniform(cfg["n_experts"], cfg["seed"], layer, TID_BIAS, cfg["bias_lo"], cfg["bias_hi"])
    nb = cfg.get("bias_boost_n", 0)
    if nb:
        # binary32 add, the same operation the device generator performs
        b[:nb] = (b[:nb] + np.float32(cfg["bias_boost"])).astype(np.float32)
    return b


def tokens(cfg: dict, n_tok: int | None = None) -> np.ndarray:
    """The layer-0 input x [n_tok, hidden]."""
    T = cfg["n_tok"] if n_tok is None else n_tok
    H = cfg["hidden"]
    n = normal(T * H, cfg["seed"], 0, TID_X, 1.0).reshape(T, H)
    if cfg["x_kind"] == "normal":
        return n
    base = normal(H, cfg["seed"], 0, TID_X_BASE, 1.0)
    half = (np.float32(0.5) * n).astype(np.float32)
    return (base[None, :] + half).astype(np.float32)


def expert_shape(cfg: dict, m: int, shared: bool = False):
    inter = cfg["shared_inter"] if shared else cfg["inter"]
    return (cfg["hidden"], inter) if m == DOWN else (inter, cfg["hidden"])


def expert_matrix(cfg: dict, layer: int, e: int, m: int, shared: bool = False) -> np.ndarray:
    """F32 weights of routed expert e (or shared expert e) matrix m in {GATE, UP, DOWN}."""
    rows, cols = expert_shape(cfg, m, shared)
    tid = tid_shared(e, m) if shared else tid_expert(e, m)
    return normal(rows * cols, cfg["seed"], layer, tid, cfg["sigma_expert"]).reshape(rows, cols)


def expert_rows(cfg: dict, layer: int, e: int, m: int, rows, shared: bool = False) -> np.ndarray:
    _, cols = expert_shape(cfg, m, shared)
    tid = tid_shared(e, m) if shared else tid_expert(e, m)
    return normal_rows(rows, cols, cfg["seed"], layer, tid, cfg["sigma_expert"])


# ---------------------------------------------------------------------------
# device (torch CUDA tensors); the stream is torch's current stream

def _stream():
    import torch
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"synth device generator failed in {what} (cudaError {rc})")


def dev_normal(out, seed: int, layer: int, tid: int, sigma: float, i0: int = 0):
    _check(_dev().synth_dev_normal(out.data_ptr(), out.numel(), i0, key(seed, layer, tid), sigma,
                                   _stream()), "normal")
    return out


def dev_uniform(out, seed: int, layer: int, tid: int, a: float, b: float, i0: int = 0):
    _check(_dev().synth_dev_uniform(out.data_ptr(), out.numel(), i0, key(seed, layer, tid), a, b,
                                    _stream()), "uniform")
    return out


def dev_router_w(cfg: dict, layer: int = 0, device="cuda"):
    import torch
    out = torch.empty(cfg["n_experts"], cfg["hidden"], dtype=torch.float32, device=device)
    return dev_normal(out, cfg["seed"], layer, TID_ROUTER, cfg["sigma_router"])


def dev_bias(cfg: dict, layer: int = 0, device="cuda"):
    import torch
    out = torch.empty(cfg["n_experts"], dtype=torch.float32, device=device)
    dev_uniform(out, cfg["seed"], layer, TID_BIAS, cfg["bias_lo"], cfg["bias_hi"])
    nb = min(cfg.get("bias_boost_n", 0), cfg["n_experts"])
    if nb:
        _check(_dev().synth_dev_add_range(out.data_ptr(), nb, cfg["bias_boost"], _stream()), "add")
    return out


def dev_tokens(cfg: dict, n_tok: int | None = None, device="cuda"):
    import torch
    T = cfg["n_tok"] if n_tok is None else n_tok
    H = cfg["hidden"]
    x = torch.empty(T, H, dtype=torch.float32, device=device)
    dev_normal(x, cfg["seed"], 0, TID_X, 1.0)
    if cfg["x_kind"] != "normal":
        base = torch.empty(H, dtype=torch.float32, device=device)
        dev_normal(base, cfg["seed"], 0, TID_X_BASE, 1.0)
        _check(_dev().synth_dev_axpy_base(x.data_ptr(), base.data_ptr(), T, H, 0.5, _stream()),
               "axpy")
    return x


def dev_expert_matrix(out, cfg: dict, layer: int, e: int, m: int, shared: bool = False):
    tid = tid_shared(e, m) if shared else tid_expert(e, m)
    return dev_normal(out, cfg["seed"], layer, tid, cfg["sigma_expert"])
