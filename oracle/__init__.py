"""The oracle: a plain single-threaded C implementation of one MoE layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library (``int4_weight_only_sigmoid_b200``) never imports
it and shares no code with it.

This module is argument marshalling only: every number is computed by
``coli_oracle.c`` (numpy arrays in, numpy arrays out).  ``build()`` compiles
the C source with ``-O2 -ffp-contract=off -fno-fast-math`` so that each float
expression there is exactly one IEEE binary32 operation.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "coli_oracle.c")
LIB = os.path.join(HERE, "libcoli_oracle.so")

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-fvisibility=hidden", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library (gcc) if it is missing or stale."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB)
        f32, i64, i32, vp = C.c_float, C.c_int64, C.c_int32, C.c_void_p
        for name, res, args in [
            ("ora_exp", f32, [f32]),
            ("ora_sigmoid", f32, [f32]),
            ("ora_silu", f32, [f32]),
            ("ora_exp_n", None, [vp, i64, vp]),
            ("ora_sigmoid_n", None, [vp, i64, vp]),
            ("ora_silu_n", None, [vp, i64, vp]),
            ("ora_pack_int4", None, [vp, i64, vp]),
            ("ora_unpack_int4", None, [vp, i64, vp]),
            ("ora_quantize_rows_int4", None, [vp, i64, i64, vp, vp]),
            ("ora_quantize_rows_int8", None, [vp, i64, i64, vp, vp]),
            ("ora_block_isums_int8", None, [vp, vp, i64, vp]),
            ("ora_quantize_act_q8", None, [vp, i64, i64, vp, vp]),
            ("ora_e4m3_to_f32", f32, [C.c_uint8]),
            ("ora_requantize_fp8_int4", None, [vp, vp, i64, i64, i64, vp, vp]),
            ("ora_router_logit", f32, [vp, vp, i64]),
            ("ora_route", None, [vp, vp, vp, i64, i64, i64, i32, i32, f32, vp, vp, vp]),
            ("ora_bucket", None, [vp, i64, i32, i32, vp, vp, vp]),
            ("ora_block_isums", None, [vp, vp, i64, vp]),
            ("ora_row_dot", f32, [vp, f32, vp, vp, i64]),
            ("ora_expert_ffn_token", None, [vp, i64, i64, vp, vp, vp, vp, vp]),
            ("ora_expert_ffn", None, [vp, i64, i64, vp, vp, i64, vp]),
            ("ora_moe_layer", C.c_int, [vp, vp, i64, vp, vp, vp]),
            ("ora_rmsnorm", None, [vp, i64, i64, f32, vp]),
            ("ora_residual_add", None, [vp, vp, i64, vp]),
        ]:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


class _Expert(C.Structure):
    _fields_ = [("gate_q", C.c_void_p), ("gate_s", C.c_void_p), ("up_q", C.c_void_p),
                ("up_s", C.c_void_p), ("down_q", C.c_void_p), ("down_s", C.c_void_p), ("bits", C.c_int32)]


class _Layer(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("inter", C.c_int32), ("n_experts", C.c_int32),
                ("top_k", C.c_int32), ("n_shared", C.c_int32), ("shared_inter", C.c_int32),
                ("norm_topk_prob", C.c_int32), ("routed_scaling_factor", C.c_float),
                ("w_router", C.c_void_p), ("bias", C.c_void_p), ("experts", C.c_void_p),
                ("shared", C.c_void_p)]


@dataclass
class QExpert:
    """One expert's weights, row-major [out x in]: packed int4 (in/2 bytes
    per row, bits=4) or int8 (in bytes per row, bits=8), one F32 scale per row."""
    gate_q: np.ndarray
    gate_s: np.ndarray
    up_q: np.ndarray
    up_s: np.ndarray
    down_q: np.ndarray
    down_s: np.ndarray
    bits: int = 4

    def _struct(self) -> _Expert:
        return _Expert(_p(self.gate_q), _p(self.gate_s), _p(self.up_q), _p(self.up_s),
                       _p(self.down_q), _p(self.down_s), int(self.bits))


# ---------------------------------------------------------------------------
# scalar functions

def exp(x: float) -> float:
    return lib().ora_exp(float(x))


def sigmoid(x: float) -> float:
    return lib().ora_sigmoid(float(x))


def silu(x: float) -> float:
    return lib().ora_silu(float(x))


def _map(fn, x: np.ndarray) -> np.ndarray:
    x = _f32(x)
    y = np.empty_like(x)
    fn(_p(x), x.size, _p(y))
    return y


def exp_array(x: np.ndarray) -> np.ndarray:
    return _map(lib().ora_exp_n, x)


def sigmoid_array(x: np.ndarray) -> np.ndarray:
    return _map(lib().ora_sigmoid_n, x)


def silu_array(x: np.ndarray) -> np.ndarray:
    return _map(lib().ora_silu_n, x)


# ---------------------------------------------------------------------------
# quantisers

def pack_int4(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    out = np.empty(q.size // 2, np.uint8)
    lib().ora_pack_int4(_p(q), q.size, _p(out))
    return out


def unpack_int4(packed: np.ndarray, n: int | None = None) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n = packed.size * 2 if n is None else n
    out = np.empty(n, np.int8)
    lib().ora_unpack_int4(_p(packed), n, _p(out))
    return out


def quantize_rows_int4(w: np.ndarray):
    w = _f32(w)
    rows, cols = w.shape
    q = np.empty((rows, cols // 2), np.uint8)
    s = np.empty(rows, np.float32)
    lib().ora_quantize_rows_int4(_p(w), rows, cols, _p(q), _p(s))
    return q, s


def quantize_rows_int8(w: np.ndarray):
    """Per-row int8 weights: (q int8 [rows x cols], scale F32 [rows])."""
    w = _f32(w)
    rows, cols = w.shape
    q = np.empty((rows, cols), np.int8)
    s = np.empty(rows, np.float32)
    lib().ora_quantize_rows_int8(_p(w), rows, cols, _p(q), _p(s))
    return q, s


def block_isums_int8(qrow: np.ndarray, xq: np.ndarray) -> np.ndarray:
    qrow = np.ascontiguousarray(qrow, np.int8)
    xq = np.ascontiguousarray(xq, np.int8)
    out = np.empty(len(xq) // 32, np.int32)
    lib().ora_block_isums_int8(_p(qrow), _p(xq), len(xq), _p(out))
    return out


def e4m3_to_f32(codes) -> np.ndarray:
    """Values of e4m3 byte codes (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, np.uint8).ravel()
    return np.array([lib().ora_e4m3_to_f32(int(b)) for b in c], np.float32).reshape(np.shape(codes))


def requantize_fp8_int4(w8: np.ndarray, block_scale: np.ndarray, block: int = 128):
    """FP8 (e4m3 codes, [rows x cols] uint8) with per-block F32 factors
    ([ceil(rows/block) x ceil(cols/block)]) -> packed int4 rows + F32 row
    scales (the converter's flow: dequantise to F32, then int4 per row)."""
    w8 = np.ascontiguousarray(w8, np.uint8)
    rows, cols = w8.shape
    bs = np.ascontiguousarray(block_scale, np.float32)
    assert bs.shape == (-(-rows // block), -(-cols // block))
    q = np.empty((rows, cols // 2), np.uint8)
    s = np.empty(rows, np.float32)
    lib().ora_requantize_fp8_int4(_p(w8), _p(bs), rows, cols, block, _p(q), _p(s))
    return q, s


def quantize_act_q8(x: np.ndarray):
    x = _f32(x)
    if x.ndim == 1:
        x = x[None, :]
    n, dim = x.shape
    q = np.empty((n, dim), np.int8)
    d = np.empty((n, dim // 32), np.float32)
    lib().ora_quantize_act_q8(_p(x), n, dim, _p(q), _p(d))
    return q, d


# ---------------------------------------------------------------------------
# router and bucketing

def router_logit(x: np.ndarray, w: np.ndarray) -> float:
    x, w = _f32(x), _f32(w)
    return lib().ora_router_logit(_p(x), _p(w), x.size)


def route(x, w_router, bias, top_k: int, norm_topk_prob: bool, rsf: float):
    """Returns (scores [T,E], idx [T,K] int32 in rank order, weights [T,K])."""
    x, w_router, bias = _f32(x), _f32(w_router), _f32(bias)
    T, H = x.shape
    E = w_router.shape[0]
    scores = np.empty((T, E), np.float32)
    idx = np.empty((T, top_k), np.int32)
    wts = np.empty((T, top_k), np.float32)
    lib().ora_route(_p(x), _p(w_router), _p(bias), T, E, H, top_k, int(bool(norm_topk_prob)),
                    float(rsf), _p(scores), _p(idx), _p(wts))
    return scores, idx, wts


def bucket(idx: np.ndarray, n_experts: int):
    """Returns (counts [E], offsets [E+1], perm [T*K]) with perm sorted by (expert, token)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    counts = np.empty(n_experts, np.int32)
    offsets = np.empty(n_experts + 1, np.int32)
    perm = np.empty(T * K, np.int32)
    lib().ora_bucket(_p(idx), T, K, n_experts, _p(counts), _p(offsets), _p(perm))
    return counts, offsets, perm


# ---------------------------------------------------------------------------
# integer dots and the expert

def block_isums(qrow: np.ndarray, xq: np.ndarray) -> np.ndarray:
    qrow = np.ascontiguousarray(qrow, np.uint8)
    xq = np.ascontiguousarray(xq, np.int8)
    out = np.empty(xq.size // 32, np.int32)
    lib().ora_block_isums(_p(qrow), _p(xq), xq.size, _p(out))
    return out


def row_dot(qrow, s_w: float, xq, xd) -> float:
    qrow = np.ascontiguousarray(qrow, np.uint8)
    xq = np.ascontiguousarray(xq, np.int8)
    xd = _f32(xd)
    return lib().ora_row_dot(_p(qrow), float(s_w), _p(xq), _p(xd), xq.size)


def expert_ffn_token(ex: QExpert, xq: np.ndarray, xd: np.ndarray):
    """Returns (y [hidden], hq [inter] int8, hd [inter/32]) for one Q8 token."""
    hidden = xq.size
    inter = ex.gate_s.size
    xq = np.ascontiguousarray(xq, np.int8).ravel()
    xd = _f32(xd).ravel()
    y = np.empty(hidden, np.float32)
    hq = np.empty(inter, np.int8)
    hd = np.empty(inter // 32, np.float32)
    s = ex._struct()
    lib().ora_expert_ffn_token(C.addressof(s), hidden, inter, _p(xq), _p(xd), _p(y), _p(hq), _p(hd))
    return y, hq, hd


def expert_ffn(ex: QExpert, xq: np.ndarray, xd: np.ndarray) -> np.ndarray:
    xq = np.ascontiguousarray(xq, np.int8)
    xd = _f32(xd)
    T, hidden = xq.shape
    inter = ex.gate_s.size
    y = np.empty((T, hidden), np.float32)
    s = ex._struct()
    lib().ora_expert_ffn(C.addressof(s), hidden, inter, _p(xq), _p(xd), T, _p(y))
    return y


def moe_layer(cfg: dict, w_router, bias, experts: dict, shared: list, x: np.ndarray):
    """One layer forward.  ``experts`` maps expert id -> QExpert; only the ids
    the routing selects need to be present.  Returns (out, idx, w)."""
    x = _f32(x)
    T, H = x.shape
    E, K = cfg["n_experts"], cfg["top_k"]
    w_router, bias = _f32(w_router), _f32(bias)
    arr = (_Expert * E)()
    for e, ex in experts.items():
        arr[e] = ex._struct()
    n_sh = len(shared)
    sh = (_Expert * max(n_sh, 1))()
    for i, ex in enumerate(shared):
        sh[i] = ex._struct()
    L = _Layer(H, cfg["inter"], E, K, n_sh, cfg.get("shared_inter", cfg["inter"]),
               int(bool(cfg["norm_topk_prob"])), float(cfg["routed_scaling_factor"]),
               _p(w_router), _p(bias), C.addressof(arr), C.addressof(sh))
    out = np.empty((T, H), np.float32)
    idx = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float32)
    rc = lib().ora_moe_layer(C.addressof(L), _p(x), T, _p(out), _p(idx), _p(w))
    if rc != 0:
        raise KeyError("the routing selected an expert that was not supplied")
    return out, idx, w


def rmsnorm(x: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    x = _f32(x)
    T, H = x.shape
    y = np.empty_like(x)
    lib().ora_rmsnorm(_p(x), T, H, float(eps), _p(y))
    return y


def residual_add(x: np.ndarray, m: np.ndarray) -> np.ndarray:
    x, m = _f32(x), _f32(m)
    out = np.empty_like(x)
    lib().ora_residual_add(_p(x), _p(m), x.size, _p(out))
    return out
