"""ctypes binding of oracle/latent_moe_ref.c, the plain-C FP64 reference of the block.

TEST INFRASTRUCTURE ONLY (like the rest of oracle/): the tests, smoke() and bench.py's CPU
baseline may call it. build() compiles the C file with gcc (IEEE double, no contraction of
multiply-adds into fused ones), in place; a missing compiler or library raises.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "latent_moe_ref.c")
LIB = os.path.join(HERE, "liblatent_moe_ref.so")
CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]

_lib: Optional[ctypes.CDLL] = None


class RefNvfp4(ctypes.Structure):
    """One NVFP4 expert tensor [E, out, in]: codes [E, out, in/2] (low nibble = even
    element), E4M3 block scales [E, out, in/16], float32 matrix scales [E]."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("matrix_scale", ctypes.c_void_p)]


class RefCfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("D", ctypes.c_int), ("L", ctypes.c_int), ("I", ctypes.c_int),
                ("E", ctypes.c_int), ("k", ctypes.c_int), ("eps", ctypes.c_double),
                ("router_mode", ctypes.c_int), ("logit_scale", ctypes.c_double),
                ("routed_scaling", ctypes.c_double), ("bias", ctypes.c_void_p), ("norm_mode", ctypes.c_int),
                ("gamma_shared", ctypes.c_int), ("pre_gain", ctypes.c_void_p), ("pre_eps", ctypes.c_double)]


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(["gcc", *CFLAGS, SRC, "-o", LIB + ".tmp", "-lm"], check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        L.ref_latent_moe_forward.argtypes = [ctypes.POINTER(RefCfg)] + [ctypes.c_void_p] * 11
        L.ref_latent_moe_forward.restype = ctypes.c_int
        L.ref_latent_moe_forward_nvfp4.argtypes = [ctypes.POINTER(RefCfg)] + [ctypes.c_void_p] * 11
        L.ref_latent_moe_forward_nvfp4.restype = ctypes.c_int
        L.ref_e2m1_value.argtypes = [ctypes.c_uint]
        L.ref_e2m1_value.restype = ctypes.c_double
        L.ref_e4m3_value.argtypes = [ctypes.c_uint]
        L.ref_e4m3_value.restype = ctypes.c_double
        _lib = L
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def e2m1_value(code: int) -> float:
    return float(lib().ref_e2m1_value(int(code)))


def e4m3_value(byte: int) -> float:
    return float(lib().ref_e4m3_value(int(byte)))


def _u8(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.uint8)


def _f32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().float().numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def latent_moe_forward_c(x, W_router, W_pool, experts, gamma, W_unpool, k: int, eps: float,
                         router_bias=None, router_mode: str = "softmax", logit_scale: float = 1.0,
                         routed_scaling: float = 1.0, norm_mode: str = "centred", pre_norm_gain=None,
                         pre_norm_eps: float = 1e-5, nvfp4: bool = False) -> Dict[str, np.ndarray]:
    """The block on every row of x [T, D]; experts = (W_gate [E, I, L], W_up [E, I, L],
    W_down [E, L, I]), or with nvfp4=True three (codes, block scales, matrix scales) triples
    that the C code decodes itself; gamma [E, L] or [L]. Returns out [T, D], idx [T, k],
    g [T, k]."""
    x, Wr, Wp, Wu_ = _f64(x), _f64(W_router), _f64(W_pool), _f64(W_unpool)
    gam = _f64(gamma)
    T, D = x.shape
    E = Wr.shape[0]
    L = Wp.shape[0]
    keep = []
    if nvfp4:
        mats = []
        for codes, scales, ms in experts:
            c8, s8, m32 = _u8(codes), _u8(scales), _f32(ms)
            assert c8.shape[:2] == s8.shape[:2] and c8.shape[2] * 2 == s8.shape[2] * 16 and m32.shape == (E,)
            keep += [c8, s8, m32]
            mats.append(RefNvfp4(c8.ctypes.data, s8.ctypes.data, m32.ctypes.data))
        I = experts[0][0].shape[1]
        assert tuple(experts[0][0].shape) == (E, I, L // 2) and tuple(experts[2][0].shape) == (E, L, I // 2)
    else:
        Wg, Wup, Wd = (_f64(m) for m in experts)
        I = Wg.shape[1]
        assert Wg.shape == (E, I, L) and Wup.shape == (E, I, L) and Wd.shape == (E, L, I)
    assert Wr.shape == (E, D) and Wp.shape == (L, D) and Wu_.shape == (D, L)
    assert gam.shape in ((E, L), (L,))
    bias = None if router_bias is None else _f64(router_bias)
    pre = None if pre_norm_gain is None else _f64(pre_norm_gain)
    c = RefCfg(T=T, D=D, L=L, I=I, E=E, k=k, eps=eps, router_mode={"softmax": 0, "sigmoid": 1}[router_mode],
               logit_scale=logit_scale, routed_scaling=routed_scaling,
               bias=None if bias is None else bias.ctypes.data,
               norm_mode={"centred": 0, "input_scaled": 1}[norm_mode], gamma_shared=int(gam.ndim == 1),
               pre_gain=None if pre is None else pre.ctypes.data, pre_eps=pre_norm_eps)
    out = np.zeros((T, D))
    idx = np.zeros((T, k), dtype=np.int32)
    g = np.zeros((T, k))
    p = lambda a: a.ctypes.data  # noqa: E731
    if nvfp4:
        rc = lib().ref_latent_moe_forward_nvfp4(ctypes.byref(c), p(x), p(Wr), p(Wp), *[ctypes.addressof(m) for m in mats],
                                                p(gam), p(Wu_), p(out), p(idx), p(g))
    else:
        rc = lib().ref_latent_moe_forward(ctypes.byref(c), p(x), p(Wr), p(Wp), p(Wg), p(Wup), p(Wd), p(gam), p(Wu_),
                                          p(out), p(idx), p(g))
    if rc != 0:
        raise ValueError("the C reference rejected the configuration")
    return {"out": out, "idx": idx.astype(np.int64), "g": g}
