"""ctypes view of the C oracle (zo_oracle.c) over numpy arrays.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's CPU-baseline
leg import this package.  See zo_oracle.c for the sources and readings each function
follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        u32, u64, i32, i64 = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_int, ctypes.c_int64
        vp, f32, f64 = ctypes.c_void_p, ctypes.c_float, ctypes.c_double
        L.zo_oracle_philox4x32_10.argtypes = [vp, vp, vp]
        L.zo_oracle_probe_sign.argtypes = [u64, u32, u32, i64]
        L.zo_oracle_probe_sign.restype = i32
        L.zo_oracle_pack_probe.argtypes = [u64, u32, u32, i64, vp]
        L.zo_oracle_perturb_f32.argtypes = [vp, i64, i64, u64, u32, u32, i32, f32, vp]
        L.zo_oracle_perturb_bf16.argtypes = [vp, i64, i64, u64, u32, u32, i32, f32, vp]
        L.zo_oracle_quad_loss.argtypes = [vp, vp, i64]
        L.zo_oracle_quad_loss.restype = f64
        L.zo_oracle_precond.argtypes = [vp, vp, vp, i32, f64, f64, f64, f64, vp, vp, vp, vp]
        L.zo_oracle_precond.restype = i32
        for nm in ("zo_oracle_update_f64_f32", "zo_oracle_update_f64_bf16",
                   "zo_oracle_update_mirror_f32", "zo_oracle_update_mirror_bf16"):
            getattr(L, nm).argtypes = [vp, i64, i64, vp, i32, u64, u32]
        L.zo_oracle_f32_to_bf16.argtypes = [f32]
        L.zo_oracle_f32_to_bf16.restype = ctypes.c_uint16
        _LIB = L
    return _LIB


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def philox4x32_10(ctr, key):
    """One Philox4x32-10 block: 4 uint32 counter words, 2 key words -> 4 words."""
    c = _c(ctr, np.uint32)
    k = _c(key, np.uint32)
    out = np.zeros(4, np.uint32)
    lib().zo_oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def probe_sign(seed, step, probe, j):
    return lib().zo_oracle_probe_sign(seed, step, probe, j)


def pack_probe(seed, step, probe, M):
    out = np.zeros((M + 7) // 8, np.uint8)
    lib().zo_oracle_pack_probe(seed, step, probe, M, _ptr(out))
    return out


def probe_signs(seed, step, probe, M):
    """z_probe as an int8 vector of +/-1 (unpacked from the packed probe)."""
    bits = np.unpackbits(pack_probe(seed, step, probe, M), bitorder="little")[:M]
    return (1 - 2 * bits.astype(np.int8)).astype(np.int8)


def perturb(theta, seed, step, probe, sign, eps, j0=0):
    """P = rd(theta + sign*eps*z_probe); theta is float32 or bf16 bits (uint16) and its
    element k is global parameter j0 + k."""
    M = theta.size
    if theta.dtype == np.float32:
        t = _c(theta, np.float32)
        out = np.empty_like(t)
        lib().zo_oracle_perturb_f32(_ptr(t), j0, M, seed, step, probe, sign, eps, _ptr(out))
    elif theta.dtype == np.uint16:
        t = _c(theta, np.uint16)
        out = np.empty_like(t)
        lib().zo_oracle_perturb_bf16(_ptr(t), j0, M, seed, step, probe, sign, eps, _ptr(out))
    else:
        raise TypeError("theta must be float32 or bf16 bits (uint16)")
    return out


def quad_loss(P, D):
    P = _c(P, np.float32)
    D = _c(D, np.float32)
    return lib().zo_oracle_quad_loss(_ptr(P), _ptr(D), P.size)


def precond(loss_plus, loss_minus, loss0, eps, lr, damping, alpha=0.1):
    """Returns dict(g, c, w, a) in fp64, or None if a loss is not finite."""
    lp = _c(loss_plus, np.float64)
    lm = _c(loss_minus, np.float64)
    n = lp.size
    l0 = None if loss0 is None else np.array([loss0], np.float64)
    g, c, w, a = (np.zeros(n, np.float64) for _ in range(4))
    rc = lib().zo_oracle_precond(_ptr(lp), _ptr(lm), None if l0 is None else _ptr(l0), n,
                                 float(eps), float(lr), float(damping), float(alpha),
                                 _ptr(g), _ptr(c), _ptr(w), _ptr(a))
    if rc != 0:
        return None
    return {"g": g, "c": c, "w": w, "a": a}


def update_f64(theta, a, seed, step, j0=0):
    """theta' = rd(theta - sum_i a_i z_i) with the probe sum in fp64 (new array); element
    k of theta is global parameter j0 + k."""
    a = _c(a, np.float64)
    t = np.array(theta, copy=True)
    if t.dtype == np.float32:
        lib().zo_oracle_update_f64_f32(_ptr(t), j0, t.size, _ptr(a), a.size, seed, step)
    elif t.dtype == np.uint16:
        lib().zo_oracle_update_f64_bf16(_ptr(t), j0, t.size, _ptr(a), a.size, seed, step)
    else:
        raise TypeError("theta must be float32 or bf16 bits (uint16)")
    return t


def update_mirror(theta, a32, seed, step, j0=0):
    """theta' in the fixed fp32 order (groups of 8 probes) from fp32 coefficients;
    element k of theta is global parameter j0 + k."""
    a32 = _c(a32, np.float32)
    t = np.array(theta, copy=True)
    if t.dtype == np.float32:
        lib().zo_oracle_update_mirror_f32(_ptr(t), j0, t.size, _ptr(a32), a32.size, seed, step)
    elif t.dtype == np.uint16:
        lib().zo_oracle_update_mirror_bf16(_ptr(t), j0, t.size, _ptr(a32), a32.size, seed, step)
    else:
        raise TypeError("theta must be float32 or bf16 bits (uint16)")
    return t


def f32_to_bf16(x):
    """Round float32 values to bf16 (RNE) with the oracle's own rounding."""
    x = np.asarray(x, np.float32).ravel()
    L = lib()
    return np.array([L.zo_oracle_f32_to_bf16(float(v)) for v in x], np.uint16)


def bf16_to_f32(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)
