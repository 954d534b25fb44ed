"""CPU oracle for the fused sigmoid-gating Gated DeltaNet decode update.

TEST INFRASTRUCTURE ONLY.  The oracle checks the CUDA path; only the tests,
the smoke check and the benchmark's CPU-baseline leg may import it.  It is a
plain single-threaded C loop nest (``gdn_oracle.c``) evaluated in fp64, with
an fp32 twin used only to size rounding drift.  This module marshals numpy
arrays into it through ctypes; it holds none of the method's arithmetic.

What it computes, and the passages it follows, is stated in ``gdn_oracle.h``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

L2NORM_QK = 1
WRITE_INTERMEDIATE = 2
NO_FINAL_WRITEBACK = 4

BAD_SLOT = 1
BAD_SEQLENS = 2

_LIBS = {}


def _load(path=None):
    """Load the oracle library (building it first when ``path`` is None)."""
    key = path or "default"
    if key not in _LIBS:
        lib = ctypes.CDLL(path or _build.build())
        p = ctypes.c_void_p
        i32 = ctypes.c_int32
        for name in ("gdn_oracle_update", "gdn_oracle_update_f32", "gdn_oracle_update_fin"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [p, p, p, p, p, p, p, p, p, p, p, p,
                           i32, i32, i32, i32, i32, i32, i32, i32,
                           ctypes.c_double, ctypes.c_uint32, p, p, p]
        for name in ("gdn_oracle_gating", "gdn_oracle_gating_f32", "gdn_oracle_gating_fin"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [p, p, p, p, i32, i32, p, p]
        _LIBS[key] = lib
    return _LIBS[key]


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def _c(x, dtype):
    arr = np.ascontiguousarray(x)
    if arr.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {arr.dtype}")
    return arr


def _variant(lib, base, precision, inputs_f32):
    if inputs_f32:
        if precision != "f64":
            raise ValueError("fp32 inputs are supported by the fp64 oracle only")
        return getattr(lib, base + "_fin"), np.float32
    return (getattr(lib, base) if precision == "f64" else getattr(lib, base + "_f32")), np.uint16


def gating(a, b, A_log, dt_bias, *, precision="f64", library=None):
    """g = -exp(A_log) softplus(a + dt_bias) and beta = sigmoid(b), [..., HV]
    each; a, b are uint16 bf16 patterns or float32 values."""
    lib = _load(library)
    inputs_f32 = np.asarray(a).dtype == np.float32
    fn, in_dt = _variant(lib, "gdn_oracle_gating", precision, inputs_f32)
    real = np.float64 if precision == "f64" else np.float32
    HV = np.asarray(a).shape[-1]
    a_ = _c(a, in_dt).reshape(-1, HV)
    b_ = _c(b, in_dt).reshape(-1, HV)
    T_tot = a_.shape[0]
    g = np.empty((T_tot, HV), dtype=real)
    beta = np.empty((T_tot, HV), dtype=real)
    rc = fn(_ptr(a_), _ptr(b_), _ptr(_c(A_log, np.float32)), _ptr(_c(dt_bias, np.float32)), T_tot, HV,
            _ptr(g), _ptr(beta))
    if rc < 0:
        raise ValueError(f"oracle gating rejected its arguments (code {rc})")
    return g, beta


def update(q, k, v, a, b, A_log, dt_bias, state_pool, state_indices,
           cu_seqlens=None, *, scale=None, flags=L2NORM_QK, precision="f64",
           fill=np.nan, library=None, g=None, beta=None):
    """Run the oracle on host arrays.

    q, k: uint16 bf16 patterns (or float32 values), shape [..., H, K] with
    leading dims [T_tot] or [N, T]; v: [..., HV, V]; a, b: [..., HV] (same
    element type as q); A_log, dt_bias: float32 [HV]; state_pool: float32
    [num_slots, HV, K, V]; state_indices: int32 [N]; cu_seqlens: int32 [N+1]
    or None (then q has leading dims [N, T]).  With ``g`` and ``beta``
    (float32, [T_tot, HV]) the gates are taken from them instead (the
    recurrence of the unfused pair); a, b, A_log, dt_bias may then be None.

    Returns ``(status, out, state_out, inter)``: the oracle's status mask,
    out [T_tot, HV, V], the pool after the call [num_slots, HV, K, V] and,
    when WRITE_INTERMEDIATE is set, the per-token states [T_tot, HV, K, V]
    (else None), all in the requested precision.  Rows the oracle does not
    write keep ``fill``.  ``library`` names another build of the same C
    source (the tests use it to run deliberately broken copies).
    """
    real = np.float64 if precision == "f64" else np.float32
    lib = _load(library)
    inputs_f32 = np.asarray(q).dtype == np.float32
    fn, in_dt = _variant(lib, "gdn_oracle_update", precision, inputs_f32)
    given = g is not None or beta is not None

    H, K = q.shape[-2:]
    HV, V = v.shape[-2:]
    state_indices = _c(state_indices, np.int32).reshape(-1)
    N = state_indices.shape[0]
    if cu_seqlens is None:
        if q.ndim != 4:
            raise ValueError("without cu_seqlens q must be [N, T, H, K]")
        T_fixed = q.shape[1]
        T_tot = N * T_fixed
    else:
        cu_seqlens = _c(cu_seqlens, np.int32).reshape(-1)
        T_fixed = -1
        T_tot = int(np.prod(q.shape[:-2]))
    q = _c(q, in_dt).reshape(T_tot, H, K)
    k = _c(k, in_dt).reshape(T_tot, H, K)
    v = _c(v, in_dt).reshape(T_tot, HV, V)
    if given:
        g = _c(g, np.float32).reshape(T_tot, HV)
        beta = _c(beta, np.float32).reshape(T_tot, HV)
        a = b = A_log = dt_bias = None
    else:
        a = _c(a, in_dt).reshape(T_tot, HV)
        b = _c(b, in_dt).reshape(T_tot, HV)
        A_log = _c(A_log, np.float32).reshape(HV)
        dt_bias = _c(dt_bias, np.float32).reshape(HV)
    state_pool = _c(state_pool, np.float32)
    num_slots = state_pool.shape[0]
    if state_pool.shape != (num_slots, HV, K, V):
        raise ValueError(f"state_pool shape {state_pool.shape}")
    if scale is None:
        scale = 1.0 / np.sqrt(K)

    out = np.full((T_tot, HV, V), fill, dtype=real)
    state_out = np.empty((num_slots, HV, K, V), dtype=real)
    inter = None
    if flags & WRITE_INTERMEDIATE:
        inter = np.full((T_tot, HV, K, V), fill, dtype=real)

    status = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(A_log),
                _ptr(dt_bias), _ptr(g), _ptr(beta), _ptr(state_pool), _ptr(state_indices),
                _ptr(cu_seqlens), N, T_fixed, T_tot, H, HV, K, V, num_slots,
                float(scale), int(flags), _ptr(out), _ptr(state_out), _ptr(inter))
    if status < 0:
        raise ValueError(f"oracle rejected its arguments (code {status})")
    return status, out, state_out, inter


def library_path() -> str:
    return os.path.abspath(_build.LIB_PATH)
