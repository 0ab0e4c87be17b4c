"""fp64 CPU oracle for the selective scan (S6) -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline /
reference legs may import this package.  It shares no code with the CUDA
library in ``selective_state_space_50_b200`` and never touches a GPU.

The arithmetic lives in ``ssm_oracle.c`` (plain sequential C in double
precision, OpenMP over (batch, channel) pairs); this module compiles it with
gcc and wraps it with ctypes over numpy float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "libssm_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compiles ssm_oracle.c into libssm_oracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC",
                               "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.c_void_p
        i = ctypes.c_int
        lib.ssm_oracle_fwd.argtypes = [i, i, i, i] + [dp] * 8 + [i, i, dp, dp, dp, i]
        lib.ssm_oracle_fwd.restype = i
        lib.ssm_oracle_bwd.argtypes = [i, i, i, i] + [dp] * 8 + [i] + [dp] * 9 + [i, i]
        lib.ssm_oracle_bwd.restype = i
        lib.ssm_oracle_max_threads.restype = i
        _lib = lib
    return _lib


def _p(x: Optional[np.ndarray]):
    if x is None:
        return None
    assert x.dtype == np.float64 and x.flags.c_contiguous
    return x.ctypes.data


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def max_threads() -> int:
    return int(_load().ssm_oracle_max_threads())


def fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
        zoh=False, h0=None, nthreads: int = 0):
    """Returns (out [b,d,L], last_state [b,d,N]) in float64."""
    u, delta, A, B, C = map(_f64, (u, delta, A, B, C))
    D, z, delta_bias, h0 = map(_f64, (D, z, delta_bias, h0))
    batch, dim, L = u.shape
    N = A.shape[1]
    assert delta.shape == u.shape and A.shape == (dim, N)
    assert B.shape == (batch, N, L) and C.shape == (batch, N, L)
    out = np.empty_like(u)
    last = np.empty((batch, dim, N))
    rc = _load().ssm_oracle_fwd(batch, dim, L, N, _p(u), _p(delta), _p(A), _p(B), _p(C),
                                _p(D), _p(z), _p(delta_bias), int(bool(delta_softplus)),
                                int(bool(zoh)), _p(h0), _p(out), _p(last), int(nthreads))
    assert rc == 0
    return out, last


def step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
         zoh=False):
    """One step of the recurrence from `state` ([b,d,N]): u, delta, z are
    [b,d], B, C [b,N].  It is the forward over a single time step started
    from h0 = state.  Returns (out [b,d], new_state [b,d,N]) in float64."""
    u, delta, B, C = (np.asarray(x, dtype=np.float64) for x in (u, delta, B, C))
    out, last = fwd(u[..., None], delta[..., None], A, B[..., None], C[..., None], D,
                    None if z is None else np.asarray(z, dtype=np.float64)[..., None],
                    delta_bias, delta_softplus, zoh=zoh, h0=state)
    return out[..., 0], last


def bwd(u, delta, A, B, C, D, z, delta_bias, delta_softplus, dout, zoh=False,
        nthreads: int = 0) -> Dict[str, np.ndarray]:
    """Returns a dict of float64 gradients: du, ddelta, dA, dB, dC and, where the
    matching input is given, dD, dz, ddelta_bias."""
    u, delta, A, B, C, dout = map(_f64, (u, delta, A, B, C, dout))
    D, z, delta_bias = map(_f64, (D, z, delta_bias))
    batch, dim, L = u.shape
    N = A.shape[1]
    g = {"du": np.empty_like(u), "ddelta": np.empty_like(u), "dA": np.empty((dim, N)),
         "dB": np.empty((batch, N, L)), "dC": np.empty((batch, N, L))}
    g["dD"] = np.empty(dim) if D is not None else None
    g["dz"] = np.empty_like(u) if z is not None else None
    g["ddelta_bias"] = np.empty(dim) if delta_bias is not None else None
    rc = _load().ssm_oracle_bwd(batch, dim, L, N, _p(u), _p(delta), _p(A), _p(B), _p(C),
                                _p(D), _p(z), _p(delta_bias), int(bool(delta_softplus)),
                                _p(dout), _p(g["du"]), _p(g["ddelta"]), _p(g["dA"]),
                                _p(g["dB"]), _p(g["dC"]), _p(g["dD"]), _p(g["dz"]),
                                _p(g["ddelta_bias"]), int(bool(zoh)), int(nthreads))
    if rc != 0:
        raise MemoryError("oracle bwd: allocation failed")
    return {k: v for k, v in g.items() if v is not None}


def fwd_workload(inputs: Dict[str, np.ndarray], w, nthreads: int = 0):
    """Runs fwd on the fp64 values of a generated workload dict."""
    return fwd(inputs["u_f64"], inputs["delta_f64"], inputs["A_f64"], inputs["B_f64"],
               inputs["C_f64"], inputs["D_f64"] if w.has_D else None,
               inputs["z_f64"] if w.has_z else None,
               inputs["delta_bias_f64"] if w.has_bias else None, w.softplus,
               nthreads=nthreads)


def bwd_workload(inputs: Dict[str, np.ndarray], w, nthreads: int = 0):
    return bwd(inputs["u_f64"], inputs["delta_f64"], inputs["A_f64"], inputs["B_f64"],
               inputs["C_f64"], inputs["D_f64"] if w.has_D else None,
               inputs["z_f64"] if w.has_z else None,
               inputs["delta_bias_f64"] if w.has_bias else None, w.softplus,
               inputs["dout_f64"], nthreads=nthreads)


# ------------------------------------------------------------------ selection projections
# The selection mechanism makes B, C and the step size functions of the input
# (Mamba paper review on booiljung.github.io, "3.2 선택적 스캔(Selective Scan)
# 알고리즘", §1.2: B_t = Linear_N(x_t), C_t = Linear_N(x_t),
# Δ_t = Softplus(Parameter + Linear_1(x_t)); honbul.tistory.com, "Mamba" §2:
# B_t = s_B(x_t), C_t = s_C(x_t), Δ_t = softplus(Δ + s_Δ(x_t))).  The step-size
# projection is taken as a rank-R factorisation Linear_D(Linear_R(x)): R = 1
# with an all-ones up-projection is the pages' Broadcast_D(Linear_1(x)).  The
# Parameter (the per-channel bias) and the softplus stay in the scan.

def bf16_round(v) -> np.ndarray:
    """Round-to-nearest-even to bfloat16 of float64 values (through float32,
    as an fp32 accumulator would be stored), returned as float64."""
    f = np.ascontiguousarray(v, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    r = ((bits + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    out = r.astype(np.uint32).view(np.float32).astype(np.float64)
    # NaN/Inf inputs keep their class (the rounding above would not carry them)
    special = ~np.isfinite(f)
    out[special] = f[special]
    return out


def projections(x, W_x, W_dt, dt_rank: int, dstate: int, store_low_bf16: bool = True):
    """x [b, D, L]; W_x [R + 2N, D]; W_dt [D, R].

    For every batch row and step t: xdbl_t = W_x x_t (one Linear over the
    channels), split into the low-rank step-size input dt_low_t = xdbl_t[0:R],
    B_t = xdbl_t[R:R+N] and C_t = xdbl_t[R+N:R+2N]; then delta_t = W_dt dt_low_t.
    dt_low is an intermediate stored in bfloat16 before the second Linear
    (store_low_bf16); the second product uses those stored values.

    Returns float64 (dt_low [b,R,L], delta [b,D,L], B [b,N,L], C [b,N,L]),
    unrounded apart from the stored intermediate."""
    x, W_x, W_dt = map(_f64, (x, W_x, W_dt))
    batch, dim, L = x.shape
    R, N = int(dt_rank), int(dstate)
    assert W_x.shape == (R + 2 * N, dim) and W_dt.shape == (dim, R)
    xdbl = np.matmul(W_x[None, :, :], x)                 # [b, R+2N, L]
    dt_low = xdbl[:, :R]
    B = xdbl[:, R:R + N]
    C = xdbl[:, R + N:]
    low = bf16_round(dt_low) if store_low_bf16 else dt_low
    delta = np.matmul(W_dt[None, :, :], low)             # [b, D, L]
    return (np.ascontiguousarray(dt_low), np.ascontiguousarray(delta),
            np.ascontiguousarray(B), np.ascontiguousarray(C))


# ------------------------------------------------------------------ sequence segments
# A sequence split into segments is reassembled from per-segment summaries with
# the associative operator of the two-level scan (booiljung.github.io, "3.2
# 선택적 스캔(Selective Scan) 알고리즘", §2.2: (a_j, b_j) • (a_i, b_i) =
# (a_j a_i, a_j b_i + b_j)).  Segment s, run from a zero state, ends in state
# e_s; its decay product over the segment is prod_t exp(Δ_t A) = exp(A Σ_t Δ_t).

def delta_sums(delta, delta_bias=None, delta_softplus=True) -> np.ndarray:
    """Σ_t Δ_t per (batch, channel) of one segment: [b, D, L] -> [b, D]."""
    r = _f64(delta) + (0.0 if delta_bias is None else _f64(delta_bias)[None, :, None])
    dt = np.logaddexp(0.0, r) if delta_softplus else r
    return dt.sum(axis=2)


def combine_carries(A, dsums, h_ends, h0=None) -> np.ndarray:
    """Exclusive scan of segment summaries in sequence order.

    A [D, N]; dsums [S, b, D]; h_ends [S, b, D, N] (each segment's end state
    from a zero start).  Returns h_in [S, b, D, N], the state entering each
    segment: h_in[0] = h0 (zero if None), h_in[s+1] = exp(A dsums[s]) h_in[s]
    + h_ends[s]."""
    A, dsums, h_ends = map(_f64, (A, dsums, h_ends))
    S = dsums.shape[0]
    out = np.empty_like(h_ends)
    h = np.zeros_like(h_ends[0]) if h0 is None else _f64(h0).copy()
    for s in range(S):
        out[s] = h
        decay = np.exp(dsums[s][:, :, None] * A[None, :, :])
        h = decay * h + h_ends[s]
    return out
