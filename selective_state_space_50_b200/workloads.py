"""Seeded synthetic inputs for the selective scan (S6).

This module is shared by the fp64 oracle tests, the GPU parity tests and the
benchmark. It holds only random-number generation and the workload recipes
(shapes and value distributions); none of the scan's arithmetic lives here.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used counter-style: element i of stream k
is mix(key_k + (i + 1) * GAMMA), where mix is SplitMix64's output function
and key_k = mix(seed * GAMMA + k).  Uniforms take the top 53 bits.  Normals
use the Box-Muller transform (Box & Muller, 1958) on consecutive uniform
pairs, keeping both the cosine and the sine output.

bf16 inputs are produced by rounding the fp64 draw to fp32 and then to bf16
with round-to-nearest-even; the oracle receives exactly those rounded values
promoted to fp64, so both sides see identical inputs.

Tensor layouts (all row-major / C-contiguous):
    u, delta, z, dout : [batch, dim, seqlen]
    B, C              : [batch, dstate, seqlen]   (shared over dim)
    A                 : [dim, dstate]
    D, delta_bias     : [dim]
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import math
import os
from typing import Dict, Optional

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream ids: one independent counter stream per tensor.
STREAMS = {"delta_bias": 1, "D": 2, "A": 3, "u": 4, "delta": 5, "z": 6,
           "B": 7, "C": 8, "dout": 9, "delta0": 10, "x": 11, "W_x": 12, "W_dt": 13}

_CHUNK = 1 << 22  # elements generated per numpy pass (bounds host memory)


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.array([(seed * int(GAMMA) + stream) & (2**64 - 1)], dtype=np.uint64)
        return _mix(s)[0]


def _uniform_block(key: np.uint64, start: int, count: int) -> np.ndarray:
    """Uniforms in [0, 1) for counters start .. start+count-1."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        x = _mix(key + idx * GAMMA)
    return (x >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def _parallel(fn, starts):
    """Runs fn(start) for every chunk start; numpy releases the GIL inside the
    ufuncs, so chunks run concurrently.  Results do not depend on scheduling."""
    if len(starts) <= 1:
        for s in starts:
            fn(s)
        return
    with _cf.ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
        list(ex.map(fn, starts))


def uniform(seed: int, stream: int, n: int, lo: float = 0.0, hi: float = 1.0) -> np.ndarray:
    key = _key(seed, stream)
    out = np.empty(n, dtype=np.float64)

    def fill(s):
        c = min(_CHUNK, n - s)
        out[s:s + c] = lo + (hi - lo) * _uniform_block(key, s, c)
    _parallel(fill, list(range(0, n, _CHUNK)))
    return out


def normal(seed: int, stream: int, n: int, std: float = 1.0) -> np.ndarray:
    """Standard normals by Box-Muller; pair k uses uniforms 2k and 2k+1."""
    key = _key(seed, stream)
    out = np.empty(n, dtype=np.float64)
    npairs = (n + 1) // 2

    def fill(s):
        c = min(_CHUNK, npairs - s)
        uu = _uniform_block(key, 2 * s, 2 * c).reshape(c, 2)
        r = np.sqrt(-2.0 * np.log1p(-uu[:, 0]))  # 1-u1 in (0, 1]
        th = (2.0 * math.pi) * uu[:, 1]
        pair = np.empty((c, 2), dtype=np.float64)
        pair[:, 0] = r * np.cos(th)
        pair[:, 1] = r * np.sin(th)
        flat = pair.reshape(-1)
        lo = 2 * s
        take = min(2 * c, n - lo)
        out[lo:lo + take] = flat[:take] * std
    _parallel(fill, list(range(0, npairs, _CHUNK)))
    return out


# ---------------------------------------------------------------- bf16 rounding

def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 -> bf16 (round to nearest even); returns uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    rounding = np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))
    nan = np.isnan(f)
    out = ((b + rounding) >> np.uint64(16)).astype(np.uint16)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- workloads

@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic selective-scan problem (shape + distributions)."""
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    io_dtype: str            # "f32" or "bf16"
    seed: int
    has_z: bool = True
    has_D: bool = True
    has_bias: bool = True
    softplus: bool = True
    D_dist: str = "ones"     # "ones" | "u0.5_1.5"
    A_dist: str = "neg_n1"   # "neg_n1": A[d,n] = -(n+1); "neg_lognormal": -exp(N(0,1))
    bias_dist: str = "expm1_u"   # "expm1_u": log(expm1(U[1e-3, 0.1])); "long_memory"; "step_u"
    delta_std: float = 1.0
    delta_abs: bool = False  # |N(0, std)| raw deltas (for callers passing Δ without softplus)

    @property
    def elems(self) -> int:
        return self.batch * self.dim * self.seqlen

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# Five workloads: a tiny fp32 case, the Mamba-130M and Mamba-2.8B layer shapes,
# a long-context small-batch case and the fwd+bwd case at the 130M shape.
WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload("tiny_f32", 2, 256, 64, 16, "f32", seed=1000,
                         D_dist="ones"),
    "mamba130m_layer": Workload("mamba130m_layer", 8, 2048, 1536, 16, "bf16",
                                seed=1001, D_dist="u0.5_1.5"),
    "mamba2p8b_layer": Workload("mamba2p8b_layer", 4, 2048, 5120, 16, "bf16",
                                seed=1002, D_dist="u0.5_1.5"),
    "long_context": Workload("long_context", 1, 131072, 2048, 16, "bf16",
                             seed=1003, D_dist="u0.5_1.5",
                             bias_dist="long_memory", delta_std=0.1),
    "mamba130m_layer_fwdbwd": Workload("mamba130m_layer_fwdbwd", 8, 2048, 1536,
                                       16, "bf16", seed=1004, D_dist="u0.5_1.5"),
}


def _cast(x: np.ndarray, io_dtype: str):
    """Returns (device-side array in io dtype, fp64 array of the same values)."""
    if io_dtype == "f32":
        f = x.astype(np.float32)
        return f, f.astype(np.float64)
    bits = round_to_bf16_bits(x)
    return bits, bf16_bits_to_f64(bits)


def generate(w: Workload, with_dout: bool = False,
             channels: Optional[slice] = None) -> Dict[str, np.ndarray]:
    """Draws every input of workload `w`.

    Returns a dict with, for each tensor name, the io-dtype array under
    `name` (float32, or uint16 bf16 bit patterns) and the exact fp64 values
    under `name + "_f64"`.  A, D and delta_bias are always fp32 on the
    device side.  `channels` optionally restricts the per-channel tensors
    (u, delta, z, dout, A, D, delta_bias) to a slice of dim; B and C are
    shared over dim and are always returned whole.
    """
    b, L, Dm, N = w.batch, w.seqlen, w.dim, w.dstate
    out: Dict[str, np.ndarray] = {}

    def put32(name, x):
        f = x.astype(np.float32)
        out[name] = f
        out[name + "_f64"] = f.astype(np.float64)

    # delta_bias
    if w.bias_dist == "step_u":
        # the bias is itself a step size in [1e-3, 0.1] (no softplus applied)
        put32("delta_bias", uniform(w.seed, STREAMS["delta_bias"], Dm, 1e-3, 0.1))
        d0 = None
    elif w.bias_dist == "expm1_u":
        d0 = uniform(w.seed, STREAMS["delta_bias"], Dm, 1e-3, 0.1)
    elif w.bias_dist == "long_memory":
        # log-uniform step size in [1.5e-4, 4.5e-3]
        d0 = np.exp(uniform(w.seed, STREAMS["delta_bias"], Dm,
                            math.log(1.5e-4), math.log(4.5e-3)))
    else:
        raise ValueError(w.bias_dist)
    if d0 is not None:
        put32("delta_bias", np.log(np.expm1(d0)))

    if w.D_dist == "ones":
        put32("D", np.ones(Dm))
    else:
        put32("D", uniform(w.seed, STREAMS["D"], Dm, 0.5, 1.5))

    if w.A_dist == "neg_n1":
        A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (Dm, 1))
    elif w.A_dist == "neg_lognormal":
        A = -np.exp(normal(w.seed, STREAMS["A"], Dm * N)).reshape(Dm, N)
    else:
        raise ValueError(w.A_dist)
    put32("A", A)

    def per_channel(stream, std=1.0):
        x = normal(w.seed, stream, b * Dm * L, std).reshape(b, Dm, L)
        return x

    names = ["u", "delta", "z"] + (["dout"] if with_dout else [])
    for name in names:
        x = per_channel(STREAMS[name], w.delta_std if name == "delta" else 1.0)
        if name == "delta" and w.delta_abs:
            x = np.abs(x)
        dev, f64 = _cast(x, w.io_dtype)
        out[name], out[name + "_f64"] = dev, f64
    for name in ("B", "C"):
        x = normal(w.seed, STREAMS[name], b * N * L).reshape(b, N, L)
        dev, f64 = _cast(x, w.io_dtype)
        out[name], out[name + "_f64"] = dev, f64

    if channels is not None:
        for name in list(out):
            base = name[:-4] if name.endswith("_f64") else name
            if base in ("u", "delta", "z", "dout"):
                out[name] = np.ascontiguousarray(out[name][:, channels, :])
            elif base in ("A", "D", "delta_bias"):
                out[name] = np.ascontiguousarray(out[name][channels])
    return out


def to_torch(inputs: Dict[str, np.ndarray], w: Workload, device):
    """Device tensors (io dtype / fp32) of a generated workload; optional
    inputs the workload leaves out map to None."""
    import torch

    def dev(x):
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(x)).to(device)
    d = {k: dev(inputs[k]) for k in ("u", "delta", "z", "B", "C", "dout", "A", "D", "delta_bias")
         if k in inputs}
    if not w.has_z:
        d["z"] = None
    if not w.has_D:
        d["D"] = None
    if not w.has_bias:
        d["delta_bias"] = None
    return d


# ---------------------------------------------------------------- projections

def generate_projection(batch: int, dim: int, seqlen: int, dstate: int, dt_rank: int,
                        seed: int) -> Dict[str, np.ndarray]:
    """Inputs of the selection projections, all bf16 (uint16 bit patterns,
    with the exact values under name + "_f64"):

        x    [batch, dim, seqlen] ~ N(0, 1)          (the scan's input u)
        W_x  [dt_rank + 2 dstate, dim] ~ N(0, 1/dim)  (rows: dt_low, B, C)
        W_dt [dim, dt_rank] ~ N(0, 1/dt_rank)

    The weight scales keep every projected value near unit variance, like
    the scan's own synthetic delta, B and C."""
    out: Dict[str, np.ndarray] = {}
    M = dt_rank + 2 * dstate
    draws = {
        "x": normal(seed, STREAMS["x"], batch * dim * seqlen).reshape(batch, dim, seqlen),
        "W_x": normal(seed, STREAMS["W_x"], M * dim, 1.0 / math.sqrt(dim)).reshape(M, dim),
        "W_dt": normal(seed, STREAMS["W_dt"], dim * dt_rank,
                       1.0 / math.sqrt(dt_rank)).reshape(dim, dt_rank),
    }
    for name, x in draws.items():
        out[name], out[name + "_f64"] = _cast(x, "bf16")
    return out
