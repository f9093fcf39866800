"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

The stream itself is implemented in ``tw_synth.c`` (SplitMix64 counters,
Box–Muller normals, a partial Fisher–Yates shuffle); this module only builds
and calls it.  It contains none of the ternary layer's arithmetic.

Workload recipe (the shapes of a Qwen2.5-1.5B-sized decoder, 28 layers x 7
projections, hidden size 1536, MLP width 8960, 256-wide k/v projections):

* weights  W[N, K] ~ N(0, 0.02^2), one independent stream per (layer, proj);
* activations x[M, K] ~ N(0, 1), one independent stream per (layer, proj);
  with ``outliers=True`` floor(0.01*K) channels, chosen by a seeded shuffle
  per (layer, proj) and shared by every token row, are multiplied by 20.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

BASE_SEED = 20261202
KIND_W, KIND_X, KIND_OUTLIER = 1, 2, 3

# (name, N, K): y = x @ W.T with W [N x K].
PROJECTIONS = (
    ("q", 1536, 1536),
    ("k", 256, 1536),
    ("v", 256, 1536),
    ("o", 1536, 1536),
    ("gate", 8960, 1536),
    ("up", 8960, 1536),
    ("down", 1536, 8960),
)
N_LAYERS = 28

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tw_synth.c")
_LIB = os.path.join(_HERE, "libtw_synth.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or (
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC)):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off",
                        "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"],
                       check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, p = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        lib.tws_output.restype = u64
        lib.tws_output.argtypes = [u64, u64]
        lib.tws_key.restype = u64
        lib.tws_key.argtypes = [u64, i64, i64, i64]
        lib.tws_normal_f32.restype = None
        lib.tws_normal_f32.argtypes = [u64, i64, i64, ctypes.c_double, p]
        lib.tws_choose.restype = None
        lib.tws_choose.argtypes = [u64, i64, i64, p]
        _lib = lib
    return _lib


def stream_key(layer: int, proj: int, kind: int, base: int = BASE_SEED) -> int:
    return int(_load().tws_key(base, layer, proj, kind))


def raw_outputs(key: int, start: int, n: int) -> np.ndarray:
    lib = _load()
    return np.array([lib.tws_output(key, start + i) for i in range(n)],
                    dtype=np.uint64)


def normal(key: int, n: int, sigma: float = 1.0, offset: int = 0) -> np.ndarray:
    out = np.empty(n, np.float32)
    _load().tws_normal_f32(key, offset, n, float(sigma), out.ctypes.data)
    return out


def choose(key: int, K: int, count: int) -> np.ndarray:
    out = np.empty(count, np.int64)
    _load().tws_choose(key, K, count, out.ctypes.data)
    return out


def weights(layer: int, proj: int, N: int, K: int, sigma: float = 0.02,
            rows: slice | None = None) -> np.ndarray:
    """W [N, K] float32 for (layer, proj); ``rows`` limits generation."""
    key = stream_key(layer, proj, KIND_W)
    r0, r1 = (0, N) if rows is None else (rows.start or 0, rows.stop)
    return normal(key, (r1 - r0) * K, sigma, offset=r0 * K).reshape(r1 - r0, K)


def outlier_channels(layer: int, proj: int, K: int) -> np.ndarray:
    return np.sort(choose(stream_key(layer, proj, KIND_OUTLIER), K, K // 100))


def activations(layer: int, proj: int, M: int, K: int,
                outliers: bool = True) -> np.ndarray:
    """x [M, K] float32 for (layer, proj)."""
    x = normal(stream_key(layer, proj, KIND_X), M * K, 1.0).reshape(M, K)
    if outliers:
        x[:, outlier_channels(layer, proj, K)] *= np.float32(20.0)
    return x


def sweep_shapes(n_layers: int = N_LAYERS):
    """[(layer, proj_index, name, N, K)] in decoder order."""
    return [(l, p, name, N, K) for l in range(n_layers)
            for p, (name, N, K) in enumerate(PROJECTIONS)]
