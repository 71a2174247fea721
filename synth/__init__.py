"""Seeded synthetic inputs for the MoE-layer forward pass.

This module serves both sides of every parity check (the CUDA library and the
CPU oracle) and holds none of the layer's arithmetic: it draws numbers
(Philox4x32-10 + Box-Muller, in ``philox.c``) and lays them out as the
workloads' tensors.  Rounding to bf16 and encoding to e4m3 use PyTorch's own
CPU casts (library routines), not code shared with either side.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "philox.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None

# One stream id per tensor role; element index is the Philox counter.
STREAM_X = 1
STREAM_ROUTER_W = 2
STREAM_ROUTER_B = 3
STREAM_W_GATE_UP = 4
STREAM_W_DOWN = 5
STREAM_WS_GATE_UP = 6
STREAM_WS_DOWN = 7
STREAM_ZIPF_RANK = 8


def build(force: bool = False) -> str:
    """Compile ``philox.c`` into ``libsynth.so`` (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.synth_philox4x32_10.argtypes = [ctypes.POINTER(ctypes.c_uint32)] * 2 + [
            ctypes.POINTER(ctypes.c_uint32)]
        L.synth_philox4x32_10.restype = None
        L.synth_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64,
                                       ctypes.c_uint64, ctypes.c_double, ctypes.c_double,
                                       ctypes.c_void_p]
        L.synth_normal_f32.restype = None
        L.synth_uniform_f64.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64,
                                        ctypes.c_uint64, ctypes.c_void_p]
        L.synth_uniform_f64.restype = None
        _lib = L
    return _lib


def philox4x32_10(counter, key):
    """One Philox4x32-10 block: 4 counter words, 2 key words -> 4 words."""
    c = (ctypes.c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in counter])
    k = (ctypes.c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    o = (ctypes.c_uint32 * 4)()
    lib().synth_philox4x32_10(c, k, o)
    return [int(v) for v in o]


def normal_f32(seed: int, stream: int, n: int, sigma: float = 1.0, mean: float = 0.0,
               start: int = 0, out: np.ndarray | None = None) -> np.ndarray:
    if out is None:
        out = np.empty(n, dtype=np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == n
    lib().synth_normal_f32(seed, stream, start, n, sigma, mean, out.ctypes.data)
    return out


def uniform_f64(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    lib().synth_uniform_f64(seed, stream, start, n, out.ctypes.data)
    return out


_CHUNK = 1 << 25  # elements per generation chunk (128 MB of fp32)


def normal_bf16(seed: int, stream: int, shape, sigma: float = 1.0):
    """N(0, sigma^2) tensor, drawn in fp32, rounded to bf16 by torch's cast."""
    import torch
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16)
    buf = np.empty(min(n, _CHUNK), dtype=np.float32)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        normal_f32(seed, stream, m, sigma, start=s, out=buf[:m])
        out[s:s + m] = torch.from_numpy(buf[:m]).to(torch.bfloat16)
    return out.view(*shape)


def normal_fp32_tensor(seed: int, stream: int, shape, sigma: float = 1.0):
    import torch
    n = int(np.prod(shape))
    return torch.from_numpy(normal_f32(seed, stream, n, sigma)).view(*shape)


def normal_e4m3_blockscaled(seed: int, stream: int, groups: int, rows: int, cols: int,
                            sigma: float, block: int = 128):
    """FP8 e4m3 weights with fp32 block scales, as an offline-quantised model
    would ship them: for every ``block x block`` tile of each [rows, cols] matrix
    the scale is amax/448 (1 if the tile is all zero) and the codes are torch's
    round-to-nearest-even cast of w/scale.  Returns (codes u8 [groups,rows,cols],
    scales f32 [groups, rows/block, cols/block])."""
    import torch
    assert rows % block == 0 and cols % block == 0
    codes = torch.empty(groups, rows, cols, dtype=torch.uint8)
    scales = torch.empty(groups, rows // block, cols // block, dtype=torch.float32)
    per = rows * cols
    buf = np.empty(per, dtype=np.float32)
    for g in range(groups):
        normal_f32(seed, stream, per, sigma, start=g * per, out=buf)
        w = torch.from_numpy(buf).view(rows // block, block, cols // block, block)
        amax = w.abs().amax(dim=(1, 3))
        s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        q = (w / s[:, None, :, None]).to(torch.float8_e4m3fn)
        codes[g] = q.view(torch.uint8).reshape(rows, cols)
        scales[g] = s
    return codes, scales


from .workloads import WORKLOADS, Workload, make_inputs  # noqa: E402,F401
