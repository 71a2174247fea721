"""CPU oracle for one MoE layer's forward pass (ctypes binding of moe_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The CUDA library never imports it and
it never imports the CUDA library.  Every function restates, in double
precision and one token at a time, what the layer computes; see the header
of ``moe_oracle.c`` for the readings of the pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2, OpenMP over tokens, no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                           "-std=c11", _SRC, "-o", tmp, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_double.restype = ctypes.c_double
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_double.restype = ctypes.c_double
        L.oracle_float_to_e4m3_sat.argtypes = [ctypes.c_float]
        L.oracle_float_to_e4m3_sat.restype = ctypes.c_uint8
        L.oracle_router_logits.argtypes = [_P, _P, _I, _I, _P, _P, _I, _P]
        L.oracle_router_logits.restype = None
        L.oracle_topk.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P]
        L.oracle_topk.restype = None
        L.oracle_route.argtypes = [_P, _P, _I, _I, _I, _P, _P, _P, _P]
        L.oracle_route.restype = _I
        L.oracle_moe_tokens_bf16.argtypes = [_P, _I, _P, _P, _I, _P, _P, _I, _P, _P, _I, _P, _I,
                                             _P]
        L.oracle_moe_tokens_bf16.restype = None
        L.oracle_quant_row_e4m3.argtypes = [_P, _I, _P, _P]
        L.oracle_quant_row_e4m3.restype = None
        L.oracle_moe_tokens_fp8.argtypes = [_P, _I, _P, _P, _I, _P, _P, _P, _P, _I, _P, _P, _P,
                                            _P, _I, _P, _I, _P]
        L.oracle_moe_tokens_fp8.restype = None
        L.oracle_round_bf16.argtypes = [_P, ctypes.c_size_t, _P]
        L.oracle_round_bf16.restype = None
        L.oracle_max_threads.argtypes = []
        L.oracle_max_threads.restype = _I
        _lib = L
    return _lib


def max_threads() -> int:
    """Threads the oracle's token loops run on (OpenMP's current maximum)."""
    return int(lib().oracle_max_threads())


# ------------------------------------------------------------------ helpers

def _np(a, dtype):
    """A C-contiguous numpy array of ``dtype`` (torch tensors viewed bitwise)."""
    if a is None:
        return None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                a = a.view(torch.int16).numpy().view(np.uint16)
            elif a.dtype == torch.float8_e4m3fn:
                a = a.view(torch.uint8).numpy()
            else:
                a = a.numpy()
    except ImportError:
        pass
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        same_width_ints = (a.dtype.itemsize == np.dtype(dtype).itemsize
                           and a.dtype.kind in "iu" and np.dtype(dtype).kind in "iu")
        a = a.view(dtype) if same_width_ints else a.astype(dtype)
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data


def bf16_to_f64(bits) -> np.ndarray:
    b = _np(bits, np.uint16)
    f = (b.astype(np.uint32) << 16).view(np.float32)
    with np.errstate(invalid="ignore"):     # signalling-NaN patterns widen quietly
        return f.astype(np.float64)


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(bits)


def double_to_bf16(v: float) -> int:
    return lib().oracle_double_to_bf16(v)


def e4m3_to_double(code: int) -> float:
    return lib().oracle_e4m3_to_double(code)


def float_to_e4m3(v: float) -> int:
    return lib().oracle_float_to_e4m3_sat(v)


# ------------------------------------------------------------- the method

def router_logits(x, valid, router_w, router_b=None) -> np.ndarray:
    """a1: fp32 logits [T, E] (double sums, one rounding)."""
    xb = _np(x, np.uint16)
    T, H = xb.shape
    Wr = _np(router_w, np.float32)
    E = Wr.shape[0]
    v = None if valid is None else _np(valid, np.uint8)
    b = None if router_b is None else _np(router_b, np.float32)
    out = np.empty((T, E), dtype=np.float32)
    lib().oracle_router_logits(_ptr(xb), _ptr(v), T, H, _ptr(Wr), _ptr(b), E, _ptr(out))
    return out


def topk(logits, valid, k: int, renorm: bool = True):
    """a2: ids int32 [T, k] (descending logit, ties to the lower index) and
    weights float64 [T, k]; padding rows give -1 / 0."""
    l = _np(logits, np.float32)
    T, E = l.shape
    v = None if valid is None else _np(valid, np.uint8)
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    lib().oracle_topk(_ptr(l), _ptr(v), T, E, k, int(bool(renorm)), _ptr(ids), _ptr(w))
    return ids, w


def route(ids, valid, E: int):
    """a3: counts [E], offsets [E+1], perm [Tv*k], inv [T*k] (int32)."""
    idn = _np(ids, np.int32)
    T, k = idn.shape
    v = None if valid is None else _np(valid, np.uint8)
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(max(T * k, 1), dtype=np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    n = lib().oracle_route(_ptr(idn), _ptr(v), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm),
                           _ptr(inv))
    return counts, offsets, perm[:n].copy(), inv


def moe_tokens(inputs: dict, ids, w, tokens=None) -> np.ndarray:
    """a4-a6 before the final rounding: float64 [n, H] accumulators for the
    given tokens (all tokens when None), routed by (ids, w)."""
    x = _np(inputs["x"], np.uint16)
    T, H = x.shape
    idn = _np(ids, np.int32)
    wn = _np(w, np.float64)
    k = idn.shape[1]
    tok = np.arange(T, dtype=np.int32) if tokens is None else _np(tokens, np.int32)
    acc = np.empty((len(tok), H), dtype=np.float64)
    wl = inputs["workload"]
    if wl.wtype == "bf16":
        Wgu = _np(inputs["w_gate_up"], np.uint16)
        Wd = _np(inputs["w_down"], np.uint16)
        Wsgu = _np(inputs.get("ws_gate_up"), np.uint16)
        Wsd = _np(inputs.get("ws_down"), np.uint16)
        lib().oracle_moe_tokens_bf16(_ptr(x), H, _ptr(idn), _ptr(wn), k, _ptr(Wgu), _ptr(Wd),
                                     wl.I, _ptr(Wsgu), _ptr(Wsd), wl.Is if wl.S else 0,
                                     _ptr(tok), len(tok), _ptr(acc))
    else:
        g = lambda name, dt: _np(inputs.get(name), dt)  # noqa: E731
        lib().oracle_moe_tokens_fp8(
            _ptr(x), H, _ptr(idn), _ptr(wn), k,
            _ptr(g("w_gate_up", np.uint8)), _ptr(g("s_gate_up", np.float32)),
            _ptr(g("w_down", np.uint8)), _ptr(g("s_down", np.float32)), wl.I,
            _ptr(g("ws_gate_up", np.uint8)), _ptr(g("ss_gate_up", np.float32)),
            _ptr(g("ws_down", np.uint8)), _ptr(g("ss_down", np.float32)), wl.Is if wl.S else 0,
            _ptr(tok), len(tok), _ptr(acc))
    return acc


def round_bf16(acc) -> np.ndarray:
    """bf16 bit patterns (uint16) of round-to-nearest-even(acc)."""
    a = np.ascontiguousarray(acc, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().oracle_round_bf16(_ptr(a), a.size, _ptr(out))
    return out


def quant_row_e4m3(v) -> tuple[np.ndarray, np.ndarray]:
    """1x128 activation quantisation of one fp32 row: (codes u8, scales f32)."""
    a = np.ascontiguousarray(v, dtype=np.float32)
    q = np.empty(a.size, dtype=np.uint8)
    s = np.empty(a.size // 128, dtype=np.float32)
    lib().oracle_quant_row_e4m3(_ptr(a), a.size, _ptr(q), _ptr(s))
    return q, s


def forward(inputs: dict, k: int | None = None, tokens=None, logits=None, renorm: bool = True):
    """The whole layer: routing from ``logits`` when given (for example the
    GPU's own logits, so that both sides route identically), else from the
    oracle's logits.  Returns a dict with logits, ids, w, counts, offsets,
    perm, inv, acc (float64 [n, H]) and out (bf16 bits, uint16 [n, H])."""
    wl = inputs["workload"]
    k = wl.k if k is None else k
    valid = inputs["valid"]
    if logits is None:
        logits = router_logits(inputs["x"], valid, inputs["router_w"], inputs["router_b"])
    else:
        logits = _np(logits, np.float32)
    ids, w = topk(logits, valid, k, renorm)
    counts, offsets, perm, inv = route(ids, valid, wl.E)
    acc = moe_tokens(inputs, ids, w, tokens)
    return {"logits": logits, "ids": ids, "w": w, "counts": counts, "offsets": offsets,
            "perm": perm, "inv": inv, "acc": acc, "out": round_bf16(acc)}
