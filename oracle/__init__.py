"""CPU oracle for the fused MXFP4 routed-MoE layer (test infrastructure).

This package is TEST INFRASTRUCTURE: only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` import it.  The
product (the CUDA library and its Python binding) never does, and shares no
code with it.

It is a thin ctypes wrapper around ``moe_oracle.c`` (plain C, IEEE double,
one pthread per token range), which is built with gcc on first use.  Every
function states the passage of the pages it follows in the C source:

* routing: softmax -> top-k (lowest index wins ties) -> renormalise
  (TokenSpeed-kernel README, "Public API"; fusedtok description, "Operators",
  "API stability");
* grouping: stable counting sort of (token, slot) pairs by expert;
* FC1 -> SwiGLU -> FC2 -> weighted combine with MXFP4 weights
  (tokenspeed-situ description, intro, "Supported contract", "Activation
  precision (w4a16 vs w4a8)"; mxfp6-sm120 description, "Execution model");
* a shared expert added to every token with weight 1, held as extra expert slots
  (mxfp6-sm120 description, path table: routed/shared reduction);
* the same layer with the routing given (precomputed top-k, global expert ids)
  for one contiguous local expert shard, whose partial outputs add up to the
  layer (tokenspeed-situ description, "Supported contract");
* MX codecs per the OCP Microscaling Formats v1.0 specification.

Parity pins (what ties this oracle to something other than itself) are in
``tests/test_oracle_mx.py``, ``tests/test_oracle_routing.py``,
``tests/test_oracle_layer.py``, ``tests/test_oracle_routed.py`` and
``tests/test_oracle_shared.py``; ``tests/test_oracle_mutations.py`` shows that
they catch planted mistakes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
# ORACLE_PLANT_MISTAKE=n (tests only) builds a copy with one deliberate mistake planted,
# so that tests/test_oracle_mutations.py can show the pins catch it.
_PLANT = int(os.environ.get("ORACLE_PLANT_MISTAKE", "0") or 0)
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so" if _PLANT == 0 else f"liboracle_plant{_PLANT}.so")
_lock = threading.Lock()
_lib = None

FMT_E2M1 = 0
FMT_E4M3 = 1
ACT_BF16 = 0
ACT_MXFP8 = 1


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into a shared library (gcc, no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
               "-fno-fast-math", "-D_GNU_SOURCE", f"-DORACLE_PLANT_MISTAKE={_PLANT}", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_e2m1_decode.argtypes, lib.oracle_e2m1_decode.restype = [ctypes.c_uint8], dbl
        lib.oracle_e4m3_decode.argtypes, lib.oracle_e4m3_decode.restype = [ctypes.c_uint8], dbl
        lib.oracle_e8m0_decode.argtypes, lib.oracle_e8m0_decode.restype = [ctypes.c_uint8], dbl
        lib.oracle_round_bf16.argtypes, lib.oracle_round_bf16.restype = [dbl], dbl
        lib.oracle_bf16_bits.argtypes, lib.oracle_bf16_bits.restype = [dbl], ctypes.c_uint16
        lib.oracle_mx_quantize.argtypes = [P, i64, i64, i32, P, P, i32]
        lib.oracle_mx_quantize.restype = i32
        lib.oracle_route.argtypes = [P, i32, i32, P, P]
        lib.oracle_route.restype = None
        lib.oracle_group.argtypes = [i32, i32, i32, P, P, P, P]
        lib.oracle_group.restype = None
        lib.oracle_moe_forward.argtypes = [i32] * 6 + [P] * 6 + [P, i32, P, P, P, P, i32]
        lib.oracle_moe_forward.restype = i32
        lib.oracle_moe_forward_shared.argtypes = [i32] * 7 + [P] * 6 + [P, i32, P, P, P, P, i32]
        lib.oracle_moe_forward_shared.restype = i32
        lib.oracle_moe_forward_routed.argtypes = [i32] * 6 + [P, P, P, i32] + [P] * 4 + [P, i32, P, P, P, P, i32]
        lib.oracle_moe_forward_routed.restype = i32
        _lib = lib
        return lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- MX codecs
def e2m1_decode(code: int) -> float:
    return _load().oracle_e2m1_decode(code)


def e4m3_decode(code: int) -> float:
    return _load().oracle_e4m3_decode(code)


def e8m0_decode(byte: int) -> float:
    return _load().oracle_e8m0_decode(byte)


def round_bf16(v: float) -> float:
    return _load().oracle_round_bf16(float(v))


def mx_quantize(v: np.ndarray, fmt: int, nthreads: int | None = None):
    """Quantise float32 [rows, K] along K. Returns (codes u8, scales u8).

    fmt FMT_E2M1: codes [rows, K/2], two per byte, element 2i in the low nibble.
    fmt FMT_E4M3: codes [rows, K].  scales: [rows, K/32] E8M0 bytes.
    """
    v = np.ascontiguousarray(v, dtype=np.float32)
    lead = v.shape[:-1]
    K = v.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    ncode = K // 2 if fmt == FMT_E2M1 else K
    codes = np.empty(lead + (ncode,), dtype=np.uint8)
    scales = np.empty(lead + (K // 32,), dtype=np.uint8)
    rc = _load().oracle_mx_quantize(_ptr(v), rows, K, fmt, _ptr(codes), _ptr(scales),
                                    nthreads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_mx_quantize rejected rows={rows} K={K} fmt={fmt}")
    return codes, scales


def mx_dequantize(codes: np.ndarray, scales: np.ndarray, fmt: int) -> np.ndarray:
    """Decode MX codes + E8M0 scales into float64 [..., K] with the oracle's tables."""
    lib = _load()
    if fmt == FMT_E2M1:
        table = np.array([lib.oracle_e2m1_decode(c) for c in range(16)], dtype=np.float64)
        lo = table[codes & 0xF]
        hi = table[codes >> 4]
        vals = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))
    else:
        table = np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)
        vals = table[codes]
    stab = np.array([lib.oracle_e8m0_decode(b) for b in range(256)], dtype=np.float64)
    s = np.repeat(stab[scales], 32, axis=-1)
    return vals * s


# ---------------------------------------------------------------- routing
def route(logits: np.ndarray, k: int):
    """Top-k softmax routing for every row of float32 [T, E]. Returns (ids i32 [T,k], w f32 [T,k])."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    lib = _load()
    for t in range(T):
        lib.oracle_route(_ptr(logits[t]), E, k, _ptr(ids[t]), _ptr(w[t]))
    return ids, w


def group(ids: np.ndarray, E: int):
    """Group (token, slot) pairs by expert. Returns (counts [E], offsets [E+1], sorted_pair [T*k])."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    sorted_pair = np.empty(T * k, dtype=np.int32)
    _load().oracle_group(T, k, E, _ptr(ids), _ptr(counts), _ptr(offsets), _ptr(sorted_pair))
    return counts, offsets, sorted_pair


# ---------------------------------------------------------------- the layer
def moe_forward(x_bf16_bits: np.ndarray, logits: np.ndarray, w1: np.ndarray, w1s: np.ndarray,
                w2: np.ndarray, w2s: np.ndarray, top_k: int, act_mode: int = ACT_BF16,
                tokens=None, nthreads: int | None = None, exact: bool = False, num_shared: int = 0):
    """Evaluate the layer per token.

    x_bf16_bits: uint16 [T, H] (bf16 bit patterns); logits f32 [T, E];
    w1 u8 [E + S, 2I, H/2], w1s u8 [E + S, 2I, H/32]; w2 u8 [E + S, H, I/2], w2s u8 [E + S, H, I/32],
    S = num_shared: the shared expert's chunks in slots E.. (added to every token with weight 1).
    tokens: optional list of token indices to evaluate (default: all).
    Returns (out bf16 bits uint16 [n, H], ids i32 [n, k + S], w f32 [n, k + S]), plus, with
    exact=True, the float64 output before its final bf16 rounding as a fourth item.
    """
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, H = x.shape
    E = logits.shape[1]
    S = int(num_shared)
    I = w2.shape[2] * 2
    for a in (w1, w1s, w2, w2s):
        assert a.dtype == np.uint8 and a.flags["C_CONTIGUOUS"]
    assert w1.shape == (E + S, 2 * I, H // 2) and w1s.shape == (E + S, 2 * I, H // 32)
    assert w2.shape == (E + S, H, I // 2) and w2s.shape == (E + S, H, I // 32)
    if tokens is None:
        tok_arr = None
        n = T
    else:
        tok_arr = np.ascontiguousarray(tokens, dtype=np.int32)
        n = int(tok_arr.shape[0])
    out = np.empty((n, H), dtype=np.uint16)
    ids = np.empty((n, top_k + S), dtype=np.int32)
    w = np.empty((n, top_k + S), dtype=np.float32)
    out_exact = np.empty((n, H), dtype=np.float64) if exact else None
    tail = (_ptr(tok_arr) if tok_arr is not None else None, n, _ptr(out), _ptr(ids), _ptr(w),
            _ptr(out_exact) if exact else None, nthreads or default_threads())
    if S:
        rc = _load().oracle_moe_forward_shared(T, H, I, E, S, top_k, act_mode, _ptr(x), _ptr(logits), _ptr(w1),
                                               _ptr(w1s), _ptr(w2), _ptr(w2s), *tail)
    else:
        rc = _load().oracle_moe_forward(T, H, I, E, top_k, act_mode, _ptr(x), _ptr(logits), _ptr(w1), _ptr(w1s),
                                        _ptr(w2), _ptr(w2s), *tail)
    if rc != 0:
        raise ValueError("oracle_moe_forward rejected its arguments")
    if exact:
        return out, ids, w, out_exact
    return out, ids, w


def moe_forward_routed(x_bf16_bits: np.ndarray, topk_ids: np.ndarray, topk_w: np.ndarray, local_offset: int,
                       w1: np.ndarray, w1s: np.ndarray, w2: np.ndarray, w2s: np.ndarray,
                       act_mode: int = ACT_BF16, tokens=None, nthreads: int | None = None):
    """Evaluate the layer per token with the routing given (precomputed top-k, global ids).

    topk_ids i32 [T, k] global expert ids, topk_w f32 [T, k]; the weights w1..w2s hold the
    local shard of E experts, global ids [local_offset, local_offset + E).  Pairs outside the
    shard contribute nothing (the result is the shard's partial output).
    Returns (out bf16 bits uint16 [n, H], exact float64 [n, H], local ids i32 [n, k] (-1: not local)).
    """
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    tw = np.ascontiguousarray(topk_w, dtype=np.float32)
    T, H = x.shape
    k = ids.shape[1]
    E = w1.shape[0]
    I = w2.shape[2] * 2
    for a in (w1, w1s, w2, w2s):
        assert a.dtype == np.uint8 and a.flags["C_CONTIGUOUS"]
    assert ids.shape == (T, k) and tw.shape == (T, k)
    assert w1.shape == (E, 2 * I, H // 2) and w1s.shape == (E, 2 * I, H // 32)
    assert w2.shape == (E, H, I // 2) and w2s.shape == (E, H, I // 32)
    tok_arr = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = T if tok_arr is None else int(tok_arr.shape[0])
    out = np.empty((n, H), dtype=np.uint16)
    out_exact = np.empty((n, H), dtype=np.float64)
    ids_loc = np.empty((n, k), dtype=np.int32)
    w_out = np.empty((n, k), dtype=np.float32)
    rc = _load().oracle_moe_forward_routed(
        T, H, I, E, k, act_mode, _ptr(x), _ptr(ids), _ptr(tw), int(local_offset), _ptr(w1), _ptr(w1s), _ptr(w2),
        _ptr(w2s), _ptr(tok_arr) if tok_arr is not None else None, n, _ptr(out), _ptr(ids_loc), _ptr(w_out),
        _ptr(out_exact), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_moe_forward_routed rejected its arguments")
    return out, out_exact, ids_loc


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
