"""CPU oracle for the packed low-bit products -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The GPU library never imports, links
or executes it, and it imports nothing from the GPU library.

The arithmetic lives in ``lowbit_oracle.c`` (plain single-threaded C, double
precision for the float formats, int64-then-wrap for the 2-bit network); this
module only compiles it with gcc and marshals numpy arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lowbit_oracle.c")
_LIB = os.path.join(_HERE, "liblowbit_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, strict IEEE: no fast-math, no FMA
    contraction) into oracle/liblowbit_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
            "-ffp-contract=off", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
    lib.orc_f16_to_f64.restype = ctypes.c_double
    lib.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.orc_bf16_to_f64.restype = ctypes.c_double
    for name in ("orc_q1_pack", "orc_q1_unpack", "orc_int4_pack", "orc_int4_unpack",
                 "orc_q2_pack", "orc_q2_unpack", "orc_t3_pack", "orc_t3_unpack"):
        getattr(lib, name).argtypes = [P, I64, I64, P]
        getattr(lib, name).restype = ctypes.c_int
    for name in ("orc_q1_gemv", "orc_int4_gemv", "orc_t3_gemv"):
        getattr(lib, name).argtypes = [P, P, P, I64, I64, I64, P, P]
        getattr(lib, name).restype = ctypes.c_int
    for name in ("orc_q1_gemv_at", "orc_int4_gemv_at", "orc_t3_gemv_at"):
        getattr(lib, name).argtypes = [P, P, P, I64, P, P, I64, P, P]
        getattr(lib, name).restype = ctypes.c_int
    lib.orc_q1_weight.argtypes = [P, P, I64, I64, I64]
    lib.orc_q1_weight.restype = ctypes.c_double
    lib.orc_t3_weight.argtypes = [P, P, I64, I64, I64]
    lib.orc_t3_weight.restype = ctypes.c_double
    lib.orc_int4_weight.argtypes = [P, P, I64, I64, I64]
    lib.orc_int4_weight.restype = ctypes.c_double
    lib.orc_q2_weight.argtypes = [P, I64, I64, I64]
    lib.orc_q2_weight.restype = ctypes.c_int
    lib.orc_q2_layer.argtypes = [P, I64, I64, P, ctypes.c_int, P]
    lib.orc_q2_layer.restype = None
    lib.orc_q2_layer_muladd16.argtypes = [P, I64, I64, P, ctypes.c_int, P]
    lib.orc_q2_layer_muladd16.restype = None
    lib.orc_argmax16.argtypes = [P, I64]
    lib.orc_argmax16.restype = ctypes.c_int32
    lib.orc_q2_mlp_forward.argtypes = [P, P, ctypes.c_int, P, I64, P, P, ctypes.c_int]
    lib.orc_q2_mlp_forward.restype = ctypes.c_int
    lib.orc_z80_generate.argtypes = [P, P, ctypes.c_int, P, I64, I64, P, I64, P, P]
    lib.orc_z80_generate.restype = ctypes.c_int
    lib.orc_trigram_encode.argtypes = [ctypes.c_char_p, P]
    lib.orc_trigram_encode.restype = None
    lib.orc_rmsnorm.argtypes = [P, P, I64, I64, ctypes.c_double, P]
    lib.orc_rmsnorm.restype = None
    lib.orc_f64_to_f16.argtypes = [ctypes.c_double]
    lib.orc_f64_to_f16.restype = ctypes.c_uint16
    for name in ("orc_q1_quantize", "orc_int4_quantize"):
        getattr(lib, name).argtypes = [P, I64, I64, P, P]
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# -- scalar decoders ---------------------------------------------------------

def f16_to_f64(bits: int) -> float:
    return _load().orc_f16_to_f64(int(bits) & 0xFFFF)


def bf16_to_f64(bits: int) -> float:
    return _load().orc_bf16_to_f64(int(bits) & 0xFFFF)


# -- packers -----------------------------------------------------------------

_PACK = {"q1": ("orc_q1_pack", "orc_q1_unpack", 8),
         "q2": ("orc_q2_pack", "orc_q2_unpack", 4),
         "int4": ("orc_int4_pack", "orc_int4_unpack", 2),
         "t3": ("orc_t3_pack", "orc_t3_unpack", None)}


def packed_cols(fmt: str, cols: int) -> int:
    """Bytes of one packed row: cols / per_byte, or 26 per 128 for ternary."""
    per = _PACK[fmt][2]
    return 26 * (cols // 128) if per is None else cols // per


def pack(fmt: str, codes: np.ndarray) -> np.ndarray:
    """codes int8 [rows][cols] -> packed uint8 [rows][packed_cols(fmt, cols)]."""
    fn, _, per = _PACK[fmt]
    codes = _c(codes, np.int8)
    rows, cols = codes.shape
    if per is None and cols % 128 != 0:
        raise ValueError(f"oracle {fn}: cols must be a multiple of 128")
    out = np.zeros((rows, packed_cols(fmt, cols)), np.uint8)
    rc = getattr(_load(), fn)(_ptr(codes), rows, cols, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle {fn} rejected the codes (shape {codes.shape})")
    return out


def unpack(fmt: str, packed: np.ndarray, cols: int) -> np.ndarray:
    _, fn, per = _PACK[fmt]
    packed = _c(packed, np.uint8)
    rows = packed.shape[0]
    out = np.zeros((rows, cols), np.int8)
    rc = getattr(_load(), fn)(_ptr(packed), rows, cols, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle {fn} rejected cols={cols}")
    return out


# -- float-format products -----------------------------------------------------

def q1_gemv(bits, scales, x, want_abs=False):
    """bits uint8 [N][K/8], scales uint16 (fp16 bits) [N][K/128],
    x uint16 (bf16 bits) [M][K] -> y float64 [M][N] (and sum |w x|)."""
    bits, scales, x = _c(bits, np.uint8), _c(scales, np.uint16), _c(x, np.uint16)
    M, K = x.shape
    N = bits.shape[0]
    y = np.zeros((M, N), np.float64)
    ab = np.zeros((M, N), np.float64)
    rc = _load().orc_q1_gemv(_ptr(bits), _ptr(scales), _ptr(x), M, N, K, _ptr(y), _ptr(ab))
    if rc != 0:
        raise ValueError("oracle q1_gemv: K must be a multiple of 128")
    return (y, ab) if want_abs else y


def q1_gemv_at(bits, scales, x, ms, ns):
    bits, scales, x = _c(bits, np.uint8), _c(scales, np.uint16), _c(x, np.uint16)
    ms, ns = _c(ms, np.int64), _c(ns, np.int64)
    K = x.shape[1]
    y = np.zeros(len(ms), np.float64)
    ab = np.zeros(len(ms), np.float64)
    rc = _load().orc_q1_gemv_at(_ptr(bits), _ptr(scales), _ptr(x), K, _ptr(ms), _ptr(ns),
                                len(ms), _ptr(y), _ptr(ab))
    if rc != 0:
        raise ValueError("oracle q1_gemv_at: K must be a multiple of 128")
    return y, ab


def q1_weight(bits, scales, K, n, k) -> float:
    bits, scales = _c(bits, np.uint8), _c(scales, np.uint16)
    return _load().orc_q1_weight(_ptr(bits), _ptr(scales), K, n, k)


def int4_gemv(q, scales, x, want_abs=False):
    """q uint8 [N][K/2], scales uint16 (fp16 bits) [N][K/64], x bf16 bits [M][K]."""
    q, scales, x = _c(q, np.uint8), _c(scales, np.uint16), _c(x, np.uint16)
    M, K = x.shape
    N = q.shape[0]
    y = np.zeros((M, N), np.float64)
    ab = np.zeros((M, N), np.float64)
    rc = _load().orc_int4_gemv(_ptr(q), _ptr(scales), _ptr(x), M, N, K, _ptr(y), _ptr(ab))
    if rc != 0:
        raise ValueError("oracle int4_gemv: K must be a multiple of 64")
    return (y, ab) if want_abs else y


def int4_gemv_at(q, scales, x, ms, ns):
    q, scales, x = _c(q, np.uint8), _c(scales, np.uint16), _c(x, np.uint16)
    ms, ns = _c(ms, np.int64), _c(ns, np.int64)
    K = x.shape[1]
    y = np.zeros(len(ms), np.float64)
    ab = np.zeros(len(ms), np.float64)
    rc = _load().orc_int4_gemv_at(_ptr(q), _ptr(scales), _ptr(x), K, _ptr(ms), _ptr(ns),
                                  len(ms), _ptr(y), _ptr(ab))
    if rc != 0:
        raise ValueError("oracle int4_gemv_at: K must be a multiple of 64")
    return y, ab


def t3_gemv(packed, scales, x, want_abs=False):
    """packed uint8 [N][26 K/128], scales uint16 (fp16 bits) [N][K/128], x bf16 bits [M][K]."""
    packed, scales, x = _c(packed, np.uint8), _c(scales, np.uint16), _c(x, np.uint16)
    M, K = x.shape
    N = packed.shape[0]
    y = np.zeros((M, N), np.float64)
    ab = np.zeros((M, N), np.float64)
    rc = _load().orc_t3_gemv(_ptr(packed), _ptr(scales), _ptr(x), M, N, K, _ptr(y), _ptr(ab))
    if rc != 0:
        raise ValueError("oracle t3_gemv: K must be a multiple of 128")
    return (y, ab) if want_abs else y


def t3_gemv_at(packed, scales, x, ms, ns):
    packed, scales, x = _c(packed, np.uint8), _c(scales, np.uint16), _c(x, np.uint16)
    ms, ns = _c(ms, np.int64), _c(ns, np.int64)
    K = x.shape[1]
    y = np.zeros(len(ms), np.float64)
    ab = np.zeros(len(ms), np.float64)
    rc = _load().orc_t3_gemv_at(_ptr(packed), _ptr(scales), _ptr(x), K, _ptr(ms), _ptr(ns),
                                len(ms), _ptr(y), _ptr(ab))
    if rc != 0:
        raise ValueError("oracle t3_gemv_at: K must be a multiple of 128")
    return y, ab


def t3_weight(packed, scales, K, n, k) -> float:
    packed, scales = _c(packed, np.uint8), _c(scales, np.uint16)
    return _load().orc_t3_weight(_ptr(packed), _ptr(scales), K, n, k)


def int4_weight(q, scales, K, n, k) -> float:
    q, scales = _c(q, np.uint8), _c(scales, np.uint16)
    return _load().orc_int4_weight(_ptr(q), _ptr(scales), K, n, k)


# -- 2-bit integer network -------------------------------------------------------

def q2_layer(packed, in_dim, out_dim, a, hidden, muladd16=False):
    packed, a = _c(packed, np.uint8), _c(a, np.int16)
    out = np.zeros(out_dim, np.int16)
    fn = _load().orc_q2_layer_muladd16 if muladd16 else _load().orc_q2_layer
    fn(_ptr(packed), in_dim, out_dim, _ptr(a), int(bool(hidden)), _ptr(out))
    return out


def q2_mlp_forward(packed_layers, dims, x, muladd16=False):
    """packed_layers: list of uint8 [dims[l+1]][dims[l]/4]; x int16 [batch][dims[0]].
    Returns (logits int16 [batch][dims[-1]], argmax int32 [batch])."""
    layers = [_c(p, np.uint8) for p in packed_layers]
    dims_a = _c(dims, np.int32)
    x = _c(x, np.int16)
    batch = x.shape[0]
    ptrs = (ctypes.c_void_p * len(layers))(*[p.ctypes.data for p in layers])
    logits = np.zeros((batch, int(dims_a[-1])), np.int16)
    am = np.zeros(batch, np.int32)
    rc = _load().orc_q2_mlp_forward(ctypes.cast(ptrs, ctypes.c_void_p), _ptr(dims_a),
                                    len(layers), _ptr(x), batch, _ptr(logits), _ptr(am),
                                    int(bool(muladd16)))
    if rc != 0:
        raise ValueError("oracle q2_mlp_forward rejected dims")
    return logits, am


def argmax16(v) -> int:
    v = _c(v, np.int16)
    return int(_load().orc_argmax16(_ptr(v), len(v)))


def z80_generate(packed_layers, dims, queries, charset, max_new):
    """Autoregressive replies: queries uint8 [batch][qlen] (0-padded text),
    charset uint8 [dims[-1]] (byte 0 = end of reply).  Returns (replies uint8
    [batch][max_new], 0 past each end; lengths int32 [batch])."""
    layers = [_c(p, np.uint8) for p in packed_layers]
    dims_a = _c(dims, np.int32)
    queries = _c(queries, np.uint8)
    charset = _c(charset, np.uint8)
    batch, qlen = queries.shape
    ptrs = (ctypes.c_void_p * len(layers))(*[p.ctypes.data for p in layers])
    reply = np.zeros((batch, max_new), np.uint8)
    lens = np.zeros(batch, np.int32)
    rc = _load().orc_z80_generate(ctypes.cast(ptrs, ctypes.c_void_p), _ptr(dims_a), len(layers), _ptr(queries),
                                  batch, qlen, _ptr(charset), max_new, _ptr(reply), _ptr(lens))
    if rc != 0:
        raise ValueError("oracle z80_generate rejected its sizes")
    return reply, lens


def trigram_encode(text: str) -> np.ndarray:
    out = np.zeros(128, np.int16)
    _load().orc_trigram_encode(text.encode("utf-8"), _ptr(out))
    return out


# -- glue ------------------------------------------------------------------------

def rmsnorm(a, b=None, eps=1e-6):
    """a (and b) float32 [M][D] -> r float64 [M][D]; v = a + b when b is given."""
    a = _c(a, np.float32)
    M, D = a.shape
    r = np.zeros((M, D), np.float64)
    bp = None
    if b is not None:
        b = _c(b, np.float32)
        bp = _ptr(b)
    _load().orc_rmsnorm(_ptr(a), bp, M, D, eps, _ptr(r))
    return r


def f64_to_f16(v: float) -> int:
    """IEEE binary16 bits of v: nearest, ties to even; |v| >= 65504 saturates."""
    return int(_load().orc_f64_to_f16(float(v)))


def q1_quantize(w):
    """float32 [N][K] -> (codes int8 {0,1} [N][K], fp16 scale bits [N][K/128]):
    sign w >= 0 -> 1, scale = fp16(mean |w| over each 128-group)."""
    w = _c(w, np.float32)
    N, K = w.shape
    codes = np.zeros((N, K), np.int8)
    scales = np.zeros((N, K // 128), np.uint16)
    if _load().orc_q1_quantize(_ptr(w), N, K, _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("oracle q1_quantize: K must be a multiple of 128")
    return codes, scales


def int4_quantize(w):
    """float32 [N][K] -> (codes int8 [-8,7] [N][K], fp16 scale bits [N][K/64]):
    d = fp16(max|w| / 7) per 64-group, q = clamp(rint(w / d), -8, 7)."""
    w = _c(w, np.float32)
    N, K = w.shape
    codes = np.zeros((N, K), np.int8)
    scales = np.zeros((N, K // 64), np.uint16)
    if _load().orc_int4_quantize(_ptr(w), N, K, _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("oracle int4_quantize: K must be a multiple of 64")
    return codes, scales
