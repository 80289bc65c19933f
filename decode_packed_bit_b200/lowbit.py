"""Python binding of liblowbit.so (include/lowbit.h): argument marshalling only.

Every function has the name of the C entry point it calls.  Tensors are
torch CUDA tensors (torch supplies device memory and streams; every step of
the computation runs in the library's own kernels).  fp16/bf16 operands may
be given as float16/bfloat16 tensors or as int16/uint16 bit patterns.  A
non-OK status raises LowbitError.  There is no fallback: if the shared
library is missing, loading fails with an error.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblowbit.so")

LOWBIT_OK = 0
LOWBIT_ERR_INVALID_ARG = 1
LOWBIT_ERR_MISALIGNED = 2
LOWBIT_ERR_UNSUPPORTED_SHAPE = 3
LOWBIT_ERR_CUDA = 4

LOWBIT_FMT_Q1_G128 = 1
LOWBIT_FMT_Q2 = 2
LOWBIT_FMT_INT4_G64 = 3
LOWBIT_FMT_TERNARY_G128 = 4
FORMATS = {"q1": LOWBIT_FMT_Q1_G128, "q2": LOWBIT_FMT_Q2, "int4": LOWBIT_FMT_INT4_G64, "t3": LOWBIT_FMT_TERNARY_G128}

# (name, restype, argtypes) of every symbol include/lowbit.h declares.
P, I32, I64, SZ, F32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
SYMBOLS = [
    ("lowbit_status_string", ctypes.c_char_p, [I32]),
    ("lowbit_version", I32, []),
    ("lowbit_fault_flags", I32, []),
    ("lowbit_pack", I32, [I32, P, I64, I64, P, P]),
    ("lowbit_unpack", I32, [I32, P, I64, I64, P, P]),
    ("lowbit_quantize", I32, [I32, P, I64, I64, P, P, P]),
    ("lowbit_q1g128_workspace_bytes", SZ, [I32, I32, I32]),
    ("lowbit_q1g128_gemv", I32, [P, P, P, P, I32, I32, I32, P, SZ, P]),
    ("lowbit_q1g128_act_bytes", SZ, [I32, I32]),
    ("lowbit_q1g128_act_workspace_bytes", SZ, [I32, I32, I32, I32]),
    ("lowbit_q1g128_prepare_act", I32, [P, I32, I32, P, SZ, P]),
    ("lowbit_q1g128_gemv_act", I32, [P, P, P, P, I32, I32, I32, P, SZ, P]),
    ("lowbit_q1g128_gemv_act_group", I32, [P, P, P, P, I32, I32, I32, I32, P, SZ, P]),
    ("lowbit_q1g128_group_workspace_bytes", SZ, [I32, I32, I32, I32]),
    ("lowbit_q1g128_gemv_group", I32, [P, P, P, P, I32, I32, I32, I32, P, SZ, P]),
    ("lowbit_q1g128_gemv_noalloc", I32, [P, P, P, P, I32, I32, I32, P]),
    ("lowbit_int4g64_gemm", I32, [P, P, P, P, I32, I32, I32, P]),
    ("lowbit_int4g64_gemm_group", I32, [P, P, P, P, I32, I32, I32, I32, P]),
    ("lowbit_t3g128_gemv", I32, [P, P, P, P, I32, I32, I32, P]),
    ("lowbit_t3g128_gemv_group", I32, [P, P, P, P, I32, I32, I32, I32, P]),
    ("lowbit_q2_mlp_forward", I32, [P, P, I32, P, I32, P, P, P]),
    ("lowbit_z80_generate", I32, [P, P, I32, P, I32, I32, P, I32, P, P, P]),
    ("lowbit_rmsnorm_bf16", I32, [P, P, I32, I32, F32, P, P]),
    ("lowbit_q1g128_stack_workspace_bytes", SZ, [I32, I32, I32]),
    ("lowbit_q1g128_stack_step", I32, [P, P, I32, I32, I32, P, F32, P, SZ, P, P, P]),
]

_lib = None


class LowbitError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().lowbit_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m decode_packed_bit_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SYMBOLS:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != LOWBIT_OK:
        raise LowbitError(status, where)


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _fmt(fmt):
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def lowbit_fault_flags() -> int:
    return int(lib().lowbit_fault_flags())


# -- packing ----------------------------------------------------------------------

def lowbit_pack(fmt, codes, packed, stream=None):
    rows, cols = codes.shape
    _check(lib().lowbit_pack(_fmt(fmt), _ptr(codes), rows, cols, _ptr(packed), _stream(stream)),
           "lowbit_pack")


def lowbit_unpack(fmt, packed, codes, stream=None):
    rows, cols = codes.shape
    _check(lib().lowbit_unpack(_fmt(fmt), _ptr(packed), rows, cols, _ptr(codes), _stream(stream)),
           "lowbit_unpack")


def lowbit_quantize(fmt, w, packed, scales, stream=None):
    """float32 weights [rows][cols] -> packed codes and FP16 scale bits ("q1" or "int4")."""
    rows, cols = w.shape
    _check(lib().lowbit_quantize(_fmt(fmt), _ptr(w), rows, cols, _ptr(packed), _ptr(scales), _stream(stream)),
           "lowbit_quantize")


# -- Q1_0_g128 --------------------------------------------------------------------

def lowbit_q1g128_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().lowbit_q1g128_workspace_bytes(M, N, K))


def lowbit_q1g128_act_bytes(M: int, K: int) -> int:
    return int(lib().lowbit_q1g128_act_bytes(M, K))


def lowbit_q1g128_act_workspace_bytes(R: int, M: int, N: int, K: int) -> int:
    return int(lib().lowbit_q1g128_act_workspace_bytes(R, M, N, K))


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def lowbit_q1g128_gemv(w_bits, w_scales, x, y, workspace=None, stream=None):
    M, K = x.shape
    N = w_bits.shape[0]
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lowbit_q1g128_gemv(_ptr(w_bits), _ptr(w_scales), _ptr(x), _ptr(y), M, N, K,
                                    _ptr(workspace), wsb, _stream(stream)), "lowbit_q1g128_gemv")


def lowbit_q1g128_prepare_act(x, act, stream=None):
    M, K = x.shape
    _check(lib().lowbit_q1g128_prepare_act(_ptr(x), M, K, _ptr(act), act.numel() * act.element_size(),
                                           _stream(stream)), "lowbit_q1g128_prepare_act")


def lowbit_q1g128_gemv_act(w_bits, w_scales, act, y, M: int, workspace=None, stream=None):
    """workspace: zero-filled before its first use (calls leave it zeroed)."""
    N = w_bits.shape[0]
    K = w_bits.shape[1] * 8
    _check(lib().lowbit_q1g128_gemv_act(_ptr(w_bits), _ptr(w_scales), _ptr(act), _ptr(y), M, N, K,
                                        _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "lowbit_q1g128_gemv_act")


def _ptr_array(ts):
    arr = (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])
    return ctypes.cast(arr, ctypes.c_void_p), arr


def lowbit_q1g128_gemv_act_group(w_bits, w_scales, act, ys, M: int, workspace=None, stream=None):
    """w_bits, w_scales, ys: equal-length lists of tensors (one per matrix)."""
    R = len(w_bits)
    N = w_bits[0].shape[0]
    K = w_bits[0].shape[1] * 8
    pb, kb = _ptr_array(w_bits)
    ps, ks = _ptr_array(w_scales)
    py, ky = _ptr_array(ys)
    _check(lib().lowbit_q1g128_gemv_act_group(pb, ps, _ptr(act), py, R, M, N, K, _ptr(workspace),
                                              _nbytes(workspace), _stream(stream)),
           "lowbit_q1g128_gemv_act_group")


def lowbit_q1g128_group_workspace_bytes(R: int, M: int, N: int, K: int) -> int:
    return lib().lowbit_q1g128_group_workspace_bytes(R, M, N, K)


def lowbit_q1g128_gemv_group(w_bits, w_scales, x, ys, workspace=None, stream=None):
    """y_r = W_r x for equal-length lists of weight tensors and outputs; x [M][K]
    bf16 bits.  workspace: lowbit_q1g128_group_workspace_bytes(R, M, N, K)
    bytes (None when that is 0)."""
    R = len(w_bits)
    M, K = x.shape
    N = w_bits[0].shape[0]
    pb, kb = _ptr_array(w_bits)
    ps, ks = _ptr_array(w_scales)
    py, ky = _ptr_array(ys)
    _check(lib().lowbit_q1g128_gemv_group(pb, ps, _ptr(x), py, R, M, N, K, _ptr(workspace), _nbytes(workspace),
                                          _stream(stream)),
           "lowbit_q1g128_gemv_group")


def lowbit_q1g128_gemv_noalloc(w_bits, w_scales, x, y, stream=None):
    """The product without a workspace (scratch in the library's own fixed
    device array; K <= 32768 at M = 1; calls must not overlap on the GPU)."""
    M, K = x.shape
    N = w_bits.shape[0]
    _check(lib().lowbit_q1g128_gemv_noalloc(_ptr(w_bits), _ptr(w_scales), _ptr(x), _ptr(y), M, N, K,
                                            _stream(stream)), "lowbit_q1g128_gemv_noalloc")


# -- INT4_G64 ---------------------------------------------------------------------

def lowbit_int4g64_gemm(w_q, w_scales, x, y, stream=None):
    M, K = x.shape
    N = w_q.shape[0]
    _check(lib().lowbit_int4g64_gemm(_ptr(w_q), _ptr(w_scales), _ptr(x), _ptr(y), M, N, K, _stream(stream)),
           "lowbit_int4g64_gemm")


def lowbit_int4g64_gemm_group(w_q, w_scales, x, ys, stream=None):
    """y_r = W_r x for equal-length lists of INT4_G64 weights (uint8 [N][K/2],
    fp16 bits [N][K/64]) and fp32 outputs [M][N]; x [M][K] bf16 bits."""
    R = len(w_q)
    M, K = x.shape
    N = w_q[0].shape[0]
    pq, kq = _ptr_array(w_q)
    ps, ks = _ptr_array(w_scales)
    py, ky = _ptr_array(ys)
    _check(lib().lowbit_int4g64_gemm_group(pq, ps, _ptr(x), py, R, M, N, K, _stream(stream)),
           "lowbit_int4g64_gemm_group")


# -- ternary, FP16 scale per 128 ---------------------------------------------------

def lowbit_t3g128_gemv(w, w_scales, x, y, stream=None):
    """w uint8 [N][26 K/128], w_scales fp16 bits [N][K/128], x bf16 [M][K], y fp32 [M][N]."""
    M, K = x.shape
    N = w.shape[0]
    _check(lib().lowbit_t3g128_gemv(_ptr(w), _ptr(w_scales), _ptr(x), _ptr(y), M, N, K, _stream(stream)),
           "lowbit_t3g128_gemv")


def lowbit_t3g128_gemv_group(w, w_scales, x, ys, stream=None):
    R = len(w)
    M, K = x.shape
    N = w[0].shape[0]
    pw, kw = _ptr_array(w)
    ps, ks = _ptr_array(w_scales)
    py, ky = _ptr_array(ys)
    _check(lib().lowbit_t3g128_gemv_group(pw, ps, _ptr(x), py, R, M, N, K, _stream(stream)),
           "lowbit_t3g128_gemv_group")


# -- Q2 MLP -----------------------------------------------------------------------

def lowbit_q2_mlp_forward(w_packed, dims, x, logits, argmax=None, stream=None):
    n_layers = len(w_packed)
    ptrs = (ctypes.c_void_p * n_layers)(*[w.data_ptr() for w in w_packed])
    dims_c = (ctypes.c_int32 * (n_layers + 1))(*[int(d) for d in dims])
    _check(lib().lowbit_q2_mlp_forward(ctypes.cast(ptrs, ctypes.c_void_p), ctypes.cast(dims_c, ctypes.c_void_p),
                                       n_layers, _ptr(x), x.shape[0], _ptr(logits), _ptr(argmax),
                                       _stream(stream)), "lowbit_q2_mlp_forward")


def lowbit_z80_generate(w_packed, dims, queries, charset, reply, reply_len, stream=None):
    """Autoregressive replies: queries uint8 [batch][qlen] (0-padded text),
    charset: bytes or a uint8 sequence of dims[-1] entries (0 = end of reply),
    reply uint8 [batch][max_new], reply_len int32 [batch]."""
    n_layers = len(w_packed)
    ptrs = (ctypes.c_void_p * n_layers)(*[w.data_ptr() for w in w_packed])
    dims_c = (ctypes.c_int32 * (n_layers + 1))(*[int(d) for d in dims])
    cs = bytes(bytearray(int(c) for c in charset))
    cs_c = ctypes.create_string_buffer(cs, len(cs))
    batch, qlen = queries.shape
    max_new = reply.shape[1]
    _check(lib().lowbit_z80_generate(ctypes.cast(ptrs, ctypes.c_void_p), ctypes.cast(dims_c, ctypes.c_void_p),
                                     n_layers, _ptr(queries), batch, qlen, ctypes.cast(cs_c, ctypes.c_void_p),
                                     max_new, _ptr(reply), _ptr(reply_len), _stream(stream)),
           "lowbit_z80_generate")


# -- glue -------------------------------------------------------------------------

def lowbit_rmsnorm_bf16(a, b, out, eps=1e-6, stream=None):
    M, D = a.shape
    _check(lib().lowbit_rmsnorm_bf16(_ptr(a), _ptr(b), M, D, float(eps), _ptr(out), _stream(stream)),
           "lowbit_rmsnorm_bf16")


# -- the fused decode step of a Q1 stack ------------------------------------------

def lowbit_q1g128_stack_workspace_bytes(n_layers: int, hidden: int, ffn: int) -> int:
    return int(lib().lowbit_q1g128_stack_workspace_bytes(n_layers, hidden, ffn))


def lowbit_q1g128_stack_step(w_bits, w_scales, x, hidden, ffn, workspace, eps=1e-6, record_inputs=None,
                             record_outputs=None, stream=None):
    """w_bits / w_scales: lists of 7 * n_layers device tensors (q, k, v, o, gate, up, down per layer)."""
    n = len(w_bits)
    bits, bits_keep = _ptr_array(w_bits)
    scales, scales_keep = _ptr_array(w_scales)
    wsb = workspace.numel() * workspace.element_size()
    _check(lib().lowbit_q1g128_stack_step(bits, scales, n // 7, hidden, ffn, _ptr(x), float(eps), _ptr(workspace), wsb,
                                          _ptr(record_inputs), _ptr(record_outputs), _stream(stream)),
           "lowbit_q1g128_stack_step")

