"""The C-ABI library loads, exports every symbol include/lowbit.h declares,
and rejects bad arguments on the host before any CUDA call.  CPU only: no
call here reaches a kernel launch (every case fails validation or is an
empty no-op)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

from decode_packed_bit_b200 import build as lb_build


@pytest.fixture(scope="module")
def L():
    lb_build.build()
    from decode_packed_bit_b200 import lowbit
    return lowbit.lib()


def _header_symbols():
    with open(os.path.join(ROOT, "include", "lowbit.h")) as f:
        txt = f.read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lowbit_[a-z0-9_]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(L):
    from decode_packed_bit_b200 import lowbit
    declared = _header_symbols()
    assert len(declared) >= 12
    bound = {name for name, _, _ in lowbit.SYMBOLS}
    for name in declared:
        assert hasattr(L, name), f"{name} missing from liblowbit.so"
        assert name in bound, f"{name} has no Python binding"


def test_status_strings(L):
    for s in range(5):
        assert L.lowbit_status_string(s)
    assert L.lowbit_status_string(99) == b"unknown status"
    assert L.lowbit_version() >= 100


FAKE = ctypes.c_void_p(0x10000)      # aligned, never dereferenced: validation fails first
MIS = ctypes.c_void_p(0x10008)


def test_pack_validation(L):
    assert L.lowbit_pack(7, FAKE, 4, 8, FAKE, None) == 1               # bad format
    assert L.lowbit_pack(1, FAKE, 4, 12, FAKE, None) == 3              # cols % 8
    assert L.lowbit_pack(2, FAKE, 4, 6, FAKE, None) == 3               # cols % 4
    assert L.lowbit_pack(3, FAKE, 4, 3, FAKE, None) == 3               # cols % 2
    assert L.lowbit_pack(1, None, 4, 8, FAKE, None) == 1               # null
    assert L.lowbit_pack(1, MIS, 4, 8, FAKE, None) == 2                # misaligned
    assert L.lowbit_pack(1, None, 0, 8, None, None) == 0               # empty: no-op
    assert L.lowbit_unpack(1, FAKE, -1, 8, FAKE, None) == 1
    assert L.lowbit_unpack(3, FAKE, 4, 8, MIS, None) == 2


def test_q1_validation(L):
    g = L.lowbit_q1g128_gemv
    assert g(FAKE, FAKE, FAKE, FAKE, 0, 16, 128, None, 0, None) == 1   # M < 1
    assert g(FAKE, FAKE, FAKE, FAKE, 17, 16, 128, None, 0, None) == 1  # M > 16
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 16, 192, None, 0, None) == 3   # K % 128
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 0, 128, None, 0, None) == 1    # N < 1
    assert g(None, FAKE, FAKE, FAKE, 1, 16, 128, None, 0, None) == 1   # null
    assert g(FAKE, FAKE, MIS, FAKE, 1, 16, 128, None, 0, None) == 2    # misaligned x
    # one-launch shapes need no workspace; the persistent M = 1 kernel (very
    # many rows, 148 SMs when no device is visible) reads a prepared activation
    assert L.lowbit_q1g128_workspace_bytes(1, 4096, 4096) == 0
    assert L.lowbit_q1g128_workspace_bytes(4, 4096, 4096) == 0
    big = 2 * 148 * 2 * 8 * 32
    need = L.lowbit_q1g128_workspace_bytes(1, big, 1024)
    assert need > 0
    assert g(FAKE, FAKE, FAKE, FAKE, 1, big, 1024, FAKE, need - 1, None) == 1
    assert g(FAKE, FAKE, FAKE, FAKE, 1, big, 1024, None, need, None) == 1
    assert g(FAKE, FAKE, FAKE, FAKE, 1, big, 1024, MIS, need, None) == 2
    # the allocation-free form: K beyond its fixed scratch is refused at M = 1
    # for every N, before any dispatch
    na = L.lowbit_q1g128_gemv_noalloc
    for n in (16, 4096, big):
        assert na(FAKE, FAKE, FAKE, FAKE, 1, n, 32768 + 128, None) == 3
    assert na(FAKE, FAKE, FAKE, FAKE, 0, 16, 128, None) == 1
    assert na(FAKE, FAKE, MIS, FAKE, 1, 16, 128, None) == 2
    assert L.lowbit_q1g128_workspace_bytes(1, 16, 100) == 0            # invalid shape -> 0
    assert L.lowbit_q1g128_act_bytes(1, 4096) > 0
    assert L.lowbit_q1g128_prepare_act(FAKE, 1, 100, FAKE, 1 << 20, None) == 3
    assert L.lowbit_q1g128_prepare_act(FAKE, 1, 128, FAKE, 0, None) == 1
    assert L.lowbit_q1g128_act_workspace_bytes(1, 1, 4096, 4096) == 0
    assert L.lowbit_q1g128_gemv_act(FAKE, FAKE, None, FAKE, 1, 16, 128, None, 0, None) == 1
    assert L.lowbit_q1g128_gemv_act(FAKE, FAKE, MIS, FAKE, 1, 16, 128, None, 0, None) == 2
    ptrs = (ctypes.c_void_p * 2)(0x10000, 0x10000)
    pp = ctypes.cast(ptrs, ctypes.c_void_p)
    grp = L.lowbit_q1g128_gemv_act_group
    assert grp(pp, pp, FAKE, pp, 0, 1, 16, 256, None, 0, None) == 1      # R < 1
    assert grp(pp, pp, FAKE, pp, 257, 1, 16, 256, None, 0, None) == 1    # R > 256
    bad = (ctypes.c_void_p * 2)(0x10000, 0)
    assert grp(pp, ctypes.cast(bad, ctypes.c_void_p), FAKE, pp, 2, 1, 16, 256, None, 0, None) == 1


def test_int4_validation(L):
    g = L.lowbit_int4g64_gemm
    assert g(FAKE, FAKE, FAKE, FAKE, 1, 16, 96, None) == 3    # K % 64
    assert g(FAKE, FAKE, FAKE, FAKE, 0, 16, 64, None) == 1
    assert g(FAKE, None, FAKE, FAKE, 1, 16, 64, None) == 1
    assert g(FAKE, FAKE, FAKE, MIS, 1, 16, 64, None) == 2


def test_q2_and_glue_validation(L):
    layers = (ctypes.c_void_p * 3)(0x10000, 0x10000, 0x10000)
    dims = (ctypes.c_int32 * 4)(256, 192, 128, 40)
    lp = ctypes.cast(layers, ctypes.c_void_p)
    dp = ctypes.cast(dims, ctypes.c_void_p)
    f = L.lowbit_q2_mlp_forward
    assert f(lp, dp, 3, FAKE, 0, FAKE, None, None) == 0                 # empty batch
    assert f(lp, dp, 0, FAKE, 4, FAKE, None, None) == 1                 # no layers
    assert f(lp, dp, 3, FAKE, 4, None, None, None) == 1                 # null logits
    bad = (ctypes.c_int32 * 4)(250, 192, 128, 40)
    assert f(lp, ctypes.cast(bad, ctypes.c_void_p), 3, FAKE, 4, FAKE, None, None) == 3
    big = (ctypes.c_int32 * 4)(1024, 1024, 1024, 40)                    # 512 KiB of weights
    assert f(lp, ctypes.cast(big, ctypes.c_void_p), 3, FAKE, 4, FAKE, None, None) == 3
    mis = (ctypes.c_void_p * 3)(0x10000, 0x10004, 0x10000)
    assert f(ctypes.cast(mis, ctypes.c_void_p), dp, 3, FAKE, 4, FAKE, None, None) == 2
    n = L.lowbit_rmsnorm_bf16
    assert n(FAKE, None, 1, 12, 1e-6, FAKE, None) == 3
    assert n(FAKE, None, 1, 16, -1.0, FAKE, None) == 1
    assert n(FAKE, MIS, 1, 16, 1e-6, FAKE, None) == 2


def test_quantize_validation(L):
    q = L.lowbit_quantize
    assert q(7, FAKE, 4, 128, FAKE, FAKE, None) == 1                   # bad format
    assert q(2, FAKE, 4, 128, FAKE, FAKE, None) == 3                   # Q2: no rule on the pages
    assert q(1, FAKE, 4, 64, FAKE, FAKE, None) == 3                    # Q1: cols % 128
    assert q(3, FAKE, 4, 96, FAKE, FAKE, None) == 3                    # INT4: cols % 64
    assert q(1, None, 4, 128, FAKE, FAKE, None) == 1                   # null weights
    assert q(3, FAKE, 4, 128, FAKE, None, None) == 1                   # null scales
    assert q(1, FAKE, 4, 128, MIS, FAKE, None) == 2                    # misaligned output
    assert q(1, None, 0, 128, None, None, None) == 0                   # empty: no-op
    assert q(3, FAKE, -1, 128, FAKE, FAKE, None) == 1


def test_group_validation(L):
    ptrs = (ctypes.c_void_p * 2)(0x10000, 0x10000)
    pp = ctypes.cast(ptrs, ctypes.c_void_p)
    misp = ctypes.cast((ctypes.c_void_p * 2)(0x10000, 0x10008), ctypes.c_void_p)
    g = L.lowbit_q1g128_gemv_group
    assert g(pp, pp, FAKE, pp, 0, 1, 16, 256, None, 0, None) == 1       # R < 1
    assert g(pp, pp, FAKE, pp, 257, 1, 16, 256, None, 0, None) == 1     # R > 256
    assert g(pp, pp, None, pp, 2, 1, 16, 256, None, 0, None) == 1       # null x
    assert g(pp, pp, MIS, pp, 2, 1, 16, 256, None, 0, None) == 2        # misaligned x
    assert g(pp, pp, FAKE, misp, 2, 1, 16, 256, None, 0, None) == 2     # misaligned y[1]
    assert g(pp, pp, FAKE, pp, 2, 1, 16, 200, None, 0, None) == 3       # K % 128
    assert g(pp, pp, FAKE, pp, 2, 17, 16, 256, None, 0, None) == 1      # M > 16
    # a small group needs the prepared activation in the workspace
    need = L.lowbit_q1g128_group_workspace_bytes(2, 1, 16, 256)
    assert need > 0
    assert g(pp, pp, FAKE, pp, 2, 1, 16, 256, None, need, None) == 1
    assert g(pp, pp, FAKE, pp, 2, 1, 16, 256, FAKE, need - 1, None) == 1
    # groups the persistent kernels take need none (148 SMs when no device is visible)
    assert L.lowbit_q1g128_group_workspace_bytes(10, 1, 4096, 1024) == 0
    assert L.lowbit_q1g128_group_workspace_bytes(40, 4, 4096, 1024) == 0
    assert L.lowbit_q1g128_group_workspace_bytes(40, 16, 4096, 1024) == 0
    i = L.lowbit_int4g64_gemm_group
    assert i(pp, pp, FAKE, pp, 0, 1, 16, 128, None) == 1       # R < 1
    assert i(pp, pp, None, pp, 2, 1, 16, 128, None) == 1       # null x
    assert i(pp, pp, FAKE, misp, 2, 1, 16, 128, None) == 2     # misaligned y[1]
    assert i(pp, pp, FAKE, pp, 2, 1, 16, 96, None) == 3        # K % 64


def test_stack_step_validation(L):
    """Every case fails before the pointer loop, so nothing reaches a launch."""
    ptrs = (ctypes.c_void_p * 14)(*([0x10000] * 14))
    pp = ctypes.cast(ptrs, ctypes.c_void_p)
    s = L.lowbit_q1g128_stack_step
    ws = L.lowbit_q1g128_stack_workspace_bytes(2, 1536, 2560)
    assert ws >= 256 + 2 * 2560 * 4
    assert s(pp, pp, 2, 1536, 2560, None, 1e-6, FAKE, ws, None, None, None) == 1      # null x
    assert s(pp, pp, 0, 1536, 2560, FAKE, 1e-6, FAKE, ws, None, None, None) == 1      # no layers
    assert s(pp, pp, 74, 1536, 2560, FAKE, 1e-6, FAKE, ws, None, None, None) == 1     # too many layers
    assert s(pp, pp, 2, 2560, 1536, FAKE, 1e-6, FAKE, ws, None, None, None) == 1      # ffn < hidden
    assert s(pp, pp, 2, 768, 2560, FAKE, 1e-6, FAKE, ws, None, None, None) == 3       # hidden % 512
    assert s(pp, pp, 2, 1536, 2816, FAKE, 1e-6, FAKE, ws, None, None, None) == 3      # ffn % 512
    assert s(pp, pp, 2, 1536, 2560, FAKE, 1e-6, FAKE, ws - 1, None, None, None) == 1  # workspace too small
    assert s(pp, pp, 2, 1536, 2560, MIS, 1e-6, FAKE, ws, None, None, None) == 2       # misaligned x


def test_z80_generate_validation(L):
    layers = (ctypes.c_void_p * 3)(0x10000, 0x10000, 0x10000)
    lp = ctypes.cast(layers, ctypes.c_void_p)
    dims = (ctypes.c_int32 * 4)(256, 192, 128, 40)
    dp = ctypes.cast(dims, ctypes.c_void_p)
    cs = ctypes.create_string_buffer(40)
    csp = ctypes.cast(cs, ctypes.c_void_p)
    f = L.lowbit_z80_generate
    assert f(lp, dp, 3, FAKE, 0, 32, csp, 8, FAKE, FAKE, None) == 0         # no conversations: no-op
    assert f(lp, dp, 3, FAKE, 4, 32, None, 8, FAKE, FAKE, None) == 1        # no character set
    assert f(lp, dp, 3, FAKE, 4, 0, csp, 8, FAKE, FAKE, None) == 1          # qlen < 1
    assert f(lp, dp, 3, FAKE, 4, 32, csp, 251, FAKE, FAKE, None) == 1       # max_new > 250
    assert f(lp, dp, 3, FAKE, 4, 32, csp, 8, None, FAKE, None) == 1         # null reply
    assert f(lp, dp, 3, MIS, 4, 32, csp, 8, FAKE, FAKE, None) == 2          # misaligned queries
    bad = (ctypes.c_int32 * 4)(128, 192, 128, 40)                           # input is not 256 buckets
    assert f(lp, ctypes.cast(bad, ctypes.c_void_p), 3, FAKE, 4, 32, csp, 8, FAKE, FAKE, None) == 3
    wide = (ctypes.c_int32 * 4)(256, 512, 128, 40)                          # a width above 256
    assert f(lp, ctypes.cast(wide, ctypes.c_void_p), 3, FAKE, 4, 32, csp, 8, FAKE, FAKE, None) == 3
