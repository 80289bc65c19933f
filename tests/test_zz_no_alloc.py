"""The allocation-free Q1 entry point, through the C ABI.

lowbit_q1g128_gemv_noalloc serves callers that cannot allocate device memory
(it keeps its scratch in a fixed array inside the library).  This file is
collected last on purpose: if it fails, a run that stops at the first
failure has already run every other test.  It must pass both alone in a
fresh process and after the rest of the suite."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from parity_util import check_float, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(cuda_device):
    from decode_packed_bit_b200 import build
    build.build()
    from decode_packed_bit_b200 import lowbit
    return lowbit.lib()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _reference(L, bits, scales, x, y):
    """The existing entry point, with a caller-provided workspace."""
    M, K = x.shape
    N = bits.shape[0]
    nws = L.lowbit_q1g128_workspace_bytes(M, N, K)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.lowbit_q1g128_gemv(_p(bits), _p(scales), _p(x), _p(y), M, N, K, _p(ws), nws, st) == 0


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(L):
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two different problems back to back: the second call reuses the array
    # the first one left filled
    for call, (N, K, seed) in enumerate([(4096, 4096, 71), (1000, 5120, 72)]):
        scales_h = synth.q1_scales(seed, N, K)
        x_h = synth.bf16_normal(seed, (1, K))
        bits = dev(synth.q1_packed_random(seed, N, K))
        scales = dev(scales_h)
        x = dev(x_h)
        y_new = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
        y_ref = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
        assert L.lowbit_q1g128_gemv_noalloc(_p(bits), _p(scales), _p(x), _p(y_new), 1, N, K, st) == 0
        _reference(L, bits, scales, x, y_ref)
        torch.cuda.synchronize()
        a, b = host(y_new)[0].astype(np.float64), host(y_ref)[0].astype(np.float64)
        # sum_k |w x| = sum_g d[n][g] * sum_{k in g} |x_k| (every |w| is the group scale)
        xabs = np.abs(synth.bf16_bits_to_f32(x_h[0]).astype(np.float64)).reshape(K // 128, 128).sum(axis=1)
        absdot = scales_h.view(np.float16).astype(np.float64) @ xabs
        # the float bar of the parity tests, with the existing entry point as reference
        check_float(a, b, absdot, f"noalloc call {call}")


def test_noalloc_rejects_k_beyond_its_scratch(L):
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    fake = ctypes.c_void_p(0x10000)
    # validation fails before anything is launched
    assert L.lowbit_q1g128_gemv_noalloc(fake, fake, fake, fake, 1, 16, 32768 + 256, st) == 3
