"""The allocation-free Q1 entry point, through the C ABI.

lowbit_q1g128_gemv_noalloc serves callers that cannot allocate device memory
(a plugin under a host framework that owns every device allocation, or a
deployment that reserves all device memory up front): where its product
needs scratch it uses a fixed array inside the library instead of a caller
workspace.  This file is collected last on purpose: if it fails, a run that
stops at the first failure has already run every other test.  It must pass
both alone in a fresh process and after the rest of the suite.

Every buffer handed to the library here is a real device allocation of the
size the shape needs, so even a wrong status could not make a kernel touch
memory it does not own."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import check_float, dev, host, sample_pairs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(cuda_device):
    from decode_packed_bit_b200 import build
    build.build()
    from decode_packed_bit_b200 import lowbit
    return lowbit.lib()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _reference(L, bits, scales, x, y):
    """The existing entry point, with a caller-provided workspace."""
    M, K = x.shape
    N = bits.shape[0]
    nws = L.lowbit_q1g128_workspace_bytes(M, N, K)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    assert L.lowbit_q1g128_gemv(_p(bits), _p(scales), _p(x), _p(y), M, N, K, _p(ws), nws, _stream()) == 0


def _scratch_rows():
    """Rows of a single M = 1 matrix large enough that the product takes the
    persistent kernel, which reads a prepared activation (the scratch)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return 2 * sms * 2 * 8 * 32


def test_noalloc_matches_workspace_entry_and_oracle_on_two_calls_in_a_row(L):
    # Three calls back to back: the first and last go through the library's
    # scratch array (the second one reusing what the first left there), the
    # middle one is a one-launch shape that needs no scratch.
    big = _scratch_rows()
    cases = [(big, 1024, 71), (4096, 4096, 72), (big, 2048, 73)]
    assert L.lowbit_q1g128_workspace_bytes(1, big, 1024) > 0      # these shapes do use scratch
    assert L.lowbit_q1g128_workspace_bytes(1, 4096, 4096) == 0
    for call, (N, K, seed) in enumerate(cases):
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        bits = torch.randint(0, 256, (N, K // 8), generator=g, device="cuda", dtype=torch.uint8)
        scales = (torch.randn((N, K // 128), generator=g, device="cuda") * 0.02).abs().half().view(torch.int16)
        x_h = synth.bf16_normal(seed, (1, K))
        x = dev(x_h)
        y_new = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
        y_ref = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
        assert L.lowbit_q1g128_gemv_noalloc(_p(bits), _p(scales), _p(x), _p(y_new), 1, N, K, _stream()) == 0
        _reference(L, bits, scales, x, y_ref)
        torch.cuda.synchronize()
        a, b = host(y_new)[0].astype(np.float64), host(y_ref)[0].astype(np.float64)
        assert np.isfinite(a).all(), f"call {call}: an output was not written"
        # against the existing entry point: the float bar, with sum |w x| as scale
        b_np, s_np = host(bits), host(scales).view(np.uint16)
        xabs = np.abs(synth.bf16_bits_to_f32(x_h[0]).astype(np.float64)).reshape(K // 128, 128).sum(axis=1)
        absdot = s_np.view(np.float16).astype(np.float64) @ xabs
        check_float(a, b, absdot, f"noalloc call {call} vs workspace entry")
        # against the FP64 oracle, on sampled rows (first and last included)
        ms, ns = sample_pairs(1, N, 256, seed)
        y64, ab = oracle.q1_gemv_at(b_np, s_np, x_h, ms, ns)
        check_float(a[ns], y64, ab, f"noalloc call {call} vs oracle")


def test_noalloc_rejects_k_beyond_its_scratch(L):
    N, K = 16, 32768 + 256
    bits = torch.zeros((N, K // 8), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((N, K // 128), dtype=torch.int16, device="cuda")
    x = torch.zeros((1, K), dtype=torch.int16, device="cuda")
    y = torch.full((1, N), -7.0, dtype=torch.float32, device="cuda")
    assert L.lowbit_q1g128_gemv_noalloc(_p(bits), _p(scales), _p(x), _p(y), 1, N, K, _stream()) == 3
    torch.cuda.synchronize()
    assert bool((y == -7.0).all())          # nothing was enqueued
