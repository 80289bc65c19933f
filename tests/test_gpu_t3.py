"""GPU parity of the ternary format (FP16 scale per 128, base-3 bytes):
packing and unpacking bit-exact against the oracle, and the product within
the float bar (relative L2 <= 1e-5, per element |diff| <= 2e-3 sum|w x|)
against the FP64 oracle, through the C ABI: the streaming kernel (single
calls with K slices, grouped calls, ragged row blocks), the plain kernel for
other shapes, special activations and the benchmark's grouped launch."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import check_float, dev, host, sample_pairs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lb(cuda_device):
    from decode_packed_bit_b200 import build
    build.build()
    from decode_packed_bit_b200 import lowbit
    return lowbit


@pytest.mark.parametrize("rows,cols", [(1, 128), (37, 1024), (300, 1152), (5, 4096)])
def test_t3_pack_unpack_bitexact(lb, rows, cols):
    codes = synth.t3_codes(200 + rows, rows, cols)
    ref = oracle.pack("t3", codes)
    packed = torch.zeros(ref.shape, dtype=torch.uint8, device="cuda")
    lb.lowbit_pack("t3", dev(codes), packed)
    back = torch.zeros((rows, cols), dtype=torch.int8, device="cuda")
    lb.lowbit_unpack("t3", packed, back)
    torch.cuda.synchronize()
    assert np.array_equal(host(packed), ref)
    assert np.array_equal(host(back), codes)


def test_t3_unpack_every_byte_value(lb):
    # every byte value (valid or not) at every position of a group
    packed = np.zeros((256, 32), np.uint8)
    packed[:, :26] = (np.arange(256)[:, None] + np.arange(26)[None, :] * 7) % 256
    packed = np.ascontiguousarray(packed[:, :26])
    ref = oracle.unpack("t3", packed, 128)
    out = torch.zeros((256, 128), dtype=torch.int8, device="cuda")
    pk = torch.zeros((256, 32), dtype=torch.uint8, device="cuda")
    pk[:, :26] = dev(packed)
    lb.lowbit_unpack("t3", pk[:, :26].contiguous(), out)
    torch.cuda.synchronize()
    assert np.array_equal(host(out), ref)


def _run(lb, packed, scales, x, N):
    M, K = x.shape
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    lb.lowbit_t3g128_gemv(dev(packed), dev(scales), dev(x), y)
    torch.cuda.synchronize()
    return host(y)


@pytest.mark.parametrize("M", [1, 2, 5])
@pytest.mark.parametrize("N,K", [(1, 128), (333, 384), (77, 1024), (1000, 2048), (40, 3072)])
def test_t3_small_full_compare(lb, M, N, K):
    codes = synth.t3_codes(300 + N + M, N, K)
    packed = oracle.pack("t3", codes)
    scales = synth.q1_scales(300 + N, N, K)
    x = synth.bf16_normal(300 + M, (M, K))
    y = _run(lb, packed, scales, x, N)
    y64, ab = oracle.t3_gemv(packed, scales, x, want_abs=True)
    check_float(y, y64, ab, f"t3 M={M} N={N} K={K}")


@pytest.mark.parametrize("N,K", [(4096, 4096), (5120, 5120), (17408, 5120), (5120, 17408), (100, 8192)])
def test_t3_m1_streaming_sampled(lb, N, K):
    """Single calls on the streaming kernel: too few row blocks to fill the
    GPU, so K is cut into slices whose partial sums are added."""
    packed, scales = synth.torch_t3_layer(400, N, K, N + K, torch.device("cuda"))
    x = synth.bf16_normal(400 + K, (1, K))
    y = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
    lb.lowbit_t3g128_gemv(packed, scales.view(torch.int16), dev(x), y)
    torch.cuda.synchronize()
    yh = host(y)
    assert np.isfinite(yh).all()
    ms, ns = sample_pairs(1, N, 200, K)
    y64, ab = oracle.t3_gemv_at(host(packed), host(scales.view(torch.int16)).view(np.uint16), x, ms, ns)
    check_float(yh[ms, ns], y64, ab, f"t3 single {N}x{K}")


@pytest.mark.parametrize("R,N,K,xkind", [(169, 4096, 4096, "normal"), (40, 1000, 2048, "normal"),
                                         (20, 4096, 1024, "extreme"), (3, 515, 1152, "normal")])
def test_t3_group(lb, R, N, K, xkind):
    """Grouped calls: the benchmark's launch (169 sets of 4096x4096), ragged
    row blocks, large and tiny activations in one group, and a K the
    streaming kernel does not take."""
    mats = [synth.torch_t3_layer(500 + R, N, K, r, torch.device("cuda")) for r in range(R)]
    x = synth.bf16_normal(500 + R, (1, K)).copy()
    if xkind == "extreme":
        x[0, ::3] = synth.to_bf16_bits(np.full(len(x[0, ::3]), 3.0e4))
        x[0, 1::7] = synth.to_bf16_bits(np.full(len(x[0, 1::7]), 1.0e-20))
    ys = [torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(R)]
    lb.lowbit_t3g128_gemv_group([m for m, _ in mats], [s.view(torch.int16) for _, s in mats], dev(x), ys)
    torch.cuda.synchronize()
    assert all(bool(torch.isfinite(y).all()) for y in ys)
    for r in (0, R // 2, R - 1):
        p, s = host(mats[r][0]), host(mats[r][1].view(torch.int16)).view(np.uint16)
        ms, ns = sample_pairs(1, N, 128, r)
        y64, ab = oracle.t3_gemv_at(p, s, x, ms, ns)
        check_float(host(ys[r])[ms, ns], y64, ab, f"t3 group R={R} {N}x{K} r={r}")


def test_t3_special_inputs(lb):
    N, K = 64, 1024
    codes = synth.t3_codes(600, N, K)
    packed = oracle.pack("t3", codes)
    scales = synth.q1_scales(600, N, K)
    zero = np.zeros((1, K), np.uint16)
    assert np.array_equal(_run(lb, packed, scales, zero, N), np.zeros((1, N), np.float32))
    for k in (0, 4, 5, 124, 125, 127, 128, 1023):
        onehot = np.zeros((1, K), np.uint16)
        onehot[0, k] = 0x3F80
        y = _run(lb, packed, scales, onehot, N)[0]
        ref = np.array([oracle.t3_weight(packed, scales, K, n, k) for n in range(N)])
        assert np.array_equal(y.astype(np.float64), ref), k
