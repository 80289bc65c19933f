"""GPU parity: every product of the library against the CPU oracle, through
the C ABI, on seeded inputs.  Integer work (packing, the 2-bit MLP) must be
bit-exact; float formats must meet relative L2 <= 1e-5 and per element
|diff| <= 2e-3 * sum|w x| against the FP64 oracle."""
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


def _sync():
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# packing: bit-exact, all formats
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt,per", [("q1", 8), ("q2", 4), ("int4", 2)])
@pytest.mark.parametrize("rows,cols", [(1, 16), (37, 1024), (300, 136 * 8), (5, 4096)])
def test_pack_unpack_bitexact(lb, fmt, per, rows, cols):
    seed = 100 + rows
    if fmt == "q1":
        codes = synth.q1_codes(seed, rows, cols)
    elif fmt == "q2":
        codes = synth.rng(seed, 0).integers(0, 4, size=(rows, cols), dtype=np.int8)
    else:
        codes = synth.int4_codes(seed, rows, cols)
    ref = oracle.pack(fmt, codes)
    packed = torch.zeros((rows, cols // per), dtype=torch.uint8, device="cuda")
    lb.lowbit_pack(fmt, dev(codes), packed)
    back = torch.zeros((rows, cols), dtype=torch.int8, device="cuda")
    lb.lowbit_unpack(fmt, packed, back)
    _sync()
    assert np.array_equal(host(packed), ref)
    assert np.array_equal(host(back), codes)


def _quant_inputs(seed, rows, cols, special):
    g = np.random.default_rng(seed)
    w = (g.standard_normal((rows, cols)) * g.uniform(1e-3, 5.0, (rows, 1))).astype(np.float32)
    if special:
        w[0, :128] = 0.0                                   # a zero group
        w[1, :8] = [-0.0, 0.0, np.nan, np.inf, -np.inf, 1e30, -1e-30, 7.0]
        w[2, :64] = 1e-6                                   # subnormal FP16 scales
        w[3, :64] = 3.0e5                                  # saturating scales
    return w


@pytest.mark.parametrize("fmt,group", [("q1", 128), ("int4", 64)])
@pytest.mark.parametrize("rows,cols,special", [(37, 1280, False), (300, 4096, False), (8, 512, True)])
def test_quantize_bitexact(lb, fmt, group, rows, cols, special):
    """lowbit_quantize against the oracle's quantiser + packer: every packed
    byte and every FP16 scale bit-exact."""
    w = _quant_inputs(5100 + rows, rows, cols, special)
    per = 8 if fmt == "q1" else 2
    packed = torch.zeros((rows, cols // per), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((rows, cols // group), dtype=torch.int16, device="cuda")
    lb.lowbit_quantize(fmt, torch.from_numpy(w).cuda(), packed, scales)
    _sync()
    codes, sref = oracle.q1_quantize(w) if fmt == "q1" else oracle.int4_quantize(w)
    assert np.array_equal(host(scales).view(np.uint16), sref)
    assert np.array_equal(host(packed), oracle.pack(fmt, codes))


def test_quantize_then_product(lb):
    """Quantise on the GPU, then multiply: matches the oracle's product of the
    oracle-quantised weights (same bits in, so the float bar applies)."""
    N, K = 256, 2048
    w = _quant_inputs(5200, N, K, False)
    x = synth.bf16_normal(5200, (1, K))
    bits = torch.zeros((N, K // 8), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((N, K // 128), dtype=torch.int16, device="cuda")
    lb.lowbit_quantize("q1", torch.from_numpy(w).cuda(), bits, sc)
    y = torch.zeros((1, N), dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(16, lb.lowbit_q1g128_workspace_bytes(1, N, K)), dtype=torch.uint8, device="cuda")
    lb.lowbit_q1g128_gemv(bits, sc, dev(x), y, workspace=ws)
    _sync()
    codes, sref = oracle.q1_quantize(w)
    y64, ab = oracle.q1_gemv(oracle.pack("q1", codes), sref, x, want_abs=True)
    check_float(host(y), y64, ab, "quantise then Q1 product")


def test_quantize_rejects_q2_and_ragged(lb):
    from decode_packed_bit_b200.lowbit import LowbitError
    w = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
    out = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((4, 2), dtype=torch.int16, device="cuda")
    with pytest.raises(LowbitError):
        lb.lowbit_quantize("q2", w, out, sc)
    with pytest.raises(LowbitError):
        lb.lowbit_quantize("q1", torch.zeros((4, 96), dtype=torch.float32, device="cuda"), out, sc)


@pytest.mark.parametrize("fmt,per", [("q1", 8), ("q2", 4), ("int4", 2)])
def test_unpack_every_byte_value(lb, fmt, per):
    allb = np.tile(np.arange(256, dtype=np.uint8), 16).reshape(16, 256)   # 16-byte aligned rows
    cols = 256 * per
    ref = oracle.unpack(fmt, allb, cols)
    out = torch.zeros((16, cols), dtype=torch.int8, device="cuda")
    lb.lowbit_unpack(fmt, dev(allb), out)
    repacked = torch.zeros((16, 256), dtype=torch.uint8, device="cuda")
    lb.lowbit_pack(fmt, out, repacked)
    _sync()
    assert np.array_equal(host(out), ref)
    assert np.array_equal(host(repacked), allb)


# ---------------------------------------------------------------------------
# Q1_0_g128
# ---------------------------------------------------------------------------

def _q1_problem(seed, M, N, K):
    codes = synth.q1_codes(seed, N, K)
    bits = oracle.pack("q1", codes)
    scales = synth.q1_scales(seed, N, K)
    x = synth.bf16_normal(seed, (M, K))
    return bits, scales, x


def _run_q1(lb, bits, scales, x, N, use_act=False):
    M, K = x.shape
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    bits_d, scales_d, x_d = dev(bits), dev(scales), dev(x)
    if use_act:
        act = torch.zeros(lb.lowbit_q1g128_act_bytes(M, K), dtype=torch.uint8, device="cuda")
        nws = lb.lowbit_q1g128_act_workspace_bytes(1, M, N, K)
        ws = torch.zeros(nws, dtype=torch.uint8, device="cuda") if nws else None
        lb.lowbit_q1g128_prepare_act(x_d, act)
        lb.lowbit_q1g128_gemv_act(bits_d, scales_d, act, y, M, workspace=ws)
    else:
        nws = lb.lowbit_q1g128_workspace_bytes(M, N, K)
        # garbage-filled on purpose: the one-shot call needs no initialised workspace
        ws = torch.full((nws,), 0xA5, dtype=torch.uint8, device="cuda") if nws else None
        lb.lowbit_q1g128_gemv(bits_d, scales_d, x_d, y, workspace=ws)
    _sync()
    return host(y)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("N,K", [(1, 128), (333, 384), (1000, 1024), (77, 2176)])
def test_q1_small_full_compare(lb, M, N, K):
    bits, scales, x = _q1_problem(1000 + M * 7 + N, M, N, K)
    y = _run_q1(lb, bits, scales, x, N)
    y64, ab = oracle.q1_gemv(bits, scales, x, want_abs=True)
    check_float(y, y64, ab, f"q1 M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [2, 7, 8, 9, 16])
@pytest.mark.parametrize("N,K", [(129, 256), (1000, 2048), (300, 5120), (77, 17408)])
def test_q1_small_batch_tensor_core(lb, M, N, K):
    """2 <= M <= 16 with K % 256 == 0 takes the bf16 tensor-core kernel: one
    or two batch tiles, ragged row blocks, one or several K slices."""
    bits, scales, x = _q1_problem(1700 + M, M, N, K)
    y = _run_q1(lb, bits, scales, x, N)
    if N * K <= 1000 * 2048:
        y64, ab = oracle.q1_gemv(bits, scales, x, want_abs=True)
        check_float(y, y64, ab, f"q1 small-M M={M} N={N} K={K}")
    else:
        ms, ns = sample_pairs(M, N, 160, M)
        y64, ab = oracle.q1_gemv_at(bits, scales, x, ms, ns)
        check_float(y[ms, ns], y64, ab, f"q1 small-M M={M} N={N} K={K}")
    assert np.isfinite(y).all()


@pytest.mark.parametrize("M", [1, 4, 16])
def test_q1_prepared_activation_matches_direct(lb, M):
    N, K = 515, 1280
    bits, scales, x = _q1_problem(2000 + M, M, N, K)
    y1 = _run_q1(lb, bits, scales, x, N)
    y2 = _run_q1(lb, bits, scales, x, N, use_act=True)
    assert np.array_equal(y1, y2)


def test_q1_act_workspace_reused_across_calls(lb):
    """One prepared activation and one split-K workspace shared by several
    products in a row: the arrival counters must come back to zero."""
    K = 4096
    x = synth.bf16_normal(2500, (1, K))
    act = torch.zeros(lb.lowbit_q1g128_act_bytes(1, K), dtype=torch.uint8, device="cuda")
    lb.lowbit_q1g128_prepare_act(dev(x), act)
    ws = torch.zeros(max(lb.lowbit_q1g128_act_workspace_bytes(1, 1, N, K) for N in (4096, 1000, 5120)),
                     dtype=torch.uint8, device="cuda")
    for rep, N in enumerate((4096, 1000, 5120, 4096)):
        bits = synth.q1_packed_random(2500 + rep, N, K)
        scales = synth.q1_scales(2500 + rep, N, K)
        y = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
        lb.lowbit_q1g128_gemv_act(dev(bits), dev(scales), act, y, 1, workspace=ws)
        _sync()
        ms, ns = sample_pairs(1, N, 200, rep)
        y64, ab = oracle.q1_gemv_at(bits, scales, x, ms, ns)
        check_float(host(y)[ms, ns], y64, ab, f"q1 reuse {rep}")
    cnt_region = host(ws)
    assert not np.isnan(host(y)).any()
    del cnt_region


@pytest.mark.parametrize("R,N,K", [(3, 515, 1280), (20, 4096, 4096), (2, 17408, 512), (5, 33, 17408),
                                   (40, 300, 3072), (200, 200, 2048)])
def test_q1_group_matches_oracle_and_single_calls(lb, R, N, K):
    """R matrices that read one prepared activation, in one launch."""
    x = synth.bf16_normal(2600 + R, (1, K))
    x_d = dev(x)
    act = torch.zeros(lb.lowbit_q1g128_act_bytes(1, K), dtype=torch.uint8, device="cuda")
    lb.lowbit_q1g128_prepare_act(x_d, act)
    mats = [(synth.q1_packed_random(2600 + r, N, K), synth.q1_scales(2600 + r, N, K)) for r in range(R)]
    bits_d = [dev(b) for b, _ in mats]
    scales_d = [dev(s) for _, s in mats]
    ys = [torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(R)]
    ws = torch.zeros(max(16, lb.lowbit_q1g128_act_workspace_bytes(R, 1, N, K)), dtype=torch.uint8,
                     device="cuda")
    lb.lowbit_q1g128_gemv_act_group(bits_d, scales_d, act, ys, 1, workspace=ws)
    _sync()
    for r in (0, R // 2, R - 1):
        b, s = mats[r]
        ms, ns = sample_pairs(1, N, 120, r)
        y64, ab = oracle.q1_gemv_at(b, s, x, ms, ns)
        check_float(host(ys[r])[ms, ns], y64, ab, f"q1 group R={R} r={r}")
        # a lone call may split K differently (another fp32 summation order)
        single = _run_q1(lb, b, s, x, N)
        np.testing.assert_allclose(single, host(ys[r]), rtol=0, atol=1e-5 * float(np.abs(host(ys[r])).max()))


@pytest.mark.parametrize("R,N,K,xkind", [(40, 4096, 1024, "normal"), (148, 1024, 5120, "normal"),
                                         (38, 4096, 17408, "normal"), (48, 4096, 2048, "extreme")])
def test_q1_large_group(lb, R, N, K, xkind):
    """Groups with >= 4736 32-row cells: on 148 SMs these take the persistent
    kernel with 1024-k steps.  Sampled rows of three matrices against the
    oracle; every output is finite and written."""
    x = synth.bf16_normal(2700 + R, (1, K)).copy()
    if xkind == "extreme":  # large and tiny activations in the same groups
        x[0, ::3] = synth.to_bf16_bits(np.full(len(x[0, ::3]), 3.0e4))
        x[0, 1::7] = synth.to_bf16_bits(np.full(len(x[0, 1::7]), 1.0e-20))
    act = torch.zeros(lb.lowbit_q1g128_act_bytes(1, K), dtype=torch.uint8, device="cuda")
    lb.lowbit_q1g128_prepare_act(dev(x), act)
    g = torch.Generator(device="cuda")
    g.manual_seed(2700 + R)
    bits_d = [torch.randint(0, 256, (N, K // 8), generator=g, device="cuda", dtype=torch.uint8) for _ in range(R)]
    scales_d = [(torch.randn((N, K // 128), generator=g, device="cuda") * 0.02).abs().half().view(torch.int16)
                for _ in range(R)]
    ys = [torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(R)]
    lb.lowbit_q1g128_gemv_act_group(bits_d, scales_d, act, ys, 1)
    _sync()
    assert all(bool(torch.isfinite(y).all()) for y in ys)
    for r in (0, R // 2, R - 1):
        b, s = host(bits_d[r]), host(scales_d[r]).view(np.uint16)
        ms, ns = sample_pairs(1, N, 96, r)
        y64, ab = oracle.q1_gemv_at(b, s, x, ms, ns)
        check_float(host(ys[r])[ms, ns], y64, ab, f"q1 large group R={R} N={N} K={K} r={r}")


@pytest.mark.parametrize("R,M,N,K", [(40, 1, 4096, 1024), (38, 1, 4096, 17408), (160, 1, 1024, 3072),
                                     (40, 4, 4096, 1024), (40, 2, 4096, 2048), (30, 3, 4096, 1024),
                                     (12, 16, 5120, 5120), (40, 9, 1000, 2048),
                                     (3, 1, 515, 1280), (2, 2, 300, 2048), (10, 8, 256, 1024),
                                     (3, 13, 1100, 512)])
def test_q1_group_from_x(lb, R, M, N, K):
    """lowbit_q1g128_gemv_group: one launch when the shape allows (the first
    eight cases on 148 SMs: the persistent bit-plane kernel for M = 1, 4, 2
    and 3 (four vectors, one of them zero), then the persistent small-batch
    bf16 kernel with ragged rows and a partial batch tile); groups with too
    few row blocks for it at M >= 2 run the split-K kernel, up to 8 matrices
    per launch (the last three cases: 2, 8 + 2 and 3 matrices, ragged rows);
    M = 1 otherwise: prepare + group product in the workspace.  Sampled
    outputs of three matrices against the oracle."""
    x = synth.bf16_normal(2800 + R, (M, K))
    g = torch.Generator(device="cuda")
    g.manual_seed(2800 + R)
    bits_d = [torch.randint(0, 256, (N, K // 8), generator=g, device="cuda", dtype=torch.uint8) for _ in range(R)]
    scales_d = [(torch.randn((N, K // 128), generator=g, device="cuda") * 0.02).abs().half().view(torch.int16)
                for _ in range(R)]
    ys = [torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(R)]
    need = lb.lowbit_q1g128_group_workspace_bytes(R, M, N, K)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda") if need else None
    lb.lowbit_q1g128_gemv_group(bits_d, scales_d, dev(x), ys, workspace=ws)
    _sync()
    assert all(bool(torch.isfinite(y).all()) for y in ys)
    for r in (0, R // 2, R - 1):
        b, s = host(bits_d[r]), host(scales_d[r]).view(np.uint16)
        ms, ns = sample_pairs(M, N, 96, r)
        y64, ab = oracle.q1_gemv_at(b, s, x, ms, ns)
        check_float(host(ys[r])[ms, ns], y64, ab, f"q1 group from x R={R} M={M} N={N} K={K} r={r}")


def test_q1_special_inputs(lb):
    N, K = 64, 512
    bits, scales, _ = _q1_problem(3000, 1, N, K)
    zero = np.zeros((1, K), np.uint16)
    assert np.array_equal(_run_q1(lb, bits, scales, zero, N), np.zeros((1, N), np.float32))
    for k in (0, 5, 127, 128, 511):
        onehot = np.zeros((1, K), np.uint16)
        onehot[0, k] = 0x3F80
        y = _run_q1(lb, bits, scales, onehot, N)[0]
        ref = np.array([oracle.q1_weight(bits, scales, K, n, k) for n in range(N)])
        assert np.array_equal(y.astype(np.float64), ref)
    # extreme magnitudes: large and tiny activations in the same group
    x = synth.bf16_normal(3001, (1, K)).copy()
    x[0, ::3] = synth.to_bf16_bits(np.full(len(x[0, ::3]), 3.0e4))
    x[0, 1::7] = synth.to_bf16_bits(np.full(len(x[0, 1::7]), 1.0e-20))
    y = _run_q1(lb, bits, scales, x, N)
    y64, ab = oracle.q1_gemv(bits, scales, x, want_abs=True)
    check_float(y, y64, ab, "q1 extreme magnitudes")


def test_q1_4096_square_full(lb):
    """The 4096x4096 M=1 GEMV, every output compared."""
    seed = synth.SEED_BASE + synth.W_Q1_4096
    bits, scales, x = _q1_problem(seed, 1, 4096, 4096)
    y = _run_q1(lb, bits, scales, x, 4096)
    y64, ab = oracle.q1_gemv(bits, scales, x, want_abs=True)
    check_float(y, y64, ab, "q1 4096^2")


@pytest.mark.parametrize("shape", synth.Q1_SWEEP_SHAPES)
@pytest.mark.parametrize("M", [1, 4, 16])
def test_q1_layer_shapes_sampled(lb, shape, M):
    N, K = shape
    seed = synth.SEED_BASE + synth.W_Q1_SWEEP
    bits = synth.q1_packed_random(seed, N, K, tag=N + K)
    scales = synth.q1_scales(seed, N, K, tag=N + K)
    x = synth.bf16_normal(seed, (M, K), tag=M)
    y = _run_q1(lb, bits, scales, x, N)
    ms, ns = sample_pairs(M, N, 160, seed + M)
    y64, ab = oracle.q1_gemv_at(bits, scales, x, ms, ns)
    check_float(y[ms, ns], y64, ab, f"q1 {shape} M={M}")


# ---------------------------------------------------------------------------
# INT4_G64
# ---------------------------------------------------------------------------

def _run_int4(lb, q, scales, x, N):
    M, K = x.shape
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    lb.lowbit_int4g64_gemm(dev(q), dev(scales), dev(x), y)
    _sync()
    return host(y)


@pytest.mark.parametrize("M", [2, 9, 17, 32])
@pytest.mark.parametrize("N,K", [(129, 128), (300, 4096), (77, 11008)])
def test_int4_small_batch_tensor_core(lb, M, N, K):
    """2 <= M <= 32 with K % 128 == 0 takes the bf16 tensor-core kernel: one
    to four batch tiles, ragged row blocks, one or several K slices."""
    seed = 4400 + M * 7 + N
    codes = synth.int4_codes(seed, N, K)
    q = oracle.pack("int4", codes)
    scales = synth.int4_scales(seed, N, K)
    x = synth.bf16_normal(seed, (M, K))
    y = _run_int4(lb, q, scales, x, N)
    y64, ab = oracle.int4_gemv(q, scales, x, want_abs=True)
    check_float(y, y64, ab, f"int4 small-M M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [1, 2, 7, 16, 32, 33, 64, 128, 130, 256, 300])
@pytest.mark.parametrize("N,K", [(1, 64), (333, 448), (1000, 1024)])
def test_int4_small_full_compare(lb, M, N, K):
    seed = 4000 + M * 13 + N
    codes = synth.int4_codes(seed, N, K)
    q = oracle.pack("int4", codes)
    scales = synth.int4_scales(seed, N, K)
    x = synth.bf16_normal(seed, (M, K))
    y = _run_int4(lb, q, scales, x, N)
    y64, ab = oracle.int4_gemv(q, scales, x, want_abs=True)
    check_float(y, y64, ab, f"int4 M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [1, 32, 256])
def test_int4_11008x4096_sampled(lb, M):
    seed = synth.SEED_BASE + synth.W_INT4
    N, K = synth.INT4_N, synth.INT4_K
    codes = synth.int4_codes(seed, N, K)
    q = oracle.pack("int4", codes)
    scales = synth.int4_scales(seed, N, K)
    x = synth.bf16_normal(seed, (M, K), tag=M)
    y = _run_int4(lb, q, scales, x, N)
    ms, ns = sample_pairs(M, N, 200, seed + M)
    y64, ab = oracle.int4_gemv_at(q, scales, x, ms, ns)
    check_float(y[ms, ns], y64, ab, f"int4 11008x4096 M={M}")
    assert lb.lowbit_fault_flags() == 0


@pytest.mark.parametrize("R,M,N,K", [(17, 1, 11008, 4096), (80, 1, 1024, 1024), (7, 1, 11008, 11008),
                                     (17, 32, 11008, 4096), (40, 5, 1000, 1024), (10, 17, 4096, 512),
                                     (40, 1, 1024, 1024), (3, 32, 300, 512), (2, 1, 300, 448),
                                     (10, 8, 256, 512), (9, 24, 1000, 256)])
def test_int4_group(lb, R, M, N, K):
    """lowbit_int4g64_gemm_group: the persistent kernels for the first six
    cases on 148 SMs (M = 1, then small batches with ragged rows and partial
    batch tiles); at 2 <= M <= 32 groups with too few row blocks run the
    split-K kernel, up to 8 matrices per launch (3, 8 + 2 and 8 + 1 matrices
    here); single calls for the rest.  Sampled outputs of three
    matrices against the oracle, and the group equals single calls up to fp32
    summation order."""
    x = synth.bf16_normal(4800 + R, (M, K))
    g = torch.Generator(device="cuda")
    g.manual_seed(4800 + R)
    q_d = [torch.randint(0, 256, (N, K // 2), generator=g, device="cuda", dtype=torch.uint8) for _ in range(R)]
    s_d = [(torch.randn((N, K // 64), generator=g, device="cuda") * 0.01).abs().half().view(torch.int16)
           for _ in range(R)]
    ys = [torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(R)]
    x_d = dev(x)
    lb.lowbit_int4g64_gemm_group(q_d, s_d, x_d, ys)
    _sync()
    assert all(bool(torch.isfinite(y).all()) for y in ys)
    for r in (0, R // 2, R - 1):
        q, s = host(q_d[r]), host(s_d[r]).view(np.uint16)
        ms, ns = sample_pairs(M, N, 96, r)
        y64, ab = oracle.int4_gemv_at(q, s, x, ms, ns)
        check_float(host(ys[r])[ms, ns], y64, ab, f"int4 group R={R} M={M} N={N} K={K} r={r}")
        single = torch.empty((M, N), dtype=torch.float32, device="cuda")
        lb.lowbit_int4g64_gemm(q_d[r], s_d[r], x_d, single)
        _sync()
        ref = host(ys[r])
        np.testing.assert_allclose(host(single), ref, rtol=0, atol=1e-5 * float(np.abs(ref).max()))
    assert lb.lowbit_fault_flags() == 0


# ---------------------------------------------------------------------------
# Z80-style 2-bit MLP: bit-exact
# ---------------------------------------------------------------------------

def _run_q2(lb, packed, dims, x, with_argmax=True):
    batch = x.shape[0]
    logits = torch.full((batch, dims[-1]), -1, dtype=torch.int16, device="cuda")
    am = torch.full((batch,), -1, dtype=torch.int32, device="cuda") if with_argmax else None
    w_d = [dev(p) for p in packed]
    lb.lowbit_q2_mlp_forward(w_d, dims, dev(x), logits, am)
    _sync()
    return host(logits), (host(am) if with_argmax else None)


def test_q2_mlp_1024_vectors_bitexact(lb):
    seed = synth.SEED_BASE + synth.W_Q2_MLP
    dims = synth.Q2_DIMS
    packed = [oracle.pack("q2", c) for c in synth.q2_codes(seed, dims)]
    x = synth.q2_inputs(seed, 1024)
    logits, am = _run_q2(lb, packed, dims, x)
    ref_l, ref_a = oracle.q2_mlp_forward(packed, dims, x)
    assert np.array_equal(logits, ref_l)
    assert np.array_equal(am, ref_a)


@pytest.mark.parametrize("batch", [1, 7, 9, 100, 5000])
def test_q2_mlp_ragged_batches_and_overflow(lb, batch):
    dims = (256, 192, 128, 40)
    packed = [oracle.pack("q2", c) for c in synth.q2_codes(77, dims)]
    g = synth.rng(77, 5)
    x = g.integers(-32768, 32768, size=(batch, 256)).astype(np.int16)   # forces 16-bit wrap
    logits, am = _run_q2(lb, packed, dims, x)
    ref_l, ref_a = oracle.q2_mlp_forward(packed, dims, x)
    assert np.array_equal(logits, ref_l)
    assert np.array_equal(am, ref_a)
    lg2, none = _run_q2(lb, packed, dims, x, with_argmax=False)
    assert np.array_equal(lg2, ref_l) and none is None


@pytest.mark.parametrize("dims", [(4, 4), (8, 12, 4), (64, 1024, 32, 1), (1024, 16, 1024), (200, 256, 152),
                                  (256, 96, 255 // 4 * 4, 44)])
def test_q2_mlp_other_topologies(lb, dims):
    codes = [synth.rng(88, l).integers(0, 4, size=(dims[l + 1], dims[l]), dtype=np.int8)
             for l in range(len(dims) - 1)]
    packed = [oracle.pack("q2", c) for c in codes]
    x = synth.rng(88, 9).integers(-3000, 3000, size=(19, dims[0])).astype(np.int16)
    logits, am = _run_q2(lb, packed, dims, x)
    ref_l, ref_a = oracle.q2_mlp_forward(packed, dims, x)
    assert np.array_equal(logits, ref_l)
    assert np.array_equal(am, ref_a)


# ---------------------------------------------------------------------------
# RMS-norm glue
# ---------------------------------------------------------------------------

def _bf16_ulp(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 1e-38)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("M,D,two", [(1, 5120, False), (8, 17408, True), (3, 64, True)])
def test_rmsnorm_bf16_within_half_ulp(lb, M, D, two):
    g = synth.rng(99, D)
    a = (g.standard_normal((M, D)) * 0.7).astype(np.float32)
    b = g.standard_normal((M, D)).astype(np.float32) if two else None
    out = torch.zeros((M, D), dtype=torch.int16, device="cuda")
    lb.lowbit_rmsnorm_bf16(dev(a), dev(b) if two else None, out, eps=1e-6)
    _sync()
    got = synth.bf16_bits_to_f32(host(out).view(np.uint16)).astype(np.float64)
    r64 = oracle.rmsnorm(a, b, eps=1e-6)
    # round-to-nearest to bf16 of an fp32 result: at most half a bf16 ulp
    # plus the fp32 error of the normalisation itself
    tol = 0.5 * _bf16_ulp(r64) + 1e-6 * np.abs(r64) + 1e-30
    assert (np.abs(got - r64) <= tol).all()


# ---------------------------------------------------------------------------
# the launches bench.py times, in its exact configuration
# ---------------------------------------------------------------------------

def _bench_sets_check(lb, mats, x, ys, what):
    """Sampled outputs of the first, middle and last matrix against the
    oracle; every output of every matrix written and finite."""
    assert all(bool(torch.isfinite(y).all()) for y in ys), f"{what}: an output was not written"
    M = x.shape[0]
    R = len(mats)
    for r in (0, R // 2, R - 1):
        b, s = host(mats[r][0]), host(mats[r][1]).view(np.uint16)
        N = b.shape[0]
        ms, ns = sample_pairs(M, N, 128, 9000 + r)
        y64, ab = oracle.q1_gemv_at(b, s, x, ms, ns)
        check_float(host(ys[r])[ms, ns], y64, ab, f"{what} r={r}")


def test_bench_headline_launch(lb):
    """The headline launch: R = bench.q1_4096_sets(L2) (169 on B200)
    4096x4096 matrices drawn as the bench draws them, one grouped call from
    x, with the workspace the bench passes."""
    import bench
    N = K = 4096
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    R = bench.q1_4096_sets(l2)
    seed = synth.SEED_BASE + synth.W_Q1_4096
    mats = [synth.torch_q1_layer(seed, N, K, r, torch.device("cuda")) for r in range(R)]
    x = synth.bf16_normal(seed, (1, K))
    ys = [torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(R)]
    need = lb.lowbit_q1g128_group_workspace_bytes(R, 1, N, K)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda") if need else None
    lb.lowbit_q1g128_gemv_group([b for b, _ in mats], [s for _, s in mats], dev(x), ys, workspace=ws)
    _sync()
    _bench_sets_check(lb, mats, x, ys, f"bench headline R={R}")
    # the single-call figure's launch: lowbit_q1g128_gemv on one of the matrices
    y1 = torch.full((1, N), float("nan"), dtype=torch.float32, device="cuda")
    nws = lb.lowbit_q1g128_workspace_bytes(1, N, K)
    lb.lowbit_q1g128_gemv(mats[R - 1][0], mats[R - 1][1], dev(x), y1,
                          workspace=torch.zeros(nws, dtype=torch.uint8, device="cuda") if nws else None)
    _sync()
    _bench_sets_check(lb, [mats[R - 1]], x, [y1], "bench single call")


@pytest.mark.parametrize("shape", synth.Q1_SWEEP_SHAPES)
@pytest.mark.parametrize("M", [1, 4, 16])
def test_bench_sweep_launch(lb, shape, M):
    """The layer-shape sweep's grouped launches (108 sets of 5120x5120, 32 of
    the FFN shapes on B200), drawn and sized as the bench does."""
    import bench
    N, K = shape
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    R = bench.sweep_sets(N, K, l2)
    seed = synth.SEED_BASE + synth.W_Q1_SWEEP
    mats = [synth.torch_q1_layer(seed, N, K, r, torch.device("cuda")) for r in range(R)]
    x = synth.bf16_normal(seed, (M, K), tag=M)
    ys = [torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(R)]
    need = lb.lowbit_q1g128_group_workspace_bytes(R, M, N, K)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda") if need else None
    lb.lowbit_q1g128_gemv_group([b for b, _ in mats], [s for _, s in mats], dev(x), ys, workspace=ws)
    _sync()
    _bench_sets_check(lb, mats, x, ys, f"bench sweep {shape} M={M} R={R}")
    del mats, ys
    torch.cuda.empty_cache()
