"""Pins for the CPU oracle: every check here compares the oracle with
something other than itself -- the pages' fixed facts (tests/golden), an
emulation of the Z80 listing's instructions, library routines (numpy's
unpackbits / float16, torch's bfloat16, numpy matmul), closed forms and
brute-force enumeration.  No GPU is used."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden


# ---------------------------------------------------------------------------
# scalar decoders
# ---------------------------------------------------------------------------

def test_f16_decode_all_patterns_match_numpy():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(p)) for p in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decode_all_patterns_match_torch():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_f64(int(p)) for p in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------------------
# Q1_0_g128
# ---------------------------------------------------------------------------

def test_q1_format_facts_from_page():
    g = {r[0]: float(r[1]) for r in read_golden("q1_format.txt")}
    K, N = 4096, 8
    codes = synth.q1_codes(1, N, K)
    packed = oracle.pack("q1", codes)
    scales = synth.q1_scales(1, N, K)
    bits = 8 * (packed.nbytes + scales.nbytes)
    assert bits / (N * K) == g["bits_per_weight"]
    assert g["sign_bits_per_weight"] + g["scale_bits"] / g["group_size"] == g["bits_per_weight"]
    assert round(16 / (bits / (N * K)), 1) == g["ratio_vs_fp16"]
    assert scales.shape == (N, K // int(g["group_size"]))


def test_q1_unpack_all_bytes_matches_numpy_unpackbits():
    allb = np.arange(256, dtype=np.uint8).reshape(256, 1)
    got = oracle.unpack("q1", allb, 8)
    ref = np.unpackbits(allb, axis=1, bitorder="little").astype(np.int8)
    assert np.array_equal(got, ref)
    assert np.array_equal(oracle.pack("q1", got), allb)


def test_q1_pack_roundtrip_random():
    codes = synth.q1_codes(2, 33, 1024)
    p = oracle.pack("q1", codes)
    assert np.array_equal(oracle.unpack("q1", p, 1024), codes)
    with pytest.raises(ValueError):
        oracle.pack("q1", np.full((1, 8), 2, np.int8))


def _np_q1_dense(bits, scales, K):
    signs = np.where(np.unpackbits(bits, axis=1, bitorder="little")[:, :K] == 1, 1.0, -1.0)
    d = np.repeat(scales.view(np.float16).astype(np.float64), 128, axis=1)
    return signs * d


def test_q1_gemv_matches_numpy_matmul():
    M, N, K = 3, 37, 384
    bits = oracle.pack("q1", synth.q1_codes(3, N, K))
    scales = synth.q1_scales(3, N, K)
    x = synth.bf16_normal(3, (M, K))
    y, ab = oracle.q1_gemv(bits, scales, x, want_abs=True)
    W = _np_q1_dense(bits, scales, K)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    np.testing.assert_allclose(y, xf @ W.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ab, np.abs(xf) @ np.abs(W).T, rtol=1e-12)


def test_q1_onehot_probe_reads_back_every_weight():
    N, K = 5, 256
    bits = oracle.pack("q1", synth.q1_codes(4, N, K))
    scales = synth.q1_scales(4, N, K)
    one = 0x3F80  # bf16 1.0
    for k in (0, 1, 7, 8, 127, 128, 200, 255):
        x = np.zeros((1, K), np.uint16)
        x[0, k] = one
        y = oracle.q1_gemv(bits, scales, x)[0]
        for n in range(N):
            bit = (int(bits[n, k // 8]) >> (k % 8)) & 1
            d = float(scales[n, k // 128:k // 128 + 1].view(np.float16)[0])
            assert y[n] == (d if bit else -d)


def test_q1_all_ones_closed_form():
    N, K = 9, 512
    bits = oracle.pack("q1", synth.q1_codes(5, N, K))
    scales = synth.q1_scales(5, N, K)
    x = np.full((1, K), 0x3F80, np.uint16)
    y = oracle.q1_gemv(bits, scales, x)[0]
    for n in range(N):
        exp = 0.0
        for g in range(K // 128):
            pop = sum(bin(int(b)).count("1") for b in bits[n, 16 * g:16 * g + 16])
            exp += float(scales[n, g:g + 1].view(np.float16)[0]) * (2 * pop - 128)
        assert y[n] == exp


def test_q1_unit_scales_integer_x_exact_int64():
    N, K = 16, 256
    codes = synth.q1_codes(6, N, K)
    bits = oracle.pack("q1", codes)
    scales = np.full((N, K // 128), 0x3C00, np.uint16)  # fp16 1.0
    xi = synth.rng(6, 99).integers(-100, 101, size=(2, K))
    x = synth.to_bf16_bits(xi.astype(np.float64))
    y = oracle.q1_gemv(bits, scales, x)
    ref = xi.astype(np.int64) @ (2 * codes.astype(np.int64) - 1).T
    assert np.array_equal(y, ref.astype(np.float64))


def test_q1_bruteforce_all_sign_patterns_of_one_byte():
    # x_k = 2^k on k = 0..7 and 0 elsewhere; sum_k (2 b_k - 1) 2^k = 2 v - 255.
    K = 128
    x = np.zeros((1, K), np.uint16)
    x[0, :8] = synth.to_bf16_bits(2.0 ** np.arange(8))
    scales = np.full((1, 1), 0x3C00, np.uint16)
    for v in range(256):
        bits = np.zeros((1, K // 8), np.uint8)
        bits[0, 0] = v
        assert oracle.q1_gemv(bits, scales, x)[0, 0] == 2 * v - 255


def test_q1_gemv_at_equals_full():
    M, N, K = 2, 11, 256
    bits = oracle.pack("q1", synth.q1_codes(7, N, K))
    scales = synth.q1_scales(7, N, K)
    x = synth.bf16_normal(7, (M, K))
    y = oracle.q1_gemv(bits, scales, x)
    ms = np.array([0, 1, 1, 0])
    ns = np.array([0, 10, 3, 5])
    ys, _ = oracle.q1_gemv_at(bits, scales, x, ms, ns)
    assert np.array_equal(ys, y[ms, ns])


# ---------------------------------------------------------------------------
# INT4-g64
# ---------------------------------------------------------------------------

def test_int4_group_fact_and_layout():
    g = {r[0]: int(r[1]) for r in read_golden("int4_group.txt")}
    assert g["group_size"] == 64 and g["values_per_byte"] == 2
    codes = synth.int4_codes(1, 4, 128)
    assert codes.min() >= g["code_min"] and codes.max() <= g["code_max"]
    scales = synth.int4_scales(1, 4, 128)
    assert scales.shape == (4, 128 // g["group_size"])


def test_int4_unpack_all_bytes_sign_extension():
    allb = np.arange(256, dtype=np.uint8).reshape(256, 1)
    got = oracle.unpack("int4", allb, 2)
    lo = (allb[:, 0].astype(np.int8) << 4) >> 4           # arithmetic shift sign-extends
    hi = allb[:, 0].astype(np.int8) >> 4
    assert np.array_equal(got[:, 0], lo)
    assert np.array_equal(got[:, 1], hi)
    assert np.array_equal(oracle.pack("int4", got), allb)


def test_int4_all_nibble_pairs_roundtrip():
    pairs = np.array([[a, b] for a in range(-8, 8) for b in range(-8, 8)], np.int8)
    p = oracle.pack("int4", pairs)
    assert np.array_equal(oracle.unpack("int4", p, 2), pairs)
    with pytest.raises(ValueError):
        oracle.pack("int4", np.array([[8, 0]], np.int8))


def test_int4_gemv_matches_numpy_matmul():
    M, N, K = 4, 29, 320
    codes = synth.int4_codes(8, N, K)
    q = oracle.pack("int4", codes)
    scales = synth.int4_scales(8, N, K)
    x = synth.bf16_normal(8, (M, K))
    y, ab = oracle.int4_gemv(q, scales, x, want_abs=True)
    W = codes.astype(np.float64) * np.repeat(scales.view(np.float16).astype(np.float64), 64, axis=1)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    np.testing.assert_allclose(y, xf @ W.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ab, np.abs(xf) @ np.abs(W).T, rtol=1e-12)


def _int4_numpy_weights(q, scales, K):
    """Weights decoded with numpy alone: low nibble = even k, high = odd k,
    sign-extended by arithmetic shifts; times the fp16 scale of k // 64."""
    lo = (q.astype(np.int8) << 4) >> 4
    hi = q.astype(np.int8) >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(q.shape[0], K).astype(np.float64)
    return codes * np.repeat(scales.view(np.float16).astype(np.float64), 64, axis=1)


def test_int4_gemv_at_matches_numpy_at_every_element():
    """The sampled-output form checks the INT4 parity tests at full size: at
    every (m, n) of a small product it must equal a numpy matmul of weights
    decoded independently of the oracle (so a wrong row, batch or scale
    index in it fails here)."""
    M, N, K = 3, 13, 448
    q = synth.rng(12, 0).integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = synth.int4_scales(12, N, K)
    x = synth.bf16_normal(12, (M, K))
    W = _int4_numpy_weights(q, scales, K)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = xf @ W.T
    mm, nn = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    ys, ab = oracle.int4_gemv_at(q, scales, x, mm.ravel(), nn.ravel())
    np.testing.assert_allclose(ys, ref.ravel(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ab, (np.abs(xf) @ np.abs(W).T).ravel(), rtol=1e-12)
    # the same elements in the reverse order: no state carried between them
    ys_rev, _ = oracle.int4_gemv_at(q, scales, x, mm.ravel()[::-1], nn.ravel()[::-1])
    assert np.array_equal(ys_rev, ys[::-1])


def test_int4_gemv_at_hand_computed_element():
    """One output worked by hand: row 1 holds q = +3 at k = 0 (low nibble),
    q = -2 at k = 65 (high nibble of byte 32, second group) and 0 elsewhere;
    scales 0.5 and 0.25; x = 1.0 at k = 0 and 2.0 at k = 65, batch row 1.
    y[1][1] = 3 * 0.5 * 1 + (-2) * 0.25 * 2 = 0.5."""
    N, K = 2, 128
    q = np.zeros((N, K // 2), np.uint8)
    q[1, 0] = 0x03            # k = 0: +3
    q[1, 32] = 0xE0           # k = 65: high nibble 0xE = -2
    q[0, :] = 0x77            # row 0: +7 everywhere (must not leak into row 1)
    scales = np.array([[0x3C00, 0x3C00], [0x3800, 0x3400]], np.uint16)   # 1, 1 | 0.5, 0.25
    x = np.zeros((2, K), np.uint16)
    x[1, 0] = 0x3F80          # 1.0
    x[1, 65] = 0x4000         # 2.0
    x[0, :] = 0x3F80          # batch row 0: all ones (must not leak into batch row 1)
    ys, ab = oracle.int4_gemv_at(q, scales, x, np.array([1, 0, 1]), np.array([1, 0, 0]))
    assert ys[0] == 0.5 and ab[0] == 2.5
    assert ys[1] == 7 * 128                       # row 0, all-ones x: 7 per weight, scale 1
    assert ys[2] == 7 * 1.0 + 7 * 2.0             # row 0 against batch row 1


def test_int4_group_isolation_probe():
    # Only group g has a non-zero scale: y must equal d * sum over that group.
    N, K = 3, 256
    codes = synth.int4_codes(9, N, K)
    q = oracle.pack("int4", codes)
    x = np.full((1, K), 0x3F80, np.uint16)
    for g in range(K // 64):
        scales = np.zeros((N, K // 64), np.uint16)
        scales[:, g] = 0x3C00
        y = oracle.int4_gemv(q, scales, x)[0]
        assert np.array_equal(y, codes[:, 64 * g:64 * g + 64].sum(axis=1).astype(np.float64))


# ---------------------------------------------------------------------------
# Z80-style 2-bit integer MLP
# ---------------------------------------------------------------------------

def _z80_unpack_byte(byte):
    """Emulate the page's listing on an 8-bit A register: `and 03h; sub 2`
    gives one weight, `rrca` twice rotates the next field into place."""
    a = byte
    out = []
    for _ in range(4):
        w = ((a & 0x03) - 2) & 0xFF
        out.append(w - 256 if w >= 128 else w)
        for _ in range(2):                      # rrca: bit 0 -> bit 7 and carry
            a = ((a >> 1) | ((a & 1) << 7)) & 0xFF
    return out


def test_q2_code_map_from_page():
    cmap = {int(c): int(w) for c, w in read_golden("q2_code_map.txt")}
    assert cmap == {0: -2, 1: -1, 2: 0, 3: 1}
    for code, w in cmap.items():
        packed = np.array([[code]], np.uint8)   # code in the first field
        assert oracle.unpack("q2", packed, 4)[0, 0] == code
        assert _z80_unpack_byte(code)[0] == w


def test_q2_unpack_matches_z80_listing_for_every_byte():
    cmap = {int(c): int(w) for c, w in read_golden("q2_code_map.txt")}
    allb = np.arange(256, dtype=np.uint8).reshape(256, 1)
    codes = oracle.unpack("q2", allb, 4)
    for v in range(256):
        assert [cmap[int(c)] for c in codes[v]] == _z80_unpack_byte(v)
    assert np.array_equal(oracle.pack("q2", codes), allb)


def _z80_sra2(v16):
    """`sra h; rr l` twice on the 16-bit pair HL, bit by bit."""
    h, l = (v16 >> 8) & 0xFF, v16 & 0xFF
    for _ in range(2):
        carry = h & 1
        h = ((h >> 1) | (h & 0x80)) & 0xFF      # sra h keeps the sign bit
        l = ((l >> 1) | (carry << 7)) & 0xFF    # rr l takes the carry
    v = (h << 8) | l
    return v - 65536 if v >= 32768 else v


def test_q2_shift_matches_z80_sra_rr_pair_exhaustive():
    # out layer with one +1 weight on input 0: acc = a0, out = shift(a0).
    packed = np.array([[0b10101011]], np.uint8)  # codes 3,2,2,2 -> +1,0,0,0
    vals = np.arange(-32768, 32768, 37, dtype=np.int64)
    for v in vals:
        a = np.array([v, 5, -5, 1], np.int16)
        got = int(oracle.q2_layer(packed, 4, 1, a, hidden=False)[0])
        assert got == _z80_sra2(int(v) & 0xFFFF)
        assert got == int(v) // 4


def test_q2_bruteforce_one_byte_all_codes():
    a = np.array([1, 10, 100, 1000], np.int16)
    for v in range(256):
        packed = np.array([[v]], np.uint8)
        ws = _z80_unpack_byte(v)
        acc = sum(w * int(x) for w, x in zip(ws, a))
        got = int(oracle.q2_layer(packed, 4, 1, a, hidden=False)[0])
        assert got == acc // 4


def _np_q2_layer(codes, a, hidden):
    acc = (codes.astype(np.int64) - 2) @ a.astype(np.int64)
    v = ((acc + 32768) % 65536) - 32768
    z = v // 4
    return np.maximum(z, 0) if hidden else z


def test_q2_layer_matches_numpy_and_muladd16_with_overflow():
    g = synth.rng(11, 0)
    for trial in range(20):
        cin, cout = 64, 24
        codes = g.integers(0, 4, size=(cout, cin), dtype=np.int8)
        # large activations force 16-bit wrap-around
        a = g.integers(-32768, 32768, size=cin).astype(np.int16)
        packed = oracle.pack("q2", codes)
        for hidden in (True, False):
            ref = _np_q2_layer(codes, a, hidden)
            assert np.array_equal(oracle.q2_layer(packed, cin, cout, a, hidden), ref)
            assert np.array_equal(oracle.q2_layer(packed, cin, cout, a, hidden, muladd16=True), ref)


def test_q2_forward_matches_numpy_stack_and_relu_placement():
    rows = {r[0]: r[1:] for r in read_golden("q2_topology.txt")}
    dims = tuple(int(d) for d in rows["layers"])
    assert dims == synth.Q2_DIMS
    layers = synth.q2_codes(12, dims)
    packed = [oracle.pack("q2", c) for c in layers]
    x = synth.q2_inputs(12, 64)
    logits, am = oracle.q2_mlp_forward(packed, dims, x)
    logits16, am16 = oracle.q2_mlp_forward(packed, dims, x, muladd16=True)
    assert np.array_equal(logits, logits16) and np.array_equal(am, am16)
    for b in range(x.shape[0]):
        a = x[b].astype(np.int64)
        for l, c in enumerate(layers):
            a = _np_q2_layer(c, a, hidden=(l < len(layers) - 1))
        assert np.array_equal(logits[b], a)
        assert am[b] == int(np.argmax(a))        # numpy argmax: first maximum
    assert (logits < 0).any()                    # no ReLU on the output layer


def test_q2_mac_count_order_from_page():
    rows = {r[0]: r[1:] for r in read_golden("q2_topology.txt")}
    dims = [int(v) for v in rows["layers"]]
    macs = sum(dims[i] * dims[i + 1] for i in range(len(dims) - 1))
    assert macs == 78848
    order = int(rows["macs_per_char_order"][0])
    assert order / 10 < macs < order * 10
    assert int(rows["query_buckets"][0]) + int(rows["context_buckets"][0]) == dims[0]


def test_argmax_ties_lowest_index():
    assert oracle.argmax16(np.array([3, 7, 7, -1], np.int16)) == 1
    assert oracle.argmax16(np.array([-5, -5], np.int16)) == 0


def test_trigram_relations_from_page():
    for rel, a, b in read_golden("trigram_examples.txt"):
        va, vb = oracle.trigram_encode(a), oracle.trigram_encode(b)
        assert va.shape == (128,) and (va % 32 == 0).all() and va.sum() > 0
        if rel == "equal":
            assert np.array_equal(va, vb)
        else:
            shared = np.minimum(va, vb).sum()
            assert shared >= 0.4 * min(va.sum(), vb.sum())
    # case-insensitive and whitespace-insensitive
    assert np.array_equal(oracle.trigram_encode("Hello  There "), oracle.trigram_encode("hello there"))


def test_q2_inputs_shape_the_trigram_distribution():
    x = synth.q2_inputs(13, 32)
    assert x.shape == (32, 256)
    for half in (x[:, :128], x[:, 128:]):
        assert ((half != 0).sum(axis=1) == 8).all()
        assert set(np.unique(half[half != 0]).tolist()) <= {32, 64, 96}


# ---------------------------------------------------------------------------
# RMS normalisation glue
# ---------------------------------------------------------------------------

def test_rmsnorm_matches_numpy_and_closed_forms():
    g = synth.rng(14, 0)
    a = g.standard_normal((3, 640)).astype(np.float32)
    b = g.standard_normal((3, 640)).astype(np.float32)
    for bb in (None, b):
        v = a.astype(np.float64) + (0.0 if bb is None else bb.astype(np.float64))
        ref = v / np.sqrt(np.mean(v * v, axis=1, keepdims=True) + 1e-6)
        np.testing.assert_allclose(oracle.rmsnorm(a, bb), ref, rtol=1e-13)
    c = np.full((1, 64), 3.0, np.float32)
    np.testing.assert_allclose(oracle.rmsnorm(c), 3.0 / np.sqrt(9.0 + 1e-6), rtol=1e-15)
    r = oracle.rmsnorm(a * 1000.0)
    np.testing.assert_allclose(r, oracle.rmsnorm(a), rtol=1e-5)


# ---------------------------------------------------------------------------
# the autoregressive reply loop
# ---------------------------------------------------------------------------

# index 0 ends a reply; then space, A-Z, 0-9, '?', '!' (40 outputs)
CHARSET = np.frombuffer(b"\0 ABCDEFGHIJKLMNOPQRSTUVWXYZ0123456789?!", np.uint8)


def _queries(texts, qlen=32):
    q = np.zeros((len(texts), qlen), np.uint8)
    for i, t in enumerate(texts):
        b = t.encode()
        q[i, :len(b)] = np.frombuffer(b, np.uint8)
    return q


def _counting_net():
    """256 -> 4 -> 40.  Hidden units 0 and 1 sum the 128 context buckets,
    unit 2 the 128 query buckets (weight +1 = code 3; every other weight is
    0 = code 2).  Output 0 (end of reply) adds units 0 and 1, output 2 ('A')
    reads unit 2.  With n query trigrams and a reply of t letters 'A' (one
    word: t trigrams), every trigram adds 32, so after the shifts
    logit[end] = 4 t and logit['A'] = 2 n: the reply is 'A' * ceil(n / 2)."""
    dims = (256, 4, 40)
    c1 = np.full((4, 256), 2, np.int8)
    c1[0, 128:] = 3
    c1[1, 128:] = 3
    c1[2, :128] = 3
    c2 = np.full((40, 4), 2, np.int8)
    c2[0, 0] = 3
    c2[0, 1] = 3
    c2[2, 2] = 3
    return dims, [oracle.pack("q2", c1), oracle.pack("q2", c2)]


def test_reply_loop_closed_form_on_a_counting_network():
    dims, packed = _counting_net()
    texts = ["hi", "hello there", "do you dream", "are you a robot", "x", "abcdefghijklmnopq"]
    reply, lens = oracle.z80_generate(packed, dims, _queries(texts), CHARSET, 40)
    for i, t in enumerate(texts):
        n = sum(len(w) for w in t.split())            # one trigram per letter of a padded word
        want = -(-n // 2)
        assert lens[i] == want, (t, lens[i], want)
        assert bytes(reply[i, :want]) == b"A" * want
        assert not reply[i, want:].any()
    # a cap shorter than the natural length stops the reply there
    reply, lens = oracle.z80_generate(packed, dims, _queries(["abcdefghijklmnopq"]), CHARSET, 3)
    assert lens[0] == 3 and bytes(reply[0]) == b"AAA"


def test_reply_loop_word_order_invariance_from_page():
    """The page: reordered words give the same bucket vector, so the same
    reply; the query's last byte may be used without a terminator."""
    dims = synth.Q2_DIMS
    packed = [oracle.pack("q2", c) for c in synth.q2_codes(31, dims)]
    a = _queries(["hello there", "there hello", "are you a robot", "robot a you are"], qlen=16)
    r, n = oracle.z80_generate(packed, dims, a, CHARSET, 24)
    assert np.array_equal(r[0], r[1]) and n[0] == n[1]
    assert np.array_equal(r[2], r[3]) and n[2] == n[3]
    full = _queries(["abcdefghijklmnop"], qlen=16)      # no terminating 0 inside the row
    r2, n2 = oracle.z80_generate(packed, dims, full, CHARSET, 8)
    r3, n3 = oracle.z80_generate(packed, dims, _queries(["abcdefghijklmnop"], qlen=20), CHARSET, 8)
    assert np.array_equal(r2, r3) and np.array_equal(n2, n3)


def test_reply_loop_degenerate_cases():
    dims = (256, 8, 40)
    zero = [oracle.pack("q2", np.full((8, 256), 2, np.int8)), oracle.pack("q2", np.full((40, 8), 2, np.int8))]
    q = _queries(["hello"])
    # all logits 0: the argmax is output 0, the end symbol: empty reply
    r, n = oracle.z80_generate(zero, dims, q, CHARSET, 10)
    assert n[0] == 0 and not r.any()
    # with no end symbol at index 0, the same network repeats charset[0]
    cs = CHARSET.copy()
    cs[0] = ord("Z")
    r, n = oracle.z80_generate(zero, dims, q, cs, 10)
    assert n[0] == 10 and bytes(r[0]) == b"Z" * 10
    r, n = oracle.z80_generate(zero, dims, q, cs, 0)
    assert r.shape == (1, 0) and n[0] == 0
    with pytest.raises(ValueError):
        oracle.z80_generate(zero, (128, 8, 40), q, CHARSET, 4)   # the input must be 128 + 128 buckets


def test_reply_loop_matches_stepwise_recomposition():
    """The loop against the same steps driven from Python through the
    separately pinned pieces (trigram encoder, network, argmax)."""
    dims = synth.Q2_DIMS
    packed = [oracle.pack("q2", c) for c in synth.q2_codes(32, dims)]
    texts = ["hello", "what is your name", "ok", "r u human", "tell me a joke", ""]
    q = _queries(texts)
    r, n = oracle.z80_generate(packed, dims, q, CHARSET, 30)
    for i, t in enumerate(texts):
        qb = oracle.trigram_encode(t)
        out = ""
        for _ in range(30):
            x = np.concatenate([qb, oracle.trigram_encode(out)])[None, :]
            _, am = oracle.q2_mlp_forward(packed, dims, x)
            ch = int(CHARSET[am[0]])
            if ch == 0:
                break
            out += chr(ch)
        assert n[i] == len(out) and bytes(r[i, :n[i]]) == out.encode(), (t, out)


# ---------------------------------------------------------------------------
# ternary, FP16 scale per 128 (base-3 bytes)
# ---------------------------------------------------------------------------

def _np_t3_codes(packed, K):
    """Codes decoded with numpy alone: group g's byte j < 25 holds k = 5j..5j+4
    as base-3 digits (least significant first), byte 25 holds k = 125..127."""
    N = packed.shape[0]
    G = K // 128
    b = packed.reshape(N, G, 26).astype(np.int64)
    digits = np.stack([(b // 3 ** i) % 3 for i in range(5)], axis=-1)   # [N][G][26][5]
    flat = digits.reshape(N, G, 130)[:, :, :128]                          # byte 25 keeps 3 digits
    return (flat - 1).reshape(N, K).astype(np.int8)


def test_t3_size_matches_the_page():
    g = {r[0]: float(r[1]) for r in read_golden("ternary_size.txt")}
    N, K = 4, 1024
    codes = synth.rng(40, 0).integers(-1, 2, size=(N, K), dtype=np.int8)
    packed = oracle.pack("t3", codes)
    bpw = 8 * (packed.nbytes + 2 * N * K // int(g["group_size"])) / (N * K)
    assert bpw == 1.75
    assert round(g["q1_model_gb"] * bpw / g["q1_bits_per_weight"], 1) == g["ternary_model_gb"]
    # the 2-bit alternative would not fit the page's figure
    two_bit = 2 + g["scale_bits"] / g["group_size"]
    assert round(g["q1_model_gb"] * two_bit / g["q1_bits_per_weight"], 1) != g["ternary_model_gb"]


def test_t3_every_byte_value_decodes_like_numpy_base3():
    # one group per row; byte 7 of row v takes the value v (k = 35..39)
    rows = 243
    packed = np.full((rows, 26), 121, np.uint8)   # 121 = 11111 in base 3: all zero weights
    packed[:, 25] = 13                            # 111 in base 3
    packed[:, 7] = np.arange(rows, dtype=np.uint8)
    got = oracle.unpack("t3", packed, 128)
    assert np.array_equal(got, _np_t3_codes(packed, 128))
    assert not got[:, :35].any() and not got[:, 40:].any()
    # all 3^5 patterns appear once: the byte is a bijection onto {-1,0,1}^5
    assert len({tuple(r) for r in got[:, 35:40]}) == 243
    assert np.array_equal(oracle.pack("t3", got), packed)
    # the last byte of a group: 27 values, three weights
    last = np.full((27, 26), 121, np.uint8)
    last[:, 25] = np.arange(27, dtype=np.uint8)
    got = oracle.unpack("t3", last, 128)
    assert len({tuple(r) for r in got[:, 125:128]}) == 27 and not got[:, :125].any()
    assert np.array_equal(oracle.pack("t3", got), last)


def test_t3_pack_roundtrip_and_range():
    codes = synth.rng(41, 0).integers(-1, 2, size=(9, 640), dtype=np.int8)
    p = oracle.pack("t3", codes)
    assert p.shape == (9, 26 * 5) and p.max() < 243
    assert np.array_equal(oracle.unpack("t3", p, 640), codes)
    assert np.array_equal(_np_t3_codes(p, 640), codes)
    with pytest.raises(ValueError):
        oracle.pack("t3", np.full((1, 128), 2, np.int8))
    with pytest.raises(ValueError):
        oracle.pack("t3", np.zeros((1, 96), np.int8))


def test_t3_gemv_matches_numpy_at_every_element():
    M, N, K = 3, 21, 384
    codes = synth.rng(42, 0).integers(-1, 2, size=(N, K), dtype=np.int8)
    packed = oracle.pack("t3", codes)
    scales = synth.q1_scales(42, N, K)
    x = synth.bf16_normal(42, (M, K))
    W = _np_t3_codes(packed, K).astype(np.float64) * np.repeat(scales.view(np.float16).astype(np.float64), 128, 1)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    y, ab = oracle.t3_gemv(packed, scales, x, want_abs=True)
    np.testing.assert_allclose(y, xf @ W.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ab, np.abs(xf) @ np.abs(W).T, rtol=1e-12)
    mm, nn = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    ys, _ = oracle.t3_gemv_at(packed, scales, x, mm.ravel(), nn.ravel())
    np.testing.assert_allclose(ys, (xf @ W.T).ravel(), rtol=1e-12, atol=1e-12)


def test_t3_bruteforce_one_byte_patterns():
    # x_k = 4^i on k = 5 + i (byte 1 of the group), 0 elsewhere: sum_i w_i 4^i
    # identifies the pattern; every pattern is reached by some byte value
    K = 128
    x = np.zeros((1, K), np.uint16)
    x[0, 5:10] = synth.to_bf16_bits(4.0 ** np.arange(5))
    scales = np.full((1, 1), 0x3C00, np.uint16)
    seen = set()
    for v in range(243):
        packed = np.full((1, 26), 121, np.uint8)
        packed[0, 25] = 13
        packed[0, 1] = v
        y = oracle.t3_gemv(packed, scales, x)[0, 0]
        want = sum((((v // 3 ** i) % 3) - 1) * 4 ** i for i in range(5))
        assert y == want
        seen.add(y)
    assert len(seen) == 243
