"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no part of the packed-weight arithmetic: it only draws
random codes, scales and activations with the distributions of the five
workloads and returns them as plain integer arrays (codes) or IEEE bit
patterns (fp16 scales, bf16 activations).  Packing, unpacking and every
product are done elsewhere -- by the GPU library or by the oracle.

Seeds: workload i uses base seed 0x5EED0000 + i, and every tensor of a
workload draws from its own sub-stream (``SeedSequence([base, stream])``),
so adding a tensor never shifts the others.
"""
from __future__ import annotations

import numpy as np

SEED_BASE = 0x5EED0000

# Sub-stream ids, one per tensor role.
S_CODES, S_SCALES, S_X, S_BUCKETS, S_VALUES, S_ROWS = range(6)

# Workload indices (the order the five workloads are listed in, then the
# ternary format).
W_Q2_MLP, W_Q1_4096, W_Q1_SWEEP, W_Q1_STACK, W_INT4, W_T3 = range(6)

Q2_DIMS = (256, 192, 128, 40)
Q1_SWEEP_SHAPES = ((5120, 5120), (17408, 5120), (5120, 17408))
STACK_HIDDEN, STACK_FFN, STACK_LAYERS = 5120, 17408, 64
# q, k, v, o, gate, up, down: (N, K) of each projection of one layer.
STACK_PROJ = (("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120), ("o", 5120, 5120),
              ("gate", 17408, 5120), ("up", 17408, 5120), ("down", 5120, 17408))
INT4_N, INT4_K = 11008, 4096


def rng(seed: int, stream: int, *extra: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, *extra])))


def to_bf16_bits(a) -> np.ndarray:
    """Round float values to bfloat16 (through float32, round-to-nearest-even
    on the dropped 16 bits) and return the uint16 bit patterns."""
    f = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (f >> 16) & 1
    r = ((f + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(a, dtype=np.float32))
    r[nan] = 0x7FC0
    return r


def to_f16_bits(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64).astype(np.float16).view(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact: bf16 is the top half)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# -- Q1_0_g128 ---------------------------------------------------------------------

def q1_codes(seed: int, N: int, K: int, tag: int = 0) -> np.ndarray:
    """Sign codes, Bernoulli(0.5), int8 {0,1} [N][K]."""
    return rng(seed, S_CODES, tag).integers(0, 2, size=(N, K), dtype=np.int8)


def q1_packed_random(seed: int, N: int, K: int, tag: int = 0) -> np.ndarray:
    """Uniform random bytes [N][K/8]: the same distribution as packing
    Bernoulli(0.5) codes (every bit independent and fair), drawn directly in
    packed form for weight sets too large to materialise as codes."""
    return rng(seed, S_CODES, tag).integers(0, 256, size=(N, K // 8), dtype=np.uint8)


def q1_scales(seed: int, N: int, K: int, tag: int = 0, sigma: float = 0.02) -> np.ndarray:
    """fp16 bits [N][K/128] of |N(0, sigma)|."""
    return to_f16_bits(np.abs(rng(seed, S_SCALES, tag).normal(0.0, sigma, size=(N, K // 128))))


def bf16_normal(seed: int, shape, tag: int = 0) -> np.ndarray:
    """bf16 bits of N(0, 1) samples."""
    return to_bf16_bits(rng(seed, S_X, tag).standard_normal(size=shape))


# -- INT4-g64 ----------------------------------------------------------------------

def int4_codes(seed: int, N: int, K: int, tag: int = 0) -> np.ndarray:
    """int8 codes uniform in [-8, 7], [N][K]."""
    return rng(seed, S_CODES, tag).integers(-8, 8, size=(N, K), dtype=np.int8)


def int4_scales(seed: int, N: int, K: int, tag: int = 0, sigma: float = 0.01) -> np.ndarray:
    """fp16 bits [N][K/64] of |N(0, sigma)|."""
    return to_f16_bits(np.abs(rng(seed, S_SCALES, tag).normal(0.0, sigma, size=(N, K // 64))))


# -- 2-bit MLP -----------------------------------------------------------------------

def q2_codes(seed: int, dims=Q2_DIMS):
    """One int8 code matrix per layer, uniform in {0,1,2,3}, [dims[l+1]][dims[l]]."""
    return [rng(seed, S_CODES, l).integers(0, 4, size=(dims[l + 1], dims[l]), dtype=np.int8)
            for l in range(len(dims) - 1)]


def q2_inputs(seed: int, batch: int, halves: int = 2, buckets: int = 128,
              active: int = 8, values=(32, 64, 96)) -> np.ndarray:
    """Trigram-bucket shaped int16 vectors [batch][halves*buckets]: in each
    half (query, context) `active` distinct buckets hold a value drawn
    uniformly from `values`; every other bucket is 0."""
    g = rng(seed, S_BUCKETS)
    out = np.zeros((batch, halves * buckets), np.int16)
    vals = np.asarray(values, np.int16)
    for b in range(batch):
        for h in range(halves):
            idx = g.choice(buckets, size=active, replace=False)
            out[b, h * buckets + idx] = vals[g.integers(0, len(vals), size=active)]
    return out


# -- device-side generation for weight sets of gigabytes --------------------------------

def torch_q1_layer(seed: int, N: int, K: int, tag: int, device):
    """(packed bits uint8 [N][K/8], fp16 scales [N][K/128]) drawn on `device`
    with torch's counter-based generator, for weight sets too large to draw
    on the host.  Every bit is a fair coin; scales are |N(0, 0.02)|."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000003 + tag) & 0x7FFFFFFFFFFFFFFF)
    bits = torch.randint(0, 256, (N, K // 8), generator=g, device=device, dtype=torch.uint8)
    scales = (torch.randn((N, K // 128), generator=g, device=device) * 0.02).abs().half()
    return bits, scales


# -- chat prompts for the reply loop ---------------------------------------------------

# Output index -> character of the 40-output network: 0 ends a reply, then
# space, A-Z, 0-9, '?', '!'.
CHARSET = b"\0 ABCDEFGHIJKLMNOPQRSTUVWXYZ0123456789?!"


def chat_queries(seed: int, batch: int, qlen: int = 32, words=(1, 5), wlen=(1, 8)) -> np.ndarray:
    """Prompts as 0-padded bytes [batch][qlen]: `words` words of `wlen`
    letters each (a-z, a quarter of them upper-case, an occasional '?'),
    separated by one or two spaces and cut to qlen bytes."""
    g = rng(seed, S_ROWS)
    out = np.zeros((batch, qlen), np.uint8)
    letters = np.frombuffer(b"abcdefghijklmnopqrstuvwxyz", np.uint8)
    for b in range(batch):
        parts = []
        for _ in range(int(g.integers(words[0], words[1] + 1))):
            w = letters[g.integers(0, 26, size=int(g.integers(wlen[0], wlen[1] + 1)))].copy()
            up = g.random(len(w)) < 0.25
            w[up] -= 32
            parts.append(bytes(w) + (b"?" if g.random() < 0.1 else b""))
        text = b"".join(p + (b"  " if g.random() < 0.2 else b" ") for p in parts).rstrip(b" ")[:qlen]
        out[b, :len(text)] = np.frombuffer(text, np.uint8)
    return out


# -- ternary, FP16 scale per 128 ---------------------------------------------------

def t3_codes(seed: int, N: int, K: int, tag: int = 0, p_zero: float = 1 / 3) -> np.ndarray:
    """Codes in {-1, 0, +1} [N][K]: 0 with probability p_zero, else a fair sign."""
    g = rng(seed, S_CODES, tag)
    z = g.random((N, K)) < p_zero
    s = g.integers(0, 2, size=(N, K), dtype=np.int8) * 2 - 1
    return np.where(z, 0, s).astype(np.int8)


def torch_t3_layer(seed: int, N: int, K: int, tag: int, device):
    """(packed base-3 bytes uint8 [N][26 K/128], fp16 scales [N][K/128]) drawn
    on `device`: every byte uniform over the 243 valid values (each of its
    five trits uniform and independent), the last byte of a group over its
    27; scales |N(0, 0.02)|."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000033 + tag) & 0x7FFFFFFFFFFFFFFF)
    G = K // 128
    b = torch.randint(0, 243, (N, G, 26), generator=g, device=device, dtype=torch.int16)
    b[:, :, 25] = torch.randint(0, 27, (N, G), generator=g, device=device, dtype=torch.int16)
    packed = b.to(torch.uint8).reshape(N, 26 * G).contiguous()
    scales = (torch.randn((N, G), generator=g, device=device) * 0.02).abs().half()
    return packed, scales
