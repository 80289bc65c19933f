"""GPU parity of the autoregressive reply loop (lowbit_z80_generate) against
the oracle's loop: every reply byte and every length bit-exact, on the
1024-conversation prompt mix, ragged tiles, replies that end early and
replies cut at max_new, long and unterminated prompts, and the counting
network whose replies have a closed form."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lb(cuda_device):
    from decode_packed_bit_b200 import build
    build.build()
    from decode_packed_bit_b200 import lowbit
    return lowbit


CS = np.frombuffer(synth.CHARSET, np.uint8)


def _gen(lb, packed, dims, queries, charset, max_new):
    batch = queries.shape[0]
    reply = torch.full((batch, max(max_new, 1)), 0xEE, dtype=torch.uint8, device="cuda")[:, :max_new]
    reply = reply.contiguous()
    lens = torch.full((batch,), -1, dtype=torch.int32, device="cuda")
    lb.lowbit_z80_generate([dev(p) for p in packed], dims, dev(queries), charset, reply, lens)
    torch.cuda.synchronize()
    return host(reply), host(lens)


def _check(lb, packed, dims, queries, charset, max_new):
    r, n = _gen(lb, packed, dims, queries, charset, max_new)
    ro, no = oracle.z80_generate(packed, dims, queries, charset, max_new)
    assert np.array_equal(n, no), f"lengths differ at {np.nonzero(n != no)[0][:8]}"
    assert np.array_equal(r, ro), f"replies differ at {np.nonzero((r != ro).any(axis=1))[0][:8]}"
    return n


@pytest.mark.parametrize("batch,max_new,seed", [(1024, 24, 1), (300, 40, 2), (31, 7, 3), (1, 250, 4)])
def test_replies_bitexact(lb, batch, max_new, seed):
    dims = synth.Q2_DIMS
    packed = [oracle.pack("q2", c) for c in synth.q2_codes(synth.SEED_BASE + synth.W_Q2_MLP + seed, dims)]
    q = synth.chat_queries(seed, batch)
    n = _check(lb, packed, dims, q, CS, max_new)
    # the mix must exercise both ways a reply ends
    if batch >= 300:
        assert (n < max_new).any() and (n == max_new).any()


def test_replies_with_skewed_networks(lb):
    """Code distributions that make the end symbol likely or rare."""
    dims = synth.Q2_DIMS
    q = synth.chat_queries(11, 200)
    for probs, seed in (((0.1, 0.2, 0.3, 0.4), 5), ((0.4, 0.3, 0.2, 0.1), 6), ((0.0, 0.1, 0.8, 0.1), 7)):
        g = synth.rng(seed, 0)
        codes = [g.choice(4, size=(dims[l + 1], dims[l]), p=probs).astype(np.int8) for l in range(len(dims) - 1)]
        packed = [oracle.pack("q2", c) for c in codes]
        _check(lb, packed, dims, q, CS, 32)


def test_replies_long_and_unterminated_prompts(lb):
    dims = synth.Q2_DIMS
    packed = [oracle.pack("q2", c) for c in synth.q2_codes(77, dims)]
    qlen = 300
    q = np.zeros((4, qlen), np.uint8)
    q[0, :280] = ord("Q")                                         # one 280-letter word: 255 kept
    q[1, :] = np.frombuffer((b"ab " * 100)[:qlen], np.uint8)      # fills the row, no 0 byte
    q[2, :5] = np.frombuffer(b"HeLLo", np.uint8)
    q[3, :3] = np.frombuffer(b"   ", np.uint8)                    # only spaces: empty query
    _check(lb, packed, dims, q, CS, 20)


def test_replies_counting_network_closed_form(lb):
    dims = (256, 4, 40)
    c1 = np.full((4, 256), 2, np.int8)
    c1[0, 128:] = 3
    c1[1, 128:] = 3
    c1[2, :128] = 3
    c2 = np.full((40, 4), 2, np.int8)
    c2[0, 0] = c2[0, 1] = 3
    c2[2, 2] = 3
    packed = [oracle.pack("q2", c1), oracle.pack("q2", c2)]
    q = synth.chat_queries(21, 100)
    r, n = _gen(lb, packed, dims, q, CS, 64)
    for i in range(100):
        text = bytes(q[i]).split(b"\0")[0].decode()
        want = min(64, -(-sum(len(w) for w in text.split()) // 2))
        assert n[i] == want and bytes(r[i, :want]) == b"A" * want and not r[i, want:].any()


def test_replies_edge_sizes(lb):
    dims = synth.Q2_DIMS
    packed = [oracle.pack("q2", c) for c in synth.q2_codes(78, dims)]
    q = synth.chat_queries(22, 40)
    r, n = _gen(lb, packed, dims, q, CS, 0)                      # no characters allowed
    assert r.shape == (40, 0) and (n == 0).all()
    r, n = _gen(lb, packed, dims, q[:0], CS, 8)                  # no conversations: no-op
    assert r.shape == (0, 8)
    from decode_packed_bit_b200.lowbit import LowbitError
    with pytest.raises(LowbitError):                             # the input must be 256 buckets
        _gen(lb, packed, (128, 192, 128, 40), q, CS, 4)
