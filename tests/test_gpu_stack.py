"""The 64-layer Q1_0_g128 projection stack (hidden 5120, ffn 17408), one
decode step at M = 1 and M = 8, checked teacher-forced: every recorded
projection against the FP64 oracle on sampled output rows, given the bf16
input it actually received; every normalisation against the oracle's RMS
norm fed the same fp32 input."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import check_float, host

pytestmark = pytest.mark.gpu

H, F, L = synth.STACK_HIDDEN, synth.STACK_FFN, synth.STACK_LAYERS


@pytest.fixture(scope="module")
def stack_weights(cuda_device):
    from decode_packed_bit_b200 import build
    build.build()
    from decode_packed_bit_b200.stack import Q1Layer
    seed = synth.SEED_BASE + synth.W_Q1_STACK
    layers = []
    for li in range(L):
        w = {}
        for pi, (name, n, k) in enumerate(synth.STACK_PROJ):
            w[name] = synth.torch_q1_layer(seed, n, k, li * 16 + pi, cuda_device)
        layers.append(Q1Layer(w))
    return layers


def _bf16_ulp(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 1e-38)))
    return 2.0 ** (e - 7)


def _next_input_key(li, name):
    nxt = {"q": (li, "k"), "k": (li, "v"), "v": (li, "o"), "o": (li, "gate"), "gate+up": (li, "down"),
           "down": (li + 1, "q")}
    return nxt[name]


def _run(stack_weights, M, which, fused=False):
    from decode_packed_bit_b200.stack import Q1Stack, StackRecord
    st = Q1Stack(stack_weights, H, F, M, "cuda")
    x0 = synth.bf16_normal(synth.SEED_BASE + synth.W_Q1_STACK, (M, H), tag=M)
    st.x.copy_(torch.from_numpy(x0.view(np.int16)).view(torch.bfloat16).cuda())
    rec = StackRecord(which=which)
    if fused:
        st.step_fused(record=rec)
    else:
        st.step(record=rec)
    torch.cuda.synchronize()
    return st, rec


def _check_projections(stack_weights, rec, M, rows_per_proj, seed):
    g = np.random.default_rng(seed)
    for (li, name), xin in rec.inputs.items():
        if (li, name) not in rec.outputs:
            continue
        bits, scales = stack_weights[li].w[name]
        N = bits.shape[0]
        rows = np.unique(np.concatenate([[0, N - 1], g.integers(0, N, size=rows_per_proj)]))
        b = host(bits[torch.as_tensor(rows, device=bits.device)])
        s = host(scales[torch.as_tensor(rows, device=bits.device)].view(torch.int16)).view(np.uint16)
        x = host(xin.view(torch.int16)).view(np.uint16)
        ms = np.repeat(np.arange(M), len(rows))
        ns = np.tile(np.arange(len(rows)), M)
        y64, ab = oracle.q1_gemv_at(b, s, x, ms, ns)
        yg = host(rec.outputs[(li, name)])[:, rows].reshape(-1)
        check_float(yg, y64, ab, f"stack M={M} layer {li} {name}")


def _check_glue(rec, M):
    checked = 0
    for (li, name), v in rec.norm_in.items():
        key = _next_input_key(li, name)
        if key not in rec.inputs:
            continue
        if name == "gate+up":
            a, b = host(v[0]), host(v[1])
            r64 = oracle.rmsnorm(a, b, eps=1e-6)
        else:
            r64 = oracle.rmsnorm(host(v), None, eps=1e-6)
        got = synth.bf16_bits_to_f32(host(rec.inputs[key].view(torch.int16)).view(np.uint16)).astype(np.float64)
        tol = 0.5 * _bf16_ulp(r64) + 1e-6 * np.abs(r64) + 1e-30
        assert (np.abs(got - r64) <= tol).all(), f"normalisation after layer {li} {name}"
        checked += 1
    assert checked > 0


def test_stack_m1_all_layers_teacher_forced(stack_weights):
    st, rec = _run(stack_weights, 1, which=None)
    assert st.bytes_per_step == 3350200320
    assert len(rec.outputs) == 7 * L
    _check_projections(stack_weights, rec, 1, rows_per_proj=12, seed=11)
    _check_glue(rec, 1)
    assert torch.isfinite(st.x.float()).all()


def test_stack_m8_sampled_layers_teacher_forced(stack_weights):
    layers = [0, 1, 9, 23, 40, 55, 62, 63]
    which = {(li, name) for li in layers for name, _, _ in synth.STACK_PROJ}
    which |= {(li + 1, "q") for li in layers if li + 1 < L}
    st, rec = _run(stack_weights, 8, which=which)
    _check_projections(stack_weights, rec, 8, rows_per_proj=6, seed=12)
    _check_glue(rec, 8)
    assert torch.isfinite(st.x.float()).all()


def test_stack_m1_one_launch_teacher_forced(stack_weights):
    """lowbit_q1g128_stack_step: all 448 projections and their
    normalisations in one cooperative launch, checked like the per-call
    step, plus the step output against the oracle's last normalisation."""
    from decode_packed_bit_b200 import lowbit as lb
    st, rec = _run(stack_weights, 1, which=None, fused=True)
    assert lb.lowbit_fault_flags() == 0
    assert len(rec.outputs) == 7 * L
    # layer 0's q input is the step input itself
    x0 = synth.bf16_normal(synth.SEED_BASE + synth.W_Q1_STACK, (1, H), tag=1)
    assert np.array_equal(host(rec.inputs[(0, "q")].view(torch.int16)).view(np.uint16), x0)
    _check_projections(stack_weights, rec, 1, rows_per_proj=12, seed=13)
    _check_glue(rec, 1)
    # the step output: the last down output, normalised
    r64 = oracle.rmsnorm(host(rec.norm_in[(L - 1, "down")]), None, eps=1e-6)
    got = synth.bf16_bits_to_f32(host(st.x.view(torch.int16)).view(np.uint16)).astype(np.float64)
    tol = 0.5 * _bf16_ulp(r64) + 1e-6 * np.abs(r64) + 1e-30
    assert (np.abs(got - r64) <= tol).all()


@pytest.mark.parametrize("hidden,ffn,n_layers", [(1024, 8192, 2), (2048, 3072, 3), (1536, 2560, 2)])
def test_stack_one_launch_other_widths(cuda_device, hidden, ffn, n_layers):
    """The one-launch step at widths whose K-slice counts (2 and 16, 4 and
    6, 3 and 5 slices of 512) differ from the 5120/17408 stack's (10 and
    34), so every CTA's slice, rank and share of the blocks take other
    values; checked teacher-forced like the full stack, plus the step
    output."""
    from decode_packed_bit_b200 import build
    build.build()
    from decode_packed_bit_b200 import lowbit as lb
    from decode_packed_bit_b200.stack import Q1Layer, Q1Stack, StackRecord
    seed = synth.SEED_BASE + synth.W_Q1_STACK + 7 * hidden + ffn
    shapes = [("q", hidden, hidden), ("k", hidden, hidden), ("v", hidden, hidden), ("o", hidden, hidden),
              ("gate", ffn, hidden), ("up", ffn, hidden), ("down", hidden, ffn)]
    layers = [Q1Layer({name: synth.torch_q1_layer(seed, n, k, li * 16 + pi, cuda_device)
                       for pi, (name, n, k) in enumerate(shapes)}) for li in range(n_layers)]
    st = Q1Stack(layers, hidden, ffn, 1, "cuda")
    assert st.fused_supported()
    x0 = synth.bf16_normal(seed, (1, hidden), tag=1)
    st.x.copy_(torch.from_numpy(x0.view(np.int16)).view(torch.bfloat16).cuda())
    rec = StackRecord(which=None)
    st.step_fused(record=rec)
    torch.cuda.synchronize()
    assert lb.lowbit_fault_flags() == 0
    assert len(rec.outputs) == 7 * n_layers
    _check_projections(layers, rec, 1, rows_per_proj=16, seed=17)
    _check_glue(rec, 1)
    r64 = oracle.rmsnorm(host(rec.norm_in[(n_layers - 1, "down")]), None, eps=1e-6)
    got = synth.bf16_bits_to_f32(host(st.x.view(torch.int16)).view(np.uint16)).astype(np.float64)
    tol = 0.5 * _bf16_ulp(r64) + 1e-6 * np.abs(r64) + 1e-30
    assert (np.abs(got - r64) <= tol).all()


def test_stack_refuses_more_slices_than_resident_ctas(cuda_device):
    """Every 512-k slice of the ffn-wide input needs a CTA of its own (one
    per SM).  With one slice more than that the launcher returns
    LOWBIT_ERR_UNSUPPORTED_SHAPE before it clears the workspace or launches;
    the buffers are real (small, never read)."""
    from decode_packed_bit_b200 import build
    build.build()
    from decode_packed_bit_b200 import lowbit as lb
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    hidden, ffn = 512, 512 * (sms + 1)
    ws_bytes = lb.lowbit_q1g128_stack_workspace_bytes(1, hidden, ffn)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=cuda_device)
    bufs = [torch.zeros(16, dtype=torch.uint8, device=cuda_device) for _ in range(14)]
    x = torch.zeros(hidden, dtype=torch.int16, device=cuda_device)
    bits, keep_b = lb._ptr_array(bufs[:7])
    scales, keep_s = lb._ptr_array(bufs[7:])
    status = lb.lib().lowbit_q1g128_stack_step(bits, scales, 1, hidden, ffn, lb._ptr(x), 1e-6, lb._ptr(ws),
                                               ws_bytes, None, None, lb._stream(None))
    torch.cuda.synchronize()
    assert status == 3
    assert lb.lowbit_fault_flags() == 0
    # one slice per SM is still taken by the one-launch step's planner
    from decode_packed_bit_b200.stack import Q1Stack
    assert not Q1Stack([], hidden, ffn, 1, cuda_device).fused_supported()
    assert Q1Stack([], hidden, 512 * sms, 1, cuda_device).fused_supported()
