"""A decode step through a stack of Q1_0_g128 linear projections.

Each layer applies q, k, v, o (hidden -> hidden), then gate and up (hidden
-> ffn, both reading the same input; their outputs are added), then down
(ffn -> hidden).  Between consecutive projections the fp32 output is
RMS-normalised (unit gain, eps 1e-6) and rounded to bf16, which is the
next projection's input; the last down output, normalised, is the next
layer's input.  Every product and normalisation runs in liblowbit.so
through the C ABI; this module only sequences the calls on one stream
(and can therefore be captured in a CUDA graph).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import lowbit as lb

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass
class Q1Layer:
    """Packed weights of one layer: name -> (bits uint8 [N][K/8], scales fp16 [N][K/128])."""
    w: dict


@dataclass
class StackRecord:
    """Optional capture of every projection's bf16 input and fp32 output,
    for (layer, projection) pairs in `which` (None: all)."""
    which: set | None = None
    inputs: dict = field(default_factory=dict)
    outputs: dict = field(default_factory=dict)
    norm_in: dict = field(default_factory=dict)    # fp32 inputs of each normalisation

    def want(self, layer, name):
        return self.which is None or (layer, name) in self.which


class Q1Stack:
    def __init__(self, layers, hidden: int, ffn: int, M: int, device, eps: float = 1e-6):
        self.layers = layers
        self.hidden, self.ffn, self.M, self.eps = hidden, ffn, M, eps
        dev = torch.device(device)
        bf = torch.bfloat16
        self.x = torch.empty((M, hidden), dtype=bf, device=dev)        # step input / output
        self.xh = torch.empty((M, hidden), dtype=bf, device=dev)       # normalised hidden-size activation
        self.xf = torch.empty((M, ffn), dtype=bf, device=dev)          # normalised ffn-size activation
        self.th = torch.empty((M, hidden), dtype=torch.float32, device=dev)
        self.tg = torch.empty((M, ffn), dtype=torch.float32, device=dev)
        self.tu = torch.empty((M, ffn), dtype=torch.float32, device=dev)
        ws = max(lb.lowbit_q1g128_workspace_bytes(M, n, k) for n, k in
                 ((hidden, hidden), (ffn, hidden), (hidden, ffn)))
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        self.act = torch.empty(max(lb.lowbit_q1g128_act_bytes(M, hidden), 256), dtype=torch.uint8, device=dev)
        gws = lb.lowbit_q1g128_act_workspace_bytes(2, M, ffn, hidden)
        self.gws = torch.empty(max(gws, 256), dtype=torch.uint8, device=dev)
        grp = lb.lowbit_q1g128_group_workspace_bytes(2, M, ffn, hidden)
        self.grp_ws = torch.empty(grp, dtype=torch.uint8, device=dev) if grp else None

    @property
    def bytes_per_step(self) -> int:
        total = 0
        for layer in self.layers:
            for bits, scales in layer.w.values():
                total += bits.numel() + scales.numel() * 2
        return total

    def launches_per_step(self) -> int:
        # per layer, M = 1: 5 one-shot products (prepare + product), 1 prepare
        # + 1 grouped product for gate/up, 6 normalisations; M > 1: 5 products,
        # 1 grouped product for gate/up, 6 normalisations
        per = 5 * 2 + 2 + 6 if self.M == 1 else 6 + 6
        return per * len(self.layers)

    def fused_supported(self) -> bool:
        if not (self.M == 1 and self.hidden % 512 == 0 and self.ffn % 512 == 0):
            return False
        # one CTA per SM, and every 512-k slice of the ffn-wide input needs one
        dev = self.x.device
        return dev.type != "cuda" or self.ffn // 512 <= torch.cuda.get_device_properties(dev).multi_processor_count

    def step_fused(self, stream=None, record: StackRecord | None = None):
        """The same step as step() at M = 1, as one launch of
        lowbit_q1g128_stack_step (every projection and normalisation inside)."""
        if not hasattr(self, "_fused_ws"):
            dev = self.x.device
            self._fused_ws = torch.empty(
                lb.lowbit_q1g128_stack_workspace_bytes(len(self.layers), self.hidden, self.ffn), dtype=torch.uint8,
                device=dev)
            self._fused_bits = [layer.w[name][0] for layer in self.layers for name in PROJ]
            self._fused_scales = [layer.w[name][1] for layer in self.layers for name in PROJ]
        rin = rout = None
        if record is not None:
            n = 7 * len(self.layers)
            rin = torch.zeros((n, self.ffn), dtype=torch.bfloat16, device=self.x.device)
            rout = torch.zeros((n, self.ffn), dtype=torch.float32, device=self.x.device)
        lb.lowbit_q1g128_stack_step(self._fused_bits, self._fused_scales, self.x, self.hidden, self.ffn,
                                    self._fused_ws, eps=self.eps, record_inputs=rin, record_outputs=rout,
                                    stream=stream)
        if record is not None:
            H, F = self.hidden, self.ffn
            for li in range(len(self.layers)):
                for pi, name in enumerate(PROJ):
                    i = 7 * li + pi
                    K = F if name == "down" else H
                    N = F if name in ("gate", "up") else H
                    if not record.want(li, name):
                        continue
                    record.inputs[(li, name)] = rin[i, :K].reshape(1, K).clone()
                    record.outputs[(li, name)] = rout[i, :N].reshape(1, N).clone()
                    if name in ("q", "k", "v", "o", "down"):
                        record.norm_in[(li, name)] = rout[i, :N].reshape(1, N).clone()
                if record.want(li, "gate") or record.want(li, "up"):
                    record.norm_in[(li, "gate+up")] = (rout[7 * li + 4, :F].reshape(1, F).clone(),
                                                       rout[7 * li + 5, :F].reshape(1, F).clone())
        return self.x

    def step(self, stream=None, record: StackRecord | None = None):
        """One decode step: self.x (bf16 [M][hidden]) -> self.x."""
        M = self.M
        for li, layer in enumerate(self.layers):
            src = self.x
            for name in ("q", "k", "v", "o"):
                bits, scales = layer.w[name]
                if record is not None and record.want(li, name):
                    record.inputs[(li, name)] = src.clone()
                lb.lowbit_q1g128_gemv(bits, scales, src, self.th, workspace=self.ws, stream=stream)
                if record is not None and record.want(li, name):
                    record.outputs[(li, name)] = self.th.clone()
                    record.norm_in[(li, name)] = self.th.clone()
                lb.lowbit_rmsnorm_bf16(self.th, None, self.xh, eps=self.eps, stream=stream)
                src = self.xh
            # gate and up read the same normalised activation
            gb, gs = layer.w["gate"]
            ub, us = layer.w["up"]
            if record is not None and (record.want(li, "gate") or record.want(li, "up")):
                record.inputs[(li, "gate")] = src.clone()
                record.inputs[(li, "up")] = src.clone()
            if M == 1:
                lb.lowbit_q1g128_prepare_act(src, self.act, stream=stream)
                lb.lowbit_q1g128_gemv_act_group([gb, ub], [gs, us], self.act, [self.tg, self.tu], M,
                                                workspace=self.gws, stream=stream)
            else:
                lb.lowbit_q1g128_gemv_group([gb, ub], [gs, us], src, [self.tg, self.tu],
                                            workspace=self.grp_ws, stream=stream)
            if record is not None and (record.want(li, "gate") or record.want(li, "up")):
                record.outputs[(li, "gate")] = self.tg.clone()
                record.outputs[(li, "up")] = self.tu.clone()
                record.norm_in[(li, "gate+up")] = (self.tg.clone(), self.tu.clone())
            lb.lowbit_rmsnorm_bf16(self.tg, self.tu, self.xf, eps=self.eps, stream=stream)
            db, ds = layer.w["down"]
            if record is not None and record.want(li, "down"):
                record.inputs[(li, "down")] = self.xf.clone()
            lb.lowbit_q1g128_gemv(db, ds, self.xf, self.th, workspace=self.ws, stream=stream)
            if record is not None and record.want(li, "down"):
                record.outputs[(li, "down")] = self.th.clone()
                record.norm_in[(li, "down")] = self.th.clone()
            lb.lowbit_rmsnorm_bf16(self.th, None, self.x, eps=self.eps, stream=stream)
        return self.x
