"""torch.nn front end of libi8linear: an int8 decomposed replacement for nn.Linear.

Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at scale"
(Hugging Face blog), section "用法" (usage): a linear layer whose fp16 weight is quantised
to int8 when it is moved to the GPU -- codes CB in [-127, 127] plus one fp32 scale SCB per
output channel, from which the weight is recovered as CB * SCB / 127 -- and whose forward
runs the mixed-precision decomposition with an outlier threshold (6.0 by default); and the
helper that swaps the nn.Linear layers of a model for such layers, leaving named ones
(typically the output head) in fp16.

Inference only: the forward has no backward (the blog's fp16-weight training mode is not
built), so outputs never require grad.  Everything numerical runs in the library's CUDA
kernels; this module allocates tensors and marshals arguments.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import torch

from . import abi


class Linear8bitLt(torch.nn.Module):
    """y = x W^T + b computed as the LLM.int8() decomposition of x (fp16) and W.

    Buffers (saved and restored by ``state_dict``): ``CB`` int8 [out, in] (the weight's
    codes), ``SCB`` fp32 [out] (per-output-channel absmax), ``bias`` fp16 [out] or absent.
    The fp16 weight itself is not kept once quantised.

    ``forward(x)``: x fp16 [..., in] on the layer's CUDA device; the leading dimensions are
    flattened into T tokens of one call (T <= 16 takes the one-launch decode kernel, larger T
    the tensor-core GEMM).  The outlier columns are found per call from x.
    """

    def __init__(self, in_features: int, out_features: int, bias: bool = True,
                 threshold: float = 6.0, device=None):
        super().__init__()
        if in_features <= 0 or out_features <= 0 or in_features % 16 != 0:
            raise ValueError("in_features must be a positive multiple of 16 (row pitch of the "
                             "int8 weight for TMA); out_features positive")
        self.in_features = in_features
        self.out_features = out_features
        self.threshold = float(threshold)
        self.register_buffer("CB", torch.zeros((out_features, in_features), dtype=torch.int8,
                                               device=device))
        self.register_buffer("SCB", torch.zeros((out_features,), dtype=torch.float32,
                                                device=device))
        if bias:
            self.register_buffer("bias", torch.zeros((out_features,), dtype=torch.float16,
                                                     device=device))
        else:
            self.register_buffer("bias", None)
        self._ws: Dict[torch.device, torch.Tensor] = {}

    @classmethod
    def from_linear(cls, linear: torch.nn.Linear, threshold: float = 6.0) -> "Linear8bitLt":
        """Quantise an fp16 nn.Linear that lives on a CUDA device."""
        w = linear.weight
        if not w.is_cuda:
            raise ValueError("the weight must be on a CUDA device (it is quantised there)")
        m = cls(linear.in_features, linear.out_features, bias=linear.bias is not None,
                threshold=threshold, device=w.device)
        m.quantize_(w.detach(), None if linear.bias is None else linear.bias.detach())
        return m

    @torch.no_grad()
    def quantize_(self, weight: torch.Tensor, bias: Optional[torch.Tensor] = None):
        """Quantise an fp16 [out, in] weight (on this layer's CUDA device) into CB / SCB."""
        if weight.shape != (self.out_features, self.in_features):
            raise ValueError("weight shape %s, expected %s"
                             % (tuple(weight.shape), (self.out_features, self.in_features)))
        if weight.device != self.CB.device:
            raise ValueError("weight on %s, layer on %s" % (weight.device, self.CB.device))
        abi.i8_quantize_weight(weight.to(torch.float16).contiguous(), self.CB, self.SCB)
        if bias is not None:
            if self.bias is None:
                raise ValueError("layer was built without bias")
            self.bias.copy_(bias.to(torch.float16))
        return self

    def dequantized_weight(self) -> torch.Tensor:
        """The weight the layer computes with, CB * SCB / 127 (fp32), for inspection."""
        return self.CB.float() * (self.SCB.float() / 127.0)[:, None]

    def _workspace(self, T: int) -> torch.Tensor:
        need = abi.i8_linear_workspace_size(T, self.out_features, self.in_features)
        dev = self.CB.device
        ws = self._ws.get(dev)
        if ws is None or ws.numel() < need:
            ws = torch.empty((need,), dtype=torch.uint8, device=dev)
            self._ws[dev] = ws
        return ws

    @torch.no_grad()
    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if x.dtype != torch.float16:
            raise TypeError("input must be fp16 (got %s)" % x.dtype)
        if x.shape[-1] != self.in_features:
            raise ValueError("last input dimension %d, expected %d"
                             % (x.shape[-1], self.in_features))
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features).contiguous()
        T = x2.shape[0]
        out = torch.empty((T, self.out_features), dtype=torch.float16, device=x2.device)
        if T > 0:
            abi.i8_linear_forward(x2, self.CB, self.SCB, self.bias, self.threshold, out,
                                  self._workspace(T))
        return out.reshape(*lead, self.out_features)

    def extra_repr(self) -> str:
        return "in_features=%d, out_features=%d, bias=%s, threshold=%g" % (
            self.in_features, self.out_features, self.bias is not None, self.threshold)


def replace_linear_with_int8(model: torch.nn.Module, threshold: float = 6.0,
                             skip: Iterable[str] = ("lm_head",)) -> torch.nn.Module:
    """Swap every nn.Linear of `model` (weights on a CUDA device) for a Linear8bitLt, in
    place, except modules whose name (last path component) is in `skip`.  Returns `model`."""
    skip = set(skip)
    for name, child in list(model.named_children()):
        if isinstance(child, torch.nn.Linear) and name not in skip:
            setattr(model, name, Linear8bitLt.from_linear(child, threshold=threshold))
        elif name not in skip:
            replace_linear_with_int8(child, threshold=threshold, skip=skip)
    return model
