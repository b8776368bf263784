"""torch.nn front end of libi8linear: an int8 decomposed replacement for nn.Linear.

Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at scale"
(Hugging Face blog), section "用法" (usage): a linear layer whose fp16 weight is quantised
to int8 when it is moved to the GPU -- codes CB in [-127, 127] plus one fp32 scale SCB per
output channel, from which the weight is recovered as CB * SCB / 127 -- and whose forward
runs the mixed-precision decomposition with an outlier threshold (6.0 by default); and the
helper that swaps the nn.Linear layers of a model for such layers, leaving named ones
(typically the output head) in fp16.

The blog also names a mode that keeps the fp16 weights for mixed-precision training
(``has_fp16_weights=True``): the weight stays an fp16 parameter, is re-quantised by every
forward, and gradients pass straight through the quantisation -- the blog gives no
gradient formulas, so the plainest reading is taken: the backward of y = x W^T + b, i.e.
dx = dy W, dW = dy^T x, db = sum(dy), with fp16 operands.  Without fp16 weights the layer
still passes dx = dy W' back (W' = CB * SCB / 127, the weight it computes with), so layers
before it can train.  Forward and backward run in the library's CUDA kernels: the two
backward products on the tcgen05 tensor cores (i8_linear_backward_input / _weight), the
bias gradient and W' in HBM-bound passes (i8_bias_grad, i8_dequantize_weight).  The
backward needs out_features % 8 == 0 (the row pitch of dy must suit TMA).

Serving with systematic outliers (the blog's observation that the same few feature
dimensions carry the outliers call after call): ``outlier_cache_cols > 0`` keeps the
weight's codes in the outlier columns (CB_o) in a device cache across forwards
(``i8_linear_forward_cached``), so a call whose outlier set matches the cached one skips
their gather; outputs are bit-identical to the uncached layer.

``code_format="e4m3"`` selects the FP8 variant of the decomposition (e4m3 codes scaled by
448 / absmax, the library's ``i8_*_e4m3`` calls); CB then holds e4m3 codes as uint8.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import torch

from . import abi


class _Int8LinearFn(torch.autograd.Function):
    """Forward: the decomposed int8 layer (CUDA library).  Backward: straight through the
    quantisation, the library's fp16 tensor-core products."""

    @staticmethod
    def forward(ctx, x2, weight, bias, layer):
        out = layer._forward_kernel(x2)
        ctx.layer = layer
        ctx.save_for_backward(x2, weight)
        ctx.has_bias = bias is not None
        return out

    @staticmethod
    def backward(ctx, gy):
        x2, weight = ctx.saved_tensors
        layer = ctx.layer
        gy = gy.to(torch.float16).contiguous()
        T, N = gy.shape
        K = layer.in_features
        dev = gy.device
        gx = gw = gb = None
        want_x = ctx.needs_input_grad[0]
        want_w = weight is not None and ctx.needs_input_grad[1]
        want_b = ctx.has_bias and ctx.needs_input_grad[2]
        if T == 0:
            z = lambda *shape: torch.zeros(shape, dtype=torch.float16, device=dev)  # noqa: E731
            return (z(0, K) if want_x else None, z(N, K) if want_w else None,
                    z(N) if want_b else None, None)
        if N % 8:
            raise NotImplementedError("the backward needs out_features % 8 == 0 (got %d): "
                                      "the row pitch of dy must be a multiple of 16 bytes" % N)
        with torch.cuda.device(dev):
            if want_x:
                w = (weight.detach().contiguous() if weight is not None
                     else layer.dequantized_weight())
                gx = torch.empty((T, K), dtype=torch.float16, device=dev)
                abi.i8_linear_backward_input(gy, w, gx)
            if want_w:
                gw = torch.empty((N, K), dtype=torch.float16, device=dev)
                abi.i8_linear_backward_weight(gy, x2.detach(), gw)
            if want_b:
                gb = torch.empty((N,), dtype=torch.float16, device=dev)
                abi.i8_bias_grad(gy, gb)
        return gx, gw, gb, None


class Linear8bitLt(torch.nn.Module):
    """y = x W^T + b computed as the LLM.int8() decomposition of x (fp16) and W.

    Buffers (saved and restored by ``state_dict``): ``CB`` int8 [out, in] (the weight's
    codes), ``SCB`` fp32 [out] (per-output-channel absmax), ``bias`` fp16 [out] or absent.
    The fp16 weight itself is not kept once quantised.

    ``forward(x)``: x fp16 [..., in] on the layer's CUDA device; the leading dimensions are
    flattened into T tokens of one call (T <= 16 takes the one-launch decode kernel, larger T
    the tensor-core GEMM).  The outlier columns are found per call from x.

    ``outlier_cache_cols``: capacity (columns) of the outlier cache, 0 = no cache.  The cache
    is not part of the state dict; ``quantize_`` and ``load_state_dict`` empty it, as they
    rewrite CB in place (write CB through neither, and call ``invalidate_outlier_cache``).
    """

    def __init__(self, in_features: int, out_features: int, bias: bool = True,
                 threshold: float = 6.0, device=None, has_fp16_weights: bool = False,
                 outlier_cache_cols: int = 0, code_format: str = "int8"):
        super().__init__()
        if code_format not in ("int8", "e4m3"):
            raise ValueError("code_format must be 'int8' or 'e4m3'")
        if code_format == "e4m3" and outlier_cache_cols:
            raise ValueError("the outlier cache serves the int8 forward only")
        self.code_format = code_format
        if in_features <= 0 or out_features <= 0 or in_features % 16 != 0:
            raise ValueError("in_features must be a positive multiple of 16 (row pitch of the "
                             "int8 weight for TMA); out_features positive")
        if outlier_cache_cols < 0:
            raise ValueError("outlier_cache_cols must be >= 0")
        if outlier_cache_cols and has_fp16_weights:
            raise ValueError("the outlier cache needs fixed codes: not with has_fp16_weights "
                             "(every forward re-quantises the weight)")
        self.in_features = in_features
        self.out_features = out_features
        self.threshold = float(threshold)
        self.outlier_cache_cols = int(outlier_cache_cols)
        self._ocache: Dict[torch.device, torch.Tensor] = {}
        cb_dtype = torch.uint8 if code_format == "e4m3" else torch.int8
        self.register_buffer("CB", torch.zeros((out_features, in_features), dtype=cb_dtype,
                                               device=device))
        self.register_buffer("SCB", torch.zeros((out_features,), dtype=torch.float32,
                                                device=device))
        self.has_fp16_weights = bool(has_fp16_weights)
        if self.has_fp16_weights:
            # training mode: fp16 master weight (and bias) as parameters, CB / SCB derived
            self.weight = torch.nn.Parameter(
                torch.zeros((out_features, in_features), dtype=torch.float16, device=device))
            self.bias = (torch.nn.Parameter(torch.zeros((out_features,), dtype=torch.float16,
                                                        device=device)) if bias else None)
        elif bias:
            self.register_buffer("bias", torch.zeros((out_features,), dtype=torch.float16,
                                                     device=device))
        else:
            self.register_buffer("bias", None)
        self._ws: Dict[torch.device, torch.Tensor] = {}

    @classmethod
    def from_linear(cls, linear: torch.nn.Linear, threshold: float = 6.0,
                    has_fp16_weights: bool = False,
                    outlier_cache_cols: int = 0, code_format: str = "int8") -> "Linear8bitLt":
        """Quantise an nn.Linear that lives on a CUDA device (weights cast to fp16)."""
        w = linear.weight
        if not w.is_cuda:
            raise ValueError("the weight must be on a CUDA device (it is quantised there)")
        m = cls(linear.in_features, linear.out_features, bias=linear.bias is not None,
                threshold=threshold, device=w.device, has_fp16_weights=has_fp16_weights,
                outlier_cache_cols=outlier_cache_cols, code_format=code_format)
        if has_fp16_weights:
            with torch.no_grad():
                m.weight.copy_(w.detach().to(torch.float16))
                if linear.bias is not None:
                    m.bias.copy_(linear.bias.detach().to(torch.float16))
        else:
            m.quantize_(w.detach(), None if linear.bias is None else linear.bias.detach())
        return m

    @torch.no_grad()
    def quantize_(self, weight: torch.Tensor, bias: Optional[torch.Tensor] = None):
        """Quantise an fp16 [out, in] weight (on this layer's CUDA device) into CB / SCB
        (inference mode; with fp16 weights every forward does this from ``weight``)."""
        if weight.shape != (self.out_features, self.in_features):
            raise ValueError("weight shape %s, expected %s"
                             % (tuple(weight.shape), (self.out_features, self.in_features)))
        if weight.device != self.CB.device:
            raise ValueError("weight on %s, layer on %s" % (weight.device, self.CB.device))
        self._quantize(weight.to(torch.float16).contiguous())
        self.invalidate_outlier_cache()
        if bias is not None:
            if self.bias is None:
                raise ValueError("layer was built without bias")
            self.bias.copy_(bias.to(torch.float16))
        return self

    def _quantize(self, weight16: torch.Tensor):
        with torch.cuda.device(self.CB.device):   # the library launches on the current device
            if self.code_format == "e4m3":
                abi.i8_quantize_weight_e4m3(weight16, self.CB, self.SCB)
            else:
                abi.i8_quantize_weight(weight16, self.CB, self.SCB)

    def dequantized_weight(self) -> torch.Tensor:
        """The weight the layer computes with, fp16 [out, in], from the library's kernel:
        CB * SCB / 127, or for e4m3 codes their values * SCB / 448 (the layer must be on a
        CUDA device)."""
        if not self.CB.is_cuda:
            raise ValueError("dequantized_weight() runs on the layer's CUDA device")
        W = torch.empty((self.out_features, self.in_features), dtype=torch.float16,
                        device=self.CB.device)
        with torch.cuda.device(self.CB.device):
            abi.i8_dequantize_weight(self.CB, self.SCB, W)
        return W

    def _workspace(self, T: int) -> torch.Tensor:
        size = (abi.i8_linear_workspace_size_e4m3 if self.code_format == "e4m3"
                else abi.i8_linear_workspace_size)
        need = size(T, self.out_features, self.in_features)
        dev = self.CB.device
        ws = self._ws.get(dev)
        if ws is None or ws.numel() < need:
            ws = torch.empty((need,), dtype=torch.uint8, device=dev)
            self._ws[dev] = ws
        return ws

    def invalidate_outlier_cache(self):
        """Empty the outlier cache (needed after CB changed in place)."""
        for c in self._ocache.values():
            with torch.cuda.device(c.device):
                abi.i8_outlier_cache_reset(c)

    def _outlier_cache(self) -> torch.Tensor:
        dev = self.CB.device
        c = self._ocache.get(dev)
        if c is None:
            need = abi.i8_outlier_cache_size(self.out_features, self.in_features,
                                             self.outlier_cache_cols)
            c = torch.empty((need,), dtype=torch.uint8, device=dev)
            with torch.cuda.device(dev):
                abi.i8_outlier_cache_reset(c)
            self._ocache[dev] = c
        return c

    def _load_from_state_dict(self, *args, **kwargs):
        super()._load_from_state_dict(*args, **kwargs)
        self.invalidate_outlier_cache()

    def _forward_kernel(self, x2: torch.Tensor) -> torch.Tensor:
        """One i8_linear_forward(_cached) call on a [T, in] fp16 input (no autograd)."""
        T = x2.shape[0]
        out = torch.empty((T, self.out_features), dtype=torch.float16, device=x2.device)
        if T > 0:
            with torch.cuda.device(self.CB.device):
                self._launch_forward(x2, out)
        return out

    def _launch_forward(self, x2: torch.Tensor, out: torch.Tensor):
        T = x2.shape[0]
        bias = None if self.bias is None else self.bias.detach()
        if self.code_format == "e4m3":
            abi.i8_linear_forward_e4m3(x2, self.CB, self.SCB, bias, self.threshold, out,
                                       self._workspace(T))
        elif self.outlier_cache_cols > 0:
            abi.i8_linear_forward_cached(x2, self.CB, self.SCB, bias, self.threshold, out,
                                         self._workspace(T), self._outlier_cache())
        else:
            abi.i8_linear_forward(x2, self.CB, self.SCB, bias, self.threshold, out,
                                  self._workspace(T))

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if x.dtype != torch.float16:
            raise TypeError("input must be fp16 (got %s)" % x.dtype)
        if x.shape[-1] != self.in_features:
            raise ValueError("last input dimension %d, expected %d"
                             % (x.shape[-1], self.in_features))
        if x.device != self.CB.device:
            raise ValueError("input on %s, layer on %s" % (x.device, self.CB.device))
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features).contiguous()
        if self.has_fp16_weights:
            with torch.no_grad():  # the weight may have changed since the last forward
                self._quantize(self.weight.detach().contiguous())
        w = self.weight if self.has_fp16_weights else None
        if torch.is_grad_enabled() and (x2.requires_grad or (w is not None and w.requires_grad)):
            y = _Int8LinearFn.apply(x2, w, self.bias, self)
        else:
            y = self._forward_kernel(x2)
        return y.reshape(*lead, self.out_features)

    def extra_repr(self) -> str:
        return ("in_features=%d, out_features=%d, bias=%s, threshold=%g, has_fp16_weights=%s, "
                "outlier_cache_cols=%d, code_format=%s"
                % (self.in_features, self.out_features, self.bias is not None, self.threshold,
                   self.has_fp16_weights, self.outlier_cache_cols, self.code_format))


def replace_linear_with_int8(model: torch.nn.Module, threshold: float = 6.0,
                             skip: Iterable[str] = ("lm_head",),
                             has_fp16_weights: bool = False,
                             outlier_cache_cols: int = 0,
                             code_format: str = "int8") -> torch.nn.Module:
    """Swap every nn.Linear of `model` (weights on a CUDA device) for a Linear8bitLt, in
    place, except modules whose name (last path component) is in `skip`.  Returns `model`."""
    skip = set(skip)
    for name, child in list(model.named_children()):
        if isinstance(child, torch.nn.Linear) and name not in skip:
            setattr(model, name, Linear8bitLt.from_linear(child, threshold=threshold,
                                                          has_fp16_weights=has_fp16_weights,
                                                          outlier_cache_cols=outlier_cache_cols,
                                                          code_format=code_format))
        elif name not in skip:
            replace_linear_with_int8(child, threshold=threshold, skip=skip,
                                     has_fp16_weights=has_fp16_weights,
                                     outlier_cache_cols=outlier_cache_cols,
                                     code_format=code_format)
    return model
