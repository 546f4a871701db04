"""A linear layer whose forward is the LLM.int8() decomposed matmul.

Restates the int8 layer of the "LLM.int8()" page (brain.gartu.xyz), "Exemple
pratique": a drop-in replacement for ``nn.Linear(in, out, bias)`` that keeps its
weight quantised to int8 (prepared once), takes the outlier threshold alpha
(6.0 by default), and computes y = x W + b with the columns of x above alpha
in fp16.  The fp16 weight is kept as well: its rows in the outlier set feed
the fp16 product.  Prepared with a calibrated set of outlier input dimensions
(``static_rows``), the layer instead keeps only the fp16 rows of those
dimensions and drops the fp16 weight; the outliers sit in a few fixed
feature dimensions ("LLM.int8() — 大模型激活值里藏着几个超大异常通道").  All
arithmetic runs in libint8mm.so; this module only holds the tensors and
marshals them.
"""
from __future__ import annotations

import torch

from . import Weight, int8mm_forward_bias, int8mm_free, int8mm_prepare_weight, int8mm_prepare_weight_static


class Linear8bitLt(torch.nn.Module):
    """y = x W + b for fp16 x [..., in_features] on a CUDA device.

    ``weight`` is stored as [in_features, out_features] fp16 (the method's W,
    K x N row-major), ``bias`` as [out_features] fp16 or None.  The int8 codes
    are prepared on the first forward, or by ``prepare()``; call it again after
    changing ``weight`` in place.
    """

    def __init__(self, in_features: int, out_features: int, bias: bool = True, threshold: float = 6.0,
                 device=None):
        super().__init__()
        self.in_features = int(in_features)
        self.out_features = int(out_features)
        self.threshold = float(threshold)
        dev = torch.device("cuda") if device is None else torch.device(device)
        self.weight = torch.nn.Parameter(
            torch.zeros((self.in_features, self.out_features), dtype=torch.float16, device=dev), requires_grad=False)
        self.bias = (torch.nn.Parameter(torch.zeros(self.out_features, dtype=torch.float16, device=dev),
                                        requires_grad=False) if bias else None)
        self._w: Weight | None = None

    @classmethod
    def from_linear(cls, linear: torch.nn.Linear, threshold: float = 6.0, static_rows=None,
                    max_outliers: int = 256) -> "Linear8bitLt":
        """The int8 layer of an ``nn.Linear`` (whose weight is [out, in]);
        ``static_rows`` / ``max_outliers`` as for ``prepare``."""
        m = cls(linear.in_features, linear.out_features, bias=linear.bias is not None, threshold=threshold,
                device=linear.weight.device)
        with torch.no_grad():
            m.weight.copy_(linear.weight.detach().t())
            if linear.bias is not None:
                m.bias.copy_(linear.bias.detach())
        m.prepare(static_rows, max_outliers)
        return m

    def prepare(self, static_rows=None, max_outliers: int = 256) -> None:
        """Quantise the current weight (per-column scales and int8 codes).

        With ``static_rows`` (the calibrated outlier input dimensions, indices
        into in_features) the memory-saving weight is prepared instead and the
        fp16 ``weight`` is dropped (set to None): the layer keeps the int8
        codes, the fp16 rows of those dimensions and room for
        ``max_outliers`` outlier rows per forward; an outlier dimension
        outside the set uses its row rebuilt from the int8 codes."""
        if self.weight is None:
            raise RuntimeError("the fp16 weight was dropped by a static prepare")
        old, self._w = self._w, None
        if old is not None:
            int8mm_free(old)
        if static_rows is None:
            self._w = int8mm_prepare_weight(self.weight.data)
        else:
            self._w = int8mm_prepare_weight_static(self.weight.data, list(static_rows), max_outliers)
            self.weight = None

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if x.dtype != torch.float16 or not x.is_cuda:
            raise TypeError("Linear8bitLt takes fp16 CUDA activations")
        if x.shape[-1] != self.in_features:
            raise ValueError(f"last dimension {x.shape[-1]} != in_features {self.in_features}")
        if self._w is None:
            self.prepare()
        x2 = x.reshape(-1, self.in_features)
        if not x2.is_contiguous():
            raise ValueError("x must be contiguous in its last dimension")
        b = None if self.bias is None else self.bias.data
        y = int8mm_forward_bias(self._w, x2, self.threshold, b)
        return y.reshape(*x.shape[:-1], self.out_features)

    def extra_repr(self) -> str:
        return (f"in_features={self.in_features}, out_features={self.out_features}, "
                f"bias={self.bias is not None}, threshold={self.threshold}")
