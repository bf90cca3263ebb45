"""PyTorch autograd glue over the C ABI: the layer as a torch.autograd.Function and
an nn.Module holding its weights.

Marshalling only.  The forward runs moe_forward_ws with MOE_PATH_TRAIN when a
gradient is needed (moe_forward otherwise), the backward runs moe_backward_ws
on the workspace the forward kept; every step is the library's kernels.

The layer is the one of include/moe.h: router scores Wg x, top-k with softmax
gates over the k, SwiGLU experts W2 (SiLU(W1 x) * W3 x), gate-weighted sum
("Mistral/Mixtral architecture" page, section "MoEの数学 — ルーターとゲーティング機構").
With alpha != 0 the gradient also holds the load-balance loss alpha E sum f p of
the batch's routing (subsection "ロードバランス損失"); its value comes from
moe_route_stats.
"""
from __future__ import annotations

import math

import torch

from . import (MOE_DTYPE_BF16, MOE_DTYPE_F32, MOE_PATH_TRAIN, moe_backward_ws, moe_forward, moe_forward_ws,
               moe_train_workspace_size)


class MoEFunction(torch.autograd.Function):
    """out = MoE(x) with weights (Wg, W1, W3, W2); gradients for x and every weight.

    Weight gradients are summed in fp32 and rounded once to each weight's dtype
    (for bf16 weights, inside the GEMM epilogue).
    """

    @staticmethod
    def forward(ctx, x, Wg, W1, W3, W2, k: int, alpha: float = 0.0):
        T, d = x.shape
        E, F, _ = W1.shape
        code = MOE_DTYPE_BF16 if x.dtype == torch.bfloat16 else MOE_DTYPE_F32
        ws = torch.empty(max(moe_train_workspace_size(T, d, F, E, k, code), 1), dtype=torch.uint8, device=x.device)
        out = moe_forward_ws(x, Wg, W1, W3, W2, k, path=MOE_PATH_TRAIN, workspace=ws)
        ctx.save_for_backward(x, Wg, W1, W3, W2)
        ctx.ws, ctx.k, ctx.alpha = ws, k, float(alpha)
        return out

    @staticmethod
    def backward(ctx, dout):
        x, Wg, W1, W3, W2 = ctx.saved_tensors
        wd = torch.bfloat16 if W1.dtype == torch.bfloat16 else torch.float32
        g, _ = moe_backward_ws(x, Wg, W1, W3, W2, dout.contiguous(), ctx.k, ctx.ws, alpha=ctx.alpha, wgrad_dtype=wd)
        ctx.ws = None
        return (g["dx"], g["dWg"].to(Wg.dtype), g["dW1"].to(W1.dtype), g["dW3"].to(W3.dtype), g["dW2"].to(W2.dtype),
                None, None)


class SparseMoE(torch.nn.Module):
    """The MoE feed-forward layer with its weights as parameters (nn.Linear layouts):
    Wg [E][d], W1 [E][F][d], W3 [E][F][d], W2 [E][d][F].  Input [..., d]."""

    def __init__(self, d: int, ffn: int, E: int = 8, k: int = 2, alpha: float = 0.0, dtype=torch.bfloat16,
                 device="cuda"):
        super().__init__()
        self.k, self.alpha = k, alpha
        kw = dict(dtype=dtype, device=device)
        self.Wg = torch.nn.Parameter(torch.randn(E, d, **kw) / math.sqrt(d))
        self.W1 = torch.nn.Parameter(torch.randn(E, ffn, d, **kw) / math.sqrt(d))
        self.W3 = torch.nn.Parameter(torch.randn(E, ffn, d, **kw) / math.sqrt(d))
        self.W2 = torch.nn.Parameter(torch.randn(E, d, ffn, **kw) / math.sqrt(ffn))

    def forward(self, x):
        shape = x.shape
        x2 = x.reshape(-1, shape[-1]).contiguous()
        weights = (self.Wg, self.W1, self.W3, self.W2)
        if torch.is_grad_enabled() and (x2.requires_grad or any(w.requires_grad for w in weights)):
            out = MoEFunction.apply(x2, *weights, self.k, self.alpha)
        else:
            out = moe_forward(x2, *(w.detach() for w in weights), self.k)
        return out.reshape(shape)
