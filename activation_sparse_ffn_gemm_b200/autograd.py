"""PyTorch autograd wrapper of the TwELL gated FFN.

``twell_ffn(X, W_g, b_g, W_u, W_d)`` computes Y = (ReLU(X W_g^T + b_g) * (X W_u^T)) W_d^T
through twell_ffn_fwd and, when autograd asks for gradients, twell_ffn_bwd over
the hybrid state the forward kept. With ``lam > 0`` the backward also adds the
gradient of lam * sum(ReLU(z)), the L1 penalty on the gate activations that
induces the sparsity ([aimodelsnavi] "Technical Explanation": ReLU gate with L1
regularisation); the penalty's value itself is not returned (sum the state's
stored g if it is needed). Gradients come back in the dtype of each input
(bf16 for bf16 tensors), computed in fp32 by the kernels.
"""

from __future__ import annotations

import torch

from . import HybridState, ffn_bwd, ffn_fwd, transpose_wd


class TwellFFNFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W_g, b_g, W_u, W_d, K: int, lam: float, dense_min: int):
        shape = X.shape
        X2 = X.reshape(-1, shape[-1]).contiguous()
        M, f = X2.shape[0], W_g.shape[0]
        W_dt = transpose_wd(W_d)
        st = HybridState(M, f, 128, K, None, X.device, with_u=True, dense_min=dense_min)
        Y, st = ffn_fwd(X2, W_g, b_g, W_u, W_d, K=K, W_dt=W_dt, state=st)
        ctx.save_for_backward(X2, W_g, b_g, W_u, W_d, W_dt)
        ctx.state, ctx.lam, ctx.shape = st, float(lam), shape
        return Y.reshape(*shape[:-1], W_d.shape[0])

    @staticmethod
    def backward(ctx, dY):
        X2, W_g, b_g, W_u, W_d, W_dt = ctx.saved_tensors
        dY2 = dY.reshape(-1, dY.shape[-1]).to(torch.bfloat16).contiguous()
        g = ffn_bwd(X2, W_g, W_u, W_d, ctx.state, dY2, lam=ctx.lam, W_dt=W_dt, with_db=True)
        ctx.state = None
        need = ctx.needs_input_grad
        out = (g["dX"].to(X2.dtype).reshape(ctx.shape) if need[0] else None,
               g["dW_g"].to(W_g.dtype) if need[1] else None,
               g["db_g"].to(b_g.dtype) if need[2] else None,
               g["dW_u"].to(W_u.dtype) if need[3] else None,
               g["dW_d"].to(W_d.dtype) if need[4] else None)
        return out + (None, None, None)


def twell_ffn(X, W_g, b_g, W_u, W_d, K: int = 8, lam: float = 0.0, dense_min: int = 0):
    """Y = TwELL gated FFN of X [..., d_model] (bf16 CUDA tensors), differentiable
    in X, W_g, b_g, W_u and W_d. K: ELL slots per (row, 128-wide tile);
    dense_min: rows with at least this many active units go to the dense backup
    (0: only rows with a tile over K); lam: weight of the L1 penalty on ReLU(z)."""
    return TwellFFNFunction.apply(X, W_g, b_g, W_u, W_d, int(K), float(lam), int(dense_min))
