"""Training objective: the negative log-likelihood of gold segmentations,
log Z_b - score_b(y*) (Streaming Structured Inference with Flash-SemiCRF,
technical summary section 3), as a torch.autograd.Function over the library's
kernels.

Forward: prefix scan, streaming forward (log Z) and the gold-score kernel.
Backward: the library's backward with weights g (gradient of g . log Z) and the
gold backward with weights -g (adds the gradient of -g . score).  Argument
marshalling only; every step runs in libsemicrf.so.
"""
from __future__ import annotations

import torch

from . import backward, forward, gold_backward, gold_score, new_workspace, prefix_scan, WS_TRAIN


class SemiCRFNLL(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, A, D, lengths, labels, seg_start, ckpt_interval=0):
        B, T, C = x.shape
        K = D.shape[0]
        xc = x.detach().contiguous().float()
        Ac = A.detach().contiguous().float()
        Dc = D.detach().contiguous().float()
        ws = new_workspace(B, T, K, C, WS_TRAIN, ckpt_interval, device=x.device)
        S, _ = prefix_scan(xc, lengths, ws=ws)
        logZ, ws = forward(S, Ac, Dc, lengths, ws=ws, ckpt_interval=ckpt_interval)
        score = gold_score(S, Ac, Dc, lengths, labels, seg_start, ws)
        ctx.save_for_backward(S, Ac, Dc, lengths, labels, seg_start, ws)
        ctx.ckpt_interval = ckpt_interval
        ctx.dtypes = (x.dtype, A.dtype, D.dtype)
        return logZ - score

    @staticmethod
    def backward(ctx, g):
        S, Ac, Dc, lengths, labels, seg_start, ws = ctx.saved_tensors
        g = g.detach().to(torch.float64).contiguous()
        dX, dA, dD = backward(S, Ac, Dc, lengths, ws, grad_logZ=g, ckpt_interval=ctx.ckpt_interval)
        gold_backward(lengths, labels, seg_start, ws, dX, dA, dD, grad_score=(-g).contiguous())
        tx, tA, tD = ctx.dtypes
        return dX.to(tx), dA.to(tA), dD.to(tD), None, None, None, None
