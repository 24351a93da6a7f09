"""Training objective: the negative log-likelihood of gold segmentations,
log Z_b - score_b(y*) (Streaming Structured Inference with Flash-SemiCRF,
technical summary section 3), as a torch.autograd.Function over the library's
kernels.

Forward: semicrf_nll -- prefix scan, streaming forward with checkpoints (log Z),
the gold-score kernel and nll = log Z - score, all on the device.
Backward: semicrf_nll_backward -- the checkpointed backward with the upstream
weights g and the gold-segmentation counts with weights -g.  Argument
marshalling only; every step runs in libsemicrf.so.  The checkpointed pair is
used (not the side-by-side step) because the upstream weights are known only
when the backward runs, and the pair keeps O(sqrt(T) K C) state between the two.
"""
from __future__ import annotations

import torch

from . import WS_TRAIN, new_workspace, nll, nll_backward, prefix_scan


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
        out, _, _ = nll(S, Ac, Dc, lengths, labels, seg_start, ws, ckpt_interval=ckpt_interval)
        ctx.save_for_backward(S, Ac, Dc, lengths, labels, seg_start, ws)
        ctx.ckpt_interval = ckpt_interval
        ctx.dtypes = (x.dtype, A.dtype, D.dtype)
        return out

    @staticmethod
    def backward(ctx, g):
        S, Ac, Dc, lengths, labels, seg_start, ws = ctx.saved_tensors
        g = g.detach().to(torch.float64).contiguous()
        dX, dA, dD = nll_backward(S, Ac, Dc, lengths, labels, seg_start, ws, grad_nll=g,
                                  ckpt_interval=ctx.ckpt_interval)
        tx, tA, tD = ctx.dtypes
        return dX.to(tx), dA.to(tA), dD.to(tD), None, None, None, None
