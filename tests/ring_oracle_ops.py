"""Block computations of the ring schedule done by the fp64 oracle, on CPU torch
tensors: the CPU tests run the ring schedule (and, with gloo ranks, its
point-to-point exchange) with these in place of the library's kernels.
Test-only."""
import numpy as np
import torch

import oracle


def _np(t):
    return t.detach().cpu().double().numpy()


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a))


class OracleOps:
    def fwd(self, q, k, v, scale, causal):
        o, lse = oracle.attn_fwd(_np(q), _np(k), _np(v), scale=scale, causal=causal)
        return _t(o), _t(lse)

    def new_fwd_acc(self, q):
        B, n, H, d = q.shape
        return torch.zeros((B, n, H, d), dtype=torch.float64), torch.zeros((B, H, n), dtype=torch.float64)

    def new_out(self, q):
        return torch.zeros(q.shape, dtype=torch.float64)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, out, row0):
        rows = slice(row0, row0 + o_part.shape[1])
        if first:
            o, lse = _np(o_part), _np(lse_part)
        else:
            o, lse = oracle.merge_partials([_np(o_acc[:, rows]), _np(o_part)],
                                           [_np(lse_acc[:, :, rows]), _np(lse_part)])
        o_acc[:, rows] = _t(o)
        lse_acc[:, :, rows] = _t(lse)
        if out is not None:
            out[:, rows] = o_acc[:, rows]

    def bwd(self, q, k, v, o, lse, do, scale, causal):
        return tuple(_t(x) for x in oracle.attn_bwd_given_stats(_np(q), _np(k), _np(v), _np(do), _np(o),
                                                                _np(lse), scale=scale, causal=causal))

    def new_grad_acc(self, x):
        return torch.zeros(x.shape, dtype=torch.float64)

    def accumulate(self, acc, part, first, row0):
        rows = slice(row0, row0 + part.shape[1])
        if first:
            acc[:, rows] = part
        else:
            acc[:, rows] += part

    def finish_grad(self, acc, like):
        return acc.clone()
