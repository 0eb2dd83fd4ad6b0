"""Ring (context-parallel) exact attention: one long sequence split across
ranks (zocula.com fla guide, the flame bullets and the glossary entry on
context parallelism: long contexts are divided over several GPUs).

Rank r of R holds rows [r n, (r + 1) n) of q, k, v (and o, lse, dO for the
backward), n = N / R.  It keeps its query rows; the key/value slices travel
around the ring, rank r passing what it holds to rank r + 1 after each step,
so at step t it holds slice (r - t) mod R.  Each (query slice, key slice)
pair is an ordinary attention call of the library:

* causal: the diagonal pair (slice r) is causal attention of two equal
  slices; slices before it are seen whole; slices after it are hidden and
  skipped (the plain reading of "causal" for the whole sequence, i.e. key j
  visible to query i iff j <= i, split into blocks).  Non-causal: every pair
  is seen whole.  Sliding windows are not supported here.
* forward: fa_fwd gives each pair's (O_t, LSE_t); fa_lse_merge folds them,
  in step order, into an fp32 running result (abeam.tech FlashAttention
  summary, "computing softmax blockwise correctly", applied to whole key
  slices).
* backward: fa_bwd of a pair, given the full rows' O and LSE, gives that
  key slice's share of dQ and its dK / dV; dQ shares add up on the rank, and
  each key slice's dK / dV accumulators travel with it and reach its owner
  after the last step (one more pass along the ring).  All sums run in fp32
  (fa_grad_accumulate) in a fixed order, so results are the same on every
  run.

The slices land in this rank's own memory before any kernel reads them
(NCCL point-to-point sends / receives through torch.distributed, or copies
in the single-process emulation); no kernel reads another GPU's memory.

Two sets of entry points share the per-rank steps: ``ring_attention_forward`` /
``ring_attention_backward`` run one rank of a torch.distributed process group
(the exchange of step t + 1's slice overlaps step t's kernels);
``local_ring_forward`` / ``local_ring_backward`` run all R ranks in one
process, the exchange being a copy (tests, and single-GPU measurement).
``ops`` supplies the block computations -- by default the library's kernels
(``LibraryOps``); there is no other implementation in the package.
"""
import math

__all__ = ["block_mode", "LibraryOps", "ForwardRank", "BackwardRank", "ring_attention_forward",
           "ring_attention_backward", "local_ring_forward", "local_ring_backward"]


def block_mode(r, src, causal):
    """How query slice r attends to key slice src of an equal split:
    'full', 'causal' (the diagonal pair) or None (every key hidden)."""
    if not causal or src < r:
        return "full"
    return "causal" if src == r else None


class LibraryOps:
    """The block computations on CUDA tensors through the library's C ABI."""

    def __init__(self):
        from . import attention_backward, attention_forward, grad_accumulate, lse_merge
        self._fwd, self._bwd = attention_forward, attention_backward
        self._merge, self._acc = lse_merge, grad_accumulate

    def fwd(self, q, k, v, scale, causal):
        return self._fwd(q, k, v, scale=scale, causal=causal)

    def new_fwd_acc(self, q):
        import torch
        B, n, H, d = q.shape
        return (torch.empty((B, n, H, d), dtype=torch.float32, device=q.device),
                torch.empty((B, H, n), dtype=torch.float32, device=q.device))

    def new_out(self, q):
        import torch
        return torch.empty_like(q)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, out):
        self._merge(o_acc, lse_acc, o_part, lse_part, first=first, out=out)

    def bwd(self, q, k, v, o, lse, do, scale, causal):
        return self._bwd(q, k, v, o, lse, do, scale=scale, causal=causal)

    def new_grad_acc(self, x):
        import torch
        return torch.empty(x.shape, dtype=torch.float32, device=x.device)

    def accumulate(self, acc, part, first):
        self._acc(acc, part, first=first)

    def finish_grad(self, acc, like):
        import torch
        out = torch.empty_like(like)
        self._acc(acc, None, out=out)
        return out


class ForwardRank:
    """Rank r's forward steps: step(t, k_slice, v_slice) for t = 0 .. R - 1,
    then result() -> (o, lse) of its query rows over the whole sequence."""

    def __init__(self, r, R, q, ops, scale, causal):
        self.r, self.R, self.q, self.ops = r, R, q, ops
        self.scale, self.causal = scale, causal
        active = [t for t in range(R) if block_mode(r, (r - t) % R, causal)]
        self.last = active[-1]  # always >= 0: the diagonal pair (t = 0) is seen
        self.o_acc, self.lse_acc = ops.new_fwd_acc(q)
        self.out = ops.new_out(q)
        self.first = True

    def step(self, t, k, v):
        mode = block_mode(self.r, (self.r - t) % self.R, self.causal)
        if mode is None:
            return
        o_p, lse_p = self.ops.fwd(self.q, k, v, self.scale, mode == "causal")
        self.ops.merge(self.o_acc, self.lse_acc, o_p, lse_p, self.first, self.out if t == self.last else None)
        self.first = False

    def result(self):
        return self.out, self.lse_acc


class BackwardRank:
    """Rank r's backward steps.  step(t, k, v, dk_acc, dv_acc) adds the pair's
    shares: dQ into this rank's accumulator, dK / dV into the travelling
    accumulators of the key slice (the slice's owner initialises them at
    t = 0, the diagonal pair, which every rank computes)."""

    def __init__(self, r, R, q, o, lse, do, ops, scale, causal):
        self.r, self.R = r, R
        self.q, self.o, self.lse, self.do = q, o, lse, do
        self.ops, self.scale, self.causal = ops, scale, causal
        self.dq_acc = ops.new_grad_acc(q)

    def step(self, t, k, v, dk_acc, dv_acc):
        mode = block_mode(self.r, (self.r - t) % self.R, self.causal)
        if mode is None:
            return
        dq, dk, dv = self.ops.bwd(self.q, k, v, self.o, self.lse, self.do, self.scale, mode == "causal")
        self.ops.accumulate(self.dq_acc, dq, t == 0)
        self.ops.accumulate(dk_acc, dk, t == 0)
        self.ops.accumulate(dv_acc, dv, t == 0)

    def dq(self):
        return self.ops.finish_grad(self.dq_acc, self.q)


def _default_scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


# ------------------------------------------------------------ all ranks in one process

def local_ring_forward(qs, ks, vs, scale=None, causal=False, ops=None):
    """Forward of R ranks emulated in one process (lists of per-rank slices);
    returns the lists of per-rank o and lse."""
    ops = ops or LibraryOps()
    R = len(qs)
    scale = _default_scale(qs[0], scale)
    ranks = [ForwardRank(r, R, qs[r], ops, scale, causal) for r in range(R)]
    kv = [(ks[r], vs[r]) for r in range(R)]
    for t in range(R):
        for r in range(R):
            ranks[r].step(t, *kv[r])
        if t < R - 1:  # rank r receives what rank r - 1 held, in its own buffer
            kv = [(kv[(r - 1) % R][0].clone(), kv[(r - 1) % R][1].clone()) for r in range(R)]
    res = [x.result() for x in ranks]
    return [o for o, _ in res], [lse for _, lse in res]


def local_ring_backward(qs, ks, vs, os_, lses, dos, scale=None, causal=False, ops=None):
    """Backward of R ranks emulated in one process; returns lists of per-rank
    dq, dk, dv (each rank's own slices)."""
    ops = ops or LibraryOps()
    R = len(qs)
    scale = _default_scale(qs[0], scale)
    ranks = [BackwardRank(r, R, qs[r], os_[r], lses[r], dos[r], ops, scale, causal) for r in range(R)]
    carry = [(ks[r], vs[r], ops.new_grad_acc(ks[r]), ops.new_grad_acc(vs[r])) for r in range(R)]
    for t in range(R):
        for r in range(R):
            ranks[r].step(t, *carry[r])
        # every slice moves on; after the last step this returns it to its owner
        carry = [tuple(x.clone() for x in carry[(r - 1) % R]) for r in range(R)]
    dq = [x.dq() for x in ranks]
    dk = [ops.finish_grad(carry[r][2], ks[r]) for r in range(R)]
    dv = [ops.finish_grad(carry[r][3], vs[r]) for r in range(R)]
    return dq, dk, dv


# ------------------------------------------------------------ one rank of a process group

def _shift(tensors, group=None):
    """Send `tensors` to the next rank of the ring and receive the previous
    rank's into new buffers; returns (requests, received)."""
    import torch
    import torch.distributed as dist
    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt, prv = (r + 1) % R, (r - 1) % R
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    recv = [torch.empty_like(x) for x in tensors]
    ops = [dist.P2POp(dist.isend, x.contiguous(), nxt, group) for x in tensors]
    ops += [dist.P2POp(dist.irecv, x, prv, group) for x in recv]
    return dist.batch_isend_irecv(ops), recv


def _wait(reqs):
    for q in reqs:
        q.wait()


def ring_attention_forward(q, k, v, scale=None, causal=False, group=None, ops=None):
    """This rank's (o, lse) of ring attention over a torch.distributed group.
    The next key/value slice is exchanged while this step's kernels run."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    R, r = dist.get_world_size(group), dist.get_rank(group)
    me = ForwardRank(r, R, q, ops, _default_scale(q, scale), causal)
    kv = (k, v)
    for t in range(R):
        pending = _shift(kv, group) if t < R - 1 else None
        me.step(t, *kv)
        if pending is not None:
            _wait(pending[0])
            kv = tuple(pending[1])
    return me.result()


def ring_attention_backward(q, k, v, o, lse, do, scale=None, causal=False, group=None, ops=None):
    """This rank's (dq, dk, dv) of ring attention over a torch.distributed
    group: dq of its query rows, dk / dv of its own key/value rows (summed
    over every rank's queries).  The next key/value slice is exchanged while
    this step's kernels run; the dK / dV accumulators follow after the step."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    R, r = dist.get_world_size(group), dist.get_rank(group)
    me = BackwardRank(r, R, q, o, lse, do, ops, _default_scale(q, scale), causal)
    kv = (k, v)
    acc = (ops.new_grad_acc(k), ops.new_grad_acc(v))
    for t in range(R):
        pending = _shift(kv, group) if t < R - 1 else None
        me.step(t, kv[0], kv[1], acc[0], acc[1])
        reqs, got = _shift(acc, group)
        _wait(reqs)
        acc = tuple(got)
        if pending is not None:
            _wait(pending[0])
            kv = tuple(pending[1])
    return me.dq(), ops.finish_grad(acc[0], k), ops.finish_grad(acc[1], v)
