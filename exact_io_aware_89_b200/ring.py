"""Ring (context-parallel) exact attention: one long sequence split across
ranks (zocula.com fla guide, the flame bullets and the glossary entry on
context parallelism: long contexts are divided over several GPUs).

The sequence of N rows is cut into equal chunks.  In the 'contiguous'
layout rank r of R holds chunk r of R (rows [r n, (r + 1) n), n = N / R); in
the 'zigzag' layout it holds chunks r and 2R - 1 - r of 2R, one from each end,
so that under a causal mask every rank has the same work at every step (with
contiguous chunks rank R - 1 does 2R - 1 times rank 0's work).  A
rank keeps its query rows (and o, lse, dO for the backward); the key/value
chunks travel around the ring, rank r passing what it holds to rank r + 1
after each step, so at step t it holds rank (r - t) mod R's.  Each (query
chunk, key chunk) pair is an ordinary attention call of the library:

* causal: the diagonal pair (a chunk against itself) is causal attention of
  two equal chunks; earlier key chunks are seen whole; later ones are hidden
  and skipped (the plain reading of "causal" for the whole sequence, i.e.
  key j visible to query i iff j <= i, split into blocks).  Non-causal: every
  pair is seen whole.  Sliding windows are not supported here.
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

__all__ = ["block_mode", "rank_chunks", "LibraryOps", "ForwardRank", "BackwardRank",
           "ring_attention_forward", "ring_attention_backward", "local_ring_forward", "local_ring_backward"]

LAYOUTS = ("contiguous", "zigzag")


def block_mode(qc, kc, causal):
    """How query chunk qc attends to key chunk kc of an equal split of the
    sequence: 'full', 'causal' (the diagonal pair) or None (every key hidden)."""
    if not causal or kc < qc:
        return "full"
    return "causal" if kc == qc else None


def rank_chunks(r, R, layout="contiguous"):
    """The sequence chunks rank r of R holds, in its row order.  'contiguous':
    the r-th of R equal chunks.  'zigzag': chunks r and 2R - 1 - r of 2R, which
    gives every rank the same causal work at every step."""
    if layout == "contiguous":
        return [r]
    if layout == "zigzag":
        return [r, 2 * R - 1 - r]
    raise ValueError("layout must be one of %s" % (LAYOUTS,))


def _split(x, n, dim=1):
    """The rank's rows as n equal chunks, each a contiguous tensor."""
    if n == 1:
        return [x]
    size = x.shape[dim] // n
    return [x.narrow(dim, i * size, size).contiguous() for i in range(n)]


def _join(xs, dim=1):
    if len(xs) == 1:
        return xs[0]
    import torch
    return torch.cat(xs, dim=dim)


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


def _schedule(r, R, layout, causal):
    """[(t, query chunk position, key chunk position, mode)] of rank r's
    visible pairs, in the order they are computed: steps, then query chunks,
    then key chunks."""
    mine = rank_chunks(r, R, layout)
    out = []
    for t in range(R):
        theirs = rank_chunks((r - t) % R, R, layout)
        for i, qc in enumerate(mine):
            for j, kc in enumerate(theirs):
                mode = block_mode(qc, kc, causal)
                if mode is not None:
                    out.append((t, i, j, mode))
    return out


class ForwardRank:
    """Rank r's forward steps: step(t, k_chunks, v_chunks) for t = 0 .. R - 1
    with the key/value chunks held at step t, then result() -> (o, lse) of its
    query rows over the whole sequence, in its row order."""

    def __init__(self, r, R, q, ops, scale, causal, layout="contiguous"):
        self.r, self.R, self.ops = r, R, ops
        self.scale, self.causal, self.layout = scale, causal, layout
        self.qs = _split(q, len(rank_chunks(r, R, layout)))
        self.sched = _schedule(r, R, layout, causal)
        # the last pair of each query chunk writes its rounded output
        self.last = {}
        for t, i, j, _ in self.sched:
            self.last[i] = (t, j)
        self.acc = [ops.new_fwd_acc(x) for x in self.qs]
        self.out = [ops.new_out(x) for x in self.qs]
        self.first = [True] * len(self.qs)

    def step(self, t, ks, vs):
        for tt, i, j, mode in self.sched:
            if tt != t:
                continue
            o_p, lse_p = self.ops.fwd(self.qs[i], ks[j], vs[j], self.scale, mode == "causal")
            o_acc, lse_acc = self.acc[i]
            self.ops.merge(o_acc, lse_acc, o_p, lse_p, self.first[i],
                           self.out[i] if self.last[i] == (t, j) else None)
            self.first[i] = False

    def result(self):
        return _join(self.out, 1), _join([lse for _, lse in self.acc], 2)


class BackwardRank:
    """Rank r's backward steps.  step(t, k_chunks, v_chunks, dk_accs,
    dv_accs) adds each visible pair's shares: dQ into this rank's
    accumulators, dK / dV into the travelling accumulators of the key chunks
    (every rank computes the diagonal pairs of its own chunks at t = 0, so the
    owner initialises them then)."""

    def __init__(self, r, R, q, o, lse, do, ops, scale, causal, layout="contiguous"):
        n = len(rank_chunks(r, R, layout))
        self.r, self.R, self.ops = r, R, ops
        self.scale, self.causal, self.layout = scale, causal, layout
        self.qs, self.os, self.dos = _split(q, n), _split(o, n), _split(do, n)
        self.lses = _split(lse, n, dim=2)
        self.sched = _schedule(r, R, layout, causal)
        self.dq_acc = [ops.new_grad_acc(x) for x in self.qs]
        self.dq_first = [True] * n

    def step(self, t, ks, vs, dk_accs, dv_accs):
        kv_first = [t == 0] * len(ks)
        for tt, i, j, mode in self.sched:
            if tt != t:
                continue
            dq, dk, dv = self.ops.bwd(self.qs[i], ks[j], vs[j], self.os[i], self.lses[i], self.dos[i],
                                      self.scale, mode == "causal")
            self.ops.accumulate(self.dq_acc[i], dq, self.dq_first[i])
            self.ops.accumulate(dk_accs[j], dk, kv_first[j])
            self.ops.accumulate(dv_accs[j], dv, kv_first[j])
            self.dq_first[i] = False
            kv_first[j] = False

    def dq(self):
        return _join([self.ops.finish_grad(a, x) for a, x in zip(self.dq_acc, self.qs)], 1)


def _default_scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


# ------------------------------------------------------------ all ranks in one process

def local_ring_forward(qs, ks, vs, scale=None, causal=False, ops=None, layout="contiguous"):
    """Forward of R ranks emulated in one process (lists of per-rank rows, in
    each rank's row order for the layout); returns the lists of per-rank o and
    lse."""
    ops = ops or LibraryOps()
    R = len(qs)
    scale = _default_scale(qs[0], scale)
    n = len(rank_chunks(0, R, layout))
    ranks = [ForwardRank(r, R, qs[r], ops, scale, causal, layout) for r in range(R)]
    kv = [(_split(ks[r], n), _split(vs[r], n)) for r in range(R)]
    for t in range(R):
        for r in range(R):
            ranks[r].step(t, *kv[r])
        if t < R - 1:  # rank r receives what rank r - 1 held, in its own buffers
            kv = [tuple([x.clone() for x in part] for part in kv[(r - 1) % R]) for r in range(R)]
    res = [x.result() for x in ranks]
    return [o for o, _ in res], [lse for _, lse in res]


def local_ring_backward(qs, ks, vs, os_, lses, dos, scale=None, causal=False, ops=None, layout="contiguous"):
    """Backward of R ranks emulated in one process; returns lists of per-rank
    dq, dk, dv (each rank's own rows, in its row order)."""
    ops = ops or LibraryOps()
    R = len(qs)
    scale = _default_scale(qs[0], scale)
    n = len(rank_chunks(0, R, layout))
    ranks = [BackwardRank(r, R, qs[r], os_[r], lses[r], dos[r], ops, scale, causal, layout) for r in range(R)]
    carry = []
    for r in range(R):
        kc, vc = _split(ks[r], n), _split(vs[r], n)
        carry.append((kc, vc, [ops.new_grad_acc(x) for x in kc], [ops.new_grad_acc(x) for x in vc]))
    for t in range(R):
        for r in range(R):
            ranks[r].step(t, *carry[r])
        # every chunk moves on; after the last step this returns it to its owner
        carry = [tuple([x.clone() for x in part] for part in carry[(r - 1) % R]) for r in range(R)]
    dq = [x.dq() for x in ranks]
    dk = [_join([ops.finish_grad(a, x) for a, x in zip(carry[r][2], carry[r][0])], 1) for r in range(R)]
    dv = [_join([ops.finish_grad(a, x) for a, x in zip(carry[r][3], carry[r][1])], 1) for r in range(R)]
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


def ring_attention_forward(q, k, v, scale=None, causal=False, group=None, ops=None, layout="contiguous"):
    """This rank's (o, lse) of ring attention over a torch.distributed group,
    its rows in the layout's order.  The next key/value chunks are exchanged
    while this step's kernels run."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    R, r = dist.get_world_size(group), dist.get_rank(group)
    n = len(rank_chunks(r, R, layout))
    me = ForwardRank(r, R, q, ops, _default_scale(q, scale), causal, layout)
    kc, vc = _split(k, n), _split(v, n)
    for t in range(R):
        pending = _shift(kc + vc, group) if t < R - 1 else None
        me.step(t, kc, vc)
        if pending is not None:
            _wait(pending[0])
            kc, vc = pending[1][:n], pending[1][n:]
    return me.result()


def ring_attention_backward(q, k, v, o, lse, do, scale=None, causal=False, group=None, ops=None,
                            layout="contiguous"):
    """This rank's (dq, dk, dv) of ring attention over a torch.distributed
    group: dq of its query rows, dk / dv of its own key/value rows (summed
    over every rank's queries), in the layout's row order.  The next
    key/value chunks are exchanged while this step's kernels run; the dK / dV
    accumulators follow after the step."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    R, r = dist.get_world_size(group), dist.get_rank(group)
    n = len(rank_chunks(r, R, layout))
    me = BackwardRank(r, R, q, o, lse, do, ops, _default_scale(q, scale), causal, layout)
    kc, vc = _split(k, n), _split(v, n)
    dk_acc = [ops.new_grad_acc(x) for x in kc]
    dv_acc = [ops.new_grad_acc(x) for x in vc]
    for t in range(R):
        pending = _shift(kc + vc, group) if t < R - 1 else None
        me.step(t, kc, vc, dk_acc, dv_acc)
        reqs, got = _shift(dk_acc + dv_acc, group)
        _wait(reqs)
        dk_acc, dv_acc = got[:n], got[n:]
        if pending is not None:
            _wait(pending[0])
            kc, vc = pending[1][:n], pending[1][n:]
    like_k = _split(k, n)
    dk = _join([ops.finish_grad(a, x) for a, x in zip(dk_acc, like_k)], 1)
    dv = _join([ops.finish_grad(a, x) for a, x in zip(dv_acc, like_k)], 1)
    return me.dq(), dk, dv
