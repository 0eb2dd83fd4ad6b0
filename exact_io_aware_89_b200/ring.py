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
after each step, so at step t it holds rank (r - t) mod R's.  Between a
query chunk and a key chunk:

* causal: the diagonal pair (a chunk against itself) is causal attention of
  two equal chunks; earlier key chunks are seen whole; later ones are hidden
  and skipped (the plain reading of "causal" for the whole sequence, i.e.
  key j visible to query i iff j <= i, split into blocks).  Non-causal: every
  pair is seen whole.  Sliding windows are not supported here.
* the visible pairs of one step are one ordinary attention call of the
  library over a range of the rank's rows.  Zig-zag, rank r holding chunks
  lo = r, hi = 2R - 1 - r, and rank s's keys: s = r, causal attention over
  all of its rows (its chunks are in sequence order); s < r, all query rows
  against chunk s alone, whole; s > r, the hi rows against all of s's keys,
  whole.  Contiguous: the whole rows, whole or causal, or nothing.
* forward: fa_fwd gives each call's (O_t, LSE_t); fa_lse_merge folds them,
  in step order, into an fp32 running result (abeam.tech FlashAttention
  summary, "computing softmax blockwise correctly", applied to whole key
  slices).
* backward: fa_bwd of a call, given the full rows' O and LSE, gives those
  keys' share of dQ and their dK / dV; dQ shares add up on the rank, and
  each rank's dK / dV accumulators travel with its keys and reach their owner
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

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, out, row0):
        self._merge(o_acc, lse_acc, o_part, lse_part, first=first, out=out, row0=row0)

    def bwd(self, q, k, v, o, lse, do, scale, causal):
        return self._bwd(q, k, v, o, lse, do, scale=scale, causal=causal)

    def new_grad_acc(self, x):
        import torch
        return torch.empty(x.shape, dtype=torch.float32, device=x.device)

    def accumulate(self, acc, part, first, row0):
        self._acc(acc, part, first=first, row0=row0)

    def finish_grad(self, acc, like):
        import torch
        out = torch.empty_like(like)
        self._acc(acc, None, out=out)
        return out


def _chunk_pairs(r, R, t, layout, causal):
    """{(query chunk position, key chunk position): mode} of the visible pairs
    of rank r at step t, when it holds rank (r - t) mod R's keys / values."""
    theirs = rank_chunks((r - t) % R, R, layout)
    out = {}
    for i, qc in enumerate(rank_chunks(r, R, layout)):
        for j, kc in enumerate(theirs):
            mode = block_mode(qc, kc, causal)
            if mode is not None:
                out[(i, j)] = mode
    return out


def _calls(pairs, n):
    """Attention calls covering the visible chunk pairs of one step, each over
    a range of the rank's rows: [((i0, i1), (j0, j1), causal)], ranges of
    chunk positions.  One call when the pairs form a rectangle seen whole, or
    when they are the whole square with the diagonal causal, below it whole and
    above it hidden (a rank's chunks are in sequence order, so that is causal
    attention over all of its rows); otherwise one call per pair."""
    if not pairs:
        return []
    I = sorted({i for i, _ in pairs})
    J = sorted({j for _, j in pairs})
    ranges = I == list(range(I[0], I[-1] + 1)) and J == list(range(J[0], J[-1] + 1))
    if ranges and all(pairs.get((i, j)) == "full" for i in I for j in J):
        return [((I[0], I[-1] + 1), (J[0], J[-1] + 1), False)]
    square = {(i, j): "causal" if i == j else "full" for i in range(n) for j in range(i + 1)}
    if pairs == square:
        return [((0, n), (0, n), True)]
    return [((i, i + 1), (j, j + 1), mode == "causal") for (i, j), mode in sorted(pairs.items())]


def _schedule(r, R, layout, causal):
    """[(t, query chunk range, key chunk range, causal)]: rank r's attention
    calls in the order they run.  Both layouts need one call per step (none
    at the hidden steps of the contiguous layout)."""
    n = len(rank_chunks(r, R, layout))
    return [(t,) + call for t in range(R) for call in _calls(_chunk_pairs(r, R, t, layout, causal), n)]


def _take_first(seen, rng):
    """Whether a call over chunk range rng is the first to reach its rows (all
    or none of them must have been reached before); marks them reached."""
    before = {seen[i] for i in range(*rng)}
    if len(before) != 1:
        raise RuntimeError("a call reaches rows of which only some were reached before")
    for i in range(*rng):
        seen[i] = True
    return not before.pop()


class _Rows:
    """Row ranges (in chunk positions) of a rank's tensors, each a contiguous
    tensor: the tensor itself for all rows (and, for one batch, a view of
    any range of dim 1), else a copy."""

    def __init__(self, n_chunks, rows):
        self.n, self.c = n_chunks, rows // n_chunks

    def __call__(self, x, rng, dim=1):
        if tuple(rng) == (0, self.n):
            return x
        return x.narrow(dim, rng[0] * self.c, (rng[1] - rng[0]) * self.c).contiguous()


class ForwardRank:
    """Rank r's forward steps: step(t, k, v) for t = 0 .. R - 1 with the
    key/value rows held at step t, then result() -> (o, lse) of its query rows
    over the whole sequence, in its row order."""

    def __init__(self, r, R, q, ops, scale, causal, layout="contiguous"):
        self.r, self.R, self.ops = r, R, ops
        self.scale, self.causal, self.layout = scale, causal, layout
        n = len(rank_chunks(r, R, layout))
        self.rows = _Rows(n, q.shape[1])
        self.q = q
        self.q_rows = {}
        self.sched = _schedule(r, R, layout, causal)
        # the last call that reaches each query chunk writes its rounded output
        self.last = {}
        for idx, (_, qr, _, _) in enumerate(self.sched):
            for i in range(*qr):
                self.last[i] = idx
        self.o_acc, self.lse_acc = ops.new_fwd_acc(q)
        self.out = ops.new_out(q)
        self.seen = [False] * n

    def step(self, t, k, v):
        for idx, (tt, qr, kr, causal) in enumerate(self.sched):
            if tt != t:
                continue
            if qr not in self.q_rows:
                self.q_rows[qr] = self.rows(self.q, qr)
            o_p, lse_p = self.ops.fwd(self.q_rows[qr], self.rows(k, kr), self.rows(v, kr), self.scale, causal)
            write = any(self.last[i] == idx for i in range(*qr))
            self.ops.merge(self.o_acc, self.lse_acc, o_p, lse_p, _take_first(self.seen, qr),
                           self.out if write else None, qr[0] * self.rows.c)

    def result(self):
        return self.out, self.lse_acc


class BackwardRank:
    """Rank r's backward steps.  step(t, k, v, dk_acc, dv_acc) adds each call's
    shares: dQ into this rank's accumulator, dK / dV into the travelling
    accumulators of the key rows it holds (every rank reaches all of its own
    key rows at t = 0, so the owner initialises them then)."""

    def __init__(self, r, R, q, o, lse, do, ops, scale, causal, layout="contiguous"):
        n = len(rank_chunks(r, R, layout))
        self.r, self.R, self.ops, self.n = r, R, ops, n
        self.scale, self.causal, self.layout = scale, causal, layout
        self.rows = _Rows(n, q.shape[1])
        self.q, self.o, self.lse, self.do = q, o, lse, do
        self.q_rows = {}
        self.sched = _schedule(r, R, layout, causal)
        self.dq_acc = ops.new_grad_acc(q)
        self.dq_seen = [False] * n

    def step(self, t, k, v, dk_acc, dv_acc):
        kv_seen = [t != 0] * self.n
        for tt, qr, kr, causal in self.sched:
            if tt != t:
                continue
            if qr not in self.q_rows:
                self.q_rows[qr] = (self.rows(self.q, qr), self.rows(self.o, qr), self.rows(self.lse, qr, 2),
                                   self.rows(self.do, qr))
            q, o, lse, do = self.q_rows[qr]
            dq, dk, dv = self.ops.bwd(q, self.rows(k, kr), self.rows(v, kr), o, lse, do, self.scale, causal)
            c = self.rows.c
            self.ops.accumulate(self.dq_acc, dq, _take_first(self.dq_seen, qr), qr[0] * c)
            first = _take_first(kv_seen, kr)
            self.ops.accumulate(dk_acc, dk, first, kr[0] * c)
            self.ops.accumulate(dv_acc, dv, first, kr[0] * c)
        if not all(kv_seen):
            raise RuntimeError("the first step must reach every key row of the rank")

    def dq(self):
        return self.ops.finish_grad(self.dq_acc, self.q)


def _default_scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


# ------------------------------------------------------------ all ranks in one process

class _NoTimer:
    def start(self, t, r):
        pass

    def stop(self, t, r):
        pass


def local_ring_forward(qs, ks, vs, scale=None, causal=False, ops=None, layout="contiguous", timer=None):
    """Forward of R ranks emulated in one process (lists of per-rank rows, in
    each rank's row order for the layout); returns the lists of per-rank o and
    lse.  ``timer.start(t, r)`` / ``timer.stop(t, r)``, if given, bracket rank
    r's work at step t."""
    ops = ops or LibraryOps()
    timer = timer or _NoTimer()
    R = len(qs)
    scale = _default_scale(qs[0], scale)
    ranks = [ForwardRank(r, R, qs[r], ops, scale, causal, layout) for r in range(R)]
    kv = [(ks[r], vs[r]) for r in range(R)]
    for t in range(R):
        for r in range(R):
            timer.start(t, r)
            ranks[r].step(t, *kv[r])
            timer.stop(t, r)
        if t < R - 1:  # rank r receives what rank r - 1 held, in its own buffers
            kv = [tuple(x.clone() for x in kv[(r - 1) % R]) for r in range(R)]
    res = [x.result() for x in ranks]
    return [o for o, _ in res], [lse for _, lse in res]


def local_ring_backward(qs, ks, vs, os_, lses, dos, scale=None, causal=False, ops=None, layout="contiguous",
                        timer=None):
    """Backward of R ranks emulated in one process; returns lists of per-rank
    dq, dk, dv (each rank's own rows, in its row order).  ``timer`` as in
    local_ring_forward."""
    ops = ops or LibraryOps()
    timer = timer or _NoTimer()
    R = len(qs)
    scale = _default_scale(qs[0], scale)
    ranks = [BackwardRank(r, R, qs[r], os_[r], lses[r], dos[r], ops, scale, causal, layout) for r in range(R)]
    carry = [(ks[r], vs[r], ops.new_grad_acc(ks[r]), ops.new_grad_acc(vs[r])) for r in range(R)]
    for t in range(R):
        for r in range(R):
            timer.start(t, r)
            ranks[r].step(t, *carry[r])
            timer.stop(t, r)
        # every rank's rows move on; after the last step this returns them to their owner
        carry = [tuple(x.clone() for x in carry[(r - 1) % R]) for r in range(R)]
    dq = [x.dq() for x in ranks]
    dk = [ops.finish_grad(carry[r][2], carry[r][0]) for r in range(R)]
    dv = [ops.finish_grad(carry[r][3], carry[r][1]) for r in range(R)]
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
    its rows in the layout's order.  The next key/value rows are exchanged
    while this step's kernels run."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    R, r = dist.get_world_size(group), dist.get_rank(group)
    me = ForwardRank(r, R, q, ops, _default_scale(q, scale), causal, layout)
    for t in range(R):
        pending = _shift([k, v], group) if t < R - 1 else None
        me.step(t, k, v)
        if pending is not None:
            _wait(pending[0])
            k, v = pending[1]
    return me.result()


def ring_attention_backward(q, k, v, o, lse, do, scale=None, causal=False, group=None, ops=None,
                            layout="contiguous"):
    """This rank's (dq, dk, dv) of ring attention over a torch.distributed
    group: dq of its query rows, dk / dv of its own key/value rows (summed
    over every rank's queries), in the layout's row order.  The next
    key/value rows are exchanged while this step's kernels run; the dK / dV
    accumulators follow after the step."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    R, r = dist.get_world_size(group), dist.get_rank(group)
    me = BackwardRank(r, R, q, o, lse, do, ops, _default_scale(q, scale), causal, layout)
    like_k, like_v = k, v
    dk_acc, dv_acc = ops.new_grad_acc(k), ops.new_grad_acc(v)
    for t in range(R):
        pending = _shift([k, v], group) if t < R - 1 else None
        me.step(t, k, v, dk_acc, dv_acc)
        reqs, got = _shift([dk_acc, dv_acc], group)
        _wait(reqs)
        dk_acc, dv_acc = got
        if pending is not None:
            _wait(pending[0])
            k, v = pending[1]
    return me.dq(), ops.finish_grad(dk_acc, like_k), ops.finish_grad(dv_acc, like_v)
