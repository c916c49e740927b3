"""Partitions of the path over ranks (one process per GPU, torch.distributed).

The pages give the path no collective; the Baidu guide ("A Guide to Sparse
Attention in Large Models", section 4.2) warns that index-based sparsity is
unfriendly to tensor and sequence parallelism, because every query may need
any earlier key.  The two partitions here are the ones the path allows:

* Prefill, query rows.  The N query rows of one causal sequence are cut into
  ``world`` contiguous chunks of about equal work (the causal rows grow with
  their position, so later chunks are shorter).  Each rank starts with an
  equal shard of the sequence's k, v and index keys kI, and one all-gather
  gives every rank the whole key range; rank r then runs the path for its
  rows t0..t1-1 as the last t1 - t0 queries of a t1-key sequence (keys past t1
  are never needed).  That all-gather is the only exchange; remote rows are
  copied into this GPU's memory before any kernel reads them.
* Decode, sequences.  Whole sequences are dealt to ranks, longest first to the
  least loaded rank.  The step has no exchange; the outputs are collected in
  batch order by one all-gather when a caller needs them on every rank.

Nothing here computes any part of the method: it picks bounds, moves rows
and hands each rank's share to a plan (``pipeline.PrefillPlan`` /
``DecodePlan`` by default).
"""

from __future__ import annotations

import numpy as np


def prefill_row_cost(N, K, W, Hq, d, H_I, D_I, block=None, keep=None) -> np.ndarray:
    """Work of each query row t = 0..N-1 in flops: the indexer over the row's
    scored keys (every causal key, or for the two-stage selection its coarse
    blocks and its candidates) plus the attention over min(t+1, K+W) keys."""
    t = np.arange(N, dtype=np.float64)
    if block is None:
        scored = t + 1
    else:
        scored = np.floor(t / block) + np.minimum(np.floor(t / block), keep) * block + (t % block) + 1
    return 2.0 * scored * H_I * D_I + 4.0 * np.minimum(t + 1, K + W) * Hq * d


def causal_chunk_bounds(cost, world: int) -> list:
    """Bounds 0 = b[0] <= b[1] <= ... <= b[world] = N of contiguous row chunks
    whose summed costs are as equal as cutting between rows allows: chunk r
    ends at the first row whose cumulative cost reaches (r+1)/world of the
    total."""
    cost = np.asarray(cost, dtype=np.float64)
    N = len(cost)
    if world < 1:
        raise ValueError("world must be >= 1")
    cum = np.cumsum(cost)
    total = cum[-1] if N else 0.0
    bounds = [0]
    for r in range(1, world):
        cut = int(np.searchsorted(cum, total * r / world, side="left")) + 1
        bounds.append(min(N, max(bounds[-1], cut)))
    bounds.append(N)
    return bounds


def key_shard_bounds(N: int, world: int) -> list:
    """Equal contiguous shards of the N key rows (the last may be shorter)."""
    per = -(-N // world) if world else 0
    return [min(N, r * per) for r in range(world)] + [N]


def decode_assignment(lengths, world: int) -> list:
    """Sequence indices per rank: longest first, each to the rank with the
    least cached tokens so far (ties to the lower rank); each rank's list is
    ascending."""
    lengths = [int(x) for x in lengths]
    load = [0] * world
    owned = [[] for _ in range(world)]
    for b in sorted(range(len(lengths)), key=lambda i: (-lengths[i], i)):
        r = min(range(world), key=lambda i: (load[i], i))
        owned[r].append(b)
        load[r] += lengths[b]
    return [sorted(o) for o in owned]


def gather_chunks(local, bounds, group=None):
    """The [bounds[-1], ...] tensor whose rows bounds[r] .. bounds[r+1]-1 are
    rank r's `local` rows (chunks may differ in length, and may be empty):
    one all_gather of chunks padded to the longest.  Rows travel as raw bytes,
    so any element type works on any backend."""
    import torch
    import torch.distributed as dist
    world = len(bounds) - 1
    N = bounds[-1]
    per = max(bounds[r + 1] - bounds[r] for r in range(world)) if world else 0
    row_shape = tuple(local.shape[1:])
    row_bytes = (int(np.prod(row_shape)) if row_shape else 1) * local.element_size()
    raw = local.contiguous().view(torch.uint8).reshape(local.shape[0], row_bytes)
    pad = torch.zeros((max(per, 1), row_bytes), dtype=torch.uint8, device=local.device)
    pad[:raw.shape[0]] = raw
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    rows = torch.cat([parts[r][:bounds[r + 1] - bounds[r]] for r in range(world)], dim=0)
    return rows.contiguous().view(local.dtype).reshape((N,) + row_shape)


def all_gather_rows(shard, N: int, world: int, group=None):
    """The full [N, ...] tensor from every rank's equal shard (rows
    key_shard_bounds(N, world)[r] .. [r+1] on rank r)."""
    return gather_chunks(shard, key_shard_bounds(N, world), group)


class ShardedPrefill:
    """One rank's share of a prefill step over a query-row partition.

    N queries at positions 0..N-1 of one causal sequence; rank `rank` of
    `world` owns rows t0 = bounds[rank] .. t1 = bounds[rank + 1] - 1 and the key
    shard key_shard_bounds(N, world)[rank] .. [rank + 1].
    make_plan(T, S) -> an object with .run(q, k, v, qI, w, kI) for T queries at
    the last T of S keys (default: pipeline.PrefillPlan)."""

    def __init__(self, N, Hq, d, H_I, D_I, K, W, rank, world, block=None, keep=None, group=None,
                 device="cuda", make_plan=None):
        self.N, self.rank, self.world, self.group = N, rank, world, group
        cost = prefill_row_cost(N, K, W, Hq, d, H_I, D_I, block, keep)
        self.bounds = causal_chunk_bounds(cost, world)
        self.t0, self.t1 = self.bounds[rank], self.bounds[rank + 1]
        self.key_bounds = key_shard_bounds(N, world)
        T, S = self.t1 - self.t0, self.t1
        if make_plan is None:
            from .pipeline import PrefillPlan
            make_plan = lambda T, S: PrefillPlan(T, Hq, d, H_I, D_I, K, W, block=block, keep=keep,
                                                 device=device, S=S)
        self.plan = make_plan(T, S) if T > 0 else None

    def gather_keys(self, k_shard, v_shard, kI_shard):
        """Every rank's key shards -> this rank's key range 0..t1-1."""
        full = [all_gather_rows(x, self.N, self.world, self.group) for x in (k_shard, v_shard, kI_shard)]
        return [x[:self.t1] for x in full]

    def run(self, q_rows, qI_rows, w_rows, k_shard, v_shard, kI_shard):
        """q_rows / qI_rows / w_rows: this rank's query rows t0..t1-1;
        *_shard: this rank's key shard.  Returns the plan's output for the
        rank's rows (None when the rank owns no row)."""
        k, v, kI = self.gather_keys(k_shard, v_shard, kI_shard)
        if self.plan is None:
            return None
        return self.plan.run(q_rows, k, v, qI_rows, w_rows, kI)

    def collect(self, rows):
        """Every rank's result rows (this rank's: `rows`, [t1 - t0, ...], any
        dtype) -> the full [N, ...] tensor on every rank, in query order."""
        return gather_chunks(rows, self.bounds, self.group)


class ShardedDecode:
    """One rank's share of a decode step over a batch split.

    Whole sequences are dealt by decode_assignment (longest first to the rank
    with the fewest cached tokens); each rank holds the caches of its own
    sequences and runs its plan on them alone, so the step itself has no
    exchange.  select() picks this rank's rows out of a batch-ordered array,
    collect() puts every rank's result rows back in batch order on every
    rank (one all_gather)."""

    def __init__(self, lengths, rank, world, group=None):
        self.lengths = [int(x) for x in lengths]
        self.rank, self.world, self.group = rank, world, group
        self.owned_by = decode_assignment(self.lengths, world)
        self.owned = self.owned_by[rank]
        counts = [len(o) for o in self.owned_by]
        self.bounds = [0] + list(np.cumsum(counts).astype(int))
        # batch index of each row of the gathered tensor
        self.order = [b for o in self.owned_by for b in o]

    def select(self, x):
        """Rows of this rank's sequences (ascending batch index) of a
        batch-ordered array or tensor."""
        return x[self.owned]

    def collect(self, rows):
        """This rank's result rows ([len(owned), ...]) -> the batch-ordered
        [B, ...] tensor on every rank."""
        import torch
        gathered = gather_chunks(rows, self.bounds, self.group)
        out = torch.empty_like(gathered)
        out[torch.as_tensor(self.order, dtype=torch.long, device=gathered.device)] = gathered
        return out
