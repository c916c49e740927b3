"""The three-stage step built from the C-ABI calls, with buffers allocated once.

A plan owns its intermediate buffers (torch device tensors) and enqueues the
library's kernels on one stream; the host does no arithmetic of the method.

    PrefillPlan    indexer -> top-K -> sparse attention for one causal
                   sequence (optionally the two-stage coarse/fine selection)
    DecodePlan     one new query per sequence over a contiguous or paged
                   KV cache: indexer -> top-K -> split-K attention + merge
    HostPipeline   steps fed from and read back to pinned host memory, the
                   copies of neighbouring steps overlapped with the kernels

``stages(inputs)`` returns the step as a list of (name, launch) pairs, one
per C-ABI call, so that callers can time each kernel; ``run`` executes them.
"""

from __future__ import annotations

import math

import torch

from . import (sa_block_scores_workspace_bytes, sa_coarse_block_counts, sa_decode_workspace_bytes,
               sa_indexer_scores, sa_indexer_scores_blocks, sa_indexer_scores_fp8, sa_indexer_topk_decode,
               sa_pool_index_keys,
               sa_prefill_workspace_bytes, sa_sparse_attn_decode, sa_sparse_attn_prefill, sa_topk_select,
               sa_topk_select_blocks)


def _ld(n: int) -> int:
    return max(4, (n + 3) // 4 * 4)


class PrefillPlan:
    """Buffers for N queries of one causal sequence of S keys (default S = N):
    the queries sit at the last N positions, S - N .. S - 1 (S > N is one
    rank's chunk of a longer sequence, see ``shard``).
    Inputs: dict with q [N,Hq,d], qI [N,H_I,D_I], w [N,H_I] and k/v [S,d],
    kI [S,D_I].
    index_fp8: qI and kI are e4m3 bytes (uint8) and the indexer runs in FP8
    (single-stage selection only)."""

    def __init__(self, N, Hq, d, H_I, D_I, K, W, block=None, keep=None, row_blocks=1, index_fp8=False,
                 device="cuda", S=None):
        if index_fp8 and block is not None:
            raise ValueError("the FP8 indexer serves the single-stage selection")
        S = N if S is None else int(S)
        if S < N:
            raise ValueError("a plan's N queries are the last N of its S keys (S >= N)")
        self.N, self.S, self.Hq, self.d, self.H_I, self.D_I, self.K, self.W = N, S, Hq, d, H_I, D_I, K, W
        self.index = sa_indexer_scores_fp8 if index_fp8 else sa_indexer_scores
        self.block, self.keep = block, keep
        # single-stage only: score and select the queries in row_blocks blocks,
        # so that a block's scores are still in L2 when top-K reads them
        self.row_blocks = max(1, int(row_blocks)) if (block is None and S == N) else 1
        self.scale = 1.0 / math.sqrt(d)
        dev = torch.device(device)
        i32, f32 = torch.int32, torch.float32
        self.topk = torch.empty((N, K), dtype=i32, device=dev)
        self.out = torch.empty((N, Hq, d), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((N, Hq), dtype=f32, device=dev)
        self.dev_status = torch.zeros(1, dtype=i32, device=dev)
        # The masked tensor-core attention (selected by passing its bitmap
        # workspace) runs one CTA per 256 query-head rows; below one CTA per SM
        # the gathered kernel is faster.
        groups = N * Hq // 256
        sms = torch.cuda.get_device_properties(dev).multi_processor_count if dev.type == "cuda" else 148
        self.attn_ws_bytes = sa_prefill_workspace_bytes(N, S, K, W, Hq, d) if groups >= sms else 0
        self.attn_ws = (torch.empty(self.attn_ws_bytes, dtype=torch.uint8, device=dev)
                        if self.attn_ws_bytes else None)
        if block is None:
            self.ld = _ld(S)
            self.scores = torch.empty((N, self.ld), dtype=f32, device=dev)
        else:
            self.nb = S // block
            self.ld_coarse = _ld(self.nb)
            self.kB = torch.empty((max(self.nb, 1), D_I), dtype=torch.bfloat16, device=dev)
            self.n_blocks = torch.empty(N, dtype=i32, device=dev)
            self.coarse = torch.empty((N, self.ld_coarse), dtype=f32, device=dev)
            self.blocks = torch.empty((N, keep), dtype=i32, device=dev)
            self.ld_cand = _ld(keep * block + block)
            self.fine = torch.empty((N, self.ld_cand), dtype=f32, device=dev)
            self.ws_bytes = sa_block_scores_workspace_bytes(N, S, keep)
            self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)

    def stages(self, x, stream=None):
        N, S, K, ds, H, D = self.N, self.S, self.K, self.dev_status, self.H_I, self.D_I
        attn = ("attention", lambda: sa_sparse_attn_prefill(
            x["q"], x["k"], x["v"], self.topk, K, self.W, N, S, self.Hq, self.d, self.scale, self.out,
            self.lse, self.attn_ws, self.attn_ws_bytes, ds, stream))
        if self.block is None and self.row_blocks > 1:
            # queries t0..t1-1 are the last t1 - t0 of a t1-key causal sequence
            bounds = [N * b // self.row_blocks for b in range(self.row_blocks + 1)]
            out = []
            for b in range(self.row_blocks):
                t0, t1 = bounds[b], bounds[b + 1]
                if t1 <= t0:
                    continue
                out.append(("indexer", lambda t0=t0, t1=t1: self.index(
                    x["qI"][t0:t1], x["w"][t0:t1], x["kI"], None, 0, 0, 64, 1, t1 - t0, t1, H, D, None,
                    self.scores[t0:t1], self.ld, ds, stream)))
                out.append(("topk", lambda t0=t0, t1=t1: sa_topk_select(
                    self.scores[t0:t1], self.ld, t1 - t0, t1, None, None, 0, K, self.topk[t0:t1], ds, stream)))
            return out + [attn]
        if self.block is None:
            return [
                ("indexer", lambda: self.index(x["qI"], x["w"], x["kI"], None, 0, 0, 64, 1, N, S, H, D,
                                               None, self.scores, self.ld, ds, stream)),
                ("topk", lambda: sa_topk_select(self.scores, self.ld, N, S, None, None, 0, K, self.topk, ds,
                                                stream)),
                attn]
        blk, keep = self.block, self.keep
        return [
            ("pool", lambda: sa_pool_index_keys(x["kI"], S, D, blk, self.kB, stream)),
            ("block_counts", lambda: sa_coarse_block_counts(N, S, blk, self.n_blocks, stream)),
            ("coarse_indexer", lambda: sa_indexer_scores(x["qI"], x["w"], self.kB, None, 0, 0, 64, 1, N, self.nb,
                                                         H, D, self.n_blocks, self.coarse, self.ld_coarse, ds,
                                                         stream)),
            ("coarse_topk", lambda: sa_topk_select(self.coarse, self.ld_coarse, N, self.nb, self.n_blocks, None,
                                                   0, keep, self.blocks, ds, stream)),
            ("fine_indexer", lambda: sa_indexer_scores_blocks(x["qI"], x["w"], x["kI"], N, S, H, D, self.blocks,
                                                              keep, blk, self.fine, self.ld_cand, self.workspace,
                                                              self.ws_bytes, ds, stream)),
            ("fine_topk", lambda: sa_topk_select_blocks(self.fine, self.ld_cand, N, S, self.blocks, keep, blk, K,
                                                        self.topk, ds, stream)),
            attn]

    def run(self, q, k, v, qI, w, kI, stream=None):
        for _, fn in self.stages(dict(q=q, k=k, v=v, qI=qI, w=w, kI=kI), stream):
            fn()
        return self.out

    def launches(self) -> int:
        """Kernels one run() enqueues: indexer + top-K (per row block), or for
        the two-stage selection pool, block counts, coarse indexer, coarse
        top-k, the fine scores' invert count / scan / scatter and block
        kernel, and the fine top-K over the kept block ids (9); then the
        attention."""
        attn = 2 if self.attn_ws is not None else 1   # (selection bitmap +) attention
        return (2 * self.row_blocks if self.block is None else 9) + attn


class DecodePlan:
    """Buffers for B sequences, one query each, over a contiguous ([B, S_max, *])
    or paged (pools [P, 64, *] + page_table [B, max_pages]) cache.
    Inputs: dict with q [B,Hq,d], k/v/kI caches, qI [B,H_I,D_I], w [B,H_I],
    lengths [B] int32 and, when paged, page_table.
    index_fp8: the qI and kI cache hold e4m3 bytes (uint8); FP8 indexer."""

    def __init__(self, B, Hq, d, H_I, D_I, K, W, S_max, paged=False, max_pages=0, pool_pages=0,
                 index_fp8=False, fused=None, device="cuda"):
        self.B, self.Hq, self.d, self.H_I, self.D_I, self.K, self.W = B, Hq, d, H_I, D_I, K, W
        self.index = sa_indexer_scores_fp8 if index_fp8 else sa_indexer_scores
        self.paged, self.max_pages, self.pool_pages = paged, max_pages, pool_pages
        self.S = max_pages * 64 if paged else S_max
        self.S_max = S_max
        # fused=True: indexer and top-K in one kernel (the scores never leave
        # shared memory).  It takes bf16 operands, H_I <= 8, D_I in (64, 128)
        # and rows of at most 262144 keys.  It is not the default: on the
        # decode workloads the two kernels apart are faster (the fused kernel
        # holds one CTA per SM for the whole select, so its key reads run at
        # about half the separate indexer's rate).
        fusable = not index_fp8 and H_I <= 8 and D_I in (64, 128) and self.S <= 262144
        self.fused = False if fused is None else bool(fused)
        if self.fused and not fusable:
            raise ValueError("the fused indexer + top-K takes bf16 operands, H_I <= 8, D_I in (64, 128) and "
                             "rows of at most 262144 keys")
        self.scale = 1.0 / math.sqrt(d)
        dev = torch.device(device)
        self.ld = _ld(self.S)
        self.scores = None if self.fused else torch.empty((B, self.ld), dtype=torch.float32, device=dev)
        self.topk = torch.empty((B, K), dtype=torch.int32, device=dev)
        self.out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        self.ws_bytes = sa_decode_workspace_bytes(B, Hq, d, K, W)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=dev)

    def stages(self, x, stream=None):
        ds, pt = self.dev_status, x.get("page_table")
        if self.fused:
            select = [("indexer_topk", lambda: sa_indexer_topk_decode(
                x["qI"], x["w"], x["kI"], pt, self.max_pages, self.pool_pages, 64, self.B, self.S, self.H_I,
                self.D_I, x["lengths"], self.K, self.topk, ds, stream))]
        else:
            select = [
                ("indexer", lambda: self.index(x["qI"], x["w"], x["kI"], pt, self.max_pages, self.pool_pages,
                                               64, self.B, 1, self.S, self.H_I, self.D_I, x["lengths"],
                                               self.scores, self.ld, ds, stream)),
                ("topk", lambda: sa_topk_select(self.scores, self.ld, self.B, self.S, x["lengths"], None, 0,
                                                self.K, self.topk, ds, stream))]
        return select + [
            ("attention", lambda: sa_sparse_attn_decode(
                x["q"], x["k"], x["v"], pt, self.max_pages, self.pool_pages, 64, self.S_max, x["lengths"],
                self.topk, self.K, self.W, self.B, self.Hq, self.d, self.scale, self.out, self.lse,
                self.workspace, self.ws_bytes, ds, stream)),
        ]

    def run(self, q, k_cache, v_cache, qI, w, kI, seq_lens, page_table=None, stream=None):
        x = dict(q=q, k=k_cache, v=v_cache, qI=qI, w=w, kI=kI, lengths=seq_lens, page_table=page_table)
        for _, fn in self.stages(x, stream):
            fn()
        return self.out

    def launches(self) -> int:
        """Kernels one run() enqueues: the fused indexer + top-K (or, unfused,
        the indexer and the top-K), then the attention of
        sa_sparse_attn_decode.  That is one kernel when a thread-block cluster
        of G = min(16, max(1, ceil((K+W)/128), ceil(Hq/8))) CTAs per sequence
        leaves each CTA at most 1024 keys (partials merged in distributed
        shared memory), else a split-K kernel and a merge kernel."""
        kw = self.K + self.W
        G = min(16, max(1, -(-kw // 128), -(-self.Hq // 8)))
        return (1 if self.fused else 2) + (1 if -(-kw // G) <= 1024 else 2)


class HostPipeline:
    """Steps whose inputs come from pinned host memory and whose output goes
    back to pinned host memory, with the copies running under the kernels.

    Two plans (two sets of device buffers) alternate.  Step i uploads its
    inputs into set i % 2 on an upload stream, runs the path on the compute
    stream and downloads the plan's output on a download stream.  Its upload
    waits only for step i - 2's compute (the set's previous reader), and its
    compute waits for its own upload and for step i - 2's download (the set's
    previous output).  So step i + 1's upload and step i - 1's download overlap
    step i's kernels, and each step still moves all of its own bytes.

    make_plan: () -> a PrefillPlan / DecodePlan (anything with .stages and .out)
    host_inputs: name -> pinned host tensor, the shapes and dtypes of one step's inputs
    resident: name -> device tensor that every step reads in place (e.g. a KV cache)
    """

    def __init__(self, make_plan, host_inputs, resident=None, device="cuda"):
        dev = torch.device(device)
        self.plans = [make_plan(), make_plan()]
        self.inputs = []
        for _ in range(2):
            x = {k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in host_inputs.items()}
            x.update(resident or {})
            self.inputs.append(x)
        self.up, self.comp, self.down = (torch.cuda.Stream(device=dev) for _ in range(3))
        self.stages = [p.stages(x, self.comp) for p, x in zip(self.plans, self.inputs)]
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]
        self.up_done, self.comp_done, self.down_done = ev(), ev(), ev()
        self.used = [False, False]

    def run(self, step_inputs, step_outputs, before_compute=None):
        """step_inputs[i]: name -> pinned host tensor; step_outputs[i]: pinned host
        tensor shaped like plan.out.  before_compute(i), if given, runs on the
        compute stream ahead of step i's kernels.  Returns without waiting;
        synchronize (or wait on self.down) before reading the outputs."""
        for i, (hin, hout) in enumerate(zip(step_inputs, step_outputs)):
            b = i % 2
            with torch.cuda.stream(self.up):
                if self.used[b]:
                    self.up.wait_event(self.comp_done[b])
                for k, t in hin.items():
                    self.inputs[b][k].copy_(t, non_blocking=True)
                self.up_done[b].record(self.up)
            with torch.cuda.stream(self.comp):
                self.comp.wait_event(self.up_done[b])
                if self.used[b]:
                    self.comp.wait_event(self.down_done[b])
                if before_compute is not None:
                    before_compute(i)
                for _, fn in self.stages[b]:
                    fn()
                self.comp_done[b].record(self.comp)
            with torch.cuda.stream(self.down):
                self.down.wait_event(self.comp_done[b])
                hout.copy_(self.plans[b].out, non_blocking=True)
                self.down_done[b].record(self.down)
            self.used[b] = True

    def dev_status(self) -> int:
        """OR of both plans' device status words (synchronizes)."""
        return int(self.plans[0].dev_status.item()) | int(self.plans[1].dev_status.item())
