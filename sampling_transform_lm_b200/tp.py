"""Vocabulary-parallel tensor parallelism of the scoring core.

"Consolidate sampling-transform scoring on one shared chunked core" (xorl PR
74, "What this PR does", item 2: ordinary vocabulary-parallel body TP is
handled inside the core -- chunk-local results are combined in rank order,
hidden gradients are summed across vocabulary ranks, weight-shard gradients
stay local). Rank k of the group holds W's vocabulary rows [k Vl, (k + 1) Vl).

Two forms of the forward, per row chunk:

* ``merge`` (the default): per-row statistics cross the ranks instead of
  logits. Each rank forms its shard's scaled logits [Tc, Vl]; the row maxima
  are combined by max, the 4096-bucket count histograms by sum; every rank
  then plans each row identically (the top-k bucket, a bracket of buckets that
  certainly holds the top-p crossing, the min-p threshold), and one pass over
  its shard forms float64 sums (combined by sum), the smallest kept and
  overall keys (by min) and the composite keys of the planned buckets (by an
  all-gather); every rank sorts and scans the merged keys and places the cuts.
  About 16 KB of counts plus the planned buckets' keys move per row, against
  4 V bytes of logits for the gather. Where the certain bracket holds more
  keys than one sort, up to 2048 keys around the estimated crossing are
  gathered and the finish checks that they hold it; rows it flags are
  resolved by the gather form.
* ``gather``: the ranks' blocks are all-gathered, interleaved in rank order
  into full rows and the support program runs on them on every rank (the
  pages' form, with its full re-sort on every rank).

The backward forms the dZ of this rank's vocabulary only, keeps its dW shard
and sums the partial dH over the group.

``VocabParallel`` holds the order of the steps and the collectives; the
per-rank operations come from ``ops`` (the library's kernels by default), so
the orchestration can be exercised with stand-ins on CPU ranks.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


class LibraryOps:
    """The per-rank steps on the GPU, through the library's C ABI."""

    def __init__(self):
        import sampling_transform_lm_b200 as sts

        self.sts = sts

    def empty(self, shape, like):
        return torch.empty(shape, dtype=torch.float32, device=like.device)

    def shard_logits(self, H, W_shard, temperature, t0, rows, out):
        # s = (H . W_shard^T) / tau for rows [t0, t0 + rows), written to out [rows, Vl]
        self.sts.sts_scaled_logits(H, W_shard, temperature, t0=t0, rows=rows, out=out)

    def gather(self, blocks, out):
        self.sts.sts_gather_vocab_shards(blocks, out)

    def resolve(self, S, V, target, temperature, top_k, top_p, min_p, entropy):
        lp, saved, _ = self.sts.sts_resolve_logits(S, target, temperature, top_k, top_p, min_p,
                                                   V=V, entropy=entropy, check=True)
        return lp, saved

    # the statistics merge's per-rank stages
    def row_max(self, local):
        return self.sts.sts_tp_row_max(local)

    def count(self, local, m):
        return self.sts.sts_tp_count(local, m)

    def sort_cap(self):
        return self.sts.sts_tp_constants()["sort_cap"]

    def exact(self, local, vocab_offset, V, target, temperature, top_k, top_p, min_p, m, counts,
              cap):
        return self.sts.sts_tp_exact(local, vocab_offset, V, target, temperature, top_k, top_p,
                                     min_p, m, counts, cap=cap)

    def finish(self, V, target, temperature, top_k, top_p, min_p, m, rec, cand, ncand):
        lp, saved, need, ws = self.sts.sts_tp_finish(V, target, temperature, top_k, top_p, min_p, m,
                                                     rec["plan"], rec["sums"], rec["keys"],
                                                     rec["ylogit"], cand, ncand)
        self.sts.sts_get_status(ws, raise_on_error=True)
        return lp, saved, need

    def backward_shard(self, H, W_shard, target, temperature, top_k, top_p, min_p, saved, grad,
                       vocab_offset):
        return self.sts.sts_backward_shard(H, W_shard, target, temperature, top_k, top_p, min_p,
                                           saved, grad, vocab_offset=vocab_offset, check=True)


class VocabParallel:
    """Forward and backward of the scoring core with W sharded by vocabulary
    over ``group`` (all ranks hold the same rows, H and metadata)."""

    def __init__(self, group=None, ops=None, row_chunk=4096, mode="merge"):
        if row_chunk % 128:
            raise ValueError("row_chunk must be a multiple of 128 (the projection's row tiles)")
        if mode not in ("merge", "gather"):
            raise ValueError("mode is 'merge' or 'gather'")
        self.group = group
        self.ops = ops if ops is not None else LibraryOps()
        self.row_chunk = row_chunk
        self.mode = mode
        self.gathered_rows = 0  # rows the merge handed to the gather form (diagnostic)

    def _world(self):
        return dist.get_world_size(self.group), dist.get_rank(self.group)

    def forward(self, H, W_shard, target, temperature, top_k, top_p, min_p, entropy=False):
        """Returns (logprob [T], saved per-row scalars) for the full vocabulary
        of world * Vl tokens; identical on every rank. The entropy output
        takes the gather form."""
        world, rank = self._world()
        T, Vl = H.shape[0], W_shard.shape[0]
        V = world * Vl
        ops = self.ops
        parts = []
        for t0 in range(0, T, self.row_chunk):
            rows = min(self.row_chunk, T - t0)
            local = ops.empty((rows, Vl), H)
            ops.shard_logits(H, W_shard, temperature, t0, rows, local)
            sl = slice(t0, t0 + rows)
            meta = (target[sl], temperature[sl], top_k[sl], top_p[sl], min_p[sl])
            if self.mode == "merge" and not entropy:
                parts.append(self._merge_chunk(local, rank, world, V, meta))
            else:
                parts.append(self._gather_chunk(local, world, V, meta, entropy))
        logprob = torch.cat([p[0] for p in parts])
        saved = {k: torch.cat([p[1][k] for p in parts]) for k in parts[0][1]}
        return logprob, saved

    def _gather_chunk(self, local, world, V, meta, entropy):
        ops = self.ops
        rows, Vl = local.shape
        blocks = ops.empty((world, rows, Vl), local)
        dist.all_gather(list(blocks.unbind(0)), local, group=self.group)
        full = ops.empty((rows, V), local)
        ops.gather(blocks, full)  # rank order: columns [k Vl, (k + 1) Vl) from rank k
        return ops.resolve(full, V, *meta, entropy)

    def _merge_chunk(self, local, rank, world, V, meta):
        ops, g = self.ops, self.group
        rows, Vl = local.shape
        m = ops.row_max(local)
        dist.all_reduce(m, op=dist.ReduceOp.MAX, group=g)
        counts = ops.count(local, m)
        dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=g)
        # keys one rank may gather per row: its share of one sort with room for
        # an uneven split (a rank over it sends the row to the gather form)
        sort_cap = ops.sort_cap()
        cap = min(sort_cap, (3 * sort_cap) // (2 * world) + 256)
        rec = ops.exact(local, rank * Vl, V, *meta, m, counts, cap)
        dist.all_reduce(rec["sums"], op=dist.ReduceOp.SUM, group=g)
        dist.all_reduce(rec["keys"], op=dist.ReduceOp.MIN, group=g)
        dist.all_reduce(rec["ylogit"], op=dist.ReduceOp.SUM, group=g)
        cand = torch.empty((world,) + tuple(rec["cand"].shape), dtype=rec["cand"].dtype,
                           device=rec["cand"].device)
        dist.all_gather(list(cand.unbind(0)), rec["cand"], group=g)
        ncand = torch.empty((world, rows), dtype=rec["ncand"].dtype, device=rec["ncand"].device)
        dist.all_gather(list(ncand.unbind(0)), rec["ncand"], group=g)
        lp, saved, need = ops.finish(V, *meta, m, rec, cand, ncand)
        # the flags are computed from merged records: every rank takes the same branch
        need_rows = need.bool()
        if bool(need_rows.any()):
            self.gathered_rows += int(need_rows.sum())
            lp_g, saved_g = self._gather_chunk(local, world, V, meta, False)
            lp = torch.where(need_rows, lp_g, lp)
            saved = {k: torch.where(need_rows.view(-1, *([1] * (v.dim() - 1))), saved_g[k], v)
                     for k, v in saved.items()}
        return lp, saved

    def backward(self, H, W_shard, target, temperature, top_k, top_p, min_p, saved, grad):
        """Returns (dH [T, d] summed over the group, this rank's dW shard)."""
        _, rank = self._world()
        offset = rank * W_shard.shape[0]
        dH, dW = self.ops.backward_shard(H, W_shard, target, temperature, top_k, top_p, min_p,
                                         saved, grad, offset)
        dist.all_reduce(dH, group=self.group)
        return dH, dW
