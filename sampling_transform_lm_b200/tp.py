"""Vocabulary-parallel tensor parallelism of the scoring core.

"Consolidate sampling-transform scoring on one shared chunked core" (xorl PR
74), "What this PR does", item 2: ordinary vocabulary-parallel body TP is
handled inside the core -- chunk-local logits are gathered in rank order,
hidden gradients are summed across vocabulary ranks, weight-shard gradients
stay local. Rank k of the group holds W's vocabulary rows [k Vl, (k + 1) Vl).

Per row chunk the forward forms this rank's scaled logits [Tc, Vl], all-gathers
the ranks' blocks, interleaves them in rank order into full rows and runs the
support program on them (every rank, identically: the pages' "full re-sort on
every rank"); the backward forms the dZ of this rank's vocabulary only, keeps
its dW shard and sums the partial dH over the group.

``VocabParallel`` holds the order of the steps; the per-rank operations come
from ``ops`` (the library's kernels by default), so the orchestration can be
exercised with stand-ins on CPU ranks.
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

    def backward_shard(self, H, W_shard, target, temperature, top_k, top_p, min_p, saved, grad,
                       vocab_offset):
        return self.sts.sts_backward_shard(H, W_shard, target, temperature, top_k, top_p, min_p,
                                           saved, grad, vocab_offset=vocab_offset, check=True)


class VocabParallel:
    """Forward and backward of the scoring core with W sharded by vocabulary
    over ``group`` (all ranks hold the same rows, H and metadata)."""

    def __init__(self, group=None, ops=None, row_chunk=4096):
        if row_chunk % 128:
            raise ValueError("row_chunk must be a multiple of 128 (the projection's row tiles)")
        self.group = group
        self.ops = ops if ops is not None else LibraryOps()
        self.row_chunk = row_chunk

    def _world(self):
        return dist.get_world_size(self.group), dist.get_rank(self.group)

    def forward(self, H, W_shard, target, temperature, top_k, top_p, min_p, entropy=False):
        """Returns (logprob [T], saved per-row scalars) for the full vocabulary
        of world * Vl tokens; identical on every rank."""
        world, _ = self._world()
        T, Vl = H.shape[0], W_shard.shape[0]
        V = world * Vl
        ops = self.ops
        parts = []
        for t0 in range(0, T, self.row_chunk):
            rows = min(self.row_chunk, T - t0)
            local = ops.empty((rows, Vl), H)
            ops.shard_logits(H, W_shard, temperature, t0, rows, local)
            blocks = ops.empty((world, rows, Vl), H)
            dist.all_gather(list(blocks.unbind(0)), local, group=self.group)
            full = ops.empty((rows, V), H)
            ops.gather(blocks, full)  # rank order: columns [k Vl, (k + 1) Vl) from rank k
            sl = slice(t0, t0 + rows)
            parts.append(ops.resolve(full, V, target[sl], temperature[sl], top_k[sl], top_p[sl],
                                     min_p[sl], entropy))
        logprob = torch.cat([p[0] for p in parts])
        saved = {k: torch.cat([p[1][k] for p in parts]) for k in parts[0][1]}
        return logprob, saved

    def backward(self, H, W_shard, target, temperature, top_k, top_p, min_p, saved, grad):
        """Returns (dH [T, d] summed over the group, this rank's dW shard)."""
        _, rank = self._world()
        offset = rank * W_shard.shape[0]
        dH, dW = self.ops.backward_shard(H, W_shard, target, temperature, top_k, top_p, min_p,
                                         saved, grad, offset)
        dist.all_reduce(dH, group=self.group)
        return dH, dW
