"""KV-sharded decode of one CSA layer: a sequence's compressed entries split over G ranks.

"Техотчёт DeepSeek-V4 (2026)", section "Гибридное внимание: CSA и HCA", CSA steps 2-3
(top-k selection over all compressed entries, then attention over the selected entries,
the window and the sink), run with the entries in G contiguous shards, one per GPU:

1. every rank scores its shard and keeps its local top-k with the exact scores
   (lightning_index with score_out);
2. the G x k candidates are all-gathered and shard_topk_merge picks the global top-k
   (the union of the local top-k sets holds it), giving each rank the ids in its shard;
3. every rank attends to its selected rows (rank 0 also to the window and the sink; the
   others pass a sink of -1e30 and no window, so that a rank without rows weighs nothing);
4. the G partial outputs and their log-sum-exps are all-gathered and attn_merge_shards
   combines them into the attention over the union.

The two exchanges are all-gathers of k (index, score) pairs and of one output row per head
(latency-bound over NVLink).  Every arithmetic step runs in the library's kernels; this
module only orders the calls and the exchanges.  `gather(t)` must return the G ranks'
tensors stacked on a new leading axis (torch.distributed.all_gather_into_tensor over the
ranks, or a concatenation when one process emulates the ranks).
"""
from __future__ import annotations

import torch

from . import _native as N

NO_SINK = -1.0e30


def shard_bounds(n_entries: int, G: int) -> list:
    """Contiguous shards of n_entries entries: shard g holds [bounds[g], bounds[g+1])."""
    return [(n_entries * g) // G for g in range(G + 1)]


class ShardState:
    """One rank's resident part of a sequence batch: its cache and indexer-key shards and
    the buffers of the two exchanges."""

    def __init__(self, rank, G, bounds, cache, kI, kI_scale, B, H, HI, dv, k, W, device="cuda"):
        self.rank, self.G, self.bounds = rank, G, bounds
        self.cache, self.kI, self.kI_scale = cache, kI, kI_scale     # [B, n_g, ...] contiguous
        self.n_local = bounds[rank + 1] - bounds[rank]
        i32 = dict(dtype=torch.int32, device=device)
        self.n_entries = torch.full((B,), self.n_local, **i32)
        self.bounds_dev = torch.tensor(bounds, **i32)
        self.idx = torch.empty(B, 1, k, **i32)
        self.score = torch.empty(B, 1, k, dtype=torch.float32, device=device)
        self.local_sel = torch.empty(G, B, k, **i32)
        self.iws = torch.empty(N.lightning_index_workspace_size(B, 1, max(self.n_local, 1), k), dtype=torch.uint8,
                               device=device)
        self.out = torch.empty(B, H, dv, dtype=cache.dtype, device=device)
        self.lse = torch.empty(B, H, dtype=torch.float32, device=device)
        self.aws = torch.empty(N.attn_decode_workspace_size(B, H, dv, k + W), dtype=torch.uint8, device=device)
        self.sink_off = torch.full((H,), NO_SINK, dtype=torch.float32, device=device)
        # a decode query sees every entry of the sequence: in the shard's own numbering,
        # a position at which all n_local entries are complete (m = 4)
        self.q_pos_all = torch.full((B, 1), 4 * max(self.n_local, 1) - 1, **i32)


def local_candidates(st: ShardState, qI, qI_scale, w, k, ifmt, ops=N):
    """Step 1: this rank's local top-k of its shard with exact scores (st.idx, st.score)."""
    ops.lightning_index(qI, qI_scale, w, st.kI, st.kI_scale, st.n_entries, st.q_pos_all, k, ifmt, st.idx, st.iws,
                        score_out=st.score, m=4)
    return st.idx[:, 0], st.score[:, 0]


def local_attention(st: ShardState, idx_all, score_all, q, win, win_len, sink, sm_scale, dv, ops=N):
    """Steps 2-3: the global top-k from all ranks' candidates ([G, B, k] each), then the
    attention over this rank's selected rows (st.out, st.lse)."""
    ops.shard_topk_merge(idx_all, score_all, st.bounds_dev, st.local_sel)
    first = st.rank == 0
    ops.sparse_attn_decode(q, st.cache, st.local_sel[st.rank], win if first else None,
                           win_len if first else None, sink if first else st.sink_off, sm_scale, dv, st.out,
                           lse=st.lse, workspace=st.aws)
    return st.out, st.lse


def merge_outputs(o_all, lse_all, out, ops=N):
    """Step 4: the attention over the union of the rows from the ranks' partial outputs."""
    ops.attn_merge_shards(o_all, lse_all, out)


def kv_sharded_decode(st: ShardState, q, qI, qI_scale, w, win, win_len, sink, k, ifmt, sm_scale, dv, gather, out,
                      ops=N):
    """One decode step of this rank (the query sees every entry).  q [B, H, d_k];
    qI / qI_scale / w the indexer query; win / win_len / sink as sparse_attn_decode.
    Writes the merged attention output into out [B, H, dv] and returns this rank's
    selected local ids [B, k]."""
    idx, score = local_candidates(st, qI, qI_scale, w, k, ifmt, ops)
    o, lse = local_attention(st, gather(idx), gather(score), q, win, win_len, sink, sm_scale, dv, ops)
    merge_outputs(gather(o), gather(lse), out, ops)
    return st.local_sel[st.rank]
