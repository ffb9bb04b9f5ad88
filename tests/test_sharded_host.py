"""The KV-sharded decode's orchestration on CPU with two and three gloo ranks.

Each rank holds a contiguous shard of a sequence batch's compressed entries.  The steps
(local top-k with exact scores, the all-gather of the candidates, the global top-k, the
attention over the rank's selected rows with the window and the sink on rank 0 only, the
all-gather of the partial outputs and their log-sum-exp merge) run here with CPU stand-ins
for the library's kernels, written from the definitions with the oracle's functions; the
merged result must equal the unsharded oracle: the same selected entries and the same
attention output.  A case where one shard holds none of the selected entries checks that
such a rank (sink -1e30, no rows) weighs nothing.

"Техотчёт DeepSeek-V4 (2026)", section "Гибридное внимание: CSA и HCA", CSA steps 2-3.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


class OracleOps:
    """CPU stand-ins with the binding's signatures (float64 tensors)."""

    @staticmethod
    def lightning_index(qI, qI_scale, w, kI, kI_scale, n_entries, q_pos, k, ifmt, idx_out, ws, score_out=None, m=4):
        from oracle import csa_oracle as O
        for b in range(w.shape[0]):
            I = O.indexer_scores(qI[b].numpy(), w[b].numpy(), kI[b].numpy(), "f32")[0]
            ne = O.n_eligible(int(q_pos[b, 0]), m, int(n_entries[b]))
            sel = O.topk(I, ne, k)
            idx_out[b, 0] = torch.from_numpy(sel.astype(np.int32))
            score_out[b, 0] = torch.from_numpy(np.where(sel >= 0, I[np.maximum(sel, 0)], 0.0))

    @staticmethod
    def shard_topk_merge(idx_all, score_all, bounds, local_out):
        G, B, k = idx_all.shape
        for b in range(B):
            gid, sc = [], []
            for g in range(G):
                for i in range(k):
                    if idx_all[g, b, i] >= 0:
                        gid.append(int(bounds[g]) + int(idx_all[g, b, i]))
                        sc.append(float(score_all[g, b, i]))
            order = sorted(range(len(gid)), key=lambda i: (-sc[i], gid[i]))[:k]
            chosen = sorted(gid[i] for i in order)
            for g in range(G):
                mine = [x - int(bounds[g]) for x in chosen if bounds[g] <= x < bounds[g + 1]]
                local_out[g, b] = -1
                local_out[g, b, :len(mine)] = torch.tensor(mine, dtype=torch.int32)

    @staticmethod
    def sparse_attn_decode(q, cache, idx, win, win_len, sink, sm_scale, dv, out, lse=None, workspace=None):
        from oracle import csa_oracle as O
        for b in range(q.shape[0]):
            sel = idx[b][idx[b] >= 0].numpy()
            rows = cache[b].numpy()[sel]
            if win is not None:
                rows = np.concatenate([rows, win[b].numpy()[:int(win_len[b])]], axis=0)
            o, l = O.attention(q[b].numpy(), rows, sink.numpy(), sm_scale, dv)
            out[b] = torch.from_numpy(o)
            lse[b] = torch.from_numpy(l)

    @staticmethod
    def attn_merge_shards(o_all, lse_all, out):
        L = torch.logsumexp(lse_all, dim=0)
        out.copy_((torch.exp(lse_all - L)[..., None] * o_all).sum(dim=0))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed, dead_shard):
    g = torch.Generator().manual_seed(seed)
    B, N, H, d, dv, HI, dI, k, W = 2, 300, 4, 64, 48, 2, 32, 16, 8
    x = dict(qI=torch.randn(B, 1, HI, dI, generator=g, dtype=torch.float64),
             w=torch.rand(B, 1, HI, generator=g, dtype=torch.float64),
             kI=torch.randn(B, N, dI, generator=g, dtype=torch.float64),
             cache=torch.randn(B, N, d, generator=g, dtype=torch.float64),
             q=torch.randn(B, H, d, generator=g, dtype=torch.float64),
             win=torch.randn(B, W, d, generator=g, dtype=torch.float64),
             win_len=torch.tensor([W, 3], dtype=torch.int32),
             sink=torch.randn(H, generator=g, dtype=torch.float64))
    if dead_shard:
        # the queries point away from the last 200 entries' keys: their scores are all 0
        x["qI"] = x["qI"].abs()
        x["kI"][:, :100] = x["kI"][:, :100].abs() + 0.1
        x["kI"][:, 100:] = -x["kI"][:, 100:].abs() - 0.1
    return x, dict(B=B, N=N, H=H, d=d, dv=dv, k=k, W=W, sm_scale=d ** -0.5)


def _worker(rank, world, port, out_dir, seed, dead_shard):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from compressed_sparse_long_csa_b200 import sharded as S
        x, D = _problem(seed, dead_shard)
        bounds = S.shard_bounds(D["N"], world)
        lo, hi = bounds[rank], bounds[rank + 1]
        st = S.ShardState(rank, world, bounds, x["cache"][:, lo:hi].contiguous(), x["kI"][:, lo:hi].contiguous(),
                          None, D["B"], D["H"], 2, D["dv"], D["k"], D["W"], device="cpu")
        st.out, st.lse = st.out.double(), st.lse.double()

        def gather(t):
            parts = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(parts, t.contiguous())
            return torch.stack(parts)

        out = torch.empty(D["B"], D["H"], D["dv"], dtype=torch.float64)
        sel = S.kv_sharded_decode(st, x["q"], x["qI"], None, x["w"], x["win"], x["win_len"], x["sink"], D["k"], 0,
                                  D["sm_scale"], D["dv"], gather, out, ops=OracleOps)
        glob = torch.where(sel >= 0, sel + lo, sel)
        allsel = gather(glob)
        if rank == 0:
            np.save(os.path.join(out_dir, "out.npy"), out.numpy())
            np.save(os.path.join(out_dir, "sel.npy"), allsel.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world,dead_shard", [(2, False), (3, False), (2, True)])
def test_sharded_decode_equals_unsharded(tmp_path, world, dead_shard):
    from oracle import csa_oracle as O
    seed = 11 + world
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), seed, dead_shard), nprocs=world,
                       join=True, start_method="spawn")
    out = np.load(tmp_path / "out.npy")
    sel = np.load(tmp_path / "sel.npy")                     # [world, B, k] global ids, -1 pads
    x, D = _problem(seed, dead_shard)
    for b in range(D["B"]):
        I = O.indexer_scores(x["qI"][b].numpy(), x["w"][b].numpy(), x["kI"][b].numpy(), "f32")[0]
        ref = O.topk(I, D["N"], D["k"])
        got = np.sort(sel[:, b][sel[:, b] >= 0])
        assert np.array_equal(got, ref), (b, got, ref)
        rows = np.concatenate([x["cache"][b].numpy()[ref], x["win"][b].numpy()[:int(x["win_len"][b])]], axis=0)
        o, _ = O.attention(x["q"][b].numpy(), rows, x["sink"].numpy(), D["sm_scale"], D["dv"])
        np.testing.assert_allclose(out[b], o, rtol=1e-10, atol=1e-12)
    if dead_shard:
        assert not (sel[1] >= 0).any()                      # the second shard selected nothing


def test_shard_bounds_cover_the_entries_contiguously():
    from compressed_sparse_long_csa_b200 import sharded as S
    for n, G in [(16384, 2), (16384, 3), (7, 4), (262144, 8)]:
        b = S.shard_bounds(n, G)
        assert b[0] == 0 and b[-1] == n and len(b) == G + 1
        sizes = [b[g + 1] - b[g] for g in range(G)]
        assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1
