"""The KV-sharded decode's kernels on one GPU, the G ranks emulated in turn.

Each emulated rank holds a contiguous shard of the 64K decode workload's entries (cache
rows and FP8 indexer keys); the exchanges become concatenations.  The merged selection must
be the exact top-k of all entries (ties within 1e-6 * |I_k|, as the unsharded acceptance),
and the merged output the attention over those rows, the window and the sink (bf16
tolerances), as computed by the fp64 oracle.

"Техотчёт DeepSeek-V4 (2026)", section "Гибридное внимание: CSA и HCA", CSA steps 2-3.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import csa_inputs as CI
from oracle import csa_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_sparse_long_csa_b200 as csa
    from compressed_sparse_long_csa_b200 import sharded as S
    from compressed_sparse_long_csa_b200 import steps


@pytest.mark.parametrize("G", [2, 3, 4])
def test_kv_sharded_decode_on_one_gpu(G):
    wl = CI.make_workload(1, scale={"B": 4, "T": 65536})
    D = wl.dims
    B, N, H, HI, dv, k, W = D["B"], D["N"], D["H"], D["HI"], D["dv"], D["k"], D["W"]
    T = steps.upload(wl)
    bounds = S.shard_bounds(N, G)
    states = []
    for g in range(G):
        lo, hi = bounds[g], bounds[g + 1]
        states.append(S.ShardState(g, G, bounds, T["cache"][:, lo:hi].contiguous(), T["kI"][:, lo:hi].contiguous(),
                                   T["kI_scale"][:, lo:hi].contiguous(), B, H, HI, dv, k, W))
    cands = [S.local_candidates(st, T["qI"], T["qI_scale"], T["w"], k, csa.CSA_IFMT_E4M3) for st in states]
    idx_all = torch.stack([c[0] for c in cands])
    score_all = torch.stack([c[1] for c in cands])
    parts = [S.local_attention(st, idx_all, score_all, T["q"][:, 0], T["win"], T["win_len"], T["sink"],
                               D["sm_scale"], dv) for st in states]
    out = torch.empty(B, H, dv, dtype=torch.bfloat16, device="cuda")
    S.merge_outputs(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]), out)
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    sel = torch.stack([st.local_sel[g] + (st.local_sel[g] >= 0) * bounds[g] for g, st in enumerate(states)])
    sel = sel.cpu().numpy()                                              # [G, B, k] global ids, -1 pads
    x = wl.tensors
    qn, winn, cache = O.decode_bf16(x["q"][:, 0]), O.decode_bf16(x["win"]), x["cache"]
    for b in range(B):
        I = O.indexer_scores(x["qI"][b], x["w"][b], x["kI"][b], "e4m3", x["qI_scale"][b], x["kI_scale"][b])[0]
        ref = O.topk(I, N, k)
        got = np.sort(sel[:, b][sel[:, b] >= 0])
        assert got.size == k and np.all(np.diff(got) > 0)
        if not np.array_equal(got, ref):
            Ik = np.sort(I)[::-1][k - 1]
            for e in set(got.tolist()) ^ set(ref.tolist()):
                assert abs(I[e] - Ik) <= 1e-6 * abs(Ik), (b, e)
        rows = np.concatenate([O.decode_bf16(cache[b][got]), winn[b]], axis=0)
        o, _ = O.attention(qn[b], rows, x["sink"].astype(np.float64), D["sm_scale"], dv)
        o = O.store(o, "bf16")
        g_ = out[b].float().cpu().numpy()
        err = np.abs(g_ - o)
        assert err.max() <= 2e-2 and err.sum() / np.abs(o).sum() <= 2e-3, (b, err.max(), err.sum() / np.abs(o).sum())
