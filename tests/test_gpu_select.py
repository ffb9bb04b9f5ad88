"""GPU: the exact top-k of the lightning indexer on decode rows ("Техотчёт DeepSeek-V4
(2026)", section "Гибридное внимание: CSA и HCA", CSA step 2), the cases the workload
tests do not reach: rows of different eligible counts, just above and at k; every key
identical (all scores tie: the lowest indices win); scores packed into one narrow range
(more candidates than the selection stages on chip); the exact scores returned with the
selection; rows around the sizes whose scores take several bulk copies; rows longer than one
CTA stages (34 816 entries), which a cluster selects over chunks of the row: ragged eligible
counts across the chunks, a row at or below k beside longer ones, all scores tied (the
counted search of the k-th key and the fp32 order), the exact scores.  Expected values come
from the oracle only.
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


def _run(qI, qs, w, kI, ks, n_entries, q_pos, k, fmt, score_out=False):
    """lightning_index on host arrays; returns (idx [B, k], scores or None, device error word)."""
    B, n_max = kI.shape[0], kI.shape[1]
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    idx = torch.empty(B, 1, k, dtype=torch.int32, device="cuda")
    so = torch.empty(B, 1, k, dtype=torch.float32, device="cuda") if score_out else None
    ws = torch.empty(csa.lightning_index_workspace_size(B, 1, n_max, k), dtype=torch.uint8, device="cuda")
    ifmt = csa.CSA_IFMT_E4M3 if fmt == "e4m3" else csa.CSA_IFMT_MXFP4
    csa.lightning_index(dev(qI), dev(qs), dev(w), dev(kI), dev(ks), dev(n_entries.astype(np.int32)),
                        dev(q_pos.astype(np.int32)), k, ifmt, idx, ws, score_out=so)
    torch.cuda.synchronize()
    err = csa.read_device_error()
    return idx[:, 0].cpu().numpy(), (so[:, 0].cpu().numpy() if so is not None else None), err


def _oracle(qI, qs, w, kI, ks, b, n, fmt):
    return O.indexer_scores(qI[b], w[b], kI[b], fmt, qs[b], ks[b])[0][:n]


def _keys(fmt, x):
    return CI.quant_e4m3_rows(x) if fmt == "e4m3" else CI.quant_mxfp4_rows(x)


def _check_exact(g, I, n, k):
    """The selection must be the oracle's exactly: ascending, ties to the lower index."""
    exp = O.topk(I, n, k)
    assert np.array_equal(g, exp), (np.setdiff1d(g, exp)[:8], np.setdiff1d(exp, g)[:8])


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
def test_decode_rows_of_different_eligible_counts(fmt):
    g = torch.Generator().manual_seed(41)
    B, N, k = 5, 6000, 512
    qI, qs = _keys(fmt, torch.randn(B, 1, 64, 128, generator=g))
    kI, ks = _keys(fmt, torch.randn(B, N, 128, generator=g))
    w = torch.rand(B, 1, 64, generator=g).numpy()
    n_entries = np.array([6000, 513, 512, 3001, 40])
    q_pos = 4 * n_entries - 1                        # the current token completes entry n - 1
    idx, _, err = _run(qI, qs, w, kI, ks, n_entries, q_pos, k, fmt)
    assert err == 0
    for b in range(B):
        _check_exact(idx[b], _oracle(qI, qs, w, kI, ks, b, n_entries[b], fmt), n_entries[b], k)


def test_all_scores_tie_and_lowest_indices_win():
    """Every key identical: every score is the same, so the k lowest indices are the
    selection (the candidate band outgrows its buffer here, which is flagged)."""
    g = torch.Generator().manual_seed(42)
    B, N, k = 2, 9000, 512
    qI, qs = _keys("e4m3", torch.randn(B, 1, 64, 128, generator=g))
    kI, ks = _keys("e4m3", torch.randn(1, 1, 128, generator=g).expand(B, N, 128).contiguous())
    w = torch.rand(B, 1, 64, generator=g).numpy()
    n_entries = np.array([N, N])
    idx, _, err = _run(qI, qs, w, kI, ks, n_entries, 4 * n_entries - 1, k, "e4m3")
    assert err & ~0x8 == 0                            # only CSA_DEVERR_BAND may be set
    assert np.array_equal(idx, np.tile(np.arange(k), (B, 1)))


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
def test_narrow_score_range_many_candidates(fmt):
    """Keys = one shared direction plus a little noise: the scores of 40 000 entries fall
    into one or two histogram bins, so the candidates outnumber the on-chip buffer and the
    selection works from the list in L2."""
    g = torch.Generator().manual_seed(43)
    B, N, k = 2, 40000, 1024
    qI, qs = _keys(fmt, torch.randn(B, 1, 64, 128, generator=g))
    base = torch.randn(B, 1, 128, generator=g)
    kI, ks = _keys(fmt, base + 0.1 * torch.randn(B, N, 128, generator=g))   # ~5000-27000 in bin T, band ~200
    w = torch.rand(B, 1, 64, generator=g).numpy()
    n_entries = np.array([N, N - 17])
    idx, _, err = _run(qI, qs, w, kI, ks, n_entries, 4 * n_entries - 1, k, fmt)
    assert err == 0
    for b in range(B):
        I = _oracle(qI, qs, w, kI, ks, b, n_entries[b], fmt)
        _check_exact(idx[b], I, n_entries[b], k)


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
def test_score_out_is_the_exact_score_of_each_selected_entry(fmt):
    g = torch.Generator().manual_seed(44)
    B, N, k = 3, 5000, 256
    qI, qs = _keys(fmt, torch.randn(B, 1, 64, 128, generator=g))
    kI, ks = _keys(fmt, torch.randn(B, N, 128, generator=g))
    w = torch.rand(B, 1, 64, generator=g).numpy()
    n_entries = np.array([N, 200, 2500])
    idx, so, err = _run(qI, qs, w, kI, ks, n_entries, 4 * n_entries - 1, k, fmt, score_out=True)
    assert err == 0
    for b in range(B):
        I = _oracle(qI, qs, w, kI, ks, b, n_entries[b], fmt)
        _check_exact(idx[b], I, n_entries[b], k)
        sel = idx[b][idx[b] >= 0]
        assert np.array_equal(so[b][:sel.size], I[sel].astype(np.float32))
        assert np.all(so[b][sel.size:] == 0)


@pytest.mark.parametrize("N", [24576, 24577])
def test_rows_at_and_above_the_staged_size(N):
    g = torch.Generator().manual_seed(45)
    B, k = 2, 1024
    qI, qs = _keys("e4m3", torch.randn(B, 1, 64, 128, generator=g))
    kI, ks = _keys("e4m3", torch.randn(B, N, 128, generator=g))
    w = torch.rand(B, 1, 64, generator=g).numpy()
    n_entries = np.array([N, N - 1000])
    idx, _, err = _run(qI, qs, w, kI, ks, n_entries, 4 * n_entries - 1, k, "e4m3")
    assert err == 0
    for b in range(B):
        _check_exact(idx[b], _oracle(qI, qs, w, kI, ks, b, n_entries[b], "e4m3"), n_entries[b], k)


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
def test_rows_longer_than_one_cta_stages(fmt):
    """Rows of 70 000 entries: chunks of one cluster; eligible counts that end inside a chunk,
    on a chunk boundary region and far below the row's length, one at most k."""
    g = torch.Generator().manual_seed(47)
    B, N, k = 4, 70000, 1024
    qI, qs = _keys(fmt, torch.randn(B, 1, 64, 128, generator=g))
    kI, ks = _keys(fmt, torch.randn(B, N, 128, generator=g))
    w = torch.rand(B, 1, 64, generator=g).numpy()
    n_entries = np.array([N, 40001, 1000, 34817])
    idx, so, err = _run(qI, qs, w, kI, ks, n_entries, 4 * n_entries - 1, k, fmt, score_out=True)
    assert err == 0
    for b in range(B):
        I = _oracle(qI, qs, w, kI, ks, b, n_entries[b], fmt)
        _check_exact(idx[b], I, n_entries[b], k)
        sel = idx[b][idx[b] >= 0]
        assert np.array_equal(so[b][:sel.size], I[sel].astype(np.float32))
        assert np.all(so[b][sel.size:] == 0)


def test_long_rows_all_scores_tie():
    """Every key identical on rows a cluster selects in chunks: the k-th key comes from the
    counted search, the band outgrows its buffer (flagged), and the k lowest indices win
    across the chunks."""
    g = torch.Generator().manual_seed(48)
    B, N, k = 2, 50000, 512
    qI, qs = _keys("e4m3", torch.randn(B, 1, 64, 128, generator=g))
    kI, ks = _keys("e4m3", torch.randn(1, 1, 128, generator=g).expand(B, N, 128).contiguous())
    w = torch.rand(B, 1, 64, generator=g).numpy()
    n_entries = np.array([N, N - 3])
    idx, _, err = _run(qI, qs, w, kI, ks, n_entries, 4 * n_entries - 1, k, "e4m3")
    assert err & ~0x8 == 0                            # only CSA_DEVERR_BAND may be set
    assert np.array_equal(idx, np.tile(np.arange(k), (B, 1)))


def test_rows_beyond_the_chunked_cluster_size():
    """600 000 entries, more than 16 chunks of 34 816 scores, so the histogram-seeded
    selection (several CTAs per row, the last one finishes) takes the row.  Every key is a
    power of two a_s (1, 2, 4 or 8) times one fixed key v with e2m1 values, so each MXFP4 key
    decodes exactly to a_s v and every score is exactly a_s times the score of v (positive
    head weights): the top-k is every entry of the highest level, then the lowest indices
    of the next, with no oracle pass over 600 000 entries (ties flag CSA_DEVERR_BAND)."""
    g = torch.Generator().manual_seed(49)
    B, N, k = 1, 600000, 1024
    n = N - 5
    qI, qs = _keys("mxfp4", torch.randn(B, 1, 64, 128, generator=g))
    e2m1 = torch.tensor([0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    v = e2m1[torch.randint(0, 7, (128,), generator=g)] * torch.where(torch.rand(128, generator=g) < 0.5, -1.0, 1.0)
    level = torch.full((N,), 2.0)
    level[torch.rand(N, generator=g) < 0.3] = 4.0
    level[torch.rand(N, generator=g) < 0.2] = 1.0
    top = torch.randperm(n, generator=g)[:700]
    level[top] = 8.0
    kI, ks = _keys("mxfp4", (level[:, None] * v[None, :])[None])
    w = torch.rand(B, 1, 64, generator=g).numpy()
    # the construction, checked on the oracle: the four levels score exactly 1, 2, 4, 8 times v's
    kl, kls = _keys("mxfp4", (torch.tensor([1.0, 2.0, 4.0, 8.0])[:, None] * v[None, :])[None])
    I_l = O.indexer_scores(qI[0], w[0], kl[0], "mxfp4", qs[0], kls[0])[0]
    assert I_l[0] > 0 and np.array_equal(I_l / I_l[0], [1.0, 2.0, 4.0, 8.0])
    lv = level[:n].numpy()
    order = np.lexsort((np.arange(n), -lv))
    exp = np.sort(order[:k])
    idx, _, err = _run(qI, qs, w, kI, ks, np.array([n]), 4 * np.array([n]) - 1, k, "mxfp4")
    assert err & ~0x8 == 0                            # only CSA_DEVERR_BAND may be set
    assert np.array_equal(idx[0], exp)


def _run_rows(qI, qs, w, kI, ks, n_entries, q_pos, k, fmt, m=4, exact_ws=False):
    """lightning_index on prefill rows (Tq > 3): idx [B, Tq, k] and the device error word;
    exact_ws: a workspace of exactly lightning_index_workspace_size_exact bytes."""
    B, Tq = qI.shape[0], qI.shape[1]
    n_max = kI.shape[1]
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    idx = torch.empty(B, Tq, k, dtype=torch.int32, device="cuda")
    ifmt = csa.CSA_IFMT_E4M3 if fmt == "e4m3" else csa.CSA_IFMT_MXFP4
    size = (csa.lightning_index_workspace_size_exact(B, Tq, n_max, k, ifmt, qI.shape[2], qI.shape[3]) if exact_ws
            else csa.lightning_index_workspace_size(B, Tq, n_max, k))
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    csa.lightning_index(dev(qI), dev(qs), dev(w), dev(kI), dev(ks), dev(n_entries.astype(np.int32)),
                        dev(q_pos.astype(np.int32)), k, ifmt, idx, ws, m=m)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), csa.read_device_error()


@pytest.mark.parametrize("k,exact_ws", [(1024, False), (300, False), (1024, True)])
def test_prefill_rows_streaming_selection(k, exact_ws):
    """640 query rows of one sequence (160 groups of four: the scoring kernel keeps candidate
    lists instead of writing scores), rows whose eligible count is below and above k; the
    selection of sampled rows equals the oracle's exact top-k."""
    g = torch.Generator().manual_seed(46)
    N, Tq = 8192, 640
    qI, qs = _keys("e4m3", torch.randn(1, Tq, 64, 128, generator=g))
    kI, ks = _keys("e4m3", torch.randn(1, N, 128, generator=g))
    w = torch.rand(1, Tq, 64, generator=g).numpy()
    n_entries = np.array([N])
    q_pos = np.concatenate([np.arange(0, 4 * 2000, 4 * 2000 // 40)[:40],          # eligible 0 .. ~1950
                            4 * N - Tq + 40 + np.arange(Tq - 40)])                 # eligible ~8000 .. N
    q_pos = q_pos[None, :]
    if exact_ws:      # the streamed rows' workspace holds no score matrix
        assert (csa.lightning_index_workspace_size(1, Tq, N, k) -
                csa.lightning_index_workspace_size_exact(1, Tq, N, k, csa.CSA_IFMT_E4M3, 64, 128)) >= Tq * N * 4
    idx, err = _run_rows(qI, qs, w, kI, ks, n_entries, q_pos, k, "e4m3", exact_ws=exact_ws)
    assert err == 0
    rows = list(range(0, 40, 3)) + list(range(40, Tq, 37)) + [Tq - 1]
    I = O.indexer_scores(qI[0][rows], w[0][rows], kI[0], "e4m3", qs[0][rows], ks[0])
    for i, t in enumerate(rows):
        n = O.n_eligible(int(q_pos[0, t]), 4, N)
        _check_exact(idx[0, t], I[i][:n], n, k)
