"""Pins of the oracle's workload passes (run_csa_prefill, run_csa_decode, run_hca_decode).

The step functions (compression, indexer, top-k, attention) are pinned in
test_oracle_pins.py.  The passes add logic of their own: the window slice of the raw
rows, the eligible-entry count of each query position, the substitution of a freshly
compressed entry into the selected rows, and the write of the fresh HCA entry before
the dense pass.  These tests fix that logic against facts that do not come from the
passes themselves:

* prefill / decode consistency: decoding token p after a prefill of the tokens before
  its block gives row p of one prefill over all tokens ("Техотчёт DeepSeek-V4 (2026)",
  "Отказоустойчивая генерация": regenerating from the stored prefix reproduces the
  same state), and a prefill chunk after a context gives the rows of the whole prefill;
* hand-sized cases whose window rows and eligible / selected entries are listed by
  hand in the test ("Гибридное внимание: CSA и HCA": entry s pools tokens 4s-4..4s+3,
  so it is complete once token 4s+3 is seen; the window is the last W raw tokens);
* fresh-entry cases: the row a decode step compresses, not the stale cache row, is
  attended when it is selected (CSA) and always (HCA).
All arithmetic here is fp64, and the caches handed from one pass to the next are kept in fp64.
"""
from __future__ import annotations

import numpy as np
import pytest

import csa_inputs as CI
from oracle import csa_oracle as O

M = 4


def _tokens(T, d, H, HI, dI, seed):
    """Per-token inputs of one sequence: compressor series, queries, raw latents."""
    r = np.random.default_rng(seed)
    f = lambda *s, std=1.0: (r.standard_normal(s) * std).astype(np.float32)
    return dict(Ca=f(T, d), Cb=f(T, d), Za=f(T, d, std=1.5), Zb=f(T, d, std=1.5), q=f(T, H, d), qI=f(T, HI, dI),
                w=r.uniform(size=(T, HI)).astype(np.float32), raw=f(T, d),
                Ba=f(M, d, std=0.1), Bb=f(M, d, std=0.1), sink=f(H), kI=f(T // M, dI))


def _dims(**kw):
    d = kw["d"]
    base = dict(B=1, dk=d, dv=d, m=M, sm_scale=1.0 / np.sqrt(d), dtype="f32", ifmt="f32")
    base.update(kw)
    base.setdefault("n_max", base["N"])
    return base


def _prefill_wl(x, t0, t1, ctx_cache, W, k, H, HI, dI):
    """Prefill of tokens t0..t1-1 of the sequence x (t0 a multiple of M); entries before
    t0/M come from ctx_cache; the raw rows passed start at max(0, t0 - (W - 1))."""
    d = x["Ca"].shape[1]
    T, Tq, N, e0 = t1, t1 - t0, t1 // M, t0 // M
    raw_pos0 = max(0, t0 - (W - 1))
    cache = np.full((1, N, d), 1e3)                        # rows the compressor must overwrite
    if e0:
        cache[0, :e0] = ctx_cache[:e0]
    pb = slice(t0 - M, t0) if t0 else slice(0, M)
    t = dict(Ca=x["Ca"][None, t0:t1], Cb=x["Cb"][None, t0:t1], Za=x["Za"][None, t0:t1], Zb=x["Zb"][None, t0:t1],
             prev_Cb=x["Cb"][None, pb], prev_Zb=x["Zb"][None, pb], Ba=x["Ba"], Bb=x["Bb"], cache=cache,
             q=x["q"][None, t0:t1], qI=x["qI"][None, t0:t1], w=x["w"][None, t0:t1], kI=x["kI"][None, :N],
             raw=x["raw"][None, raw_pos0:t1], sink=x["sink"])
    dims = _dims(T=T, Tq=Tq, N=N, d=d, H=H, HI=HI, dI=dI, k=k, W=W, q_pos0=t0, raw_pos0=raw_pos0, entry0=e0)
    return CI.Workload("hand_prefill", "csa_prefill", dims, t)


def _decode_wl(x, p, cache_rows, W, k, H, HI, dI, stale=1e3):
    """Decode of token p (p + 1 a multiple of M: the token completes block (p+1)/M - 1);
    entries before that block come from cache_rows, the block's own row holds `stale`."""
    d = x["Ca"].shape[1]
    T = p + 1
    N = T // M
    e0 = N - 1
    b0 = M * e0
    cache = np.full((1, N, d), stale)                      # fp64: the stored entries stay exact
    cache[0, :e0] = cache_rows[:e0]
    lo = max(0, p - W + 1)
    # entry 0 has no b-half: its prev rows exist only as placeholders the pass must ignore
    prev_C = x["Cb"][None, b0 - M:b0] if b0 else np.full((1, M, d), 1e3, np.float32)
    prev_Z = x["Zb"][None, b0 - M:b0] if b0 else np.full((1, M, d), 1e3, np.float32)
    t = dict(Ca=x["Ca"][None, b0:T], Cb=x["Cb"][None, b0:T], Za=x["Za"][None, b0:T], Zb=x["Zb"][None, b0:T],
             prev_Cb=prev_C, prev_Zb=prev_Z, Ba=x["Ba"], Bb=x["Bb"], cache=cache,
             q=x["q"][None, p:p + 1], qI=x["qI"][None, p:p + 1], w=x["w"][None, p:p + 1],
             qI_scale=np.ones((1, 1, HI), np.float32), kI=x["kI"][None, :N], kI_scale=np.ones((1, N), np.float32),
             win=x["raw"][None, lo:T], sink=x["sink"])
    dims = _dims(T=T, Tq=1, N=N, d=d, H=H, HI=HI, dI=dI, k=k, W=W, q_pos0=p, entry0=e0)
    return CI.Workload("hand_decode", "csa_decode", dims, t)


SIZES = dict(H=2, HI=2, dI=4)


def test_decode_after_prefill_equals_one_prefill():
    """T = 48, W = 8, k = 3: decode token 47 after a prefill of tokens 0..43 equals row 47
    of one prefill of all 48 tokens (selected set, output and lse)."""
    x = _tokens(48, 8, seed=7, **SIZES)
    full = O.run_csa_prefill(_prefill_wl(x, 0, 48, None, 8, 3, **SIZES))
    pre = O.run_csa_prefill(_prefill_wl(x, 0, 44, None, 8, 3, **SIZES))
    dec = O.run_csa_decode(_decode_wl(x, 47, pre["cache"], 8, 3, **SIZES))
    assert np.array_equal(dec["idx"][0], full["idx"][47])
    np.testing.assert_allclose(dec["entry"][0][0], full["cache"][11], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dec["out"][0], full["out"][47], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dec["lse"][0], full["lse"][47], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(dec["scores"][0][:12], full["scores"][47][:12])


@pytest.mark.parametrize("p", [3, 7, 23, 35, 47])
def test_every_block_end_decode_equals_prefill_row(p):
    """The same at every block end, including the first block (entry 0 has no b-half and
    the window is clipped at token 0) and windows shorter than W."""
    W, k = 8, 3
    x = _tokens(48, 8, seed=11, **SIZES)
    full = O.run_csa_prefill(_prefill_wl(x, 0, 48, None, W, k, **SIZES))
    ctx = np.zeros((12, 8))
    if p + 1 > M:
        ctx = O.run_csa_prefill(_prefill_wl(x, 0, p + 1 - M, None, W, k, **SIZES))["cache"]
    dec = O.run_csa_decode(_decode_wl(x, p, ctx, W, k, **SIZES))
    assert np.array_equal(dec["idx"][0], full["idx"][p])
    np.testing.assert_allclose(dec["out"][0], full["out"][p], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dec["lse"][0], full["lse"][p], rtol=0, atol=1e-12)


def test_prefill_chunk_after_context_equals_whole_prefill_rows():
    """A 16-token chunk after a 32-token context (raw rows from token 25 on, entries 0..7
    from the context) gives rows 32..47 of the whole prefill, and the same entries 8..11."""
    W, k = 8, 3
    x = _tokens(48, 8, seed=3, **SIZES)
    full = O.run_csa_prefill(_prefill_wl(x, 0, 48, None, W, k, **SIZES))
    ctx = O.run_csa_prefill(_prefill_wl(x, 0, 32, None, W, k, **SIZES))["cache"]
    chunk = O.run_csa_prefill(_prefill_wl(x, 32, 48, ctx, W, k, **SIZES))
    np.testing.assert_allclose(chunk["cache"], full["cache"], rtol=0, atol=1e-12)
    for tq in range(16):
        assert np.array_equal(chunk["idx"][tq], full["idx"][32 + tq])
        np.testing.assert_allclose(chunk["out"][tq], full["out"][32 + tq], rtol=0, atol=1e-12)
        np.testing.assert_allclose(chunk["lse"][tq], full["lse"][32 + tq], rtol=0, atol=1e-12)


# -------------------------------------------------------------- hand-sized, rows listed

def _hand_prefill(W=3, k=2):
    """T = 12 tokens, N = 3 entries.  Indexer keys and queries are set by hand so that
    every query scores the entries 1, 3, 2 (I = sum_j w_j * ReLU(q_j . k_s) with one
    head of weight 1 and keys e_0 * (1, 3, 2))."""
    x = _tokens(12, 8, seed=5, **SIZES)
    x["kI"] = np.zeros((3, 4), np.float32)
    x["kI"][:, 0] = [1.0, 3.0, 2.0]
    x["qI"] = np.zeros((12, 2, 4), np.float32)
    x["qI"][:, 0, 0] = 1.0
    x["w"] = np.tile(np.array([1.0, 0.5], np.float32), (12, 1))
    return x, O.run_csa_prefill(_prefill_wl(x, 0, 12, None, W, k, **SIZES))


# query position -> (eligible entries, selected entries, window positions), by hand:
# entry s is complete at token 4s+3; k = 2 keeps the two best of (1, 3, 2); W = 3
HAND_ROWS = {
    0: ([], [], [0]),
    2: ([], [], [0, 1, 2]),
    3: ([0], [0], [1, 2, 3]),
    6: ([0], [0], [4, 5, 6]),
    7: ([0, 1], [0, 1], [5, 6, 7]),
    10: ([0, 1], [0, 1], [8, 9, 10]),
    11: ([0, 1, 2], [1, 2], [9, 10, 11]),
}


@pytest.mark.parametrize("p", sorted(HAND_ROWS))
def test_hand_sized_prefill_rows(p):
    x, res = _hand_prefill()
    elig, sel, win = HAND_ROWS[p]
    assert O.n_eligible(p, M, 3) == len(elig)
    assert res["idx"][p].tolist() == sel + [-1] * (2 - len(sel))
    entries = O.csa_compress(*(x[n].astype(np.float64) for n in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb")))
    rows = np.concatenate([entries[sel], x["raw"][win].astype(np.float64)], axis=0)
    o, lse = O.attention(x["q"][p], rows, x["sink"], 1.0 / np.sqrt(8), 8)
    np.testing.assert_allclose(res["out"][p], o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(res["lse"][p], lse, rtol=0, atol=1e-13)


def test_hand_sized_decode_rows():
    """Decode of token 11 with W = 3, k = 2: selected entries {1, 2} (2 is the fresh one),
    window rows 9, 10, 11."""
    x, _ = _hand_prefill()
    ent = O.csa_compress(*(x[n].astype(np.float64) for n in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb")))
    dec = O.run_csa_decode(_decode_wl(x, 11, ent, 3, 2, **SIZES))
    assert dec["idx"][0].tolist() == [1, 2]
    rows = np.concatenate([ent[[1, 2]], x["raw"][[9, 10, 11]].astype(np.float64)], axis=0)
    o, lse = O.attention(x["q"][11], rows, x["sink"], 1.0 / np.sqrt(8), 8)
    np.testing.assert_allclose(dec["out"][0], o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dec["lse"][0], lse, rtol=0, atol=1e-13)


# -------------------------------------------------------------- fresh entries

def test_csa_decode_attends_the_fresh_entry_not_the_stale_row():
    """Entry N-1 (the block the current token completes) scores highest; the cache holds
    a stale row there.  The output uses the freshly compressed row (uniform gates: the
    mean of the 8 source tokens), and differs from attending to the stale row."""
    W, k = 4, 2
    x = _tokens(16, 8, seed=9, **SIZES)
    for n in ("Za", "Zb", "Ba", "Bb"):
        x[n][:] = 0.0
    x["kI"] = np.zeros((4, 4), np.float32)
    x["kI"][:, 0] = [1.0, 0.5, 2.0, 9.0]
    x["qI"][:] = 0.0
    x["qI"][:, 0, 0] = 1.0
    ent = O.csa_compress(*(x[n].astype(np.float64) for n in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb")))
    stale = 0.25
    dec = O.run_csa_decode(_decode_wl(x, 15, ent, W, k, stale=stale, **SIZES))
    assert dec["idx"][0].tolist() == [2, 3]
    fresh = np.concatenate([x["Cb"][8:12], x["Ca"][12:16]]).astype(np.float64).mean(axis=0)   # block mean
    np.testing.assert_allclose(dec["entry"][0][0], fresh, rtol=0, atol=1e-12)
    win = x["raw"][12:16].astype(np.float64)
    o, _ = O.attention(x["q"][15], np.concatenate([ent[[2]], fresh[None], win]), x["sink"], 1 / np.sqrt(8), 8)
    np.testing.assert_allclose(dec["out"][0], o, rtol=0, atol=1e-12)
    o_stale, _ = O.attention(x["q"][15], np.concatenate([ent[[2]], np.full((1, 8), stale), win]), x["sink"],
                             1 / np.sqrt(8), 8)
    assert np.abs(dec["out"][0] - o_stale).max() > 1e-3


def _hca_wl(N, mp, W, stale, seed, uniform=False):
    d, H = 8, 2
    r = np.random.default_rng(seed)
    f = lambda *s, std=1.0: (r.standard_normal(s) * std).astype(np.float32)
    cache = f(1, N, d)
    cache[0, N - 1] = stale
    t = dict(cache=cache, C=f(1, mp, d), Z=f(1, mp, d, std=2.0), bias=f(mp, d, std=0.1), q=f(1, 1, H, d),
             win=f(1, W, d), sink=f(H))
    if uniform:
        t["Z"][:] = 0.0
        t["bias"][:] = 0.0
    dims = dict(B=1, T=N * mp, Tq=1, N=N, n_max=N, d=d, dk=d, dv=d, H=H, W=W, m_prime=mp, sm_scale=1 / np.sqrt(d),
                dtype="f32", q_pos0=N * mp - 1, entry0=N - 1)
    return CI.Workload("hand_hca", "hca_decode", dims, t)


def test_hca_decode_rows_listed_by_hand():
    """HCA decode with N = 3 entries of m' = 4 tokens and uniform gates: the rows are cache
    entries 0 and 1, the mean of the fresh chunk (not the stale row 2), and the window."""
    wl = _hca_wl(3, 4, 5, stale=7.0, seed=2, uniform=True)
    t = wl.tensors
    res = O.run_hca_decode(wl)
    fresh = t["C"][0].astype(np.float64).mean(axis=0)
    np.testing.assert_allclose(res["entry"][0][0], fresh, rtol=0, atol=1e-12)
    rows = np.concatenate([t["cache"][0, [0, 1]].astype(np.float64), fresh[None], t["win"][0].astype(np.float64)])
    o, lse = O.attention(t["q"][0, 0], rows, t["sink"], 1 / np.sqrt(8), 8)
    np.testing.assert_allclose(res["out"][0], o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(res["lse"][0], lse, rtol=0, atol=1e-13)


def test_hca_decode_equals_csa_decode_with_every_entry():
    """The dense HCA pass equals the sparse attention over the selection of every entry
    (top-k with k = N, computed by the CSA passes' own attention step) with the fresh entry
    substituted, for gated (non-uniform) compression."""
    wl = _hca_wl(6, 8, 3, stale=-3.0, seed=4)
    t = wl.tensors
    res = O.run_hca_decode(wl)
    fresh = O.hca_compress(t["C"][0].astype(np.float64), t["Z"][0].astype(np.float64), t["bias"].astype(np.float64), 8)
    cache = t["cache"][0].astype(np.float64).copy()
    cache[5] = fresh[0]
    sel = O.topk(np.arange(6, dtype=np.float64), 6, 6)
    assert sel.tolist() == list(range(6))
    o, lse = O.attention(t["q"][0, 0], np.concatenate([cache[sel], t["win"][0]]), t["sink"], 1 / np.sqrt(8), 8)
    np.testing.assert_allclose(res["out"][0], o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(res["lse"][0], lse, rtol=0, atol=1e-13)


# -------------------------------------------------------------- fresh key and window ring

def test_decode_fresh_key_and_ring_row_equal_a_prefill_row():
    """A decode token brings its block's indexer activations and its raw latent: the pass
    must produce the entry's key from the activations (the pinned index_key_compress) and
    put the raw latent at ring slot position mod W.  The same sequence as a prefill (E4M3
    indexer, the keys given as inputs, including the one the activations produce) must give
    the same selection, output and lse for that token; the window ring holds positions
    p - W + 1 .. p at slots pos mod W (in ring order, not position order)."""
    W, k, m = 8, 3, 4
    r = np.random.default_rng(31)
    x = _tokens(48, 8, seed=31, **SIZES)
    d, HI, dI = 8, 2, 32
    # an E4M3 indexer: queries and keys quantised with per-row scales
    qf = r.standard_normal((48, HI, dI))
    x["qI8"], x["qIs"] = O.quantise_index_keys(qf.reshape(48 * HI, dI), "e4m3")[:2]
    x["qI8"] = x["qI8"].reshape(48, HI, dI)
    x["qIs"] = x["qIs"].reshape(48, HI)
    kf = r.standard_normal((12, dI))
    kI8, kIs = O.quantise_index_keys(kf, "e4m3")[:2]
    act = {n: r.standard_normal((4, dI)) * (2.0 if n.startswith("Z") else 1.0) for n in ("Ca", "Cb", "Za", "Zb")}
    act.update(prev_Cb=r.standard_normal((4, dI)), prev_Zb=2 * r.standard_normal((4, dI)),
               Ba=0.1 * r.standard_normal((4, dI)), Bb=0.1 * r.standard_normal((4, dI)))
    # the key of entry 11 as the activations give it
    fresh8, fresh_s = O.index_key_compress(act["Ca"], act["Cb"], act["Za"], act["Zb"], act["Ba"], act["Bb"], "e4m3",
                                           act["prev_Cb"], act["prev_Zb"], 11, m)[:2]
    kI_full, kIs_full = kI8.copy(), kIs.copy()
    kI_full[11], kIs_full[11] = fresh8[0], fresh_s[0]
    # the prefill of all 48 tokens with the full key set
    pre = _prefill_wl(x, 0, 48, None, W, k, H=2, HI=HI, dI=dI)
    pre.dims["ifmt"] = "e4m3"
    pre.tensors.update(qI=x["qI8"][None], qI_scale=x["qIs"][None], kI=kI_full[None], kI_scale=kIs_full[None])
    full = O.run_csa_prefill(pre)
    # the decode of token 47: stale key row 11 and stale ring slot 47 mod 8 = 7
    ctx = O.run_csa_prefill(_prefill_wl(x, 0, 44, None, W, k, **SIZES))["cache"]
    dec = _decode_wl(x, 47, ctx, W, k, H=2, HI=HI, dI=dI)
    dec.dims.update(ifmt="e4m3", win_slot=47 % W)
    ring = np.full((1, W, d), 5.0)
    for pos in range(40, 47):
        ring[0, pos % W] = x["raw"][pos]
    stale_k = kI8.copy()
    stale_k[11] = 0x38                                        # 1.0 everywhere: not the produced key
    dec.tensors.update(qI=x["qI8"][None, 47:48], qI_scale=x["qIs"][None, 47:48], kI=stale_k[None],
                       kI_scale=kIs[None], win=ring, raw_new=x["raw"][None, 47],
                       **{n + "I": v[None] for n, v in act.items() if n not in ("Ba", "Bb")},
                       BaI=act["Ba"], BbI=act["Bb"])
    res = O.run_csa_decode(dec)
    assert np.array_equal(res["idx"][0], full["idx"][47])
    np.testing.assert_allclose(res["out"][0], full["out"][47], rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["lse"][0], full["lse"][47], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(res["scores"][0], full["scores"][47][:12])


def test_hca_decode_ring_row():
    """The HCA pass puts raw_new at ring slot win_slot: equal to the window with that row in place."""
    wl = _hca_wl(4, 4, 6, stale=1.5, seed=8)
    t = wl.tensors
    ref = O.run_hca_decode(wl)
    r = np.random.default_rng(9)
    new = r.standard_normal((1, 8)).astype(np.float32)
    wl2 = _hca_wl(4, 4, 6, stale=1.5, seed=8)
    wl2.tensors["win"] = t["win"].copy()
    wl2.tensors["win"][0, 3] = 99.0                           # stale
    wl2.tensors["raw_new"] = new
    wl2.dims["win_slot"] = 3
    res = O.run_hca_decode(wl2)
    wl3 = _hca_wl(4, 4, 6, stale=1.5, seed=8)
    wl3.tensors["win"] = t["win"].copy()
    wl3.tensors["win"][0, 3] = new[0]
    exp = O.run_hca_decode(wl3)
    np.testing.assert_array_equal(res["out"][0], exp["out"][0])
    assert np.abs(res["out"][0] - ref["out"][0]).max() > 0       # the row mattered
