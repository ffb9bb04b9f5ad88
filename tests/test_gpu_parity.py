"""GPU parity: every step of the hot path through the C ABI vs the fp64 oracle.

Acceptance (written from the workload contract):
* top-k index sets equal, except that an index in one set and not the other must
  have an oracle score within 1e-6 * |I_k| of the oracle's k-th score I_k;
* bf16 outputs: max-abs <= 2e-2 and mean-rel (sum|g-o| / sum|o|) <= 2e-3;
* fp32 (tiny workload): max-abs <= 1e-4.
Inputs come from csa_inputs only; expected values only from oracle/.
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
    from compressed_sparse_long_csa_b200 import steps


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _within(g, o, dtype, what):
    err = np.abs(g - o)
    if dtype == "f32":
        assert err.max() <= 1e-4, (what, err.max())
    else:
        assert err.max() <= 2e-2, (what, err.max())
        assert err.sum() / max(np.abs(o).sum(), 1e-30) <= 2e-3, (what, err.sum() / np.abs(o).sum())


def check_close(g, o, dtype, what):
    """Compare a stored GPU result with the oracle, twice, with the same bounds: against
    the exact fp64 value, and against that value rounded to the storage format (bf16
    round-to-nearest-even), which is the best a stored result can be, so that the second
    comparison measures the kernel's own error."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    assert np.all(np.isfinite(g)), what
    _within(g, o, dtype, what + " (exact oracle)")
    _within(g, O.store(o, dtype), dtype, what + " (oracle rounded to storage)")


def check_topk(g, o, scores, n_elig, k, what=""):
    g = np.asarray(g)
    valid = g[g >= 0]
    cnt = min(k, n_elig)
    assert valid.size == cnt, (what, valid.size, cnt)
    assert np.all(g[cnt:] == -1), what
    assert np.all(np.diff(valid) > 0), what          # ascending, no duplicates
    assert valid.size == 0 or (valid.min() >= 0 and valid.max() < n_elig), what
    ov = np.asarray(o)[np.asarray(o) >= 0]
    if np.array_equal(valid, ov):
        return
    s = np.asarray(scores[:n_elig], np.float64)
    order = np.lexsort((np.arange(n_elig), -s))
    Ik = s[order[cnt - 1]]
    for x in set(valid.tolist()) ^ set(ov.tolist()):
        assert abs(s[x] - Ik) <= 1e-6 * abs(Ik), (what, x, s[x], Ik)


def run(wl):
    T = steps.upload(wl)
    steps.run_step(wl.kind, T, wl.dims)
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    return T


# ----------------------------------------------------------------------------- CSA prefill

def _sampled_rows(Tq, n, seed):
    """The first 8 and last 8 query rows of the chunk plus seeded rows between them."""
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(8, Tq - 8), n - 16, replace=False)
    return sorted(set(range(8)) | set(range(Tq - 8, Tq)) | set(int(x) for x in mid))


PREFILL_CASES = {
    "tiny_fp32": (0, None, None),
    "prefill_small": (3, {"ctx": 4096, "Tq": 256, "k": 256}, None),
    "prefill_full_sampled": (3, None, _sampled_rows(4096, 256, 33)),
}


def _prefill_oracle(wl, rows, chunk=32):
    """run_csa_prefill over the sampled rows, a few at a time (its per-head dot products
    for all rows at once would not fit the host's memory at the full size)."""
    if rows is None:
        return O.run_csa_prefill(wl, rows)
    ref = None
    for c0 in range(0, len(rows), chunk):
        part = O.run_csa_prefill(wl, rows[c0:c0 + chunk])
        if ref is None:
            ref = part
        else:
            for key in ("idx", "out", "lse", "scores"):
                ref[key].update(part[key])
    return ref


@pytest.mark.parametrize("case", list(PREFILL_CASES))
def test_csa_prefill(case):
    i, sc, rows = PREFILL_CASES[case]
    wl = CI.make_workload(i, scale=sc)
    D = wl.dims
    T = run(wl)
    ref = _prefill_oracle(wl, rows)
    rows = list(range(D["Tq"])) if rows is None else rows
    e0 = D["entry0"]
    n_new = D["Tq"] // D["m"]
    check_close(_np(T["cache"][0, e0:e0 + n_new]), ref["cache"][e0:e0 + n_new], D["dtype"], "compress")
    idx = T["idx"][0].cpu().numpy()
    out = T["out"][0]
    lse = _np(T["lse"][0])
    for tq in rows:
        ne = O.n_eligible(D["q_pos0"] + tq, D["m"], D["N"])
        check_topk(idx[tq], ref["idx"][tq], ref["scores"][tq], ne, D["k"], f"row {tq}")
    g = np.stack([_np(out[tq]) for tq in rows])
    o = np.stack([ref["out"][tq] for tq in rows])
    check_close(g, o, D["dtype"], "attention out")
    np.testing.assert_allclose(lse[rows], np.stack([ref["lse"][tq] for tq in rows]), atol=2e-3, rtol=0)


# ----------------------------------------------------------------------------- CSA decode

DECODE_CASES = {
    "csa_decode_small": (1, {"B": 3, "T": 8192}),
    "csa_decode_full": (1, None),
    "pair_small": (4, {"B": 2, "T": 65536}),
    "pair_full": (4, None),
}


@pytest.mark.parametrize("case", list(DECODE_CASES))
def test_csa_decode(case):
    i, sc = DECODE_CASES[case]
    wl = CI.make_workload(i, scale=sc)
    D = wl.dims
    T = run(wl)
    ref = O.run_csa_decode(wl)
    for b in range(D["B"]):
        check_close(_np(T["cache"][b, D["entry0"]]), ref["entry"][b][0], D["dtype"], f"compress b{b}")
        check_topk(T["idx"][b, 0].cpu().numpy(), ref["idx"][b], ref["scores"][b], D["N"], D["k"], f"b{b}")
    g = np.stack([_np(T["out"][b, 0]) for b in range(D["B"])])
    o = np.stack([ref["out"][b] for b in range(D["B"])])
    check_close(g, o, D["dtype"], "attention out")
    np.testing.assert_allclose(_np(T["lse"][:, 0]), np.stack([ref["lse"][b] for b in range(D["B"])]),
                               atol=2e-3, rtol=0)
    if wl.kind == "hybrid_pair":
        href = O.run_hca_decode(wl, prefix="h_")
        for b in range(D["B"]):
            check_close(_np(T["h_cache"][b, D["entry0_h"]]), href["entry"][b][0], D["dtype"], f"hca compress b{b}")
        g = np.stack([_np(T["h_out"][b, 0]) for b in range(D["B"])])
        o = np.stack([href["out"][b] for b in range(D["B"])])
        check_close(g, o, D["dtype"], "hca out")


# ----------------------------------------------------------------------------- HCA decode

HCA_CASES = {
    "hca_small_ragged": (2, {"B": 3, "T": 128 * 300}),
    "hca_full": (2, None),
}


@pytest.mark.parametrize("case", list(HCA_CASES))
def test_hca_decode(case):
    i, sc = HCA_CASES[case]
    wl = CI.make_workload(i, scale=sc)
    D = wl.dims
    T = run(wl)
    ref = O.run_hca_decode(wl)
    for b in range(D["B"]):
        check_close(_np(T["cache"][b, D["entry0"]]), ref["entry"][b][0], D["dtype"], f"compress b{b}")
    g = np.stack([_np(T["out"][b, 0]) for b in range(D["B"])])
    o = np.stack([ref["out"][b] for b in range(D["B"])])
    check_close(g, o, D["dtype"], "hca out")
    np.testing.assert_allclose(_np(T["lse"][:, 0]), np.stack([ref["lse"][b] for b in range(D["B"])]),
                               atol=2e-3, rtol=0)


@pytest.mark.parametrize("case", list(HCA_CASES))
def test_fused_hca_step_equals_separate_calls(case):
    """hca_compress_attn_decode (attention started while the compression runs) gives
    bit-for-bit the results of hca_compress followed by hca_attn_decode."""
    i, sc = HCA_CASES[case]
    wl = CI.make_workload(i, scale=sc)
    D = wl.dims
    T = steps.upload(wl)
    cache0 = T["cache"].clone()
    csa.hca_compress(T["C"], T["Z"], T["bias"], T["entry0"], T["cache"], D["m_prime"])
    csa.hca_attn_decode(T["q"][:, 0], T["cache"], T["n_entries"], T["win"], T["win_len"], T["sink"], D["sm_scale"],
                        D["dv"], T["out"][:, 0], T["lse"][:, 0], T["aws"])
    torch.cuda.synchronize()
    out_sep, lse_sep, cache_sep = T["out"].clone(), T["lse"].clone(), T["cache"].clone()
    T["cache"].copy_(cache0)
    T["out"].zero_()
    csa.hca_compress_attn_decode(T["C"], T["Z"], T["bias"], T["entry0"], T["q"][:, 0], T["cache"], T["n_entries"],
                                 T["win"], T["win_len"], T["sink"], D["sm_scale"], D["dv"], T["out"][:, 0],
                                 T["lse"][:, 0], T["aws"], m_prime=D["m_prime"])
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    assert torch.equal(T["cache"], cache_sep)
    assert torch.equal(T["out"], out_sep)
    assert torch.equal(T["lse"], lse_sep)


# ----------------------------------------------------------------------------- edge cases

def test_decode_ragged_window_pad_indices_and_determinism():
    wl = CI.make_workload(1, scale={"B": 3, "T": 4096, "k": 600})
    D = wl.dims
    T = steps.upload(wl)
    d = D["d"]
    # idx with -1 slots and duplicates-free arbitrary order; ragged window lengths
    rng = np.random.default_rng(0)
    idx = np.full((3, 600), -1, np.int32)
    for b, cnt in enumerate([600, 17, 0]):
        idx[b, :cnt] = rng.choice(D["N"], cnt, replace=False)
    win_len = np.array([128, 5, 0], np.int32)
    T["idx"] = torch.from_numpy(idx).cuda().view(3, 1, 600)
    T["win_len"] = torch.from_numpy(win_len).cuda()
    outs = []
    for _ in range(2):
        csa.sparse_attn_decode(T["q"][:, 0], T["cache"], T["idx"][:, 0], T["win"], T["win_len"], T["sink"],
                               D["sm_scale"], D["dv"], T["out"][:, 0], T["lse"][:, 0], T["aws"])
        torch.cuda.synchronize()
        outs.append(T["out"].clone())
    assert torch.equal(outs[0], outs[1])                 # run-to-run bitwise determinism
    assert csa.read_device_error() == 0
    cache = O.decode_bf16(wl.tensors["cache"])
    win = O.decode_bf16(wl.tensors["win"])
    sink = wl.tensors["sink"].astype(np.float64)
    for b in range(3):
        sel = idx[b][idx[b] >= 0]
        rows = np.concatenate([cache[b][sel], win[b][:win_len[b]]], axis=0)
        o, lse = O.attention(O.decode_bf16(wl.tensors["q"][b, 0]), rows, sink, D["sm_scale"], D["dv"])
        check_close(_np(T["out"][b, 0]), o, "bf16", f"b{b}")
    # b = 2 has no rows at all: the sink takes all the weight -> zero output
    assert torch.count_nonzero(T["out"][2, 0]) == 0


def test_decode_out_of_range_index_is_flagged_not_faulted():
    wl = CI.make_workload(1, scale={"B": 2, "T": 4096, "k": 64})
    D = wl.dims
    T = steps.upload(wl)
    idx = torch.arange(64, dtype=torch.int32, device="cuda").repeat(2, 1)
    idx[1, 5] = D["N"] + 7                                # outside the cache: skipped and reported
    csa.sparse_attn_decode(T["q"][:, 0], T["cache"], idx, T["win"], T["win_len"], T["sink"], D["sm_scale"],
                           D["dv"], T["out"][:, 0], T["lse"][:, 0], T["aws"])
    torch.cuda.synchronize()
    assert csa.read_device_error() & 0x1
    assert csa.read_device_error() == 0                   # reading clears the word


def test_hca_ragged_entry_counts():
    wl = CI.make_workload(2, scale={"B": 3, "T": 128 * 256})
    D = wl.dims
    T = steps.upload(wl)
    n_ent = np.array([256, 1, 100], np.int32)
    win_len = np.array([128, 3, 64], np.int32)
    T["n_entries"] = torch.from_numpy(n_ent).cuda()
    T["win_len"] = torch.from_numpy(win_len).cuda()
    csa.hca_attn_decode(T["q"][:, 0], T["cache"], T["n_entries"], T["win"], T["win_len"], T["sink"], D["sm_scale"],
                        D["dv"], T["out"][:, 0], T["lse"][:, 0], T["aws"])
    torch.cuda.synchronize()
    cache = O.decode_bf16(wl.tensors["cache"])
    win = O.decode_bf16(wl.tensors["win"])
    for b in range(3):
        rows = np.concatenate([cache[b][:n_ent[b]], win[b][:win_len[b]]], axis=0)
        o, _ = O.attention(O.decode_bf16(wl.tensors["q"][b, 0]), rows, wl.tensors["sink"].astype(np.float64),
                           D["sm_scale"], D["dv"])
        check_close(_np(T["out"][b, 0]), o, "bf16", f"b{b}")


def test_topk_select_exact_with_ties_nan_and_ragged_rows():
    rng = np.random.default_rng(5)
    R, n, k = 7, 5000, 300
    s = rng.integers(0, 50, size=(R, n)).astype(np.float32)      # heavy ties
    s[1] = rng.standard_normal(n).astype(np.float32)
    s[2, ::7] = np.nan
    s[3] = 0.0
    n_valid = np.array([5000, 4999, 3000, 300, 299, 1, 0], np.int32)
    S = torch.from_numpy(s).cuda()
    out = torch.empty(R, k, dtype=torch.int32, device="cuda")
    csa.topk_select(S, torch.from_numpy(n_valid).cuda(), k, out)
    torch.cuda.synchronize()
    g = out.cpu().numpy()
    for r in range(R):
        nv = n_valid[r]
        row = np.where(np.isnan(s[r, :nv]), -np.inf, s[r, :nv]).astype(np.float64)
        exp = O.topk(row, nv, k)
        assert np.array_equal(g[r], exp), r


def test_lightning_index_score_out_and_k_equals_n():
    wl = CI.make_workload(1, scale={"B": 2, "T": 2048, "k": 512})     # N = 512 = k: everything selected
    D = wl.dims
    T = steps.upload(wl)
    so = torch.empty(2, 1, 512, dtype=torch.float32, device="cuda")
    csa.lightning_index(T["qI"], T["qI_scale"], T["w"], T["kI"], T["kI_scale"], T["n_entries"], T["q_pos"], 512,
                        csa.CSA_IFMT_E4M3, T["idx"], T["iws"], score_out=so)
    torch.cuda.synchronize()
    assert np.array_equal(T["idx"][:, 0].cpu().numpy(), np.tile(np.arange(512), (2, 1)))
    for b in range(2):
        I = O.indexer_scores(wl.tensors["qI"][b], wl.tensors["w"][b], wl.tensors["kI"][b], "e4m3",
                             wl.tensors["qI_scale"][b], wl.tensors["kI_scale"][b])[0]
        np.testing.assert_allclose(so[b, 0].cpu().numpy(), I, rtol=1e-6)


def _dequant_rows(codes, scale, fmt):
    if fmt == "e4m3":
        return O.decode_e4m3(codes) * np.asarray(scale, np.float64)[..., None]
    v = O.decode_e2m1_packed(codes)
    return v * np.repeat(O.decode_ue8m0(scale), 32, axis=-1)


@pytest.mark.parametrize("wid,sc", [(1, {"B": 4, "T": 65536}), (3, {"ctx": 16384, "Tq": 64, "k": 1024}),
                                    (4, {"B": 2, "T": 262144})])
def test_indexer_fp32_score_error_within_band_bound(wid, sc):
    """The exact top-k trusts |S32 - S| <= eps * U * knmax (U = sum_j w_j ||q_j||,
    knmax >= max_s ||k_s||).  Measure the fp32 scores the scoring kernel leaves in
    the workspace against the exact oracle scores and check the bound with margin."""
    wl = CI.make_workload(wid, scale=sc)
    D = wl.dims
    T = steps.upload(wl)
    fmt = D["ifmt"]
    csa.lightning_index(T["qI"], T["qI_scale"], T["w"], T["kI"], T["kI_scale"], T["n_entries"], T["q_pos"], D["k"],
                        csa.CSA_IFMT_E4M3 if fmt == "e4m3" else csa.CSA_IFMT_MXFP4, T["idx"], T["iws"])
    torch.cuda.synchronize()
    B, Tq, N = D["B"], D["Tq"], D["N"]
    ld = (N + 63) // 64 * 64
    S32 = T["iws"][:B * Tq * ld * 4].view(torch.float32).view(B, Tq, ld).double().cpu().numpy()
    off = (B * Tq * ld * 4 + 255) // 256 * 256
    knmax = T["iws"][off:off + 4 * B].view(torch.float32).double().cpu().numpy()
    worst = 0.0
    for b in range(B):
        qv = _dequant_rows(wl.tensors["qI"][b], wl.tensors["qI_scale"][b], fmt)
        U = (wl.tensors["w"][b] * np.sqrt((qv ** 2).sum(-1))).sum(-1)                  # [Tq]
        kn = np.sqrt((_dequant_rows(wl.tensors["kI"][b], wl.tensors["kI_scale"][b], fmt) ** 2).sum(-1))
        assert knmax[b] >= kn.max() * (1 - 1e-6)
        I = O.indexer_scores(wl.tensors["qI"][b], wl.tensors["w"][b], wl.tensors["kI"][b], fmt,
                             wl.tensors["qI_scale"][b], wl.tensors["kI_scale"][b])
        for t in range(Tq):
            ne = O.n_eligible(D["q_pos0"] + t, D["m"], N)
            err = np.abs(S32[b, t, :ne] - I[t, :ne]) / (U[t] * knmax[b])
            worst = max(worst, float(err.max()))
    print(f"max |S32-S| / (U knmax) = {worst:.3e}")
    assert worst <= 1.0 / 131072 / 4        # the kernel's eps (2^-17) with a 4x margin
