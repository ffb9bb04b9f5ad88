"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: closed forms
(uniform gates give the block mean, [P1] exercise 2), exact integer arithmetic
(FP8 / MXFP4 dot products through Python fractions), independent library
routines (torch's float8 / bfloat16 decoders, torch's scaled-dot-product
attention in float64, a full Python sort for top-k), locality / invariance
properties, and the entry counts of [P1] exercise 1.

[P1] "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section
     "Гибридное внимание: CSA и HCA" and "Что сделать руками".
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# ---------------------------------------------------------------- formats

def test_e4m3_table_matches_torch_decoder():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.decode_e4m3(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours)) and nan.sum() == 2
    assert np.array_equal(ref[~nan], ours[~nan])


def test_e4m3_landmarks():
    t = O.E4M3
    assert t[0x38] == 1.0 and t[0xB8] == -1.0
    assert t[0x7E] == 448.0                 # largest finite
    assert t[0x01] == 2.0 ** -9             # smallest subnormal
    assert t[0x08] == 2.0 ** -6             # smallest normal


def test_e2m1_grid_and_ue8m0():
    assert list(O.E2M1[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(O.E2M1[8:]) == [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]
    assert O.decode_ue8m0(np.array([127, 128, 120], np.uint8)).tolist() == [1.0, 2.0, 2.0 ** -7]
    # low nibble is element 0
    v = O.decode_e2m1_packed(np.array([[0x72]], np.uint8))
    assert v.tolist() == [[1.0, 6.0]]


def test_bf16_decode_and_round_match_torch():
    x = torch.from_numpy(rng.standard_normal(4096).astype(np.float32) * 10)
    bits = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.decode_bf16(bits), x.to(torch.bfloat16).to(torch.float64).numpy())
    # rounding of float32 inputs (no double rounding possible) agrees with torch's RNE cast
    assert np.array_equal(O.round_to_bf16(x.numpy().astype(np.float64)),
                          x.to(torch.bfloat16).to(torch.float64).numpy())
    # an exact tie goes to the even mantissa
    one_plus_half_ulp = 1.0 + 2.0 ** -8
    assert O.round_to_bf16(np.array([one_plus_half_ulp]))[0] == 1.0
    assert O.round_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


# ---------------------------------------------------------------- a1: CSA compression

def _csa_inputs(T, d, m=4, seed=0):
    r = np.random.default_rng(seed)
    return [r.standard_normal((T, d)) for _ in range(4)] + \
           [0.1 * r.standard_normal((m, d)) for _ in range(2)] + \
           [r.standard_normal((m, d)), r.standard_normal((m, d))]


def test_csa_uniform_gates_give_block_means():
    """[P1] exercise 2: with equal gates the pooling is a plain average of the 2m sources."""
    T, d, m = 32, 5, 4
    Ca, Cb, _, _, _, _, pCb, _ = _csa_inputs(T, d)
    Z = np.zeros((T, d)); B = np.zeros((m, d)); pZ = np.zeros((m, d))
    # chunk at sequence start: entry 0 averages its 4 a-sources only
    out = O.csa_compress(Ca, Cb, Z, Z, B, B, None, None, 0, m)
    assert out.shape == (T // m, d)
    np.testing.assert_allclose(out[0], Ca[0:4].mean(axis=0), rtol=0, atol=1e-14)
    for i in range(1, T // m):
        ref = np.concatenate([Cb[4 * i - 4:4 * i], Ca[4 * i:4 * i + 4]]).mean(axis=0)
        np.testing.assert_allclose(out[i], ref, rtol=0, atol=1e-14)
    # a chunk later in the sequence takes the b-half of entry 0 from prev_Cb
    out2 = O.csa_compress(Ca, Cb, Z, Z, B, B, pCb, pZ, 7, m)
    np.testing.assert_allclose(out2[0], np.concatenate([pCb, Ca[0:4]]).mean(axis=0), atol=1e-14)


def test_csa_one_hot_gate_selects_source():
    T, d, m = 16, 3, 4
    Ca, Cb, _, _, _, _, pCb, _ = _csa_inputs(T, d, seed=1)
    Za = np.zeros((T, d)); Zb = np.zeros((T, d)); B = np.zeros((m, d))
    Zb[5, 1] = 1e4                    # b-series token 5 is a source of entry 2 (tokens 4..7)
    Za[9, 2] = 1e4                    # a-series token 9 belongs to entry 2 (tokens 8..11)
    out = O.csa_compress(Ca, Cb, Za, Zb, B, B, None, None, 0, m)
    assert out[2, 1] == pytest.approx(Cb[5, 1], abs=1e-12)
    assert out[2, 2] == pytest.approx(Ca[9, 2], abs=1e-12)


def test_csa_window_alignment_and_overlap():
    """Token t is an a-source of entry t//m and a b-source of entry t//m + 1 only:
    entry i pools tokens [4i-4, 4i+4) ([P1] step 1: overlapping 2m windows, stride m)."""
    T, d, m = 32, 4, 4
    args = _csa_inputs(T, d, seed=2)
    base = O.csa_compress(*args[:6], None, None, 0, m)
    for t in [0, 5, 13, 31]:
        for series in (0, 1):             # perturb C^a (a-series) or C^b (b-series)
            pert = [a.copy() for a in args[:6]]
            pert[series][t] += 1.0
            out = O.csa_compress(*pert, None, None, 0, m)
            changed = set(np.nonzero(np.abs(out - base).max(axis=1) > 0)[0].tolist())
            expect = {t // m} if series == 0 else ({t // m + 1} if t // m + 1 < T // m else set())
            assert changed == expect, (t, series, changed)


def test_csa_convex_and_shift_invariant():
    T, d, m = 24, 6, 4
    Ca, Cb, Za, Zb, Ba, Bb, pCb, pZb = _csa_inputs(T, d, seed=3)
    out = O.csa_compress(Ca, Cb, Za, Zb, Ba, Bb, pCb, pZb, 3, m)
    # adding one constant to every gate logit of a component changes nothing
    out2 = O.csa_compress(Ca, Cb, Za + 3.7, Zb + 3.7, Ba, Bb, pCb, pZb + 3.7, 3, m)
    np.testing.assert_allclose(out, out2, rtol=0, atol=1e-13)
    # constant values are reproduced exactly
    c = np.full((T, d), 2.5)
    out3 = O.csa_compress(c, c, Za, Zb, Ba, Bb, np.full((m, d), 2.5), pZb, 3, m)
    np.testing.assert_allclose(out3, 2.5, atol=1e-14)
    # every output lies inside the range of its sources
    for i in range(T // m):
        src = np.concatenate([pCb if i == 0 else Cb[4 * i - 4:4 * i], Ca[4 * i:4 * i + 4]])
        assert np.all(out[i] <= src.max(axis=0) + 1e-12) and np.all(out[i] >= src.min(axis=0) - 1e-12)


def test_csa_chunked_equals_whole():
    """Compressing a sequence in two chunks (the second with the first's last b-block
    as prev) equals compressing it whole: the KV-cache append is consistent."""
    T, d, m = 40, 3, 4
    Ca, Cb, Za, Zb, Ba, Bb, _, _ = _csa_inputs(T, d, seed=4)
    whole = O.csa_compress(Ca, Cb, Za, Zb, Ba, Bb, None, None, 0, m)
    c = 16
    p1 = O.csa_compress(Ca[:c], Cb[:c], Za[:c], Zb[:c], Ba, Bb, None, None, 0, m)
    p2 = O.csa_compress(Ca[c:], Cb[c:], Za[c:], Zb[c:], Ba, Bb, Cb[c - m:c], Zb[c - m:c], c // m, m)
    np.testing.assert_allclose(np.concatenate([p1, p2]), whole, rtol=0, atol=1e-15)


# ---------------------------------------------------------------- a2: HCA compression

def test_hca_uniform_gates_give_block_means_and_no_overlap():
    T, d, mp = 384, 4, 128
    r = np.random.default_rng(5)
    C = r.standard_normal((T, d))
    out = O.hca_compress(C, np.zeros((T, d)), np.zeros((mp, d)), mp)
    assert out.shape == (3, d)
    for i in range(3):
        np.testing.assert_allclose(out[i], C[mp * i:mp * (i + 1)].mean(axis=0), atol=1e-14)
    Z = r.standard_normal((T, d)); bias = 0.1 * r.standard_normal((mp, d))
    base = O.hca_compress(C, Z, bias, mp)
    C2 = C.copy(); C2[200] += 1
    changed = np.nonzero(np.abs(O.hca_compress(C2, Z, bias, mp) - base).max(axis=1))[0]
    assert changed.tolist() == [1]


def test_hca_one_hot():
    T, d, mp = 128, 2, 128
    r = np.random.default_rng(6)
    C = r.standard_normal((T, d)); Z = np.zeros((T, d)); bias = np.zeros((mp, d))
    bias[77, 0] = 1e4
    out = O.hca_compress(C, Z, bias, mp)
    assert out[0, 0] == pytest.approx(C[77, 0], abs=1e-12)


def test_exercise1_entry_counts():
    """[P1] "Что сделать руками" exercise 1: entries at a 1M context for m=4 and m'=128."""
    with open(os.path.join(GOLDEN, "exercise1_entry_counts.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for ctx, m, count in rows:
        ctx, m, count = int(ctx), int(m), int(count)
        assert O.n_eligible(ctx - 1, m, 1 << 40) == count
        T = m * 2
        out = O.hca_compress(np.zeros((T, 1)), np.zeros((T, 1)), np.zeros((m, 1)), m) if m > 4 else \
            O.csa_compress(*[np.zeros((T, 1))] * 4, np.zeros((m, 1)), np.zeros((m, 1)), None, None, 0, m)
        assert out.shape[0] == T // m       # the sequence shrinks exactly m times


# ---------------------------------------------------------------- a3: indexer

def _e4m3_fraction(code: int) -> Fraction:
    """Exact value of an e4m3 code from integer fields (independent of the table)."""
    s = -1 if code & 0x80 else 1
    e = (code >> 3) & 0xF
    mant = code & 7
    if e == 0:
        return Fraction(s * mant, 8 * 64)
    return s * Fraction(8 + mant, 8) * (Fraction(2) ** (e - 7))


def test_fp8_head_dots_exact():
    r = np.random.default_rng(7)
    q = r.integers(0, 256, size=(2, 3, 16), dtype=np.uint8)
    k = r.integers(0, 256, size=(5, 16), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x3F            # no NaN codes
    k[(k & 0x7F) == 0x7F] = 0x3F
    qs = np.array([[0.5, 0.25, 2.0], [1.0, 4.0, 0.125]])
    ks = np.array([1.0, 0.5, 2.0, 0.25, 8.0])
    D = O.head_dots(q, k, "e4m3", qs, ks)
    for t in range(2):
        for j in range(3):
            for s in range(5):
                exact = sum(_e4m3_fraction(int(a)) * _e4m3_fraction(int(b)) for a, b in zip(q[t, j], k[s]))
                assert D[t, j, s] == float(Fraction(qs[t, j]) * Fraction(ks[s]) * exact)


def test_mxfp4_head_dots_exact():
    r = np.random.default_rng(8)
    qp = r.integers(0, 256, size=(1, 2, 32), dtype=np.uint8)     # d_I = 64 -> 2 blocks
    kp = r.integers(0, 256, size=(3, 32), dtype=np.uint8)
    qsc = r.integers(120, 135, size=(1, 2, 2), dtype=np.uint8)
    ksc = r.integers(120, 135, size=(3, 2), dtype=np.uint8)
    grid = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]

    def val(nib):
        return (-1 if nib & 8 else 1) * grid[nib & 7]

    D = O.head_dots(qp, kp, "mxfp4", qsc, ksc)
    for j in range(2):
        for s in range(3):
            tot = Fraction(0)
            for c in range(64):
                qb = int(qp[0, j, c // 2]); kb = int(kp[s, c // 2])
                qn = qb & 0xF if c % 2 == 0 else qb >> 4
                kn = kb & 0xF if c % 2 == 0 else kb >> 4
                blk = c // 32
                sc = Fraction(2) ** (int(qsc[0, j, blk]) - 127) * Fraction(2) ** (int(ksc[s, blk]) - 127)
                tot += sc * val(qn) * val(kn)
            assert D[0, j, s] == float(tot)


def test_indexer_relu_weighting():
    """I = sum_j w_j max(0, D_j): heads with negative dots contribute nothing, and the
    score is linear in w ([P1] CSA step 2 'оценки с ReLU'; [P3] ReLU-scored dot)."""
    r = np.random.default_rng(9)
    q = r.standard_normal((3, 4, 8)); k = r.standard_normal((10, 8)); w = r.uniform(size=(3, 4))
    I = O.indexer_scores(q, w, k, "f32")
    D = np.einsum("tjc,sc->tjs", q, k)
    for t in range(3):
        for s in range(10):
            pos = [j for j in range(4) if D[t, j, s] > 0]
            assert I[t, s] == pytest.approx(sum(w[t, j] * D[t, j, s] for j in pos), rel=1e-13, abs=1e-15)
    assert np.all(I >= 0)
    np.testing.assert_allclose(O.indexer_scores(q, 3 * w, k, "f32"), 3 * I, rtol=1e-14)


def test_eligibility():
    # entry s is complete once its last source token m*s+m-1 has been seen
    assert O.n_eligible(2, 4, 100) == 0
    assert O.n_eligible(3, 4, 100) == 1
    assert O.n_eligible(7, 4, 100) == 2
    assert O.n_eligible(10 ** 6, 4, 5) == 5


# ---------------------------------------------------------------- a4: top-k

def test_topk_equals_full_sort():
    r = np.random.default_rng(10)
    for trial in range(200):
        n = int(r.integers(1, 40)); k = int(r.integers(1, 12)); ne = int(r.integers(0, n + 1))
        s = r.integers(0, 6, size=n).astype(np.float64)        # many exact ties
        got = O.topk(s, ne, k)
        ref = sorted(range(ne), key=lambda i: (-s[i], i))[:k]
        exp = sorted(ref) + [-1] * (k - len(ref))
        assert got.tolist() == exp


def test_topk_bf16_rounds_before_selecting():
    """Scores 1 + 2^-9 and 1 + 2^-8 round to the bf16 key 1.0 (ulp 2^-7), so they tie with
    an exact 1.0 and the lowest indices win; 1 + 3 * 2^-8 rounds up to 1 + 2^-7."""
    s = np.array([1.0, 1.0 + 2.0 ** -8, 0.5, 1.0 + 2.0 ** -9, 1.0 + 3 * 2.0 ** -8, 0.25])
    assert O.topk(s, 6, 2).tolist() == [1, 4]                # exact: the two largest
    assert O.topk(s, 6, 3).tolist() == [1, 3, 4]
    assert O.topk_bf16(s, 6, 2).tolist() == [0, 4]           # bf16: 1+3*2^-8 -> 1+2^-7, then ties at 1.0
    assert O.topk_bf16(s, 6, 3).tolist() == [0, 1, 4]
    assert O.topk_bf16(s, 3, 5).tolist() == [0, 1, 2, -1, -1]
    # keys already on the bf16 grid select exactly as topk does
    g = O.round_to_bf16(np.random.default_rng(2).normal(size=300))
    assert np.array_equal(O.topk_bf16(g, 300, 40), O.topk(g, 300, 40))


def test_topk_invariant_to_positive_weight_scale():
    r = np.random.default_rng(11)
    q = r.standard_normal((2, 4, 8)); k = r.standard_normal((50, 8)); w = r.uniform(size=(2, 4))
    a = O.indexer_scores(q, w, k, "f32"); b = O.indexer_scores(q, 0.37 * w, k, "f32")
    for t in range(2):
        assert np.array_equal(O.topk(a[t], 50, 7), O.topk(b[t], 50, 7))


# ---------------------------------------------------------------- a5/a6: attention

def _sdpa_with_sink(q, rows, sink, scale, dv):
    """torch's scaled_dot_product_attention (float64) with the sink as one extra
    key of value zero whose logit is set through an additive mask."""
    H, dk = q.shape
    R = rows.shape[0]
    K = torch.zeros(1, 1, R + 1, dk, dtype=torch.float64)
    K[0, 0, :R] = torch.from_numpy(rows)
    V = torch.zeros(1, 1, R + 1, dv, dtype=torch.float64)
    V[0, 0, :R] = torch.from_numpy(rows[:, :dv])
    Q = torch.from_numpy(q).reshape(1, H, 1, dk)
    mask = torch.zeros(1, H, 1, R + 1, dtype=torch.float64)
    mask[0, :, 0, R] = torch.from_numpy(sink)
    out = torch.nn.functional.scaled_dot_product_attention(
        Q, K.expand(1, H, R + 1, dk), V.expand(1, H, R + 1, dv), attn_mask=mask, scale=scale)
    return out[0, :, 0, :].numpy()


def test_attention_matches_library_sdpa():
    r = np.random.default_rng(12)
    H, dk, dv, R = 4, 12, 8, 30
    q = r.standard_normal((H, dk)); rows = r.standard_normal((R, dk)); sink = r.standard_normal(H)
    o, lse = O.attention(q, rows, sink, 0.3, dv)
    np.testing.assert_allclose(o, _sdpa_with_sink(q, rows, sink, 0.3, dv), rtol=1e-12, atol=1e-13)
    # lse matches an independent log-sum-exp over logits and sink
    from scipy.special import logsumexp
    L = 0.3 * q @ rows.T
    np.testing.assert_allclose(lse, logsumexp(np.concatenate([L, sink[:, None]], axis=1), axis=1), rtol=1e-13)


def test_attention_without_sink_is_dense_softmax_attention():
    """k = all entries, no window, sink = -inf: plain dense attention over the compressed KV."""
    r = np.random.default_rng(13)
    H, dk, dv, R = 3, 16, 16, 20
    q = r.standard_normal((H, dk)); rows = r.standard_normal((R, dk))
    o, _ = O.attention(q, rows, np.full(H, -np.inf), 0.25, dv)
    Q = torch.from_numpy(q).reshape(1, H, 1, dk)
    Kt = torch.from_numpy(rows).reshape(1, 1, R, dk).expand(1, H, R, dk)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, Kt, Kt, scale=0.25)[0, :, 0].numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_attention_weights_sum_to_one_with_sink():
    r = np.random.default_rng(14)
    H, dk, R = 5, 8, 17
    q = r.standard_normal((H, dk)); sink = r.standard_normal(H)
    rows = r.standard_normal((R, dk)); rows[:, :1] = 1.0        # value dim 0 is constant 1
    o, lse = O.attention(q, rows, sink, 0.5, 1)
    # o = sum_r p_r * 1 = 1 - p_sink, with p_sink = e^{sink - lse}
    np.testing.assert_allclose(o[:, 0] + np.exp(sink - lse), 1.0, rtol=0, atol=1e-14)


def test_attention_special_cases():
    r = np.random.default_rng(15)
    H, dk, dv = 2, 6, 4
    q = r.standard_normal((H, dk)); row = r.standard_normal((1, dk))
    o, _ = O.attention(q, row, np.full(H, -np.inf), 1.0, dv)
    np.testing.assert_allclose(o, np.repeat(row[:, :dv], H, axis=0), atol=1e-15)
    rows = r.standard_normal((9, dk))
    o_big, _ = O.attention(q, rows, np.full(H, 1e6), 1.0, dv)         # sink -> +inf
    assert np.abs(o_big).max() < 1e-300
    perm = r.permutation(9)
    a, _ = O.attention(q, rows, np.zeros(H), 1.0, dv)
    b, _ = O.attention(q, rows[perm], np.zeros(H), 1.0, dv)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


def test_hca_is_sparse_attention_with_all_entries():
    """HCA dense attention = CSA sparse attention with idx = every entry ([P1] HCA paragraph)."""
    r = np.random.default_rng(16)
    N, dk, H, dv = 12, 8, 2, 6
    cache = r.standard_normal((N, dk)); win = r.standard_normal((3, dk)); q = r.standard_normal((H, dk))
    sink = r.standard_normal(H)
    idx = O.topk(np.zeros(N), N, N)
    assert idx.tolist() == list(range(N))
    a, _ = O.attention(q, np.concatenate([cache, win]), sink, 0.3, dv)
    b, _ = O.attention(q, np.concatenate([cache[idx], win]), sink, 0.3, dv)
    np.testing.assert_array_equal(a, b)


def test_window_range():
    assert O.window_range(0, 16) == (0, 1)
    assert O.window_range(5, 16) == (0, 6)
    assert O.window_range(100, 16) == (85, 101)


# ---------------------------------------------------------------- indexer-key producer
# [P1] section "FP4 с учётом квантования": the indexer's Q·K activations are cached in
# FP4 (MXFP4, 1x32 tiles); the keys of compressed entries come from CSA step 1's pooling.

def _e4m3_cases():
    mags = O.E4M3_MAGS
    mids = (mags[1:] + mags[:-1]) / 2                       # every rounding tie
    r = np.random.default_rng(7)
    rand = np.exp(r.uniform(np.log(2.0 ** -12), np.log(448.0), 4000))
    v = np.concatenate([mags, mids, rand, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)])
    v = v[v <= 448.0]
    return np.concatenate([v, -v])


def test_e4m3_encoder_matches_torch_cast():
    """torch's float8_e4m3fn cast (round to nearest even) is an independent encoder in the
    finite range; it keeps the sign of a value that rounds to zero, the oracle writes +0."""
    v = _e4m3_cases()
    ref = torch.tensor(v, dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref = np.where(ref == 0x80, 0, ref)
    assert np.array_equal(O.encode_e4m3(v), ref)


def test_e4m3_encoder_landmarks_and_saturation():
    v = np.array([1.0, 17.0, 19.0, 2.0 ** -10, 3 * 2.0 ** -10, 448.0, 464.0, 1e6, -1e6, -1e-5, -2.0 ** -9])
    # 17 ties 16 (even mantissa) / 18; 19 ties 18 / 20 (even); 2^-10 ties 0 / 2^-9
    assert O.encode_e4m3(v).tolist() == [0x38, 0x58, 0x5A, 0x00, 0x02, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x81]


def test_e2m1_encoder_ties_and_saturation():
    # grid 0 .5 1 1.5 2 3 4 6 (codes 0..7); ties go to the even code
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 0.26, 4.9, -0.1, -0.3, -6.0, -100.0])
    assert O.encode_e2m1(v).tolist() == [0, 2, 2, 4, 4, 6, 6, 7, 1, 6, 0, 9, 15, 15]


def test_mx_exponent_is_smallest_power_covering_amax():
    f32_above_6 = float(np.nextafter(np.float32(6.0), np.float32(7.0)))
    a = np.array([6.0, f32_above_6, 3.0, 0.0, 1.5, 1.5000001, 1e-45, 6.0 * 2.0 ** 100])
    assert O.mx_exponent(a).tolist() == [0, 1, -1, -127, -2, -1, -127, 100]
    r = np.random.default_rng(3)
    amax = np.exp(r.uniform(-30, 30, 500))
    e = O.mx_exponent(amax)
    assert np.all(amax <= 6.0 * np.ldexp(1.0, e)) and np.all(amax > 6.0 * np.ldexp(1.0, e - 1))


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
def test_quantised_keys_are_nearest_grid_values(fmt):
    """Brute force: every code decodes to a grid value at least as close to y as any
    other; the row (block) maximum lands at the top of the grid."""
    r = np.random.default_rng(11)
    x = r.normal(size=(24, 128)) * np.exp(r.uniform(-8, 8, size=(24, 1)))
    x[3] = 0.0                                              # an all-zero row
    codes, scales, y = O.quantise_index_keys(x, fmt)
    if fmt == "e4m3":
        grid = O.E4M3_MAGS
        dq = O.decode_e4m3(codes)
        assert scales[3] == 1.0 and not codes[3].any()
        live = np.abs(x).max(axis=1) > 0
        assert np.all(np.abs(y[live]).max(axis=1) == pytest.approx(448.0, rel=1e-6))
        # half a step of the grid: 2^-4 relative for normals, 2^-10 absolute (in units of the
        # scale) among subnormals, plus the fp32 rounding of x and y
        s64 = scales[:, None].astype(np.float64)
        assert np.all(np.abs(dq * s64 - x) <= 2.0 ** -4 * np.abs(x) + 2.0 ** -10 * s64 + 2.0 ** -22 * np.abs(x))
    else:
        grid = O.E2M1_MAGS
        dq = O.decode_e2m1_packed(codes)
        assert not codes[3].any() and np.all(scales[3] == 0)
        top = np.abs(y).reshape(24, 4, 32).max(axis=2)
        live = top > 0
        assert np.all((top[live] > 3.0) & (top[live] <= 6.0))
    dist = np.abs(np.abs(y)[..., None] - grid).min(axis=-1)
    assert np.allclose(np.abs(np.abs(dq) - np.abs(y)), dist, rtol=0, atol=0)
    assert np.all((np.sign(dq) == np.sign(y)) | (dq == 0))


def test_index_key_compress_constant_rows_give_grid_codes():
    """C constant along tokens: any gates give that constant (weights sum to one), so
    rows that sit on the code grid come back as exactly those codes."""
    r = np.random.default_rng(5)
    m, d, n = 4, 64, 3
    e4 = O.E4M3_MAGS[r.integers(1, 126, size=(n, d))] * np.where(r.random((n, d)) < 0.5, -1, 1)
    e4[:, 0] = 448.0
    row = np.repeat(e4, m, axis=0)                           # [n*m, d]: token 4i+t carries entry i's row
    Z = lambda: r.normal(0, 2, size=(n * m, d))
    B = lambda: r.normal(0, 0.1, size=(m, d))
    prev = np.repeat(e4[:1], m, axis=0)
    codes, scales, y, x = O.index_key_compress(row, np.concatenate([row[m:], prev]), Z(), Z(), B(), B(),
                                               "e4m3", prev_Cb=prev, prev_Zb=r.normal(size=(m, d)),
                                               first_entry=0)
    # entry 0 pools only its own a-block; entries 1.. pool the b-series of block i-1,
    # which carries row i here (Cb is shifted by one block), so every entry sees one value
    assert np.array_equal(scales, np.ones(n, np.float32))
    assert np.array_equal(O.decode_e4m3(codes), e4)
    g = O.E2M1_MAGS[r.integers(0, 8, size=(n, d))] * np.where(r.random((n, d)) < 0.5, -1, 1)
    g[:, ::32] = 6.0
    rowg = np.repeat(g * 4.0, m, axis=0)
    codes, scales, y, x = O.index_key_compress(rowg, np.concatenate([rowg[m:], rowg[:m]]), Z(), Z(), B(), B(),
                                               "mxfp4")
    assert np.all(scales == 129)                             # 2^2 covers 24 = 6 * 4
    assert np.array_equal(O.decode_e2m1_packed(codes), g + 0.0)


# ---------------------------------------------------------------- grouped output projection
# [P1] CSA step 4 and table "Конфигурации" (g groups, intermediate width, hidden size d).

def test_grouped_projection_is_a_block_diagonal_projection():
    """The grouped first stage is one projection by the block-diagonal matrix of the group
    matrices (built by scipy's block_diag) of the flattened head outputs."""
    from scipy.linalg import block_diag
    r = np.random.default_rng(21)
    T, H, dv, g, d_mid, d = 3, 8, 4, 4, 5, 6
    o = r.normal(size=(T, H, dv))
    W1 = r.normal(size=(g * d_mid, (H // g) * dv))
    W2 = r.normal(size=(d, g * d_mid))
    u, y = O.grouped_out_proj(o, W1, W2, g, dtype="f64")
    Bd = block_diag(*[W1[j * d_mid:(j + 1) * d_mid] for j in range(g)])     # [g*d_mid, H*dv]
    np.testing.assert_allclose(u, o.reshape(T, H * dv) @ Bd.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, (o.reshape(T, H * dv) @ Bd.T) @ W2.T, rtol=1e-12, atol=1e-12)


def test_grouped_projection_locality_and_rounding():
    """A change to one head reaches only its group's intermediate columns; u is rounded to
    bf16 before the second stage reads it."""
    r = np.random.default_rng(22)
    T, H, dv, g, d_mid, d = 2, 8, 4, 4, 3, 5
    o = r.normal(size=(T, H, dv))
    W1 = r.normal(size=(g * d_mid, (H // g) * dv))
    W2 = r.normal(size=(d, g * d_mid))
    u0, _ = O.grouped_out_proj(o, W1, W2, g, dtype="f64")
    o2 = o.copy()
    o2[:, 5] += 1.0                                          # head 5 is in group 2 (heads 4, 5)
    u1, _ = O.grouped_out_proj(o2, W1, W2, g, dtype="f64")
    changed = np.nonzero(np.any(u1 != u0, axis=0))[0]
    assert changed.tolist() == list(range(2 * d_mid, 3 * d_mid))
    ub, yb = O.grouped_out_proj(o, W1, W2, g, dtype="bf16")
    assert np.array_equal(ub, O.round_to_bf16(u0))
    assert np.array_equal(yb, O.round_to_bf16(O.round_to_bf16(u0) @ W2.T))


# ---------------------------------------------------------------- FP8 KV storage
# [P3] section "Гибридный attention: CSA и HCA": FP8 KV entries, BF16 RoPE dimensions.

def test_kv8_rows_layout_scale_and_error_bound():
    r = np.random.default_rng(41)
    x = r.normal(size=(40, 576)) * np.exp(r.uniform(-6, 6, size=(40, 1)))
    x[7] = 0.0
    q = O.quantise_latent_fp8(x)
    assert q.shape == (40, 656) and not q[:, 641:].any()
    e = q[:, 640].astype(np.int64) - 127
    amax = np.abs(x[:, :512].astype(np.float32).astype(np.float64)).max(axis=1)
    live = amax > 0
    assert np.all(amax[live] <= 448.0 * np.ldexp(1.0, e[live]))
    assert np.all(amax[live] > 448.0 * np.ldexp(1.0, e[live] - 1))
    assert e[7] == -126 and not q[7, :640].any()
    dq = O.dequantise_latent_fp8(q)
    # the codes are torch's float8 cast of x * 2^-e (up to the sign of zero)
    y = x[:, :512].astype(np.float32).astype(np.float64) * np.ldexp(1.0, -e)[:, None]
    ref = torch.tensor(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(np.where(ref == 0x80, 0, ref), q[:, :512])
    # nope: within half an e4m3 step (2^-4 relative; 2^-10 * 2^e among subnormals)
    s = np.ldexp(1.0, e)[:, None]
    assert np.all(np.abs(dq[:, :512] - x[:, :512]) <= 2.0 ** -4 * np.abs(x[:, :512]) + 2.0 ** -10 * s + 1e-30)
    # rope: torch's bf16 rounding of the fp32 value
    rb = torch.tensor(x[:, 512:].astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(dq[:, 512:], rb)
    # every dequantised value is a bf16 value (the attention kernel's exact operand)
    assert np.array_equal(O.round_to_bf16(dq), dq)


def test_kv8_rows_on_grid_round_trip_exactly():
    r = np.random.default_rng(42)
    codes = r.integers(0, 0x7F, size=(5, 512)).astype(np.uint8) | np.where(r.random((5, 512)) < 0.5, 0x80, 0).astype(np.uint8)
    codes[:, 3] = 0x7E                                      # 448 somewhere in every row
    e = np.array([-3, 0, 4, -126 + 9, 20])
    x = np.zeros((5, 576))
    x[:, :512] = O.decode_e4m3(codes) * np.ldexp(1.0, e)[:, None]
    x[:, 512:] = O.round_to_bf16(r.normal(size=(5, 64)))
    q = O.quantise_latent_fp8(x)
    assert np.array_equal(q[:, 640].astype(np.int64) - 127, e)
    assert np.array_equal(O.dequantise_latent_fp8(q), np.where(x == 0, 0.0, x))
