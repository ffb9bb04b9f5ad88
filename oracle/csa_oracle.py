"""fp64 CPU oracle for the CSA / HCA attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA library: it decodes the stored number formats itself, and every step
below is the plain definition written out in float64 with numpy.

Sources (DeepSeek-V4 technical report as digested on the web):

[P1] "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста" (ai.flicky.cc),
     section "Гибридное внимание: CSA и HCA": "CSA: сжать в 4 раза и выбрать
     top-k" steps 1-3, "HCA: сжать в 128 раз, но смотреть на всё", the table
     "Конфигурации", section "FP4 с учётом квантования", and "Что сделать
     руками" exercises 1-2.
[P3] aixai.ru blog post "deepseek-v4-million-token-context-agents", section
     "Гибридный attention: CSA и HCA" (softmax-gated pooling with a learnable
     positional bias; ReLU-scored multi-head dot product; FP8/BF16 KV storage).
[P4] "Технический отчёт DeepSeek-V4 — часть 1/2" (aifinder.ae): CSA is MLA with
     a sliding window; every 2m tokens are pooled with stride m; attention sink;
     partial RoPE on the last 64 of the 576 latent dims.

Readings where the pages are silent (the same readings bind the CUDA path):

* CSA entry i pools the b-series of block i-1 (tokens 4i-4..4i-1) and the
  a-series of block i (tokens 4i..4i+3): 2m = 8 sources.  Entry 0 has no
  b-half; its softmax runs over the 4 a-sources only.
* Positional biases are indexed by the offset j of a token inside its block:
  B^a[j], B^b[j] (j < m) for CSA and B[j] (j < m') for HCA.
* A compressed entry is visible to the query at absolute position p iff all its
  sources are <= p: entry s is eligible iff m*s + m - 1 <= p.
* Top-k orders eligible entries by (score descending, index ascending) and
  pads with -1 when fewer than k are eligible; the oracle reports the selected
  set in ascending index order.
* The window holds the raw latents of positions max(0, p-W+1)..p (the current
  token included); raw rows and compressed rows are separate softmax terms.
* The sink is a per-head logit with a zero value vector: it only enlarges the
  softmax denominator.
* Keys are the full d_k = 576 latent row, values its first d_v = 512 dims (MLA:
  one latent serves as K and V for every head, MQA).
* Indexer: I[t,s] = sum_j w[t,j] * max(0, sq[t,j] * sk[s] * <q8[t,j], k8[s]>)
  for FP8 with per-row scales; for MXFP4 the block scales multiply each
  32-element partial dot product.  No extra global score scale is applied.
* Stored results (compressed cache rows, attention outputs) are rounded to the
  storage format (bf16, round-to-nearest-even) when the workload is bf16.
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# number formats (decoded from their definitions)
# ---------------------------------------------------------------------------

def _e4m3_table() -> np.ndarray:
    """All 256 FP8 e4m3 codes as float64 (bias 7, 3 mantissa bits, no infinities;
    codes 0x7F / 0xFF are NaN, exponent field 0 is subnormal: mant/8 * 2^-6)."""
    t = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        mant = c & 0x7
        if e == 0xF and mant == 0x7:
            t[c] = np.nan
        elif e == 0:
            t[c] = s * (mant / 8.0) * 2.0 ** -6
        else:
            t[c] = s * (1.0 + mant / 8.0) * 2.0 ** (e - 7)
    return t


def _e2m1_table() -> np.ndarray:
    """All 16 FP4 e2m1 codes (bias 1, 1 mantissa bit, exponent 0 subnormal: mant * 0.5)."""
    t = np.empty(16, dtype=np.float64)
    for c in range(16):
        s = -1.0 if c & 0x8 else 1.0
        e = (c >> 1) & 0x3
        mant = c & 0x1
        t[c] = s * (mant * 0.5 if e == 0 else (1.0 + mant / 2.0) * 2.0 ** (e - 1))
    return t


E4M3 = _e4m3_table()
E2M1 = _e2m1_table()


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 storage bits (uint16) -> float64 (the upper half of an fp32 word)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    return E4M3[codes.astype(np.intp)]


def decode_e2m1_packed(packed: np.ndarray) -> np.ndarray:
    """[..., d/2] bytes -> [..., d] values; element 2i is the low nibble."""
    lo = E2M1[(packed & 0xF).astype(np.intp)]
    hi = E2M1[(packed >> 4).astype(np.intp)]
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.float64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def decode_ue8m0(codes: np.ndarray) -> np.ndarray:
    return np.ldexp(1.0, codes.astype(np.int64) - 127)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (8 significant bits, ties to even), as float64."""
    x = np.asarray(x, dtype=np.float64)
    mant, ex = np.frexp(x)                      # x = mant * 2^ex, 0.5 <= |mant| < 1
    return np.ldexp(np.rint(mant * 256.0) / 256.0, ex)


def bf16_bits_of(x: np.ndarray) -> np.ndarray:
    """float64 values already on the bf16 grid -> uint16 storage bits."""
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def load(t: np.ndarray, dtype: str) -> np.ndarray:
    """Stored tensor -> float64 values (bf16 arrive as uint16 bits, fp32 as float32)."""
    if dtype == "bf16":
        return decode_bf16(t)
    return np.asarray(t, dtype=np.float64)


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round a result to the storage format of the workload (values stay float64)."""
    return round_to_bf16(x) if dtype == "bf16" else np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# a1: CSA compression  ([P1] CSA step 1 and exercise 2; [P3]; [P4])
# ---------------------------------------------------------------------------

def csa_compress(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb=None, prev_Zb=None, first_entry=0, m=4):
    """Compress a chunk of T_new = n*m tokens that starts at token m*first_entry.

    Ca, Cb, Za, Zb: [T_new, d] float64; Ba, Bb: [m, d]; prev_Cb/prev_Zb: [m, d]
    b-series of the block before the chunk (ignored when first_entry == 0).
    Returns the n entries first_entry .. first_entry+n-1 as [n, d] float64.

    Entry i, component c:  softmax over the sources s of (Z_s,c + B_s,c), then
    sum of weight * C_s,c, where the sources are the b-series of block i-1 with
    biases Bb[0..m-1] and the a-series of block i with biases Ba[0..m-1].
    """
    T_new, d = Ca.shape
    assert T_new % m == 0
    n = T_new // m
    out = np.empty((n, d), dtype=np.float64)
    for j in range(n):
        a_C = Ca[j * m:(j + 1) * m]
        a_L = Za[j * m:(j + 1) * m] + Ba
        if j > 0:
            b_C = Cb[(j - 1) * m:j * m]
            b_L = Zb[(j - 1) * m:j * m] + Bb
        elif first_entry > 0:
            b_C = prev_Cb
            b_L = prev_Zb + Bb
        else:
            b_C = None
        if b_C is None:
            C_src, L_src = a_C, a_L
        else:
            C_src = np.concatenate([b_C, a_C], axis=0)
            L_src = np.concatenate([b_L, a_L], axis=0)
        M = L_src.max(axis=0)
        e = np.exp(L_src - M)
        out[j] = (e * C_src).sum(axis=0) / e.sum(axis=0)
    return out


# ---------------------------------------------------------------------------
# a2: HCA compression  ([P1] "HCA: сжать в 128 раз ..."; [P3])
# ---------------------------------------------------------------------------

def hca_compress(C, Z, bias, m_prime=128):
    """C, Z: [T_new, d] (T_new a multiple of m'), bias: [m', d] -> [T_new/m', d].

    Entry i: softmax over its m' tokens of (Z + bias[j]) per component, then the
    weighted sum of C; blocks do not overlap.
    """
    T_new, d = C.shape
    assert T_new % m_prime == 0
    n = T_new // m_prime
    out = np.empty((n, d), dtype=np.float64)
    for i in range(n):
        L = Z[i * m_prime:(i + 1) * m_prime] + bias
        M = L.max(axis=0)
        e = np.exp(L - M)
        out[i] = (e * C[i * m_prime:(i + 1) * m_prime]).sum(axis=0) / e.sum(axis=0)
    return out


# ---------------------------------------------------------------------------
# a3: lightning indexer  ([P1] CSA step 2 and "FP4 с учётом квантования"; [P3])
# ---------------------------------------------------------------------------

def _dots(qv, kv):
    """D[t, j, s] = sum_c qv[t, j, c] * kv[s, c] (a library float64 matmul)."""
    Tq, HI, dI = qv.shape
    return (qv.reshape(Tq * HI, dI) @ kv.T).reshape(Tq, HI, kv.shape[0])


def head_dots(q, k, fmt, q_scale=None, k_scale=None):
    """Per-head dot products D[t, j, s] = <q[t,j], k[s]> with dequantisation scales.

    fmt "f32":   q [Tq, H_I, d_I] float, k [N, d_I] float (no scales).
    fmt "e4m3":  q codes [Tq, H_I, d_I], q_scale [Tq, H_I]; k codes [N, d_I], k_scale [N].
                 D = sq * sk * sum_c q8*k8 (the integer-grid sum is exact in float64).
    fmt "mxfp4": q packed [Tq, H_I, d_I/2], q_scale ue8m0 [Tq, H_I, d_I/32]; k likewise.
                 D = sum over 32-blocks b of sq_b * sk_b * sum_{c in b} q4*k4.
    """
    if fmt == "f32":
        qv = np.asarray(q, dtype=np.float64)
        kv = np.asarray(k, dtype=np.float64)
        return _dots(qv, kv)
    if fmt == "e4m3":
        qv = decode_e4m3(q)
        kv = decode_e4m3(k)
        raw = _dots(qv, kv)                                    # exact: 43-bit span < 53
        return (np.asarray(q_scale, np.float64)[:, :, None]
                * np.asarray(k_scale, np.float64)[None, None, :]) * raw
    if fmt == "mxfp4":
        qv = decode_e2m1_packed(q)
        kv = decode_e2m1_packed(k)
        Tq, HI, dI = qv.shape
        N = kv.shape[0]
        nb = dI // 32
        qs = decode_ue8m0(q_scale)                             # [Tq, HI, nb]
        ks = decode_ue8m0(k_scale)                             # [N, nb]
        D = np.zeros((Tq, HI, N), dtype=np.float64)
        for b in range(nb):
            part = _dots(qv[:, :, 32 * b:32 * (b + 1)], kv[:, 32 * b:32 * (b + 1)])
            D += qs[:, :, b][:, :, None] * ks[:, b][None, None, :] * part
        return D
    raise ValueError(fmt)


def indexer_scores(q, w, k, fmt, q_scale=None, k_scale=None):
    """I[t, s] = sum_j w[t, j] * max(0, D[t, j, s]), heads summed in order j = 0..H_I-1."""
    D = head_dots(q, k, fmt, q_scale, k_scale)
    R = np.maximum(D, 0.0)
    w = np.asarray(w, dtype=np.float64)
    I = np.zeros((D.shape[0], D.shape[2]), dtype=np.float64)
    for j in range(D.shape[1]):
        I += w[:, j][:, None] * R[:, j, :]
    return I


def n_eligible(pos, m, n_entries):
    """Entries whose m source tokens are all <= pos: floor((pos+1)/m), capped at n_entries."""
    return min(int(n_entries), (int(pos) + 1) // m)


# ---------------------------------------------------------------------------
# indexer-key producer  ([P1] section "FP4 с учётом квантования": the indexer's
# Q·K activations are cached and multiplied in FP4, MXFP4 with 1x32 tiles; the
# keys of the compressed entries come from CSA step 1's gated pooling)
#
# Readings: the pooled value is quantised directly (no bf16 intermediate), and
# every quantisation decision is taken on that value as an fp32 number, the
# precision of the CUDA kernel: E4M3 scale = fp32(amax / 448) (1 for an
# all-zero row) and y = fp32(x / scale); MXFP4 exponent e = the smallest integer
# with amax <= 6 * 2^e over each 32-block (clamped to [-127, 127]; -127 for an
# all-zero block) and y = x * 2^-e.  Codes round y to the nearest grid value,
# ties to the even code, saturating at the largest finite value; a value that
# rounds to zero gets the +0 code.
# ---------------------------------------------------------------------------

def _encode_nearest(y, mags, sign_bit):
    """Codes of the grid values nearest to y; mags[c] is the magnitude of code c, increasing.

    Ties go to the even code; |y| beyond the last magnitude saturates to it."""
    a = np.minimum(np.abs(np.asarray(y, dtype=np.float64)), mags[-1])
    hi = np.clip(np.searchsorted(mags, a, side="left"), 0, len(mags) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo = a - mags[lo]
    dhi = mags[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.int64)
    neg = (np.asarray(y) < 0) & (code != 0)
    return (code | np.where(neg, sign_bit, 0)).astype(np.uint8)


E4M3_MAGS = E4M3[:0x7F].copy()        # codes 0x00..0x7E: 0 .. 448, increasing
E2M1_MAGS = E2M1[:8].copy()           # codes 0..7: 0, .5, 1, 1.5, 2, 3, 4, 6


def encode_e4m3(y):
    return _encode_nearest(y, E4M3_MAGS, 0x80)


def encode_e2m1(y):
    return _encode_nearest(y, E2M1_MAGS, 0x8)


def mx_exponent(amax):
    """Smallest integer e with amax <= 6 * 2^e (exact comparisons), clamped to [-127, 127];
    -127 for amax == 0."""
    amax = np.asarray(amax, dtype=np.float64)
    out = np.full(amax.shape, -127, dtype=np.int64)
    for idx in np.ndindex(amax.shape):
        a = float(amax[idx])
        if a == 0.0:
            continue
        e = math.frexp(a)[1] - 3                 # 6 * 2^e < a here
        while 6.0 * 2.0 ** e < a:
            e += 1
        out[idx] = min(max(e, -127), 127)
    return out


def quantise_index_keys(x, fmt):
    """Quantise pooled rows x [n, d] (float64) to the lightning indexer's key format.

    Returns (codes, scales, y): E4M3 -> codes uint8 [n, d], scales float32 [n];
    MXFP4 -> codes uint8 [n, d/2] (element 2i in the low nibble), scales ue8m0
    uint8 [n, d/32].  y is the pre-rounding value on the code grid (float64)."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    n, d = x32.shape
    if fmt == "e4m3":
        amax = np.abs(x32).max(axis=1)
        scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
        y = (x32 / scale[:, None]).astype(np.float32).astype(np.float64)
        return encode_e4m3(y), scale, y
    if fmt == "mxfp4":
        assert d % 32 == 0
        blk = x32.reshape(n, d // 32, 32).astype(np.float64)
        e = mx_exponent(np.abs(blk).max(axis=2))                        # [n, d/32]
        y = (blk * np.ldexp(1.0, -e)[:, :, None]).reshape(n, d)
        c = encode_e2m1(y)
        packed = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
        return packed, (e + 127).astype(np.uint8), y
    raise ValueError(fmt)


def index_key_compress(Ca, Cb, Za, Zb, Ba, Bb, fmt, prev_Cb=None, prev_Zb=None, first_entry=0, m=4):
    """Indexer keys of the entries a chunk completes: csa_compress of the indexer
    activations, then quantise_index_keys.  Returns (codes, scales, y, x)."""
    x = csa_compress(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, first_entry, m)
    codes, scales, y = quantise_index_keys(x, fmt)
    return codes, scales, y, x


# ---------------------------------------------------------------------------
# FP8 KV storage  ([P3] section "Гибридный attention: CSA и HCA": KV entries are
# stored in FP8, only the RoPE dimensions stay in BF16)
#
# Reading (the pages give no layout or scale): a 576-wide latent row is stored as
# 656 bytes: its first 512 values as e4m3 codes of x * 2^-e, the 64 RoPE values as
# bf16 (nearest even), then one byte e + 127 and 15 zero bytes.  e is the smallest
# integer with max|x[:512]| <= 448 * 2^e, clamped to [-126, 127]; a power of two,
# so every stored value times 2^e is exactly a bf16 value.  Decisions are taken on
# the row as fp32 values, as for the indexer keys.
# ---------------------------------------------------------------------------

KV8_ROW_BYTES = 656


def kv8_exponent(amax):
    """Smallest integer e with amax <= 448 * 2^e (exact comparisons), clamped to [-126, 127]."""
    amax = np.asarray(amax, dtype=np.float64)
    out = np.full(amax.shape, -126, dtype=np.int64)
    for idx in np.ndindex(amax.shape):
        a = float(amax[idx])
        if a == 0.0:
            continue
        e = math.frexp(a)[1] - 10                # 448 * 2^e < a here
        while 448.0 * 2.0 ** e < a:
            e += 1
        out[idx] = min(max(e, -126), 127)
    return out


def quantise_latent_fp8(x):
    """Rows x [n, 576] (float64) -> stored FP8 rows [n, 656] uint8."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    n = x32.shape[0]
    assert x32.shape[1] == 576
    nope = x32[:, :512].astype(np.float64)
    e = kv8_exponent(np.abs(nope).max(axis=1))
    codes = encode_e4m3(nope * np.ldexp(1.0, -e)[:, None])
    rope = bf16_bits_of(round_to_bf16(x32[:, 512:].astype(np.float64)))
    out = np.zeros((n, KV8_ROW_BYTES), dtype=np.uint8)
    out[:, :512] = codes
    out[:, 512:640] = rope.astype("<u2").view(np.uint8).reshape(n, 128)
    out[:, 640] = (e + 127).astype(np.uint8)
    return out


def dequantise_latent_fp8(rows8):
    """Stored FP8 rows [n, 656] -> the latent values [n, 576] they hold (float64, exact)."""
    rows8 = np.asarray(rows8, dtype=np.uint8)
    e = rows8[:, 640].astype(np.int64) - 127
    nope = decode_e4m3(rows8[:, :512]) * np.ldexp(1.0, e)[:, None]
    rope = decode_bf16(np.ascontiguousarray(rows8[:, 512:640]).view("<u2"))
    return np.concatenate([nope, rope], axis=1)


# ---------------------------------------------------------------------------
# grouped output projection  ([P1] CSA step 4: the head outputs are split into g
# groups, each group is projected to an intermediate width, and the concatenation is
# projected to the hidden size; table "Конфигурации": g = 16, width 1024, d = 7168)
# ---------------------------------------------------------------------------

def grouped_out_proj(o, W1, W2, g, dtype="bf16"):
    """o [T, H, dv], W1 [g*d_mid, (H/g)*dv], W2 [d, g*d_mid] (float64 values).

    Group j holds heads j*H/g .. (j+1)*H/g - 1; its outputs, concatenated in head order,
    are multiplied by rows j*d_mid .. (j+1)*d_mid - 1 of W1.  The intermediate u is stored
    (rounded to the storage format) before W2 reads it.  Returns (u, y), both stored."""
    T, H, dv = o.shape
    d_mid = W1.shape[0] // g
    hg = H // g
    u = np.empty((T, g * d_mid), dtype=np.float64)
    for j in range(g):
        xj = o[:, j * hg:(j + 1) * hg, :].reshape(T, hg * dv)
        u[:, j * d_mid:(j + 1) * d_mid] = xj @ W1[j * d_mid:(j + 1) * d_mid].T
    u = store(u, dtype)
    y = store(u @ W2.T, dtype)
    return u, y


# ---------------------------------------------------------------------------
# a4: top-k  ([P1] CSA step 2; k from table "Конфигурации")
# ---------------------------------------------------------------------------

def topk(scores_row, n_elig, k):
    """Indices of the k largest of scores_row[:n_elig], ties to the lower index,
    returned in ascending index order and padded with -1 to length k."""
    n_elig = int(n_elig)
    s = np.asarray(scores_row[:n_elig], dtype=np.float64)
    order = np.lexsort((np.arange(n_elig), -s))              # primary: -score, secondary: index
    sel = np.sort(order[:min(k, n_elig)])
    out = np.full(k, -1, dtype=np.int64)
    out[:sel.size] = sel
    return out


def topk_bf16(scores_row, n_elig, k):
    """Top-k over bf16 keys ([P1] "FP4 с учётом квантования": the indexer's scores are
    converted from FP32 to BF16 before the selection): each exact score rounded to the
    nearest bf16 value (ties to even), then topk over those keys, so scores closer than
    the bf16 resolution tie and the lower index wins."""
    return topk(round_to_bf16(np.asarray(scores_row[:int(n_elig)], dtype=np.float64)), n_elig, k)


# ---------------------------------------------------------------------------
# a5 / a6: attention over compressed entries + window + sink  ([P1] CSA step 3,
# HCA paragraph and sliding window; [P4] MLA latent, SWA, attention sink)
# ---------------------------------------------------------------------------

def attention(q, rows, sink, sm_scale, dv):
    """q: [H, d_k]; rows: [R, d_k] key rows (values = rows[:, :dv]); sink: [H].

    Returns (o [H, dv], lse [H]) with
    o_h = sum_r e^{l_r - M} v_r / (e^{sink_h - M} + sum_r e^{l_r - M}),
    l_r = sm_scale * <q_h, k_r>, M = max(sink_h, max_r l_r),
    lse_h = M + log(e^{sink_h - M} + sum_r e^{l_r - M}).
    """
    q = np.asarray(q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    sink = np.asarray(sink, dtype=np.float64)
    L = sm_scale * (q @ rows.T)                                  # [H, R]
    M = np.maximum(sink, L.max(axis=1) if L.shape[1] else -np.inf)
    P = np.exp(L - M[:, None])
    es = np.exp(sink - M)
    den = es + P.sum(axis=1)
    o = (P @ rows[:, :dv]) / den[:, None]
    lse = M + np.log(den)
    return o, lse


def window_range(pos, W):
    """Absolute positions of the raw window of the query at pos: [max(0,pos-W+1), pos]."""
    return max(0, pos - W + 1), pos + 1


# ---------------------------------------------------------------------------
# workload-level passes (compose the steps above)
# ---------------------------------------------------------------------------

def run_csa_prefill(wl, rows=None):
    """CSA prefill of Tq tokens (workloads 0 and 3).

    Returns dict(cache [N, d] float64 rows as stored, scores-free idx {t: [k]},
    out {t: [H, dv]}, lse {t: [H]}) for the query rows ``rows`` (default: all).
    """
    D = wl.dims
    t = wl.tensors
    dt = D["dtype"]; m = D["m"]; k = D["k"]; W = D["W"]
    e0 = D["entry0"]
    cache = load(t["cache"][0], dt).copy() if "cache" in t else np.zeros((D["N"], D["d"]))
    new = csa_compress(load(t["Ca"][0], dt), load(t["Cb"][0], dt), load(t["Za"][0], dt),
                       load(t["Zb"][0], dt), load(t["Ba"], "f32"), load(t["Bb"], "f32"),
                       load(t["prev_Cb"][0], dt), load(t["prev_Zb"][0], dt), e0, m)
    cache[e0:e0 + new.shape[0]] = store(new, dt)
    Tq = D["Tq"]
    rows = list(range(Tq)) if rows is None else list(rows)
    ifmt = D["ifmt"]
    qI = t["qI"][0][rows]
    w = t["w"][0][rows]
    if ifmt == "f32":
        I = indexer_scores(qI, w, t["kI"][0], "f32")
    else:
        I = indexer_scores(qI, w, t["kI"][0], ifmt, t["qI_scale"][0][rows], t["kI_scale"][0])
    raw = load(t["raw"][0], dt)
    q = t["q"][0]
    res = dict(cache=cache, idx={}, out={}, lse={}, scores={})
    for r_i, tq in enumerate(rows):
        pos = D["q_pos0"] + tq
        ne = n_eligible(pos, m, D["N"])
        sel = topk(I[r_i], ne, k)
        lo, hi = window_range(pos, W)
        win = raw[lo - D["raw_pos0"]:hi - D["raw_pos0"]]
        kv = np.concatenate([cache[sel[sel >= 0]], win], axis=0)
        o, lse = attention(load(q[tq], dt), kv, load(t["sink"], "f32"), D["sm_scale"], D["dv"])
        res["idx"][tq] = sel
        res["out"][tq] = o
        res["lse"][tq] = lse
        res["scores"][tq] = I[r_i]
    return res


def _window(t, D, b, p, dt):
    """The raw window rows of sequence b.  A decode token's own raw latent (raw_new, when the
    workload gives it) goes into its ring slot win_slot = position mod W; the window is a set
    of rows, so their order does not matter."""
    win = load(t[p + "win"][b], dt)
    if p + "raw_new" in t:
        win = win.copy()
        win[D["win_slot"]] = load(t[p + "raw_new"][b], dt)
    return win


def run_csa_decode(wl, batches=None, prefix=""):
    """CSA decode step (workload 1, CSA half of 4): compress the block completed
    by the current token into entry N-1, index, select top-k, attend."""
    D = wl.dims
    t = wl.tensors
    dt = D["dtype"]; m = D["m"]; k = D["k"]; N = D["N"]
    e0 = D["entry0"]
    pos = D["q_pos0"]
    batches = range(D["B"]) if batches is None else batches
    res = dict(entry={}, idx={}, out={}, lse={}, scores={})
    for b in batches:
        new = csa_compress(load(t["Ca"][b], dt), load(t["Cb"][b], dt), load(t["Za"][b], dt),
                           load(t["Zb"][b], dt), load(t["Ba"], "f32"), load(t["Bb"], "f32"),
                           load(t["prev_Cb"][b], dt), load(t["prev_Zb"][b], dt), e0, m)
        entry = store(new, dt)
        ifmt = D["ifmt"]
        kI_b, kIs_b = t["kI"][b], t["kI_scale"][b]
        if "CaI" in t:
            # the key of the fresh entry comes from the block's indexer activations
            codes, scales, _, _ = index_key_compress(
                load(t["CaI"][b], dt), load(t["CbI"][b], dt), load(t["ZaI"][b], dt), load(t["ZbI"][b], dt),
                load(t["BaI"], "f32"), load(t["BbI"], "f32"), ifmt, load(t["prev_CbI"][b], dt),
                load(t["prev_ZbI"][b], dt), e0, m)
            kI_b, kIs_b = kI_b.copy(), kIs_b.copy()
            kI_b[e0:e0 + codes.shape[0]] = codes
            kIs_b[e0:e0 + codes.shape[0]] = scales
        I = indexer_scores(t["qI"][b], t["w"][b], kI_b, ifmt, t["qI_scale"][b], kIs_b)[0]
        sel = topk(I, n_eligible(pos, m, N), k)
        cache_b = t["cache"][b]
        rows_sel = load(cache_b[np.clip(sel[sel >= 0], 0, N - 1)], dt)
        # entry e0 is the freshly compressed one
        for r_i, s in enumerate(sel[sel >= 0]):
            if e0 <= s < e0 + entry.shape[0]:
                rows_sel[r_i] = entry[s - e0]
        kv = np.concatenate([rows_sel, _window(t, D, b, "", dt)], axis=0)
        o, lse = attention(load(t["q"][b][0], dt), kv, load(t["sink"], "f32"), D["sm_scale"], D["dv"])
        res["entry"][b] = entry
        res["idx"][b] = sel
        res["out"][b] = o
        res["lse"][b] = lse
        res["scores"][b] = I
    return res


def run_hca_decode(wl, batches=None, prefix=""):
    """HCA decode step (workload 2, HCA half of 4): compress the fresh m'-token chunk
    into entry N-1, then dense attention over all N entries + window + sink."""
    D = wl.dims
    t = wl.tensors
    p = prefix
    dt = D["dtype"]
    N = D["Nh"] if p else D["N"]
    e0 = D["entry0_h"] if p else D["entry0"]
    mp = D["m_prime"]
    batches = range(D["B"]) if batches is None else batches
    res = dict(entry={}, out={}, lse={})
    for b in batches:
        new = hca_compress(load(t[p + "C"][b], dt), load(t[p + "Z"][b], dt), load(t[p + "bias"], "f32"), mp)
        entry = store(new, dt)
        cache = load(t[p + "cache"][b], dt).copy()
        cache[e0:e0 + entry.shape[0]] = entry
        kv = np.concatenate([cache[:N], _window(t, D, b, p, dt)], axis=0)
        o, lse = attention(load(t[p + "q"][b][0], dt), kv, load(t[p + "sink"], "f32"), D["sm_scale"], D["dv"])
        res["entry"][b] = entry
        res["out"][b] = o
        res["lse"][b] = lse
    return res
