"""GPU parity of the indexer-key producer (index_key_compress) against the fp64 oracle.

[P1] "Техотчёт DeepSeek-V4 (2026)", section "FP4 с учётом квантования": the indexer's
Q·K activations are cached in FP4 (MXFP4, 1x32 tiles); the keys of the compressed
entries are the CSA step-1 pooling of those activations, quantised.

Codes are bytes, so they must match exactly, with one allowance that the arithmetic
forces: the kernel pools in fp32 and the oracle in fp64, so a pooled value that lies
within the fp32 pooling error of a rounding midpoint may land on either neighbour.  A
mismatch is accepted only for adjacent codes whose midpoint is that close to the
oracle's pre-rounding value; the same holds for an MXFP4 block whose maximum sits that
close to a power-of-two boundary of its exponent.  Scales of E4M3 rows match to the
same relative error.
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

FMT = {"e4m3": 1, "mxfp4": 2}
POOL_REL = 4e-6          # fp32 pooling error bound, relative to the largest source magnitude


def _dev(a, dtype):
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def _src_max(t, dtype, b, j, first_entry):
    """Largest |C| over the 8 sources of chunk entry j of sequence b, per component."""
    ld = lambda x: O.load(x, dtype)
    a = np.abs(ld(t["Ca"][b, 4 * j:4 * j + 4])).max(axis=0)
    if j > 0:
        return np.maximum(a, np.abs(ld(t["Cb"][b, 4 * j - 4:4 * j])).max(axis=0))
    if first_entry > 0:
        return np.maximum(a, np.abs(ld(t["prev_Cb"][b])).max(axis=0))
    return a


def run_case(t, entry0, n_max, fmt, dtype, d_I):
    B, T_new, _ = t["Ca"].shape
    n = T_new // 4
    dv = {k: _dev(v, dtype if k not in ("Ba", "Bb") else "f32") for k, v in t.items()}
    e0 = torch.tensor(entry0, dtype=torch.int32, device="cuda")
    width = d_I if fmt == "e4m3" else d_I // 2
    kI = torch.full((B, n_max, width), 0xAB, dtype=torch.uint8, device="cuda")
    ks = (torch.full((B, n_max), -3.0, dtype=torch.float32, device="cuda") if fmt == "e4m3"
          else torch.full((B, n_max, d_I // 32), 0xAB, dtype=torch.uint8, device="cuda"))
    csa.index_key_compress(dv["Ca"], dv["Cb"], dv["Za"], dv["Zb"], dv["Ba"], dv["Bb"], dv["prev_Cb"], dv["prev_Zb"],
                           e0, kI, ks, FMT[fmt])
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    g_codes, g_scales = kI.cpu().numpy(), ks.cpu().numpy()
    flips = 0
    for b in range(B):
        ld = lambda x: O.load(x, dtype)
        codes, scales, y, x = O.index_key_compress(ld(t["Ca"][b]), ld(t["Cb"][b]), ld(t["Za"][b]), ld(t["Zb"][b]),
                                                   t["Ba"].astype(np.float64), t["Bb"].astype(np.float64), fmt,
                                                   ld(t["prev_Cb"][b]), ld(t["prev_Zb"][b]), entry0[b])
        rows = slice(entry0[b], entry0[b] + n)
        tol_x = np.stack([POOL_REL * _src_max(t, dtype, b, j, entry0[b]) for j in range(n)])   # [n, d_I]
        flips += compare_keys(g_codes[b, rows], g_scales[b, rows], codes, scales, y, x, tol_x, fmt)
        # rows outside the chunk keep their contents
        keep = np.ones(n_max, bool)
        keep[rows] = False
        assert np.all(g_codes[b, keep] == 0xAB)
        assert np.all(g_scales[b, keep] == (-3.0 if fmt == "e4m3" else 0xAB))
    assert flips <= 1e-3 * B * n * d_I, flips           # midpoint cases stay rare
    return flips


def _unpack(c, fmt):
    if fmt == "e4m3":
        return c.astype(np.int64)
    out = np.empty(c.shape[:-1] + (2 * c.shape[-1],), np.int64)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def compare_keys(gc, gs, oc, os_, y, x, tol_x, fmt):
    """Exact codes, except adjacent codes around a midpoint within the pooling error."""
    n, d = x.shape
    mags = O.E4M3_MAGS if fmt == "e4m3" else O.E2M1_MAGS
    sign = 0x80 if fmt == "e4m3" else 0x8
    g = _unpack(gc, fmt)
    o = _unpack(oc, fmt)
    if fmt == "e4m3":
        s = os_.astype(np.float64)
        # the row maximum carries the same relative error into the scale
        assert np.allclose(gs, os_, rtol=1e-5, atol=0), np.abs(gs / os_ - 1).max()
        tol_y = tol_x / s[:, None] + 1e-5 * np.abs(y)
        live = np.ones_like(g, bool)
    else:
        e = os_.astype(np.int64) - 127
        ge = gs.astype(np.int64) - 127
        live = np.repeat(ge == e, 32, axis=1)
        if not live.all():
            # a different exponent only where the oracle's block maximum is that close to
            # a boundary 6 * 2^e of the exponent search
            amax = np.abs(x.astype(np.float32).astype(np.float64)).reshape(n, d // 32, 32).max(axis=2)
            tol_a = tol_x.reshape(n, d // 32, 32).max(axis=2)
            bad = ge != e
            near = (np.abs(amax - 6.0 * np.ldexp(1.0, e)) <= tol_a) | (np.abs(amax - 6.0 * np.ldexp(1.0, e - 1)) <= tol_a)
            assert np.all(near[bad]), "MX exponent differs away from a boundary"
        tol_y = tol_x * np.ldexp(1.0, -np.repeat(e, 32, axis=1))
    mism = (g != o) & live
    if mism.any():
        gm, om = g[mism] & ~sign, o[mism] & ~sign
        ym, tm = y[mism], tol_y[mism]
        assert np.all(np.abs(gm - om) == 1), "codes more than one step apart"
        mid = (mags[gm] + mags[om]) / 2
        assert np.all(np.abs(np.abs(ym) - mid) <= tm), "a code differs away from a rounding midpoint"
    # where the magnitude is non-zero, the GPU's sign is the value's sign
    nz = ((g & ~sign) > 0) & live & (np.abs(y) > tol_y)
    assert np.all(((g & sign) != 0)[nz] == (y < 0)[nz])
    # a value that rounds to zero is stored as +0
    assert not np.any(g == sign)
    return int(mism.sum()) + int((~live).sum())


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
def test_decode_append_one_entry_per_sequence(fmt):
    """The decode step: each of 16 sequences completes one entry; entry 0 (no b-half), the
    last cache row and rows in between."""
    B, n_max = 16, 64
    t = CI.index_key_inputs(41, B, 4, 128, "bf16")
    entry0 = [0, 1, 63, 17, 2, 30, 31, 32, 5, 6, 62, 40, 41, 3, 9, 12]
    run_case(t, entry0, n_max, fmt, "bf16", 128)


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
def test_prefill_chunk_with_wide_magnitude_spread(fmt):
    """A 4096-token chunk (1024 entries: several CTAs and a ragged grid) appended after
    8192 entries, and one from the start of a sequence; token magnitudes over 2^+-12,
    so the MX exponents cover a wide range."""
    t = CI.index_key_inputs(42, 2, 4096, 128, "bf16", spread=12.0)
    flips = run_case(t, [8192, 0], 8192 + 1024, fmt, "bf16", 128)
    assert flips <= 8


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
@pytest.mark.parametrize("d_I,dtype", [(32, "f32"), (64, "f32"), (128, "f32"), (64, "bf16"), (256, "bf16")])
def test_other_widths_and_fp32_inputs(fmt, d_I, dtype):
    t = CI.index_key_inputs(43 + d_I, 3, 36, d_I, dtype)
    run_case(t, [0, 4, 100], 109, fmt, dtype, d_I)


@pytest.mark.parametrize("fmt", ["e4m3", "mxfp4"])
def test_zero_and_on_grid_entries_are_exact(fmt):
    """An all-zero entry gives code 0 with the zero-row scale; entries whose sources carry
    one constant row that sits on the code grid come back as exactly those codes."""
    d, n = 128, 4
    t = CI.index_key_inputs(44, 1, 4 * n, d, "f32")
    r = np.random.default_rng(9)
    if fmt == "e4m3":
        grid = O.E4M3_MAGS[r.integers(1, 126, size=(n, d))] * np.where(r.random((n, d)) < 0.5, -1, 1)
        grid[:, 5] = 448.0
    else:
        # block maxima 32 = 4 * 2^3, away from the exponent boundaries 24 and 48
        grid = 8.0 * O.E2M1_MAGS[r.integers(0, 7, size=(n, d))] * np.where(r.random((n, d)) < 0.5, -1, 1)
        grid[:, ::32] = -32.0
    grid[2] = 0.0
    rows = np.repeat(grid, 4, axis=0).astype(np.float32)          # token 4i+j carries row i
    t["Ca"] = rows[None]
    t["Cb"] = np.concatenate([rows[4:], rows[:4]])[None]          # b-series of block i-1 carries row i
    t["prev_Cb"] = rows[None, :4]
    flips = run_case(t, [7], 16, fmt, "f32", d)
    assert flips == 0


def test_out_of_range_entry_is_flagged_not_written():
    """entry0 beyond the cache: the kernel skips the rows and sets the entry error bit."""
    t = CI.index_key_inputs(45, 2, 8, 128, "bf16")
    dv = {k: _dev(v, "bf16" if k not in ("Ba", "Bb") else "f32") for k, v in t.items()}
    kI = torch.full((2, 16, 128), 0xAB, dtype=torch.uint8, device="cuda")
    ks = torch.full((2, 16), -3.0, dtype=torch.float32, device="cuda")
    e0 = torch.tensor([15, 3], dtype=torch.int32, device="cuda")        # row 16 of sequence 0 is outside
    csa.index_key_compress(dv["Ca"], dv["Cb"], dv["Za"], dv["Zb"], dv["Ba"], dv["Bb"], dv["prev_Cb"], dv["prev_Zb"],
                           e0, kI, ks, FMT["e4m3"])
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0x10
    g = kI.cpu().numpy()
    assert np.all(g[0, :15] == 0xAB) and not np.all(g[0, 15] == 0xAB)   # entry 15 written, 16 skipped
    assert not np.all(g[1, 3:5] == 0xAB)
