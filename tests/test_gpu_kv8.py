"""GPU parity of the FP8 KV cache calls (sparse_attn_decode_kv8, hca_attn_decode_kv8).

[P3] aixai.ru digest, section "Гибридный attention: CSA и HCA": KV entries are stored in
FP8 and only the RoPE dimensions in BF16.  The stored row is exactly codes * 2^e followed
by the bf16 RoPE values, so (1) the FP8 call must return exactly what the bf16 call
returns on a bf16 cache holding those decoded rows, and (2) both must match the fp64
oracle's attention over the decoded rows within the bf16 output tolerances.
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


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _check(g, o, what):
    g = np.asarray(g, np.float64)
    o = O.store(np.asarray(o, np.float64), "bf16")
    err = np.abs(g - o)
    assert np.all(np.isfinite(g)), what
    assert err.max() <= 2e-2, (what, err.max())
    assert err.sum() / np.abs(o).sum() <= 2e-3, (what, err.sum() / np.abs(o).sum())


def _kv8_cache(wl, key="cache"):
    x = torch.from_numpy(O.decode_bf16(wl.tensors[key]).astype(np.float32))
    c8 = CI.quant_latent_fp8_rows(x)                                    # [B, N, 656]
    deq = O.dequantise_latent_fp8(c8.reshape(-1, 656)).reshape(c8.shape[0], c8.shape[1], 576)
    return c8, deq


@pytest.mark.parametrize("B,T,k", [(4, 65536, 512), (3, 8192, 1024)])
def test_sparse_decode_kv8(B, T, k):
    wl = CI.make_workload(1, scale={"B": B, "T": T, "k": k})
    D = wl.dims
    N, H, dv, W = D["N"], D["H"], D["dv"], D["W"]
    c8, deq = _kv8_cache(wl)
    r = np.random.default_rng(B * 7 + k)
    idx = np.stack([np.sort(r.choice(N, size=k, replace=False)) for _ in range(B)]).astype(np.int32)
    idx[0, -37:] = -1                                                   # unused slots
    idx[1, 5] = 0                                                       # entry 0
    win_len = np.array([W, 1, 77, 128][:B], np.int32)
    q, win, sink = _bf16_dev(wl.tensors["q"][:, 0]), _bf16_dev(wl.tensors["win"]), torch.from_numpy(wl.tensors["sink"]).cuda()
    ws = torch.empty(csa.attn_decode_workspace_size(B, H, dv, k + W), dtype=torch.uint8, device="cuda")
    idx_d, wl_d = torch.from_numpy(idx).cuda(), torch.from_numpy(win_len).cuda()
    out8 = torch.empty(B, H, dv, dtype=torch.bfloat16, device="cuda")
    csa.sparse_attn_decode_kv8(q, torch.from_numpy(c8).cuda(), idx_d, win, wl_d, sink, D["sm_scale"], dv, out8,
                               workspace=ws)
    # the bf16 call on a bf16 cache holding the decoded rows
    cache16 = torch.from_numpy(deq.astype(np.float32)).to(torch.bfloat16).cuda()
    out16 = torch.empty_like(out8)
    csa.sparse_attn_decode(q, cache16, idx_d, win, wl_d, sink, D["sm_scale"], dv, out16, workspace=ws)
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    assert torch.equal(out8, out16)
    qn = O.decode_bf16(wl.tensors["q"][:, 0])
    winn = O.decode_bf16(wl.tensors["win"])
    for b in range(B):
        sel = idx[b][idx[b] >= 0]
        rows = np.concatenate([deq[b][sel], winn[b][:win_len[b]]], axis=0)
        o, _ = O.attention(qn[b], rows, wl.tensors["sink"].astype(np.float64), D["sm_scale"], dv)
        _check(out8[b].float().cpu().numpy(), o, f"kv8 sparse b={b}")


@pytest.mark.parametrize("B,T", [(2, 1 << 20), (3, 1 << 17)])
def test_hca_decode_kv8(B, T):
    wl = CI.make_workload(2, scale={"B": B, "T": T})
    D = wl.dims
    N, H, dv, W = D["N"], D["H"], D["dv"], D["W"]
    c8, deq = _kv8_cache(wl)
    n_entries = np.array([N, N - 77, 1][:B], np.int32)                  # ragged, down to one entry
    win_len = np.array([W, 13, 0][:B], np.int32)
    q, win, sink = _bf16_dev(wl.tensors["q"][:, 0]), _bf16_dev(wl.tensors["win"]), torch.from_numpy(wl.tensors["sink"]).cuda()
    ws = torch.empty(csa.attn_decode_workspace_size(B, H, dv, N + W), dtype=torch.uint8, device="cuda")
    ne_d, wl_d = torch.from_numpy(n_entries).cuda(), torch.from_numpy(win_len).cuda()
    out8 = torch.empty(B, H, dv, dtype=torch.bfloat16, device="cuda")
    csa.hca_attn_decode_kv8(q, torch.from_numpy(c8).cuda(), ne_d, win, wl_d, sink, D["sm_scale"], dv, out8,
                            workspace=ws)
    cache16 = torch.from_numpy(deq.astype(np.float32)).to(torch.bfloat16).cuda()
    out16 = torch.empty_like(out8)
    csa.hca_attn_decode(q, cache16, ne_d, win, wl_d, sink, D["sm_scale"], dv, out16, workspace=ws)
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    assert torch.equal(out8, out16)
    qn = O.decode_bf16(wl.tensors["q"][:, 0])
    winn = O.decode_bf16(wl.tensors["win"])
    for b in range(B):
        rows = np.concatenate([deq[b][:n_entries[b]], winn[b][:win_len[b]]], axis=0)
        o, _ = O.attention(qn[b], rows, wl.tensors["sink"].astype(np.float64), D["sm_scale"], dv)
        _check(out8[b].float().cpu().numpy(), o, f"kv8 dense b={b}")


# ----------------------------------------------------------------------------- the FP8 writer

def _compare_rows(g8, o8, x, tol_x):
    """Stored bytes must match, except where the fp32 pooling error (tol_x per component)
    can carry a value across a rounding midpoint (codes, bf16 RoPE) or the row maximum
    across an exponent boundary 448 * 2^e."""
    x32 = x.astype(np.float32).astype(np.float64)
    ge, oe = g8[:, 640].astype(np.int64) - 127, o8[:, 640].astype(np.int64) - 127
    assert not g8[:, 641:].any()
    amax = np.abs(x32[:, :512]).max(axis=1)
    tol_a = tol_x[:, :512].max(axis=1)
    bad = ge != oe
    near = (np.abs(amax - 448.0 * np.ldexp(1.0, oe)) <= tol_a) | (np.abs(amax - 448.0 * np.ldexp(1.0, oe - 1)) <= tol_a)
    assert np.all(near[bad]), "row exponent differs away from a boundary"
    flips = int(bad.sum()) * 512
    ok = ~bad
    gc, oc = g8[ok, :512].astype(np.int64), o8[ok, :512].astype(np.int64)
    mism = gc != oc
    if mism.any():
        y = x32[ok, :512] * np.ldexp(1.0, -oe[ok])[:, None]
        ty = tol_x[ok, :512] * np.ldexp(1.0, -oe[ok])[:, None]
        gm, om = gc[mism] & 0x7F, oc[mism] & 0x7F
        assert np.all(np.abs(gm - om) == 1), "codes more than one step apart"
        mid = (O.E4M3_MAGS[gm] + O.E4M3_MAGS[om]) / 2
        assert np.all(np.abs(np.abs(y[mism]) - mid) <= ty[mism]), "a code differs away from a midpoint"
        flips += int(mism.sum())
    gr = O.decode_bf16(np.ascontiguousarray(g8[:, 512:640]).view("<u2"))
    orr = O.decode_bf16(np.ascontiguousarray(o8[:, 512:640]).view("<u2"))
    rm = gr != orr
    if rm.any():
        mid = (gr[rm] + orr[rm]) / 2
        assert np.all(np.abs(x32[:, 512:][rm] - mid) <= tol_x[:, 512:][rm]), "a RoPE value differs away from a midpoint"
        flips += int(rm.sum())
    return flips


@pytest.mark.parametrize("B,T_new,entry0,dtype", [
    (16, 4, [0, 1, 63, 17, 2, 30, 31, 32, 5, 6, 62, 40, 41, 3, 9, 12], "bf16"),   # the decode append
    (2, 1024, [8192, 0], "bf16"),                                               # a chunk of 256 entries
    (3, 36, [0, 4, 100], "f32"),
])
def test_csa_compress_kv8(B, T_new, entry0, dtype):
    n = T_new // 4
    n_max = max(entry0) + n
    t = CI.index_key_inputs(61 + B, B, T_new, 576, dtype, spread=4.0)
    dev = {k: (torch.from_numpy(np.ascontiguousarray(v)).cuda() if v.dtype == np.float32
               else _bf16_dev(v)) for k, v in t.items()}
    c8 = torch.full((B, n_max, 656), 0xAB, dtype=torch.uint8, device="cuda")
    e0 = torch.tensor(entry0, dtype=torch.int32, device="cuda")
    csa.csa_compress_kv8(dev["Ca"], dev["Cb"], dev["Za"], dev["Zb"], dev["Ba"], dev["Bb"], dev["prev_Cb"],
                         dev["prev_Zb"], e0, c8)
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    g = c8.cpu().numpy()
    flips = 0
    for b in range(B):
        ld = lambda a: O.load(a, dtype)
        x = O.csa_compress(ld(t["Ca"][b]), ld(t["Cb"][b]), ld(t["Za"][b]), ld(t["Zb"][b]),
                           t["Ba"].astype(np.float64), t["Bb"].astype(np.float64), ld(t["prev_Cb"][b]),
                           ld(t["prev_Zb"][b]), entry0[b])
        srcmax = []
        for j in range(n):
            a = np.abs(ld(t["Ca"][b, 4 * j:4 * j + 4])).max(axis=0)
            if j > 0:
                a = np.maximum(a, np.abs(ld(t["Cb"][b, 4 * j - 4:4 * j])).max(axis=0))
            elif entry0[b] > 0:
                a = np.maximum(a, np.abs(ld(t["prev_Cb"][b])).max(axis=0))
            srcmax.append(a)
        tol_x = 4e-6 * np.stack(srcmax)
        rows = slice(entry0[b], entry0[b] + n)
        flips += _compare_rows(g[b, rows], O.quantise_latent_fp8(x), x, tol_x)
        keep = np.ones(n_max, bool)
        keep[rows] = False
        assert np.all(g[b, keep] == 0xAB)
    assert flips <= 1e-3 * B * n * 576, flips
