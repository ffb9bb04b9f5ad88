"""Seeded synthetic workloads for the CSA / HCA attention hot path.

This module is shared by the fp64 oracle and by the CUDA path, and it holds none
of the method's arithmetic: it only draws random numbers and stores them in the
number formats the method consumes (bf16, fp32, FP8 e4m3 with a per-row fp32
scale, MXFP4 = e2m1 with a ue8m0 scale per 32 elements).  Every tensor is
returned as a host numpy array holding the raw storage bits:

* fp32 -> ``float32``; bf16 -> ``uint16`` bit patterns; e4m3 -> ``uint8`` codes;
* MXFP4 values -> ``uint8`` with two e2m1 codes per byte (element 2i in the low
  nibble, 2i+1 in the high nibble); ue8m0 scales -> ``uint8`` biased exponents.

The workloads follow the shapes and distributions of the DeepSeek-V4 technical
report digest ("Техотчёт DeepSeek-V4 (2026)", section "Гибридное внимание: CSA и
HCA" and table "Конфигурации"): m = 4, m' = 128, a 128-token window, top-k 512
or 1024, 128 query heads with a 576-wide MLA latent (512 content + 64 RoPE
dims), 64 indexer heads of width 128.  The five named workloads are:

0. ``tiny_prefill_fp32``  – 256-token CSA prefill in fp32 (d = 64, 4 heads).
1. ``csa_decode_64k``     – CSA decode, batch 16, 65,536-token context, FP8 indexer.
2. ``hca_decode_1m``      – HCA decode, batch 4, 1,048,576-token context.
3. ``csa_prefill_4k``     – CSA prefill of 4,096 tokens after a 131,072-token context.
4. ``hybrid_pair_1m``     – one CSA layer (MXFP4 indexer) + one HCA layer, batch 8, 1M context.

Random draws use ``torch.Generator`` on the CPU (seeded, deterministic across
machines for a given torch version); rounding to bf16 / e4m3 uses torch's own
round-to-nearest-even casts; e2m1 rounding is written out below.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

__all__ = [
    "WORKLOADS", "make_workload", "Workload",
    "bf16_bits", "fp32", "quant_e4m3_rows", "quant_mxfp4_rows", "index_key_inputs", "out_proj_inputs", "quant_latent_fp8_rows",
]

# --------------------------------------------------------------------------
# storage-format helpers (input preparation only)
# --------------------------------------------------------------------------

def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """fp32 tensor -> bf16 storage bits (uint16), round-to-nearest-even."""
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def fp32(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float32).numpy().copy()


def quant_e4m3_rows(x: torch.Tensor):
    """Quantise the last axis of ``x`` to FP8 e4m3 with one fp32 scale per row.

    scale = amax(|row|) / 448 (1 for an all-zero row); codes = RNE(row / scale)
    saturated to +-448.  Returns (codes uint8 [..., d], scale float32 [...]).
    """
    x = x.to(torch.float32)
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp(-448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.numpy().copy(), scale.numpy().astype(np.float32).copy()


def quant_latent_fp8_rows(x: torch.Tensor) -> np.ndarray:
    """576-wide latent rows -> 656-byte FP8 rows: bytes 0..511 the e4m3 codes (torch's
    round-to-nearest-even cast, +0 for values that round to zero) of x[:512] / 2^e with e
    the smallest integer such that max|x[:512]| <= 448 * 2^e (clamped to [-126, 127]);
    bytes 512..639 x[512:] as bf16 (little endian); byte 640 = e + 127; the rest zero."""
    x = x.to(torch.float32)
    lead = x.shape[:-1]
    nope = x[..., :512]
    amax = nope.abs().amax(dim=-1)
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.full_like(amax, -126.0))
    e = torch.where((amax > 0) & (amax > 448.0 * torch.exp2(e)), e + 1, e)
    e = torch.where((amax > 0) & (amax <= 448.0 * torch.exp2(e - 1)), e - 1, e)
    e = e.clamp(-126, 127)
    codes = (nope / torch.exp2(e).unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    codes = torch.where(codes == 0x80, torch.zeros_like(codes), codes)
    out = torch.zeros(*lead, 656, dtype=torch.uint8)
    out[..., :512] = codes
    rope = x[..., 512:].to(torch.bfloat16).contiguous().view(torch.uint8)
    out[..., 512:640] = rope.reshape(*lead, 128)
    out[..., 640] = (e + 127).to(torch.uint8)
    return out.numpy()


def _e2m1_rne_codes(y: torch.Tensor) -> torch.Tensor:
    """|y| <= 6 -> e2m1 code (sign in bit 3, magnitude code 0..7 for the grid
    0, .5, 1, 1.5, 2, 3, 4, 6), round to nearest with ties to the even code.

    The midpoints between grid neighbours are .25 .75 1.25 1.75 2.5 3.5 5; at a
    midpoint the even code wins, so the comparison is strict ('>') where the lower
    neighbour is even and inclusive ('>=') where the upper neighbour is even.
    """
    a = y.abs()
    mag = ((a > 0.25).to(torch.uint8) + (a >= 0.75).to(torch.uint8) + (a > 1.25).to(torch.uint8)
           + (a >= 1.75).to(torch.uint8) + (a > 2.5).to(torch.uint8) + (a >= 3.5).to(torch.uint8)
           + (a > 5.0).to(torch.uint8))
    sign = ((y < 0) & (mag > 0)).to(torch.uint8) << 3
    return mag | sign


def quant_mxfp4_rows(x: torch.Tensor):
    """Quantise the last axis (a multiple of 32) to MXFP4.

    Per 32-element block: scale = 2^ceil(log2(amax/6)) stored as a ue8m0 biased
    exponent (127 + e); values = e2m1 RNE(x / scale).  Returns
    (packed uint8 [..., d/2], scales uint8 [..., d/32]).
    """
    x = x.to(torch.float32)
    d = x.shape[-1]
    assert d % 32 == 0
    blk = x.reshape(*x.shape[:-1], d // 32, 32)
    amax = blk.abs().amax(dim=-1)
    e = torch.where(amax > 0, torch.ceil(torch.log2(amax / 6.0)), torch.full_like(amax, -127.0))
    # guard against log2 rounding: make sure amax / 2^e <= 6
    e = torch.where((amax > 0) & (amax / torch.exp2(e) > 6.0), e + 1, e)
    e = e.clamp(-127, 127)
    y = blk / torch.exp2(e).unsqueeze(-1)
    codes = _e2m1_rne_codes(y).reshape(*x.shape[:-1], d)
    lo = codes[..., 0::2]
    hi = codes[..., 1::2]
    packed = (lo | (hi << 4)).to(torch.uint8)
    scales = (e + 127).to(torch.uint8)
    return packed.numpy().copy(), scales.numpy().copy()


# --------------------------------------------------------------------------
# workload descriptions
# --------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    kind: str                      # "csa_prefill" | "csa_decode" | "hca_decode" | "hybrid_pair"
    dims: dict
    tensors: dict = field(default_factory=dict)


WORKLOADS = {
    0: "tiny_prefill_fp32",
    1: "csa_decode_64k",
    2: "hca_decode_1m",
    3: "csa_prefill_4k",
    4: "hybrid_pair_1m",
}


class _Rng:
    def __init__(self, seed: int):
        self.g = torch.Generator().manual_seed(seed)

    def normal(self, shape, std=1.0):
        return torch.randn(*shape, generator=self.g, dtype=torch.float32) * std

    def uniform(self, shape):
        return torch.rand(*shape, generator=self.g, dtype=torch.float32)


def _csa_compressor_inputs(r: _Rng, B, T_new, d, m, gate_std, to_store):
    t = {}
    t["Ca"] = to_store(r.normal((B, T_new, d)))
    t["Cb"] = to_store(r.normal((B, T_new, d)))
    t["Za"] = to_store(r.normal((B, T_new, d), gate_std))
    t["Zb"] = to_store(r.normal((B, T_new, d), gate_std))
    t["prev_Cb"] = to_store(r.normal((B, m, d)))
    t["prev_Zb"] = to_store(r.normal((B, m, d), gate_std))
    t["Ba"] = fp32(r.normal((m, d), 0.1))
    t["Bb"] = fp32(r.normal((m, d), 0.1))
    return t


def _decode_fresh_inputs(r: _Rng, t: dict, dims: dict, B: int, dI: int, d: int, m: int, W: int, ifmt: str):
    """What a decode token brings besides its query (drawn after every other tensor, so the
    rest of the workload is unchanged): the indexer activations of the block it completes
    (CaI .. prev_ZbI ~ N(0, 1), gates ~ N(0, 2), biases BaI, BbI ~ N(0, 0.1)), from which
    the key of the fresh entry is produced in the step, and its raw latent raw_new ~ N(0, 1),
    which the step writes into the window ring at slot q_pos0 mod W.  The workload's kI row
    of the fresh entry and win row of that slot are stale inputs the step overwrites."""
    ki = _csa_compressor_inputs(r, B, m, dI, m, 2.0, bf16_bits)
    for k, v in ki.items():
        t[k + "I"] = v
    t["raw_new"] = bf16_bits(r.normal((B, d)))
    dims["win_slot"] = dims["q_pos0"] % W
    dims["key_fmt"] = ifmt


def index_key_inputs(seed: int, B: int, T_new: int, d_I: int = 128, dtype: str = "bf16",
                     gate_std: float = 2.0, spread: float = 0.0) -> dict:
    """Indexer activations and gates for the indexer-key producer (the CSA pooling with
    m = 4 over width d_I): Ca, Cb, prev_Cb ~ N(0, 1) times a per-token magnitude
    2^u, u ~ U(-spread, spread) (spread = 0: plain N(0, 1)); Za, Zb, prev_Zb ~ N(0,
    gate_std); Ba, Bb ~ N(0, 0.1) fp32.  Stored as bf16 bits or fp32 (``dtype``)."""
    r = _Rng(seed)
    to_store = bf16_bits if dtype == "bf16" else fp32
    t = _csa_compressor_inputs(r, B, T_new, d_I, 4, gate_std, lambda x: x)
    if spread > 0:
        for name in ("Ca", "Cb", "prev_Cb"):
            x = t[name]
            t[name] = x * torch.exp2((r.uniform(x.shape[:-1] + (1,)) * 2 - 1) * spread)
    return {k: (to_store(v) if isinstance(v, torch.Tensor) else v) for k, v in t.items()}


def out_proj_inputs(seed: int, T: int, H: int = 128, dv: int = 512, g: int = 16, d_mid: int = 1024,
                    d: int = 7168) -> dict:
    """Inputs of the grouped output projection, stored as bf16 bits: head outputs
    o [T, H, dv] ~ N(0, 1), W1 [g*d_mid, (H/g)*dv] ~ N(0, 1/((H/g)*dv)) and
    W2 [d, g*d_mid] ~ N(0, 1/(g*d_mid)) (random initialisation of that scale keeps the
    outputs near unit size)."""
    r = _Rng(seed)
    k1, k2 = (H // g) * dv, g * d_mid
    return {"o": bf16_bits(r.normal((T, H, dv))),
            "W1": bf16_bits(r.normal((g * d_mid, k1), 1.0 / math.sqrt(k1))),
            "W2": bf16_bits(r.normal((d, k2), 1.0 / math.sqrt(k2)))}


def make_workload(i: int, seed: int | None = None, scale: dict | None = None) -> Workload:
    """Build workload ``i`` (0..4) with the given seed (default: seed = i).

    ``scale`` may override size entries (for example ``{"B": 2, "T": 8192}``)
    to produce the same structure at a size the oracle finishes quickly; the
    structure (which token completes a block, window length, k) is kept.
    """
    seed = i if seed is None else seed
    sc = dict(scale or {})
    r = _Rng(seed)
    if i == 0:
        n = sc.get("T", 256); d = 64; H = 4; HI = 2; dI = 32; k = sc.get("k", 8); W = 16; m = 4
        assert n % m == 0
        N = n // m
        dims = dict(B=1, T=n, Tq=n, N=N, n_max=N, d=d, dk=d, dv=d, H=H, HI=HI, dI=dI, k=k, W=W,
                    m=m, sm_scale=1.0 / math.sqrt(d), dtype="f32", ifmt="f32", q_pos0=0,
                    raw_pos0=0, entry0=0)
        t = _csa_compressor_inputs(r, 1, n, d, m, 1.0, fp32)
        t["q"] = fp32(r.normal((1, n, H, d)))
        t["qI"] = fp32(r.normal((1, n, HI, dI)))
        t["w"] = fp32(r.uniform((1, n, HI)))
        t["kI"] = fp32(r.normal((1, N, dI)))
        t["raw"] = fp32(r.normal((1, n, d)))
        t["sink"] = fp32(r.normal((H,)))
        return Workload(WORKLOADS[0], "csa_prefill", dims, t)

    if i == 1:
        B = sc.get("B", 16); T = sc.get("T", 65536); k = sc.get("k", 512)
        d = 576; dv = 512; H = 128; HI = 64; dI = 128; W = 128; m = 4
        N = T // m
        dims = dict(B=B, T=T, Tq=1, N=N, n_max=N, d=d, dk=d, dv=dv, H=H, HI=HI, dI=dI, k=k, W=W,
                    m=m, sm_scale=1.0 / math.sqrt(d), dtype="bf16", ifmt="e4m3",
                    q_pos0=T - 1, entry0=N - 1)
        # the current token (position T-1) completes block N-1: compress its 4 tokens
        t = _csa_compressor_inputs(r, B, m, d, m, 2.0, bf16_bits)
        cache = r.normal((B, N, d))
        t["cache"] = bf16_bits(cache)          # entry N-1 is overwritten by the compressor
        t["q"] = bf16_bits(r.normal((B, 1, H, d)))
        t["win"] = bf16_bits(r.normal((B, W, d)))
        t["qI"], t["qI_scale"] = quant_e4m3_rows(r.normal((B, 1, HI, dI)))
        t["kI"], t["kI_scale"] = quant_e4m3_rows(r.normal((B, N, dI)))
        t["w"] = fp32(r.uniform((B, 1, HI)))
        t["sink"] = fp32(r.normal((H,)))
        _decode_fresh_inputs(r, t, dims, B, dI, d, m, W, "e4m3")
        return Workload(WORKLOADS[1], "csa_decode", dims, t)

    if i == 2:
        B = sc.get("B", 4); T = sc.get("T", 1 << 20)
        d = 576; dv = 512; H = 128; W = 128; mp = 128
        N = T // mp
        dims = dict(B=B, T=T, Tq=1, N=N, n_max=N, d=d, dk=d, dv=dv, H=H, W=W, m_prime=mp,
                    sm_scale=1.0 / math.sqrt(d), dtype="bf16", q_pos0=T - 1, entry0=N - 1)
        t = {}
        t["cache"] = bf16_bits(r.normal((B, N, d)))   # entry N-1 comes from the fresh chunk
        t["C"] = bf16_bits(r.normal((B, mp, d)))
        t["Z"] = bf16_bits(r.normal((B, mp, d), 2.0))
        t["bias"] = fp32(r.normal((mp, d), 0.1))
        t["q"] = bf16_bits(r.normal((B, 1, H, d)))
        t["win"] = bf16_bits(r.normal((B, W, d)))
        t["sink"] = fp32(r.normal((H,)))
        t["raw_new"] = bf16_bits(r.normal((B, d)))
        dims["win_slot"] = (T - 1) % W
        return Workload(WORKLOADS[2], "hca_decode", dims, t)

    if i == 3:
        B = 1; ctx = sc.get("ctx", 131072); Tq = sc.get("Tq", 4096); k = sc.get("k", 1024)
        d = 576; dv = 512; H = 128; HI = 64; dI = 128; W = 128; m = 4
        T = ctx + Tq
        assert ctx % m == 0 and Tq % m == 0
        N = T // m; N0 = ctx // m
        raw_pos0 = max(0, ctx - (W - 1))
        dims = dict(B=B, T=T, Tq=Tq, N=N, n_max=N, d=d, dk=d, dv=dv, H=H, HI=HI, dI=dI, k=k, W=W,
                    m=m, sm_scale=1.0 / math.sqrt(d), dtype="bf16", ifmt="e4m3",
                    q_pos0=ctx, raw_pos0=raw_pos0, entry0=N0, ctx=ctx)
        t = _csa_compressor_inputs(r, B, Tq, d, m, 1.0, bf16_bits)
        t["cache"] = bf16_bits(r.normal((B, N, d)))   # entries N0.. come from the compressor
        t["kI"], t["kI_scale"] = quant_e4m3_rows(r.normal((B, N, dI)))
        t["qI"], t["qI_scale"] = quant_e4m3_rows(r.normal((B, Tq, HI, dI)))
        t["w"] = fp32(r.uniform((B, Tq, HI)))
        t["q"] = bf16_bits(r.normal((B, Tq, H, d)))
        t["raw"] = bf16_bits(r.normal((B, T - raw_pos0, d)))
        t["sink"] = fp32(r.normal((H,)))
        return Workload(WORKLOADS[3], "csa_prefill", dims, t)

    if i == 4:
        B = sc.get("B", 8); T = sc.get("T", 1 << 20); k = sc.get("k", 1024)
        d = 576; dv = 512; H = 128; HI = 64; dI = 128; W = 128; m = 4; mp = 128
        N = T // m; Nh = T // mp
        dims = dict(B=B, T=T, Tq=1, N=N, n_max=N, Nh=Nh, d=d, dk=d, dv=dv, H=H, HI=HI, dI=dI,
                    k=k, W=W, m=m, m_prime=mp, sm_scale=1.0 / math.sqrt(d), dtype="bf16",
                    ifmt="mxfp4", q_pos0=T - 1, entry0=N - 1, entry0_h=Nh - 1)
        t = _csa_compressor_inputs(r, B, m, d, m, 2.0, bf16_bits)
        t["cache"] = bf16_bits(r.normal((B, N, d)))
        t["q"] = bf16_bits(r.normal((B, 1, H, d)))
        t["win"] = bf16_bits(r.normal((B, W, d)))
        t["qI"], t["qI_scale"] = quant_mxfp4_rows(r.normal((B, 1, HI, dI)))
        t["kI"], t["kI_scale"] = quant_mxfp4_rows(r.normal((B, N, dI)))
        t["w"] = fp32(r.uniform((B, 1, HI)))
        t["sink"] = fp32(r.normal((H,)))
        # HCA layer of the pair
        t["h_cache"] = bf16_bits(r.normal((B, Nh, d)))
        t["h_C"] = bf16_bits(r.normal((B, mp, d)))
        t["h_Z"] = bf16_bits(r.normal((B, mp, d), 2.0))
        t["h_bias"] = fp32(r.normal((mp, d), 0.1))
        t["h_q"] = bf16_bits(r.normal((B, 1, H, d)))
        t["h_win"] = bf16_bits(r.normal((B, W, d)))
        t["h_sink"] = fp32(r.normal((H,)))
        _decode_fresh_inputs(r, t, dims, B, dI, d, m, W, "mxfp4")
        t["h_raw_new"] = bf16_bits(r.normal((B, d)))
        return Workload(WORKLOADS[4], "hybrid_pair", dims, t)

    raise ValueError(f"unknown workload {i}")
