"""The seeded input generator: determinism and the storage formats it writes."""
import numpy as np
import torch

import csa_inputs as CI
from oracle import csa_oracle as O


def test_deterministic():
    a = CI.make_workload(0)
    b = CI.make_workload(0)
    for k in a.tensors:
        assert np.array_equal(a.tensors[k], b.tensors[k]), k


def test_e4m3_rows_roundtrip():
    x = torch.randn(64, 128, generator=torch.Generator().manual_seed(3))
    codes, scale = CI.quant_e4m3_rows(x)
    v = O.decode_e4m3(codes) * scale[:, None]
    # every row uses the full range: its largest magnitude maps to 448
    assert np.all(np.abs(O.decode_e4m3(codes)).max(axis=1) == 448.0)
    # error within half an e4m3 ulp (relative 2^-4) of each value
    err = np.abs(v - x.numpy()) / np.maximum(np.abs(x.numpy()), 2.0 ** -6 * scale[:, None])
    assert err.max() <= 2.0 ** -4 + 1e-7


def test_mxfp4_rows_rne_and_scales():
    x = torch.tensor([[0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0] + [0.0] * 23 + [6.0]])
    packed, sc = CI.quant_mxfp4_rows(x)
    assert sc.tolist() == [[127]]                      # amax 6 -> scale 2^0
    v = O.decode_e2m1_packed(packed)
    assert v[0, :8].tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -4.0]   # ties to even codes
    y = torch.randn(16, 128, generator=torch.Generator().manual_seed(4)) * 3
    p, s = CI.quant_mxfp4_rows(y)
    deq = O.decode_e2m1_packed(p) * np.repeat(O.decode_ue8m0(s), 32, axis=-1)
    blk = y.numpy().reshape(16, 4, 32)
    amax = np.abs(blk).max(axis=-1)
    assert np.all(amax / O.decode_ue8m0(s) <= 6.0) and np.all(amax / O.decode_ue8m0(s) > 3.0)
    assert np.abs(deq - y.numpy()).max() <= (O.decode_ue8m0(s).max() * 1.0)


def test_workload_shapes_small():
    w = CI.make_workload(1, scale={"B": 2, "T": 4096})
    t, D = w.tensors, w.dims
    assert t["cache"].shape == (2, 1024, 576) and t["cache"].dtype == np.uint16
    assert t["kI"].shape == (2, 1024, 128) and t["kI_scale"].shape == (2, 1024)
    assert D["entry0"] == 1023 and D["q_pos0"] == 4095
    w4 = CI.make_workload(4, scale={"B": 1, "T": 8192})
    assert w4.tensors["kI"].shape == (1, 2048, 64) and w4.tensors["kI_scale"].shape == (1, 2048, 4)


def test_fp8_latent_rows_of_the_generator_match_the_oracle_format():
    """The generator's FP8 cache rows (torch casts) equal the oracle's own quantiser (its
    e4m3 encoder and exponent search) on rows of widely different magnitudes."""
    import torch
    from oracle import csa_oracle as O
    g = torch.Generator().manual_seed(5)
    x = torch.randn(64, 576, generator=g) * torch.exp(torch.randn(64, 1, generator=g) * 4)
    x[9] = 0.0
    assert np.array_equal(CI.quant_latent_fp8_rows(x), O.quantise_latent_fp8(x.double().numpy()))


def test_added_generators_are_seeded_and_shaped():
    a = CI.index_key_inputs(3, 2, 8, 128, "bf16", spread=4.0)
    b = CI.index_key_inputs(3, 2, 8, 128, "bf16", spread=4.0)
    assert all(np.array_equal(a[k], b[k]) for k in a)
    assert a["Ca"].shape == (2, 8, 128) and a["Ca"].dtype == np.uint16
    assert a["prev_Cb"].shape == (2, 4, 128) and a["Ba"].shape == (4, 128) and a["Ba"].dtype == np.float32
    c = CI.index_key_inputs(4, 2, 8, 128, "bf16")
    assert not np.array_equal(a["Ca"], c["Ca"])
    x = CI.out_proj_inputs(5, 3, H=8, dv=16, g=4, d_mid=128, d=256)
    assert x["o"].shape == (3, 8, 16) and x["W1"].shape == (512, 32) and x["W2"].shape == (256, 512)
    y = CI.out_proj_inputs(5, 3, H=8, dv=16, g=4, d_mid=128, d=256)
    assert all(np.array_equal(x[k], y[k]) for k in x)


def test_row_quantisers_of_the_generator_match_the_oracle():
    """The generator's E4M3 and MXFP4 row quantisers (torch casts, its own e2m1 rounding)
    and the oracle's key quantiser (its own nearest-grid encoders and exponent search)
    agree on the same fp32 rows, up to the sign of a value that rounds to zero."""
    import torch
    from oracle import csa_oracle as O
    g = torch.Generator().manual_seed(8)
    x = torch.randn(40, 128, generator=g) * torch.exp(torch.randn(40, 1, generator=g) * 3)
    x[3] = 0.0
    c_gen, s_gen = CI.quant_e4m3_rows(x)
    c_orc, s_orc, _ = O.quantise_index_keys(x.double().numpy(), "e4m3")
    assert np.array_equal(s_gen, s_orc)
    assert np.array_equal(np.where(c_gen == 0x80, 0, c_gen), c_orc)
    p_gen, e_gen = CI.quant_mxfp4_rows(x)
    p_orc, e_orc, _ = O.quantise_index_keys(x.double().numpy(), "mxfp4")
    assert np.array_equal(e_gen, e_orc)
    lo, hi = p_gen & 0xF, p_gen >> 4
    lo = np.where(lo == 0x8, 0, lo)
    hi = np.where(hi == 0x8, 0, hi)
    assert np.array_equal((lo | (hi << 4)).astype(np.uint8), p_orc)
