"""GPU: csa_decode_append (one launch for a decode token's cache entry, indexer key and
window-ring row) gives bit for bit what the separate calls give: csa_compress of the
block, index_key_compress of the block's indexer activations, and a copy of the raw
latent into ring slot win_slot.  window_append alone does the last part.  Expected values
come from the library's own separate calls (same arithmetic) and from the inputs."""
from __future__ import annotations

import pytest
import torch

import csa_inputs as CI

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_sparse_long_csa_b200 as csa
    from compressed_sparse_long_csa_b200 import steps


@pytest.mark.parametrize("wid,sc", [(1, {"B": 3, "T": 8192}), (4, {"B": 2, "T": 65536})])
def test_fused_append_equals_separate_calls(wid, sc):
    wl = CI.make_workload(wid, scale=sc)
    D = wl.dims
    T = steps.upload(wl)
    fmt = steps._ifmt(D)
    cache0, kI0, ks0, win0 = T["cache"].clone(), T["kI"].clone(), T["kI_scale"].clone(), T["win"].clone()
    # the separate calls on copies
    cache_s, kI_s, ks_s = cache0.clone(), kI0.clone(), ks0.clone()
    csa.csa_compress(T["Ca"], T["Cb"], T["Za"], T["Zb"], T["Ba"], T["Bb"], T["prev_Cb"], T["prev_Zb"], T["entry0"],
                     cache_s, m=4)
    csa.index_key_compress(T["CaI"], T["CbI"], T["ZaI"], T["ZbI"], T["BaI"], T["BbI"], T["prev_CbI"], T["prev_ZbI"],
                           T["entry0"], kI_s, ks_s, fmt)
    # the fused call
    steps._decode_append(T, D, None)
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    assert torch.equal(T["cache"], cache_s)
    assert torch.equal(T["kI"], kI_s)
    assert torch.equal(T["kI_scale"], ks_s)
    slot = D["win_slot"]
    win_exp = win0.clone()
    win_exp[:, slot] = T["raw_new"]
    assert torch.equal(T["win"], win_exp)
    # the key really changed (the workload's row was stale)
    assert not torch.equal(T["kI"], kI0)


def test_window_append_and_a_bad_slot_is_flagged():
    g = torch.Generator().manual_seed(3)
    B, W, d = 3, 16, 576
    win = torch.randn(B, W, d, generator=g).to(torch.bfloat16).cuda()
    new = torch.randn(B, d, generator=g).to(torch.bfloat16).cuda()
    slot = torch.tensor([0, 15, 7], dtype=torch.int32, device="cuda")
    exp = win.clone()
    exp[torch.arange(B), slot.long()] = new
    csa.window_append(new, win, slot)
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    assert torch.equal(win, exp)
    bad = torch.tensor([0, 16, -1], dtype=torch.int32, device="cuda")
    before = win.clone()
    csa.window_append(new, win, bad)
    torch.cuda.synchronize()
    assert csa.read_device_error() & 0x2                      # CSA_DEVERR_WINDOW
    assert torch.equal(win[1:], before[1:])                   # the bad slots were skipped
