"""GPU: a device-side wait that cannot end gives up with an error status.

Every kernel of the library waits on CTA-local mbarriers with a time limit.  The probe
kernel waits on a barrier that nothing completes, with a 1 ms limit: the wait must give
up, the error word must carry CSA_DEVERR_TIMEOUT, and the context must stay usable (a
following attention call is correct and raises no error).  No copy or MMA is in flight
in the probe, so nothing is left running when it returns.
"""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import csa_inputs as CI
from oracle import csa_oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_sparse_long_csa_b200 as csa
    from compressed_sparse_long_csa_b200 import steps

CSA_DEVERR_TIMEOUT = 0x4


def test_wait_that_cannot_end_times_out_and_the_device_stays_usable():
    csa.read_device_error()                                  # start from a clear word
    t0 = time.perf_counter()
    csa.wait_probe(1_000_000)                               # 1 ms limit
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert csa.read_device_error() & CSA_DEVERR_TIMEOUT
    assert dt < 1.0                                          # it gave up, it did not hang
    # a normal call afterwards: correct, and no error raised
    wl = CI.make_workload(1, scale={"B": 2, "T": 4096, "k": 64})
    D = wl.dims
    T = steps.upload(wl)
    idx = torch.arange(64, dtype=torch.int32, device="cuda").repeat(2, 1)
    csa.sparse_attn_decode(T["q"][:, 0], T["cache"], idx, T["win"], T["win_len"], T["sink"], D["sm_scale"], D["dv"],
                           T["out"][:, 0], T["lse"][:, 0], T["aws"])
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    cache, win = O.decode_bf16(wl.tensors["cache"]), O.decode_bf16(wl.tensors["win"])
    for b in range(2):
        o, _ = O.attention(O.decode_bf16(wl.tensors["q"][b, 0]), np.concatenate([cache[b][:64], win[b]]),
                           wl.tensors["sink"].astype(np.float64), D["sm_scale"], D["dv"])
        g = T["out"][b, 0].float().cpu().numpy()
        assert np.abs(g - o).max() <= 2e-2


def test_wait_probe_rejects_limits_out_of_range():
    with pytest.raises(csa.CsaError):
        csa.wait_probe(10)                                   # below 1 us
    with pytest.raises(csa.CsaError):
        csa.wait_probe(5_000_000_000)                        # above the library's 2 s
