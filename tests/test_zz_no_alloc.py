"""sparse_attn_decode_noalloc: the decode attention for callers that cannot allocate
device memory (code inside another framework's memory pool, latency-critical paths
that must never call cudaMalloc).  It must give the same results as
sparse_attn_decode with a caller workspace, call after call, although every call
reuses the library's one fixed scratch buffer.

This file is collected last so that, if it fails, a run stopping at the first
failure has already run every other test.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import pytest
import torch

import csa_inputs as CI

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_sparse_long_csa_b200 as csa
    from compressed_sparse_long_csa_b200 import _native as N
    from compressed_sparse_long_csa_b200 import steps


def _close(g, ref):
    """The tolerance of the parity tests (bf16 outputs): max-abs 2e-2, mean-rel 2e-3."""
    g = g.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g))
    assert err.max() <= 2e-2, err.max()
    assert err.sum() / max(np.abs(ref).sum(), 1e-30) <= 2e-3


def _call_noalloc(T, D, idx, out, lse):
    """Call the entry point through the C ABI directly."""
    q = T["q"][:, 0]
    B, H, d_k = q.shape
    st = N.lib.sparse_attn_decode_noalloc(
        q.data_ptr(), T["cache"].data_ptr(), idx.data_ptr(), T["win"].data_ptr(), T["win_len"].data_ptr(),
        T["sink"].data_ptr(), B, H, d_k, D["dv"], T["cache"].shape[1], idx.shape[1], T["win"].shape[1],
        C.c_float(D["sm_scale"]), N.CSA_BF16, out.data_ptr(), lse.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == 0, N.lib.csa_status_string(st)


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    wl = CI.make_workload(1, scale={"B": 3, "T": 8192})         # 3 x 640 rows: several KV splits
    D = wl.dims
    T = steps.upload(wl)
    B, H, dv = D["B"], D["H"], D["dv"]
    assert N.lib.attn_decode_workspace_size(B, H, dv, D["k"] + D["W"]) <= N.NOALLOC_SCRATCH_BYTES
    rng = np.random.default_rng(3)
    for call in range(2):
        # a different selection each call: stale partials from the last call must not leak in
        idx = torch.from_numpy(np.stack([np.sort(rng.choice(D["N"], D["k"], replace=False)) for _ in range(B)])
                               .astype(np.int32)).cuda()
        ref_out = torch.empty(B, H, dv, dtype=torch.bfloat16, device="cuda")
        ref_lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
        csa.sparse_attn_decode(T["q"][:, 0], T["cache"], idx, T["win"], T["win_len"], T["sink"], D["sm_scale"], dv,
                               ref_out, ref_lse, T["aws"])
        out = torch.full((B, H, dv), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        _call_noalloc(T, D, idx, out, lse)
        torch.cuda.synchronize()
        _close(out, ref_out)
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=2e-3, rtol=0)
    assert csa.read_device_error() == 0


def test_noalloc_rejects_requests_beyond_its_buffer():
    # 200 sequences of 128 heads need more partials than the fixed buffer holds:
    # the call is refused on the host before any device work.
    need = N.lib.attn_decode_workspace_size(200, 128, 512, 640)
    assert need > N.NOALLOC_SCRATCH_BYTES
    st = N.lib.sparse_attn_decode_noalloc(None, None, None, None, None, None, 200, 128, 576, 512, 16384, 512, 128,
                                          C.c_float(0.04), N.CSA_BF16, None, None, None)
    assert st == 6            # CSA_ERR_WORKSPACE
