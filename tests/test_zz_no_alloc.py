"""sparse_attn_decode_noalloc: the decode attention for callers that cannot allocate
device memory (code inside another framework's memory pool, latency-critical paths
that must never call cudaMalloc).  It must give the same results as
sparse_attn_decode with a caller workspace, call after call, although every call
reuses the library's one fixed scratch buffer: both run the same deterministic
kernels on the same inputs, so the results must be bit-for-bit equal (a stale partial
left in the shared buffer by an earlier call would change low bits).

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


def _call_noalloc(q, cache, idx, win, win_len, sink, sm_scale, dv, out, lse):
    """Call the entry point through the C ABI directly."""
    B, H, d_k = q.shape
    dtype = N.CSA_BF16 if q.dtype == torch.bfloat16 else N.CSA_F32
    st = N.lib.sparse_attn_decode_noalloc(
        q.data_ptr(), cache.data_ptr(), idx.data_ptr(), win.data_ptr(), win_len.data_ptr(), sink.data_ptr(),
        B, H, d_k, dv, cache.shape[1], idx.shape[1], win.shape[1], C.c_float(sm_scale), dtype, out.data_ptr(),
        lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, N.lib.csa_status_string(st)


def _bf16_inputs():
    wl = CI.make_workload(1, scale={"B": 3, "T": 8192})         # 3 x 640 rows: several KV splits
    D = wl.dims
    T = steps.upload(wl)
    return dict(q=T["q"][:, 0], cache=T["cache"], win=T["win"], win_len=T["win_len"], sink=T["sink"],
                sm_scale=D["sm_scale"], dv=D["dv"], N=D["N"], k=D["k"], aws=T["aws"])


def _fp32_inputs():
    """The CUDA-core path: fp32 storage, 4 heads of width 64 (the tiny workload's shape)."""
    g = torch.Generator().manual_seed(21)
    B, H, d, N, k, W = 3, 4, 64, 256, 24, 16
    f = lambda *s: torch.randn(*s, generator=g).cuda()
    return dict(q=f(B, H, d), cache=f(B, N, d), win=f(B, W, d), win_len=torch.full((B,), W, dtype=torch.int32).cuda(),
                sink=f(H), sm_scale=1 / 8.0, dv=d, N=N, k=k,
                aws=torch.empty(max(1, N_ws(B, H, d, k + W)), dtype=torch.uint8, device="cuda"))


def N_ws(B, H, dv, rows):
    return N.lib.attn_decode_workspace_size(B, H, dv, rows)


@pytest.mark.parametrize("case", ["bf16_full", "bf16_pads_ragged_window", "fp32_cuda_core"])
def test_noalloc_equals_workspace_entry_point_on_consecutive_calls(case):
    x = _fp32_inputs() if case == "fp32_cuda_core" else _bf16_inputs()
    q, B, H, dv, k = x["q"], x["q"].shape[0], x["q"].shape[1], x["dv"], x["k"]
    assert N_ws(B, H, dv, k + x["win"].shape[1]) <= N.NOALLOC_SCRATCH_BYTES
    if case == "bf16_pads_ragged_window":
        x["win_len"] = torch.tensor([128, 5, 0], dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(3)
    for call in range(2):
        # a different selection each call: stale partials from the last call must not leak in
        idx = np.stack([np.sort(rng.choice(x["N"], k, replace=False)) for _ in range(B)]).astype(np.int32)
        if case == "bf16_pads_ragged_window":
            idx[0, 300 + 50 * call:] = -1
            idx[1, :] = -1
        idx = torch.from_numpy(idx).cuda()
        ref_out = torch.empty(B, H, dv, dtype=q.dtype, device="cuda")
        ref_lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
        csa.sparse_attn_decode(q, x["cache"], idx, x["win"], x["win_len"], x["sink"], x["sm_scale"], dv,
                               ref_out, ref_lse, x["aws"])
        out = torch.full((B, H, dv), float("nan"), dtype=q.dtype, device="cuda")
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _call_noalloc(q, x["cache"], idx, x["win"], x["win_len"], x["sink"], x["sm_scale"], dv, out, lse)
        torch.cuda.synchronize()
        if call > 0:
            # the first call may load the module that holds the fixed buffer; later calls
            # take no device memory
            assert torch.cuda.mem_get_info()[0] == free_before
        assert torch.equal(out, ref_out), call
        assert torch.equal(lse, ref_lse), call
    assert csa.read_device_error() == 0


def test_noalloc_rejects_requests_beyond_its_buffer():
    # 200 sequences of 128 heads need more partials than the fixed buffer holds:
    # the call is refused on the host before any device work.
    need = N.lib.attn_decode_workspace_size(200, 128, 512, 640)
    assert need > N.NOALLOC_SCRATCH_BYTES
    st = N.lib.sparse_attn_decode_noalloc(None, None, None, None, None, None, 200, 128, 576, 512, 16384, 512, 128,
                                          C.c_float(0.04), N.CSA_BF16, None, None, None)
    assert st == 6            # CSA_ERR_WORKSPACE
