"""GPU parity of the grouped output projection (grouped_out_proj) against the fp64 oracle.

[P1] "Техотчёт DeepSeek-V4 (2026)", section "Гибридное внимание: CSA и HCA", CSA step 4,
and table "Конфигурации" (g = 16 groups, intermediate width 1024, head size 512, d = 7168).
Both outputs are bf16: max-abs <= 2e-2 and mean-rel <= 2e-3 against the oracle's values
rounded to bf16, as for the attention outputs.
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


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _close(g, o, what):
    g = np.asarray(g, np.float64)
    err = np.abs(g - o)
    assert np.all(np.isfinite(g)), what
    assert err.max() <= 2e-2, (what, err.max())
    assert err.sum() / np.abs(o).sum() <= 2e-3, (what, err.sum() / np.abs(o).sum())


CASES = {
    # name: (T, H, dv, g, d_mid, d, use workspace)
    "pro_decode_16": (16, 128, 512, 16, 1024, 7168, True),
    "pro_decode_16_no_split": (16, 128, 512, 16, 1024, 7168, False),
    "flash_decode_5": (5, 64, 512, 8, 1024, 4096, True),
    "one_token": (1, 128, 512, 16, 1024, 1024, True),
    "ragged_300_tokens": (300, 128, 64, 16, 128, 1024, True),
    "prefill_1100_tokens": (1100, 32, 128, 4, 256, 512, True),
}


@pytest.mark.parametrize("case", list(CASES))
def test_grouped_out_proj(case):
    T, H, dv, g, d_mid, d, use_ws = CASES[case]
    x = CI.out_proj_inputs(31, T, H, dv, g, d_mid, d)
    o, W1, W2 = _dev(x["o"]), _dev(x["W1"]), _dev(x["W2"])
    u = torch.full((T, g * d_mid), 7.0, dtype=torch.bfloat16, device="cuda")
    y = torch.full((T, d), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = None
    if use_ws:
        nb = csa.grouped_out_proj_workspace_size(T, g, d_mid, d)
        ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    csa.grouped_out_proj(o, W1, W2, g, u, y, ws)
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    ou, oy = O.grouped_out_proj(O.decode_bf16(x["o"]), O.decode_bf16(x["W1"]), O.decode_bf16(x["W2"]), g)
    _close(u.float().cpu().numpy(), ou, "u")
    _close(y.float().cpu().numpy(), oy, "y")


def test_grouped_out_proj_is_deterministic():
    T, H, dv, g, d_mid, d = 16, 128, 512, 16, 1024, 2048
    x = CI.out_proj_inputs(32, T, H, dv, g, d_mid, d)
    o, W1, W2 = _dev(x["o"]), _dev(x["W1"]), _dev(x["W2"])
    ws = torch.empty(csa.grouped_out_proj_workspace_size(T, g, d_mid, d), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        u = torch.empty((T, g * d_mid), dtype=torch.bfloat16, device="cuda")
        y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
        csa.grouped_out_proj(o, W1, W2, g, u, y, ws)
        outs.append(y.clone())
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
