"""GPU: the dense MMA rate probe used for the scoring kernels' tensor rooflines runs at
both indexer formats without a device error, and its rate lies between a tenth of the
nominal dense figure and 1.5 times it (a probe far above the nominal figure would not be
doing the work it counts)."""
from __future__ import annotations

import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import compressed_sparse_long_csa_b200 as csa


@pytest.mark.parametrize("fmt,n,nominal", [("e4m3", 256, 4500.0), ("mxfp4", 64, 9000.0)])
def test_tensor_peak_probe_rate(fmt, n, nominal):
    ifmt = csa.CSA_IFMT_E4M3 if fmt == "e4m3" else csa.CSA_IFMT_MXFP4
    iters = 2000
    csa.tensor_peak_probe(ifmt, 10)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    csa.tensor_peak_probe(ifmt, iters)
    e1.record()
    torch.cuda.synchronize()
    assert csa.read_device_error() == 0
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tflops = 2.0 * 128 * n * 128 * iters * sms / (e0.elapsed_time(e1) * 1e-3) / 1e12
    print(f"{fmt}: {tflops:.0f} TFLOP/s")
    assert nominal / 10 < tflops < 1.5 * nominal


def test_tensor_peak_probe_rejects_bad_arguments():
    with pytest.raises(csa.CsaError):
        csa.tensor_peak_probe(csa.CSA_IFMT_F32, 10)
    with pytest.raises(csa.CsaError):
        csa.tensor_peak_probe(csa.CSA_IFMT_E4M3, 0)
