"""Host logic of bench.py: the algorithmic bytes and FLOPs that the roofline divides by.

The per-step figures are derived in the scope table's measurement section from the
workloads' shapes (decode: every byte of the indexer keys, the selected or all cache rows,
the window, the query and the output once; prefill: the FP8 indexer and bf16 attention
contractions over the eligible pairs); bench.py's accounting must reproduce them.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

COMMON = dict(d=576, dk=576, dv=512, H=128, HI=64, dI=128, W=128, m=4, m_prime=128)


def test_decode_64k_bytes_per_step():
    D = dict(COMMON, B=16, T=65536, N=16384, n_max=16384, k=512, ifmt="e4m3")
    ab = bench.algorithmic_bytes(1, D)
    # 16 x (2.16 MB keys + 0.59 MB rows + 0.15 MB window + 0.28 MB q/out) ~ 51.0 MB
    assert sum(ab.values()) == pytest.approx(51.0e6, rel=0.02)
    assert ab["indexer"] == pytest.approx(16 * 16384 * 132, rel=0.01)


def test_hca_decode_1m_bytes_per_step():
    D = dict(COMMON, B=4, T=1 << 20, N=8192, n_max=8192)
    ab = bench.algorithmic_bytes(2, D)
    # 4 x (9.44 MB cache + 0.29 MB chunk + 0.15 MB window + 0.28 MB q/out) ~ 40.9 MB
    assert sum(ab.values()) == pytest.approx(40.9e6, rel=0.02)


def test_hybrid_pair_bytes_per_step():
    D = dict(COMMON, B=8, T=1 << 20, N=262144, n_max=262144, Nh=8192, k=1024, ifmt="mxfp4")
    ab = bench.algorithmic_bytes(4, D)
    # 8 x (19.4 MB CSA + 9.9 MB HCA) ~ 234 MB; the MXFP4 keys are 64 + 4 bytes per entry
    assert sum(ab.values()) == pytest.approx(234e6, rel=0.02)
    assert ab["indexer"] == pytest.approx(8 * 262144 * 68, rel=0.01)


def test_prefill_flops():
    ctx, Tq = 131072, 4096
    D = dict(COMMON, B=1, T=ctx + Tq, Tq=Tq, N=(ctx + Tq) // 4, n_max=(ctx + Tq) // 4, k=1024, ifmt="e4m3",
             q_pos0=ctx)
    fl = bench.algorithmic_flops(3, D)
    # eligible pairs sum_p floor((p+1)/4) = 136.3 M; x 2 x 64 heads x 128 = 2.23 TFLOP (FP8)
    assert fl["indexer"] == pytest.approx(2.23e12, rel=0.01)
    # 4096 queries x 128 heads x (1024 + 128) rows x 2 x (576 + 512) = 1.31 TFLOP (bf16)
    assert fl["attention"] == pytest.approx(1.31e12, rel=0.01)
