"""Host-only checks of the C ABI: the library loads, exports every declared entry
point, and rejects invalid arguments with the documented status codes before any
device work (these calls never reach a kernel, so they run without a GPU)."""
import ctypes as C
import os
import re

import pytest

import compressed_sparse_long_csa_b200 as csa
from compressed_sparse_long_csa_b200 import _native as N

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "csa.h")
OK, ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_UNSUP, ERR_WS, ERR_CUDA = range(8)


def declared_functions():
    src = open(HDR).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\**\s+\**([a-z_0-9]+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert {"csa_compress", "hca_compress", "lightning_index", "topk_select", "sparse_attn_decode",
            "sparse_attn_prefill", "hca_attn_decode", "hca_compress_attn_decode", "index_key_compress",
            "lightning_index_bf16", "grouped_out_proj", "sparse_attn_decode_kv8",
            "hca_attn_decode_kv8", "csa_compress_kv8", "shard_topk_merge", "attn_merge_shards"} <= set(names)
    for n in names:
        assert hasattr(N.lib, n), n


def test_header_is_plain_c(tmp_path):
    """The boundary is a C ABI: the header compiles as C99 with no C++ in it."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "h.c"
    src.write_text('#include "%s"\nint main(void) { return csa_abi_version() > 0 ? 0 : 1; }\n' % HDR)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_program_links_every_declared_call(tmp_path):
    """A plain C program that takes the address of every declared call links against the
    shared library and runs (csa_abi_version is host-only, so no GPU is needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(csa.lib_path)
    names = declared_functions()
    src = tmp_path / "link.c"
    src.write_text('#include "%s"\nint main(void) {\n  const void* f[] = {%s};\n'
                   '  unsigned i;\n  for (i = 0; i < sizeof f / sizeof f[0]; ++i) if (!f[i]) return 2;\n'
                   '  return csa_abi_version() == %d ? 0 : 1;\n}\n'
                   % (HDR, ", ".join("(const void*)%s" % n for n in names), N.lib.csa_abi_version()))
    exe = tmp_path / "link"
    r = subprocess.run([cc, "-std=c99", str(src), "-o", str(exe), "-L" + libdir, "-lcsa_b200",
                        "-Wl,--allow-shlib-undefined", "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0


def test_launch_counter_is_host_side_and_ignores_refused_calls():
    before = N.lib.csa_launch_count()
    assert N.lib.topk_select(None, 100, None, 4, 100, 8, FAKE, None, 0, None) == ERR_NULL
    assert N.lib.csa_launch_count() == before


def test_version_and_strings():
    assert N.lib.csa_abi_version() == 1
    for s in range(8):
        assert N.lib.csa_status_string(s).startswith(b"CSA_")


FAKE = 1 << 20          # a 16-byte aligned non-null address that is never dereferenced on the host


def compress(**kw):
    args = dict(Ca=FAKE, Cb=FAKE, Za=FAKE, Zb=FAKE, Ba=FAKE, Bb=FAKE, pCb=FAKE, pZb=FAKE, e0=FAKE, cache=FAKE,
                n_max=64, B=1, T=16, d=64, m=4, dtype=0)
    args.update(kw)
    a = args
    return N.lib.csa_compress(a["Ca"], a["Cb"], a["Za"], a["Zb"], a["Ba"], a["Bb"], a["pCb"], a["pZb"], a["e0"],
                              a["cache"], a["n_max"], a["B"], a["T"], a["d"], a["m"], a["dtype"], None)


def test_compress_validation():
    assert compress(Ca=None) == ERR_NULL
    assert compress(e0=None) == ERR_NULL
    assert compress(Cb=FAKE + 4) == ERR_ALIGN
    assert compress(dtype=7) == ERR_DTYPE
    assert compress(T=15) == ERR_SHAPE          # not a multiple of m
    assert compress(m=0) == ERR_SHAPE
    assert compress(m=17) == ERR_SHAPE
    assert compress(d=6) == ERR_SHAPE           # rows must stay 16-byte aligned
    assert compress(dtype=1, d=12) == ERR_SHAPE


def index_keys(**kw):
    a = dict(Ca=FAKE, Cb=FAKE, Za=FAKE, Zb=FAKE, Ba=FAKE, Bb=FAKE, pCb=FAKE, pZb=FAKE, e0=FAKE, kI=FAKE, ks=FAKE,
             n_max=64, B=1, T=16, d=128, m=4, dtype=1, ifmt=1)
    a.update(kw)
    return N.lib.index_key_compress(a["Ca"], a["Cb"], a["Za"], a["Zb"], a["Ba"], a["Bb"], a["pCb"], a["pZb"],
                                    a["e0"], a["kI"], a["ks"], a["n_max"], a["B"], a["T"], a["d"], a["m"],
                                    a["dtype"], a["ifmt"], None)


def test_index_key_compress_validation():
    before = N.lib.csa_launch_count()
    assert index_keys(kI=None) == ERR_NULL
    assert index_keys(ks=None) == ERR_NULL
    assert index_keys(e0=None) == ERR_NULL
    assert index_keys(ks=FAKE + 4) == ERR_ALIGN
    assert index_keys(ifmt=0) == ERR_DTYPE          # keys are quantised: E4M3 or MXFP4 only
    assert index_keys(ifmt=3) == ERR_DTYPE
    assert index_keys(dtype=2) == ERR_DTYPE
    assert index_keys(m=8) == ERR_UNSUP             # the CSA rate only
    assert index_keys(T=18) == ERR_SHAPE
    assert index_keys(d=96) == ERR_UNSUP            # threads of an entry: a power of two within a warp
    assert index_keys(d=256, dtype=0) == ERR_UNSUP
    assert index_keys(B=0) == ERR_SHAPE
    assert N.lib.csa_launch_count() == before


def test_indexer_validation():
    def call(**kw):
        a = dict(qI=FAKE, qs=FAKE, w=FAKE, kI=FAKE, ks=FAKE, ne=FAKE, qp=FAKE, m=4, B=1, Tq=1, HI=64, dI=128,
                 n_max=1024, k=64, ifmt=1, idx=FAKE, so=None, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return N.lib.lightning_index(a["qI"], a["qs"], a["w"], a["kI"], a["ks"], a["ne"], a["qp"], a["m"], a["B"],
                                     a["Tq"], a["HI"], a["dI"], a["n_max"], a["k"], a["ifmt"], a["idx"], a["so"],
                                     a["ws"], a["wsb"], None)
    assert call(ifmt=9) == ERR_DTYPE
    assert call(dI=48) == ERR_SHAPE
    assert call(HI=65) == ERR_SHAPE
    assert call(k=4096) == ERR_SHAPE
    assert call(qs=None) == ERR_NULL
    assert call(ifmt=0, qs=None, ks=None) != ERR_NULL      # fp32 operands need no scales
    assert call(wsb=16) == ERR_WS
    assert call(ws=None) == ERR_WS
    assert call(qI=FAKE + 8) == ERR_ALIGN       # vector loads of the query and key rows
    assert call(kI=FAKE + 4) == ERR_ALIGN
    need = N.lib.lightning_index_workspace_size(2, 3, 1000, 64)
    assert need >= 2 * 3 * 1000 * 4


def test_indexer_bf16_validation():
    def call(**kw):
        a = dict(qI=FAKE, qs=FAKE, w=FAKE, kI=FAKE, ks=FAKE, ne=FAKE, qp=FAKE, m=4, B=1, Tq=1, HI=64, dI=128,
                 n_max=1024, k=64, ifmt=1, idx=FAKE, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return N.lib.lightning_index_bf16(a["qI"], a["qs"], a["w"], a["kI"], a["ks"], a["ne"], a["qp"], a["m"],
                                          a["B"], a["Tq"], a["HI"], a["dI"], a["n_max"], a["k"], a["ifmt"], a["idx"],
                                          a["ws"], a["wsb"], None)
    before = N.lib.csa_launch_count()
    assert call(ifmt=9) == ERR_DTYPE
    assert call(k=0) == ERR_SHAPE
    assert call(idx=None) == ERR_NULL
    assert call(ks=None) == ERR_NULL
    assert call(wsb=16) == ERR_WS
    assert call(kI=FAKE + 4) == ERR_ALIGN
    assert N.lib.csa_launch_count() == before


def test_grouped_out_proj_validation():
    def call(**kw):
        a = dict(o=FAKE, T=16, H=128, dv=512, g=16, dm=1024, W1=FAKE, W2=FAKE, d=7168, u=FAKE, y=FAKE, ws=None, wsb=0)
        a.update(kw)
        return N.lib.grouped_out_proj(a["o"], a["T"], a["H"], a["dv"], a["g"], a["dm"], a["W1"], a["W2"], a["d"],
                                      a["u"], a["y"], a["ws"], a["wsb"], None)
    before = N.lib.csa_launch_count()
    assert call(o=None) == ERR_NULL
    assert call(y=FAKE + 2) == ERR_ALIGN
    assert call(T=0) == ERR_SHAPE
    assert call(g=3) == ERR_SHAPE                   # heads split evenly into groups
    assert call(dm=1000) == ERR_UNSUP               # intermediate rows in whole 128-row tiles
    assert call(d=7000) == ERR_UNSUP
    assert call(dv=4, H=16, g=16) == ERR_UNSUP      # K of a group: whole 64-element stages
    assert call(ws=FAKE + 8, wsb=64) == ERR_ALIGN
    assert N.lib.csa_launch_count() == before
    assert N.lib.grouped_out_proj_workspace_size(16, 16, 1024, 7168) == 8 * 16 * 16384 * 4
    assert N.lib.grouped_out_proj_workspace_size(4096, 16, 1024, 7168) == 0   # large batches need no split


def test_shard_merge_validation():
    before = N.lib.csa_launch_count()
    assert N.lib.shard_topk_merge(FAKE, FAKE, FAKE, 9, 4, 64, FAKE, None) == ERR_SHAPE      # at most 8 shards
    assert N.lib.shard_topk_merge(FAKE, FAKE, FAKE, 4, 4, 2048, FAKE, None) == ERR_SHAPE   # G * k <= 4096
    assert N.lib.shard_topk_merge(FAKE, FAKE, None, 2, 4, 64, FAKE, None) == ERR_NULL
    assert N.lib.attn_merge_shards(FAKE, FAKE, 2, 64, 512, 7, FAKE, None, None) == ERR_DTYPE
    assert N.lib.attn_merge_shards(FAKE, None, 2, 64, 512, 1, FAKE, None, None) == ERR_NULL
    assert N.lib.attn_merge_shards(FAKE, FAKE, 0, 64, 512, 1, FAKE, None, None) == ERR_SHAPE
    assert N.lib.csa_launch_count() == before


def test_kv8_compress_validation():
    def call(**kw):
        a = dict(d=576, m=4, dtype=1, T=16, c8=FAKE)
        a.update(kw)
        return N.lib.csa_compress_kv8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, a["c8"], 64, 2, a["T"],
                                      a["d"], a["m"], a["dtype"], None)
    before = N.lib.csa_launch_count()
    assert call(d=512) == ERR_UNSUP
    assert call(m=8) == ERR_UNSUP
    assert call(T=18) == ERR_SHAPE
    assert call(c8=None) == ERR_NULL
    assert call(c8=FAKE + 8) == ERR_ALIGN
    assert call(dtype=5) == ERR_DTYPE
    assert N.lib.csa_launch_count() == before


def test_kv8_attention_validation():
    """FP8 rows exist only on the tensor-core shapes; the checks run before any launch."""
    before = N.lib.csa_launch_count()
    args = lambda H, dk, dv: (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, H, dk, dv, 1024, 64, 16, 0.05, FAKE, None,
                              FAKE, 1 << 30, None)
    assert N.lib.sparse_attn_decode_kv8(*args(64, 576, 512)) == ERR_UNSUP
    assert N.lib.sparse_attn_decode_kv8(*args(128, 64, 64)) == ERR_UNSUP
    a = list(args(128, 576, 512))
    a[1] = None
    assert N.lib.sparse_attn_decode_kv8(*a) == ERR_NULL
    h = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 128, 576, 256, 1024, 16, 0.05, FAKE, None, FAKE, 1 << 30, None)
    assert N.lib.hca_attn_decode_kv8(*h) == ERR_UNSUP
    assert N.lib.csa_launch_count() == before


def test_attention_validation():
    def call(**kw):
        a = dict(q=FAKE, cache=FAKE, idx=FAKE, win=FAKE, wl=FAKE, sink=FAKE, B=2, H=128, dk=576, dv=512,
                 n_max=4096, k=512, W=128, scale=0.04, dtype=1, out=FAKE, lse=None, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return N.lib.sparse_attn_decode(a["q"], a["cache"], a["idx"], a["win"], a["wl"], a["sink"], a["B"], a["H"],
                                        a["dk"], a["dv"], a["n_max"], a["k"], a["W"], a["scale"], a["dtype"],
                                        a["out"], a["lse"], a["ws"], a["wsb"], None)
    assert call(H=129) == ERR_SHAPE
    assert call(dv=640) == ERR_SHAPE
    assert call(dk=580) == ERR_SHAPE
    assert call(dtype=3) == ERR_DTYPE
    assert call(idx=None) == ERR_NULL
    assert call(wl=None) == ERR_NULL
    assert call(out=FAKE + 2) == ERR_ALIGN
    assert call(scale=float("nan")) == ERR_SHAPE
    assert call(ws=None, wsb=0) == ERR_WS
    assert N.lib.attn_decode_workspace_size(16, 128, 512, 640) > 0


def test_fused_hca_step_validation_before_any_launch():
    def call(**kw):
        a = dict(C=FAKE, Z=FAKE, bias=FAKE, e0=FAKE, T_new=128, mp=128, q=FAKE, cache=FAKE, ne=FAKE, win=FAKE,
                 wl=FAKE, sink=FAKE, B=2, H=128, dk=576, dv=512, n_max=8192, W=128, scale=0.04, dtype=1, out=FAKE,
                 lse=None, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return N.lib.hca_compress_attn_decode(a["C"], a["Z"], a["bias"], a["e0"], a["T_new"], a["mp"], a["q"],
                                              a["cache"], a["ne"], a["win"], a["wl"], a["sink"], a["B"], a["H"],
                                              a["dk"], a["dv"], a["n_max"], a["W"], a["scale"], a["dtype"], a["out"],
                                              a["lse"], a["ws"], a["wsb"], None)
    before = N.lib.csa_launch_count()
    assert call(T_new=100) == ERR_SHAPE        # not a multiple of m'
    assert call(mp=2048) == ERR_SHAPE
    assert call(e0=None) == ERR_NULL
    assert call(C=FAKE + 8) == ERR_ALIGN
    assert call(ne=None) == ERR_NULL
    assert call(dv=640) == ERR_SHAPE
    assert call(ws=None, wsb=0) == ERR_WS
    assert N.lib.csa_launch_count() == before  # nothing was launched, not even the compression


def test_topk_validation():
    assert N.lib.topk_select(FAKE, 100, None, 4, 100, 4096, FAKE, None, 0, None) == ERR_SHAPE
    assert N.lib.topk_select(FAKE, 50, None, 4, 100, 8, FAKE, None, 0, None) == ERR_SHAPE   # ld < n
    assert N.lib.topk_select(None, 100, None, 4, 100, 8, FAKE, None, 0, None) == ERR_NULL


def test_package_has_no_cpu_fallback():
    # the binding exposes only library calls; importing never pulls in the oracle
    import sys
    assert not any(m.startswith("oracle") for m in sys.modules if m.startswith("oracle") and
                   getattr(sys.modules[m], "__file__", "").startswith(os.path.dirname(csa.__file__)))
    src = open(os.path.join(os.path.dirname(csa.__file__), "_native.py")).read() + \
        open(os.path.join(os.path.dirname(csa.__file__), "steps.py")).read()
    assert "oracle" not in src


def test_exact_indexer_workspace_drops_the_score_region_only_for_streamed_prefill_rows():
    """lightning_index_workspace_size_exact: the 4096-token prefill chunk (E4M3, 64 x 128,
    k 1024) needs no [rows, n_max] fp32 score region; decode rows, MXFP4 keys, k above 1024
    and too few query groups to fill the device keep the full size (host-side sizes only)."""
    full = csa.lightning_index_workspace_size
    exact = csa.lightning_index_workspace_size_exact
    E, M = csa.CSA_IFMT_E4M3, csa.CSA_IFMT_MXFP4
    B, Tq, N, k = 1, 4096, 33792, 1024
    assert full(B, Tq, N, k) - exact(B, Tq, N, k, E, 64, 128) >= Tq * N * 4
    assert exact(B, Tq, N, k, E, 64, 128) >= Tq * 2048 * 8          # the candidate lists stay
    for args in [(16, 1, 16384, 512, E), (8, 1, 262144, 1024, M), (B, Tq, N, k, M), (B, Tq, N, 2048, E),
                 (1, 8, N, k, E)]:
        b, t, n, kk, f = args
        assert exact(b, t, n, kk, f, 64, 128) == full(b, t, n, kk), args
    assert exact(B, Tq, N, k, E, 32, 128) == full(B, Tq, N, k)
    assert exact(0, Tq, N, k, E, 64, 128) == 0


def test_exact_indexer_workspace_is_what_the_call_checks():
    """The streamed prefill call accepts exactly lightning_index_workspace_size_exact bytes and
    refuses one byte less; with score_out it needs the full size (both refusals happen
    before any device work)."""
    B, Tq, n_max, k, E = 1, 4096, 33792, 1024, csa.CSA_IFMT_E4M3
    exact = csa.lightning_index_workspace_size_exact(B, Tq, n_max, k, E, 64, 128)
    full = csa.lightning_index_workspace_size(B, Tq, n_max, k)

    def call(wsb, so=None):
        return N.lib.lightning_index(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, B, Tq, 64, 128, n_max, k, E, FAKE, so,
                                     FAKE, wsb, None)
    assert call(exact - 1) == ERR_WS
    assert call(exact, so=FAKE) == ERR_WS        # score_out: the scores are written, so the full size
    assert exact < full
