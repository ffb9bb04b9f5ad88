"""Throughput of the CSA / HCA hot path on B200.

By default every workload runs in one invocation and prints one JSON line each:
HCA decode at 1M context, the CSA prefill chunk, the hybrid pair at 1M context, and
last the headline, CSA decode at a 64K context (batch 16 sequences, 16,384
compressed entries, m = 4, 128 query heads of width 576/512, FP8 indexer with 64
heads of width 128, top-k 512, window 128, attention sink).  A decode step is one
token for every sequence: csa_compress (the block the token completes) ->
lightning_index (scores + exact top-k) -> sparse_attn_decode (+ split combine);
the HCA step compresses the fresh 128-token chunk and attends to every entry; the
prefill step compresses the 4096-token chunk, selects per query and attends.
Inputs are synthetic (seeded) and resident in HBM; the timed steps rotate over
enough copies of the inputs that every step reads them from HBM (the rows beyond the
step, timed alone, flush L2 before every call instead).  ``--workload NAME`` runs one workload.

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample
of the same workloads.  Under torchrun each rank runs its own batch (independent
sequences: weak scaling, no data-path collective); rank 0 prints the lines.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    "csa_decode_64k": 1,
    "hca_decode_1m": 2,
    "csa_prefill_4k": 3,
    "hybrid_pair_1m": 4,
}
METRIC = "CSA/HCA decode tokens/s and HBM GB/s (% roofline) at 64K-1M ctx; prefill TFLOP/s"
L2_BYTES = 126 * 1024 * 1024

# DRAM bytes (read + write) per call of the dominant ABI call, summed over its kernels, from
# the ncu captures summarised under profiles/ (None until a capture of the current kernels).
TENSOR_PEAKS = {}   # measured once per single-GPU run (measure_tensor_peaks)

TRAFFIC = {
    # profiles/csa_decode_64k_dram_traffic.md: indexer_tc_kernel<1,6> 34 773 632 + indexer_select_row 1 369 984
    ("csa_decode_64k", "indexer"): 36143616,
    # profiles/hybrid_pair_1m_dram_traffic.md: indexer_mxf4_kernel 142 688 000 read + 5 062 784 written (its
    # scores) + indexer_select_dist 8 670 080
    ("hybrid_pair_1m", "indexer"): 156420864,
    # profiles/hca_decode_1m_launches.md: attn_tc_kernel 39 008 896 read + 2 304 written (the combine's
    # reads are L2 hits in the timed step; under ncu the caches are flushed before each kernel)
    ("hca_decode_1m", "attention"): 39011200,
    # profiles/csa_prefill_4k_launches.md: attn_tc_kernel 831 254 272 read (cache rows, queries, raw
    # window) + 513 781 248 written (the 537 MB bf16 output, partly still in L2 at the kernel's end)
    ("csa_prefill_4k", "attention"): 1345035520,
}


def workload_config(name, D):
    """The workload a line is measured on (shared by both arms)."""
    return {"workload": name, "batch": D["B"], "context": D["T"], "entries": D["N"], "query_tokens": D.get("Tq", 1),
            "top_k": D.get("k"), "window": D["W"], "heads": D["H"], "d_k": D["dk"], "d_v": D["dv"],
            "indexer": D.get("ifmt")}


def algorithmic_flops(wid, D):
    """Prefill multiply-adds x 2 of the tensor-core contractions (valid rows only)."""
    if wid != 3:
        return {}
    import numpy as np
    Tq, H, dk, dv, k, W, m = D["Tq"], D["H"], D["dk"], D["dv"], D["k"], D["W"], D["m"]
    pos = D["q_pos0"] + np.arange(Tq)
    n_elig = np.minimum(D["N"], (pos + 1) // m)
    rows = np.minimum(n_elig, k) + np.minimum(pos + 1, W)
    return {"attention": float(2 * H * (dk + dv) * rows.sum()),
            "indexer": float(2 * D["HI"] * D["dI"] * n_elig.sum())}


def algorithmic_bytes(wid, D):
    """Bytes the method must move per step (each input / output byte once)."""
    B = D["B"]
    if wid in (1, 4):
        N, d, k, W, H, dv, dI = D["N"], D["d"], D["k"], D["W"], D["H"], D["dv"], D["dI"]
        kI_row = dI + 4 if D["ifmt"] == "e4m3" else dI // 2 + dI // 32
        per = dict(
            # the block's 4 series x 4 tokens + biases + the entry; its key's 4 x 4 indexer
            # activations + key row; the raw row into the window
            compress=(4 * 4 * d * 2) + 8 * 4 * d + d * 2 + (4 * 4 * dI * 2 + kI_row) + 2 * d * 2,
            indexer=N * kI_row + 64 * (dI + 4) + 64 * 4,
            attention=k * d * 2 + W * d * 2 + H * d * 2 + H * dv * 2,
        )
        tot = {kk: v * B for kk, v in per.items()}
        if wid == 4:
            Nh = D["Nh"]
            tot["hca"] = B * (Nh * d * 2 + W * d * 2 + H * d * 2 + H * dv * 2 + 2 * 128 * d * 2)
        return tot
    if wid == 2:
        N, d, W, H, dv = D["N"], D["d"], D["W"], D["H"], D["dv"]
        return dict(compress=B * 2 * 128 * d * 2, attention=B * (N * d * 2 + W * d * 2 + H * d * 2 + H * dv * 2))
    if wid == 3:
        Tq, d, H, dv, N = D["Tq"], D["d"], D["H"], D["dv"], D["N"]
        return dict(compress=4 * Tq * d * 2, indexer=N * 132 + Tq * 64 * 132,
                    attention=Tq * H * d * 2 + Tq * H * dv * 2 + N * d * 2)
    raise ValueError(wid)


def measure_tensor_peaks(csa):
    """Dense MMA rate at the indexer's operand formats and shapes, measured by the library's
    probe (operands resident in shared memory, one CTA per SM, CUDA events around three
    launches after a warm-up), with the nominal dense figures beside it."""
    import torch
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    res = {}
    for name, fmt, n, iters, nominal in (("fp8_e4m3", csa.CSA_IFMT_E4M3, 256, 4000, 4500.0),
                                         ("mxfp4", csa.CSA_IFMT_MXFP4, 64, 16000, 9000.0)):
        csa.tensor_peak_probe(fmt, 100)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(3):
            csa.tensor_peak_probe(fmt, iters)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 3
        flops = 2.0 * 128 * n * 128 * iters * sms
        res[name] = {"tflops": flops / (ms * 1e-3) / 1e12, "nominal_tflops": nominal,
                     "shape": f"M 128, N {n}, K 128 x {iters} per SM, {sms} SMs"}
    return res


def sample_clocks(stop, out):
    cmd = ["nvidia-smi", "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
           "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
           "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
           "--format=csv,noheader,nounits", "-lms", "100"]
    try:
        p = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
    except OSError:
        return
    dev = os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0]
    try:
        while not stop.is_set():
            line = p.stdout.readline()
            if not line:
                break
            out.append(line.strip())
    finally:
        p.terminate()
        try:
            p.wait(timeout=5)
        except Exception:
            p.kill()


def summarize_clocks(lines, local_index=None):
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for l in lines:
        f = [x.strip() for x in l.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1])); mx = float(f[2])
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower().startswith("active"):
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
    sm.sort()
    return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons)}


def rank_seed(wid, rank):
    """Each rank draws its own batch of the workload (independent sequences)."""
    return wid + 1000 * rank


def max_over_ranks(x, world, device):
    """The slowest rank's value: every timing is taken per rank on its own device."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, world, ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (ms * 1e-3)


def run_reference(args, wid, name):
    """Time the fp64 oracle on host cores on a bounded sample of the workload."""
    import numpy as np
    import csa_inputs as CI
    from oracle import csa_oracle as O
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    scale = None
    wl = CI.make_workload(wid, scale=scale)
    D = wl.dims
    cores = os.cpu_count()
    sample_b = list(range(min(D["B"], 1 if wid == 4 else 4)))   # the pair's MXFP4 decode costs ~1 s a sequence
    sample_rows = [int(r) for r in np.linspace(0, D["Tq"] - 1, 4)] if wid == 3 else []
    t0 = time.perf_counter()
    steps_done = 0
    for _ in range(max(1, args.steps)):
        if wid in (1, 4):
            O.run_csa_decode(wl, batches=sample_b)
            if wid == 4:
                O.run_hca_decode(wl, batches=sample_b, prefix="h_")
        elif wid == 2:
            O.run_hca_decode(wl, batches=sample_b)
        else:
            O.run_csa_prefill(wl, rows=sample_rows)
        steps_done += 1
    dt = time.perf_counter() - t0
    tokens = steps_done * (len(sample_rows) if wid == 3 else len(sample_b))
    sample = (f"{len(sample_rows)} of {D['Tq']} query tokens per step (compression of the whole chunk included)"
              if wid == 3 else f"{len(sample_b)} of {D['B']} sequences per step, full context")
    value = tokens / dt
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / steps_done * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(name, D),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# the order of the lines of a default run: the headline workload comes last
ORDER = ["hca_decode_1m", "csa_prefill_4k", "hybrid_pair_1m", "csa_decode_64k"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="all", choices=["all"] + list(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    names = ORDER if args.workload == "all" else [args.workload]
    for name in names:
        if args.impl == "reference":
            run_reference(args, WORKLOADS[name], name)
        else:
            run_ours(args, WORKLOADS[name], name)


def check_device(csa, name, where):
    """Raise if a kernel flagged an error (the library's device error word) since the last check."""
    import torch
    torch.cuda.synchronize()
    e = csa.read_device_error()
    if e:
        raise RuntimeError(f"{name}: device error word 0x{e:x} after the {where}")


def run_ours(args, wid, name):
    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    import compressed_sparse_long_csa_b200 as csa
    if world == 1 and "v" not in TENSOR_PEAKS:
        TENSOR_PEAKS["v"] = measure_tensor_peaks(csa)
    from compressed_sparse_long_csa_b200 import steps
    import csa_inputs as CI

    wl = CI.make_workload(wid, seed=rank_seed(wid, rank))
    D = wl.dims
    T = steps.upload(wl)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def l2_flush():
        # write 256 MB (twice the L2), then read it back so that L2 holds clean lines and the
        # timed kernels do not pay for write-backs of the flush itself (used by the single-call
        # characterisations of the rows beyond the step)
        flush.zero_()
        flush.view(torch.float32).sum()

    # Timed steps rotate over n_copies copies of the step's inputs (every tensor the workload
    # defines: caches, keys, queries, window, compressor inputs), enough that the bytes read
    # between two uses of a copy are at least three times the 126 MB L2: each step's inputs
    # come from HBM, while the kernels' instructions stay warm as in a serving loop.  Outputs
    # and workspaces are shared (every step rewrites them).
    step_bytes = sum(algorithmic_bytes(wid, D).values())
    n_copies = int(min(16, max(2, -(-3 * L2_BYTES // step_bytes))))
    Ts = [T]
    for _ in range(n_copies - 1):
        Tc = dict(T)
        for k in wl.tensors:
            Tc[k] = T[k].clone()
        Ts.append(Tc)

    # The four ABI calls of a step (compress / indexer / attention / hca), each captured once
    # per copy into a CUDA graph so that host-side launch cost stays out of the device
    # timeline; events between the graph launches attribute the time to the calls.
    p = "h_"

    def part_compress(T):
        if "CaI" in T:
            steps._decode_append(T, D, None)      # cache entry, its key and the window row, one launch
        elif wid in (1, 3, 4):
            csa.csa_compress(T["Ca"], T["Cb"], T["Za"], T["Zb"], T["Ba"], T["Bb"], T["prev_Cb"], T["prev_Zb"],
                             T["entry0"], T["cache"], m=D["m"])
        else:
            if "raw_new" in T:
                csa.window_append(T["raw_new"], T["win"], T["win_slot"])
            csa.hca_compress(T["C"], T["Z"], T["bias"], T["entry0"], T["cache"], D["m_prime"])

    def part_indexer(T):
        if wid in (1, 3, 4):
            csa.lightning_index(T["qI"], T.get("qI_scale"), T["w"], T["kI"], T.get("kI_scale"), T["n_entries"],
                                T["q_pos"], D["k"], steps._ifmt(D), T["idx"], T["iws"], m=D["m"])

    def part_attention(T):
        if wid == 3:
            csa.sparse_attn_prefill(T["q"], T["q_pos"], T["cache"], T["idx"], T["raw"], T["raw_pos0"], D["W"],
                                    T["sink"], D["sm_scale"], D["dv"], T["out"], T["lse"])
        elif wid in (1, 4):
            csa.sparse_attn_decode(T["q"][:, 0], T["cache"], T["idx"][:, 0], T["win"], T["win_len"], T["sink"],
                                   D["sm_scale"], D["dv"], T["out"][:, 0], T["lse"][:, 0], T["aws"])
        else:
            csa.hca_attn_decode(T["q"][:, 0], T["cache"], T["n_entries"], T["win"], T["win_len"], T["sink"],
                                D["sm_scale"], D["dv"], T["out"][:, 0], T["lse"][:, 0], T["aws"])

    def part_hca(T):
        if wid == 4:
            steps.hca_decode_step(T, D, prefix=p)

    parts = [part_compress, part_indexer, part_attention, part_hca]
    for _ in range(max(3, args.warmup)):        # eager warm-up (also resolves every lazy setup step)
        for Tc in Ts:
            for f in parts:
                f(Tc)
    torch.cuda.synchronize()
    n0 = csa.launch_count()
    for f in parts:                              # one more eager step: count the library's kernels
        f(T)
    launches_step = csa.launch_count() - n0
    torch.cuda.synchronize()
    check_device(csa, name, "eager warm-up")
    # the whole step as one CUDA graph per copy (the timed quantity), and one graph per ABI
    # call and copy (timed separately, for the per-call breakdown)
    active = {1: [1, 1, 1, 0], 2: [1, 0, 1, 0], 3: [1, 1, 1, 0], 4: [1, 1, 1, 1]}[wid]   # calls a step makes
    graphs, g_steps = [], []
    for Tc in Ts:
        gl = []
        for f, on in zip(parts, active):
            g = None
            if on:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    f(Tc)
            gl.append(g)
        graphs.append(gl)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            steps.run_step(wl.kind, Tc, D)   # the step as a user runs it (compressor append on a side stream)
        g_steps.append(g)
    torch.cuda.synchronize()

    def step_parts(evs, c):
        evs[0].record()
        for i, g in enumerate(graphs[c]):
            if g is not None:
                g.replay()
            evs[i + 1].record()

    def mk(n=5):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    for w in range(max(3, args.warmup)):
        for c in range(n_copies):
            g_steps[c].replay()
        step_parts(mk(), w % n_copies)
    torch.cuda.synchronize()
    check_device(csa, name, "graph warm-up")

    clock_lines, stop = [], threading.Event()
    th = threading.Thread(target=sample_clocks, args=(stop, clock_lines), daemon=True)
    th.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for i in range(args.steps):
        g_steps[i % n_copies].replay()
    ev1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    stop.set()
    th.join(timeout=10)
    ev_list = []                             # per-call breakdown (not part of the timed quantity)
    for i in range(max(10, n_copies)):
        evs = mk()
        step_parts(evs, i % n_copies)
        ev_list.append(evs)
    torch.cuda.synchronize()
    per = np.array([[ev[i].elapsed_time(ev[i + 1]) for i in range(4)] for ev in ev_list])   # ms
    total_ms = max_over_ranks(float(ev0.elapsed_time(ev1)), world, "cuda")
    ms_per_step = total_ms / args.steps
    tokens_per_step = D["B"] * (D["Tq"] if wid == 3 else 1)
    value = job_rate(tokens_per_step, world, ms_per_step)

    # ---- e2e through the public API with host buffers (max over ranks too)
    check_device(csa, name, "timed steps")
    e2e_ms, h2d, d2h, h2d_gbs = measure_e2e(args, wid, wl, Ts, D, csa, steps)
    check_device(csa, name, "e2e")
    e2e_ms = max_over_ranks(e2e_ms, world, "cuda")
    e2e = {"value": job_rate(tokens_per_step, world, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "h2d_link_gbs": h2d_gbs, "h2d_copy_ms": h2d / h2d_gbs * 1e-6}
    ab = algorithmic_bytes(wid, D)
    comp = ["compress", "indexer", "attention", "hca"]
    mean_ms = per.mean(axis=0)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    src = "measured" if peaks else "fallback"
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    bf16_peak = peaks.get("bf16_tflops", 1590.0)
    tpeaks = TENSOR_PEAKS.get("v") if world == 1 else None
    # the dominant ABI call by time; decode calls are HBM-bound, prefill calls tensor-bound
    # (the FP8 indexer against the measured FP8 MMA rate, else twice the measured bf16 peak,
    # the nominal dense ratio)
    cand = [c for c in comp if c in ab]
    dom = max(cand, key=lambda c: mean_ms[comp.index(c)])
    dom_ms = float(mean_ms[comp.index(dom)])
    fl = algorithmic_flops(wid, D)
    if wid == 3 and dom in fl:
        if dom == "indexer" and tpeaks:
            peak, psrc = tpeaks["fp8_e4m3"]["tflops"], "measured fp8 MMA probe"
        else:
            peak = bf16_peak * (2.0 if dom == "indexer" else 1.0)
            psrc = src + (" bf16 x 2 (fp8)" if dom == "indexer" else " bf16 burst")
        achieved = fl[dom] / (dom_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": psrc, "traffic": TRAFFIC.get((name, dom))}
    else:
        achieved = ab[dom] / (dom_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "peak_source": src, "traffic": TRAFFIC.get((name, dom))}
    # the indexer's tensor-side fraction beside its HBM one: its dot-product FLOPs (every
    # eligible entry x 64 heads x d_I) against the measured MMA rate of its format
    idx_tensor = None
    if tpeaks and wid in (1, 3, 4):
        fmt_key = "fp8_e4m3" if D["ifmt"] == "e4m3" else "mxfp4"
        if fmt_key in tpeaks:
            idx_fl = fl.get("indexer") if wid == 3 else float(2 * D["HI"] * D["dI"] * D["N"] * D["B"])
            a_tf = idx_fl / (float(mean_ms[comp.index("indexer")]) * 1e-3) / 1e12
            idx_tensor = {"achieved": a_tf, "peak": tpeaks[fmt_key]["tflops"], "unit": "TFLOP/s",
                          "frac": a_tf / tpeaks[fmt_key]["tflops"], "nominal_peak": tpeaks[fmt_key]["nominal_tflops"],
                          "peak_source": "measured " + fmt_key + " MMA probe"}
    extra = None
    if world == 1:
        # the rows beyond the step, each timed alone on this GPU (single-GPU characterisations:
        # a multi-rank run skips them)
        extra = measure_index_keys(wid, D, csa, l2_flush, hbm_peak, src)
        bf = measure_bf16_index(wid, D, T, csa, steps, l2_flush, float(mean_ms[comp.index("indexer")]))
        if bf:
            extra = dict(extra or {}, **bf)
        extra = dict(extra or {}, **measure_out_proj(D, T, csa, l2_flush, hbm_peak, bf16_peak, src))
        kv = measure_kv8_attention(wid, wl, D, T, csa, l2_flush, float(mean_ms[comp.index("attention")]), hbm_peak,
                                   src)
        if kv:
            extra.update(kv)
        check_device(csa, name, "rows beyond the step")
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(name, D), launch="one CUDA graph per step",
                       l2=f"inputs rotated over {n_copies} copies ({n_copies * step_bytes / 1e6:.0f} MB, over 3x the "
                          f"126 MB L2 between reuses); no flush"),
        "hbm_gbs_step": sum(ab.values()) / (ms_per_step * 1e-3) / 1e9,
        "hbm_frac_step": sum(ab.values()) / (ms_per_step * 1e-3) / 1e9 / hbm_peak,
        "breakdown_ms": {c: float(m) for c, m in zip(comp, mean_ms)},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": launches_step * args.steps,
        "clocks": summarize_clocks(clock_lines),
    }
    if idx_tensor:
        line["indexer_tensor"] = idx_tensor
    if tpeaks:
        line["tensor_peaks"] = tpeaks
    if extra:
        line["next_rows"] = extra
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wid, wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    # release this workload's graphs and buffers before the next one
    del g_steps, graphs, T, Ts
    import gc
    gc.collect()
    torch.cuda.empty_cache()
    if world > 1:
        dist.barrier()
        if name == ORDER[-1] or args.workload != "all":
            dist.destroy_process_group()


def measure_index_keys(wid, D, csa, l2_flush, hbm_peak, peak_src, reps=20):
    """The indexer-key producer for the entries this workload's step completes (one per
    sequence in decode, Tq/4 in the prefill chunk), timed alone: one call captured in a
    CUDA graph, L2 flushed before each replay, CUDA events around it.  Not part of the
    step's timed quantity."""
    import numpy as np
    import torch
    import csa_inputs as CI
    if wid not in (1, 3, 4):
        return None
    B, T_new, d_I = D["B"], (D["Tq"] if wid == 3 else D["m"]), D["dI"]
    mx = D["ifmt"] == "mxfp4"
    t = CI.index_key_inputs(977, B, T_new, d_I, "bf16")
    dev = {k: (torch.from_numpy(v).cuda() if v.dtype == np.float32
               else torch.from_numpy(v.view(np.int16)).cuda().view(torch.bfloat16)) for k, v in t.items()}
    n_max = D["n_max"]
    e0 = torch.full((B,), D["entry0"], dtype=torch.int32, device="cuda")
    kI = torch.empty((B, n_max, d_I // 2 if mx else d_I), dtype=torch.uint8, device="cuda")
    ks = (torch.empty((B, n_max, d_I // 32), dtype=torch.uint8, device="cuda") if mx
          else torch.empty((B, n_max), dtype=torch.float32, device="cuda"))
    fmt = csa.CSA_IFMT_MXFP4 if mx else csa.CSA_IFMT_E4M3

    def call():
        csa.index_key_compress(dev["Ca"], dev["Cb"], dev["Za"], dev["Zb"], dev["Ba"], dev["Bb"], dev["prev_Cb"],
                               dev["prev_Zb"], e0, kI, ks, fmt)

    for _ in range(3):
        call()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    ms = []
    for _ in range(reps):
        l2_flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        ms.append((a, b))
    torch.cuda.synchronize()
    us = float(np.mean([a.elapsed_time(b) for a, b in ms])) * 1e3
    n = B * (T_new // 4)
    # algorithmic bytes: every source row read once (4 series of the chunk plus the two
    # b-series rows before it), biases, and the key rows written
    nbytes = (4 * B * T_new * d_I + 2 * B * 4 * d_I) * 2 + 2 * 4 * d_I * 4 + n * ((d_I // 2 + d_I // 32) if mx else (d_I + 4))
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"index_key_compress": {"entries": n, "format": D["ifmt"], "us": us, "bytes": nbytes,
                                   "achieved_gbs": gbs, "frac": gbs / hbm_peak, "peak_source": peak_src,
                                   "l2": "flushed before every call",
                                   "timing": "CUDA events around one graph replay of the call (launch included)"}}


def measure_bf16_index(wid, D, T, csa, steps, l2_flush, exact_ms, reps=20):
    """lightning_index_bf16 on this workload's indexer inputs, timed alone like the
    per-call breakdown (one graph replay after an L2 flush), and its recall against the
    exact selection of the same inputs (the step's own index output)."""
    import numpy as np
    import torch
    if wid not in (1, 3, 4):
        return None
    exact = T["idx"].clone()
    idx = torch.empty_like(T["idx"])
    # the bf16-key call writes its scores: the full workspace (the step's may omit that region)
    ws = torch.empty(csa.lightning_index_workspace_size(D["B"], D["Tq"], D["n_max"], D["k"]), dtype=torch.uint8,
                     device="cuda")

    def call():
        csa.lightning_index_bf16(T["qI"], T.get("qI_scale"), T["w"], T["kI"], T.get("kI_scale"), T["n_entries"],
                                 T["q_pos"], D["k"], steps._ifmt(D), idx, ws, m=D["m"])

    for _ in range(3):
        call()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    evs = []
    for _ in range(reps):
        l2_flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    us = float(np.mean([a.elapsed_time(b) for a, b in evs])) * 1e3
    e, f = exact.cpu().numpy().reshape(-1, D["k"]), idx.cpu().numpy().reshape(-1, D["k"])
    hit = sum(np.intersect1d(f[r][f[r] >= 0], e[r][e[r] >= 0]).size for r in range(e.shape[0]))
    recall = hit / max(int((e >= 0).sum()), 1)
    return {"lightning_index_bf16": {"us": us, "exact_us": exact_ms * 1e3, "speedup": exact_ms * 1e3 / us,
                                     "recall_vs_exact": recall, "l2": "flushed before every call",
                                     "timing": "CUDA events around one graph replay of the call (launch included)"}}


def measure_out_proj(D, T, csa, l2_flush, hbm_peak, bf16_peak, peak_src, reps=10):
    """The grouped output projection (16 groups -> 1024 -> 7168, the Pro sizes) applied to
    this step's attention output, timed alone (one graph replay after an L2 flush).  Few
    tokens stream 369 MB of weights (HBM-bound); a prefill chunk is tensor-bound."""
    import numpy as np
    import torch
    import csa_inputs as CI
    H, dv, g, d_mid, d = D["H"], D["dv"], 16, 1024, 7168
    o = T["out"].reshape(-1, H, dv)
    n_tok = o.shape[0]
    x = CI.out_proj_inputs(4242, 1, H, dv, g, d_mid, d)
    W1 = torch.from_numpy(x["W1"].view(np.int16)).cuda().view(torch.bfloat16)
    W2 = torch.from_numpy(x["W2"].view(np.int16)).cuda().view(torch.bfloat16)
    u = torch.empty((n_tok, g * d_mid), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((n_tok, d), dtype=torch.bfloat16, device="cuda")
    nb = csa.grouped_out_proj_workspace_size(n_tok, g, d_mid, d)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None

    def call():
        csa.grouped_out_proj(o, W1, W2, g, u, y, ws)

    for _ in range(3):
        call()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        call()
    evs = []
    for _ in range(reps):
        l2_flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        gr.replay()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    us = float(np.mean([a.elapsed_time(b) for a, b in evs])) * 1e3
    wbytes = (W1.numel() + W2.numel()) * 2
    nbytes = wbytes + n_tok * (H * dv + 2 * g * d_mid + d) * 2
    flops = 2.0 * n_tok * (W1.numel() + W2.numel())
    res = {"tokens": n_tok, "us": us, "bytes": nbytes, "achieved_gbs": nbytes / (us * 1e-6) / 1e9,
           "tflops": flops / (us * 1e-6) / 1e12, "peak_source": peak_src, "l2": "flushed before every call",
           "timing": "CUDA events around one graph replay of the call (launch included)"}
    if n_tok <= 256:
        res.update(bound="hbm", frac=res["achieved_gbs"] / hbm_peak)
    else:
        res.update(bound="tensor", frac=res["tflops"] / bf16_peak)
    del W1, W2
    return {"grouped_out_proj": res}


def measure_kv8_attention(wid, wl, D, T, csa, l2_flush, bf16_ms, hbm_peak, peak_src, reps=20):
    """The decode attention of this step over an FP8 copy of the cache (656-byte rows made
    by the input generator from the same values), timed alone like the per-call breakdown,
    beside the bf16 call's time."""
    import numpy as np
    import torch
    import csa_inputs as CI
    if wid not in (1, 2):
        return None
    bits = wl.tensors["cache"]
    x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float()
    c8 = torch.from_numpy(CI.quant_latent_fp8_rows(x)).cuda()
    del x
    B, H, dv, W = D["B"], D["H"], D["dv"], D["W"]
    out = torch.empty(B, H, dv, dtype=torch.bfloat16, device="cuda")

    def call():
        if wid == 1:
            csa.sparse_attn_decode_kv8(T["q"][:, 0], c8, T["idx"][:, 0], T["win"], T["win_len"], T["sink"],
                                       D["sm_scale"], dv, out, workspace=T["aws"])
        else:
            csa.hca_attn_decode_kv8(T["q"][:, 0], c8, T["n_entries"], T["win"], T["win_len"], T["sink"],
                                    D["sm_scale"], dv, out, workspace=T["aws"])

    for _ in range(3):
        call()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    evs = []
    for _ in range(reps):
        l2_flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    us = float(np.mean([a.elapsed_time(b) for a, b in evs])) * 1e3
    rows = D["k"] if wid == 1 else D["N"]
    nbytes = B * (rows * 656 + W * 1152 + H * 576 * 2 + H * dv * 2)
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"attention_kv8": {"us": us, "bf16_us": bf16_ms * 1e3, "speedup": bf16_ms * 1e3 / us, "bytes": nbytes,
                              "achieved_gbs": gbs, "frac": gbs / hbm_peak, "peak_source": peak_src,
                              "l2": "flushed before every call",
                              "timing": "CUDA events around one graph replay of the call (launch included)"}}


def measure_e2e(args, wid, wl, Ts, D, csa, steps):
    """Same step through the public API, every step's inputs copied from pinned host
    memory and its results read back inside the timed region.  Two buffer sets: the
    copies of step i+1's inputs and of step i-1's results run on their own streams while
    step i computes (what a serving loop does); the region ends when the last result is
    on the host.  The packed buffers hold exactly the tensors the step reads as input
    and writes as result; every other tensor (caches, workspaces) stays resident, and the
    steps rotate over the resident copies as the device-timed steps do.  Each step's calls
    are one CUDA graph launch (captured per buffer set and resident copy)."""
    import torch
    T = Ts[0]
    # a decode step brings its block's compressor and indexer activations, its query and its
    # raw latent (appended to the resident window ring by the library); the window's other
    # rows, the caches and the keys stay resident
    fresh = ["CaI", "CbI", "ZaI", "ZbI", "raw_new"]
    per_step_in = {1: ["Ca", "Cb", "Za", "Zb", "q", "qI", "qI_scale", "w"] + fresh,
                   2: ["C", "Z", "q", "raw_new"], 3: ["Ca", "Cb", "Za", "Zb", "q", "qI", "qI_scale", "w"],
                   4: ["Ca", "Cb", "Za", "Zb", "q", "qI", "qI_scale", "w"] + fresh + ["h_C", "h_Z", "h_q", "h_raw_new"]}[wid]
    outs = ["out", "idx"] if wid != 2 else ["out"]
    if wid == 4:
        outs.append("h_out")
    # the step's inputs (and its results) are packed into one buffer each, so that a
    # step moves one host-to-device and one device-to-host copy
    def layout(names):
        off, lay = 0, {}
        for k in names:
            nb = T[k].numel() * T[k].element_size()
            lay[k] = (off, nb)
            off += (nb + 255) // 256 * 256
        return lay, off

    def views(buf, lay):
        return {k: buf[o:o + nb].view(T[k].dtype).view(T[k].shape) for k, (o, nb) in lay.items()}

    lay_in, n_in = layout(per_step_in)
    lay_out, n_out = layout(outs)
    host_in = torch.empty(n_in, dtype=torch.uint8).pin_memory()
    for k, v in views(host_in, lay_in).items():
        v.copy_(T[k].cpu())
    dev_in = [host_in.to("cuda") for _ in range(2)]       # valid inputs for the warm-up and capture runs
    dev_out = [torch.empty(n_out, dtype=torch.uint8, device="cuda") for _ in range(2)]
    host_out = [torch.empty(n_out, dtype=torch.uint8).pin_memory() for _ in range(2)]
    io = [dict(views(dev_in[j], lay_in), **views(dev_out[j], lay_out)) for j in range(2)]
    h2d = sum(nb for _, nb in lay_in.values())
    d2h = sum(nb for _, nb in lay_out.values())
    n = max(6, min(args.steps, 20))
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_comp = [torch.cuda.Event(), torch.cuda.Event()]
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]
    # the step's calls, captured once per (buffer set, resident copy) into a CUDA graph, as a
    # serving loop would: each step is then one launch from the host
    step_graphs = {}
    for j in range(2):
        for c in range(len(Ts)):
            Tjc = dict(Ts[c], **io[j])
            steps.run_step(wl.kind, Tjc, D)                # warm (and resolve lazy set-up) outside capture
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                steps.run_step(wl.kind, Tjc, D)
            step_graphs[(j, c)] = g
    torch.cuda.synchronize()

    def run(nsteps, e0=None, e1=None):
        if e0 is not None:
            e0.record(comp)
        s_in.wait_stream(comp)
        s_out.wait_stream(comp)
        for i in range(nsteps):
            j = i & 1
            ev_in = torch.cuda.Event()
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[j])          # step i-2 has read this set's inputs
                dev_in[j].copy_(host_in, non_blocking=True)
                ev_in.record(s_in)
            comp.wait_event(ev_in)
            if i >= 2:
                comp.wait_event(ev_out[j])              # step i-2's results have left this set
            step_graphs[(j, i % len(Ts))].replay()      # the step's calls on set j and resident copy i
            ev_comp[j].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[j])
                host_out[j].copy_(dev_out[j], non_blocking=True)
                ev_out[j].record(s_out)
        comp.wait_stream(s_out)
        comp.wait_stream(s_in)
        if e1 is not None:
            e1.record(comp)

    run(2)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    run(n, e0, e1)
    torch.cuda.synchronize()
    # the host link alone: the same packed input copy, back to back (the e2e roofline)
    link = []
    for _ in range(3):
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s_in):
            a.record(s_in)
            for _ in range(n):
                dev_in[0].copy_(host_in, non_blocking=True)
            b_.record(s_in)
        torch.cuda.synchronize()
        link.append(a.elapsed_time(b_) / n)
    h2d_gbs = h2d / (min(link) * 1e-3) / 1e9
    return e0.elapsed_time(e1) / n, h2d, d2h, h2d_gbs


def cpu_baseline(wid, wl, min_s=3.0, max_reps=20):
    """The oracle as it stands on the host cores, on a bounded sample of the workload:
    the sample (whole sequences of a decode step, query rows of the prefill chunk with
    the chunk's compression) is repeated until at least min_s seconds have passed, and
    the rate is taken over all repeats."""
    from oracle import csa_oracle as O
    D = wl.dims
    sample = list(range(min(D["B"], 2)))
    rows = list(range(8))
    reps, t0 = 0, time.perf_counter()
    while reps < max_reps and (reps == 0 or time.perf_counter() - t0 < min_s):
        if wid in (1, 4):
            O.run_csa_decode(wl, batches=sample)
            if wid == 4:
                O.run_hca_decode(wl, batches=sample, prefix="h_")
        elif wid == 2:
            O.run_hca_decode(wl, batches=sample)
        else:
            O.run_csa_prefill(wl, rows=rows)
        reps += 1
    dt = time.perf_counter() - t0
    toks = (len(sample) if wid != 3 else len(rows)) * reps
    what = (f"{len(rows)} query rows of the chunk (with the chunk's compression)" if wid == 3
            else f"{len(sample)} of {D['B']} sequences, full context")
    return {"value": toks / dt, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{what}, repeated {reps}x ({dt:.1f} s)"}


if __name__ == "__main__":
    main()
