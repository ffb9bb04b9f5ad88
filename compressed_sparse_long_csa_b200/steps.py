"""One pass of the CSA / HCA hot path as a sequence of C-ABI calls.

A *step* is what one attention layer does for one batch:

* CSA decode (one new token per sequence that completes an m-token block):
  csa_compress (entry N-1, appended to the cache) -> lightning_index (scores +
  exact top-k) -> sparse_attn_decode (selected entries + window + sink).
* HCA decode (the token completes an m'-token chunk): hca_compress (entry N-1)
  -> hca_attn_decode (all entries + window + sink).
* CSA prefill chunk: csa_compress (the chunk's entries) -> lightning_index (per
  query eligibility) -> sparse_attn_prefill.
* Hybrid pair: a CSA decode step then an HCA decode step.

The functions take a dict of device tensors (see ``upload``) and only issue the
calls; every number is computed by the library's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _native as N

_INT_META = ("entry0", "q_pos", "n_entries", "win_len", "raw_pos0", "h_entry0", "h_n_entries", "h_win_len", "win_slot")


def _to_device(name, arr, device):
    if arr.dtype == np.uint16:          # bf16 storage bits
        return torch.from_numpy(arr.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def upload(wl, device="cuda"):
    """Copy a csa_inputs.Workload to the device and allocate outputs/workspaces."""
    D = wl.dims
    T = {k: _to_device(k, v, device) for k, v in wl.tensors.items()}
    B, Tq = D["B"], D["Tq"]
    i32 = dict(dtype=torch.int32, device=device)
    lat = torch.bfloat16 if D["dtype"] == "bf16" else torch.float32
    kind = wl.kind
    if kind in ("csa_decode", "csa_prefill", "hybrid_pair"):
        if "cache" not in T:                           # tiny prefill: the cache starts empty
            T["cache"] = torch.zeros(B, D["N"], D["d"], dtype=lat, device=device)
        T["entry0"] = torch.full((B,), D["entry0"], **i32)
        T["n_entries"] = torch.full((B,), D["N"], **i32)
        T["q_pos"] = (D["q_pos0"] + torch.arange(Tq, dtype=torch.int32)).repeat(B, 1).to(device)
        T["idx"] = torch.empty(B, Tq, D["k"], **i32)
        # the exact call's own size: prefill rows that stream candidates need no score region
        T["iws"] = torch.empty(N.lightning_index_workspace_size_exact(B, Tq, D["n_max"], D["k"], _ifmt(D), D["HI"],
                                                                       D["dI"]), dtype=torch.uint8, device=device)
        T["out"] = torch.empty(B, Tq, D["H"], D["dv"], dtype=lat, device=device)
        T["lse"] = torch.empty(B, Tq, D["H"], dtype=torch.float32, device=device)
        if kind == "csa_prefill":
            T["raw_pos0"] = torch.full((B,), D["raw_pos0"], **i32)
        else:
            T["win_len"] = torch.full((B,), D["W"], **i32)
            if "win_slot" in D:
                T["win_slot"] = torch.full((B,), D["win_slot"], **i32)
            T["aws"] = torch.empty(max(1, N.attn_decode_workspace_size(B, D["H"], D["dv"], D["k"] + D["W"])),
                                   dtype=torch.uint8, device=device)
    if kind in ("hca_decode", "hybrid_pair"):
        p = "h_" if kind == "hybrid_pair" else ""
        if "win_slot" in D and "win_slot" not in T:
            T["win_slot"] = torch.full((B,), D["win_slot"], **i32)
        Nh = D["Nh"] if p else D["N"]
        T[p + "entry0"] = torch.full((B,), D["entry0_h"] if p else D["entry0"], **i32)
        T[p + "n_entries"] = torch.full((B,), Nh, **i32)
        T[p + "win_len"] = torch.full((B,), D["W"], **i32)
        T[p + "out"] = torch.empty(B, 1, D["H"], D["dv"], dtype=lat, device=device)
        T[p + "lse"] = torch.empty(B, 1, D["H"], dtype=torch.float32, device=device)
        T[p + "aws"] = torch.empty(max(1, N.attn_decode_workspace_size(B, D["H"], D["dv"], Nh + D["W"])),
                                   dtype=torch.uint8, device=device)
    return T


def _ifmt(D):
    return {"f32": N.CSA_IFMT_F32, "e4m3": N.CSA_IFMT_E4M3, "mxfp4": N.CSA_IFMT_MXFP4}[D["ifmt"]]


_SIDE = {}


def _side_stream(device):
    """A second stream per device for work that is independent of the main chain."""
    key = torch.device(device).index
    if key not in _SIDE:
        _SIDE[key] = torch.cuda.Stream(device=device)
    return _SIDE[key]


def _decode_append(T, D, stream):
    """The decode token's appends in one launch: the block it completes pooled into the
    cache, the indexer key of that block, and its raw latent into the window ring (the key
    is read by the indexer, so this runs before it)."""
    keys = (T["CaI"], T["CbI"], T["ZaI"], T["ZbI"], T["BaI"], T["BbI"], T["prev_CbI"], T["prev_ZbI"], T["kI"],
            T["kI_scale"], _ifmt(D))
    N.csa_decode_append(T["Ca"], T["Cb"], T["Za"], T["Zb"], T["Ba"], T["Bb"], T["prev_Cb"], T["prev_Zb"],
                        T["entry0"], T["cache"], keys=keys, window=(T["raw_new"], T["win"], T["win_slot"]),
                        stream=stream)


def _csa_layer(T, D, stream, attend):
    """One CSA layer.  A decode token with its indexer activations and raw latent: one
    launch appends the cache entry, its key and the window row, then the indexer and the
    attention.  Otherwise the compressor's cache append and the lightning indexer are
    independent (the indexer scores the given indexer keys; the new cache entry is read
    only by the attention), so the append runs on a side stream while the indexer runs on
    the main one; the attention waits for both."""
    main = stream if stream is not None else torch.cuda.current_stream()
    if "CaI" in T:
        _decode_append(T, D, main)
        N.lightning_index(T["qI"], T.get("qI_scale"), T["w"], T["kI"], T.get("kI_scale"), T["n_entries"],
                          T["q_pos"], D["k"], _ifmt(D), T["idx"], T["iws"], m=D["m"], stream=main)
        attend(main)
        return
    side = _side_stream(main.device)
    fork = torch.cuda.Event()
    fork.record(main)
    side.wait_event(fork)
    N.csa_compress(T["Ca"], T["Cb"], T["Za"], T["Zb"], T["Ba"], T["Bb"], T["prev_Cb"], T["prev_Zb"],
                   T["entry0"], T["cache"], m=D["m"], stream=side)
    join = torch.cuda.Event()
    join.record(side)
    N.lightning_index(T["qI"], T.get("qI_scale"), T["w"], T["kI"], T.get("kI_scale"), T["n_entries"], T["q_pos"],
                      D["k"], _ifmt(D), T["idx"], T["iws"], m=D["m"], stream=main)
    main.wait_event(join)
    attend(main)


def csa_decode_step(T, D, stream=None):
    _csa_layer(T, D, stream, lambda st: N.sparse_attn_decode(
        T["q"][:, 0], T["cache"], T["idx"][:, 0], T["win"], T["win_len"], T["sink"], D["sm_scale"], D["dv"],
        T["out"][:, 0], T["lse"][:, 0], T["aws"], stream=st))


def hca_decode_step(T, D, stream=None, prefix=""):
    """The fresh chunk's compression and the dense attention as one call (the attention
    streams the other entries while the compression runs); the token's raw latent, when
    given, goes into the window ring first."""
    p = prefix
    if p + "raw_new" in T:
        N.window_append(T[p + "raw_new"], T[p + "win"], T["win_slot"], stream=stream)
    N.hca_compress_attn_decode(T[p + "C"], T[p + "Z"], T[p + "bias"], T[p + "entry0"], T[p + "q"][:, 0],
                               T[p + "cache"], T[p + "n_entries"], T[p + "win"], T[p + "win_len"], T[p + "sink"],
                               D["sm_scale"], D["dv"], T[p + "out"][:, 0], T[p + "lse"][:, 0], T[p + "aws"],
                               m_prime=D["m_prime"], stream=stream)


def csa_prefill_step(T, D, stream=None):
    _csa_layer(T, D, stream, lambda st: N.sparse_attn_prefill(
        T["q"], T["q_pos"], T["cache"], T["idx"], T["raw"], T["raw_pos0"], D["W"], T["sink"], D["sm_scale"], D["dv"],
        T["out"], T["lse"], stream=st))


def hybrid_pair_step(T, D, stream=None):
    csa_decode_step(T, D, stream)
    hca_decode_step(T, D, stream, prefix="h_")


STEPS = {"csa_decode": csa_decode_step, "hca_decode": hca_decode_step, "csa_prefill": csa_prefill_step,
         "hybrid_pair": hybrid_pair_step}


def run_step(kind, T, D, stream=None):
    STEPS[kind](T, D, stream)
