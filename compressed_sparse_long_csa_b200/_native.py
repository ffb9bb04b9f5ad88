"""ctypes binding of libcsa_b200.so (argument marshalling only)."""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libcsa_b200.so")
if not os.path.exists(lib_path):
    raise ImportError(f"{lib_path} is missing: build it with `python -m compressed_sparse_long_csa_b200.build`")
lib = C.CDLL(lib_path)

CSA_F32, CSA_BF16 = 0, 1
CSA_IFMT_F32, CSA_IFMT_E4M3, CSA_IFMT_MXFP4 = 0, 1, 2

_vp, _i32, _i64, _f32, _sz = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t

_SIGS = {
    "csa_abi_version": ([], _i32),
    "csa_status_string": ([_i32], C.c_char_p),
    "csa_read_device_error": ([_vp, C.POINTER(C.c_uint32)], _i32),
    "csa_launch_count": ([], C.c_uint64),
    "csa_wait_probe": ([C.c_uint64, _vp], _i32),
    "csa_tensor_peak_probe": ([_i32, _i32, _vp], _i32),
    "csa_compress": ([_vp] * 10 + [_i64, _i32, _i32, _i32, _i32, _i32, _vp], _i32),
    "csa_compress_kv8": ([_vp] * 10 + [_i64, _i32, _i32, _i32, _i32, _i32, _vp], _i32),
    "csa_decode_append": ([_vp] * 10 + [_i64, _i32] + [_vp] * 10 + [_i32, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _vp], _i32),
    "window_append": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp], _i32),
    "index_key_compress": ([_vp] * 11 + [_i64, _i32, _i32, _i32, _i32, _i32, _i32, _vp], _i32),
    "shard_topk_merge": ([_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp], _i32),
    "attn_merge_shards": ([_vp, _vp, _i32, _i64, _i32, _i32, _vp, _vp, _vp], _i32),
    "grouped_out_proj_workspace_size": ([_i32, _i32, _i32, _i32], _sz),
    "grouped_out_proj": ([_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp], _i32),
    "hca_compress": ([_vp] * 5 + [_i64, _i32, _i32, _i32, _i32, _i32, _vp], _i32),
    "lightning_index_workspace_size": ([_i32, _i32, _i64, _i32], _sz),
    "lightning_index_workspace_size_exact": ([_i32, _i32, _i64, _i32, _i32, _i32, _i32], _sz),
    "lightning_index": ([_vp] * 7 + [_i32, _i32, _i32, _i32, _i32, _i64, _i32, _i32, _vp, _vp, _vp, _sz, _vp], _i32),
    "lightning_index_bf16": ([_vp] * 7 + [_i32, _i32, _i32, _i32, _i32, _i64, _i32, _i32, _vp, _vp, _sz, _vp], _i32),
    "topk_select_workspace_size": ([_i32, _i64, _i32], _sz),
    "topk_select": ([_vp, _i64, _vp, _i32, _i64, _i32, _vp, _vp, _sz, _vp], _i32),
    "attn_decode_workspace_size": ([_i32, _i32, _i32, _i64], _sz),
    "sparse_attn_decode": ([_vp] * 6 + [_i32, _i32, _i32, _i32, _i64, _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp], _i32),
    "hca_attn_decode": ([_vp] * 6 + [_i32, _i32, _i32, _i32, _i64, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp], _i32),
    "sparse_attn_decode_kv8": ([_vp] * 6 + [_i32, _i32, _i32, _i32, _i64, _i32, _i32, _f32, _vp, _vp, _vp, _sz, _vp], _i32),
    "hca_attn_decode_kv8": ([_vp] * 6 + [_i32, _i32, _i32, _i32, _i64, _i32, _f32, _vp, _vp, _vp, _sz, _vp], _i32),
    "hca_compress_attn_decode": ([_vp] * 4 + [_i32, _i32] + [_vp] * 6 + [_i32, _i32, _i32, _i32, _i64, _i32, _f32, _i32,
                                                                      _vp, _vp, _vp, _sz, _vp], _i32),
    "sparse_attn_decode_noalloc": ([_vp] * 6 + [_i32, _i32, _i32, _i32, _i64, _i32, _i32, _f32, _i32, _vp, _vp, _vp], _i32),
    "sparse_attn_prefill": ([_vp] * 5 + [_i64, _vp, _vp] + [_i32] * 5 + [_i64, _i32, _i32, _f32, _i32, _vp, _vp, _vp, _sz, _vp], _i32),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class CsaError(RuntimeError):
    pass


def _check(status: int, name: str):
    if status != 0:
        raise CsaError(f"{name}: {lib.csa_status_string(status).decode()}")


def _p(t):
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t):
    return CSA_BF16 if t.dtype == torch.bfloat16 else CSA_F32


def csa_decode_append(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, entry0, cache, keys=None, window=None, stream=None):
    """One decode step's appends in one launch (see csa.h).  keys = (CaI, CbI, ZaI, ZbI, BaI,
    BbI, prev_CbI, prev_ZbI, kI, kI_scale, ifmt) or None; window = (raw_new, win, win_slot) or None."""
    B, _, d = Ca.shape
    kp = [None] * 10
    d_I, ifmt = 0, CSA_IFMT_E4M3
    if keys is not None:
        kp = [_p(t) for t in keys[:10]]
        d_I, ifmt = keys[0].shape[-1], keys[10]
    raw_new, win, slot, W = None, None, None, 0
    if window is not None:
        raw_new, win, slot = window
        W = win.shape[1]
    _check(lib.csa_decode_append(_p(Ca), _p(Cb), _p(Za), _p(Zb), _p(Ba), _p(Bb), _p(prev_Cb), _p(prev_Zb), _p(entry0),
                                 _p(cache), cache.shape[1], d, *kp, d_I, ifmt, _p(raw_new), _p(win), _p(slot), W, B,
                                 _dtype_code(Ca), _stream(stream)), "csa_decode_append")


def window_append(raw_new, win, win_slot, stream=None):
    B, W, d = win.shape
    _check(lib.window_append(_p(raw_new), _p(win), _p(win_slot), B, W, d, _dtype_code(win), _stream(stream)),
           "window_append")


def wait_probe(limit_ns: int, stream=None):
    """One kernel whose wait can never end, bounded by limit_ns (sets CSA_DEVERR_TIMEOUT)."""
    _check(lib.csa_wait_probe(int(limit_ns), _stream(stream)), "csa_wait_probe")


def tensor_peak_probe(ifmt, iters, stream=None):
    """Dense MMA rate probe at the indexer's operand formats (see csa_tensor_peak_probe)."""
    _check(lib.csa_tensor_peak_probe(int(ifmt), int(iters), _stream(stream)), "csa_tensor_peak_probe")


def launch_count() -> int:
    """Kernels the library has enqueued in this process (a captured launch counts once)."""
    return int(lib.csa_launch_count())


def read_device_error(stream=None) -> int:
    v = C.c_uint32(0)
    _check(lib.csa_read_device_error(_stream(stream), C.byref(v)), "csa_read_device_error")
    return int(v.value)


def csa_compress(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, entry0, cache, m=4, stream=None):
    B, T_new, d = Ca.shape
    _check(lib.csa_compress(_p(Ca), _p(Cb), _p(Za), _p(Zb), _p(Ba), _p(Bb), _p(prev_Cb), _p(prev_Zb),
                            _p(entry0), _p(cache), cache.shape[1], B, T_new, d, m, _dtype_code(Ca),
                            _stream(stream)), "csa_compress")


def index_key_compress(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, entry0, kI, kI_scale, ifmt, m=4, stream=None):
    B, T_new, d_I = Ca.shape
    _check(lib.index_key_compress(_p(Ca), _p(Cb), _p(Za), _p(Zb), _p(Ba), _p(Bb), _p(prev_Cb), _p(prev_Zb),
                                  _p(entry0), _p(kI), _p(kI_scale), kI.shape[1], B, T_new, d_I, m,
                                  _dtype_code(Ca), ifmt, _stream(stream)), "index_key_compress")


def shard_topk_merge(idx_parts, score_parts, bounds, local_idx_out, stream=None):
    """idx_parts / score_parts [G, R, k]; bounds [G+1] int32; local_idx_out [G, R, k]."""
    G, R, k = idx_parts.shape
    _check(lib.shard_topk_merge(_p(idx_parts), _p(score_parts), _p(bounds), G, R, k, _p(local_idx_out),
                                _stream(stream)), "shard_topk_merge")


def attn_merge_shards(o_parts, lse_parts, out, lse_out=None, stream=None):
    """o_parts [G, rows, dv] (any leading shape flattened to rows); lse_parts [G, rows]."""
    G = o_parts.shape[0]
    dv = o_parts.shape[-1]
    rows = o_parts[0].numel() // dv
    _check(lib.attn_merge_shards(_p(o_parts), _p(lse_parts), G, rows, dv, _dtype_code(o_parts), _p(out),
                                 _p(lse_out), _stream(stream)), "attn_merge_shards")


def grouped_out_proj_workspace_size(T, g, d_mid, d):
    return lib.grouped_out_proj_workspace_size(T, g, d_mid, d)


def grouped_out_proj(o, W1, W2, g, u, y, workspace=None, stream=None):
    """o [T, H, dv] bf16; W1 [g*d_mid, (H/g)*dv]; W2 [d, g*d_mid]; writes u [T, g*d_mid], y [T, d]."""
    T, H, dv = o.shape
    d_mid = W1.shape[0] // g
    d = W2.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.grouped_out_proj(_p(o), T, H, dv, g, d_mid, _p(W1), _p(W2), d, _p(u), _p(y), _p(workspace), ws_bytes,
                                _stream(stream)), "grouped_out_proj")


def csa_compress_kv8(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, entry0, cache8, m=4, stream=None):
    """cache8: [B, n_max, 656] uint8 FP8 rows (see csa.h)."""
    B, T_new, d = Ca.shape
    _check(lib.csa_compress_kv8(_p(Ca), _p(Cb), _p(Za), _p(Zb), _p(Ba), _p(Bb), _p(prev_Cb), _p(prev_Zb),
                                _p(entry0), _p(cache8), cache8.shape[1], B, T_new, d, m, _dtype_code(Ca),
                                _stream(stream)), "csa_compress_kv8")


def hca_compress(C_, Z, bias, entry0, cache, m_prime=128, stream=None):
    B, T_new, d = C_.shape
    _check(lib.hca_compress(_p(C_), _p(Z), _p(bias), _p(entry0), _p(cache), cache.shape[1], B, T_new, d,
                            m_prime, _dtype_code(C_), _stream(stream)), "hca_compress")


def lightning_index_workspace_size(B, Tq, n_max, k):
    return int(lib.lightning_index_workspace_size(B, Tq, n_max, k))


def lightning_index_workspace_size_exact(B, Tq, n_max, k, ifmt, H_I, d_I):
    return int(lib.lightning_index_workspace_size_exact(B, Tq, n_max, k, ifmt, H_I, d_I))


def lightning_index(qI, qI_scale, w, kI, kI_scale, n_entries, q_pos, k, ifmt, idx_out, workspace,
                    score_out=None, m=4, stream=None):
    B, Tq, H_I = w.shape
    n_max = kI.shape[1]
    d_I = qI.shape[-1] * (2 if ifmt == CSA_IFMT_MXFP4 else 1)
    _check(lib.lightning_index(_p(qI), _p(qI_scale), _p(w), _p(kI), _p(kI_scale), _p(n_entries), _p(q_pos), m,
                               B, Tq, H_I, d_I, n_max, k, ifmt, _p(idx_out), _p(score_out), _p(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)), "lightning_index")


def lightning_index_bf16(qI, qI_scale, w, kI, kI_scale, n_entries, q_pos, k, ifmt, idx_out, workspace, m=4,
                         stream=None):
    B, Tq, H_I = w.shape
    n_max = kI.shape[1]
    d_I = qI.shape[-1] * (2 if ifmt == CSA_IFMT_MXFP4 else 1)
    _check(lib.lightning_index_bf16(_p(qI), _p(qI_scale), _p(w), _p(kI), _p(kI_scale), _p(n_entries), _p(q_pos), m,
                                    B, Tq, H_I, d_I, n_max, k, ifmt, _p(idx_out), _p(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "lightning_index_bf16")


def topk_select(scores, n_valid, k, idx_out, stream=None):
    R, n = scores.shape
    _check(lib.topk_select(_p(scores), scores.stride(0), _p(n_valid), R, n, k, _p(idx_out), None, 0,
                           _stream(stream)), "topk_select")


def attn_decode_workspace_size(B, H, d_v, rows_max):
    return int(lib.attn_decode_workspace_size(B, H, d_v, rows_max))


def _ws(workspace):
    if workspace is None:
        return None, 0
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def sparse_attn_decode(q, cache, idx, win, win_len, sink, sm_scale, d_v, out, lse=None, workspace=None,
                       stream=None):
    B, H, d_k = q.shape
    W = win.shape[1] if win is not None else 0
    k = idx.shape[1] if idx is not None else 0
    wp, wb = _ws(workspace)
    _check(lib.sparse_attn_decode(_p(q), _p(cache), _p(idx), _p(win), _p(win_len), _p(sink), B, H, d_k, d_v,
                                  cache.shape[1], k, W, sm_scale, _dtype_code(q), _p(out), _p(lse), wp, wb,
                                  _stream(stream)), "sparse_attn_decode")


def hca_attn_decode(q, cache, n_entries, win, win_len, sink, sm_scale, d_v, out, lse=None, workspace=None,
                    stream=None):
    B, H, d_k = q.shape
    W = win.shape[1] if win is not None else 0
    wp, wb = _ws(workspace)
    _check(lib.hca_attn_decode(_p(q), _p(cache), _p(n_entries), _p(win), _p(win_len), _p(sink), B, H, d_k, d_v,
                               cache.shape[1], W, sm_scale, _dtype_code(q), _p(out), _p(lse), wp, wb,
                               _stream(stream)), "hca_attn_decode")


def sparse_attn_decode_kv8(q, cache8, idx, win, win_len, sink, sm_scale, d_v, out, lse=None, workspace=None,
                           stream=None):
    """cache8: [B, n_max, 656] uint8 FP8 rows (see csa.h)."""
    B, H, d_k = q.shape
    W = win.shape[1] if win is not None else 0
    k = idx.shape[1] if idx is not None else 0
    wp, wb = _ws(workspace)
    _check(lib.sparse_attn_decode_kv8(_p(q), _p(cache8), _p(idx), _p(win), _p(win_len), _p(sink), B, H, d_k, d_v,
                                      cache8.shape[1], k, W, sm_scale, _p(out), _p(lse), wp, wb, _stream(stream)),
           "sparse_attn_decode_kv8")


def hca_attn_decode_kv8(q, cache8, n_entries, win, win_len, sink, sm_scale, d_v, out, lse=None, workspace=None,
                        stream=None):
    B, H, d_k = q.shape
    W = win.shape[1] if win is not None else 0
    wp, wb = _ws(workspace)
    _check(lib.hca_attn_decode_kv8(_p(q), _p(cache8), _p(n_entries), _p(win), _p(win_len), _p(sink), B, H, d_k,
                                   d_v, cache8.shape[1], W, sm_scale, _p(out), _p(lse), wp, wb, _stream(stream)),
           "hca_attn_decode_kv8")


def hca_compress_attn_decode(C_, Z, bias, entry0, q, cache, n_entries, win, win_len, sink, sm_scale, d_v, out,
                             lse=None, workspace=None, m_prime=128, stream=None):
    """hca_compress of the fresh chunk (C_, Z) then hca_attn_decode, as one call."""
    B, H, d_k = q.shape
    T_new = C_.shape[1]
    W = win.shape[1] if win is not None else 0
    wp, wb = _ws(workspace)
    _check(lib.hca_compress_attn_decode(_p(C_), _p(Z), _p(bias), _p(entry0), T_new, m_prime, _p(q), _p(cache),
                                        _p(n_entries), _p(win), _p(win_len), _p(sink), B, H, d_k, d_v, cache.shape[1],
                                        W, sm_scale, _dtype_code(q), _p(out), _p(lse), wp, wb, _stream(stream)),
           "hca_compress_attn_decode")


def sparse_attn_prefill(q, q_pos, cache, idx, raw, raw_pos0, W, sink, sm_scale, d_v, out, lse=None,
                        workspace=None, stream=None):
    B, Tq, H, d_k = q.shape
    k = idx.shape[2] if idx is not None else 0
    wp, wb = _ws(workspace)
    _check(lib.sparse_attn_prefill(_p(q), _p(q_pos), _p(cache), _p(idx), _p(raw), raw.shape[1], _p(raw_pos0),
                                   _p(sink), B, Tq, H, d_k, d_v, cache.shape[1], k, W, sm_scale, _dtype_code(q),
                                   _p(out), _p(lse), wp, wb, _stream(stream)), "sparse_attn_prefill")


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def sparse_attn_decode_noalloc(q, cache, idx, win, win_len, sink, sm_scale, d_v, out, lse=None, stream=None):
    """sparse_attn_decode for callers that cannot allocate: the split partials use the
    library's own fixed device buffer (NOALLOC_SCRATCH_BYTES).  Calls that overlap on
    the GPU race on that buffer; the first call on a device should precede capture."""
    B, H, d_k = q.shape
    W = win.shape[1] if win is not None else 0
    k = idx.shape[1] if idx is not None else 0
    _check(lib.sparse_attn_decode_noalloc(_p(q), _p(cache), _p(idx), _p(win), _p(win_len), _p(sink), B, H, d_k,
                                          d_v, cache.shape[1], k, W, sm_scale, _dtype_code(q), _p(out), _p(lse),
                                          _stream(stream)), "sparse_attn_decode_noalloc")
