// Internal arguments of the attention kernels.
#pragma once
#include "common.cuh"

#include <cuda_fp16.h>

namespace csa {

struct AttnArgs {
  const void* q;              // [B*Tq, H, dk]
  const void* cache;          // [B, n_max, dk]
  const int32_t* idx;         // [B*Tq, k] (sparse) or null (dense: entries 0..n_entries[b]-1)
  const int32_t* n_entries;   // [B] (dense)
  int k;                      // sparse: index slots per query; dense: unused
  const void* win;            // decode: [B, W, dk]; prefill: raw [B, t_raw, dk]
  const int32_t* win_len;     // decode: [B]
  const int32_t* q_pos;       // prefill: [B*Tq]
  const int32_t* raw_pos0;    // prefill: [B]
  int64_t t_raw;
  int W;
  int prefill;
  const float* sink;          // [H]
  int B, Tq, H, dk, dv;
  int64_t n_max;
  float sm_scale;
  void* out;                  // [B*Tq, H, dv]
  float* lse;                 // [B*Tq, H] or null
  float* part;                // split partials: [B*Tq, splits] blocks of attn_part_block(H, dv) floats
  int part_fp16;              // partial block format (see attn_part_block)
  int splits;
  int rows_per_split;         // CUDA-core path: contiguous virtual rows per split (the
                              // tensor-core path deals 64-row tiles to the splits round-robin)
  int n_seg_a;                // virtual rows in segment A (k or n_max)
  int cluster_combine;        // tensor-core path: splits merged inside a thread-block cluster
  const int32_t* dep_entry0;  // dense decode after a compression kernel in the same stream: it
  int dep_rows;               // writes rows dep_entry0[b] .. +dep_rows-1 (null: wait for it at once)
  int kv8;                    // cache rows are 656-byte FP8 rows (tensor-core kernel only)
  int idx_late;               // sparse decode: only idx may come from the preceding kernel; each
                              // split takes its tiles last to first (the window's first) and waits
                              // for that kernel just before it resolves an index (tensor-core kernel)
  unsigned* err;
};

// Floats per (query, split, head) record of the split partials: o[dv], m, l, 2 pad,
// so that every record starts on a 16-byte boundary (vector stores).
__host__ __device__ inline int attn_part_stride(int dv) { return dv + 4; }
// Floats per (query, split) block of the split partials.  Two formats fit in it:
//   0 (CUDA-core kernel): per head [H][attn_part_stride(dv)] fp32: o[dv], m, l, 2 pad;
//   1 (tensor-core kernel): o as fp16 at [dv/8][H][8] (a warp's heads store contiguous
//     16-byte pieces), each half row divided by l and by a power of two that puts its
//     largest magnitude in [0.5, 1); then per head a float4 {m, l, p_lo, p_hi}, the powers
//     of two of columns [0, dv/2) and [dv/2, dv).  o = stored * p * l.
__host__ __device__ inline size_t attn_part_block(int H, int dv) { return (size_t)H * attn_part_stride(dv); }
// format 1: offset (in halves) of values c..c+3 of head h (c a multiple of 4)
__host__ __device__ inline size_t attn_part16_val(int H, int h, int c) { return ((size_t)(c >> 3) * H + h) * 8 + (c & 7); }
// format 1: offset (in floats) of the record of head h
__host__ __device__ inline size_t attn_part16_rec(int H, int dv, int h) { return (size_t)dv * H / 2 + 4 * (size_t)h; }

// Number of virtual rows of a query: compressed segment + window segment.
__host__ __device__ inline int64_t attn_virtual_rows(const AttnArgs& a) { return (int64_t)a.n_seg_a + a.W; }

// Resolve virtual row v of query `row` to a latent row pointer (null = not a row).
template <typename T>
__device__ __forceinline__ const T* attn_row_ptr(const AttnArgs& a, int row, int v) {
  const int b = row / a.Tq;
  if (v < a.n_seg_a) {
    int e;
    if (a.idx) {
      e = a.idx[(size_t)row * a.k + v];
      if (e < 0) return nullptr;
      if ((int64_t)e >= a.n_max) { raise_err(a.err, CSA_DEVERR_INDEX); return nullptr; }
    } else {
      int n = a.n_entries[b];
      if ((int64_t)n > a.n_max) n = (int)a.n_max;
      if (v >= n) return nullptr;
      e = v;
    }
    return (const T*)a.cache + ((size_t)b * a.n_max + e) * a.dk;
  }
  const int w = v - a.n_seg_a;
  if (!a.prefill) {
    int wl = a.win_len[b];
    if (wl > a.W) wl = a.W;
    if (w >= wl) return nullptr;
    return (const T*)a.win + ((size_t)b * a.W + w) * a.dk;
  }
  const int pos = a.q_pos[row];
  const int lo = pos - a.W + 1 < 0 ? 0 : pos - a.W + 1;
  const int p = lo + w;
  if (p > pos) return nullptr;
  const int64_t r = (int64_t)p - a.raw_pos0[b];
  if (r < 0 || r >= a.t_raw) { raise_err(a.err, CSA_DEVERR_WINDOW); return nullptr; }
  return (const T*)a.win + ((size_t)b * a.t_raw + r) * a.dk;
}

// Same resolution as attn_row_ptr, as (tensor, row) for TMA: which = 0 for the cache
// ([B*n_max] rows), 1 for the window / raw buffer ([B*W] or [B*t_raw] rows), -1 when
// virtual row v of query `row` is not a row.
__device__ __forceinline__ int attn_row_coord(const AttnArgs& a, int row, int v, int* y) {
  const int b = row / a.Tq;
  if (v < a.n_seg_a) {
    int e;
    if (a.idx) {
      e = a.idx[(size_t)row * a.k + v];
      if (e < 0) return -1;
      if ((int64_t)e >= a.n_max) { raise_err(a.err, CSA_DEVERR_INDEX); return -1; }
    } else {
      int n = a.n_entries[b];
      if ((int64_t)n > a.n_max) n = (int)a.n_max;
      if (v >= n) return -1;
      e = v;
    }
    *y = (int)((int64_t)b * a.n_max + e);
    return 0;
  }
  const int w = v - a.n_seg_a;
  if (!a.prefill) {
    int wl = a.win_len[b];
    if (wl > a.W) wl = a.W;
    if (w >= wl) return -1;
    *y = b * a.W + w;
    return 1;
  }
  const int pos = a.q_pos[row];
  const int lo = pos - a.W + 1 < 0 ? 0 : pos - a.W + 1;
  const int p = lo + w;
  if (p > pos) return -1;
  const int64_t r = (int64_t)p - a.raw_pos0[b];
  if (r < 0 || r >= a.t_raw) { raise_err(a.err, CSA_DEVERR_WINDOW); return -1; }
  *y = (int)((int64_t)b * a.t_raw + r);
  return 1;
}

int attn_choose_splits(int n_queries, int H, int64_t rows, bool tc_path);
// Rows of each split (the last split takes the rest); a multiple of 64 on the tensor-core path.
int attn_rows_per_split(int64_t rows, int splits, bool tc_path);

cudaError_t launch_attention_cuda_core(AttnArgs a, int dtype, cudaStream_t st);
cudaError_t launch_attention_tc(AttnArgs a, cudaStream_t st, bool* used, bool* combined);
cudaError_t launch_attn_combine(const AttnArgs& a, int dtype, cudaStream_t st);

}  // namespace csa
