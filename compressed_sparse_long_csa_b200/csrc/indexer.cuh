// Internal arguments of the indexer / top-k kernels.
#pragma once
#include "common.cuh"

namespace csa {

struct IndexerArgs {
  const void* qI;
  const void* qI_scale;
  const float* w;
  const void* kI;
  const void* kI_scale;
  const int32_t* n_entries;   // [B]
  const int32_t* q_pos;       // [B*Tq]
  int m;
  int B, Tq, H_I, d_I;
  int64_t n_max;
  int k;
  int ifmt;
  float* scores;              // workspace [B*Tq, ld] fp32 scores
  int64_t ld;
  unsigned* knmax;            // workspace [B]: bits of max_s ||k_s||_2 (dequantised)
  unsigned* keyrange;         // workspace [B*Tq][2]: max order key, max of ~order key (= ~min) of the row's scores
  int kpart;                  // > 0: knmax [B*Tq][kpart] and keyrange [B*Tq][kpart][2] hold one partial per
                              // (row, entry split), each written by its scoring CTA (nothing to zero), and
                              // the scoring kernel may overlap a preceding decode append (it waits for it
                              // before the tile of each row's newest entry); 0: one atomic slot each
  int32_t* idx_out;           // [B*Tq, k]
  float* score_out;           // [B*Tq, k] or null
  unsigned* err;
  float eps_dot;              // bound on |fp32 dot - exact| / (||q|| ||k||) of the scoring path
  int score_bf16;             // 1: scores are rounded to bf16 before they are stored (lightning_index_bf16)
  // decode rows (Tq <= 3) only, else null: the histogram-seeded selection (select_hist.cu)
  unsigned* hist;             // [B*Tq][4096] coarse score histogram (order key >> 20), zeroed per call
  unsigned* fhist;            // [B*Tq][65536] fine score histogram (order key >> 16), zeroed per call
  unsigned* counters;         // [B*Tq][256]: certain entries, CTAs done, overflow, per-CTA band counts; zeroed
  unsigned* bitmap;           // [B*Tq][ld/32] certain entries
  void* cand;                 // [B*Tq][ld] band entries, 16 bytes each (order key, entry id, exact score)
  // prefill rows of the streaming selection (indexer_tc.cu, select_row.cu), else null:
  uint2* stream_cand;         // [B*Tq][IDX_STREAM_CAP] (order key, entry id) of each row's candidates
  uint4* stream_meta;         // [B*Tq]: candidates, threshold key, U (float bits), key-norm bound (float bits)
};

// Candidates one prefill row keeps while it is scored (the streaming selection).
constexpr int IDX_STREAM_CAP = 2048;
constexpr int IDX_STREAM_KMAX = 1024;        // largest k the streaming selection takes

// Entries of one selection row: n_valid[row] (topk_select), else the indexer's
// eligibility min(n_entries[b], (q_pos[row] + 1) / m) when q_pos is set, else n_cap;
// always clamped to [0, n_cap].
struct RowCount {
  const int32_t* n_valid = nullptr;
  const int32_t* q_pos = nullptr;
  const int32_t* n_entries = nullptr;
  int m = 1, Tq = 1;
  __device__ __forceinline__ int operator()(int row, int64_t n_cap) const {
    int n = (int)(n_cap < 0x7fffffff ? n_cap : 0x7fffffff);
    if (n_valid) {
      n = n_valid[row];
    } else if (q_pos) {
      const int pos = q_pos[row];
      const int ne = pos < 0 ? 0 : (pos + 1) / m;
      const int nb = n_entries[row / Tq];
      n = ne < nb ? ne : nb;
    }
    if ((int64_t)n > n_cap) n = (int)n_cap;
    return n < 0 ? 0 : n;
  }
};

__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// The key-norm bound of row `row` (sequence b) and its scores' order-key range (max key,
// max of ~key), from the per-split partials when kpart > 0.
__device__ __forceinline__ float load_knmax(const IndexerArgs& a, int row, int b) {
  if (a.kpart == 0) return __uint_as_float(__ldcg(a.knmax + b));
  uint32_t m = 0u;
  for (int s = 0; s < a.kpart; ++s) m = max(m, __ldcg(a.knmax + (size_t)row * a.kpart + s));
  return __uint_as_float(m);
}
__device__ __forceinline__ void load_keyrange(const IndexerArgs& a, int row, uint32_t* mx, uint32_t* nmn) {
  if (a.kpart == 0) {
    *mx = __ldcg(a.keyrange + 2 * (size_t)row);
    *nmn = __ldcg(a.keyrange + 2 * (size_t)row + 1);
    return;
  }
  uint32_t x = 0u, y = 0u;
  for (int s = 0; s < a.kpart; ++s) {
    x = max(x, __ldcg(a.keyrange + 2 * ((size_t)row * a.kpart + s)));
    y = max(y, __ldcg(a.keyrange + 2 * ((size_t)row * a.kpart + s) + 1));
  }
  *mx = x;
  *nmn = y;
}

// Number of entries visible to query row `row` (= b*Tq + t): all m sources <= pos.
__device__ __forceinline__ int row_eligible(const IndexerArgs& a, int row) {
  const int b = row / a.Tq;
  const int pos = a.q_pos[row];
  int ne = pos < 0 ? 0 : (pos + 1) / a.m;
  int n = a.n_entries[b];
  if ((int64_t)n > a.n_max) n = (int)a.n_max;
  if (n < 0) n = 0;
  return ne < n ? ne : n;
}

// Per-thread running order-key range of the scores a thread writes (flushed once, at
// the end of a kernel, by flush_key_range).
struct KeyRange {
  uint32_t mx = 0u, nmn = 0u;           // max key, max of ~key (= ~min key)
  __device__ __forceinline__ void add(float score) {
    const uint32_t k = f32_order_key(score);
    mx = max(mx, k);
    nmn = max(nmn, ~k);
  }
};
// Merge a warp's ranges for `row` into the workspace (one atomic pair per warp; all 32
// lanes call; lanes that recorded nothing hold zeros, which change nothing).
__device__ __forceinline__ void flush_key_range(unsigned* keyrange, int row, const KeyRange& r) {
  const uint32_t mx = __reduce_max_sync(0xffffffffu, r.mx);
  const uint32_t mn = __reduce_max_sync(0xffffffffu, r.nmn);
  if ((threadIdx.x & 31) == 0 && (mx | mn) != 0u) {
    atomicMax(keyrange + 2 * (size_t)row, mx);
    atomicMax(keyrange + 2 * (size_t)row + 1, mn);
  }
}

// Record the order-key range of a warp's scores for `row` (one atomic pair per warp).
// Lanes without a score pass valid = false.  All 32 lanes must call.
__device__ __forceinline__ void record_key_range(unsigned* keyrange, int row, float score, bool valid) {
  const uint32_t key = f32_order_key(score);
  const uint32_t mx = __reduce_max_sync(0xffffffffu, valid ? key : 0u);
  const uint32_t mn = __reduce_max_sync(0xffffffffu, valid ? ~key : 0u);
  const bool any = __any_sync(0xffffffffu, valid);
  if (any && (threadIdx.x & 31) == 0) {
    atomicMax(keyrange + 2 * (size_t)row, mx);
    atomicMax(keyrange + 2 * (size_t)row + 1, mn);
  }
}

cudaError_t launch_indexer_scores_cuda_core(const IndexerArgs& a, cudaStream_t st);
cudaError_t launch_indexer_scores_tc(IndexerArgs& a, cudaStream_t st, bool* used);   // sets a.eps_dot
cudaError_t launch_indexer_select(const IndexerArgs& a, cudaStream_t st);
cudaError_t launch_topk_select(const float* scores, int64_t ld, RowCount rc, int R, int64_t n,
                               int k, int32_t* idx_out, cudaStream_t st, unsigned* err);
// Cluster paths (select.cu); cudaErrorNotSupported when a row does not fit one cluster.
cudaError_t launch_indexer_select_cluster(const IndexerArgs& a, cudaStream_t st);
// Histogram-seeded selection of decode rows (select_hist.cu); cudaErrorNotSupported when
// the scoring path wrote no histogram.
cudaError_t launch_indexer_select_hist(const IndexerArgs& a, cudaStream_t st);
// One-CTA-per-row selection of decode rows over the staged fp32 scores (select_row.cu);
// cudaErrorNotSupported for other shapes.
cudaError_t launch_indexer_select_row(const IndexerArgs& a, cudaStream_t st);
// The exact selection of prefill rows from the candidates the streaming scoring kernel kept
// (select_row.cu, one CTA per row).
cudaError_t launch_indexer_select_stream(const IndexerArgs& a, cudaStream_t st);
// Whether the streaming scoring + selection takes these rows (E4M3 keys of width 128, 64
// heads, at least four queries per sequence, a grid that fills the GPU, k small enough).
bool indexer_stream_applies(const IndexerArgs& a);
// knmax[b] = the largest key norm of sequence b (E4M3 keys of width 128; knmax zeroed before).
cudaError_t launch_key_norm_max(const IndexerArgs& a, cudaStream_t st);
int64_t indexer_select_row_max_entries();
// Rows longer than one CTA stages: one cluster per row over chunks of it (select_row.cu).
// indexer_select_dist_clusters: its cluster size for these rows, 0 when it does not apply.
int indexer_select_dist_clusters(const IndexerArgs& a);
cudaError_t launch_indexer_select_dist(const IndexerArgs& a, cudaStream_t st);
cudaError_t launch_topk_select_cluster(const float* scores, int64_t ld, RowCount rc, int R, int64_t n,
                                       int k, int32_t* idx_out, cudaStream_t st);

}  // namespace csa
