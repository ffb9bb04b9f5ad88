// KV-sharded decode of one sequence over G GPUs: the two merge steps.
//
// The compressed entries of a sequence are split into G contiguous shards, one per GPU.
// Every GPU scores its shard and keeps its local top-k with the exact scores
// (lightning_index with score_out); after an all-gather of those G x k candidates,
// shard_topk_merge selects the global top-k ("Техотчёт DeepSeek-V4 (2026)", section
// "Гибридное внимание: CSA и HCA", CSA step 2: the k largest I[t,s], ties to the lower
// entry index) and hands every GPU the ids that fall in its shard.  Every GPU then attends
// to its share (the window and the sink on GPU 0 only), and attn_merge_shards combines the
// G partial outputs by their log-sum-exp: with lse_g = log(sum over shard g's rows of
// e^{l_r}, plus e^{sink} on GPU 0) and o_g = that shard's normalised output,
//   out = sum_g e^{lse_g - L} o_g,   L = log sum_g e^{lse_g},
// which is the attention over the union of the rows (CSA step 3).
#include <cuda_bf16.h>

#include "../../include/csa.h"
#include "common.cuh"

namespace csa {
namespace {

constexpr int SM_THREADS = 512;
constexpr int SM_CAP = CSA_SHARD_MAX_CANDIDATES;   // G * k candidates per row at most
static_assert(CSA_SHARD_MAX_G <= 8, "per-shard counts cnt[] below hold G + 1 entries");

// In-place ascending bitonic sort of n (a power of two, <= SM_CAP) keys in shared memory.
__device__ void bitonic_sort(unsigned long long* key, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n / 2; i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const unsigned long long a = key[lo], b = key[hi];
        if ((a > b) == up) { key[lo] = b; key[hi] = a; }
      }
    }
  }
  __syncthreads();
}

// One CTA per query row.  Candidates: idx_parts[g][row][i] (local id, -1 = none) with
// score_parts[g][row][i]; bounds[g] is shard g's first global entry.  Key of a candidate:
// (inverted fp32 order key of the score) << 32 | global id, so that an ascending sort
// puts the larger score first and, among equal scores, the lower entry id first.
__global__ void __launch_bounds__(SM_THREADS)
shard_topk_merge_kernel(const int32_t* __restrict__ idx_parts, const float* __restrict__ score_parts,
                        const int32_t* __restrict__ bounds, int G, int R, int k, int32_t* __restrict__ local_out) {
  __shared__ unsigned long long key[SM_CAP];
  __shared__ int cnt[CSA_SHARD_MAX_G + 1];
  const int row = blockIdx.x;
  const int n = G * k;
  int np = 1;
  while (np < n) np <<= 1;
  for (int i = threadIdx.x; i < np; i += blockDim.x) {
    unsigned long long kk = ~0ull;
    if (i < n) {
      const int g = i / k, s = i - g * k;
      const size_t off = ((size_t)g * R + row) * k + s;
      const int32_t li = idx_parts[off];
      if (li >= 0) {
        const uint32_t sk = ~f32_order_key(score_parts[off]);
        kk = ((unsigned long long)sk << 32) | (uint32_t)(bounds[g] + li);
      }
    }
    key[i] = kk;
  }
  bitonic_sort(key, np);
  // the first k keys that are not padding are the selection: re-sort them by entry id
  int kp = 1;
  while (kp < k) kp <<= 1;
  for (int i = threadIdx.x; i < kp; i += blockDim.x) {
    const unsigned long long kk = i < k ? key[i] : ~0ull;
    key[i] = kk == ~0ull ? ~0ull : (kk & 0xFFFFFFFFull);
  }
  // (entries past kp are not read again)
  bitonic_sort(key, kp);
  if (threadIdx.x <= G) cnt[threadIdx.x] = 0;
  __syncthreads();
  // the selected ids of shard g form one run of the sorted list: its start is the number
  // of selected ids below bounds[g]
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    const unsigned long long v = key[i];
    if (v == ~0ull) continue;
    for (int g = 1; g <= G; ++g)
      if ((long long)v < (long long)bounds[g]) { atomicAdd(&cnt[g], 1); break; }
  }
  __syncthreads();
  // cnt[g] = selected ids in shard g-1; prefix sums give each shard's run
  for (int g = 0; g < G; ++g) {
    int start = 0;
    for (int h = 1; h <= g; ++h) start += cnt[h];
    const int c = cnt[g + 1];
    int32_t* out = local_out + ((size_t)g * R + row) * k;
    for (int i = threadIdx.x; i < k; i += blockDim.x)
      out[i] = i < c ? (int32_t)((long long)key[start + i] - bounds[g]) : -1;
  }
}

// One warp per (row, head): out = sum_g e^{lse_g - L} o_g, L = log sum_g e^{lse_g}.
template <typename T>
__global__ void __launch_bounds__(256)
attn_merge_shards_kernel(const T* __restrict__ o_parts, const float* __restrict__ lse_parts, int G, int64_t rows,
                         int dv, T* __restrict__ out, float* __restrict__ lse_out) {
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float M = -INFINITY;
  for (int g = 0; g < G; ++g) M = fmaxf(M, lse_parts[(size_t)g * rows + r]);
  float den = 0.f;
  for (int g = 0; g < G; ++g) den += M == -INFINITY ? 0.f : __expf(lse_parts[(size_t)g * rows + r] - M);
  const float L = den > 0.f ? M + __logf(den) : -INFINITY;
  for (int c = lane; c < dv; c += 32) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) {
      const float lg = lse_parts[(size_t)g * rows + r];
      const float w = L == -INFINITY ? 0.f : __expf(lg - L);
      acc = fmaf(w, Elem<T>::ld(o_parts + ((size_t)g * rows + r) * dv + c), acc);
    }
    Elem<T>::st(out + (size_t)r * dv + c, acc);
  }
  if (lane == 0 && lse_out) lse_out[r] = L;
}

}  // namespace

cudaError_t launch_shard_topk_merge(const int32_t* idx_parts, const float* score_parts, const int32_t* bounds,
                                    int G, int R, int k, int32_t* local_out, cudaStream_t st) {
  note_launch();
  shard_topk_merge_kernel<<<R, SM_THREADS, 0, st>>>(idx_parts, score_parts, bounds, G, R, k, local_out);
  return cudaGetLastError();
}

cudaError_t launch_attn_merge_shards(const void* o_parts, const float* lse_parts, int G, int64_t rows, int dv,
                                     int dtype, void* out, float* lse_out, cudaStream_t st) {
  const dim3 grid((unsigned)((rows * 32 + 255) / 256));
  note_launch();
  if (dtype == CSA_BF16)
    attn_merge_shards_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)o_parts, lse_parts, G, rows,
                                                                  dv, (__nv_bfloat16*)out, lse_out);
  else
    attn_merge_shards_kernel<float><<<grid, 256, 0, st>>>((const float*)o_parts, lse_parts, G, rows, dv,
                                                          (float*)out, lse_out);
  return cudaGetLastError();
}

}  // namespace csa
