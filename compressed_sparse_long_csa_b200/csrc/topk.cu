// Exact top-k selection of compressed entries: the single-CTA path for rows longer
// than one thread-block cluster holds (select.cu has the cluster path used otherwise).
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 2 (the indexer keeps the top-k compressed blocks;
// k = 512 / 1024 from table "Конфигурации").  Ties go to the lower entry index and
// the selected set is written in ascending index order, padded with -1.
//
// One CTA of 1024 threads per query row, scores read from global memory:
//  1. range-aware histogram passes over monotone fp32 keys give the exact k-th
//     largest fp32 score tau (MSB-first radix select as the fallback);
//  2a. topk_select: entries with key > tau are in; the first `remaining` entries
//     with key == tau (ascending index) complete the set.
//  2b. lightning_index: the fp32 scores carry a bounded error E (accumulation in the
//     scoring kernel).  Entries above tau + 2E are certainly in, entries below
//     tau - 2E certainly out; the band between is re-scored exactly in fp64 from
//     the quantised operands (FP8/FP4 products and their sums are exact in fp64)
//     and ranked by (score desc, index asc).
//  3. The chosen indices are written in ascending order.
#include "indexer.cuh"

namespace csa {

constexpr int TK_THREADS = 1024;
constexpr int TK_KMAX = 2048;
constexpr int AMB_CAP = 2048;

constexpr int HB = 2048;          // histogram bins of the range-aware select (11-bit digits)

struct TopkShared {
  uint32_t hist[HB];
  uint32_t wtot[32];
  int32_t sel[TK_KMAX];
  int32_t amb[AMB_CAP];
  double amb_s[AMB_CAP];
  double contrib[32][64];
  double kd[32][128];          // key rows being re-scored (exact fp64 values of the codes)
  double ksd[32][4];           // their scales: E4M3 row scale in [0], MXFP4 block scales in [0..3]
  double qd[64 * 129];         // query row codes as fp64 (padded rows: conflict-free per-head reads)
  float qsc[64 * 4];
  float w[64];
  uint32_t digit, remaining, n_sel, n_amb;
  uint32_t hT, hcgt, hcT, kmax_s, kmin_s;
  float U;
};

__device__ __forceinline__ int block_excl_scan_flag(bool f, uint32_t* wtot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, f);
  const int pre = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) wtot[warp] = __popc(bal);
  __syncthreads();
  int wpre = 0, tot = 0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
    const int v = (int)wtot[i];
    if (i < warp) wpre += v;
    tot += v;
  }
  __syncthreads();
  *total = tot;
  return wpre + pre;
}

// Histogram select over the range of the keys.  All keys share the bits above the
// highest bit h where kmin and kmax differ, so the digit is bits [lo, h] of the key
// (lo = max(0, h-10)): at most 2048 bins, spread over the keys' actual range.  Bins
// are counted with warp-aggregated shared-memory atomics.  Returns the bin T that
// holds the k-th largest key: key_lo..key_hi are the bin's key bounds, *c_gt the
// number of keys above the bin and *c_T the number inside it.
struct BinSel {
  uint32_t key_lo, key_hi;
  int c_gt, c_T;
  bool exact;                     // every key of the bin is the same key
};

template <typename KeyFn>
__device__ BinSel hist_select(TopkShared& sh, int n, int k, KeyFn key, uint32_t kmin, uint32_t kmax) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  BinSel r;
  const uint32_t diff = kmin ^ kmax;
  if (diff == 0u) {
    r.key_lo = r.key_hi = kmax; r.c_gt = 0; r.c_T = n; r.exact = true;
    return r;
  }
  const int h = 31 - __clz(diff);
  const int lo = h >= 10 ? h - 10 : 0;
  const uint32_t nbm = (1u << (h - lo + 1)) - 1u;
  for (int i = tid; i < HB; i += blockDim.x) sh.hist[i] = 0u;
  __syncthreads();
  const int iters = (n + (int)blockDim.x - 1) / (int)blockDim.x;
  for (int it = 0; it < iters; ++it) {
    const int i = it * blockDim.x + tid;
    const uint32_t dg = i < n ? (key(i) >> lo) & nbm : 0xFFFFFFFFu;
    const unsigned peers = __match_any_sync(0xffffffffu, dg);
    if (dg != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[dg], (uint32_t)__popc(peers));
  }
  __syncthreads();
  // suffix sums over bins: thread t owns bins 2t (lower) and 2t+1 (upper)
  const uint32_t b0 = sh.hist[2 * tid], b1 = sh.hist[2 * tid + 1];
  uint32_t v = b0 + b1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_down_sync(0xffffffffu, v, o);
    if (lane + o < 32) v += x;
  }
  if (lane == 0) sh.wtot[warp] = v;                 // warp total (suffix from lane 0)
  __syncthreads();
  uint32_t above_w = 0;
  for (int w = warp + 1; w < (int)(blockDim.x >> 5); ++w) above_w += sh.wtot[w];
  const uint32_t after = v - (b0 + b1) + above_w;  // keys in bins above this thread's pair
  const uint32_t kk = (uint32_t)k;
  if (after < kk && kk <= after + b1) { sh.hT = 2 * tid + 1; sh.hcgt = after; sh.hcT = b1; }
  if (after + b1 < kk && kk <= after + b1 + b0) { sh.hT = 2 * tid; sh.hcgt = after + b1; sh.hcT = b0; }
  __syncthreads();
  const uint32_t T = sh.hT;
  const uint32_t pre = (h + 1 >= 32) ? 0u : (kmax & ~((2u << h) - 1u));
  r.key_lo = pre | (T << lo);
  r.key_hi = r.key_lo | ((1u << lo) - 1u);
  r.c_gt = (int)sh.hcgt;
  r.c_T = (int)sh.hcT;
  r.exact = lo == 0;
  __syncthreads();
  return r;
}

// Block min / max of the keys.
template <typename KeyFn>
__device__ void key_range(TopkShared& sh, int n, KeyFn key, uint32_t* kmin, uint32_t* kmax) {
  uint32_t mx = 0u, mn = 0xFFFFFFFFu;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t x = key(i);
    mx = max(mx, x);
    mn = min(mn, x);
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  mn = __reduce_min_sync(0xffffffffu, mn);
  if (threadIdx.x == 0) { sh.kmax_s = 0u; sh.kmin_s = 0xFFFFFFFFu; }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) { atomicMax(&sh.kmax_s, mx); atomicMin(&sh.kmin_s, mn); }
  __syncthreads();
  *kmin = sh.kmin_s;
  *kmax = sh.kmax_s;
  __syncthreads();
}

// Radix select: the k-th largest key among key(0..n-1).  Returns tau; *remaining =
// how many entries equal to tau belong to the top-k.
template <typename KeyFn>
__device__ uint32_t radix_select(TopkShared& sh, int n, uint32_t k, KeyFn key, uint32_t* remaining_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0, remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) {
      const uint32_t kk = key(i);
      if ((kk & mask) == prefix) atomicAdd(&sh.hist[(kk >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8], loc = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { c[q] = sh.hist[lane * 8 + q]; loc += c[q]; }
      uint32_t incl = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += v;
      }
      uint32_t above = incl - loc;
#pragma unroll
      for (int q = 7; q >= 0; --q) {
        if (above < remaining && remaining <= above + c[q]) {
          sh.digit = (uint32_t)(lane * 8 + q);
          sh.remaining = remaining - above;
        }
        above += c[q];
      }
    }
    __syncthreads();
    prefix |= sh.digit << shift;
    mask |= 0xFFu << shift;
    remaining = sh.remaining;
    __syncthreads();
  }
  *remaining_out = remaining;
  return prefix;
}

__device__ void block_sort_asc(int32_t* v, int n_pow2) {
  for (int size = 2; size <= n_pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < (n_pow2 >> 1); t += blockDim.x) {
        const int i = (t / stride) * stride * 2 + (t % stride);
        const int j = i + stride;
        const bool asc = (i & size) == 0;
        const int32_t a = v[i], b = v[j];
        if ((a > b) == asc) { v[i] = b; v[j] = a; }
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// Sort sel[0..cnt) ascending and write k outputs (-1 padded).
__device__ void write_sorted(TopkShared& sh, int cnt, int k, int32_t* out) {
  const int np = next_pow2(cnt < 2 ? 2 : cnt);
  for (int i = cnt + threadIdx.x; i < np; i += blockDim.x) sh.sel[i] = 0x7fffffff;
  __syncthreads();
  block_sort_asc(sh.sel, np);
  for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < cnt ? sh.sel[i] : -1;
}

// ------------------------------------------------------------------ topk_select (fp32 keys)
// Exact top-k of one row held in global memory (all threads of the CTA call it).
__device__ void topk_select_global_row(TopkShared& sh, const float* S, int n, int k, int32_t* out) {
  auto key = [&](int i) { return f32_order_key(S[i]); };
  if (threadIdx.x == 0) sh.n_sel = 0;
  __syncthreads();
  uint32_t kmin, kmax;
  key_range(sh, n, key, &kmin, &kmax);
  const BinSel bs = hist_select(sh, n, k, key, kmin, kmax);
  if (bs.c_T <= AMB_CAP) {
    // keys above the bin are in; the bin's keys are ranked exactly in shared memory
    if (threadIdx.x == 0) { sh.n_sel = 0; sh.n_amb = 0; }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t x = key(i);
      if (x > bs.key_hi) {
        const uint32_t slot = atomicAdd(&sh.n_sel, 1u);
        if (slot < (uint32_t)k) sh.sel[slot] = i;
      } else if (x >= bs.key_lo) {
        const uint32_t slot = atomicAdd(&sh.n_amb, 1u);
        if (slot < AMB_CAP) sh.amb[slot] = i;
      }
    }
    __syncthreads();
    const int n_gt = min((int)sh.n_sel, k), nc = min((int)sh.n_amb, AMB_CAP), need = k - n_gt;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) sh.hist[c] = key(sh.amb[c]);   // bin keys, staged
    __syncthreads();
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
      const int ic = sh.amb[c];
      const uint32_t xc = sh.hist[c];
      int rank = 0;
      for (int j = 0; j < nc; ++j) {
        const uint32_t xj = sh.hist[j];
        rank += (xj > xc) || (xj == xc && sh.amb[j] < ic);
      }
      if (rank < need) sh.sel[n_gt + rank] = ic;
    }
    __syncthreads();
    write_sorted(sh, k, k, out);
    return;
  }
  // many keys in one bin (heavy ties): exact multi-pass radix select over the row
  if (threadIdx.x == 0) sh.n_sel = 0;
  __syncthreads();
  uint32_t remaining;
  const uint32_t tau = radix_select(sh, n, (uint32_t)k, key, &remaining);
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    if (key(i) > tau) {
      const uint32_t slot = atomicAdd(&sh.n_sel, 1u);
      if (slot < (uint32_t)k) sh.sel[slot] = i;
    }
  __syncthreads();
  const int n_gt = min((int)sh.n_sel, k);
  // ties at tau: the `remaining` lowest indices, found by an ordered pass
  int taken = 0;
  for (int base = 0; base < n && taken < (int)remaining; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const bool f = i < n && key(i) == tau;
    int tot;
    const int pos = block_excl_scan_flag(f, sh.wtot, &tot);
    if (f && taken + pos < (int)remaining) sh.sel[n_gt + taken + pos] = i;
    taken += tot;
  }
  __syncthreads();
  write_sorted(sh, k, k, out);
}

__global__ void __launch_bounds__(TK_THREADS)
topk_select_kernel(const float* __restrict__ scores, int64_t ld, RowCount rc, int64_t n_cap, int k,
                   int32_t* __restrict__ idx_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  const int row = blockIdx.x;
  const float* S = scores + (size_t)row * ld;
  const int n = rc(row, n_cap);
  int32_t* out = idx_out + (size_t)row * k;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? i : -1;
    return;
  }
  topk_select_global_row(sh, S, n, k, out);
}

// ------------------------------------------------------------------ indexer selection
// Exact fp64 score of entry s for query row `row`, computed by one warp; the head
// contributions are summed in order j = 0..H_I-1.
__device__ double rescore_entry(const IndexerArgs& a, TopkShared& sh, int row, int s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = row / a.Tq;
  const int HI = a.H_I, dI = a.d_I, nb = dI / 32;
  const size_t koff = (size_t)b * a.n_max + s;
  double* kd = sh.kd[warp];
  for (int c = lane; c < dI; c += 32) {
    float v;
    if (a.ifmt == CSA_IFMT_F32) v = ((const float*)a.kI)[koff * dI + c];
    else if (a.ifmt == CSA_IFMT_E4M3) v = e4m3_to_float(((const uint8_t*)a.kI)[koff * dI + c]);
    else {
      const uint8_t byte = ((const uint8_t*)a.kI)[koff * (dI / 2) + c / 2];
      v = e2m1_to_float((c & 1) ? (byte >> 4) : (byte & 0xF));
    }
    kd[c] = (double)v;
  }
  __syncwarp();
  double ks = 1.0;
  double kblk[4] = {1.0, 1.0, 1.0, 1.0};
  if (a.ifmt == CSA_IFMT_E4M3) ks = (double)((const float*)a.kI_scale)[koff];
  if (a.ifmt == CSA_IFMT_MXFP4)
    for (int bb = 0; bb < nb; ++bb) kblk[bb] = (double)ue8m0_to_float(((const uint8_t*)a.kI_scale)[koff * nb + bb]);
  for (int j = lane; j < HI; j += 32) {
    const double* qj = sh.qd + j * 129;
    double D;
    if (a.ifmt == CSA_IFMT_MXFP4) {
      D = 0.0;
      for (int bb = 0; bb < nb; ++bb) {
        double part = 0.0;
        for (int c = bb * 32; c < bb * 32 + 32; ++c) part = fma(qj[c], kd[c], part);
        D += ((double)sh.qsc[j * nb + bb] * kblk[bb]) * part;
      }
    } else {
      double raw = 0.0;
      for (int c = 0; c < dI; ++c) raw = fma(qj[c], kd[c], raw);
      D = (a.ifmt == CSA_IFMT_E4M3) ? ((double)sh.qsc[j] * ks) * raw : raw;
    }
    sh.contrib[warp][j] = (double)sh.w[j] * fmax(D, 0.0);
  }
  __syncwarp();
  double S = 0.0;
  if (lane == 0)
    for (int j = 0; j < HI; ++j) S += sh.contrib[warp][j];
  S = __shfl_sync(0xffffffffu, S, 0);
  __syncwarp();
  return S;
}

// Exact fp64 scores of the entries ids[0..n) of query row `row`, into out[0..n),
// computed by the whole CTA: key rows are staged 32 at a time, then every thread
// computes (candidate, head) dot products with four independent accumulators (the
// partial sums of FP8 / FP4 products are exact in fp64, so their order does not
// matter), and one thread per candidate adds the head terms in order j = 0..H_I-1.
__device__ void rescore_block(const IndexerArgs& a, TopkShared& sh, int row, const int32_t* ids, int n,
                              double* out) {
  const int b = row / a.Tq;
  const int HI = a.H_I, dI = a.d_I, nb = dI / 32;
  for (int base = 0; base < n; base += 32) {
    const int cnt = min(32, n - base);
    for (int i = threadIdx.x; i < cnt * dI; i += blockDim.x) {
      const int c = i / dI, d = i - c * dI;
      const size_t koff = (size_t)b * a.n_max + ids[base + c];
      float v;
      if (a.ifmt == CSA_IFMT_F32) v = ((const float*)a.kI)[koff * dI + d];
      else if (a.ifmt == CSA_IFMT_E4M3) v = e4m3_to_float(((const uint8_t*)a.kI)[koff * dI + d]);
      else {
        const uint8_t byte = ((const uint8_t*)a.kI)[koff * (dI / 2) + d / 2];
        v = e2m1_to_float((d & 1) ? (byte >> 4) : (byte & 0xF));
      }
      sh.kd[c][d] = (double)v;
    }
    for (int c = threadIdx.x; c < cnt; c += blockDim.x) {
      const size_t koff = (size_t)b * a.n_max + ids[base + c];
      if (a.ifmt == CSA_IFMT_E4M3) sh.ksd[c][0] = (double)((const float*)a.kI_scale)[koff];
      else if (a.ifmt == CSA_IFMT_MXFP4)
        for (int bb = 0; bb < nb; ++bb) sh.ksd[c][bb] = (double)ue8m0_to_float(((const uint8_t*)a.kI_scale)[koff * nb + bb]);
      else sh.ksd[c][0] = 1.0;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < cnt * HI; p += blockDim.x) {
      const int c = p / HI, j = p - c * HI;
      const double* qj = sh.qd + j * 129;
      const double* kc = sh.kd[c];
      double D;
      if (a.ifmt == CSA_IFMT_MXFP4) {
        D = 0.0;
        for (int bb = 0; bb < nb; ++bb) {
          double p0 = 0.0, p1 = 0.0, p2 = 0.0, p3 = 0.0;
#pragma unroll
          for (int d = bb * 32; d < bb * 32 + 32; d += 4) {
            p0 = fma(qj[d], kc[d], p0); p1 = fma(qj[d + 1], kc[d + 1], p1);
            p2 = fma(qj[d + 2], kc[d + 2], p2); p3 = fma(qj[d + 3], kc[d + 3], p3);
          }
          D += ((double)sh.qsc[j * nb + bb] * sh.ksd[c][bb]) * ((p0 + p1) + (p2 + p3));
        }
      } else {
        double p0 = 0.0, p1 = 0.0, p2 = 0.0, p3 = 0.0;
        for (int d = 0; d < dI; d += 4) {
          p0 = fma(qj[d], kc[d], p0); p1 = fma(qj[d + 1], kc[d + 1], p1);
          p2 = fma(qj[d + 2], kc[d + 2], p2); p3 = fma(qj[d + 3], kc[d + 3], p3);
        }
        const double raw = (p0 + p1) + (p2 + p3);
        D = (a.ifmt == CSA_IFMT_E4M3) ? ((double)sh.qsc[j] * sh.ksd[c][0]) * raw : raw;
      }
      sh.contrib[c][j] = (double)sh.w[j] * fmax(D, 0.0);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < cnt; c += blockDim.x) {
      double S = 0.0;
      for (int j = 0; j < HI; ++j) S += sh.contrib[c][j];
      out[base + c] = S;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(TK_THREADS)
indexer_select_kernel(IndexerArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  const int row = blockIdx.x;
  const int b = row / a.Tq;
  const int HI = a.H_I, dI = a.d_I, nb = dI / 32;
  const int k = a.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = row_eligible(a, row);
  int32_t* out = a.idx_out + (size_t)row * k;
  float* sout = a.score_out ? a.score_out + (size_t)row * k : nullptr;

  // stage the query row (codes as exact floats) and its scales / weights
  for (int i = threadIdx.x; i < HI * dI; i += blockDim.x) {
    const int j = i / dI, c = i % dI;
    const size_t qoff = (size_t)row * HI + j;
    float v;
    if (a.ifmt == CSA_IFMT_F32) v = ((const float*)a.qI)[qoff * dI + c];
    else if (a.ifmt == CSA_IFMT_E4M3) v = e4m3_to_float(((const uint8_t*)a.qI)[qoff * dI + c]);
    else {
      const uint8_t byte = ((const uint8_t*)a.qI)[qoff * (dI / 2) + c / 2];
      v = e2m1_to_float((c & 1) ? (byte >> 4) : (byte & 0xF));
    }
    sh.qd[j * 129 + c] = (double)v;
  }
  for (int i = threadIdx.x; i < HI; i += blockDim.x) {
    sh.w[i] = a.w[(size_t)row * HI + i];
    if (a.ifmt == CSA_IFMT_E4M3) sh.qsc[i] = ((const float*)a.qI_scale)[(size_t)row * HI + i];
    if (a.ifmt == CSA_IFMT_MXFP4)
      for (int bb = 0; bb < nb; ++bb)
        sh.qsc[i * nb + bb] = ue8m0_to_float(((const uint8_t*)a.qI_scale)[((size_t)row * HI + i) * nb + bb]);
  }
  if (threadIdx.x == 0) { sh.n_sel = 0; sh.n_amb = 0; }
  __syncthreads();

  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? i : -1;
    if (sout) {
      for (int i = warp; i < k; i += (int)(blockDim.x >> 5)) {
        float v = 0.f;
        if (i < n) v = (float)rescore_entry(a, sh, row, i);
        if (lane == 0) sout[i] = v;
      }
    }
    return;
  }

  // U = sum_j w_j ||q_j|| (dequantised): with max_s ||k_s|| it bounds sum_c |q_c k_c|.
  if (warp == 0) {
    float u = 0.f;
    for (int j = lane; j < HI; j += 32) {
      float n2 = 0.f;
      for (int c = 0; c < dI; ++c) {
        float v = (float)sh.qd[j * 129 + c];
        if (a.ifmt == CSA_IFMT_E4M3) v *= sh.qsc[j];
        if (a.ifmt == CSA_IFMT_MXFP4) v *= sh.qsc[j * nb + c / 32];
        n2 = fmaf(v, v, n2);
      }
      u += fabsf(sh.w[j]) * sqrtf(n2);      // |w|: the bound holds for any sign
    }
    u = warp_sum(u);
    if (lane == 0) sh.U = u * 1.0001f;
  }
  const float* S = a.scores + (size_t)row * a.ld;
  // the scoring kernel recorded this row's key range; the k-th largest fp32 score
  // lies in histogram bin [f_lo, f_hi]
  uint32_t kmax, knmn;
  load_keyrange(a, row, &kmax, &knmn);
  const uint32_t kmin = ~knmn;
  const BinSel bs = hist_select(sh, n, k, [&](int i) { return f32_order_key(S[i]); }, kmin, kmax);
  const float f_lo = f32_from_order_key(bs.key_lo), f_hi = f32_from_order_key(bs.key_hi);
  const float knmax = load_knmax(a, row, b);
  const float E = a.eps_dot * sh.U * knmax + 1.52587890625e-05f * fmaxf(fabsf(f_lo), fabsf(f_hi));  // 2^-16 |tau|
  // every score is within E of its exact value, so entries above f_hi + 2E are in and
  // entries below f_lo - 2E are out; the band between is re-scored exactly
  const float hi = f_hi + 2.f * E, lo = f_lo - 2.f * E;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float v = S[i];
    if (v > hi) {
      const uint32_t slot = atomicAdd(&sh.n_sel, 1u);
      if (slot < (uint32_t)k) sh.sel[slot] = i;
    } else if (v >= lo) {
      const uint32_t slot = atomicAdd(&sh.n_amb, 1u);
      if (slot < AMB_CAP) sh.amb[slot] = i;
    }
  }
  __syncthreads();
  const int n_in = min((int)sh.n_sel, k);
  int n_amb = (int)sh.n_amb;
  if (n_amb > AMB_CAP) {
    if (threadIdx.x == 0) raise_err(a.err, CSA_DEVERR_BAND);
    n_amb = AMB_CAP;
  }
  const int need = k - n_in;
  rescore_block(a, sh, row, sh.amb, n_amb, sh.amb_s);
  for (int i = threadIdx.x; i < n_amb; i += blockDim.x) {
    const double si = sh.amb_s[i];
    const int ii = sh.amb[i];
    int rank = 0;
    for (int j = 0; j < n_amb; ++j) {
      const double sj = sh.amb_s[j];
      rank += (sj > si) || (sj == si && sh.amb[j] < ii);
    }
    if (rank < need) sh.sel[n_in + rank] = ii;
  }
  __syncthreads();
  const int cnt = min(k, n_in + min(need, n_amb));
  write_sorted(sh, cnt, k, out);
  if (sout) {
    __syncthreads();
    rescore_block(a, sh, row, sh.sel, cnt, sh.amb_s);
    for (int i = threadIdx.x; i < k; i += blockDim.x) sout[i] = i < cnt ? (float)sh.amb_s[i] : 0.f;
  }
}

static void set_smem_attr(const void* fn) {
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(TopkShared));
}

cudaError_t launch_indexer_select(const IndexerArgs& a, cudaStream_t st) {
  if (a.hist) {
    const cudaError_t eh = launch_indexer_select_hist(a, st);
    if (eh != cudaErrorNotSupported) return eh;
  }
  const cudaError_t e = launch_indexer_select_cluster(a, st);
  if (e != cudaErrorNotSupported) return e;
  set_smem_attr((const void*)indexer_select_kernel);
  note_launch();
  indexer_select_kernel<<<a.B * a.Tq, TK_THREADS, sizeof(TopkShared), st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_topk_select(const float* scores, int64_t ld, RowCount rc, int R, int64_t n,
                               int k, int32_t* idx_out, cudaStream_t st, unsigned* err) {
  (void)err;
  const cudaError_t e = launch_topk_select_cluster(scores, ld, rc, R, n, k, idx_out, st);
  if (e != cudaErrorNotSupported) return e;
  set_smem_attr((const void*)topk_select_kernel);
  note_launch();
  topk_select_kernel<<<R, TK_THREADS, sizeof(TopkShared), st>>>(scores, ld, rc, n, k, idx_out);
  return cudaGetLastError();
}

}  // namespace csa
