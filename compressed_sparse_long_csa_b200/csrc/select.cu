// Exact top-k selection of compressed entries on a thread-block cluster per query row.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 2 (the indexer keeps the top-k compressed blocks;
// k = 512 / 1024 from table "Конфигурации").  Ties go to the lower entry index and
// the selected set is written in ascending index order, padded with -1.
//
// A row of n scores is split over the C CTAs (C <= 8) of one cluster: CTA r holds
// entries [r*chunk, (r+1)*chunk) in shared memory.  The CTAs combine their partial
// results through distributed shared memory:
//  1. the key range [kmin, kmax] of the row (monotone fp32 order keys);
//  2. 2048-bin histograms over the current key range [lo, hi]: bin = (key - lo) >> s
//     with the smallest s that fits (at least half the bins are in use; no division);
//     the bin holding the k-th largest key
//     becomes the next range until it holds at most SL_CAP keys or one key value;
//  3. topk_select: the keys of that bin, gathered by every CTA, give the exact k-th
//     largest fp32 key tau (lightning_index refines the bin to at most 64 keys and
//     uses its bounds [tau_lo, tau_hi] instead);
//  4a. topk_select: keys above tau are in; of the keys equal to tau, the lowest
//      indices complete the set (CTA rank order is index order);
//  4b. lightning_index: the fp32 scores carry a bounded error E (accumulation in the
//      scoring kernel), so the k-th largest exact score lies in [tau_lo - E, tau_hi + E].
//      Entries above tau_hi + 2E are certainly in, entries below tau_lo - 2E certainly
//      out.  The key range comes from the scoring kernel, which records it.  Every CTA re-scores its own band entries exactly in
//      fp64 from the quantised operands (FP8 / FP4 products and their sums are exact
//      in fp64; the per-head terms are then added in head order, as the definition
//      does), and the band is ranked by (exact score desc, index asc).
//  5. selections are kept as bitmaps (one ballot per 32 entries); cluster-wide prefix
//     counts give each CTA its output offset and a scan over the bitmap words writes
//     the indices in ascending order.
// Every pass over the entries is a rolled loop: this kernel runs its code once per
// row, and code that runs once costs its instruction fetch, so the code is kept small.
#include "indexer.cuh"
#include "tc.cuh"

#include <algorithm>
#include <cooperative_groups.h>
#include <map>
#include <mutex>
#include <tuple>

namespace csa {

namespace cg = cooperative_groups;

namespace {

constexpr int SL_T = 512;              // threads per CTA (128 registers each: no spills)
constexpr int SL_W = SL_T / 32;
constexpr int SL_BINS = 2048;          // histogram bins
constexpr int SL_CAP = 1024;           // threshold-bin keys / band entries gathered per row
constexpr int SL_CMAX = 8;             // CTAs per cluster (portable cluster size)
constexpr int SL_CHUNK = 34 * 1024;    // entries per CTA at most
constexpr int SL_QPT = 8192 / SL_T;    // query-row elements per thread (H_I * d_I <= 8192)
constexpr int SL_BAND_CT = 64;         // the indexer refines the threshold bin down to this many keys
constexpr int SL_WORDS = SL_CHUNK / 32;
constexpr int SL_RR = 32;              // entries re-scored per round
constexpr int SL_QLD = 132;            // padded row length (doubles) of the staged query / key rows

struct SelFixed {
  uint32_t hist[2][SL_BINS];           // read by peers (double-buffered across refinement rounds)
  uint32_t keys[SL_CAP];               // read by peers: this CTA's keys of the threshold bin
  uint32_t gkeys[SL_CAP];              // all keys of the threshold bin
  uint32_t bits_a[SL_WORDS];           // selected (indexer: sure, then also chosen band) / above tau
  uint32_t bits_b[SL_WORDS];           // plain select: equal to tau
  int32_t band_id[SL_CAP];             // read by peers: this CTA's band entries
  double band_s[SL_CAP];               // read by peers: their exact scores
  int32_t gband_id[SL_CAP];
  double gband_s[SL_CAP];
  uint32_t wtot[SL_W];
  uint32_t red[2];
  uint32_t pub[4];                     // read by peers
  uint32_t pcnt[SL_CMAX][2];
  int goff[SL_CMAX + 1];               // start of each CTA's part in a gathered list
  uint32_t cgt, cT, tau, tlo, thi, cnt, n_sure;
  alignas(8) uint64_t ldbar;           // completion of the bulk copy of the scores
  float qsc[64 * 4];
  float w[64];
  float U;
};

// Re-scoring scratch (see sl_resc_sep for where it lives).
struct Resc {
  double qd[64 * SL_QLD];              // query row codes as fp64 (rows padded: conflict-free fragment reads)
  double kd[SL_RR][SL_QLD];            // key rows being re-scored (one round)
  double contrib[SL_RR][65];           // their per-head terms (rows padded)
  float ksc[SL_RR][4];                 // their scales (E4M3 row scale in [0], MXFP4 block scales)
};

constexpr size_t SL_FIXED = (sizeof(SelFixed) + 127) & ~size_t(127);
// The re-scoring scratch gets its own region after the scores when both fit (the query
// row is then staged while the scores land), else it overlays them.
__host__ __device__ constexpr size_t sl_score_bytes(int chunk) { return ((size_t)chunk * 4 + 127) & ~size_t(127); }
__host__ __device__ constexpr bool sl_resc_sep(int chunk) { return SL_FIXED + sl_score_bytes(chunk) + sizeof(Resc) <= 232448; }


__device__ __forceinline__ void sl_sync(cg::cluster_group cl, unsigned C) {
  if (C == 1) __syncthreads();
  else cl.sync();
}

// Block-wide exclusive scan of one int per thread (all threads call).
__device__ __forceinline__ int sl_excl_scan(int v, uint32_t* wtot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) wtot[warp] = (uint32_t)incl;
  __syncthreads();
  int wpre = 0, tot = 0;
  if (lane < SL_W) {
    const int x = (int)wtot[lane];
    wpre = (lane < warp) ? x : 0;
    tot = x;
  }
  for (int o = 16; o > 0; o >>= 1) {
    wpre += __shfl_xor_sync(0xffffffffu, wpre, o);
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
  }
  __syncthreads();
  *total = tot;
  return wpre + incl - v;
}

// Word `slot` of CTA p's published values, p < C.
__device__ __forceinline__ uint32_t sl_peer(cg::cluster_group cl, const uint32_t* pub, int slot, int p) {
  return cl.map_shared_rank(pub, p)[slot];
}

// Concatenate every CTA's list (CTA p's count in its pub[slot]) into dst in rank order;
// returns the total (at most cap).
// The offsets are set by sl_gather_offsets (one thread, then a barrier).
// Peer loads in these helpers are unrolled over SL_CMAX and predicated, so that all of
// them are in flight at once (a loop over the runtime cluster size issued them one by one).
__device__ __forceinline__ void sl_gather_offsets(SelFixed& sh, cg::cluster_group cl, unsigned C, int slot) {
  const int t = threadIdx.x;
  if (t <= SL_CMAX) {
    int sum = 0;
#pragma unroll
    for (int p = 0; p < SL_CMAX; ++p)
      if (p < t && p < (int)C) sum += (int)sl_peer(cl, sh.pub, slot, p);
    sh.goff[t] = sum;
  }
}
template <typename T>
__device__ __forceinline__ int sl_gather(SelFixed& sh, cg::cluster_group cl, unsigned C, T* list, T* dst, int cap) {
  const int total = min(sh.goff[SL_CMAX], cap);
  for (int i = threadIdx.x; i < total; i += SL_T) {
    int p = 0;
    while (p + 1 < (int)C && sh.goff[p + 1] <= i) ++p;
    dst[i] = cl.map_shared_rank(list, p)[i - sh.goff[p]];
  }
  return total;
}

// Key range [lo, hi] of the row over every CTA's entries sv[0..m).
__device__ __forceinline__ void sl_key_range(SelFixed& sh, const float* sv, int m, cg::cluster_group cluster,
                                          uint32_t* lo_out, uint32_t* hi_out) {
  const int tid = threadIdx.x, lane = tid & 31;
  const unsigned C = cluster.num_blocks();
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  for (int i = tid; i < m; i += SL_T) {
    const uint32_t x = f32_order_key(sv[i]);
    mn = min(mn, x);
    mx = max(mx, x);
  }
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (tid == 0) { sh.red[0] = 0xFFFFFFFFu; sh.red[1] = 0u; }
  __syncthreads();
  if (lane == 0) { atomicMin(&sh.red[0], mn); atomicMax(&sh.red[1], mx); }
  __syncthreads();
  if (tid == 0) { sh.pub[0] = sh.red[0]; sh.pub[1] = sh.red[1]; }
  sl_sync(cluster, C);
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
  for (int p = 0; p < SL_CMAX; ++p) {
    if (p < (int)C) {
      lo = min(lo, sl_peer(cluster, sh.pub, 0, p));
      hi = max(hi, sl_peer(cluster, sh.pub, 1, p));
    }
  }
  *lo_out = lo;
  *hi_out = hi;
}

// Histogram refinement (step 2): [*lo, *hi] holds the k-th largest key of the row; on
// return it is a bin of at most stop_ct keys (or one key value), *want is the rank of
// the k-th largest key from the top among the keys inside it and *cT their number.
// Every CTA of the cluster calls it with the same arguments and gets the same results.
__device__ __forceinline__ void sl_refine(SelFixed& sh, const float* sv, int m, int k, int stop_ct,
                                       cg::cluster_group cluster, uint32_t* lo_io, uint32_t* hi_io, int* want_out,
                                       uint32_t* ct_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned C = cluster.num_blocks();
  uint32_t lo = *lo_io, hi = *hi_io;
  int want = k;
  uint32_t cT = 0;
  for (int round = 0; round < 6; ++round) {
    uint32_t* H = sh.hist[round & 1];
    reinterpret_cast<uint4*>(H)[tid] = make_uint4(0u, 0u, 0u, 0u);   // 4 bins per thread
    // bins of 2^sh keys: the smallest shift with (hi - lo) >> sh < SL_BINS
    const int range_bits = 32 - __clz(hi - lo);              // 0 when lo == hi
    const int shf = range_bits > 11 ? range_bits - 11 : 0;
    __syncthreads();
#pragma unroll 4
    for (int i = tid; i < m; i += SL_T) {
      const uint32_t x = f32_order_key(sv[i]);
      if (x >= lo && x <= hi) atomicAdd(&H[(x - lo) >> shf], 1u);
    }
    sl_sync(cluster, C);
    uint4 hb = make_uint4(0u, 0u, 0u, 0u);
    {
      uint4 xs[SL_CMAX];
#pragma unroll
      for (int p = 0; p < SL_CMAX; ++p)
        xs[p] = p < (int)C ? reinterpret_cast<const uint4*>(cluster.map_shared_rank(H, p))[tid] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int p = 0; p < SL_CMAX; ++p) { hb.x += xs[p].x; hb.y += xs[p].y; hb.z += xs[p].z; hb.w += xs[p].w; }
    }
    // suffix counts: bins above 4*tid+3 belong to higher threads
    const uint32_t mine = hb.x + hb.y + hb.z + hb.w;
    uint32_t vsum = mine;
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_down_sync(0xffffffffu, vsum, o);
      if (lane + o < 32) vsum += x;
    }
    if (lane == 0) sh.wtot[warp] = vsum;
    __syncthreads();
    uint32_t above_w = 0;
    if (lane < SL_W && lane > warp) above_w = sh.wtot[lane];
    above_w = __reduce_add_sync(0xffffffffu, above_w);
    uint32_t after = vsum - mine + above_w;                 // keys in bins > 4*tid+3
    const uint32_t kk = (uint32_t)want;
    const uint32_t cb[4] = {hb.w, hb.z, hb.y, hb.x};        // bins 4t+3, 4t+2, 4t+1, 4t
    int bin = -1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (bin < 0 && after < kk && kk <= after + cb[q]) { bin = 4 * tid + 3 - q; sh.cgt = after; sh.cT = cb[q]; }
      after += cb[q];
    }
    if (bin >= 0) {
      // key bounds of bin T
      sh.tlo = lo + ((uint32_t)bin << shf);
      const uint64_t top = (uint64_t)sh.tlo + ((1ull << shf) - 1ull);
      sh.thi = top < (uint64_t)hi ? (uint32_t)top : hi;
    }
    __syncthreads();
    want -= (int)sh.cgt;
    cT = sh.cT;
    lo = sh.tlo;
    hi = sh.thi;
    __syncthreads();                                       // sh.* is rewritten next round
    if (lo == hi || cT <= (uint32_t)stop_ct) break;
  }
  *lo_io = lo;
  *hi_io = hi;
  *want_out = want;
  *ct_out = cT;
}

// Step 3: the exact k-th largest key, given the bin [lo, hi] that holds it at rank
// `want` from the top (the bin holds at most SL_CAP keys).
__device__ __forceinline__ uint32_t sl_exact_tau(SelFixed& sh, const float* sv, int m, cg::cluster_group cluster,
                                              uint32_t lo, uint32_t hi, int want) {
  const int tid = threadIdx.x;
  const unsigned C = cluster.num_blocks();
  if (lo == hi) return lo;
  if (tid == 0) { sh.cnt = 0; sh.tau = lo; }
  __syncthreads();
  for (int i = tid; i < m; i += SL_T) {
    const uint32_t x = f32_order_key(sv[i]);
    if (x >= lo && x <= hi) {
      const uint32_t s = atomicAdd(&sh.cnt, 1u);
      if (s < (uint32_t)SL_CAP) sh.keys[s] = x;
    }
  }
  __syncthreads();
  if (tid == 0) sh.pub[2] = min(sh.cnt, (uint32_t)SL_CAP);
  sl_sync(cluster, C);
  sl_gather_offsets(sh, cluster, C, 2);
  __syncthreads();
  const int ng = sl_gather(sh, cluster, C, sh.keys, sh.gkeys, SL_CAP);
  __syncthreads();
  for (int i = tid; i < ng; i += SL_T) {
    const uint32_t xi = sh.gkeys[i];
    int gt = 0, ge = 0;
    for (int j = 0; j < ng; ++j) {
      const uint32_t xj = sh.gkeys[j];
      gt += xj > xi;
      ge += xj >= xi;
    }
    if (gt < want && want <= ge) sh.tau = xi;             // every such xi is the same key
  }
  __syncthreads();
  return sh.tau;
}

// Load this CTA's scores S[0, m) into sv (16-byte vectors when aligned).
__device__ __forceinline__ void sl_load(const float* __restrict__ S, int m, bool vec, float* sv) {
  if (vec) {
    const int m4 = m & ~3;
#pragma unroll 4
    for (int i = threadIdx.x * 4; i < m4; i += SL_T * 4)
      *reinterpret_cast<float4*>(sv + i) = *reinterpret_cast<const float4*>(S + i);
    for (int i = m4 + threadIdx.x; i < m; i += SL_T) sv[i] = S[i];
  } else {
#pragma unroll 4
    for (int i = threadIdx.x; i < m; i += SL_T) sv[i] = S[i];
  }
}

// Writes this CTA's selected entries (bitmap sel over nwords words, entry ids base + bit
// index) at out[off ...] in ascending order; returns the CTA's count.
__device__ __forceinline__ int sl_write(SelFixed& sh, const uint32_t* sel, int nwords, int base, int off, int k, int32_t* out) {
  const int wpt = (nwords + SL_T - 1) / SL_T;            // words per thread (contiguous)
  const int w0 = threadIdx.x * wpt, w1 = min(nwords, w0 + wpt);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(sel[w]);
  int tot;
  int pos = off + sl_excl_scan(cnt, sh.wtot, &tot);
  for (int w = w0; w < w1; ++w)
    for (uint32_t bits = sel[w]; bits; bits &= bits - 1) {
      if (pos < k) out[pos] = base + 32 * w + __ffs(bits) - 1;
      ++pos;
    }
  return tot;
}

// ------------------------------------------------------------------ plain top-k
__global__ void __launch_bounds__(SL_T, 1)
topk_cluster_kernel(const float* __restrict__ scores, int64_t ld, RowCount rc, int64_t n_cap,
                    int k, int32_t* __restrict__ idx_out, int chunk, int vec) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SelFixed& sh = *reinterpret_cast<SelFixed*>(smem_raw);
  float* sv = reinterpret_cast<float*>(smem_raw + SL_FIXED);
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned C = cluster.num_blocks(), r = cluster.block_rank();
  const int row = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  tc::griddep_wait();                                      // every input may come from the previous kernel
  const int n = rc(row, n_cap);
  int32_t* out = idx_out + (size_t)row * k;
  if (n <= k) {
    if (r == 0)
      for (int i = tid; i < k; i += SL_T) out[i] = i < n ? i : -1;
    return;                                                // uniform over the cluster: no DSMEM use
  }
  const int lo = (int)r * chunk;
  const int m = max(0, min(n - lo, chunk));
  sl_load(scores + (size_t)row * ld + lo, m, vec != 0, sv);
  __syncthreads();
  uint32_t lo_k, hi_k, cT;
  int want;
  sl_key_range(sh, sv, m, cluster, &lo_k, &hi_k);
  sl_refine(sh, sv, m, k, SL_CAP, cluster, &lo_k, &hi_k, &want, &cT);
  const uint32_t tau = sl_exact_tau(sh, sv, m, cluster, lo_k, hi_k, want);
  // bitmaps: above tau, equal to tau
  const int nwords = (m + 31) / 32;
  int gt = 0, eq = 0;
  for (int w = warp; w < nwords; w += SL_W) {
    const int i = 32 * w + lane;
    const uint32_t x = i < m ? f32_order_key(sv[i]) : 0u;
    const uint32_t ba = __ballot_sync(0xffffffffu, i < m && x > tau);
    const uint32_t bb = __ballot_sync(0xffffffffu, i < m && x == tau);
    if (lane == 0) { sh.bits_a[w] = ba; sh.bits_b[w] = bb; gt += __popc(ba); eq += __popc(bb); }
  }
  int gt_tot, eq_tot;
  sl_excl_scan(gt, sh.wtot, &gt_tot);
  sl_excl_scan(eq, sh.wtot, &eq_tot);
  if (tid == 0) { sh.pub[0] = (uint32_t)gt_tot; sh.pub[1] = (uint32_t)eq_tot; }
  sl_sync(cluster, C);
  int gp[SL_CMAX], ep[SL_CMAX];
#pragma unroll
  for (int p = 0; p < SL_CMAX; ++p) {
    gp[p] = p < (int)C ? (int)sl_peer(cluster, sh.pub, 0, p) : 0;
    ep[p] = p < (int)C ? (int)sl_peer(cluster, sh.pub, 1, p) : 0;
  }
  int all_gt = 0;
#pragma unroll
  for (int p = 0; p < SL_CMAX; ++p) all_gt += gp[p];
  const int eq_need = k - all_gt;
  int eqp = 0, off = 0, quota = 0;
#pragma unroll
  for (int p = 0; p < SL_CMAX; ++p) {
    const int q = max(0, min(eq_need - eqp, ep[p]));
    if (p < (int)r) off += gp[p] + q;
    if (p == (int)r) quota = q;
    eqp += ep[p];
  }
  // keep the first `quota` entries equal to tau (index order)
  {
    const int wpt = (nwords + SL_T - 1) / SL_T;
    const int w0 = tid * wpt, w1 = min(nwords, w0 + wpt);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(sh.bits_b[w]);
    int tot;
    int seen = sl_excl_scan(c, sh.wtot, &tot);
    for (int w = w0; w < w1; ++w) {
      uint32_t keep = 0u;
      for (uint32_t bits = sh.bits_b[w]; bits; bits &= bits - 1) {
        if (seen < quota) keep |= bits & (0u - bits);
        ++seen;
      }
      sh.bits_a[w] |= keep;
    }
  }
  __syncthreads();
  sl_write(sh, sh.bits_a, nwords, lo, off, k, out);
  sl_sync(cluster, C);                                     // peers may still read pub
}

// ------------------------------------------------------------------ indexer selection
// D (8x8) += A (8x4, row-major) * B (4x8, column-major), fp64 tensor-core MMA.  Lane l
// holds A[l/4][l%4], B[l%4][l/4] and D[l/4][2(l%4)], D[l/4][2(l%4)+1].
__device__ __forceinline__ void dmma_884(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d0), "+d"(d1) : "d"(a), "d"(b));
}

// What the exact re-scoring reads of the key side, passed by value: taking the address of
// a kernel parameter would copy the whole argument block to local memory.
struct RescKeys {
  const void* kI;
  const void* kI_scale;
  int64_t n_max;
  int HI, dI;
};

// Exact fp64 scores of entries ids[0..cnt) (cnt <= SL_RR) into out[0..cnt), by the whole
// CTA (all threads call; barriers inside).  The query row is staged in rs.qd / sh.qsc /
// sh.w.  The per-head dot products of FP8 / FP4 codes are exact in fp64 in any order, so
// they run on the fp64 tensor cores: every warp takes (8 entries x 8 heads) tiles over
// K = d_I.  Each head's term w_j * max(D_j, 0) is formed as the definition does, and the
// terms are added in order j = 0..H_I-1.
template <int F>
__device__ __noinline__ void sl_rescore_round(const RescKeys a, SelFixed& sh, Resc& rs, int b, const int32_t* ids,
                                              int cnt, double* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int HI = a.HI, dI = a.dI, nb = dI / 32;
  // ---- key rows (zeros past cnt): element idx = tid + SL_T*u is (entry idx / d_I,
  // dim idx % d_I); all loads first, then consecutive threads store consecutive doubles
  const int lgd = __ffs(dI) - 1;
  float xv[SL_RR * 128 / SL_T];
#pragma unroll
  for (int u = 0; u < SL_RR * 128 / SL_T; ++u) {
    const int idx = tid + SL_T * u;
    const int c = idx >> lgd, d = idx & (dI - 1);
    xv[u] = 0.f;
    if (c < cnt) {
      const size_t koff = (size_t)b * a.n_max + ids[c];
      if (F == CSA_IFMT_E4M3) xv[u] = e4m3_to_float(((const uint8_t*)a.kI)[koff * dI + d]);
      else if (F == CSA_IFMT_MXFP4) {
        const uint8_t byte = ((const uint8_t*)a.kI)[koff * (dI / 2) + (d >> 1)];
        xv[u] = e2m1_to_float((d & 1) ? (byte >> 4) : (byte & 0xF));
      } else xv[u] = ((const float*)a.kI)[koff * dI + d];
    }
  }
  float scl = 0.f;
  const int nsc = (F == CSA_IFMT_MXFP4) ? nb : 1;
  if (tid < SL_RR * nsc) {
    const int c = tid / nsc, q = tid - c * nsc;
    if (c < cnt) {
      const size_t koff = (size_t)b * a.n_max + ids[c];
      if (F == CSA_IFMT_E4M3) scl = ((const float*)a.kI_scale)[koff];
      if (F == CSA_IFMT_MXFP4) scl = ue8m0_to_float(((const uint8_t*)a.kI_scale)[koff * nb + q]);
    }
  }
#pragma unroll
  for (int u = 0; u < SL_RR * 128 / SL_T; ++u) {
    const int idx = tid + SL_T * u;
    if (idx < SL_RR * dI) rs.kd[idx >> lgd][idx & (dI - 1)] = (double)xv[u];
  }
  if (tid < SL_RR * nsc) rs.ksc[tid / nsc][tid % nsc] = scl;
  __syncthreads();
  // ---- (8 entries x 8 heads) tiles: tile = (group, head block)
  const int g = lane >> 2, t = lane & 3;
  const int n_hb = (HI + 7) / 8, n_grp = (cnt + 7) / 8;
  const int n_blk = (F == CSA_IFMT_MXFP4) ? nb : 1;
  const int ks_blk = dI / 4 / n_blk;
  for (int tile = warp; tile < n_grp * n_hb; tile += SL_W) {
    const int grp = tile / n_hb, hb = tile - grp * n_hb;
    const double* arow = rs.qd + (8 * hb + g) * SL_QLD;      // A[m][k]: head 8hb+g, dim k = t
    const double* brow = rs.kd[8 * grp + g];                 // B[k][n]: entry 8grp+g, dim k = t
    const int j = 8 * hb + g;
    const int c0 = 8 * grp + 2 * t;
    double D0 = 0.0, D1 = 0.0;
    for (int bb = 0; bb < n_blk; ++bb) {
      double P0 = 0.0, P1 = 0.0, Q0 = 0.0, Q1 = 0.0;         // two chains: even / odd k-steps
      const int k0 = bb * ks_blk;
#pragma unroll 4
      for (int ks = 0; ks < ks_blk; ks += 2) {
        dmma_884(P0, P1, arow[4 * (k0 + ks) + t], brow[4 * (k0 + ks) + t]);
        dmma_884(Q0, Q1, arow[4 * (k0 + ks + 1) + t], brow[4 * (k0 + ks + 1) + t]);
      }
      P0 += Q0;                                              // exact: all partial sums are
      P1 += Q1;                                              // multiples of the code grid
      if (F == CSA_IFMT_MXFP4) {
        const double qs = (j < HI) ? (double)sh.qsc[j * nb + bb] : 0.0;
        D0 += (qs * (double)rs.ksc[c0][bb]) * P0;
        D1 += (qs * (double)rs.ksc[c0 + 1][bb]) * P1;
      } else {
        D0 = P0;
        D1 = P1;
      }
    }
    if (j < HI) {
      if (F == CSA_IFMT_E4M3) {
        D0 = ((double)sh.qsc[j] * (double)rs.ksc[c0][0]) * D0;
        D1 = ((double)sh.qsc[j] * (double)rs.ksc[c0 + 1][0]) * D1;
      }
      rs.contrib[c0][j] = (double)sh.w[j] * fmax(D0, 0.0);
      rs.contrib[c0 + 1][j] = (double)sh.w[j] * fmax(D1, 0.0);
    }
  }
  __syncthreads();
  // ---- head terms added in order, one thread per entry
  if (tid < cnt) {
    const double* cr = rs.contrib[tid];
    double S = 0.0;
    int j = 0;
    for (; j + 8 <= HI; j += 8) {
      double v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = cr[j + q];
#pragma unroll
      for (int q = 0; q < 8; ++q) S += v[q];
    }
    for (; j < HI; ++j) S += cr[j];
    out[tid] = S;
  }
  __syncthreads();
}

template <int F>
__device__ __forceinline__ void sl_rescore_list(const RescKeys a, SelFixed& sh, Resc& rs, int b, const int32_t* ids,
                                                int n, double* out) {
  for (int c0 = 0; c0 < n; c0 += SL_RR) sl_rescore_round<F>(a, sh, rs, b, ids + c0, min(SL_RR, n - c0), out + c0);
}

// Stage the query row codes (held in registers, element tid + SL_T*e) as fp64:
// consecutive threads store consecutive doubles; rows up to the next multiple of 8 heads
// are zero (fp64 MMA fragments read them).
__device__ __forceinline__ void sl_stage_query(Resc& rs, const float (&qx)[SL_QPT], int total, int lgd, int HI, int dI) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int e = 0; e < SL_QPT; ++e) {
    const int i = tid + SL_T * e;
    if (i < total) rs.qd[(i >> lgd) * SL_QLD + (i & (dI - 1))] = (double)qx[e];
  }
  const int hpad = (HI + 7) / 8 * 8;
  for (int i = total + tid; i < hpad * dI; i += SL_T) rs.qd[(i >> lgd) * SL_QLD + (i & (dI - 1))] = 0.0;
}

template <int F>
__global__ void __launch_bounds__(SL_T, 1)
indexer_select_cluster_kernel(IndexerArgs a, int chunk) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SelFixed& sh = *reinterpret_cast<SelFixed*>(smem_raw);
  float* sv = reinterpret_cast<float*>(smem_raw + SL_FIXED);
  const bool resc_sep = sl_resc_sep(chunk);
  Resc& rs = *reinterpret_cast<Resc*>(smem_raw + SL_FIXED + (resc_sep ? sl_score_bytes(chunk) : 0));
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned C = cluster.num_blocks(), r = cluster.block_rank();
  const int row = blockIdx.x / C;
  const int b = row / a.Tq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.k;
  const int HI = a.H_I, dI = a.d_I, nb = dI / 32;
  const int n = row_eligible(a, row);
  int32_t* out = a.idx_out + (size_t)row * k;
  float* sout = a.score_out ? a.score_out + (size_t)row * k : nullptr;
  const RescKeys rk{a.kI, a.kI_scale, a.n_max, a.H_I, a.d_I};
  const int lo = (int)r * chunk;
  const int m = max(0, min(n - lo, chunk));
  tc::griddep_launch_dependents();
  // ---- the query row (written before the scoring kernel started: read before waiting
  // for it): codes into registers (staged into shared memory once the scores are
  // classified), scales and weights, and U = sum_j |w_j| ||q_j|| for the error bound
  const int m4 = (n > k) ? (m & ~3) : 0;
  const float* srow = a.scores + (size_t)row * a.ld + lo;
  if (tid == 0) {
    tc::mbar_init(&sh.ldbar, 1);
    tc::fence_mbar_init();
  }
  const int total = HI * dI, lgd = __ffs(dI) - 1;
  const size_t r0 = (size_t)row * total;
  float qx[SL_QPT];
#pragma unroll
  for (int e = 0; e < SL_QPT; ++e) {
    const int i = tid + SL_T * e;
    qx[e] = 0.f;
    if (i < total) {
      if (F == CSA_IFMT_E4M3) qx[e] = e4m3_to_float(((const uint8_t*)a.qI)[r0 + i]);
      else if (F == CSA_IFMT_MXFP4) {
        const uint8_t byte = ((const uint8_t*)a.qI)[(r0 + i) >> 1];
        qx[e] = e2m1_to_float((i & 1) ? (byte >> 4) : (byte & 0xF));
      } else qx[e] = ((const float*)a.qI)[r0 + i];
    }
  }
  // weights and scales, and the words of this warp's heads for U = sum_j |w_j| ||q_j||
  // (warp w takes heads w, w + SL_W, ...; lane l holds elements [epl*l, epl*l + epl)):
  // every load of the prologue is issued before any is used
  constexpr int EPL = (F == CSA_IFMT_MXFP4) ? 8 : 4;
  float w_r = 0.f, qs_r[4] = {0.f, 0.f, 0.f, 0.f};
  if (tid < HI) {
    w_r = a.w[(size_t)row * HI + tid];
    if (F == CSA_IFMT_E4M3) qs_r[0] = ((const float*)a.qI_scale)[(size_t)row * HI + tid];
    if (F == CSA_IFMT_MXFP4) {
#pragma unroll
      for (int bb = 0; bb < 4; ++bb)
        if (bb < nb) qs_r[bb] = ue8m0_to_float(((const uint8_t*)a.qI_scale)[((size_t)row * HI + tid) * nb + bb]);
    }
  }
  uint4 qv[64 / SL_W];
#pragma unroll
  for (int h = 0; h < 64 / SL_W; ++h) {
    const int j = warp + SL_W * h;
    qv[h] = make_uint4(0u, 0u, 0u, 0u);
    if (j < HI && lane * EPL < dI) {
      const size_t e0 = r0 + (size_t)j * dI + lane * EPL;
      if (F == CSA_IFMT_E4M3) qv[h].x = *reinterpret_cast<const uint32_t*>((const uint8_t*)a.qI + e0);
      else if (F == CSA_IFMT_MXFP4) qv[h].x = *reinterpret_cast<const uint32_t*>((const uint8_t*)a.qI + e0 / 2);
      else qv[h] = *reinterpret_cast<const uint4*>((const float*)a.qI + e0);
    }
  }
  // ---- the scoring kernel's outputs: key-norm bound and key range (the scores follow
  // by one bulk copy into shared memory, the tail by plain loads)
  tc::griddep_wait();
  // the scores go into shared memory first (one bulk copy, the tail by plain loads); the
  // head-norm bound below runs while they travel (tid 0 initialised the barrier itself)
  if (tid == 0) {
    tc::mbar_arrive_expect_tx(&sh.ldbar, (uint32_t)m4 * 4u);
    for (int o = 0; o < m4; o += 8192) {
      const uint32_t bytes = (uint32_t)min(8192, m4 - o) * 4u;
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(tc::smem_u32(sv + o)), "l"(srow + o), "r"(bytes), "r"(tc::smem_u32(&sh.ldbar)) : "memory");
    }
  }
  if (n > k && tid < m - m4) sv[m4 + tid] = srow[m4 + tid];
  const float knmax = load_knmax(a, row, b);
  // the key range the scoring kernel recorded (exact min / max over the row's eligible entries)
  uint32_t hi_k, lo_k;
  load_keyrange(a, row, &hi_k, &lo_k);
  lo_k = ~lo_k;
  if (tid < HI) {
    sh.w[tid] = w_r;
    if (F == CSA_IFMT_E4M3) sh.qsc[tid] = qs_r[0];
    if (F == CSA_IFMT_MXFP4) {
#pragma unroll
      for (int bb = 0; bb < 4; ++bb)
        if (bb < nb) sh.qsc[tid * nb + bb] = qs_r[bb];
    }
  }
  if (tid == 0) sh.U = 0.f;
  __syncthreads();                                         // w, scales, U = 0 and the barrier init are visible
  {
    float n2[64 / SL_W];
#pragma unroll
    for (int h = 0; h < 64 / SL_W; ++h) {
      const int j = warp + SL_W * h;
      float acc = 0.f;
      if (j < HI && lane * EPL < dI) {
        if (F == CSA_IFMT_E4M3) {
          for (int e = 0; e < 4; ++e) { const float x = e4m3_to_float((qv[h].x >> (8 * e)) & 0xFFu); acc = fmaf(x, x, acc); }
          acc *= sh.qsc[j] * sh.qsc[j];
        } else if (F == CSA_IFMT_MXFP4) {
          for (int e = 0; e < 8; ++e) { const float x = e2m1_to_float((qv[h].x >> (4 * e)) & 0xFu); acc = fmaf(x, x, acc); }
          const float sc = sh.qsc[j * nb + (lane * 8) / 32];
          acc *= sc * sc;
        } else {
          acc = __uint_as_float(qv[h].x) * __uint_as_float(qv[h].x) + __uint_as_float(qv[h].y) * __uint_as_float(qv[h].y) +
                __uint_as_float(qv[h].z) * __uint_as_float(qv[h].z) + __uint_as_float(qv[h].w) * __uint_as_float(qv[h].w);
        }
      }
      n2[h] = acc;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int h = 0; h < 64 / SL_W; ++h) n2[h] += __shfl_xor_sync(0xffffffffu, n2[h], o);
    }
    float uw = 0.f;
#pragma unroll
    for (int h = 0; h < 64 / SL_W; ++h) {
      const int j = warp + SL_W * h;
      if (j < HI) uw += fabsf(sh.w[j]) * sqrtf(n2[h]);     // |w|: the bound holds for any sign
    }
    if (lane == 0) atomicAdd(&sh.U, uw);                   // read after the barriers below
  }
  if (resc_sep) sl_stage_query(rs, qx, total, lgd, HI, dI);   // covered by the barrier below
  // the scores have landed (bounded wait; on a timeout the error word is set)
  if (n > k && m4 > 0) {
    const bool ok = tc::mbar_wait(&sh.ldbar, 0);
    if (!ok && tid == 0) raise_err(a.err, CSA_DEVERR_TIMEOUT);
  }
  __syncthreads();
  if (n <= k) {
    // every eligible entry is selected; CTA r scores the slots [r*k/C, (r+1)*k/C)
    if (r == 0)
      for (int i = tid; i < k; i += SL_T) out[i] = i < n ? i : -1;
    if (sout) {
      if (!resc_sep) sl_stage_query(rs, qx, total, lgd, HI, dI);
      const int s0 = (int)((int64_t)k * r / C), s1 = (int)((int64_t)k * (r + 1) / C);
      for (int c0 = s0; c0 < s1; c0 += SL_CAP) {
        const int cnt = min(SL_CAP, s1 - c0);
        __syncthreads();
        for (int i = tid; i < cnt; i += SL_T) sh.band_id[i] = min(c0 + i, max(n - 1, 0));
        __syncthreads();
        sl_rescore_list<F>(rk, sh, rs, b, sh.band_id, cnt, sh.band_s);
        for (int i = tid; i < cnt; i += SL_T) sout[c0 + i] = (c0 + i < n) ? (float)sh.band_s[i] : 0.f;
      }
    }
    return;                                                // uniform over the cluster: no DSMEM use
  }
  // the bin [tau_lo, tau_hi] that holds the k-th largest fp32 score (at most SL_BAND_CT
  // scores, or one value); the band is that bin widened by 2E on both sides
  uint32_t cT;
  int want;
  sl_refine(sh, sv, m, k, SL_BAND_CT, cluster, &lo_k, &hi_k, &want, &cT);
  const float tau_lo = f32_from_order_key(lo_k), tau_hi = f32_from_order_key(hi_k);
  const float E = a.eps_dot * sh.U * 1.0001f * knmax + 1.52587890625e-05f * fmaxf(fabsf(tau_lo), fabsf(tau_hi));
  const float band_hi = tau_hi + 2.f * E, band_lo = tau_lo - 2.f * E;
  // ---- classify: sure (above the band) as a bitmap, band entries as a list
  if (tid == 0) { sh.cnt = 0; sh.n_sure = 0; }
  __syncthreads();
  const int nwords = (m + 31) / 32;
  int my_sure = 0;
  for (int w = warp; w < nwords; w += SL_W) {
    const int i = 32 * w + lane;
    const float v = i < m ? sv[i] : 0.f;
    const bool sure = i < m && v > band_hi;
    const bool band = i < m && !sure && v >= band_lo;
    const uint32_t ba = __ballot_sync(0xffffffffu, sure);
    if (lane == 0) { sh.bits_a[w] = ba; my_sure += __popc(ba); }
    if (band) {
      const uint32_t s = atomicAdd(&sh.cnt, 1u);
      if (s < (uint32_t)SL_CAP) sh.band_id[s] = lo + i;
    }
  }
  if (lane == 0 && my_sure) atomicAdd(&sh.n_sure, (uint32_t)my_sure);
  __syncthreads();                                         // sv is dead from here on
  const uint32_t nb_raw = sh.cnt;
  const int n_band = (int)min(nb_raw, (uint32_t)SL_CAP);
  if (nb_raw > (uint32_t)SL_CAP && tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
  if (!resc_sep) sl_stage_query(rs, qx, total, lgd, HI, dI);
  // ---- exact scores of this CTA's band entries (the first round's barrier covers the staging)
  sl_rescore_list<F>(rk, sh, rs, b, sh.band_id, n_band, sh.band_s);
  if (tid == 0) { sh.pub[0] = sh.n_sure; sh.pub[1] = (uint32_t)n_band; }
  sl_sync(cluster, C);
  // ---- gather every CTA's band and rank all of it (each CTA reaches the same verdicts)
  int ng = n_band;
  const int32_t* gid = sh.band_id;
  const double* gsc = sh.band_s;
  if (C > 1) {
    sl_gather_offsets(sh, cluster, C, 1);
    __syncthreads();
    ng = sl_gather(sh, cluster, C, sh.band_id, sh.gband_id, SL_CAP);
    sl_gather(sh, cluster, C, sh.band_s, sh.gband_s, SL_CAP);
    gid = sh.gband_id;
    gsc = sh.gband_s;
  }
  if (tid < SL_CMAX) {
    sh.pcnt[tid][0] = (unsigned)tid < C ? sl_peer(cluster, sh.pub, 0, tid) : 0u;
    sh.pcnt[tid][1] = 0u;
  }
  __syncthreads();
  int all_sure = 0;
#pragma unroll
  for (int p = 0; p < SL_CMAX; ++p) all_sure += (int)sh.pcnt[p][0];
  const int need = k - all_sure;
  for (int i = tid; i < ng; i += SL_T) {
    const double si = gsc[i];
    const int ii = gid[i];
    int rank = 0;
    for (int j = 0; j < ng; ++j) {
      const double sj = gsc[j];
      rank += (sj > si) || (sj == si && gid[j] < ii);
    }
    if (rank < need) {
      const int owner = ii / chunk;
      atomicAdd(&sh.pcnt[owner][1], 1u);
      if (owner == (int)r) atomicOr(&sh.bits_a[(ii - lo) >> 5], 1u << ((ii - lo) & 31));
    }
  }
  __syncthreads();
  int off = 0, tot_all = 0;
  for (int p = 0; p < (int)C; ++p) {
    const int c = (int)(sh.pcnt[p][0] + sh.pcnt[p][1]);
    if (p < (int)r) off += c;
    tot_all += c;
  }
  // ---- write the selected entries of this CTA in ascending order
  const int mine = sl_write(sh, sh.bits_a, nwords, lo, off, k, out);
  if (r == 0)
    for (int i = tot_all + tid; i < k; i += SL_T) out[i] = -1;
  if (sout) {
    // this CTA's selected entries, SL_CAP at a time (the gathered band arrays as scratch)
    const int p0 = off, p1 = min(k, off + mine);
    for (int c0 = p0; c0 < p1; c0 += SL_CAP) {
      const int cnt = min(SL_CAP, p1 - c0);
      __syncthreads();
      for (int i = tid; i < cnt; i += SL_T) sh.gband_id[i] = out[c0 + i];
      __syncthreads();
      sl_rescore_list<F>(rk, sh, rs, b, sh.gband_id, cnt, sh.gband_s);
      for (int i = tid; i < cnt; i += SL_T) sout[c0 + i] = (float)sh.gband_s[i];
    }
    if (r == 0)
      for (int i = tot_all + tid; i < k; i += SL_T) sout[i] = 0.f;
  }
  sl_sync(cluster, C);                                     // peers may still read band_id / band_s / pub
}

// Cluster size and chunk: the fewest CTAs (at most SL_CMAX) whose shared memory holds
// the row, more when there are few rows; chunk is a multiple of 1024 entries.
bool sl_plan(int64_t n, int rows, int* C, int* chunk) {
  const int64_t c = (n + SL_CHUNK - 1) / SL_CHUNK;
  if (c > SL_CMAX) return false;
  int64_t cc = c < 1 ? 1 : c;
  // few rows: up to four CTAs per row (their passes over the scores are shorter, their
  // band re-scoring is shared), while each CTA keeps at least 4096 entries
  if ((int64_t)rows * cc < num_sms()) {
    int64_t want = num_sms() / rows;
    if (want > 4) want = 4;
    while (want > cc && (n + want - 1) / want < 4096) --want;
    if (want > cc) cc = want;
  }
  int64_t ch = (n + cc - 1) / cc;
  ch = (ch + 1023) / 1024 * 1024;
  if (ch < 1024) ch = 1024;
  *C = (int)cc;
  *chunk = (int)ch;
  return true;
}

template <typename Kern, typename... Args>
cudaError_t sl_launch(Kern kern, int rows, int C, size_t smem, cudaStream_t st, Args... args) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * C);
  cfg.blockDim = dim3(SL_T);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the prologue overlaps the previous kernel's tail; the
  // kernels wait (griddepcontrol.wait) before reading anything that kernel writes
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // a cluster of C CTAs of this size must fit on the GPU (checked once per kernel, C and size)
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, size_t>, bool> fits;
  {
    std::lock_guard<std::mutex> g(mu);
    const auto key = std::make_tuple((const void*)kern, C, smem);
    auto it = fits.find(key);
    if (it == fits.end()) {
      int n_clusters = 0;
      const bool ok = cudaOccupancyMaxActiveClusters(&n_clusters, kern, &cfg) == cudaSuccess && n_clusters > 0;
      cudaGetLastError();
      it = fits.emplace(key, ok).first;
    }
    if (!it->second) return cudaErrorNotSupported;
  }
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

static_assert(SL_FIXED + sizeof(Resc) <= 232448 && SL_FIXED + (size_t)SL_CHUNK * 4 <= 232448,
              "shared memory budget of one CTA (227 KB)");

}  // namespace

// Returns cudaErrorNotSupported when the row is too long for one cluster (the caller
// then uses the single-CTA global-memory path).
cudaError_t launch_indexer_select_cluster(const IndexerArgs& a, cudaStream_t st) {
  int C, chunk;
  const int rows = a.B * a.Tq;
  if (a.H_I > 64 || a.d_I > 128 || a.H_I * a.d_I > SL_QPT * SL_T || !sl_plan(a.n_max, rows, &C, &chunk) || (a.ld % 4) != 0 ||
      ((uintptr_t)a.scores & 15) != 0 || (int64_t)rows * C > 0x7fffffffLL)
    return cudaErrorNotSupported;
  const size_t region = sl_resc_sep(chunk) ? sl_score_bytes(chunk) + sizeof(Resc) : std::max((size_t)chunk * 4, sizeof(Resc));
  if (a.ifmt == CSA_IFMT_E4M3) return sl_launch(indexer_select_cluster_kernel<CSA_IFMT_E4M3>, rows, C, SL_FIXED + region, st, a, chunk);
  if (a.ifmt == CSA_IFMT_MXFP4) return sl_launch(indexer_select_cluster_kernel<CSA_IFMT_MXFP4>, rows, C, SL_FIXED + region, st, a, chunk);
  return sl_launch(indexer_select_cluster_kernel<CSA_IFMT_F32>, rows, C, SL_FIXED + region, st, a, chunk);
}

cudaError_t launch_topk_select_cluster(const float* scores, int64_t ld, RowCount rc, int R, int64_t n,
                                       int k, int32_t* idx_out, cudaStream_t st) {
  int C, chunk;
  if (!sl_plan(n, R, &C, &chunk) || (int64_t)R * C > 0x7fffffffLL) return cudaErrorNotSupported;
  const int vec = (ld % 4 == 0) && (((uintptr_t)scores & 15) == 0);
  return sl_launch(topk_cluster_kernel, R, C, SL_FIXED + (size_t)chunk * 4, st, scores, ld, rc, n, k, idx_out,
                   chunk, vec);
}

}  // namespace csa
