// Exact top-k of the lightning indexer's decode rows, seeded by a score histogram.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 2: the indexer keeps the k compressed entries with the
// largest scores I[t,s] (k = 512 / 1024 from table "Конфигурации").  Ties go to the
// lower entry index; the selected set is written in ascending index order, padded with -1.
//
// The tensor-core scoring kernels write every eligible fp32 score of a row and, from their
// epilogues, a 4096-bin histogram of the scores' monotone order keys (bin = key >> 20:
// sign, exponent and the top three mantissa bits).  This kernel then needs one pass over
// the scores and no refinement chain over the whole row:
//
//  A. (every CTA; P CTAs share a row, each owns a contiguous chunk of entries)
//     1. The bin T that holds the k-th largest fp32 score follows from the histogram
//        (a suffix count over the bins).
//     2. The fp32 scores carry an error below E = eps * U * knmax + 2^-16 |tau| (eps of the
//        scoring path, U = sum_j |w_j| ||q_j||, knmax >= every key norm; the second term
//        covers the epilogue's head sum), so with tau anywhere in bin T = [b_lo, b_hi],
//        entries above b_hi + 2 E_max are certainly selected and entries below
//        b_lo - 2 E_max certainly not (E_max: E at |tau| = max(|b_lo|, |b_hi|)).
//     3. The CTA marks its certain entries in the row's bitmap, appends the rest of its
//        entries inside [b_lo - 2 E_max, b_hi + 2 E_max] to the row's candidate list, and
//        counts the certain ones.  The last CTA of the row to finish (an atomic counter
//        after a memory fence; no CTA waits for another) carries on alone.
//  B. (last CTA of the row)
//     4. tau = the exact fp32 k'-th largest candidate score, k' = k - (certain entries),
//        by radix refinement of the candidates' order keys (2048 bins per round).
//     5. Candidates above tau + 2E are in, below tau - 2E out; the band between is
//        re-scored exactly in fp64 from the quantised operands (FP8 / FP4 products and
//        their sums are exact in fp64; the per-head terms w_j * max(D_j, 0) are then added
//        in head order, as the definition does, so the scores equal the oracle's bit for
//        bit) and ranked by (exact score desc, index asc).
//     6. The row's bitmap (certain entries plus the chosen candidates) is scanned in
//        ascending order and the indices are written.
// A band larger than its buffer falls back to the fp32 order (score desc, index asc) and
// sets CSA_DEVERR_BAND.
#include "indexer.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int SH_T = 256;                // threads per CTA
constexpr int SH_W = SH_T / 32;
constexpr int SH_BINS = 4096;            // level-1 bins (key >> 20), written by the scoring epilogues
constexpr int SH_BINS2 = 2048;           // refinement bins
constexpr int SH_CCAP = 4096;            // candidates staged in shared memory (more stay in L2)
constexpr int SH_BAND = 512;             // band entries re-scored exactly
constexpr int SH_BMW = 8192;             // bitmap words handled per output pass (262 144 entries)

struct ShSmem {
  double qd[128][64];                    // query codes as fp64, [dim][head]: lanes read consecutive heads
  double krow[SH_W][128];                // one key row per warp (re-scoring)
  double contrib[SH_W][64];              // one entry's per-head terms per warp
  uint2 cand[SH_CCAP];                   // (order key, entry id)
  uint32_t bm[SH_BMW];                   // output bitmap chunk
  uint32_t tie[SH_BMW];                  // fallback: band entries equal to tau
  uint32_t hist2[SH_BINS2];
  int32_t band_id[SH_BAND];
  double band_s[SH_BAND];
  uint8_t band_take[SH_BAND];            // band entry chosen (rank by exact score, then index)
  float w[64];
  float qsc[64 * 4];
  uint32_t wred[SH_W][4];
  uint32_t bins_above, bin_T, cnt, cnt2, ties, last, lo, hi;
  int want;
  float U;
};

// Block-wide inclusive scan of one value per thread; *total = the sum over the block.
__device__ __forceinline__ uint32_t sh_scan(uint32_t v, uint32_t (*wred)[4], uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  __syncthreads();
  if (lane == 31) wred[warp][0] = incl;
  __syncthreads();
  uint32_t pre = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < SH_W; ++w) {
    const uint32_t x = wred[w][0];
    pre += (w < warp) ? x : 0u;
    tot += x;
  }
  *total = tot;
  return pre + incl;
}

// The bin holding the want-th largest key, bins[0..nb) with nb = SH_T * per; thread t holds
// bins [per*t, per*t + per) in cnt[].  Returns (through smem) the bin, the count of keys in
// bins above it, and want minus that count.  All threads call.
template <int PER>
__device__ __forceinline__ void sh_find_bin(ShSmem& sm, const uint32_t (&cnt)[PER], uint32_t want) {
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) mine += cnt[i];
  if (threadIdx.x == 0) { sm.bin_T = 0u; sm.bins_above = 0u; }   // (a consistent histogram always sets them)
  uint32_t tot;
  const uint32_t incl = sh_scan(mine, sm.wred, &tot);
  uint32_t above = tot - incl;                           // keys in the bins of higher threads
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    if (above < want && want <= above + cnt[i]) {
      sm.bin_T = (uint32_t)(PER * threadIdx.x + i);
      sm.bins_above = above;
    }
    above += cnt[i];
  }
  __syncthreads();
}

// What the exact re-scoring reads (passed by value: the address of a kernel parameter
// would copy the argument block to local memory).
struct KeySide {
  const void* kI;
  const void* kI_scale;
  int64_t n_max;
  int HI, dI;
};

// Exact fp64 score of entry `id` of sequence b, by one warp; the query row is staged in
// sm.qd / sm.qsc / sm.w.  Lane l forms the dot products of heads l and l + 32 over the key
// row (exact: every partial sum is a multiple of the code grid's product unit and spans
// fewer than 53 bits), applies the scales as the definition does, and lane 0 adds the
// head terms w_j * max(D_j, 0) in order j = 0..H_I-1.  Returns the score on lane 0.
template <int F>
__device__ __noinline__ double sh_exact_score(const KeySide ks, ShSmem& sm, int b, int id) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double* kr = sm.krow[warp];
  const size_t koff = (size_t)b * ks.n_max + id;
  const int dI = ks.dI, nb = dI / 32;
  // key codes of the row as fp64
  for (int c = lane; c < dI; c += 32) {
    double v;
    if (F == CSA_IFMT_E4M3) {
      v = (double)e4m3_to_float(((const uint8_t*)ks.kI)[koff * dI + c]);
    } else {
      const uint8_t byte = ((const uint8_t*)ks.kI)[koff * (dI / 2) + (c >> 1)];
      v = (double)e2m1_to_float((c & 1) ? (byte >> 4) : (byte & 0xF));
    }
    kr[c] = v;
  }
  double kscale[4] = {0.0, 0.0, 0.0, 0.0};
  if (F == CSA_IFMT_E4M3) {
    kscale[0] = (double)((const float*)ks.kI_scale)[koff];
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q < nb) kscale[q] = (double)ue8m0_to_float(((const uint8_t*)ks.kI_scale)[koff * nb + q]);
  }
  __syncwarp();
  for (int h = 0; h < 2; ++h) {
    const int j = lane + 32 * h;
    if (j < ks.HI) {
      double D = 0.0;
      if (F == CSA_IFMT_E4M3) {
        double acc = 0.0;
#pragma unroll 8
        for (int c = 0; c < dI; ++c) acc = fma(sm.qd[c][j], kr[c], acc);
        D = ((double)sm.qsc[j] * kscale[0]) * acc;
      } else {
        for (int q = 0; q < nb; ++q) {
          double part = 0.0;
#pragma unroll 8
          for (int c = 32 * q; c < 32 * q + 32; ++c) part = fma(sm.qd[c][j], kr[c], part);
          D += ((double)sm.qsc[j * nb + q] * kscale[q]) * part;
        }
      }
      sm.contrib[warp][j] = (double)sm.w[j] * fmax(D, 0.0);
    }
  }
  __syncwarp();
  double S = 0.0;
  if (lane == 0)
    for (int j = 0; j < ks.HI; ++j) S += sm.contrib[warp][j];
  __syncwarp();
  return S;
}

template <int F>
__global__ void __launch_bounds__(SH_T, 1)
indexer_select_hist_kernel(IndexerArgs a, int P, int chunk) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ShSmem& sm = *reinterpret_cast<ShSmem*>(smem_raw);
  const int row = blockIdx.x / P, part = blockIdx.x - row * P;
  const int b = row / a.Tq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.k, HI = a.H_I, dI = a.d_I, nb = dI / 32;
  const KeySide ks{a.kI, a.kI_scale, a.n_max, a.H_I, a.d_I};
  int32_t* out = a.idx_out + (size_t)row * k;
  float* sout = a.score_out ? a.score_out + (size_t)row * k : nullptr;
  uint32_t* hist = a.hist + (size_t)row * SH_BINS;
  uint32_t* ctr = a.counters + (size_t)row * 4;              // [0] candidates, [1] certain, [2] CTAs done
  uint32_t* bitmap = a.bitmap + (size_t)row * (a.ld / 32);
  uint2* cand_g = a.cand + (size_t)row * a.ld;
  tc::griddep_launch_dependents();

  // ---- prologue (inputs only; overlaps the scoring kernel): weights, query scales and
  // U = sum_j |w_j| ||q_j||.  Thread t takes 32 elements of head t / 4.
  const size_t qrow = (size_t)row * HI * dI;
  if (tid < HI) {
    sm.w[tid] = a.w[(size_t)row * HI + tid];
    if (F == CSA_IFMT_E4M3) sm.qsc[tid] = ((const float*)a.qI_scale)[(size_t)row * HI + tid];
    else
      for (int q = 0; q < nb; ++q) sm.qsc[tid * nb + q] = ue8m0_to_float(((const uint8_t*)a.qI_scale)[((size_t)row * HI + tid) * nb + q]);
  }
  if (tid == 0) sm.U = 0.f;
  __syncthreads();
  {
    const int j = tid >> 2, q = tid & 3;
    float ss = 0.f;
    if (j < HI && 32 * q < dI) {
      if (F == CSA_IFMT_E4M3) {
        const uint4* p = reinterpret_cast<const uint4*>((const uint8_t*)a.qI + qrow + (size_t)j * dI + 32 * q);
        const uint4 v0 = p[0], v1 = p[1];
        const uint32_t wds[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int e = 0; e < 32; ++e) { const float x = e4m3_to_float((wds[e >> 2] >> (8 * (e & 3))) & 0xFFu); ss = fmaf(x, x, ss); }
        ss *= sm.qsc[j] * sm.qsc[j];
      } else {
        const uint4 v = *reinterpret_cast<const uint4*>((const uint8_t*)a.qI + (qrow + (size_t)j * dI + 32 * q) / 2);
        const uint32_t wds[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 32; ++e) { const float x = e2m1_to_float((wds[e >> 3] >> (4 * (e & 7))) & 0xFu); ss = fmaf(x, x, ss); }
        const float sc = sm.qsc[j * nb + q];
        ss *= sc * sc;
      }
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    float u = (q == 0 && j < HI) ? fabsf(sm.w[j]) * sqrtf(ss) : 0.f;
    u = warp_sum(u);
    if (lane == 0) atomicAdd(&sm.U, u);
  }
  const int n = row_eligible(a, row);
  tc::griddep_wait();                                        // the scores, the histogram, knmax
  __syncthreads();
  if (n <= k) {
    // every eligible entry is selected
    if (part == 0) {
      for (int i = tid; i < k; i += SH_T) out[i] = i < n ? i : -1;
      if (sout) {
        // exact scores of entries 0..n-1 (one warp per entry) need the staged query row
        for (int i = tid; i < 128 * 64; i += SH_T) {
          const int c = i >> 6, j = i & 63;
          double v = 0.0;
          if (j < HI && c < dI) {
            if (F == CSA_IFMT_E4M3) v = (double)e4m3_to_float(((const uint8_t*)a.qI)[qrow + (size_t)j * dI + c]);
            else {
              const uint8_t byte = ((const uint8_t*)a.qI)[(qrow + (size_t)j * dI + c) >> 1];
              v = (double)e2m1_to_float((c & 1) ? (byte >> 4) : (byte & 0xF));
            }
          }
          sm.qd[c][j] = v;
        }
        __syncthreads();
        for (int i = warp; i < k; i += SH_W) {
          const double s = i < n ? sh_exact_score<F>(ks, sm, b, i) : 0.0;
          if (lane == 0) sout[i] = (float)s;
        }
      }
    }
    return;
  }

  // ---- A1: the bin T of the k-th largest score (thread t holds bins 16t .. 16t+15)
  {
    uint32_t cnt[SH_BINS / SH_T];
    const uint4* hp = reinterpret_cast<const uint4*>(hist + (SH_BINS / SH_T) * tid);
#pragma unroll
    for (int v = 0; v < SH_BINS / SH_T / 4; ++v) {
      const uint4 x = hp[v];
      cnt[4 * v] = x.x; cnt[4 * v + 1] = x.y; cnt[4 * v + 2] = x.z; cnt[4 * v + 3] = x.w;
    }
    sh_find_bin<SH_BINS / SH_T>(sm, cnt, (uint32_t)k);
  }
  const uint32_t T = sm.bin_T;
  const float knmax = __uint_as_float(a.knmax[b]);
  const float b_lo = f32_from_order_key(T << 20), b_hi = f32_from_order_key((T << 20) | 0xFFFFFu);
  const float EU = a.eps_dot * sm.U * 1.0001f * knmax;
  const float E_max = (EU + 1.52587890625e-05f * fmaxf(fabsf(b_lo), fabsf(b_hi))) * 1.0001f;
  const float hi_thr = b_hi + 2.f * E_max, lo_thr = b_lo - 2.f * E_max;

  // ---- A2: classify this CTA's chunk (whole bitmap words: chunk % 32 == 0)
  const int c0 = part * chunk, c1 = min(n, c0 + chunk);
  const float* srow = a.scores + (size_t)row * a.ld;
  uint32_t n_sure = 0;
  for (int base = c0 + 32 * warp; base < c0 + chunk && base < (int)a.ld; base += 32 * SH_W) {
    const int i = base + lane;
    const float s = i < c1 ? srow[i] : 0.f;
    const bool sure = i < c1 && s > hi_thr;
    const bool cnd = i < c1 && !sure && s >= lo_thr;
    const uint32_t bs = __ballot_sync(0xffffffffu, sure);
    const uint32_t bc = __ballot_sync(0xffffffffu, cnd);
    if (lane == 0) bitmap[base >> 5] = bs;
    n_sure += __popc(bs);
    if (bc) {
      uint32_t off = 0;
      if (lane == 0) off = atomicAdd(&ctr[0], (uint32_t)__popc(bc));
      off = __shfl_sync(0xffffffffu, off, 0);
      if (cnd) cand_g[off + __popc(bc & ((1u << lane) - 1u))] = make_uint2(f32_order_key(s), (uint32_t)i);
    }
  }
  if (lane == 0 && n_sure) atomicAdd(&ctr[1], n_sure);
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = (atomicAdd(&ctr[2], 1u) == (uint32_t)(P - 1)) ? 1u : 0u;
  __syncthreads();
  if (!sm.last) return;
  __threadfence();

  // ---- B: the last CTA of the row.  Stage the query row as fp64 (for the re-scoring).
  for (int i = tid; i < 128 * 64; i += SH_T) {
    const int c = i >> 6, j = i & 63;
    double v = 0.0;
    if (j < HI && c < dI) {
      if (F == CSA_IFMT_E4M3) v = (double)e4m3_to_float(((const uint8_t*)a.qI)[qrow + (size_t)j * dI + c]);
      else {
        const uint8_t byte = ((const uint8_t*)a.qI)[(qrow + (size_t)j * dI + c) >> 1];
        v = (double)e2m1_to_float((c & 1) ? (byte >> 4) : (byte & 0xF));
      }
    }
    sm.qd[c][j] = v;
  }
  const uint32_t nc = *(volatile uint32_t*)&ctr[0];
  const uint32_t n_sure_all = *(volatile uint32_t*)&ctr[1];
  const bool staged = nc <= (uint32_t)SH_CCAP;
  // candidates: staged in shared memory when they fit, else read from L2 each pass
  auto cget = [&](uint32_t i) { return staged ? sm.cand[i] : __ldcg(cand_g + i); };
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (uint32_t i = tid; i < nc; i += SH_T) {
    const uint2 c = __ldcg(cand_g + i);
    if (staged) sm.cand[i] = c;
    kmin = min(kmin, c.x);
    kmax = max(kmax, c.x);
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (tid == 0) { sm.lo = 0xFFFFFFFFu; sm.hi = 0u; }
  __syncthreads();
  if (lane == 0) { atomicMin(&sm.lo, kmin); atomicMax(&sm.hi, kmax); }
  __syncthreads();
  // ---- B4: tau = the exact want-th largest candidate key
  uint32_t lo = sm.lo, hi = sm.hi;
  uint32_t want = (uint32_t)k - n_sure_all;
  for (int round = 0; round < 4 && lo != hi; ++round) {
    const int range_bits = 32 - __clz(hi - lo);
    const int shf = range_bits > 11 ? range_bits - 11 : 0;
    for (int i = tid; i < SH_BINS2; i += SH_T) sm.hist2[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < nc; i += SH_T) {
      const uint32_t x = cget(i).x;
      if (x >= lo && x <= hi) atomicAdd(&sm.hist2[(x - lo) >> shf], 1u);
    }
    __syncthreads();
    uint32_t cnt[SH_BINS2 / SH_T];
#pragma unroll
    for (int i = 0; i < SH_BINS2 / SH_T; ++i) cnt[i] = sm.hist2[(SH_BINS2 / SH_T) * tid + i];
    sh_find_bin<SH_BINS2 / SH_T>(sm, cnt, want);
    want -= sm.bins_above;
    const uint32_t nlo = lo + (sm.bin_T << shf);
    const uint64_t top = (uint64_t)nlo + ((1ull << shf) - 1ull);
    hi = top < (uint64_t)hi ? (uint32_t)top : hi;
    lo = nlo;
    __syncthreads();
  }
  const float tau = f32_from_order_key(lo);
  const float E = (EU + 1.52587890625e-05f * fabsf(tau)) * 1.0001f;
  const float band_hi = tau + 2.f * E, band_lo = tau - 2.f * E;
  // ---- B5: in / band; the band is re-scored exactly and ranked
  if (tid == 0) { sm.cnt = 0u; sm.cnt2 = 0u; sm.ties = 0u; }
  __syncthreads();
  uint32_t my_in = 0, my_above = 0;
  for (uint32_t i = tid; i < nc; i += SH_T) {
    const uint2 c = cget(i);
    const float s = f32_from_order_key(c.x);
    if (s > band_hi) {
      ++my_in;
    } else if (s >= band_lo) {
      my_above += s > tau ? 1u : 0u;
      const uint32_t o = atomicAdd(&sm.cnt, 1u);
      if (o < (uint32_t)SH_BAND) sm.band_id[o] = (int32_t)c.y;
    }
  }
  uint32_t n_in, n_above_tau;
  sh_scan(my_in, sm.wred, &n_in);
  sh_scan(my_above, sm.wred, &n_above_tau);
  const uint32_t n_band = sm.cnt;
  const uint32_t need = (uint32_t)k - n_sure_all - n_in;    // >= 1: tau itself is in the band
  const bool exact = n_band <= (uint32_t)SH_BAND;
  if (!exact && tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
  if (exact) {
    for (uint32_t i = warp; i < n_band; i += SH_W) {
      const double s = sh_exact_score<F>(ks, sm, b, sm.band_id[i]);
      if (lane == 0) sm.band_s[i] = s;
    }
    __syncthreads();
    for (uint32_t i = tid; i < n_band; i += SH_T) {
      const double si = sm.band_s[i];
      const int id = sm.band_id[i];
      uint32_t rank = 0;
      for (uint32_t j = 0; j < n_band; ++j) {
        const double sj = sm.band_s[j];
        rank += (sj > si) || (sj == si && sm.band_id[j] < id);
      }
      sm.band_take[i] = rank < need ? 1 : 0;
    }
    __syncthreads();
  }
  // ---- B6: ascending write, SH_BMW bitmap words (32 * SH_BMW entries) per pass
  const int nwords = (n + 31) >> 5;
  uint32_t written = 0;
  // fallback (band beyond its buffer): band entries above tau are in, and the first
  // (need - those) entries equal to tau in index order
  const uint32_t quota = need > n_above_tau ? need - n_above_tau : 0u;
  for (int w0 = 0; w0 < nwords; w0 += SH_BMW) {
    const int w1 = min(nwords, w0 + SH_BMW);
    const int e0 = 32 * w0, e1 = 32 * w1;
    for (int w = w0 + tid; w < w1; w += SH_T) { sm.bm[w - w0] = __ldcg(bitmap + w); sm.tie[w - w0] = 0u; }
    __syncthreads();
    for (uint32_t i = tid; i < nc; i += SH_T) {
      const uint2 c = cget(i);
      const int id = (int)c.y;
      if (id < e0 || id >= e1) continue;
      const float s = f32_from_order_key(c.x);
      bool take = s > band_hi;
      if (!exact && !take && s >= band_lo) {
        take = s > tau;
        if (s == tau) atomicOr(&sm.tie[(id - e0) >> 5], 1u << ((id - e0) & 31));
      }
      if (take) atomicOr(&sm.bm[(id - e0) >> 5], 1u << ((id - e0) & 31));
    }
    if (exact) {
      for (uint32_t i = tid; i < n_band; i += SH_T) {
        const int id = sm.band_id[i];
        if (sm.band_take[i] && id >= e0 && id < e1) atomicOr(&sm.bm[(id - e0) >> 5], 1u << ((id - e0) & 31));
      }
    }
    __syncthreads();
    const int nw = w1 - w0, wpt = (nw + SH_T - 1) / SH_T;
    const int a0 = tid * wpt, a1 = min(nw, a0 + wpt);
    if (!exact) {
      uint32_t c = 0;
      for (int w = a0; w < a1; ++w) c += __popc(sm.tie[w]);
      uint32_t tot;
      uint32_t seen = sh_scan(c, sm.wred, &tot) - c + sm.ties;     // ties of earlier passes first
      for (int w = a0; w < a1; ++w) {
        uint32_t keep = 0u;
        for (uint32_t bits = sm.tie[w]; bits; bits &= bits - 1) {
          if (seen < quota) keep |= bits & (0u - bits);
          ++seen;
        }
        sm.bm[w] |= keep;
      }
      __syncthreads();
      if (tid == 0) sm.ties += tot;
    }
    // prefix counts over the words (contiguous words per thread) and the write
    uint32_t c = 0;
    for (int w = a0; w < a1; ++w) c += __popc(sm.bm[w]);
    uint32_t tot;
    uint32_t pos = written + sh_scan(c, sm.wred, &tot) - c;
    for (int w = a0; w < a1; ++w)
      for (uint32_t bits = sm.bm[w]; bits; bits &= bits - 1) {
        if (pos < (uint32_t)k) out[pos] = e0 + 32 * w + __ffs(bits) - 1;
        ++pos;
      }
    written += tot;
    __syncthreads();
  }
  for (uint32_t i = written + tid; i < (uint32_t)k; i += SH_T) out[i] = -1;
  if (written != (uint32_t)k && tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
  if (sout) {
    __syncthreads();
    for (int i = warp; i < k; i += SH_W) {
      const int id = __ldcg(out + i);
      const double s = id >= 0 ? sh_exact_score<F>(ks, sm, b, id) : 0.0;
      if (lane == 0) sout[i] = (float)s;
    }
  }
}

}  // namespace

// Launch plan: P CTAs per row, one wave over the SMs when the rows allow, each CTA a
// multiple of 32 entries.  Returns cudaErrorNotSupported for shapes this path does not
// take (the caller then runs the cluster selection).
cudaError_t launch_indexer_select_hist(const IndexerArgs& a, cudaStream_t st) {
  if (!a.hist || a.H_I > 64 || a.d_I > 128 || (a.ifmt != CSA_IFMT_E4M3 && a.ifmt != CSA_IFMT_MXFP4))
    return cudaErrorNotSupported;
  const int rows = a.B * a.Tq;
  int P = num_sms() / rows;
  if (P < 1) P = 1;
  const int64_t min_chunk = 1024;
  if ((int64_t)P * min_chunk > a.n_max) P = (int)((a.n_max + min_chunk - 1) / min_chunk);
  if (P < 1) P = 1;
  int64_t chunk = (a.n_max + P - 1) / P;
  chunk = (chunk + 31) / 32 * 32;
  P = (int)((a.n_max + chunk - 1) / chunk);
  if ((int64_t)rows * P > 0x7fffffffLL) return cudaErrorNotSupported;
  const size_t smem = sizeof(ShSmem);
  auto kern = a.ifmt == CSA_IFMT_E4M3 ? indexer_select_hist_kernel<CSA_IFMT_E4M3> : indexer_select_hist_kernel<CSA_IFMT_MXFP4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * P);
  cfg.blockDim = dim3(SH_T);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  // programmatic dependent launch: the prologue (query row, U) overlaps the scoring kernel
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, a, P, (int)chunk);
}

static_assert(sizeof(ShSmem) <= 232448, "shared memory budget of one CTA (227 KB)");

}  // namespace csa
