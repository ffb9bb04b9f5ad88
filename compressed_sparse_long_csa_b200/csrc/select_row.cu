// Exact top-k of the lightning indexer's decode rows: one thread-block cluster per row, the
// row's scores staged in every CTA's shared memory.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 2: the indexer keeps the k compressed entries with the
// largest scores I[t,s] (k = 512 / 1024 from table "Конфигурации").  Ties go to the
// lower entry index; the selected set is written in ascending index order, padded with -1.
//
// The tensor-core scoring kernel writes the row's fp32 scores (L2-resident at decode
// sizes), their order-key range and a bound on the key norms.  Every CTA of the row's
// cluster then does the same selection work on its own copy of the scores (the passes are
// shared-memory bound and run side by side), and the exact re-scoring of the band is split
// over the CTAs:
//   1. bulk-copy the n scores into shared memory while the query codes become integers;
//   2. histogram the scores' monotone order keys over the row's key range (4096 bins,
//      bin = (key - lo) >> s): the bin holding the k-th largest key, [b_lo, b_hi];
//   3. every fp32 score differs from the exact one by less than
//      E = (eps + 2^-19) U knmax + 2^-16 |tau|  (eps: the MMA dot product's bound, 2^-19: the
//      epilogue's head sum and weight rounding, 2^-16 |tau|: the final scale; U = sum_j
//      |w_j| ||q_j||, knmax >= every key norm).  One pass marks the entries above
//      b_hi + 2E as certain and lists the ones in [b_lo - 2E, b_hi + 2E] as candidates;
//   4. the exact k-th largest fp32 key tau comes from the candidates (at most two more
//      histograms over the bin); the exact k-th largest score lies in [tau - E, tau + E], so
//      candidates above tau + 2E are certain too and the band [tau - 2E, tau + 2E] holds
//      every entry whose order is in doubt (a few dozen at most at these sizes);
//   5. the band's exact scores: FP8 / FP4 codes times a power of two are small integers, so
//      each head's dot product is an exact integer sum (64-bit multiply-adds for E4M3, 32-bit
//      for the FP4 blocks); the head's term w_j * max(D_j, 0) is then formed in fp64 as the
//      definition does and the terms are added in head order, so each score equals the
//      oracle's bit for bit.  CTA c of the cluster re-scores band entries c, c + C, ... and
//      stores them into the first CTA's shared memory;
//   6. the first CTA ranks the band by (exact score desc, index asc), takes its first
//      k - (certain entries), and writes the row's bitmap out in ascending order.
// A band or candidate list larger than its buffer (heavy ties) is handled on the whole
// row: the fp32 order (score desc, index asc) decides the band, and CSA_DEVERR_BAND is set.
#include "indexer.cuh"
#include "tc.cuh"

#include <cooperative_groups.h>
#include <map>
#include <mutex>

namespace cg = cooperative_groups;

namespace csa {
namespace {

constexpr int SR_T = 512;                 // threads per CTA
constexpr int SR_W = SR_T / 32;
constexpr int SR_CMAX = 8;                // CTAs per cluster
constexpr int SR_HB = 4096;               // bins of the first histogram
constexpr int SR_HB2 = 2048;              // bins of the refinements
constexpr int SR_CCAP = 2048;             // candidates listed
constexpr int SR_BCAP = 512;              // band entries re-scored exactly (at most one per thread: the sort)
constexpr int SR_RB = 8;                  // entries re-scored at once (one per thread of a head's eight)
constexpr int SR_NMAX = 34816;            // most scores a row stages in shared memory (and bitmap bits)
constexpr int SR_CHUNK = 16384;           // bytes per bulk copy (the first histogram starts on the first)
constexpr int SR_KLD = 160;               // staged key row: dims 16 g .. 16 g + 15 at word 20 g (no bank conflicts)
static_assert(SR_RB == 8, "the re-scoring gives each of a head's eight threads one entry");
constexpr int SR_TLD = 66;                // per-head term row stride (the ordered sums read rows side by side)
constexpr int SD_CMAX = 16;               // CTAs per cluster of the chunked selection (above 8: non-portable size)
constexpr int SD_LCAP = 1024;             // candidates (or band entries) one CTA of it lists

// What the CTAs of a chunked-selection cluster tell each other: every CTA stores its entry c
// of each array into every CTA of the cluster, and reads them after the next cluster barrier.
struct SdXchg {
  uint32_t fail[SD_CMAX];                 // a score copy that did not land
  uint32_t stot[SD_CMAX];                 // total of the histogram slice the CTA summed
  uint32_t nsure[SD_CMAX], ncand[SD_CMAX];  // certain entries marked and candidates listed in its chunk
  uint32_t nsure2[SD_CMAX], nband[SD_CMAX];  // after a counted search of tau: entries above the band, band entries
  uint32_t cnt[2][SD_CMAX][2];            // counting rounds (two buffers: a round's values are read before the
                                          // barrier that ends the next one)
};

struct SrSmem {
  uint32_t hist[SR_HB];
  uint32_t bm[SR_NMAX / 32];              // selection bitmap
  uint32_t tb[SR_NMAX / 32];              // fp32-order fallback: entries equal to tau
  int32_t cid[SR_CCAP];                   // candidates
  uint32_t ckey[SR_CCAP];
  int32_t bid[SR_BCAP];                   // band entries, ascending index
  int32_t bid_raw[SR_BCAP];
  double bs[SR_BCAP];                     // their exact scores (stored by every CTA of the cluster)
  alignas(16) int32_t kint[SR_RB][SR_KLD];            // key codes of a re-scoring batch as integers (16 dims per 20 words)
  float ksc[SR_RB][4];                    // their scales
  double term[SR_RB][SR_TLD];             // their per-head terms
  double rs[SR_RB];                       // their exact scores
  int32_t rid[SR_RB];
  float w[64];
  float qsc[64 * 4];
  uint32_t wred[SR_W];
  alignas(8) uint64_t bar[(SR_NMAX * 4 + SR_CHUNK - 1) / SR_CHUNK];   // one per bulk copy
  uint32_t bin, above, ccnt, bcnt, nsure, fail;
  uint32_t kr_mx, kr_nmn, kn;             // the row's key range and key-norm bound (reduced over partials)
  float U;
  // chunked selection only
  uint32_t hsum[SR_HB / 2];               // the cluster's histogram: this CTA's slice of it (C >= 2)
  int32_t lid[SD_LCAP];                   // this chunk's candidates (row indices) and their keys
  uint32_t lkey[SD_LCAP];
  SdXchg x;
  uint32_t sure[SD_CMAX], win[SD_CMAX];   // per chunk: entries selected for certain, band entries chosen
  uint32_t tot;
  alignas(16) float sc[1];                // the row's scores (sized at launch)
};
static_assert(sizeof(SrSmem) - sizeof(float) + SR_NMAX * sizeof(float) + 1024 <= 232448,
              "the largest staged row fits one CTA's shared memory");

// Block-wide inclusive scan of one value per thread; *total = the block's sum.  All threads call.
__device__ __forceinline__ uint32_t sr_scan(uint32_t v, uint32_t* wred, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  __syncthreads();
  if (lane == 31) wred[warp] = incl;
  __syncthreads();
  uint32_t pre = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < SR_W; ++w) {
    const uint32_t x = wred[w];
    pre += w < warp ? x : 0u;
    tot += x;
  }
  *total = tot;
  return pre + incl;
}

// The bin of sm.hist[0, PER * SR_T) holding the want-th largest key: sets sm.bin and
// sm.above (keys in higher bins).  All threads call.
template <int PER>
__device__ __forceinline__ void sr_find_bin(SrSmem& sm, uint32_t want) {
  uint32_t c[PER], mine = 0;
  if (PER % 4 == 0) {
#pragma unroll
    for (int i = 0; i < PER; i += 4) {
      const uint4 v = reinterpret_cast<const uint4*>(sm.hist + PER * threadIdx.x)[i / 4];
      c[i] = v.x; c[(i + 1) % PER] = v.y; c[(i + 2) % PER] = v.z; c[(i + 3) % PER] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < PER; ++i) c[i] = sm.hist[PER * threadIdx.x + i];
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) mine += c[i];
  if (threadIdx.x == 0) { sm.bin = 0u; sm.above = 0u; }
  uint32_t tot;
  const uint32_t incl = sr_scan(mine, sm.wred, &tot);
  uint32_t above = tot - incl;                               // keys in the bins of higher threads
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    if (above < want && want <= above + c[i]) {
      sm.bin = (uint32_t)(PER * threadIdx.x + i);
      sm.above = above;
    }
    above += c[i];
  }
  __syncthreads();
}

// The band's exact scores sm.bs[0, nbnd) replaced in place by monotone 64-bit keys (x + 0.0
// folds -0 into +0; exact scores are never NaN), so that ranking compares integers instead of
// running on the fp64 pipe.  All threads call (one barrier).
__device__ __forceinline__ void sr_band_keys(SrSmem& sm, uint32_t nbnd) {
  for (uint32_t i = threadIdx.x; i < nbnd; i += SR_T) {
    const uint64_t u = (uint64_t)__double_as_longlong(sm.bs[i] + 0.0);
    reinterpret_cast<uint64_t*>(sm.bs)[i] = (u >> 63) ? ~u : (u | 0x8000000000000000ull);
  }
  __syncthreads();
}

// Histogram shift: the smallest s with (width - 1) >> s < 2^log2_bins.
__device__ __forceinline__ int sr_shift(uint64_t width, int log2_bins) {
  const int bits = width <= 1 ? 0 : 64 - __clzll((long long)(width - 1));
  return bits > log2_bins ? bits - log2_bins : 0;
}

// Exact fp64 scores of entries sm.rid[0, cnt) (cnt <= SR_RB) of sequence b into sm.rs, by
// the whole CTA (all threads call; barriers inside).  Thread t owns head t / 8 and dims
// [16 (t % 8), +16), whose query codes it holds as integers in qi (E4M3: value * 2^9; FP4:
// value * 2).  A head's dot product is an exact integer (E4M3: |sum| < 2^43 in 64 bits,
// then * 2^-18; FP4: each 32-dim block below 2^13 in 32 bits, then * 2^-2); the head term
// and the ordered head sum follow the definition in fp64.
template <int F>
__device__ __forceinline__ void sr_rescore(SrSmem& sm, const IndexerArgs& a, int b, int cnt, const int (&qi)[16]) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int HI = a.H_I, dI = a.d_I, nb = dI / 32;
  // ---- stage the key codes: thread t converts 4 codes of entry t / 32
  if (tid < 32 * SR_RB) {
    const int e = tid >> 5;
    if (e < cnt && 4 * lane < dI) {
      const size_t koff = (size_t)b * a.n_max + sm.rid[e];
      int* kr = sm.kint[e];
      if (F == CSA_IFMT_E4M3) {
        const uint32_t v = *(reinterpret_cast<const uint32_t*>((const uint8_t*)a.kI + koff * dI) + lane);
        const int4 w4 = make_int4((int)(e4m3_to_float(v & 0xFFu) * 512.f), (int)(e4m3_to_float((v >> 8) & 0xFFu) * 512.f),
                                  (int)(e4m3_to_float((v >> 16) & 0xFFu) * 512.f), (int)(e4m3_to_float(v >> 24) * 512.f));
        *reinterpret_cast<int4*>(kr + 20 * (lane >> 2) + 4 * (lane & 3)) = w4;
      } else {
        const uint32_t v = *(reinterpret_cast<const uint16_t*>((const uint8_t*)a.kI + koff * (dI / 2)) + lane);
        const int4 w4 = make_int4((int)(e2m1_to_float(v & 0xFu) * 2.f), (int)(e2m1_to_float((v >> 4) & 0xFu) * 2.f),
                                  (int)(e2m1_to_float((v >> 8) & 0xFu) * 2.f), (int)(e2m1_to_float((v >> 12) & 0xFu) * 2.f));
        *reinterpret_cast<int4*>(kr + 20 * (lane >> 2) + 4 * (lane & 3)) = w4;
      }
      if (lane < 4) {
        float s = 0.f;
        if (F == CSA_IFMT_E4M3) s = lane == 0 ? ((const float*)a.kI_scale)[koff] : 0.f;
        else s = lane < nb ? ue8m0_to_float(((const uint8_t*)a.kI_scale)[koff * nb + lane]) : 0.f;
        sm.ksc[e][lane] = s;
      }
    }
  }
  __syncthreads();
  // ---- per-head terms: the batch's entries as independent chains
  const int j = tid >> 3, g = tid & 7;
  const bool live = j < HI && 16 * g < dI;
  if (F == CSA_IFMT_E4M3) {
    long long acc[SR_RB];
#pragma unroll
    for (int e = 0; e < SR_RB; ++e) acc[e] = 0;
    if (live) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int e = 0; e < SR_RB; ++e) {
          if (e < cnt) {
            const int4 kv = reinterpret_cast<const int4*>(sm.kint[e] + 20 * g)[u];
            long long x = acc[e];
            x += (long long)qi[4 * u] * kv.x;
            x += (long long)qi[4 * u + 1] * kv.y;
            x += (long long)qi[4 * u + 2] * kv.z;
            x += (long long)qi[4 * u + 3] * kv.w;
            acc[e] = x;
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < SR_RB; ++e) {
      if (e < cnt) {
        long long x = acc[e];
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        acc[e] = x;
      }
    }
    // every lane of the head holds the sums: thread g forms the term of entry g (the fp64
    // pipe is narrow on this GPU, so the terms go to all lanes rather than one per head)
    long long mine = 0;
#pragma unroll
    for (int e = 0; e < SR_RB; ++e) mine = e == g ? acc[e] : mine;
    if (j < HI && g < cnt) {
      const double D = ((double)sm.qsc[j] * (double)sm.ksc[g][0]) * ((double)mine * 3.814697265625e-06);   // 2^-18
      sm.term[g][j] = (double)sm.w[j] * fmax(D, 0.0);
    }
  } else {
    int acc[SR_RB];
#pragma unroll
    for (int e = 0; e < SR_RB; ++e) acc[e] = 0;
    if (live) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int e = 0; e < SR_RB; ++e) {
          if (e < cnt) {
            const int4 kv = reinterpret_cast<const int4*>(sm.kint[e] + 20 * g)[u];
            acc[e] += qi[4 * u] * kv.x + qi[4 * u + 1] * kv.y + qi[4 * u + 2] * kv.z + qi[4 * u + 3] * kv.w;
          }
        }
      }
    }
    // the 32-dim block q of a head sums lanes 2q and 2q + 1 of its eight; thread g takes the
    // block sums of entry g and forms its term (blocks added in order)
    int P[4] = {0, 0, 0, 0};
#pragma unroll
    for (int e = 0; e < SR_RB; ++e) {
      if (e < cnt) {
        const int x = acc[e] + __shfl_xor_sync(0xffffffffu, acc[e], 1);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int pq = __shfl_sync(0xffffffffu, x, (lane & ~7) | (2 * q));
          P[q] = e == g ? pq : P[q];
        }
      }
    }
    if (j < HI && g < cnt) {
      double D = 0.0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q >= nb) break;
        const double t = ((double)sm.qsc[j * nb + q] * (double)sm.ksc[g][q]) * ((double)P[q] * 0.25);
        D = q == 0 ? t : D + t;
      }
      sm.term[g][j] = (double)sm.w[j] * fmax(D, 0.0);
    }
  }
  __syncthreads();
  if (tid < cnt) {
    double S = 0.0;
    for (int jj = 0; jj < HI; ++jj) S += sm.term[tid][jj];
    sm.rs[tid] = S;
  }
  __syncthreads();
}

// The row kernels' prologue (inputs only; it overlaps the scoring kernel): head weights and
// query scales into shared memory, the copy barriers, zeroed counters, thread t's query codes
// (head t / 8, dims [16 (t % 8), +16)) as integers in qi, and U = sum_j |w_j| ||q_j|| added
// into sm.U (complete after the caller's next barrier).  All threads call.
template <int F>
__device__ __forceinline__ void sr_prologue(SrSmem& sm, const IndexerArgs& a, int row, int (&qi)[16]) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int HI = a.H_I, dI = a.d_I, nb = dI / 32;
  if (tid < HI) {
    sm.w[tid] = a.w[(size_t)row * HI + tid];
    if (F == CSA_IFMT_E4M3) sm.qsc[tid] = ((const float*)a.qI_scale)[(size_t)row * HI + tid];
    else
      for (int q = 0; q < nb; ++q)
        sm.qsc[tid * nb + q] = ue8m0_to_float(((const uint8_t*)a.qI_scale)[((size_t)row * HI + tid) * nb + q]);
  }
  if (tid == 0) {
    for (int c = 0; c < (SR_NMAX * 4 + SR_CHUNK - 1) / SR_CHUNK; ++c) tc::mbar_init(&sm.bar[c], 1);
    tc::fence_mbar_init();
    sm.U = 0.f;
    sm.ccnt = 0u;
    sm.bcnt = 0u;
    sm.nsure = 0u;
    sm.fail = 0u;
  }
  // thread t: head t / 8, dims [16 (t % 8), +16)
  const int qj = tid >> 3, qs = tid & 7;
  const bool qlive = qj < HI && 16 * qs < dI;
  float qv[16];
  {
    const size_t qrow = (size_t)row * HI * dI;
    if (F == CSA_IFMT_E4M3) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (qlive) v = *reinterpret_cast<const uint4*>((const uint8_t*)a.qI + qrow + (size_t)qj * dI + 16 * qs);
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) qv[i] = e4m3_to_float((wd[i >> 2] >> (8 * (i & 3))) & 0xFFu);
#pragma unroll
      for (int i = 0; i < 16; ++i) qi[i] = (int)(qv[i] * 512.f);                // exact: codes are multiples of 2^-9
    } else {
      uint2 v = make_uint2(0u, 0u);
      if (qlive) v = *reinterpret_cast<const uint2*>((const uint8_t*)a.qI + (qrow + (size_t)qj * dI + 16 * qs) / 2);
      const uint32_t wd[2] = {v.x, v.y};
#pragma unroll
      for (int i = 0; i < 16; ++i) qv[i] = e2m1_to_float((wd[i >> 3] >> (4 * (i & 7))) & 0xFu);
#pragma unroll
      for (int i = 0; i < 16; ++i) qi[i] = (int)(qv[i] * 2.f);                  // exact: codes are multiples of 1/2
    }
  }
  __syncthreads();                                           // w, scales, the barrier, U = 0
  {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) ss = fmaf(qv[i], qv[i], ss);
    if (qlive) {
      const float sc = F == CSA_IFMT_E4M3 ? sm.qsc[qj] : sm.qsc[qj * nb + (16 * qs) / 32];
      ss *= sc * sc;
    } else {
      ss = 0.f;
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    float u = (qs == 0 && qj < HI) ? fabsf(sm.w[qj]) * sqrtf(ss) : 0.f;
    u = warp_sum(u);
    if (lane == 0) atomicAdd(&sm.U, u);
  }
}

template <int F>
__global__ void __launch_bounds__(SR_T, 1)
indexer_select_row_kernel(IndexerArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SrSmem& sm = *reinterpret_cast<SrSmem*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks(), crank = (int)cluster.block_rank();
  const bool leader = crank == 0;
  const int row = blockIdx.x / C, b = row / a.Tq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.k;
  int32_t* out = a.idx_out + (size_t)row * k;
  float* sout = a.score_out ? a.score_out + (size_t)row * k : nullptr;

  // ---- prologue (inputs only; overlaps the scoring kernel)
  int qi[16];
  sr_prologue<F>(sm, a, row, qi);
  const int n = row_eligible(a, row);
  tc::griddep_wait();                                        // the scores, their key range, knmax
  tc::griddep_launch_dependents();

  if (n <= k) {
    // every eligible entry is selected (the first CTA writes)
    if (!leader) return;
    for (int i = tid; i < k; i += SR_T) out[i] = i < n ? i : -1;
    if (sout) {
      __syncthreads();
      for (int i0 = 0; i0 < k; i0 += SR_RB) {
        const int cnt = max(0, min(SR_RB, n - i0));
        if (tid < SR_RB) sm.rid[tid] = i0 + tid;
        __syncthreads();
        if (cnt > 0) sr_rescore<F>(sm, a, b, cnt, qi);
        if (tid < SR_RB && i0 + tid < k) sout[i0 + tid] = tid < cnt ? (float)sm.rs[tid] : 0.f;
        __syncthreads();
      }
    }
    return;
  }

  // ---- 1. the row's scores into shared memory, in 16 KB copies
  const uint32_t bytes = (uint32_t)(((n + 3) & ~3) * 4);      // whole 16-byte units (ld is a multiple of 64)
  const int nch = (int)((bytes + SR_CHUNK - 1) / SR_CHUNK);
  if (tid == 0) {
    const char* src = (const char*)(a.scores + (size_t)row * a.ld);
    for (int c = 0; c < nch; ++c) {
      const uint32_t o = (uint32_t)c * SR_CHUNK;
      const uint32_t len = bytes - o < (uint32_t)SR_CHUNK ? bytes - o : (uint32_t)SR_CHUNK;
      tc::mbar_arrive_expect_tx(&sm.bar[c], len);
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(tc::smem_u32((char*)sm.sc + o)), "l"(src + o), "r"(len), "r"(tc::smem_u32(&sm.bar[c]))
                   : "memory");
    }
  }
  for (int i = tid; i < SR_HB; i += SR_T) sm.hist[i] = 0u;
  if (warp == 0) {
    // the scoring kernel's key range and key-norm bound: one value, or one per split
    uint32_t x = 0u, y = 0u, z = 0u;
    if (a.kpart == 0) {
      if (lane == 0) {
        x = __ldcg(a.keyrange + 2 * (size_t)row);
        y = __ldcg(a.keyrange + 2 * (size_t)row + 1);
        z = __ldcg(a.knmax + b);
      }
    } else {
      for (int s = lane; s < a.kpart; s += 32) {
        const size_t slot = (size_t)row * a.kpart + s;
        x = max(x, __ldcg(a.keyrange + 2 * slot));
        y = max(y, __ldcg(a.keyrange + 2 * slot + 1));
        z = max(z, __ldcg(a.knmax + slot));
      }
    }
    x = __reduce_max_sync(0xffffffffu, x);
    y = __reduce_max_sync(0xffffffffu, y);
    z = __reduce_max_sync(0xffffffffu, z);
    if (lane == 0) sm.kr_mx = x, sm.kr_nmn = y, sm.kn = z;
  }
  __syncthreads();
  const uint32_t klo = ~sm.kr_nmn, khi = sm.kr_mx;
  const float knmax = __uint_as_float(sm.kn);
  const float* sc = sm.sc;
  const float4* sc4 = reinterpret_cast<const float4*>(sc);
  const int nw = (n + 31) >> 5;
  // ---- 2. histogram over the row's key range, each copy as soon as it lands
  const bool ranged = klo <= khi;
  const uint32_t lo = ranged ? klo : 0u;
  const uint32_t hi = ranged ? khi : 0xFFFFFFFFu;
  const int s1 = sr_shift((uint64_t)(hi - lo) + 1u, 12);
  const int n4 = (n + 3) >> 2;
  bool ok = true;
  for (int c = 0; c < nch && ok; ++c) {
    ok = tc::mbar_wait(&sm.bar[c], 0);
    if (!ok) break;
    const int e4 = min(n4, (c + 1) * (SR_CHUNK / 16));
#pragma unroll 2
    for (int i4 = c * (SR_CHUNK / 16) + tid; i4 < e4; i4 += SR_T) {
      const float4 v = sc4[i4];
      const float x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t key = f32_order_key(x[u]);
        const uint32_t bin = key >= lo ? min((key - lo) >> s1, (uint32_t)(SR_HB - 1)) : 0u;
        if (4 * i4 + u < n) atomicAdd(&sm.hist[bin], 1u);
      }
    }
  }
  const bool landed = __syncthreads_and(ok);
  bool band_ok = false;                                      // the exact path applies
  uint32_t nbnd = 0;
  if (!landed) {
    if (tid == 0) {
      raise_err(a.err, CSA_DEVERR_TIMEOUT);
      for (int c = 0; c < nch; ++c) tc::mbar_wait(&sm.bar[c], 0);   // the copies may still be writing
      sm.fail = 1u;
    }
    __syncthreads();
  } else {
    sr_find_bin<SR_HB / SR_T>(sm, (uint32_t)k);
    uint32_t want = (uint32_t)k - sm.above;
    const uint32_t blo = lo + (sm.bin << s1);
    const uint64_t bhi64 = (uint64_t)blo + ((1ull << s1) - 1u);
    const uint32_t bhi = bhi64 > (uint64_t)hi ? max(hi, blo) : (uint32_t)bhi64;

    // ---- 3. certain entries above the bin, candidates around it
    const float EU = (a.eps_dot + 1.9073486328125e-06f) * sm.U * knmax * 1.0002f;
    const float f_lo = f32_from_order_key(blo), f_hi = f32_from_order_key(bhi);
    const float E2max = 2.f * ((EU + 1.52587890625e-05f * fmaxf(fabsf(f_lo), fabsf(f_hi))) * 1.0002f);
    const float sure_thr = __fadd_ru(f_hi, E2max), cand_lo = __fsub_rd(f_lo, E2max);
    // four entries per lane: a warp covers four bitmap words per step
    uint32_t n_sure = 0;
    for (int base = 128 * warp; base < n; base += 128 * SR_W) {
      const int i0 = base + 4 * lane;
      const float4 v = i0 < n ? sc4[i0 >> 2] : make_float4(0.f, 0.f, 0.f, 0.f);
      const float x[4] = {v.x, v.y, v.z, v.w};
      uint32_t nsur = 0u, ncan = 0u;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool valid = i0 + u < n;
        const bool sure = valid && x[u] > sure_thr;
        const bool cand = valid && !sure && x[u] >= cand_lo;
        nsur |= (sure ? 1u : 0u) << u;
        ncan |= (cand ? 1u : 0u) << u;
      }
      uint32_t ws = nsur << (4 * (lane & 7));                  // lanes 8w .. 8w+7 form word w of the step
      ws |= __shfl_xor_sync(0xffffffffu, ws, 1);
      ws |= __shfl_xor_sync(0xffffffffu, ws, 2);
      ws |= __shfl_xor_sync(0xffffffffu, ws, 4);
      const int wd = (base >> 5) + (lane >> 3);
      if ((lane & 7) == 0 && wd < nw) sm.bm[wd] = ws;
      n_sure += __popc(nsur);
      const uint32_t cc = __popc(ncan);
      if (__any_sync(0xffffffffu, cc != 0u)) {
        uint32_t incl = cc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t off = 0;
        if (lane == 31) off = atomicAdd(&sm.ccnt, incl);
        off = __shfl_sync(0xffffffffu, off, 31) + incl - cc;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if ((ncan >> u) & 1u) {
            if (off < (uint32_t)SR_CCAP) {
              sm.cid[off] = i0 + u;
              sm.ckey[off] = f32_order_key(x[u]);
            }
            ++off;
          }
      }
    }
    n_sure = __reduce_add_sync(0xffffffffu, n_sure);
    if (lane == 0 && n_sure) atomicAdd(&sm.nsure, n_sure);
    __syncthreads();
    const uint32_t ncand = sm.ccnt;
    const bool listed = ncand <= (uint32_t)SR_CCAP;          // else the whole row is the candidate source
    const uint32_t nsrc = listed ? ncand : (uint32_t)n;

    // ---- 4. the exact k-th largest key inside [blo, bhi]: by ranking the bin's candidates
    // when they are few, else by histograms over the bin
    uint32_t cur = blo;
    uint64_t width = (uint64_t)(bhi - blo) + 1u;
    if (listed && ncand <= (uint32_t)SR_T) {
      if (tid < (int)ncand) {
        const uint32_t kt = sm.ckey[tid];
        if (kt >= blo && kt <= bhi) {
          uint32_t gt = 0, eq_before = 0;
          for (uint32_t j2 = 0; j2 < ncand; ++j2) {
            const uint32_t kj = sm.ckey[j2];
            const bool inb = kj >= blo && kj <= bhi;
            gt += (inb && kj > kt) ? 1u : 0u;
            eq_before += (inb && kj == kt && j2 < (uint32_t)tid) ? 1u : 0u;
          }
          if (gt + eq_before == want - 1u) { sm.bin = kt; sm.above = gt; }
        }
      }
      __syncthreads();
      cur = sm.bin;
      want -= sm.above;
      width = 1;
    }
    while (width > 1) {
      const int s2 = sr_shift(width, 11);
      for (int i = tid; i < SR_HB2; i += SR_T) sm.hist[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < nsrc; i += SR_T) {
        const uint32_t key = listed ? sm.ckey[i] : f32_order_key(sc[i]);
        if (key >= cur && (uint64_t)(key - cur) < width) atomicAdd(&sm.hist[(key - cur) >> s2], 1u);
      }
      __syncthreads();
      sr_find_bin<SR_HB2 / SR_T>(sm, want);
      want -= sm.above;
      cur += sm.bin << s2;
      const uint64_t nwid = 1ull << s2;
      width = nwid < width ? nwid : width;
    }
    const uint32_t tkey = cur;
    const uint32_t quota = want;                             // keys equal to tau that the fp32 order takes
    const float tau = f32_from_order_key(tkey);
    const float E2 = 2.f * ((EU + 1.52587890625e-05f * fabsf(tau)) * 1.0002f);
    const float band_hi = __fadd_ru(tau, E2), band_lo = __fsub_rd(tau, E2);

    // the certain candidates, and the band
    for (uint32_t i = tid; i < nsrc; i += SR_T) {
      const int id = listed ? sm.cid[i] : (int)i;
      const float s = listed ? f32_from_order_key(sm.ckey[i]) : sc[i];
      if (!listed && (s > sure_thr || s < cand_lo)) continue;      // certain already, or out
      if (s > band_hi) {
        atomicOr(&sm.bm[id >> 5], 1u << (id & 31));
        atomicAdd(&sm.nsure, 1u);
      } else if (s >= band_lo) {
        const uint32_t off = atomicAdd(&sm.bcnt, 1u);
        if (off < (uint32_t)SR_BCAP) sm.bid_raw[off] = id;
      }
    }
    __syncthreads();
    nbnd = sm.bcnt;
    band_ok = nbnd <= (uint32_t)SR_BCAP;
    if (band_ok) {
      // ---- 5. the band in ascending index order (the same list in every CTA), exact scores
      if (tid < (int)nbnd) {
        const int id = sm.bid_raw[tid];
        int pos = 0;
        for (uint32_t j2 = 0; j2 < nbnd; ++j2) pos += sm.bid_raw[j2] < id ? 1 : 0;
        sm.bid[pos] = id;
      }
      __syncthreads();
      // this CTA's share: band entries crank, crank + C, ...
      const int mine = (int)nbnd > crank ? ((int)nbnd - crank + C - 1) / C : 0;
      for (int i0 = 0; i0 < mine; i0 += SR_RB) {
        const int cnt = min(SR_RB, mine - i0);
        if (tid < cnt) sm.rid[tid] = sm.bid[crank + (i0 + tid) * C];
        __syncthreads();
        sr_rescore<F>(sm, a, b, cnt, qi);
        if (tid < cnt) *cluster.map_shared_rank(&sm.bs[crank + (i0 + tid) * C], 0) = sm.rs[tid];
      }
    } else if (leader) {
      // ---- the fp32 order over the whole row: every entry above tau, then the first
      // `quota` equal to it by index
      raise_err(a.err, CSA_DEVERR_BAND);
      for (int w0 = warp; w0 < nw; w0 += SR_W) {
        const int i = 32 * w0 + lane;
        const uint32_t key = i < n ? f32_order_key(sc[i]) : 0u;
        const uint32_t ab = __ballot_sync(0xffffffffu, i < n && key > tkey);
        const uint32_t eq = __ballot_sync(0xffffffffu, i < n && key == tkey);
        if (lane == 0) { sm.bm[w0] = ab; sm.tb[w0] = eq; }
      }
      __syncthreads();
      const int wpt = (nw + SR_T - 1) / SR_T, a0 = tid * wpt, a1 = min(nw, a0 + wpt);
      uint32_t c = 0;
      for (int w = a0; w < a1; ++w) c += __popc(sm.tb[w]);
      uint32_t tot;
      uint32_t seen = sr_scan(c, sm.wred, &tot) - c;
      for (int w = a0; w < a1; ++w) {
        uint32_t keep = 0u;
        for (uint32_t bits = sm.tb[w]; bits; bits &= bits - 1) {
          if (seen < quota) keep |= bits & (0u - bits);
          ++seen;
        }
        sm.bm[w] |= keep;
      }
    }
  }
  if (!landed && tid == 0 && !leader) *cluster.map_shared_rank(&sm.fail, 0) = 1u;
  // every CTA of the cluster arrives here exactly once: then the band's exact scores (and a
  // failed copy anywhere) are in the first CTA's shared memory
  if (C > 1) cluster.sync();
  else __syncthreads();
  if (!leader) return;
  if (sm.fail) {
    for (int i = tid; i < k; i += SR_T) out[i] = -1;
    return;
  }
  if (band_ok) {
    // ---- 6. rank the band by (exact score desc, index asc); the first k - certain are chosen
    const uint32_t need = (uint32_t)k - sm.nsure;
    sr_band_keys(sm, nbnd);
    const uint64_t* bk = reinterpret_cast<const uint64_t*>(sm.bs);
    for (uint32_t i = warp; i < nbnd; i += SR_W) {
      const int id = sm.bid[i];
      const uint64_t s = bk[i];
      uint32_t rank = 0;
      for (uint32_t j0 = 0; j0 < nbnd; j0 += 32) {
        const uint32_t j2 = j0 + lane;
        const bool better = j2 < nbnd && (bk[j2] > s || (bk[j2] == s && sm.bid[j2] < id));
        rank += __popc(__ballot_sync(0xffffffffu, better));
      }
      if (lane == 0 && rank < need) atomicOr(&sm.bm[id >> 5], 1u << (id & 31));
    }
  }
  __syncthreads();

  // ---- ascending write
  const int wpt = (nw + SR_T - 1) / SR_T, a0 = tid * wpt, a1 = min(nw, a0 + wpt);
  uint32_t c = 0;
  for (int w = a0; w < a1; ++w) c += __popc(sm.bm[w]);
  uint32_t written;
  uint32_t pos = sr_scan(c, sm.wred, &written) - c;
  for (int w = a0; w < a1; ++w)
    for (uint32_t bits = sm.bm[w]; bits; bits &= bits - 1) {
      if (pos < (uint32_t)k) out[pos] = 32 * w + __ffs(bits) - 1;
      ++pos;
    }
  for (uint32_t i = written + tid; i < (uint32_t)k; i += SR_T) out[i] = -1;
  if (written != (uint32_t)k && tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
  if (sout) {
    // the exact score of every selected entry (the output is written: read it back)
    __syncthreads();
    for (int i0 = 0; i0 < k; i0 += SR_RB) {
      const int cnt = max(0, min(SR_RB, (int)written - i0));
      if (tid < SR_RB) sm.rid[tid] = (i0 + tid < (int)written) ? __ldcg(out + i0 + tid) : 0;
      __syncthreads();
      if (cnt > 0) sr_rescore<F>(sm, a, b, cnt, qi);
      if (tid < SR_RB && i0 + tid < k) sout[i0 + tid] = tid < cnt ? (float)sm.rs[tid] : 0.f;
      __syncthreads();
    }
  }
}

// The exact selection of a prefill row from the candidates the streaming scoring kernel kept
// (indexer_tc.cu): every entry of the row whose order key is at least the list's threshold,
// with the U and key-norm bound that threshold was computed from.  The k-th largest fp32 key
// tau is at least the threshold, so it is the k-th largest of the list; the band
// [tau - 2E, tau + 2E] (E from the same U and bound) lies above the threshold, so the list
// holds all of it.  Then as the row selection: certain entries into the row's bitmap, the
// band re-scored exactly and ranked, the bitmap written in ascending order.  One CTA per row.
template <int F>
__global__ void __launch_bounds__(SR_T, 1)
indexer_select_stream_kernel(IndexerArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SrSmem& sm = *reinterpret_cast<SrSmem*>(smem_raw);
  const int row = blockIdx.x, b = row / a.Tq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.k, HI = a.H_I, dI = a.d_I, nb = dI / 32;
  int32_t* out = a.idx_out + (size_t)row * k;

  // ---- prologue (inputs only): weights, query scales, the query codes as integers
  if (tid < HI) {
    sm.w[tid] = a.w[(size_t)row * HI + tid];
    if (F == CSA_IFMT_E4M3) sm.qsc[tid] = ((const float*)a.qI_scale)[(size_t)row * HI + tid];
    else
      for (int q = 0; q < nb; ++q)
        sm.qsc[tid * nb + q] = ue8m0_to_float(((const uint8_t*)a.qI_scale)[((size_t)row * HI + tid) * nb + q]);
  }
  if (tid == 0) { sm.bcnt = 0u; sm.nsure = 0u; sm.ccnt = 0u; }
  const int qj = tid >> 3, qs = tid & 7;
  const bool qlive = qj < HI && 16 * qs < dI;
  int qi[16];
  {
    const size_t qrow = (size_t)row * HI * dI;
    if (F == CSA_IFMT_E4M3) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (qlive) v = *reinterpret_cast<const uint4*>((const uint8_t*)a.qI + qrow + (size_t)qj * dI + 16 * qs);
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) qi[i] = (int)(e4m3_to_float((wd[i >> 2] >> (8 * (i & 3))) & 0xFFu) * 512.f);
    } else {
      uint2 v = make_uint2(0u, 0u);
      if (qlive) v = *reinterpret_cast<const uint2*>((const uint8_t*)a.qI + (qrow + (size_t)qj * dI + 16 * qs) / 2);
      const uint32_t wd[2] = {v.x, v.y};
#pragma unroll
      for (int i = 0; i < 16; ++i) qi[i] = (int)(e2m1_to_float((wd[i >> 3] >> (4 * (i & 7))) & 0xFu) * 2.f);
    }
  }
  const int n = row_eligible(a, row);
  tc::griddep_wait();                                        // the candidate lists
  tc::griddep_launch_dependents();
  if (n <= k) {
    for (int i = tid; i < k; i += SR_T) out[i] = i < n ? i : -1;
    return;
  }
  const uint4 meta = __ldcg(a.stream_meta + row);
  const uint32_t nc = min(meta.x & 0x7FFFFFFFu, (uint32_t)SR_CCAP);
  const uint32_t thr = meta.y;
  const float U = __uint_as_float(meta.z), knmax = __uint_as_float(meta.w);
  if ((meta.x >> 31) && tid == 0) raise_err(a.err, CSA_DEVERR_BAND);      // a list overflowed: entries were lost
  const uint2* cand = a.stream_cand + (size_t)row * IDX_STREAM_CAP;
  for (uint32_t i = tid; i < nc; i += SR_T) {
    const uint2 c = __ldcg(cand + i);
    sm.ckey[i] = c.x;
    sm.cid[i] = (int32_t)c.y;
  }
  const int nw = (n + 31) >> 5;
  for (int w = tid; w < nw; w += SR_T) { sm.bm[w] = 0u; sm.tb[w] = 0u; }
  for (int i = tid; i < SR_HB; i += SR_T) sm.hist[i] = 0u;
  // the candidates' key range
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  __syncthreads();
  for (uint32_t i = tid; i < nc; i += SR_T) { mn = min(mn, sm.ckey[i]); mx = max(mx, sm.ckey[i]); }
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (tid == 0) { sm.bin = 0xFFFFFFFFu; sm.above = 0u; }
  __syncthreads();
  if (lane == 0) { atomicMin(&sm.bin, mn); atomicMax(&sm.above, mx); }
  __syncthreads();
  const uint32_t lo = sm.bin, hi = max(sm.above, sm.bin);
  // ---- the exact k-th largest key among the candidates
  uint32_t want = (uint32_t)k, cur = lo;
  uint64_t width = (uint64_t)(hi - lo) + 1u;
  bool first = true;
  while (width > 1) {
    const int sh = sr_shift(width, first ? 12 : 11);
    if (!first) {
      for (int i = tid; i < SR_HB2; i += SR_T) sm.hist[i] = 0u;
      __syncthreads();
    }
    for (uint32_t i = tid; i < nc; i += SR_T) {
      const uint32_t key = sm.ckey[i];
      if (key >= cur && (uint64_t)(key - cur) < width) atomicAdd(&sm.hist[(key - cur) >> sh], 1u);
    }
    __syncthreads();
    if (first) sr_find_bin<SR_HB / SR_T>(sm, want);
    else sr_find_bin<SR_HB2 / SR_T>(sm, want);
    want -= sm.above;
    cur += sm.bin << sh;
    const uint64_t nwid = 1ull << sh;
    width = nwid < width ? nwid : width;
    first = false;
  }
  const uint32_t tkey = cur, quota = want;
  const float tau = f32_from_order_key(tkey);
  const float EU = (a.eps_dot + 1.9073486328125e-06f) * U * knmax * 1.0002f;
  const float E2 = 2.f * ((EU + 1.52587890625e-05f * fabsf(tau)) * 1.0002f);
  const float band_hi = __fadd_ru(tau, E2), band_lo = __fsub_rd(tau, E2);
  if (f32_order_key(band_lo) < thr && tid == 0) raise_err(a.err, CSA_DEVERR_BAND);   // cannot happen: same U, bound
  // ---- certain entries and the band
  for (uint32_t i = tid; i < nc; i += SR_T) {
    const int id = sm.cid[i];
    const float s = f32_from_order_key(sm.ckey[i]);
    if (s > band_hi) {
      atomicOr(&sm.bm[id >> 5], 1u << (id & 31));
      atomicAdd(&sm.nsure, 1u);
    } else if (s >= band_lo) {
      const uint32_t off = atomicAdd(&sm.bcnt, 1u);
      if (off < (uint32_t)SR_BCAP) sm.bid_raw[off] = id;
    }
  }
  __syncthreads();
  const uint32_t nbnd = sm.bcnt;
  if (nbnd <= (uint32_t)SR_BCAP) {
    if (tid < (int)nbnd) {
      const int id = sm.bid_raw[tid];
      int pos = 0;
      for (uint32_t j2 = 0; j2 < nbnd; ++j2) pos += sm.bid_raw[j2] < id ? 1 : 0;
      sm.bid[pos] = id;
    }
    __syncthreads();
    for (uint32_t i0 = 0; i0 < nbnd; i0 += SR_RB) {
      const int cnt = (int)min((uint32_t)SR_RB, nbnd - i0);
      if (tid < cnt) sm.rid[tid] = sm.bid[i0 + tid];
      __syncthreads();
      sr_rescore<F>(sm, a, b, cnt, qi);
      if (tid < cnt) sm.bs[i0 + tid] = sm.rs[tid];
    }
    __syncthreads();
    const uint32_t need = (uint32_t)k - sm.nsure;
    sr_band_keys(sm, nbnd);
    const uint64_t* bk = reinterpret_cast<const uint64_t*>(sm.bs);
    for (uint32_t i = warp; i < nbnd; i += SR_W) {
      const int id = sm.bid[i];
      const uint64_t sc = bk[i];
      uint32_t rank = 0;
      for (uint32_t j0 = 0; j0 < nbnd; j0 += 32) {
        const uint32_t j2 = j0 + lane;
        const bool better = j2 < nbnd && (bk[j2] > sc || (bk[j2] == sc && sm.bid[j2] < id));
        rank += __popc(__ballot_sync(0xffffffffu, better));
      }
      if (lane == 0 && rank < need) atomicOr(&sm.bm[id >> 5], 1u << (id & 31));
    }
  } else {
    // the fp32 order among the candidates: every key above tau, then the first `quota` equal
    // to it by index
    if (tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
    for (uint32_t i = tid; i < nc; i += SR_T) {
      const int id = sm.cid[i];
      const uint32_t key = sm.ckey[i];
      if (key > tkey) atomicOr(&sm.bm[id >> 5], 1u << (id & 31));
      else if (key == tkey) atomicOr(&sm.tb[id >> 5], 1u << (id & 31));
    }
    __syncthreads();
    // (the certain entries marked above all have keys above tau, so the words hold exactly
    // the keys above tau); now the first `quota` ties
    const int wpt = (nw + SR_T - 1) / SR_T, a0 = tid * wpt, a1 = min(nw, a0 + wpt);
    uint32_t c = 0;
    for (int w = a0; w < a1; ++w) c += __popc(sm.tb[w]);
    uint32_t tot;
    uint32_t seen = sr_scan(c, sm.wred, &tot) - c;
    for (int w = a0; w < a1; ++w) {
      uint32_t keep = 0u;
      for (uint32_t bits = sm.tb[w]; bits; bits &= bits - 1) {
        if (seen < quota) keep |= bits & (0u - bits);
        ++seen;
      }
      sm.bm[w] |= keep;
    }
  }
  __syncthreads();
  // ---- ascending write
  const int wpt = (nw + SR_T - 1) / SR_T, a0 = tid * wpt, a1 = min(nw, a0 + wpt);
  uint32_t c = 0;
  for (int w = a0; w < a1; ++w) c += __popc(sm.bm[w]);
  uint32_t written;
  uint32_t pos = sr_scan(c, sm.wred, &written) - c;
  for (int w = a0; w < a1; ++w)
    for (uint32_t bits = sm.bm[w]; bits; bits &= bits - 1) {
      if (pos < (uint32_t)k) out[pos] = 32 * w + __ffs(bits) - 1;
      ++pos;
    }
  for (uint32_t i = written + tid; i < (uint32_t)k; i += SR_T) out[i] = -1;
  if (written != (uint32_t)k && tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
}

// ---- rows longer than one CTA stages: the chunked selection ---------------------------------
// One cluster of C CTAs (2 to 16) per row; CTA c stages entries [c L, c L + L) of the row
// (L a multiple of 128) and the CTAs share what the one-CTA selection computes alone:
//   1. each CTA histograms its chunk's order keys over the row's key range (4096 bins);
//   2. CTA c sums slice c of the bins over the cluster and tells every CTA the slice's total;
//      every CTA then finds the slice holding the k-th largest key and reads that slice's
//      bins from its owner: the bin [b_lo, b_hi] and the keys above it;
//   3. each CTA marks its chunk's certain entries (above b_hi + 2E) in its own bitmap and
//      lists its candidates (within 2E of the bin); every CTA gathers all candidates (in
//      chunk order), so every CTA finds the same tau, band and certain candidates;
//   4. the band is re-scored exactly (entries c, c + C, ... on CTA c) and every exact score
//      is stored into every CTA; each CTA ranks the band, and from the per-chunk counts (the
//      same in every CTA) writes its chunk's selected entries at their place in the output.
// When the candidates do not fit the lists, tau comes from a counted search instead (32
// rounds of per-chunk counts of the keys above a trial key) and each chunk lists its own band
// entries; a band larger than its buffer makes the row take the fp32 order (score desc, index
// asc) and sets CSA_DEVERR_BAND.  Every CTA takes the same branches, so all of them meet at
// every cluster barrier, and none reads another's shared memory after the last one.

__device__ __forceinline__ void sd_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
__device__ __forceinline__ void sd_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Value v of this CTA into slot crank of array field of every CTA of the cluster (threads < C).
__device__ __forceinline__ void sd_tell(cg::cluster_group& cluster, uint32_t* field, int crank, int C, uint32_t v) {
  if ((int)threadIdx.x < C) *cluster.map_shared_rank(field + crank, (unsigned)threadIdx.x) = v;
}

// The number of this chunk's keys (sm.sc[0, len)) for which pred holds, to every thread.
template <typename P>
__device__ __forceinline__ uint32_t sd_count(SrSmem& sm, int len, P pred) {
  uint32_t c = 0;
  for (int i = threadIdx.x; i < len; i += SR_T) c += pred(f32_order_key(sm.sc[i])) ? 1u : 0u;
  uint32_t tot;
  sr_scan(c, sm.wred, &tot);
  return tot;
}

// The fp32 order over the row (every key above tkey, then the first of those equal to it by
// index, k in all): this chunk's bitmap, and per chunk the entries it selects in sm.sure
// (sm.win zero).  One counting round.
__device__ void sd_fp32_order(SrSmem& sm, cg::cluster_group& cluster, int C, int crank, int len, int k,
                              uint32_t tkey, int& rnd) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = (len + 31) >> 5;
  for (int w0 = warp; w0 < nw; w0 += SR_W) {
    const int i = 32 * w0 + lane;
    const uint32_t key = i < len ? f32_order_key(sm.sc[i]) : 0u;
    const uint32_t ab = __ballot_sync(0xffffffffu, i < len && key > tkey);
    const uint32_t eq = __ballot_sync(0xffffffffu, i < len && key == tkey);
    if (lane == 0) { sm.bm[w0] = ab; sm.tb[w0] = eq; }
  }
  __syncthreads();
  const int wpt = (nw + SR_T - 1) / SR_T, a0 = tid * wpt, a1 = min(nw, a0 + wpt);
  uint32_t g = 0, e = 0;
  for (int w = a0; w < a1; ++w) { g += __popc(sm.bm[w]); e += __popc(sm.tb[w]); }
  uint32_t gt, eqt;
  sr_scan(g, sm.wred, &gt);
  const uint32_t e_before = sr_scan(e, sm.wred, &eqt) - e;
  const int r = rnd & 1;
  if (tid < C) {
    uint32_t* px = &cluster.map_shared_rank(&sm.x, (unsigned)tid)->cnt[r][crank][0];
    px[0] = gt;
    px[1] = eqt;
  }
  cluster.sync();
  ++rnd;
  uint32_t G = 0, pre = 0;
  for (int p = 0; p < C; ++p) {
    G += sm.x.cnt[r][p][0];
    if (p < crank) pre += sm.x.cnt[r][p][1];
  }
  const uint32_t quota = (uint32_t)k > G ? (uint32_t)k - G : 0u;
  const uint32_t take = quota > pre ? min(quota - pre, eqt) : 0u;
  uint32_t seen = e_before;
  for (int w = a0; w < a1; ++w) {
    uint32_t keep = 0u;
    for (uint32_t bits = sm.tb[w]; bits; bits &= bits - 1) {
      if (seen < take) keep |= bits & (0u - bits);
      ++seen;
    }
    sm.bm[w] |= keep;
  }
  if (tid < C) {
    uint32_t before = 0;
    for (int p = 0; p < tid; ++p) before += sm.x.cnt[r][p][1];
    const uint32_t eq_p = sm.x.cnt[r][tid][1];
    sm.sure[tid] = sm.x.cnt[r][tid][0] + (quota > before ? min(quota - before, eq_p) : 0u);
    sm.win[tid] = 0u;
  }
  __syncthreads();
}

template <int F>
__global__ void __launch_bounds__(SR_T, 1)
indexer_select_dist_kernel(IndexerArgs a, int L) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SrSmem& sm = *reinterpret_cast<SrSmem*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks(), crank = (int)cluster.block_rank();
  const bool leader = crank == 0;
  const int row = blockIdx.x / C, b = row / a.Tq;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = a.k;
  int32_t* out = a.idx_out + (size_t)row * k;
  float* sout = a.score_out ? a.score_out + (size_t)row * k : nullptr;

  // ---- prologue (inputs only; overlaps the scoring kernel)
  int qi[16];
  sr_prologue<F>(sm, a, row, qi);
  sd_arrive_relaxed();                                       // paired with the wait before the first remote access
  const int n = row_eligible(a, row);
  tc::griddep_wait();                                        // the scores, their key range, knmax
  tc::griddep_launch_dependents();

  if (n <= k) {
    // every eligible entry is selected (the first CTA writes)
    sd_wait();
    if (!leader) return;
    for (int i = tid; i < k; i += SR_T) out[i] = i < n ? i : -1;
    if (sout) {
      __syncthreads();
      for (int i0 = 0; i0 < k; i0 += SR_RB) {
        const int cnt = max(0, min(SR_RB, n - i0));
        if (tid < SR_RB) sm.rid[tid] = i0 + tid;
        __syncthreads();
        if (cnt > 0) sr_rescore<F>(sm, a, b, cnt, qi);
        if (tid < SR_RB && i0 + tid < k) sout[i0 + tid] = tid < cnt ? (float)sm.rs[tid] : 0.f;
        __syncthreads();
      }
    }
    return;
  }

  // ---- 1. this chunk's scores into shared memory, in 16 KB copies; its histogram
  const int base = crank * L;
  const int len = max(0, min(L, n - base));
  const uint32_t bytes = (uint32_t)(((len + 3) & ~3) * 4);    // whole 16-byte units (ld and L are multiples of 64)
  const int nch = (int)((bytes + SR_CHUNK - 1) / SR_CHUNK);
  if (tid == 0) {
    const char* src = (const char*)(a.scores + (size_t)row * a.ld + base);
    for (int c = 0; c < nch; ++c) {
      const uint32_t o = (uint32_t)c * SR_CHUNK;
      const uint32_t cl = bytes - o < (uint32_t)SR_CHUNK ? bytes - o : (uint32_t)SR_CHUNK;
      tc::mbar_arrive_expect_tx(&sm.bar[c], cl);
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(tc::smem_u32((char*)sm.sc + o)), "l"(src + o), "r"(cl), "r"(tc::smem_u32(&sm.bar[c]))
                   : "memory");
    }
  }
  for (int i = tid; i < SR_HB; i += SR_T) sm.hist[i] = 0u;
  if (warp == 0) {
    // the scoring kernel's key range and key-norm bound: one value, or one per split
    uint32_t x = 0u, y = 0u, z = 0u;
    if (a.kpart == 0) {
      if (lane == 0) {
        x = __ldcg(a.keyrange + 2 * (size_t)row);
        y = __ldcg(a.keyrange + 2 * (size_t)row + 1);
        z = __ldcg(a.knmax + b);
      }
    } else {
      for (int s = lane; s < a.kpart; s += 32) {
        const size_t slot = (size_t)row * a.kpart + s;
        x = max(x, __ldcg(a.keyrange + 2 * slot));
        y = max(y, __ldcg(a.keyrange + 2 * slot + 1));
        z = max(z, __ldcg(a.knmax + slot));
      }
    }
    x = __reduce_max_sync(0xffffffffu, x);
    y = __reduce_max_sync(0xffffffffu, y);
    z = __reduce_max_sync(0xffffffffu, z);
    if (lane == 0) sm.kr_mx = x, sm.kr_nmn = y, sm.kn = z;
  }
  __syncthreads();
  const uint32_t klo = ~sm.kr_nmn, khi = sm.kr_mx;
  const float knmax = __uint_as_float(sm.kn);
  const float* sc = sm.sc;
  const float4* sc4 = reinterpret_cast<const float4*>(sc);
  const int nw = (len + 31) >> 5;
  const bool ranged = klo <= khi;
  const uint32_t lo = ranged ? klo : 0u;
  const uint32_t hi = ranged ? khi : 0xFFFFFFFFu;
  const int s1 = sr_shift((uint64_t)(hi - lo) + 1u, 12);
  const int n4 = (len + 3) >> 2;
  bool ok = true;
  for (int c = 0; c < nch && ok; ++c) {
    ok = tc::mbar_wait(&sm.bar[c], 0);
    if (!ok) break;
    const int e4 = min(n4, (c + 1) * (SR_CHUNK / 16));
#pragma unroll 2
    for (int i4 = c * (SR_CHUNK / 16) + tid; i4 < e4; i4 += SR_T) {
      const float4 v = sc4[i4];
      const float xv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t key = f32_order_key(xv[u]);
        const uint32_t bin = key >= lo ? min((key - lo) >> s1, (uint32_t)(SR_HB - 1)) : 0u;
        if (4 * i4 + u < len) atomicAdd(&sm.hist[bin], 1u);
      }
    }
  }
  const bool landed = __syncthreads_and(ok);
  if (!landed && tid == 0) {
    raise_err(a.err, CSA_DEVERR_TIMEOUT);
    for (int c = 0; c < nch; ++c) tc::mbar_wait(&sm.bar[c], 0);   // the copies may still be writing
  }
  sd_wait();                                                 // every CTA of the cluster runs
  sd_tell(cluster, sm.x.fail, crank, C, landed ? 0u : 1u);
  cluster.sync();                                            // (1) histograms, failures
  {
    uint32_t anyfail = 0u;
    for (int p = 0; p < C; ++p) anyfail |= sm.x.fail[p];
    if (anyfail) {
      if (leader)
        for (int i = tid; i < k; i += SR_T) out[i] = -1;
      return;
    }
  }

  // ---- 2. slice crank of the cluster's histogram; then the bin of the k-th largest key
  const int S = SR_HB / C;
  {
    uint32_t part = 0;
    for (int i = tid; i < S; i += SR_T) {
      const int bin = crank * S + i;
      uint32_t r[SD_CMAX];
#pragma unroll
      for (int p = 0; p < SD_CMAX; ++p) r[p] = p < C ? *cluster.map_shared_rank(&sm.hist[bin], (unsigned)p) : 0u;
      uint32_t v = 0;
#pragma unroll
      for (int p = 0; p < SD_CMAX; ++p) v += r[p];
      sm.hsum[i] = v;
      part += v;
    }
    uint32_t stot;
    sr_scan(part, sm.wred, &stot);
    sd_tell(cluster, sm.x.stot, crank, C, stot);
  }
  cluster.sync();                                            // (2) slices and their totals
  uint32_t above = 0;
  int ss = C - 1;
  for (; ss > 0; --ss) {
    const uint32_t t = sm.x.stot[ss];
    if (above + t >= (uint32_t)k) break;
    above += t;
  }
  {
    const uint32_t* oh = cluster.map_shared_rank(sm.hsum, (unsigned)ss);
    for (int i = tid; i < SR_HB; i += SR_T) sm.hist[i] = i < S ? oh[i] : 0u;
  }
  __syncthreads();
  if (S >= 2048) sr_find_bin<4>(sm, (uint32_t)k - above);
  else if (S == 1024) sr_find_bin<2>(sm, (uint32_t)k - above);
  else sr_find_bin<1>(sm, (uint32_t)k - above);
  uint32_t want = (uint32_t)k - above - sm.above;
  const uint32_t gbin = (uint32_t)(ss * S) + sm.bin;
  const uint32_t blo = lo + (gbin << s1);
  const uint64_t bhi64 = (uint64_t)blo + ((1ull << s1) - 1u);
  const uint32_t bhi = bhi64 > (uint64_t)hi ? max(hi, blo) : (uint32_t)bhi64;

  // ---- 3. this chunk's certain entries above the bin, and its candidates around it
  const float EU = (a.eps_dot + 1.9073486328125e-06f) * sm.U * knmax * 1.0002f;
  const float f_lo = f32_from_order_key(blo), f_hi = f32_from_order_key(bhi);
  const float E2max = 2.f * ((EU + 1.52587890625e-05f * fmaxf(fabsf(f_lo), fabsf(f_hi))) * 1.0002f);
  const float sure_thr = __fadd_ru(f_hi, E2max), cand_lo = __fsub_rd(f_lo, E2max);
  {
    uint32_t n_sure = 0;
    for (int cb = 128 * warp; cb < len; cb += 128 * SR_W) {
      const int i0 = cb + 4 * lane;
      const float4 v = i0 < len ? sc4[i0 >> 2] : make_float4(0.f, 0.f, 0.f, 0.f);
      const float xv[4] = {v.x, v.y, v.z, v.w};
      uint32_t nsur = 0u, ncan = 0u;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool valid = i0 + u < len;
        const bool sure = valid && xv[u] > sure_thr;
        const bool cand = valid && !sure && xv[u] >= cand_lo;
        nsur |= (sure ? 1u : 0u) << u;
        ncan |= (cand ? 1u : 0u) << u;
      }
      uint32_t ws = nsur << (4 * (lane & 7));                  // lanes 8w .. 8w+7 form word w of the step
      ws |= __shfl_xor_sync(0xffffffffu, ws, 1);
      ws |= __shfl_xor_sync(0xffffffffu, ws, 2);
      ws |= __shfl_xor_sync(0xffffffffu, ws, 4);
      const int wd = (cb >> 5) + (lane >> 3);
      if ((lane & 7) == 0 && wd < nw) sm.bm[wd] = ws;
      n_sure += __popc(nsur);
      const uint32_t cc = __popc(ncan);
      if (__any_sync(0xffffffffu, cc != 0u)) {
        uint32_t incl = cc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t off = 0;
        if (lane == 31) off = atomicAdd(&sm.ccnt, incl);
        off = __shfl_sync(0xffffffffu, off, 31) + incl - cc;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if ((ncan >> u) & 1u) {
            if (off < (uint32_t)SD_LCAP) {
              sm.lid[off] = base + i0 + u;
              sm.lkey[off] = f32_order_key(xv[u]);
            }
            ++off;
          }
      }
    }
    n_sure = __reduce_add_sync(0xffffffffu, n_sure);
    if (lane == 0 && n_sure) atomicAdd(&sm.nsure, n_sure);
  }
  __syncthreads();
  if (tid < C) {
    SdXchg* px = cluster.map_shared_rank(&sm.x, (unsigned)tid);
    px->nsure[crank] = sm.nsure;
    px->ncand[crank] = sm.ccnt;
  }
  cluster.sync();                                            // (3) chunk counts and candidate lists
  uint32_t ncand = 0;
  bool lovf = false;
  for (int p = 0; p < C; ++p) {
    ncand += sm.x.ncand[p];
    lovf = lovf || sm.x.ncand[p] > (uint32_t)SD_LCAP;
  }
  const bool listed = !lovf && ncand <= (uint32_t)SR_CCAP;
  int rnd = 0;
  uint32_t tkey;
  if (listed) {
    // every chunk's candidates, in chunk order (each thread's remote loads independent)
    for (uint32_t f = tid; f < ncand; f += SR_T) {
      int p = 0;
      uint32_t o = 0;
      while (f >= o + sm.x.ncand[p]) o += sm.x.ncand[p++];
      sm.cid[f] = cluster.map_shared_rank(sm.lid, (unsigned)p)[f - o];
      sm.ckey[f] = cluster.map_shared_rank(sm.lkey, (unsigned)p)[f - o];
    }
    __syncthreads();
    // ---- the exact k-th largest key inside [blo, bhi]: by ranking the bin's candidates
    // when they are few, else by histograms over the bin
    uint32_t cur = blo;
    uint64_t width = (uint64_t)(bhi - blo) + 1u;
    if (ncand <= (uint32_t)SR_T) {
      if (tid < (int)ncand) {
        const uint32_t kt = sm.ckey[tid];
        if (kt >= blo && kt <= bhi) {
          uint32_t gt = 0, eq_before = 0;
          for (uint32_t j2 = 0; j2 < ncand; ++j2) {
            const uint32_t kj = sm.ckey[j2];
            const bool inb = kj >= blo && kj <= bhi;
            gt += (inb && kj > kt) ? 1u : 0u;
            eq_before += (inb && kj == kt && j2 < (uint32_t)tid) ? 1u : 0u;
          }
          if (gt + eq_before == want - 1u) { sm.bin = kt; sm.above = gt; }
        }
      }
      __syncthreads();
      cur = sm.bin;
      want -= sm.above;
      width = 1;
    }
    while (width > 1) {
      const int s2 = sr_shift(width, 11);
      for (int i = tid; i < SR_HB2; i += SR_T) sm.hist[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < ncand; i += SR_T) {
        const uint32_t key = sm.ckey[i];
        if (key >= cur && (uint64_t)(key - cur) < width) atomicAdd(&sm.hist[(key - cur) >> s2], 1u);
      }
      __syncthreads();
      sr_find_bin<SR_HB2 / SR_T>(sm, want);
      want -= sm.above;
      cur += sm.bin << s2;
      const uint64_t nwid = 1ull << s2;
      width = nwid < width ? nwid : width;
    }
    tkey = cur;
  } else {
    // counted search: the largest key t with at least k keys >= t
    uint32_t tlo = 0u, thi = 0xFFFFFFFFu;
    while (tlo < thi) {
      const uint32_t mid = tlo + (uint32_t)(((uint64_t)thi - tlo + 1u) >> 1);
      const uint32_t c = sd_count(sm, len, [&](uint32_t key) { return key >= mid; });
      const int r = rnd & 1;
      if (tid < C) cluster.map_shared_rank(&sm.x, (unsigned)tid)->cnt[r][crank][0] = c;
      cluster.sync();
      ++rnd;
      uint32_t tot = 0;
      for (int p = 0; p < C; ++p) tot += sm.x.cnt[r][p][0];
      if (tot >= (uint32_t)k) tlo = mid;
      else thi = mid - 1u;
    }
    tkey = tlo;
  }
  const float tau = f32_from_order_key(tkey);
  const float E2 = 2.f * ((EU + 1.52587890625e-05f * fabsf(tau)) * 1.0002f);
  const float band_hi = __fadd_ru(tau, E2), band_lo = __fsub_rd(tau, E2);

  // ---- the band and the certain candidates (the same lists in every CTA)
  if (tid < C) { sm.sure[tid] = 0u; sm.win[tid] = 0u; }
  if (tid == 0) { sm.bcnt = 0u; sm.ccnt = 0u; }
  __syncthreads();
  bool band_ok;
  if (listed) {
    for (uint32_t i = tid; i < ncand; i += SR_T) {
      const int id = sm.cid[i];
      const float s = f32_from_order_key(sm.ckey[i]);
      if (s > band_hi) {
        const int owner = id / L;
        atomicAdd(&sm.sure[owner], 1u);
        if (owner == crank) atomicOr(&sm.bm[(id - base) >> 5], 1u << ((id - base) & 31));
      } else if (s >= band_lo) {
        const uint32_t o = atomicAdd(&sm.bcnt, 1u);
        if (o < (uint32_t)SR_BCAP) sm.bid_raw[o] = id;
      }
    }
    __syncthreads();
    if (tid < C) sm.sure[tid] += sm.x.nsure[tid];
    band_ok = sm.bcnt <= (uint32_t)SR_BCAP;
  } else {
    // this chunk from scratch: the bitmap of the entries above the band, its band entries
    uint32_t nab = 0;
    for (int w0 = warp; w0 < nw; w0 += SR_W) {
      const int i = 32 * w0 + lane;
      const float s = i < len ? sc[i] : 0.f;
      const bool ab = i < len && s > band_hi;
      const bool inb = i < len && !ab && s >= band_lo;
      const uint32_t m = __ballot_sync(0xffffffffu, ab);
      if (lane == 0) sm.bm[w0] = m;
      nab += lane == 0 ? __popc(m) : 0u;
      if (inb) {
        const uint32_t o = atomicAdd(&sm.ccnt, 1u);
        if (o < (uint32_t)SD_LCAP) sm.lid[o] = base + i;
      }
    }
    nab = __reduce_add_sync(0xffffffffu, nab);
    if (lane == 0 && nab) atomicAdd(&sm.bcnt, nab);
    __syncthreads();
    if (tid < C) {
      SdXchg* px = cluster.map_shared_rank(&sm.x, (unsigned)tid);
      px->nsure2[crank] = sm.bcnt;
      px->nband[crank] = sm.ccnt;
    }
    cluster.sync();                                          // chunk band lists
    uint32_t nbt = 0;
    bool bovf = false;
    for (int p = 0; p < C; ++p) {
      nbt += sm.x.nband[p];
      bovf = bovf || sm.x.nband[p] > (uint32_t)SD_LCAP;
    }
    band_ok = !bovf && nbt <= (uint32_t)SR_BCAP;
    __syncthreads();                                         // sm.bcnt read above
    if (band_ok) {
      for (uint32_t f = tid; f < nbt; f += SR_T) {
        int p = 0;
        uint32_t o = 0;
        while (f >= o + sm.x.nband[p]) o += sm.x.nband[p++];
        sm.bid_raw[f] = cluster.map_shared_rank(sm.lid, (unsigned)p)[f - o];
      }
    }
    if (tid == 0) sm.bcnt = nbt;
    if (tid < C) sm.sure[tid] = sm.x.nsure2[tid];
    __syncthreads();
  }

  const uint32_t nbnd = sm.bcnt;
  if (band_ok) {
    // ---- 4. the band in ascending index order, exact scores into every CTA, ranking
    if (tid < (int)nbnd) {
      const int id = sm.bid_raw[tid];
      int pos = 0;
      for (uint32_t j2 = 0; j2 < nbnd; ++j2) pos += sm.bid_raw[j2] < id ? 1 : 0;
      sm.bid[pos] = id;
    }
    __syncthreads();
    const int mine = (int)nbnd > crank ? ((int)nbnd - crank + C - 1) / C : 0;
    for (int i0 = 0; i0 < mine; i0 += SR_RB) {
      const int cnt = min(SR_RB, mine - i0);
      if (tid < cnt) sm.rid[tid] = sm.bid[crank + (i0 + tid) * C];
      __syncthreads();
      sr_rescore<F>(sm, a, b, cnt, qi);
      if (tid < cnt)
        for (int p = 0; p < C; ++p) *cluster.map_shared_rank(&sm.bs[crank + (i0 + tid) * C], (unsigned)p) = sm.rs[tid];
    }
    cluster.sync();                                          // (4) every exact score in every CTA
    uint32_t nsure = 0;
    for (int p = 0; p < C; ++p) nsure += sm.sure[p];
    const uint32_t need = (uint32_t)k > nsure ? (uint32_t)k - nsure : 0u;
    sr_band_keys(sm, nbnd);
    const uint64_t* bk = reinterpret_cast<const uint64_t*>(sm.bs);
    for (uint32_t i = warp; i < nbnd; i += SR_W) {
      const int id = sm.bid[i];
      const uint64_t s = bk[i];
      uint32_t rank = 0;
      for (uint32_t j0 = 0; j0 < nbnd; j0 += 32) {
        const uint32_t j2 = j0 + lane;
        const bool better = j2 < nbnd && (bk[j2] > s || (bk[j2] == s && sm.bid[j2] < id));
        rank += __popc(__ballot_sync(0xffffffffu, better));
      }
      if (lane == 0 && rank < need) {
        const int owner = id / L;
        atomicAdd(&sm.win[owner], 1u);
        if (owner == crank) atomicOr(&sm.bm[(id - base) >> 5], 1u << ((id - base) & 31));
      }
    }
    __syncthreads();
  } else {
    if (leader && tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
    sd_fp32_order(sm, cluster, C, crank, len, k, tkey, rnd);
  }

  // ---- this chunk's selected entries at their place in the ascending output
  uint32_t offset = 0, total = 0;
  for (int p = 0; p < C; ++p) {
    const uint32_t cp = sm.sure[p] + sm.win[p];
    offset += p < crank ? cp : 0u;
    total += cp;
  }
  const int wpt = (nw + SR_T - 1) / SR_T, a0 = tid * wpt, a1 = min(nw, a0 + wpt);
  uint32_t c = 0;
  for (int w = a0; w < a1; ++w) c += __popc(sm.bm[w]);
  uint32_t mine_cnt;
  uint32_t pos = offset + sr_scan(c, sm.wred, &mine_cnt) - c;
  for (int w = a0; w < a1; ++w)
    for (uint32_t bits = sm.bm[w]; bits; bits &= bits - 1) {
      if (pos < (uint32_t)k) out[pos] = base + 32 * w + __ffs(bits) - 1;
      ++pos;
    }
  for (uint32_t i = total + (uint32_t)(crank * SR_T + tid); i < (uint32_t)k; i += (uint32_t)(C * SR_T)) out[i] = -1;
  if (leader && tid == 0 && total != (uint32_t)k) raise_err(a.err, CSA_DEVERR_BAND);
  if (sout) {
    // the exact score of each entry this CTA wrote (read back from the output)
    __syncthreads();
    const uint32_t end = min((uint32_t)k, offset + mine_cnt);
    for (uint32_t i0 = offset; i0 < end; i0 += SR_RB) {
      const int cnt = (int)min((uint32_t)SR_RB, end - i0);
      if (tid < cnt) sm.rid[tid] = __ldcg(out + i0 + tid);
      __syncthreads();
      sr_rescore<F>(sm, a, b, cnt, qi);
      if (tid < cnt) sout[i0 + tid] = (float)sm.rs[tid];
      __syncthreads();
    }
    for (uint32_t i = total + (uint32_t)(crank * SR_T + tid); i < (uint32_t)k; i += (uint32_t)(C * SR_T)) sout[i] = 0.f;
  }
}

}  // namespace

size_t indexer_select_row_smem(int64_t n_max) {
  return offsetof(SrSmem, sc) + (size_t)((n_max + 31) / 32 * 32) * sizeof(float);
}

// One cluster of C CTAs per row (up to 8, while the rows leave SMs for them), launched with
// programmatic dependent launch (the prologue overlaps the scoring kernel).
// cudaErrorNotSupported for shapes this path does not take.
cudaError_t launch_indexer_select_row(const IndexerArgs& a, cudaStream_t st) {
  if (a.H_I > 64 || a.d_I > 128 || (a.ifmt != CSA_IFMT_E4M3 && a.ifmt != CSA_IFMT_MXFP4) || a.n_max > SR_NMAX ||
      a.score_bf16 || !a.keyrange)
    return cudaErrorNotSupported;
  const size_t smem = indexer_select_row_smem(a.n_max);
  auto kern = a.ifmt == CSA_IFMT_E4M3 ? indexer_select_row_kernel<CSA_IFMT_E4M3> : indexer_select_row_kernel<CSA_IFMT_MXFP4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows = a.B * a.Tq;
  int C = num_sms() / rows;
  C = C < 1 ? 1 : (C >= SR_CMAX ? SR_CMAX : (C >= 4 ? 4 : (C >= 2 ? 2 : 1)));
  // the largest cluster size whose clusters for every row are resident at once (a cluster
  // that waits for another to finish would serialise the rows), checked once per size
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(SR_T);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  static std::mutex mu;
  static std::map<std::pair<int, size_t>, int> resident;
  for (; C > 1; C >>= 1) {
    std::lock_guard<std::mutex> g(mu);
    const auto key = std::make_pair(C * (a.ifmt == CSA_IFMT_E4M3 ? 1 : -1), smem);
    auto it = resident.find(key);
    if (it == resident.end()) {
      cfg.gridDim = dim3(rows * C);
      attr[1].val.clusterDim.x = C;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess) nc = 0;
      cudaGetLastError();
      it = resident.emplace(key, nc).first;
    }
    if (it->second >= rows) break;
  }
  cfg.gridDim = dim3(rows * C);
  attr[1].val.clusterDim.x = C;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, a);
}

int64_t indexer_select_row_max_entries() { return SR_NMAX; }

namespace {
struct SdPlan {
  int C = 0, L = 0;
  size_t smem = 0;
};
// The chunked selection's cluster size for these rows: the largest C in {16, 8, 4, 2} whose
// chunks fit one CTA's staging buffer and whose clusters for every row are resident at once
// (else the largest whose clusters fit at all); C = 0 when the rows do not fit.
SdPlan sd_plan(const IndexerArgs& a) {
  SdPlan best;
  if (a.H_I > 64 || a.d_I > 128 || (a.ifmt != CSA_IFMT_E4M3 && a.ifmt != CSA_IFMT_MXFP4) || a.score_bf16 ||
      !a.keyrange || a.n_max <= SR_NMAX)
    return best;
  auto kern = a.ifmt == CSA_IFMT_E4M3 ? indexer_select_dist_kernel<CSA_IFMT_E4M3> : indexer_select_dist_kernel<CSA_IFMT_MXFP4>;
  const int rows = a.B * a.Tq;
  static std::mutex mu;
  static std::map<std::pair<int, size_t>, int> resident;
  std::lock_guard<std::mutex> g(mu);
  for (int C = SD_CMAX; C >= 2; C >>= 1) {
    const int64_t per = (a.n_max + C - 1) / C;
    const int L = (int)((per + 127) / 128 * 128);
    if (L > SR_NMAX) break;                                  // smaller clusters only make the chunks longer
    SdPlan P;
    P.C = C;
    P.L = L;
    P.smem = offsetof(SrSmem, sc) + (size_t)L * sizeof(float);
    const auto key = std::make_pair(C * (a.ifmt == CSA_IFMT_E4M3 ? 1 : -1), P.smem);
    auto it = resident.find(key);
    if (it == resident.end()) {
      int nc = 0;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem) == cudaSuccess &&
          cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(rows * C);
        cfg.blockDim = dim3(SR_T);
        cfg.dynamicSmemBytes = P.smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess) nc = 0;
      }
      cudaGetLastError();
      it = resident.emplace(key, nc).first;
    }
    if (it->second >= rows) return P;
    if (it->second >= 1 && best.C == 0) best = P;
  }
  return best;
}
}  // namespace

int indexer_select_dist_clusters(const IndexerArgs& a) { return sd_plan(a).C; }

// One cluster per row over chunks of the row (rows longer than one CTA stages), launched with
// programmatic dependent launch.  cudaErrorNotSupported for rows this path does not take.
cudaError_t launch_indexer_select_dist(const IndexerArgs& a, cudaStream_t st) {
  const SdPlan P = sd_plan(a);
  if (P.C == 0) return cudaErrorNotSupported;
  auto kern = a.ifmt == CSA_IFMT_E4M3 ? indexer_select_dist_kernel<CSA_IFMT_E4M3> : indexer_select_dist_kernel<CSA_IFMT_MXFP4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.Tq * P.C);
  cfg.blockDim = dim3(SR_T);
  cfg.dynamicSmemBytes = P.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = P.C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, a, P.L);
}

cudaError_t launch_indexer_select_stream(const IndexerArgs& a, cudaStream_t st) {
  if (!a.stream_cand || !a.stream_meta || a.H_I > 64 || a.d_I > 128 || a.n_max > SR_NMAX || a.k > IDX_STREAM_KMAX ||
      (a.ifmt != CSA_IFMT_E4M3 && a.ifmt != CSA_IFMT_MXFP4))
    return cudaErrorNotSupported;
  const size_t smem = offsetof(SrSmem, sc);
  auto kern = a.ifmt == CSA_IFMT_E4M3 ? indexer_select_stream_kernel<CSA_IFMT_E4M3>
                                      : indexer_select_stream_kernel<CSA_IFMT_MXFP4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.B * a.Tq);
  cfg.blockDim = dim3(SR_T);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, a);
}

static_assert(offsetof(SrSmem, sc) % 16 == 0, "bulk copy destination");
static_assert(offsetof(SrSmem, sc) + SR_NMAX * sizeof(float) <= 232448, "shared memory budget of one CTA (227 KB)");
static_assert(SR_CCAP >= IDX_STREAM_CAP, "a streaming candidate list fits the candidate buffers");

}  // namespace csa
