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
constexpr int SH_RB = 32;                // entries re-scored per batch
constexpr int SH_DLD = 132;              // bytes per staged digit row (128 dims + 4: conflict-free fragments)
constexpr int SH_CTR0 = 4;               // row counters: [1] certain entries, [2] CTAs done, [4 + p] CTA p's candidates
constexpr int SH_CTR_STRIDE = 256;       // words of counters per row (so at most 252 CTAs per row)

struct ShSmem {
  int8_t qdig[3][64][SH_DLD];            // query codes as integer digits (see sh_digits), [plane][head][dim]
  int8_t kdig[3][SH_RB][SH_DLD];         // key codes of one batch, [plane][entry][dim]
  double contrib[SH_RB][65];             // the batch's per-head terms
  double rs_out[SH_RB];                  // the batch's exact scores
  float ksc[SH_RB][4];                   // their scales (E4M3 row scale in [0], MXFP4 block scales)
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
  uint32_t coff[260];                    // gathered position of each classifying CTA's candidates
  uint32_t bins_above, bin_T, cnt, cnt2, ties, last, lo, hi;
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

// ---- exact dot products of quantised codes on the integer tensor cores
//
// An E4M3 value times 2^9 is an integer V with |V| < 2^18 (subnormals: the 3-bit mantissa;
// normals: (8 + mantissa) << (exponent - 1)); V splits into three signed 7-bit digits,
// V = d0 + 2^7 d1 + 2^14 d2.  For two code vectors of 128 dims,
//   sum_c q_c k_c = 2^-18 sum_{a,b} 2^{7(a+b)} sum_c dq_{a,c} dk_{b,c},
// where every inner sum (128 products of 7-bit digits, |.| < 2^21) is exact in an int32
// accumulator of the int8 MMA, the weighted sum is exact in int64 (|.| < 2^53 since
// sum_c |Vq Vk| < 2^43) and so is its conversion to fp64.  An e2m1 value times 2 is an
// integer in [-12, 12]: one digit, and each 32-dim block's sum is 2^-2 times an exact int32.
// So the per-head dot products equal the oracle's exact fp64 values bit for bit.
template <int F>
__device__ __forceinline__ void sh_digits(uint32_t code, int (&d)[3]) {
  int v, neg;
  if (F == CSA_IFMT_E4M3) {
    const int e = (code >> 3) & 0xF, mnt = code & 7;
    v = e == 0 ? mnt : (8 + mnt) << (e - 1);
    neg = (code >> 7) & 1;
  } else {
    const int e = (code >> 1) & 3, mnt = code & 1;
    v = e == 0 ? mnt : (2 + mnt) << (e - 1);
    neg = (code >> 3) & 1;
  }
  const int a = v & 127, b = (v >> 7) & 127, c = v >> 14;
  d[0] = neg ? -a : a;
  d[1] = neg ? -b : b;
  d[2] = neg ? -c : c;
}
__device__ __forceinline__ uint32_t sh_pack4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) | ((uint32_t)(d & 0xFF) << 24);
}
// D (16x8 s32) += A (16x32 s8, row) * B (32x8 s8, col)
__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Digits of `cnt` rows of 128 codes (E4M3 bytes, or MXFP4 bytes of two codes) into
// dst[plane][row][dim]; thread t converts 16 codes of row t / 8 per step.
template <int F>
__device__ __forceinline__ void sh_stage_digits(int8_t (*dst)[SH_DLD], size_t plane_stride, const uint8_t* const* rows,
                                                int cnt, int dI) {
  for (int u = threadIdx.x; u < cnt * 8; u += SH_T) {
    const int r = u >> 3, seg = u & 7;
    uint32_t wd[4] = {0u, 0u, 0u, 0u};
    if (16 * seg < dI && rows[r]) {
      if (F == CSA_IFMT_E4M3) {
        const uint4 v = *reinterpret_cast<const uint4*>(rows[r] + 16 * seg);
        wd[0] = v.x; wd[1] = v.y; wd[2] = v.z; wd[3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(rows[r] + 8 * seg);
        wd[0] = v.x; wd[1] = v.y;
      }
    }
    int dg[16][3];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t code = F == CSA_IFMT_E4M3 ? (wd[i >> 2] >> (8 * (i & 3))) & 0xFFu : (wd[i >> 3] >> (4 * (i & 7))) & 0xFu;
      sh_digits<F>(code, dg[i]);
    }
#pragma unroll
    for (int p = 0; p < (F == CSA_IFMT_E4M3 ? 3 : 1); ++p) {
      uint32_t* o = reinterpret_cast<uint32_t*>(&dst[r][16 * seg] + p * plane_stride);
#pragma unroll
      for (int w = 0; w < 4; ++w) o[w] = sh_pack4(dg[4 * w][p], dg[4 * w + 1][p], dg[4 * w + 2][p], dg[4 * w + 3][p]);
    }
  }
}

// Exact fp64 scores of entries ids[0..cnt) (cnt <= SH_RB) of sequence b into sm.rs_out, by
// the whole CTA (all threads call; barriers inside).  The query digits are in sm.qdig.  Warp w computes (16 heads x 8 entries) tiles with the int8 MMA; the
// per-head values are then formed as the definition does (E4M3: (sq * sk) * raw; MXFP4: the
// block terms (qs * ks) * P_b added in block order), each head's term w_j * max(D_j, 0) is
// written, and one thread per entry adds the terms in order j = 0..H_I-1.
template <int F>
__device__ __noinline__ void sh_rescore(const KeySide ks, ShSmem& sm, const void* qI, size_t qrow, int b,
                                        const int32_t* ids, int cnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dI = ks.dI, nb = dI / 32, HI = ks.HI;
  const int rowbytes = F == CSA_IFMT_E4M3 ? dI : dI / 2;
  __shared__ const uint8_t* rowp[64];
  (void)qI; (void)qrow;                                     // the query digits are staged in the prologue
  __syncthreads();
  if (tid < SH_RB) rowp[tid] = tid < cnt ? (const uint8_t*)ks.kI + ((size_t)b * ks.n_max + ids[tid]) * rowbytes : nullptr;
  if (tid < SH_RB * 4) {
    const int e2 = tid >> 2, q2 = tid & 3;
    float v = 0.f;
    if (e2 < cnt) {
      const size_t koff = (size_t)b * ks.n_max + ids[e2];
      if (F == CSA_IFMT_E4M3) v = q2 == 0 ? ((const float*)ks.kI_scale)[koff] : 0.f;
      else v = q2 < nb ? ue8m0_to_float(((const uint8_t*)ks.kI_scale)[koff * nb + q2]) : 0.f;
    }
    sm.ksc[e2][q2] = v;
  }
  __syncthreads();
  sh_stage_digits<F>(sm.kdig[0], sizeof(sm.kdig[0]), rowp, SH_RB, dI);
  __syncthreads();
  // ---- tiles: 4 head tiles x ceil(cnt / 8) entry tiles over the 8 warps
  const int g = lane >> 2, tig = lane & 3;
  const int ntile = (cnt + 7) / 8;
  for (int job = warp; job < 4 * ntile; job += SH_W) {
    const int mt = job & 3, nt = job >> 2;
    // E4M3: one accumulator per digit pair (a, b), so that no MMA waits for another; MXFP4:
    // one per 32-dim block
    constexpr int NACC = F == CSA_IFMT_E4M3 ? 9 : 4;
    int acc[NACC][4];
#pragma unroll
    for (int i = 0; i < NACC; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0;
#pragma unroll
    for (int kst = 0; kst < 4; ++kst) {
      const int kc = 32 * kst + 4 * tig;
      if (F == CSA_IFMT_E4M3) {
        uint32_t bq[3][2];
#pragma unroll
        for (int pb = 0; pb < 3; ++pb) {
          const int8_t* kb = &sm.kdig[pb][8 * nt + g][kc];
          bq[pb][0] = *reinterpret_cast<const uint32_t*>(kb);
          bq[pb][1] = *reinterpret_cast<const uint32_t*>(kb + 16);
        }
#pragma unroll
        for (int pa = 0; pa < 3; ++pa) {
          const int8_t* qa = &sm.qdig[pa][16 * mt + g][kc];
          const uint32_t a0 = *reinterpret_cast<const uint32_t*>(qa);
          const uint32_t a1 = *reinterpret_cast<const uint32_t*>(qa + 8 * SH_DLD);
          const uint32_t a2 = *reinterpret_cast<const uint32_t*>(qa + 16);
          const uint32_t a3 = *reinterpret_cast<const uint32_t*>(qa + 8 * SH_DLD + 16);
#pragma unroll
          for (int pb = 0; pb < 3; ++pb) mma_s8(acc[3 * pa + pb], a0, a1, a2, a3, bq[pb][0], bq[pb][1]);
        }
      } else {
        const int8_t* qa = &sm.qdig[0][16 * mt + g][kc];
        const int8_t* kb = &sm.kdig[0][8 * nt + g][kc];
        mma_s8(acc[kst], *reinterpret_cast<const uint32_t*>(qa), *reinterpret_cast<const uint32_t*>(qa + 8 * SH_DLD),
               *reinterpret_cast<const uint32_t*>(qa + 16), *reinterpret_cast<const uint32_t*>(qa + 8 * SH_DLD + 16),
               *reinterpret_cast<const uint32_t*>(kb), *reinterpret_cast<const uint32_t*>(kb + 16));
      }
    }
    // accumulator element i: head 16 mt + g + 8 (i >> 1), entry 8 nt + 2 tig + (i & 1)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = 16 * mt + g + 8 * (i >> 1), e = 8 * nt + 2 * tig + (i & 1);
      if (j >= HI || e >= cnt) continue;
      double D;
      if (F == CSA_IFMT_E4M3) {
        // sum over digit pairs of 2^(7 (a + b)) x the pair's exact int32 sum, exact in int64
        const long long tot = (long long)acc[0][i] + (((long long)acc[1][i] + acc[3][i]) << 7) +
                              (((long long)acc[2][i] + acc[4][i] + acc[6][i]) << 14) +
                              (((long long)acc[5][i] + acc[7][i]) << 21) + ((long long)acc[8][i] << 28);
        const double raw = (double)tot * 0x1p-18;                  // exact: |tot| < 2^53
        D = ((double)sm.qsc[j] * (double)sm.ksc[e][0]) * raw;
      } else {
        D = 0.0;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < nb) D += ((double)sm.qsc[j * nb + q] * (double)sm.ksc[e][q]) * ((double)acc[q][i] * 0.25);
      }
      sm.contrib[e][j] = (double)sm.w[j] * fmax(D, 0.0);
    }
  }
  __syncthreads();
  if (tid < cnt) {
    double S = 0.0;
    for (int jj = 0; jj < HI; ++jj) S += sm.contrib[tid][jj];
    sm.rs_out[tid] = S;
  }
  __syncthreads();
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
  uint32_t* ctr = a.counters + (size_t)row * SH_CTR_STRIDE;
  uint32_t* bitmap = a.bitmap + (size_t)row * (a.ld / 32);
  uint2* cand_g = a.cand + (size_t)row * a.ld;
  tc::griddep_launch_dependents();

  // ---- prologue (inputs only; overlaps the scoring kernel): weights, query scales, the
  // query row in registers as fp64 (thread t: head t / 4, dims [32 (t % 4), +32)) and
  // U = sum_j |w_j| ||q_j||
  const size_t qrow = (size_t)row * HI * dI;
  if (tid < HI) {
    sm.w[tid] = a.w[(size_t)row * HI + tid];
    if (F == CSA_IFMT_E4M3) sm.qsc[tid] = ((const float*)a.qI_scale)[(size_t)row * HI + tid];
    else
      for (int q = 0; q < nb; ++q) sm.qsc[tid * nb + q] = ue8m0_to_float(((const uint8_t*)a.qI_scale)[((size_t)row * HI + tid) * nb + q]);
  }
  if (tid == 0) sm.U = 0.f;
  {
    // thread t: head t / 4, dims [32 (t % 4), +32) (one MXFP4 scale block)
    const int j = tid >> 2, q = tid & 3;
    float ss = 0.f;
    uint32_t wds[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (j < HI && 32 * q < dI) {
      if (F == CSA_IFMT_E4M3) {
        const uint4* p = reinterpret_cast<const uint4*>((const uint8_t*)a.qI + qrow + (size_t)j * dI + 32 * q);
        const uint4 v0 = p[0], v1 = p[1];
        wds[0] = v0.x; wds[1] = v0.y; wds[2] = v0.z; wds[3] = v0.w; wds[4] = v1.x; wds[5] = v1.y; wds[6] = v1.z; wds[7] = v1.w;
      } else {
        const uint4 v = *reinterpret_cast<const uint4*>((const uint8_t*)a.qI + (qrow + (size_t)j * dI + 32 * q) / 2);
        wds[0] = v.x; wds[1] = v.y; wds[2] = v.z; wds[3] = v.w;
      }
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float x = F == CSA_IFMT_E4M3 ? e4m3_to_float((wds[e >> 2] >> (8 * (e & 3))) & 0xFFu)
                                         : e2m1_to_float((wds[e >> 3] >> (4 * (e & 7))) & 0xFu);
      ss = fmaf(x, x, ss);
    }
    __syncthreads();                                         // w, scales, U = 0
    if (j < HI && 32 * q < dI) {
      const float sc = F == CSA_IFMT_E4M3 ? sm.qsc[j] : sm.qsc[j * nb + q];
      ss *= sc * sc;
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    float u = (q == 0 && j < HI) ? fabsf(sm.w[j]) * sqrtf(ss) : 0.f;
    u = warp_sum(u);
    if (lane == 0) atomicAdd(&sm.U, u);
  }
  // the query row's integer digits for the exact re-scoring (inputs only: before the wait)
  {
    __shared__ const uint8_t* qrows[64];
    if (tid < 64) qrows[tid] = tid < HI ? (const uint8_t*)a.qI + (F == CSA_IFMT_E4M3 ? qrow + (size_t)tid * dI : (qrow + (size_t)tid * dI) / 2) : nullptr;
    __syncthreads();
    sh_stage_digits<F>(sm.qdig[0], sizeof(sm.qdig[0]), qrows, 64, dI);
  }
  const int n = row_eligible(a, row);
  tc::griddep_wait();                                        // the scores, the histogram, knmax
  __syncthreads();
  if (n <= k) {
    // every eligible entry is selected
    if (part == 0) {
      for (int i = tid; i < k; i += SH_T) out[i] = i < n ? i : -1;
      if (sout) {
        for (int i0 = 0; i0 < k; i0 += SH_RB) {
          const int cnt = max(0, min(SH_RB, n - i0));
          if (tid < SH_RB) sm.band_id[tid] = i0 + tid;
          __syncthreads();
          sh_rescore<F>(ks, sm, a.qI, qrow, b, sm.band_id, cnt);
          if (tid < SH_RB && i0 + tid < k) sout[i0 + tid] = tid < cnt ? (float)sm.rs_out[tid] : 0.f;
          __syncthreads();
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

  // ---- A2: classify this CTA's chunk (whole bitmap words: chunk % 32 == 0): certain entries
  // into the row's bitmap, candidates into this CTA's own region [c0, c0 + count) of the row's
  // list (no place to reserve: the region holds the whole chunk), the count into ctr[4 + part]
  const int c0 = part * chunk, c1 = min(n, c0 + chunk);
  const float* srow = a.scores + (size_t)row * a.ld;
  const int c_end = min(c0 + chunk, (int)a.ld);
  constexpr int SH_WPT = 8;                                  // words per warp per round
  uint2* my_cand = cand_g + c0;
  if (tid == 0) sm.cnt = 0u;
  __syncthreads();
  uint32_t n_sure = 0;
  for (int base0 = c0 + 32 * warp; base0 < c_end; base0 += SH_WPT * 32 * SH_W) {
    float sv[SH_WPT];
#pragma unroll
    for (int u = 0; u < SH_WPT; ++u) {
      const int i = base0 + u * 32 * SH_W + lane;
      sv[u] = i < c1 ? __ldcg(srow + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < SH_WPT; ++u) {
      const int base = base0 + u * 32 * SH_W;
      const bool in = base < c_end && base + lane < c1;
      const bool sure = in && sv[u] > hi_thr;
      const bool cnd = in && !sure && sv[u] >= lo_thr;
      const uint32_t bs = __ballot_sync(0xffffffffu, sure);
      const uint32_t bc = __ballot_sync(0xffffffffu, cnd);
      if (lane == 0 && base < c_end) bitmap[base >> 5] = bs;
      n_sure += __popc(bs);
      if (bc) {
        uint32_t off = 0;
        if (lane == 0) off = atomicAdd(&sm.cnt, (uint32_t)__popc(bc));
        off = __shfl_sync(0xffffffffu, off, 0);
        if (cnd) my_cand[off + __popc(bc & ((1u << lane) - 1u))] = make_uint2(f32_order_key(sv[u]), (uint32_t)(base + lane));
      }
    }
  }
  if (lane == 0 && n_sure) atomicAdd(&ctr[1], n_sure);
  __syncthreads();
  if (tid == 0) ctr[SH_CTR0 + part] = sm.cnt;
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = (atomicAdd(&ctr[2], 1u) == (uint32_t)(P - 1)) ? 1u : 0u;
  __syncthreads();
  if (!sm.last) return;
  __threadfence();

  // ---- B: the last CTA of the row.  The candidates' places: CTA p's count at ctr[4 + p],
  // its list at p * chunk; sm.coff[p] = the first candidate of CTA p in the gathered order.
  const uint32_t n_sure_all = __ldcg(&ctr[1]);
  {
    const uint32_t cp = tid < P ? __ldcg(&ctr[SH_CTR0 + tid]) : 0u;
    uint32_t tot;
    const uint32_t incl = sh_scan(cp, sm.wred, &tot);
    if (tid < P) sm.coff[tid] = incl - cp;
    if (tid == 0) { sm.coff[P] = tot; sm.cnt = tot; }
  }
  __syncthreads();
  const uint32_t nc = sm.cnt;
  const bool staged = nc <= (uint32_t)SH_CCAP;
  // candidate i: staged in shared memory when they all fit, else found in its CTA's region
  auto cget = [&](uint32_t i) -> uint2 {
    if (staged) return sm.cand[i];
    int lo_p = 0, hi_p = P;                                  // the last p with coff[p] <= i
    while (hi_p - lo_p > 1) {
      const int mid = (lo_p + hi_p) >> 1;
      if (sm.coff[mid] <= i) lo_p = mid; else hi_p = mid;
    }
    return __ldcg(cand_g + (size_t)lo_p * chunk + (i - sm.coff[lo_p]));
  };
  // ---- B4: one histogram of the candidates over [lo_thr, hi_thr] (2048 bins of 2^shf keys,
  // built while they are gathered); its bin [tau_lo, tau_hi] holding the want-th largest
  // candidate is narrower than the error margin, so the band is that bin widened by 2E
  uint32_t lo = f32_order_key(lo_thr), hi = f32_order_key(hi_thr);
  uint32_t want = (uint32_t)k - n_sure_all;
  int shf;
  {
    const int range_bits = 32 - __clz(hi - lo);
    shf = range_bits > 11 ? range_bits - 11 : 0;
  }
  for (int i = tid; i < SH_BINS2; i += SH_T) sm.hist2[i] = 0u;
  __syncthreads();
  {
    // every thread's candidates at once (their loads are independent): candidate i lives in
    // the region of the last CTA p with coff[p] <= i
    constexpr int GU = 4;
    for (uint32_t i0 = 0; i0 < nc; i0 += GU * SH_T) {
      uint2 c[GU];
#pragma unroll
      for (int u = 0; u < GU; ++u) {
        const uint32_t i = i0 + u * SH_T + tid;
        c[u] = make_uint2(0u, 0u);
        if (i < nc) {
          int lo_p = 0, hi_p = P;
          while (hi_p - lo_p > 1) {
            const int mid = (lo_p + hi_p) >> 1;
            if (sm.coff[mid] <= i) lo_p = mid; else hi_p = mid;
          }
          c[u] = __ldcg(cand_g + (size_t)lo_p * chunk + (i - sm.coff[lo_p]));
        }
      }
#pragma unroll
      for (int u = 0; u < GU; ++u) {
        const uint32_t i = i0 + u * SH_T + tid;
        if (i >= nc) continue;
        if (staged) sm.cand[i] = c[u];
        if (c[u].x >= lo && c[u].x <= hi) atomicAdd(&sm.hist2[(c[u].x - lo) >> shf], 1u);
      }
    }
  }
  __syncthreads();
  {
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
  const float tau_lo = f32_from_order_key(lo), tau_hi = f32_from_order_key(hi);
  const float E = (EU + 1.52587890625e-05f * fmaxf(fabsf(tau_lo), fabsf(tau_hi))) * 1.0001f;
  const float band_hi = tau_hi + 2.f * E, band_lo = tau_lo - 2.f * E;
  // ---- B5: in / band; the band is re-scored exactly and ranked
  if (tid == 0) { sm.cnt = 0u; sm.ties = 0u; }
  __syncthreads();
  uint32_t my_in = 0;
  for (uint32_t i = tid; i < nc; i += SH_T) {
    const uint2 c = cget(i);
    const float s = f32_from_order_key(c.x);
    if (s > band_hi) {
      ++my_in;
    } else if (s >= band_lo) {
      const uint32_t o = atomicAdd(&sm.cnt, 1u);
      if (o < (uint32_t)SH_BAND) sm.band_id[o] = (int32_t)c.y;
    }
  }
  uint32_t n_in;
  sh_scan(my_in, sm.wred, &n_in);
  const uint32_t n_band = sm.cnt;
  const uint32_t need = (uint32_t)k - n_sure_all - n_in;    // >= 1: the want-th candidate is in the band
  const bool exact = n_band <= (uint32_t)SH_BAND;
  float tau = tau_lo;                                        // the fallback's exact fp32 k-th score
  uint32_t n_above_tau = 0;
  if (exact) {
    for (uint32_t i0 = 0; i0 < n_band; i0 += SH_RB) {
      const int cnt = (int)min((uint32_t)SH_RB, n_band - i0);
      sh_rescore<F>(ks, sm, a.qI, qrow, b, sm.band_id + i0, cnt);
      if (tid < cnt) sm.band_s[i0 + tid] = sm.rs_out[tid];
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
  } else {
    // the band outgrew its buffer (heavy ties): fall back to the fp32 order.  Refine the bin
    // to the exact fp32 want-th largest candidate tau, then count the band entries above it.
    if (tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
    for (int round = 0; round < 4 && lo != hi; ++round) {
      const int range_bits = 32 - __clz(hi - lo);
      const int sh2 = range_bits > 11 ? range_bits - 11 : 0;
      for (int i = tid; i < SH_BINS2; i += SH_T) sm.hist2[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < nc; i += SH_T) {
        const uint32_t x = cget(i).x;
        if (x >= lo && x <= hi) atomicAdd(&sm.hist2[(x - lo) >> sh2], 1u);
      }
      __syncthreads();
      uint32_t cnt[SH_BINS2 / SH_T];
#pragma unroll
      for (int i = 0; i < SH_BINS2 / SH_T; ++i) cnt[i] = sm.hist2[(SH_BINS2 / SH_T) * tid + i];
      sh_find_bin<SH_BINS2 / SH_T>(sm, cnt, want);
      want -= sm.bins_above;
      const uint32_t nlo = lo + (sm.bin_T << sh2);
      const uint64_t top = (uint64_t)nlo + ((1ull << sh2) - 1ull);
      hi = top < (uint64_t)hi ? (uint32_t)top : hi;
      lo = nlo;
      __syncthreads();
    }
    tau = f32_from_order_key(lo);
    uint32_t my_above = 0;
    for (uint32_t i = tid; i < nc; i += SH_T) {
      const float s = f32_from_order_key(cget(i).x);
      my_above += (s > tau && s <= band_hi) ? 1u : 0u;
    }
    sh_scan(my_above, sm.wred, &n_above_tau);
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
    // the exact score of every selected entry (the output is written: read it back)
    __syncthreads();
    for (int i0 = 0; i0 < k; i0 += SH_RB) {
      const int cnt = min(SH_RB, (int)written - i0);
      if (tid < SH_RB) sm.band_id[tid] = (i0 + tid < k) ? __ldcg(out + i0 + tid) : 0;
      __syncthreads();
      if (cnt > 0) sh_rescore<F>(ks, sm, a.qI, qrow, b, sm.band_id, cnt);
      if (tid < SH_RB && i0 + tid < k) sout[i0 + tid] = tid < cnt ? (float)sm.rs_out[tid] : 0.f;
      __syncthreads();
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
  if ((int64_t)rows * P > 0x7fffffffLL || P > SH_CTR_STRIDE - SH_CTR0) return cudaErrorNotSupported;
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

static_assert(sizeof(ShSmem) + 1024 <= 232448, "shared memory budget of one CTA (227 KB, with 1 KB of row pointers)");

}  // namespace csa
