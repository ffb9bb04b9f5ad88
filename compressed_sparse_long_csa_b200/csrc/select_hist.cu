// Exact top-k of the lightning indexer's decode rows, seeded by two score histograms.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 2: the indexer keeps the k compressed entries with the
// largest scores I[t,s] (k = 512 / 1024 from table "Конфигурации").  Ties go to the
// lower entry index; the selected set is written in ascending index order, padded with -1.
//
// The tensor-core scoring kernels write every eligible fp32 score of a row and two
// histograms of the scores' monotone order keys: a coarse one of 4096 bins (key >> 20: sign,
// exponent, three mantissa bits; built in shared memory, flushed once per CTA) and a fine
// one of 65 536 bins (key >> 16; one reduction per score).  Then:
//
//  A. (every CTA; P CTAs share a row, each owns a contiguous chunk of entries)
//     1. The coarse bin T and, inside it, the fine bin F that hold the k-th largest fp32
//        score follow from suffix counts.
//     2. The fp32 scores carry an error below E = eps * U * knmax + 2^-16 |tau| (eps of the
//        scoring path, U = sum_j |w_j| ||q_j||, knmax >= every key norm; the second term
//        covers the epilogue's head sum), so with the k-th score tau anywhere in F =
//        [f_lo, f_hi]: entries above f_hi + 2 E_max are certainly selected, entries below
//        f_lo - 2 E_max certainly not (E_max: E at |tau| = max(|f_lo|, |f_hi|)), and the
//        band between holds every entry whose order is in doubt: a fine bin's worth, a few
//        dozen at these sizes.
//     3. The CTA marks its certain entries in the row's bitmap, and re-scores its band
//        entries exactly in fp64 from the quantised operands (FP8 / FP4 products and their
//        sums are exact in fp64 in any order; the per-head terms w_j * max(D_j, 0) are then
//        added in head order, as the definition does, so the scores equal the oracle's bit
//        for bit).  It writes (key, index, exact score) of its band entries to its own region
//        of the row's list and its counts; the last CTA of the row to finish (an atomic
//        counter after a memory fence; no CTA waits for another) carries on alone.
//  B. (last CTA of the row)
//     4. The band entries are ranked by (exact score desc, index asc); the first
//        k - (certain entries) are selected.
//     5. The row's bitmap (certain entries plus the chosen band entries) is scanned in
//        ascending order and the indices are written.
// A CTA whose band outgrows its re-scoring buffer (heavy ties) makes the row fall back to
// the fp32 order (score desc, index asc) over the band, and sets CSA_DEVERR_BAND.
#include "indexer.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int SH_T = 256;                // threads per CTA
constexpr int SH_W = SH_T / 32;
constexpr int SH_BINS = 4096;            // coarse bins (key >> 20), written by the scoring epilogues
constexpr int SH_FINE = 16;              // fine bins (key >> 16) per coarse bin
constexpr int SH_BLOC = 64;              // band entries one CTA re-scores
constexpr int SH_BCAP = 4096;            // band entries the last CTA ranks in shared memory
constexpr int SH_RB = 16;                // entries re-scored per batch
constexpr int SH_KLD = 144;              // staged key row: 4 segments of 32 dims, 36 words apart
constexpr int SH_BMW = 8192;             // bitmap words handled per output pass (262 144 entries)
constexpr int SH_BINS2 = 2048;           // fallback refinement bins
constexpr int SH_CTR0 = 4;               // row counters: [1] certain, [2] CTAs done, [3] overflow, [4 + p] band of CTA p
constexpr int SH_CTR_STRIDE = 256;       // words of counters per row (so at most 252 CTAs per row)

// One band entry: the order key of its fp32 score, its index, its exact score.
struct BandEnt {
  uint32_t key;
  int32_t id;
  double s;
};
static_assert(sizeof(BandEnt) == 16, "band entries are 16-byte records");

struct ShSmem {
  alignas(16) int32_t krow[SH_RB][SH_KLD];   // key rows of one re-scoring batch as integers (E4M3: value * 2^9,
                                            // FP4: value * 2), 32-dim segments 36 words apart
  double contrib[SH_RB][65];             // their per-head terms
  double rs_out[SH_RB];                  // their exact scores
  float ksc[SH_RB][4];                   // their scales (E4M3 row scale in [0], MXFP4 block scales)
  int32_t rid[SH_RB];                    // their indices
  BandEnt band[SH_BCAP];                 // A: this CTA's first SH_BLOC band entries; B: every band entry
  uint32_t bm[SH_BMW + SH_BMW / 32];     // output bitmap chunk (word w at w + w / 32: conflict-free runs)
  uint32_t tie[SH_BMW + SH_BMW / 32];    // exact path: the band's verdicts; fallback: entries equal to tau
  uint32_t hist2[SH_BINS2];              // fallback refinement
  uint32_t boff[SH_CTR_STRIDE + 1];      // gathered position of each CTA's band entries
  float w[64];
  float qsc[64 * 4];
  uint32_t wred[SH_W][4];
  uint32_t bins_above, bin_T, cnt, ties, last, ovf;
  float U;
};

// Padded place of bitmap word w: a thread's run of consecutive words is read without bank conflicts.
__device__ __forceinline__ int bmi(int w) { return w + (w >> 5); }

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

// The bin holding the want-th largest key; thread t holds bins [PER t, PER t + PER) in
// cnt[].  Sets sm.bin_T and sm.bins_above (the keys in higher bins).  All threads call.
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

// Exact fp64 scores of the entries sm.rid[0..cnt) (cnt <= SH_RB) of sequence b into
// sm.rs_out, by the whole CTA (all threads call; barriers inside).  Thread t holds, in qi,
// the query codes of head j = t / 4 over dims [32 q, 32 q + 32), q = t % 4 (one MXFP4
// scale block), as integers (E4M3: value * 2^9; FP4: value * 2).  Its partial dot product
// with a key row is then an exact integer (E4M3: below 2^43 in 64 bits; FP4: below 2^13);
// the four partials of a head are combined as the definition does (E4M3: their exact sum
// * 2^-18 times sq * sk; MXFP4: the block terms (qs * ks) * P_b, P_b = partial * 2^-2,
// added in block order), each head's term w_j * max(D_j, 0) is formed, and one thread per
// entry adds the terms in order.
template <int F>
__device__ __forceinline__ void sh_rescore(const KeySide ks, ShSmem& sm, const int (&qi)[32], int b, int cnt) {
  const int tid = threadIdx.x;
  const int j = tid >> 2, q = tid & 3;
  const int dI = ks.dI, nb = dI / 32, HI = ks.HI;
  // ---- stage the key rows: thread t converts 16 codes of entry t / 8
  if (tid < SH_RB * 8) {
    const int e = tid >> 3, seg = tid & 7;
    if (e < cnt && 16 * seg < dI) {
      const size_t koff = (size_t)b * ks.n_max + sm.rid[e];
      int* kr = sm.krow[e] + 36 * (seg >> 1) + 16 * (seg & 1);
      if (F == CSA_IFMT_E4M3) {
        const uint4 v = *reinterpret_cast<const uint4*>((const uint8_t*)ks.kI + koff * dI + 16 * seg);
        const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 16; ++i) kr[i] = (int)(e4m3_to_float((wd[i >> 2] >> (8 * (i & 3))) & 0xFFu) * 512.f);
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>((const uint8_t*)ks.kI + koff * (dI / 2) + 8 * seg);
        const uint32_t wd[2] = {v.x, v.y};
#pragma unroll
        for (int i = 0; i < 16; ++i) kr[i] = (int)(e2m1_to_float((wd[i >> 3] >> (4 * (i & 7))) & 0xFu) * 2.f);
      }
    }
  } else if (tid < SH_RB * 8 + SH_RB * 4) {
    const int u = tid - SH_RB * 8, e2 = u >> 2, q2 = u & 3;
    float v = 0.f;
    if (e2 < cnt) {
      const size_t koff = (size_t)b * ks.n_max + sm.rid[e2];
      if (F == CSA_IFMT_E4M3) v = q2 == 0 ? ((const float*)ks.kI_scale)[koff] : 0.f;
      else v = q2 < nb ? ue8m0_to_float(((const uint8_t*)ks.kI_scale)[koff * nb + q2]) : 0.f;
    }
    sm.ksc[e2][q2] = v;
  }
  __syncthreads();
  // ---- per-head terms, two entries at a time
  const bool live = j < HI && 32 * q < dI;
  const double wj = (j < HI) ? (double)sm.w[j] : 0.0;
  for (int e0 = 0; e0 < cnt; e0 += 2) {
    long long acc[2] = {0, 0};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int4* kr = reinterpret_cast<const int4*>(sm.krow[min(e0 + u, cnt - 1)] + 36 * q);
      if (live) {
        long long x = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int4 kv = kr[i];
          if (F == CSA_IFMT_E4M3) {
            x += (long long)qi[4 * i] * kv.x;
            x += (long long)qi[4 * i + 1] * kv.y;
            x += (long long)qi[4 * i + 2] * kv.z;
            x += (long long)qi[4 * i + 3] * kv.w;
          } else {
            x += qi[4 * i] * kv.x + qi[4 * i + 1] * kv.y + qi[4 * i + 2] * kv.z + qi[4 * i + 3] * kv.w;
          }
        }
        acc[u] = x;
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = min(e0 + u, cnt - 1);
      double D;
      if (F == CSA_IFMT_E4M3) {
        long long raw = acc[u] + __shfl_xor_sync(0xffffffffu, acc[u], 1);
        raw += __shfl_xor_sync(0xffffffffu, raw, 2);                                // exact
        D = live ? ((double)sm.qsc[j] * (double)sm.ksc[e][0]) * ((double)raw * 3.814697265625e-06) : 0.0;   // 2^-18
      } else {
        const double t = live ? ((double)sm.qsc[j * nb + q] * (double)sm.ksc[e][q]) * ((double)acc[u] * 0.25) : 0.0;
        const double t1 = __shfl_down_sync(0xffffffffu, t, 1);
        const double t2 = __shfl_down_sync(0xffffffffu, t, 2);
        const double t3 = __shfl_down_sync(0xffffffffu, t, 3);
        D = ((t + t1) + t2) + t3;                                               // block order (lane q = 0)
      }
      if (q == 0 && j < HI && e0 + u < cnt) sm.contrib[e][j] = wj * fmax(D, 0.0);
    }
  }
  __syncthreads();
  if (tid < cnt) {
    // the terms in registers first, then added in head order
    double t[64];
#pragma unroll
    for (int jj = 0; jj < 64; ++jj) t[jj] = jj < HI ? sm.contrib[tid][jj] : 0.0;
    double S = 0.0;
#pragma unroll
    for (int jj = 0; jj < 64; ++jj)
      if (jj < HI) S += t[jj];
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
  const uint32_t* hist = a.hist + (size_t)row * SH_BINS;
  const uint32_t* fhist = a.fhist + (size_t)row * SH_BINS * SH_FINE;
  uint32_t* ctr = a.counters + (size_t)row * SH_CTR_STRIDE;
  uint32_t* bitmap = a.bitmap + (size_t)row * (a.ld / 32);
  BandEnt* band_g = reinterpret_cast<BandEnt*>(a.cand) + (size_t)row * a.ld;
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
  if (tid == 0) { sm.U = 0.f; sm.cnt = 0u; sm.ovf = 0u; }
  float qr[32];
  int qi[32];
  {
    const int j = tid >> 2, q = tid & 3;
#pragma unroll
    for (int i = 0; i < 32; ++i) qr[i] = 0.f;
    if (j < HI && 32 * q < dI) {
      if (F == CSA_IFMT_E4M3) {
        const uint4* p = reinterpret_cast<const uint4*>((const uint8_t*)a.qI + qrow + (size_t)j * dI + 32 * q);
        const uint4 v0 = p[0], v1 = p[1];
        const uint32_t wds[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int e = 0; e < 32; ++e) qr[e] = e4m3_to_float((wds[e >> 2] >> (8 * (e & 3))) & 0xFFu);
      } else {
        const uint4 v = *reinterpret_cast<const uint4*>((const uint8_t*)a.qI + (qrow + (size_t)j * dI + 32 * q) / 2);
        const uint32_t wds[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 32; ++e) qr[e] = e2m1_to_float((wds[e >> 3] >> (4 * (e & 7))) & 0xFu);
      }
    }
    __syncthreads();                                         // w, scales, U = 0
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) ss = fmaf(qr[e], qr[e], ss);
#pragma unroll
    for (int e = 0; e < 32; ++e) qi[e] = (int)(qr[e] * (F == CSA_IFMT_E4M3 ? 512.f : 2.f));   // exact integers
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
  const int n = row_eligible(a, row);
  tc::griddep_wait();                                        // the scores, the histograms, knmax
  __syncthreads();
  if (n <= k) {
    // every eligible entry is selected
    if (part == 0) {
      for (int i = tid; i < k; i += SH_T) out[i] = i < n ? i : -1;
      if (sout) {
        for (int i0 = 0; i0 < k; i0 += SH_RB) {
          const int cnt = max(0, min(SH_RB, n - i0));
          if (tid < SH_RB) sm.rid[tid] = i0 + tid;
          __syncthreads();
          if (cnt > 0) sh_rescore<F>(ks, sm, qi, b, cnt);
          if (tid < SH_RB && i0 + tid < k) sout[i0 + tid] = tid < cnt ? (float)sm.rs_out[tid] : 0.f;
          __syncthreads();
        }
      }
    }
    return;
  }

  // ---- A1: the coarse bin T (thread t holds bins 16t .. 16t+15), then the fine bin inside it
  {
    uint32_t cnt[SH_BINS / SH_T];
    const uint4* hp = reinterpret_cast<const uint4*>(hist + (SH_BINS / SH_T) * tid);
#pragma unroll
    for (int v = 0; v < SH_BINS / SH_T / 4; ++v) {
      const uint4 x = __ldcg(hp + v);
      cnt[4 * v] = x.x; cnt[4 * v + 1] = x.y; cnt[4 * v + 2] = x.z; cnt[4 * v + 3] = x.w;
    }
    sh_find_bin<SH_BINS / SH_T>(sm, cnt, (uint32_t)k);
  }
  const uint32_t T = sm.bin_T;
  const uint32_t want_T = (uint32_t)k - sm.bins_above;
  if (warp == 0) {
    // the 16 fine bins of T, from the top: lane i (< 16) holds fine bin 15 - i
    const uint32_t c = lane < SH_FINE ? __ldcg(fhist + (size_t)T * SH_FINE + (SH_FINE - 1 - lane)) : 0u;
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    const bool here = lane < SH_FINE && incl - c < want_T && want_T <= incl;
    const uint32_t hb = __ballot_sync(0xffffffffu, here);
    if (lane == 0) sm.bin_T = hb ? T * SH_FINE + (SH_FINE - 1 - (__ffs(hb) - 1)) : T * SH_FINE;
  }
  __syncthreads();
  const uint32_t Fb = sm.bin_T;                             // the fine bin of the k-th score
  const float knmax = __uint_as_float(a.knmax[b]);
  const float f_lo = f32_from_order_key(Fb << 16), f_hi = f32_from_order_key((Fb << 16) | 0xFFFFu);
  const float EU = a.eps_dot * sm.U * 1.0001f * knmax;
  const float E_max = (EU + 1.52587890625e-05f * fmaxf(fabsf(f_lo), fabsf(f_hi))) * 1.0001f;
  const float band_hi = f_hi + 2.f * E_max, band_lo = f_lo - 2.f * E_max;

  // ---- A2: classify this CTA's chunk (whole bitmap words: chunk % 32 == 0): certain entries
  // into the row's bitmap, band entries into this CTA's own region [c0, c0 + count) of the
  // row's list (the region holds the whole chunk) and, the first SH_BLOC, into shared memory
  const int c0 = part * chunk, c1 = min(n, c0 + chunk);
  const float* srow = a.scores + (size_t)row * a.ld;
  const int c_end = min(c0 + chunk, (int)a.ld);
  constexpr int SH_WPT = 8;                                  // words per warp per round
  BandEnt* my_band = band_g + c0;
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
      const bool sure = in && sv[u] > band_hi;
      const bool bnd = in && !sure && sv[u] >= band_lo;
      const uint32_t bs = __ballot_sync(0xffffffffu, sure);
      const uint32_t bb = __ballot_sync(0xffffffffu, bnd);
      if (lane == 0 && base < c_end) bitmap[base >> 5] = bs;
      n_sure += __popc(bs);
      if (bb) {
        uint32_t off = 0;
        if (lane == 0) off = atomicAdd(&sm.cnt, (uint32_t)__popc(bb));
        off = __shfl_sync(0xffffffffu, off, 0) + __popc(bb & ((1u << lane) - 1u));
        if (bnd) {
          const BandEnt be{f32_order_key(sv[u]), base + lane, 0.0};
          my_band[off] = be;
          if (off < (uint32_t)SH_BLOC) {
            sm.band[off] = be;
            // its key row is re-scored next: start bringing it into L2
            const size_t koff = (size_t)b * a.n_max + (base + lane);
            const char* kp = (const char*)a.kI + koff * (F == CSA_IFMT_E4M3 ? dI : dI / 2);
            asm volatile("prefetch.global.L2 [%0];" ::"l"(kp));
          }
        }
      }
    }
  }
  if (lane == 0 && n_sure) atomicAdd(&ctr[1], n_sure);
  __syncthreads();
  // ---- A3: exact scores of this CTA's band entries
  const uint32_t nb_mine = sm.cnt;
  if (nb_mine <= (uint32_t)SH_BLOC) {
    for (uint32_t i0 = 0; i0 < nb_mine; i0 += SH_RB) {
      const int cnt = (int)min((uint32_t)SH_RB, nb_mine - i0);
      if (tid < cnt) sm.rid[tid] = sm.band[i0 + tid].id;
      __syncthreads();
      sh_rescore<F>(ks, sm, qi, b, cnt);
      if (tid < cnt) my_band[i0 + tid].s = sm.rs_out[tid];
    }
  } else if (tid == 0) {
    atomicOr(&ctr[3], 1u);                                   // the row falls back to the fp32 order
  }
  if (tid == 0) ctr[SH_CTR0 + part] = nb_mine;
  __threadfence();
  __syncthreads();
  if (tid == 0) sm.last = (atomicAdd(&ctr[2], 1u) == (uint32_t)(P - 1)) ? 1u : 0u;
  __syncthreads();
  if (!sm.last) return;
  __threadfence();

  // ---- B: the last CTA of the row.  Band entries of CTA p: ctr[4 + p] of them at p * chunk.
  const uint32_t n_sure_all = __ldcg(&ctr[1]);
  bool fallback = __ldcg(&ctr[3]) != 0u;
  {
    const uint32_t cp = tid < P ? __ldcg(&ctr[SH_CTR0 + tid]) : 0u;
    uint32_t tot;
    const uint32_t incl = sh_scan(cp, sm.wred, &tot);
    if (tid < P) sm.boff[tid] = incl - cp;
    if (tid == 0) { sm.boff[P] = tot; sm.cnt = tot; sm.ties = 0u; }
  }
  __syncthreads();
  const uint32_t nbt = sm.cnt;
  const uint32_t need = (uint32_t)k - n_sure_all;            // >= 1, <= nbt
  if (nbt > (uint32_t)SH_BMW) fallback = true;               // more verdicts than their buffer holds
  const bool staged = nbt <= (uint32_t)SH_BCAP;
  // band entry i: in the region of the last CTA p with boff[p] <= i
  auto bsrc = [&](uint32_t i) -> const uint4* {
    int lo_p = 0, hi_p = P;
    while (hi_p - lo_p > 1) {
      const int mid = (lo_p + hi_p) >> 1;
      if (sm.boff[mid] <= i) lo_p = mid; else hi_p = mid;
    }
    return reinterpret_cast<const uint4*>(band_g + (size_t)lo_p * chunk + (i - sm.boff[lo_p]));
  };
  auto bget = [&](uint32_t i) -> BandEnt {
    if (staged) return sm.band[i];
    const uint4 raw = __ldcg(bsrc(i));
    BandEnt e;
    e.key = raw.x;
    e.id = (int32_t)raw.y;
    e.s = __hiloint2double((int)raw.w, (int)raw.z);
    return e;
  };
  if (staged)
    for (uint32_t i = tid; i < nbt; i += SH_T) *reinterpret_cast<uint4*>(&sm.band[i]) = __ldcg(bsrc(i));
  const int nwords = (n + 31) >> 5;
  const bool one_pass = nwords <= SH_BMW;                    // the bitmap words come in with the band
  if (one_pass)
    for (int w = tid; w < nwords; w += SH_T) sm.bm[bmi(w)] = __ldcg(bitmap + w);
  __syncthreads();
  // fallback: the exact fp32 need-th largest band key tau and the count above it
  uint32_t tau_key = 0u, n_above_tau = 0u;
  if (fallback) {
    if (tid == 0) raise_err(a.err, CSA_DEVERR_BAND);
    uint32_t lo = f32_order_key(band_lo), hi = f32_order_key(band_hi), want = need;
    for (int round = 0; round < 4 && lo != hi; ++round) {
      const int range_bits = 32 - __clz(hi - lo);
      const int sh2 = range_bits > 11 ? range_bits - 11 : 0;
      for (int i = tid; i < SH_BINS2; i += SH_T) sm.hist2[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < nbt; i += SH_T) {
        const uint32_t x = bget(i).key;
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
    tau_key = lo;
    uint32_t my_above = 0;
    for (uint32_t i = tid; i < nbt; i += SH_T) my_above += bget(i).key > tau_key ? 1u : 0u;
    sh_scan(my_above, sm.wred, &n_above_tau);
  }
  const uint32_t quota = need > n_above_tau ? need - n_above_tau : 0u;   // fallback: ties at tau by index
  // exact path: rank every band entry by (exact score desc, index asc), one warp per entry and
  // 32 others per step (64-bit monotone keys of the scores: integer compares); sm.tie holds
  // the verdicts (1 = chosen) until the output loop clears it
  if (!fallback) {
    auto okey = [](double x) -> unsigned long long {
      const unsigned long long u = (unsigned long long)__double_as_longlong(x);
      return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
    };
    for (uint32_t i = warp; i < nbt; i += SH_W) {
      const BandEnt be = bget(i);
      const unsigned long long ki = okey(be.s);
      uint32_t rank = 0;
      for (uint32_t j0 = 0; j0 < nbt; j0 += 32) {
        const uint32_t jx = j0 + lane;
        bool better = false;
        if (jx < nbt) {
          const BandEnt o = bget(jx);
          const unsigned long long kj = okey(o.s);
          better = kj > ki || (kj == ki && o.id < be.id);
        }
        rank += __popc(__ballot_sync(0xffffffffu, better));
      }
      if (lane == 0 && i < (uint32_t)SH_BMW) sm.tie[i] = rank < need ? 1u : 0u;
    }
    __syncthreads();
  }
  // ---- B4 / B5: ascending write, SH_BMW bitmap words (32 * SH_BMW entries) per pass
  uint32_t written = 0;
  for (int w0 = 0; w0 < nwords; w0 += SH_BMW) {
    const int w1 = min(nwords, w0 + SH_BMW);
    const int e0 = 32 * w0, e1 = 32 * w1;
    if (!one_pass) {
      for (int w = w0 + tid; w < w1; w += SH_T) sm.bm[bmi(w - w0)] = __ldcg(bitmap + w);
      __syncthreads();                                       // every word is in before any bit is set
    }
    if (!fallback) {
      // the chosen band entries of this range (verdicts in sm.tie[i], from the ranking above)
      for (uint32_t i = tid; i < nbt; i += SH_T) {
        const BandEnt be = bget(i);
        const bool take = i < (uint32_t)SH_BMW ? sm.tie[i] != 0u : false;
        if (take && be.id >= e0 && be.id < e1) atomicOr(&sm.bm[bmi((be.id - e0) >> 5)], 1u << ((be.id - e0) & 31));
      }
    } else {
      for (int w = w0 + tid; w < w1; w += SH_T) sm.tie[bmi(w - w0)] = 0u;
      __syncthreads();                                       // the cleared words before any tie bit
      for (uint32_t i = tid; i < nbt; i += SH_T) {
        const BandEnt be = bget(i);
        if (be.id < e0 || be.id >= e1) continue;
        if (be.key > tau_key) atomicOr(&sm.bm[bmi((be.id - e0) >> 5)], 1u << ((be.id - e0) & 31));
        if (be.key == tau_key) atomicOr(&sm.tie[bmi((be.id - e0) >> 5)], 1u << ((be.id - e0) & 31));
      }
    }
    __syncthreads();
    const int nw = w1 - w0, wpt = (nw + SH_T - 1) / SH_T;
    const int a0 = tid * wpt, a1 = min(nw, a0 + wpt);
    if (fallback) {
      uint32_t c = 0;
      for (int w = a0; w < a1; ++w) c += __popc(sm.tie[bmi(w)]);
      uint32_t tot;
      uint32_t seen = sh_scan(c, sm.wred, &tot) - c + sm.ties;     // ties of earlier passes first
      for (int w = a0; w < a1; ++w) {
        uint32_t keep = 0u;
        for (uint32_t bits = sm.tie[bmi(w)]; bits; bits &= bits - 1) {
          if (seen < quota) keep |= bits & (0u - bits);
          ++seen;
        }
        sm.bm[bmi(w)] |= keep;
      }
      __syncthreads();
      if (tid == 0) sm.ties += tot;
    }
    // prefix counts over the words (contiguous words per thread) and the write
    uint32_t c = 0;
    for (int w = a0; w < a1; ++w) c += __popc(sm.bm[bmi(w)]);
    uint32_t tot;
    uint32_t pos = written + sh_scan(c, sm.wred, &tot) - c;
    for (int w = a0; w < a1; ++w)
      for (uint32_t bits = sm.bm[bmi(w)]; bits; bits &= bits - 1) {
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
      const int cnt = max(0, min(SH_RB, (int)written - i0));
      if (tid < SH_RB) sm.rid[tid] = (i0 + tid < k) ? __ldcg(out + i0 + tid) : 0;
      __syncthreads();
      if (cnt > 0) sh_rescore<F>(ks, sm, qi, b, cnt);
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
  if (!a.hist || !a.fhist || a.H_I > 64 || a.d_I > 128 || (a.ifmt != CSA_IFMT_E4M3 && a.ifmt != CSA_IFMT_MXFP4))
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

static_assert(sizeof(ShSmem) <= 232448, "shared memory budget of one CTA (227 KB)");

}  // namespace csa
