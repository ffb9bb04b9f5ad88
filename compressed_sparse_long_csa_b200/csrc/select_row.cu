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
constexpr int SR_BCAP = 128;              // band entries re-scored exactly
constexpr int SR_RB = 8;                  // entries re-scored at once
constexpr int SR_NMAX = 34816;            // most scores a row stages in shared memory (and bitmap bits)
constexpr int SR_CHUNK = 16384;           // bytes per bulk copy (the first histogram starts on the first)
constexpr int SR_KLD = 160;               // staged key row: dims 16 g .. 16 g + 15 at word 20 g (no bank conflicts)
constexpr int SR_TLD = 66;                // per-head term row stride (the ordered sums read rows side by side)

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
  alignas(16) float sc[1];                // the row's scores (sized at launch)
};

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
    if (g == 0 && j < HI) {
      const double wj = (double)sm.w[j], qs = (double)sm.qsc[j];
#pragma unroll
      for (int e = 0; e < SR_RB; ++e)
        if (e < cnt) {
          const double D = (qs * (double)sm.ksc[e][0]) * ((double)acc[e] * 3.814697265625e-06);   // 2^-18
          sm.term[e][j] = wj * fmax(D, 0.0);
        }
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
#pragma unroll
    for (int e = 0; e < SR_RB; ++e) {
      if (e < cnt) {
        const int x = acc[e] + __shfl_xor_sync(0xffffffffu, acc[e], 1);   // the 32-dim block of lanes g, g ^ 1
        // the block partials at the head's first lane, in block order
        const int p1 = __shfl_down_sync(0xffffffffu, x, 2);
        const int p2 = __shfl_down_sync(0xffffffffu, x, 4);
        const int p3 = __shfl_down_sync(0xffffffffu, x, 6);
        if (g == 0 && j < HI) {
          const int P[4] = {x, p1, p2, p3};
          double D = 0.0;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q >= nb) break;
            const double t = ((double)sm.qsc[j * nb + q] * (double)sm.ksc[e][q]) * ((double)P[q] * 0.25);
            D = q == 0 ? t : D + t;
          }
          sm.term[e][j] = (double)sm.w[j] * fmax(D, 0.0);
        }
      }
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
  const int k = a.k, HI = a.H_I, dI = a.d_I, nb = dI / 32;
  int32_t* out = a.idx_out + (size_t)row * k;
  float* sout = a.score_out ? a.score_out + (size_t)row * k : nullptr;

  // ---- prologue (inputs only; overlaps the scoring kernel)
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
  int qi[16];
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
  const int n = row_eligible(a, row);
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
    for (uint32_t i = warp; i < nbnd; i += SR_W) {
      const int id = sm.bid[i];
      const double s = sm.bs[i];
      uint32_t rank = 0;
      for (uint32_t j0 = 0; j0 < nbnd; j0 += 32) {
        const uint32_t j2 = j0 + lane;
        const bool better = j2 < nbnd && (sm.bs[j2] > s || (sm.bs[j2] == s && sm.bid[j2] < id));
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
    for (uint32_t i = warp; i < nbnd; i += SR_W) {
      const int id = sm.bid[i];
      const double sc = sm.bs[i];
      uint32_t rank = 0;
      for (uint32_t j0 = 0; j0 < nbnd; j0 += 32) {
        const uint32_t j2 = j0 + lane;
        const bool better = j2 < nbnd && (sm.bs[j2] > sc || (sm.bs[j2] == sc && sm.bid[j2] < id));
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
