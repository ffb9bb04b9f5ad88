// Lightning indexer scores on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 2 (DSA lightning indexer, ReLU scores I[t,s]) and
// section "FP4 с учётом квантования" (low-precision Q·K of the indexer).
//
// Per sequence b the scores are a GEMM with the entries on M and (query, head) on
// N:  D[s, (g, j)] = sum_c k8[s, c] * q8[g, j, c]  (E4M3 x E4M3 -> FP32 in TMEM),
// followed by an epilogue that turns each TMEM row (one entry) into
//   I[g, s] = sk[s] * sum_j (w[g, j] * sq[g, j]) * max(0, D[s, (g, j)]),
// i.e. the ReLU, the head weighting and the head sum happen in registers, one
// entry per thread, and only one fp32 score per (query, entry) is written.
//
// CTA = (split of the entry tiles, group of G queries, sequence).  Warp roles:
// warp 0 issues TMA loads of 128-entry x 128-byte key tiles (128-byte swizzle)
// into a STAGES-deep ring (the first ones before the CTA's setup barrier); warp 1 owns
// the TMEM allocation and one lane issues the tcgen05.mma (M = 128, N = 64 G, K = 32,
// four per tile) into a ring of accumulators; warps 4..11 run the epilogue as two
// warpgroups that take alternate tiles.  Every wait is bounded: on timeout the CTA
// raises CSA_DEVERR_TIMEOUT, drains its own copies and exits.
#include "indexer.cuh"
#include "tc.cuh"

#include <cudaTypedefs.h>
#include <type_traits>

namespace csa {

namespace {

constexpr int IT_ROWS = 128;     // entries per tile (MMA M)
constexpr int IT_KB = 128;       // bytes per key row (d_I = 128 FP8 values)
constexpr int IT_TILE_BYTES = IT_ROWS * IT_KB;

struct IdxTcParams {
  IndexerArgs a;
  int n_qg;            // query groups per sequence
  int tiles;           // ceil(n_max / 128)
  int tiles_per_split;
};

constexpr int IT_THREADS = 384;  // warp 0 TMA, warp 1 MMA, warps 4..11 epilogue (two warpgroups)

// The score histograms that seed the decode selection (select_hist.cu): coarse bins are the
// top 12 bits of a score's monotone order key, fine bins the top 16.  A CTA counts its scores
// in a window of IT_FWIN fine bins in shared memory (16-aligned, anchored on the first score
// it sees: a row's scores span a few hundred fine bins) and adds the window to the row's
// fine and coarse histograms once, at the end; a score outside the window goes to them
// directly.
constexpr int IT_HBINS = 4096;
constexpr int IT_FWIN = 2048;
constexpr uint32_t IT_FNONE = 0xFFFFFFFFu;

// Count one score (order key) of row `row` (all lanes call; `valid` lanes count).
__device__ __forceinline__ void hist_count(uint32_t* fwin, uint32_t* fbase, const IndexerArgs& a, size_t row,
                                           uint32_t key, bool valid) {
  if (!valid) return;
  const uint32_t fb = key >> 16;
  uint32_t base = *(volatile uint32_t*)fbase;
  if (base == IT_FNONE) {
    const uint32_t lo = fb > (uint32_t)(IT_FWIN / 2) ? ((fb - IT_FWIN / 2) & ~15u) : 0u;
    const uint32_t want = lo < 65536u - IT_FWIN ? lo : 65536u - IT_FWIN;
    const uint32_t old = atomicCAS(fbase, IT_FNONE, want);
    base = old == IT_FNONE ? want : old;
  }
  const uint32_t o = fb - base;
  if (o < (uint32_t)IT_FWIN) {
    atomicAdd(fwin + o, 1u);
  } else {
    atomicAdd(a.fhist + row * (IT_HBINS * 16) + fb, 1u);
    atomicAdd(a.hist + row * IT_HBINS + (fb >> 4), 1u);
  }
}

// Add a CTA's window to the row's histograms (all threads of the CTA call, after a barrier).
__device__ __forceinline__ void hist_flush(const uint32_t* fwin, uint32_t fbase, const IndexerArgs& a, size_t row) {
  if (fbase == IT_FNONE) return;
  uint32_t* gf = a.fhist + row * (IT_HBINS * 16) + fbase;
  for (int i = threadIdx.x; i < IT_FWIN; i += blockDim.x) {
    const uint32_t c = fwin[i];
    if (c) atomicAdd(gf + i, c);
  }
  for (int g = threadIdx.x; g < IT_FWIN / 16; g += blockDim.x) {
    uint32_t c = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) c += fwin[16 * g + i];
    if (c) atomicAdd(a.hist + row * IT_HBINS + (fbase >> 4) + g, c);
  }
}

// ---- the streaming selection of prefill rows --------------------------------------------
// A CTA of the four-query kernel scores every eligible entry of its rows (one entry split),
// so instead of writing the scores it keeps, per row, the entries whose order key is at
// least a running threshold (IDX_STREAM_CAP of them in shared memory).  When a row's list has
// less than two tiles' worth of room, the 256 epilogue threads compact it: the k-th largest
// key of the list lies in a histogram bin [b_lo, ...]; the exact k-th largest score of the
// row can only be larger, and an entry below it by more than the error band 2E can never be
// selected, so the threshold rises to b_lo - 2E(b_lo) (rounded down; x - 2E(x) grows with x)
// and the entries below it leave.  At the end the lists go to the workspace with the
// threshold, U and the key-norm bound they used, and the selection kernel finishes each row
// from its list (select_row.cu).  No score leaves the SM.
constexpr int IT_PF = 4;                   // key scales fetched this many tiles (of a thread's own) ahead
constexpr int ST_T = 256;                  // epilogue threads (warps 4..11)
constexpr int ST_HB = 2048;                // bins of the compaction histograms (all rows)
constexpr int ST_PAIRS = 2;                // pairs of tiles between two meetings of the epilogue threads
static_assert(IDX_STREAM_CAP - 2 * ST_PAIRS * IT_ROWS > IDX_STREAM_KMAX,
              "a compacted list (about k entries) leaves room for the appends until the next meeting");

template <int G>
struct StreamBuf {
  uint32_t ckey[G][IDX_STREAM_CAP];        // order keys of the kept entries
  int32_t cid[G][IDX_STREAM_CAP];          // their indices
  uint32_t hist[ST_HB];
  unsigned long long ccnt;                  // the rows' list lengths, 16 bits each
  uint32_t thr[G], ovf[G];
  float U[G];
  uint32_t kmaxbits;
  uint32_t red[G][ST_T / 32];
  uint32_t lo[G], hi[G], bin[G];
};
struct StreamNone {};
static_assert(IDX_STREAM_CAP + 2 * 2 * 128 < 65536, "the packed 16-bit list lengths cannot carry");

template <int G, int STAGES, bool HIST, bool STREAM = false>
struct IdxSmem {
  alignas(1024) uint8_t q[G * 64 * IT_KB];
  alignas(1024) uint8_t k[STAGES][IT_TILE_BYTES];
  uint32_t fwin[HIST ? IT_FWIN : 1];
  uint32_t fbase;
  alignas(8) uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[4];
  uint64_t tempty[4];
  uint64_t qfull;
  uint32_t tmem_base;
  int abort_flag;
  int t_begin, t_end;
  int issued0;          // tile loads issued before the setup barrier
  int n_elig[G];
  int row[G];
  int t_dep;            // tile of the row's newest entry (partial-slot mode), else -1
  uint32_t part[3];     // the CTA's key range (max key, max ~key) and key-norm bound (partial-slot mode)
  alignas(16) float wq[G][64];
  typename std::conditional<STREAM, StreamBuf<G>, StreamNone>::type st;
};

// The weighted ReLU head sum of one entry (TMEM lane = the thread's entry) for query g of the
// accumulator at column `col`: four partial sums over the heads (j mod 4).
__device__ __forceinline__ float head_sum(uint32_t tmem_lane_col, const float* wq) {
  float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q16 = 0; q16 < 4; ++q16) {
    uint32_t v[16];
    tc::tmem_ld16(tmem_lane_col + q16 * 16, v);
    // the 16 weights as four 16-byte loads, in flight with the TMEM load (one load per
    // weight exposed its latency 64 times per tile)
    const float4* w4p = reinterpret_cast<const float4*>(wq + q16 * 16);
    float4 w4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) w4[u] = w4p[u];
    tc::tmem_ld_wait();
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      part[0] = fmaf(w4[u].x, fmaxf(__uint_as_float(v[4 * u]), 0.f), part[0]);
      part[1] = fmaf(w4[u].y, fmaxf(__uint_as_float(v[4 * u + 1]), 0.f), part[1]);
      part[2] = fmaf(w4[u].z, fmaxf(__uint_as_float(v[4 * u + 2]), 0.f), part[2]);
      part[3] = fmaf(w4[u].w, fmaxf(__uint_as_float(v[4 * u + 3]), 0.f), part[3]);
    }
  }
  return (part[0] + part[1]) + (part[2] + part[3]);
}

// Barrier of the 256 epilogue threads (named barrier 1; the producer and MMA warps go on).
__device__ __forceinline__ void ep_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Length of row g's list (16 bits of the packed counts; a list that overflowed keeps counting
// to at most IDX_STREAM_CAP + 2 * ST_PAIRS * 128 < 2^16).
template <int G>
__device__ __forceinline__ uint32_t st_count(const StreamBuf<G>& st, int g) {
  return (uint32_t)((*(volatile const unsigned long long*)&st.ccnt >> (16 * g)) & 0xFFFFull);
}

// Exclusive scan of G values per epilogue thread at once; tot[g] = the sums.
template <int G>
__device__ __forceinline__ void ep_scan_g(const uint32_t (&v)[G], uint32_t (&excl)[G], uint32_t (&tot)[G],
                                          uint32_t (*red)[ST_T / 32]) {
  const int te = threadIdx.x - 128, lane = te & 31, w = te >> 5;
  uint32_t incl[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    incl[g] = v[g];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, incl[g], o);
      if (lane >= o) incl[g] += x;
    }
  }
  ep_sync();
  if (lane == 31)
#pragma unroll
    for (int g = 0; g < G; ++g) red[g][w] = incl[g];
  ep_sync();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    uint32_t pre = 0, t = 0;
#pragma unroll
    for (int i = 0; i < ST_T / 32; ++i) {
      const uint32_t x = red[g][i];
      pre += i < w ? x : 0u;
      t += x;
    }
    excl[g] = pre + incl[g] - v[g];
    tot[g] = t;
  }
}

// Compact every row's list at once: raise each row's threshold to b_lo - 2E(b_lo), b_lo the
// lower edge of the histogram bin (512 bins over the list's key range) that holds the list's
// k-th largest key, and drop the entries below it.  A row with at most k entries keeps all.
template <int G>
__device__ __noinline__ void ep_compact_all(StreamBuf<G>& st, uint32_t k, const float (&EU)[G]) {
  constexpr int HB = ST_HB / G;             // bins per row
  const int te = threadIdx.x - 128, lane = te & 31;
  uint32_t n[G], mn[G], mx[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    n[g] = min(st_count(st, g), (uint32_t)IDX_STREAM_CAP);
    mn[g] = 0xFFFFFFFFu;
    mx[g] = 0u;
    for (uint32_t i = te; i < n[g]; i += ST_T) {
      const uint32_t key = st.ckey[g][i];
      mn[g] = min(mn[g], key);
      mx[g] = max(mx[g], key);
    }
    mn[g] = __reduce_min_sync(0xffffffffu, mn[g]);
    mx[g] = __reduce_max_sync(0xffffffffu, mx[g]);
  }
  if (te < G) { st.lo[te] = 0xFFFFFFFFu; st.hi[te] = 0u; st.bin[te] = 0u; }
  for (int i = te; i < ST_HB; i += ST_T) st.hist[i] = 0u;
  ep_sync();
  if (lane == 0)
#pragma unroll
    for (int g = 0; g < G; ++g) { atomicMin(&st.lo[g], mn[g]); atomicMax(&st.hi[g], mx[g]); }
  ep_sync();
  int sh[G];
  uint32_t lo[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    lo[g] = st.lo[g];
    const uint64_t width = st.hi[g] >= lo[g] ? (uint64_t)(st.hi[g] - lo[g]) + 1u : 1u;
    const int bits = width <= 1 ? 0 : 64 - __clzll((long long)(width - 1));
    constexpr int LB = HB == 2048 ? 11 : HB == 1024 ? 10 : 9;
    sh[g] = bits > LB ? bits - LB : 0;
    for (uint32_t i = te; i < n[g]; i += ST_T) atomicAdd(&st.hist[g * HB + ((st.ckey[g][i] - lo[g]) >> sh[g])], 1u);
  }
  ep_sync();
  // the bin of the k-th largest key of each row: thread t holds bins [HB/ST_T * t, +HB/ST_T)
  constexpr int PER = HB / ST_T;
  {
    uint32_t c[G][PER], mine[G], excl[G], tot[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      mine[g] = 0u;
#pragma unroll
      for (int i = 0; i < PER; ++i) { c[g][i] = st.hist[g * HB + PER * te + i]; mine[g] += c[g][i]; }
    }
    ep_scan_g<G>(mine, excl, tot, st.red);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      uint32_t above = tot[g] - excl[g] - mine[g];
#pragma unroll
      for (int i = PER - 1; i >= 0; --i) {
        if (above < k && k <= above + c[g][i]) st.bin[g] = (uint32_t)(PER * te + i);
        above += c[g][i];
      }
    }
  }
  ep_sync();
  uint32_t thr[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    thr[g] = st.thr[g];
    if (n[g] > k) {
      const float x = f32_from_order_key(lo[g] + (st.bin[g] << sh[g]));
      const float E2 = 2.f * ((EU[g] + 1.52587890625e-05f * fabsf(x)) * 1.0002f);
      thr[g] = max(thr[g], f32_order_key(__fsub_rd(x, E2)));
    }
  }
  // in place: thread t keeps slots t, t + 256, ... of every row (conflict-free reads; the list's
  // order does not matter)
  constexpr int SL = IDX_STREAM_CAP / ST_T;
  uint32_t kk[G][SL], keep[G], cnt[G], pos[G], tot2[G];
  int32_t ii[G][SL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    keep[g] = 0u;
#pragma unroll
    for (int u = 0; u < SL; ++u) {
      const uint32_t i = te + ST_T * u;
      const bool v = i < n[g];
      kk[g][u] = v ? st.ckey[g][i] : 0u;
      ii[g][u] = v ? st.cid[g][i] : 0;
      keep[g] |= (v && kk[g][u] >= thr[g] ? 1u : 0u) << u;
    }
    cnt[g] = __popc(keep[g]);
  }
  ep_scan_g<G>(cnt, pos, tot2, st.red);                  // its barriers order the reads above before the writes
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int u = 0; u < SL; ++u)
      if ((keep[g] >> u) & 1u) {
        st.ckey[g][pos[g]] = kk[g][u];
        st.cid[g][pos[g]] = ii[g][u];
        ++pos[g];
      }
    if (te == 0) st.thr[g] = thr[g];
  }
  if (te == 0) {
    unsigned long long c = 0ull;
#pragma unroll
    for (int g = 0; g < G; ++g) c |= (unsigned long long)tot2[g] << (16 * g);
    st.ccnt = c;
  }
  ep_sync();
}

template <int G, int STAGES, bool HIST, bool STREAM = false>
__global__ void __launch_bounds__(IT_THREADS, G == 1 ? 2 : 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ, IdxTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  using Sm = IdxSmem<G, STAGES, HIST, STREAM>;
  Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const IndexerArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, qg = blockIdx.y, b = blockIdx.z;
  constexpr int N = 64 * G;
  constexpr int NACC = (G == 1) ? 4 : 2;     // accumulators in TMEM
  constexpr uint32_t NCOLS = NACC * N;       // a power of two >= 32

  if (threadIdx.x == 0) {
    tc::prefetch_tmap(&tmK);                 // descriptor fetches overlap the setup
    tc::prefetch_tmap(&tmQ);
    for (int s = 0; s < STAGES; ++s) { tc::mbar_init(&sm.full[s], 1); tc::mbar_init(&sm.empty[s], 1); }
    for (int s = 0; s < NACC; ++s) { tc::mbar_init(&sm.tfull[s], 1); tc::mbar_init(&sm.tempty[s], 4); }
    tc::mbar_init(&sm.qfull, 1);
    tc::fence_mbar_init();
    sm.abort_flag = 0;
    int max_elig = 0;
    for (int g = 0; g < G; ++g) {
      const int t = qg * G + g;
      int ne = 0, row = b * a.Tq;
      if (t < a.Tq) { row = b * a.Tq + t; ne = row_eligible(a, row); }
      sm.n_elig[g] = ne;
      sm.row[g] = row;
      max_elig = ne > max_elig ? ne : max_elig;
    }
    const int t_lim = (max_elig + IT_ROWS - 1) / IT_ROWS;
    int t0 = split * p.tiles_per_split, t1 = t0 + p.tiles_per_split;
    if (t1 > t_lim) t1 = t_lim;
    sm.t_begin = t0;
    sm.t_end = t1 > t0 ? t1 : t0;
    // partial-slot mode (one query per CTA): a preceding decode append may still be writing
    // the row's newest key, so its tile is loaded only after waiting for that grid
    sm.t_dep = (G == 1 && a.kpart > 0 && max_elig > 0) ? (max_elig - 1) / IT_ROWS : -1;
    sm.part[0] = sm.part[1] = sm.part[2] = 0u;
    // the query tile and the first key tiles go out before the setup barrier (a stage's
    // first use needs no release)
    int n0 = sm.t_end - t0 < STAGES ? sm.t_end - t0 : STAGES;
    if (sm.t_dep >= t0 && sm.t_dep < t0 + n0) n0 = sm.t_dep - t0;
    if (sm.t_end > t0) {                      // (n0 may be 0: the first tile waits for the append)
      tc::mbar_arrive_expect_tx(&sm.qfull, G * 64 * IT_KB);
      tc::tma_load_2d(sm.q, &tmQ, &sm.qfull, 0, (b * a.Tq + qg * G) * 64);
      for (int it = 0; it < n0; ++it) {
        tc::mbar_arrive_expect_tx(&sm.full[it], IT_TILE_BYTES);
        tc::tma_load_2d(sm.k[it], &tmK, &sm.full[it], 0, (int)(b * a.n_max) + (t0 + it) * IT_ROWS);
      }
    }
    sm.issued0 = n0;
  }
  if (HIST) {
    for (int i = threadIdx.x; i < IT_FWIN; i += blockDim.x) sm.fwin[i] = 0u;
    if (threadIdx.x == 0) sm.fbase = IT_FNONE;
  }
  for (int i = threadIdx.x; i < G * 64; i += blockDim.x) {
    const int g = i / 64, j = i % 64;
    const int t = qg * G + g;
    float v = 0.f;
    if (t < a.Tq && j < a.H_I) {
      const size_t o = ((size_t)b * a.Tq + t) * a.H_I + j;
      v = a.w[o] * ((const float*)a.qI_scale)[o];
    }
    sm.wq[g][j] = v;
  }
  if (warp == 1) { tc::tmem_alloc(&sm.tmem_base, NCOLS); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  tc::griddep_launch_dependents();           // the selection kernel may start its prologue
  const uint32_t tmem = sm.tmem_base;
  const int t_begin = sm.t_begin, n_t = sm.t_end - sm.t_begin;

  if (warp == 0) {
    if (lane == 0 && n_t > 0) {
      int issued = sm.issued0;
      for (int it = issued; it < n_t; ++it) {
        const int st = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!tc::mbar_wait(&sm.empty[st], ph ^ 1)) { atomicExch(&sm.abort_flag, 1); break; }
        if (*(volatile int*)&sm.abort_flag) break;
        if (t_begin + it == sm.t_dep) tc::griddep_wait();
        tc::mbar_arrive_expect_tx(&sm.full[st], IT_TILE_BYTES);
        tc::tma_load_2d(sm.k[st], &tmK, &sm.full[st], 0, (int)(b * a.n_max) + (t_begin + it) * IT_ROWS);
        ++issued;
      }
      // drain: wait (bounded) for every copy this thread started before the CTA may exit
      tc::mbar_wait(&sm.qfull, 0);
      for (int it = (issued > STAGES ? issued - STAGES : 0); it < issued; ++it)
        tc::mbar_wait(&sm.full[it % STAGES], (it / STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t ID = tc::idesc(tc::FMT_E4M3, tc::FMT_E4M3, IT_ROWS, N);
      bool ok = tc::mbar_wait(&sm.qfull, 0);
      int last_issued = -1;
      const uint32_t q_addr = tc::smem_u32(sm.q);
      for (int it = 0; ok && it < n_t; ++it) {
        const int st = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        const int acc = it % NACC;
        const uint32_t aph = (it / NACC) & 1;
        if (!tc::mbar_wait(&sm.tempty[acc], aph ^ 1)) { ok = false; break; }
        if (!tc::mbar_wait(&sm.full[st], ph)) { ok = false; break; }
        if (*(volatile int*)&sm.abort_flag) { ok = false; break; }
        tc::fence_after_sync();
        const uint64_t kd = tc::desc_k_sw128(tc::smem_u32(sm.k[st])), qd = tc::desc_k_sw128(q_addr);
#pragma unroll
        for (int ks = 0; ks < IT_KB / 32; ++ks)
          tc::mma_f8f6f4(tmem + acc * N, kd + (uint64_t)((ks * 32) >> 4), qd + (uint64_t)((ks * 32) >> 4), ID,
                         ks > 0 ? 1u : 0u);
        tc::mma_commit(&sm.empty[st]);
        tc::mma_commit(&sm.tfull[acc]);
        last_issued = it;
      }
      if (!ok) {
        atomicExch(&sm.abort_flag, 1);
        // let the last issued MMA finish before the TMEM is released
        if (last_issued >= 0) tc::mbar_wait(&sm.tfull[last_issued % NACC], (last_issued / NACC) & 1);
      }
    }
  } else if (warp >= 4 && !STREAM) {
    // epilogue warpgroup e takes tiles e, e+2, ...; quarter q = warp % 4 reads TMEM lanes 32q..32q+31
    const int e = (warp - 4) >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const float* kscale = (const float*)a.kI_scale;
    float kmax = 0.f;
    const int t_dep = sm.t_dep;
    // the key scale of the group's next tile is loaded before waiting for the current accumulator
    auto load_scale = [&](int it) {
      const int s = (t_begin + it) * IT_ROWS + r;
      if (it < n_t && t_begin + it == t_dep) tc::griddep_wait();
      return (it < n_t && s < a.n_max) ? __ldcg(kscale + (size_t)b * a.n_max + s) : 0.f;
    };
    // IT_PF of the group's tiles ahead: a scale fetched one group tile ahead tied the tile
    // rate to the memory latency (about 0.5 us per tile whatever the ring depth)
    float skq[IT_PF];
#pragma unroll
    for (int d = 0; d < IT_PF; ++d) skq[d] = load_scale(e + 2 * d);
    // partial-slot mode: no global write before the preceding grid has finished (it may
    // still read this workspace)
    if (G == 1 && a.kpart > 0) tc::griddep_wait();
    KeyRange kr[G];
    for (int it = e; it < n_t; it += 2) {
      const int acc = it % NACC;
      const uint32_t aph = (it / NACC) & 1;
      const float sk = skq[0];
#pragma unroll
      for (int d = 0; d + 1 < IT_PF; ++d) skq[d] = skq[d + 1];
      skq[IT_PF - 1] = load_scale(it + 2 * IT_PF);
      bool ok = tc::mbar_wait(&sm.tfull[acc], aph) && !*(volatile int*)&sm.abort_flag;
      ok = __all_sync(0xffffffffu, ok);               // the TMEM loads below are warp-collective
      if (!ok) { atomicExch(&sm.abort_flag, 1); break; }
      tc::fence_after_sync();
      const int s = (t_begin + it) * IT_ROWS + r;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float val = head_sum(tmem + ((uint32_t)(quarter * 32) << 16) + acc * N + g * 64, sm.wq[g]);
        const bool valid = s < sm.n_elig[g];
        const float sc = a.score_bf16 ? round_bf16(val * sk) : val * sk;
        if (valid) {
          a.scores[(size_t)sm.row[g] * a.ld + s] = sc;
          kmax = fmaxf(kmax, sk);
          kr[g].add(sc);
        }
        if (HIST && a.hist) hist_count(sm.fwin, &sm.fbase, a, (size_t)sm.row[g], f32_order_key(sc), valid);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.tempty[acc]);
    }
    // |k8| <= 448 per element, so ||k_s|| <= sk * 448 * sqrt(d_I)
    kmax = warp_max(kmax);
    if (t_dep >= 0 || (G == 1 && a.kpart > 0)) {
      // the CTA's partials, reduced in shared memory and written to its own slots at the end
      const uint32_t mx = __reduce_max_sync(0xffffffffu, kr[0].mx), mn = __reduce_max_sync(0xffffffffu, kr[0].nmn);
      if (lane == 0) {
        atomicMax(&sm.part[0], mx);
        atomicMax(&sm.part[1], mn);
        if (kmax > 0.f) atomicMax(&sm.part[2], __float_as_uint(kmax * 448.f * 11.3137085f * 1.0001f));
      }
    } else {
#pragma unroll
      for (int g = 0; g < G; ++g) flush_key_range(a.keyrange, sm.row[g], kr[g]);
      if (lane == 0 && kmax > 0.f) atomicMax(a.knmax + b, __float_as_uint(kmax * 448.f * 11.3137085f * 1.0001f));
    }
  } else if (warp >= 4) {
    if constexpr (STREAM) {
      // the streaming selection (see StreamBuf): candidates instead of scores
      StreamBuf<G>& st = sm.st;
      const int e = (warp - 4) >> 2, quarter = warp & 3;
      const int r = quarter * 32 + lane, te = threadIdx.x - 128;
      const float* kscale = (const float*)a.kI_scale;
      if (te < G) { st.thr[te] = 0u; st.ovf[te] = 0u; st.U[te] = 0.f; }
      if (te == 0) st.ccnt = 0ull;
      if (te == 0) st.kmaxbits = 0u;
      ep_sync();
      // the sequence's key-norm bound (key_norm_max_kernel, before this kernel), and
      // U = sum_j |w_j| ||q_j|| per row (thread te: head te / 4, dims [32 (te % 4), +32))
      {
        if (te == 0) st.kmaxbits = __ldcg(a.knmax + b);
        const int j = te >> 2, q = te & 3;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const int t = qg * G + g;
          float ss = 0.f;
          if (t < a.Tq) {
            const uint4* qp = reinterpret_cast<const uint4*>((const uint8_t*)a.qI +
                                                             (((size_t)b * a.Tq + t) * 64 + j) * IT_KB + 32 * q);
            const uint4 v0 = __ldg(qp), v1 = __ldg(qp + 1);
            const uint32_t wd[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float x = e4m3_to_float((wd[i >> 2] >> (8 * (i & 3))) & 0xFFu);
              ss = fmaf(x, x, ss);
            }
          }
          ss += __shfl_xor_sync(0xffffffffu, ss, 1);
          ss += __shfl_xor_sync(0xffffffffu, ss, 2);
          float u = (q == 0 && t < a.Tq) ? fabsf(sm.wq[g][j]) * sqrtf(ss) : 0.f;   // wq = w * sq
          u = warp_sum(u);
          if (lane == 0) atomicAdd(&st.U[g], u);
        }
      }
      ep_sync();
      const float knmax = __uint_as_float(st.kmaxbits);
      float EU[G];
#pragma unroll
      for (int g = 0; g < G; ++g) EU[g] = (a.eps_dot + 1.9073486328125e-06f) * st.U[g] * knmax * 1.0002f;
      auto load_scale = [&](int it) {
        const int s = (t_begin + it) * IT_ROWS + r;
        return (it < n_t && s < a.n_max) ? __ldg(kscale + (size_t)b * a.n_max + s) : 0.f;
      };
      float sk_next = load_scale(e);
      bool alive = true;
      const int npairs = (n_t + 1) >> 1;
      // the epilogue threads meet every ST_PAIRS pairs of tiles; a list with less room than
      // those pairs can append is compacted there
      for (int ip = 0; ip < npairs; ++ip) {
        const int it = 2 * ip + e;
        if (it < n_t && alive) {
          const int acc = it % NACC;
          const uint32_t aph = (it / NACC) & 1;
          const float sk = sk_next;
          sk_next = load_scale(it + 2);
          bool ok = tc::mbar_wait(&sm.tfull[acc], aph) && !*(volatile int*)&sm.abort_flag;
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) {
            atomicExch(&sm.abort_flag, 1);
            alive = false;
          } else {
            tc::fence_after_sync();
            const int s = (t_begin + it) * IT_ROWS + r;
            // every row's entries first, then one shared-memory atomic per warp reserves the
            // slots of all rows at once (the four row counts are 16-bit fields of one word)
            uint32_t key[G], bt[G];
            unsigned long long inc = 0ull;
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float val = head_sum(tmem + ((uint32_t)(quarter * 32) << 16) + acc * N + g * 64, sm.wq[g]);
              key[g] = f32_order_key(val * sk);
              bt[g] = __ballot_sync(0xffffffffu, s < sm.n_elig[g] && key[g] >= st.thr[g]);
              inc |= (unsigned long long)__popc(bt[g]) << (16 * g);
            }
            if (inc) {
              unsigned long long old = 0ull;
              if (lane == 0) old = atomicAdd(&st.ccnt, inc);
              old = __shfl_sync(0xffffffffu, old, 0);
#pragma unroll
              for (int g = 0; g < G; ++g) {
                if (!((bt[g] >> lane) & 1u)) continue;
                const uint32_t off = (uint32_t)((old >> (16 * g)) & 0xFFFFull) + __popc(bt[g] & ((1u << lane) - 1u));
                if (off < (uint32_t)IDX_STREAM_CAP) {
                  st.ckey[g][off] = key[g];
                  st.cid[g][off] = s;
                } else {
                  st.ovf[g] = 1u;
                }
              }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.tempty[acc]);
          }
        }
        if (ip % ST_PAIRS == ST_PAIRS - 1 || ip == npairs - 1) {
          ep_sync();
          // (the decision reads shared memory after the barrier: every epilogue thread takes it alike)
          bool full = false;
#pragma unroll
          for (int g = 0; g < G; ++g) full = full || st_count(st, g) > (uint32_t)(IDX_STREAM_CAP - 2 * ST_PAIRS * IT_ROWS);
          if (full) ep_compact_all<G>(st, (uint32_t)a.k, EU);
        }
      }
      // the lists, and what the selection needs to finish them
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int t = qg * G + g;
        if (t >= a.Tq) continue;
        const size_t row = (size_t)b * a.Tq + t;
        const uint32_t n = min(st_count(st, g), (uint32_t)IDX_STREAM_CAP);
        for (uint32_t i = te; i < n; i += ST_T)
          a.stream_cand[row * IDX_STREAM_CAP + i] = make_uint2(st.ckey[g][i], (uint32_t)st.cid[g][i]);
        if (te == 0)
          a.stream_meta[row] = make_uint4(n | (st.ovf[g] ? 0x80000000u : 0u), st.thr[g], __float_as_uint(st.U[g]),
                                          __float_as_uint(knmax));
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (sm.abort_flag && threadIdx.x == 0) raise_err(a.err, CSA_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, NCOLS);
  }
  if (G == 1 && !STREAM && a.kpart > 0 && threadIdx.x == 0) {
    // a CTA that never reached the newest tile still waits once, so that this grid ends
    // after the append it may overlap (the kernels after it rely on that order)
    tc::griddep_wait();
    const size_t slot = (size_t)sm.row[0] * a.kpart + split;
    a.keyrange[2 * slot] = sm.part[0];
    a.keyrange[2 * slot + 1] = sm.part[1];
    a.knmax[slot] = sm.part[2];
  }
  if (HIST && a.hist) hist_flush(sm.fwin, sm.fbase, a, (size_t)sm.row[0]);
}

// ------------------------------------------------------------------------------------------
// MXFP4 operands ("FP4 с учётом квантования": the indexer's Q·K path in FP4).  Same
// structure as the E4M3 kernel, with the native block-scaled MMA: packed e2m1 key tiles
// (64-byte rows, 64-byte swizzle) and one ue8m0 scale per 32 elements applied inside the
// tensor core.  The scale factors go to TMEM with tcgen05.st: for M rows, row m's four
// scale bytes (k-blocks 0..3) sit in 32-bit column m/32 of lane m%32, replicated in all
// four lane quarters; warps 12..15 (one per quarter) write them for every tile.  Each tile
// is two MMAs of K = 64 (k-blocks 0-1, then 2-3: scale byte 0, then byte 2).
constexpr int MX_KB = 64;                 // bytes per packed key row (128 e2m1)
constexpr int MX_TILE_BYTES = IT_ROWS * MX_KB;

template <int STAGES>
struct MxSmem {
  alignas(1024) uint8_t q[64 * MX_KB];
  alignas(1024) uint8_t k[STAGES][MX_TILE_BYTES];
  uint32_t fwin[IT_FWIN];
  uint32_t fbase;
  alignas(8) uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t sfa_full[STAGES];
  uint64_t tfull[4];
  uint64_t tempty[4];
  uint64_t qfull;
  uint64_t sfb_ready;
  uint32_t tmem_base;
  int abort_flag;
  int t_begin, t_end;
  int issued0;          // tile loads issued before the setup barrier
  int n_elig;
  int t_dep;            // tile of the row's newest entry (partial-slot mode), else -1
  uint32_t part[3];     // the CTA's key range (max key, max ~key) and key-norm bound (partial-slot mode)
  alignas(16) float w[64];
};

// TMEM columns (256: two CTAs share an SM): two accumulators [0, 128), q scales at 128,
// key-scale ring at 136 + 4 * stage
constexpr uint32_t MX_SFB = 128, MX_SFA = 136, MX_COLS = 256;
constexpr int MX_NACC = 2;
constexpr int MX_THREADS = 512;   // warp 0 TMA, 1 MMA, 4..11 epilogue (two warpgroups), 12..15 scale writers

template <int STAGES>
__global__ void __launch_bounds__(MX_THREADS, 2)
indexer_mxf4_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ, IdxTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  using Sm = MxSmem<STAGES>;
  Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const IndexerArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, t = blockIdx.y, b = blockIdx.z;     // one query per CTA
  const int row = b * a.Tq + t;
  constexpr int N = 64;
  const uint32_t* ksc = (const uint32_t*)a.kI_scale;                  // 4 ue8m0 bytes per entry
  const uint32_t* qsc = (const uint32_t*)a.qI_scale;                  // 4 ue8m0 bytes per head

  if (threadIdx.x == 0) {
    tc::prefetch_tmap(&tmK);                 // descriptor fetches overlap the setup
    tc::prefetch_tmap(&tmQ);
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&sm.full[s], 1); tc::mbar_init(&sm.empty[s], 1); tc::mbar_init(&sm.sfa_full[s], 4);
    }
    for (int s = 0; s < MX_NACC; ++s) { tc::mbar_init(&sm.tfull[s], 1); tc::mbar_init(&sm.tempty[s], 4); }
    tc::mbar_init(&sm.qfull, 1);
    tc::mbar_init(&sm.sfb_ready, 4);
    tc::fence_mbar_init();
    sm.abort_flag = 0;
    const int ne = row_eligible(a, row);
    sm.n_elig = ne;
    const int t_lim = (ne + IT_ROWS - 1) / IT_ROWS;
    int t0 = split * p.tiles_per_split, t1 = t0 + p.tiles_per_split;
    if (t1 > t_lim) t1 = t_lim;
    sm.t_begin = t0;
    sm.t_end = t1 > t0 ? t1 : t0;
    // partial-slot mode: the tile of the row's newest entry waits for a preceding decode append
    sm.t_dep = (a.kpart > 0 && ne > 0) ? (ne - 1) / IT_ROWS : -1;
    sm.part[0] = sm.part[1] = sm.part[2] = 0u;
    // the query tile and the first key tiles go out before the setup barrier
    int n0 = sm.t_end - t0 < STAGES ? sm.t_end - t0 : STAGES;
    if (sm.t_dep >= t0 && sm.t_dep < t0 + n0) n0 = sm.t_dep - t0;
    if (sm.t_end > t0) {                      // (n0 may be 0: the first tile waits for the append)
      tc::mbar_arrive_expect_tx(&sm.qfull, 64 * MX_KB);
      tc::tma_load_2d(sm.q, &tmQ, &sm.qfull, 0, row * 64);
      for (int it = 0; it < n0; ++it) {
        tc::mbar_arrive_expect_tx(&sm.full[it], MX_TILE_BYTES);
        tc::tma_load_2d(sm.k[it], &tmK, &sm.full[it], 0, (int)(b * a.n_max) + (t0 + it) * IT_ROWS);
      }
    }
    sm.issued0 = n0;
  }
  if (threadIdx.x < 64) sm.w[threadIdx.x] = threadIdx.x < a.H_I ? a.w[(size_t)row * a.H_I + threadIdx.x] : 0.f;
  for (int i = threadIdx.x; i < IT_FWIN; i += blockDim.x) sm.fwin[i] = 0u;
  if (threadIdx.x == 0) sm.fbase = IT_FNONE;
  if (warp == 1) { tc::tmem_alloc(&sm.tmem_base, MX_COLS); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  tc::griddep_launch_dependents();           // the selection kernel may start its prologue
  const uint32_t tmem = sm.tmem_base;
  const int t_begin = sm.t_begin, n_t = sm.t_end - sm.t_begin;

  if (warp == 0) {
    if (lane == 0 && n_t > 0) {
      int issued = sm.issued0;
      for (int it = issued; it < n_t; ++it) {
        const int st = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!tc::mbar_wait(&sm.empty[st], ph ^ 1)) { atomicExch(&sm.abort_flag, 1); break; }
        if (*(volatile int*)&sm.abort_flag) break;
        if (t_begin + it == sm.t_dep) tc::griddep_wait();
        tc::mbar_arrive_expect_tx(&sm.full[st], MX_TILE_BYTES);
        tc::tma_load_2d(sm.k[st], &tmK, &sm.full[st], 0, (int)(b * a.n_max) + (t_begin + it) * IT_ROWS);
        ++issued;
      }
      tc::mbar_wait(&sm.qfull, 0);
      for (int it = (issued > STAGES ? issued - STAGES : 0); it < issued; ++it)
        tc::mbar_wait(&sm.full[it % STAGES], (it / STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t ID0 = tc::idesc_mxf4(IT_ROWS, N, 0, 0);
      constexpr uint32_t ID1 = tc::idesc_mxf4(IT_ROWS, N, 2, 2);
      bool ok = tc::mbar_wait(&sm.qfull, 0) && tc::mbar_wait(&sm.sfb_ready, 0);
      int last_issued = -1;
      const uint32_t q_addr = tc::smem_u32(sm.q);
      for (int it = 0; ok && it < n_t; ++it) {
        const int st = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        const int acc = it % MX_NACC;
        const uint32_t aph = (it / MX_NACC) & 1;
        if (!tc::mbar_wait(&sm.tempty[acc], aph ^ 1) || !tc::mbar_wait(&sm.full[st], ph) ||
            !tc::mbar_wait(&sm.sfa_full[st], ph) || *(volatile int*)&sm.abort_flag) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t k_addr = tc::smem_u32(sm.k[st]);
        const uint32_t sfa = tmem + MX_SFA + 4 * st, sfb = tmem + MX_SFB;
        tc::mma_mxf4(tmem + acc * N, tc::desc_k_sw64(k_addr), tc::desc_k_sw64(q_addr), ID0, sfa, sfb, 0u);
        tc::mma_mxf4(tmem + acc * N, tc::desc_k_sw64(k_addr + 32), tc::desc_k_sw64(q_addr + 32), ID1, sfa, sfb, 1u);
        tc::mma_commit(&sm.empty[st]);
        tc::mma_commit(&sm.tfull[acc]);
        last_issued = it;
      }
      if (!ok) {
        atomicExch(&sm.abort_flag, 1);
        if (last_issued >= 0) tc::mbar_wait(&sm.tfull[last_issued % MX_NACC], (last_issued / MX_NACC) & 1);
      }
    }
  } else if (warp >= 12) {
    // scale-factor writers, one warp per lane quarter (all quarters hold the same data)
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    if (n_t > 0) {
      // query scales: heads lane and lane + 32
      tc::tmem_st2(tmem + lane_base + MX_SFB, __ldg(qsc + (size_t)row * 64 + lane), __ldg(qsc + (size_t)row * 64 + 32 + lane));
      tc::tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.sfb_ready);
    }
    auto load4 = [&](int it, uint32_t* v) {
      const int s0 = (t_begin + it) * IT_ROWS + lane;
      if (it < n_t && t_begin + it == sm.t_dep) tc::griddep_wait();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int s = s0 + 32 * c;
        v[c] = (it < n_t && s < a.n_max) ? __ldcg(ksc + (size_t)b * a.n_max + s) : 0u;
      }
    };
    // the scales of IT_PF tiles ahead (one tile ahead tied the tile rate to the memory latency)
    uint32_t nxt[IT_PF][4];
#pragma unroll
    for (int d = 0; d < IT_PF; ++d) load4(d, nxt[d]);
    for (int it = 0; it < n_t; ++it) {
      const int st = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      uint32_t cur[4] = {nxt[0][0], nxt[0][1], nxt[0][2], nxt[0][3]};
#pragma unroll
      for (int d = 0; d + 1 < IT_PF; ++d)
#pragma unroll
        for (int c = 0; c < 4; ++c) nxt[d][c] = nxt[d + 1][c];
      load4(it + IT_PF, nxt[IT_PF - 1]);
      bool ok = tc::mbar_wait(&sm.empty[st], ph ^ 1) && !*(volatile int*)&sm.abort_flag;
      if (!__all_sync(0xffffffffu, ok)) { atomicExch(&sm.abort_flag, 1); break; }
      tc::fence_after_sync();
      tc::tmem_st4(tmem + lane_base + MX_SFA + 4 * st, cur[0], cur[1], cur[2], cur[3]);
      tc::tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.sfa_full[st]);
    }
  } else if (warp >= 4) {
    // epilogue warpgroup e takes tiles e, e+2, ...; quarter q = warp % 4 reads TMEM lanes 32q..32q+31
    const int e = (warp - 4) >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    float kb = 0.f;
    auto load_sc = [&](int it) {
      const int s = (t_begin + it) * IT_ROWS + r;
      if (it < n_t && t_begin + it == sm.t_dep) tc::griddep_wait();
      return (it < n_t && s < a.n_max) ? __ldcg(ksc + (size_t)b * a.n_max + s) : 0u;
    };
    uint32_t scq[IT_PF];
#pragma unroll
    for (int d = 0; d < IT_PF; ++d) scq[d] = load_sc(e + 2 * d);
    if (a.kpart > 0) tc::griddep_wait();                   // no global write before the preceding grid ends
    KeyRange kr;
    for (int it = e; it < n_t; it += 2) {
      const int acc = it % MX_NACC;
      const uint32_t aph = (it / MX_NACC) & 1;
      const int s = (t_begin + it) * IT_ROWS + r;
      const bool valid = s < sm.n_elig;
      const uint32_t sc = scq[0];
#pragma unroll
      for (int d = 0; d + 1 < IT_PF; ++d) scq[d] = scq[d + 1];
      scq[IT_PF - 1] = load_sc(it + 2 * IT_PF);
      // ||k_s|| <= 6 * sqrt(32 * sum_b scale_b^2): |e2m1| <= 6
      if (valid) {
        float ss = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) { const float f = ue8m0_to_float((sc >> (8 * q)) & 0xFFu); ss = fmaf(f, f, ss); }
        kb = fmaxf(kb, 6.f * sqrtf(32.f * ss));
      }
      bool ok = tc::mbar_wait(&sm.tfull[acc], aph) && !*(volatile int*)&sm.abort_flag;
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) { atomicExch(&sm.abort_flag, 1); break; }
      tc::fence_after_sync();
      float part[4] = {0.f, 0.f, 0.f, 0.f};
      // 16 heads at a time: their accumulator columns and weights (four 16-byte loads) in
      // flight together (the kernel runs at 64 registers)
#pragma unroll
      for (int q16 = 0; q16 < 4; ++q16) {
        uint32_t v[16];
        tc::tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + acc * N + q16 * 16, v);
        const float4* w4p = reinterpret_cast<const float4*>(&sm.w[q16 * 16]);
        float4 w4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) w4[u] = w4p[u];
        tc::tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          part[0] = fmaf(w4[u].x, fmaxf(__uint_as_float(v[4 * u]), 0.f), part[0]);
          part[1] = fmaf(w4[u].y, fmaxf(__uint_as_float(v[4 * u + 1]), 0.f), part[1]);
          part[2] = fmaf(w4[u].z, fmaxf(__uint_as_float(v[4 * u + 2]), 0.f), part[2]);
          part[3] = fmaf(w4[u].w, fmaxf(__uint_as_float(v[4 * u + 3]), 0.f), part[3]);
        }
      }
      const float val = a.score_bf16 ? round_bf16((part[0] + part[1]) + (part[2] + part[3]))
                                     : (part[0] + part[1]) + (part[2] + part[3]);
      if (valid) {
        a.scores[(size_t)row * a.ld + s] = val;
        kr.add(val);
      }
      if (a.hist) hist_count(sm.fwin, &sm.fbase, a, (size_t)row, f32_order_key(val), valid);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.tempty[acc]);
    }
    kb = warp_max(kb);
    if (a.kpart > 0) {
      const uint32_t mx = __reduce_max_sync(0xffffffffu, kr.mx), mn = __reduce_max_sync(0xffffffffu, kr.nmn);
      if (lane == 0) {
        atomicMax(&sm.part[0], mx);
        atomicMax(&sm.part[1], mn);
        if (kb > 0.f) atomicMax(&sm.part[2], __float_as_uint(kb * 1.0001f));
      }
    } else {
      flush_key_range(a.keyrange, row, kr);
      if (lane == 0 && kb > 0.f) atomicMax(a.knmax + b, __float_as_uint(kb * 1.0001f));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (sm.abort_flag && threadIdx.x == 0) raise_err(a.err, CSA_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, MX_COLS);
  }
  if (a.kpart > 0 && threadIdx.x == 0) {
    tc::griddep_wait();                                      // this grid ends after the append
    const size_t slot = (size_t)row * a.kpart + split;
    a.keyrange[2 * slot] = sm.part[0];
    a.keyrange[2 * slot + 1] = sm.part[1];
    a.knmax[slot] = sm.part[2];
  }
  if (a.hist) hist_flush(sm.fwin, sm.fbase, a, (size_t)row);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

// 2D byte tensor: rows of 128 bytes, box = box_rows x 128 bytes, 128-byte swizzle.
bool make_map_rows128(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2D byte tensor: rows of 64 bytes, box = box_rows x 64 bytes, 64-byte swizzle.
bool make_map_rows64(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {64, rows};
  cuuint64_t strides[1] = {64};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A launch with programmatic stream serialization (the kernel may start while the previous
// one in the stream runs; it waits for it with griddepcontrol.wait before dependent reads).
template <typename K, typename... Args>
cudaError_t launch_pdl(K kern, dim3 grid, int threads, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

cudaError_t launch_mxf4(const IndexerArgs& a, cudaStream_t st, bool* used, int* kpart_out) {
  constexpr int STAGES = 8;
  IdxTcParams p{};
  p.a = a;
  p.n_qg = a.Tq;
  p.tiles = (int)((a.n_max + IT_ROWS - 1) / IT_ROWS);
  const int64_t ctas = (int64_t)a.B * a.Tq;
  int splits = (int)(2 * num_sms() / ctas);         // one wave: two CTAs per SM
  if (a.kpart > 0 && splits > a.kpart) splits = a.kpart;   // the partial slots a row has
  if (splits > p.tiles) splits = p.tiles;
  if (splits < 1) splits = 1;
  p.tiles_per_split = (p.tiles + splits - 1) / splits;
  splits = (p.tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  CUtensorMap mk, mq;
  if (!make_map_rows64(&mk, a.kI, (uint64_t)a.B * a.n_max, IT_ROWS)) return cudaSuccess;
  if (!make_map_rows64(&mq, a.qI, (uint64_t)a.B * a.Tq * 64, 64)) return cudaSuccess;
  const size_t smem = sizeof(MxSmem<STAGES>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(indexer_mxf4_kernel<STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  if (a.kpart > 0) p.a.kpart = splits;
  dim3 grid(splits, a.Tq, a.B);
  note_launch();
  *used = true;
  if (a.kpart > 0) {
    *kpart_out = splits;
    return launch_pdl(indexer_mxf4_kernel<STAGES>, grid, MX_THREADS, smem, st, mk, mq, p);
  }
  indexer_mxf4_kernel<STAGES><<<grid, MX_THREADS, smem, st>>>(mk, mq, p);
  return cudaGetLastError();
}

template <int G, int STAGES, bool HIST, bool STREAM = false>
cudaError_t launch_g(const IndexerArgs& a, cudaStream_t st, bool* used, int* kpart_out) {
  IdxTcParams p{};
  p.a = a;
  if (G != 1) p.a.kpart = 0;
  p.n_qg = (a.Tq + G - 1) / G;
  p.tiles = (int)((a.n_max + IT_ROWS - 1) / IT_ROWS);
  // decode-like shapes: split the entry tiles so that the grid fills the SMs once
  // (two CTAs per SM for the one-query variant, one for the four-query variant); the
  // streaming selection keeps every entry of a row in one CTA
  const int64_t ctas = (int64_t)a.B * p.n_qg;
  const int64_t slots = G == 1 ? 2 * num_sms() : num_sms();
  int splits = STREAM ? 1 : (int)(slots / ctas);
  if (G == 1 && a.kpart > 0 && splits > a.kpart) splits = a.kpart;
  if (splits > p.tiles) splits = p.tiles;
  if (splits < 1) splits = 1;
  p.tiles_per_split = (p.tiles + splits - 1) / splits;
  splits = (p.tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  CUtensorMap mk, mq;
  if (!make_map_rows128(&mk, a.kI, (uint64_t)a.B * a.n_max, IT_ROWS)) return cudaSuccess;
  if (!make_map_rows128(&mq, a.qI, (uint64_t)a.B * a.Tq * 64, 64 * G)) return cudaSuccess;
  const size_t smem = sizeof(IdxSmem<G, STAGES, HIST, STREAM>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<G, STAGES, HIST, STREAM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (G == 1 && a.kpart > 0) p.a.kpart = splits;
  dim3 grid(splits, p.n_qg, a.B);
  note_launch();
  *used = true;
  if (G == 1 && a.kpart > 0) {
    *kpart_out = splits;
    return launch_pdl(indexer_tc_kernel<G, STAGES, HIST, STREAM>, grid, IT_THREADS, smem, st, mk, mq, p);
  }
  indexer_tc_kernel<G, STAGES, HIST, STREAM><<<grid, IT_THREADS, smem, st>>>(mk, mq, p);
  return cudaGetLastError();
}

}  // namespace

// The largest key norm of each sequence, for the streaming selection's error bound: one
// thread per entry forms sk * sqrt(sum of its squared E4M3 codes) (fp32, times 1.0001 for the
// rounding of 128 squares, the root and the product) and the warps' maxima go to knmax[b]
// (zeroed by the caller) as float bits.  Tighter than the scale-only bound sk * 448 * sqrt(d_I)
// by the ratio of a row's largest code to its root-mean-square code.
__global__ void __launch_bounds__(256) key_norm_max_kernel(const uint8_t* __restrict__ kI, const float* __restrict__ ks,
                                                           int64_t n_max, unsigned* knmax) {
  const int b = blockIdx.y;
  const int64_t s = (int64_t)blockIdx.x * 256 + threadIdx.x;
  float nrm = 0.f;
  if (s < n_max) {
    const uint4* p = reinterpret_cast<const uint4*>(kI + ((size_t)b * n_max + s) * IT_KB);
    float ss = 0.f;
#pragma unroll
    for (int v = 0; v < IT_KB / 16; ++v) {
      const uint4 x = __ldg(p + v);
      const uint32_t wd[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float c = e4m3_to_float((wd[i >> 2] >> (8 * (i & 3))) & 0xFFu);
        ss = fmaf(c, c, ss);
      }
    }
    nrm = __ldg(ks + (size_t)b * n_max + s) * sqrtf(ss) * 1.0001f;
  }
  nrm = warp_max(nrm);
  if ((threadIdx.x & 31) == 0 && nrm > 0.f) atomicMax(knmax + b, __float_as_uint(nrm));
}

cudaError_t launch_key_norm_max(const IndexerArgs& a, cudaStream_t st) {
  dim3 grid((unsigned)((a.n_max + 255) / 256), a.B);
  note_launch();
  key_norm_max_kernel<<<grid, 256, 0, st>>>((const uint8_t*)a.kI, (const float*)a.kI_scale, a.n_max, a.knmax);
  return cudaGetLastError();
}

bool indexer_stream_applies(const IndexerArgs& a) {
  if (a.ifmt != CSA_IFMT_E4M3 || a.H_I != 64 || a.d_I != 128 || a.Tq < 4 || a.score_bf16 || a.score_out) return false;
  if (a.k > IDX_STREAM_KMAX || ((uintptr_t)a.kI & 15) || ((uintptr_t)a.qI & 15)) return false;
  if ((int64_t)a.B * a.n_max > 0x7fffffffLL || (int64_t)a.B * a.Tq * 64 > 0x7fffffffLL) return false;
  // one CTA per four queries holds all of their entries: enough of them to fill the GPU
  return (int64_t)a.B * ((a.Tq + 3) / 4) >= num_sms();
}

// Tensor-core scores for E4M3 operands with 64 heads of width 128; other shapes
// return *used = false and run on the CUDA-core path.
cudaError_t launch_indexer_scores_tc(IndexerArgs& a, cudaStream_t st, bool* used) {
  *used = false;
  if (a.ifmt == CSA_IFMT_MXFP4 && a.H_I == 64 && a.d_I == 128) {
    if (((uintptr_t)a.kI & 15) || ((uintptr_t)a.qI & 15) || ((uintptr_t)a.kI_scale & 3) || ((uintptr_t)a.qI_scale & 3))
      return cudaSuccess;
    if ((int64_t)a.B * a.n_max > 0x7fffffffLL || (int64_t)a.B * a.Tq * 64 > 0x7fffffffLL) return cudaSuccess;
    // same bound as the E4M3 kernel
    a.eps_dot = 1.0f / 131072.0f;
    int kp = 0;
    const cudaError_t e = launch_mxf4(a, st, used, &kp);
    if (*used) a.kpart = kp;
    return e;
  }
  if (a.ifmt != CSA_IFMT_E4M3 || a.H_I != 64 || a.d_I != 128) return cudaSuccess;
  if (((uintptr_t)a.kI & 15) || ((uintptr_t)a.qI & 15)) return cudaSuccess;
  if ((int64_t)a.B * a.n_max > 0x7fffffffLL || (int64_t)a.B * a.Tq * 64 > 0x7fffffffLL) return cudaSuccess;
  // Bound on |fp32 MMA dot - exact| relative to ||q|| ||k||: the worst case of a 128-term
  // fp32 accumulation of exact products (128 * 2^-24 = 2^-17).  Measured on B200: <= 5e-9
  // relative to the bound's scale (test_indexer_fp32_score_error_within_band_bound).
  a.eps_dot = 1.0f / 131072.0f;
  // a.kpart on return: the partial slots per row the launch wrote (0: the shared atomic slots)
  int kp = 0;
  cudaError_t e;
  if (a.stream_cand) e = launch_g<4, 6, false, true>(a, st, used, &kp);
  else if (a.Tq >= 4) e = launch_g<4, 6, false>(a, st, used, &kp);
  // decode rows: the score histogram for the selection (one fewer ring stage makes room
  // for it at two CTAs per SM)
  else if (a.hist) e = launch_g<1, 5, true>(a, st, used, &kp);
  else e = launch_g<1, 6, false>(a, st, used, &kp);
  if (*used) a.kpart = kp;
  return e;
}

}  // namespace csa
