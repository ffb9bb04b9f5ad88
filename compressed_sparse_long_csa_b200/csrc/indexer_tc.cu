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

template <int G, int STAGES, bool HIST>
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
  alignas(16) float wq[G][64];
};

template <int G, int STAGES, bool HIST>
__global__ void __launch_bounds__(IT_THREADS, G == 1 ? 2 : 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ, IdxTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  using Sm = IdxSmem<G, STAGES, HIST>;
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
    // the query tile and the first key tiles go out before the setup barrier (a stage's
    // first use needs no release)
    const int n0 = sm.t_end - t0 < STAGES ? sm.t_end - t0 : STAGES;
    if (n0 > 0) {
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
  } else if (warp >= 4) {
    // epilogue warpgroup e takes tiles e, e+2, ...; quarter q = warp % 4 reads TMEM lanes 32q..32q+31
    const int e = (warp - 4) >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const float* kscale = (const float*)a.kI_scale;
    float kmax = 0.f;
    // the key scale of the group's next tile is loaded before waiting for the current accumulator
    auto load_scale = [&](int it) {
      const int s = (t_begin + it) * IT_ROWS + r;
      return (it < n_t && s < a.n_max) ? __ldg(kscale + (size_t)b * a.n_max + s) : 0.f;
    };
    float sk_next = load_scale(e);
    KeyRange kr[G];
    for (int it = e; it < n_t; it += 2) {
      const int acc = it % NACC;
      const uint32_t aph = (it / NACC) & 1;
      const float sk = sk_next;
      sk_next = load_scale(it + 2);
      bool ok = tc::mbar_wait(&sm.tfull[acc], aph) && !*(volatile int*)&sm.abort_flag;
      ok = __all_sync(0xffffffffu, ok);               // the TMEM loads below are warp-collective
      if (!ok) { atomicExch(&sm.abort_flag, 1); break; }
      tc::fence_after_sync();
      const int s = (t_begin + it) * IT_ROWS + r;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        // four partial sums over the heads (j mod 4)
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q16 = 0; q16 < 4; ++q16) {
          uint32_t v[16];
          const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + acc * N + g * 64 + q16 * 16;
          tc::tmem_ld16(ta, v);
          // the 16 weights as four 16-byte loads, in flight with the TMEM load (one load per
          // weight exposed its latency 64 times per tile)
          const float4* w4p = reinterpret_cast<const float4*>(&sm.wq[g][q16 * 16]);
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
        const float val = (part[0] + part[1]) + (part[2] + part[3]);
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
#pragma unroll
    for (int g = 0; g < G; ++g) flush_key_range(a.keyrange, sm.row[g], kr[g]);
    // |k8| <= 448 per element, so ||k_s|| <= sk * 448 * sqrt(d_I)
    kmax = warp_max(kmax);
    if (lane == 0 && kmax > 0.f) atomicMax(a.knmax + b, __float_as_uint(kmax * 448.f * 11.3137085f * 1.0001f));
  }
  tc::fence_before_sync();
  __syncthreads();
  if (sm.abort_flag && threadIdx.x == 0) raise_err(a.err, CSA_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, NCOLS);
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
    // the query tile and the first key tiles go out before the setup barrier
    const int n0 = sm.t_end - t0 < STAGES ? sm.t_end - t0 : STAGES;
    if (n0 > 0) {
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
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int s = s0 + 32 * c;
        v[c] = (it < n_t && s < a.n_max) ? __ldg(ksc + (size_t)b * a.n_max + s) : 0u;
      }
    };
    uint32_t nxt[4];
    load4(0, nxt);
    for (int it = 0; it < n_t; ++it) {
      const int st = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      uint32_t cur[4] = {nxt[0], nxt[1], nxt[2], nxt[3]};
      load4(it + 1, nxt);
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
      return (it < n_t && s < a.n_max) ? __ldg(ksc + (size_t)b * a.n_max + s) : 0u;
    };
    uint32_t sc_next = load_sc(e);
    KeyRange kr;
    for (int it = e; it < n_t; it += 2) {
      const int acc = it % MX_NACC;
      const uint32_t aph = (it / MX_NACC) & 1;
      const int s = (t_begin + it) * IT_ROWS + r;
      const bool valid = s < sm.n_elig;
      const uint32_t sc = sc_next;
      sc_next = load_sc(it + 2);
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
    flush_key_range(a.keyrange, row, kr);
    kb = warp_max(kb);
    if (lane == 0 && kb > 0.f) atomicMax(a.knmax + b, __float_as_uint(kb * 1.0001f));
  }
  tc::fence_before_sync();
  __syncthreads();
  if (sm.abort_flag && threadIdx.x == 0) raise_err(a.err, CSA_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, MX_COLS);
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

cudaError_t launch_mxf4(const IndexerArgs& a, cudaStream_t st, bool* used) {
  constexpr int STAGES = 8;
  IdxTcParams p{};
  p.a = a;
  p.n_qg = a.Tq;
  p.tiles = (int)((a.n_max + IT_ROWS - 1) / IT_ROWS);
  const int64_t ctas = (int64_t)a.B * a.Tq;
  int splits = (int)(2 * num_sms() / ctas);         // one wave: two CTAs per SM
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
  dim3 grid(splits, a.Tq, a.B);
  note_launch();
  indexer_mxf4_kernel<STAGES><<<grid, MX_THREADS, smem, st>>>(mk, mq, p);
  *used = true;
  return cudaGetLastError();
}

template <int G, int STAGES, bool HIST>
cudaError_t launch_g(const IndexerArgs& a, cudaStream_t st, bool* used) {
  IdxTcParams p{};
  p.a = a;
  p.n_qg = (a.Tq + G - 1) / G;
  p.tiles = (int)((a.n_max + IT_ROWS - 1) / IT_ROWS);
  // decode-like shapes: split the entry tiles so that the grid fills the SMs once
  // (two CTAs per SM for the one-query variant, one for the four-query variant)
  const int64_t ctas = (int64_t)a.B * p.n_qg;
  const int64_t slots = G == 1 ? 2 * num_sms() : num_sms();
  int splits = (int)(slots / ctas);
  if (splits > p.tiles) splits = p.tiles;
  if (splits < 1) splits = 1;
  p.tiles_per_split = (p.tiles + splits - 1) / splits;
  splits = (p.tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  CUtensorMap mk, mq;
  if (!make_map_rows128(&mk, a.kI, (uint64_t)a.B * a.n_max, IT_ROWS)) return cudaSuccess;
  if (!make_map_rows128(&mq, a.qI, (uint64_t)a.B * a.Tq * 64, 64 * G)) return cudaSuccess;
  const size_t smem = sizeof(IdxSmem<G, STAGES, HIST>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<G, STAGES, HIST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(splits, p.n_qg, a.B);
  note_launch();
  indexer_tc_kernel<G, STAGES, HIST><<<grid, IT_THREADS, smem, st>>>(mk, mq, p);
  *used = true;
  return cudaGetLastError();
}

}  // namespace

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
    return launch_mxf4(a, st, used);
  }
  if (a.ifmt != CSA_IFMT_E4M3 || a.H_I != 64 || a.d_I != 128) return cudaSuccess;
  if (((uintptr_t)a.kI & 15) || ((uintptr_t)a.qI & 15)) return cudaSuccess;
  if ((int64_t)a.B * a.n_max > 0x7fffffffLL || (int64_t)a.B * a.Tq * 64 > 0x7fffffffLL) return cudaSuccess;
  // Bound on |fp32 MMA dot - exact| relative to ||q|| ||k||: the worst case of a 128-term
  // fp32 accumulation of exact products (128 * 2^-24 = 2^-17).  Measured on B200: <= 5e-9
  // relative to the bound's scale (test_indexer_fp32_score_error_within_band_bound).
  a.eps_dot = 1.0f / 131072.0f;
  if (a.Tq >= 4) return launch_g<4, 6, false>(a, st, used);
  // decode rows: the score histogram for the selection (one fewer ring stage makes room
  // for it at two CTAs per SM)
  if (a.hist) return launch_g<1, 5, true>(a, st, used);
  return launch_g<1, 6, false>(a, st, used);
}

}  // namespace csa
