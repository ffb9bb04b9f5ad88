// Sparse / dense MQA attention over compressed entries + window + sink on the
// 5th-generation tensor cores (tcgen05, sm_100a), bf16 operands, fp32 accumulation.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA": CSA step 3 (every compressed entry is key and value for all
// query heads) and the HCA paragraph (dense attention over the compressed entries);
// "Технический отчёт DeepSeek-V4 — часть 1/2": the 576-wide MLA latent (keys use all
// 576 dims, values the first 512), the sliding-window branch and the attention sink.
//
// Shape covered: 128 heads, d_k = 576, d_v = 512.  A CTA handles one query token, one
// half of the heads (64, the MMA M dimension) and one split of the KV rows.  With M = 64
// an accumulator occupies lanes 0-15 of each 32-lane TMEM quarter, so O (64 heads x 512
// values: lanes 0-15, columns 0-511) and the double-buffered logits S (64 heads x 64 rows:
// lanes 16-31, columns 0-127) share the 512 TMEM columns.  Per tile of 64 KV rows:
//   1. a loader group brings the full 1152-byte rows into its own stage of a two-stage
//      ring, laid out in 128-byte swizzle atoms: rows that are one contiguous run of a
//      tensor come as nine 64-row TMA boxes, gathered rows as 16-byte cp.async (the
//      fastest way to gather scattered rows that was measured on B200);
//   2. one thread issues S = Q K^T (M=64, N=64, 36 steps of K=16) into TMEM;
//   3. softmax threads (one per head, TMEM lanes 16-31) run an online softmax with a
//      lazily raised running max and write P to shared memory as two bf16 parts,
//      P_hi = bf16(P) and P_lo = bf16(P - P_hi) (the second into the tile's RoPE atom,
//      which only S reads);
//   4. O += P_hi V + P_lo V (M=64, N=2x256, K=2x64; V is read MN-major from the same tile).
// At the end, threads of TMEM lanes 0-15 normalise O (one split), or write the split
// partial (o, m, l) to the workspace.  The CTAs of one query's head half form a
// thread-block cluster (at most 8 splits): after a cluster barrier each merges a slice
// of the heads from every split's partial, read back from L2 (distributed shared memory
// moved these partials at about 40 GB/s per SM, several times slower).  Without a
// cluster attn_combine merges them.  Every wait is bounded (CSA_DEVERR_TIMEOUT).
#include "attention.cuh"
#include "tc.cuh"

#include <cooperative_groups.h>
#include <cudaTypedefs.h>
#include <map>
#include <mutex>

namespace csa {

namespace {

constexpr int AT_ROWS = 64;              // KV rows per tile (N of QK^T, K of PV)
constexpr int AT_H = 128;                // heads per query
constexpr int AT_HC = 64;                // heads per CTA (MMA M)
constexpr int AT_ATOMS = 9;              // 576 dims = 9 atoms of 64 dims (128 bytes)
constexpr int AT_CHUNKS = AT_ATOMS * 8;  // 16-byte chunks per row
constexpr int AT_GROUP = 96;             // threads per loader group; group g fills stage g (15 warps in
                                         // all: 128 registers per thread, where 17 warps get 96)
constexpr int AT_SMW = 8;                // softmax warps: two warpgroups, one per half of the tile's columns
constexpr int AT_MMAW = AT_SMW;          // the MMA warp
constexpr int AT_LDW = AT_SMW + 1;       // first loader warp
constexpr int AT_THREADS = (AT_SMW + 1) * 32 + 2 * AT_GROUP;
constexpr float AT_RESCALE_THRESH = 8.0f;  // base-2 units: O is rescaled once the max grows 256-fold
constexpr int ATOM = AT_ROWS * 128;      // one 64-row x 128-byte swizzle atom
constexpr unsigned long long NO_RUN = ~0ull;

struct AtSmem {
  alignas(1024) uint8_t q[AT_ATOMS][AT_HC * 128];          // 72 KB
  alignas(1024) uint8_t kv[2][AT_ATOMS][ATOM];             // 144 KB
  alignas(1024) uint8_t p[AT_HC * 128];                    // P: 64 heads x 64 rows bf16
  const __nv_bfloat16* rowp[2][AT_ROWS];
  unsigned long long run_key[2][2];   // per stage and loader warp: (tensor << 32 | first row) or NO_RUN
  uint32_t vmask[2][2];  // per stage: bit j of word j / 32 set when row j of the tile is valid
  uint32_t k8mask[2][2]; // per stage: row j is an FP8 cache row, expanded to bf16 in place
  alignas(8) uint64_t full[2];
  uint64_t empty[2];
  uint64_t sfull[2];
  uint64_t sfree[2];
  uint64_t pfull;
  uint64_t pdone;
  uint64_t qfull;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int ld_stop[2];       // per loader group: 1 + the iteration at which it stops (0 = running)
  float lx[2][AT_HC];   // softmax row sums of each warpgroup's columns
};

static_assert(sizeof(AtSmem) + 1024 <= 232448, "shared memory budget of one CTA (227 KB)");

struct AtMaps {
  CUtensorMap q;       // [B*Tq*128 rows, 576] bf16, box 64 x 64
  CUtensorMap cache;   // [B*n_max rows, 576],   box 64 x 64
  CUtensorMap win;     // [window / raw rows, 576], box 64 x 64
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_zero16(uint32_t dst, const void* any) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, 0;" ::"r"(dst), "l"(any) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 2^x by the MUFU.EX2 unit (ex2.approx; relative error about 2^-22, far below the bf16
// rounding of P)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// byte offset of 16-byte chunk c of row j in a 128-byte-swizzled atom
__device__ __forceinline__ uint32_t sw128_off(int j, int c) { return (j >> 3) * 1024 + (j & 7) * 128 + ((c ^ (j & 7)) << 4); }

// ---- FP8 cache rows (656 bytes: 512 e4m3 codes of x / 2^e, 64 bf16 RoPE values, the byte
// e + 127).  The gather puts a row's 64 codes of atom a into the second half of the row's
// own 128-byte line of atom a (unswizzled), its RoPE values straight into atom 8, and its
// exponent byte into the first bytes of each of its eight code lines; a thread then expands
// one (row, atom) line in place: it reads the exponent and the line's codes before it writes
// the line, and no other thread touches the line, so no barrier is needed inside the
// expansion (512 lines per tile over the group's 96 threads).  codes * 2^e are exact bf16
// values: the MMA sees the stored row.
constexpr int KV8_ROW = 656;

__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t pair, float mult) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(pair));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * mult, f.y * mult);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ void kv8_expand(uint32_t kv0, const uint32_t* k8mask, int lg) {
  for (int u = lg; u < 8 * AT_ROWS; u += AT_GROUP) {
    const int j = u & (AT_ROWS - 1), a = u / AT_ROWS;
    if (!((k8mask[j >> 5] >> (j & 31)) & 1u)) continue;
    const uint32_t atom = kv0 + a * ATOM;
    const uint32_t line = atom + j * 128;
    uint32_t sc, cw[16];
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(sc) : "r"(line) : "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i)
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(cw[4 * i]), "=r"(cw[4 * i + 1]), "=r"(cw[4 * i + 2]), "=r"(cw[4 * i + 3])
                   : "r"(line + 64 + 16 * i) : "memory");
    const float mult = __uint_as_float((sc & 0xFFu) << 23);          // 2^e
#pragma unroll
    for (int i = 0; i < 8; ++i) {                                   // bf16 chunk i: codes 8i .. 8i+7
      const uint32_t w0 = cw[2 * i], w1 = cw[2 * i + 1];
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                   ::"r"(atom + sw128_off(j, i)), "r"(e4m3x2_to_bf16x2(w0 & 0xFFFFu, mult)),
                     "r"(e4m3x2_to_bf16x2(w0 >> 16, mult)), "r"(e4m3x2_to_bf16x2(w1 & 0xFFFFu, mult)),
                     "r"(e4m3x2_to_bf16x2(w1 >> 16, mult)) : "memory");
    }
  }
}

// TMEM: O at lane offset 0, columns [0, 512); S buffers at lane offset 16, columns 0 and 64.
constexpr uint32_t TM_S_LANE = 16u << 16, TM_COLS = 512;

// KV8: the cache rows are FP8 rows (a separate instance, so that the bf16 gather loop
// carries no test for them).
template <bool KV8>
__global__ void __launch_bounds__(AT_THREADS, 1)
attn_tc_kernel(const __grid_constant__ AtMaps maps, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AtSmem& sm = *reinterpret_cast<AtSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hh = blockIdx.x / a.splits, split = blockIdx.x - hh * a.splits;   // a cluster spans the splits
  const int row = blockIdx.y;                       // query row b*Tq + t
  const int64_t nrows = attn_virtual_rows(a);
  // The 64-row tiles of the query's virtual rows are dealt to the splits round-robin
  // (split s takes tiles s, s + S, ...), so the gathered top-k tiles and the contiguous
  // window tiles (one TMA copy each, several times faster) spread evenly over the splits.
  const int tiles_all = (int)((nrows + AT_ROWS - 1) / AT_ROWS);
  const int n_t = split < tiles_all ? (tiles_all - split + a.splits - 1) / a.splits : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&sm.full[s], AT_GROUP);
      tc::mbar_init(&sm.empty[s], 1);
      tc::mbar_init(&sm.sfull[s], 1);
      tc::mbar_init(&sm.sfree[s], AT_SMW);
      sm.ld_stop[s] = 0;
    }
    tc::mbar_init(&sm.pfull, AT_SMW);
    tc::mbar_init(&sm.pdone, 1);
    tc::mbar_init(&sm.qfull, 1);
    tc::mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == AT_MMAW) { tc::tmem_alloc(&sm.tmem_base, TM_COLS); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // The setup above overlaps the previous kernel's tail; every input may come from it,
  // except after a compression kernel that writes known rows (dep_entry0): then only the
  // loader of a tile holding them waits, just before loading it.
  const bool dep_rows_only = a.dep_entry0 != nullptr;
  const bool idx_late = a.idx_late != 0 && !dep_rows_only;
  if (!dep_rows_only && !idx_late) tc::griddep_wait();
  // the tile of a split's it-th step
  auto tile_of = [&](int it) { return split + (idx_late ? n_t - 1 - it : it) * a.splits; };
  tc::griddep_launch_dependents();
  const uint32_t tmem = sm.tmem_base;
  // The sink logit, needed only at the end, is loaded now: with one split by every softmax
  // thread for its head, else by threads [0, hp) for the heads they merge.
  const int merge_hp = (AT_HC + a.splits - 1) / a.splits, merge_h0 = split * merge_hp;
  float sink_pre = 0.f;
  if (a.splits == 1) {
    if (warp < AT_SMW) sink_pre = a.sink[hh * AT_HC + (warp & 3) * 16 + (lane & 15)];
  } else if ((int)threadIdx.x < merge_hp && merge_h0 + (int)threadIdx.x < AT_HC) {
    sink_pre = a.sink[hh * AT_HC + merge_h0 + threadIdx.x];
  }

  if (warp >= AT_LDW) {
    // ------------------------------------------------------------------ loader group g (96 threads)
    // Group g loads tiles g, g+2, ... into stage g; the two groups never wait on each other.
    const int g = (warp - AT_LDW) / (AT_GROUP / 32);
    const int lg = threadIdx.x - AT_LDW * 32 - g * AT_GROUP;
    if (g == 0 && lg == 0) {
      tc::prefetch_tmap(&maps.q);
      tc::prefetch_tmap(&maps.cache);
      tc::prefetch_tmap(&maps.win);
      tc::mbar_arrive_expect_tx(&sm.qfull, AT_ATOMS * AT_HC * 128);
      for (int at = 0; at < AT_ATOMS; ++at) tc::tma_load_2d(sm.q[at], &maps.q, &sm.qfull, 64 * at, row * AT_H + hh * AT_HC);
    }
    // row coordinates of the next tile, resolved into registers before its stage is free
    int which = -1, y = 0;
    bool idx_ready = !idx_late;
    auto coord = [&](int t) {
      which = -1;
      y = 0;
      if (lg < AT_ROWS) {
        const int64_t v = (int64_t)tile_of(t) * AT_ROWS + lg;
        if (!idx_ready && v < a.n_seg_a) {
          tc::griddep_wait();                         // the indices come from the preceding kernel
          idx_ready = true;
        }
        if (v < nrows) which = attn_row_coord(a, row, (int)v, &y);
      }
    };
    if (g < n_t) coord(g);
    // rows the preceding compression writes (dense decode): [dep0, dep1) of this sequence
    int64_t dep0 = 0, dep1 = 0;
    bool dep_done = !dep_rows_only;
    if (dep_rows_only) {
      dep0 = a.dep_entry0[row / a.Tq];
      dep1 = dep0 + a.dep_rows;
    }
    int issued = 0;                                   // tiles this group started (for the drain)
    for (int it = g, i = 0; it < n_t; it += 2, ++i) {
      const bool go = tc::mbar_wait(&sm.empty[g], (i & 1) ^ 1) && !*(volatile int*)&sm.abort_flag;
      if (!go) sm.ld_stop[g] = i + 1;      // the group leaves together at this iteration's barrier
      if (lg < AT_ROWS) {
        const bool r8 = KV8 && which == 0;                   // an FP8 cache row
        const __nv_bfloat16* base = which == 1 ? (const __nv_bfloat16*)a.win : (const __nv_bfloat16*)a.cache;
        sm.rowp[g][lg] = which < 0 ? nullptr
                         : r8 ? reinterpret_cast<const __nv_bfloat16*>((const uint8_t*)a.cache + (size_t)y * KV8_ROW)
                              : base + (size_t)y * 576;
        const uint32_t vb = __ballot_sync(0xffffffffu, which >= 0);
        const uint32_t kb = __ballot_sync(0xffffffffu, r8);
        if ((lg & 31) == 0) { sm.vmask[g][lg >> 5] = vb; sm.k8mask[g][lg >> 5] = kb; }
        // the tile is one contiguous run when all 64 rows are valid bf16 rows of one tensor
        // with y - lg the same everywhere; each warp checks its 32 rows
        const unsigned long long key =
            which >= 0 && !r8 ? ((unsigned long long)which << 32) | (unsigned)(y - lg) : NO_RUN;
        int same = 0;
        __match_all_sync(0xffffffffu, key, &same);
        if ((lg & 31) == 0) sm.run_key[g][lg >> 5] = same ? key : NO_RUN;
      }
      named_bar(1 + g, AT_GROUP);
      const int stop = *(volatile int*)&sm.ld_stop[g];
      if (stop != 0 && stop <= i + 1) break;
      if (!dep_done) {
        const int64_t r0 = (int64_t)tile_of(it) * AT_ROWS;   // the tile's cache rows
        if (r0 < dep1 && r0 + AT_ROWS > dep0) {
          tc::griddep_wait();                         // every thread of the group loads
          dep_done = true;
        }
      }
      const unsigned long long k0 = sm.run_key[g][0];
      const bool run = k0 != NO_RUN && k0 == sm.run_key[g][1];
      if (run) {
        if (lg == 0) {
          tc::mbar_arrive_expect_tx(&sm.full[g], AT_ATOMS * ATOM);
          const CUtensorMap* m = (k0 >> 32) == 1 ? &maps.win : &maps.cache;
          const int y0 = (int)(unsigned)(k0 & 0xffffffffu);
          for (int at = 0; at < AT_ATOMS; ++at) tc::tma_load_2d(sm.kv[g][at], m, &sm.full[g], 64 * at, y0);
        } else {
          tc::mbar_arrive(&sm.full[g]);
        }
      } else {
        const uint32_t kv0 = tc::smem_u32(sm.kv[g][0]);
        const bool any8 = KV8 && (sm.k8mask[g][0] | sm.k8mask[g][1]) != 0u;
        for (int p = lg; p < AT_ROWS * AT_CHUNKS; p += AT_GROUP) {
          const int j = p / AT_CHUNKS, c = p - j * AT_CHUNKS;
          const __nv_bfloat16* rp = sm.rowp[g][j];
          if (any8 && ((sm.k8mask[g][j >> 5] >> (j & 31)) & 1u)) {
            const uint8_t* rb = reinterpret_cast<const uint8_t*>(rp);
            if (c < 32) cp_async16(kv0 + (c >> 2) * ATOM + j * 128 + 64 + (c & 3) * 16, rb + c * 16);
            else if (c < 40) cp_async16(kv0 + 8 * ATOM + sw128_off(j, c - 32), rb + 512 + (c - 32) * 16);
            else if (c < 48) cp_async16(kv0 + (c - 40) * ATOM + j * 128, rb + 640);   // exponent, per line
            continue;
          }
          const uint32_t dst = kv0 + (c >> 3) * ATOM + sw128_off(j, c & 7);
          if (rp) cp_async16(dst, rp + c * 8);
          else cp_async_zero16(dst, a.cache);
        }
        cp_async_commit();
      }
      ++issued;
      // resolve the group's next tile while the copies are in flight
      if (it + 2 < n_t) coord(it + 2);
      if (!run) {
        cp_async_wait_all();
        if (KV8 && (sm.k8mask[g][0] | sm.k8mask[g][1]) != 0u) {   // the same for the whole group
          named_bar(1 + g, AT_GROUP);                         // every thread's copies have landed
          kv8_expand(tc::smem_u32(sm.kv[g][0]), sm.k8mask[g], lg);
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&sm.full[g]);
      }
    }
    cp_async_wait_all();
    // drain: no TMA write of this CTA may be in flight when the CTA exits
    if (lg == 0) {
      if (g == 0) tc::mbar_wait(&sm.qfull, 0);
      if (issued > 0) tc::mbar_wait(&sm.full[g], (issued - 1) & 1);
    }
  } else if (warp == AT_MMAW) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); lane 0 decides, one
    // elected lane (always the same) issues every MMA and commit.
    constexpr uint32_t ID_S = tc::idesc(tc::FMT_BF16, tc::FMT_BF16, AT_HC, AT_ROWS);
    constexpr uint32_t ID_O = tc::idesc(tc::FMT_BF16, tc::FMT_BF16, AT_HC, 256, 0, 1);
    bool ok = n_t == 0 || tc::mbar_wait(&sm.qfull, 0);
    ok = __all_sync(0xffffffffu, ok);
    // Descriptors are formed once; an MMA's operands are these plus compile-time offsets
    // (the 14-bit address field of a descriptor cannot carry: shared memory < 256 KB).
    const uint64_t q_d0 = tc::desc_k_sw128(tc::smem_u32(sm.q[0]));
    const uint64_t k_d0 = tc::desc_k_sw128(tc::smem_u32(sm.kv[0][0])), k_d1 = tc::desc_k_sw128(tc::smem_u32(sm.kv[1][0]));
    const uint64_t p_d0 = tc::desc_k_sw128(tc::smem_u32(sm.p));
    // P's low part of tile st sits in the stage's RoPE atom (free once S has read it)
    const uint64_t pl_d0 = tc::desc_k_sw128(tc::smem_u32(sm.kv[0][AT_ATOMS - 1])),
                   pl_d1 = tc::desc_k_sw128(tc::smem_u32(sm.kv[1][AT_ATOMS - 1]));
    const uint64_t v_d0 = tc::desc_mn_sw128(tc::smem_u32(sm.kv[0][0]), ATOM, 1024),
                   v_d1 = tc::desc_mn_sw128(tc::smem_u32(sm.kv[1][0]), ATOM, 1024);
    // Event-driven issue: S(ns) once its tile has landed and its S buffer is free, PV(np)
    // once P(np) is ready, in order; a PV never waits behind the next tile's load.
    int ns = 0, np = 0;
    uint64_t t_idle = tc::now_ns();
    uint32_t spins = 0;
    while (ok && np < n_t) {
      bool prog = false;
      if (ns < n_t) {
        const int st = ns & 1;
        const uint32_t ph = (ns >> 1) & 1;
        bool ready = false;
        if (lane == 0) ready = tc::mbar_try_wait(&sm.full[st], ph) && tc::mbar_try_wait(&sm.sfree[st], ph ^ 1);
        if (__shfl_sync(0xffffffffu, (int)ready, 0)) {
          tc::fence_after_sync();
          const uint32_t d = tmem + TM_S_LANE + st * AT_ROWS;
          const uint64_t kd = st ? k_d1 : k_d0;
          // S = Q K^T over 9 atoms x 4 k-steps of 16 (atoms of Q and of the tile are 8 KB apart)
          if (tc::elect_one()) tc::mma_f16_c<false>(d, q_d0, kd, ID_S);
#pragma unroll
          for (int i = 1; i < AT_ATOMS * 4; ++i) {
            const uint64_t off = (uint64_t)(((i >> 2) * ATOM + (i & 3) * 32) >> 4);
            if (tc::elect_one()) tc::mma_f16_c<true>(d, q_d0 + off, kd + off, ID_S);
          }
          if (tc::elect_one()) tc::mma_commit(&sm.sfull[st]);
          __syncwarp();
          ++ns;
          prog = true;
        }
      }
      if (np < ns) {
        bool ready = false;
        if (lane == 0) ready = tc::mbar_try_wait(&sm.pfull, np & 1);
        if (__shfl_sync(0xffffffffu, (int)ready, 0)) {
          // O += (P_hi + P_lo)_np V_np: value dims 0-255 (atoms 0-3) and 256-511 (atoms 4-7);
          // the two bf16 parts of P are two K ranges over the same V rows
          const int st = np & 1;
          tc::fence_after_sync();
          const uint64_t vd = st ? v_d1 : v_d0;
          const uint64_t pl = st ? pl_d1 : pl_d0;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint64_t vh = vd + (uint64_t)((4 * half * ATOM) >> 4);
            if (tc::elect_one()) {
              if (np > 0) tc::mma_f16_c<true>(tmem + 256 * half, p_d0, vh, ID_O);
              else tc::mma_f16_c<false>(tmem + 256 * half, p_d0, vh, ID_O);
            }
#pragma unroll
            for (int ks = 1; ks < AT_ROWS / 16; ++ks)
              if (tc::elect_one())
                tc::mma_f16_c<true>(tmem + 256 * half, p_d0 + (uint64_t)((ks * 32) >> 4), vh + (uint64_t)((ks * 16 * 128) >> 4), ID_O);
#pragma unroll
            for (int ks = 0; ks < AT_ROWS / 16; ++ks)
              if (tc::elect_one())
                tc::mma_f16_c<true>(tmem + 256 * half, pl + (uint64_t)((ks * 32) >> 4), vh + (uint64_t)((ks * 16 * 128) >> 4), ID_O);
          }
          if (tc::elect_one()) {
            tc::mma_commit(&sm.empty[st]);
            tc::mma_commit(&sm.pdone);
          }
          __syncwarp();
          ++np;
          prog = true;
        }
      }
      if (prog) {
        spins = 0;
      } else if ((++spins & 63u) == 0u) {
        bool stop = false;
        if (lane == 0) {
          const uint64_t t = tc::now_ns();
          if (spins == 64u) t_idle = t;
          stop = *(volatile int*)&sm.abort_flag || t - t_idle > tc::WAIT_LIMIT_NS;
        }
        if (__shfl_sync(0xffffffffu, (int)stop, 0)) ok = false;
      }
    }
    if (!ok && lane == 0) atomicExch(&sm.abort_flag, 1);
    // every MMA the elected lane issued has completed before the CTA frees TMEM
    if (tc::elect_one()) tc::mma_commit(&sm.drain);
    __syncwarp();
    tc::mbar_wait(&sm.drain, 0);
  } else {
    // ------------------------------------------------------------------ softmax + epilogue, warps 0-7
    // TMEM quarter q = warp % 4: lanes 16-31 hold the logits of heads 16q .. 16q+15 (S), lanes
    // 0-15 the output rows of the same heads (O).  Warpgroup wg = warp / 4 exponentiates the
    // tile's columns [32wg, 32wg+32): each S lane takes 16 of them and hands the other 16 to
    // its O lane (lane - 16), which is otherwise idle here.  Both warpgroups read all 64
    // logits, so they reach the same running max without exchanging it.
    const int wg = warp >> 2, quarter = warp & 3;
    const bool is_s = lane >= 16;
    const int hl = quarter * 16 + (lane & 15);      // head within the CTA
    const int h = hh * AT_HC + hl;                  // head within the query
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    // logits are kept in the base-2 domain (scale x log2 e): P = 2^(s - m); the running max
    // and the partial's m leave it (x ln 2) at the end
    const float scale2 = a.sm_scale * 1.4426950408889634f;
    float m_run = -INFINITY, l_run = 0.f;           // S lanes: running max, this warpgroup's row sum
    bool ok = true;
    for (int it = 0; it < n_t; ++it) {
      const int st = it & 1;
      const uint32_t ph = (it >> 1) & 1;
      bool w = tc::mbar_wait(&sm.sfull[st], ph) && tc::mbar_wait(&sm.full[st], ph);
      w = __all_sync(0xffffffffu, w && !*(volatile int*)&sm.abort_flag);
      if (!w) { ok = false; break; }
      tc::fence_after_sync();
      float s[AT_ROWS];
      {
        uint32_t v[AT_ROWS];
        tc::tmem_ld64(tmem + lane_base + st * AT_ROWS, v);     // lanes 16-31: S; lanes 0-15: unused
#pragma unroll
        for (int j = 0; j < AT_ROWS; ++j) s[j] = __uint_as_float(v[j]);
      }
      // scaled logits, invalid rows at -inf (a full tile skips the mask), and their max
      // over four independent chains
      const uint32_t vm0 = sm.vmask[st][0], vm1 = sm.vmask[st][1];
#pragma unroll
      for (int j = 0; j < AT_ROWS; ++j) s[j] *= scale2;
      if ((vm0 & vm1) != 0xffffffffu) {
#pragma unroll
        for (int j = 0; j < AT_ROWS; ++j)
          if (!((j < 32 ? vm0 >> j : vm1 >> (j - 32)) & 1u)) s[j] = -INFINITY;
      }
      float mq[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int j = 4; j < AT_ROWS; ++j) mq[j & 3] = fmaxf(mq[j & 3], s[j]);
      const float mt = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      // online softmax with a lazily raised running max (S lanes decide; O lanes follow)
      bool need_rescale = false;
      float alpha = 1.f;
      if (is_s && (mt > m_run + AT_RESCALE_THRESH || (m_run == -INFINITY && mt != -INFINITY))) {
        const float m_new = fmaxf(mt, m_run);
        alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new);
        need_rescale = (m_run != -INFINITY);
        m_run = m_new;
      }
      // the O row of head hl sits in lane (lane & 15) of the same warp
      const float alpha_o = __shfl_sync(0xffffffffu, alpha, (lane & 15) + 16);
      const float m_use = __shfl_sync(0xffffffffu, m_run, (lane & 15) + 16);
      const bool rescale_any = __any_sync(0xffffffffu, need_rescale);
      // this thread's 16 logits: S lanes keep the first 16 of the warpgroup's 32 columns,
      // O lanes receive the second 16 from their S lane
      float pv[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float a0 = wg ? s[32 + q] : s[q];
        const float a1 = wg ? s[48 + q] : s[16 + q];
        const float moved = __shfl_down_sync(0xffffffffu, a1, 16);
        pv[q] = is_s ? a0 : moved;
      }
      // P in registers first, as two bf16 parts (hi = P rounded, lo = the remainder rounded:
      // their sum carries P to about 2^-17 where bf16 alone gives 2^-9, which would use a
      // third of the output's error budget); the normaliser sums the parts the MMA sees.
      // This overlaps the previous PV, which owns the shared P tile and O until it completes.
      uint32_t w8[8], l8[8];
      float psum = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float p0 = (m_use == -INFINITY) ? 0.f : ex2_approx(pv[2 * u] - m_use);
        const float p1 = (m_use == -INFINITY) ? 0.f : ex2_approx(pv[2 * u + 1] - m_use);
        const __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
        const float h0 = __low2float(hb), h1 = __high2float(hb);
        const __nv_bfloat162 lb = __floats2bfloat162_rn(p0 - h0, p1 - h1);
        psum += (h0 + __low2float(lb)) + (h1 + __high2float(lb));
        w8[u] = *reinterpret_cast<const uint32_t*>(&hb);
        l8[u] = *reinterpret_cast<const uint32_t*>(&lb);
      }
      const float po = __shfl_up_sync(0xffffffffu, psum, 16);   // the O lane's part, to its S lane
      if (is_s) l_run = l_run * alpha + psum + po;
      if (it >= 1) {
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.pdone, (it - 1) & 1))) { ok = false; break; }
        tc::fence_after_sync();
      }
      if (rescale_any) {
        // A 32x32b store writes all 32 lanes, so the S lanes write back what they read.
        // That is harmless only while no MMA writes an S buffer: this tile's buffer is not
        // released yet, and the next tile's S must have landed.  Warpgroup wg rescales O
        // columns [256wg, 256wg+256).
        if (it + 1 < n_t) {
          if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.sfull[st ^ 1], ((it + 1) >> 1) & 1))) { ok = false; break; }
          tc::fence_after_sync();
        }
#pragma unroll 1
        for (int c = 4 * wg; c < 4 * wg + 4; ++c) {
          uint32_t v[64];
          tc::tmem_ld64(tmem + lane_base + c * 64, v);
          const float f = is_s ? 1.f : alpha_o;
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_st16(tmem + lane_base + c * 64 + q * 16, v + q * 16);
        }
        tc::tmem_st_wait();
      }
      {
        // P_hi into the P tile, P_lo into this stage's RoPE atom (S of this tile, its only
        // reader, has completed: sfull[st] was waited on above)
        const uint32_t pbase = tc::smem_u32(sm.p), lbase = tc::smem_u32(sm.kv[st][AT_ATOMS - 1]);
        const int c0 = 4 * wg + (is_s ? 0 : 2);     // 16-byte chunks (8 columns) of the P row
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pbase + sw128_off(hl, c0 + cc)), "r"(w8[4 * cc]),
                       "r"(w8[4 * cc + 1]), "r"(w8[4 * cc + 2]), "r"(w8[4 * cc + 3]) : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(lbase + sw128_off(hl, c0 + cc)), "r"(l8[4 * cc]),
                       "r"(l8[4 * cc + 1]), "r"(l8[4 * cc + 2]), "r"(l8[4 * cc + 3]) : "memory");
        }
      }
      // release this tile's S buffer and hand P (and a rescaled O) to the MMA thread
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&sm.sfree[st]);
        tc::mbar_arrive(&sm.pfull);
      }
    }
    // ---- epilogue: wait for the last PV, then normalise or write the split partial
    if (ok && n_t > 0) ok = __all_sync(0xffffffffu, tc::mbar_wait(&sm.pdone, (n_t - 1) & 1));
    if (!ok) atomicExch(&sm.abort_flag, 1);
    tc::fence_after_sync();
    const bool have_o = ok && n_t > 0;
    // the row sum is the two warpgroups' parts; the O lanes take m and l from the S lanes
    if (is_s) sm.lx[wg][hl] = l_run;
    named_bar(3, AT_SMW * 32);
    const float l_tot = sm.lx[0][hl] + sm.lx[1][hl];
    const float m_h = __shfl_sync(0xffffffffu, m_run, (lane & 15) + 16) * 0.6931471805599453f;
    const float l_h = __shfl_sync(0xffffffffu, l_tot, (lane & 15) + 16);
    if (a.splits == 1) {
      const float sk = sink_pre;
      const float mh = have_o ? m_h : -INFINITY;
      const float M = fmaxf(sk, mh);
      float den = 0.f, f = 0.f;
      if (M != -INFINITY) {
        f = (mh == -INFINITY) ? 0.f : __expf(mh - M);
        den = __expf(sk - M) + l_h * f;
      }
      const float inv = den > 0.f ? f / den : 0.f;
      __nv_bfloat16* o = (__nv_bfloat16*)a.out + ((size_t)row * AT_H + h) * 512;
#pragma unroll 1
      for (int c = 4 * wg; c < 4 * wg + 4; ++c) {
        uint32_t v[64];
        if (have_o) {
          tc::tmem_ld64(tmem + lane_base + c * 64, v);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = 0u;
        }
        if (!is_s) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float f8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) f8[j] = __uint_as_float(v[q * 8 + j]) * inv;
            Elem<__nv_bfloat16>::st_vec(o + c * 64 + q * 8, f8);
          }
        }
      }
      if (a.lse && !is_s && wg == 0) a.lse[(size_t)row * AT_H + h] = den > 0.f ? M + logf(den) : -INFINITY;
    } else {
      // Split partial, format 1 of attn_part_block: this thread's half row (256 values)
      // divided by l and by the power of two that puts its largest magnitude in [0.5, 1),
      // stored as fp16 at [512/8][128 heads][8], so that the 16 O lanes of a warp (16
      // consecutive heads) store 256 contiguous bytes.
      float* blk = a.part + ((size_t)row * a.splits + split) * attn_part_block(AT_H, 512);
      float amax = 0.f;
#pragma unroll 1
      for (int c = 4 * wg; c < 4 * wg + 4 && have_o; ++c) {
        uint32_t v[64];
        tc::tmem_ld64(tmem + lane_base + c * 64, v);
#pragma unroll
        for (int j = 0; j < 64; ++j) amax = fmaxf(amax, fabsf(__uint_as_float(v[j])));
      }
      const float inv_l = (have_o && l_h > 0.f) ? 1.f / l_h : 0.f;
      int e2 = 0;
      frexpf(amax * inv_l, &e2);
      const float f = inv_l * ldexpf(1.f, -e2);
      uint4* d16 = reinterpret_cast<uint4*>(blk) + h;
#pragma unroll 1
      for (int c = 4 * wg; c < 4 * wg + 4; ++c) {
        uint32_t v[64];
        if (have_o) {
          tc::tmem_ld64(tmem + lane_base + c * 64, v);
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = 0u;
        }
        if (!is_s) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint32_t w4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const __half2 hv = __floats2half2_rn(__uint_as_float(v[8 * q + 2 * u]) * f,
                                                   __uint_as_float(v[8 * q + 2 * u + 1]) * f);
              w4[u] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            d16[(size_t)(c * 8 + q) * AT_H] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      if (!is_s) {
        float* rec = blk + 512 * AT_H / 2 + 4 * (size_t)h;
        if (wg == 0) {
          rec[0] = have_o ? m_h : -INFINITY;
          rec[1] = have_o ? l_h : 0.f;
        }
        rec[2 + wg] = ldexpf(1.f, e2);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (sm.abort_flag && threadIdx.x == 0) raise_err(a.err, CSA_DEVERR_TIMEOUT);
  if (warp == AT_MMAW) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TM_COLS);
  }
  if (a.cluster_combine) {
    // Merge heads [h0, h1) of this head half from every split's partial.  The partials are
    // in the workspace (L2): a cluster barrier (release / acquire at cluster scope) orders
    // their stores before these loads, which bypass L1.
    namespace cg = cooperative_groups;
    cg::this_cluster().sync();
    const int S = a.splits;
    const int hp = merge_hp, h0 = merge_h0, h1 = min(AT_HC, h0 + hp);
    const size_t blkn = attn_part_block(AT_H, 512);
    const float* blk0 = a.part + (size_t)row * S * blkn;      // split p: blk0 + p * blkn
    const int hg0 = hh * AT_HC + h0;                          // first merged head within the query
    const int nh = h1 > h0 ? h1 - h0 : 1;                     // heads merged here (the last slice may be short)
    const int items = h1 > h0 ? nh * (512 / 8) : 0;           // (8-column piece, head), heads fastest
    float* wts = reinterpret_cast<float*>(&sm.q[0][0]);       // [head][half][split] merge weights (Q is idle)
    constexpr int OT_PITCH = 1040;                            // bytes per staged output row (16-byte multiple)
    uint8_t* ot = &sm.q[0][0] + 4096;                         // [head][512] bf16 output rows
    // the first item's partials are loaded before the weights are known
    uint4 x[8];
    int it = threadIdx.x;
    auto load_item = [&](int i) {
      const int hr = i % nh, c8 = i / nh;
#pragma unroll
      for (int p = 0; p < 8; ++p)
        x[p] = (p < S && i < items)
                   ? __ldcg(reinterpret_cast<const uint4*>(blk0 + p * blkn) + (size_t)c8 * AT_H + hg0 + hr)
                   : make_uint4(0u, 0u, 0u, 0u);
    };
    load_item(it);
    if ((int)threadIdx.x < h1 - h0) {
      const int hl = h0 + threadIdx.x;
      const float sk = sink_pre;
      float4 rc[8];
#pragma unroll
      for (int p = 0; p < 8; ++p)
        rc[p] = p < S ? __ldcg(reinterpret_cast<const float4*>(blk0 + p * blkn + 512 * AT_H / 2) + hh * AT_HC + hl)
                      : make_float4(-INFINITY, 0.f, 0.f, 0.f);
      float M = sk;
#pragma unroll
      for (int p = 0; p < 8; ++p) M = fmaxf(M, rc[p].x);
      float den = 0.f;
      if (M != -INFINITY) {
        den = __expf(sk - M);
#pragma unroll
        for (int p = 0; p < 8; ++p)
          if (rc[p].x != -INFINITY) den += rc[p].y * __expf(rc[p].x - M);
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const float w = (rc[p].x == -INFINITY || M == -INFINITY) ? 0.f : __expf(rc[p].x - M) * inv * rc[p].y;
        wts[(hl - h0) * 16 + p] = w * rc[p].z;
        wts[(hl - h0) * 16 + 8 + p] = w * rc[p].w;
      }
      if (a.lse) a.lse[(size_t)row * AT_H + hh * AT_HC + hl] = den > 0.f ? M + logf(den) : -INFINITY;
    }
    __syncthreads();
    for (; it < items; it += AT_THREADS) {
      const int hr = it % nh, c8 = it / nh;
      const float* wr = wts + hr * 16 + (c8 >= 32 ? 8 : 0);
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const float wgt = wr[p];
        const uint32_t u[4] = {x[p].x, x[p].y, x[p].z, x[p].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&u[q]));
          acc[2 * q] = fmaf(wgt, f2.x, acc[2 * q]);
          acc[2 * q + 1] = fmaf(wgt, f2.y, acc[2 * q + 1]);
        }
      }
      if (it + AT_THREADS < items) load_item(it + AT_THREADS);
      uint32_t pk[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        pk[q] = *reinterpret_cast<uint32_t*>(&b2);
      }
      *reinterpret_cast<uint4*>(ot + hr * OT_PITCH + c8 * 16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    __syncthreads();
    // the merged rows leave in 16-byte pieces, 1 KB contiguous per head
    for (int i = threadIdx.x; i < (h1 - h0) * 64; i += AT_THREADS) {
      const int hr = i >> 6, ch = i & 63;
      const uint4 v = *reinterpret_cast<const uint4*>(ot + hr * OT_PITCH + ch * 16);
      *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(a.out) + ((size_t)row * AT_H + hg0 + hr) * 1024 + ch * 16) = v;
    }
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_attn() {
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

// [rows, 576] bf16 latent rows (1152-byte pitch), box = 64 dims x 64 rows, 128-byte swizzle.
bool make_latent_map(CUtensorMap* m, const void* base, uint64_t rows) {
  auto enc = get_encode_attn();
  if (!enc || rows == 0) return false;
  cuuint64_t dims[2] = {576, rows};
  cuuint64_t strides[1] = {576 * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attention_tc(AttnArgs a, cudaStream_t st, bool* used, bool* combined) {
  *used = false;
  *combined = false;
  if (a.H != AT_H || a.dk != 576 || a.dv != 512) return cudaSuccess;
  if ((uintptr_t)a.q & 15 || (uintptr_t)a.cache & 15 || (a.win && ((uintptr_t)a.win & 15))) return cudaSuccess;
  if ((int64_t)a.B * a.n_max > 0x7fffffffLL || (int64_t)a.B * a.Tq * AT_H > 0x7fffffffLL) return cudaSuccess;
  AtMaps maps;
  const uint64_t win_rows = a.prefill ? (uint64_t)a.B * a.t_raw : (uint64_t)a.B * a.W;
  if (!make_latent_map(&maps.q, a.q, (uint64_t)a.B * a.Tq * AT_H)) return cudaSuccess;
  if (a.kv8) maps.cache = maps.q;                    // FP8 rows are gathered, never loaded by TMA
  else if (!make_latent_map(&maps.cache, a.cache, (uint64_t)a.B * a.n_max)) return cudaSuccess;
  if (a.win && win_rows > 0) {
    if (!make_latent_map(&maps.win, a.win, win_rows)) return cudaSuccess;
  } else {
    maps.win = maps.cache;                           // no row is ever resolved to the window tensor
  }
  const size_t smem = sizeof(AtSmem) + 1024;
  auto kern = a.kv8 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.splits, a.B * a.Tq);
  cfg.blockDim = dim3(AT_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait in the kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = a.splits;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  a.cluster_combine = 0;
  if (a.splits >= 2 && a.splits <= 8) {
    // merge the splits in a cluster when such clusters fit (checked once per split count)
    static std::mutex mu;
    static std::map<std::pair<int, int>, bool> fits;
    std::lock_guard<std::mutex> g(mu);
    const auto key = std::make_pair(a.splits, a.kv8);
    auto it = fits.find(key);
    if (it == fits.end()) {
      int n = 0;
      const bool ok = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0;
      cudaGetLastError();
      it = fits.emplace(key, ok).first;
    }
    a.cluster_combine = it->second ? 1 : 0;
  }
  cfg.numAttrs = a.cluster_combine ? 2 : 1;
  note_launch();
  e = cudaLaunchKernelEx(&cfg, kern, maps, a);
  *used = true;
  *combined = a.cluster_combine != 0;
  return e;
}

}  // namespace csa
