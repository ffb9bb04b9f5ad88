// Sparse / dense MQA attention over compressed entries + window + sink on the
// 5th-generation tensor cores (tcgen05, sm_100a), bf16 operands, fp32 accumulation.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA": CSA step 3 (every compressed entry is key and value for all
// query heads) and the HCA paragraph (dense attention over the compressed entries);
// "Технический отчёт DeepSeek-V4 — часть 1/2": the 576-wide MLA latent (keys use all
// 576 dims, values the first 512), the sliding-window branch and the attention sink.
//
// Shape covered: 128 heads, d_k = 576, d_v = 512.  The 128 heads are the MMA M
// dimension.  One query token and one KV split are handled by a cluster of two CTAs
// that split the latent dims: CTA r holds value dims [256r, 256r+256) and RoPE dims
// [512+32r, 512+32r+32) of q and of every KV row (288 dims, 576 bytes), so each KV
// byte is read once.  Per tile of 64 KV rows:
//   1. loader warps gather the rows' 576-byte halves with 16-byte cp.async into a
//      two-stage ring laid out for the UMMA descriptors (128-byte swizzle for the 256
//      value dims, 64-byte swizzle for the 32 RoPE dims);
//   2. one thread issues S_r = Q_r K_r^T (M=128, N=64, 18 MMAs of K=16) into a
//      double-buffered TMEM accumulator;
//   3. softmax warps (thread = head) read S_r from TMEM, send it to the peer CTA's
//      shared memory, receive the peer's half, and add them (same order of operands
//      in both CTAs, so both see bitwise identical logits), then run an online softmax
//      with a lazily updated running max, write P (bf16) to shared memory;
//   4. O_r += P V_r (M=128, N=256, K=64, V read MN-major from the same tile).
// O_r lives in TMEM (256 columns); at the end it is normalised (one split) or written
// as a split partial (m, l, o) for attn_combine.
//
// Every wait is bounded (CSA_DEVERR_TIMEOUT on expiry) and the CTA pair meets at a
// cluster barrier before exit so no CTA leaves while its peer may still touch its
// shared memory.  No TMA multicast is used.
#include "attention.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int AT_ROWS = 64;              // KV rows per tile (N of QK^T, K of PV)
constexpr int AT_H = 128;                // heads (M)
constexpr int AT_VD = 256;               // value dims per CTA
constexpr int AT_RD = 32;                // RoPE dims per CTA
constexpr int AT_CHUNKS = (AT_VD + AT_RD) * 2 / 16;   // 36 16-byte chunks per half row
constexpr int AT_STAGES = 2;
constexpr int AT_LOADER_THREADS = 96;    // warps 0, 2, 3
constexpr float AT_RESCALE_THRESH = 8.0f;

struct AtSmem {
  // Q half: 4 value atoms [128 rows x 128 B] (SW128) + RoPE part [128 rows x 64 B] (SW64)
  alignas(1024) uint8_t qv[4][AT_H * 128];
  alignas(1024) uint8_t qr[AT_H * 64];
  // KV ring: per stage 4 value atoms [64 x 128 B] + RoPE [64 x 64 B]
  alignas(1024) uint8_t kv[AT_STAGES][4][AT_ROWS * 128];
  alignas(1024) uint8_t kr[AT_STAGES][AT_ROWS * 64];
  // P (bf16, 128 heads x 64 rows, SW128 K-major)
  alignas(1024) uint8_t p[AT_H * 128];
  // partial logits received from the peer, double buffered
  alignas(16) float x[2][AT_H][AT_ROWS];
  uint8_t valid[AT_STAGES][AT_ROWS];
  const __nv_bfloat16* rowp[2][AT_ROWS];   // resolved row pointers of the current / next tile
  alignas(8) uint64_t full[AT_STAGES];
  uint64_t empty[AT_STAGES];
  uint64_t sfull[2];
  uint64_t sfree[2];
  uint64_t xfull[2];
  uint64_t xempty[2];
  uint64_t pfull;
  uint64_t pdone;
  uint64_t qready;
  uint32_t tmem_base;
  int abort_flag;
  int ld_stop;          // written only by loader threads, read by them after a named barrier
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_peer(uint32_t local_addr, uint32_t peer) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(peer));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, 10000;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(tc::smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t limit = 200000u) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait_cluster(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
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
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// SW64 K-major descriptor: 64-byte rows, 8-row groups 512 bytes apart.
__device__ __forceinline__ uint64_t desc_k_sw64(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(512u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)4u << 61;                      // SWIZZLE_64B
  return d;
}

// byte offset of 16-byte chunk c of row j in a 128-byte-swizzled atom / 64-byte-swizzled block
__device__ __forceinline__ uint32_t sw128_off(int j, int c) { return (j >> 3) * 1024 + (j & 7) * 128 + ((c ^ (j & 7)) << 4); }
__device__ __forceinline__ uint32_t sw64_off(int j, int c) { return (j >> 3) * 512 + (j & 7) * 64 + ((c ^ ((j >> 1) & 3)) << 4); }

static_assert(sizeof(AtSmem) + 1024 <= 232448, "shared memory budget of one CTA (227 KB)");

// TMEM column map: O at [0, 256), S buffers at 256 and 320.
constexpr uint32_t TM_O = 0, TM_S = 256, TM_COLS = 512;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(256, 1)
attn_tc_kernel(AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AtSmem& sm = *reinterpret_cast<AtSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const int split = blockIdx.x >> 1;
  const int row = blockIdx.y;                       // query row b*Tq + t
  const int64_t nrows = attn_virtual_rows(a);
  const int64_t v0 = (int64_t)split * a.rows_per_split;
  int64_t v1 = v0 + a.rows_per_split;
  if (v1 > nrows) v1 = nrows;
  const int n_t = v1 > v0 ? (int)((v1 - v0 + AT_ROWS - 1) / AT_ROWS) : 0;
  const __nv_bfloat16* qrow = (const __nv_bfloat16*)a.q + (size_t)row * AT_H * 576;

  if (threadIdx.x == 0) {
    for (int s = 0; s < AT_STAGES; ++s) {
      tc::mbar_init(&sm.full[s], AT_LOADER_THREADS);
      tc::mbar_init(&sm.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&sm.sfull[s], 1);
      tc::mbar_init(&sm.sfree[s], 4);
      tc::mbar_init(&sm.xfull[s], AT_H);          // 128 remote arrivals from the peer's softmax threads
      tc::mbar_init(&sm.xempty[s], AT_H);
    }
    tc::mbar_init(&sm.pfull, AT_H);
    tc::mbar_init(&sm.pdone, 1);
    tc::mbar_init(&sm.qready, AT_LOADER_THREADS);
    sm.abort_flag = 0;
    sm.ld_stop = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) { tc::tmem_alloc(&sm.tmem_base, TM_COLS); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  cluster_sync_all();                                // peer barriers initialised before any remote arrive
  tc::fence_after_sync();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0 || warp == 2 || warp == 3) {
    // ------------------------------------------------------------------ loaders
    const int lt = warp == 0 ? lane : (warp - 1) * 32 + lane;       // 0..95
    // Q half (128 heads x 36 chunks)
    for (int p = lt; p < AT_H * AT_CHUNKS; p += AT_LOADER_THREADS) {
      const int h = p / AT_CHUNKS, c = p % AT_CHUNKS;
      uint32_t dst;
      const __nv_bfloat16* src;
      if (c < 32) {
        dst = tc::smem_u32(sm.qv[c >> 3]) + sw128_off(h, c & 7);
        src = qrow + (size_t)h * 576 + AT_VD * rank + c * 8;
      } else {
        dst = tc::smem_u32(sm.qr) + sw64_off(h, c - 32);
        src = qrow + (size_t)h * 576 + 512 + AT_RD * rank + (c - 32) * 8;
      }
      cp_async16(dst, src, true);
    }
    cp_async_commit();
    cp_async_wait<0>();
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&sm.qready);
    bool ok = true;
    // row pointers are resolved once per tile (one idx lookup per row, in parallel) and
    // the next tile's are resolved while the current tile's copies are in flight
    auto resolve = [&](int t, int buf) {
      if (lt < AT_ROWS) {
        const int64_t v = v0 + (int64_t)t * AT_ROWS + lt;
        sm.rowp[buf][lt] = (v < v1) ? attn_row_ptr<__nv_bfloat16>(a, row, (int)v) : nullptr;
      }
    };
    if (n_t > 0) resolve(0, 0);
    named_bar(1, AT_LOADER_THREADS);
    for (int it = 0; it < n_t; ++it) {
      const int st = it % AT_STAGES;
      const uint32_t ph = (it / AT_STAGES) & 1;
      // all loader threads take the same decision: ld_stop is written only by loader
      // threads before the barrier and read after it
      const bool go = tc::mbar_wait(&sm.empty[st], ph ^ 1) && !*(volatile int*)&sm.abort_flag;
      if (!go) sm.ld_stop = 1;
      named_bar(1, AT_LOADER_THREADS);
      if (*(volatile int*)&sm.ld_stop) { ok = false; break; }
      for (int p = lt; p < AT_ROWS * AT_CHUNKS; p += AT_LOADER_THREADS) {
        const int j = p / AT_CHUNKS, c = p % AT_CHUNKS;
        const __nv_bfloat16* rp = sm.rowp[it & 1][j];
        if (c == 0) sm.valid[st][j] = rp != nullptr;
        uint32_t dst;
        const __nv_bfloat16* src;
        if (c < 32) {
          dst = tc::smem_u32(sm.kv[st][c >> 3]) + sw128_off(j, c & 7);
          src = rp ? rp + AT_VD * rank + c * 8 : qrow;
        } else {
          dst = tc::smem_u32(sm.kr[st]) + sw64_off(j, c - 32);
          src = rp ? rp + 512 + AT_RD * rank + (c - 32) * 8 : qrow;
        }
        cp_async16(dst, src, rp != nullptr);
      }
      cp_async_commit();
      if (it + 1 < n_t) resolve(it + 1, (it + 1) & 1);
      cp_async_wait<0>();
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&sm.full[st]);
      named_bar(1, AT_LOADER_THREADS);               // next pointers visible; current buffer free
    }
    if (!ok) atomicExch(&sm.abort_flag, 1);
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t ID_S = tc::idesc(tc::FMT_BF16, tc::FMT_BF16, AT_H, AT_ROWS);
      constexpr uint32_t ID_O = tc::idesc(tc::FMT_BF16, tc::FMT_BF16, AT_H, AT_VD, 0, 1);
      bool ok = tc::mbar_wait(&sm.qready, 0);
      int last_commit = -1;
      for (int it = 0; ok && it <= n_t; ++it) {
        if (it < n_t) {
          const int st = it % AT_STAGES;
          const uint32_t ph = (it / AT_STAGES) & 1;
          const int sb = it & 1;
          const uint32_t sph = (it >> 1) & 1;
          if (!tc::mbar_wait(&sm.full[st], ph) || !tc::mbar_wait(&sm.sfree[sb], sph ^ 1) ||
              *(volatile int*)&sm.abort_flag) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t d = tmem + TM_S + sb * AT_ROWS;
          int step = 0;
#pragma unroll
          for (int at = 0; at < 4; ++at) {
            const uint32_t qa = tc::smem_u32(sm.qv[at]), ka = tc::smem_u32(sm.kv[st][at]);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks, ++step)
              tc::mma_f16(d, tc::desc_k_sw128(qa + ks * 32), tc::desc_k_sw128(ka + ks * 32), ID_S, step > 0);
          }
          const uint32_t qa = tc::smem_u32(sm.qr), ka = tc::smem_u32(sm.kr[st]);
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) tc::mma_f16(d, desc_k_sw64(qa + ks * 32), desc_k_sw64(ka + ks * 32), ID_S, 1u);
          tc::mma_commit(&sm.sfull[sb]);
        }
        if (it >= 1) {
          // O += P_{it-1} V_{it-1}
          const int pt = it - 1;
          const int st = pt % AT_STAGES;
          if (!tc::mbar_wait(&sm.pfull, pt & 1) || *(volatile int*)&sm.abort_flag) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t pa = tc::smem_u32(sm.p), va = tc::smem_u32(sm.kv[st][0]);
#pragma unroll
          for (int ks = 0; ks < AT_ROWS / 16; ++ks)
            tc::mma_f16(tmem + TM_O, tc::desc_k_sw128(pa + ks * 32),
                        tc::desc_mn_sw128(va + ks * 16 * 128, AT_ROWS * 128, 1024), ID_O, (pt > 0 || ks > 0) ? 1u : 0u);
          tc::mma_commit(&sm.empty[st]);
          tc::mma_commit(&sm.pdone);
          last_commit = pt;
        }
      }
      if (!ok) {
        atomicExch(&sm.abort_flag, 1);
        if (last_commit >= 0) tc::mbar_wait(&sm.pdone, last_commit & 1);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax (thread = head)
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float scale = a.sm_scale;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    const uint32_t peer_x0 = map_peer(tc::smem_u32(&sm.x[0][h][0]), peer);
    const uint32_t peer_x1 = map_peer(tc::smem_u32(&sm.x[1][h][0]), peer);
    const uint32_t peer_xfull0 = map_peer(tc::smem_u32(&sm.xfull[0]), peer);
    const uint32_t peer_xfull1 = map_peer(tc::smem_u32(&sm.xfull[1]), peer);
    const uint32_t peer_xempty0 = map_peer(tc::smem_u32(&sm.xempty[0]), peer);
    const uint32_t peer_xempty1 = map_peer(tc::smem_u32(&sm.xempty[1]), peer);
    for (int it = 0; it < n_t; ++it) {
      const int sb = it & 1;
      const uint32_t sph = (it >> 1) & 1;
      const int st = it % AT_STAGES;
      bool w = tc::mbar_wait(&sm.sfull[sb], sph) && tc::mbar_wait(&sm.full[st], (it / AT_STAGES) & 1);
      w = __all_sync(0xffffffffu, w && !*(volatile int*)&sm.abort_flag);
      if (!w) { ok = false; break; }
      tc::fence_after_sync();
      float s[AT_ROWS];
      {
        uint32_t v[AT_ROWS];
        tc::tmem_ld64(tmem + lane_base + TM_S + sb * AT_ROWS, v);
#pragma unroll
        for (int j = 0; j < AT_ROWS; ++j) s[j] = __uint_as_float(v[j]);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.sfree[sb]);
      // send the partial logits to the peer (its buffer sb must have been drained)
      if (it >= 2) {
        if (!mbar_wait_cluster(&sm.xempty[sb], ((it - 2) >> 1) & 1)) { ok = false; }
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const uint32_t px = sb ? peer_x1 : peer_x0;
#pragma unroll
      for (int j = 0; j < AT_ROWS; j += 4) st_cluster_v4(px + j * 4, s[j], s[j + 1], s[j + 2], s[j + 3]);
      mbar_arrive_remote(sb ? peer_xfull1 : peer_xfull0);
      // receive the peer's partial logits
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(&sm.xfull[sb], sph))) { ok = false; break; }
      float mt = -INFINITY;
      const float4* mine = reinterpret_cast<const float4*>(&sm.x[sb][h][0]);
#pragma unroll
      for (int j4 = 0; j4 < AT_ROWS / 4; ++j4) {
        const float4 o = mine[j4];
        const float po[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j4 * 4 + u;
          // rank 0 adds (own + peer) = (S0 + S1); rank 1 adds (peer + own) = (S0 + S1)
          const float tot = rank == 0 ? (s[j] + po[u]) : (po[u] + s[j]);
          const float l = sm.valid[st][j] ? tot * scale : -INFINITY;
          s[j] = l;
          mt = fmaxf(mt, l);
        }
      }
      mbar_arrive_remote(sb ? peer_xempty1 : peer_xempty0);
      // online softmax with a lazily raised running max (identical decisions in both CTAs)
      bool need_rescale = false;
      float alpha = 1.f;
      if (mt > m_run + AT_RESCALE_THRESH || (m_run == -INFINITY && mt != -INFINITY)) {
        const float m_new = fmaxf(mt, m_run);
        alpha = (m_run == -INFINITY) ? 0.f : __expf(m_run - m_new);
        need_rescale = (m_run != -INFINITY);
        m_run = m_new;
      }
      // P buffer and O are owned by the previous PV until it completes
      if (it >= 1) {
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&sm.pdone, (it - 1) & 1))) { ok = false; break; }
        tc::fence_after_sync();
      }
      if (__any_sync(0xffffffffu, need_rescale)) {
        // O *= alpha for this row (alpha == 1 for lanes that did not need it)
#pragma unroll 1
        for (int c = 0; c < AT_VD / 64; ++c) {
          uint32_t v[64];
          tc::tmem_ld64(tmem + lane_base + TM_O + c * 64, v);
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha);
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_st16(tmem + lane_base + TM_O + c * 64 + q * 16, v + q * 16);
        }
        tmem_st_wait();
      }
      l_run *= alpha;
      float psum = 0.f;
      const uint32_t pbase = tc::smem_u32(sm.p);
#pragma unroll
      for (int c = 0; c < AT_ROWS / 8; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float p0 = (m_run == -INFINITY) ? 0.f : __expf(s[c * 8 + 2 * u] - m_run);
          const float p1 = (m_run == -INFINITY) ? 0.f : __expf(s[c * 8 + 2 * u + 1] - m_run);
          __nv_bfloat162 hb = __floats2bfloat162_rn(p0, p1);
          psum += __low2float(hb) + __high2float(hb);     // the normaliser uses the rounded P
          w4[u] = *reinterpret_cast<uint32_t*>(&hb);
        }
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pbase + sw128_off(h, c)), "r"(w4[0]),
                     "r"(w4[1]), "r"(w4[2]), "r"(w4[3]) : "memory");
      }
      l_run += psum;
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.pfull);
    }
    // ---- epilogue: wait for the last PV, then normalise or write the split partial
    if (ok && n_t > 0) ok = __all_sync(0xffffffffu, tc::mbar_wait(&sm.pdone, (n_t - 1) & 1));
    if (!ok) atomicExch(&sm.abort_flag, 1);
    tc::fence_after_sync();
    const int dv0 = AT_VD * rank;
    if (a.splits == 1) {
      const float sk = a.sink[h];
      const float M = fmaxf(sk, m_run);
      float den = 0.f, f = 0.f;
      if (M != -INFINITY) {
        f = (m_run == -INFINITY) ? 0.f : __expf(m_run - M);
        den = __expf(sk - M) + l_run * f;
      }
      const float inv = den > 0.f ? f / den : 0.f;
      __nv_bfloat16* o = (__nv_bfloat16*)a.out + ((size_t)row * AT_H + h) * 512 + dv0;
#pragma unroll 1
      for (int c = 0; c < AT_VD / 64; ++c) {
        uint32_t v[64];
        if (ok && n_t > 0) {
          tc::tmem_ld64(tmem + lane_base + TM_O + c * 64, v);
        } else {
          for (int j = 0; j < 64; ++j) v[j] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float f8[8];
          for (int j = 0; j < 8; ++j) f8[j] = __uint_as_float(v[q * 8 + j]) * inv;
          Elem<__nv_bfloat16>::st_vec(o + c * 64 + q * 8, f8);
        }
      }
      if (a.lse && rank == 0) a.lse[(size_t)row * AT_H + h] = den > 0.f ? M + logf(den) : -INFINITY;
    } else {
      float* P = a.part + (((size_t)row * a.splits + split) * AT_H + h) * attn_part_stride(512);
#pragma unroll 1
      for (int c = 0; c < AT_VD / 64; ++c) {
        uint32_t v[64];
        if (ok && n_t > 0) {
          tc::tmem_ld64(tmem + lane_base + TM_O + c * 64, v);
        } else {
          for (int j = 0; j < 64; ++j) v[j] = 0u;
        }
        float4* d4 = reinterpret_cast<float4*>(P + dv0 + c * 64);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          d4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]), __uint_as_float(v[4 * j + 2]),
                              __uint_as_float(v[4 * j + 3]));
      }
      if (rank == 0) { P[512] = m_run; P[513] = l_run; }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (sm.abort_flag && threadIdx.x == 0) raise_err(a.err, CSA_DEVERR_TIMEOUT);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, TM_COLS);
  }
  cluster_sync_all();                                 // the peer may still read our barriers / buffers
}

}  // namespace

cudaError_t launch_attention_tc(AttnArgs a, cudaStream_t st, bool* used) {
  *used = false;
  if (a.H != AT_H || a.dk != 576 || a.dv != 512) return cudaSuccess;
  if ((uintptr_t)a.q & 15 || (uintptr_t)a.cache & 15 || (a.win && ((uintptr_t)a.win & 15))) return cudaSuccess;
  const size_t smem = sizeof(AtSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(2 * a.splits, a.B * a.Tq);
  attn_tc_kernel<<<grid, 256, smem, st>>>(a);
  *used = true;
  return cudaGetLastError();
}

}  // namespace csa
