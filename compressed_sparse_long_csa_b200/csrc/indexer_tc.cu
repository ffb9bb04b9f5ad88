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
// into a STAGES-deep ring; warp 1 owns the TMEM allocation and one lane issues the
// tcgen05.mma (M = 128, N = 64 G, K = 32, four per tile) into a double-buffered
// accumulator; warps 4..7 run the epilogue.  Every wait is bounded: on timeout the
// CTA raises CSA_DEVERR_TIMEOUT, drains its own copies and exits.
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

template <int G, int STAGES>
struct IdxSmem {
  alignas(1024) uint8_t q[G * 64 * IT_KB];
  alignas(1024) uint8_t k[STAGES][IT_TILE_BYTES];
  alignas(8) uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t qfull;
  uint32_t tmem_base;
  int abort_flag;
  int t_begin, t_end;
  int n_elig[G];
  int row[G];
  float wq[G][64];
};

template <int G, int STAGES>
__global__ void __launch_bounds__(256, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ, IdxTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  using Sm = IdxSmem<G, STAGES>;
  Sm& sm = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const IndexerArgs& a = p.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, qg = blockIdx.y, b = blockIdx.z;
  constexpr int N = 64 * G;
  constexpr uint32_t NCOLS = 2 * N;          // two accumulators; power of two >= 32

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { tc::mbar_init(&sm.full[s], 1); tc::mbar_init(&sm.empty[s], 1); }
    for (int s = 0; s < 2; ++s) { tc::mbar_init(&sm.tfull[s], 1); tc::mbar_init(&sm.tempty[s], 4); }
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
  const uint32_t tmem = sm.tmem_base;
  const int t_begin = sm.t_begin, n_t = sm.t_end - sm.t_begin;

  if (warp == 0) {
    if (lane == 0 && n_t > 0) {
      tc::prefetch_tmap(&tmK);
      tc::prefetch_tmap(&tmQ);
      tc::mbar_arrive_expect_tx(&sm.qfull, G * 64 * IT_KB);
      tc::tma_load_2d(sm.q, &tmQ, &sm.qfull, 0, (b * a.Tq + qg * G) * 64);
      int issued = 0;
      for (int it = 0; it < n_t; ++it) {
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
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!tc::mbar_wait(&sm.tempty[acc], aph ^ 1)) { ok = false; break; }
        if (!tc::mbar_wait(&sm.full[st], ph)) { ok = false; break; }
        if (*(volatile int*)&sm.abort_flag) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t k_addr = tc::smem_u32(sm.k[st]);
#pragma unroll
        for (int ks = 0; ks < IT_KB / 32; ++ks)
          tc::mma_f8f6f4(tmem + acc * N, tc::desc_k_sw128(k_addr + ks * 32), tc::desc_k_sw128(q_addr + ks * 32), ID,
                         ks > 0 ? 1u : 0u);
        tc::mma_commit(&sm.empty[st]);
        tc::mma_commit(&sm.tfull[acc]);
        last_issued = it;
      }
      if (!ok) {
        atomicExch(&sm.abort_flag, 1);
        // let the last issued MMA finish before the TMEM is released
        if (last_issued >= 0) tc::mbar_wait(&sm.tfull[last_issued & 1], (last_issued >> 1) & 1);
      }
    }
  } else if (warp >= 4) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const float* kscale = (const float*)a.kI_scale;
    float kmax = 0.f;
    for (int it = 0; it < n_t; ++it) {
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      bool ok = tc::mbar_wait(&sm.tfull[acc], aph) && !*(volatile int*)&sm.abort_flag;
      ok = __all_sync(0xffffffffu, ok);               // the TMEM loads below are warp-collective
      if (!ok) { atomicExch(&sm.abort_flag, 1); break; }
      tc::fence_after_sync();
      const int s = (t_begin + it) * IT_ROWS + r;
      const float sk = (s < a.n_max) ? kscale[(size_t)b * a.n_max + s] : 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float val = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t v[16];
          tc::tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + acc * N + g * 64 + c * 16, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) val = fmaf(sm.wq[g][c * 16 + j], fmaxf(__uint_as_float(v[j]), 0.f), val);
        }
        if (s < sm.n_elig[g]) {
          a.scores[(size_t)sm.row[g] * a.ld + s] = val * sk;
          kmax = fmaxf(kmax, sk);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sm.tempty[acc]);
    }
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

template <int G, int STAGES>
cudaError_t launch_g(const IndexerArgs& a, cudaStream_t st, bool* used) {
  IdxTcParams p{};
  p.a = a;
  p.n_qg = (a.Tq + G - 1) / G;
  p.tiles = (int)((a.n_max + IT_ROWS - 1) / IT_ROWS);
  // decode-like shapes: split the entry tiles so that the grid covers the 148 SMs
  const int64_t ctas = (int64_t)a.B * p.n_qg;
  int splits = (int)((148 + ctas - 1) / ctas);
  if (splits > p.tiles) splits = p.tiles;
  if (splits < 1) splits = 1;
  p.tiles_per_split = (p.tiles + splits - 1) / splits;
  splits = (p.tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  CUtensorMap mk, mq;
  if (!make_map_rows128(&mk, a.kI, (uint64_t)a.B * a.n_max, IT_ROWS)) return cudaSuccess;
  if (!make_map_rows128(&mq, a.qI, (uint64_t)a.B * a.Tq * 64, 64 * G)) return cudaSuccess;
  const size_t smem = sizeof(IdxSmem<G, STAGES>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<G, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(splits, p.n_qg, a.B);
  indexer_tc_kernel<G, STAGES><<<grid, 256, smem, st>>>(mk, mq, p);
  *used = true;
  return cudaGetLastError();
}

}  // namespace

// Tensor-core scores for E4M3 operands with 64 heads of width 128; other shapes
// return *used = false and run on the CUDA-core path.
cudaError_t launch_indexer_scores_tc(const IndexerArgs& a, cudaStream_t st, bool* used) {
  *used = false;
  if (a.ifmt != CSA_IFMT_E4M3 || a.H_I != 64 || a.d_I != 128) return cudaSuccess;
  if (((uintptr_t)a.kI & 15) || ((uintptr_t)a.qI & 15)) return cudaSuccess;
  if ((int64_t)a.B * a.n_max > 0x7fffffffLL || (int64_t)a.B * a.Tq * 64 > 0x7fffffffLL) return cudaSuccess;
  // Bound on |fp32 MMA dot - exact| relative to ||q|| ||k||: twice the worst case of a
  // 128-term fp32 accumulation (128 * 2^-24).  Measured on B200: <= 5e-9 relative to the
  // bound's scale (test_indexer_fp32_score_error_within_band_bound).
  const_cast<IndexerArgs&>(a).eps_dot = 1.0f / 65536.0f;
  if (a.Tq >= 4) return launch_g<4, 6>(a, st, used);
  return launch_g<1, 8>(a, st, used);
}

}  // namespace csa
