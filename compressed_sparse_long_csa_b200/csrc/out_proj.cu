// Grouped output projection of the attention heads.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное внимание:
// CSA и HCA", CSA step 4: with many query heads (n_h = 128 for Pro) one projection of
// their concatenated outputs into the hidden size d would be expensive, so the heads are
// split into g groups (16 for Pro), each group's outputs are projected to an intermediate
// width of 1024, and only the concatenation of those is projected to d (table
// "Конфигурации": head size c = 512, d = 7168 for Pro).
//
//   u[t, j*d_mid + i] = sum_k W1[j*d_mid + i, k] * o[t, heads of group j][k]    (k < (H/g)*c)
//   y[t, r]           = sum_k W2[r, k] * u[t, k]                                (k < g*d_mid)
//
// Both stages are one kernel: a tcgen05 GEMM with the weights as the M operand (128 weight
// rows per CTA) and the tokens as N (up to 256 per CTA), so that a decode batch of a few
// tokens still fills the MMA: D^T[rows, tokens] = W[rows, K] * X[tokens, K]^T.  Weight and
// token tiles arrive by TMA (128-byte swizzle, no multicast) through a ring of stages; one
// elected lane of the MMA warp issues K = 16 steps into a TMEM accumulator; all four warps
// drain it (warp w holds weight rows 32w .. 32w+31) and store bf16 rows of y (or u), or
// fp32 partials when K is split across CTAs (few tokens: the weight stream then spreads
// over more SMs) and a second kernel adds the partials in a fixed order.
#include "common.cuh"
#include "tc.cuh"

#include <cudaTypedefs.h>

namespace csa {
namespace {

constexpr int OP_BM = 128;          // weight rows per CTA (MMA M)
constexpr int OP_BK = 64;           // K per stage: one 128-byte swizzled row of bf16
constexpr int OP_THREADS = 128;     // warp 0: TMA producer, warp 1: MMA issue; all four drain TMEM
constexpr int OP_SMEM_RING = 196608;

struct OpParams {
  int T;                // tokens
  int K;                // reduction length of one output row
  int rows_per_group;   // weight rows that read the same K slice of X (X column offset = group * K)
  int R;                // weight rows = output columns
  int N;                // token tile (multiple of 16, <= 256)
  int stages;
  int k_split;          // CTAs along K (fp32 partials when > 1)
  int k_per_split;      // multiple of OP_BK
  int tmem_cols;
  __nv_bfloat16* y;     // [T, R] bf16 (k_split == 1)
  float* part;          // [k_split, T, R] fp32 (k_split > 1)
  unsigned* err;
};

__global__ void __launch_bounds__(OP_THREADS, 1)
out_proj_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, OpParams p) {
  extern __shared__ unsigned char smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int a_bytes = OP_BM * OP_BK * 2;
  const int b_bytes = p.N * OP_BK * 2;
  const int stage_bytes = a_bytes + b_bytes;                 // a multiple of 1024 (N % 16 == 0)
  uint64_t* full = reinterpret_cast<uint64_t*>(base + (size_t)p.stages * stage_bytes);
  uint64_t* empty = full + p.stages;
  uint64_t* done = empty + p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * OP_BM, t0 = blockIdx.y * p.N, ks = blockIdx.z;
  const int wk0 = ks * p.k_per_split;
  const int xk0 = (row0 / p.rows_per_group) * p.K + wk0;
  const int n_k = p.k_per_split / OP_BK;

  if (threadIdx.x == 0) {
    tc::prefetch_tmap(&tmW);
    tc::prefetch_tmap(&tmX);
    for (int s = 0; s < p.stages; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
    tc::mbar_init(done, 1);
    tc::fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 1) { tc::tmem_alloc(tmem_slot, (uint32_t)p.tmem_cols); tc::tmem_relinquish(); }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // the weights are read-only inputs; the tokens (o, or u of the first stage) may come
  // from the previous kernel: wait for it before the first token tile
  tc::griddep_wait();

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_k; ++it) {
        const int st = it % p.stages;
        const uint32_t ph = (it / p.stages) & 1;
        if (!tc::mbar_wait(&empty[st], ph ^ 1)) { atomicExch(abort_flag, 1); break; }
        if (*(volatile int*)abort_flag) break;
        uint8_t* a = base + (size_t)st * stage_bytes;
        tc::mbar_arrive_expect_tx(&full[st], (uint32_t)stage_bytes);
        tc::tma_load_2d(a, &tmW, &full[st], wk0 + it * OP_BK, row0);
        tc::tma_load_2d(a + a_bytes, &tmX, &full[st], xk0 + it * OP_BK, t0);
        ++issued;
      }
      // every copy this thread started lands before the CTA may leave (bounded waits)
      for (int it = (issued > p.stages ? issued - p.stages : 0); it < issued; ++it)
        tc::mbar_wait(&full[it % p.stages], (it / p.stages) & 1);
    }
  } else if (warp == 1) {
    const uint32_t ID = tc::idesc(tc::FMT_BF16, tc::FMT_BF16, OP_BM, 16) + (uint32_t)(((p.N >> 3) - 2) << 17);
    int it = 0;
    for (; it < n_k; ++it) {
      const int st = it % p.stages;
      if (!tc::mbar_wait(&full[st], (it / p.stages) & 1)) { atomicExch(abort_flag, 1); break; }
      tc::fence_after_sync();
      const uint32_t a = tc::smem_u32(base + (size_t)st * stage_bytes);
      const uint64_t ad = tc::desc_k_sw128(a), bd = tc::desc_k_sw128(a + a_bytes);
#pragma unroll
      for (int kk = 0; kk < OP_BK / 16; ++kk)
        if (tc::elect_one()) tc::mma_f16(tmem, ad + 2 * kk, bd + 2 * kk, ID, (it | kk) != 0);
      __syncwarp();
      if (tc::elect_one()) tc::mma_commit(&empty[st]);      // the stage is free once these MMAs read it
      __syncwarp();
    }
    if (tc::elect_one()) tc::mma_commit(done);                // the accumulator is final
    __syncwarp();
  }
  // ---- epilogue: warp w drains TMEM lanes 32w .. 32w+31 (weight rows row0 + 32w + lane)
  const bool ok = tc::mbar_wait(done, 0);
  tc::fence_after_sync();
  __syncwarp();
  const bool live = ok && !*(volatile int*)abort_flag;
  if (!live && threadIdx.x == 0) raise_err(p.err, CSA_DEVERR_TIMEOUT);
  const int r = row0 + 32 * warp + lane;
  for (int c = 0; c < p.N; c += 16) {
    uint32_t v[16];
    __syncwarp();                                           // the TMEM load is warp-collective
    tc::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c, v);
    tc::tmem_ld_wait();
    if (!live || r >= p.R) continue;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int t = t0 + c + j;
      if (t >= p.T) break;
      if (p.k_split == 1) p.y[(size_t)t * p.R + r] = __float2bfloat16_rn(__uint_as_float(v[j]));
      else p.part[((size_t)ks * p.T + t) * p.R + r] = __uint_as_float(v[j]);
    }
  }
  tc::griddep_launch_dependents();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
}

// y[t, r] = bf16(sum over splits s = 0, 1, ... of part[s, t, r]), 4 outputs per thread.
__global__ void __launch_bounds__(256)
out_proj_reduce_kernel(const float* __restrict__ part, int k_split, int64_t n, __nv_bfloat16* __restrict__ y) {
  tc::griddep_wait();
  const int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= n) return;
  float4 acc = *reinterpret_cast<const float4*>(part + i);
  for (int s = 1; s < k_split; ++s) {
    const float4 x = *reinterpret_cast<const float4*>(part + (size_t)s * n + i);
    acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
  *reinterpret_cast<__nv_bfloat162*>(y + i) = lo;
  *reinterpret_cast<__nv_bfloat162*>(y + i + 2) = hi;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_op() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)ptr;
  }
  return fn;
}

// [rows, cols] bf16 with a row pitch of ld elements; box = 64 columns x box_rows rows,
// 128-byte swizzle; rows past the end read as zero.
bool make_op_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  auto enc = get_encode_op();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One GEMM stage: out[T, R] (+ partials) = W[R, K] applied to X, group g of the weight
// rows reading columns [g*K, (g+1)*K) of X ([T, ldx]).
cudaError_t launch_stage(const void* W, int R, int K, int rows_per_group, const void* X, int64_t ldx, int64_t x_cols,
                         int T, __nv_bfloat16* out, float* part, size_t part_elems, cudaStream_t st, unsigned* err) {
  OpParams p{};
  p.T = T; p.K = K; p.rows_per_group = rows_per_group; p.R = R; p.err = err; p.y = out;
  p.N = T <= 256 ? (T + 15) / 16 * 16 : (T <= 2048 ? 128 : 256);
  const int stage_bytes = (OP_BM + p.N) * OP_BK * 2;
  p.stages = OP_SMEM_RING / stage_bytes;
  if (p.stages > 12) p.stages = 12;
  p.tmem_cols = p.N <= 32 ? 32 : (p.N <= 64 ? 64 : (p.N <= 128 ? 128 : 256));
  const int row_blocks = (R + OP_BM - 1) / OP_BM;
  const int t_blocks = (T + p.N - 1) / p.N;
  // few CTAs: split K (each split streams its share of the weights) while the partials stay small
  int ksplit = 1;
  const int k_steps = K / OP_BK;
  while (part && row_blocks * t_blocks * ksplit * 2 <= num_sms() && k_steps % (ksplit * 2) == 0 &&
         (size_t)ksplit * 2 * T * R <= part_elems)
    ksplit *= 2;
  p.k_split = ksplit;
  p.k_per_split = K / ksplit;
  p.part = part;
  CUtensorMap mw, mx;
  if (!make_op_map(&mw, W, (uint64_t)R, (uint64_t)K, (uint64_t)K, OP_BM)) return cudaErrorInvalidValue;
  if (!make_op_map(&mx, X, (uint64_t)T, (uint64_t)x_cols, (uint64_t)ldx, (uint32_t)p.N)) return cudaErrorInvalidValue;
  const size_t smem = (size_t)p.stages * stage_bytes + 1024 + 256;
  cudaError_t e = cudaFuncSetAttribute(out_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(row_blocks, t_blocks, ksplit);
  cfg.blockDim = dim3(OP_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait in the kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  e = cudaLaunchKernelEx(&cfg, out_proj_kernel, mw, mx, p);
  if (e != cudaSuccess || ksplit == 1) return e;
  const int64_t n = (int64_t)T * R;
  cfg.gridDim = dim3((unsigned)((n / 4 + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  note_launch();
  return cudaLaunchKernelEx(&cfg, out_proj_reduce_kernel, (const float*)part, ksplit, n, out);
}

}  // namespace

size_t out_proj_partial_elems(int T, int R_max) { return (size_t)8 * T * R_max; }

cudaError_t launch_grouped_out_proj(const void* o, int T, int H, int dv, int g, int d_mid, const void* W1,
                                    const void* W2, int d, void* u, void* y, float* part, size_t part_elems,
                                    cudaStream_t st, unsigned* err) {
  const int K1 = (H / g) * dv;
  // stage 1: u = blockdiag(W1_0 .. W1_{g-1}) o, the groups' weight rows stacked
  cudaError_t e = launch_stage(W1, g * d_mid, K1, d_mid, o, (int64_t)H * dv, (int64_t)H * dv, T,
                               (__nv_bfloat16*)u, part, part_elems, st, err);
  if (e != cudaSuccess) return e;
  // stage 2: y = W2 u
  return launch_stage(W2, d, g * d_mid, d, u, (int64_t)g * d_mid, (int64_t)g * d_mid, T, (__nv_bfloat16*)y, part,
                      part_elems, st, err);
}

}  // namespace csa
