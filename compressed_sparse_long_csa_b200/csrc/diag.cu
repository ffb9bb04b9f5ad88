// Diagnostic kernels (no counterpart in the pages).
//
// csa_wait_probe: a kernel whose one wait can never end, run with a short limit, so that a
// caller can see the library's bounded waits give up with an error status instead of hanging.
//
// Every kernel of the library that waits (on a TMA copy, a tensor-core MMA, a peer warp)
// waits through tc::mbar_wait_limit on a CTA-local mbarrier.  This kernel initialises such
// a barrier for one arrival that nothing makes, waits on its first phase with the caller's
// limit, and on the timeout sets CSA_DEVERR_TIMEOUT and returns.  No copy or MMA is in
// flight, so the CTA exits cleanly and the context stays usable.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

__global__ void wait_probe_kernel(uint64_t limit_ns, unsigned* err) {
  __shared__ alignas(8) uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  const bool ok = tc::mbar_wait_limit(&bar, 0, limit_ns);   // phase 0 never completes
  if (!ok && threadIdx.x == 0) raise_err(err, CSA_DEVERR_TIMEOUT);
}

// csa_tensor_peak_probe: the dense tcgen05 MMA rate at the indexer kernels' own shapes,
// operands resident in shared memory (nothing else runs): E4M3 x E4M3 -> f32
// (kind::f8f6f4, M 128, N 256, K 32 per instruction, the prefill scoring shape) and MXFP4
// (kind::mxf4.block_scale, M 128, N 64, K 64, ue8m0 scales in TMEM, the decode scoring
// shape).  One CTA per SM; one thread issues iters x 128 K of MMAs into one accumulator,
// commits, and every wait is bounded.  The operand values are constants (the rate does not
// depend on them).
constexpr int PK_THREADS = 128;
constexpr uint32_t PK_SFB = 128, PK_SFA = 136;

template <int F>
__global__ void __launch_bounds__(PK_THREADS, 1) tensor_peak_kernel(int iters, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  constexpr int N = F == CSA_IFMT_E4M3 ? 256 : 64;
  constexpr int ROWB = F == CSA_IFMT_E4M3 ? 128 : 64;        // bytes per operand row (K = 128 codes)
  constexpr uint32_t COLS = F == CSA_IFMT_E4M3 ? 256 : 256;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A = base;
  uint8_t* B = base + 128 * ROWB;
  __shared__ alignas(8) uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // E4M3 0x38 = 1.0; e2m1 nibbles 0x2 = 1.0
  const uint32_t fill = F == CSA_IFMT_E4M3 ? 0x38383838u : 0x22222222u;
  for (int i = threadIdx.x; i < (128 + N) * ROWB / 16; i += PK_THREADS)
    reinterpret_cast<uint4*>(base)[i] = make_uint4(fill, fill, fill, fill);
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) { tc::tmem_alloc(&tmem_base, COLS); tc::tmem_relinquish(); }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_base;
  if (F == CSA_IFMT_MXFP4) {
    // scale 2^0 for every 32-block: A's 4 columns and B's 2, in every lane quarter
    const uint32_t lb = (uint32_t)(warp * 32) << 16, one = 0x7F7F7F7Fu;
    tc::tmem_st4(tmem + lb + PK_SFA, one, one, one, one);
    tc::tmem_st2(tmem + lb + PK_SFB, one, one);
    tc::tmem_st_wait();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1 && lane == 0) {
    if (F == CSA_IFMT_E4M3) {
      constexpr uint32_t ID = tc::idesc(tc::FMT_E4M3, tc::FMT_E4M3, 128, N);
      const uint64_t ad = tc::desc_k_sw128(tc::smem_u32(A)), bd = tc::desc_k_sw128(tc::smem_u32(B));
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_f8f6f4(tmem, ad + (uint64_t)(2 * ks), bd + (uint64_t)(2 * ks), ID, (it | ks) ? 1u : 0u);
      }
    } else {
      constexpr uint32_t ID0 = tc::idesc_mxf4(128, N, 0, 0), ID1 = tc::idesc_mxf4(128, N, 2, 2);
      const uint32_t a_addr = tc::smem_u32(A), b_addr = tc::smem_u32(B);
      const uint64_t a0 = tc::desc_k_sw64(a_addr), b0 = tc::desc_k_sw64(b_addr);
      const uint64_t a1 = tc::desc_k_sw64(a_addr + 32), b1 = tc::desc_k_sw64(b_addr + 32);
      for (int it = 0; it < iters; ++it) {
        tc::mma_mxf4(tmem, a0, b0, ID0, tmem + PK_SFA, tmem + PK_SFB, it ? 1u : 0u);
        tc::mma_mxf4(tmem, a1, b1, ID1, tmem + PK_SFA, tmem + PK_SFB, 1u);
      }
    }
    tc::mma_commit(&bar);
    if (!tc::mbar_wait(&bar, 0)) {
      raise_err(err, CSA_DEVERR_TIMEOUT);
      tc::mbar_wait(&bar, 0);                  // the MMAs must finish before the TMEM is freed
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, COLS);
}

}  // namespace

cudaError_t launch_tensor_peak_probe(int ifmt, int iters, cudaStream_t st, unsigned* err) {
  // room for one CTA per SM (each holds all 256 TMEM columns it allocates)
  const size_t smem = 120 * 1024;
  auto kern = ifmt == CSA_IFMT_E4M3 ? tensor_peak_kernel<CSA_IFMT_E4M3> : tensor_peak_kernel<CSA_IFMT_MXFP4>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  note_launch();
  kern<<<num_sms(), PK_THREADS, smem, st>>>(iters, err);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(uint64_t limit_ns, cudaStream_t st, unsigned* err) {
  note_launch();
  wait_probe_kernel<<<1, 32, 0, st>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace csa
