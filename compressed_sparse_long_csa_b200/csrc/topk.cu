// Exact top-k selection of compressed entries.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 2 (the indexer keeps the top-k compressed blocks;
// k = 512 / 1024 from table "Конфигурации").  Ties go to the lower entry index and
// the selected set is written in ascending index order, padded with -1.
//
// One CTA of 1024 threads per query row:
//  1. MSB-first radix select (4 passes of 8 bits) over monotone fp32 keys gives the
//     exact k-th largest fp32 score tau.
//  2a. topk_select: entries with key > tau are in; the first `remaining` entries
//     with key == tau (ascending index) complete the set.
//  2b. lightning_index: the fp32 scores carry a bounded error E (accumulation in the
//     scoring kernel).  Entries above tau + 2E are certainly in, entries below
//     tau - 2E certainly out; the band between is re-scored exactly in fp64 from
//     the quantised operands (FP8/FP4 products and their sums are exact in fp64)
//     and ranked by (score desc, index asc).
//  3. The chosen indices are sorted ascending (bitonic sort in shared memory).
#include "indexer.cuh"

namespace csa {

constexpr int TK_THREADS = 1024;
constexpr int TK_KMAX = 2048;
constexpr int AMB_CAP = 2048;

struct TopkShared {
  uint32_t hist[256];
  uint32_t wtot[32];
  int32_t sel[TK_KMAX];
  int32_t amb[AMB_CAP];
  double amb_s[AMB_CAP];
  double contrib[32][64];
  double kd[32][128];          // per-warp key row being re-scored (exact fp64 values of the codes)
  double qd[64 * 129];         // query row codes as fp64 (padded rows: conflict-free per-head reads)
  float qsc[64 * 4];
  float w[64];
  uint32_t digit, remaining, n_sel, n_amb;
  float U;
};

__device__ __forceinline__ int block_excl_scan_flag(bool f, uint32_t* wtot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, f);
  const int pre = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) wtot[warp] = __popc(bal);
  __syncthreads();
  int wpre = 0, tot = 0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
    const int v = (int)wtot[i];
    if (i < warp) wpre += v;
    tot += v;
  }
  __syncthreads();
  *total = tot;
  return wpre + pre;
}

// Radix select: the k-th largest key among key(0..n-1).  Returns tau; *remaining =
// how many entries equal to tau belong to the top-k.
template <typename KeyFn>
__device__ uint32_t radix_select(TopkShared& sh, int n, uint32_t k, KeyFn key, uint32_t* remaining_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0, remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += blockDim.x) sh.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) {
      const uint32_t kk = key(i);
      if ((kk & mask) == prefix) atomicAdd(&sh.hist[(kk >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8], loc = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { c[q] = sh.hist[lane * 8 + q]; loc += c[q]; }
      uint32_t incl = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
        if (lane + o < 32) incl += v;
      }
      uint32_t above = incl - loc;
#pragma unroll
      for (int q = 7; q >= 0; --q) {
        if (above < remaining && remaining <= above + c[q]) {
          sh.digit = (uint32_t)(lane * 8 + q);
          sh.remaining = remaining - above;
        }
        above += c[q];
      }
    }
    __syncthreads();
    prefix |= sh.digit << shift;
    mask |= 0xFFu << shift;
    remaining = sh.remaining;
    __syncthreads();
  }
  *remaining_out = remaining;
  return prefix;
}

__device__ void block_sort_asc(int32_t* v, int n_pow2) {
  for (int size = 2; size <= n_pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < (n_pow2 >> 1); t += blockDim.x) {
        const int i = (t / stride) * stride * 2 + (t % stride);
        const int j = i + stride;
        const bool asc = (i & size) == 0;
        const int32_t a = v[i], b = v[j];
        if ((a > b) == asc) { v[i] = b; v[j] = a; }
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// Sort sel[0..cnt) ascending and write k outputs (-1 padded).
__device__ void write_sorted(TopkShared& sh, int cnt, int k, int32_t* out) {
  const int np = next_pow2(cnt < 2 ? 2 : cnt);
  for (int i = cnt + threadIdx.x; i < np; i += blockDim.x) sh.sel[i] = 0x7fffffff;
  __syncthreads();
  block_sort_asc(sh.sel, np);
  for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < cnt ? sh.sel[i] : -1;
}

// ------------------------------------------------------------------ topk_select (fp32 keys)
__global__ void __launch_bounds__(TK_THREADS)
topk_select_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ n_valid,
                   int64_t n_cap, int k, int32_t* __restrict__ idx_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  const int row = blockIdx.x;
  const float* S = scores + (size_t)row * ld;
  int n = n_valid ? n_valid[row] : (int)n_cap;
  if ((int64_t)n > n_cap) n = (int)n_cap;
  if (n < 0) n = 0;
  int32_t* out = idx_out + (size_t)row * k;
  if (threadIdx.x == 0) sh.n_sel = 0;
  __syncthreads();
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? i : -1;
    return;
  }
  uint32_t remaining;
  const uint32_t tau = radix_select(sh, n, (uint32_t)k, [&](int i) { return f32_order_key(S[i]); }, &remaining);
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    if (f32_order_key(S[i]) > tau) {
      const uint32_t slot = atomicAdd(&sh.n_sel, 1u);
      if (slot < (uint32_t)k) sh.sel[slot] = i;
    }
  __syncthreads();
  const int n_gt = min((int)sh.n_sel, k);
  // ties at tau: the `remaining` lowest indices, found by an ordered pass
  int taken = 0;
  for (int base = 0; base < n && taken < (int)remaining; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const bool f = i < n && f32_order_key(S[i]) == tau;
    int tot;
    const int pos = block_excl_scan_flag(f, sh.wtot, &tot);
    if (f && taken + pos < (int)remaining) sh.sel[n_gt + taken + pos] = i;
    taken += tot;
  }
  __syncthreads();
  write_sorted(sh, k, k, out);
}

// ------------------------------------------------------------------ indexer selection
// Exact fp64 score of entry s for query row `row`, computed by one warp; the head
// contributions are summed in order j = 0..H_I-1.
__device__ double rescore_entry(const IndexerArgs& a, TopkShared& sh, int row, int s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = row / a.Tq;
  const int HI = a.H_I, dI = a.d_I, nb = dI / 32;
  const size_t koff = (size_t)b * a.n_max + s;
  double* kd = sh.kd[warp];
  for (int c = lane; c < dI; c += 32) {
    float v;
    if (a.ifmt == CSA_IFMT_F32) v = ((const float*)a.kI)[koff * dI + c];
    else if (a.ifmt == CSA_IFMT_E4M3) v = e4m3_to_float(((const uint8_t*)a.kI)[koff * dI + c]);
    else {
      const uint8_t byte = ((const uint8_t*)a.kI)[koff * (dI / 2) + c / 2];
      v = e2m1_to_float((c & 1) ? (byte >> 4) : (byte & 0xF));
    }
    kd[c] = (double)v;
  }
  __syncwarp();
  double ks = 1.0;
  double kblk[4] = {1.0, 1.0, 1.0, 1.0};
  if (a.ifmt == CSA_IFMT_E4M3) ks = (double)((const float*)a.kI_scale)[koff];
  if (a.ifmt == CSA_IFMT_MXFP4)
    for (int bb = 0; bb < nb; ++bb) kblk[bb] = (double)ue8m0_to_float(((const uint8_t*)a.kI_scale)[koff * nb + bb]);
  for (int j = lane; j < HI; j += 32) {
    const double* qj = sh.qd + j * 129;
    double D;
    if (a.ifmt == CSA_IFMT_MXFP4) {
      D = 0.0;
      for (int bb = 0; bb < nb; ++bb) {
        double part = 0.0;
        for (int c = bb * 32; c < bb * 32 + 32; ++c) part = fma(qj[c], kd[c], part);
        D += ((double)sh.qsc[j * nb + bb] * kblk[bb]) * part;
      }
    } else {
      double raw = 0.0;
      for (int c = 0; c < dI; ++c) raw = fma(qj[c], kd[c], raw);
      D = (a.ifmt == CSA_IFMT_E4M3) ? ((double)sh.qsc[j] * ks) * raw : raw;
    }
    sh.contrib[warp][j] = (double)sh.w[j] * fmax(D, 0.0);
  }
  __syncwarp();
  double S = 0.0;
  if (lane == 0)
    for (int j = 0; j < HI; ++j) S += sh.contrib[warp][j];
  S = __shfl_sync(0xffffffffu, S, 0);
  __syncwarp();
  return S;
}

__global__ void __launch_bounds__(TK_THREADS)
indexer_select_kernel(IndexerArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  const int row = blockIdx.x;
  const int b = row / a.Tq;
  const int HI = a.H_I, dI = a.d_I, nb = dI / 32;
  const int k = a.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n = row_eligible(a, row);
  int32_t* out = a.idx_out + (size_t)row * k;
  float* sout = a.score_out ? a.score_out + (size_t)row * k : nullptr;

  // stage the query row (codes as exact floats) and its scales / weights
  for (int i = threadIdx.x; i < HI * dI; i += blockDim.x) {
    const int j = i / dI, c = i % dI;
    const size_t qoff = (size_t)row * HI + j;
    float v;
    if (a.ifmt == CSA_IFMT_F32) v = ((const float*)a.qI)[qoff * dI + c];
    else if (a.ifmt == CSA_IFMT_E4M3) v = e4m3_to_float(((const uint8_t*)a.qI)[qoff * dI + c]);
    else {
      const uint8_t byte = ((const uint8_t*)a.qI)[qoff * (dI / 2) + c / 2];
      v = e2m1_to_float((c & 1) ? (byte >> 4) : (byte & 0xF));
    }
    sh.qd[j * 129 + c] = (double)v;
  }
  for (int i = threadIdx.x; i < HI; i += blockDim.x) {
    sh.w[i] = a.w[(size_t)row * HI + i];
    if (a.ifmt == CSA_IFMT_E4M3) sh.qsc[i] = ((const float*)a.qI_scale)[(size_t)row * HI + i];
    if (a.ifmt == CSA_IFMT_MXFP4)
      for (int bb = 0; bb < nb; ++bb)
        sh.qsc[i * nb + bb] = ue8m0_to_float(((const uint8_t*)a.qI_scale)[((size_t)row * HI + i) * nb + bb]);
  }
  if (threadIdx.x == 0) { sh.n_sel = 0; sh.n_amb = 0; }
  __syncthreads();

  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? i : -1;
    if (sout) {
      for (int i = warp; i < k; i += (int)(blockDim.x >> 5)) {
        float v = 0.f;
        if (i < n) v = (float)rescore_entry(a, sh, row, i);
        if (lane == 0) sout[i] = v;
      }
    }
    return;
  }

  // U = sum_j w_j ||q_j|| (dequantised): with max_s ||k_s|| it bounds sum_c |q_c k_c|.
  if (warp == 0) {
    float u = 0.f;
    for (int j = lane; j < HI; j += 32) {
      float n2 = 0.f;
      for (int c = 0; c < dI; ++c) {
        float v = (float)sh.qd[j * 129 + c];
        if (a.ifmt == CSA_IFMT_E4M3) v *= sh.qsc[j];
        if (a.ifmt == CSA_IFMT_MXFP4) v *= sh.qsc[j * nb + c / 32];
        n2 = fmaf(v, v, n2);
      }
      u += sh.w[j] * sqrtf(n2);
    }
    u = warp_sum(u);
    if (lane == 0) sh.U = u * 1.0001f;
  }
  const float* S = a.scores + (size_t)row * a.ld;
  uint32_t remaining;
  const uint32_t tau_key = radix_select(sh, n, (uint32_t)k, [&](int i) { return f32_order_key(S[i]); }, &remaining);
  const float tau = f32_from_order_key(tau_key);
  const float knmax = __uint_as_float(a.knmax[b]);
  const float E = a.eps_dot * sh.U * knmax + 1.52587890625e-05f * fabsf(tau);   // 2^-16 |tau|
  const float hi = tau + 2.f * E, lo = tau - 2.f * E;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float v = S[i];
    if (v > hi) {
      const uint32_t slot = atomicAdd(&sh.n_sel, 1u);
      if (slot < (uint32_t)k) sh.sel[slot] = i;
    } else if (v >= lo) {
      const uint32_t slot = atomicAdd(&sh.n_amb, 1u);
      if (slot < AMB_CAP) sh.amb[slot] = i;
    }
  }
  __syncthreads();
  const int n_in = min((int)sh.n_sel, k);
  int n_amb = (int)sh.n_amb;
  if (n_amb > AMB_CAP) {
    if (threadIdx.x == 0) raise_err(a.err, CSA_DEVERR_BAND);
    n_amb = AMB_CAP;
  }
  const int need = k - n_in;
  for (int i = warp; i < n_amb; i += (int)(blockDim.x >> 5)) {
    const double v = rescore_entry(a, sh, row, sh.amb[i]);
    if (lane == 0) sh.amb_s[i] = v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n_amb; i += blockDim.x) {
    const double si = sh.amb_s[i];
    const int ii = sh.amb[i];
    int rank = 0;
    for (int j = 0; j < n_amb; ++j) {
      const double sj = sh.amb_s[j];
      rank += (sj > si) || (sj == si && sh.amb[j] < ii);
    }
    if (rank < need) sh.sel[n_in + rank] = ii;
  }
  __syncthreads();
  const int cnt = min(k, n_in + min(need, n_amb));
  write_sorted(sh, cnt, k, out);
  if (sout) {
    __syncthreads();
    for (int i = warp; i < k; i += (int)(blockDim.x >> 5)) {
      float v = 0.f;
      if (i < cnt) v = (float)rescore_entry(a, sh, row, sh.sel[i]);
      if (lane == 0) sout[i] = v;
    }
  }
}

static void set_smem_attr(const void* fn) {
  cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(TopkShared));
}

cudaError_t launch_indexer_select(const IndexerArgs& a, cudaStream_t st) {
  set_smem_attr((const void*)indexer_select_kernel);
  indexer_select_kernel<<<a.B * a.Tq, TK_THREADS, sizeof(TopkShared), st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_topk_select(const float* scores, int64_t ld, const int32_t* n_valid, int R, int64_t n,
                               int k, int32_t* idx_out, cudaStream_t st, unsigned* err) {
  (void)err;
  set_smem_attr((const void*)topk_select_kernel);
  topk_select_kernel<<<R, TK_THREADS, sizeof(TopkShared), st>>>(scores, ld, n_valid, n, k, idx_out);
  return cudaGetLastError();
}

}  // namespace csa
