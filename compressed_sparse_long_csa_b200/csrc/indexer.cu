// Lightning indexer scores, CUDA-core path.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 2 (DSA lightning indexer: ReLU-gated scores
// I[t,s] over the compressed entries) and section "FP4 с учётом квантования"
// (Q·K of the indexer in FP4).  I[t,s] = sum_j w[t,j] * max(0, D[t,j,s]) with
// D the dequantised per-head dot product.
//
// This path computes fp32 scores with exact operand products (e4m3 x e4m3 and
// e2m1 x e2m1 products are exact in fp32) and sequential fp32 accumulation; it
// serves the fp32 operand format and any shape the tensor-core kernel does not
// cover.  Alongside the scores it records max_s ||k_s|| per sequence, which bounds
// the accumulation error used by the exact top-k band (topk.cu).
#include "common.cuh"
#include "indexer.cuh"

namespace csa {

constexpr int IDX_TILE = 128;

// grid (ceil(n_max/128), B*Tq <= 65535), 128 threads; dynamic smem: q [H_I][d_I] + k tile [128][d_I+1] floats
__global__ void __launch_bounds__(IDX_TILE)
indexer_scores_cuda_core(IndexerArgs a) {
  extern __shared__ float smem[];
  const int row = blockIdx.y;                 // b*Tq + t
  const int b = row / a.Tq;
  const int HI = a.H_I, dI = a.d_I;
  float* qs = smem;                           // [HI][dI] codes (or values) as float
  float* ks = smem + HI * dI;                 // [128][dI+1]
  __shared__ float qscale[64 * 4];            // e4m3: [HI]; mxfp4: [HI][dI/32]
  __shared__ float wsh[64];

  const int n_elig = row_eligible(a, row);
  const int s0 = blockIdx.x * IDX_TILE;
  if (s0 >= n_elig) return;
  const int nb = dI / 32;

  // ---- stage the query row
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
    qs[j * dI + c] = v;
  }
  for (int i = threadIdx.x; i < HI; i += blockDim.x) {
    wsh[i] = a.w[(size_t)row * HI + i];
    if (a.ifmt == CSA_IFMT_E4M3) qscale[i] = ((const float*)a.qI_scale)[(size_t)row * HI + i];
    if (a.ifmt == CSA_IFMT_MXFP4)
      for (int bb = 0; bb < nb; ++bb)
        qscale[i * nb + bb] = ue8m0_to_float(((const uint8_t*)a.qI_scale)[((size_t)row * HI + i) * nb + bb]);
  }
  // ---- stage the key tile
  const int ntile = min(IDX_TILE, n_elig - s0);
  for (int i = threadIdx.x; i < IDX_TILE * dI; i += blockDim.x) {
    const int r = i / dI, c = i % dI;
    float v = 0.f;
    if (r < ntile) {
      const size_t koff = (size_t)b * a.n_max + s0 + r;
      if (a.ifmt == CSA_IFMT_F32) v = ((const float*)a.kI)[koff * dI + c];
      else if (a.ifmt == CSA_IFMT_E4M3) v = e4m3_to_float(((const uint8_t*)a.kI)[koff * dI + c]);
      else {
        const uint8_t byte = ((const uint8_t*)a.kI)[koff * (dI / 2) + c / 2];
        v = e2m1_to_float((c & 1) ? (byte >> 4) : (byte & 0xF));
      }
    }
    ks[r * (dI + 1) + c] = v;
  }
  __syncthreads();

  const int r = threadIdx.x;
  const bool has = r < ntile;
  const int s = s0 + (has ? r : 0);
  const size_t koff = (size_t)b * a.n_max + s;
  const float* kr = ks + r * (dI + 1);
  float kscale = 1.f;
  float kblk[4] = {1.f, 1.f, 1.f, 1.f};
  if (a.ifmt == CSA_IFMT_E4M3) kscale = ((const float*)a.kI_scale)[koff];
  if (a.ifmt == CSA_IFMT_MXFP4)
    for (int bb = 0; bb < nb; ++bb) kblk[bb] = ue8m0_to_float(((const uint8_t*)a.kI_scale)[koff * nb + bb]);

  // dequantised key norm (bounds the accumulation error of this path and the MMA path)
  float kn2 = 0.f;
  for (int c = 0; c < dI; ++c) {
    float v = kr[c];
    if (a.ifmt == CSA_IFMT_E4M3) v *= kscale;
    if (a.ifmt == CSA_IFMT_MXFP4) v *= kblk[c / 32];
    kn2 = fmaf(v, v, kn2);
  }
  if (has) atomicMax(a.knmax + b, __float_as_uint(sqrtf(kn2) * 1.0001f));

  float score = 0.f;
  for (int j = 0; j < HI; ++j) {
    const float* qj = qs + j * dI;
    float D;
    if (a.ifmt == CSA_IFMT_MXFP4) {
      D = 0.f;
      for (int bb = 0; bb < nb; ++bb) {
        float part = 0.f;                    // exact: e2m1 products on a 1/4 grid
        for (int c = bb * 32; c < bb * 32 + 32; ++c) part = fmaf(qj[c], kr[c], part);
        D = fmaf(qscale[j * nb + bb] * kblk[bb], part, D);
      }
    } else {
      float dot = 0.f;
      for (int c = 0; c < dI; ++c) dot = fmaf(qj[c], kr[c], dot);
      D = (a.ifmt == CSA_IFMT_E4M3) ? (qscale[j] * kscale) * dot : dot;
    }
    score = fmaf(wsh[j], fmaxf(D, 0.f), score);
  }
  if (a.score_bf16) score = round_bf16(score);
  if (has) a.scores[(size_t)row * a.ld + s] = score;
  record_key_range(a.keyrange, row, score, has);
}

cudaError_t launch_indexer_scores_cuda_core(const IndexerArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)a.H_I * a.d_I * 4 + (size_t)IDX_TILE * (a.d_I + 1) * 4;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaFuncSetAttribute(indexer_scores_cuda_core, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    attr_set[dev] = true;
  }
  dim3 grid((unsigned)((a.n_max + IDX_TILE - 1) / IDX_TILE), a.B * a.Tq);
  note_launch();
  indexer_scores_cuda_core<<<grid, IDX_TILE, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa
