// Attention over selected / all compressed entries + raw sliding window + sink,
// CUDA-core path, and the split-KV combine.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA": CSA step 3 (MQA: every compressed entry is key and value
// for all query heads), the HCA paragraph (dense attention over the compressed
// entries) and the 128-token window of uncompressed entries; "Технический отчёт
// DeepSeek-V4 — часть 1/2": MLA latent (keys use all 576 dims, values the first
// 512), sliding-window branch and attention sink.
//
// The CUDA-core path runs fp32 math for any head count / width (it is the only
// path for fp32 storage); the tcgen05 path (attention_tc.cu) covers bf16 with
// 128 heads of width 576/512.  Both write the same split partials
// (m, l, unnormalised o) which attn_combine merges with the sink.
#include "attention.cuh"

namespace csa {

constexpr int CC_ROWS = 32;    // rows per shared-memory tile
constexpr int CC_HG = 8;       // heads per CTA (one warp each)
constexpr int CC_MAXD = 576;

// grid (splits, ceil(H/8), B*Tq), 256 threads.  dynamic smem: [32][dk] floats.
template <typename T>
__global__ void __launch_bounds__(256)
attn_cuda_core_kernel(AttnArgs a) {
  extern __shared__ float Ks[];               // [CC_ROWS][dk]
  __shared__ const T* rowp[CC_ROWS];
  const int split = blockIdx.x, hg = blockIdx.y, row = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = hg * CC_HG + warp;
  const int dk = a.dk, dv = a.dv;
  const bool hv = h < a.H;
  const int nq = (dk + 31) / 32, nv = (dv + 31) / 32;

  float qr[CC_MAXD / 32];
  float o[CC_MAXD / 32];
#pragma unroll
  for (int i = 0; i < CC_MAXD / 32; ++i) {
    const int c = lane + 32 * i;
    qr[i] = (hv && i < nq && c < dk) ? Elem<T>::ld((const T*)a.q + ((size_t)row * a.H + h) * dk + c) : 0.f;
    o[i] = 0.f;
  }
  float m_run = -INFINITY, l_run = 0.f;
  const int64_t nrows = attn_virtual_rows(a);
  const int64_t v0 = (int64_t)split * a.rows_per_split;
  const int64_t v1 = min(nrows, v0 + a.rows_per_split);
  const float scale = a.sm_scale;

  for (int64_t t0 = v0; t0 < v1; t0 += CC_ROWS) {
    __syncthreads();
    if (threadIdx.x < CC_ROWS) {
      const int64_t v = t0 + threadIdx.x;
      rowp[threadIdx.x] = (v < v1) ? attn_row_ptr<T>(a, row, (int)v) : nullptr;
    }
    __syncthreads();
    const int vecs = dk / Elem<T>::VEC;
    for (int i = threadIdx.x; i < CC_ROWS * vecs; i += blockDim.x) {
      const int r = i / vecs, c = (i % vecs) * Elem<T>::VEC;
      float tmp[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (rowp[r]) Elem<T>::ld_vec(rowp[r] + c, tmp);
#pragma unroll
      for (int u = 0; u < Elem<T>::VEC; ++u) Ks[r * dk + c + u] = tmp[u];
    }
    __syncthreads();
    if (!hv) continue;
    float logit = -INFINITY;
    for (int r = 0; r < CC_ROWS; ++r) {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < CC_MAXD / 32; ++i) {
        const int c = lane + 32 * i;
        if (i < nq && c < dk) part = fmaf(qr[i], Ks[r * dk + c], part);
      }
      part = warp_sum(part) * scale;
      if (lane == r) logit = rowp[r] ? part : -INFINITY;
    }
    const float mx = warp_max(logit);
    const float m_new = fmaxf(m_run, mx);
    if (m_new == -INFINITY) continue;
    const float alpha = __expf(m_run - m_new);
    const float p = __expf(logit - m_new);
    l_run = l_run * alpha + warp_sum(p);
#pragma unroll
    for (int i = 0; i < CC_MAXD / 32; ++i) o[i] *= alpha;
    for (int r = 0; r < CC_ROWS; ++r) {
      const float pr = __shfl_sync(0xffffffffu, p, r);
      if (pr == 0.f) continue;
#pragma unroll
      for (int i = 0; i < CC_MAXD / 32; ++i) {
        const int c = lane + 32 * i;
        if (i < nv && c < dv) o[i] = fmaf(pr, Ks[r * dk + c], o[i]);
      }
    }
    m_run = m_new;
  }
  if (!hv) return;
  if (a.splits == 1) {
    const float sk = a.sink[h];
    const float M = fmaxf(sk, m_run);
    float den = 0.f, f = 0.f;
    if (M != -INFINITY) {
      f = (m_run == -INFINITY) ? 0.f : __expf(m_run - M);
      den = __expf(sk - M) + l_run * f;
    }
    const float inv = den > 0.f ? f / den : 0.f;
#pragma unroll
    for (int i = 0; i < CC_MAXD / 32; ++i) {
      const int c = lane + 32 * i;
      if (i < nv && c < dv) Elem<T>::st((T*)a.out + ((size_t)row * a.H + h) * dv + c, o[i] * inv);
    }
    if (a.lse && lane == 0) a.lse[(size_t)row * a.H + h] = den > 0.f ? M + logf(den) : -INFINITY;
  } else {
    float* P = a.part + (((size_t)row * a.splits + split) * a.H + h) * attn_part_stride(dv);
#pragma unroll
    for (int i = 0; i < CC_MAXD / 32; ++i) {
      const int c = lane + 32 * i;
      if (i < nv && c < dv) P[c] = o[i];
    }
    if (lane == 0) { P[dv] = m_run; P[dv + 1] = l_run; }
  }
}

// out = sum_s e^{m_s-M} o_s / (e^{sink-M} + sum_s e^{m_s-M} l_s), M = max(sink, max_s m_s).
// grid (B*Tq, H), 128 threads.
template <typename T>
__global__ void __launch_bounds__(128)
attn_combine_kernel(AttnArgs a) {
  __shared__ float wsh[2][64];         // per split and half row: exp(m_s - M) / den (x l_s p_s in format 1)
  __shared__ float stat[2];            // M, den
  const int row = blockIdx.x, h = blockIdx.y;
  const int dv = a.dv, S = a.splits, H = a.H;
  const size_t sstride = attn_part_block(H, dv);
  const float* B0 = a.part + (size_t)row * S * sstride;     // block of split s: B0 + s * sstride
  // the splits' (m, l) once, by the first warp
  if (threadIdx.x < 32) {
    auto rec_m = [&](int s) { return a.part_fp16 ? B0[s * sstride + attn_part16_rec(H, dv, h)]
                                                 : B0[s * sstride + (size_t)h * attn_part_stride(dv) + dv]; };
    auto rec_l = [&](int s) { return a.part_fp16 ? B0[s * sstride + attn_part16_rec(H, dv, h) + 1]
                                                 : B0[s * sstride + (size_t)h * attn_part_stride(dv) + dv + 1]; };
    float M = a.sink[h];
    for (int s = threadIdx.x; s < S; s += 32) M = fmaxf(M, rec_m(s));
    M = warp_max(M);
    const float sk = a.sink[h];
    float den = 0.f;
    if (M != -INFINITY) {
      for (int s = threadIdx.x; s < S; s += 32) {
        const float ms = rec_m(s);
        if (ms != -INFINITY) den += rec_l(s) * __expf(ms - M);
      }
      den = warp_sum(den) + __expf(sk - M);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int s = threadIdx.x; s < S; s += 32) {
      const float ms = rec_m(s);
      const float w = (ms == -INFINITY || M == -INFINITY) ? 0.f : __expf(ms - M) * inv;
      if (a.part_fp16) {
        const float* r = B0 + s * sstride + attn_part16_rec(H, dv, h);
        wsh[0][s] = w * r[1] * r[2];
        wsh[1][s] = w * r[1] * r[3];
      } else {
        wsh[0][s] = w;
        wsh[1][s] = w;
      }
    }
    if (threadIdx.x == 0) { stat[0] = M; stat[1] = den; }
  }
  __syncthreads();
  // four values per thread and step, the splits' loads issued four at a time
  for (int c = 4 * threadIdx.x; c < dv; c += 4 * blockDim.x) {
    const float* wc = wsh[(a.part_fp16 && 2 * c >= dv) ? 1 : 0];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto load = [&](int s) -> float4 {
      if (a.part_fp16) {
        const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const __half*>(B0 + s * sstride) +
                                                        attn_part16_val(H, h, c));
        const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        return make_float4(lo.x, lo.y, hi.x, hi.y);
      }
      return *reinterpret_cast<const float4*>(B0 + s * sstride + (size_t)h * attn_part_stride(dv) + c);
    };
    int s = 0;
    for (; s + 4 <= S; s += 4) {
      float4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = load(s + u);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float wgt = wc[s + u];
        acc.x = fmaf(wgt, x[u].x, acc.x); acc.y = fmaf(wgt, x[u].y, acc.y);
        acc.z = fmaf(wgt, x[u].z, acc.z); acc.w = fmaf(wgt, x[u].w, acc.w);
      }
    }
    for (; s < S; ++s) {
      const float4 x = load(s);
      const float wgt = wc[s];
      acc.x = fmaf(wgt, x.x, acc.x); acc.y = fmaf(wgt, x.y, acc.y);
      acc.z = fmaf(wgt, x.z, acc.z); acc.w = fmaf(wgt, x.w, acc.w);
    }
    T* o = (T*)a.out + ((size_t)row * a.H + h) * dv + c;
    Elem<T>::st(o, acc.x);
    Elem<T>::st(o + 1, acc.y);
    Elem<T>::st(o + 2, acc.z);
    Elem<T>::st(o + 3, acc.w);
  }
  if (a.lse && threadIdx.x == 0)
    a.lse[(size_t)row * a.H + h] = stat[1] > 0.f ? stat[0] + logf(stat[1]) : -INFINITY;
}

// The tensor-core kernel's partials (format 1: fp16 values, 128 heads, d_v = 512) into bf16
// outputs.  grid (B*Tq, 64): two heads per CTA, one 8-value piece per thread.  Every
// split's piece is loaded before the weights are known (16 splits at a time).
constexpr int C16_CHUNK = 16;
__global__ void __launch_bounds__(128)
attn_combine16_kernel(AttnArgs a) {
  __shared__ float wsh[2][2][64];      // [head][half][split]
  const int row = blockIdx.x, hp = threadIdx.x >> 6, c8 = threadIdx.x & 63;
  const int h = blockIdx.y * 2 + hp;
  const int S = a.splits;
  const size_t sstride = attn_part_block(128, 512);
  const float sk = a.sink[h];
  const float* B0 = a.part + (size_t)row * S * sstride;
  const uint4* v0 = reinterpret_cast<const uint4*>(B0) + (size_t)c8 * 128 + h;   // split s: + s * sstride / 4
  uint4 x[C16_CHUNK];
#pragma unroll
  for (int u = 0; u < C16_CHUNK; ++u)
    x[u] = u < S ? __ldcg(v0 + (size_t)u * (sstride / 4)) : make_uint4(0u, 0u, 0u, 0u);
  // weights: the first warp of each head's pair of warps
  if ((threadIdx.x & 63) < 32) {
    const int lane = threadIdx.x & 31;
    float4 rc[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int s2 = lane + 32 * q;
      rc[q] = s2 < S ? __ldcg(reinterpret_cast<const float4*>(B0 + s2 * sstride + attn_part16_rec(128, 512, h)))
                     : make_float4(-INFINITY, 0.f, 0.f, 0.f);
    }
    float M = fmaxf(sk, fmaxf(rc[0].x, rc[1].x));
    M = warp_max(M);
    float den = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int q = 0; q < 2; ++q)
        if (rc[q].x != -INFINITY) den += rc[q].y * __expf(rc[q].x - M);
      den = warp_sum(den) + __expf(sk - M);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int s2 = lane + 32 * q;
      const float w = (rc[q].x == -INFINITY || M == -INFINITY) ? 0.f : __expf(rc[q].x - M) * inv * rc[q].y;
      wsh[hp][0][s2] = w * rc[q].z;
      wsh[hp][1][s2] = w * rc[q].w;
    }
    if (a.lse && lane == 0) a.lse[(size_t)row * 128 + h] = den > 0.f ? M + logf(den) : -INFINITY;
  }
  __syncthreads();
  const float* wr = wsh[hp][c8 >= 32 ? 1 : 0];
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int s0 = 0; s0 < S; s0 += C16_CHUNK) {
    if (s0 > 0) {
#pragma unroll
      for (int u = 0; u < C16_CHUNK; ++u)
        x[u] = s0 + u < S ? __ldcg(v0 + (size_t)(s0 + u) * (sstride / 4)) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < C16_CHUNK; ++u) {
      const float wgt = s0 + u < S ? wr[s0 + u] : 0.f;
      const uint32_t q4[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&q4[q]));
        acc[2 * q] = fmaf(wgt, f2.x, acc[2 * q]);
        acc[2 * q + 1] = fmaf(wgt, f2.y, acc[2 * q + 1]);
      }
    }
  }
  uint32_t pk[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
    pk[q] = *reinterpret_cast<uint32_t*>(&b2);
  }
  *reinterpret_cast<uint4*>((__nv_bfloat16*)a.out + ((size_t)row * 128 + h) * 512 + c8 * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

int attn_choose_splits(int n_queries, int H, int64_t rows, bool tc_path) {
  int64_t s;
  const int64_t tiles = (rows + 63) / 64;
  if (tc_path) {
    // one wave of CTAs (two per query and split, one CTA per SM), splits of at least two
    // 64-row tiles, and the tiles spread as evenly as whole tiles allow
    s = num_sms() / (2 * (int64_t)n_queries);
    if (s > tiles / 2) s = tiles / 2;
    if (s > 64) s = 64;                      // attn_combine_kernel keeps 64 splits' weights
    if (s < 1) s = 1;
    const int64_t per = (tiles + s - 1) / s;
    s = (tiles + per - 1) / per;
  } else {
    // aim for >= 2 waves of CTAs
    const int64_t ctas_per_split = (int64_t)n_queries * ((H + CC_HG - 1) / CC_HG);
    s = (2 * (int64_t)num_sms() + ctas_per_split - 1) / ctas_per_split;
  }
  if (s > tiles) s = tiles;
  if (s < 1) s = 1;
  if (s > 64) s = 64;
  return (int)s;
}

int attn_rows_per_split(int64_t rows, int splits, bool tc_path) {
  int64_t r = (rows + splits - 1) / splits;
  if (tc_path) r = (r + 63) / 64 * 64;     // the tensor-core kernel takes whole 64-row tiles
  return (int)(r < 1 ? 1 : r);
}

cudaError_t launch_attention_cuda_core(AttnArgs a, int dtype, cudaStream_t st) {
  const size_t smem = (size_t)CC_ROWS * a.dk * sizeof(float);
  dim3 grid(a.splits, (a.H + CC_HG - 1) / CC_HG, a.B * a.Tq);
  if (dtype == CSA_BF16) {
    cudaFuncSetAttribute(attn_cuda_core_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
    note_launch();
    attn_cuda_core_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(attn_cuda_core_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
    note_launch();
    attn_cuda_core_kernel<float><<<grid, 256, smem, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_attn_combine(const AttnArgs& a, int dtype, cudaStream_t st) {
  if (a.part_fp16 && dtype == CSA_BF16 && a.H == 128 && a.dv == 512 && a.splits <= 64) {
    // a plain launch: launched early, its CTAs would wait on the few SMs the attention
    // grid leaves free and then run there
    note_launch();
    attn_combine16_kernel<<<dim3(a.B * a.Tq, 64), 128, 0, st>>>(a);
    return cudaGetLastError();
  }
  dim3 grid(a.B * a.Tq, a.H);
  note_launch();
  if (dtype == CSA_BF16) {
    attn_combine_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(a);
  } else {
    attn_combine_kernel<float><<<grid, 128, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace csa
