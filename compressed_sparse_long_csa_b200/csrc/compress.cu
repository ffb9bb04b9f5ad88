// CSA and HCA gated-pooling compressors fused with the KV-cache append.
//
// "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста", section "Гибридное
// внимание: CSA и HCA", CSA step 1 (two value series C^a, C^b and two gate series
// Z^a, Z^b; a per-component softmax over the 2m sources of gate + positional bias;
// shifted, overlapping a/b windows so that each entry draws on 2m tokens) and the
// HCA paragraph (m' = 128 tokens per entry, no overlap).
//
// Both kernels are HBM-bound: every input element is read exactly once and every
// output element written once, with 16-byte vector accesses.  Softmax statistics
// are kept per component in fp32 with a streaming (running max / sum) update.
#include <type_traits>

#include "common.cuh"

namespace csa {

// Streaming softmax-weighted sum over sources for VEC components at once.
struct PoolAcc {
  float M[8], S[8], A[8];
  __device__ __forceinline__ void init(int vec) {
#pragma unroll
    for (int i = 0; i < 8; ++i) { M[i] = -INFINITY; S[i] = 0.f; A[i] = 0.f; }
  }
  __device__ __forceinline__ void add(const float* c, const float* z, const float* b, int vec) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < vec) {
        const float l = z[i] + b[i];
        const float Mn = fmaxf(M[i], l);
        const float a = __expf(M[i] - Mn);
        const float e = __expf(l - Mn);
        S[i] = S[i] * a + e;
        A[i] = A[i] * a + e * c[i];
        M[i] = Mn;
      }
    }
  }
};

// One thread per (entry, VEC-wide component group).  grid.y = batch.
template <typename T>
__global__ void __launch_bounds__(256)
csa_compress_kernel(const T* __restrict__ Ca, const T* __restrict__ Cb, const T* __restrict__ Za,
                    const T* __restrict__ Zb, const float* __restrict__ Ba, const float* __restrict__ Bb,
                    const T* __restrict__ pCb, const T* __restrict__ pZb, const int32_t* __restrict__ entry0,
                    T* __restrict__ cache, int64_t n_max, int T_new, int d, int m, unsigned* err) {
  constexpr int VEC = Elem<T>::VEC;
  const int b = blockIdx.y;
  const int groups = d / VEC;
  const int n_blk = T_new / m;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (int64_t)n_blk * groups) return;
  const int j = (int)(gid / groups);
  const int c0 = (int)(gid % groups) * VEC;
  const int e = entry0[b] + j;
  if (e < 0 || (int64_t)e >= n_max) { raise_err(err, CSA_DEVERR_ENTRY); return; }

  const size_t seq = (size_t)b * T_new * d;
  PoolAcc acc;
  acc.init(VEC);
  float cv[VEC], zv[VEC], bv[8];
  // b-half: previous block (in the chunk, or prev_* for the chunk's first entry; none for entry 0)
  if (e > 0) {
    for (int t = 0; t < m; ++t) {
      const T* cp; const T* zp;
      if (j > 0) {
        const size_t off = seq + (size_t)((j - 1) * m + t) * d + c0;
        cp = Cb + off; zp = Zb + off;
      } else {
        const size_t off = ((size_t)b * m + t) * d + c0;
        cp = pCb + off; zp = pZb + off;
      }
      Elem<T>::ld_vec(cp, cv);
      Elem<T>::ld_vec(zp, zv);
#pragma unroll
      for (int i = 0; i < VEC; ++i) bv[i] = Bb[t * d + c0 + i];
      acc.add(cv, zv, bv, VEC);
    }
  }
  // a-half: own block
  for (int t = 0; t < m; ++t) {
    const size_t off = seq + (size_t)(j * m + t) * d + c0;
    Elem<T>::ld_vec(Ca + off, cv);
    Elem<T>::ld_vec(Za + off, zv);
#pragma unroll
    for (int i = 0; i < VEC; ++i) bv[i] = Ba[t * d + c0 + i];
    acc.add(cv, zv, bv, VEC);
  }
  float out[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) out[i] = acc.A[i] / acc.S[i];
  Elem<T>::st_vec(cache + ((size_t)b * n_max + e) * d + c0, out);
}

// m = 4 (the CSA rate): all 16 source vectors and 8 bias vectors of a thread are
// loaded before any arithmetic, so a thread waits for one memory round trip instead
// of one per source.  Pools components c0 .. c0+VEC-1 of chunk entry j into out[];
// returns the entry's index in the cache, or -1 (error word set) when it is outside
// [0, n_max).
template <typename T>
__device__ __forceinline__ int pool_m4(const T* __restrict__ Ca, const T* __restrict__ Cb,
                                       const T* __restrict__ Za, const T* __restrict__ Zb,
                                       const float* __restrict__ Ba, const float* __restrict__ Bb,
                                       const T* __restrict__ pCb, const T* __restrict__ pZb,
                                       const int32_t* __restrict__ entry0, int64_t n_max, int T_new, int d,
                                       int b, int j, int c0, float* out, unsigned* err) {
  constexpr int VEC = Elem<T>::VEC;
  constexpr int M = 4;
  const int e0 = entry0[b];                // in flight with the source loads below
  const size_t seq = (size_t)b * T_new * d;
  float c[2 * M][VEC], z[2 * M][VEC], bias[2 * M][VEC];
#pragma unroll
  for (int t = 0; t < M; ++t) {
    const T *cp, *zp;
    if (j > 0) {
      const size_t off = seq + (size_t)((j - 1) * M + t) * d + c0;
      cp = Cb + off; zp = Zb + off;
    } else {
      const size_t off = ((size_t)b * M + t) * d + c0;
      cp = pCb + off; zp = pZb + off;
    }
    // the previous block's rows are read even for entry 0 (they exist; their terms are
    // dropped below), so no load waits for entry0
    Elem<T>::ld_vec(cp, c[t]);
    Elem<T>::ld_vec(zp, z[t]);
    const size_t off = seq + (size_t)(j * M + t) * d + c0;
    Elem<T>::ld_vec(Ca + off, c[M + t]);
    Elem<T>::ld_vec(Za + off, z[M + t]);
    const float4* bb = reinterpret_cast<const float4*>(Bb + t * d + c0);
    const float4* ba = reinterpret_cast<const float4*>(Ba + t * d + c0);
#pragma unroll
    for (int q = 0; q < VEC / 4; ++q) {
      const float4 x = bb[q], y = ba[q];
      bias[t][4 * q] = x.x; bias[t][4 * q + 1] = x.y; bias[t][4 * q + 2] = x.z; bias[t][4 * q + 3] = x.w;
      bias[M + t][4 * q] = y.x; bias[M + t][4 * q + 1] = y.y; bias[M + t][4 * q + 2] = y.z; bias[M + t][4 * q + 3] = y.w;
    }
  }
  const int e = e0 + j;
  if (e < 0 || (int64_t)e >= n_max) { raise_err(err, CSA_DEVERR_ENTRY); return -1; }
  const bool has_b = e > 0;
#pragma unroll
  for (int i = 0; i < VEC; ++i) {
    float mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < 2 * M; ++t)
      if (has_b || t >= M) mx = fmaxf(mx, z[t][i] + bias[t][i]);
    float S = 0.f, A = 0.f;
#pragma unroll
    for (int t = 0; t < 2 * M; ++t) {
      if (has_b || t >= M) {
        const float w = __expf(z[t][i] + bias[t][i] - mx);
        S += w;
        A = fmaf(w, c[t][i], A);
      }
    }
    out[i] = A / S;
  }
  return e;
}

// One thread per (entry, VEC-wide component group), m = 4.  grid.y = batch.
template <typename T>
__global__ void __launch_bounds__(256)
csa_compress_m4_kernel(const T* __restrict__ Ca, const T* __restrict__ Cb, const T* __restrict__ Za,
                       const T* __restrict__ Zb, const float* __restrict__ Ba, const float* __restrict__ Bb,
                       const T* __restrict__ pCb, const T* __restrict__ pZb, const int32_t* __restrict__ entry0,
                       T* __restrict__ cache, int64_t n_max, int T_new, int d, unsigned* err) {
  constexpr int VEC = Elem<T>::VEC;
  const int b = blockIdx.y;
  const int groups = d / VEC;
  const int n_blk = T_new / 4;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (int64_t)n_blk * groups) return;
  const int j = (int)(gid / groups);
  const int c0 = (int)(gid % groups) * VEC;
  float out[VEC];
  const int e = pool_m4<T>(Ca, Cb, Za, Zb, Ba, Bb, pCb, pZb, entry0, n_max, T_new, d, b, j, c0, out, err);
  if (e < 0) return;
  Elem<T>::st_vec(cache + ((size_t)b * n_max + e) * d + c0, out);
}

// ---- indexer-key producer -------------------------------------------------------------------
// "Техотчёт DeepSeek-V4 (2026)", section "FP4 с учётом квантования": the indexer's Q·K path
// caches its activations in FP4 (MXFP4, one scale per 1x32 tile).  The key of a compressed
// entry is the CSA step-1 pooling (m = 4) of the indexer activations, quantised in this
// kernel's epilogue to the format lightning_index reads:
//   E4M3:  scale = amax(|row|) / 448 (1 for an all-zero row), code = RNE(x / scale), one fp32
//          scale per row;
//   MXFP4: per 32 components, e = the smallest integer with amax <= 6 * 2^e (clamped to
//          [-127, 127]), code = RNE_e2m1(x * 2^-e), scale byte e + 127.
// Every decision is taken on the fp32 pooled value (IEEE division for E4M3, an exact power
// of two for MXFP4); the hardware conversion rounds to nearest even and saturates, and a
// value that rounds to zero is written as +0.  The d / VEC threads of an entry (a power of
// two <= 32, an aligned lane group) share the amax through shuffles.
__device__ __forceinline__ uint32_t e4m3x2_rn(float lo, float hi) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(hi), "f"(lo));
  uint32_t v = h;
  if ((v & 0x7Fu) == 0) v &= 0xFF00u;                    // +0, not -0
  if ((v & 0x7F00u) == 0) v &= 0x00FFu;
  return v;
}

__device__ __forceinline__ uint32_t e2m1x2_rn(float lo, float hi) {
  uint32_t v;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(v) : "f"(hi), "f"(lo));
  if ((v & 0x7u) == 0) v &= 0xF0u;
  if ((v & 0x70u) == 0) v &= 0x0Fu;
  return v;
}

// The MX exponent of a block maximum, from its fp32 fields: amax = f * 2^E, f in [1, 2),
// and 6 * 2^e = 1.5 * 2^(e+2), so e = E - 2 when f <= 1.5, else E - 1.
__device__ __forceinline__ int mx_exponent(float amax) {
  const uint32_t u = __float_as_uint(amax);
  const int E = (int)((u >> 23) & 0xFFu);
  if (E == 0) return -127;                                // zero or subnormal: below 2^-127 * 6
  const int e = (u & 0x7FFFFFu) > 0x400000u ? E - 128 : E - 129;
  return e < -127 ? -127 : e;
}

template <int VEC, int FMT>
__device__ __forceinline__ void store_index_key(const float (&x)[VEC], size_t row, int d, int g, int tpe,
                                                unsigned gmask, uint8_t* __restrict__ kI, void* __restrict__ kI_scale);

template <typename T, int FMT>
__global__ void __launch_bounds__(256)
index_key_compress_kernel(const T* __restrict__ Ca, const T* __restrict__ Cb, const T* __restrict__ Za,
                          const T* __restrict__ Zb, const float* __restrict__ Ba, const float* __restrict__ Bb,
                          const T* __restrict__ pCb, const T* __restrict__ pZb, const int32_t* __restrict__ entry0,
                          uint8_t* __restrict__ kI, void* __restrict__ kI_scale, int64_t n_max, int T_new, int d,
                          unsigned* err) {
  constexpr int VEC = Elem<T>::VEC;
  const int b = blockIdx.y;
  const int tpe = d / VEC;                                // threads per entry
  const int n_blk = T_new / 4;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (int64_t)n_blk * tpe) return;               // whole lane groups leave together
  const int j = (int)(gid / tpe);
  const int g = (int)(gid % tpe);
  const int c0 = g * VEC;
  const int lane = threadIdx.x & 31;
  const unsigned gmask = tpe == 32 ? 0xFFFFFFFFu : ((1u << tpe) - 1u) << (lane & ~(tpe - 1));
  float x[VEC];
  const int e = pool_m4<T>(Ca, Cb, Za, Zb, Ba, Bb, pCb, pZb, entry0, n_max, T_new, d, b, j, c0, x, err);
  if (e < 0) return;                                      // the same for the whole group
  store_index_key<VEC, FMT>(x, (size_t)b * n_max + e, d, g, tpe, gmask, kI, kI_scale);
}

// The quantised key of one pooled entry: thread g of the entry's tpe threads (an aligned lane
// group, mask gmask) holds components [g * VEC, g * VEC + VEC) in x.
template <int VEC, int FMT>
__device__ __forceinline__ void store_index_key(const float (&x)[VEC], size_t row, int d, int g, int tpe,
                                                unsigned gmask, uint8_t* __restrict__ kI, void* __restrict__ kI_scale) {
  const int c0 = g * VEC;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VEC; ++i) amax = fmaxf(amax, fabsf(x[i]));
  if (FMT == CSA_IFMT_E4M3) {
    for (int o = tpe >> 1; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, o));
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint32_t w[VEC / 4];
#pragma unroll
    for (int q = 0; q < VEC / 4; ++q)
      w[q] = e4m3x2_rn(__fdiv_rn(x[4 * q], scale), __fdiv_rn(x[4 * q + 1], scale)) |
             (e4m3x2_rn(__fdiv_rn(x[4 * q + 2], scale), __fdiv_rn(x[4 * q + 3], scale)) << 16);
    uint8_t* dst = kI + row * d + c0;
    if (VEC == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[VEC / 4 - 1]);
    else *reinterpret_cast<uint32_t*>(dst) = w[0];
    if (g == 0) reinterpret_cast<float*>(kI_scale)[row] = scale;
  } else {
    constexpr int TPB = 32 / VEC;                         // threads per 32-component block
    for (int o = TPB >> 1; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, o));
    const int ex = mx_exponent(amax);
    const float inv = __uint_as_float((uint32_t)(127 - ex) << 23);     // 2^-ex, exact: -ex in [-126, 127]
    uint32_t w = 0;
#pragma unroll
    for (int q = 0; q < VEC / 2; ++q) w |= e2m1x2_rn(x[2 * q] * inv, x[2 * q + 1] * inv) << (8 * q);
    uint8_t* dst = kI + row * (d / 2) + c0 / 2;
    if (VEC == 8) *reinterpret_cast<uint32_t*>(dst) = w;
    else *reinterpret_cast<uint16_t*>(dst) = (uint16_t)w;
    if (g % TPB == 0) reinterpret_cast<uint8_t*>(kI_scale)[row * (d / 32) + c0 / 32] = (uint8_t)(ex + 127);
  }
}

// ---- one decode step's appends in one launch --------------------------------------------------
// The token that completes block e = entry0[b] (m = 4) of sequence b brings three writes:
//   warps 0..2  the CSA pooling of the block into cache row e (pool_m4, d / VEC threads);
//   warp 3      the indexer key of the same block (pool_m4 of the indexer activations, then
//               store_index_key; d_I / VEC threads), when CaI is given;
//   warps 4..6  the token's raw latent into slot win_slot[b] of the window ring, when raw_new
//               is given (the attention reads the window's rows in any order).
// One CTA per sequence.
template <typename T, int FMT>
__global__ void __launch_bounds__(224)
decode_append_kernel(const T* __restrict__ Ca, const T* __restrict__ Cb, const T* __restrict__ Za,
                     const T* __restrict__ Zb, const float* __restrict__ Ba, const float* __restrict__ Bb,
                     const T* __restrict__ pCb, const T* __restrict__ pZb, const int32_t* __restrict__ entry0,
                     T* __restrict__ cache, int64_t n_max, int d,
                     const T* __restrict__ CaI, const T* __restrict__ CbI, const T* __restrict__ ZaI,
                     const T* __restrict__ ZbI, const float* __restrict__ BaI, const float* __restrict__ BbI,
                     const T* __restrict__ pCbI, const T* __restrict__ pZbI, uint8_t* __restrict__ kI,
                     void* __restrict__ kI_scale, int d_I,
                     const T* __restrict__ raw_new, T* __restrict__ win, const int32_t* __restrict__ win_slot, int W,
                     unsigned* err) {
  // a dependent lightning_index may start now: it reads the key written here (each row's
  // newest entry) only after waiting for this grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int VEC = Elem<T>::VEC;
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < 3) {
    const int g = threadIdx.x;
    if (g < d / VEC) {
      float out[VEC];
      const int e = pool_m4<T>(Ca, Cb, Za, Zb, Ba, Bb, pCb, pZb, entry0, n_max, 4, d, b, 0, g * VEC, out, err);
      if (e >= 0) Elem<T>::st_vec(cache + ((size_t)b * n_max + e) * d + g * VEC, out);
    }
  } else if (warp == 3) {
    const int tpe = d_I / VEC;
    if (CaI && lane < tpe) {
      const unsigned gmask = tpe == 32 ? 0xFFFFFFFFu : (1u << tpe) - 1u;
      float x[VEC];
      const int e = pool_m4<T>(CaI, CbI, ZaI, ZbI, BaI, BbI, pCbI, pZbI, entry0, n_max, 4, d_I, b, 0, lane * VEC, x, err);
      if (e >= 0) store_index_key<VEC, FMT>(x, (size_t)b * n_max + e, d_I, lane, tpe, gmask, kI, kI_scale);
    }
  } else {
    const int g = threadIdx.x - 128;
    if (raw_new && g < d / VEC) {
      const int slot = win_slot[b];
      if (slot < 0 || slot >= W) {
        if (g == 0) raise_err(err, CSA_DEVERR_WINDOW);
      } else {
        float v[VEC];
        Elem<T>::ld_vec(raw_new + (size_t)b * d + g * VEC, v);
        Elem<T>::st_vec(win + ((size_t)b * W + slot) * d + g * VEC, v);
      }
    }
  }
}

// The raw latent of the current token into slot win_slot[b] of sequence b's window ring.
template <typename T>
__global__ void __launch_bounds__(96)
window_append_kernel(const T* __restrict__ raw_new, T* __restrict__ win, const int32_t* __restrict__ win_slot, int W,
                     int d, unsigned* err) {
  constexpr int VEC = Elem<T>::VEC;
  const int b = blockIdx.x;
  for (int g = threadIdx.x; g < d / VEC; g += blockDim.x) {
    const int slot = win_slot[b];
    if (slot < 0 || slot >= W) {
      if (g == 0) raise_err(err, CSA_DEVERR_WINDOW);
      return;
    }
    float v[VEC];
    Elem<T>::ld_vec(raw_new + (size_t)b * d + g * VEC, v);
    Elem<T>::st_vec(win + ((size_t)b * W + slot) * d + g * VEC, v);
  }
}

// One CTA per (entry, slab of 8*VEC components, batch): 8 component groups x 32 token lanes.
// Each thread pools tokens tl, tl+32, ... of its group; the 32 partial (M, S, A) are merged
// in shared memory.
template <typename T>
__global__ void __launch_bounds__(256)
hca_compress_kernel(const T* __restrict__ C, const T* __restrict__ Z, const float* __restrict__ bias,
                    const int32_t* __restrict__ entry0, T* __restrict__ cache, int64_t n_max,
                    int T_new, int d, int mp, unsigned* err) {
  constexpr int VEC = Elem<T>::VEC;
  constexpr int SLAB = 8 * VEC;
  __shared__ float sM[32][SLAB + 1], sS[32][SLAB + 1], sA[32][SLAB + 1];
  // a dependent attention kernel (hca_compress_attn_decode) may start now: it reads the
  // rows written here only after waiting for this grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int j = blockIdx.x;          // entry within chunk
  const int b = blockIdx.z;
  const int g = threadIdx.x & 7;     // component group inside slab
  const int tl = threadIdx.x >> 3;   // token lane 0..31
  const int e = entry0[b] + j;
  const bool valid_e = !(e < 0 || (int64_t)e >= n_max);
  if (!valid_e) {
    if (threadIdx.x == 0) raise_err(err, CSA_DEVERR_ENTRY);
    return;
  }
  // slabs of SLAB components: blockIdx.y, blockIdx.y + gridDim.y, ...
  for (int slab = blockIdx.y; slab * SLAB < d; slab += gridDim.y) {
    const int c0 = slab * SLAB + g * VEC;
    const bool active = c0 < d;
    PoolAcc acc;
    acc.init(VEC);
    if (active) {
      float cv[VEC], zv[VEC], bv[8];
      for (int t = tl; t < mp; t += 32) {
        const size_t off = ((size_t)b * T_new + (size_t)j * mp + t) * d + c0;
        Elem<T>::ld_vec(C + off, cv);
        Elem<T>::ld_vec(Z + off, zv);
#pragma unroll
        for (int i = 0; i < VEC; ++i) bv[i] = bias[(size_t)t * d + c0 + i];
        acc.add(cv, zv, bv, VEC);
      }
    }
#pragma unroll
    for (int i = 0; i < VEC; ++i) {
      sM[tl][g * VEC + i] = acc.M[i];
      sS[tl][g * VEC + i] = acc.S[i];
      sA[tl][g * VEC + i] = acc.A[i];
    }
    __syncthreads();
    if (threadIdx.x < SLAB) {
      const int col = threadIdx.x;
      const int c = slab * SLAB + col;
      if (c < d) {
        float M = -INFINITY;
        for (int l = 0; l < 32; ++l) M = fmaxf(M, sM[l][col]);
        float S = 0.f, A = 0.f;
        for (int l = 0; l < 32; ++l) {
          const float a = (sS[l][col] > 0.f) ? __expf(sM[l][col] - M) : 0.f;
          S += sS[l][col] * a;
          A += sA[l][col] * a;
        }
        Elem<T>::st(cache + ((size_t)b * n_max + e) * d + c, A / S);
      }
    }
    __syncthreads();                 // the partials of the next slab reuse the shared arrays
  }
}

// ---- CSA compression into an FP8 cache ----------------------------------------------------
// "Гибридный attention: CSA и HCA" of the aixai.ru digest: KV entries are stored in FP8,
// only the RoPE dimensions in BF16.  One warp per entry pools its 576 components (chunk
// lane + 32 p of VEC components, p = 0, 1, ...) with the m = 4 pooling above and writes the
// 656-byte row: the e4m3 codes of x[0:512] * 2^-e (round to nearest even, saturating, +0 for
// values that round to zero), x[512:576] as bf16 and the byte e + 127, where e is the
// smallest integer with max|x[0:512]| <= 448 * 2^e (clamped to [-126, 127]): from the fields
// of amax = f * 2^E (f in [1, 2)), 448 * 2^e = 1.75 * 2^(e+8), so e = E - 8 when f <= 1.75,
// else E - 7.  The decisions are taken on the fp32 pooled values.
__device__ __forceinline__ int kv8_exponent(float amax) {
  const uint32_t u = __float_as_uint(amax);
  const int E = (int)((u >> 23) & 0xFFu);
  if (E == 0) return -126;                                // zero or subnormal: the smallest exponent
  const int e = (u & 0x7FFFFFu) > 0x600000u ? E - 134 : E - 135;
  return e < -126 ? -126 : (e > 127 ? 127 : e);
}

template <typename T>
__global__ void __launch_bounds__(256)
csa_compress_kv8_kernel(const T* __restrict__ Ca, const T* __restrict__ Cb, const T* __restrict__ Za,
                        const T* __restrict__ Zb, const float* __restrict__ Ba, const float* __restrict__ Bb,
                        const T* __restrict__ pCb, const T* __restrict__ pZb, const int32_t* __restrict__ entry0,
                        uint8_t* __restrict__ cache8, int64_t n_max, int T_new, unsigned* err) {
  constexpr int VEC = Elem<T>::VEC, D = 576, NCH = D / VEC, NOPE = 512 / VEC, PER = (NCH + 31) / 32;
  const int b = blockIdx.y, lane = threadIdx.x & 31;
  const int j = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (j >= T_new / 4) return;                            // whole warps
  float x[PER][VEC];
  int e = -1;
#pragma unroll
  for (int p = 0; p < PER; ++p) {
    const int ch = lane + 32 * p;
    if (ch < NCH) {
      const int ep = pool_m4<T>(Ca, Cb, Za, Zb, Ba, Bb, pCb, pZb, entry0, n_max, T_new, D, b, j, ch * VEC, x[p], err);
      if (p == 0) e = ep;
    }
  }
  if (e < 0) return;                                      // the same for the whole warp
  float amax = 0.f;
#pragma unroll
  for (int p = 0; p < PER; ++p)
    if (lane + 32 * p < NOPE)
#pragma unroll
      for (int i = 0; i < VEC; ++i) amax = fmaxf(amax, fabsf(x[p][i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const int ex = kv8_exponent(amax);
  const float inv = __uint_as_float((uint32_t)(127 - ex) << 23);    // 2^-ex, exact: 127 - ex in [0, 253]
  uint8_t* row = cache8 + ((size_t)b * n_max + e) * 656;
#pragma unroll
  for (int p = 0; p < PER; ++p) {
    const int ch = lane + 32 * p;
    if (ch < NOPE) {
      uint32_t w[VEC / 4];
#pragma unroll
      for (int q = 0; q < VEC / 4; ++q)
        w[q] = e4m3x2_rn(x[p][4 * q] * inv, x[p][4 * q + 1] * inv) |
               (e4m3x2_rn(x[p][4 * q + 2] * inv, x[p][4 * q + 3] * inv) << 16);
      if (VEC == 8) *reinterpret_cast<uint2*>(row + ch * VEC) = make_uint2(w[0], w[VEC / 4 - 1]);
      else *reinterpret_cast<uint32_t*>(row + ch * VEC) = w[0];
    } else if (ch < NCH) {
      uint32_t w[VEC / 2];
#pragma unroll
      for (int q = 0; q < VEC / 2; ++q) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(x[p][2 * q], x[p][2 * q + 1]);
        w[q] = *reinterpret_cast<const uint32_t*>(&h);
      }
      uint8_t* dst = row + 512 + (ch - NOPE) * VEC * 2;
      if (VEC == 8) *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1 % (VEC / 2)], w[2 % (VEC / 2)], w[3 % (VEC / 2)]);
      else *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1 % (VEC / 2)]);
    }
  }
  if (lane == 0) *reinterpret_cast<uint4*>(row + 640) = make_uint4((uint32_t)(ex + 127), 0u, 0u, 0u);
}

cudaError_t launch_csa_compress_kv8(const void* Ca, const void* Cb, const void* Za, const void* Zb, const float* Ba,
                                    const float* Bb, const void* pCb, const void* pZb, const int32_t* entry0,
                                    void* cache8, int64_t n_max, int B, int T_new, int dtype, cudaStream_t st,
                                    unsigned* err) {
  const int64_t warps = T_new / 4;
  const int threads = warps < 8 ? (int)warps * 32 : 256;
  dim3 grid((unsigned)((warps * 32 + threads - 1) / threads), B);
  note_launch();
  if (dtype == CSA_BF16) {
    using T = __nv_bfloat16;
    csa_compress_kv8_kernel<T><<<grid, threads, 0, st>>>((const T*)Ca, (const T*)Cb, (const T*)Za, (const T*)Zb, Ba,
                                                         Bb, (const T*)pCb, (const T*)pZb, entry0, (uint8_t*)cache8,
                                                         n_max, T_new, err);
  } else {
    csa_compress_kv8_kernel<float><<<grid, threads, 0, st>>>((const float*)Ca, (const float*)Cb, (const float*)Za,
                                                             (const float*)Zb, Ba, Bb, (const float*)pCb,
                                                             (const float*)pZb, entry0, (uint8_t*)cache8, n_max,
                                                             T_new, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                                const float* Ba, const float* Bb, const void* pCb, const void* pZb,
                                const int32_t* entry0, void* cache, int64_t n_max, int B, int T_new,
                                int d, int m, int dtype, cudaStream_t st, unsigned* err) {
  const int n_blk = T_new / m;
  if (m == 4) {
    const int vec = dtype == CSA_BF16 ? 8 : 4;
    const int64_t work = (int64_t)n_blk * (d / vec);
    const int threads = work < 256 ? (int)((work + 31) / 32 * 32) : 256;
    dim3 grid((unsigned)((work + threads - 1) / threads), B);
    if (dtype == CSA_BF16) {
      using T = __nv_bfloat16;
      note_launch();
      csa_compress_m4_kernel<T><<<grid, threads, 0, st>>>((const T*)Ca, (const T*)Cb, (const T*)Za, (const T*)Zb, Ba,
                                                          Bb, (const T*)pCb, (const T*)pZb, entry0, (T*)cache, n_max,
                                                          T_new, d, err);
    } else {
      note_launch();
      csa_compress_m4_kernel<float><<<grid, threads, 0, st>>>((const float*)Ca, (const float*)Cb, (const float*)Za,
                                                              (const float*)Zb, Ba, Bb, (const float*)pCb,
                                                              (const float*)pZb, entry0, (float*)cache, n_max, T_new,
                                                              d, err);
    }
    return cudaGetLastError();
  }
  if (dtype == CSA_BF16) {
    using T = __nv_bfloat16;
    const int64_t work = (int64_t)n_blk * (d / 8);
    dim3 grid((unsigned)((work + 255) / 256), B);
    note_launch();
    csa_compress_kernel<T><<<grid, 256, 0, st>>>((const T*)Ca, (const T*)Cb, (const T*)Za, (const T*)Zb,
                                                 Ba, Bb, (const T*)pCb, (const T*)pZb, entry0, (T*)cache,
                                                 n_max, T_new, d, m, err);
  } else {
    const int64_t work = (int64_t)n_blk * (d / 4);
    dim3 grid((unsigned)((work + 255) / 256), B);
    note_launch();
    csa_compress_kernel<float><<<grid, 256, 0, st>>>((const float*)Ca, (const float*)Cb, (const float*)Za,
                                                     (const float*)Zb, Ba, Bb, (const float*)pCb,
                                                     (const float*)pZb, entry0, (float*)cache, n_max,
                                                     T_new, d, m, err);
  }
  return cudaGetLastError();
}

cudaError_t launch_index_key_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                                     const float* Ba, const float* Bb, const void* pCb, const void* pZb,
                                     const int32_t* entry0, void* kI, void* kI_scale, int64_t n_max, int B,
                                     int T_new, int d, int dtype, int ifmt, cudaStream_t st, unsigned* err) {
  const int vec = dtype == CSA_BF16 ? 8 : 4;
  const int64_t work = (int64_t)(T_new / 4) * (d / vec) * B;
  // every thread waits for one round trip of its 16 source loads: spread small grids over
  // more SMs with smaller CTAs
  const int64_t per_seq = work / B;
  const int threads = per_seq < 256 ? (int)((per_seq + 31) / 32 * 32) : (work < 256LL * num_sms() ? 128 : 256);
  dim3 grid((unsigned)((per_seq + threads - 1) / threads), B);
  auto go = [&](auto tag, auto fmt) {
    using T = decltype(tag);
    note_launch();
    index_key_compress_kernel<T, decltype(fmt)::value><<<grid, threads, 0, st>>>(
        (const T*)Ca, (const T*)Cb, (const T*)Za, (const T*)Zb, Ba, Bb, (const T*)pCb, (const T*)pZb, entry0,
        (uint8_t*)kI, kI_scale, n_max, T_new, d, err);
  };
  using E4 = std::integral_constant<int, CSA_IFMT_E4M3>;
  using MX = std::integral_constant<int, CSA_IFMT_MXFP4>;
  if (dtype == CSA_BF16) {
    if (ifmt == CSA_IFMT_E4M3) go(__nv_bfloat16(), E4()); else go(__nv_bfloat16(), MX());
  } else {
    if (ifmt == CSA_IFMT_E4M3) go(float(), E4()); else go(float(), MX());
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_append(const void* Ca, const void* Cb, const void* Za, const void* Zb, const float* Ba,
                                 const float* Bb, const void* pCb, const void* pZb, const int32_t* entry0,
                                 void* cache, int64_t n_max, int d, const void* CaI, const void* CbI,
                                 const void* ZaI, const void* ZbI, const float* BaI, const float* BbI,
                                 const void* pCbI, const void* pZbI, void* kI, void* kI_scale, int d_I, int ifmt,
                                 const void* raw_new, void* win, const int32_t* win_slot, int W, int B, int dtype,
                                 cudaStream_t st, unsigned* err) {
  auto go = [&](auto tag, auto fmt) {
    using T = decltype(tag);
    note_launch();
    decode_append_kernel<T, decltype(fmt)::value><<<B, 224, 0, st>>>(
        (const T*)Ca, (const T*)Cb, (const T*)Za, (const T*)Zb, Ba, Bb, (const T*)pCb, (const T*)pZb, entry0,
        (T*)cache, n_max, d, (const T*)CaI, (const T*)CbI, (const T*)ZaI, (const T*)ZbI, BaI, BbI, (const T*)pCbI,
        (const T*)pZbI, (uint8_t*)kI, kI_scale, d_I, (const T*)raw_new, (T*)win, win_slot, W, err);
  };
  using E4 = std::integral_constant<int, CSA_IFMT_E4M3>;
  using MX = std::integral_constant<int, CSA_IFMT_MXFP4>;
  if (dtype == CSA_BF16) {
    if (ifmt == CSA_IFMT_MXFP4) go(__nv_bfloat16(), MX()); else go(__nv_bfloat16(), E4());
  } else {
    if (ifmt == CSA_IFMT_MXFP4) go(float(), MX()); else go(float(), E4());
  }
  return cudaGetLastError();
}

cudaError_t launch_window_append(const void* raw_new, void* win, const int32_t* win_slot, int W, int B, int d,
                                 int dtype, cudaStream_t st, unsigned* err) {
  auto go = [&](auto tag) {
    using T = decltype(tag);
    note_launch();
    window_append_kernel<T><<<B, 96, 0, st>>>((const T*)raw_new, (T*)win, win_slot, W, d, err);
  };
  if (dtype == CSA_BF16) go(__nv_bfloat16()); else go(float());
  return cudaGetLastError();
}

cudaError_t launch_hca_compress(const void* C, const void* Z, const float* bias, const int32_t* entry0,
                                void* cache, int64_t n_max, int B, int T_new, int d, int mp, int dtype,
                                cudaStream_t st, unsigned* err, int max_ctas) {
  const int n_blk = T_new / mp;
  // slab groups per entry: every slab its own CTA, or fewer CTAs that loop over slabs
  // when max_ctas bounds the grid (it runs beside an attention grid that fills the SMs)
  auto groups = [&](int slabs) {
    int gy = slabs;
    if (max_ctas > 0) {
      const int64_t per = (int64_t)max_ctas / ((int64_t)n_blk * B);
      gy = (int)(per < 1 ? 1 : (per < slabs ? per : slabs));
    }
    return gy;
  };
  if (dtype == CSA_BF16) {
    using T = __nv_bfloat16;
    dim3 grid(n_blk, groups((d + 63) / 64), B);
    note_launch();
    hca_compress_kernel<T><<<grid, 256, 0, st>>>((const T*)C, (const T*)Z, bias, entry0, (T*)cache, n_max,
                                                 T_new, d, mp, err);
  } else {
    dim3 grid(n_blk, groups((d + 31) / 32), B);
    note_launch();
    hca_compress_kernel<float><<<grid, 256, 0, st>>>((const float*)C, (const float*)Z, bias, entry0,
                                                     (float*)cache, n_max, T_new, d, mp, err);
  }
  return cudaGetLastError();
}

}  // namespace csa
