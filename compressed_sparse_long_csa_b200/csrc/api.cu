// extern "C" entry points of libcsa_b200: host-side validation, workspace layout
// and dispatch to the kernels.  Nothing here allocates device memory or
// synchronises (except csa_read_device_error, which is documented to).
#include <math.h>
#include <atomic>
#include <mutex>

#include "attention.cuh"
#include "indexer.cuh"

namespace csa {
cudaError_t launch_csa_compress(const void*, const void*, const void*, const void*, const float*, const float*,
                                const void*, const void*, const int32_t*, void*, int64_t, int, int, int, int,
                                int, cudaStream_t, unsigned*);
cudaError_t launch_hca_compress(const void*, const void*, const float*, const int32_t*, void*, int64_t, int,
                                int, int, int, int, cudaStream_t, unsigned*, int max_ctas);
cudaError_t launch_csa_compress_kv8(const void*, const void*, const void*, const void*, const float*, const float*,
                                    const void*, const void*, const int32_t*, void*, int64_t, int, int, int,
                                    cudaStream_t, unsigned*);
cudaError_t launch_shard_topk_merge(const int32_t*, const float*, const int32_t*, int, int, int, int32_t*,
                                    cudaStream_t);
cudaError_t launch_attn_merge_shards(const void*, const float*, int, int64_t, int, int, void*, float*, cudaStream_t);
size_t out_proj_partial_elems(int T, int R_max);
cudaError_t launch_grouped_out_proj(const void* o, int T, int H, int dv, int g, int d_mid, const void* W1,
                                    const void* W2, int d, void* u, void* y, float* part, size_t part_elems,
                                    cudaStream_t st, unsigned* err);
cudaError_t launch_wait_probe(uint64_t limit_ns, cudaStream_t st, unsigned* err);
cudaError_t launch_tensor_peak_probe(int ifmt, int iters, cudaStream_t st, unsigned* err);
cudaError_t launch_decode_append(const void*, const void*, const void*, const void*, const float*, const float*,
                                 const void*, const void*, const int32_t*, void*, int64_t, int, const void*,
                                 const void*, const void*, const void*, const float*, const float*, const void*,
                                 const void*, void*, void*, int, int, const void*, void*, const int32_t*, int, int,
                                 int, cudaStream_t, unsigned*);
cudaError_t launch_window_append(const void*, void*, const int32_t*, int, int, int, int, cudaStream_t, unsigned*);
cudaError_t launch_index_key_compress(const void*, const void*, const void*, const void*, const float*,
                                      const float*, const void*, const void*, const int32_t*, void*, void*, int64_t,
                                      int, int, int, int, int, cudaStream_t, unsigned*);
}  // namespace csa

using namespace csa;

// Per-device error word (see CSA_DEVERR_* in csa.h).
__device__ unsigned int g_csa_device_error = 0u;

namespace {

constexpr int kMaxDevices = 64;
unsigned* g_err_ptr[kMaxDevices] = {nullptr};
std::mutex g_err_mu;

unsigned* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_csa_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = (unsigned*)p;
  }
  return g_err_ptr[dev];
}

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline cudaStream_t S(void* s) { return (cudaStream_t)s; }
inline csa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }
inline int elem_size(int dtype) { return dtype == CSA_BF16 ? 2 : 4; }

#define REQUIRE(cond, code) do { if (!(cond)) return (code); } while (0)
#define REQUIRE_PTR(p) do { if (!(p)) return CSA_ERR_NULL; if (!aligned16(p)) return CSA_ERR_ALIGN; } while (0)

// tensor-core paths may be disabled (for A/B testing) through this environment variable
bool tc_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("CSA_B200_DISABLE_TC");
    v = (e && e[0] == '1') ? 0 : 1;
  }
  return v == 1;
}

std::atomic<uint64_t> g_launches{0};

}  // namespace

void csa::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int csa::num_sms() {
  static const int n = [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        v > 0)
      return v;
    cudaGetLastError();
    return 148;
  }();
  return n;
}

extern "C" {

int csa_abi_version(void) { return CSA_ABI_VERSION; }

uint64_t csa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* csa_status_string(int s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_NULL: return "CSA_ERR_NULL: a required pointer is NULL";
    case CSA_ERR_SHAPE: return "CSA_ERR_SHAPE: a size is out of range or sizes are inconsistent";
    case CSA_ERR_DTYPE: return "CSA_ERR_DTYPE: unsupported storage or operand format";
    case CSA_ERR_ALIGN: return "CSA_ERR_ALIGN: a device pointer is not 16-byte aligned";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED: no kernel for this combination of sizes";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE: workspace missing or too small";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA: a CUDA runtime call or launch failed";
    default: return "unknown csa_status";
  }
}

csa_status csa_read_device_error(void* stream, uint32_t* out) {
  REQUIRE(out, CSA_ERR_NULL);
  unsigned* w = device_error_word();
  REQUIRE(w, CSA_ERR_CUDA);
  unsigned h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, w, sizeof(unsigned), cudaMemcpyDeviceToHost, S(stream));
  if (e == cudaSuccess) e = cudaMemsetAsync(w, 0, sizeof(unsigned), S(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(S(stream));
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  *out = h;
  return CSA_OK;
}

csa_status csa_tensor_peak_probe(int ifmt, int iters, void* stream) {
  REQUIRE(ifmt == CSA_IFMT_E4M3 || ifmt == CSA_IFMT_MXFP4, CSA_ERR_DTYPE);
  REQUIRE(iters >= 1 && iters <= 1000000, CSA_ERR_SHAPE);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  return cuda_status(launch_tensor_peak_probe(ifmt, iters, S(stream), err));
}

csa_status csa_wait_probe(uint64_t limit_ns, void* stream) {
  REQUIRE(limit_ns >= 1000u && limit_ns <= 2000000000ull, CSA_ERR_SHAPE);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  return cuda_status(launch_wait_probe(limit_ns, S(stream), err));
}

// ----------------------------------------------------------------------------- compressors
csa_status csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb, const float* Ba,
                        const float* Bb, const void* prev_Cb, const void* prev_Zb, const int32_t* entry0,
                        void* cache, int64_t n_max, int B, int T_new, int d, int m, int dtype, void* stream) {
  REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_DTYPE);
  REQUIRE(B >= 1 && B <= 65535 && T_new >= 1 && d >= 1 && m >= 1 && m <= 16 && n_max >= 1, CSA_ERR_SHAPE);
  REQUIRE(T_new % m == 0, CSA_ERR_SHAPE);
  REQUIRE(d % (dtype == CSA_BF16 ? 8 : 4) == 0, CSA_ERR_SHAPE);
  REQUIRE_PTR(Ca); REQUIRE_PTR(Cb); REQUIRE_PTR(Za); REQUIRE_PTR(Zb); REQUIRE_PTR(Ba); REQUIRE_PTR(Bb);
  REQUIRE_PTR(prev_Cb); REQUIRE_PTR(prev_Zb); REQUIRE_PTR(cache);
  REQUIRE(entry0, CSA_ERR_NULL);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  return cuda_status(launch_csa_compress(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, entry0, cache, n_max, B,
                                         T_new, d, m, dtype, S(stream), err));
}

csa_status csa_compress_kv8(const void* Ca, const void* Cb, const void* Za, const void* Zb, const float* Ba,
                            const float* Bb, const void* prev_Cb, const void* prev_Zb, const int32_t* entry0,
                            void* cache8, int64_t n_max, int B, int T_new, int d, int m, int dtype, void* stream) {
  REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_DTYPE);
  REQUIRE(B >= 1 && B <= 65535 && T_new >= 1 && n_max >= 1, CSA_ERR_SHAPE);
  REQUIRE(d == 576 && m == 4, CSA_ERR_UNSUPPORTED);
  REQUIRE(T_new % m == 0, CSA_ERR_SHAPE);
  REQUIRE_PTR(Ca); REQUIRE_PTR(Cb); REQUIRE_PTR(Za); REQUIRE_PTR(Zb); REQUIRE_PTR(Ba); REQUIRE_PTR(Bb);
  REQUIRE_PTR(prev_Cb); REQUIRE_PTR(prev_Zb); REQUIRE_PTR(cache8);
  REQUIRE(entry0, CSA_ERR_NULL);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  return cuda_status(launch_csa_compress_kv8(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, entry0, cache8, n_max, B,
                                             T_new, dtype, S(stream), err));
}

csa_status csa_decode_append(const void* Ca, const void* Cb, const void* Za, const void* Zb, const float* Ba,
                             const float* Bb, const void* prev_Cb, const void* prev_Zb, const int32_t* entry0,
                             void* cache, int64_t n_max, int d, const void* CaI, const void* CbI, const void* ZaI,
                             const void* ZbI, const float* BaI, const float* BbI, const void* prev_CbI,
                             const void* prev_ZbI, void* kI, void* kI_scale, int d_I, int ifmt, const void* raw_new,
                             void* win, const int32_t* win_slot, int W, int B, int dtype, void* stream) {
  REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_DTYPE);
  const int vec = dtype == CSA_BF16 ? 8 : 4;
  REQUIRE(B >= 1 && B <= 65535 && n_max >= 1 && d >= 1, CSA_ERR_SHAPE);
  REQUIRE(d % vec == 0 && d / vec <= 96, CSA_ERR_UNSUPPORTED);
  REQUIRE_PTR(Ca); REQUIRE_PTR(Cb); REQUIRE_PTR(Za); REQUIRE_PTR(Zb); REQUIRE_PTR(Ba); REQUIRE_PTR(Bb);
  REQUIRE_PTR(prev_Cb); REQUIRE_PTR(prev_Zb); REQUIRE_PTR(cache);
  REQUIRE(entry0, CSA_ERR_NULL);
  if (CaI) {
    REQUIRE(ifmt == CSA_IFMT_E4M3 || ifmt == CSA_IFMT_MXFP4, CSA_ERR_DTYPE);
    REQUIRE(d_I == 32 || d_I == 64 || d_I == 128 || (d_I == 256 && dtype == CSA_BF16), CSA_ERR_UNSUPPORTED);
    REQUIRE_PTR(CbI); REQUIRE_PTR(ZaI); REQUIRE_PTR(ZbI); REQUIRE_PTR(BaI); REQUIRE_PTR(BbI);
    REQUIRE_PTR(prev_CbI); REQUIRE_PTR(prev_ZbI); REQUIRE_PTR(kI); REQUIRE_PTR(kI_scale);
  }
  if (raw_new) {
    REQUIRE(W >= 1 && W <= 4096, CSA_ERR_SHAPE);
    REQUIRE_PTR(win);
    REQUIRE(win_slot, CSA_ERR_NULL);
  }
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  return cuda_status(launch_decode_append(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, entry0, cache, n_max, d, CaI, CbI,
                                          ZaI, ZbI, BaI, BbI, prev_CbI, prev_ZbI, kI, kI_scale, d_I, ifmt, raw_new, win,
                                          win_slot, W, B, dtype, S(stream), err));
}

csa_status window_append(const void* raw_new, void* win, const int32_t* win_slot, int B, int W, int d, int dtype,
                         void* stream) {
  REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_DTYPE);
  REQUIRE(B >= 1 && B <= 65535 && W >= 1 && W <= 4096 && d >= 1, CSA_ERR_SHAPE);
  REQUIRE(d % (dtype == CSA_BF16 ? 8 : 4) == 0, CSA_ERR_SHAPE);
  REQUIRE_PTR(raw_new); REQUIRE_PTR(win);
  REQUIRE(win_slot, CSA_ERR_NULL);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  return cuda_status(launch_window_append(raw_new, win, win_slot, W, B, d, dtype, S(stream), err));
}

csa_status hca_compress(const void* C, const void* Z, const float* bias, const int32_t* entry0, void* cache,
                        int64_t n_max, int B, int T_new, int d, int m_prime, int dtype, void* stream) {
  REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_DTYPE);
  REQUIRE(B >= 1 && B <= 65535 && T_new >= 1 && d >= 1 && m_prime >= 1 && m_prime <= 1024 && n_max >= 1,
          CSA_ERR_SHAPE);
  REQUIRE(T_new % m_prime == 0 && T_new / m_prime <= 2147483647, CSA_ERR_SHAPE);
  REQUIRE(d % (dtype == CSA_BF16 ? 8 : 4) == 0, CSA_ERR_SHAPE);
  REQUIRE_PTR(C); REQUIRE_PTR(Z); REQUIRE_PTR(bias); REQUIRE_PTR(cache);
  REQUIRE(entry0, CSA_ERR_NULL);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  return cuda_status(launch_hca_compress(C, Z, bias, entry0, cache, n_max, B, T_new, d, m_prime, dtype,
                                         S(stream), err, 0));
}

csa_status index_key_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb, const float* Ba,
                              const float* Bb, const void* prev_Cb, const void* prev_Zb, const int32_t* entry0,
                              void* kI, void* kI_scale, int64_t n_max, int B, int T_new, int d_I, int m, int dtype,
                              int ifmt, void* stream) {
  REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_DTYPE);
  REQUIRE(ifmt == CSA_IFMT_E4M3 || ifmt == CSA_IFMT_MXFP4, CSA_ERR_DTYPE);
  REQUIRE(B >= 1 && B <= 65535 && T_new >= 1 && n_max >= 1, CSA_ERR_SHAPE);
  REQUIRE(m == 4, CSA_ERR_UNSUPPORTED);
  REQUIRE(T_new % m == 0, CSA_ERR_SHAPE);
  // d_I / (components per thread) threads share an entry: a power of two within a warp
  REQUIRE(d_I == 32 || d_I == 64 || d_I == 128 || (d_I == 256 && dtype == CSA_BF16), CSA_ERR_UNSUPPORTED);
  REQUIRE_PTR(Ca); REQUIRE_PTR(Cb); REQUIRE_PTR(Za); REQUIRE_PTR(Zb); REQUIRE_PTR(Ba); REQUIRE_PTR(Bb);
  REQUIRE_PTR(prev_Cb); REQUIRE_PTR(prev_Zb); REQUIRE_PTR(kI); REQUIRE_PTR(kI_scale);
  REQUIRE(entry0, CSA_ERR_NULL);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  return cuda_status(launch_index_key_compress(Ca, Cb, Za, Zb, Ba, Bb, prev_Cb, prev_Zb, entry0, kI, kI_scale,
                                               n_max, B, T_new, d_I, dtype, ifmt, S(stream), err));
}

// ----------------------------------------------------------------------------- indexer / top-k
static int64_t idx_ld(int64_t n_max) { return (int64_t)round_up((size_t)n_max, 64); }

// Decode rows (at most this many queries per sequence) select through the score histogram
// (select_hist.cu), which needs its own workspace regions.
constexpr int kHistMaxTq = 3;
constexpr size_t kHistBins = 4096;
constexpr size_t kHistFine = 16;          // fine bins per coarse bin
constexpr size_t kHistCounters = 256;     // per row: certain count, CTAs done, per-CTA candidate counts

// Workspace layout of lightning_index (each region 256-byte aligned):
//   scores [R][ld] fp32 | knmax [B] | keyrange [R][2] | (decode rows:) hist [R][4096] |
//   fhist [R][65536] | counters [R][256] | bitmap [R][ld/32] | band [R][ld] x 16 bytes
// R = B * Tq.  knmax .. counters is one contiguous region, zeroed by one memset per call.
// Decode rows that take the one-cluster-per-row selection use knmax and keyrange as
// [R][kpart] partial slots (kpart <= kKpartCap(R)), written whole by the scoring kernel.
constexpr int kKpartSlots = 512;          // at least two scoring CTAs per SM on any device
static int kpart_cap(size_t R) { return R >= (size_t)kKpartSlots ? 1 : (int)(kKpartSlots / R); }
struct IdxWs {
  size_t scores, knmax, keyrange, hist, fhist, counters, bitmap, cand, end, zero_end, scand, smeta;
};
// with_scores = false (prefill rows of the streamed selection only): no score region.
static IdxWs idx_ws_layout(int B, int Tq, int64_t n_max, bool with_scores = true) {
  const size_t R = (size_t)B * Tq, ld = (size_t)idx_ld(n_max);
  IdxWs L{};
  L.scores = 0;
  L.knmax = with_scores ? round_up(R * ld * sizeof(float), 256) : 0;
  const size_t slots = Tq <= kHistMaxTq ? R * kpart_cap(R) : R;
  L.keyrange = L.knmax + round_up((slots > (size_t)B ? slots : (size_t)B) * sizeof(unsigned), 256);
  L.hist = L.keyrange + round_up(slots * 2 * sizeof(unsigned), 256);
  L.fhist = L.counters = L.bitmap = L.cand = L.end = L.zero_end = L.hist;
  if (Tq <= kHistMaxTq) {
    L.fhist = L.hist + round_up(R * kHistBins * sizeof(unsigned), 256);
    L.counters = L.fhist + round_up(R * kHistBins * kHistFine * sizeof(unsigned), 256);
    L.zero_end = L.counters + R * kHistCounters * sizeof(unsigned);
    L.bitmap = L.counters + round_up(R * kHistCounters * sizeof(unsigned), 256);
    L.cand = L.bitmap + round_up(R * (ld / 32) * sizeof(unsigned), 256);
    L.end = L.cand + round_up(R * ld * 16, 256);
  } else {
    // prefill rows: the streaming selection's candidate lists and their summaries
    L.scand = L.hist;
    L.smeta = L.scand + round_up(R * IDX_STREAM_CAP * sizeof(uint2), 256);
    L.end = L.smeta + round_up(R * sizeof(uint4), 256);
  }
  return L;
}

size_t lightning_index_workspace_size(int B, int Tq, int64_t n_max, int k) {
  (void)k;
  if (B < 1 || Tq < 1 || n_max < 1) return 0;
  return idx_ws_layout(B, Tq, n_max).end;
}

// Prefill rows that the streamed selection takes (the exact call without score_out) need no
// score region.  The same test decides the call's layout.
static bool idx_streamed_shape(int B, int Tq, int64_t n_max, int k, int ifmt, int H_I, int d_I) {
  if (!tc_enabled() || Tq <= kHistMaxTq) return false;
  IndexerArgs a{};
  a.B = B; a.Tq = Tq; a.n_max = n_max; a.k = k; a.ifmt = ifmt; a.H_I = H_I; a.d_I = d_I;
  return indexer_stream_applies(a);
}

size_t lightning_index_workspace_size_exact(int B, int Tq, int64_t n_max, int k, int ifmt, int H_I, int d_I) {
  if (B < 1 || Tq < 1 || n_max < 1) return 0;
  return idx_ws_layout(B, Tq, n_max, !idx_streamed_shape(B, Tq, n_max, k, ifmt, H_I, d_I)).end;
}

static csa_status run_lightning_index(const void* qI, const void* qI_scale, const float* w, const void* kI,
                                      const void* kI_scale, const int32_t* n_entries, const int32_t* q_pos, int m,
                                      int B, int Tq, int H_I, int d_I, int64_t n_max, int k, int ifmt,
                                      int32_t* idx_out, float* score_out, void* workspace, size_t ws_bytes,
                                      void* stream, bool bf16_scores) {
  REQUIRE(ifmt == CSA_IFMT_F32 || ifmt == CSA_IFMT_E4M3 || ifmt == CSA_IFMT_MXFP4, CSA_ERR_DTYPE);
  REQUIRE(B >= 1 && Tq >= 1 && (int64_t)B * Tq <= 65535 && H_I >= 1 && H_I <= 64 && m >= 1, CSA_ERR_SHAPE);
  REQUIRE(d_I == 32 || d_I == 64 || d_I == 128, CSA_ERR_SHAPE);
  REQUIRE(k >= 1 && k <= 2048 && n_max >= 1 && n_max <= (1 << 24), CSA_ERR_SHAPE);
  REQUIRE_PTR(qI); REQUIRE_PTR(w); REQUIRE_PTR(kI); REQUIRE_PTR(idx_out);
  if (ifmt != CSA_IFMT_F32) { REQUIRE_PTR(qI_scale); REQUIRE_PTR(kI_scale); }
  if (score_out) REQUIRE(aligned16(score_out), CSA_ERR_ALIGN);
  REQUIRE(aligned16(qI) && aligned16(kI), CSA_ERR_ALIGN);
  REQUIRE(n_entries && q_pos, CSA_ERR_NULL);
  // the streamed prefill selection writes no scores: its layout has no score region
  const bool streamed = !bf16_scores && !score_out && idx_streamed_shape(B, Tq, n_max, k, ifmt, H_I, d_I);
  const IdxWs L = idx_ws_layout(B, Tq, n_max, !streamed);
  REQUIRE(workspace && ws_bytes >= L.end, CSA_ERR_WORKSPACE);
  REQUIRE(aligned16(workspace), CSA_ERR_ALIGN);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);

  IndexerArgs a{};
  a.qI = qI; a.qI_scale = qI_scale; a.w = w; a.kI = kI; a.kI_scale = kI_scale;
  a.n_entries = n_entries; a.q_pos = q_pos; a.m = m;
  a.B = B; a.Tq = Tq; a.H_I = H_I; a.d_I = d_I; a.n_max = n_max; a.k = k; a.ifmt = ifmt;
  a.ld = idx_ld(n_max);
  char* ws = (char*)workspace;
  a.scores = (float*)(ws + L.scores);
  a.knmax = (unsigned*)(ws + L.knmax);
  a.keyrange = (unsigned*)(ws + L.keyrange);
  a.idx_out = idx_out; a.score_out = score_out; a.err = err;
  a.score_bf16 = bf16_scores ? 1 : 0;
  // decode rows of the exact call (the bf16-key call selects on the stored keys with the
  // plain top-k): rows that fit one CTA's shared memory take the one-cluster-per-row selection
  // over the staged scores, longer rows the same over chunks staged across a cluster (no
  // histograms either way); rows beyond that the histogram-seeded one
  const bool decode_rows = Tq <= kHistMaxTq && !bf16_scores;
  const bool row_fits = n_max <= indexer_select_row_max_entries();
  const bool row_path = decode_rows && (ifmt == CSA_IFMT_E4M3 || ifmt == CSA_IFMT_MXFP4) &&
                        (row_fits || indexer_select_dist_clusters(a) > 0);
  const bool hist_path = decode_rows && !row_path;
  // prefill rows that one CTA per four queries scores completely: the streaming selection
  // (candidates instead of scores; nothing to zero)
  if (streamed) {
    a.stream_cand = reinterpret_cast<uint2*>(ws + L.scand);
    a.stream_meta = reinterpret_cast<uint4*>(ws + L.smeta);
  }
  const bool stream_path = a.stream_cand != nullptr;
  if (hist_path) {
    a.hist = (unsigned*)(ws + L.hist);
    a.fhist = (unsigned*)(ws + L.fhist);
    a.counters = (unsigned*)(ws + L.counters);
    a.bitmap = (unsigned*)(ws + L.bitmap);
    a.cand = ws + L.cand;
  }
  // zeroed per call: the key-norm bound and key ranges, and the histograms and counters when
  // used; the streaming path needs only the bound (its pre-pass takes the keys' actual norms);
  // the row path's scoring kernel writes per-split partial slots whole (nothing to zero) and
  // starts by programmatic dependent launch (it waits for the preceding kernel before the
  // tile of each row's newest entry and before its first write)
  const size_t zero_bytes = (hist_path ? L.zero_end : stream_path ? L.keyrange : L.hist) - L.knmax;
  cudaError_t e = cudaSuccess;
  if (row_path && tc_enabled()) a.kpart = kpart_cap((size_t)B * Tq);
  else e = cudaMemsetAsync(ws + L.knmax, 0, zero_bytes, S(stream));
  if (e == cudaSuccess && stream_path) e = launch_key_norm_max(a, S(stream));
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  bool used_tc = false;
  if (tc_enabled()) {
    e = launch_indexer_scores_tc(a, S(stream), &used_tc);       // sets a.eps_dot (and a.kpart) of its path
    if (e != cudaSuccess) return CSA_ERR_CUDA;
  }
  if (!used_tc && a.kpart > 0) {
    // no tensor-core launch took these rows: the shared slots, zeroed, for the CUDA-core path
    a.kpart = 0;
    e = cudaMemsetAsync(ws + L.knmax, 0, zero_bytes, S(stream));
    if (e != cudaSuccess) return CSA_ERR_CUDA;
  }
  if (!used_tc) a.hist = a.fhist = nullptr;                    // the CUDA-core scores come without histograms
  if (!used_tc) {
    // sequential fp32 FMA accumulation of d_I exact products: |err| <= (d_I+2) u sum|q c k c|
    a.eps_dot = (float)(d_I + 4) * 5.9604645e-08f * 1.25f;
    e = launch_indexer_scores_cuda_core(a, S(stream));
    if (e != cudaSuccess) return CSA_ERR_CUDA;
  }
  if (bf16_scores) {
    // the stored keys are the selection's keys: a plain exact top-k over them
    RowCount rc;
    rc.q_pos = q_pos; rc.n_entries = n_entries; rc.m = m; rc.Tq = Tq;
    return cuda_status(launch_topk_select(a.scores, a.ld, rc, B * Tq, n_max, k, idx_out, S(stream), err));
  }
  if (stream_path) {
    if (!used_tc) return CSA_ERR_CUDA;                          // the streaming kernel always takes these rows
    return cuda_status(launch_indexer_select_stream(a, S(stream)));
  }
  if (row_path && used_tc) {
    const cudaError_t er = row_fits ? launch_indexer_select_row(a, S(stream)) : launch_indexer_select_dist(a, S(stream));
    if (er != cudaErrorNotSupported) return cuda_status(er);
  }
  return cuda_status(launch_indexer_select(a, S(stream)));
}

csa_status lightning_index(const void* qI, const void* qI_scale, const float* w, const void* kI,
                           const void* kI_scale, const int32_t* n_entries, const int32_t* q_pos, int m, int B,
                           int Tq, int H_I, int d_I, int64_t n_max, int k, int ifmt, int32_t* idx_out,
                           float* score_out, void* workspace, size_t ws_bytes, void* stream) {
  return run_lightning_index(qI, qI_scale, w, kI, kI_scale, n_entries, q_pos, m, B, Tq, H_I, d_I, n_max, k, ifmt,
                             idx_out, score_out, workspace, ws_bytes, stream, false);
}

csa_status lightning_index_bf16(const void* qI, const void* qI_scale, const float* w, const void* kI,
                                const void* kI_scale, const int32_t* n_entries, const int32_t* q_pos, int m, int B,
                                int Tq, int H_I, int d_I, int64_t n_max, int k, int ifmt, int32_t* idx_out,
                                void* workspace, size_t ws_bytes, void* stream) {
  return run_lightning_index(qI, qI_scale, w, kI, kI_scale, n_entries, q_pos, m, B, Tq, H_I, d_I, n_max, k, ifmt,
                             idx_out, nullptr, workspace, ws_bytes, stream, true);
}

size_t topk_select_workspace_size(int R, int64_t n, int k) {
  (void)R; (void)n; (void)k;
  return 0;
}

csa_status topk_select(const float* scores, int64_t ld, const int32_t* n_valid, int R, int64_t n, int k,
                       int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream) {
  (void)workspace; (void)ws_bytes;
  REQUIRE(R >= 1 && n >= 1 && n <= (1 << 24) && ld >= n && k >= 1 && k <= 2048, CSA_ERR_SHAPE);
  REQUIRE_PTR(scores); REQUIRE_PTR(idx_out);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  RowCount rc;
  rc.n_valid = n_valid;
  return cuda_status(launch_topk_select(scores, ld, rc, R, n, k, idx_out, S(stream), err));
}

// ----------------------------------------------------------------------------- KV-sharded decode
csa_status shard_topk_merge(const int32_t* idx_parts, const float* score_parts, const int32_t* bounds, int G, int R,
                            int k, int32_t* local_idx_out, void* stream) {
  REQUIRE(G >= 1 && G <= CSA_SHARD_MAX_G && R >= 1 && R <= 65535 && k >= 1 && (int64_t)G * k <= CSA_SHARD_MAX_CANDIDATES,
          CSA_ERR_SHAPE);
  REQUIRE(idx_parts && score_parts && bounds && local_idx_out, CSA_ERR_NULL);
  return cuda_status(launch_shard_topk_merge(idx_parts, score_parts, bounds, G, R, k, local_idx_out, S(stream)));
}

csa_status attn_merge_shards(const void* o_parts, const float* lse_parts, int G, int64_t rows, int dv, int dtype,
                             void* out, float* lse_out, void* stream) {
  REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_DTYPE);
  REQUIRE(G >= 1 && G <= CSA_SHARD_MAX_G && rows >= 1 && rows <= (1LL << 31) && dv >= 1 && dv <= 4096, CSA_ERR_SHAPE);
  REQUIRE(o_parts && lse_parts && out, CSA_ERR_NULL);
  return cuda_status(launch_attn_merge_shards(o_parts, lse_parts, G, rows, dv, dtype, out, lse_out, S(stream)));
}

// ----------------------------------------------------------------------------- output projection
size_t grouped_out_proj_workspace_size(int T, int g, int d_mid, int d) {
  if (T < 1 || T > 256 || g < 1 || d_mid < 1 || d < 1) return 0;
  const int R = g * d_mid > d ? g * d_mid : d;
  return out_proj_partial_elems(T, R) * sizeof(float);
}

csa_status grouped_out_proj(const void* o, int T, int H, int dv, int g, int d_mid, const void* W1, const void* W2,
                            int d, void* u, void* y, void* workspace, size_t ws_bytes, void* stream) {
  REQUIRE(T >= 1 && H >= 1 && dv >= 1 && g >= 1 && d_mid >= 1 && d >= 1, CSA_ERR_SHAPE);
  REQUIRE(H % g == 0, CSA_ERR_SHAPE);
  REQUIRE(((int64_t)(H / g) * dv) % 64 == 0 && d_mid % 128 == 0 && d % 128 == 0, CSA_ERR_UNSUPPORTED);
  REQUIRE((int64_t)H * dv <= (1 << 20) && (int64_t)g * d_mid <= (1 << 20) && d <= (1 << 20), CSA_ERR_SHAPE);
  REQUIRE((int64_t)T * H * dv < (1LL << 40), CSA_ERR_SHAPE);
  REQUIRE_PTR(o); REQUIRE_PTR(W1); REQUIRE_PTR(W2); REQUIRE_PTR(u); REQUIRE_PTR(y);
  if (workspace) REQUIRE(aligned16(workspace), CSA_ERR_ALIGN);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  const size_t part_elems = workspace ? ws_bytes / sizeof(float) : 0;
  return cuda_status(launch_grouped_out_proj(o, T, H, dv, g, d_mid, W1, W2, d, u, y, (float*)workspace, part_elems,
                                             S(stream), err));
}

// ----------------------------------------------------------------------------- attention
static bool attn_tc_shape(int dtype, int H, int dk, int dv) {
  return dtype == CSA_BF16 && H == 128 && dk == 576 && dv == 512;
}

static int decode_splits(int B, int H, int64_t rows_max) {
  const int s1 = attn_choose_splits(B, H, rows_max, false);
  const int s2 = attn_choose_splits(B, H, rows_max, true);
  return s1 > s2 ? s1 : s2;
}

size_t attn_decode_workspace_size(int B, int H, int d_v, int64_t rows_max) {
  if (B < 1 || H < 1 || d_v < 1 || rows_max < 1) return 0;
  const int s = decode_splits(B, H, rows_max);
  return round_up((size_t)B * s * H * attn_part_stride(d_v) * sizeof(float), 256);
}

static csa_status attn_common_checks(const void* q, const void* cache, const void* win, const float* sink, int B,
                                     int H, int d_k, int d_v, int64_t n_max, int W, int dtype, void* out,
                                     float* lse) {
  REQUIRE(dtype == CSA_F32 || dtype == CSA_BF16, CSA_ERR_DTYPE);
  REQUIRE(B >= 1 && H >= 1 && H <= 128 && d_k >= 1 && d_k <= 576 && d_v >= 1 && d_v <= d_k, CSA_ERR_SHAPE);
  REQUIRE(d_k % 8 == 0 && d_v % 4 == 0 && n_max >= 1 && W >= 0 && W <= 4096, CSA_ERR_SHAPE);
  REQUIRE_PTR(q); REQUIRE_PTR(cache); REQUIRE_PTR(sink); REQUIRE_PTR(out);
  if (W > 0) REQUIRE_PTR(win);
  if (lse) REQUIRE(aligned16(lse), CSA_ERR_ALIGN);
  return CSA_OK;
}

static csa_status run_attention(AttnArgs& a, int dtype, void* workspace, size_t ws_bytes, bool decode,
                                cudaStream_t st) {
  const int64_t rows = attn_virtual_rows(a);
  const bool tc = tc_enabled() && attn_tc_shape(dtype, a.H, a.dk, a.dv);
  if (decode) {
    a.splits = attn_choose_splits(a.B * a.Tq, a.H, rows, tc);
  } else {
    a.splits = 1;
  }
  a.rows_per_split = attn_rows_per_split(rows, a.splits, tc);
  a.splits = (int)((rows + a.rows_per_split - 1) / a.rows_per_split);
  if (a.splits < 1) a.splits = 1;
  a.part = (float*)workspace;
  bool used = false, combined = false;
  cudaError_t e = cudaSuccess;
  a.part_fp16 = 0;
  if (a.kv8 && !tc) return CSA_ERR_UNSUPPORTED;
  if (tc) e = launch_attention_tc(a, st, &used, &combined);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  if (a.kv8 && !used) return CSA_ERR_UNSUPPORTED;  // FP8 rows have no CUDA-core path
  if (used) a.part_fp16 = 1;                   // the tensor-core kernel's partial format
  if (!used) {
    if (tc) {  // the tensor-core path declined: recompute the split plan for the CUDA-core path
      a.splits = decode ? attn_choose_splits(a.B * a.Tq, a.H, rows, false) : 1;
      a.rows_per_split = attn_rows_per_split(rows, a.splits, false);
    }
    e = launch_attention_cuda_core(a, dtype, st);
    if (e != cudaSuccess) return CSA_ERR_CUDA;
  }
  if (a.splits > 1 && !combined) return cuda_status(launch_attn_combine(a, dtype, st));
  return CSA_OK;
}

static csa_status sparse_decode(const void* q, const void* cache, const int32_t* idx, const void* win,
                                const int32_t* win_len, const float* sink, int B, int H, int d_k, int d_v,
                                int64_t n_max, int k, int W, float sm_scale, int dtype, void* out, float* lse,
                                void* workspace, size_t ws_bytes, void* stream, int kv8) {
  csa_status s = attn_common_checks(q, cache, win, sink, B, H, d_k, d_v, n_max, W, dtype, out, lse);
  if (s != CSA_OK) return s;
  REQUIRE(k >= 0 && k <= 65536 && B <= 65535, CSA_ERR_SHAPE);
  REQUIRE(k == 0 || idx, CSA_ERR_NULL);
  REQUIRE(W == 0 || win_len, CSA_ERR_NULL);
  REQUIRE(isfinite(sm_scale), CSA_ERR_SHAPE);
  REQUIRE(workspace && ws_bytes >= attn_decode_workspace_size(B, H, d_v, (int64_t)k + W), CSA_ERR_WORKSPACE);
  REQUIRE(aligned16(workspace), CSA_ERR_ALIGN);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  AttnArgs a{};
  a.q = q; a.cache = cache; a.idx = idx; a.k = k; a.n_seg_a = k; a.win = win; a.win_len = win_len;
  a.W = W; a.prefill = 0; a.sink = sink; a.B = B; a.Tq = 1; a.H = H; a.dk = d_k; a.dv = d_v; a.n_max = n_max;
  a.sm_scale = sm_scale; a.out = out; a.lse = lse; a.err = err; a.kv8 = kv8;
  a.idx_late = 1;
  return run_attention(a, dtype, workspace, ws_bytes, true, S(stream));
}

csa_status sparse_attn_decode(const void* q, const void* cache, const int32_t* idx, const void* win,
                              const int32_t* win_len, const float* sink, int B, int H, int d_k, int d_v,
                              int64_t n_max, int k, int W, float sm_scale, int dtype, void* out, float* lse,
                              void* workspace, size_t ws_bytes, void* stream) {
  return sparse_decode(q, cache, idx, win, win_len, sink, B, H, d_k, d_v, n_max, k, W, sm_scale, dtype, out, lse,
                       workspace, ws_bytes, stream, 0);
}

csa_status sparse_attn_decode_kv8(const void* q, const void* cache8, const int32_t* idx, const void* win,
                                  const int32_t* win_len, const float* sink, int B, int H, int d_k, int d_v,
                                  int64_t n_max, int k, int W, float sm_scale, void* out, float* lse,
                                  void* workspace, size_t ws_bytes, void* stream) {
  REQUIRE(attn_tc_shape(CSA_BF16, H, d_k, d_v), CSA_ERR_UNSUPPORTED);
  return sparse_decode(q, cache8, idx, win, win_len, sink, B, H, d_k, d_v, n_max, k, W, sm_scale, CSA_BF16, out,
                       lse, workspace, ws_bytes, stream, 1);
}

static csa_status hca_decode(const void* q, const void* cache, const int32_t* n_entries, const void* win,
                             const int32_t* win_len, const float* sink, int B, int H, int d_k, int d_v,
                             int64_t n_max, int W, float sm_scale, int dtype, void* out, float* lse,
                             void* workspace, size_t ws_bytes, void* stream, int kv8) {
  csa_status s = attn_common_checks(q, cache, win, sink, B, H, d_k, d_v, n_max, W, dtype, out, lse);
  if (s != CSA_OK) return s;
  REQUIRE(n_max <= (1 << 24) && B <= 65535, CSA_ERR_SHAPE);
  REQUIRE(n_entries, CSA_ERR_NULL);
  REQUIRE(W == 0 || win_len, CSA_ERR_NULL);
  REQUIRE(isfinite(sm_scale), CSA_ERR_SHAPE);
  REQUIRE(workspace && ws_bytes >= attn_decode_workspace_size(B, H, d_v, n_max + W), CSA_ERR_WORKSPACE);
  REQUIRE(aligned16(workspace), CSA_ERR_ALIGN);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  AttnArgs a{};
  a.q = q; a.cache = cache; a.idx = nullptr; a.n_entries = n_entries; a.n_seg_a = (int)n_max;
  a.win = win; a.win_len = win_len; a.W = W; a.prefill = 0; a.sink = sink; a.B = B; a.Tq = 1; a.H = H;
  a.dk = d_k; a.dv = d_v; a.n_max = n_max; a.sm_scale = sm_scale; a.out = out; a.lse = lse; a.err = err;
  a.kv8 = kv8;
  return run_attention(a, dtype, workspace, ws_bytes, true, S(stream));
}

csa_status hca_attn_decode(const void* q, const void* cache, const int32_t* n_entries, const void* win,
                           const int32_t* win_len, const float* sink, int B, int H, int d_k, int d_v,
                           int64_t n_max, int W, float sm_scale, int dtype, void* out, float* lse,
                           void* workspace, size_t ws_bytes, void* stream) {
  return hca_decode(q, cache, n_entries, win, win_len, sink, B, H, d_k, d_v, n_max, W, sm_scale, dtype, out, lse,
                    workspace, ws_bytes, stream, 0);
}

csa_status hca_attn_decode_kv8(const void* q, const void* cache8, const int32_t* n_entries, const void* win,
                               const int32_t* win_len, const float* sink, int B, int H, int d_k, int d_v,
                               int64_t n_max, int W, float sm_scale, void* out, float* lse, void* workspace,
                               size_t ws_bytes, void* stream) {
  REQUIRE(attn_tc_shape(CSA_BF16, H, d_k, d_v), CSA_ERR_UNSUPPORTED);
  return hca_decode(q, cache8, n_entries, win, win_len, sink, B, H, d_k, d_v, n_max, W, sm_scale, CSA_BF16, out,
                    lse, workspace, ws_bytes, stream, 1);
}

csa_status hca_compress_attn_decode(const void* C, const void* Z, const float* bias, const int32_t* entry0, int T_new,
                                    int m_prime, const void* q, void* cache, const int32_t* n_entries, const void* win,
                                    const int32_t* win_len, const float* sink, int B, int H, int d_k, int d_v,
                                    int64_t n_max, int W, float sm_scale, int dtype, void* out, float* lse,
                                    void* workspace, size_t ws_bytes, void* stream) {
  // every argument of both calls is checked before the first launch
  csa_status s = attn_common_checks(q, cache, win, sink, B, H, d_k, d_v, n_max, W, dtype, out, lse);
  if (s != CSA_OK) return s;
  REQUIRE(n_max <= (1 << 24) && B <= 65535, CSA_ERR_SHAPE);
  REQUIRE(n_entries, CSA_ERR_NULL);
  REQUIRE(W == 0 || win_len, CSA_ERR_NULL);
  REQUIRE(isfinite(sm_scale), CSA_ERR_SHAPE);
  REQUIRE(workspace && ws_bytes >= attn_decode_workspace_size(B, H, d_v, n_max + W), CSA_ERR_WORKSPACE);
  REQUIRE(aligned16(workspace), CSA_ERR_ALIGN);
  REQUIRE(T_new >= 1 && m_prime >= 1 && m_prime <= 1024 && T_new % m_prime == 0, CSA_ERR_SHAPE);
  REQUIRE(d_k % (dtype == CSA_BF16 ? 8 : 4) == 0, CSA_ERR_SHAPE);
  REQUIRE_PTR(C); REQUIRE_PTR(Z); REQUIRE_PTR(bias);
  REQUIRE(entry0, CSA_ERR_NULL);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  // the full compression grid: capping it (CTAs that loop over their slabs) left room for
  // the whole attention grid but made the compression the longest chain
  cudaError_t e = launch_hca_compress(C, Z, bias, entry0, cache, n_max, B, T_new, d_k, m_prime, dtype, S(stream), err, 0);
  if (e != cudaSuccess) return CSA_ERR_CUDA;
  AttnArgs a{};
  a.q = q; a.cache = cache; a.idx = nullptr; a.n_entries = n_entries; a.n_seg_a = (int)n_max;
  a.win = win; a.win_len = win_len; a.W = W; a.prefill = 0; a.sink = sink; a.B = B; a.Tq = 1; a.H = H;
  a.dk = d_k; a.dv = d_v; a.n_max = n_max; a.sm_scale = sm_scale; a.out = out; a.lse = lse; a.err = err;
  a.dep_entry0 = entry0;
  a.dep_rows = T_new / m_prime;
  return run_attention(a, dtype, workspace, ws_bytes, true, S(stream));
}

csa_status sparse_attn_prefill(const void* q, const int32_t* q_pos, const void* cache, const int32_t* idx,
                               const void* raw, int64_t t_raw, const int32_t* raw_pos0, const float* sink, int B,
                               int Tq, int H, int d_k, int d_v, int64_t n_max, int k, int W, float sm_scale,
                               int dtype, void* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  csa_status s = attn_common_checks(q, cache, raw, sink, B, H, d_k, d_v, n_max, W, dtype, out, lse);
  if (s != CSA_OK) return s;
  REQUIRE(Tq >= 1 && (int64_t)B * Tq <= 65535 && k >= 0 && k <= 65536, CSA_ERR_SHAPE);
  REQUIRE(k == 0 || idx, CSA_ERR_NULL);
  REQUIRE(q_pos, CSA_ERR_NULL);
  REQUIRE(W == 0 || (raw_pos0 && t_raw >= 1), CSA_ERR_NULL);
  REQUIRE(isfinite(sm_scale), CSA_ERR_SHAPE);
  unsigned* err = device_error_word();
  REQUIRE(err, CSA_ERR_CUDA);
  AttnArgs a{};
  a.q = q; a.cache = cache; a.idx = idx; a.k = k; a.n_seg_a = k; a.win = raw; a.q_pos = q_pos;
  a.raw_pos0 = raw_pos0; a.t_raw = t_raw; a.W = W; a.prefill = 1; a.sink = sink; a.B = B; a.Tq = Tq; a.H = H;
  a.dk = d_k; a.dv = d_v; a.n_max = n_max; a.sm_scale = sm_scale; a.out = out; a.lse = lse; a.err = err;
  return run_attention(a, dtype, workspace, ws_bytes, false, S(stream));
}

}  // extern "C"
