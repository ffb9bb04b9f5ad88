/*
 * csa.h — C ABI of the B200 (sm_100a) CSA / HCA attention hot path.
 *
 * The operations follow the DeepSeek-V4 technical report as digested in
 * "Техотчёт DeepSeek-V4 (2026): миллион токенов контекста" (ai.flicky.cc),
 * section "Гибридное внимание: CSA и HCA" (CSA steps 1-3, the HCA paragraph,
 * the 128-token sliding window), table "Конфигурации" (m = 4, m' = 128,
 * top-k 512 / 1024, 128 heads of width 512) and section "FP4 с учётом
 * квантования" (FP4 indexer path); plus "Технический отчёт DeepSeek-V4 — часть
 * 1/2" (aifinder.ae) for the MLA latent (576 = 512 + 64 RoPE dims), the window
 * branch and the attention sink.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer named as device memory must be a CUDA device pointer on the
 *   current device; sizes are element counts.  All tensors are dense, row-major
 *   (C order) with the shapes given; the library never allocates, frees or
 *   synchronises: outputs and workspaces belong to the caller.
 * - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *   NULL = the legacy default stream).  It returns CSA_OK once its kernels are
 *   enqueued.  Arguments are validated on the host BEFORE any launch; an invalid
 *   argument returns an error code and enqueues nothing.
 * - Device-side checks (an index out of range, a window row outside the raw
 *   buffer, a bounded wait that gave up, a top-k candidate band that overflowed)
 *   never fault: the offending access is skipped and a bit is OR-ed into a
 *   per-device error word that csa_read_device_error() returns and clears.
 * - Latent rows (compressor inputs, KV cache, window, queries, outputs) are
 *   stored as CSA_BF16 or CSA_F32 (dtype argument).  Biases, sinks, indexer
 *   weights and FP8 scales are always fp32.
 * - 16-byte alignment is required of every device pointer; row widths must keep
 *   rows 16-byte aligned (d * element size % 16 == 0).
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSA_ABI_VERSION 1

typedef enum csa_status {
  CSA_OK = 0,
  CSA_ERR_NULL = 1,        /* a required pointer is NULL                              */
  CSA_ERR_SHAPE = 2,       /* a size is out of range or sizes are inconsistent         */
  CSA_ERR_DTYPE = 3,       /* unsupported storage / operand format                     */
  CSA_ERR_ALIGN = 4,       /* a device pointer is not 16-byte aligned                  */
  CSA_ERR_UNSUPPORTED = 5, /* no kernel for this combination of sizes                  */
  CSA_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than the *_workspace_size()    */
  CSA_ERR_CUDA = 7         /* a CUDA runtime call or launch failed                     */
} csa_status;

typedef enum csa_dtype { CSA_F32 = 0, CSA_BF16 = 1 } csa_dtype;

/* Operand format of the lightning indexer (queries and keys use the same one). */
typedef enum csa_ifmt {
  CSA_IFMT_F32 = 0,   /* fp32 values, no scales                                      */
  CSA_IFMT_E4M3 = 1,  /* FP8 e4m3 codes (1 byte) + one fp32 scale per row             */
  CSA_IFMT_MXFP4 = 2  /* e2m1 codes packed 2 per byte (element 2i in the low nibble) +
                         one ue8m0 scale byte (2^(code-127)) per 32 consecutive elements */
} csa_ifmt;

/* Bits of the per-device error word. */
#define CSA_DEVERR_INDEX    0x1u  /* a KV / entry index outside [0, n_max): row skipped   */
#define CSA_DEVERR_WINDOW   0x2u  /* a window row outside the raw buffer: row skipped    */
#define CSA_DEVERR_TIMEOUT  0x4u  /* a bounded device-side wait gave up                  */
#define CSA_DEVERR_BAND     0x8u  /* top-k candidate band exceeded its capacity          */
#define CSA_DEVERR_ENTRY    0x10u /* a compressor output entry outside [0, n_max): skipped */

int csa_abi_version(void);
const char* csa_status_string(int status);

/* Reads the calling device's error word into *out (host pointer), then clears
 * it.  Synchronises `stream` (the only call that does).                       */
csa_status csa_read_device_error(void* stream, uint32_t* out);

/* Number of kernels the library has enqueued in this process (all devices and
 * streams; a launch captured into a CUDA graph counts once, at capture).  The
 * paper has no counterpart: it lets a caller check which work ran on the GPU.  */
uint64_t csa_launch_count(void);

/* Device-side waits.  Every kernel that waits (for a TMA copy, a tensor-core MMA or
 * another warp of its CTA) waits on a CTA-local mbarrier with a time limit of 2 s; a
 * wait that runs out sets CSA_DEVERR_TIMEOUT, the kernel waits (again bounded) for its
 * own copies in flight, releases its tensor memory and returns.
 * csa_wait_probe launches one CTA whose single wait nothing can complete, with the
 * limit limit_ns (1e3 .. 2e9 ns, CSA_ERR_SHAPE otherwise): after it the error word
 * holds CSA_DEVERR_TIMEOUT and the device stays usable.  The paper has no
 * counterpart: it lets a caller check that a wait that cannot end returns an error. */
csa_status csa_wait_probe(uint64_t limit_ns, void* stream);

/* csa_tensor_peak_probe — the dense tensor-core rate at the indexer's operand formats,
 * for the rooflines of the scoring kernels.  One CTA per SM issues iters x 128 of K of
 * MMAs on operands resident in shared memory (nothing is read from or written to global
 * memory except the error word): ifmt = CSA_IFMT_E4M3 runs kind::f8f6f4, M 128, N 256
 * (2 * 128 * 256 * 128 * iters FLOP per SM); CSA_IFMT_MXFP4 runs kind::mxf4.block_scale,
 * M 128, N 64 (2 * 128 * 64 * 128 * iters FLOP per SM).  Time it with events on the stream.
 * iters in 1 .. 1e6 (CSA_ERR_SHAPE otherwise); other formats CSA_ERR_DTYPE.  A wait that
 * gives up sets CSA_DEVERR_TIMEOUT.  The pages have no counterpart: it measures the GPU,
 * not the method. */
csa_status csa_tensor_peak_probe(int ifmt, int iters, void* stream);

/* ---------------------------------------------------------------------------
 * csa_compress — CSA token-axis compression fused with the KV-cache append.
 * ("Гибридное внимание: CSA и HCA", CSA step 1: two KV series C^a, C^b and two
 * gate series Z^a, Z^b; per component a softmax over the 2m sources of
 * (Z + learnable positional bias), then the weighted sum; the a/b windows are
 * shifted so that entry i draws on 2m tokens and the length still shrinks m×.)
 *
 * Entry e of a sequence pools, per component c, the b-series of tokens
 * m*e-m .. m*e-1 (bias Bb[j]) and the a-series of tokens m*e .. m*e+m-1
 * (bias Ba[j]), j = offset inside the block.  Entry 0 has no b-half.
 *
 *   Ca, Cb, Za, Zb  device [B, T_new, d] dtype: the chunk's tokens, which start
 *                   at token m*entry0[b] of sequence b; T_new % m == 0
 *   Ba, Bb          device [m, d] fp32 positional biases
 *   prev_Cb, prev_Zb device [B, m, d] dtype: b-series of the block just before
 *                   the chunk (always allocated; its values count only where
 *                   entry0[b] > 0)
 *   entry0          device [B] int32: index of the chunk's first entry
 *   cache           device [B, n_max, d] dtype: rows entry0[b] .. entry0[b]+T_new/m-1
 *                   are written (outputs rounded to nearest-even for bf16)
 * Supported: m in 1..16, d % 8 == 0 (bf16) or d % 4 == 0 (f32).
 * ------------------------------------------------------------------------- */
csa_status csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                        const float* Ba, const float* Bb,
                        const void* prev_Cb, const void* prev_Zb,
                        const int32_t* entry0, void* cache, int64_t n_max,
                        int B, int T_new, int d, int m, int dtype, void* stream);

/* csa_compress_kv8 — csa_compress (m = 4, d = 576) writing the FP8 cache rows that
 * sparse_attn_decode_kv8 reads ("Гибридный attention: CSA и HCA" of the aixai.ru
 * digest: KV entries in FP8, RoPE dimensions in BF16).  Row entry0[b] + i of
 * cache8 [B, n_max, 656] receives the 656-byte form of the pooled fp32 row (layout
 * and exponent rule at sparse_attn_decode_kv8); codes round to nearest even and
 * saturate, a value that rounds to zero gets code 0.  Other arguments as csa_compress.
 * Supported: d == 576 and m == 4 (CSA_ERR_UNSUPPORTED otherwise).                   */
csa_status csa_compress_kv8(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                            const float* Ba, const float* Bb,
                            const void* prev_Cb, const void* prev_Zb,
                            const int32_t* entry0, void* cache8, int64_t n_max,
                            int B, int T_new, int d, int m, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * csa_decode_append — the cache and window appends of one decode step, in one launch.
 * The current token completes block entry0[b] (m = 4) of sequence b; the call writes
 *   - cache row entry0[b]: csa_compress of that block (Ca, Cb, Za, Zb [B, 4, d], the
 *     previous block's b-series prev_Cb, prev_Zb [B, 4, d], biases Ba, Bb [4, d]);
 *   - when CaI != NULL, indexer key row entry0[b] of kI / kI_scale: index_key_compress of
 *     the block's indexer activations (CaI .. prev_ZbI [B, 4, d_I], BaI, BbI [4, d_I]) in
 *     format ifmt ("FP4 с учётом квантования": the keys of compressed entries are cached);
 *   - when raw_new != NULL, window row win_slot[b] of win [B, W, d]: the token's raw latent
 *     raw_new [B, d] ("Гибридное внимание: CSA и HCA": the sliding window of uncompressed
 *     entries).  The window is a ring: the token at position p goes to slot p mod W, and
 *     the attention calls read its rows in any order.  A slot outside [0, W) is skipped
 *     and sets CSA_DEVERR_WINDOW.
 * Each part is the same arithmetic as its own call (csa_compress with T_new = 4,
 * index_key_compress, a row copy).
 * Supported: d / (8 for bf16, 4 for f32) <= 96; d_I as index_key_compress.
 * ------------------------------------------------------------------------- */
csa_status csa_decode_append(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                             const float* Ba, const float* Bb, const void* prev_Cb, const void* prev_Zb,
                             const int32_t* entry0, void* cache, int64_t n_max, int d,
                             const void* CaI, const void* CbI, const void* ZaI, const void* ZbI,
                             const float* BaI, const float* BbI, const void* prev_CbI, const void* prev_ZbI,
                             void* kI, void* kI_scale, int d_I, int ifmt,
                             const void* raw_new, void* win, const int32_t* win_slot, int W,
                             int B, int dtype, void* stream);

/* window_append — the window part of csa_decode_append alone (for the HCA window):
 * win[b, win_slot[b], :] = raw_new[b, :], raw_new [B, d], win [B, W, d].              */
csa_status window_append(const void* raw_new, void* win, const int32_t* win_slot, int B, int W, int d,
                         int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * hca_compress — HCA compression ("HCA: сжать в 128 раз, но смотреть на всё":
 * the same gated pooling with m' tokens per entry and no overlap).
 *
 *   C, Z    device [B, T_new, d] dtype, T_new % m_prime == 0, starting at token
 *           m_prime*entry0[b]
 *   bias    device [m_prime, d] fp32
 *   cache   device [B, n_max, d]: rows entry0[b] .. entry0[b]+T_new/m_prime-1 written
 * Supported: m_prime in 1..1024.
 * ------------------------------------------------------------------------- */
csa_status hca_compress(const void* C, const void* Z, const float* bias,
                        const int32_t* entry0, void* cache, int64_t n_max,
                        int B, int T_new, int d, int m_prime, int dtype, void* stream);

/* ---------------------------------------------------------------------------
 * index_key_compress — the indexer keys of the entries a chunk completes
 * ("FP4 с учётом квантования": the indexer's Q·K activations are cached and
 * multiplied in FP4, MXFP4 with 1x32 tiles; the keys belong to the compressed
 * entries, so they come from the CSA step-1 pooling of the indexer activations).
 *
 * The pooling is csa_compress's with m = 4, over indexer activations of width
 * d_I; the pooled fp32 row is quantised in the same kernel to the format that
 * lightning_index reads:
 *   CSA_IFMT_E4M3:  scale = amax(|row|)/448 (1 for an all-zero row), one fp32
 *                   per row; code = round-to-nearest-even(x / scale) in e4m3;
 *   CSA_IFMT_MXFP4: per 32 components e = the smallest integer with
 *                   amax <= 6 * 2^e (clamped to [-127, 127]; -127 for zeros),
 *                   scale byte e + 127; code = RNE e2m1 of x * 2^-e.
 * Decisions are made on the fp32 pooled values; a value that rounds to zero is
 * written as +0 (code 0).
 *
 *   Ca, Cb, Za, Zb   device [B, T_new, d_I] dtype (indexer activations and gates)
 *   Ba, Bb           device [4, d_I] fp32 positional biases
 *   prev_Cb, prev_Zb device [B, 4, d_I] dtype (as in csa_compress)
 *   entry0           device [B] int32: index of the chunk's first entry
 *   kI               device [B, n_max, d_I] bytes (E4M3) or [B, n_max, d_I/2] (MXFP4)
 *   kI_scale         device [B, n_max] fp32 (E4M3) or [B, n_max, d_I/32] bytes (MXFP4)
 *                    rows entry0[b] .. entry0[b]+T_new/4-1 are written; an entry
 *                    outside [0, n_max) is skipped and sets CSA_DEVERR_ENTRY
 * Supported: m == 4 (CSA_ERR_UNSUPPORTED otherwise), d_I in {32, 64, 128} (and
 * 256 for bf16).  All pointers 16-byte aligned.
 * ------------------------------------------------------------------------- */
csa_status index_key_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                              const float* Ba, const float* Bb,
                              const void* prev_Cb, const void* prev_Zb,
                              const int32_t* entry0, void* kI, void* kI_scale, int64_t n_max,
                              int B, int T_new, int d_I, int m, int dtype, int ifmt, void* stream);

/* ---------------------------------------------------------------------------
 * KV-sharded decode of one sequence over G GPUs: the two merge steps.  The
 * entries are split into G contiguous shards (shard g holds global entries
 * bounds[g] .. bounds[g+1]-1).  Every GPU runs lightning_index on its shard with
 * score_out, the candidates are all-gathered, and:
 *
 * shard_topk_merge — the global top-k ("Гибридное внимание: CSA и HCA", CSA step 2:
 *   the k largest scores, ties to the lower entry id) of the G x k candidates.
 *     idx_parts   device [G, R, k] int32 local ids (-1 = no candidate)
 *     score_parts device [G, R, k] fp32 their scores (lightning_index score_out)
 *     bounds      device [G + 1] int32 shard boundaries (global entry ids)
 *     local_idx_out device [G, R, k] int32: for shard g, the selected entries of
 *                 that shard as local ids in ascending order, -1 padded
 *   Supported: G <= CSA_SHARD_MAX_G, G * k <= CSA_SHARD_MAX_CANDIDATES, R <= 65535.
 *
 * attn_merge_shards — the attention over the union of the shards' rows from the
 *   shards' outputs o_g (each normalised over its own rows) and their lse_g:
 *   out = sum_g e^{lse_g - L} o_g, L = log sum_g e^{lse_g} (written to lse_out if
 *   not NULL).  The sink and the window belong to one shard; the others pass a
 *   very negative finite sink (e.g. -1e30), so that a shard without rows returns
 *   o = 0 with lse = -1e30 and weighs nothing.
 *     o_parts device [G, rows, dv] dtype;  lse_parts device [G, rows] fp32
 *     out device [rows, dv] dtype (rows = B * H)
 * Both calls accept 1 <= G <= CSA_SHARD_MAX_G (CSA_ERR_SHAPE otherwise).
 * ------------------------------------------------------------------------- */
#define CSA_SHARD_MAX_G 8                 /* shards G of one sequence, both merges       */
#define CSA_SHARD_MAX_CANDIDATES 4096     /* G * k of shard_topk_merge                   */
csa_status shard_topk_merge(const int32_t* idx_parts, const float* score_parts, const int32_t* bounds,
                            int G, int R, int k, int32_t* local_idx_out, void* stream);
csa_status attn_merge_shards(const void* o_parts, const float* lse_parts, int G, int64_t rows, int dv,
                             int dtype, void* out, float* lse_out, void* stream);

/* ---------------------------------------------------------------------------
 * grouped_out_proj — the grouped output projection after the attention
 * ("Гибридное внимание: CSA и HCA", CSA step 4: the n_h head outputs are split
 * into g groups, each group is projected to an intermediate width d_mid, and the
 * concatenation of the groups is projected to the hidden size d; table
 * "Конфигурации": g = 16, d_mid = 1024, head size 512, d = 7168 for Pro).
 *
 *   u[t, j*d_mid + i] = sum_k W1[j*d_mid + i, k] * o[t, j*(H/g)*dv + k],  k < (H/g)*dv
 *   y[t, r]           = sum_k W2[r, k] * u[t, k],                          k < g*d_mid
 *
 *   o   device [T, H, dv] bf16 (the attention output; o[t] read as one row of H*dv)
 *   W1  device [g*d_mid, (H/g)*dv] bf16 (group j's matrix is rows j*d_mid ..)
 *   W2  device [d, g*d_mid] bf16
 *   u   device [T, g*d_mid] bf16, written (the intermediate, rounded to bf16)
 *   y   device [T, d] bf16, written (fp32 accumulation, rounded to nearest even)
 *   workspace  NULL, or >= grouped_out_proj_workspace_size(T, g, d_mid, d) bytes:
 *              with it, batches of at most 256 tokens split the weight stream
 *              over more SMs (fp32 partials added in a fixed order)
 * Supported: (H/g)*dv % 64 == 0, d_mid % 128 == 0, d % 128 == 0
 * (CSA_ERR_UNSUPPORTED otherwise).  All pointers 16-byte aligned.
 * ------------------------------------------------------------------------- */
size_t grouped_out_proj_workspace_size(int T, int g, int d_mid, int d);
csa_status grouped_out_proj(const void* o, int T, int H, int dv, int g, int d_mid,
                            const void* W1, const void* W2, int d, void* u, void* y,
                            void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * lightning_index — indexer scores and top-k selection of compressed entries
 * ("Гибридное внимание: CSA и HCA", CSA step 2: the DSA lightning indexer
 * scores I[t,s] with a ReLU and keeps the top-k compressed blocks; FP4 Q·K
 * path from "FP4 с учётом квантования").
 *
 *   I[t,s] = sum_j w[t,j] * max(0, <q[t,j], k[s]>)   (dequantised operands)
 *
 * Query t of sequence b at absolute position pos = q_pos[b*Tq+t] sees entries
 * s < min(n_entries[b], (pos+1)/m) (all of an entry's tokens are <= pos).  The
 * k entries with the largest I are returned, ties to the lower index, in
 * ascending index order, padded with -1.  Selection is exact: tensor-core fp32
 * scores pick a candidate band which is re-scored exactly on CUDA cores
 * (integer dot products of the E4M3 / MXFP4 codes, fp64 for F32 operands).
 *
 * Stream order: for decode rows (Tq <= 3, E4M3 or MXFP4) the scoring kernel is
 * launched with programmatic dependent launch.  It may start while the kernel
 * before it in the stream is still running, and it waits for that kernel to
 * finish before it reads the key tile holding each row's newest eligible
 * entry and before any write.  So the preceding kernel may produce only those
 * newest keys (csa_decode_append does); every other input must be complete
 * before it starts, as it is after any kernel that does not trigger its
 * dependents early.
 *
 *   qI       device [B, Tq, H_I, d_I] (F32: fp32; E4M3: bytes; MXFP4: [.., d_I/2] bytes)
 *   qI_scale E4M3: device [B, Tq, H_I] fp32; MXFP4: [B, Tq, H_I, d_I/32] bytes; F32: NULL
 *   w        device [B, Tq, H_I] fp32 head weights
 *   kI       device [B, n_max, d_I] (same format; MXFP4 [B, n_max, d_I/2])
 *   kI_scale E4M3: device [B, n_max] fp32; MXFP4: [B, n_max, d_I/32] bytes; F32: NULL
 *   n_entries device [B] int32, q_pos device [B, Tq] int32
 *   idx_out  device [B, Tq, k] int32;  score_out device [B, Tq, k] fp32 or NULL
 *            (the fp64 score of each selected entry rounded to fp32; 0 for pads)
 *   workspace >= lightning_index_workspace_size(B, Tq, n_max, k) bytes (or, with
 *            score_out NULL, lightning_index_workspace_size_exact(...) bytes)
 * Supported: B*Tq <= 65535, H_I <= 64, d_I in {32, 64, 128}, k <= 2048,
 * n_max <= 2^24.  qI, kI, score_out and workspace must be 16-byte aligned
 * (CSA_ERR_ALIGN otherwise).
 * ------------------------------------------------------------------------- */
size_t lightning_index_workspace_size(int B, int Tq, int64_t n_max, int k);
/* The bytes lightning_index itself (score_out NULL) needs for these shapes on the current
 * device: prefill rows whose selection streams candidates instead of scores (E4M3 keys,
 * H_I 64, d_I 128, k <= 1024, Tq >= 4 and enough rows to fill the device) need no score
 * region, about B*Tq*n_max*4 bytes less; otherwise the same as
 * lightning_index_workspace_size.  A call with score_out, or lightning_index_bf16, needs
 * lightning_index_workspace_size.  0 for empty shapes. */
size_t lightning_index_workspace_size_exact(int B, int Tq, int64_t n_max, int k, int ifmt, int H_I, int d_I);
csa_status lightning_index(const void* qI, const void* qI_scale, const float* w,
                           const void* kI, const void* kI_scale,
                           const int32_t* n_entries, const int32_t* q_pos, int m,
                           int B, int Tq, int H_I, int d_I, int64_t n_max, int k, int ifmt,
                           int32_t* idx_out, float* score_out,
                           void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * lightning_index_bf16 — the same scores rounded to bf16 before the top-k
 * ("FP4 с учётом квантования": the indexer's scores are converted from FP32 to
 * BF16, which makes the top-k selection faster while keeping nearly all of the
 * needed entries).  Not the exact selection of lightning_index: the k largest
 * bf16 keys bf16(I[t,s]) are kept, ties to the lower index, so entries whose
 * scores differ by less than the bf16 resolution are ordered by index.  I is
 * the scoring kernel's fp32 score (rounded to nearest even); a score within
 * the fp32 accumulation error of a bf16 rounding midpoint may round either way.
 * Arguments, layouts, workspace and errors as lightning_index (no score_out).
 * ------------------------------------------------------------------------- */
csa_status lightning_index_bf16(const void* qI, const void* qI_scale, const float* w,
                                const void* kI, const void* kI_scale,
                                const int32_t* n_entries, const int32_t* q_pos, int m,
                                int B, int Tq, int H_I, int d_I, int64_t n_max, int k, int ifmt,
                                int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * topk_select — exact top-k of fp32 scores (CSA step 2's selection on its own).
 *   scores   device [R, ld] fp32; row r has n_valid[r] valid leading entries
 *   idx_out  device [R, k] int32: the k largest, ties to the lower index,
 *            ascending index order, -1 padding.  NaN ranks below every number.
 * Supported: k <= 2048, n <= 2^24.
 * ------------------------------------------------------------------------- */
size_t topk_select_workspace_size(int R, int64_t n, int k);
csa_status topk_select(const float* scores, int64_t ld, const int32_t* n_valid,
                       int R, int64_t n, int k, int32_t* idx_out,
                       void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Attention over compressed entries + raw window + sink ("Гибридное внимание:
 * CSA и HCA", CSA step 3: every compressed entry is key and value for all query
 * heads (MQA); the 128-token window of uncompressed entries; the attention sink
 * and the 576 = 512 + 64 latent of "Технический отчёт DeepSeek-V4 — часть 1/2").
 *
 * For head h of a query, over the row set R (selected / all compressed entries
 * plus window rows):  l_r = sm_scale * <q_h, row_r[0:d_k]>,
 *   out_h = sum_r e^{l_r - M} row_r[0:d_v] / (e^{sink_h - M} + sum_r e^{l_r - M}),
 *   M = max(sink_h, max_r l_r),   lse_h = M + log(e^{sink_h-M} + sum_r e^{l_r-M}).
 * Pass sink = -INFINITY for no sink.  out is rounded to dtype; lse is fp32.
 * Supported: H <= 128, d_v <= d_k <= 576, d_k % 8 == 0.  The tcgen05 path runs
 * for bf16 with H == 128, d_k == 576, d_v == 512; other shapes run a CUDA-core path.
 * ------------------------------------------------------------------------- */

/* Workspace for the split-KV partials of the decode calls: sparse_attn_decode needs
 * attn_decode_workspace_size(B, H, d_v, k + W) bytes and hca_attn_decode
 * attn_decode_workspace_size(B, H, d_v, n_max + W); CSA_ERR_WORKSPACE otherwise.
 * sparse_attn_prefill takes no workspace (pass NULL, 0).                         */
size_t attn_decode_workspace_size(int B, int H, int d_v, int64_t rows_max);

/* sparse_attn_decode — one query token per sequence.
 *   q       device [B, H, d_k];  cache device [B, n_max, d_k]
 *   idx     device [B, k] int32 entry ids (-1 = unused slot)
 *   win     device [B, W, d_k]: raw latents of the last win_len[b] positions
 *   win_len device [B] int32 (0..W)
 *   sink    device [H] fp32
 *   out     device [B, H, d_v];  lse device [B, H] fp32 or NULL
 * Ordering: when the preceding kernel in the stream allows programmatic dependent
 * launch (lightning_index's selection does), this call overlaps it and waits for it
 * only before it reads idx: q, cache, win, win_len and sink must not be written by that
 * kernel (they may be written by any earlier one).                                   */
csa_status sparse_attn_decode(const void* q, const void* cache, const int32_t* idx,
                              const void* win, const int32_t* win_len, const float* sink,
                              int B, int H, int d_k, int d_v, int64_t n_max, int k, int W,
                              float sm_scale, int dtype, void* out, float* lse,
                              void* workspace, size_t ws_bytes, void* stream);

/* hca_attn_decode — dense attention over entries 0..n_entries[b]-1 + window.
 *   n_entries device [B] int32 (<= n_max); other arguments as sparse_attn_decode. */
csa_status hca_attn_decode(const void* q, const void* cache, const int32_t* n_entries,
                           const void* win, const int32_t* win_len, const float* sink,
                           int B, int H, int d_k, int d_v, int64_t n_max, int W,
                           float sm_scale, int dtype, void* out, float* lse,
                           void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * sparse_attn_decode_kv8 / hca_attn_decode_kv8 — the same attention over an FP8
 * cache ("Гибридный attention: CSA и HCA" of the aixai.ru digest: KV entries are
 * stored in FP8, only the RoPE dimensions in BF16).
 *
 *   cache8  device [B, n_max, 656] bytes per entry: bytes 0..511 the e4m3 codes of
 *           row[0:512] / 2^e, bytes 512..639 row[512:576] as bf16 (little endian),
 *           byte 640 = e + 127 (e in [-126, 127]), bytes 641..655 zero.  The stored
 *           row is codes * 2^e (exact) followed by the bf16 RoPE values.
 * The window rows stay bf16 ([B, W, d_k]).  Each FP8 row is expanded to bf16 in
 * shared memory as it is gathered; the arithmetic is that of the bf16 calls.
 * Other arguments as sparse_attn_decode / hca_attn_decode with dtype bf16.
 * Supported: H == 128, d_k == 576, d_v == 512 (CSA_ERR_UNSUPPORTED otherwise).
 * ------------------------------------------------------------------------- */
csa_status sparse_attn_decode_kv8(const void* q, const void* cache8, const int32_t* idx,
                                  const void* win, const int32_t* win_len, const float* sink,
                                  int B, int H, int d_k, int d_v, int64_t n_max, int k, int W,
                                  float sm_scale, void* out, float* lse,
                                  void* workspace, size_t ws_bytes, void* stream);
csa_status hca_attn_decode_kv8(const void* q, const void* cache8, const int32_t* n_entries,
                               const void* win, const int32_t* win_len, const float* sink,
                               int B, int H, int d_k, int d_v, int64_t n_max, int W,
                               float sm_scale, void* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream);

/* hca_compress_attn_decode — one HCA decode step: hca_compress of the fresh chunk
 * into the cache, then hca_attn_decode over entries 0..n_entries[b]-1 (which include
 * the fresh rows) + window + sink; the same results as the two calls in that order.
 * The attention kernel starts while the compression runs: its CTAs stream the rows the
 * compression does not write and wait for the compression only before the tile that
 * holds rows entry0[b] .. entry0[b] + T_new/m_prime - 1.
 *   C, Z, bias, entry0, T_new, m_prime  as hca_compress (d = d_k, same dtype as q)
 *   other arguments                     as hca_attn_decode                          */
csa_status hca_compress_attn_decode(const void* C, const void* Z, const float* bias,
                                    const int32_t* entry0, int T_new, int m_prime,
                                    const void* q, void* cache, const int32_t* n_entries,
                                    const void* win, const int32_t* win_len, const float* sink,
                                    int B, int H, int d_k, int d_v, int64_t n_max, int W,
                                    float sm_scale, int dtype, void* out, float* lse,
                                    void* workspace, size_t ws_bytes, void* stream);

/* sparse_attn_prefill — Tq query tokens per sequence, each with its own index set.
 *   q        device [B, Tq, H, d_k];  q_pos device [B, Tq] int32 absolute positions
 *   idx      device [B, Tq, k] int32 (-1 = unused)
 *   raw      device [B, t_raw, d_k]: raw latents of positions raw_pos0[b] ..
 *            raw_pos0[b]+t_raw-1 (raw_pos0 device [B] int32)
 *   The window of a query at pos is positions max(0, pos-W+1) .. pos.
 *   out      device [B, Tq, H, d_v];  lse device [B, Tq, H] fp32 or NULL       */
csa_status sparse_attn_prefill(const void* q, const int32_t* q_pos, const void* cache,
                               const int32_t* idx, const void* raw, int64_t t_raw,
                               const int32_t* raw_pos0, const float* sink,
                               int B, int Tq, int H, int d_k, int d_v, int64_t n_max, int k,
                               int W, float sm_scale, int dtype, void* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * sparse_attn_decode_noalloc — sparse_attn_decode without a caller workspace.
 * The paper has no counterpart to this call; it exists for callers that cannot
 * allocate device memory: code running inside another framework's memory pool,
 * latency-critical paths that must never call cudaMalloc (which can synchronise
 * the device), or deployments whose device memory is budgeted up front.
 *
 * Arguments, results and rules are those of sparse_attn_decode, minus the
 * workspace.  The split-KV partials go to a buffer the library owns: a fixed
 * array of CSA_NOALLOC_SCRATCH_BYTES in device memory, held by every GPU that
 * loads the library until the process exits.
 * - Limit: when attn_decode_workspace_size(B, H, d_v, k + W) exceeds
 *   CSA_NOALLOC_SCRATCH_BYTES the call returns CSA_ERR_WORKSPACE and enqueues
 *   nothing.  Example: batch 16 with 128 heads, d_v = 512 and k + W = 640 needs
 *   about 17 MB.
 * - The first call on each device looks up the buffer's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture: inside a capture the lookup can fail, and the
 *   call then returns CSA_ERR_CUDA.  Later calls only read the cached address.
 * - The cached address belongs to the device's primary context: after
 *   cudaDeviceReset on that device the address is stale, and so is the error
 *   word every call uses.  Do not call the library after a reset in the same
 *   process.
 * - All calls on a device share the one buffer, and it keeps the last call's
 *   contents.  Every call rewrites all it reads, so nothing must be cleared.
 *   Calls that overlap on the GPU (different streams, or different host threads
 *   on the same device) race on the buffer: serialise them.
 * - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 * ------------------------------------------------------------------------- */
#define CSA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
csa_status sparse_attn_decode_noalloc(const void* q, const void* cache, const int32_t* idx,
                                      const void* win, const int32_t* win_len, const float* sink,
                                      int B, int H, int d_k, int d_v, int64_t n_max, int k, int W,
                                      float sm_scale, int dtype, void* out, float* lse, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA_B200_H */
