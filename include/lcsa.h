/*
 * lcsa.h - C ABI of liblcsa, the B200 (sm_100a) hot path of the DeepSeek-V4
 * hybrid compressed attention: CSA (compressed sparse attention) and HCA
 * (heavily compressed attention).
 *
 * Sources, cited below by tag (web pages about DeepSeek-V4):
 *   [p1] "DeepSeek V4的4个技巧", section 1 "技巧1：混合注意力"
 *   [p2] "深度解析 DeepSeek-V4：百万级长文本的低成本突破", sections
 *        "CSA：Compressed Sparse Attention" (Step 1 Compress, Step 2 Select,
 *        ASCII figure), "HCA：Heavily Compressed Attention",
 *        "Sliding Window Branch", "Attention Sink"
 *   [p3] untitled classical-Chinese paraphrase page: the "Partial RoPE",
 *        "Attention sink", "第一步/第二步/第三步" step sentences, and the
 *        strict-causality, HCA-no-overlap and sliding-window sentences
 *   [p4] "DeepSeek V4 技术架构深度解析", section "二、CSA + HCA" (with
 *        "KV Cache优化细节")
 *
 * Conventions shared by every call
 *   - Every tensor argument is a DEVICE pointer, allocated and owned by the
 *     caller; the library never allocates device memory.  Tensors are dense
 *     row-major with the last dimension contiguous.  Every tensor pointer and
 *     every row must be 16-byte aligned (rows of D elements: D*elem % 16 == 0).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous and stream-ordered.
 *   - Argument errors are detected on the host before anything is launched and
 *     returned synchronously (LCSA_ERR_INVALID_ARG / LCSA_ERR_UNSUPPORTED /
 *     LCSA_ERR_WORKSPACE); a failed launch returns LCSA_ERR_CUDA.  Problems a
 *     kernel detects while running (a bounded wait that gave up, an index out
 *     of range) are written to a per-device status word that
 *     lcsa_get_device_status() reads; the kernel skips the bad access.
 *   - Positions are absolute token positions (int64).  Compressed entry j of a
 *     stride-m cache sits at position j*m and is visible to the query at
 *     position t iff j < floor(t/m) ([p3] strict causality: a query never sees
 *     the tokens of its own compressed block).
 *   - Storage dtypes: LCSA_BF16 (BF16 storage, FP32 arithmetic) or LCSA_FP32.
 *     BF16 with the layer's shapes (H=64, D=512, R=64; indexer H_I=64,
 *     D_I=128) runs on tcgen05 tensor cores; other shapes and FP32 run on
 *     FP32 CUDA-core kernels.  There is no CPU path: without a CUDA device every
 *     compute call returns LCSA_ERR_CUDA.
 */
#ifndef LCSA_H
#define LCSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LCSA_OK = 0,
  LCSA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size           */
  LCSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented combination         */
  LCSA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required    */
  LCSA_ERR_CUDA = 4,          /* launch failure / no device                    */
  LCSA_ERR_DEVICE = 5         /* device status word holds an error             */
} lcsa_status;

typedef enum { LCSA_FP32 = 0, LCSA_BF16 = 1 } lcsa_dtype;

/* Device status codes (lcsa_get_device_status). */
#define LCSA_DEV_OK 0
#define LCSA_DEV_TIMEOUT 1        /* a bounded mbarrier / flag wait gave up     */
#define LCSA_DEV_BAD_INDEX 2      /* a selected index was >= Nc (skipped)       */

const char* lcsa_version(void);
const char* lcsa_status_string(lcsa_status s);

/* Number of kernels this library has launched in the calling process (all
 * devices, all streams).  Benchmarks read it before and after a timed region
 * to report how many of the library's kernels ran inside it. */
uint64_t lcsa_kernel_launches(void);

/* Synchronises `stream`, returns the current device's status word in *code
 * (LCSA_DEV_*) and clears it.  Returns LCSA_ERR_DEVICE when *code != 0. */
lcsa_status lcsa_get_device_status(void* stream, int* code);

/* Limit of every bounded wait (an mbarrier or a pipeline hand-off) in the
 * library's kernels on the current device, in nanoseconds of the GPU's global
 * timer: a wait that lasts longer gives up, the kernel records
 * LCSA_DEV_TIMEOUT, stops issuing work, lets its copies in flight land, frees
 * its tensor memory and returns, so the context stays usable.  Default 2 s;
 * ns = 0 restores it.  A synchronous copy to the device: call it outside
 * stream capture, with no library kernel running on the device. */
lcsa_status lcsa_set_wait_limit_ns(uint64_t ns);

/* Test hook of the bounded waits: the next launch of the grouped output
 * projection's GEMM kernel (lcsa_grouped_out_proj's first GEMM) leaves the
 * pipeline stage of k-chunk `chunk` of its first CTA unfilled (no copy, no
 * arrival), so every wait on that stage runs out.  The call then returns,
 * lcsa_get_device_status reports LCSA_DEV_TIMEOUT and the output is
 * undefined; later calls are unaffected.  chunk < 0 clears a pending hook. */
void lcsa_test_withhold_stage(int chunk);

/* How CSA sparse attention on BF16 entries stages its selected rows (the
 * entries chosen by top-k, [p2] CSA Step 3; the pages leave the copy
 * mechanism open): mode 0 (default) gathers each 64-row tile with 16-byte
 * cp.async copies from all producer warps; mode 1 uses TMA tile::gather4
 * (four 128-byte rows per copy, 128 copies per tile, issued by the same
 * warps).  Both give identical results; mode 0 is the faster on B200 and
 * mode 1 is kept for measurement.  Process-wide; applies to calls issued
 * after it.  Any other value: LCSA_ERR_INVALID_ARG. */
lcsa_status lcsa_set_attn_gather(int mode);

/* How lcsa_indexer_topk_mxfp4 feeds its MXFP4 keys to the tensor cores
 * (the pages give the FP4 QK path, [p2] "FP4 Quantization-Aware Training",
 * not its kernel): mode 0 (default) stages every key as FP8 E4M3 relative
 * to its largest block scale before an E4M3 MMA; mode 1 hands calls of one
 * or two query rows per sequence (decode) to a block-scaled MMA that reads
 * the E2M1 codes and their UE8M0 block scales as they are.  Scores agree to
 * FP32 rounding order, and mode 1 stays exact where mode 0 rounds a block
 * more than 2^13 below its entry's largest; mode 0 is the faster on B200.
 * Process-wide; applies to calls issued after it.  Any other value:
 * LCSA_ERR_INVALID_ARG. */
lcsa_status lcsa_set_fp4_mma(int mode);

/* ------------------------------------------------------------------------
 * KV compression ([p2] CSA Step 1: m consecutive tokens merged into one entry
 * with learned softmax weights; [p2] HCA: m' = 128 tokens per entry; [p3]
 * "第一步，KV压缩" and the sentence that HCA pools every m' tokens without
 * CSA's overlap).
 *
 *   c[b,j,d] = sum_{i in S_j} softmax_{i in S_j}(gate[b,i,d]) * kv[b,i,d]
 *   CSA: S_j = [(j-1)m, (j+1)m) clipped at 0 (window 2m, stride m)
 *   HCA: S_j = [j m, (j+1) m)              (non-overlapping)
 * for j < floor(T/m) (entries exist only for complete own-blocks).  With
 * rms_weight != NULL the entry is RMS-normalised, c / sqrt(mean(c^2)+eps) * w
 * ([p2] "Attention Sink" section: RMSNorm on the compressed KV entries).
 *
 *   kv   [B,T,D] dtype          gate [B,T,D] dtype (gate_per_channel=1) or
 *                               [B,T] dtype (one logit per token, =0)
 *   out  [B,floor(T/m),D] out_dtype
 * Constraints: D*elem % 16 == 0, m >= 1, T >= 0.
 * ------------------------------------------------------------------------ */
lcsa_status lcsa_csa_compress(const void* kv, const void* gate, int gate_per_channel,
                              int B, int T, int D, int m, lcsa_dtype dtype,
                              const float* rms_weight, float rms_eps,
                              void* out, lcsa_dtype out_dtype, void* stream);
lcsa_status lcsa_hca_compress(const void* kv, const void* gate, int gate_per_channel,
                              int B, int T, int D, int m, lcsa_dtype dtype,
                              const float* rms_weight, float rms_eps,
                              void* out, lcsa_dtype out_dtype, void* stream);

/* ------------------------------------------------------------------------
 * Incremental KV compression for decode: the pooling above, for the entries
 * whose windows a buffer of recent raw rows covers.  A decode loop appends
 * entry j = t/m - 1 of a CSA or HCA cache once the token at position t-1 has
 * arrived and t % m == 0 (the pages' m-token compression applied as tokens
 * arrive; the window ring of raw rows kept for the sliding-window branch
 * holds every token such an entry needs when W >= window).
 *
 * Computes c[b,j,:] for j in [j0, j0 + n_entries) with
 *   S_j = [(j+1)m - window, (j+1)m) clipped at 0
 * (window 2m for CSA, m for HCA; any window >= 1).  Buffer row i of every
 * sequence holds position kv_pos0 + i, and every position of every S_j must
 * lie in [kv_pos0, kv_pos0 + Tkv).
 *
 *   kv    [B,Tkv,D] dtype          gate [B,Tkv,D] dtype (gate_per_channel=1)
 *                                  or [B,Tkv] dtype (=0)
 *   cache [B,cache_rows,D] out_dtype; entry j is written at row j, nothing
 *         else is touched
 * Returns LCSA_ERR_INVALID_ARG when a window leaves the buffer, when
 * j0 < 0 or j0 + n_entries > cache_rows, or on the layout constraints of
 * lcsa_csa_compress.  Buffers are caller-owned; the call is stream-ordered.
 * ------------------------------------------------------------------------ */
lcsa_status lcsa_compress_entries(const void* kv, const void* gate, int gate_per_channel,
                                  int B, int Tkv, int D, int64_t kv_pos0, int m, int window,
                                  int64_t j0, int n_entries, lcsa_dtype dtype,
                                  const float* rms_weight, float rms_eps,
                                  void* cache, int64_t cache_rows, lcsa_dtype out_dtype, void* stream);

/* ------------------------------------------------------------------------
 * Top-k selection ([p2] CSA Step 2 and its ASCII figure: keep only the top-k
 * scored entries; [p1] section 1: the top 2048 blocks).
 *
 * For every row r: the k column indices of the largest scores among columns
 * [0, n_valid[r]), ties broken to the lower index, written ascending to
 * idx_out[r, 0:k] and padded with -1 when n_valid[r] < k.  -0.0 equals +0.0.
 * Scores must not be NaN.  The selection is exact (radix select on the
 * order-preserving 32-bit key), so two calls on identical scores agree bit
 * for bit with any other exact implementation.
 *
 *   scores  [rows, ld] fp32 (row stride ld >= n_cols)
 *   n_valid [rows] int32 device, or NULL (= n_cols for every row)
 *   idx_out [rows, k] int32
 *
 * lcsa_topk_workspace returns the device scratch (bytes, 16-byte aligned)
 * that lets rows longer than 32768 columns take the two-phase path (top k of
 * every 32768-column chunk, then of their union); it is 0 when that path does
 * not apply (short rows, k not a multiple of 4, more than 32768/k chunks).
 * Without it, long rows use a single-phase kernel with the same result.
 * The workspace is owned by the caller and must stay valid until the work on
 * `stream` is done.
 * ------------------------------------------------------------------------ */
size_t lcsa_topk_workspace(int rows, int n_cols, int k);
lcsa_status lcsa_topk_from_scores(const float* scores, int rows, int n_cols, int64_t ld,
                                  const int32_t* n_valid, int k, int32_t* idx_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Lightning Indexer + top-k ([p2] CSA Step 2; [p3] "第二步，lightning indexer
 * + top-k选择" and the sentence on scoring every compressed block against
 * each query token; [p4] "二、CSA + HCA": the indexer QK path and its scores).
 *
 *   s[b,t,j] = sum_h w[b,t,h] * relu(q_I[b,t,h,:] . k_I[b,j,:]),  j < N_vis(t)
 *   N_vis(t) = min(Nc, floor(t/m)),  t = q_pos0 + row
 * then the top-k of every row as lcsa_topk_from_scores does, on the FP32
 * scores.  BF16 inputs are multiplied exactly and accumulated in FP32.
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* q_idx;     /* [B,Tq,H_I,D_I] dtype                                 */
  const float* w;        /* [B,Tq,H_I] fp32 head weights                          */
  const void* k_idx;     /* [B,Nc,D_I] dtype, one indexer key per entry            */
  int B, Tq, Nc, H_I, D_I;
  lcsa_dtype dtype;
  int64_t q_pos0;        /* absolute position of query row 0 (every sequence)    */
  int m;                 /* entry stride, for the visibility rule                */
  int k;                 /* entries kept per query                               */
  int32_t* idx_out;      /* [B,Tq,k] int32, ascending, -1 padded                 */
  float* scores_out;     /* optional [B,Tq,Nc] fp32; columns >= N_vis(t) undefined */
} lcsa_indexer_args;

size_t lcsa_indexer_topk_workspace(const lcsa_indexer_args* a);
lcsa_status lcsa_indexer_topk(const lcsa_indexer_args* a, void* workspace,
                              size_t workspace_bytes, void* stream);
int lcsa_indexer_uses_tensor_cores(const lcsa_indexer_args* a);

/* ------------------------------------------------------------------------
 * MXFP4 quantisation for the FP4 indexer QK path ([p2] "FP4
 * Quantization-Aware Training": the indexer's query-key scores are computed
 * in FP4 E2M1 with block scale factors; [p4] "三、FP4量化": E2M1 = 2 exponent
 * bits + 1 mantissa bit, and the CSA indexer QK path goes from FP32 to FP4).
 * The pages give no block size or scale encoding; this is the OCP
 * Microscaling MXFP4 format:
 *   - 32 consecutive values of a row form a block with scale 2^X,
 *     X = floor(log2(max |x|)) - 2 clamped to [-127, 127] (-127 for an
 *     all-zero block), stored as the byte X + 127;
 *   - each value is the E2M1 number nearest to x / 2^X (ties to an even
 *     mantissa bit, magnitudes above 6 saturate), sign bit = (x < 0);
 *   - a block holding Inf or NaN gets scale byte 255 and zero codes.
 *
 *   x      [rows, cols] dtype (cols a multiple of 32), device, aligned to its
 *          element size
 *   codes  [rows, cols/2] uint8, device: element 2i in the low nibble of byte i
 *   scales [rows, cols/32] uint8, device
 * Codes and scales are a pure function of x (bit-exact with any other exact
 * implementation of the definition above).
 * ------------------------------------------------------------------------ */
lcsa_status lcsa_quantize_mxfp4(const void* x, int64_t rows, int cols, lcsa_dtype dtype, uint8_t* codes,
                                uint8_t* scales, void* stream);

/* ------------------------------------------------------------------------
 * Indexer + top-k on the FP4 QK path.  Same scores and selection as
 * lcsa_indexer_topk, with both sides of every dot product taken at their
 * MXFP4 values: the keys come quantised (the indexer-key cache in MXFP4,
 * e.g. written by lcsa_quantize_mxfp4 with cols = D_I), the BF16 queries are
 * quantised per (row, head) inside the call.  The products of the
 * dequantised values are exact and accumulate in FP32.  Each query head is
 * staged as FP8 E4M3 relative to its largest block scale, exact while its
 * block scales lie within 2^13 of it (a block further below rounds to the
 * E4M3 grid).  Keys are staged the same way, or, with lcsa_set_fp4_mma(1)
 * and one or two query rows per sequence (decode), read by the tensor cores
 * as E2M1 codes with their block scales (exact for any scales).  That path
 * needs k_codes 32-byte aligned (any allocation from the CUDA allocators
 * is); 16-byte aligned codes are staged.
 *
 *   q_idx     [B,Tq,64,128] BF16, 16-byte aligned; finite values
 *   w         [B,Tq,64] FP32
 *   k_codes   [B,Nc,64] uint8 (MXFP4 codes of the 128-dim keys), 16-byte aligned
 *   k_scales  [B,Nc,4] uint8, 4-byte aligned
 *   idx_out, scores_out, q_pos0, m, k: as lcsa_indexer_args
 * Only H_I = 64 and D_I = 128 (LCSA_ERR_UNSUPPORTED otherwise).  The
 * workspace (size from lcsa_indexer_topk_mxfp4_workspace) holds the score
 * chunk, the top-k scratch and the prepared queries of a chunk; a smaller
 * one processes fewer rows at a time (LCSA_ERR_WORKSPACE below one row).
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* q_idx;
  const float* w;
  const uint8_t* k_codes;
  const uint8_t* k_scales;
  int B, Tq, Nc, H_I, D_I;
  int64_t q_pos0;
  int m;
  int k;
  int32_t* idx_out;
  float* scores_out;
} lcsa_indexer_mxfp4_args;

size_t lcsa_indexer_topk_mxfp4_workspace(const lcsa_indexer_mxfp4_args* a);
lcsa_status lcsa_indexer_topk_mxfp4(const lcsa_indexer_mxfp4_args* a, void* workspace, size_t workspace_bytes,
                                   void* stream);

/* ------------------------------------------------------------------------
 * Grouped output projection ([p3] "第四步，grouped output projection" and its
 * explanation: with head dimension 512, projecting all heads straight back
 * to d would be costly, so the n_h heads are split into g groups, each group
 * is projected to an intermediate width d_g, and the concatenated groups are
 * projected back to d).  The pages give no g or d_g.
 *
 *   mid[t, j*d_g + i] = sum_k o[t, j*K + k] * w_group[j, i, k]    (K = n_h/g * c)
 *   y[t, e]           = sum_i mid[t, i] * w_out[e, i]              (i < g*d_g)
 *
 *   o       [T, n_h, c] BF16 (attention outputs; group j = heads j*n_h/g ..)
 *   w_group [g, d_g, K] BF16 (rows = outputs)
 *   w_out   [d, g*d_g]  BF16 (rows = outputs)
 *   y       [T, d]      BF16
 * BF16 operands, FP32 accumulation; mid is rounded to BF16 in the caller's
 * workspace (size from lcsa_grouped_out_proj_workspace).  Requirements: g
 * divides n_h, K and g*d_g multiples of 64, d_g and d multiples of 8, all
 * pointers 16-byte aligned (LCSA_ERR_INVALID_ARG otherwise).
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* o;
  const void* w_group;
  const void* w_out;
  void* y;
  int T, n_h, c, g, d_g, d;
} lcsa_out_proj_args;

size_t lcsa_grouped_out_proj_workspace(const lcsa_out_proj_args* a);
lcsa_status lcsa_grouped_out_proj(const lcsa_out_proj_args* a, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* ------------------------------------------------------------------------
 * Indexer + top-k without a caller workspace.  The pages have no counterpart
 * to this call: it exists for callers that cannot allocate device memory when
 * they call the library (an allocator or arena they do not own, a runtime
 * that forbids allocation after start-up, a thread that must not let
 * cudaMalloc/cudaFree synchronise the device).
 *
 * Same arguments and results as lcsa_indexer_topk, minus the workspace.  The
 * score workspace is a fixed 32 MiB array inside the library's device image,
 * held by every GPU that loads the library until the process exits; large
 * problems are processed in row chunks that fit it.  Nothing is allocated and
 * nothing needs clearing (each chunk writes the scratch it reads).
 *   - Argument errors are those of lcsa_indexer_topk, checked first.
 *   - Returns LCSA_ERR_WORKSPACE when what one query row needs does not fit
 *     32 MiB: its Nc FP32 scores (rounded up to 256 bytes), its 256-byte
 *     count and, for rows longer than 32768 columns that take the two-phase
 *     top-k, 3 x (ceil(Nc/32768) x k x 4 bytes, rounded up to 256) + 256.
 *     Nc > 8,388,544 never fits; with a two-phase row the limit is lower
 *     (e.g. about 8.34 M columns at k = 64).
 *   - The scratch array's device address belongs to the current context: it
 *     differs between contexts and changes after cudaDeviceReset.  Every call
 *     made while its stream is not being captured looks the address up in the
 *     current context (cudaGetSymbolAddress) and remembers it for that
 *     context; a call made during stream capture uses the remembered address
 *     and returns LCSA_ERR_CUDA when the current context has none.  So make
 *     one call outside capture in each context, and again after a reset,
 *     before capturing a call into a CUDA graph.
 *   - All calls in a context share the one array: calls that overlap on the
 *     GPU (different streams, or concurrent host threads without ordering)
 *     race on it.  Order them on one stream.
 * ------------------------------------------------------------------------ */
lcsa_status lcsa_indexer_topk_noalloc(const lcsa_indexer_args* a, void* stream);

/* ------------------------------------------------------------------------
 * Core attention ([p3] "第三步，core attention"; [p3] the sentence on running
 * multi-query attention over the selected blocks (CSA) and the HCA sentence on
 * dense attention over all compressed KV; [p2] "Sliding Window Branch": the
 * 128 most recent raw tokens; [p2] "Attention Sink" and [p3] "Attention
 * sink": a learnable logit per head added to the softmax denominator;
 * [p3] "Partial RoPE": rotary on the last 64 dims of queries and KV entries,
 * and the output rotated at position -i because each entry is both key and
 * value).
 *
 * For query row i of sequence b at position t = q_pos0 + i and head h:
 *   keys  = { entry j rotated at position j*m : j in sel(t) }
 *         U { raw row kv[b, s - kv_pos0] rotated at s : t-W < s <= t,
 *             kv_pos0 <= s < kv_pos0 + Tkv }
 *   sel(t) = idx[b,i,:] minus the -1 padding          (CSA, sparse)
 *          = { j : j < min(Nc, floor(t/m)) }           (HCA, dense)
 *   l_hj  = softmax_scale * rot_t(q[b,i,h]) . key_j
 *   out   = rot_{-t}( sum_j e^{l_hj} key_j / (sum_j e^{l_hj} + e^{sink_h}) )
 *   lse   = log(sum_j e^{l_hj} + e^{sink_h})
 * rot_p rotates dims [D-R, D) pairwise (2i, 2i+1) by p*base^(-2i/R); one
 * softmax covers compressed entries, window rows and the sink (shared
 * log-sum-exp).  The rotated entry is both key and value.  The CSA call trusts
 * idx for visibility (the indexer emits only visible entries); an index
 * >= Nc is skipped and flagged LCSA_DEV_BAD_INDEX.
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* q;         /* [B,Tq,H,D] dtype                                     */
  const void* ckv;       /* [B,Nc,D] dtype compressed entries (shared K=V)       */
  const int32_t* idx;    /* CSA: [B,Tq,k] int32 ascending, -1 padded; HCA: unused */
  const void* kv;        /* [B,Tkv,D] dtype raw rows at kv_pos0 .. kv_pos0+Tkv-1  */
  const float* sink;     /* [H] fp32 or NULL (no sink)                           */
  int B, Tq, H, D, R, Nc, k, Tkv;
  int64_t q_pos0, kv_pos0;
  int m;                 /* entry stride (position j*m, visibility floor(t/m))   */
  int W;                 /* sliding window (raw tokens), W >= 0                  */
  float softmax_scale;   /* 0 -> 1/sqrt(D)                                       */
  float rope_base;       /* 0 -> 10000                                           */
  lcsa_dtype dtype;
  void* out;             /* [B,Tq,H,D] out_dtype                                 */
  lcsa_dtype out_dtype;
  float* lse;            /* optional [B,Tq,H] fp32 (natural log)                 */
} lcsa_attn_args;

size_t lcsa_attn_workspace(const lcsa_attn_args* a, int sparse);
lcsa_status lcsa_csa_sparse_attn(const lcsa_attn_args* a, void* workspace,
                                 size_t workspace_bytes, void* stream);
lcsa_status lcsa_hca_dense_attn(const lcsa_attn_args* a, void* workspace,
                                size_t workspace_bytes, void* stream);
int lcsa_attn_uses_tensor_cores(const lcsa_attn_args* a);

/* ------------------------------------------------------------------------
 * FP8 entry cache ([p4] "二、CSA + HCA" / "KV Cache优化细节": the compressed
 * KV cache keeps the RoPE dims in BF16 and the rest in FP8).  The pages give
 * no FP8 variant or scale; this library's format, per entry row x[0..D):
 *   - body x[0..D-R): one E4M3 byte per value (bias 7, no infinities,
 *     largest finite 448, subnormals m * 2^-9), the value nearest to
 *     x / 2^X (ties to even, magnitudes above 448 saturate, a zero of either
 *     sign coded +0), with one scale per entry: X the smallest integer with
 *     max|body| <= 448 * 2^X, raised to at least -124 (-124 for an all-zero
 *     body), stored as the byte X + 127;
 *   - rotary dims x[D-R..D): BF16 (round to nearest even).
 * Every E4M3 * 2^X with X >= -124 is a BF16 number, so the attention calls
 * expand entries to BF16 exactly.  Bytes per entry at D=512, R=64:
 * 448 + 1 + 128 = 577 against 1024.
 *
 *   x      [rows, D] dtype (BF16 or FP32), device, aligned to its element size
 *   codes  [rows, D-R] uint8        scales [rows] uint8
 *   rope   [rows, R] BF16
 * R must be even and less than D; codes, scales and rope are a pure function
 * of x (bit-exact with any other exact implementation of the rule above).
 * ------------------------------------------------------------------------ */
typedef struct {
  const uint8_t* codes;   /* [B,Nc,D-R] E4M3, 16-byte aligned                  */
  const uint8_t* scales;  /* [B,Nc] X + 127                                    */
  const void* rope;       /* [B,Nc,R] BF16, 16-byte aligned                    */
} lcsa_fp8_entries;

lcsa_status lcsa_quantize_entries_fp8(const void* x, int64_t rows, int D, int R, lcsa_dtype dtype,
                                      uint8_t* codes, uint8_t* scales, void* rope, void* stream);

/* Core attention (as lcsa_csa_sparse_attn / lcsa_hca_dense_attn) over
 * entries held in the FP8 cache `e` instead of a->ckv (not read; may be
 * NULL).  Every other argument, the workspace (lcsa_attn_workspace) and the
 * results are those of the BF16 calls on the expanded entries.  Only the
 * tensor-core shapes (BF16 q/kv, H=64, D=512, R=64); LCSA_ERR_UNSUPPORTED
 * otherwise. */
lcsa_status lcsa_csa_sparse_attn_fp8(const lcsa_attn_args* a, const lcsa_fp8_entries* e, void* workspace,
                                     size_t workspace_bytes, void* stream);
lcsa_status lcsa_hca_dense_attn_fp8(const lcsa_attn_args* a, const lcsa_fp8_entries* e, void* workspace,
                                    size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* LCSA_H */
