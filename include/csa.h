/*
 * csa.h - C ABI of libcsa.so, the B200 (sm_100a) DeepSeek-V4 hybrid-attention
 * hot path: Compressed Sparse Attention (CSA) and Heavily Compressed
 * Attention (HCA).
 *
 * Sources, cited by page title and section:
 *   [P2] "DeepSeek V4 technical report" (agentupdate.ai, Chinese), hybrid
 *        attention section: CSA steps 1 (KV compression), 2 (Lightning
 *        Indexer + top-k), 3 (core multi-query attention); HCA paragraph.
 *   [P3] "DeepSeek V4-Pro Architecture: KV Cache Compression and
 *        Hyper-Connections Visualised" (webconsulting.at), "Key points" and
 *        "Dual Compression and Indexing".
 *   [P5] "DeepSeek V4-Pro" (lizeman.github.io llm-arch-kb), "What's new in
 *        V4 / 1. Hybrid attention: CSA + HCA replace MLA"; "5. 1M context,
 *        gradually" (YaRN extension); "Family" (V4-Flash shapes).
 *
 * Conventions shared by every entry point
 *   - Tensor pointers are DEVICE pointers owned by the caller (the binding
 *     allocates them with PyTorch).  The library never allocates or frees
 *     device memory; scratch comes from a caller-provided workspace whose
 *     size csa_workspace_bytes() reports.  Host pointers are marked "host".
 *   - Every tensor is dense, row-major, in the layout written beside it, and
 *     its base address is 16-byte aligned (CSA_ERR_INVALID_ARG otherwise).
 *   - bf16 tensors are passed as void* holding IEEE bfloat16 values; E4M3
 *     tensors as uint8_t* holding OCP FP8 E4M3 ("fn") codes.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work; they are stream-ordered, keep no
 *     state between calls and may be captured into a CUDA graph.
 *   - Ordering: the first kernel of every call starts its work only after
 *     all earlier work on the stream has completed -- including a caller's
 *     kernel that lets its dependents launch early.  (It is an ordinary
 *     launch, except in the decode steps, where it may be scheduled early
 *     but waits for the previous kernel before reading anything.)
 *     The later kernels of a call may start while their predecessor in the
 *     same call still runs (programmatic dependent launch) and read the
 *     call's inputs early; they wait for that predecessor before reading
 *     anything it writes.  Inputs therefore only need to be complete in
 *     stream order when the call is made.
 *   - Argument checks are synchronous and return an error before anything
 *     is enqueued.  A failed launch returns CSA_ERR_CUDA.  csa_last_error()
 *     returns a thread-local message for the last failure on that thread.
 *   - `dev_status` (optional, device int32) receives the first error a
 *     kernel detects on the device (an index outside the buffers it was
 *     given, a visible-entry count above the capacity, a bounded wait that
 *     gave up).  The offending access is skipped; nothing traps.  The caller
 *     reads and clears it.
 *   - No exceptions cross the ABI and there is no CPU fallback.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,       /* null/misaligned pointer, negative size, ... */
  CSA_ERR_UNSUPPORTED_SHAPE = 2, /* a size outside the supported set below */
  CSA_ERR_CAPACITY = 3,          /* a range that does not fit the given capacity */
  CSA_ERR_WORKSPACE = 4,         /* workspace missing or smaller than required */
  CSA_ERR_CUDA = 5,              /* a CUDA runtime/driver call failed */
  CSA_ERR_DEVICE_TIMEOUT = 6,    /* (dev_status) a bounded device wait gave up */
  CSA_ERR_DEVICE_INDEX = 7       /* (dev_status) an index outside its buffer */
} csa_status;

/* Shapes and constants shared by the calls of one layer.
 * Supported: d in {128, 512}; 1 <= H <= 128; H_I in {1..64}, D_I in {64, 128}
 * (indexer calls only); 1 <= k <= 2048; 0 <= window <= 1024; rope_dim in
 * {0, 32, 64} and <= d/4 (attention calls); 1 <= m <= 128 (CSA uses 4, HCA
 * 128); 0 <= overlap <= m with m + overlap <= 128; eps > 0. */
typedef struct {
  int B;               /* sequences in the batch */
  int d;               /* KV entry dim == attention head dim D ([P5]: 512) */
  int H;               /* query heads ([P5]: 128) */
  int H_I;             /* Lightning-Indexer heads ([P5]: 64) */
  int D_I;             /* Lightning-Indexer head dim ([P5]: 128) */
  int k;               /* entries kept per query ([P5]: 1024) */
  int window;          /* uncompressed sliding window W ([P5]: 128) */
  int rope_dim;        /* rotated trailing dims r ([P5]: 64) */
  int m;               /* compression ratio ([P5]: 4 for CSA, 128 for HCA) */
  float eps;           /* RMSNorm epsilon (1e-6 in the tests) */
  float softmax_scale; /* logit scale; 0 selects 1/sqrt(d) */
  const double* rope_inv_freq; /* host, [rope_dim/2] angle per position for
                                  pair j; NULL selects 10000^(-2j/rope_dim) */
  int overlap;         /* compression: tokens of block i-1 that entry i also
                          pools (0 = non-overlapping blocks; 0..m, see
                          csa_compress); b_pos then holds m + overlap values */
  int64_t entry_offset; /* the compressed cache (kv_c, idx_key, idx_scale and
                          the indexer scores) holds entries entry_offset ..
                          entry_offset + N_cap - 1 of the sequence: a shard of
                          a context split over several devices (0 = the whole
                          cache).  Local entry i is block entry_offset + i: its
                          tokens and its rotation position (entry_offset + i +
                          1)*m - 1 are the sequence's, visible counts are
                          floor((pos+1)/m) - entry_offset clamped to 0..N_cap,
                          and block ranges and indices are local.  Token rows
                          (kv_tok, idx_tok) and positions stay global. */
} csa_params;

/* Operation selector for csa_workspace_bytes(). */
typedef enum {
  CSA_OP_INDEX_TOPK = 1,
  CSA_OP_SPARSE_MQA = 2,
  CSA_OP_DENSE_MQA = 3,
  CSA_OP_PREFILL = 4,
  CSA_OP_HCA_PREFILL = 5,
  CSA_OP_CSA_DECODE_STEP = 6,
  CSA_OP_HCA_DECODE_STEP = 7
} csa_op;

/* Library version (major*100 + minor). */
int csa_version(void);

/* Thread-local message for the last non-OK status returned on this thread. */
const char* csa_last_error(void);

/* ---------------------------------------------------------------------------
 * Transfers for a decode loop (no counterpart in the method: plumbing for a
 * caller that keeps its inputs and outputs in host memory).  One
 * asynchronous copy on `stream`, in whichever direction the two addresses
 * imply (host or device memory; unified addressing); page-locked host memory
 * makes it overlap with kernels.  Ordering: stream order only, so the
 * caller orders the copy against the step that reads or writes the device
 * side (same stream, or events).  Nothing is owned or kept.
 *   csa_copy_async: `bytes` contiguous bytes.
 *   csa_copy_rows_async: `rows` rows of `row_bytes` bytes each, row r at
 *   dst + r * dst_pitch and src + r * src_pitch (pitches >= row_bytes), e.g.
 *   the new token's row of every sequence in a [B, L_cap, d] token buffer.
 * Errors: a NULL address with a non-zero size or a pitch below row_bytes ->
 * CSA_ERR_INVALID_ARG; a refused copy -> CSA_ERR_CUDA.  Zero bytes or rows
 * enqueue nothing.
 * ------------------------------------------------------------------------- */
csa_status csa_copy_async(void* dst, const void* src, size_t bytes, void* stream);
csa_status csa_copy_rows_async(void* dst, size_t dst_pitch, const void* src, size_t src_pitch,
                               size_t row_bytes, size_t rows, void* stream);

/* ---------------------------------------------------------------------------
 * YaRN RoPE frequency table (host only; no device work).  [P5] "5. 1M
 * context, gradually": the context is extended to 1,048,576 tokens with
 * YaRN, factor 16, beta_fast 32, beta_slow 1.  The pages give no formula;
 * this follows the published method (Peng et al. 2023, "YaRN: Efficient
 * Context Window Extension of Large Language Models", NTK-by-parts):
 *   theta_j  = base^(-2j/rope_dim)                 j < rope_dim/2
 *   turns_j  = original_len * theta_j / (2 pi)
 *   ramp_j   = clamp((turns_j - beta_slow) / (beta_fast - beta_slow), 0, 1)
 *   inv_freq[j] = ramp_j * theta_j + (1 - ramp_j) * theta_j / factor
 *   *logit_gain    = (1 + 0.1 ln factor)^2   (the method's attention
 *                    temperature: query and key are each scaled by
 *                    1 + 0.1 ln factor)
 *   *softmax_scale = *logit_gain / sqrt(d), rounded to binary32: the logit
 *                    scale to put in csa_params.softmax_scale
 * Pass the table as csa_params.rope_inv_freq: compression, the window
 * rotation, the query rotation and the inverse rotation of the output all
 * use it.  (original_len = 1,048,576 / 16 = 65,536 is the reading for the
 * pages' schedule.)
 *   d             head dim of the attention calls (read only when
 *                 softmax_scale is not NULL)
 *   inv_freq      host, [rope_dim/2] doubles (written)
 *   logit_gain    host, one double (written) or NULL
 *   softmax_scale host, one float (written) or NULL
 * Errors: CSA_ERR_UNSUPPORTED_SHAPE for rope_dim odd or outside 2..128;
 *         CSA_ERR_INVALID_ARG for inv_freq NULL, base <= 1, factor < 1,
 *         beta_slow < 0, beta_fast <= beta_slow, original_len <= 0, any
 *         non-finite value, or d < 1 with softmax_scale not NULL.  Nothing
 *         is written on error.
 * ------------------------------------------------------------------------- */
csa_status csa_rope_yarn(int rope_dim, double base, double factor, double beta_fast,
                         double beta_slow, double original_len, int d, double* inv_freq,
                         double* logit_gain, float* softmax_scale);

/* Workspace bytes that `op` needs for these params.
 *   Q     queries per sequence (1 for decode; T for CSA_OP_PREFILL and
 *         CSA_OP_HCA_PREFILL),
 *   N_cap capacity of the compressed cache (entries per sequence).
 * Returns 0 for invalid arguments (and sets csa_last_error). */
size_t csa_workspace_bytes(const csa_params* p, csa_op op, int Q, int64_t N_cap);

/* ---------------------------------------------------------------------------
 * KV compression, HCA form ([P2] HCA: m' = 128, blocks do not overlap;
 * [P3] "Dual Compression and Indexing": a learned weighted average per
 * block; [P5] "Hybrid attention": HCA bullet).
 *
 * For every sequence b and block i in [first_block, first_block+n_blocks)
 * the present tokens t = i*m + j (j < m, t < ctx_len[b]) are pooled:
 *   s_j   = kv_tok[b,t,:] . w_s + b_pos[j]
 *   alpha = softmax over the present j of s_j
 *   e     = RMSNorm(sum_j alpha_j kv_tok[b,t,:]) * gamma      (eps = p->eps)
 * and RoPE_{(i+1)m-1}(e) -- e rotated on its last p->rope_dim dims to the
 * position of the block's last token ([P5]: RoPE on the last 64 dims of the
 * KV) -- is stored as bf16 in kv_c[b,i,:], so that attention uses entries
 * as stored.  A block with no present token is left untouched.  (The weight
 * form and the place of the rotation are the readings taken here: the pages
 * fix neither.)  rope_dim must be 0, 32 or 64 and at most d/4.
 *
 *   kv_tok  [B, L_cap, d] bf16 (device)     token KV stream
 *   ctx_len [B] int64 (device)              tokens present per sequence
 *   w_s [d], b_pos [m], gamma [d] or NULL (ones)   fp32 (device)
 *   kv_c    [B, N_cap, d] bf16 (device)     compressed cache (written)
 * Errors: CSA_ERR_CAPACITY if first_block < 0 or first_block + n_blocks > N_cap
 *         (checked on the host); tokens at or beyond L_cap are never read.
 * ------------------------------------------------------------------------- */
csa_status hca_compress(const csa_params* p, const void* kv_tok, int64_t L_cap,
                        const int64_t* ctx_len, const float* w_s, const float* b_pos,
                        const float* gamma, int64_t first_block, int64_t n_blocks,
                        void* kv_c, int64_t N_cap, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * KV compression, CSA form ([P2] CSA step 1; [P5] CSA bullet: m = 4).
 * The KV stream is pooled exactly as hca_compress does.
 * Overlapping variant (p->overlap > 0; [P2] states "no overlap" for HCA
 * only and gives no rule for CSA, so this is the reading taken here): entry i
 * pools the window of m + overlap tokens t = i*m - overlap + j (j < m +
 * overlap), those with 0 <= t < ctx_len, scored with b_pos[j]; b_pos then
 * holds m + overlap values.  The entry is still written once its own block
 * has a token, visible once its own block is complete, and rotated to
 * (i+1)*m - 1.  The same holds for every call that compresses (the prefill
 * chunks and the decode steps).  When idx_tok is not
 * NULL, the indexer-key stream idx_tok [B, L_cap, D_I] bf16 is pooled by the
 * same operation with its own w_s_idx [D_I] and b_pos_idx [m] (no gain),
 * and each pooled row x is stored in E4M3 ([P3]: the indexer is low
 * precision): scale = max|x| / 448 in binary32 (1 when the row is zero),
 * code = E4M3 round-to-nearest-even, saturating, of x / scale.
 *   idx_key   [B, N_cap, D_I] uint8 E4M3 codes (written)
 *   idx_scale [B, N_cap] fp32 (written)
 * ------------------------------------------------------------------------- */
csa_status csa_compress(const csa_params* p, const void* kv_tok, int64_t L_cap,
                        const int64_t* ctx_len, const float* w_s, const float* b_pos,
                        const float* gamma, int64_t first_block, int64_t n_blocks,
                        void* kv_c, int64_t N_cap, const void* idx_tok,
                        const float* w_s_idx, const float* b_pos_idx, uint8_t* idx_key,
                        float* idx_scale, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Lightning Indexer + top-k ([P2] CSA step 2; [P5] CSA bullet: 64 heads of
 * dim 128, k = 1024; [P3] "Key points": ~262,000 entries narrowed to 1,024).
 *
 * For every sequence b and query q (position pos_q[b,q]) the visible
 * entries are i < n_vis = floor((pos_q+1)/m) (the block holding the query is
 * not complete and is not visible, [P5] sliding-window bullet).  Score
 * (reading of the DSA form the pages cite):
 *   score_i = sum_h w[h] * ReLU( (q_idx[h,:]*q_scale[h]) . (key[i,:]*key_scale[i]) )
 * evaluated as key_scale[i] * sum_h (w[h]*q_scale[h]) * ReLU(q_idx[h,:] . key[i,:])
 * with E4M3 products accumulated in fp32 on the tensor cores.  The k entries
 * with the largest score are kept (ties: lower index first; NaN lowest;
 * -0 == +0) and written as ascending indices, padded with -1;
 * topk_cnt = min(k, n_vis).
 *
 *   q_idx    [B, Q, H_I, D_I] uint8 E4M3 (device)
 *   q_scale  [B, Q, H_I] fp32 (device, >= 0)    w [B, Q, H_I] fp32 (device)
 *   idx_key  [B, N_cap, D_I] uint8, idx_scale [B, N_cap] fp32 (device, >= 0)
 *   pos_q    [B, Q] int64 (device)
 *   topk_idx [B, Q, k] int32 (written)          topk_cnt [B, Q] int32 (written)
 *   scores_out [B, Q, N_cap] fp32 or NULL: when given, entries i < n_vis
 *              receive the fp32 scores (others are not written).
 * Device errors: n_vis > N_cap -> CSA_ERR_CAPACITY in dev_status, clamped.
 * Sizes: N_cap <= 262144 (one cluster of 8 CTAs holds a row of scores).
 * ------------------------------------------------------------------------- */
csa_status lightning_index_topk(const csa_params* p, int Q, const uint8_t* q_idx,
                                const float* q_scale, const float* w,
                                const uint8_t* idx_key, const float* idx_scale, int64_t N_cap,
                                const int64_t* pos_q, int32_t* topk_idx, int32_t* topk_cnt,
                                float* scores_out, void* ws, size_t ws_bytes,
                                int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * The two halves of lightning_index_topk, for callers that want the scores
 * themselves or their own selection: lightning_index_scores writes the fp32
 * scores of the visible entries (others untouched); topk_select ranks the
 * first n_vis = floor((pos_q+1)/m) scores of every row with the same rule
 * and output as lightning_index_topk.  Running the two in order gives the
 * same result as lightning_index_topk.
 *   scores [B, Q, N_cap] fp32 (device; written / read).
 * ------------------------------------------------------------------------- */
csa_status lightning_index_scores(const csa_params* p, int Q, const uint8_t* q_idx,
                                  const float* q_scale, const float* w, const uint8_t* idx_key,
                                  const float* idx_scale, int64_t N_cap, const int64_t* pos_q,
                                  float* scores, int32_t* dev_status, void* stream);

csa_status topk_select(const csa_params* p, int Q, const float* scores, int64_t N_cap,
                       const int64_t* pos_q, int32_t* topk_idx, int32_t* topk_cnt,
                       int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * lightning_index_topk without a workspace.  The paper has no counterpart:
 * this is an interface variant of this library, not a step of the method.
 *
 * Same arguments, result and errors as lightning_index_topk minus scores_out,
 * ws and ws_bytes: the fp32 score matrix lives in an array that the library
 * itself holds on every device it is loaded on (8 MiB each, kept until the
 * process exits).  The call allocates no device or host memory, so callers
 * that cannot allocate can use it: code running under another memory
 * manager that has reserved the device's memory (an engine that pre-reserves
 * the HBM for its KV cache), code that may not stall the device (freeing
 * memory synchronises it), or code whose fixed interface has no workspace
 * to hand over.
 *
 * Limit: B * Q * N_cap <= 2^21 (2097152) scores -- e.g. B = 8 at N_cap =
 * 32768 or B = 4 at N_cap = 262144, one query each.  Larger calls return
 * CSA_ERR_WORKSPACE and launch nothing.
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * Every call on a device uses the same array, which keeps the last call's
 * scores; nothing in it has to start at zero (each call writes every score
 * it then ranks).  Calls that can overlap on one device -- on two streams,
 * or from two host threads -- race on the array and give wrong results:
 * order them on one stream.
 * ------------------------------------------------------------------------- */
csa_status lightning_index_topk_static(const csa_params* p, int Q, const uint8_t* q_idx,
                                       const float* q_scale, const float* w,
                                       const uint8_t* idx_key, const float* idx_scale,
                                       int64_t N_cap, const int64_t* pos_q, int32_t* topk_idx,
                                       int32_t* topk_cnt, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Shared-KV multi-query attention over selected entries + window + sink
 * ([P2] CSA step 3; [P5] "Hybrid attention": shared-KV MQA with 128 heads
 * of dim 512, sliding-window branch of 128 tokens, per-head sink logits in
 * the softmax denominator, QK RMSNorm, RoPE on the last 64 dims with inverse
 * RoPE on the output).  One query per sequence at position pos = pos_q[b].
 *
 *   qhat_h = RoPE_pos(RMSNorm(q[b,h,:]) * gamma_q)
 *   KV set = { kv_c[b,i,:] (stored rotated, see hca_compress) : i in topk_idx[b, 0..topk_cnt) }
 *          U { RoPE_t(RMSNorm(kv_tok[b,t,:]) * gamma_kv) : max(0,pos-W+1) <= t <= pos }
 *   s_hj = softmax_scale * qhat_h . v_j;  M_h = max(max_j s_hj, sink[h])
 *   out[b,h,:] = RoPE_{-pos}( sum_j e^{s_hj-M_h} v_j / (sum_j e^{s_hj-M_h} + e^{sink[h]-M_h}) )
 * stored as bf16; lse[b,h] = M_h + log(denominator) when lse is not NULL.
 * Readings (pages silent): one joint softmax over window and entries, no
 * de-duplication; compressed entries are used as stored (their pooling
 * RMSNorm is the KV norm, and they are stored rotated to their position
 * (i+1)*m-1); rotate-half pairing over the last rope_dim dims.  sink = -inf drops the sink; +inf
 * gives a zero output.
 *
 *   q [B, H, d] bf16; pos_q [B] int64; kv_c [B, N_cap, d] bf16;
 *   topk_idx [B, k] int32, topk_cnt [B] int32 (entries must be < n_vis);
 *   kv_tok [B, L_cap, d] bf16; sink [H] fp32; gamma_q, gamma_kv [d] or NULL;
 *   out [B, H, d] bf16 (written); lse [B, H] fp32 or NULL.
 * Device errors: an index >= n_vis or < -1 -> CSA_ERR_DEVICE_INDEX, skipped.
 * ------------------------------------------------------------------------- */
csa_status sparse_mqa_decode(const csa_params* p, const void* q, const int64_t* pos_q,
                             const void* kv_c, int64_t N_cap, const int32_t* topk_idx,
                             const int32_t* topk_cnt, const void* kv_tok, int64_t L_cap,
                             const float* sink, const float* gamma_q, const float* gamma_kv,
                             void* out, float* lse, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * HCA dense decode ([P2] HCA: dense attention over every compressed entry;
 * [P5] HCA bullet).  As sparse_mqa_decode with the KV set
 * { entries 0 .. n_vis-1 } U window, n_vis = min(floor((pos+1)/m), N_cap).
 * ------------------------------------------------------------------------- */
csa_status dense_mqa_decode(const csa_params* p, const void* q, const int64_t* pos_q,
                            const void* kv_c, int64_t N_cap, const void* kv_tok, int64_t L_cap,
                            const float* sink, const float* gamma_q, const float* gamma_kv,
                            void* out, float* lse, void* ws, size_t ws_bytes,
                            int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * CSA prefill chunk (B = 1): T new tokens at positions P .. P+T-1 whose KV
 * rows (kv_tok) and indexer-stream rows (idx_tok) the caller has already
 * written.  Runs, in order: csa_compress of blocks P/m .. ceil((P+T)/m)-1
 * (ctx_len = P+T); the Lightning Indexer for every new query t with its own
 * causal visible count floor((t+1)/m); top-k per query; and the sparse MQA
 * per query with its own window [max(0,t-W+1), t].  P must be a multiple
 * of m, and the cache is a whole one (entry_offset = 0).
 *   q [T, H, d] bf16, q_idx [T, H_I, D_I] E4M3, q_scale/w [T, H_I] fp32,
 *   out [T, H, d] bf16 (written), topk_idx [T, k] / topk_cnt [T] (written).
 * ------------------------------------------------------------------------- */
csa_status csa_prefill_chunk(const csa_params* p, int64_t P, int T, const void* kv_tok,
                             const void* idx_tok, int64_t L_cap, const float* w_s,
                             const float* b_pos, const float* gamma, const float* w_s_idx,
                             const float* b_pos_idx, void* kv_c, uint8_t* idx_key,
                             float* idx_scale, int64_t N_cap, const void* q,
                             const uint8_t* q_idx, const float* q_scale, const float* w,
                             const float* sink, const float* gamma_q, const float* gamma_kv,
                             int32_t* topk_idx, int32_t* topk_cnt, void* out, void* ws,
                             size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * One CSA decode step for B sequences, each at its own position ([P2] CSA
 * steps 1-3; [P5] "Hybrid attention": CSA bullet).  The caller has written
 * each sequence's new token rows (kv_tok, idx_tok row pos_q[b]); the call
 * then runs, in order:
 *   1. compression of each sequence's newest block, the one holding its
 *      query token: block pos_q[b]/m pooled over tokens up to pos_q[b] (as
 *      csa_compress; a block that is still partial is written but stays
 *      invisible until it is complete, and a later step rewrites it);
 *   2. the Lightning Indexer and top-k over the visible entries
 *      floor((pos_q[b]+1)/m) (as lightning_index_topk);
 *   3. the sparse MQA over the selection, the window and the sink (as
 *      sparse_mqa_decode).
 * Calling it for consecutive positions is the decode loop: the caches grow
 * by one compressed entry every m steps.
 *   pos_q [B] int64 (device); q [B, H, d]; q_idx [B, H_I, D_I]; q_scale, w
 *   [B, H_I]; topk_idx [B, k], topk_cnt [B] (written); out [B, H, d] bf16
 *   and lse [B, H] or NULL (written); other tensors as csa_compress and
 *   sparse_mqa_decode.
 * Workspace: csa_workspace_bytes(p, CSA_OP_CSA_DECODE_STEP, 1, N_cap).  It
 * carries state between calls that only affects speed: where the top-k
 * spreads a row over a cluster of CTAs (a few long rows), the indexer
 * counts each row's scores by their top 12 key bits into a histogram in the
 * workspace, which the top-k reads and clears.  A zero-filled workspace, or
 * one that the previous call of this function left, takes the fast path;
 * other contents cost that call a full radix selection, never a different
 * result.
 * Device errors: a newest block at or beyond N_cap -> CSA_ERR_DEVICE_INDEX
 * (not written).
 * ------------------------------------------------------------------------- */
csa_status csa_decode_step(const csa_params* p, const int64_t* pos_q, const void* kv_tok,
                           const void* idx_tok, int64_t L_cap, const float* w_s,
                           const float* b_pos, const float* gamma, const float* w_s_idx,
                           const float* b_pos_idx, void* kv_c, uint8_t* idx_key,
                           float* idx_scale, int64_t N_cap, const void* q, const uint8_t* q_idx,
                           const float* q_scale, const float* w, const float* sink,
                           const float* gamma_q, const float* gamma_kv, int32_t* topk_idx,
                           int32_t* topk_cnt, void* out, float* lse, void* ws, size_t ws_bytes,
                           int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * One HCA decode step for B sequences, each at its own position ([P2] HCA
 * paragraph; [P5] "Hybrid attention": HCA bullet): compression of each
 * sequence's newest block (block pos_q[b]/m, pooled over tokens up to
 * pos_q[b], as hca_compress), then the dense MQA over the visible entries,
 * the window and the sink (as dense_mqa_decode).
 * Workspace: csa_workspace_bytes(p, CSA_OP_HCA_DECODE_STEP, 1, N_cap).
 * ------------------------------------------------------------------------- */
csa_status hca_decode_step(const csa_params* p, const int64_t* pos_q, const void* kv_tok,
                           int64_t L_cap, const float* w_s, const float* b_pos,
                           const float* gamma, void* kv_c, int64_t N_cap, const void* q,
                           const float* sink, const float* gamma_q, const float* gamma_kv,
                           void* out, float* lse, void* ws, size_t ws_bytes,
                           int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * HCA prefill chunk (B = 1; [P2] HCA paragraph: dense attention over every
 * compressed entry, m' = 128, no overlap; [P5] "Hybrid attention": HCA
 * bullet and the sliding-window branch).  T new tokens at positions
 * P .. P+T-1 whose KV rows (kv_tok) the caller has already written.  Runs,
 * in order: hca_compress of blocks P/m .. ceil((P+T)/m)-1 with ctx_len = P+T
 * (a partial last block is pooled over its present tokens and stays
 * invisible), then for every new query t the dense MQA over its visible
 * entries 0 .. floor((t+1)/m)-1 and its window [max(0, t-W+1), t], one joint
 * softmax with the sink, inverse RoPE on the output.  P must be a multiple
 * of m; entries before P/m must already be in kv_c.
 *   kv_tok [1, L_cap, d] bf16; w_s [d], b_pos [m], gamma [d] or NULL fp32;
 *   kv_c [1, N_cap, d] bf16 (blocks P/m .. written); q [T, H, d] bf16;
 *   sink [H] fp32; gamma_q, gamma_kv [d] or NULL; out [T, H, d] bf16
 *   (written); lse [T, H] fp32 or NULL.
 * Workspace: csa_workspace_bytes(p, CSA_OP_HCA_PREFILL, T, N_cap).
 * Errors: CSA_ERR_UNSUPPORTED_SHAPE for B != 1 or T > 65535;
 *         CSA_ERR_INVALID_ARG when P is not a multiple of m or T < 1;
 *         CSA_ERR_CAPACITY when P+T > L_cap or ceil((P+T)/m) > N_cap.
 * ------------------------------------------------------------------------- */
csa_status hca_prefill_chunk(const csa_params* p, int64_t P, int T, const void* kv_tok,
                             int64_t L_cap, const float* w_s, const float* b_pos,
                             const float* gamma, void* kv_c, int64_t N_cap, const void* q,
                             const float* sink, const float* gamma_q, const float* gamma_kv,
                             void* out, float* lse, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Grouped output projection ("DeepSeek V4 technical report" (agentupdate.ai),
 * 混合注意力机制, item 分组输出投影: because the head dim is 512, the heads'
 * outputs are not projected straight back to the model dim d; the n_h heads
 * are split into g groups, each group is projected to an intermediate dim
 * d_g, and the concatenation is projected back to d.  "DeepSeek V4-Pro"
 * (llm-arch-kb), "1. Hybrid attention": g = 16, d_g = 1024.)
 *
 * For every token t (the rows of the attention output o):
 *   y[t, j*d_g + r] = sum_c W_g[j, r, c] * o[t, j*(H/g)*D + c]   j < g, r < d_g
 *   z[t, n]         = sum_i W_o[n, i] * y[t, i]                  n < d_model
 * i.e. group j reads heads j*H/g .. (j+1)*H/g - 1 of o (contiguous,
 * head-major).  No bias and no nonlinearity between the two projections (the
 * pages give none).  bf16 inputs, fp32 accumulation on the tensor cores, y
 * stored in bf16 before the second projection, z stored in bf16.  The pages
 * do not give d; any multiple of 128 is supported.
 *
 *   o   [T, H, D] bf16 (device)             attention output
 *   w_g [g, d_g, (H/g)*D] bf16 (device)     rows are outputs
 *   w_o [d_model, g*d_g] bf16 (device)      rows are outputs
 *   y   [T, g*d_g] bf16 (device, written) or NULL (then kept in the workspace)
 *   z   [T, d_model] bf16 (device, written)
 * Supported: g divides H; (H/g)*D and g*d_g multiples of 64; d_g and
 * d_model multiples of 128; T >= 1.  Anything else returns
 * CSA_ERR_UNSUPPORTED_SHAPE (or CSA_ERR_INVALID_ARG for values < 1).
 * Workspace: grouped_out_proj_workspace_bytes(T, H, D, g, d_g, d_model)
 * (0 for unsupported arguments); CSA_ERR_WORKSPACE when smaller.
 * ------------------------------------------------------------------------- */
size_t grouped_out_proj_workspace_bytes(int T, int H, int D, int g, int d_g, int d_model);

csa_status grouped_out_proj(int T, int H, int D, int g, int d_g, int d_model, const void* o,
                            const void* w_g, const void* w_o, void* y, void* z, void* ws,
                            size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * Context split: one sequence's compressed cache over G devices.
 *
 * The pages give no parallel scheme for this path ("Architectural Overview
 * of V4 Series Models" (intl.cloud.baidu.com) names only 3D-parallel
 * training as an outlook); this is this library's.  Rank r holds the entries
 * [lo_r, hi_r) of the compressed KV cache and of the indexer keys, a
 * contiguous range in rank order, described to every call by
 * csa_params.entry_offset = lo_r and N_cap = hi_r - lo_r.  One decode step:
 *   1. every rank scores its entries and keeps its local top-k
 *      (lightning_index_topk on its shard, scores_out given);
 *   2. csa_shard_candidates turns that into (score, sequence index) pairs;
 *   3. the ranks exchange the pairs and counts (an all-gather in rank order,
 *      e.g. NCCL);
 *   4. csa_merge_candidates ranks the G*k candidates: the exact top-k of the
 *      whole sequence (it lies within the union of the local top-k lists;
 *      same tie rule), and this rank's share of it as local indices;
 *   5. sparse_mqa_partials attends over this rank's share (the window only on
 *      the rank holding the newest tokens: csa_params.window = 0 elsewhere)
 *      and writes split partials instead of an output;
 *   6. the ranks exchange the partials (all-gather in rank order);
 *   7. mqa_merge_partials folds all ranks' partials, the sink and the inverse
 *      rotation into the output, identical on every rank.
 * Steps 3 and 6 are the only data exchange (B*Q*k*8 bytes of candidates and
 * B*S*H*(2d+8) bytes of partials per rank).
 * ------------------------------------------------------------------------- */

/* Candidates of one shard.  For every row (b, q) and slot j < topk_cnt:
 *   cand_score[b,q,j] = scores[b,q,topk_idx[b,q,j]],
 *   cand_idx[b,q,j]   = topk_idx[b,q,j] + p->entry_offset  (sequence index);
 * slots j >= topk_cnt get (NaN, -1).  scores [B,Q,N_cap] fp32, topk_idx
 * [B,Q,k] / topk_cnt [B,Q] int32 as lightning_index_topk writes them (all
 * device); cand_score [B,Q,k] fp32, cand_idx [B,Q,k] int32 (written).
 * Sequence indices must fit in int32 (CSA_ERR_UNSUPPORTED_SHAPE). */
csa_status csa_shard_candidates(const csa_params* p, int Q, const float* scores, int64_t N_cap,
                                const int32_t* topk_idx, const int32_t* topk_cnt,
                                float* cand_score, int32_t* cand_idx, int32_t* dev_status,
                                void* stream);

/* Global top-k over the candidates of G ranks (concatenated in rank order).
 *   cand_score [G,B,Q,k] fp32, cand_idx [G,B,Q,k] int32, cand_cnt [G,B,Q]
 *   int32 (device): the all-gathered outputs of csa_shard_candidates and the
 *   local counts.  The candidates of rank r must be ascending and below
 *   rank r+1's (true for contiguous shards in rank order).
 *   topk_idx [B,Q,k] / topk_cnt [B,Q] (written): the k best candidates by
 *   (score descending, sequence index ascending; NaN lowest), as ascending
 *   sequence indices padded with -1 -- the same selection lightning_index_topk
 *   makes over the whole sequence.
 *   local_idx [B,Q,k] / local_cnt [B,Q] (written): the selected entries in
 *   this rank's range [p->entry_offset, p->entry_offset + N_cap), as local
 *   indices (ascending, padded with -1).
 * Supported: 1 <= G <= 64 with G*k <= 24320. */
csa_status csa_merge_candidates(const csa_params* p, int Q, int G, const float* cand_score,
                                const int32_t* cand_idx, const int32_t* cand_cnt, int64_t N_cap,
                                int32_t* topk_idx, int32_t* topk_cnt, int32_t* local_idx,
                                int32_t* local_cnt, int32_t* dev_status, void* stream);

/* sparse_mqa_decode over this rank's share, stopped before the merge: the KV
 * set is the entries local_idx (topk_idx here) of this rank's cache plus,
 * when p->window > 0, the window of kv_tok; the list is cut into `splits`
 * parts (1..64), and each part's unnormalised softmax state is written:
 *   part_o  [B, splits, H, d] fp16 (device): the part's weighted sum of
 *           values divided by its own sum (before the inverse rotation),
 *   part_ml [B, splits, 2, H] fp32 (device): [.., 0, h] the part's largest
 *           logit times log2(e), [.., 1, h] its sum of 2^(logit*log2 e - max);
 *           an empty part holds (-inf, 0) and no part_o row.
 * Other arguments as sparse_mqa_decode (no sink: the merge adds it). */
csa_status sparse_mqa_partials(const csa_params* p, int splits, const void* q, const int64_t* pos_q,
                               const void* kv_c, int64_t N_cap, const int32_t* topk_idx,
                               const int32_t* topk_cnt, const void* kv_tok, int64_t L_cap,
                               const float* gamma_q, const float* gamma_kv, void* part_o,
                               float* part_ml, int32_t* dev_status, void* stream);

/* Merge of split partials [B, splits, ...] (the concatenation, in rank
 * order, of every rank's sparse_mqa_partials output for B = 1): the
 * output and log-sum-exp of one joint softmax over every part's KV set and
 * the sink, with the inverse rotation by pos_q -- what sparse_mqa_decode
 * would write for the union of the parts.  splits 1..4096. */
csa_status mqa_merge_partials(const csa_params* p, int splits, const void* part_o,
                              const float* part_ml, const int64_t* pos_q, const float* sink,
                              void* out, float* lse, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
