/*
 * hca.h -- C ABI of the B200 (sm_100a) hot path of DeepSeek-V4's hybrid
 * compressed attention: CSA (4x compression, FP4 lightning indexer, top-k)
 * and HCA (128x compression, dense), both with the 128-token sliding window.
 *
 * Sources (page titles and sections):
 *   "DeepSeek V4: Towards Highly Efficient Million Token Context
 *    Intelligence" (papers.chlience.com reading note):
 *      section 7 "CSA"  -- compressor (m = 4), lightning indexer
 *                          I_{t,s} = sum_h w_{t,h} ReLU(q_{t,h} . K_s),
 *                          Top-k selection, shared key-value MQA core
 *                          attention, sliding-window branch;
 *      section 8 "HCA"  -- compressor (m' = 128) equations
 *                          S = Softmax_row(Z + B), C^Comp_i = sum_j S_j (.) C_j,
 *                          dense attention over all compressed entries;
 *      section 9        -- KV storage (RoPE dims BF16, the rest FP8),
 *                          FP4 indexer, 128-token window.
 *   "DeepSeek-V4: a million-token context that agents can actually use"
 *    (Hugging Face blog), "Hybrid attention: CSA and HCA" and figures 3, 4.
 *
 * Conventions for every call
 *   - Returns an hca_status.  Arguments are validated on the host before
 *     anything is launched; a rejected call launches nothing.
 *   - Every pointer is a DEVICE pointer unless stated otherwise, owned by
 *     the caller, and must stay valid until the work queued on `stream`
 *     has finished.  The library allocates no device memory: scratch comes
 *     from the caller's `ws` buffer, sized by the matching *_workspace_size.
 *     The one exception is compressed_attn_decode_noalloc, whose scratch is
 *     a 16 MiB array built into the library: every device that loads the
 *     library holds it until the process exits.
 *   - Every pointer must be 16-byte aligned (HCA_ERR_INVALID_ARG otherwise).
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Calls are asynchronous and never synchronise the device.
 *   - bf16 values travel as uint16_t bit patterns.
 *   - Integer/byte results (FP8 codes, scales, top-k sets) are bit-exact
 *     reproductions of the definitions below; attention outputs are fp32-
 *     accumulated and rounded to bf16.
 *
 * KV cache layout (one cache per layer and compression ratio; structure of
 * arrays, entry e of sequence b at row b*capacity + e):
 *   codes  uint8  [B][capacity][d - d_rope]          FP8 e4m3fn
 *   scales float  [B][capacity][(d - d_rope)/group]  fp32, amax/448
 *   rope   bf16   [B][capacity][d_rope]
 * Supported layouts: (d, d_rope, group) = (512, 64, 64) and (128, 32, 32).
 */
#ifndef HCA_B200_H
#define HCA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HCA_OK = 0,
    HCA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or index  */
    HCA_ERR_UNSUPPORTED = 2,   /* valid but not implemented shape/layout       */
    HCA_ERR_CUDA = 3,          /* a CUDA launch or query failed                */
    HCA_ERR_WORKSPACE = 4,     /* ws is NULL or smaller than required          */
    HCA_ERR_SCRATCH_LIMIT = 5  /* request needs more than the library's built-in
                                  scratch (compressed_attn_decode_noalloc)     */
} hca_status;

typedef struct {
    int32_t d;             /* channels per entry (= attention head dim)       */
    int32_t d_rope;        /* trailing channels stored as bf16                 */
    int32_t scale_group;   /* FP8 channels sharing one fp32 scale              */
} hca_kv_layout;

typedef struct {
    uint8_t*  codes;
    float*    scales;
    uint16_t* rope;
    int64_t   capacity;    /* entries per sequence                             */
} hca_kv_cache;

/* Human-readable name of a status code (static string). */
const char* hca_status_string(int status);
/* The last cudaError_t seen by a call that returned HCA_ERR_CUDA (per thread). */
int hca_last_cuda_error(void);
/* Device-side error word of the current device: non-zero when a kernel gave
 * up a bounded wait on its own pipeline barriers (its outputs are then NaN;
 * index scores of the CTA that gave up are NaN, and top-k sets and counts
 * built from them are undefined).
 * Reads and clears the word; synchronises with the device.  -1 if the word
 * cannot be read. */
int hca_take_device_error(void);

/* Launch budget: a scheduling knob with no counterpart on the pages.  It
 * caps the CTAs of one decode launch so that the launch occupies only part
 * of the device and another stream's kernels run beside it:
 *   HCA_BUDGET_DENSE_DECODE / HCA_BUDGET_SPARSE_DECODE: the CTAs (splits x
 *             sequences) of a decode attention launch on the tensor-core path
 *             (d = 512, H = 64), at most max(max_ctas, B);
 *   HCA_BUDGET_DECODE_INDEX: the CTAs of the fused decode indexer
 *             (lightning_index_topk on the tensor pipe), at most
 *             max(max_ctas, B), two per SM by default.
 *   max_ctas  > 0: the cap; 0: the default
 * Process-wide; applies to workspace sizing and launches made after the
 * call, so size workspaces after setting it.  Returns the previous value,
 * or -1 for an unknown op or a negative max_ctas. */
#define HCA_BUDGET_DENSE_DECODE 0
#define HCA_BUDGET_SPARSE_DECODE 1
#define HCA_BUDGET_DECODE_INDEX 2
int hca_set_launch_budget(int op, int max_ctas);

/* Early query: a scheduling knob with no counterpart on the pages.  Decode
 * attention launches are programmatic: a launch may start while the kernel
 * queued just before it on the stream is still running, and waits for that
 * kernel before it reads anything.  With the knob on, a sparse decode
 * attention on the tensor-core path (idx != NULL, d = 512, H = 64) loads and
 * prepares its query (conversion, and with extras the RMSNorm and RoPE)
 * before that wait, so that this work overlaps the previous kernel (in the
 * decode step: the top-k select).  The query (and the extras' weights and
 * q_pos) must then be complete before the previous kernel starts, i.e.
 * written by work queued before it or on another stream that the caller's
 * stream waited on; never by the previous kernel itself.  The index list,
 * its counts and the caches are still read after the wait.
 *   on  1: on; 0: off (the default)
 * Process-wide; applies to launches made after the call.  Returns the
 * previous value, or -1 for a value other than 0 or 1. */
int hca_set_early_query(int on);

/* ------------------------------------------------------------------ */
/* Compression: softmax-gated pooling + FP8/BF16 storage.               */
/* ------------------------------------------------------------------ */
/* Pools n_blocks consecutive blocks of m tokens for each of B sequences
 * (note, section 8 equations; section 7 for m = 4) and stores each pooled
 * entry in the cache layout above (section 9).
 *
 *   x, gate   bf16 [B][x_seq_stride][d]: raw KV C and gate logits Z; row 0
 *             of each sequence is the first token of block `entry_begin`
 *             (the caller offsets the pointers), so block entry_begin+j is
 *             rows j*m .. j*m+m-1.  Requires n_blocks*m <= x_seq_stride.
 *   pos_bias  fp32 [m][d]: learned positional bias B, row i added to the
 *             gate logit of the i-th token of every block.
 *   out       entries entry_begin .. entry_begin+n_blocks-1 are written;
 *             requires entry_begin + n_blocks <= out.capacity.
 *
 * Arithmetic (fixed so results are bit-exact; the pages give no precision):
 * per channel c, z_i = fp32(gate) + bias (fp32), zmax = max z_i,
 * e_i = E(z_i - zmax) with E the Cody-Waite / degree-7-Taylor exp in fp32,
 * S and N = sum e_i and sum e_i*x_i accumulated from +0 in ascending i with
 * every product and sum rounded (no FMA), y = N / S (IEEE division).  FP8
 * channels: per group, scale = amax/448 (IEEE division; 0 when amax = 0,
 * with codes 0), code = e4m3fn(y / scale) round-to-nearest-even,
 * saturating at +-448.  RoPE channels: bf16(y), nearest-even.
 * csa_compress uses m = 4, hca_compress m = 128. */
int csa_compress(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride,
                 const float* pos_bias, int32_t B, int64_t n_blocks,
                 hca_kv_layout layout, hca_kv_cache out, int64_t entry_begin,
                 void* stream);
int hca_compress(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride,
                 const float* pos_bias, int32_t B, int64_t n_blocks,
                 hca_kv_layout layout, hca_kv_cache out, int64_t entry_begin,
                 void* stream);

/* ------------------------------------------------------------------ */
/* Section 9 extras of the stored vectors: KV entry RMSNorm and partial  */
/* RoPE.                                                                 */
/* ------------------------------------------------------------------ */
/* "DeepSeek V4 ..." note, section 9: every compressed KV entry (and query
 * head) is RMS-normalised before core attention, and RoPE is applied to the
 * last d_rope dims of the query, the KV entry and the attention output.
 *   norm_w    fp32 [d]: RMSNorm weight, or NULL for no RMSNorm
 *   norm_eps  RMSNorm epsilon
 *   inv_freq  fp32 [d_rope/2]: RoPE frequencies (pair i = dims 2i, 2i+1 of
 *             the RoPE dims, rotated by position * inv_freq[i]), or NULL for
 *             no RoPE
 * Arithmetic (fixed so stored codes stay bit-exact): the squares are rounded
 * and summed as a pairwise tree over consecutive channel pairs, r =
 * sqrt(sum / d + eps) correctly rounded, y = (y / r) * w in fp32.  RoPE:
 * the angle position * inv_freq[i] in fp64 (exact), the rotation
 * (a cos - b sin, a sin + b cos) in fp64 with every product and sum rounded,
 * then one rounding to bf16.  A compressed entry e of ratio m sits at
 * position e * m (its block's first token). */
typedef struct {
    const float* norm_w;
    float norm_eps;
    const float* inv_freq;
} hca_entry_extras;

/* csa_compress / hca_compress with the extras: the pooled entry is
 * normalised, then stored (FP8 dims as above; RoPE dims rotated to the
 * entry's position).  ex == NULL or all-NULL members: identical to the
 * plain calls. */
int csa_compress_ex(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride,
                    const float* pos_bias, int32_t B, int64_t n_blocks,
                    hca_kv_layout layout, hca_kv_cache out, int64_t entry_begin,
                    const hca_entry_extras* ex, void* stream);
int hca_compress_ex(const uint16_t* x, const uint16_t* gate, int64_t x_seq_stride,
                    const float* pos_bias, int32_t B, int64_t n_blocks,
                    hca_kv_layout layout, hca_kv_cache out, int64_t entry_begin,
                    const hca_entry_extras* ex, void* stream);

/* ------------------------------------------------------------------ */
/* The note's overlapped CSA compressor and the indexer-key compressor   */
/* (section 7: two KV streams C_a = H W_a^KV, C_b = H W_b^KV and two gate */
/* streams Z_a, Z_b; each compressed entry pools 2m adjacent entries     */
/* with row-wise softmax weights, neighbouring entries overlapping; the  */
/* indexer keys K^IComp_s come from a compressor too, stored FP4).       */
/* ------------------------------------------------------------------ */
/* Reading (the note gives no index formula): entry i pools the m = 4
 * tokens of block i-1 from stream a and the 4 tokens of block i from stream
 * b, one softmax per channel over those 8 tokens with a positional bias of
 * 8 rows (rows 0..3 for the a-half, 4..7 for the b-half); each token feeds
 * entry i through stream b and entry i+1 through stream a.
 *   xa, za, xb, zb  bf16 [B][x_seq_stride][d]: row 0 = first token of block
 *                   entry_begin; the b-half of entry entry_begin+j is rows
 *                   4j..4j+3 of xb/zb and, for j >= 1, its a-half rows
 *                   4(j-1)..4j-1 of xa/za
 *   a_prev, za_prev bf16 [B][x_seq_stride][d], rows 0..3: stream a's block
 *                   before entry_begin (the first entry's a-half), or both
 *                   NULL: the first entry has no a-half (entry_begin = 0)
 *   pos_bias        fp32 [8][d]
 * Arithmetic: as csa_compress over the 8 tokens in the order a-half
 * ascending, b-half ascending; storage as csa_compress.  Requires
 * 4 * n_blocks <= x_seq_stride and entry_begin + n_blocks <= capacity. */
int csa_compress_overlap(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                         const uint16_t* a_prev, const uint16_t* za_prev, int64_t x_seq_stride,
                         const float* pos_bias, int32_t B, int64_t n_blocks, hca_kv_layout layout,
                         hca_kv_cache out, int64_t entry_begin, void* stream);
/* Indexer keys: the same overlapped pooling over c-channel indexer-key
 * streams (c = 64 or 128), stored FP4 as lightning_index reads them:
 * k_codes uint8 [B][capacity][c/2] (element 2i in the low nibble), k_sf
 * uint8 [B][capacity][c/32] ue8m0.  Per 32-element block (the OCP MX rule
 * for e2m1): X = floor(log2 amax) - 2, clamped to [-127, 127] (amax = 0 or
 * below 2^-126: -127), byte X + 127, codes e2m1(v * 2^-X) rounded to nearest
 * even, saturating at +-6, the sign kept. */
int indexer_key_compress(const uint16_t* xa, const uint16_t* za, const uint16_t* xb, const uint16_t* zb,
                         const uint16_t* a_prev, const uint16_t* za_prev, int64_t x_seq_stride,
                         const float* pos_bias, int32_t B, int64_t n_blocks, int32_t c,
                         uint8_t* k_codes, uint8_t* k_sf, int64_t capacity, int64_t entry_begin, void* stream);

/* Raw tokens prepared for the sliding window (the state cache keeps them in
 * this form): RMSNorm and partial RoPE at each token's position, every
 * channel stored bf16 (non-RoPE dims rounded from fp32, RoPE dims from fp64).
 *   x    bf16 [n][d]; pos int32 [n] token positions; out bf16 [n][d] (may
 *        not overlap x)
 * Supported layouts: as the cache layouts above. */
int kv_token_prep(const uint16_t* x, const int32_t* pos, int64_t n, hca_kv_layout layout,
                  const hca_entry_extras* ex, uint16_t* out, void* stream);

/* ------------------------------------------------------------------ */
/* Lightning indexer (section 7, eq. I_{t,s}; section 9: FP4).          */
/* ------------------------------------------------------------------ */
/*   q_codes  uint8 [B][Tq][Hi][c/2]  FP4 e2m1, element 2i in the low nibble
 *   q_sf     uint8 [B][Tq][Hi][c/32] ue8m0 (2^(u-127)) per 32 elements
 *   w        fp32  [B][Tq][Hi]       head weights w_{t,h}
 *   k_codes  uint8 [B][Nc_cap][c/2]  one indexer key per compressed entry,
 *   k_sf     uint8 [B][Nc_cap][c/32] shared by all Hi heads
 *   q_pos    int32 [B][Tq]           absolute position t of each query
 *   scores   fp32  [B][Tq][Nc_cap]   output
 * Entry s is eligible for query t iff its block ends at or before t:
 * (s+1)*m - 1 <= t; ineligible scores are -inf.
 * dot_h = fp32 sum over blocks b = 0..c/32-1, in order, of
 *         (exact block dot) * 2^(eq_b + ek_b - 254); with all scale bytes in
 *         [123, 127] every term and partial sum is exact, so dot_h is the
 *         exact FP4 dot product.
 * score = fp32, from +0, for h = 0..Hi-1 in order: score += w_h * ReLU(dot_h)
 *         (product rounded, then sum rounded).
 * Supported: c in {64, 128}, 1 <= Hi <= 8, or Hi = 64 (the note's
 * n_h^I = 64, section 7 parameters) with c = 128 on the tensor pipe (key
 * code buffer 32-byte and scale buffer 16-byte aligned, Nc_cap a multiple of
 * 4); m >= 1. */
int lightning_index(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                    const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                    int32_t B, int32_t Tq, int64_t Nc_cap, int32_t Hi, int32_t c, int32_t m,
                    float* scores, void* stream);
/* lightning_index with the note's BF16 index scores (section 9: the top-k
 * selector's index scores in BF16 instead of FP32): score_bf16 != 0 writes
 * each score rounded to bf16 (nearest even) into scores as uint16 bit patterns
 * [B][Tq][Nc_cap] (-inf for ineligible entries); score_bf16 = 0 is
 * lightning_index (scores fp32).  BF16 scores and Hi = 64 run on the tensor
 * pipe only: c = 128, Hi in {4, 64}, key code buffer 32-byte and scale buffer
 * 16-byte aligned, Nc_cap a multiple of 4 (HCA_ERR_UNSUPPORTED otherwise). */
int lightning_index_ex(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                       const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                       int32_t B, int32_t Tq, int64_t Nc_cap, int32_t Hi, int32_t c, int32_t m,
                       int32_t score_bf16, void* scores, void* stream);

/* ------------------------------------------------------------------ */
/* Top-k selection (section 7: C^SprsComp_t = {C_s | I_{t,s} in Top-k}) */
/* ------------------------------------------------------------------ */
/*   scores  fp32 [R][Nc_cap]; row r belongs to the query at q_pos[r]
 *   q_pos   int32 [R]
 *   idx     int32 [R][k]  output: the chosen entry indices, ascending,
 *                         padded with -1
 *   count   int32 [R]     output: min(k, #eligible)
 * Eligible entries are s < min(Nc_cap, (q_pos+1)/m).  The chosen set is the
 * min(k, #eligible) largest scores under the total order (score descending,
 * index ascending): scores compare as values (+0 == -0) and equal scores go
 * to the lower index.  NaN scores are not supported.
 * Supported: 1 <= k <= 4096.
 * Workspace: topk_select_workspace_size(R, Nc_cap, k) bytes (0 when the call
 * needs none), 256-byte aligned, owned by the caller, contents need not be
 * initialised and are clobbered.  Few long rows (R * ceil(Nc_cap / 16384)
 * <= the device's SM count, Nc_cap >= 8192) and rows longer than 2^19 scores
 * go through histogram passes (the keys above the threshold bin and the
 * candidates in it gathered by one kernel over the whole device, whose last
 * CTA per row resolves the exact threshold and writes the row) and use it; otherwise a row is split over a
 * thread-block cluster of up to 16 blocks of at most 32768 scores each
 * (Nc_cap <= 2^19) and the workspace is ignored.  A row longer than 2^19
 * scores without an adequate workspace returns HCA_ERR_WORKSPACE. */
size_t topk_select_workspace_size(int32_t R, int64_t Nc_cap, int32_t k);
int topk_select(const float* scores, const int32_t* q_pos, int32_t R, int64_t Nc_cap,
                int32_t m, int32_t k, int32_t* idx, int32_t* count,
                void* ws, size_t ws_bytes, void* stream);
/* topk_select over BF16 scores (score_bf16 != 0: scores are bf16 bit
 * patterns, uint16 [R][Nc_cap]; values compare as the bf16 values, the same
 * total order, ties to the lower index), or over fp32 scores (score_bf16 = 0:
 * topk_select).  BF16 rows always take the histogram passes: a workspace of
 * topk_select_ex_workspace_size(R, Nc_cap, k, 1) bytes (256-byte aligned) is
 * required, and Nc_cap >= 1. */
size_t topk_select_ex_workspace_size(int32_t R, int64_t Nc_cap, int32_t k, int32_t score_bf16);
int topk_select_ex(const void* scores, int32_t score_bf16, const int32_t* q_pos, int32_t R, int64_t Nc_cap,
                   int32_t m, int32_t k, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ */
/* Fused decode selection: lightning_index (Tq = 1) then topk_select.   */
/* ------------------------------------------------------------------ */
/* The same results as lightning_index(..., Tq = 1, ...) followed by
 * topk_select(scores, q_pos, B, Nc_cap, m, k, ...): scores [B][Nc_cap]
 * are written, idx [B][k] and count [B] as topk_select.  With a workspace of
 * lightning_index_topk_workspace_size(B, Nc_cap, k) bytes (256-byte
 * aligned), c = 128 and Hi = 4, the indexer kernel also builds each row's
 * key histogram, which saves the top-k one pass over the scores; otherwise
 * the two calls run one after the other.  index_done (a cudaEvent_t, may
 * be NULL) is recorded on the stream once the scores are written, before the
 * top-k work: a scheduler can start other streams' work there.  Error
 * behaviour as the two calls. */
size_t lightning_index_topk_workspace_size(int32_t B, int64_t Nc_cap, int32_t k);
int lightning_index_topk(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                         const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                         int32_t B, int64_t Nc_cap, int32_t Hi, int32_t c, int32_t m, int32_t k,
                         float* scores, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                         void* index_done, void* stream);
/* lightning_index_topk with BF16 scores (score_bf16 != 0; scores uint16 bf16
 * bits, see lightning_index_ex and topk_select_ex) or fp32 scores
 * (score_bf16 = 0).  Hi may be 64 with c = 128 (fused on the tensor pipe).
 * Workspace: lightning_index_topk_ex_workspace_size(B, Nc_cap, k, score_bf16)
 * bytes, required with BF16 scores. */
size_t lightning_index_topk_ex_workspace_size(int32_t B, int64_t Nc_cap, int32_t k, int32_t score_bf16);
int lightning_index_topk_ex(const uint8_t* q_codes, const uint8_t* q_sf, const float* w,
                            const uint8_t* k_codes, const uint8_t* k_sf, const int32_t* q_pos,
                            int32_t B, int64_t Nc_cap, int32_t Hi, int32_t c, int32_t m, int32_t k,
                            int32_t score_bf16, void* scores, int32_t* idx, int32_t* count, void* ws,
                            size_t ws_bytes, void* index_done, void* stream);

/* ------------------------------------------------------------------ */
/* Core attention (section 7: shared key-value MQA + sliding window;    */
/* section 8: dense over all compressed entries).                       */
/* ------------------------------------------------------------------ */
/* Decode: one query token per sequence, H heads sharing one KV head.
 *   q        bf16 [B][H][d]
 *   kv       the sequences' compressed cache (layout above)
 *   idx      int32 [B][idx_stride]: CSA mode, the selected entries of each
 *            sequence (e.g. topk_select output); only the first n_comp[b]
 *            are read.  NULL: HCA (dense) mode, entries 0..n_comp[b]-1.
 *   n_comp   int32 [B] (device): compressed keys of each sequence
 *   max_comp host upper bound of n_comp[] (sizes the split-K plan)
 *   window   bf16 [B][W][d]: the last W raw tokens, oldest first; key =
 *            value = token (all W rows are used)
 *   out      bf16 [B][H][d];  lse fp32 [B][H] (natural log) or NULL
 * softmax_scale must be positive and finite (else HCA_ERR_INVALID_ARG).
 * Per head: o = sum_j softmax_j(scale * q.k_j) k_j over the compressed keys
 * (dequantised: code * scale, bf16 RoPE dims) and the window tokens, one
 * joint softmax.  Split-K over the keys with a log-sum-exp combine; the
 * contractions run on tensor cores with fp16 operands and fp32 accumulation.
 * Supported: H in {8, 64} for d = 128 and H = 64 for d = 512; W <= 4096. */
size_t compressed_attn_decode_workspace_size(int32_t B, int32_t H, hca_kv_layout layout,
                                             int32_t max_comp, int32_t W);
int compressed_attn_decode(const uint16_t* q, int32_t B, int32_t H,
                           hca_kv_layout layout, hca_kv_cache kv,
                           const int32_t* idx, int32_t idx_stride,
                           const int32_t* n_comp, int32_t max_comp,
                           const uint16_t* window, int32_t W,
                           float softmax_scale, uint16_t* out, float* lse,
                           void* ws, size_t ws_bytes, void* stream);

/* Decode attention for callers that cannot allocate device memory.
 * No passage of the pages corresponds to this call: it is the same
 * computation as compressed_attn_decode (same arguments minus ws/ws_bytes,
 * same split-K plan and kernels, so the same outputs), but the split-K
 * partials go to a scratch array built into the library instead of a
 * caller-provided workspace.  It is meant for code that has no way to get
 * device memory at the point of the call: for example a plug-in running
 * inside a host engine that owns every byte of device memory and forbids
 * allocation after start-up, or a latency-critical path where the implicit
 * device synchronisation of cudaMalloc/cudaFree is not acceptable.  The call
 * itself allocates nothing (no cudaMalloc, no cudaFree, no library
 * allocator).
 *   - Limit: the scratch is 16 MiB
 *     (HCA_NOALLOC_SCRATCH_BYTES); a request whose split-K workspace
 *     (compressed_attn_decode_workspace_size) exceeds it is rejected with
 *     HCA_ERR_SCRATCH_LIMIT and nothing is launched.
 *   - The scratch is a per-device global of the library: every GPU on which
 *     the library is used keeps those 16 MiB until the process exits.
 *   - Every call looks up the scratch's device address for the current
 *     device (cudaGetSymbolAddress; no allocation).  The first call on a
 *     device also loads the library's device globals there: make that first
 *     call before any stream capture.
 *   - Every call on a device shares the one scratch array, which keeps the
 *     previous call's contents; the kernels overwrite every partial they
 *     read, so nothing needs clearing.  Calls whose work overlaps on the GPU
 *     (different streams, or different host threads, without ordering
 *     between them) race on the scratch and give wrong results: order them. */
#define HCA_NOALLOC_SCRATCH_BYTES (16u << 20)
int compressed_attn_decode_noalloc(const uint16_t* q, int32_t B, int32_t H,
                                   hca_kv_layout layout, hca_kv_cache kv,
                                   const int32_t* idx, int32_t idx_stride,
                                   const int32_t* n_comp, int32_t max_comp,
                                   const uint16_t* window, int32_t W,
                                   float softmax_scale, uint16_t* out, float* lse,
                                   void* stream);

/* Chunked prefill of one sequence: Tq query tokens at positions p0..p0+Tq-1,
 * each with causal eligibility.
 *   q       bf16 [Tq][H][d]
 *   kv      the sequence's cache (B = 1), already holding every entry a
 *           query can see (including the chunk's own complete blocks)
 *   idx     int32 [Tq][idx_stride] + count int32 [Tq]: CSA mode, query i
 *           attends to idx[i][0..count[i]);  idx = NULL: HCA (dense causal)
 *           mode, query at position p attends to entries
 *           s < min(kv.capacity, (p+1)/m)  (m is only used in this mode)
 *   raw     bf16 [W-1+Tq][d]: raw tokens from position p0-(W-1) on; the
 *           window of position p is tokens max(0, p-W+1) .. p
 *   out     bf16 [Tq][H][d]
 * Same attention rule (and softmax_scale rule) as decode. */
int compressed_attn_prefill(const uint16_t* q, int32_t Tq, int32_t H, int32_t p0, int32_t m,
                            hca_kv_layout layout, hca_kv_cache kv,
                            const int32_t* idx, int32_t idx_stride, const int32_t* count,
                            const uint16_t* raw, int32_t W,
                            float softmax_scale, uint16_t* out, void* stream);

/* ------------------------------------------------------------------ */
/* Core attention with the section 9 extras.                            */
/* ------------------------------------------------------------------ */
/* "DeepSeek V4 ..." note, section 9: query-head RMSNorm, partial RoPE on the
 * query and the output, and a learnable sink logit per head that lets the
 * attention mass be below 1.
 *   q_norm_w  fp32 [d]: RMSNorm weight of every query head (fp32 arithmetic),
 *             or NULL
 *   norm_eps  its epsilon
 *   sink      fp32 [H]: per-head sink logit, on the scale of the scaled
 *             logits (natural log): p_j = e^{l_j} / (sum_i e^{l_i} + e^{sink}),
 *             or NULL
 *   inv_freq  fp32 [d_rope/2] (as hca_entry_extras), or NULL: the query's
 *             RoPE dims are rotated to its position before the logits and the
 *             output's RoPE dims rotated back by it (the keys carry their own
 *             positions, as stored)
 *   q_pos     int32 [B]: decode only, the position of each sequence's query
 *             (required with inv_freq); prefill queries sit at p0 + i
 * lse (decode) includes the sink.  ex == NULL or all-NULL members: identical
 * to the plain calls. */
typedef struct {
    const float* q_norm_w;
    float norm_eps;
    const float* sink;
    const float* inv_freq;
    const int32_t* q_pos;
    const int32_t* win_len;  /* decode: [B] valid window rows, each <= W (the
                                state cache's window before it is full: rows
                                0 .. win_len-1 hold the tokens); NULL: all W */
} hca_attn_extras;

int compressed_attn_decode_ex(const uint16_t* q, int32_t B, int32_t H,
                              hca_kv_layout layout, hca_kv_cache kv,
                              const int32_t* idx, int32_t idx_stride,
                              const int32_t* n_comp, int32_t max_comp,
                              const uint16_t* window, int32_t W,
                              float softmax_scale, const hca_attn_extras* ex,
                              uint16_t* out, float* lse,
                              void* ws, size_t ws_bytes, void* stream);
int compressed_attn_prefill_ex(const uint16_t* q, int32_t Tq, int32_t H, int32_t p0, int32_t m,
                               hca_kv_layout layout, hca_kv_cache kv,
                               const int32_t* idx, int32_t idx_stride, const int32_t* count,
                               const uint16_t* raw, int32_t W,
                               float softmax_scale, const hca_attn_extras* ex, uint16_t* out,
                               void* stream);

/* ------------------------------------------------------------------ */
/* State cache of the decode loop (section 11: a fixed-size state per     */
/* sequence holds the recent sliding-window KV entries and the            */
/* uncompressed tail of the CSA/HCA block not yet complete).             */
/* ------------------------------------------------------------------ */
/* Appends one token per sequence at position pos (the same for all B):
 *   x, gate   bf16 [B][d]: the token's raw KV and gate logits
 *   window    bf16 [B][W][d]: ring buffer, the token goes to row pos % W
 *             (win_x, if not NULL, bf16 [B][d], is written there instead of
 *             x: the token as prepared for attention, see kv_token_prep)
 *   tail_x, tail_gate  bf16 [B][m][d]: the current block's tokens, row pos % m
 *             (skipped when m == 0 or tail_x is NULL)
 * Once the token ends a block ((pos+1) % m == 0), tail_x / tail_gate hold
 * that block's m tokens in order and csa_compress / hca_compress(tail_x,
 * tail_gate, m, ..., n_blocks = 1, entry_begin = (pos+1)/m - 1) pools it. */
int kv_state_append(const uint16_t* x, const uint16_t* gate, const uint16_t* win_x, int32_t B, int32_t d,
                    int64_t pos, uint16_t* window, int32_t W, uint16_t* tail_x, uint16_t* tail_gate,
                    int32_t m, void* stream);

/* ------------------------------------------------------------------ */
/* One decode step from host memory to host memory (sections 7 and 8:    */
/* the CSA path and the HCA path of one decode position).               */
/* ------------------------------------------------------------------ */
/* Device state and buffers of the step, all owned by the caller (device
 * pointers unless stated): the CSA layer's cache, indexer keys and window,
 * the HCA layer's cache, entry counts and window, staging buffers for the
 * queries, the index scores, top-k outputs and workspaces, the outputs; and
 * for the schedule a second stream and five events (cudaStream_t /
 * cudaEvent_t as void*, created by the caller). */
typedef struct {
    int32_t B, H, Hi, c, k, W;
    float softmax_scale;
    hca_kv_layout layout;
    hca_kv_cache csa_cache;
    int64_t csa_entries;          /* entries per sequence = indexer keys per sequence    */
    const uint8_t* k_codes;       /* [B][csa_entries][c/2]                               */
    const uint8_t* k_sf;          /* [B][csa_entries][c/32]                              */
    const uint16_t* csa_window;   /* [B][W][d]                                           */
    hca_kv_cache hca_cache;
    const int32_t* hca_n;         /* [B] HCA entries per sequence                        */
    int32_t hca_max;              /* host bound of hca_n                                 */
    const uint16_t* hca_window;   /* [B][W][d]                                           */
    const int32_t* q_pos;         /* [B] query position                                  */
    uint16_t* q_csa;              /* [B][H][d] staging                                   */
    uint16_t* q_hca;              /* [B][H][d] staging                                   */
    uint8_t* iq_codes;            /* [B][Hi][c/2] staging                                */
    uint8_t* iq_sf;               /* [B][Hi][c/32] staging                               */
    float* iq_w;                  /* [B][Hi] staging                                     */
    float* scores;                /* [B][csa_entries]                                    */
    int32_t* idx;                 /* [B][k]                                              */
    int32_t* count;               /* [B]                                                 */
    void* topk_ws; size_t topk_ws_bytes;   /* lightning_index_topk_workspace_size        */
    void* ws_csa; size_t ws_csa_bytes;     /* compressed_attn_decode_workspace_size      */
    void* ws_hca; size_t ws_hca_bytes;
    uint16_t* out_csa;            /* [B][H][d]                                           */
    uint16_t* out_hca;            /* [B][H][d]                                           */
    void* side_stream;
    void* ev_fork; void* ev_index; void* ev_q; void* ev_join;
    int32_t hca_ctas;             /* CTAs of the HCA attention (its split-K plan); 0: the  */
                                  /* SMs that the top-k select's B * floor(SMs / 2 / B)    */
                                  /* CTAs leave (at least half), the rest left to the      */
                                  /* concurrent CSA chain                                  */
    void* ev_iq;                  /* marks the indexer query's copy                        */
    int32_t packed;               /* bit 0: the indexer query's codes, scales and weights */
                                  /* lie in one allocation each (host and device), in that */
                                  /* order, each from the next 16-byte boundary: one copy; */
                                  /* bit 1: out_csa and out_hca lie back to back in one    */
                                  /* allocation, h_out_csa and h_out_hca likewise, in the  */
                                  /* same order: one copy of both after the join           */
} hca_decode_step_plan;

/* Host queries in, host outputs out:
 *   h_q_csa, h_q_hca  bf16 [B][H][d]; h_iq_codes [B][Hi][c/2], h_iq_sf
 *   [B][Hi][c/32], h_iq_w fp32 [B][Hi]; h_out_csa, h_out_hca bf16 [B][H][d]
 *   (host memory; pinned for asynchronous copies).
 * Queues on the plan's side stream (give it the higher priority: it carries
 * the critical path): the indexer-query copy (one copy with plan->packed
 * bit 0, else three), lightning_index_topk, the CSA attention (after the
 * CSA-query copy) and its output copy.  On `stream`, once the indexer query
 * has crossed (ev_iq), so that the small copy the indexer waits for does not
 * share the link with the large ones: the attention-query copies and, once
 * the indexer has run, the HCA attention and its output copy (with
 * plan->packed bit 1, one copy of both outputs on `stream` after the join
 * instead).  `stream` finally waits for the side stream, so both outputs are
 * in host memory when `stream` reaches that point.  The five events of the
 * plan are the caller's (created without timing); nothing is allocated.
 * Errors as the calls it makes; HCA_ERR_INVALID_ARG also when a bit of
 * plan->packed is set but the pointers do not lie as it states. */
int hca_decode_step_host(const hca_decode_step_plan* plan, const uint16_t* h_q_csa, const uint16_t* h_q_hca,
                         const uint8_t* h_iq_codes, const uint8_t* h_iq_sf, const float* h_iq_w,
                         uint16_t* h_out_csa, uint16_t* h_out_hca, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* HCA_B200_H */
