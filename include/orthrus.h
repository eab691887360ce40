/*
 * orthrus.h — C ABI of the B200 (sm_100a) dual-view decode library.
 *
 * One decode cycle of Orthrus ("Orthrus: Memory-Efficient Parallel Token
 * Generation via Dual-View Diffusion"; the paper-notes page, §4.1) is three
 * calls on one CUDA stream:
 *
 *   orthrus_draft_block   parallel projection: the diffusion view reads the
 *                         block [anchor, mask x (K-1)] and proposes K tokens
 *                         (§4.1 step 1);
 *   orthrus_verify_block  AR verification: the frozen AR view reads
 *                         [anchor, y_1 .. y_{K-1}] in one causal forward and
 *                         writes its K/V into the cache tail (§4.1 step 2);
 *   orthrus_commit        consensus: greedy prefix match (§4.2) or rejection
 *                         sampling at T>0 (§4.3); the committed length grows
 *                         by the n in [1, K] emitted tokens (§4.1 step 3).
 *
 * orthrus_prefill builds the shared cache with the AR view (§2.2);
 * orthrus_ar_step is one step of plain AR decoding with the same kernels
 * (the baseline the method must reproduce exactly at T = 0, §4.2, §9.1);
 * orthrus_generate drives the whole loop.  Beyond the cycle:
 * orthrus_draft_block_iterative (multi-pass denoising draft, §5.4.2),
 * orthrus_block_mask_attention and orthrus_kl_lm_head (the training-side
 * dual-pass block mask and forward KL, §3.1-3.3), orthrus_tree_topw /
 * orthrus_tree_build / orthrus_verify_tree / orthrus_tree_commit (tree
 * verification over the draft's marginals, §7.5, §9.6), and
 * orthrus_adaptive_len / orthrus_commit_adaptive (a verify length set by the
 * draft rows' entropies, §7.4, §9.6).
 *
 * Conventions for every entry point:
 *   - Every pointer to tensor data is a DEVICE pointer owned by the caller
 *     unless the comment says "host".  The library never allocates or frees
 *     device memory: its scratch lives in the caller's workspace.
 *   - `stream` is a cudaStream_t passed as void*; all work is enqueued on it
 *     and the calls return without synchronising, except where stated.
 *   - Matrices are row-major [out][in] (the nn.Linear layout), in the
 *     config's dtype (bf16 or fp32).  Norm gains are [hidden] in that dtype.
 *   - Argument and capacity errors are found on the host before any launch
 *     and returned synchronously; nothing is enqueued then.  Problems that
 *     only the device can see (a token id out of range, a sequence that
 *     would overflow its pages, a non-finite log-sum-exp) set bits of a
 *     device error word and skip the offending write; orthrus_check_error
 *     and orthrus_generate report them as ORTHRUS_ERR_DEVICE_CHECK /
 *     ORTHRUS_ERR_NONFINITE.  No call aborts the process.
 *   - A context is bound to one stream at a time and is not thread-safe.
 */
#ifndef ORTHRUS_H
#define ORTHRUS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ORTHRUS_OK = 0,
    ORTHRUS_ERR_INVALID_ARG = 1,   /* null pointer, bad size or shape */
    ORTHRUS_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim) */
    ORTHRUS_ERR_CAPACITY = 3,      /* batch, K, length or workspace too large */
    ORTHRUS_ERR_CUDA = 4,          /* a CUDA runtime call failed */
    ORTHRUS_ERR_DEVICE_CHECK = 5,  /* a device-side bounds/id check fired */
    ORTHRUS_ERR_NONFINITE = 6      /* a log-sum-exp came out NaN or inf */
} orthrus_status_t;

typedef enum { ORTHRUS_BF16 = 0, ORTHRUS_FP32 = 1 } orthrus_dtype_t;

/* Device error-word bits (orthrus_check_error's *bits). */
#define ORTHRUS_DEVERR_TOKEN     0x1   /* token id outside [0, vocab) */
#define ORTHRUS_DEVERR_CAPACITY  0x2   /* position beyond the sequence's pages */
#define ORTHRUS_DEVERR_NONFINITE 0x4   /* non-finite log-sum-exp */
#define ORTHRUS_DEVERR_TIMEOUT   0x8   /* a kernel's bounded wait ran out; it stopped early */

/*
 * Model shape and run limits.  The decoder is the pages' frozen AR backbone
 * (pre-norm, RMSNorm, rotary positions, grouped-query attention, SwiGLU FFN,
 * no biases) with one extra W_Q/W_K/W_V per layer for the diffusion view
 * (paper notes §2.1).
 *   head_dim     must be 16, 32, 64 or 128; 128 for the bf16 tensor-core path.
 *   mask_token_id  id of the mask token that fills block rows 1..K-1 of a
 *                draft (paper notes §4.1 step 1); an ordinary embedding row.
 *   max_batch, max_block   largest batch and block size K a call may use.
 *   max_seq      largest committed length + K a sequence may reach; sizes the
 *                attention split buffers only (never the diffusion K/V).
 *   split_tokens KV positions per attention split, a multiple of 64; fixed
 *                for a run so a row's result never depends on the block it
 *                sits in.
 */
typedef struct {
    int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab, mask_token_id;
    int32_t dtype;                 /* orthrus_dtype_t */
    int32_t max_batch, max_block, max_seq, split_tokens;
    float rope_theta, rms_eps;
} orthrus_config_t;

/* Device pointers of one layer.  wq/wk/wv: AR view; *_diff: diffusion view
 * (paper notes §2.1).  Shapes: wq [n_q*hd][hidden], wk/wv [n_kv*hd][hidden],
 * wo [hidden][n_q*hd], w_gate/w_up [ffn][hidden], w_down [hidden][ffn]. */
typedef struct {
    const void *attn_norm, *wq, *wk, *wv, *wq_diff, *wk_diff, *wv_diff;
    const void *wo, *ffn_norm, *w_gate, *w_up, *w_down;
} orthrus_layer_weights_t;

/* embed [vocab][hidden], lm_head [vocab][hidden] (may equal embed when the
 * head is tied), final_norm [hidden]; `layers` is a HOST array of n_layers
 * entries, copied by orthrus_create. */
typedef struct {
    const void *embed, *final_norm, *lm_head;
    const orthrus_layer_weights_t *layers;
} orthrus_weights_t;

/*
 * The one shared KV cache (paper notes §2.2-2.3): AR keys (after RoPE) and
 * values only, paged.
 *   k_pages      [n_layers][num_pages][n_kv][page_size][head_dim], dtype
 *   v_pages      [n_layers][num_pages][n_kv][head_dim][page_size], dtype: V is
 *                stored transposed inside a page, so both attention products
 *                read their operand with the reduced dimension contiguous
 *   block_table  [max_batch][max_pages_per_seq] int32 page ids
 *   seq_lens     [max_batch] int32 committed length t of each sequence
 *                (the anchor's own K/V are not in the cache)
 * page_size must be a multiple of 16 (of 64 on the bf16 path).  Pages must
 * hold finite values before first use (zero them once): slots beyond a
 * sequence's length are read and then masked, and 0 * NaN would not vanish.
 */
typedef struct {
    void *k_pages, *v_pages;
    int32_t *block_table;
    int32_t *seq_lens;
    int32_t num_pages, page_size, max_pages_per_seq;
} orthrus_kv_t;

typedef struct orthrus_ctx orthrus_ctx_t;

/* Host-side statistics filled by orthrus_generate. */
typedef struct {
    int64_t cycles;         /* decode cycles (2 forwards each; 1 for plain AR) */
    int64_t forwards;       /* forward passes run after prefill */
    int64_t tokens;         /* tokens emitted, summed over the batch */
    int64_t min_tokens;     /* smallest per-sequence count reached */
} orthrus_stats_t;

/* Bytes of workspace a context needs for `cfg` (device memory the caller
 * allocates, 256-byte aligned).  Independent of any sequence length. */
orthrus_status_t orthrus_workspace_size(const orthrus_config_t *cfg, size_t *bytes);

/* Bytes of the transient diffusion K/V of one draft of `batch` sequences
 * and block size K across all layers: n_layers*batch*K*n_kv*hd*2*sizeof(dtype).
 * The pages state this is constant in the sequence length (~4.5 MiB for the
 * Qwen3-8B shape at K = 32; paper notes §2.3, §9.5). */
orthrus_status_t orthrus_transient_bytes(const orthrus_config_t *cfg, int32_t batch, int32_t K,
                                         size_t *bytes);

/* Validates cfg, copies cfg and the weight pointers (the weights themselves
 * stay caller-owned and must outlive the context), carves the workspace and
 * zeroes its counters on the current device.  Synchronous. */
orthrus_status_t orthrus_create(const orthrus_config_t *cfg, const orthrus_weights_t *weights,
                                void *workspace, size_t ws_bytes, orthrus_ctx_t **out);
orthrus_status_t orthrus_destroy(orthrus_ctx_t *ctx);

/*
 * AR prefill (paper notes §2.2): for each b < batch, runs the AR view
 * causally over tokens[b][0 .. lens[b]-2], writing their K/V into the
 * sequence's pages, sets seq_lens[b] = lens[b]-1 and anchor_out[b] =
 * tokens[b][lens[b]-1].  tokens: device [batch][tok_stride]; lens: HOST
 * [batch], each in [1, max_seq - max_block].
 */
orthrus_status_t orthrus_prefill(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, const int32_t *tokens,
                                 int32_t tok_stride, const int32_t *lens, int32_t batch,
                                 int32_t *anchor_out, void *stream);

/*
 * Parallel projection (paper notes §4.1 step 1, §3.2 mask): per sequence b,
 * the block [anchor[b], mask x (K-1)] at positions t..t+K-1 (t = seq_lens[b])
 * goes through the diffusion view; each block row attends to cache rows
 * [0, t) and to every block row.  The block's K/V stay in the workspace and
 * never enter the cache.  Writes draft [batch][K] int32: argmax per row at
 * temperature 0, else a Gumbel-max sample of softmax(logits/T) keyed by
 * (seed, *step, row).  step: device int64 (read only).
 */
orthrus_status_t orthrus_draft_block(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, const int32_t *anchor,
                                     int32_t batch, int32_t K, float temperature, uint64_t seed,
                                     const int64_t *step, int32_t *draft, void *stream);

/*
 * Iterative-denoising draft: the multi-step variant the paper-notes page
 * compares with single-step drafting (§5.4.2; the page gives no procedure).
 * Pass 0 is orthrus_draft_block; each further pass s (< iterations) runs the
 * diffusion view again on the block [anchor[b], draft[b][0] .. draft[b][K-2]]
 * of the previous pass's drafts (same positions, same mask) and overwrites
 * draft with its own argmaxes or samples; pass s keys its Gumbel noise with
 * (seed, *step, row, purpose DRAFT | s << 8).  The acceptance test that
 * follows uses the last pass's distribution, so sampled decoding stays
 * lossless.  iterations = 1 is orthrus_draft_block exactly; iterations < 1
 * returns ORTHRUS_ERR_INVALID_ARG.  Each pass is one diffusion forward and
 * one LM-head pass; the cache is never written.
 */
orthrus_status_t orthrus_draft_block_iterative(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, const int32_t *anchor,
                                               int32_t batch, int32_t K, int32_t iterations, float temperature,
                                               uint64_t seed, const int64_t *step, int32_t *draft, void *stream);

/*
 * AR verification (paper notes §4.1 step 2): per sequence, the block
 * [anchor, draft[0..K-2]] at positions t..t+K-1 through the AR view, causal
 * (row k sees cache rows [0, t+k]).  Its K/V are written into cache slots
 * t..t+K-1 (beyond the committed length until orthrus_commit).  Results stay
 * in the workspace for orthrus_commit.  The pages for t+K positions must
 * exist in block_table.
 */
orthrus_status_t orthrus_verify_block(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, const int32_t *anchor,
                                      const int32_t *draft, int32_t batch, int32_t K, float temperature,
                                      void *stream);

/*
 * Consensus and commit (paper notes §4.1 step 3, §4.2, §4.3) after a draft
 * and a verify with the same batch, K and temperature.  Greedy: accept draft
 * tokens while they equal the AR argmax; at the first mismatch j emit the AR
 * argmax.  T>0: accept row k iff u_k < p_k(y_k)/q_k(y_k); at the first
 * rejection draw the correction from norm(max(0, p_j - q_j)).  Writes
 * n_out [batch] (in [1, K]), tokens_out [batch][K] (first n valid),
 * anchor_io[b] = last emitted token, seq_lens[b] += n, and *step += 1.
 * force_n (nullable, device [batch]) overrides n (tokens emitted are then
 * the AR argmaxes), for measurements with a prescribed acceptance.
 */
orthrus_status_t orthrus_commit(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, int32_t batch, int32_t K,
                                float temperature, uint64_t seed, int64_t *step, const int32_t *force_n,
                                int32_t *n_out, int32_t *tokens_out, int32_t *anchor_io, void *stream);

/*
 * Adaptive block length (paper notes §7.4: a verify length set by the
 * draft's own uncertainty, SV's signal, named as complementary to Orthrus;
 * §9.6: a dynamic K; neither gives a rule).  Reading taken: after a draft
 * of K rows, sequence b verifies kt[b] = 1 + the number of leading drafted
 * tokens y_1, y_2, ... whose draft rows have entropy at most h_max (y_k is
 * drafted by row k-1), so 1 <= kt[b] <= K; h_max = +inf is the fixed-K
 * cycle and h_max < 0 plain AR.  Greedy decoding only: the entropy is that
 * of the row's softmax(z) at T = 1, in nats, computed inside the draft's
 * LM-head epilogue (no logits are written).
 *   kt       device int32 [batch], written
 *   entropy  device fp32 [batch][K] (nullable): the rows' entropies
 * Call after orthrus_draft_block (temperature 0) with the same batch and K;
 * then orthrus_verify_block (temperature 0, block K) and
 * orthrus_commit_adaptive.  h_max NaN returns ORTHRUS_ERR_INVALID_ARG.
 */
orthrus_status_t orthrus_adaptive_len(orthrus_ctx_t *ctx, int32_t batch, int32_t K, float h_max, int32_t *kt,
                                      float *entropy, void *stream);

/*
 * Greedy consensus and commit over the first kt[b] rows of the verified
 * block (kt as orthrus_adaptive_len writes it, clamped to [1, K]): accept
 * drafted tokens while they equal the AR argmax within those rows, at the
 * first mismatch emit the AR argmax, else emit all kt[b]; n_out, tokens_out,
 * anchor_io, seq_lens and *step as orthrus_commit at temperature 0.  The
 * verify rows kt[b] .. K-1 do not change rows below them (causal mask); their
 * K/V lie beyond the committed length and are overwritten later, so the
 * result equals a verify of kt[b] rows.
 */
orthrus_status_t orthrus_commit_adaptive(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, int32_t batch, int32_t K,
                                         const int32_t *kt, int64_t *step, int32_t *n_out, int32_t *tokens_out,
                                         int32_t *anchor_io, void *stream);

/*
 * One plain AR decoding step with the same kernels: the AR view on
 * [anchor[b]] at position seq_lens[b], then emit the argmax (T = 0) or a
 * Gumbel-max sample keyed by (seed, *step) (T > 0).  Writes token_out
 * [batch], anchor_io[b] = that token, seq_lens[b] += 1, *step += 1.
 */
orthrus_status_t orthrus_ar_step(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, int32_t batch,
                                 float temperature, uint64_t seed, int64_t *step, int32_t *token_out,
                                 int32_t *anchor_io, void *stream);

/*
 * Whole generation: prefill, then cycles of draft/verify/commit (K >= 1) or
 * plain AR steps (K == 0) until every sequence has max_new tokens.
 * prompt: device [batch][tok_stride]; lens: HOST [batch]; out: device
 * [batch][max_new].  Synchronises the stream once per cycle (to read how many
 * tokens were produced); returns a pending device error, if any.
 */
orthrus_status_t orthrus_generate(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, const int32_t *prompt,
                                  int32_t tok_stride, const int32_t *lens, int32_t batch, int32_t K,
                                  int32_t max_new, float temperature, uint64_t seed, int32_t *out,
                                  orthrus_stats_t *stats, void *stream);

/*
 * The dual-view attention on its own (paper notes §3.2 and §4.1): block of
 * K query rows per sequence at positions t..t+K-1 (t = seq_lens[b]).
 *   q       [batch][K][n_q][hd]
 *   mode 0  AR verify: keys/values are cache rows [0, t+k] for row k (the
 *           block's rows must already be in the cache at t..t+K-1);
 *   mode 1  diffusion draft: cache rows [0, t) plus all K rows of
 *           k_blk/v_blk [batch][K][n_kv][hd].
 *   out     [batch][K][n_q][hd]
 * Uses the layer-`layer` slice of the cache and the context's workspace.
 * On a bf16 head_dim-128 context whose GQA group divides 128 the tensor-core
 * kernel runs and needs q 16-byte aligned; otherwise (or when its tensor maps
 * cannot be encoded over these buffers) the call returns
 * ORTHRUS_ERR_UNSUPPORTED without launching anything, since such a context
 * holds no room for the SIMT kernel's split partials.
 */
orthrus_status_t orthrus_dual_view_attention(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, int32_t layer,
                                             int32_t mode, const void *q, const void *k_blk,
                                             const void *v_blk, int32_t batch, int32_t K, void *out,
                                             void *stream);

/*
 * orthrus_dual_view_attention for callers that cannot allocate device
 * memory.  The paper has no counterpart to this entry point; it exists for
 * deployment.  Some callers cannot hand the library a workspace: a serving
 * runtime that reserves the whole of HBM for its own pool at start-up (a
 * cudaMalloc from a plugin then fails or eats memory the pool was promised),
 * or code on a latency-critical path where cudaMalloc / cudaFree would
 * synchronise the device.  This call needs no context and no workspace: its
 * scratch lives in a fixed 16 MiB array that the library holds on every GPU
 * it is loaded on, until the process exits.  It allocates nothing.  It runs
 * the kernels, launch shapes and summation orders that
 * orthrus_dual_view_attention runs for the same config, so its output is
 * bit-identical to that entry point's (long contexts included: from max_seq
 * >= 8192 both spread a row group over several clusters).
 *
 *   cfg      model shape and limits (only the attention fields, n_layers,
 *            dtype, max_seq and split_tokens are read); q, k_blk, v_blk, out,
 *            kv, mode, layer, batch, K as for orthrus_dual_view_attention.
 *   dev_err  device pointer to a uint32 the caller owns, or NULL; it is
 *            cleared and then receives the device error bits of this call.
 *            With NULL the bits go to a word inside the fixed array.
 *
 * Capacity.  With rows = batch*K, kp = K rounded up to 64, es = 2 (bf16) or
 * 4 (fp32), S = ceil(max_seq / split_tokens) + 1 and up(x) = x rounded up to
 * 256, the call needs
 *     256 + up(4 * batch)
 *   + (mode 1 only) 2 * up(batch * n_kv * kp * head_dim * es)   (block K, V^T)
 *   + tensor-core path, max_seq >= 8192 only:
 *       up(4 * rows * n_q * head_dim * 4) + up(4 * rows * n_q * 8) + rows * n_kv * 32
 *   + SIMT path: up(rows * n_q * S * 8) + rows * n_q * S * head_dim * 4
 * bytes, and returns ORTHRUS_ERR_CAPACITY, launching nothing, when that
 * exceeds 16 MiB.  The tensor-core path is taken for bf16, head_dim 128, a
 * GQA group dividing 128, q 16-byte aligned and buffers whose tensor maps
 * encode; every other call takes the SIMT path, whose split partials are
 * then counted.  The first call on a device also looks up the array's device
 * address and sets the kernels' shared-memory limit; make that first call
 * before capturing a stream.  All calls share the one array, which keeps the
 * last call's contents, so calls whose work overlaps on the GPU (two
 * streams, or two threads) race and give wrong results: serialise them.
 */
orthrus_status_t orthrus_dual_view_attention_noalloc(const orthrus_config_t *cfg, const orthrus_kv_t *kv,
                                                    int32_t layer, int32_t mode, const void *q, const void *k_blk,
                                                    const void *v_blk, int32_t batch, int32_t K, void *out,
                                                    uint32_t *dev_err, void *stream);

/*
 * Training-side dual-pass block-masked attention (paper notes §3.1-3.2; the
 * hotdry.top page's training section): one packed training sequence of L
 * clean positions holds n_blocks anchor blocks of K positions each; block b
 * starts at anchor position anchors[b].  Query row k of block b sees the
 * clean context positions [0, anchors[b]) (their AR K/V) and all K rows of
 * its own block (their diffusion K/V, bidirectional); blocks never see one
 * another.  This is the diffusion-view kernel with one "sequence" per block,
 * all reading the same context pages.
 *   kv        block_table row 0 lists the packed context's pages, in order;
 *             its layer-`layer` slice holds the context K/V (rows [0, L));
 *             kv->seq_lens is not read.
 *   q         device [n_blocks][K][n_q][hd] (context dtype)
 *   k_blk,
 *   v_blk     device [n_blocks][K][n_kv][hd], the blocks' diffusion K/V
 *   anchors   DEVICE int32 [n_blocks], 0 <= anchors[b]; positions past the
 *             pages block_table row 0 covers raise ORTHRUS_DEVERR_CAPACITY
 *   out       device [n_blocks][K][n_q][hd]
 * Requires n_blocks >= 1 and 1 <= K <= max_block; blocks are independent
 * and are processed max_batch at a time.  Ownership and errors as for
 * orthrus_dual_view_attention.
 */
orthrus_status_t orthrus_block_mask_attention(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, int32_t layer,
                                              const void *q, const void *k_blk, const void *v_blk,
                                              const int32_t *anchors, int32_t n_blocks, int32_t K, void *out,
                                              void *stream);

/*
 * Forward KL of the distillation loss (paper notes §3.3): for each row r,
 * with the shared LM head W,
 *     KL(p_AR || p_diff) = sum_v p_AR(v) (log p_AR(v) - log p_diff(v)),
 *     p_AR = softmax(W h_ar[r]),  p_diff = softmax(W h_diff[r]),
 * over the whole vocabulary, fused into the LM-head GEMM: the logits never
 * reach memory (per vocabulary tile the epilogue keeps both views' max and
 * sum of exponentials and sum exp(z_AR - max)(z_AR - z_diff); a second
 * kernel merges the tiles).
 *   h_ar, h_diff  device [rows][hidden] (context dtype): final-normed hidden
 *                 rows of the two views at the same positions
 *   kl            device fp32 [rows]
 *   lse_ar,
 *   lse_diff      device fp32 [rows] log-sum-exps of the two views, or NULL
 * Requires 1 <= rows and 2 * rows <= max_batch * max_block.  Uses the
 * context's workspace (its activation rows and LM-head records), so it must
 * not overlap a decode call of the same context on the GPU.
 */
orthrus_status_t orthrus_kl_lm_head(orthrus_ctx_t *ctx, const void *h_ar, const void *h_diff, int32_t rows,
                                    float *kl, float *lse_ar, float *lse_diff, void *stream);

/*
 * Tree verification, the parts that do not change a forward (paper notes
 * §7.5: DDTree expands one diffusion forward's marginals best-first into a
 * tree of the top prefixes and verifies it with tree attention in one pass;
 * §9.6: the same proposed for Orthrus).  Greedy only.  A tree of R rows
 * keeps row 0 as the root (the anchor) and every other row r as a node
 * with parent[r] in [0, r) and its draft token; node r sits at position
 * t + depth(r).  A tree cycle is: the draft with the top-W candidates of its
 * rows (orthrus_draft_block_topw; or orthrus_draft_block and
 * orthrus_tree_topw over materialised logits), the tree
 * (orthrus_tree_build), its tree-masked AR forward (orthrus_verify_tree)
 * and the walk plus commit (orthrus_tree_commit).
 *
 * orthrus_tree_topw: for each of `rows` rows of fp32 logits (device,
 * [rows][vocab]) the `width` largest logits, best first (ties: lowest id),
 * ids [rows][width] int32 and vals [rows][width] fp32, and the row's
 * log-sum-exp lse [rows] fp32 (T = 1).  Requires 1 <= width <= 8,
 * width <= vocab and rows <= 65535 (ORTHRUS_ERR_CAPACITY beyond).  A
 * non-finite log-sum-exp raises ORTHRUS_DEVERR_NONFINITE.
 */
orthrus_status_t orthrus_tree_topw(orthrus_ctx_t *ctx, const float *logits, int32_t rows, int32_t width,
                                   int32_t *ids, float *vals, float *lse, void *stream);

/*
 * orthrus_draft_block_topw: the greedy draft (orthrus_draft_block at
 * temperature 0: writes draft [batch][K]) that also returns, for draft rows
 * k < depth of every sequence, the `width` largest logits best first (ties:
 * lowest id) as ids [batch][depth][width] int32 and vals fp32, and each
 * row's log-sum-exp lse [batch][depth] fp32 (T = 1) — orthrus_tree_topw's
 * outputs for those rows, taken inside the LM-head pass (each vocabulary
 * tile keeps its best width logits; a second kernel merges the tiles) so the
 * logits never reach memory.  depth = K - 1 gives the candidates
 * orthrus_tree_build takes for a tree that fits a K-row block.  Requires
 * 1 <= width <= 8, width <= vocab and 1 <= depth <= K.
 */
orthrus_status_t orthrus_draft_block_topw(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, const int32_t *anchor,
                                          int32_t batch, int32_t K, int32_t width, int32_t depth, int32_t *draft,
                                          int32_t *ids, float *vals, float *lse, void *stream);

/*
 * orthrus_tree_build: per sequence b, the best-first draft tree.  Inputs
 * (device): ids, vals [batch][depth][width] and lse [batch][depth] as
 * orthrus_tree_topw writes them for the draft rows 0 .. depth-1 (row d
 * gives the candidates for depth d + 1, log q = val - lse).  A prefix
 * scores the fp64 sum of its log q; the tree is the root plus the `nodes`
 * best prefixes of depth <= `depth`, ordered by score and then by their
 * rank sequences, rows in that order.  Outputs (device) [batch][nodes + 1]:
 * parent (-1 for the root and unused rows), token (-1 likewise),
 * node_depth, score (fp64, -inf on unused rows); n_rows [batch] = rows used
 * (fewer than nodes + 1 when fewer prefixes exist).  Requires 1 <= batch <=
 * max_batch, 0 <= depth < 128, 1 <= width <= 8, 0 <= nodes < 128.
 */
orthrus_status_t orthrus_tree_build(orthrus_ctx_t *ctx, const int32_t *ids, const float *vals, const float *lse,
                                    int32_t batch, int32_t depth, int32_t width, int32_t nodes, int32_t *parent,
                                    int32_t *token, int32_t *node_depth, double *score, int32_t *n_rows,
                                    void *stream);

/*
 * orthrus_verify_tree: the tree-masked AR verification of one tree per
 * sequence (paper notes §7.5: all the tree's nodes in one forward with tree
 * attention).  Row 0 is the anchor, row r > 0 the node with parent[r] in
 * [0, r) and token[r], as orthrus_tree_build writes them (rows with parent
 * -1 past the tree's end are unused).  Row r is rotated for position
 * t + depth(r) (t = seq_lens[b]) but its AR K/V are written to cache slot
 * t + r; it attends to cache rows [0, t) and to the block rows on its own
 * root path (its ancestors and itself), so every node's logits equal those
 * of a plain causal forward of its root path.  Writes g [batch][rows]
 * int32: each row's AR argmax (the consensus input of orthrus_tree_commit).
 * The pages for t + rows positions must exist.  Requires 1 <= rows <=
 * min(max_block, 128); a parent outside [0, r) or a token outside
 * [0, vocab) raises ORTHRUS_DEVERR_TOKEN (that row is then treated as
 * unused).  Greedy only.
 */
orthrus_status_t orthrus_verify_tree(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, const int32_t *anchor,
                                     const int32_t *parent, const int32_t *token, int32_t batch, int32_t rows,
                                     int32_t *g, void *stream);

/*
 * orthrus_tree_commit: greedy acceptance on a verified tree and the commit
 * of its accepted path.  Per sequence b (t = kv->seq_lens[b] on entry):
 * from the root, follow the lowest row whose parent is the current row and
 * whose token equals the current row's AR argmax g; emit the followed
 * tokens and then g of the last row reached (n = path length + 1); the
 * K/V of the i-th accepted node move from cache slot t + row to slot t + i
 * in every layer and KV head; kv->seq_lens[b] += n; anchor[b] = the last
 * emitted token.
 *   parent, token, g  device int32 [batch][rows] (g: the AR argmax of each
 *                     tree row's logits)
 *   n_rows            device int32 [batch]: valid rows of each tree
 *   n_out             device int32 [batch]
 *   emit              device int32 [batch][rows]: tokens 0 .. n-1
 *   anchor            device int32 [batch], written
 * Requires 1 <= batch <= max_batch and 1 <= rows <= min(max_block, 128).
 * A parent outside [0, r) or a g outside [0, vocab) raises
 * ORTHRUS_DEVERR_TOKEN; slots beyond the sequence's pages raise
 * ORTHRUS_DEVERR_CAPACITY (those rows are not moved).
 */
orthrus_status_t orthrus_tree_commit(orthrus_ctx_t *ctx, const orthrus_kv_t *kv, int32_t batch, int32_t rows,
                                     const int32_t *parent, const int32_t *token, const int32_t *n_rows,
                                     const int32_t *g, int32_t *n_out, int32_t *emit, int32_t *anchor,
                                     void *stream);

/*
 * Test and measurement hook: the logits of the last verify (which = 0) or
 * draft (which = 1) for every block row, fp32 [batch][K][vocab], computed
 * from the final hidden rows the step kept (one extra LM-head pass; the
 * decode path itself never writes logits).
 */
orthrus_status_t orthrus_debug_logits(orthrus_ctx_t *ctx, int32_t which, int32_t batch, int32_t K,
                                      float *logits, void *stream);

/*
 * Test hook: the per-row results the last verify (which = 0) or draft
 * (which = 1) left for consensus, for batch x K rows in [b][k] order —
 *   which = 0: tok = the AR argmax g_k, logprob = log p_k(y_k) of the
 *              verified token (log softmax(z/T) at T > 0, of z at T = 0),
 *              lse = log-sum-exp of z/T (of z at T = 0);
 *   which = 1: tok = the drafted token y_k (argmax, or the Gumbel-max
 *              sample at T > 0), logprob = log q_k(y_k), lse likewise of
 *              the diffusion view's logits.
 * tok (int32), logprob and lse (fp32) are device [batch][K]; any may be
 * NULL.  Device-to-device copies on the stream, no arithmetic.
 */
orthrus_status_t orthrus_debug_rows(orthrus_ctx_t *ctx, int32_t which, int32_t batch, int32_t K, int32_t *tok,
                                    float *logprob, float *lse, void *stream);

/*
 * Measurement hook.  While set, every forward of `view` (0 = AR: verify,
 * prefill and plain AR steps; 1 = diffusion draft) records caller-owned CUDA
 * events (cudaEvent_t passed as void*) on the launch stream around the
 * launches of layer `layer`: starts[i] just before and stops[i] just after
 * launch i of kernel family `family` (0 = the four projection GEMMs in the
 * order QKV, O, gate/up, down; 1 = the attention split and combine kernels
 * as one bracket).  Each family has its own probe; slots are used
 * cyclically (i = hit mod n).  n = 0 disables that family's probe.  The arrays are copied; the events must outlive the
 * probe.  Not for use while a stream is being captured.
 */
orthrus_status_t orthrus_set_probe(orthrus_ctx_t *ctx, int32_t family, int32_t layer, int32_t view,
                                   void *const *starts, void *const *stops, int32_t n);

/* Number of kernel launches the context has enqueued since orthrus_create
 * (host-side count; a CUDA-graph replay of captured calls adds nothing). */
uint64_t orthrus_launch_count(const orthrus_ctx_t *ctx);

/* Synchronises `stream`, returns and clears the device error word (*bits may
 * be NULL). */
orthrus_status_t orthrus_check_error(orthrus_ctx_t *ctx, void *stream, uint32_t *bits);

const char *orthrus_status_string(orthrus_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* ORTHRUS_H */
