// Internal declarations of the dual-view decode library: the context, the
// workspace carve-up and the kernel launchers.  Not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <unordered_map>
#include <vector>

#include "../../include/orthrus.h"

namespace orthrus {

constexpr int kTileN = 128;          // GEMM tile: output features per tile
constexpr int kTileM = 32;           // GEMM tile: token rows per tile
constexpr int kTileK = 64;           // GEMM k chunk
constexpr int kKeyTile = 64;         // attention: keys per tile
constexpr int kPrefillChunk = 128;   // prefill rows per forward
constexpr int kNumSMs = 148;
// Contexts this long spread each attention row group over up to
// kAttnMaxClusters clusters.
constexpr int kAttnTwoClusterSeq = 8192;
constexpr int kAttnMaxClusters = 4;
constexpr int kResidSlots = 8;   // most k segments of a deferred residual GEMM

// Per-(row, vocab tile) record of the fused LM-head epilogue.
struct LmPart {
    float zmax;   // max logit in the tile
    float zsum;   // sum over the tile of exp((z - zmax) / T)
    int zarg;     // lowest index attaining zmax
    float gbest;  // best z/T + Gumbel (draft / AR sampling), or best residual score
    int garg;     // its index
    float gz;     // logit at garg
    float zid;    // logit at the row's given id, NaN if the id is not in the tile
    float zez;    // draft rows: sum over the tile of exp((z - zmax) / T) * z (the entropy's mean logit)
};

// One of the kTopWMax best logits of a (row, vocab tile), for the draft's
// top-W candidates (tree verification).
struct TopRec {
    float z;
    int id;
};

// Per-(row pair, vocab tile) record of the fused forward-KL epilogue: rows
// 2i (AR view) and 2i+1 (diffusion view) of the same position.
struct KlPart {
    float ma;    // max AR logit in the tile
    float sa;    // sum over the tile of exp(z_AR - ma)
    float ta;    // sum over the tile of exp(z_AR - ma) (z_AR - z_diff)
    float md;    // max diffusion logit in the tile
    float sd;    // sum over the tile of exp(z_diff - md)
    int pad[3];
};
static_assert(sizeof(KlPart) == sizeof(LmPart), "KL records share the LM-head record buffer");

enum Epi : int { EPI_QKV = 0, EPI_RESID = 1, EPI_SWIGLU = 2, EPI_LMHEAD = 3, EPI_RESAMPLE = 4, EPI_LOGITS = 5,
                 EPI_KL = 6 };

// Where an attention / QKV call reads positions and writes K/V.
struct KvView {
    void *k_pages, *v_pages;
    const int32_t *block_table;
    int num_pages, page_size, max_pages;
};

// One GEMM launch: Y[M][N] = X[M][Kd] . W^T with a fused epilogue.
struct GemmArgs {
    const void *x;           // [M][Kd] activations, dtype
    int M, N, Kd;
    // weight rows: concatenation of up to three matrices (QKV) or, for the
    // SwiGLU epilogue, tile halves [0,64) from w[0] and [64,128) from w[1]
    const void *w[3];
    int wrows[3];
    int splits;              // partial / flag slots per (m tile, n tile): the most pieces a tile is cut into
    float *part;             // [m tile][n tile][slot] fp32 partial tiles of a cut n tile
    int *ticket;             // [m tile][n tile][slot] published flags (reset by the tile's reducer)
    unsigned *err;
    int epi;
    // EPI_RESID
    float *resid;            // [M][N] fp32, += result
    // deferred residual (tensor-core path): the k segments of each tile are
    // written to rpart[seg][row][N] and summed into resid by the next RMSNorm
    int defer;               // segments per tile (0: add in the epilogue)
    int pair;                // tensor-core path: 2 or 3 k segments per n tile, reduced inside a cluster (0: off)
    // tensor-core path: ring stages whose weight tiles are requested before
    // waiting for the predecessor grid (0: the whole ring)
    int prewait_stages;
    float *rpart;
    int rpart_rows;
    // EPI_SWIGLU
    void *act;               // [M][N/2] dtype
    // EPI_QKV
    void *q_out;             // [M][n_q*hd]
    int n_q, n_kv, hd, layer;
    int kv_to_cache;         // 1: K/V into pages at (b, pos); 0: into k_blk/v_blk
    void *k_blk, *v_blk;     // transient layouts of AttnArgs (kv_to_cache == 0)
    int kp, bmax;
    KvView kv;
    const int32_t *pos0;     // [batch] position of block row 0
    const int32_t *bt_rows;  // [batch] row of block_table for each batch entry
    int K;                   // rows per sequence in this launch
    // tree verify: row (b, k) is rotated for position pos0[b] + rope_pos[b*K + k]
    // (its depth in the tree) while its K/V still go to slot pos0[b] + k; null:
    // position = slot
    const int32_t *rope_pos;
    double rope_theta;
    const double *rope_invf; // [head_dim / 2] theta^(-2i / head_dim), computed once on the host
    // EPI_LMHEAD / EPI_RESAMPLE
    LmPart *lm;              // [M][n_vtiles]
    float inv_temp;          // 1/T (T > 0) or 0 for greedy
    uint64_t seed;
    const int64_t *step;
    int lm_mode;             // 0 verify (zid from given ids), 1 draft (Gumbel), 2 AR sample
    int draft_pass;          // lm_mode 1: pass of an iterative draft (Gumbel purpose DRAFT | pass << 8)
    int topw;                // lm_mode 1: keep each (row, tile)'s topw best logits in top (0: off)
    TopRec *top;             // [M][n_vtiles][kTopWMax]
    const int32_t *given;    // [M] id whose logit is wanted (verify), or null
    const float *lse_p, *lse_q;   // EPI_RESAMPLE: per (b, k) row
    const int32_t *rej_row;  // EPI_RESAMPLE: [batch] j or -1
    const int *any_flag;     // EPI_RESAMPLE: skip everything when 0
    float *logits;           // EPI_LOGITS: [M][N] fp32
    KlPart *kl;              // EPI_KL: [M / 2][n_vtiles]
};

struct AttnArgs {
    const void *q;           // [B*K][n_q][hd]
    void *out;               // [B*K][n_q][hd]
    // mode 1: the block's transient K/V (all layers), K as
    // [n_layers][bmax][n_kv][kp][hd] and V transposed as
    // [n_layers][bmax][n_kv][hd][kp]; rows >= K of a slice are ignored
    const void *k_blk, *v_blk;
    int kp, bmax;
    int blk_layer, blk_layers;   // layer index into, and layer count of, k_blk / v_blk
    KvView kv;
    int layer;
    const int32_t *seq_lens;  // [batch] t per sequence (positions of block row 0)
    const int32_t *bt_rows;   // [batch] block-table row
    int B, K, n_q, n_kv, hd, mode;
    // n_splits = partial-buffer stride: cache splits of the longest sequence
    // plus one slot (the last) for the diffusion block's own keys
    int split_tokens, n_splits;
    float *part;             // [B*K][n_q][n_splits][hd]
    float2 *ml;              // [B*K][n_q][n_splits]
    // tensor-core path, xz > 1: up to xz clusters per (sequence, KV head,
    // row group) merged through [xz][xrows][hd] fp32 partial rows,
    // [xz][xrows] (m, l) and a ticket per owner CTA (zero between calls);
    // xrows = row capacity x n_q.  xz == 1 (or no buffers): one cluster.
    float *xo;
    float2 *xml;
    int *xcnt;
    int xrows, xz;
    // mode 0 tree verify (K <= 128): bit j of tree_mask[(b*K + k)*4 + j/32]
    // set when block row j is row k's ancestor or row k itself; row k then
    // sees cache keys [0, t) and exactly those block keys.  Null: causal.
    const uint32_t *tree_mask;
    unsigned *err;
};

// Tensor maps are looked up by (base pointer, box rows).
struct TmapKey {
    const void *ptr;
    uint32_t box_rows;
    bool operator==(const TmapKey &o) const { return ptr == o.ptr && box_rows == o.box_rows; }
};
struct TmapKeyHash {
    size_t operator()(const TmapKey &k) const { return std::hash<const void *>()(k.ptr) ^ (size_t)k.box_rows * 0x9E3779B97F4A7C15ull; }
};

// Attention tensor maps are cached per (buffers, shape).
struct AttnMapKey {
    const void *q, *kc, *vc, *kb;
    int num_pages, page_size, K, mode, q_rows;
    bool operator==(const AttnMapKey &o) const
    {
        return q == o.q && kc == o.kc && vc == o.vc && kb == o.kb && num_pages == o.num_pages &&
               page_size == o.page_size && K == o.K && mode == o.mode && q_rows == o.q_rows;
    }
};
struct AttnMapKeyHash {
    size_t operator()(const AttnMapKey &k) const
    {
        size_t h = std::hash<const void *>()(k.q) ^ (std::hash<const void *>()(k.kc) << 1) ^
                   (std::hash<const void *>()(k.kb) << 2);
        return h ^ ((size_t)k.K * 131 + (size_t)k.mode * 7 + (size_t)k.num_pages * 1000003 + (size_t)k.q_rows);
    }
};

struct Ctx {
    orthrus_config_t cfg;
    mutable std::unordered_map<AttnMapKey, std::vector<unsigned char>, AttnMapKeyHash> amaps;
    std::unordered_map<TmapKey, CUtensorMap, TmapKeyHash> tmaps;   // bf16 TMA maps of weights and activations
    std::vector<orthrus_layer_weights_t> layers;
    const void *embed, *final_norm, *lm_head;
    int esize;               // bytes per element of the dtype
    int R;                   // decode rows: max_batch * max_block
    int Rw;                  // rows of the forward buffers: max(R, prefill chunk)
    int n_splits;            // attention split stride
    int n_vtiles;            // LM-head vocab tiles
    int dev;
    // workspace carve-up (device pointers)
    float *h;                // [Rw][d]
    void *a;                 // [Rw][d]
    void *q;                 // [Rw][n_q*hd]
    void *attn_o;            // [Rw][n_q*hd]
    void *act;               // [Rw][F]
    void *k_diff, *v_diff;   // [n_layers][max_batch][n_kv][kp][hd] and [..][hd][kp] (V transposed)
    int kp;                  // max_block rounded up to a multiple of 64
    void *fin_draft, *fin_verify;  // [R][d]
    void *res_x;             // [2*max_batch][d]
    float *attn_part;        // [Rw][n_q][n_splits][hd]
    float2 *attn_ml;         // [Rw][n_q][n_splits]
    int attn_simt_rows;      // token rows attn_part / attn_ml hold (0: none; the tensor-core attention needs none)
    float *attn_xo;          // [kAttnMaxClusters][Rw][n_q][hd] (long contexts only, else null)
    float2 *attn_xml;        // [kAttnMaxClusters][Rw][n_q]
    int *attn_xcnt;          // [Rw][n_kv][8] tickets
    int attn_xz;             // most clusters per attention row group (1: short contexts)
    float *gemm_part;
    size_t gemm_part_floats;
    int *gemm_ticket;
    void *blk_pack;          // [2][max_batch][n_kv][kp][hd]: user block K/V repacked (standalone attention)
    int gemm_tickets;
    float *resid_part;       // [kResidSlots][Rw][hidden] deferred residual segments
    double *rope_invf;       // [head_dim / 2] rotary inverse frequencies
    LmPart *lm_part;         // [max(R, 2*max_batch)][n_vtiles]
    TopRec *top_part;        // [R][n_vtiles][kTopWMax] the draft rows' per-tile top-W
    int32_t *tok;            // [Rw] block tokens
    int32_t *tree_tok, *tree_depth;   // [R] tree verify: row tokens and depths
    uint32_t *tree_mask;     // [R][4] tree verify: ancestor bit masks
    int32_t *pos0;           // [max_batch]
    int32_t *bt_rows;        // [max_batch] identity rows 0..max_batch-1
    int32_t *bt_zero;        // [max_batch] zeros (every entry reads block-table row 0)
    int32_t *prefill_row;    // [1]
    int32_t *draft;          // [R]
    float *logq, *lse_q;     // [R]
    float *ent;              // [R] entropy of each draft row's distribution
    int32_t *g;              // [R]
    float *logp, *lse_p;     // [R]
    int32_t *rej_row;        // [max_batch]
    int32_t *res_tok;        // [max_batch]
    int *any_reject;         // [1]
    unsigned *err;           // [1]
    int32_t *produced;       // [max_batch]
    int64_t *step;           // [1]
    int32_t *n_buf, *tok_buf, *anchor_buf;  // generate scratch
    // host-side measurement state
    mutable uint64_t launches = 0;
    struct Probe {
        int layer = -1, view = -1;
        std::vector<cudaEvent_t> start, stop;
        uint64_t hits = 0;
    } probe[2];                 // 0: projection GEMMs, 1: attention
};

struct Layout {
    size_t total;
    size_t off[40];
};

// workspace carve-up shared by orthrus_workspace_size and orthrus_create
size_t plan_workspace(const orthrus_config_t &c, Ctx *ctx);

bool use_tensor_cores(const orthrus_config_t &c);

// ---------------------------------------------------------------- launchers
cudaError_t launch_gemm(const Ctx &c, GemmArgs a, cudaStream_t s);
cudaError_t gemm_init_attributes();
cudaError_t gemm_tc_init_attributes();
bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool make_tmap_box(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_cols, uint32_t box_rows);
// Tensor maps of one tensor-core attention call.
struct AtMaps {
    CUtensorMap kc;   // 2-D cache K rows [slot rows][128], box {64, 64}
    CUtensorMap vc;   // 2-D cache V^T rows [dim rows][page_size], box {64, 128}
    CUtensorMap kb;   // 2-D transient K [rows][128], box {64, 64}
    CUtensorMap vb;   // 2-D transient V^T [dim rows][Kp], box {64, 128}
};
cudaError_t attn_tc_init_attributes();
cudaError_t launch_gemm_tc(const Ctx &c, const GemmArgs &a, int n_mt, int tm, int n_nt, cudaStream_t s);
// Token tiles of the tensor-core GEMM for M token rows: n_mt tiles of tm rows
// (a multiple of 32, at most 256, as even as the multiple allows).
void gemm_token_tile(int M, int *n_mt, int *tm);
constexpr int kTcTokenTileMax = 256;
int sk_max_segments(int n_nt, int chunks);
cudaError_t attention_init_attributes();
// The attention of one call: the tensor-core kernel when the shape and the
// buffers allow it (attn_tc_shape_ok and tensor maps that encode), else the
// SIMT split kernel and its combine.  Their partials (a.part / a.ml, stride
// a.n_splits) hold simt_rows token rows; a call of more rows than that
// (simt_rows = 0: none reserved) launches nothing and returns
// cudaErrorNotSupported instead of falling back.
cudaError_t launch_attention(const Ctx &c, const AttnArgs &a, cudaStream_t s, int q_rows, int simt_rows);
cudaError_t launch_attention_simt(const Ctx &c, const AttnArgs &a, cudaStream_t s);
// bf16, head_dim 128, GQA group dividing 128, pages of a multiple of 64 slots
bool attn_tc_shape_ok(int dtype, int hd, int n_q, int n_kv, int page_size);
cudaError_t launch_attn_tc_cached(const Ctx &c, const AttnArgs &a, int n_split_grid, int q_rows, cudaStream_t s);
cudaError_t launch_attn_tc(const AttnArgs &a, const AtMaps &maps, int n_split_grid, cudaStream_t s);
bool attn_tc_maps(const AttnArgs &a, int n_layers, AtMaps *m);
cudaError_t launch_embed(const Ctx &c, int mode, const int32_t *tokens, const int32_t *anchor,
                         const int32_t *draft, int B, int K, cudaStream_t s);
cudaError_t launch_rmsnorm(const Ctx &c, float *h, const void *gain, void *out, int M, int pending, cudaStream_t s);
int resid_defer_slots(const orthrus_config_t &cfg, int N, int Kd);
cudaError_t launch_lm_finalize(const Ctx &c, int mode, int B, int K, float temperature, uint64_t seed,
                               const int64_t *step, int32_t *tok_out, cudaStream_t s);
// The draft rows' top-W from the per-tile records: rows k < depth of each
// sequence to ids / vals [B][depth][W] and their log-sum-exps to lse [B][depth].
cudaError_t launch_topw_finalize(const Ctx &c, int B, int K, int depth, int W, int32_t *ids, float *vals, float *lse,
                                 cudaStream_t s);
cudaError_t launch_commit(const Ctx &c, const orthrus_kv_t &kv, int B, int K, float temperature, uint64_t seed,
                          int64_t *step, const int32_t *force_n, int32_t *n_out, int32_t *tokens_out,
                          int32_t *anchor_io, int32_t *append_out, int append_stride, int append_max,
                          cudaStream_t s, const int32_t *kt = nullptr);
cudaError_t launch_adaptive_len(const Ctx &c, int B, int K, float h_max, int32_t *kt, float *ent_out, cudaStream_t s);
cudaError_t launch_ar_commit(const Ctx &c, const orthrus_kv_t &kv, int B, int64_t *step,
                             int32_t *token_out, int32_t *anchor_io, int32_t *append_out, int append_stride,
                             int append_max, cudaStream_t s);
cudaError_t launch_set_lens(const Ctx &c, int32_t *seq_lens, int b, int value, int32_t *anchor_out,
                            const int32_t *tokens, cudaStream_t s);
cudaError_t launch_pack_block(const Ctx &c, const void *k_src, const void *v_src, void *k_dst, void *v_dst, int B,
                              int K, int kp, cudaStream_t s);
cudaError_t launch_logits_dump(const Ctx &c, const void *fin, int M, float *logits, cudaStream_t s);
// Tree verification (tree.cu): the draft tree's builder and its commit.
struct TreeBuildArgs {   // one best-first tree per sequence
    const int32_t *ids;      // [B][D][W] candidate ids, best first
    const float *vals;       // [B][D][W] their logits
    const float *lse;        // [B][D]
    int D, W, N;
    int32_t *parent, *token, *depth;   // [B][N+1]
    double *score;                     // [B][N+1]
    int32_t *n_rows;                   // [B]
};

struct TreeCommitArgs {
    KvView kv;
    int32_t *seq_lens;
    int rows, n_layers, n_kv, hd, vocab;
    const int32_t *parent, *token, *g;   // [B][rows]
    const int32_t *n_rows;               // [B]
    int32_t *n_out, *emit, *anchor;      // [B], [B][rows], [B]
    unsigned *err;
};

cudaError_t launch_tree_prep(const Ctx &c, const int32_t *anchor, const int32_t *parent, const int32_t *token, int B,
                             int R, cudaStream_t s);
cudaError_t launch_tree_topw(const Ctx &c, const float *logits, int rows, int W, int32_t *ids, float *vals,
                             float *lse, cudaStream_t s);
cudaError_t launch_tree_build(const Ctx &c, const TreeBuildArgs &a, int B, cudaStream_t s);
cudaError_t launch_tree_commit(const Ctx &c, const TreeCommitArgs &a, int B, cudaStream_t s);
cudaError_t launch_kl_lm_head(const Ctx &c, const void *h_a, const void *h_d, int rows, float *kl, float *lse_a,
                              float *lse_d, cudaStream_t s);

}  // namespace orthrus
