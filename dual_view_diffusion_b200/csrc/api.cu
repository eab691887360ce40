// C ABI of the dual-view decode library (declared in include/orthrus.h).
//
// Host orchestration only: argument checks, the workspace carve-up, and the
// order of kernel launches for prefill, the draft forward (diffusion view),
// the verify forward (AR view), consensus/commit and plain AR decoding
// ("Orthrus: Memory-Efficient Parallel Token Generation via Dual-View
// Diffusion", paper notes §2.1-§2.3 and §4.1-§4.3).  Every step of the
// arithmetic runs in the kernels.
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <type_traits>
#include <cmath>
#include <vector>

#include "common.cuh"
#include "internal.h"

struct orthrus_ctx : orthrus::Ctx {};

namespace orthrus {

cudaError_t launch_set_int(int32_t *p, int v, cudaStream_t s);
cudaError_t launch_lm_finalize_impl(const Ctx &c, int mode, int B, int K, float temperature, int32_t *tok_out,
                                    const int32_t *given, cudaStream_t s);

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static bool valid_config(const orthrus_config_t &c)
{
    if (c.n_layers < 1 || c.hidden < 1 || c.n_q_heads < 1 || c.n_kv_heads < 1 || c.ffn < 1 || c.vocab < 2)
        return false;
    if (c.n_q_heads % c.n_kv_heads) return false;
    if (c.head_dim != 16 && c.head_dim != 32 && c.head_dim != 64 && c.head_dim != 128) return false;
    if (c.mask_token_id < 0 || c.mask_token_id >= c.vocab) return false;
    if (c.dtype != ORTHRUS_BF16 && c.dtype != ORTHRUS_FP32) return false;
    if (c.max_batch < 1 || c.max_batch > 128 || c.max_block < 1 || c.max_block > 4096) return false;
    if (c.split_tokens < 64 || c.split_tokens % 64) return false;
    if (c.max_seq < c.max_block + 1) return false;
    if (!(c.rope_theta > 0.f) || !(c.rms_eps > 0.f)) return false;
    return true;
}

// Largest split-partial buffer and ticket count any projection of this
// model needs with up to `rows` token rows.
static void gemm_scratch(const orthrus_config_t &c, int rows_body, int rows_lm, size_t *floats, int *tickets)
{
    const int d = c.hidden, hq = c.n_q_heads * c.head_dim, hk = c.n_kv_heads * c.head_dim;
    struct Shape { int n_tiles, Kd, rows; };
    const Shape shapes[] = {
        {(hq + 2 * hk + kTileN - 1) / kTileN, d, rows_body},
        {(d + kTileN - 1) / kTileN, hq, rows_body},
        {(c.ffn + 63) / 64, d, rows_body},
        {(d + kTileN - 1) / kTileN, c.ffn, rows_body},
        {(c.vocab + kTileN - 1) / kTileN, d, rows_lm},
    };
    *floats = 0;
    *tickets = 1;
    for (const Shape &s : shapes) {
        const int S = (use_tensor_cores(c) && s.Kd % kTileK == 0) ? sk_max_segments(s.n_tiles, s.Kd / kTileK) : 1;
        // the largest token tiles x tile rows any M up to s.rows uses
        size_t rows_mt = 0, n_mt_max = 0;
        for (int M = 1; M <= s.rows; M += (M < 256 ? 1 : 32)) {
            int n_mt, tm;
            gemm_token_tile(M, &n_mt, &tm);
            rows_mt = std::max(rows_mt, (size_t)n_mt * tm);
            n_mt_max = std::max(n_mt_max, (size_t)n_mt);
        }
        {
            int n_mt, tm;
            gemm_token_tile(s.rows, &n_mt, &tm);
            rows_mt = std::max(rows_mt, (size_t)n_mt * tm);
            n_mt_max = std::max(n_mt_max, (size_t)n_mt);
        }
        const size_t n_mt32 = (s.rows + kTileM - 1) / kTileM;
        if (S > 1) *floats = std::max(*floats, rows_mt * s.n_tiles * S * kTileN);
        *tickets = std::max(*tickets, (int)(std::max(n_mt32, n_mt_max) * s.n_tiles * S));
    }
}

size_t plan_workspace(const orthrus_config_t &c, Ctx *x)
{
    const size_t es = c.dtype == ORTHRUS_BF16 ? 2 : 4;
    const size_t d = c.hidden, hq = (size_t)c.n_q_heads * c.head_dim, hk = (size_t)c.n_kv_heads * c.head_dim;
    const size_t F = c.ffn, L = c.n_layers, mb = c.max_batch;
    const size_t R = mb * c.max_block;
    const size_t Rw = std::max(R, (size_t)kPrefillChunk);
    const size_t Rlm = std::max(R, 2 * mb);
    // cache splits of the longest sequence plus one slot for the diffusion block
    const size_t n_splits = (c.max_seq + c.split_tokens - 1) / c.split_tokens + 1;
    const size_t kp = ((size_t)c.max_block + 63) / 64 * 64;
    const size_t n_vtiles = (c.vocab + kTileN - 1) / kTileN;
    size_t gfloats;
    int gtickets;
    gemm_scratch(c, (int)Rw, (int)Rlm, &gfloats, &gtickets);

    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
    const size_t o_h = take(Rw * d * 4), o_a = take(Rw * d * es), o_q = take(Rw * hq * es), o_o = take(Rw * hq * es);
    const size_t o_act = take(Rw * F * es);
    const size_t o_kd = take(L * mb * kp * hk * es), o_vd = take(L * mb * kp * hk * es);
    const size_t o_bp = take(2 * mb * kp * hk * es);
    const size_t o_fd = take(R * d * es), o_fv = take(R * d * es), o_rx = take(2 * mb * d * es);
    // attention partials [Rw][n_q][n_splits][hd] fp32 and [Rw][n_q][n_splits]
    // float2: only the SIMT attention uses them (the tensor-core attention
    // combines its splits on chip)
    // (pages of a multiple of 64 slots are required of the bf16 head_dim-128
    // path, so they do not decide it here)
    const bool simt_attn = !attn_tc_shape_ok(c.dtype, c.head_dim, c.n_q_heads, c.n_kv_heads, 64);
    const size_t o_part = take(simt_attn ? Rw * c.n_q_heads * n_splits * c.head_dim * 4 : 0);
    const size_t o_ml = take(simt_attn ? Rw * c.n_q_heads * n_splits * 8 : 0);
    // long contexts: the tensor-core attention spreads a row group over up
    // to kAttnMaxClusters clusters and merges them through these (one
    // ticket per owner CTA)
    const bool attn_x2 = !simt_attn && c.max_seq >= kAttnTwoClusterSeq;
    const size_t o_xo = take(attn_x2 ? kAttnMaxClusters * Rw * c.n_q_heads * c.head_dim * 4 : 0);
    const size_t o_xml = take(attn_x2 ? kAttnMaxClusters * Rw * c.n_q_heads * 8 : 0);
    const size_t o_xc = take(attn_x2 ? Rw * c.n_kv_heads * 8 * 4 : 0);
    const size_t o_gp = take(std::max(gfloats, (size_t)1) * 4), o_gt = take((size_t)gtickets * 4);
    const int rslots = std::max(resid_defer_slots(c, c.hidden, c.n_q_heads * c.head_dim), resid_defer_slots(c, c.hidden, c.ffn));
    const size_t o_rp = take((size_t)rslots * Rw * d * 4);
    const size_t o_invf = take((size_t)c.head_dim / 2 * 8);
    const size_t o_lm = take(Rlm * n_vtiles * sizeof(LmPart));
    const size_t o_top = take(R * n_vtiles * kTopWMax * sizeof(TopRec));
    const size_t o_tok = take(Rw * 4), o_pos = take(mb * 4), o_bt = take(mb * 4), o_pr = take(4);
    const size_t o_ttok = take(R * 4), o_tdep = take(R * 4), o_tmask = take(R * 16);
    const size_t o_bz = take(mb * 4);   // zeros, never written
    const size_t o_dr = take(R * 4), o_lq = take(R * 4), o_lsq = take(R * 4), o_g = take(R * 4), o_lp = take(R * 4),
                 o_lsp = take(R * 4), o_ent = take(R * 4);
    const size_t o_rj = take(mb * 4), o_rt = take(mb * 4), o_any = take(4), o_err = take(4), o_prod = take(mb * 4),
                 o_step = take(8), o_nb = take(mb * 4), o_tb = take(R * 4), o_ab = take(mb * 4);
    const size_t total = off;
    if (x) {
        char *base = (char *)nullptr;
        auto P = [&](size_t o) { return (void *)(base + o); };
        x->h = (float *)P(o_h); x->a = P(o_a); x->q = P(o_q); x->attn_o = P(o_o); x->act = P(o_act);
        x->k_diff = P(o_kd); x->v_diff = P(o_vd); x->fin_draft = P(o_fd); x->fin_verify = P(o_fv); x->res_x = P(o_rx);
        x->attn_part = (float *)P(o_part); x->attn_ml = (float2 *)P(o_ml);
        x->attn_simt_rows = simt_attn ? (int)Rw : 0;
        x->attn_xo = attn_x2 ? (float *)P(o_xo) : nullptr; x->attn_xml = attn_x2 ? (float2 *)P(o_xml) : nullptr;
        x->attn_xcnt = attn_x2 ? (int *)P(o_xc) : nullptr; x->attn_xz = attn_x2 ? kAttnMaxClusters : 1;
        x->gemm_part = (float *)P(o_gp); x->gemm_part_floats = gfloats; x->gemm_ticket = (int *)P(o_gt);
        x->gemm_tickets = gtickets; x->lm_part = (LmPart *)P(o_lm); x->top_part = (TopRec *)P(o_top);
        x->resid_part = (float *)P(o_rp);
        x->rope_invf = (double *)P(o_invf);
        x->tok = (int32_t *)P(o_tok); x->pos0 = (int32_t *)P(o_pos); x->bt_rows = (int32_t *)P(o_bt);
        x->bt_zero = (int32_t *)P(o_bz);
        x->tree_tok = (int32_t *)P(o_ttok); x->tree_depth = (int32_t *)P(o_tdep); x->tree_mask = (uint32_t *)P(o_tmask);
        x->prefill_row = (int32_t *)P(o_pr);
        x->draft = (int32_t *)P(o_dr); x->logq = (float *)P(o_lq); x->lse_q = (float *)P(o_lsq);
        x->ent = (float *)P(o_ent);
        x->g = (int32_t *)P(o_g); x->logp = (float *)P(o_lp); x->lse_p = (float *)P(o_lsp);
        x->rej_row = (int32_t *)P(o_rj); x->res_tok = (int32_t *)P(o_rt); x->any_reject = (int *)P(o_any);
        x->err = (unsigned *)P(o_err); x->produced = (int32_t *)P(o_prod); x->step = (int64_t *)P(o_step);
        x->n_buf = (int32_t *)P(o_nb); x->tok_buf = (int32_t *)P(o_tb); x->anchor_buf = (int32_t *)P(o_ab);
        x->R = (int)R; x->Rw = (int)Rw; x->n_splits = (int)n_splits; x->n_vtiles = (int)n_vtiles;
        x->kp = (int)kp; x->blk_pack = P(o_bp);
        x->esize = (int)es;
    }
    return total;
}

static void rebase(Ctx *x, char *ws)
{
    auto fix = [&](auto *&p) { p = (std::remove_reference_t<decltype(p)>)(ws + (size_t)(const char *)p); };
    fix(x->h); fix(x->a); fix(x->q); fix(x->attn_o); fix(x->act); fix(x->k_diff); fix(x->v_diff); fix(x->blk_pack);
    fix(x->fin_draft); fix(x->fin_verify); fix(x->res_x); fix(x->attn_part); fix(x->attn_ml); fix(x->gemm_part);
    fix(x->gemm_ticket); fix(x->lm_part); fix(x->top_part); fix(x->resid_part); fix(x->rope_invf); fix(x->tok); fix(x->pos0); fix(x->bt_rows); fix(x->bt_zero); fix(x->prefill_row);
    fix(x->tree_tok); fix(x->tree_depth); fix(x->tree_mask);
    fix(x->draft); fix(x->logq); fix(x->lse_q); fix(x->ent); fix(x->g); fix(x->logp); fix(x->lse_p); fix(x->rej_row);
    fix(x->res_tok); fix(x->any_reject); fix(x->err); fix(x->produced); fix(x->step); fix(x->n_buf);
    fix(x->tok_buf); fix(x->anchor_buf);
    if (x->attn_xz > 1) { fix(x->attn_xo); fix(x->attn_xml); fix(x->attn_xcnt); }
}

// TMA maps for the tensor-core GEMM: every weight matrix (128-row boxes;
// 64-row boxes for gate/up, whose tiles pair 64 gate rows with 64 up rows)
// and every activation buffer a projection reads (32-row boxes).  A matrix
// whose inner size is not a multiple of 64 gets no map and runs on the SIMT
// kernel.
static void build_tmaps(Ctx *c)
{
    const orthrus_config_t &f = c->cfg;
    const int d = f.hidden, hq = f.n_q_heads * f.head_dim, hk = f.n_kv_heads * f.head_dim, F = f.ffn;
    auto add = [&](const void *p, int rows, int cols, uint32_t box) {
        if (!p || cols % kTileK) return;
        CUtensorMap m;
        if (make_tmap(&m, p, rows, cols, box)) c->tmaps[TmapKey{p, box}] = m;
    };
    // activation buffers: one map per token-tile height the GEMM may use
    auto add_x = [&](const void *p, int rows, int cols) {
        for (uint32_t box = kTileM; box <= (uint32_t)kTcTokenTileMax; box += kTileM) add(p, rows, cols, box);
    };
    for (const orthrus_layer_weights_t &L : c->layers) {
        add(L.wq, hq, d, kTileN); add(L.wk, hk, d, kTileN); add(L.wv, hk, d, kTileN);
        add(L.wq_diff, hq, d, kTileN); add(L.wk_diff, hk, d, kTileN); add(L.wv_diff, hk, d, kTileN);
        add(L.wo, d, hq, kTileN); add(L.w_gate, F, d, 64); add(L.w_up, F, d, 64); add(L.w_down, d, F, kTileN);
    }
    add(c->lm_head, f.vocab, d, kTileN);
    add_x(c->a, c->Rw, d); add_x(c->attn_o, c->Rw, hq); add_x(c->act, c->Rw, F);
    add_x(c->fin_draft, c->R, d); add_x(c->fin_verify, c->R, d);
    add_x(c->res_x, 2 * f.max_batch, d);
}

static KvView kv_view(const orthrus_kv_t &kv)
{
    return KvView{kv.k_pages, kv.v_pages, kv.block_table, kv.num_pages, kv.page_size, kv.max_pages_per_seq};
}

// Event probe (orthrus_set_probe): bracket a launch of the probed family in
// the probed layer and view.
struct ProbeScope {
    Ctx::Probe &p;
    bool on;
    size_t slot;
    cudaStream_t s;
    ProbeScope(Ctx &c, int family, int layer, int view, cudaStream_t s_)
        : p(c.probe[family]), on(!p.start.empty() && p.layer == layer && p.view == view), slot(0), s(s_)
    {
        if (on) {
            slot = p.hits++ % p.start.size();
            cudaEventRecord(p.start[slot], s);
        }
    }
    ~ProbeScope()
    {
        if (on) cudaEventRecord(p.stop[slot], s);
    }
};

// One forward of either view over B*K rows already embedded in c.h.
//   view 0: AR W_Q/W_K/W_V, K/V written into the cache, causal (mode 0)
//   view 1: diffusion W^diff, K/V into the transient buffer, block
//           bidirectional (mode 1)
// fin (nullable): final-norm rows for the LM head.
// rope_pos / tree_mask (view 0 only, nullable): the tree-masked verify's
// per-row rotary positions (depths) and ancestor masks.
static cudaError_t forward(Ctx &c, const orthrus_kv_t &kv, int view, int B, int K, const int32_t *pos0,
                           const int32_t *bt_rows, void *fin, cudaStream_t s, const int32_t *rope_pos = nullptr,
                           const uint32_t *tree_mask = nullptr)
{
    const orthrus_config_t &f = c.cfg;
    const int M = B * K, hd = f.head_dim;
    cudaError_t e;
    // residual segments the O and down projections leave for the next RMSNorm
    int pending = 0;
    const int defer_o = resid_defer_slots(f, f.hidden, f.n_q_heads * hd), defer_dn = resid_defer_slots(f, f.hidden, f.ffn);
    for (int l = 0; l < f.n_layers; ++l) {
        const orthrus_layer_weights_t &W = c.layers[l];
        if ((e = launch_rmsnorm(c, c.h, W.attn_norm, c.a, M, pending, s)) != cudaSuccess) return e;
        GemmArgs q{};
        q.x = c.a; q.M = M; q.Kd = f.hidden;
        q.w[0] = view ? W.wq_diff : W.wq; q.w[1] = view ? W.wk_diff : W.wk; q.w[2] = view ? W.wv_diff : W.wv;
        q.wrows[0] = f.n_q_heads * hd; q.wrows[1] = q.wrows[2] = f.n_kv_heads * hd;
        q.N = q.wrows[0] + 2 * q.wrows[1];
        q.epi = EPI_QKV; q.q_out = c.q; q.n_q = f.n_q_heads; q.n_kv = f.n_kv_heads; q.hd = hd; q.layer = l;
        q.kv_to_cache = view == 0; q.k_blk = c.k_diff; q.v_blk = c.v_diff; q.kp = c.kp; q.bmax = f.max_batch;
        q.kv = kv_view(kv); q.pos0 = pos0; q.bt_rows = bt_rows; q.K = K; q.rope_theta = (double)f.rope_theta;
        q.rope_invf = c.rope_invf; q.rope_pos = view == 0 ? rope_pos : nullptr;
        {
            ProbeScope ps(c, 0, l, view, s);
            if ((e = launch_gemm(c, q, s)) != cudaSuccess) return e;
        }

        AttnArgs at{};
        at.q = c.q; at.out = c.attn_o;
        at.k_blk = c.k_diff; at.v_blk = c.v_diff; at.kp = c.kp; at.bmax = f.max_batch;
        at.blk_layer = l; at.blk_layers = f.n_layers;
        at.kv = kv_view(kv); at.layer = l; at.seq_lens = pos0; at.bt_rows = bt_rows;
        at.B = B; at.K = K; at.n_q = f.n_q_heads; at.n_kv = f.n_kv_heads; at.hd = hd; at.mode = view;
        at.split_tokens = f.split_tokens; at.n_splits = c.n_splits; at.part = c.attn_part; at.ml = c.attn_ml;
        at.xo = c.attn_xo; at.xml = c.attn_xml; at.xcnt = c.attn_xcnt; at.xrows = c.Rw * f.n_q_heads;
        at.xz = c.attn_xz;
        at.tree_mask = view == 0 ? tree_mask : nullptr;
        at.err = c.err;
        {
            ProbeScope ps(c, 1, l, view, s);
            if ((e = launch_attention(c, at, s, c.Rw, c.attn_simt_rows)) != cudaSuccess) return e;
        }

        GemmArgs o{};
        o.x = c.attn_o; o.M = M; o.N = f.hidden; o.Kd = f.n_q_heads * hd; o.w[0] = W.wo; o.wrows[0] = f.hidden;
        o.epi = EPI_RESID; o.resid = c.h; o.defer = defer_o; o.rpart = c.resid_part; o.rpart_rows = c.Rw;
        // the attention before it is latency-bound: a full ring of weight
        // requests (16 MiB over the grid) issued while it runs delays its
        // own loads more than it saves here (measured on the 8B decode step)
        o.prewait_stages = 2;
        {
            ProbeScope ps(c, 0, l, view, s);
            if ((e = launch_gemm(c, o, s)) != cudaSuccess) return e;
        }

        if ((e = launch_rmsnorm(c, c.h, W.ffn_norm, c.a, M, defer_o, s)) != cudaSuccess) return e;
        GemmArgs gu{};
        gu.x = c.a; gu.M = M; gu.N = f.ffn; gu.Kd = f.hidden; gu.w[0] = W.w_gate; gu.w[1] = W.w_up;
        gu.wrows[0] = gu.wrows[1] = f.ffn; gu.epi = EPI_SWIGLU; gu.act = c.act;
        {
            ProbeScope ps(c, 0, l, view, s);
            if ((e = launch_gemm(c, gu, s)) != cudaSuccess) return e;
        }

        GemmArgs dn{};
        dn.x = c.act; dn.M = M; dn.N = f.hidden; dn.Kd = f.ffn; dn.w[0] = W.w_down; dn.wrows[0] = f.hidden;
        dn.epi = EPI_RESID; dn.resid = c.h; dn.defer = defer_dn; dn.rpart = c.resid_part; dn.rpart_rows = c.Rw;
        {
            ProbeScope ps(c, 0, l, view, s);
            if ((e = launch_gemm(c, dn, s)) != cudaSuccess) return e;
        }
        pending = defer_dn;
    }
    if (fin) return launch_rmsnorm(c, c.h, c.final_norm, fin, M, pending, s);
    return cudaSuccess;
}

static cudaError_t lm_head(Ctx &c, const void *fin, int B, int K, int lm_mode, float temperature, uint64_t seed,
                           const int64_t *step, const int32_t *given, cudaStream_t s, int draft_pass = 0, int topw = 0)
{
    GemmArgs g{};
    g.topw = topw; g.top = c.top_part;
    g.draft_pass = draft_pass;
    g.x = fin; g.M = B * K; g.N = c.cfg.vocab; g.Kd = c.cfg.hidden; g.w[0] = c.lm_head; g.wrows[0] = c.cfg.vocab;
    g.epi = EPI_LMHEAD; g.lm = c.lm_part; g.inv_temp = temperature > 0.f ? 1.0f / temperature : 0.f;
    g.seed = seed; g.step = step; g.lm_mode = lm_mode; g.given = given; g.K = K;
    return launch_gemm(c, g, s);
}

}  // namespace orthrus

using namespace orthrus;

// cudaErrorNotSupported: a launcher found no kernel for these arguments
// (e.g. the attention's buffers admit no tensor maps and the context holds no
// room for the SIMT kernel's partials); nothing was launched.
#define CK(x)                                                                              \
    do {                                                                                   \
        cudaError_t e_ = (x);                                                              \
        if (e_ == cudaErrorNotSupported) return ORTHRUS_ERR_UNSUPPORTED;                   \
        if (e_ != cudaSuccess) return ORTHRUS_ERR_CUDA;                                    \
    } while (0)

static bool kv_ok(const orthrus_ctx_t *c, const orthrus_kv_t *kv)
{
    if (!kv || !kv->k_pages || !kv->v_pages || !kv->block_table || !kv->seq_lens) return false;
    if (kv->num_pages < 1 || kv->max_pages_per_seq < 1) return false;
    if ((uintptr_t)kv->k_pages % 16 || (uintptr_t)kv->v_pages % 16) return false;
    const int ps_mult = (c->cfg.dtype == ORTHRUS_BF16 && c->cfg.head_dim == 128) ? 64 : 16;
    if (kv->page_size < ps_mult || kv->page_size % ps_mult) return false;
    return true;
}

extern "C" {

const char *orthrus_status_string(orthrus_status_t s)
{
    switch (s) {
    case ORTHRUS_OK: return "ok";
    case ORTHRUS_ERR_INVALID_ARG: return "invalid argument";
    case ORTHRUS_ERR_UNSUPPORTED: return "unsupported configuration";
    case ORTHRUS_ERR_CAPACITY: return "capacity exceeded";
    case ORTHRUS_ERR_CUDA: return "CUDA runtime error";
    case ORTHRUS_ERR_DEVICE_CHECK: return "device-side check failed";
    case ORTHRUS_ERR_NONFINITE: return "non-finite log-sum-exp";
    }
    return "unknown status";
}

orthrus_status_t orthrus_workspace_size(const orthrus_config_t *cfg, size_t *bytes)
{
    if (!cfg || !bytes) return ORTHRUS_ERR_INVALID_ARG;
    if (!valid_config(*cfg)) return ORTHRUS_ERR_INVALID_ARG;
    *bytes = plan_workspace(*cfg, nullptr);
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_transient_bytes(const orthrus_config_t *cfg, int32_t batch, int32_t K, size_t *bytes)
{
    if (!cfg || !bytes || !valid_config(*cfg) || batch < 1 || K < 1) return ORTHRUS_ERR_INVALID_ARG;
    if (batch > cfg->max_batch || K > cfg->max_block) return ORTHRUS_ERR_CAPACITY;
    const size_t es = cfg->dtype == ORTHRUS_BF16 ? 2 : 4;
    *bytes = (size_t)cfg->n_layers * batch * K * cfg->n_kv_heads * cfg->head_dim * 2 * es;
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_create(const orthrus_config_t *cfg, const orthrus_weights_t *w, void *workspace,
                                size_t ws_bytes, orthrus_ctx_t **out)
{
    if (!cfg || !w || !workspace || !out || !w->embed || !w->final_norm || !w->lm_head || !w->layers)
        return ORTHRUS_ERR_INVALID_ARG;
    if (!valid_config(*cfg)) return ORTHRUS_ERR_INVALID_ARG;
    if ((uintptr_t)workspace % 256) return ORTHRUS_ERR_INVALID_ARG;
    for (int l = 0; l < cfg->n_layers; ++l) {
        const orthrus_layer_weights_t &L = w->layers[l];
        if (!L.attn_norm || !L.wq || !L.wk || !L.wv || !L.wq_diff || !L.wk_diff || !L.wv_diff || !L.wo ||
            !L.ffn_norm || !L.w_gate || !L.w_up || !L.w_down)
            return ORTHRUS_ERR_INVALID_ARG;
    }
    orthrus_ctx_t *c = new (std::nothrow) orthrus_ctx_t();
    if (!c) return ORTHRUS_ERR_CAPACITY;
    c->cfg = *cfg;
    const size_t need = plan_workspace(*cfg, c);
    if (ws_bytes < need) { delete c; return ORTHRUS_ERR_CAPACITY; }
    rebase(c, (char *)workspace);
    c->layers.assign(w->layers, w->layers + cfg->n_layers);
    c->embed = w->embed; c->final_norm = w->final_norm; c->lm_head = w->lm_head;
    if (cudaGetDevice(&c->dev) != cudaSuccess || gemm_init_attributes() != cudaSuccess ||
        gemm_tc_init_attributes() != cudaSuccess || attention_init_attributes() != cudaSuccess) {
        delete c;
        return ORTHRUS_ERR_CUDA;
    }
    if (cfg->dtype == ORTHRUS_BF16) build_tmaps(c);
    std::vector<int32_t> ident(cfg->max_batch);
    for (int b = 0; b < cfg->max_batch; ++b) ident[b] = b;
    // rotary inverse frequencies theta^(-2i / head_dim), in double on the host
    std::vector<double> invf(cfg->head_dim / 2);
    for (int i = 0; i < cfg->head_dim / 2; ++i) invf[i] = std::pow((double)cfg->rope_theta, -2.0 * i / cfg->head_dim);
    if (cudaMemset(workspace, 0, need) != cudaSuccess ||
        cudaMemcpy(c->bt_rows, ident.data(), ident.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->rope_invf, invf.data(), invf.size() * 8, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
        delete c;
        return ORTHRUS_ERR_CUDA;
    }
    *out = c;
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_destroy(orthrus_ctx_t *c)
{
    if (!c) return ORTHRUS_ERR_INVALID_ARG;
    delete c;
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_prefill(orthrus_ctx_t *c, const orthrus_kv_t *kv, const int32_t *tokens, int32_t stride,
                                 const int32_t *lens, int32_t batch, int32_t *anchor_out, void *stream)
{
    if (!c || !kv_ok(c, kv) || !tokens || !lens || !anchor_out || batch < 1) return ORTHRUS_ERR_INVALID_ARG;
    if (batch > c->cfg.max_batch) return ORTHRUS_ERR_CAPACITY;
    cudaStream_t s = (cudaStream_t)stream;
    for (int b = 0; b < batch; ++b) {
        if (lens[b] < 1 || lens[b] > stride) return ORTHRUS_ERR_INVALID_ARG;
        if (lens[b] - 1 + c->cfg.max_block > c->cfg.max_seq ||
            lens[b] - 1 > kv->max_pages_per_seq * kv->page_size)
            return ORTHRUS_ERR_CAPACITY;
    }
    for (int b = 0; b < batch; ++b) {
        const int n = lens[b] - 1;
        CK(launch_set_int(c->prefill_row, b, s));
        c->launches += 1;
        for (int p0 = 0; p0 < n; p0 += c->Rw) {
            const int R = std::min(c->Rw, n - p0);
            CK(launch_set_int(c->pos0, p0, s));
            c->launches += 1;
            CK(launch_embed(*c, 2, tokens + (size_t)b * stride + p0, nullptr, nullptr, 1, R, s));
            CK(forward(*c, *kv, 0, 1, R, c->pos0, c->prefill_row, nullptr, s));
        }
        CK(launch_set_lens(*c, kv->seq_lens, b, n, anchor_out, tokens + (size_t)b * stride + n, s));
        c->launches += 1;
    }
    return ORTHRUS_OK;
}

static orthrus_status_t check_step(orthrus_ctx_t *c, const orthrus_kv_t *kv, int batch, int K)
{
    if (!c || !kv_ok(c, kv) || batch < 1 || K < 1) return ORTHRUS_ERR_INVALID_ARG;
    if (batch > c->cfg.max_batch || K > c->cfg.max_block) return ORTHRUS_ERR_CAPACITY;
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_draft_block(orthrus_ctx_t *c, const orthrus_kv_t *kv, const int32_t *anchor, int32_t batch,
                                     int32_t K, float temperature, uint64_t seed, const int64_t *step, int32_t *draft,
                                     void *stream)
{
    return orthrus_draft_block_iterative(c, kv, anchor, batch, K, 1, temperature, seed, step, draft, stream);
}

orthrus_status_t orthrus_draft_block_iterative(orthrus_ctx_t *c, const orthrus_kv_t *kv, const int32_t *anchor,
                                               int32_t batch, int32_t K, int32_t iterations, float temperature,
                                               uint64_t seed, const int64_t *step, int32_t *draft, void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, K);
    if (st != ORTHRUS_OK) return st;
    if (!anchor || !draft || (temperature > 0.f && !step) || temperature < 0.f || iterations < 1)
        return ORTHRUS_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    for (int pass = 0; pass < iterations; ++pass) {
        // pass 0: [anchor, mask x (K-1)]; later passes: [anchor, previous drafts]
        CK(launch_embed(*c, pass == 0 ? 0 : 1, nullptr, anchor, pass == 0 ? nullptr : draft, batch, K, s));
        CK(forward(*c, *kv, 1, batch, K, kv->seq_lens, c->bt_rows, c->fin_draft, s));
        CK(lm_head(*c, c->fin_draft, batch, K, 1, temperature, seed, step, nullptr, s, pass));
        CK(launch_lm_finalize_impl(*c, 1, batch, K, temperature, draft, nullptr, s));
    }
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_draft_block_topw(orthrus_ctx_t *c, const orthrus_kv_t *kv, const int32_t *anchor,
                                          int32_t batch, int32_t K, int32_t width, int32_t depth, int32_t *draft,
                                          int32_t *ids, float *vals, float *lse, void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, K);
    if (st != ORTHRUS_OK) return st;
    if (!anchor || !draft || !ids || !vals || !lse || width < 1 || width > kTopWMax || width > c->cfg.vocab ||
        depth < 1 || depth > K)
        return ORTHRUS_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    CK(launch_embed(*c, 0, nullptr, anchor, nullptr, batch, K, s));
    CK(forward(*c, *kv, 1, batch, K, kv->seq_lens, c->bt_rows, c->fin_draft, s));
    CK(lm_head(*c, c->fin_draft, batch, K, 1, 0.f, 0, nullptr, nullptr, s, 0, width));
    CK(launch_lm_finalize_impl(*c, 1, batch, K, 0.f, draft, nullptr, s));
    CK(launch_topw_finalize(*c, batch, K, depth, width, ids, vals, lse, s));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_verify_block(orthrus_ctx_t *c, const orthrus_kv_t *kv, const int32_t *anchor,
                                      const int32_t *draft, int32_t batch, int32_t K, float temperature, void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, K);
    if (st != ORTHRUS_OK) return st;
    if (!anchor || !draft || temperature < 0.f) return ORTHRUS_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    CK(launch_embed(*c, 1, nullptr, anchor, draft, batch, K, s));
    CK(forward(*c, *kv, 0, batch, K, kv->seq_lens, c->bt_rows, c->fin_verify, s));
    CK(lm_head(*c, c->fin_verify, batch, K, 0, temperature, 0, nullptr, draft, s));
    CK(launch_lm_finalize_impl(*c, 0, batch, K, temperature, nullptr, draft, s));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_commit(orthrus_ctx_t *c, const orthrus_kv_t *kv, int32_t batch, int32_t K, float temperature,
                                uint64_t seed, int64_t *step, const int32_t *force_n, int32_t *n_out,
                                int32_t *tokens_out, int32_t *anchor_io, void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, K);
    if (st != ORTHRUS_OK) return st;
    if (!step || !n_out || !anchor_io || temperature < 0.f) return ORTHRUS_ERR_INVALID_ARG;
    CK(launch_commit(*c, *kv, batch, K, temperature, seed, step, force_n, n_out, tokens_out, anchor_io, nullptr, 0, 0,
                     (cudaStream_t)stream));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_adaptive_len(orthrus_ctx_t *c, int32_t batch, int32_t K, float h_max, int32_t *kt,
                                      float *entropy, void *stream)
{
    if (!c || !kt || batch < 1 || K < 1 || h_max != h_max) return ORTHRUS_ERR_INVALID_ARG;
    if (batch > c->cfg.max_batch || K > c->cfg.max_block) return ORTHRUS_ERR_CAPACITY;
    CK(launch_adaptive_len(*c, batch, K, h_max, kt, entropy, (cudaStream_t)stream));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_commit_adaptive(orthrus_ctx_t *c, const orthrus_kv_t *kv, int32_t batch, int32_t K,
                                         const int32_t *kt, int64_t *step, int32_t *n_out, int32_t *tokens_out,
                                         int32_t *anchor_io, void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, K);
    if (st != ORTHRUS_OK) return st;
    if (!kt || !step || !n_out || !anchor_io) return ORTHRUS_ERR_INVALID_ARG;
    CK(launch_commit(*c, *kv, batch, K, 0.f, 0, step, nullptr, n_out, tokens_out, anchor_io, nullptr, 0, 0,
                     (cudaStream_t)stream, kt));
    return ORTHRUS_OK;
}

static orthrus_status_t ar_step_impl(orthrus_ctx_t *c, const orthrus_kv_t *kv, int batch, float temperature,
                                     uint64_t seed, int64_t *step, int32_t *token_out, int32_t *anchor_io,
                                     int32_t *append, int stride, int amax, cudaStream_t s)
{
    CK(launch_embed(*c, 1, nullptr, anchor_io, nullptr, batch, 1, s));
    CK(forward(*c, *kv, 0, batch, 1, kv->seq_lens, c->bt_rows, c->fin_verify, s));
    CK(lm_head(*c, c->fin_verify, batch, 1, 2, temperature, seed, step, nullptr, s));
    CK(launch_lm_finalize_impl(*c, 2, batch, 1, temperature, nullptr, nullptr, s));
    CK(launch_ar_commit(*c, *kv, batch, step, token_out, anchor_io, append, stride, amax, s));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_ar_step(orthrus_ctx_t *c, const orthrus_kv_t *kv, int32_t batch, float temperature,
                                 uint64_t seed, int64_t *step, int32_t *token_out, int32_t *anchor_io, void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, 1);
    if (st != ORTHRUS_OK) return st;
    if (!step || !anchor_io || temperature < 0.f) return ORTHRUS_ERR_INVALID_ARG;
    return ar_step_impl(c, kv, batch, temperature, seed, step, token_out, anchor_io, nullptr, 0, 0,
                        (cudaStream_t)stream);
}

orthrus_status_t orthrus_set_probe(orthrus_ctx_t *c, int32_t family, int32_t layer, int32_t view,
                                   void *const *starts, void *const *stops, int32_t n)
{
    if (!c || n < 0 || (n > 0 && (!starts || !stops))) return ORTHRUS_ERR_INVALID_ARG;
    if (n > 0 && (family < 0 || family > 1 || layer < 0 || layer >= c->cfg.n_layers || view < 0 || view > 1))
        return ORTHRUS_ERR_INVALID_ARG;
    if (family < 0 || family > 1) return ORTHRUS_ERR_INVALID_ARG;
    Ctx::Probe &p = c->probe[family];
    p.start.clear();
    p.stop.clear();
    p.hits = 0;
    for (int i = 0; i < n; ++i) {
        if (!starts[i] || !stops[i]) { p.start.clear(); p.stop.clear(); return ORTHRUS_ERR_INVALID_ARG; }
        p.start.push_back((cudaEvent_t)starts[i]);
        p.stop.push_back((cudaEvent_t)stops[i]);
    }
    p.layer = layer;
    p.view = view;
    return ORTHRUS_OK;
}

uint64_t orthrus_launch_count(const orthrus_ctx_t *c) { return c ? c->launches : 0; }

orthrus_status_t orthrus_check_error(orthrus_ctx_t *c, void *stream, uint32_t *bits)
{
    if (!c) return ORTHRUS_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned h = 0;
    CK(cudaMemcpyAsync(&h, c->err, 4, cudaMemcpyDeviceToHost, s));
    CK(cudaMemsetAsync(c->err, 0, 4, s));
    CK(cudaStreamSynchronize(s));
    if (bits) *bits = h;
    if (h & ORTHRUS_DEVERR_NONFINITE) return ORTHRUS_ERR_NONFINITE;
    if (h) return ORTHRUS_ERR_DEVICE_CHECK;
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_generate(orthrus_ctx_t *c, const orthrus_kv_t *kv, const int32_t *prompt, int32_t stride,
                                  const int32_t *lens, int32_t batch, int32_t K, int32_t max_new, float temperature,
                                  uint64_t seed, int32_t *out, orthrus_stats_t *stats, void *stream)
{
    if (!c || !prompt || !lens || !out || max_new < 1 || K < 0 || temperature < 0.f) return ORTHRUS_ERR_INVALID_ARG;
    orthrus_status_t st = check_step(c, kv, batch, K > 0 ? K : 1);
    if (st != ORTHRUS_OK) return st;
    const int Kb = K > 0 ? K : 1;
    for (int b = 0; b < batch; ++b) {
        if (lens[b] < 1) return ORTHRUS_ERR_INVALID_ARG;
        const long need = (long)lens[b] - 1 + max_new + Kb;
        if (need > c->cfg.max_seq || need > (long)kv->max_pages_per_seq * kv->page_size) return ORTHRUS_ERR_CAPACITY;
    }
    cudaStream_t s = (cudaStream_t)stream;
    st = orthrus_prefill(c, kv, prompt, stride, lens, batch, c->anchor_buf, stream);
    if (st != ORTHRUS_OK) return st;
    CK(cudaMemsetAsync(c->produced, 0, (size_t)batch * 4, s));
    CK(cudaMemsetAsync(c->step, 0, 8, s));
    std::vector<int32_t> prod(batch);
    orthrus_stats_t stt{};
    for (int cycle = 0; cycle < max_new; ++cycle) {
        if (K == 0) {
            st = ar_step_impl(c, kv, batch, temperature, seed, c->step, nullptr, c->anchor_buf, out, max_new, max_new, s);
            if (st != ORTHRUS_OK) return st;
            stt.forwards += 1;
        } else {
            st = orthrus_draft_block(c, kv, c->anchor_buf, batch, K, temperature, seed, c->step, c->draft, stream);
            if (st != ORTHRUS_OK) return st;
            st = orthrus_verify_block(c, kv, c->anchor_buf, c->draft, batch, K, temperature, stream);
            if (st != ORTHRUS_OK) return st;
            CK(launch_commit(*c, *kv, batch, K, temperature, seed, c->step, nullptr, c->n_buf, c->tok_buf,
                             c->anchor_buf, out, max_new, max_new, s));
            stt.forwards += 2;
        }
        stt.cycles += 1;
        CK(cudaMemcpyAsync(prod.data(), c->produced, (size_t)batch * 4, cudaMemcpyDeviceToHost, s));
        CK(cudaStreamSynchronize(s));
        const int mn = *std::min_element(prod.begin(), prod.end());
        if (mn >= max_new) break;
    }
    for (int b = 0; b < batch; ++b) stt.tokens += std::min(prod[b], max_new);
    stt.min_tokens = *std::min_element(prod.begin(), prod.end());
    if (stats) *stats = stt;
    return orthrus_check_error(c, stream, nullptr);
}

orthrus_status_t orthrus_dual_view_attention(orthrus_ctx_t *c, const orthrus_kv_t *kv, int32_t layer, int32_t mode,
                                             const void *q, const void *k_blk, const void *v_blk, int32_t batch,
                                             int32_t K, void *out, void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, K);
    if (st != ORTHRUS_OK) return st;
    if (!q || !out || (mode != 0 && mode != 1) || (mode == 1 && (!k_blk || !v_blk)) || layer < 0 ||
        layer >= c->cfg.n_layers)
        return ORTHRUS_ERR_INVALID_ARG;
    const orthrus_config_t &f = c->cfg;
    cudaStream_t s = (cudaStream_t)stream;
    AttnArgs at{};
    if (mode == 1) {   // user layout [B][K][n_kv][hd] -> the kernels' transient layouts
        const size_t half = (size_t)f.max_batch * c->kp * f.n_kv_heads * f.head_dim * c->esize;
        CK(launch_pack_block(*c, k_blk, v_blk, c->blk_pack, (char *)c->blk_pack + half, batch, K, c->kp, s));
        at.k_blk = c->blk_pack; at.v_blk = (char *)c->blk_pack + half;
    }
    at.kp = c->kp; at.bmax = f.max_batch; at.blk_layer = 0; at.blk_layers = 1;
    at.q = q; at.out = out; at.kv = kv_view(*kv); at.layer = layer;
    at.seq_lens = kv->seq_lens; at.bt_rows = c->bt_rows; at.B = batch; at.K = K; at.n_q = f.n_q_heads;
    at.n_kv = f.n_kv_heads; at.hd = f.head_dim; at.mode = mode; at.split_tokens = f.split_tokens;
    at.n_splits = c->n_splits; at.part = c->attn_part; at.ml = c->attn_ml; at.err = c->err;
    at.xo = c->attn_xo; at.xml = c->attn_xml; at.xcnt = c->attn_xcnt; at.xrows = c->Rw * f.n_q_heads;
    at.xz = c->attn_xz;
    CK(launch_attention(*c, at, s, batch * K, c->attn_simt_rows));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_block_mask_attention(orthrus_ctx_t *c, const orthrus_kv_t *kv, int32_t layer,
                                              const void *q, const void *k_blk, const void *v_blk,
                                              const int32_t *anchors, int32_t n_blocks, int32_t K, void *out,
                                              void *stream)
{
    if (!c || !kv || !q || !k_blk || !v_blk || !anchors || !out) return ORTHRUS_ERR_INVALID_ARG;
    const orthrus_config_t &f = c->cfg;
    if (n_blocks < 1 || K < 1 || K > f.max_block || layer < 0 || layer >= f.n_layers) return ORTHRUS_ERR_INVALID_ARG;
    {   // kv->seq_lens is not read here: the block lengths are the anchors
        orthrus_kv_t k2 = *kv;
        k2.seq_lens = const_cast<int32_t *>(anchors);
        if (!kv_ok(c, &k2)) return ORTHRUS_ERR_INVALID_ARG;
    }
    cudaStream_t s = (cudaStream_t)stream;
    // the diffusion view with one sequence per block: length = the block's
    // anchor, every block on block-table row 0 (the packed context); blocks
    // are independent, so they go max_batch at a time
    const size_t half = (size_t)f.max_batch * c->kp * f.n_kv_heads * f.head_dim * c->esize;
    const size_t qrow = (size_t)K * f.n_q_heads * f.head_dim * c->esize, kvrow = (size_t)K * f.n_kv_heads * f.head_dim * c->esize;
    for (int b0 = 0; b0 < n_blocks; b0 += f.max_batch) {
        const int nb = std::min(f.max_batch, n_blocks - b0);
        CK(launch_pack_block(*c, (const char *)k_blk + b0 * kvrow, (const char *)v_blk + b0 * kvrow, c->blk_pack,
                             (char *)c->blk_pack + half, nb, K, c->kp, s));
        AttnArgs at{};
        at.k_blk = c->blk_pack; at.v_blk = (char *)c->blk_pack + half;
        at.kp = c->kp; at.bmax = f.max_batch; at.blk_layer = 0; at.blk_layers = 1;
        at.q = (const char *)q + b0 * qrow; at.out = (char *)out + b0 * qrow; at.kv = kv_view(*kv); at.layer = layer;
        at.seq_lens = anchors + b0; at.bt_rows = c->bt_zero; at.B = nb; at.K = K; at.n_q = f.n_q_heads;
        at.n_kv = f.n_kv_heads; at.hd = f.head_dim; at.mode = 1; at.split_tokens = f.split_tokens;
        at.n_splits = c->n_splits; at.part = c->attn_part; at.ml = c->attn_ml; at.err = c->err;
        at.xo = c->attn_xo; at.xml = c->attn_xml; at.xcnt = c->attn_xcnt; at.xrows = c->Rw * f.n_q_heads;
        at.xz = c->attn_xz;
        CK(launch_attention(*c, at, s, nb * K, c->attn_simt_rows));
    }
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_kl_lm_head(orthrus_ctx_t *c, const void *h_ar, const void *h_diff, int32_t rows,
                                    float *kl, float *lse_ar, float *lse_diff, void *stream)
{
    if (!c || !h_ar || !h_diff || !kl || rows < 1) return ORTHRUS_ERR_INVALID_ARG;
    if (2 * (size_t)rows > (size_t)c->cfg.max_batch * c->cfg.max_block) return ORTHRUS_ERR_CAPACITY;
    CK(launch_kl_lm_head(*c, h_ar, h_diff, rows, kl, lse_ar, lse_diff, (cudaStream_t)stream));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_tree_topw(orthrus_ctx_t *c, const float *logits, int32_t rows, int32_t width,
                                   int32_t *ids, float *vals, float *lse, void *stream)
{
    if (!c || !logits || !ids || !vals || !lse || rows < 1 || width < 1 || width > 8 || width > c->cfg.vocab)
        return ORTHRUS_ERR_INVALID_ARG;
    if (rows > 65535) return ORTHRUS_ERR_CAPACITY;
    CK(launch_tree_topw(*c, logits, rows, width, ids, vals, lse, (cudaStream_t)stream));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_tree_build(orthrus_ctx_t *c, const int32_t *ids, const float *vals, const float *lse,
                                    int32_t batch, int32_t depth, int32_t width, int32_t nodes, int32_t *parent,
                                    int32_t *token, int32_t *node_depth, double *score, int32_t *n_rows,
                                    void *stream)
{
    if (!c || !parent || !token || !node_depth || !score || !n_rows || batch < 1 || depth < 0 || depth >= 128 ||
        width < 1 || width > 8 || nodes < 0 || nodes >= 128 || (depth > 0 && (!ids || !vals || !lse)))
        return ORTHRUS_ERR_INVALID_ARG;
    if (batch > c->cfg.max_batch) return ORTHRUS_ERR_CAPACITY;
    TreeBuildArgs a{};
    a.ids = ids; a.vals = vals; a.lse = lse; a.D = depth; a.W = width; a.N = nodes;
    a.parent = parent; a.token = token; a.depth = node_depth; a.score = score; a.n_rows = n_rows;
    CK(launch_tree_build(*c, a, batch, (cudaStream_t)stream));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_verify_tree(orthrus_ctx_t *c, const orthrus_kv_t *kv, const int32_t *anchor,
                                     const int32_t *parent, const int32_t *token, int32_t batch, int32_t rows,
                                     int32_t *g, void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, rows);
    if (st != ORTHRUS_OK) return st;
    if (!anchor || !parent || !token || !g) return ORTHRUS_ERR_INVALID_ARG;
    if (rows > 128) return ORTHRUS_ERR_CAPACITY;
    cudaStream_t s = (cudaStream_t)stream;
    CK(launch_tree_prep(*c, anchor, parent, token, batch, rows, s));
    CK(launch_embed(*c, 2, c->tree_tok, nullptr, nullptr, batch, rows, s));
    CK(forward(*c, *kv, 0, batch, rows, kv->seq_lens, c->bt_rows, c->fin_verify, s, c->tree_depth, c->tree_mask));
    CK(lm_head(*c, c->fin_verify, batch, rows, 0, 0.f, 0, nullptr, nullptr, s));
    CK(launch_lm_finalize_impl(*c, 0, batch, rows, 0.f, nullptr, nullptr, s));
    CK(cudaMemcpyAsync(g, c->g, (size_t)batch * rows * 4, cudaMemcpyDeviceToDevice, s));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_tree_commit(orthrus_ctx_t *c, const orthrus_kv_t *kv, int32_t batch, int32_t rows,
                                     const int32_t *parent, const int32_t *token, const int32_t *n_rows,
                                     const int32_t *g, int32_t *n_out, int32_t *emit, int32_t *anchor,
                                     void *stream)
{
    orthrus_status_t st = check_step(c, kv, batch, rows);
    if (st != ORTHRUS_OK) return st;
    if (!parent || !token || !n_rows || !g || !n_out || !emit || !anchor) return ORTHRUS_ERR_INVALID_ARG;
    if (rows > 128) return ORTHRUS_ERR_CAPACITY;
    const orthrus_config_t &f = c->cfg;
    TreeCommitArgs a{};
    a.kv = kv_view(*kv); a.seq_lens = kv->seq_lens;
    a.rows = rows; a.n_layers = f.n_layers; a.n_kv = f.n_kv_heads; a.hd = f.head_dim; a.vocab = f.vocab;
    a.parent = parent; a.token = token; a.g = g; a.n_rows = n_rows;
    a.n_out = n_out; a.emit = emit; a.anchor = anchor; a.err = c->err;
    CK(launch_tree_commit(*c, a, batch, (cudaStream_t)stream));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_debug_rows(orthrus_ctx_t *c, int32_t which, int32_t batch, int32_t K, int32_t *tok,
                                    float *logprob, float *lse, void *stream)
{
    if (!c || (which != 0 && which != 1) || batch < 1 || K < 1) return ORTHRUS_ERR_INVALID_ARG;
    if (batch * K > c->R) return ORTHRUS_ERR_CAPACITY;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t n = (size_t)batch * K * 4;
    if (tok) CK(cudaMemcpyAsync(tok, which ? c->draft : c->g, n, cudaMemcpyDeviceToDevice, s));
    if (logprob) CK(cudaMemcpyAsync(logprob, which ? c->logq : c->logp, n, cudaMemcpyDeviceToDevice, s));
    if (lse) CK(cudaMemcpyAsync(lse, which ? c->lse_q : c->lse_p, n, cudaMemcpyDeviceToDevice, s));
    return ORTHRUS_OK;
}

orthrus_status_t orthrus_debug_logits(orthrus_ctx_t *c, int32_t which, int32_t batch, int32_t K, float *logits,
                                      void *stream)
{
    if (!c || !logits || (which != 0 && which != 1) || batch < 1 || K < 1) return ORTHRUS_ERR_INVALID_ARG;
    if (batch * K > c->R) return ORTHRUS_ERR_CAPACITY;
    CK(launch_logits_dump(*c, which ? c->fin_draft : c->fin_verify, batch * K, logits, (cudaStream_t)stream));
    return ORTHRUS_OK;
}

}  // extern "C"
