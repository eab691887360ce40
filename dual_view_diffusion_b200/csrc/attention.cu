// Dual-view attention over the one shared paged KV cache.
//
// Block of K query rows per sequence at positions t .. t+K-1; GQA groups of
// g = n_q / n_kv query heads share a KV head, so one CTA serves all K*g rows
// of a (sequence, KV head) pair and every K/V tile it stages is reused by
// all of them (paper notes §2.2-2.3: both views read the same AR cache).
//
//   mode 0 (AR verify, paper notes §4.1 step 2): row k sees cache rows
//          [0, t+k]; the block's own K/V were written into the cache tail;
//   mode 1 (diffusion draft, paper notes §3.2): row k sees cache rows
//          [0, t) and all K rows of the transient diffusion K/V.
//
// Split-KV flash decoding: split s covers absolute key positions
// [s*S, (s+1)*S) for a run-constant S, so a row meets the same splits and
// the same key tiles whatever block it belongs to; keys outside a row's
// window contribute exact zeros.  Each split writes an unnormalised partial
// (O, running max in log2 units, running sum); a second kernel combines the
// splits in order.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace orthrus {

constexpr int kAttnRowsSimt = 32;   // rows per CTA, SIMT kernel
constexpr float kLog2e = 1.4426950408889634f;

struct KeySrc {
    const void *k;       // key row (element type erased), null = zero fill
    const void *v;       // element d of the value lives at v + d * v_stride
    size_t v_stride;
};

// Source of key position p for (b, kvh).  Cache pages hold K as
// [slot][dim] and V transposed as [dim][slot]; the diffusion block's
// transient K/V (mode 1, keys t .. t+K-1) follow the same two layouts.
template <class T>
__device__ __forceinline__ KeySrc key_src(const AttnArgs &a, int b, int kvh, int t, int p, int key_end, bool block)
{
    KeySrc r{nullptr, nullptr, 0};
    if (p >= key_end) return r;
    if (block) {
        const size_t head = ((size_t)a.blk_layer * a.bmax + b) * a.n_kv + kvh;
        r.k = (const T *)a.k_blk + (head * a.kp + (p - t)) * a.hd;
        r.v = (const T *)a.v_blk + head * a.hd * a.kp + (p - t);
        r.v_stride = a.kp;
        return r;
    }
    const int pidx = p / a.kv.page_size;
    if (pidx >= a.kv.max_pages) { raise_err(a.err, ORTHRUS_DEVERR_CAPACITY); return r; }
    const int page = a.kv.block_table[(size_t)a.bt_rows[b] * a.kv.max_pages + pidx];
    if (page < 0 || page >= a.kv.num_pages) { raise_err(a.err, ORTHRUS_DEVERR_CAPACITY); return r; }
    const size_t head = ((size_t)a.layer * a.kv.num_pages + page) * a.n_kv + kvh;
    const int slot = p % a.kv.page_size;
    r.k = (const T *)a.kv.k_pages + (head * a.kv.page_size + slot) * a.hd;
    r.v = (const T *)a.kv.v_pages + head * a.hd * a.kv.page_size + slot;
    r.v_stride = a.kv.page_size;
    return r;
}

// ---------------------------------------------------------------- SIMT
// Any head_dim <= 128, any dtype: 4 warps, a warp walks its rows one by one;
// per-row running state lives in shared memory between key tiles.
template <class T>
__global__ void __launch_bounds__(128) attn_split_simt(AttnArgs a, int n_split_grid)
{
    extern __shared__ __align__(16) float fsm[];
    const int hd = a.hd, hp = hd + 1;
    float *qs = fsm;                                    // [32][hd]
    float *os = qs + kAttnRowsSimt * hd;                // [32][hd]
    float *ks = os + kAttnRowsSimt * hd;                // [64][hp]
    float *vs = ks + kKeyTile * hp;                     // [64][hp]
    float *ms = vs + kKeyTile * hp;                     // [32]
    float *ls = ms + kAttnRowsSimt;                     // [32]
    pdl_trigger();
    pdl_wait();
    // grid (kv head, sequence x row group, split): the split index varies
    // slowest, so the CTAs of splits a short sequence never reaches (they
    // exit at once) come after every working CTA; in the diffusion view the
    // last split index is the block's own keys
    const int kvh = blockIdx.x, s = blockIdx.z;
    const int rgroups = gridDim.y / a.B, b = blockIdx.y / rgroups, rg = blockIdx.y % rgroups;
    const int g = a.n_q / a.n_kv, R = a.K * g, r0 = rg * kAttnRowsSimt;
    if (r0 >= R) return;
    const int t = a.seq_lens[b];
    const bool block = a.mode == 1 && s == n_split_grid;
    int key0, key1, slot;
    if (block) {
        key0 = t; key1 = t + a.K; slot = a.n_splits - 1;
    } else {
        key0 = s * a.split_tokens;
        key1 = min(key0 + a.split_tokens, a.mode == 0 ? t + a.K : t);
        slot = s;
        if (key0 >= key1) return;
    }
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float scale = kLog2e / sqrtf((float)hd);
    const int nr = min(kAttnRowsSimt, R - r0);

    for (int idx = tid; idx < nr * hd; idx += 128) {
        const int r = idx / hd, d = idx % hd, rr = r0 + r, k = rr / g, j = rr % g;
        qs[idx] = to_f<T>(((const T *)a.q)[((size_t)(b * a.K + k) * a.n_q + kvh * g + j) * hd + d]);
        os[idx] = 0.f;
    }
    for (int r = tid; r < nr; r += 128) { ms[r] = -INFINITY; ls[r] = 0.f; }

    for (int p0 = key0; p0 < key1; p0 += kKeyTile) {
        __syncthreads();
        for (int idx = tid; idx < kKeyTile * hd; idx += 128) {
            const int row = idx / hd, d = idx % hd;
            const KeySrc src = key_src<T>(a, b, kvh, t, p0 + row, key1, block);
            ks[row * hp + d] = src.k ? to_f<T>(((const T *)src.k)[d]) : 0.f;
            vs[row * hp + d] = src.v ? to_f<T>(((const T *)src.v)[(size_t)d * src.v_stride]) : 0.f;
        }
        __syncthreads();
        for (int r = warp; r < nr; r += 4) {
            const int k = (r0 + r) / g;
            const bool tree = a.mode == 0 && a.tree_mask != nullptr;
            const int lim = (a.mode == 0 && !block && !tree) ? t + k + 1 : key1;
            float sv[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h, p = p0 + j;
                float acc = 0.f;
                for (int d = 0; d < hd; ++d) acc = fmaf(qs[r * hd + d], ks[j * hp + d], acc);
                bool see = p < lim && p < key1;
                if (tree && see && p >= t) {   // a block key: the row's ancestors and itself only
                    const int jb = p - t;
                    see = jb < 128 && ((a.tree_mask[(size_t)(b * a.K + k) * 4 + (jb >> 5)] >> (jb & 31)) & 1u);
                }
                sv[h] = see ? acc * scale : -INFINITY;
            }
            float tmax = fmaxf(sv[0], sv[1]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
            const float mo = ms[r], mn = fmaxf(mo, tmax), mu = mn == -INFINITY ? 0.f : mn;
            const float alpha = exp2f(mo - mu);
            float pv[2] = {exp2f(sv[0] - mu), exp2f(sv[1] - mu)};
            const float rs = warp_sum(pv[0] + pv[1]);
            for (int d0 = 0; d0 < hd; d0 += 32) {   // every lane joins the shuffles
                const int d = d0 + lane;
                float acc = d < hd ? os[r * hd + d] * alpha : 0.f;
                for (int j = 0; j < kKeyTile; ++j) {
                    const float pj = __shfl_sync(0xffffffffu, pv[j >> 5], j & 31);
                    if (d < hd) acc = fmaf(pj, vs[j * hp + d], acc);
                }
                if (d < hd) os[r * hd + d] = acc;
            }
            __syncwarp();
            if (lane == 0) { ms[r] = mn; ls[r] = ls[r] * alpha + rs; }
            __syncwarp();
        }
    }
    __syncthreads();
    for (int idx = tid; idx < nr * hd; idx += 128) {
        const int r = idx / hd, d = idx % hd, rr = r0 + r, k = rr / g, j = rr % g;
        const size_t rowhead = (size_t)(b * a.K + k) * a.n_q + kvh * g + j;
        a.part[(rowhead * a.n_splits + slot) * hd + d] = os[idx];
        if (d == 0) a.ml[rowhead * a.n_splits + slot] = make_float2(ms[r], ls[r]);
    }
}

// ---------------------------------------------------------------- combine
// One warp per (block row, query head): weights 2^(m_s - M) over the splits
// the sequence used, summed in split order.  Lane s holds split s's (m, l)
// (32 splits per round); each lane accumulates 4 output dims, loading the
// partial rows of 8 splits before using any of them.
template <class T>
__global__ void __launch_bounds__(256) attn_combine(AttnArgs a)
{
    pdl_trigger();
    pdl_wait();
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    const int rows = a.B * a.K * a.n_q;
    if (w >= rows) return;
    const int row = w / a.n_q, b = row / a.K;
    // cache splits the sequence reached, then (diffusion view) the block slot
    const int cache_end = a.seq_lens[b] + (a.mode == 0 ? a.K : 0);
    int n_cache = (cache_end + a.split_tokens - 1) / a.split_tokens;
    if (n_cache > a.n_splits - 1) {   // longer than the context was sized for
        if (lane == 0) raise_err(a.err, ORTHRUS_DEVERR_CAPACITY);
        n_cache = a.n_splits - 1;
    }
    const int n_used = n_cache + (a.mode == 1 ? 1 : 0);
    // slot of the i-th used split
#define SLOT(i) ((a.mode == 1 && (i) == n_cache) ? a.n_splits - 1 : (i))
    const float2 *ml = a.ml + (size_t)w * a.n_splits;
    float M = -INFINITY;
    for (int s = lane; s < n_used; s += 32) M = fmaxf(M, ml[SLOT(s)].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int s = lane; s < n_used; s += 32) L += ml[SLOT(s)].y * exp2f(ml[SLOT(s)].x - M);
    L = warp_sum(L);
    const float inv = 1.0f / L;
    const float *part = a.part + (size_t)w * a.n_splits * a.hd;
    const int c0 = lane * 4;
    const bool mine = c0 < a.hd;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n_used; s0 += 32) {
        const int sl = s0 + lane;
        const float wl = sl < n_used ? exp2f(ml[SLOT(sl)].x - M) : 0.f;
        const int cnt = min(32, n_used - s0);
        for (int j0 = 0; j0 < cnt; j0 += 8) {
            float4 v[8];
            float wt[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                wt[j] = __shfl_sync(0xffffffffu, wl, (j0 + j) & 31);
                const bool ok = mine && j0 + j < cnt;
                v[j] = ok ? *(const float4 *)(part + (size_t)SLOT(s0 + j0 + j) * a.hd + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j0 + j < cnt) {
                    acc.x = fmaf(wt[j], v[j].x, acc.x); acc.y = fmaf(wt[j], v[j].y, acc.y);
                    acc.z = fmaf(wt[j], v[j].z, acc.z); acc.w = fmaf(wt[j], v[j].w, acc.w);
                }
            }
        }
    }
#undef SLOT
    if (mine) {
        T *o = (T *)a.out + (size_t)w * a.hd + c0;
        o[0] = from_f<T>(acc.x * inv); o[1] = from_f<T>(acc.y * inv);
        o[2] = from_f<T>(acc.z * inv); o[3] = from_f<T>(acc.w * inv);
    }
}

// ---------------------------------------------------------------- host
static size_t simt_smem(int hd)
{
    return sizeof(float) * (2 * kAttnRowsSimt * hd + 2 * kKeyTile * (hd + 1) + 2 * kAttnRowsSimt);
}

cudaError_t attention_init_attributes()
{
    cudaError_t e = attn_tc_init_attributes();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_split_simt<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)simt_smem(128));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(attn_split_simt<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)simt_smem(128));
}

bool attn_tc_shape_ok(int dtype, int hd, int n_q, int n_kv, int page_size)
{
    if (dtype != ORTHRUS_BF16 || hd != 128 || n_kv < 1 || n_q % n_kv) return false;
    const int g = n_q / n_kv;
    return g >= 1 && 128 % g == 0 && page_size % 64 == 0;
}

cudaError_t launch_attention_simt(const Ctx &c, const AttnArgs &a, cudaStream_t s)
{
    const int n_split_grid = (c.cfg.max_seq + a.split_tokens - 1) / a.split_tokens;
    const int g = a.n_q / a.n_kv, R = a.K * g;
    const int rgroups = (R + kAttnRowsSimt - 1) / kAttnRowsSimt;
    dim3 grid(a.n_kv, a.B * rgroups, n_split_grid + (a.mode == 1 ? 1 : 0));
    cudaError_t e;
    if (c.cfg.dtype == ORTHRUS_BF16)
        e = launch_k(attn_split_simt<bf16>, grid, 128, simt_smem(a.hd), s, a, n_split_grid);
    else
        e = launch_k(attn_split_simt<float>, grid, 128, simt_smem(a.hd), s, a, n_split_grid);
    c.launches += 1;
    if (e != cudaSuccess) return e;
    c.launches += 1;
    const int rows = a.B * a.K * a.n_q;
    if (c.cfg.dtype == ORTHRUS_BF16) return launch_k(attn_combine<bf16>, (rows + 7) / 8, 256, 0, s, a);
    return launch_k(attn_combine<float>, (rows + 7) / 8, 256, 0, s, a);
}

// q_rows: token rows the q buffer holds (its tensor map's extent).
cudaError_t launch_attention(const Ctx &c, const AttnArgs &a, cudaStream_t s, int q_rows, int simt_rows)
{
    const int n_split_grid = (c.cfg.max_seq + a.split_tokens - 1) / a.split_tokens;
    // tensor-core path: one launch, the cluster combines and writes the output
    if (attn_tc_shape_ok(c.cfg.dtype, a.hd, a.n_q, a.n_kv, a.kv.page_size)) {
        const cudaError_t e = launch_attn_tc_cached(c, a, n_split_grid, q_rows, s);
        if (e != cudaErrorNotSupported) return e;
    }
    // the SIMT kernel writes [B*K][n_q][n_splits] partials: only into room
    // the caller reserved for them
    if (a.B * a.K > simt_rows || !a.part || !a.ml || a.n_splits < n_split_grid + 1) return cudaErrorNotSupported;
    return launch_attention_simt(c, a, s);
}

}  // namespace orthrus
