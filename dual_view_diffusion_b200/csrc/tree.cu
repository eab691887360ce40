// Tree verification over one draft's marginals ("Orthrus" paper-notes page,
// §7.5: DDTree expands one diffusion forward's marginals best-first into a
// tree of the top prefixes and verifies it with tree attention in one pass;
// §9.6: the same proposed for Orthrus's K marginals).  Greedy only.
//
//   tree_topw_kernel     per row of fp32 logits: the W best ids (ties: lowest
//                        id) with their logits, and the row's log-sum-exp
//   tree_build_kernel    one warp per sequence: the root plus the N best
//                        prefixes of depth <= D, scores = sums of log q in
//                        fp64, ordered by score and then by rank sequence
//   tree_compact_kernel  the accepted root path's K/V, from cache slot
//                        t + row to slot t + depth, every layer and KV head
//   tree_finish_kernel   the accepted tokens, n, the next anchor, seq_len += n
#include <limits.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace orthrus {

constexpr int kTreeMaxW = 8;        // candidates per depth
constexpr int kTreeMaxRows = 128;   // rows of one tree (root + nodes)
constexpr int kTreeTopwThreads = 256;

__device__ __forceinline__ bool tw_better(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// One lane's sorted list (best first) gives up its head.
__device__ __forceinline__ void tw_pop(float (&v)[kTreeMaxW], int (&i)[kTreeMaxW])
{
#pragma unroll
    for (int j = 0; j + 1 < kTreeMaxW; ++j) { v[j] = v[j + 1]; i[j] = i[j + 1]; }
    v[kTreeMaxW - 1] = -INFINITY;
    i[kTreeMaxW - 1] = INT_MAX;
}

// The warp's kTreeMaxW best entries over all lanes' sorted lists, best
// first, into ov/oi (every lane gets the same result).  Ids are distinct
// across lanes, so the winner of a round is one lane.
__device__ __forceinline__ void tw_warp_merge(float (&v)[kTreeMaxW], int (&i)[kTreeMaxW], float *ov, int *oi)
{
#pragma unroll 1
    for (int r = 0; r < kTreeMaxW; ++r) {
        float bv = v[0];
        int bi = i[0];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov2 = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi2 = __shfl_xor_sync(0xffffffffu, bi, off);
            if (tw_better(ov2, oi2, bv, bi)) { bv = ov2; bi = oi2; }
        }
        if (i[0] == bi && bi != INT_MAX) tw_pop(v, i);
        ov[r] = bv;
        oi[r] = bi;
    }
}

// Grid rows, kTreeTopwThreads threads.  z [rows][V] fp32.
__global__ void __launch_bounds__(kTreeTopwThreads) tree_topw_kernel(const float *__restrict__ z, int V, int W,
                                                                     int32_t *ids, float *vals, float *lse,
                                                                     unsigned *err)
{
    pdl_trigger();
    pdl_wait();
    __shared__ float wv[kTreeTopwThreads / 32][kTreeMaxW];
    __shared__ int wi[kTreeTopwThreads / 32][kTreeMaxW];
    __shared__ float wm[kTreeTopwThreads / 32], ws[kTreeTopwThreads / 32];
    const int row = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float *zr = z + (size_t)row * V;
    float tv[kTreeMaxW];
    int ti[kTreeMaxW];
#pragma unroll
    for (int j = 0; j < kTreeMaxW; ++j) { tv[j] = -INFINITY; ti[j] = INT_MAX; }
    float m = -INFINITY, s = 0.f;   // running max and sum of exp(x - m)
    for (int v = threadIdx.x; v < V; v += kTreeTopwThreads) {
        const float x = zr[v];
        if (x > m) { s = s * expf(m - x) + 1.f; m = x; }
        else s += expf(x - m);
        if (tw_better(x, v, tv[kTreeMaxW - 1], ti[kTreeMaxW - 1])) {   // insert, keep the list sorted
            tv[kTreeMaxW - 1] = x;
            ti[kTreeMaxW - 1] = v;
#pragma unroll
            for (int j = kTreeMaxW - 1; j > 0; --j)
                if (tw_better(tv[j], ti[j], tv[j - 1], ti[j - 1])) {
                    const float a = tv[j]; tv[j] = tv[j - 1]; tv[j - 1] = a;
                    const int b = ti[j]; ti[j] = ti[j - 1]; ti[j - 1] = b;
                }
        }
    }
    // log-sum-exp: (m, s) pairs merged across the warp, then across warps
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, off), s2 = __shfl_xor_sync(0xffffffffu, s, off);
        const float M = fmaxf(m, m2);
        s = (M == -INFINITY) ? 0.f : s * expf(m - M) + s2 * expf(m2 - M);
        m = M;
    }
    float mv[kTreeMaxW];
    int mi[kTreeMaxW];
    tw_warp_merge(tv, ti, mv, mi);
    if (lane == 0) {
        wm[warp] = m;
        ws[warp] = s;
#pragma unroll
        for (int j = 0; j < kTreeMaxW; ++j) { wv[warp][j] = mv[j]; wi[warp][j] = mi[j]; }
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int nw = kTreeTopwThreads / 32;
#pragma unroll
        for (int j = 0; j < kTreeMaxW; ++j) {
            tv[j] = lane < nw ? wv[lane][j] : -INFINITY;
            ti[j] = lane < nw ? wi[lane][j] : INT_MAX;
        }
        tw_warp_merge(tv, ti, mv, mi);
        if (lane == 0) {
            float M = -INFINITY, S = 0.f;
            for (int w = 0; w < nw; ++w) M = fmaxf(M, wm[w]);
            for (int w = 0; w < nw; ++w) S += ws[w] * expf(wm[w] - M);
            const float l = M + logf(S);
            if (!isfinite(l)) raise_err(err, ORTHRUS_DEVERR_NONFINITE);
            lse[row] = l;
            for (int j = 0; j < W; ++j) {
                ids[(size_t)row * W + j] = mi[j];
                vals[(size_t)row * W + j] = mv[j];
            }
        }
    }
}

// ------------------------------------------------------------------ builder

// Shared memory of one sequence's build (N + 1 nodes, 2N + 2 pool entries).
__host__ __device__ inline size_t tree_build_smem(int N, int D)
{
    const size_t nodes = (size_t)N + 1, pool = 2 * (size_t)N + 2;
    return nodes * 8 + pool * 8 + nodes * 4 * 3 + pool * 4 * 2 + nodes * (size_t)(D > 0 ? D : 1);
}

// Candidate a before candidate b: larger score, then the smaller rank
// sequence (parent's ranks, then the candidate's own rank; a prefix before
// its extensions).
__device__ __forceinline__ bool tb_before(int a, int b, const double *ps, const int32_t *pp, const int32_t *pr,
                                          const int32_t *dep, const unsigned char *rseq, int D)
{
    if (ps[a] != ps[b]) return ps[a] > ps[b];
    const int la = dep[pp[a]] + 1, lb = dep[pp[b]] + 1;
    for (int k = 0; k < la && k < lb; ++k) {
        const int x = k < la - 1 ? rseq[(size_t)pp[a] * D + k] : pr[a];
        const int y = k < lb - 1 ? rseq[(size_t)pp[b] * D + k] : pr[b];
        if (x != y) return x < y;
    }
    return la < lb;
}

// Grid B, one warp: lanes scan the pool, lane 0 updates it.
__global__ void __launch_bounds__(32) tree_build_kernel(TreeBuildArgs a)
{
    pdl_trigger();
    pdl_wait();
    extern __shared__ __align__(16) unsigned char tb_raw[];
    const int b = blockIdx.x, lane = threadIdx.x, D = a.D, W = a.W, N = a.N;
    const size_t nodes = (size_t)N + 1, pool = 2 * (size_t)N + 2;
    double *sc = (double *)tb_raw;                       // node scores
    double *ps = sc + nodes;                             // pool scores
    int32_t *par = (int32_t *)(ps + pool), *tok = par + nodes, *dep = tok + nodes;
    int32_t *pp = dep + nodes, *pr = pp + pool;          // pool: parent node, rank
    unsigned char *rseq = (unsigned char *)(pr + pool);  // node rank sequences [nodes][D]
    const int32_t *ids = a.ids + (size_t)b * D * W;
    const float *vals = a.vals + (size_t)b * D * W, *lse = a.lse + (size_t)b * D;
    auto lp = [&](int d, int r) { return (double)vals[d * W + r] - (double)lse[d]; };   // log q, depth d + 1
    __shared__ int np_s;
    if (lane == 0) {
        par[0] = -1; tok[0] = -1; dep[0] = 0; sc[0] = 0.0;
        np_s = 0;
        if (D > 0 && N > 0) { pp[0] = 0; pr[0] = 0; ps[0] = lp(0, 0); np_s = 1; }
    }
    __syncwarp();
    int n = 1;
    while (n <= N) {
        const int np = np_s;
        if (np == 0) break;
        int best = -1;
        for (int i = lane; i < np; i += 32)
            if (best < 0 || tb_before(i, best, ps, pp, pr, dep, rseq, D)) best = i;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const int o = __shfl_xor_sync(0xffffffffu, best, off);
            if (o >= 0 && (best < 0 || tb_before(o, best, ps, pp, pr, dep, rseq, D))) best = o;
        }
        if (lane == 0) {
            const int p = pp[best], rk = pr[best];
            const double s = ps[best];
            pp[best] = pp[np - 1]; pr[best] = pr[np - 1]; ps[best] = ps[np - 1];
            int cnt = np - 1;
            const int d = dep[p] + 1;
            par[n] = p; dep[n] = d; sc[n] = s; tok[n] = ids[(d - 1) * W + rk];
            for (int k = 0; k < d - 1; ++k) rseq[(size_t)n * D + k] = rseq[(size_t)p * D + k];
            rseq[(size_t)n * D + d - 1] = (unsigned char)rk;
            if (rk + 1 < W) { pp[cnt] = p; pr[cnt] = rk + 1; ps[cnt] = sc[p] + lp(d - 1, rk + 1); ++cnt; }
            if (d < D) { pp[cnt] = n; pr[cnt] = 0; ps[cnt] = s + lp(d, 0); ++cnt; }
            np_s = cnt;
        }
        __syncwarp();
        ++n;
    }
    const size_t o = (size_t)b * nodes;
    for (int r = lane; r < (int)nodes; r += 32) {
        const bool in = r < n;
        a.parent[o + r] = in ? par[r] : -1;
        a.token[o + r] = in ? tok[r] : -1;
        a.depth[o + r] = in ? dep[r] : -1;
        a.score[o + r] = in ? sc[r] : -INFINITY;
    }
    if (lane == 0) a.n_rows[b] = n;
}

// ------------------------------------------------------------------- commit

// The greedy walk (shared by both kernels): from the root follow the lowest
// row whose parent is the current row and whose token is the current row's
// argmax g; path[0..m] = rows visited.  Returns m; a malformed parent entry
// raises ORTHRUS_DEVERR_TOKEN and ends the walk there.
__device__ int tree_walk(const TreeCommitArgs &a, int b, int32_t *path)
{
    const int R = min(max(a.n_rows[b], 1), a.rows);
    const int32_t *par = a.parent + (size_t)b * a.rows, *tok = a.token + (size_t)b * a.rows;
    const int32_t *g = a.g + (size_t)b * a.rows;
    int cur = 0, m = 0;
    path[0] = 0;
    for (;;) {
        int next = -1;
        for (int c = cur + 1; c < R && next < 0; ++c) {
            const int p = par[c];
            if (p < 0 || p >= c) { raise_err(a.err, ORTHRUS_DEVERR_TOKEN); return m; }
            if (p == cur && tok[c] == g[cur]) next = c;
        }
        if (next < 0) return m;
        path[++m] = next;
        cur = next;
    }
}

// Grid (n_layers * n_kv, B), 128 threads.  Rows move in chunks of 32 path
// entries: a chunk's sources are all read before any of its destinations is
// written, and a destination t + i can only be the source of an earlier
// path entry (path[j] = i needs j < i), so ascending chunks are safe.
template <class T>
__global__ void __launch_bounds__(128) tree_compact_kernel(TreeCommitArgs a)
{
    __shared__ int32_t path[kTreeMaxRows];
    __shared__ int m_s, t_s;
    __shared__ T kbuf[32][128], vbuf[32][128];
    pdl_wait();   // no early trigger: tree_finish_kernel writes seq_lens, read here
    const int b = blockIdx.y, layer = blockIdx.x / a.n_kv, kvh = blockIdx.x % a.n_kv, hd = a.hd;
    if (threadIdx.x == 0) { m_s = tree_walk(a, b, path); t_s = a.seq_lens[b]; }
    __syncthreads();
    const int m = m_s, t = t_s;
    const T *kp = (const T *)a.kv.k_pages;
    const T *vp = (const T *)a.kv.v_pages;
    auto head_of = [&](int pos, int *slot) -> long long {   // -1: beyond the sequence's pages
        const int pidx = pos / a.kv.page_size;
        if (pos < 0 || pidx >= a.kv.max_pages) return -1;
        const int page = a.kv.block_table[(size_t)b * a.kv.max_pages + pidx];
        if (page < 0 || page >= a.kv.num_pages) return -1;
        *slot = pos % a.kv.page_size;
        return ((long long)layer * a.kv.num_pages + page) * a.n_kv + kvh;
    };
    for (int i0 = 1; i0 <= m; i0 += 32) {
        const int cnt = min(32, m - i0 + 1);
        for (int e = threadIdx.x; e < cnt * hd; e += blockDim.x) {
            const int i = e / hd, d = e % hd;
            int slot = 0;
            const long long hh = head_of(t + path[i0 + i], &slot);
            if (hh < 0) { raise_err(a.err, ORTHRUS_DEVERR_CAPACITY); continue; }
            kbuf[i][d] = kp[(hh * a.kv.page_size + slot) * hd + d];
            vbuf[i][d] = vp[(hh * hd + d) * a.kv.page_size + slot];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < cnt * hd; e += blockDim.x) {
            const int i = e / hd, d = e % hd;
            int slot = 0, slot_src = 0;
            const long long hh = head_of(t + i0 + i, &slot);
            if (hh < 0 || head_of(t + path[i0 + i], &slot_src) < 0) continue;
            ((T *)a.kv.k_pages)[(hh * a.kv.page_size + slot) * hd + d] = kbuf[i][d];
            ((T *)a.kv.v_pages)[(hh * hd + d) * a.kv.page_size + slot] = vbuf[i][d];
        }
        __syncthreads();
    }
}

// Grid 1, B threads (B <= max_batch): emitted tokens, n, anchor, seq_len.
__global__ void tree_finish_kernel(TreeCommitArgs a, int B)
{
    pdl_wait();
    const int b = threadIdx.x;
    if (b >= B) return;
    int32_t path[kTreeMaxRows];
    const int m = tree_walk(a, b, path);
    const int32_t *tok = a.token + (size_t)b * a.rows, *g = a.g + (size_t)b * a.rows;
    for (int i = 1; i <= m; ++i) a.emit[(size_t)b * a.rows + i - 1] = tok[path[i]];
    int last = g[path[m]];
    if (last < 0 || last >= a.vocab) { raise_err(a.err, ORTHRUS_DEVERR_TOKEN); last = 0; }
    a.emit[(size_t)b * a.rows + m] = last;
    a.n_out[b] = m + 1;
    a.anchor[b] = last;
    a.seq_lens[b] += m + 1;
}

cudaError_t launch_tree_topw(const Ctx &c, const float *logits, int rows, int W, int32_t *ids, float *vals,
                             float *lse, cudaStream_t s)
{
    c.launches += 1;
    return launch_k(tree_topw_kernel, rows, kTreeTopwThreads, 0, s, logits, c.cfg.vocab, W, ids, vals, lse, c.err);
}

cudaError_t launch_tree_build(const Ctx &c, const TreeBuildArgs &a, int B, cudaStream_t s)
{
    const size_t smem = tree_build_smem(a.N, a.D);
    if (smem > 48 * 1024) return cudaErrorInvalidValue;
    c.launches += 1;
    return launch_k(tree_build_kernel, B, 32, smem, s, a);
}

cudaError_t launch_tree_commit(const Ctx &c, const TreeCommitArgs &a, int B, cudaStream_t s)
{
    if (a.hd > 128 || a.rows > kTreeMaxRows || B > 1024) return cudaErrorInvalidValue;
    c.launches += 2;
    const dim3 grid(a.n_layers * a.n_kv, B);
    cudaError_t e = c.cfg.dtype == ORTHRUS_BF16 ? launch_k(tree_compact_kernel<bf16>, grid, 128, 0, s, a)
                                                : launch_k(tree_compact_kernel<float>, grid, 128, 0, s, a);
    if (e != cudaSuccess) return e;
    return launch_k(tree_finish_kernel, 1, B, 0, s, a, B);
}

}  // namespace orthrus
