// Tree verification over one draft's marginals ("Orthrus" paper-notes page,
// §7.5: DDTree expands one diffusion forward's marginals best-first into a
// tree of the top prefixes and verifies it with tree attention in one pass;
// §9.6: the same proposed for Orthrus's K marginals).  Greedy only.
//
//   tree_topw_kernel     per row of fp32 logits (one 8-CTA cluster): the W
//                        best ids (ties: lowest id) with their logits, and
//                        the row's log-sum-exp
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

constexpr int kTreeMaxW = kTopWMax;   // candidates per depth
constexpr int kTreeMaxRows = 128;   // rows of one tree (root + nodes)
constexpr int kTreeTopwThreads = 256;
constexpr int kTreeTopwSplit = 8;     // CTAs (one cluster) per logits row

// Up to four logits (x[0 .. n-1]) into a thread's running (max, sum of
// exp(x - max)): one rescale per group, the exponentials independent.
__device__ __forceinline__ void tw_lse4(const float (&x)[4], int n, float &m, float &s)
{
    float mc = x[0];
#pragma unroll
    for (int e = 1; e < 4; ++e)
        if (e < n) mc = fmaxf(mc, x[e]);
    if (mc > m) { s *= expf(m - mc); m = mc; }
    if (m == -INFINITY) return;   // every logit so far is -inf (a masked id): nothing to add
    float add = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e)
        if (e < n) add += expf(x[e] - m);
    s += add;
}

// The warp keeps one sorted list (every lane holds the same copy): the
// lanes' candidates (n values each, ids ascending within a lane) enter one
// at a time in (lane, element) order, each insertion the same on every lane,
// and a candidate is dropped as soon as the list's last entry passes it.  A
// warp meets about W ln(N / W) insertions over N logits, so almost every
// step is one compare per value and a ballot.  Every lane must call it.
__device__ __forceinline__ void tw_warp_insert(const float *x, const int *id, int n, float (&tv)[kTopWMax],
                                               int (&ti)[kTopWMax])
{
    const int lane = threadIdx.x & 31;
    if (ti[kTopWMax - 1] == INT_MAX) {
        // the list is not full yet (the first steps, warp-uniform): every
        // lane's candidates and one entry of the list each go into a private
        // list, and the warp merges them all at once
        float pv[kTopWMax];
        int pi[kTopWMax];
#pragma unroll
        for (int j = 0; j < kTopWMax; ++j) { pv[j] = -INFINITY; pi[j] = INT_MAX; }
        float cv = -INFINITY;
        int cid = INT_MAX;
#pragma unroll
        for (int j = 0; j < kTopWMax; ++j)
            if (j == lane) { cv = tv[j]; cid = ti[j]; }
        if (cid != INT_MAX) tw_insert(cv, cid, pv, pi);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k < n) tw_insert(x[k], id[k], pv, pi);
#pragma unroll
        for (int r = 0; r < kTopWMax; ++r) {   // round r: the warp's best remaining head
            float bv = pv[0];
            int bi = pi[0];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                if (tw_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
            }
            if (pi[0] == bi && bi != INT_MAX) tw_pop(pv, pi);
            tv[r] = bv;
            ti[r] = bi;
        }
        return;
    }
    uint32_t cm = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (k < n && tw_better(x[k], id[k], tv[kTopWMax - 1], ti[kTopWMax - 1])) cm |= 1u << k;
    for (;;) {
        const uint32_t any = __ballot_sync(0xffffffffu, cm != 0);
        if (!any) break;
        const int src = __ffs(any) - 1;
        const int e = __ffs(__shfl_sync(0xffffffffu, cm, src)) - 1;
        float xv = x[0];
        int xi = id[0];
#pragma unroll
        for (int k = 1; k < 4; ++k)
            if (k < n && k == e) { xv = x[k]; xi = id[k]; }
        xv = __shfl_sync(0xffffffffu, xv, src);
        xi = __shfl_sync(0xffffffffu, xi, src);
        tw_insert(xv, xi, tv, ti);
        if (lane == src) cm &= ~(1u << e);
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (((cm >> k) & 1u) && !tw_better(x[k], id[k], tv[kTopWMax - 1], ti[kTopWMax - 1])) cm &= ~(1u << k);
    }
}

__device__ __forceinline__ uint32_t tw_smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint32_t tw_mapa(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ float tw_ld_peer_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ int tw_ld_peer_s32(uint32_t addr)
{
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];\n" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void tw_cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Grid (kTreeTopwSplit, rows), clusters of kTreeTopwSplit CTAs along x: CTA
// s of a row's cluster takes ids [s * chunk, (s + 1) * chunk) (chunk a
// multiple of 4), each thread a sorted top list and a running (max, sum),
// merged across the CTA's warps; then CTA 0 pulls every CTA's list and
// (max, sum) from distributed shared memory and merges them.  VEC (V a
// multiple of 4, z 16-byte aligned): 16-byte loads, four in flight.
template <bool VEC>
__global__ void __launch_bounds__(kTreeTopwThreads) tree_topw_kernel(const float *__restrict__ z, int V, int W,
                                                                     int chunk, int32_t *ids, float *vals,
                                                                     float *lse, unsigned *err)
{
    pdl_trigger();
    pdl_wait();
    constexpr int nw = kTreeTopwThreads / 32;
    __shared__ float wv[nw][kTreeMaxW];
    __shared__ int wi[nw][kTreeMaxW];
    __shared__ float wm[nw], ws[nw];
    __shared__ float cv[kTreeMaxW];   // this CTA's result, read by CTA 0 of the cluster
    __shared__ int ci[kTreeMaxW];
    __shared__ float cms[2];
    const int split = blockIdx.x, row = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lo = split * chunk, hi = min(V, lo + chunk);
    const float *zr = z + (size_t)row * V;
    float tv[kTreeMaxW];
    int ti[kTreeMaxW];
#pragma unroll
    for (int j = 0; j < kTreeMaxW; ++j) { tv[j] = -INFINITY; ti[j] = INT_MAX; }
    float m = -INFINITY, s = 0.f;   // running max and sum of exp(x - m)
    // lanes walk the range in warp-uniform steps (the list is shared by the
    // warp); lanes past the end offer nothing
    if (VEC) {
        constexpr int U = 4;
        const int q0 = lo / 4, q1 = (hi + 3) / 4;   // hi is V or a multiple of 4; V % 4 == 0 here
        const float4 *z4 = (const float4 *)zr;
        for (int b0 = q0 + (threadIdx.x & ~31); b0 < q1; b0 += kTreeTopwThreads * U) {
            float4 x4[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = b0 + lane + u * kTreeTopwThreads;
                x4[u] = i < q1 ? z4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = b0 + lane + u * kTreeTopwThreads;
                const bool in = i < q1;
                const float x[4] = {in ? x4[u].x : -INFINITY, in ? x4[u].y : -INFINITY,
                                    in ? x4[u].z : -INFINITY, in ? x4[u].w : -INFINITY};
                const int id[4] = {in ? 4 * i : INT_MAX, in ? 4 * i + 1 : INT_MAX, in ? 4 * i + 2 : INT_MAX,
                                   in ? 4 * i + 3 : INT_MAX};
                if (in) tw_lse4(x, 4, m, s);
                tw_warp_insert(x, id, 4, tv, ti);
            }
        }
    } else {
        for (int b = lo + (threadIdx.x & ~31); b < hi; b += kTreeTopwThreads) {
            const int v = b + lane;
            const bool in = v < hi;
            const float x[4] = {in ? zr[v] : -INFINITY, 0.f, 0.f, 0.f};
            const int id[4] = {in ? v : INT_MAX, 0, 0, 0};
            if (in) tw_lse4(x, 1, m, s);
            tw_warp_insert(x, id, 1, tv, ti);
        }
    }
    // this CTA: (m, s) across the warp, then across warps; lists likewise
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, off), s2 = __shfl_xor_sync(0xffffffffu, s, off);
        const float M = fmaxf(m, m2);
        s = (M == -INFINITY) ? 0.f : s * expf(m - M) + s2 * expf(m2 - M);
        m = M;
    }
    float mv[kTreeMaxW];
    int mi[kTreeMaxW];
#pragma unroll
    for (int j = 0; j < kTreeMaxW; ++j) { mv[j] = tv[j]; mi[j] = ti[j]; }   // the warp's list (every lane's copy)
    if (lane == 0) {
        wm[warp] = m;
        ws[warp] = s;
#pragma unroll
        for (int j = 0; j < kTreeMaxW; ++j) { wv[warp][j] = mv[j]; wi[warp][j] = mi[j]; }
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int j = 0; j < kTreeMaxW; ++j) {
            tv[j] = lane < nw ? wv[lane][j] : -INFINITY;
            ti[j] = lane < nw ? wi[lane][j] : INT_MAX;
        }
        tw_warp_merge(tv, ti, mv, mi);
        if (lane == 0) {
            float M = -INFINITY, S = 0.f;
            for (int w = 0; w < nw; ++w) M = fmaxf(M, wm[w]);
            if (M != -INFINITY)
                for (int w = 0; w < nw; ++w) S += ws[w] * expf(wm[w] - M);
            cms[0] = M;
            cms[1] = S;
#pragma unroll
            for (int j = 0; j < kTreeMaxW; ++j) { cv[j] = mv[j]; ci[j] = mi[j]; }
        }
    }
    tw_cluster_sync();   // every CTA's result is in its shared memory
    if (split == 0 && warp == 0) {
        // lane c < kTreeTopwSplit holds CTA c's list; the same warp merge
        const bool on = lane < kTreeTopwSplit;
        const uint32_t pv = tw_mapa(tw_smem_u32(cv), on ? lane : 0), pi = tw_mapa(tw_smem_u32(ci), on ? lane : 0);
#pragma unroll
        for (int j = 0; j < kTreeMaxW; ++j) {
            tv[j] = on ? tw_ld_peer_f32(pv + 4 * j) : -INFINITY;
            ti[j] = on ? tw_ld_peer_s32(pi + 4 * j) : INT_MAX;
        }
        const uint32_t pm = tw_mapa(tw_smem_u32(cms), on ? lane : 0);
        float m1 = on ? tw_ld_peer_f32(pm) : -INFINITY, s1 = on ? tw_ld_peer_f32(pm + 4) : 0.f;
        tw_warp_merge(tv, ti, mv, mi);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m1, off), s2 = __shfl_xor_sync(0xffffffffu, s1, off);
            const float M = fmaxf(m1, m2);
            s1 = (M == -INFINITY) ? 0.f : s1 * expf(m1 - M) + s2 * expf(m2 - M);
            m1 = M;
        }
        if (lane == 0) {
            const float l = m1 + logf(s1);
            if (!isfinite(l)) raise_err(err, ORTHRUS_DEVERR_NONFINITE);
            lse[row] = l;
            for (int j = 0; j < W; ++j) {
                ids[(size_t)row * W + j] = mi[j];
                vals[(size_t)row * W + j] = mv[j];
            }
        }
    }
    tw_cluster_sync();   // no CTA leaves while CTA 0 may still read its shared memory
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

// One sequence's tree rows staged in shared memory by the whole CTA (the walk
// then reads no global memory).  Returns R, the rows in use.
__device__ int tree_stage(const TreeCommitArgs &a, int b, int32_t *par, int32_t *tok, int32_t *g)
{
    const int R = min(max(a.n_rows[b], 1), a.rows);
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        par[r] = a.parent[(size_t)b * a.rows + r];
        tok[r] = a.token[(size_t)b * a.rows + r];
        g[r] = a.g[(size_t)b * a.rows + r];
    }
    __syncthreads();
    return R;
}

// The greedy walk (both kernels, one thread): from the root follow the lowest
// row whose parent is the current row and whose token is the current row's
// argmax g; path[0..m] = rows visited.  Returns m; a malformed parent entry
// raises ORTHRUS_DEVERR_TOKEN and ends the walk there.
__device__ int tree_walk(const int32_t *par, const int32_t *tok, const int32_t *g, int R, unsigned *err,
                         int32_t *path)
{
    int cur = 0, m = 0;
    path[0] = 0;
    for (;;) {
        int next = -1;
        for (int c = cur + 1; c < R && next < 0; ++c) {
            const int p = par[c];
            if (p < 0 || p >= c) { raise_err(err, ORTHRUS_DEVERR_TOKEN); return m; }
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
    __shared__ int32_t path[kTreeMaxRows], s_par[kTreeMaxRows], s_tok[kTreeMaxRows], s_g[kTreeMaxRows];
    __shared__ int m_s, t_s;
    __shared__ T kbuf[32][128], vbuf[32][128];
    pdl_wait();   // no early trigger: tree_finish_kernel writes seq_lens, read here
    const int b = blockIdx.y, layer = blockIdx.x / a.n_kv, kvh = blockIdx.x % a.n_kv, hd = a.hd;
    const int R = tree_stage(a, b, s_par, s_tok, s_g);
    if (threadIdx.x == 0) { m_s = tree_walk(s_par, s_tok, s_g, R, a.err, path); t_s = a.seq_lens[b]; }
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

// Grid B, 128 threads: emitted tokens, n, anchor, seq_len of sequence b.
__global__ void __launch_bounds__(128) tree_finish_kernel(TreeCommitArgs a)
{
    __shared__ int32_t path[kTreeMaxRows], s_par[kTreeMaxRows], s_tok[kTreeMaxRows], s_g[kTreeMaxRows];
    pdl_wait();
    const int b = blockIdx.x;
    const int R = tree_stage(a, b, s_par, s_tok, s_g);
    if (threadIdx.x != 0) return;
    const int m = tree_walk(s_par, s_tok, s_g, R, a.err, path);
    for (int i = 1; i <= m; ++i) a.emit[(size_t)b * a.rows + i - 1] = s_tok[path[i]];
    int last = s_g[path[m]];
    if (last < 0 || last >= a.vocab) { raise_err(a.err, ORTHRUS_DEVERR_TOKEN); last = 0; }
    a.emit[(size_t)b * a.rows + m] = last;
    a.n_out[b] = m + 1;
    a.anchor[b] = last;
    a.seq_lens[b] += m + 1;
}

// Inputs of the tree-masked verify forward, per sequence b and tree row r
// (grid B, kTreeMaxRows threads): the row's token (the anchor for the
// root), its depth (the rotary position is t + depth) and its ancestor bit
// mask (bit j set for every row j on its root path, itself included).  A
// row r > 0 with parent -1 is unused (a tree smaller than the block): it
// gets the anchor, depth 0 and only its own bit.  A parent outside [0, r)
// raises ORTHRUS_DEVERR_TOKEN and leaves the row unused, as does a token
// outside [0, vocab).
__global__ void __launch_bounds__(kTreeMaxRows) tree_prep_kernel(const int32_t *anchor, const int32_t *parent,
                                                                 const int32_t *token, int R, int vocab,
                                                                 int32_t *tok, int32_t *depth, uint32_t *mask,
                                                                 unsigned *err)
{
    __shared__ int32_t s_par[kTreeMaxRows];
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x, r = threadIdx.x;
    if (r < R) s_par[r] = r == 0 ? -1 : parent[(size_t)b * R + r];
    __syncthreads();
    if (r >= R) return;
    int tk = anchor[b], dep = 0;
    uint32_t m[4] = {0u, 0u, 0u, 0u};
    m[r >> 5] |= 1u << (r & 31);
    if (r > 0 && s_par[r] != -1) {
        const int t0 = token[(size_t)b * R + r];
        bool ok = t0 >= 0 && t0 < vocab;
        int cur = r;
        while (ok && cur > 0) {   // at most r steps: parents strictly decrease
            const int p = s_par[cur];
            if (p < 0 || p >= cur) { ok = false; break; }
            m[p >> 5] |= 1u << (p & 31);
            ++dep;
            cur = p;
        }
        if (ok) {
            tk = t0;
        } else {
            raise_err(err, ORTHRUS_DEVERR_TOKEN);
            dep = 0;
            m[0] = m[1] = m[2] = m[3] = 0u;
            m[r >> 5] = 1u << (r & 31);
        }
    }
    const size_t row = (size_t)b * R + r;
    tok[row] = tk;
    depth[row] = dep;
    *(uint4 *)(mask + row * 4) = make_uint4(m[0], m[1], m[2], m[3]);
}

cudaError_t launch_tree_prep(const Ctx &c, const int32_t *anchor, const int32_t *parent, const int32_t *token, int B,
                             int R, cudaStream_t s)
{
    if (R < 1 || R > kTreeMaxRows) return cudaErrorInvalidValue;
    c.launches += 1;
    return launch_k(tree_prep_kernel, B, kTreeMaxRows, 0, s, anchor, parent, token, R, c.cfg.vocab, c.tree_tok,
                    c.tree_depth, c.tree_mask, c.err);
}

cudaError_t launch_tree_topw(const Ctx &c, const float *logits, int rows, int W, int32_t *ids, float *vals,
                             float *lse, cudaStream_t s)
{
    const int V = c.cfg.vocab;
    const bool vec = V % 4 == 0 && ((uintptr_t)logits & 15) == 0;
    const int chunk = ((V + 4 * kTreeTopwSplit - 1) / (4 * kTreeTopwSplit)) * 4;   // a multiple of 4
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kTreeTopwSplit, rows);
    cfg.blockDim = dim3(kTreeTopwThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = kTreeTopwSplit;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    c.launches += 1;
    if (vec) return cudaLaunchKernelEx(&cfg, tree_topw_kernel<true>, logits, V, W, chunk, ids, vals, lse, c.err);
    return cudaLaunchKernelEx(&cfg, tree_topw_kernel<false>, logits, V, W, chunk, ids, vals, lse, c.err);
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
    if (a.hd > 128 || a.rows > kTreeMaxRows || B > 65535) return cudaErrorInvalidValue;
    c.launches += 2;
    const dim3 grid(a.n_layers * a.n_kv, B);
    cudaError_t e = c.cfg.dtype == ORTHRUS_BF16 ? launch_k(tree_compact_kernel<bf16>, grid, 128, 0, s, a)
                                                : launch_k(tree_compact_kernel<float>, grid, 128, 0, s, a);
    if (e != cudaSuccess) return e;
    return launch_k(tree_finish_kernel, B, 128, 0, s, a);
}

}  // namespace orthrus
