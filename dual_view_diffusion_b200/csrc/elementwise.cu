// Row-wise kernels of the decode cycle: block embedding, RMSNorm, the
// LM-head reduction across vocab tiles, consensus and commit.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace orthrus {

// ---------------------------------------------------------------- embedding
// mode 0: draft block [anchor, mask x (K-1)] (paper notes §4.1 step 1)
// mode 1: verify block [anchor, draft[0 .. K-2]] (§4.1 step 2)
// mode 2: explicit tokens (prefill)
template <class T>
__global__ void embed_kernel(const T *embed, int d, int V, int mask_id, int mode, const int32_t *tokens,
                             const int32_t *anchor, const int32_t *draft, int K, int32_t *tok_out, float *h,
                             unsigned *err)
{
    pdl_trigger();
    pdl_wait();
    const int row = blockIdx.x, b = row / K, k = row % K;
    int tok;
    if (mode == 2) tok = tokens[row];
    else if (k == 0) tok = anchor[b];
    else tok = mode == 0 ? mask_id : draft[b * K + k - 1];
    if (tok < 0 || tok >= V) {
        if (threadIdx.x == 0) raise_err(err, ORTHRUS_DEVERR_TOKEN);
        tok = 0;
    }
    if (threadIdx.x == 0) tok_out[row] = tok;
    const T *src = embed + (size_t)tok * d;
    float *dst = h + (size_t)row * d;
    constexpr int E = 16 / (int)sizeof(T);   // elements per 16-byte chunk
    if (d % E == 0 && ((uintptr_t)src & 15) == 0 && ((uintptr_t)dst & 15) == 0) {
        // every chunk of the row in flight at once (one round trip to the table)
        constexpr int Q = 4;
        const int nc = d / E;
        for (int c0 = threadIdx.x; c0 < nc; c0 += Q * blockDim.x) {
            uint4 u[Q];
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const int c = c0 + q * blockDim.x;
                if (c < nc) u[q] = ((const uint4 *)src)[c];
            }
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const int c = c0 + q * blockDim.x;
                if (c >= nc) continue;
                const T *e = (const T *)&u[q];
#pragma unroll
                for (int k4 = 0; k4 < E; k4 += 4)
                    *(float4 *)(dst + (size_t)c * E + k4) =
                        make_float4(to_f<T>(e[k4]), to_f<T>(e[k4 + 1]), to_f<T>(e[k4 + 2]), to_f<T>(e[k4 + 3]));
            }
        }
    } else {
        for (int i = threadIdx.x; i < d; i += blockDim.x) dst[i] = to_f<T>(src[i]);
    }
}

// ---------------------------------------------------------------- RMSNorm
// out = h / sqrt(mean(h^2) + eps) * gain; fixed reduction order per row.
// Rows of up to 8192 elements (multiple of 4) stay in registers: every load
// is issued before the first use.
constexpr int kNormThreads = 512, kNormVec = 2;   // vector path for rows up to 4096

template <class T>
__device__ __forceinline__ void store4(T *p, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float *p, float a, float b, float c, float d)
{
    *(float4 *)p = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16 *p, float a, float b, float c, float d)
{
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *(uint32_t *)&lo;
    u.y = *(uint32_t *)&hi;
    *(uint2 *)p = u;
}

template <class T>
__device__ __forceinline__ float4 load_gain4(const T *g, int i)
{
    return make_float4(to_f<T>(g[i]), to_f<T>(g[i + 1]), to_f<T>(g[i + 2]), to_f<T>(g[i + 3]));
}

template <class T>
// pending > 0: first fold the residual segments part[s][row] (s < pending,
// in order) into h, which is written back.
__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(float *h, const T *gain, T *out, int d, float eps,
                                                               const float *part, int pending, size_t slot_stride)
{
    __shared__ float red[kNormThreads / 32];
    pdl_trigger();
    const int row = blockIdx.x, tid = threadIdx.x;
    const bool vec = (d & 3) == 0 && d <= kNormThreads * 4 * kNormVec;
    // the gain is a weight (no predecessor writes it): fetched before the
    // wait, so the output loop does not wait on a second round trip
    float4 gv[kNormVec];
    if (vec) {
#pragma unroll
        for (int j = 0; j < kNormVec; ++j) {
            const int i = (tid + j * kNormThreads) * 4;
            gv[j] = i < d ? load_gain4(gain, i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    pdl_wait();
    float *x = h + (size_t)row * d;
    float ss = 0.f;
    float4 v[kNormVec];
    if (vec) {
#pragma unroll
        for (int j = 0; j < kNormVec; ++j) {
            const int i = (tid + j * kNormThreads) * 4;
            v[j] = i < d ? *(const float4 *)(x + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (pending > 0) {
            // every segment's loads are issued before the first add
            float4 u[kResidSlots][kNormVec];
#pragma unroll
            for (int sl = 0; sl < kResidSlots; ++sl) {
                const float *p = part + sl * slot_stride + (size_t)row * d;
#pragma unroll
                for (int j = 0; j < kNormVec; ++j) {
                    const int i = (tid + j * kNormThreads) * 4;
                    u[sl][j] = (sl < pending && i < d) ? __ldcg((const float4 *)(p + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int sl = 0; sl < kResidSlots; ++sl) {
                if (sl >= pending) break;
#pragma unroll
                for (int j = 0; j < kNormVec; ++j) {
                    v[j].x += u[sl][j].x; v[j].y += u[sl][j].y; v[j].z += u[sl][j].z; v[j].w += u[sl][j].w;
                }
            }
#pragma unroll
            for (int j = 0; j < kNormVec; ++j) {
                const int i = (tid + j * kNormThreads) * 4;
                if (i < d) *(float4 *)(x + i) = v[j];
            }
        }
#pragma unroll
        for (int j = 0; j < kNormVec; ++j) {
            ss = fmaf(v[j].x, v[j].x, ss); ss = fmaf(v[j].y, v[j].y, ss);
            ss = fmaf(v[j].z, v[j].z, ss); ss = fmaf(v[j].w, v[j].w, ss);
        }
    } else {
        for (int i = tid; i < d; i += kNormThreads) {
            float xi = x[i];
            for (int sl = 0; sl < pending; ++sl) xi += part[sl * slot_stride + (size_t)row * d + i];
            if (pending > 0) x[i] = xi;
            ss = fmaf(xi, xi, ss);
        }
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kNormThreads / 32; ++w) tot += red[w];
    const float inv = 1.0f / sqrtf(tot / d + eps);
    T *o = out + (size_t)row * d;
    if (vec) {
#pragma unroll
        for (int j = 0; j < kNormVec; ++j) {
            const int i = (tid + j * kNormThreads) * 4;
            if (i < d) {
                const float4 g = gv[j];
                store4<T>(o + i, v[j].x * inv * g.x, v[j].y * inv * g.y, v[j].z * inv * g.z, v[j].w * inv * g.w);
            }
        }
    } else {
        for (int i = tid; i < d; i += kNormThreads) o[i] = from_f<T>(x[i] * inv * to_f<T>(gain[i]));
    }
}

// ---------------------------------------------------------------- LM head
// Merge the per-tile records of one row: global max / lowest argmax,
// log-sum-exp of z/T (T = 1 when greedy), Gumbel winner, logit at the
// given id.  mode 0 verify, 1 draft, 2 AR step, 3 residual resample.
struct LmArgs {
    const LmPart *part;
    int n_vtiles, B, K, mode;
    float inv_temp;
    int32_t *draft, *draft_user, *g, *res_tok;
    float *logq, *lse_q, *logp, *lse_p;
    float *ent;
    const int32_t *given, *rej_row;
    unsigned *err;
};

__global__ void __launch_bounds__(256) lm_finalize_kernel(LmArgs a)
{
    pdl_trigger();
    pdl_wait();
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    const int rows = a.mode == 3 ? a.B : a.B * a.K;
    if (w >= rows) return;
    if (a.mode == 3) {
        const int j = a.rej_row[w];
        if (j < 0) return;
        const LmPart *p = a.part + (size_t)(2 * w) * a.n_vtiles;
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int i = lane; i < a.n_vtiles; i += 32) argmax_merge(bv, bi, p[i].gbest, p[i].garg);
        warp_argmax(bv, bi);
        if (lane == 0) a.res_tok[w] = bv > -INFINITY ? bi : a.g[w * a.K + j];
        return;
    }
    const LmPart *p = a.part + (size_t)w * a.n_vtiles;
    float zm = -INFINITY;
    int za = 0x7fffffff;
    float gb = -INFINITY, gz = 0.f;
    int ga = 0x7fffffff;
    float zid = NAN;
    // (unrolled: the tiles' records are independent loads, in flight together)
#pragma unroll 4
    for (int i = lane; i < a.n_vtiles; i += 32) {
        const LmPart q = p[i];
        argmax_merge(zm, za, q.zmax, q.zarg);
        if (q.gbest > gb || (q.gbest == gb && q.garg < ga)) { gb = q.gbest; ga = q.garg; gz = q.gz; }
        if (!isnan(q.zid)) zid = q.zid;
    }
    warp_argmax(zm, za);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float gb2 = __shfl_xor_sync(0xffffffffu, gb, o);
        const int ga2 = __shfl_xor_sync(0xffffffffu, ga, o);
        const float gz2 = __shfl_xor_sync(0xffffffffu, gz, o);
        if (gb2 > gb || (gb2 == gb && ga2 < ga)) { gb = gb2; ga = ga2; gz = gz2; }
    }
    const unsigned has = __ballot_sync(0xffffffffu, !isnan(zid));
    if (has) zid = __shfl_sync(0xffffffffu, zid, __ffs(has) - 1);
    const float it = a.inv_temp > 0.f ? a.inv_temp : 1.0f;
    float s = 0.f, ez = 0.f;
#pragma unroll 4
    for (int i = lane; i < a.n_vtiles; i += 32) {
        const float f = expf((p[i].zmax - zm) * it);
        s += p[i].zsum * f;
        if (a.mode == 1) ez = fmaf(p[i].zez, f, ez);
    }
    s = warp_sum(s);
    if (a.mode == 1) ez = warp_sum(ez);
    const float lse = zm * it + logf(s);
    if (lane != 0) return;
    if (!isfinite(lse)) raise_err(a.err, ORTHRUS_DEVERR_NONFINITE);
    if (a.mode == 0) {
        a.g[w] = za;
        a.lse_p[w] = lse;
        a.logp[w] = zid * it - lse;
        if (a.given) a.draft[w] = a.given[w];
    } else if (a.mode == 1) {
        const int tok = a.inv_temp > 0.f ? ga : za;
        a.draft[w] = tok;
        if (a.draft_user) a.draft_user[w] = tok;
        a.lse_q[w] = lse;
        a.logq[w] = (a.inv_temp > 0.f ? gz : zm) * it - lse;
        // entropy of softmax(z / T): LSE(z / T) - E[z] / T
        if (a.ent) a.ent[w] = lse - it * (ez / s);
    } else {
        a.g[w] = a.inv_temp > 0.f ? ga : za;
    }
}

// The draft rows' top-W candidates (tree verification) from the LM-head
// epilogue's per-tile records: one warp per (sequence, row < depth), each
// lane a sorted top-W of the tiles it scans, merged across the warp (ties
// to the lowest id), with the row's log-sum-exp (T = 1: the draft is
// greedy).
__global__ void __launch_bounds__(256) topw_finalize_kernel(const TopRec *top, const float *lse_q, int n_vtiles, int B,
                                                            int K, int depth, int W, int32_t *ids, float *vals,
                                                            float *lse)
{
    pdl_trigger();
    pdl_wait();
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= B * depth) return;
    const int b = w / depth, k = w % depth, row = b * K + k;
    float tv[kTopWMax];
    int ti[kTopWMax];
#pragma unroll
    for (int j = 0; j < kTopWMax; ++j) { tv[j] = -INFINITY; ti[j] = INT_MAX; }
    for (int t = lane; t < n_vtiles; t += 32) {
        const TopRec *p = top + ((size_t)row * n_vtiles + t) * kTopWMax;
        for (int r = 0; r < W; ++r) {
            const TopRec q = p[r];
            if (!tw_better(q.z, q.id, tv[kTopWMax - 1], ti[kTopWMax - 1])) break;   // the tile's list is sorted
            tw_insert(q.z, q.id, tv, ti);
        }
    }
    float ov[kTopWMax];
    int oi[kTopWMax];
    tw_warp_merge(tv, ti, ov, oi);
    if (lane == 0) {
        for (int r = 0; r < W; ++r) {
            ids[(size_t)w * W + r] = oi[r];
            vals[(size_t)w * W + r] = ov[r];
        }
        lse[w] = lse_q[row];
    }
}

// ---------------------------------------------------------------- commit
struct CommitArgs {
    int B, K;
    float inv_temp;
    uint64_t seed;
    int64_t *step;
    const int32_t *force_n;
    const int32_t *kt;       // greedy: per-sequence verify length (consensus over its first kt rows), or null
    const int32_t *draft, *g, *res_tok;
    const float *logp, *logq;
    int32_t *rej_row;
    int *any_reject;
    const void *fin_verify, *fin_draft;
    void *res_x;
    int d, esize;
    int32_t *n_out, *tokens_out, *anchor_io, *seq_lens;
    int32_t *append_out, *produced;
    int append_stride, append_max;
};

// Decide n per sequence (paper notes §4.2 greedy, §4.3 sampled); for a
// sampled rejection at row j, stage the two hidden rows the residual draw
// needs (AR view, diffusion view).
__global__ void commit_decide_kernel(CommitArgs a)
{
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x, lane = threadIdx.x & 31;
    __shared__ int s_j;
    if (threadIdx.x < 32) {   // warp 0: rows k = lane, lane + 32, ... tested at once, the first failure wins
        int n = a.K, j = -1;
        if (a.force_n) {
            n = min(max(a.force_n[b], 1), a.K);
        } else if (a.inv_temp <= 0.f) {
            const int kt = a.kt ? min(max(a.kt[b], 1), a.K) : a.K;
            n = kt;
            for (int k0 = 0; k0 < kt; k0 += 32) {
                const int k = k0 + lane;
                const unsigned miss = __ballot_sync(0xffffffffu, k < kt && a.draft[b * a.K + k] != a.g[b * a.K + k]);
                if (miss) { n = k0 + __ffs(miss); break; }
            }
        } else {
            const uint32_t step = (uint32_t)*a.step;
            for (int k0 = 0; k0 < a.K; k0 += 32) {
                const int k = k0 + lane;
                bool rej = false;
                if (k < a.K) {
                    const float log_u = -neg_log_uniform(a.seed, step, rng_row(b, k), 0, PURPOSE_ACCEPT);
                    rej = !(log_u < a.logp[b * a.K + k] - a.logq[b * a.K + k]);
                }
                const unsigned r = __ballot_sync(0xffffffffu, rej);
                if (r) { j = k0 + __ffs(r) - 1; n = j + 1; break; }
            }
        }
        if (lane == 0) {
            a.n_out[b] = n;
            if (a.rej_row) a.rej_row[b] = j;
            if (j >= 0) atomicOr(a.any_reject, 1);
            s_j = j;
        }
    }
    __syncthreads();
    if (s_j >= 0 && a.res_x) {
        const size_t bytes = (size_t)a.d * a.esize;
        const char *sv = (const char *)a.fin_verify + (size_t)(b * a.K + s_j) * bytes;
        const char *sd = (const char *)a.fin_draft + (size_t)(b * a.K + s_j) * bytes;
        char *dv = (char *)a.res_x + (size_t)(2 * b) * bytes;
        for (size_t i = threadIdx.x; i < bytes; i += blockDim.x) { dv[i] = sv[i]; dv[bytes + i] = sd[i]; }
    }
}

// Emit the tokens, advance the committed length (the accepted rows' AR K/V
// are already in place: paper notes §4.1 step 3), bump the step counter.
__global__ void commit_apply_kernel(CommitArgs a)
{
    // no early pdl_trigger: later kernels read what this one writes before
    // their griddepcontrol.wait, so nothing may be scheduled until it exits
    pdl_wait();
    // one warp per sequence, a lane per emitted token
    const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (b < a.B) {
        const int n = a.n_out[b];
        const int j = a.rej_row ? a.rej_row[b] : -1;
        const bool sampled = a.inv_temp > 0.f && !a.force_n;
        const int p0 = a.append_out ? a.produced[b] : 0;
        for (int i = lane; i < n; i += 32) {
            int tok;
            if (!sampled) tok = a.g[b * a.K + i];
            else tok = (i == j) ? a.res_tok[b] : a.draft[b * a.K + i];
            if (a.tokens_out) a.tokens_out[b * a.K + i] = tok;
            if (a.append_out && p0 + i < a.append_max) a.append_out[(size_t)b * a.append_stride + p0 + i] = tok;
            if (i == n - 1) a.anchor_io[b] = tok;
        }
        __syncwarp();   // every lane has read produced[b]
        if (lane == 0) {
            if (a.append_out) a.produced[b] = p0 + n;
            a.seq_lens[b] += n;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {   // nothing in this kernel reads them
        *a.step += 1;
        if (a.any_reject) *a.any_reject = 0;
    }
}

// ---------------------------------------------------------------- AR step
__global__ void ar_commit_kernel(int B, const int32_t *g, int64_t *step, int32_t *token_out, int32_t *anchor_io,
                                 int32_t *seq_lens, int32_t *append_out, int32_t *produced, int stride, int amax)
{
    // no early pdl_trigger: later kernels read what this one writes before
    // their griddepcontrol.wait, so nothing may be scheduled until it exits
    pdl_wait();
    const int b = threadIdx.x;
    if (b < B) {
        const int tok = g[b];
        if (token_out) token_out[b] = tok;
        anchor_io[b] = tok;
        seq_lens[b] += 1;
        if (append_out) {
            if (produced[b] < amax) append_out[(size_t)b * stride + produced[b]] = tok;
            produced[b] += 1;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) *step += 1;
}

// Adaptive block length (reading of the paper-notes page §7.4 / §9.6): per
// sequence, 1 + the number of leading drafted tokens y_1, y_2, ... (y_k from
// draft row k-1) whose rows' entropies are at most h_max, at most K.
__global__ void adaptive_len_kernel(const float *ent, int B, int K, float h_max, int32_t *kt, float *ent_out)
{
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    int k = 1;
    while (k < K && ent[b * K + k - 1] <= h_max) ++k;
    kt[b] = k;
    if (ent_out)
        for (int i = 0; i < K; ++i) ent_out[b * K + i] = ent[b * K + i];
}

__global__ void set_lens_kernel(int32_t *seq_lens, int b, int value, int32_t *anchor_out, const int32_t *last_tok)
{
    // no early pdl_trigger: later kernels read what this one writes before
    // their griddepcontrol.wait, so nothing may be scheduled until it exits
    pdl_wait();
    seq_lens[b] = value;
    if (anchor_out) anchor_out[b] = *last_tok;
}

// Block K/V given as [B][K][n_kv][hd] -> K [B][n_kv][kp][hd] and V transposed
// [B][n_kv][hd][kp] (rows K .. kp-1 zero).  Grid (n_kv, B, kp / 16), 256
// threads, 16 rows per CTA: K is copied row by row, V is staged in shared
// memory and written out a dim at a time (16 consecutive rows), so the
// loads and stores of a warp touch consecutive elements; every load of a
// thread is in flight at once (hd <= 128).
template <class T>
__global__ void __launch_bounds__(256) pack_block_kernel(const T *__restrict__ ks, const T *__restrict__ vs,
                                                         T *__restrict__ kd, T *__restrict__ vd, int K, int kp,
                                                         int n_kv, int hd)
{
    constexpr int kRows = 16;
    constexpr int kPad = 4 / (int)sizeof(T);   // a 32-bit word per row: a column read walks the banks
    __shared__ T tile[kRows][128 + kPad];
    pdl_trigger();
    pdl_wait();
    const int kvh = blockIdx.x, b = blockIdx.y, k0 = blockIdx.z * kRows;
    const size_t head = (size_t)b * n_kv + kvh;
    const T z = from_f<T>(0.f);
    const int n = kRows * hd;
#pragma unroll 8
    for (int i = threadIdx.x; i < n; i += 256) {
        const int r = i / hd, d = i % hd, k = k0 + r;
        const size_t src = (((size_t)b * K + k) * n_kv + kvh) * hd + d;
        const bool in = k < K;
        kd[(head * kp + k) * hd + d] = in ? ks[src] : z;
        tile[r][d] = in ? vs[src] : z;
    }
    __syncthreads();
#pragma unroll 8
    for (int i = threadIdx.x; i < n; i += 256) {
        const int d = i / kRows, r = i % kRows;
        vd[(head * hd + d) * kp + k0 + r] = tile[r][d];
    }
}

// Rows of two views into one interleaved activation buffer: out[2r] =
// a[r], out[2r+1] = b[r] (the row pairs of the forward-KL LM-head GEMM).
template <class T>
__global__ void interleave_rows_kernel(const T *ra, const T *rb, T *out, int d)
{
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        out[(size_t)(2 * r) * d + i] = ra[(size_t)r * d + i];
        out[(size_t)(2 * r + 1) * d + i] = rb[(size_t)r * d + i];
    }
}

// Forward KL per row pair from the per-tile records of EPI_KL (paper notes
// §3.3): with M = max over tiles, S = sum_t s_t exp(m_t - M) for each view
// and T = sum_t t_t exp(ma_t - M_AR),
//     LSE = M + log S,   KL(p_AR || p_diff) = T / S_AR - (LSE_AR - LSE_diff).
struct KlArgs {
    const KlPart *part;
    int n_vtiles, rows;
    float *kl, *lse_a, *lse_d;
    unsigned *err;
};

__global__ void __launch_bounds__(256) kl_finalize_kernel(KlArgs a)
{
    pdl_trigger();
    pdl_wait();
    const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (w >= a.rows) return;
    const KlPart *p = a.part + (size_t)w * a.n_vtiles;
    float Ma = -INFINITY, Md = -INFINITY;
    for (int i = lane; i < a.n_vtiles; i += 32) {
        Ma = fmaxf(Ma, p[i].ma);
        Md = fmaxf(Md, p[i].md);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        Ma = fmaxf(Ma, __shfl_xor_sync(0xffffffffu, Ma, o));
        Md = fmaxf(Md, __shfl_xor_sync(0xffffffffu, Md, o));
    }
    float Sa = 0.f, Ta = 0.f, Sd = 0.f;
    for (int i = lane; i < a.n_vtiles; i += 32) {
        const float fa = expf(p[i].ma - Ma);
        Sa = fmaf(p[i].sa, fa, Sa);
        Ta = fmaf(p[i].ta, fa, Ta);
        Sd = fmaf(p[i].sd, expf(p[i].md - Md), Sd);
    }
    Sa = warp_sum(Sa);
    Ta = warp_sum(Ta);
    Sd = warp_sum(Sd);
    if (lane != 0) return;
    const float la = Ma + logf(Sa), ld = Md + logf(Sd);
    const float kl = Ta / Sa - (la - ld);
    if (!isfinite(kl)) raise_err(a.err, ORTHRUS_DEVERR_NONFINITE);
    a.kl[w] = kl;
    if (a.lse_a) a.lse_a[w] = la;
    if (a.lse_d) a.lse_d[w] = ld;
}

__global__ void set_int_kernel(int32_t *p, int v)
{
    // no early pdl_trigger: later kernels read what this one writes before
    // their griddepcontrol.wait, so nothing may be scheduled until it exits
    pdl_wait();
    *p = v;
}

// ---------------------------------------------------------------- host
cudaError_t launch_embed(const Ctx &c, int mode, const int32_t *tokens, const int32_t *anchor, const int32_t *draft,
                         int B, int K, cudaStream_t s)
{
    const int rows = B * K;
    c.launches += 1;
    if (c.cfg.dtype == ORTHRUS_BF16)
        return launch_k(embed_kernel<bf16>, rows, 256, 0, s, (const bf16 *)c.embed, c.cfg.hidden, c.cfg.vocab,
                        c.cfg.mask_token_id, mode, tokens, anchor, draft, K, c.tok, c.h, c.err);
    return launch_k(embed_kernel<float>, rows, 256, 0, s, (const float *)c.embed, c.cfg.hidden, c.cfg.vocab,
                    c.cfg.mask_token_id, mode, tokens, anchor, draft, K, c.tok, c.h, c.err);
}

cudaError_t launch_rmsnorm(const Ctx &c, float *h, const void *gain, void *out, int M, int pending, cudaStream_t s)
{
    c.launches += 1;
    const size_t stride = (size_t)c.Rw * c.cfg.hidden;
    if (c.cfg.dtype == ORTHRUS_BF16)
        return launch_k(rmsnorm_kernel<bf16>, M, kNormThreads, 0, s, h, (const bf16 *)gain, (bf16 *)out, c.cfg.hidden,
                        c.cfg.rms_eps, (const float *)c.resid_part, pending, stride);
    return launch_k(rmsnorm_kernel<float>, M, kNormThreads, 0, s, h, (const float *)gain, (float *)out, c.cfg.hidden,
                    c.cfg.rms_eps, (const float *)c.resid_part, pending, stride);
}

cudaError_t launch_lm_finalize_impl(const Ctx &c, int mode, int B, int K, float temperature, int32_t *tok_out,
                                    const int32_t *given, cudaStream_t s)
{
    LmArgs a;
    a.part = c.lm_part; a.n_vtiles = c.n_vtiles; a.B = B; a.K = K; a.mode = mode;
    a.inv_temp = temperature > 0.f ? 1.0f / temperature : 0.f;
    a.draft = c.draft; a.draft_user = tok_out; a.g = c.g; a.res_tok = c.res_tok;
    a.logq = c.logq; a.lse_q = c.lse_q; a.logp = c.logp; a.lse_p = c.lse_p;
    a.given = given; a.rej_row = c.rej_row; a.err = c.err; a.ent = c.ent;
    const int rows = mode == 3 ? B : B * K;
    c.launches += 1;
    return launch_k(lm_finalize_kernel, (rows + 7) / 8, 256, 0, s, a);
}

cudaError_t launch_lm_finalize(const Ctx &c, int mode, int B, int K, float temperature, uint64_t, const int64_t *,
                               int32_t *tok_out, cudaStream_t s)
{
    return launch_lm_finalize_impl(c, mode, B, K, temperature, tok_out, mode == 0 ? tok_out : nullptr, s);
}

cudaError_t launch_topw_finalize(const Ctx &c, int B, int K, int depth, int W, int32_t *ids, float *vals, float *lse,
                                 cudaStream_t s)
{
    c.launches += 1;
    return launch_k(topw_finalize_kernel, (B * depth + 7) / 8, 256, 0, s, (const TopRec *)c.top_part,
                    (const float *)c.lse_q, c.n_vtiles, B, K, depth, W, ids, vals, lse);
}

static CommitArgs commit_args(const Ctx &c, const orthrus_kv_t &kv, int B, int K, float temperature, uint64_t seed,
                              int64_t *step, const int32_t *force_n, int32_t *n_out, int32_t *tokens_out,
                              int32_t *anchor_io, int32_t *append_out, int append_stride, int append_max)
{
    CommitArgs a;
    a.B = B; a.K = K; a.inv_temp = temperature > 0.f ? 1.0f / temperature : 0.f;
    a.seed = seed; a.step = step; a.force_n = force_n; a.kt = nullptr;
    a.draft = c.draft; a.g = c.g; a.res_tok = c.res_tok; a.logp = c.logp; a.logq = c.logq;
    a.rej_row = c.rej_row; a.any_reject = c.any_reject;
    a.fin_verify = c.fin_verify; a.fin_draft = c.fin_draft; a.res_x = c.res_x;
    a.d = c.cfg.hidden; a.esize = c.esize;
    a.n_out = n_out; a.tokens_out = tokens_out; a.anchor_io = anchor_io; a.seq_lens = kv.seq_lens;
    a.append_out = append_out; a.produced = c.produced; a.append_stride = append_stride; a.append_max = append_max;
    return a;
}

cudaError_t launch_commit(const Ctx &c, const orthrus_kv_t &kv, int B, int K, float temperature, uint64_t seed,
                          int64_t *step, const int32_t *force_n, int32_t *n_out, int32_t *tokens_out,
                          int32_t *anchor_io, int32_t *append_out, int append_stride, int append_max,
                          cudaStream_t s, const int32_t *kt)
{
    CommitArgs a = commit_args(c, kv, B, K, temperature, seed, step, force_n, n_out, tokens_out, anchor_io,
                               append_out, append_stride, append_max);
    a.kt = kt;
    c.launches += 2;
    cudaError_t e = launch_k(commit_decide_kernel, B, 128, 0, s, a);
    if (e != cudaSuccess) return e;
    if (temperature > 0.f && !force_n) {
        // residual draw at the rejected row: one LM-head pass over the two
        // staged hidden rows per sequence (skipped on device when nothing
        // was rejected)
        GemmArgs g{};
        g.x = c.res_x; g.M = 2 * B; g.N = c.cfg.vocab; g.Kd = c.cfg.hidden;
        g.w[0] = c.lm_head; g.wrows[0] = c.cfg.vocab;
        g.epi = EPI_RESAMPLE; g.lm = c.lm_part; g.inv_temp = 1.0f / temperature; g.seed = seed; g.step = step;
        g.lse_p = c.lse_p; g.lse_q = c.lse_q; g.rej_row = c.rej_row; g.any_flag = c.any_reject; g.K = K;
        e = launch_gemm(c, g, s);
        if (e != cudaSuccess) return e;
        e = launch_lm_finalize_impl(c, 3, B, K, temperature, nullptr, nullptr, s);
        if (e != cudaSuccess) return e;
    }
    return launch_k(commit_apply_kernel, (B + 3) / 4, 128, 0, s, a);
}

cudaError_t launch_ar_commit(const Ctx &c, const orthrus_kv_t &kv, int B, int64_t *step, int32_t *token_out,
                             int32_t *anchor_io, int32_t *append_out, int append_stride, int append_max,
                             cudaStream_t s)
{
    c.launches += 1;
    return launch_k(ar_commit_kernel, 1, 128, 0, s, B, (const int32_t *)c.g, step, token_out, anchor_io, kv.seq_lens,
                    append_out, c.produced, append_stride, append_max);
}

cudaError_t launch_set_lens(const Ctx &, int32_t *seq_lens, int b, int value, int32_t *anchor_out,
                            const int32_t *last_tok, cudaStream_t s)
{
    return launch_k(set_lens_kernel, 1, 1, 0, s, seq_lens, b, value, anchor_out, last_tok);
}

cudaError_t launch_adaptive_len(const Ctx &c, int B, int K, float h_max, int32_t *kt, float *ent_out, cudaStream_t s)
{
    c.launches += 1;
    return launch_k(adaptive_len_kernel, (B + 127) / 128, 128, 0, s, (const float *)c.ent, B, K, h_max, kt, ent_out);
}

cudaError_t launch_set_int(int32_t *p, int v, cudaStream_t s)
{
    return launch_k(set_int_kernel, 1, 1, 0, s, p, v);
}

cudaError_t launch_pack_block(const Ctx &c, const void *k_src, const void *v_src, void *k_dst, void *v_dst, int B,
                              int K, int kp, cudaStream_t s)
{
    c.launches += 1;
    if (kp % 16 || c.cfg.head_dim > 128) return cudaErrorInvalidValue;
    const dim3 grid(c.cfg.n_kv_heads, B, kp / 16);
    if (c.cfg.dtype == ORTHRUS_BF16)
        return launch_k(pack_block_kernel<bf16>, grid, 256, 0, s, (const bf16 *)k_src, (const bf16 *)v_src,
                        (bf16 *)k_dst, (bf16 *)v_dst, K, kp, c.cfg.n_kv_heads, c.cfg.head_dim);
    return launch_k(pack_block_kernel<float>, grid, 256, 0, s, (const float *)k_src, (const float *)v_src,
                    (float *)k_dst, (float *)v_dst, K, kp, c.cfg.n_kv_heads, c.cfg.head_dim);
}

cudaError_t launch_kl_lm_head(const Ctx &c, const void *h_a, const void *h_d, int rows, float *kl, float *lse_a,
                              float *lse_d, cudaStream_t s)
{
    const int d = c.cfg.hidden;
    c.launches += 1;
    cudaError_t e = c.cfg.dtype == ORTHRUS_BF16
                        ? launch_k(interleave_rows_kernel<bf16>, rows, 256, 0, s, (const bf16 *)h_a, (const bf16 *)h_d,
                                   (bf16 *)c.a, d)
                        : launch_k(interleave_rows_kernel<float>, rows, 256, 0, s, (const float *)h_a,
                                   (const float *)h_d, (float *)c.a, d);
    if (e != cudaSuccess) return e;
    GemmArgs g{};
    g.x = c.a; g.M = 2 * rows; g.N = c.cfg.vocab; g.Kd = d;
    g.w[0] = c.lm_head; g.wrows[0] = c.cfg.vocab;
    g.epi = EPI_KL; g.kl = (KlPart *)c.lm_part;
    e = launch_gemm(c, g, s);
    if (e != cudaSuccess) return e;
    KlArgs k;
    k.part = (const KlPart *)c.lm_part; k.n_vtiles = c.n_vtiles; k.rows = rows;
    k.kl = kl; k.lse_a = lse_a; k.lse_d = lse_d; k.err = c.err;
    c.launches += 1;
    return launch_k(kl_finalize_kernel, (rows + 7) / 8, 256, 0, s, k);
}

cudaError_t launch_logits_dump(const Ctx &c, const void *fin, int M, float *logits, cudaStream_t s)
{
    GemmArgs g{};
    g.x = fin; g.M = M; g.N = c.cfg.vocab; g.Kd = c.cfg.hidden;
    g.w[0] = c.lm_head; g.wrows[0] = c.cfg.vocab;
    g.epi = EPI_LOGITS; g.logits = logits;
    return launch_gemm(c, g, s);
}

}  // namespace orthrus
