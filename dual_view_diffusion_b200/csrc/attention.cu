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

constexpr int kAttnRowsMma = 128;   // rows per CTA, tensor-core kernel (8 warps x 16)
constexpr int kAttnRowsSimt = 32;   // rows per CTA, SIMT kernel
constexpr float kLog2e = 1.4426950408889634f;

struct KeySrc {
    const void *k, *v;   // row pointers (element type erased), null = zero fill
};

// Source rows of key position p for (b, kvh); null when p is outside
// [0, key_end) or its page is not mapped.
template <class T>
__device__ __forceinline__ KeySrc key_src(const AttnArgs &a, int b, int kvh, int t, int p, int key_end)
{
    KeySrc r{nullptr, nullptr};
    if (p >= key_end) return r;
    if (a.mode == 1 && p >= t) {
        const size_t off = ((size_t)(b * a.K + (p - t)) * a.n_kv + kvh) * a.hd;
        r.k = (const T *)a.k_blk + off;
        r.v = (const T *)a.v_blk + off;
        return r;
    }
    const int pidx = p / a.kv.page_size;
    if (pidx >= a.kv.max_pages) { raise_err(a.err, ORTHRUS_DEVERR_CAPACITY); return r; }
    const int page = a.kv.block_table[(size_t)a.bt_rows[b] * a.kv.max_pages + pidx];
    if (page < 0 || page >= a.kv.num_pages) { raise_err(a.err, ORTHRUS_DEVERR_CAPACITY); return r; }
    const size_t off = (((size_t)a.layer * a.kv.num_pages + page) * a.n_kv + kvh) * (size_t)a.kv.page_size * a.hd +
                       (size_t)(p % a.kv.page_size) * a.hd;
    r.k = (const T *)a.kv.k_pages + off;
    r.v = (const T *)a.kv.v_pages + off;
    return r;
}

// ---------------------------------------------------------------- tensor cores
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};\n"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *(const uint32_t *)&v;
}

// 128-element (256-byte) rows: 16-byte chunk c of row r sits at chunk
// c ^ (r & 7), which keeps ldmatrix phases conflict-free.
__device__ __forceinline__ int swz128(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 3); }

struct AttnSmem {
    bf16 q[kAttnRowsMma * 128];
    bf16 k[2][kKeyTile * 128];
    bf16 v[2][kKeyTile * 128];
};

__global__ void __launch_bounds__(256, 1) attn_split_mma(AttnArgs a, int n_split_grid)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    AttnSmem &sm = *(AttnSmem *)smem_raw;
    pdl_trigger();
    pdl_wait();
    // grid (kv head, sequence x row group, split): the split index varies
    // slowest, so the CTAs of splits a short sequence never reaches (they
    // exit at once) come after every working CTA
    const int kvh = blockIdx.x, s = blockIdx.z;
    const int rgroups = gridDim.y / a.B, b = blockIdx.y / rgroups, rg = blockIdx.y % rgroups;
    const int g = a.n_q / a.n_kv, R = a.K * g, r0 = rg * kAttnRowsMma;
    if (r0 >= R) return;
    const int t = a.seq_lens[b];
    const int kv_len = t + a.K;
    const int key0 = s * a.split_tokens;
    const int key1 = min(key0 + a.split_tokens, kv_len);
    if (key0 >= kv_len) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // Q rows -> shared (row r = block row k * g + head j of the group)
    for (int idx = tid; idx < kAttnRowsMma * 16; idx += 256) {
        const int r = idx >> 4, ch = idx & 15, rr = r0 + r;
        const bf16 *src = (const bf16 *)a.q;
        int bytes = 0;
        if (rr < R) {
            const int k = rr / g, j = rr % g;
            src = (const bf16 *)a.q + ((size_t)(b * a.K + k) * a.n_q + kvh * g + j) * 128 + ch * 8;
            bytes = 16;
        }
        cp_async16(smem_u32(sm.q + swz128(r, ch)), src, bytes);
    }
    cp_async_commit();

    const int ntiles = (key1 - key0 + kKeyTile - 1) / kKeyTile;
    auto load_tile = [&](int buf, int ti) {
        const int p0 = key0 + ti * kKeyTile;
        const int ch = tid & 15;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = (tid >> 4) + 16 * i;
            const KeySrc src = key_src<bf16>(a, b, kvh, t, p0 + row, key1);
            const bf16 *ks = src.k ? (const bf16 *)src.k + ch * 8 : (const bf16 *)a.q;
            const bf16 *vs = src.v ? (const bf16 *)src.v + ch * 8 : (const bf16 *)a.q;
            cp_async16(smem_u32(sm.k[buf] + swz128(row, ch)), ks, src.k ? 16 : 0);
            cp_async16(smem_u32(sm.v[buf] + swz128(row, ch)), vs, src.v ? 16 : 0);
        }
    };
    load_tile(0, 0);
    cp_async_commit();

    // rows of this thread: local rows lr0 = warp*16 + lane/4 and lr0 + 8
    const int lr0 = warp * 16 + (lane >> 2);
    int lim[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rr = r0 + lr0 + 8 * h;
        const int k = min(rr, R - 1) / g;
        lim[h] = a.mode == 0 ? t + k + 1 : kv_len;
    }
    const float scale = kLog2e / sqrtf(128.f);

    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    uint32_t qf[8][4];

    for (int ti = 0; ti < ntiles; ++ti) {
        const int buf = ti & 1;
        if (ti + 1 < ntiles) load_tile(buf ^ 1, ti + 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (ti == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                ldsm_x4(smem_u32(sm.q + swz128(warp * 16 + (lane & 15), ks * 2 + (lane >> 4))), qf[ks][0], qf[ks][1],
                        qf[ks][2], qf[ks][3]);
        }
        const uint32_t kb = smem_u32(sm.k[buf]), vb = smem_u32(sm.v[buf]);
        float sc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) sc[i][j] = 0.f;
#pragma unroll
        for (int n2 = 0; n2 < 4; ++n2)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int mi = lane >> 3;
                const int key = n2 * 16 + (mi >> 1) * 8 + (lane & 7);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + 2 * swz128(key, ks * 2 + (mi & 1)), b0, b1, b2, b3);
                mma16816(sc[2 * n2], qf[ks], b0, b1);
                mma16816(sc[2 * n2 + 1], qf[ks], b2, b3);
            }
        // mask, online softmax (log2 domain)
        const int p0 = key0 + ti * kKeyTile;
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e >> 1, p = p0 + n * 8 + (lane & 3) * 2 + (e & 1);
                const float v = (p < lim[h] && p < key1) ? sc[n][e] * scale : -INFINITY;
                sc[n][e] = v;
                tmax[h] = fmaxf(tmax[h], v);
            }
        float alpha[2], mu[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 1));
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 2));
            const float mn = fmaxf(m_run[h], tmax[h]);
            mu[h] = mn == -INFINITY ? 0.f : mn;
            alpha[h] = exp2f(m_run[h] - mu[h]);
            m_run[h] = mn;
        }
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e >> 1;
                const float p = exp2f(sc[n][e] - mu[h]);
                sc[n][e] = p;
                rs[h] += p;
            }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 1);
            rs[h] += __shfl_xor_sync(0xffffffffu, rs[h], 2);
            l_run[h] = l_run[h] * alpha[h] + rs[h];
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            o[i][0] *= alpha[0]; o[i][1] *= alpha[0];
            o[i][2] *= alpha[1]; o[i][3] *= alpha[1];
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t pa[4];
            pa[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
            pa[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
            pa[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
            pa[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {
                const int mi = lane >> 3;
                const int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vb + 2 * swz128(key, 2 * dp + (mi >> 1)), b0, b1, b2, b3);
                mma16816(o[2 * dp], pa, b0, b1);
                mma16816(o[2 * dp + 1], pa, b2, b3);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    // unnormalised partials
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rr = r0 + lr0 + 8 * h;
        if (rr >= R) continue;
        const int k = rr / g, j = rr % g;
        const size_t rowhead = (size_t)(b * a.K + k) * a.n_q + kvh * g + j;
        float *dst = a.part + (rowhead * a.n_splits + s) * 128;
#pragma unroll
        for (int dn = 0; dn < 16; ++dn) {
            const int c = dn * 8 + (lane & 3) * 2;
            *(float2 *)(dst + c) = make_float2(o[dn][2 * h], o[dn][2 * h + 1]);
        }
        if ((lane & 3) == 0) a.ml[rowhead * a.n_splits + s] = make_float2(m_run[h], l_run[h]);
    }
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
    const int kvh = blockIdx.x, s = blockIdx.z;
    const int rgroups = gridDim.y / a.B, b = blockIdx.y / rgroups, rg = blockIdx.y % rgroups;
    const int g = a.n_q / a.n_kv, R = a.K * g, r0 = rg * kAttnRowsSimt;
    if (r0 >= R) return;
    const int t = a.seq_lens[b], kv_len = t + a.K;
    const int key0 = s * a.split_tokens, key1 = min(key0 + a.split_tokens, kv_len);
    if (key0 >= kv_len) return;
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
            const KeySrc src = key_src<T>(a, b, kvh, t, p0 + row, key1);
            ks[row * hp + d] = src.k ? to_f<T>(((const T *)src.k)[d]) : 0.f;
            vs[row * hp + d] = src.v ? to_f<T>(((const T *)src.v)[d]) : 0.f;
        }
        __syncthreads();
        for (int r = warp; r < nr; r += 4) {
            const int k = (r0 + r) / g;
            const int lim = a.mode == 0 ? t + k + 1 : kv_len;
            float sv[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h, p = p0 + j;
                float acc = 0.f;
                for (int d = 0; d < hd; ++d) acc = fmaf(qs[r * hd + d], ks[j * hp + d], acc);
                sv[h] = (p < lim && p < key1) ? acc * scale : -INFINITY;
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
        a.part[(rowhead * a.n_splits + s) * hd + d] = os[idx];
        if (d == 0) a.ml[rowhead * a.n_splits + s] = make_float2(ms[r], ls[r]);
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
    const int kv_len = a.seq_lens[b] + a.K;
    int n_used = (kv_len + a.split_tokens - 1) / a.split_tokens;
    if (n_used > a.n_splits) {   // longer than the context was sized for
        if (lane == 0) raise_err(a.err, ORTHRUS_DEVERR_CAPACITY);
        n_used = a.n_splits;
    }
    const float2 *ml = a.ml + (size_t)w * a.n_splits;
    float M = -INFINITY;
    for (int s = lane; s < n_used; s += 32) M = fmaxf(M, ml[s].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int s = lane; s < n_used; s += 32) L += ml[s].y * exp2f(ml[s].x - M);
    L = warp_sum(L);
    const float inv = 1.0f / L;
    const float *part = a.part + (size_t)w * a.n_splits * a.hd;
    const int c0 = lane * 4;
    const bool mine = c0 < a.hd;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n_used; s0 += 32) {
        const int sl = s0 + lane;
        const float wl = sl < n_used ? exp2f(ml[sl].x - M) : 0.f;
        const int cnt = min(32, n_used - s0);
        for (int j0 = 0; j0 < cnt; j0 += 8) {
            float4 v[8];
            float wt[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                wt[j] = __shfl_sync(0xffffffffu, wl, (j0 + j) & 31);
                const bool ok = mine && j0 + j < cnt;
                v[j] = ok ? *(const float4 *)(part + (size_t)(s0 + j0 + j) * a.hd + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
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
    cudaError_t e = cudaFuncSetAttribute(attn_split_mma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(AttnSmem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_split_simt<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)simt_smem(128));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(attn_split_simt<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)simt_smem(128));
}

cudaError_t launch_attention(const Ctx &c, const AttnArgs &a, cudaStream_t s)
{
    const int g = a.n_q / a.n_kv, R = a.K * g;
    const bool tc = c.cfg.dtype == ORTHRUS_BF16 && a.hd == 128;
    const int rows_per = tc ? kAttnRowsMma : kAttnRowsSimt;
    const int rgroups = (R + rows_per - 1) / rows_per;
    // splits reachable by any sequence this context serves
    const int n_split_grid = (c.cfg.max_seq + a.split_tokens - 1) / a.split_tokens;
    dim3 grid(a.n_kv, a.B * rgroups, n_split_grid);
    c.launches += 2;
    cudaError_t e;
    if (tc)
        e = launch_k(attn_split_mma, grid, 256, sizeof(AttnSmem), s, a, n_split_grid);
    else if (c.cfg.dtype == ORTHRUS_BF16)
        e = launch_k(attn_split_simt<bf16>, grid, 128, simt_smem(a.hd), s, a, n_split_grid);
    else
        e = launch_k(attn_split_simt<float>, grid, 128, simt_smem(a.hd), s, a, n_split_grid);
    if (e != cudaSuccess) return e;
    const int rows = a.B * a.K * a.n_q;
    if (c.cfg.dtype == ORTHRUS_BF16) return launch_k(attn_combine<bf16>, (rows + 7) / 8, 256, 0, s, a);
    return launch_k(attn_combine<float>, (rows + 7) / 8, 256, 0, s, a);
}

}  // namespace orthrus
