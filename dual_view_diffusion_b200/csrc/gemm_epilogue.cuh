// Epilogues of the projection GEMMs, shared by the tensor-core and SIMT
// mainloops: QKV with RoPE and the K/V scatter, residual add, SiLU*up, the
// LM-head reduction (max, lowest argmax, sum of exponentials, Gumbel winner,
// logit at a given id), the residual draw of sampled consensus, and a plain
// logits dump.  Each works on the finished fp32 tile tile[token][feature] in
// shared memory with kEpiThreads threads.
//
// Every loop that touches global memory is unrolled with all of its loads
// issued before their first use, and per-row metadata (positions, cache
// pages, requested ids) is staged in shared memory once per tile: a loop of
// dependent global round trips costs ~0.4 us per iteration at L2 latency,
// which would dwarf the tile's share of the weight stream.
#pragma once
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace orthrus {

constexpr int kTilePad = kTileN + 4;
constexpr int kEpiThreads = 128;
constexpr int kEpiVec = kTileM * kTileN / 4 / kEpiThreads;   // float4 chunks per thread (8)

struct SyncBlock {
    __device__ void operator()() const { __syncthreads(); }
};
// named barrier 1 over the four epilogue warps of a warp-specialised kernel
struct SyncEpilogue {
    __device__ void operator()() const { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }
};

struct Best {
    float v;
    int i;
    float z;
};

__device__ __forceinline__ void best_merge(Best &a, const Best &b)
{
    if (b.v > a.v || (b.v == a.v && b.i < a.i)) a = b;
}

__device__ __forceinline__ Best warp_best(Best b)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        Best c;
        c.v = __shfl_xor_sync(0xffffffffu, b.v, o);
        c.i = __shfl_xor_sync(0xffffffffu, b.i, o);
        c.z = __shfl_xor_sync(0xffffffffu, b.z, o);
        best_merge(b, c);
    }
    return b;
}

// Rotation angle pos * theta^(-2i/hd) reduced to [-pi, pi] in fp64 (the
// product reaches ~1e5 rad at long context), then fp32 sin/cos.
__device__ __forceinline__ void rope_sincos(int pos, double inv_freq, float &s, float &c)
{
    const double ang = (double)pos * inv_freq;
    const double k = rint(ang * 0.15915494309189535);        // 1 / (2 pi)
    const double r = fma(-k, 6.283185307179586, ang);
    sincosf((float)r, &s, &c);
}

template <class T, class Sync>
__device__ void epilogue(const GemmArgs &a, float (*tile)[kTilePad], int mt, int nt, int n_nt, int tid, Sync sync)
{
    if (a.epi == EPI_RESID) {
        if ((a.N & 3) == 0) {
            float4 v[kEpiVec];
            bool ok[kEpiVec];
#pragma unroll
            for (int j = 0; j < kEpiVec; ++j) {
                const int c = tid + j * kEpiThreads, m = c >> 5, n = nt * kTileN + (c & 31) * 4, row = mt * kTileM + m;
                ok[j] = row < a.M && n < a.N;
                if (ok[j]) v[j] = *(const float4 *)&a.resid[(size_t)row * a.N + n];
            }
#pragma unroll
            for (int j = 0; j < kEpiVec; ++j) {
                const int c = tid + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
                if (!ok[j]) continue;
                const int row = mt * kTileM + m, n = nt * kTileN + c4;
                float4 t = v[j];
                t.x += tile[m][c4]; t.y += tile[m][c4 + 1]; t.z += tile[m][c4 + 2]; t.w += tile[m][c4 + 3];
                *(float4 *)&a.resid[(size_t)row * a.N + n] = t;
            }
        } else {
            for (int idx = tid; idx < kTileM * kTileN; idx += kEpiThreads) {
                const int m = idx >> 7, nl = idx & 127, row = mt * kTileM + m, n = nt * kTileN + nl;
                if (row < a.M && n < a.N) a.resid[(size_t)row * a.N + n] += tile[m][nl];
            }
        }
    } else if (a.epi == EPI_SWIGLU) {
#pragma unroll 4
        for (int idx = tid; idx < kTileM * 64; idx += kEpiThreads) {
            const int m = idx >> 6, i = idx & 63, row = mt * kTileM + m, f = nt * 64 + i;
            if (row < a.M && f < a.N) {
                const float g = tile[m][i], u = tile[m][64 + i];
                const float s = g / (1.0f + expf(-g));
                ((T *)a.act)[(size_t)row * a.N + f] = from_f<T>(s * u);
            }
        }
    } else if (a.epi == EPI_QKV) {
        __shared__ int s_pos[kTileM], s_page[kTileM];
        __shared__ double s_invf[64];
        const int half = a.hd / 2, Nq = a.n_q * a.hd, Nk = a.n_kv * a.hd;
        if (tid < kTileM) {
            const int row = mt * kTileM + tid;
            int pos = -1, page = -1;
            if (row < a.M) {
                const int b = row / a.K, k = row % a.K;
                pos = a.pos0[b] + k;
                if (a.kv_to_cache) {
                    const int pidx = pos / a.kv.page_size;
                    if (pos >= 0 && pidx < a.kv.max_pages) {
                        page = a.kv.block_table[(size_t)a.bt_rows[b] * a.kv.max_pages + pidx];
                        if (page >= a.kv.num_pages) page = -1;
                    }
                    if (page < 0 && nt * kTileN + kTileN > Nq) raise_err(a.err, ORTHRUS_DEVERR_CAPACITY);
                }
            }
            s_pos[tid] = pos;
            s_page[tid] = page;
        } else if (tid >= 64 && tid - 64 < half) {
            s_invf[tid - 64] = pow(a.rope_theta, -2.0 * (tid - 64) / a.hd);
        }
        sync();
#pragma unroll 4
        for (int idx = tid; idx < kTileM * 64; idx += kEpiThreads) {
            const int m = idx >> 6, p = idx & 63;
            const int nl = (p / half) * a.hd + (p % half), i = p % half;
            const int n = nt * kTileN + nl, row = mt * kTileM + m;
            if (row >= a.M || n >= Nq + 2 * Nk) continue;
            float x0 = tile[m][nl], x1 = tile[m][nl + half];
            const int pos = s_pos[m];
            if (n < Nq + Nk) {   // rotary embedding on Q and K (rotate-half pairs)
                float sn, cs;
                rope_sincos(pos, s_invf[i], sn, cs);
                const float r0 = x0 * cs - x1 * sn, r1 = x1 * cs + x0 * sn;
                x0 = r0; x1 = r1;
            }
            if (n < Nq) {
                T *q = (T *)a.q_out + (size_t)row * Nq;
                q[n] = from_f<T>(x0);
                q[n + half] = from_f<T>(x1);
                continue;
            }
            const bool is_k = n < Nq + Nk;
            const int nn = n - Nq - (is_k ? 0 : Nk), kvh = nn / a.hd, d = nn % a.hd;
            // K rows are [slot][dim]; V is stored transposed, [dim][slot]
            size_t base, step;
            if (a.kv_to_cache) {
                const int page = s_page[m];
                if (page < 0) continue;
                const size_t head = ((size_t)a.layer * a.kv.num_pages + page) * a.n_kv + kvh;
                const int slot = pos % a.kv.page_size;
                if (is_k) { base = (head * a.kv.page_size + slot) * a.hd + d; step = 1; }
                else { base = (head * a.hd + d) * a.kv.page_size + slot; step = a.kv.page_size; }
            } else {
                const int b = row / a.K, k = row % a.K;
                const size_t head = ((size_t)a.layer * a.bmax + b) * a.n_kv + kvh;
                if (is_k) { base = (head * a.kp + k) * a.hd + d; step = 1; }
                else { base = (head * a.hd + d) * a.kp + k; step = a.kp; }
            }
            T *dst = (T *)(is_k ? (a.kv_to_cache ? a.kv.k_pages : a.k_blk) : (a.kv_to_cache ? a.kv.v_pages : a.v_blk));
            dst[base] = from_f<T>(x0);
            dst[base + (size_t)half * step] = from_f<T>(x1);
        }
    } else if (a.epi == EPI_LMHEAD) {
        __shared__ int s_given[kTileM];
        __shared__ uint32_t s_step;
        if (tid < kTileM) {
            const int row = mt * kTileM + tid;
            s_given[tid] = (a.given && row < a.M) ? a.given[row] : -1;
        }
        if (tid == 32) s_step = a.step ? (uint32_t)*a.step : 0u;
        sync();
        const int lane = tid & 31, warp = tid >> 5;
        const bool sampling = a.lm_mode != 0 && a.inv_temp > 0.f;
        const float it = a.inv_temp > 0.f ? a.inv_temp : 1.0f;
        const uint32_t step = s_step;
        for (int ml = 0; ml < kTileM / 4; ++ml) {
            const int m = warp * (kTileM / 4) + ml, row = mt * kTileM + m;
            if (row >= a.M) break;
            const int b = row / a.K, k = row % a.K;
            const int given = s_given[m];
            Best zb{-INFINITY, 0x7fffffff, 0.f}, gb{-INFINITY, 0x7fffffff, 0.f};
            float zid = NAN;
            float zv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int nl = lane * 4 + j, v = nt * kTileN + nl;
                zv[j] = v < a.N ? tile[m][nl] : -INFINITY;
                if (v < a.N) {
                    best_merge(zb, Best{zv[j], v, zv[j]});
                    if (v == given) zid = zv[j];
                    if (sampling) {
                        const uint32_t rr = a.lm_mode == 2 ? rng_row(b, 0) : rng_row(b, k);
                        const uint32_t pu = a.lm_mode == 2 ? PURPOSE_AR : PURPOSE_DRAFT;
                        best_merge(gb, Best{zv[j] * a.inv_temp + gumbel(a.seed, step, rr, (uint32_t)v, pu), v, zv[j]});
                    }
                }
            }
            zb = warp_best(zb);
            if (sampling) gb = warp_best(gb);
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (nt * kTileN + lane * 4 + j < a.N) s += expf((zv[j] - zb.v) * it);
            s = warp_sum(s);
            // the id's logit lives in exactly one lane (or none)
            const unsigned has = __ballot_sync(0xffffffffu, !isnan(zid));
            if (has) zid = __shfl_sync(0xffffffffu, zid, __ffs(has) - 1);
            if (lane == 0) {
                LmPart pr;
                pr.zmax = zb.v; pr.zsum = s; pr.zarg = zb.i;
                pr.gbest = gb.v; pr.garg = gb.i; pr.gz = gb.z; pr.zid = zid; pr.pad = 0;
                a.lm[(size_t)row * n_nt + nt] = pr;
            }
        }
    } else if (a.epi == EPI_LOGITS) {
#pragma unroll 4
        for (int idx = tid; idx < kTileM * kTileN; idx += kEpiThreads) {
            const int m = idx >> 7, nl = idx & 127, row = mt * kTileM + m, n = nt * kTileN + nl;
            if (row < a.M && n < a.N) a.logits[(size_t)row * a.N + n] = tile[m][nl];
        }
    } else if (a.epi == EPI_RESAMPLE) {
        // rows come in pairs (2b: AR view at the rejected row, 2b+1: diffusion
        // view at the same row); score = log max(0, p - q) + Gumbel
        __shared__ int s_j[kTileM / 2];
        __shared__ float s_lp[kTileM / 2], s_lq[kTileM / 2];
        __shared__ uint32_t s_step2;
        if (tid < kTileM / 2) {
            const int row = mt * kTileM + 2 * tid, b = row / 2;
            int j = -1;
            if (row < a.M) j = a.rej_row[b];
            s_j[tid] = j;
            s_lp[tid] = j >= 0 ? a.lse_p[b * a.K + j] : 0.f;
            s_lq[tid] = j >= 0 ? a.lse_q[b * a.K + j] : 0.f;
        }
        if (tid == 32) s_step2 = a.step ? (uint32_t)*a.step : 0u;
        sync();
        const int lane = tid & 31, warp = tid >> 5;
        const uint32_t step = s_step2;
        for (int pl = 0; pl < kTileM / 8; ++pl) {
            const int mp = warp * (kTileM / 8) + pl;        // pair index within tile
            const int m = 2 * mp, row = mt * kTileM + m, b = row / 2;
            if (row >= a.M) break;
            const int j = s_j[mp];
            if (j < 0) continue;
            const float lp = s_lp[mp], lq = s_lq[mp];
            Best gb{-INFINITY, 0x7fffffff, 0.f};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int nl = lane * 4 + jj, v = nt * kTileN + nl;
                if (v < a.N) {
                    const float r = expf(tile[m][nl] * a.inv_temp - lp) - expf(tile[m + 1][nl] * a.inv_temp - lq);
                    if (r > 0.f)
                        best_merge(gb, Best{logf(r) + gumbel(a.seed, step, rng_row(b, j), (uint32_t)v, PURPOSE_RESIDUAL),
                                            v, tile[m][nl]});
                }
            }
            gb = warp_best(gb);
            if (lane == 0) {
                LmPart pr{};
                pr.gbest = gb.v; pr.garg = gb.i; pr.gz = gb.z;
                a.lm[(size_t)row * n_nt + nt] = pr;
            }
        }
    }
}

// Split-K: publish this unit's partial tile; the CTA that completes the
// tile's set of segments sums them in segment order (so the sum never
// depends on arrival order) and runs the epilogue.  `sync` is a barrier over
// the kEpiThreads epilogue threads.  Returns true when this CTA must run the
// epilogue.
template <class Sync>
__device__ bool split_k_gather(const GemmArgs &a, float (*tile)[kTilePad], int t, int seg, int tid, int *s_last,
                               Sync sync)
{
    const int S = a.splits;
    if (S == 1) return true;
    float *slot = a.part + ((size_t)t * S + seg) * (kTileM * kTileN);
#pragma unroll
    for (int j = 0; j < kEpiVec; ++j) {
        const int c = tid + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
        __stcg((float4 *)(slot + m * kTileN + c4), *(float4 *)&tile[m][c4]);
    }
    __threadfence();
    sync();
    if (tid == 0) *s_last = (atomicAdd(&a.ticket[t], 1) == S - 1);
    sync();
    if (!*s_last) return false;
    __threadfence();
    const float *base = a.part + (size_t)t * S * (kTileM * kTileN);
    float4 acc[kEpiVec];
#pragma unroll
    for (int j = 0; j < kEpiVec; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < S; ++s) {
        float4 v[kEpiVec];
#pragma unroll
        for (int j = 0; j < kEpiVec; ++j) {
            const int c = tid + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
            v[j] = __ldcg((const float4 *)(base + (size_t)s * kTileM * kTileN + m * kTileN + c4));
        }
#pragma unroll
        for (int j = 0; j < kEpiVec; ++j) {
            acc[j].x += v[j].x; acc[j].y += v[j].y; acc[j].z += v[j].z; acc[j].w += v[j].w;
        }
    }
#pragma unroll
    for (int j = 0; j < kEpiVec; ++j) {
        const int c = tid + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
        *(float4 *)&tile[m][c4] = acc[j];
    }
    if (tid == 0) a.ticket[t] = 0;
    sync();
    return true;
}

}  // namespace orthrus
