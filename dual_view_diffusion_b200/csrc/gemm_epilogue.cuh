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

// What an epilogue can fetch before its accumulator is ready: the residual
// rows (RESID) and the per-row destinations and rotary frequencies of a
// head-sized QKV tile.  A warp-specialised kernel fills it while the tile's
// last weight chunks stream in, so only arithmetic and stores remain after.
struct QkvPre {
    int pos[kTileM];
    long long dst[kTileM];   // element offset of (row, dim 0); -1: skip the row
    double invf[64];
};
struct EpiPre {
    float resid[kTileM][kTilePad];
    QkvPre qkv;
};

// E >= 0 fixes the epilogue at compile time (each tensor-core kernel carries
// only its own epilogue's code); E < 0 dispatches on a.epi.
template <int E> __device__ __forceinline__ int epi_kind(const GemmArgs &a) { return E >= 0 ? E : a.epi; }

template <int E = -1>
__device__ __forceinline__ bool qkv_fast(const GemmArgs &a, int es)
{
    return epi_kind<E>(a) == EPI_QKV && es == 2 && a.hd == kTileN && (a.n_q * a.hd) % kTileN == 0;
}

// Q, K or V (0, 1, 2) and head of an n tile of a head-sized QKV projection
__device__ __forceinline__ void qkv_kind(const GemmArgs &a, int nt, int &kind, int &head)
{
    const int Nq = a.n_q * kTileN, Nk = a.n_kv * kTileN, n0 = nt * kTileN;
    kind = n0 < Nq ? 0 : (n0 < Nq + Nk ? 1 : 2);
    head = (n0 - (kind == 0 ? 0 : (kind == 1 ? Nq : Nq + Nk))) / kTileN;
}

__device__ inline void qkv_prepare(const GemmArgs &a, QkvPre &pre, int mt, int nt, int tid)
{
    int kind, head;
    qkv_kind(a, nt, kind, head);
    if (tid < kTileM) {
        const int row = mt * kTileM + tid;
        int pos = -1;
        long long dst = -1;
        if (row < a.M) {
            const int b = row / a.K, k = row % a.K;
            const int spos = a.pos0[b] + k;                              // cache slot
            pos = a.rope_pos ? a.pos0[b] + a.rope_pos[row] : spos;       // rotary position
            if (kind == 0) {
                dst = (long long)row * a.n_q * kTileN + head * kTileN;
            } else if (a.kv_to_cache) {
                const int pidx = spos / a.kv.page_size;
                int page = -1;
                if (spos >= 0 && pidx < a.kv.max_pages) {
                    page = a.kv.block_table[(size_t)a.bt_rows[b] * a.kv.max_pages + pidx];
                    if (page >= a.kv.num_pages) page = -1;
                }
                if (page < 0) {
                    raise_err(a.err, ORTHRUS_DEVERR_CAPACITY);
                } else {
                    const long long hh = ((long long)a.layer * a.kv.num_pages + page) * a.n_kv + head;
                    const int slot = spos % a.kv.page_size;
                    dst = kind == 1 ? (hh * a.kv.page_size + slot) * kTileN : hh * kTileN * a.kv.page_size + slot;
                }
            } else {
                const long long hh = ((long long)a.layer * a.bmax + b) * a.n_kv + head;
                dst = kind == 1 ? (hh * a.kp + k) * kTileN : hh * kTileN * a.kp + k;
            }
        }
        pre.pos[tid] = pos;
        pre.dst[tid] = dst;
    } else if (tid >= 64) {
        pre.invf[tid - 64] = a.rope_invf[tid - 64];
    }
}

template <class T, int E = -1>
__device__ void epilogue_prepare(const GemmArgs &a, EpiPre &pre, int mt, int nt, int tid)
{
    if (epi_kind<E>(a) == EPI_RESID && (a.N & 3) == 0) {
        float4 v[kEpiVec];
#pragma unroll
        for (int j = 0; j < kEpiVec; ++j) {
            const int c = tid + j * kEpiThreads, m = c >> 5, n = nt * kTileN + (c & 31) * 4, row = mt * kTileM + m;
            if (row < a.M && n < a.N) v[j] = __ldcg((const float4 *)&a.resid[(size_t)row * a.N + n]);
        }
#pragma unroll
        for (int j = 0; j < kEpiVec; ++j) {
            const int c = tid + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
            *(float4 *)&pre.resid[m][c4] = v[j];
        }
    } else if (qkv_fast<E>(a, sizeof(T))) {
        qkv_prepare(a, pre.qkv, mt, nt, tid);
    }
}

// pre: filled by epilogue_prepare for this tile (and made visible with a
// barrier), or null to fetch everything here.
// bf16 outputs: the same reduction, then the MUFU sine / cosine (absolute
// error ~4e-7 on [-pi, pi], far inside bf16 rounding) in a few instructions
__device__ __forceinline__ void rope_sincos_fast(int pos, double inv_freq, float &s, float &c)
{
    const double ang = (double)pos * inv_freq;
    const double k = rint(ang * 0.15915494309189535);
    const float r = (float)fma(-k, 6.283185307179586, ang);
    s = __sinf(r);
    c = __cosf(r);
}

template <class T, class Sync, int E = -1>
__device__ void epilogue(const GemmArgs &a, float (*tile)[kTilePad], int mt, int nt, int n_nt, int tid, Sync sync,
                         EpiPre *pre = nullptr)
{
    const int epi = epi_kind<E>(a);
    if (epi == EPI_RESID) {
        if ((a.N & 3) == 0) {
            float4 v[kEpiVec];
            bool ok[kEpiVec];
#pragma unroll
            for (int j = 0; j < kEpiVec; ++j) {
                const int c = tid + j * kEpiThreads, m = c >> 5, n = nt * kTileN + (c & 31) * 4, row = mt * kTileM + m;
                ok[j] = row < a.M && n < a.N;
                if (ok[j]) v[j] = pre ? *(const float4 *)&pre->resid[m][(c & 31) * 4]
                                      : *(const float4 *)&a.resid[(size_t)row * a.N + n];
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
    } else if (epi == EPI_SWIGLU && sizeof(T) == 2 && (a.N & 7) == 0) {
        // 8 outputs per item: gate / up float4 pairs -> one 16-byte store
#pragma unroll
        for (int j = 0; j < kTileM * 8 / kEpiThreads; ++j) {
            const int item = tid + j * kEpiThreads, m = item >> 3, i0 = (item & 7) * 8;
            const int row = mt * kTileM + m, f = nt * 64 + i0;
            if (row >= a.M || f >= a.N) continue;
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const float g0 = tile[m][i0 + e], g1 = tile[m][i0 + e + 1];
                const float u0 = tile[m][64 + i0 + e], u1 = tile[m][64 + i0 + e + 1];
                // bf16 output: the MUFU exponential and an approximate divide
                // are well inside its rounding, and keep this path short
                const float s0 = __fdividef(g0, 1.0f + __expf(-g0)), s1 = __fdividef(g1, 1.0f + __expf(-g1));
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(s0 * u0, s1 * u1);
                o[e / 2] = *(const uint32_t *)&h2;
            }
            __stcg((uint4 *)((bf16 *)a.act + (size_t)row * a.N + f), make_uint4(o[0], o[1], o[2], o[3]));
        }
    } else if (epi == EPI_SWIGLU) {
#pragma unroll 4
        for (int idx = tid; idx < kTileM * 64; idx += kEpiThreads) {
            const int m = idx >> 6, i = idx & 63, row = mt * kTileM + m, f = nt * 64 + i;
            if (row < a.M && f < a.N) {
                const float g = tile[m][i], u = tile[m][64 + i];
                const float s = g / (1.0f + expf(-g));
                ((T *)a.act)[(size_t)row * a.N + f] = from_f<T>(s * u);
            }
        }
    } else if (qkv_fast<E>(a, sizeof(T))) {
        // one tile = one head of Q, K or V (head_dim 128).  Per-row
        // destinations are resolved once; Q/K rows are rotated 8 dimension
        // pairs at a time and written with 16-byte stores; V goes to its
        // transposed layout 8 tokens at a time where they are contiguous.
        QkvPre *qp = pre ? &pre->qkv : nullptr;
        if (!qp) {
            __shared__ QkvPre s_qkv;
            qkv_prepare(a, s_qkv, mt, nt, tid);
            sync();
            qp = &s_qkv;
        }
        int kind, head;
        qkv_kind(a, nt, kind, head);
        const int vstride = a.kv_to_cache ? a.kv.page_size : a.kp;
        const int *s_pos = qp->pos;
        const long long *s_dst = qp->dst;
        const double *s_invf = qp->invf;
        if (kind < 2) {
            bf16 *base = (bf16 *)(kind == 0 ? a.q_out : (a.kv_to_cache ? a.kv.k_pages : a.k_blk));
#pragma unroll
            for (int j = 0; j < kTileM * 8 / kEpiThreads; ++j) {
                const int item = tid + j * kEpiThreads, m = item >> 3, i0 = (item & 7) * 8;
                const long long dst = s_dst[m];
                if (dst < 0) continue;
                const int pos = s_pos[m];
                uint32_t lo[4], hi[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float r[4];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        float sn, cs;
                        rope_sincos_fast(pos, s_invf[i0 + e + u], sn, cs);
                        const float x0 = tile[m][i0 + e + u], x1 = tile[m][64 + i0 + e + u];
                        r[u] = x0 * cs - x1 * sn;
                        r[2 + u] = x1 * cs + x0 * sn;
                    }
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(r[0], r[1]), h2 = __floats2bfloat162_rn(r[2], r[3]);
                    lo[e / 2] = *(const uint32_t *)&l2;
                    hi[e / 2] = *(const uint32_t *)&h2;
                }
                __stcg((uint4 *)(base + dst + i0), make_uint4(lo[0], lo[1], lo[2], lo[3]));
                __stcg((uint4 *)(base + dst + 64 + i0), make_uint4(hi[0], hi[1], hi[2], hi[3]));
            }
        } else {
            bf16 *base = (bf16 *)(a.kv_to_cache ? a.kv.v_pages : a.v_blk);
            // every 8-row group's slots consecutive and 16-byte aligned (a
            // block starting at a multiple of 8, inside one page): one 16-byte
            // store per (group, dim); otherwise (a decode block at any
            // position) each warp writes 32 consecutive slots of one dim row
            // per store instruction, lane = row
            bool vec = (vstride & 7) == 0;
#pragma unroll
            for (int tg = 0; tg < kTileM / 8; ++tg) {
                const long long d0 = s_dst[tg * 8];
                vec = vec && d0 >= 0 && (d0 & 7) == 0;
#pragma unroll
                for (int e = 1; e < 8; ++e) vec = vec && s_dst[tg * 8 + e] == d0 + e;
            }
            if (vec) {
#pragma unroll
                for (int j = 0; j < kTileM * kTileN / 8 / kEpiThreads; ++j) {
                    const int item = tid + j * kEpiThreads, tg = item & 3, d = item >> 2, m0 = tg * 8;
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(tile[m0 + e][d], tile[m0 + e + 1][d]);
                        o[e / 2] = *(const uint32_t *)&h2;
                    }
                    __stcg((uint4 *)(base + s_dst[m0] + (long long)d * vstride), make_uint4(o[0], o[1], o[2], o[3]));
                }
            } else {
                const int m = tid & 31, w = tid >> 5;
                const long long de = s_dst[m];
#pragma unroll 8
                for (int dd = 0; dd < kTileN / (kEpiThreads / 32); ++dd) {
                    const int d = w * (kTileN / (kEpiThreads / 32)) + dd;
                    if (de >= 0) base[de + (long long)d * vstride] = __float2bfloat16_rn(tile[m][d]);
                }
            }
        }
    } else if (epi == EPI_QKV) {
        __shared__ int s_pos[kTileM], s_page[kTileM], s_slot[kTileM];
        __shared__ double s_invf[64];
        const int half = a.hd / 2, Nq = a.n_q * a.hd, Nk = a.n_kv * a.hd;
        if (tid < kTileM) {
            const int row = mt * kTileM + tid;
            int pos = -1, page = -1, spos = -1;
            if (row < a.M) {
                const int b = row / a.K, k = row % a.K;
                spos = a.pos0[b] + k;                                  // cache slot
                pos = a.rope_pos ? a.pos0[b] + a.rope_pos[row] : spos; // rotary position
                if (a.kv_to_cache) {
                    const int pidx = spos / a.kv.page_size;
                    if (spos >= 0 && pidx < a.kv.max_pages) {
                        page = a.kv.block_table[(size_t)a.bt_rows[b] * a.kv.max_pages + pidx];
                        if (page >= a.kv.num_pages) page = -1;
                    }
                    if (page < 0 && nt * kTileN + kTileN > Nq) raise_err(a.err, ORTHRUS_DEVERR_CAPACITY);
                }
            }
            s_pos[tid] = pos;
            s_page[tid] = page;
            s_slot[tid] = spos;
        } else if (tid >= 64 && tid - 64 < half) {
            s_invf[tid - 64] = a.rope_invf[tid - 64];
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
                const int slot = s_slot[m] % a.kv.page_size;
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
    } else if (epi == EPI_LMHEAD) {
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
                        const uint32_t pu = a.lm_mode == 2 ? PURPOSE_AR : (PURPOSE_DRAFT | ((uint32_t)a.draft_pass << 8));
                        best_merge(gb, Best{zv[j] * a.inv_temp + gumbel(a.seed, step, rr, (uint32_t)v, pu), v, zv[j]});
                    }
                }
            }
            zb = warp_best(zb);
            if (sampling) gb = warp_best(gb);
            // sum of exp((z - max) / T), and for draft rows the same weights
            // times z (the mean logit of the row's distribution, for its
            // entropy)
            float s = 0.f, ez = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (nt * kTileN + lane * 4 + j < a.N) {
                    const float ex = expf((zv[j] - zb.v) * it);
                    s += ex;
                    ez = fmaf(ex, zv[j], ez);
                }
            s = warp_sum(s);
            if (a.lm_mode == 1) ez = warp_sum(ez);
            if (a.topw > 0) {   // this tile's topw best (z, id), best first, ties to the lowest id
                float tv[4];
                int ti[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int v = nt * kTileN + lane * 4 + j;
                    tv[j] = v < a.N ? zv[j] : -INFINITY;
                    ti[j] = v < a.N ? v : INT_MAX;
                }
#pragma unroll
                for (int i = 0; i < 3; ++i)   // a lane's four, sorted
#pragma unroll
                    for (int j = 0; j < 3 - i; ++j)
                        if (tw_better(tv[j + 1], ti[j + 1], tv[j], ti[j])) {
                            const float x = tv[j]; tv[j] = tv[j + 1]; tv[j + 1] = x;
                            const int y = ti[j]; ti[j] = ti[j + 1]; ti[j + 1] = y;
                        }
                TopRec *out = a.top + ((size_t)row * n_nt + nt) * kTopWMax;
                for (int r = 0; r < a.topw; ++r) {
                    float bv = tv[0];
                    int bi = ti[0];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                        if (tw_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
                    }
                    if (ti[0] == bi && bi != INT_MAX) {   // the owning lane gives up its head
                        tv[0] = tv[1]; tv[1] = tv[2]; tv[2] = tv[3]; tv[3] = -INFINITY;
                        ti[0] = ti[1]; ti[1] = ti[2]; ti[2] = ti[3]; ti[3] = INT_MAX;
                    }
                    if (lane == 0) out[r] = TopRec{bv, bi};
                }
            }
            // the id's logit lives in exactly one lane (or none)
            const unsigned has = __ballot_sync(0xffffffffu, !isnan(zid));
            if (has) zid = __shfl_sync(0xffffffffu, zid, __ffs(has) - 1);
            if (lane == 0) {
                LmPart pr;
                pr.zmax = zb.v; pr.zsum = s; pr.zarg = zb.i;
                pr.gbest = gb.v; pr.garg = gb.i; pr.gz = gb.z; pr.zid = zid; pr.zez = ez;
                a.lm[(size_t)row * n_nt + nt] = pr;
            }
        }
    } else if (epi == EPI_LOGITS) {
#pragma unroll 4
        for (int idx = tid; idx < kTileM * kTileN; idx += kEpiThreads) {
            const int m = idx >> 7, nl = idx & 127, row = mt * kTileM + m, n = nt * kTileN + nl;
            if (row < a.M && n < a.N) a.logits[(size_t)row * a.N + n] = tile[m][nl];
        }
    } else if (epi == EPI_KL) {
        // rows come in pairs (2i: AR view, 2i+1: diffusion view of the same
        // position, paper notes §3.3); per pair and vocabulary tile: each
        // view's max and sum of exponentials, and the AR-weighted sum of
        // z_AR - z_diff (the forward-KL numerator)
        const int lane = tid & 31, warp = tid >> 5;
        for (int pl = 0; pl < kTileM / 8; ++pl) {
            const int mp = warp * (kTileM / 8) + pl;        // pair index within tile
            const int m = 2 * mp, row = mt * kTileM + m;
            if (row >= a.M) break;
            float za[4], zd[4];
            float ma = -INFINITY, md = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int nl = lane * 4 + j;
                const bool ok = nt * kTileN + nl < a.N;
                za[j] = ok ? tile[m][nl] : -INFINITY;
                zd[j] = ok ? tile[m + 1][nl] : -INFINITY;
                ma = fmaxf(ma, za[j]);
                md = fmaxf(md, zd[j]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
                md = fmaxf(md, __shfl_xor_sync(0xffffffffu, md, o));
            }
            float sa = 0.f, ta = 0.f, sd = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (nt * kTileN + lane * 4 + j >= a.N) continue;
                const float ea = expf(za[j] - ma);
                sa += ea;
                ta = fmaf(ea, za[j] - zd[j], ta);
                sd += expf(zd[j] - md);
            }
            sa = warp_sum(sa);
            ta = warp_sum(ta);
            sd = warp_sum(sd);
            if (lane == 0) {
                KlPart pr{};
                pr.ma = ma; pr.sa = sa; pr.ta = ta; pr.md = md; pr.sd = sd;
                a.kl[(size_t)(row / 2) * n_nt + nt] = pr;
            }
        }
    } else if (epi == EPI_RESAMPLE) {
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

}  // namespace orthrus
