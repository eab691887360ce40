// Weight-streaming projections of the dual-view decoder with fused epilogues.
//
// Y[M][N] = X[M][Kd] . W^T for the K-row block of a draft or verify
// forward (paper notes §2.1: both views share every matrix except
// W_Q/W_K/W_V).  At decode sizes M = batch*K is small and the work is bound
// by streaming W from HBM, so the kernel is organised around the weights:
//
//   * persistent CTAs walk work units (m tile, n tile, k segment); each unit
//     streams a 128-row x (Kd/S) slab of W through a multi-stage cp.async
//     ring, the activations (32 rows) ride along;
//   * the k split S is a function of the matrix shape only, never of M, and
//     partial tiles are summed in segment order by whichever CTA arrives
//     last, so a token row gets bit-identical results whatever block, batch
//     or row slot it sits in (the property that makes greedy Orthrus equal
//     plain AR on the GPU, paper notes §4.2);
//   * epilogues run on the finished fp32 tile in shared memory: QKV with
//     RoPE and the K/V scatter into the paged cache or the transient
//     diffusion buffer, residual add, SiLU*up, and the LM-head reduction
//     (max, argmax, log-sum-exp terms, Gumbel-max sampling) so logits never
//     reach HBM.
//
// bf16 uses tensor cores (mma.sync m16n8k16, fp32 accumulate); fp32 uses a
// SIMT loop with the same tiling, scheduling and epilogues.
#include <math.h>
#include <stdlib.h>

#include "common.cuh"
#include "gemm_epilogue.cuh"
#include "internal.h"

namespace orthrus {

constexpr int kStages = 6;
constexpr int kGemmThreads = 128;

struct GemmShape {
    int n_mt, n_nt;
};

template <class T>
__device__ __forceinline__ const T *weight_row(const GemmArgs &a, int nt, int r)
{
    if (a.epi == EPI_SWIGLU) {
        const int half = r >> 6, f = nt * 64 + (r & 63);
        if (f >= a.wrows[half]) return nullptr;
        return (const T *)a.w[half] + (size_t)f * a.Kd;
    }
    int n = nt * kTileN + r;
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        if (n < a.wrows[s]) return (const T *)a.w[s] + (size_t)n * a.Kd;
        n -= a.wrows[s];
    }
    return nullptr;
}

// ---------------------------------------------------------------- mainloops
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};\n"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory image of a 64-element (128-byte) row: its eight 16-byte
// chunks are XOR-swizzled by the row index so ldmatrix is conflict-free.
__device__ __forceinline__ int swz(int row, int chunk) { return row * 64 + ((chunk ^ (row & 7)) << 3); }

struct MmaSmem {
    bf16 w[kStages][kTileN * kTileK];
    bf16 x[kStages][kTileM * kTileK];
};

__device__ void mainloop_mma(const GemmArgs &a, int mt, int nt, int c0, int c1, MmaSmem &sm,
                             float (*tile)[kTilePad])
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bf16 *wp[8];
    const bf16 *xp[2];
#pragma unroll
    for (int i = 0; i < 8; ++i) wp[i] = weight_row<bf16>(a, nt, (tid >> 3) + 16 * i);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int row = mt * kTileM + (tid >> 3) + 16 * i;
        xp[i] = row < a.M ? (const bf16 *)a.x + (size_t)row * a.Kd : nullptr;
    }
    const int ch = tid & 7;
    const bf16 *wbase = (const bf16 *)a.w[0];
    const bf16 *xbase = (const bf16 *)a.x;

    auto load = [&](int stage, int c) {
        const uint32_t sw = smem_u32(sm.w[stage]), sx = smem_u32(sm.x[stage]);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int row = (tid >> 3) + 16 * i;
            const bf16 *src = wp[i] ? wp[i] + (size_t)c * kTileK + ch * 8 : wbase;
            cp_async16(sw + 2 * swz(row, ch), src, wp[i] ? 16 : 0);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int row = (tid >> 3) + 16 * i;
            const bf16 *src = xp[i] ? xp[i] + (size_t)c * kTileK + ch * 8 : xbase;
            cp_async16(sx + 2 * swz(row, ch), src, xp[i] ? 16 : 0);
        }
    };

    float acc[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[i][j][k] = 0.f;

    const int n = c1 - c0;
#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < n) load(s, c0 + s);
        cp_async_commit();
    }
    for (int it = 0; it < n; ++it) {
        cp_async_wait<kStages - 2>();
        __syncthreads();
        const int st = it % kStages;
        {
            const int nx = it + kStages - 1;
            if (nx < n) load(nx % kStages, c0 + nx);
            cp_async_commit();
        }
        const uint32_t sw = smem_u32(sm.w[st]), sx = smem_u32(sm.x[st]);
#pragma unroll
        for (int ks = 0; ks < kTileK / 16; ++ks) {
            uint32_t af[2][4], bfr[4][2];
#pragma unroll
            for (int m2 = 0; m2 < 2; ++m2) {
                const int row = warp * 32 + m2 * 16 + (lane & 15);
                ldsm_x4(sw + 2 * swz(row, ks * 2 + (lane >> 4)), af[m2][0], af[m2][1], af[m2][2], af[m2][3]);
            }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                const int mi = lane >> 3;
                const int tok = (2 * np + (mi >> 1)) * 8 + (lane & 7);
                ldsm_x4(sx + 2 * swz(tok, ks * 2 + (mi & 1)), bfr[2 * np][0], bfr[2 * np][1], bfr[2 * np + 1][0],
                        bfr[2 * np + 1][1]);
            }
#pragma unroll
            for (int m2 = 0; m2 < 2; ++m2)
#pragma unroll
                for (int j = 0; j < 4; ++j) mma_bf16(acc[m2][j], af[m2], bfr[j][0], bfr[j][1]);
        }
    }
    cp_async_wait<0>();
    __syncthreads();
#pragma unroll
    for (int m2 = 0; m2 < 2; ++m2)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int f = warp * 32 + m2 * 16 + (lane >> 2) + (i >= 2 ? 8 : 0);
                const int m = j * 8 + (lane & 3) * 2 + (i & 1);
                tile[m][f] = acc[m2][j][i];
            }
}

// SIMT mainloop: thread r owns output feature r of the tile for all 32 rows.
template <class T>
__device__ void mainloop_simt(const GemmArgs &a, int mt, int nt, int k0, int k1, float *xs,
                              float (*tile)[kTilePad])
{
    const int tid = threadIdx.x;
    const T *w = weight_row<T>(a, nt, tid);
    float acc[kTileM];
#pragma unroll
    for (int m = 0; m < kTileM; ++m) acc[m] = 0.f;
    for (int kc = k0; kc < k1; kc += kTileK) {
        const int len = min(kTileK, k1 - kc);
        __syncthreads();
        for (int idx = tid; idx < kTileM * kTileK; idx += kGemmThreads) {
            const int m = idx / kTileK, kk = idx % kTileK, row = mt * kTileM + m;
            xs[idx] = (row < a.M && kk < len) ? to_f<T>(((const T *)a.x)[(size_t)row * a.Kd + kc + kk]) : 0.f;
        }
        __syncthreads();
        if (w) {
            for (int kk = 0; kk < len; ++kk) {
                const float wv = to_f<T>(w[kc + kk]);
#pragma unroll
                for (int m = 0; m < kTileM; ++m) acc[m] = fmaf(xs[m * kTileK + kk], wv, acc[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < kTileM; ++m) tile[m][tid] = acc[m];
}

// ---------------------------------------------------------------- kernel
// One-dimensional grid of persistent CTAs walking (m tile, n tile, segment)
// units in order.
template <class T, bool TC>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(GemmArgs a, int n_mt, int n_nt)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float(*tile)[kTilePad] = (float(*)[kTilePad])smem_raw;
    unsigned char *pipe = smem_raw + sizeof(float) * kTileM * kTilePad;
    __shared__ int s_last;
    if (a.epi == EPI_RESAMPLE && *a.any_flag == 0) return;

    const int S = a.splits;
    const int units = n_mt * n_nt * S;
    const int chunks = (a.Kd + kTileK - 1) / kTileK;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int seg = u % S, t = u / S, mt = t % n_mt, nt = t / n_mt;
        const int c0 = (int)((long)seg * chunks / S), c1 = (int)((long)(seg + 1) * chunks / S);
        if constexpr (TC) {
            mainloop_mma(a, mt, nt, c0, c1, *(MmaSmem *)pipe, tile);
        } else {
            mainloop_simt<T>(a, mt, nt, c0 * kTileK, min(c1 * kTileK, a.Kd), (float *)pipe, tile);
        }
        __syncthreads();
        if (!split_k_gather(a, tile, t, seg, threadIdx.x, &s_last, SyncBlock{}))
            continue;
        epilogue<T>(a, tile, mt, nt, n_nt, threadIdx.x, SyncBlock{});
        __syncthreads();
    }
}

// ---------------------------------------------------------------- host
// k segments per n tile.  A persistent CTA streams its units back to back,
// so the time is set by the busiest CTA's chunk count; each extra segment
// adds a partial tile to publish and reduce.  Cost = max chunks per CTA +
// 8 chunk-equivalents per segment (fitted to the Qwen3-8B projections on a
// B200: QKV -> 3, O -> 3, gate/up -> 2, down -> 4, LM head -> 1).  Depends on
// the matrix shape only, never on the number of token rows.
int choose_splits(int N, int Kd)
{
    const int n_nt = (N + kTileN - 1) / kTileN;
    const int chunks = (Kd + kTileK - 1) / kTileK;
    int best = 1;
    long best_cost = -1;
    for (int S = 1; S <= 16; ++S) {
        if (S > 1 && chunks / S < 4) break;
        const long units = (long)n_nt * S;
        const long per_cta = (units + kNumSMs - 1) / kNumSMs;
        const long cost = per_cta * ((chunks + S - 1) / S) + 8L * S;
        if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = S; }
    }
    return best;
}

bool use_tensor_cores(const orthrus_config_t &c) { return c.dtype == ORTHRUS_BF16; }

size_t gemm_smem_bytes(bool tc)
{
    return sizeof(float) * kTileM * kTilePad + (tc ? sizeof(MmaSmem) : sizeof(float) * kTileM * kTileK);
}

cudaError_t launch_gemm(const Ctx &c, GemmArgs a, cudaStream_t s)
{
    const bool tc = use_tensor_cores(c.cfg) && a.Kd % kTileK == 0;
    const int n_nt = a.epi == EPI_SWIGLU ? (a.N + 63) / 64 : (a.N + kTileN - 1) / kTileN;
    const int n_mt = (a.M + kTileM - 1) / kTileM;
    a.splits = tc ? choose_splits(n_nt * kTileN, a.Kd) : 1;
    if (a.splits > 1) {
        if ((size_t)n_mt * n_nt * a.splits * kTileM * kTileN > c.gemm_part_floats ||
            n_mt * n_nt > c.gemm_tickets)
            return cudaErrorInvalidValue;
    }
    a.part = c.gemm_part;
    a.ticket = c.gemm_ticket;
    a.err = c.err;
    const long units = (long)n_mt * n_nt * a.splits;
    const int grid = (int)(units < kNumSMs ? units : kNumSMs);
    const size_t smem = gemm_smem_bytes(tc);
    if (tc) {
        const cudaError_t e = launch_gemm_tc(c, a, n_mt, n_nt, grid, s);
        if (e != cudaErrorNotSupported) return e;
    }
    c.launches += 1;
    if (tc && getenv("ORTHRUS_GEMM_MMA_SYNC")) {
        gemm_kernel<bf16, true><<<grid, kGemmThreads, smem, s>>>(a, n_mt, n_nt);
    } else if (c.cfg.dtype == ORTHRUS_BF16) {
        gemm_kernel<bf16, false><<<grid, kGemmThreads, smem, s>>>(a, n_mt, n_nt);
    } else {
        gemm_kernel<float, false><<<grid, kGemmThreads, smem, s>>>(a, n_mt, n_nt);
    }
    return cudaGetLastError();
}

cudaError_t gemm_init_attributes()
{
    return cudaFuncSetAttribute(gemm_kernel<bf16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)gemm_smem_bytes(true));
}

}  // namespace orthrus
