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
// This file holds the SIMT mainloop (fp32 models, and bf16 shapes without
// tensor maps) and the host dispatch; the bf16 tensor-core mainloop
// (tcgen05, TMA, TMEM) is in gemm_tc.cu.  Both share tiling, scheduling and
// the epilogues of gemm_epilogue.cuh.
#include <math.h>

#include "common.cuh"
#include "gemm_epilogue.cuh"
#include "internal.h"

namespace orthrus {

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

// ---------------------------------------------------------------- mainloop
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
template <class T>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(GemmArgs a, int n_mt, int n_nt)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float(*tile)[kTilePad] = (float(*)[kTilePad])smem_raw;
    unsigned char *pipe = smem_raw + sizeof(float) * kTileM * kTilePad;
    __shared__ int s_last;
    pdl_trigger();
    pdl_wait();
    if (a.epi == EPI_RESAMPLE && *a.any_flag == 0) return;

    const int S = a.splits;
    const int units = n_mt * n_nt * S;
    const int chunks = (a.Kd + kTileK - 1) / kTileK;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int seg = u % S, t = u / S, mt = t % n_mt, nt = t / n_mt;
        const int c0 = (int)((long)seg * chunks / S), c1 = (int)((long)(seg + 1) * chunks / S);
        mainloop_simt<T>(a, mt, nt, c0 * kTileK, min(c1 * kTileK, a.Kd), (float *)pipe, tile);
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

size_t gemm_smem_bytes() { return sizeof(float) * kTileM * kTilePad + sizeof(float) * kTileM * kTileK; }

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
    const size_t smem = gemm_smem_bytes();
    if (tc) {
        const cudaError_t e = launch_gemm_tc(c, a, n_mt, n_nt, grid, s);
        if (e != cudaErrorNotSupported) return e;
    }
    c.launches += 1;
    if (c.cfg.dtype == ORTHRUS_BF16) return launch_k(gemm_kernel<bf16>, grid, kGemmThreads, smem, s, a, n_mt, n_nt);
    return launch_k(gemm_kernel<float>, grid, kGemmThreads, smem, s, a, n_mt, n_nt);
}

cudaError_t gemm_init_attributes() { return cudaSuccess; }

}  // namespace orthrus
