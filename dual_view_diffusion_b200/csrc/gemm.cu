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
#include <algorithm>

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
// One-dimensional grid of persistent CTAs walking (m tile, n tile) units in
// order, each over the whole k range.
template <class T>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(GemmArgs a, int n_mt, int n_nt)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float(*tile)[kTilePad] = (float(*)[kTilePad])smem_raw;
    unsigned char *pipe = smem_raw + sizeof(float) * kTileM * kTilePad;
    pdl_trigger();
    pdl_wait();
    if (a.epi == EPI_RESAMPLE && *a.any_flag == 0) return;

    const int units = n_mt * n_nt;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int mt = u % n_mt, nt = u / n_mt;
        mainloop_simt<T>(a, mt, nt, 0, a.Kd, (float *)pipe, tile);
        __syncthreads();
        epilogue<T>(a, tile, mt, nt, n_nt, threadIdx.x, SyncBlock{});
        __syncthreads();
    }
}

// ---------------------------------------------------------------- host
bool use_tensor_cores(const orthrus_config_t &c) { return c.dtype == ORTHRUS_BF16; }

// k segments per n tile of a residual GEMM whose sum is left to the next
// RMSNorm: the most that keeps n_tiles x segments within one wave of SMs
// with whole chunks per segment (0: the epilogue adds to the residual).
// A function of the matrix shape only.
int resid_defer_slots(const orthrus_config_t &cfg, int N, int Kd)
{
    if (!use_tensor_cores(cfg) || Kd % kTileK) return 0;
    const int n_nt = (N + kTileN - 1) / kTileN, chunks = Kd / kTileK;
    for (int S = std::min(kResidSlots, kNumSMs / std::max(n_nt, 1)); S >= 1; --S)
        if (chunks % S == 0) return S;
    return 0;
}

size_t gemm_smem_bytes() { return sizeof(float) * kTileM * kTilePad + sizeof(float) * kTileM * kTileK; }

cudaError_t launch_gemm(const Ctx &c, GemmArgs a, cudaStream_t s)
{
    const bool tc = use_tensor_cores(c.cfg) && a.Kd % kTileK == 0;
    const int n_nt = a.epi == EPI_SWIGLU ? (a.N + 63) / 64 : (a.N + kTileN - 1) / kTileN;
    const int n_mt = (a.M + kTileM - 1) / kTileM;
    a.part = c.gemm_part;
    a.ticket = c.gemm_ticket;
    a.err = c.err;
    if (tc) {   // stream-K split: partial and flag slots per (token tile, n tile, segment)
        int n_mt_tc, tm;
        gemm_token_tile(a.M, &n_mt_tc, &tm);
        GemmArgs t = a;
        t.splits = t.defer > 0 ? t.defer : sk_max_segments(n_nt, a.Kd / kTileK);
        // QKV: each head tile cut in 2 k segments reduced inside a 2-CTA
        // cluster when one cluster per tile fits one wave of SMs (a function
        // of the matrix shape, never of the token count; 3-CTA clusters
        // measured slower on B200).  Token tiles of TM rows (all the rows of
        // a step up to 256) ride on each weight tile; the summation order of
        // a row never depends on TM.
        t.pair = 0;
        if (a.epi == EPI_QKV && t.defer == 0)
            for (int S = 2; S >= 2 && !t.pair; --S)
                if (n_nt * S <= kNumSMs && a.Kd / kTileK >= S) t.pair = S;   // the matrix shape only
        const size_t slots = (size_t)n_mt_tc * n_nt * t.splits;
        if (t.splits > 1 && (slots * tm * kTileN > c.gemm_part_floats || slots > (size_t)c.gemm_tickets))
            return cudaErrorInvalidValue;
        const cudaError_t e = launch_gemm_tc(c, t, n_mt_tc, tm, n_nt, s);
        if (e != cudaErrorNotSupported) return e;
    }
    if (a.defer > 0) return cudaErrorInvalidValue;   // only the tensor-core kernel defers
    a.splits = 1;
    const long units = (long)n_mt * n_nt;
    const int grid = (int)(units < kNumSMs ? units : kNumSMs);
    const size_t smem = gemm_smem_bytes();
    c.launches += 1;
    if (c.cfg.dtype == ORTHRUS_BF16) return launch_k(gemm_kernel<bf16>, grid, kGemmThreads, smem, s, a, n_mt, n_nt);
    return launch_k(gemm_kernel<float>, grid, kGemmThreads, smem, s, a, n_mt, n_nt);
}

cudaError_t gemm_init_attributes() { return cudaSuccess; }

}  // namespace orthrus
