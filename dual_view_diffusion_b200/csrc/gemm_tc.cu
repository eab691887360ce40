// Projection GEMMs on the 5th-generation tensor cores (tcgen05) for bf16.
//
// Same contract as the SIMT path in gemm.cu (work units, fixed split-K per
// matrix shape, deterministic segment-order reduction, shared epilogues), with
// a Blackwell mainloop:
//
//   warp 0      producer: one thread issues TMA tile loads (W: 128 rows x 64,
//               X: 32 token rows x 64, both 128-byte swizzled) into a ring of
//               shared-memory stages, signalling an mbarrier per stage;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M = 128 weight rows,
//               N = 32 tokens, K = 16 per instruction) from shared memory into a
//               TMEM accumulator; tcgen05.commit releases each stage when the
//               MMAs reading it are done, and publishes the accumulator at the
//               end of a unit;
//   warps 2..5  epilogue: drain the accumulator with tcgen05.ld (warp w reads
//               TMEM lanes 32*(w%4) ..), stage it as fp32 in shared memory and
//               run the split-K gather and the fused epilogue.
//
// Two accumulators (2 x 32 TMEM columns) let unit i+1's MMAs run while unit i
// drains.  Every mbarrier wait is bounded: on timeout the kernel raises
// ORTHRUS_DEVERR_TIMEOUT, stops issuing, and still frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "gemm_epilogue.cuh"
#include "internal.h"

namespace orthrus {

constexpr int kTcStages = 8;
constexpr int kTcThreads = 192;
constexpr int kTcAccCols = 32;                          // TMEM columns per accumulator (N = 32)
constexpr uint32_t kStageWBytes = kTileN * kTileK * 2;  // 16 KiB
constexpr uint32_t kStageXBytes = kTileM * kTileK * 2;  // 4 KiB
constexpr long long kSpinCycles = 4000000000LL;        // ~2 s at the B200 SM clock

struct TcSmem {
    alignas(1024) unsigned char w[kTcStages][kStageWBytes];
    alignas(1024) unsigned char x[kTcStages][kStageXBytes];
    float tile[kTileM][kTilePad];
    alignas(8) uint64_t full[kTcStages], empty[kTcStages], tfull[2], tempty[2];
    uint32_t tmem_base;
    int abort;
    int s_last;
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t *b, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok) : "r"(smem_u32(b)), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait (about two seconds of SM clock); false on timeout, or when
// another role of the CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, volatile int *abort)
{
    const long long t0 = clock64();
    for (long i = 0;; ++i) {
        if (mbar_try(b, parity)) return true;
        if ((i & 255) == 255) {
            if (*abort) return false;
            if (clock64() - t0 > kSpinCycles) break;
        }
    }
    *abort = 1;
    return false;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
        ::"r"(smem_u32(dst)), "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// K-major operand, 128-byte swizzle, rows of 64 bf16: 8-row groups 1024 B
// apart (stride byte offset), leading byte offset unused (1), descriptor
// version 1, layout code 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void *p)
{
    const uint32_t a = smem_u32(p);
    return (uint64_t)((a & 0x3FFFF) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both
// K-major, N = 32, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTileM >> 3) << 17) |
                            ((uint32_t)(kTileN >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                 " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
                 ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
                 : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32])
{
    uint32_t u[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
          "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
          "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(u[i]);
}

// ---------------------------------------------------------------- kernel
struct TcMaps {
    CUtensorMap w[3];   // weight segments (QKV: Q, K, V; SwiGLU: gate, up; else w[0])
    CUtensorMap x;      // activations
};

__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(const __grid_constant__ TcMaps maps, GemmArgs a,
                                                                 int n_mt, int n_nt)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    TcSmem &sm = *(TcSmem *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    if (a.epi == EPI_RESAMPLE) {   // the flag comes from the previous kernel
        pdl_wait();
        if (*a.any_flag == 0) return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&sm.tfull[s], 1); mbar_init(&sm.tempty[s], kEpiThreads); }
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(2 * kTcAccCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    const int S = a.splits;
    const int units = n_mt * n_nt * S;
    const int chunks = a.Kd / kTileK;

    if (warp == 0) {
        if (lane == 0) {   // ------------------------------------------- producer
            // Weights never depend on earlier kernels: the first unit's first
            // stages are requested before waiting for the predecessor grid;
            // their activation tiles follow once it has completed.
            uint32_t stage = 0, phase = 0;
            int deferred = 0;   // stages whose X tile is still to be requested
            for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x) {
                const int seg = u % S, t = u / S, mt = t % n_mt, nt = t / n_mt;
                const int c0 = (int)((long)seg * chunks / S), c1 = (int)((long)(seg + 1) * chunks / S);
                // weight segment of this n tile
                int wsel = 0, wrow = nt * kTileN;
                if (a.epi != EPI_SWIGLU) {
                    while (wsel < 2 && wrow >= a.wrows[wsel]) { wrow -= a.wrows[wsel]; ++wsel; }
                }
                const bool first = u == (int)blockIdx.x;
                for (int c = c0; c < c1; ++c) {
                    if (first && deferred >= 0 && c - c0 == kTcStages) {
                        pdl_wait();
                        for (int i = 0; i < deferred; ++i)
                            tma_load_2d(sm.x[i], &maps.x, (c0 + i) * kTileK, mt * kTileM, &sm.full[i]);
                        deferred = -1;
                    }
                    if (!mbar_wait(&sm.empty[stage], phase ^ 1, abort)) break;
                    mbar_expect_tx(&sm.full[stage], kStageWBytes + kStageXBytes);
                    if (a.epi == EPI_SWIGLU) {
                        tma_load_2d(sm.w[stage], &maps.w[0], c * kTileK, nt * 64, &sm.full[stage]);
                        tma_load_2d(sm.w[stage] + kStageWBytes / 2, &maps.w[1], c * kTileK, nt * 64, &sm.full[stage]);
                    } else {
                        tma_load_2d(sm.w[stage], &maps.w[wsel], c * kTileK, wrow, &sm.full[stage]);
                    }
                    if (first && deferred >= 0) ++deferred;
                    else tma_load_2d(sm.x[stage], &maps.x, c * kTileK, mt * kTileM, &sm.full[stage]);
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
                if (first && deferred >= 0) {   // first unit shorter than the ring
                    pdl_wait();
                    for (int i = 0; i < deferred; ++i)
                        tma_load_2d(sm.x[i], &maps.x, (c0 + i) * kTileK, mt * kTileM, &sm.full[i]);
                    deferred = -1;
                }
            }
            if (deferred >= 0) pdl_wait();
            pdl_trigger();   // every load of this CTA is issued
        }
        __syncwarp();   // lanes 1..31 wait for the producer lane before the block barrier
    } else if (warp == 1) {
        if (lane == 0) {   // ------------------------------------------- MMA issuer
            uint32_t stage = 0, phase = 0;
            int local = 0;
            for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x, ++local) {
                const int seg = u % S;
                const int c0 = (int)((long)seg * chunks / S), c1 = (int)((long)(seg + 1) * chunks / S);
                const int acc = local & 1;
                const uint32_t aphase = (local >> 1) & 1;
                if (!mbar_wait(&sm.tempty[acc], aphase ^ 1, abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * kTcAccCols;
                bool ok = true;
                for (int c = c0; c < c1; ++c) {
                    if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_sw128(sm.w[stage]), bd = smem_desc_sw128(sm.x[stage]);
#pragma unroll
                    for (int k = 0; k < kTileK / 16; ++k)   // +32 bytes per k step inside the swizzle atom
                        umma_bf16(d, ad + 2 * k, bd + 2 * k, (c > c0 || k > 0) ? 1u : 0u);
                    umma_commit(&sm.empty[stage]);
                    if (++stage == kTcStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&sm.tfull[acc]);
            }
        }
        __syncwarp();   // lanes 1..31 wait for the MMA lane before the block barrier
    } else {   // --------------------------------------------------------- epilogue
        pdl_wait();                                  // the epilogues read and write predecessor data
        const int et = threadIdx.x - 64;            // 0..127
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        int local = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++local) {
            const int seg = u % S, t = u / S, mt = t % n_mt, nt = t / n_mt;
            const int acc = local & 1;
            const uint32_t aphase = (local >> 1) & 1;
            const bool ok = mbar_wait(&sm.tfull[acc], aphase, abort);
            SyncEpilogue{}();
            if (!ok || *abort) break;
            tc_fence_after();
            float r[32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + acc * kTcAccCols, r);
            tc_fence_before();
            mbar_arrive(&sm.tempty[acc]);
            const int f = q * 32 + lane;             // weight row = output feature in the tile
#pragma unroll
            for (int j = 0; j < kTileM; ++j) sm.tile[j][f] = r[j];
            SyncEpilogue{}();
            if (split_k_gather(a, sm.tile, t, seg, et, &sm.s_last, SyncEpilogue{}))
                epilogue<bf16>(a, sm.tile, mt, nt, n_nt, et, SyncEpilogue{});
            SyncEpilogue{}();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (sm.abort && threadIdx.x == 0) raise_err(a.err, ORTHRUS_DEVERR_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(2 * kTcAccCols));
    }
}

// ---------------------------------------------------------------- host
static PFN_cuTensorMapEncodeTiled_v12000 get_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    return fn;
}

// 2-D bf16 map over a row-major [rows][cols] matrix, box {box_cols, box_rows}
// (box_cols * 2 bytes <= 128), 128-byte swizzle, zero fill outside.
bool make_tmap_box(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_cols, uint32_t box_rows)
{
    auto enc = get_encoder();
    if (!enc || !ptr || ((uintptr_t)ptr & 15) || (cols * 2) % 16 || box_cols * 2 > 128) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    return make_tmap_box(m, ptr, rows, cols, 64, box_rows);
}

// 4-D view of q [rows][n_q][hd] as (dim, head in group, kv head, row), box
// {64, g, 1, ksub}: one load brings the g heads of one KV head for ksub
// consecutive block rows, ordered (row, head) = the attention CTA's rows.
bool make_tmap_q4(CUtensorMap *m, const void *q, int rows_total, int n_q, int n_kv, int hd, int ksub)
{
    auto enc = get_encoder();
    const int g = n_q / n_kv;
    if (!enc || !q || ((uintptr_t)q & 15) || (hd * 2) % 16 || g > 256 || ksub > 256) return false;
    cuuint64_t dims[4] = {(cuuint64_t)hd, (cuuint64_t)g, (cuuint64_t)n_kv, (cuuint64_t)rows_total};
    cuuint64_t strides[3] = {(cuuint64_t)hd * 2, (cuuint64_t)g * hd * 2, (cuuint64_t)n_q * hd * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)g, 1, (cuuint32_t)ksub};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t gemm_tc_smem_bytes() { return sizeof(TcSmem) + 1024; }

cudaError_t gemm_tc_init_attributes()
{
    return cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)gemm_tc_smem_bytes());
}

// Launches the tcgen05 kernel when every operand has a tensor map; returns
// cudaErrorNotSupported otherwise (the caller then uses the SIMT kernel).
cudaError_t launch_gemm_tc(const Ctx &c, const GemmArgs &a, int n_mt, int n_nt, int grid, cudaStream_t s)
{
    TcMaps maps;
    memset(&maps, 0, sizeof(maps));
    const int nseg = a.epi == EPI_SWIGLU ? 2 : 3;
    for (int i = 0; i < nseg; ++i) {
        if (!a.w[i] || a.wrows[i] == 0) continue;
        auto it = c.tmaps.find(TmapKey{a.w[i], a.epi == EPI_SWIGLU ? 64u : 128u});
        if (it == c.tmaps.end()) return cudaErrorNotSupported;
        maps.w[i] = it->second;
        if (a.epi != EPI_SWIGLU && i < 2 && a.wrows[i + 1] > 0 && a.wrows[i] % kTileN) return cudaErrorNotSupported;
    }
    auto it = c.tmaps.find(TmapKey{a.x, (uint32_t)kTileM});
    if (it == c.tmaps.end()) return cudaErrorNotSupported;
    maps.x = it->second;
    c.launches += 1;
    return launch_k(gemm_tc_kernel, grid, kTcThreads, gemm_tc_smem_bytes(), s, maps, a, n_mt, n_nt);
}

}  // namespace orthrus
