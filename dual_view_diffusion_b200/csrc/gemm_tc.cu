// Projection GEMMs on the 5th-generation tensor cores (tcgen05) for bf16.
//
// Work split ("stream-K"): the (n tile, 64-wide k chunk) pairs of one token
// tile, taken n-tile-major, are cut into G = min(148, pairs) equal contiguous
// pieces, one per CTA; token tiles repeat the same cut.  A token tile holds
// TM rows, a multiple of 32 up to 256 (one MMA's N): every token row of a
// step of up to 256 rows rides on each weight tile, so the weights stream
// from HBM once whatever the batch.  A piece
// covers the end of one n tile, whole n tiles and the start of another, so
// every SM streams the same number of weight bytes whatever the matrix shape.
// An n tile cut across pieces is reduced by the piece holding its first
// chunks: the others publish fp32 partials and a flag, and that piece sums
// them in segment order (fixed by the shape alone, never by the token count)
// before the fused epilogue.  The piece holding a tile's last chunks works on
// them first, so its partial is usually published long before it is needed.
//
//   warp 0      producer: one thread issues TMA tile loads (W: 128 rows x 64,
//               X: TM token rows x 64, both 128-byte swizzled) into a ring of
//               shared-memory stages (8 for TM = 32, fewer for wider token
//               tiles), signalling an mbarrier per stage;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M = 128 weight rows,
//               N = TM tokens, K = 16 per instruction) from shared memory into a
//               TMEM accumulator; tcgen05.commit releases each stage when the
//               MMAs reading it are done, and publishes the accumulator at the
//               end of a tile's chunks;
//   warps 2..5  epilogue: fetch what the epilogue needs (residual rows, cache
//               destinations, other pieces' partials) while the chunks stream,
//               then drain the accumulator 32 token rows at a time with
//               tcgen05.ld (warp w reads TMEM lanes 32*(w%4) ..), stage each
//               32-row chunk in shared memory and either publish it as a
//               partial or finish it.
//
// Two accumulators (2 x TM TMEM columns) let the next tile's MMAs run while
// one drains.  Every wait (mbarrier or flag) is bounded: on timeout the
// kernel raises ORTHRUS_DEVERR_TIMEOUT, stops issuing, and still frees its
// TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "gemm_epilogue.cuh"
#include "internal.h"

namespace orthrus {

constexpr int kTcStages = 8;                             // most ring stages (TM = 32)
constexpr int kTcThreads = 192;
constexpr int kTcMaxTM = 256;                           // token rows per tile: one MMA's largest N
constexpr uint32_t kStageWBytes = kTileN * kTileK * 2;  // 16 KiB
constexpr long long kSpinCycles = 4000000000LL;        // ~2 s at the B200 SM clock
// dynamic shared memory of one CTA: the 227 KiB a block may opt in to, less
// the epilogues' static shared arrays (at most 1 KiB) and 1 KiB of slack
constexpr size_t kTcSmemBudget = 225 * 1024;

// The fixed part of the shared memory; the stage ring (kStageWBytes weight
// tiles, then TM x 128-byte token tiles, stages of each) follows it at a
// 1024-byte boundary, sized per launch.
struct TcSmem {
    float tile[kTileM][kTilePad];
    EpiPre pre;                       // (cluster mode, rank 0: pre.resid lands rank 1's tile)
    float peer2[kTileM][kTilePad];    // cluster mode, rank 0: rank 2's tile
    alignas(8) uint64_t full[kTcStages], empty[kTcStages], tfull[2], tempty[2];
    uint64_t peer_full, peer_empty;   // cluster mode: the other ranks' tiles landed / this rank's was consumed
    uint32_t tmem_base;
    int abort;
    int s_last;
};
constexpr size_t kTcRingOffset = (sizeof(TcSmem) + 1023) / 1024 * 1024;

// Ring stages for token tiles of tm rows: as many as fit beside the fixed
// part, at most kTcStages.
__host__ __device__ constexpr int tc_stages(int tm)
{
    const size_t per = kStageWBytes + (size_t)tm * kTileK * 2;
    const size_t n = (kTcSmemBudget - 1024 - kTcRingOffset) / per;
    return (int)(n < (size_t)kTcStages ? n : (size_t)kTcStages);
}
// TMEM columns of the two accumulators (a power of two, at least 32)
__host__ __device__ constexpr uint32_t tc_tmem_cols(int tm)
{
    uint32_t c = 32;
    while (c < 2u * (uint32_t)tm) c <<= 1;
    return c;
}

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

// Weight tiles are read once per forward: they are loaded with an L2
// evict-first policy so that the weight stream does not push activations,
// cache pages and the other kernels' code out of L2.
__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar,
                                                 uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;\n"
        ::"r"(smem_u32(dst)), "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
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
// K-major, N = tm token rows, M = 128 weight rows.
__device__ __forceinline__ uint32_t tc_idesc(int tm)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(tm >> 3) << 17) | ((uint32_t)(kTileN >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                 " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
                 ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ uint32_t tc_cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t tc_mapa(uint32_t local, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
__device__ __forceinline__ void tc_cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed;\n" ::: "memory"); }
__device__ __forceinline__ void tc_cluster_arrive() { asm volatile("barrier.cluster.arrive;\n" ::: "memory"); }
__device__ __forceinline__ void tc_cluster_wait() { asm volatile("barrier.cluster.wait;\n" ::: "memory"); }
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

// ---------------------------------------------------------------- work split
// Piece g of G covers pairs [g*P/G, (g+1)*P/G) of the P = n_nt * chunks
// (n tile, chunk) pairs of a token tile.
struct SkShape {
    long P;
    int G, chunks, n_nt, n_mt;
    int tm;       // token rows per token tile (a multiple of 32, at most kTcMaxTM)
    int stages;   // ring stages (tc_stages(tm))
};
__host__ __device__ inline long sk_begin(const SkShape &k, int g) { return (long)g * k.P / k.G; }
// the piece holding pair x
__host__ __device__ inline int sk_piece(const SkShape &k, long x)
{
    int g = (int)((x * k.G) / k.P);
    while (g + 1 < k.G && sk_begin(k, g + 1) <= x) ++g;
    while (g > 0 && sk_begin(k, g) > x) --g;
    return g;
}
struct SkSub {
    int mt, nt, c0, c1, seg, nseg;
};
// The sub-units (token tile, n tile, chunk range) of piece g, in order.
struct SkIter {
    SkShape k;
    int g, mt, nt;
    long b, e;
    __device__ SkIter(const SkShape &k_, int g_) : k(k_), g(g_), mt(0)
    {
        b = sk_begin(k, g);
        e = sk_begin(k, g + 1);
        nt = (int)(b / k.chunks);
        if (g >= k.G || b >= e) mt = k.n_mt;
    }
    __device__ bool valid() const { return mt < k.n_mt; }
    __device__ SkSub get() const
    {
        const long tb = (long)nt * k.chunks;
        SkSub s;
        s.mt = mt;
        s.nt = nt;
        s.c0 = (int)((b > tb ? b : tb) - tb);
        s.c1 = (int)((e < tb + k.chunks ? e : tb + k.chunks) - tb);
        const int gf = sk_piece(k, tb), gl = sk_piece(k, tb + k.chunks - 1);
        s.seg = g - gf;
        s.nseg = gl - gf + 1;
        return s;
    }
    __device__ void advance()
    {
        ++nt;
        if ((long)nt * k.chunks >= e) {
            ++mt;
            nt = (int)(b / k.chunks);
        }
    }
};

// ---------------------------------------------------------------- kernel
struct TcMaps {
    CUtensorMap w[3];   // weight segments (QKV: Q, K, V; SwiGLU: gate, up; else w[0])
    CUtensorMap x;      // activations
};

__device__ __forceinline__ bool flag_wait(const int *f, volatile int *abort)
{
    const long long t0 = clock64();
    for (long i = 0;; ++i) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(f) : "memory");
        if (v) return true;
        if ((i & 63) == 63) {
            if (*abort) return false;
            if (clock64() - t0 > kSpinCycles) break;
        }
    }
    *abort = 1;
    return false;
}

// E: the epilogue (Epi), fixed at compile time.  TMF: the token tile's rows
// when fixed at compile time (32: one token tile of a decode step at batch
// 1, where the ring and the chunk loop fold to constants), or 0 for a tile
// size taken from sk.tm.
template <int E, int TMF>
__global__ void __launch_bounds__(kTcThreads, 1) gemm_tc_kernel(const __grid_constant__ TcMaps maps, GemmArgs a,
                                                                 SkShape sk)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *base = (unsigned char *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    TcSmem &sm = *(TcSmem *)base;
    if (E == EPI_RESAMPLE) {   // the flag comes from the previous kernel
        pdl_wait();
        if (*a.any_flag == 0) return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;
    const int tm = TMF ? TMF : sk.tm, nch = tm / kTileM, stages = TMF ? tc_stages(TMF) : sk.stages;
    const uint32_t xbytes = (uint32_t)tm * kTileK * 2;
    unsigned char *ring_w = base + kTcRingOffset, *ring_x = ring_w + (size_t)stages * kStageWBytes;
    const uint32_t tcols = tc_tmem_cols(tm);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(&sm.tfull[s], 1); mbar_init(&sm.tempty[s], kEpiThreads); }
        mbar_init(&sm.peer_full, 1);
        mbar_init(&sm.peer_empty, 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(tcols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int g = blockIdx.x;
    // cluster mode (a.pair = 2 or 3 CTAs per cluster): the CTAs of a cluster
    // hold the k segments of the same n tiles; ranks 1.. hand their fp32
    // tiles to rank 0 through distributed shared memory, one 32-row chunk at
    // a time.  Every CTA's barriers are initialised before any signals
    // another (start of the cluster barrier; its wait comes before the first
    // remote operation).
    const bool pair = a.pair > 1;
    const uint32_t crank = pair ? tc_cluster_rank() : 0u;
    if (pair) tc_cluster_arrive_relaxed();

    if (warp == 0) {
        if (lane == 0) {   // ------------------------------------------- producer
            // Weights never depend on earlier kernels: the first stages of
            // the ring are requested before waiting for the predecessor grid;
            // their activation tiles follow once it has completed.
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            bool waited = false;
            const uint64_t wpol = l2_evict_first();
            const int prewait = a.prewait_stages > 0 ? min(stages, a.prewait_stages) : stages;
            int def_c[kTcStages], def_mt[kTcStages];
            auto release_deferred = [&]() {
                pdl_wait();
                waited = true;
                for (int i = 0; i < issued && i < stages; ++i)
                    tma_load_2d(ring_x + (size_t)i * xbytes, &maps.x, def_c[i] * kTileK, def_mt[i] * tm, &sm.full[i]);
            };
            bool stop = false;
            for (SkIter it(sk, g); it.valid() && !stop; it.advance()) {
                const SkSub s = it.get();
                // weight segment of this n tile
                int wsel = 0, wrow = s.nt * kTileN;
                if (E != EPI_SWIGLU) {
                    while (wsel < 2 && wrow >= a.wrows[wsel]) { wrow -= a.wrows[wsel]; ++wsel; }
                }
                for (int c = s.c0; c < s.c1; ++c) {
                    if (!waited && issued == prewait) release_deferred();
                    if (!mbar_wait(&sm.empty[stage], phase ^ 1, abort) || *abort) { stop = true; break; }
                    mbar_expect_tx(&sm.full[stage], kStageWBytes + xbytes);
                    unsigned char *wdst = ring_w + (size_t)stage * kStageWBytes;
                    if (E == EPI_SWIGLU) {
                        tma_load_2d_hint(wdst, &maps.w[0], c * kTileK, s.nt * 64, &sm.full[stage], wpol);
                        tma_load_2d_hint(wdst + kStageWBytes / 2, &maps.w[1], c * kTileK, s.nt * 64, &sm.full[stage], wpol);
                    } else {
                        tma_load_2d_hint(wdst, &maps.w[wsel], c * kTileK, wrow, &sm.full[stage], wpol);
                    }
                    if (!waited) { def_c[issued] = c; def_mt[issued] = s.mt; }
                    else tma_load_2d(ring_x + (size_t)stage * xbytes, &maps.x, c * kTileK, s.mt * tm, &sm.full[stage]);
                    ++issued;
                    if (++stage == (uint32_t)stages) { stage = 0; phase ^= 1; }
                }
            }
            if (!waited) release_deferred();
            // the next kernel may be scheduled once every load of every CTA
            // is issued (triggering at the start measured slower: its CTAs
            // then compete with this grid's tail for SMs)
            pdl_trigger();
        }
        __syncwarp();   // lanes 1..31 wait for the producer lane before the block barrier
    } else if (warp == 1) {
        if (lane == 0) {   // ------------------------------------------- MMA issuer
            uint32_t stage = 0, phase = 0;
            int local = 0;
            const uint32_t idesc = tc_idesc(tm);
            for (SkIter it(sk, g); it.valid() && !*abort; it.advance(), ++local) {
                const SkSub s = it.get();
                const int acc = local & 1;
                const uint32_t aphase = (local >> 1) & 1;
                if (!mbar_wait(&sm.tempty[acc], aphase ^ 1, abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * tm;
                bool ok = true;
                for (int c = s.c0; c < s.c1; ++c) {
                    if (!mbar_wait(&sm.full[stage], phase, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_sw128(ring_w + (size_t)stage * kStageWBytes);
                    const uint64_t bd = smem_desc_sw128(ring_x + (size_t)stage * xbytes);
#pragma unroll
                    for (int k = 0; k < kTileK / 16; ++k)   // +32 bytes per k step inside the swizzle atom
                        umma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (c > s.c0 || k > 0) ? 1u : 0u);
                    umma_commit(&sm.empty[stage]);
                    if (++stage == (uint32_t)stages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&sm.tfull[acc]);
            }
        }
        __syncwarp();   // lanes 1..31 wait for the MMA lane before the block barrier
    } else {   // --------------------------------------------------------- epilogue
        pdl_wait();                                  // the epilogues read and write predecessor data
        if (pair) tc_cluster_wait();
        const int et = threadIdx.x - 64;            // 0..127
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        const int n_nt_epi = E == EPI_SWIGLU ? (a.N + 63) / 64 : (a.N + kTileN - 1) / kTileN;
        const size_t tile_f = (size_t)tm * kTileN;   // floats of one partial tile
        int local = 0;
        uint32_t hc = 0;   // cluster mode: chunk handovers so far
        for (SkIter it(sk, g); it.valid(); it.advance(), ++local) {
            const SkSub s = it.get();
            const int acc = local & 1;
            const uint32_t aphase = (local >> 1) & 1;
            const size_t slot0 = ((size_t)s.mt * sk.n_nt + s.nt) * a.splits;   // partial / flag slots of this tile
            // 32-row chunks of the token tile that hold rows below M
            const int nvalid = min(nch, (a.M - s.mt * tm + kTileM - 1) / kTileM);
            // -------- before the accumulator is ready
            bool good = !*abort;
            const bool defer = a.defer > 0;
            const bool reducer = !pair && !defer && s.seg == 0 && s.nseg > 1;
            if (reducer) {   // the other segments' partials must be published first
                for (int sg = 1; sg < s.nseg && good; ++sg) {
                    if (et == 0) good = flag_wait(a.ticket + slot0 + sg, abort);
                    SyncEpilogue{}();
                    good = good && !*abort;
                }
            }
            // segments 1.. of chunk 0, summed in order (reducer only)
            float4 rest[kEpiVec];
            auto load_rest = [&](int ch) {
#pragma unroll
                for (int j = 0; j < kEpiVec; ++j) rest[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int sg = 1; sg < s.nseg; ++sg) {
                    const float *src = a.part + (slot0 + sg) * tile_f + (size_t)ch * kTileM * kTileN;
#pragma unroll
                    for (int j = 0; j < kEpiVec; ++j) {
                        const int c = et + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
                        const float4 v = __ldcg((const float4 *)(src + m * kTileN + c4));
                        if (sg == 1) rest[j] = v;
                        else { rest[j].x += v.x; rest[j].y += v.y; rest[j].z += v.z; rest[j].w += v.w; }
                    }
                }
            };
            if (reducer && good) load_rest(0);
            if (!defer && s.seg == 0) epilogue_prepare<bf16, E>(a, sm.pre, s.mt * nch, s.nt, et);
            // -------- the accumulator
            const bool ok = good && mbar_wait(&sm.tfull[acc], aphase, abort);
            SyncEpilogue{}();
            if (!ok || *abort) break;
            tc_fence_after();
            bool stop = false;
            for (int ch = 0; ch < nch; ++ch) {
                const int mt32 = s.mt * nch + ch;   // this chunk's 32-row tile index
                const bool last = ch == nch - 1;
                if (ch >= nvalid) {   // rows past M: nothing to read or write
                    if (last) { tc_fence_before(); mbar_arrive(&sm.tempty[acc]); }
                    continue;
                }
                float r[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + acc * tm + ch * kTileM, r);
                if (last || ch + 1 >= nvalid) {   // the accumulator is drained
                    tc_fence_before();
                    if (last) mbar_arrive(&sm.tempty[acc]);
                }
                const int f = q * 32 + lane;             // weight row = output feature in the tile
                if (ch > 0) SyncEpilogue{}();            // the previous chunk's readers are done with the tile
                if (pair) {   // handover hc of this cluster: one per 32-row chunk, in the same order on every rank
                    if (crank == 0) {
                        if (et == 0) mbar_expect_tx(&sm.peer_full, (uint32_t)((a.pair - 1) * sizeof(sm.tile)));
                    } else {   // rank 0 has consumed the previous handover (so its copy out of sm.tile is done)
                        bool freed = true;
                        if (et == 0) freed = mbar_wait(&sm.peer_empty, (hc & 1) ^ 1, abort);
                        SyncEpilogue{}();
                        if (!freed || *abort) { stop = true; break; }
                    }
                }
#pragma unroll
                for (int j = 0; j < kTileM; ++j) sm.tile[j][f] = r[j];
                if (pair && crank > 0) {   // hand this chunk's segment to rank 0
                    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
                    SyncEpilogue{}();
                    if (et == 0) {
                        const float *land = crank == 1 ? &sm.pre.resid[0][0] : &sm.peer2[0][0];
                        const uint32_t dst = tc_mapa(smem_u32(land), 0), bar = tc_mapa(smem_u32(&sm.peer_full), 0);
                        asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
                                     ::"r"(dst), "r"(smem_u32(&sm.tile[0][0])), "r"((uint32_t)sizeof(sm.tile)), "r"(bar) : "memory");
                    }
                    ++hc;
                    continue;
                }
                SyncEpilogue{}();
                if (pair) {   // rank 0: rank 2 + (rank 1 + rank 0), then free the landing tiles
                    bool landed = true;
                    if (et == 0) landed = mbar_wait(&sm.peer_full, hc & 1, abort);
                    ++hc;
                    SyncEpilogue{}();
                    if (!landed || *abort) { stop = true; break; }
#pragma unroll
                    for (int j = 0; j < kEpiVec; ++j) {
                        const int c = et + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
                        float4 &o = *(float4 *)&sm.tile[m][c4];
                        const float4 p = *(const float4 *)&sm.pre.resid[m][c4];
                        o.x = p.x + o.x; o.y = p.y + o.y; o.z = p.z + o.z; o.w = p.w + o.w;
                        if (a.pair > 2) {
                            const float4 p2 = *(const float4 *)&sm.peer2[m][c4];
                            o.x = p2.x + o.x; o.y = p2.y + o.y; o.z = p2.z + o.z; o.w = p2.w + o.w;
                        }
                    }
                    SyncEpilogue{}();
                    if (et > 0 && et < a.pair)
                        asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n"
                                     ::"r"(tc_mapa(smem_u32(&sm.peer_empty), (uint32_t)et)) : "memory");
                }
                if (defer) {   // this segment of the residual update, summed later by the RMSNorm
#pragma unroll
                    for (int j = 0; j < kEpiVec; ++j) {
                        const int c = et + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
                        const int row = mt32 * kTileM + m, n = s.nt * kTileN + c4;
                        if (row < a.M && n < a.N)
                            __stcg((float4 *)(a.rpart + ((size_t)s.seg * a.rpart_rows + row) * a.N + n),
                                   *(const float4 *)&sm.tile[m][c4]);
                    }
                    continue;
                }
                if (!pair && s.seg > 0) {   // publish this segment's chunk for the tile's reducer
                    float *dst = a.part + (slot0 + s.seg) * tile_f + (size_t)ch * kTileM * kTileN;
#pragma unroll
                    for (int j = 0; j < kEpiVec; ++j) {
                        const int c = et + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
                        __stcg((float4 *)(dst + m * kTileN + c4), *(const float4 *)&sm.tile[m][c4]);
                    }
                    continue;
                }
                if (reducer) {   // (segments 1..) + segment 0
                    if (ch > 0) load_rest(ch);
#pragma unroll
                    for (int j = 0; j < kEpiVec; ++j) {
                        const int c = et + j * kEpiThreads, m = c >> 5, c4 = (c & 31) * 4;
                        float4 &o = *(float4 *)&sm.tile[m][c4];
                        o.x = rest[j].x + o.x; o.y = rest[j].y + o.y; o.z = rest[j].z + o.z; o.w = rest[j].w + o.w;
                    }
                    SyncEpilogue{}();
                }
                if (ch > 0 && !defer && s.seg == 0) {   // chunk 0's was fetched while the chunks streamed
                    epilogue_prepare<bf16, E>(a, sm.pre, mt32, s.nt, et);
                    SyncEpilogue{}();
                }
                epilogue<bf16, SyncEpilogue, E>(a, sm.tile, mt32, s.nt, n_nt_epi, et, SyncEpilogue{}, &sm.pre);
            }
            if (stop) break;
            if (!pair && !defer && s.seg > 0) {   // every chunk of this segment is out: raise its flag
                __threadfence();
                SyncEpilogue{}();
                if (et == 0) asm volatile("st.release.gpu.global.b32 [%0], %1;\n" ::"l"(a.ticket + slot0 + s.seg), "r"(1) : "memory");
            }
            if (reducer && et > 0 && et < s.nseg) a.ticket[slot0 + et] = 0;   // flags ready for the next call
            SyncEpilogue{}();
        }
        // cluster mode, ranks 1..: rank 0's last signal (its arrive after
        // consuming the last handover) lands before this CTA leaves; rank 0
        // itself waited for every copy into it, so no cluster barrier is
        // needed at the end
        if (pair && crank > 0 && hc > 0) {
            if (et == 0) mbar_wait(&sm.peer_empty, (hc - 1) & 1, abort);
            SyncEpilogue{}();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (pair && warp < 2) tc_cluster_wait();   // (their arrive at the start)
    if (sm.abort && threadIdx.x == 0) raise_err(a.err, ORTHRUS_DEVERR_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(tcols));
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

// Dynamic shared memory of a launch with token tiles of tm rows (the fixed
// part, its ring, and slack for the 1024-byte alignment of the base).
size_t gemm_tc_smem_bytes(int tm)
{
    return 1024 + kTcRingOffset + (size_t)tc_stages(tm) * (kStageWBytes + (size_t)tm * kTileK * 2);
}

void gemm_token_tile(int M, int *n_mt, int *tm)
{
    const int n = (M + kTcMaxTM - 1) / kTcMaxTM;
    const int per = (M + n - 1) / n;
    *n_mt = n;
    *tm = (per + kTileM - 1) / kTileM * kTileM;
}

template <int E> static cudaError_t set_smem()
{
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<E, kTileM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kTcSmemBudget);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(gemm_tc_kernel<E, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmemBudget);
}

template <int E>
static cudaError_t launch_tc_e(int G, size_t smem, cudaStream_t s, const TcMaps &maps, const GemmArgs &a,
                               const SkShape &k)
{
    if (k.tm == kTileM) return launch_k(gemm_tc_kernel<E, kTileM>, G, kTcThreads, smem, s, maps, a, k);
    return launch_k(gemm_tc_kernel<E, 0>, G, kTcThreads, smem, s, maps, a, k);
}

cudaError_t gemm_tc_init_attributes()
{
    cudaError_t e = set_smem<EPI_QKV>();
    if (e == cudaSuccess) e = set_smem<EPI_RESID>();
    if (e == cudaSuccess) e = set_smem<EPI_SWIGLU>();
    if (e == cudaSuccess) e = set_smem<EPI_LMHEAD>();
    if (e == cudaSuccess) e = set_smem<EPI_RESAMPLE>();
    if (e == cudaSuccess) e = set_smem<EPI_LOGITS>();
    if (e == cudaSuccess) e = set_smem<EPI_KL>();
    return e;
}

// Largest number of pieces one n tile is cut into, for n_nt tiles of
// `chunks` k chunks (the partial and flag slots per tile).
int sk_max_segments(int n_nt, int chunks)
{
    SkShape k;
    k.P = (long)n_nt * chunks;
    k.G = (int)std::min<long>(kNumSMs, k.P);
    k.chunks = chunks;
    k.n_nt = n_nt;
    k.n_mt = 1;
    int best = 1;
    for (int nt = 0; nt < n_nt; ++nt) {
        const long tb = (long)nt * chunks;
        best = std::max(best, sk_piece(k, tb + chunks - 1) - sk_piece(k, tb) + 1);
    }
    return best;
}

// Launches the tcgen05 kernel when every operand has a tensor map; returns
// cudaErrorNotSupported otherwise (the caller then uses the SIMT kernel).
// a.splits must hold sk_max_segments(n_nt, Kd / 64); n_mt token tiles of tm
// rows (gemm_token_tile).
cudaError_t launch_gemm_tc(const Ctx &c, const GemmArgs &a, int n_mt, int tm, int n_nt, cudaStream_t s)
{
    if (tm < kTileM || tm > kTcMaxTM || tm % kTileM) return cudaErrorInvalidValue;
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
    auto it = c.tmaps.find(TmapKey{a.x, (uint32_t)tm});
    if (it == c.tmaps.end()) return cudaErrorNotSupported;
    maps.x = it->second;
    SkShape k;
    k.chunks = a.Kd / kTileK;
    k.n_nt = n_nt;
    k.n_mt = n_mt;
    k.tm = tm;
    k.stages = tc_stages(tm);
    k.P = (long)n_nt * k.chunks;
    // deferred residual: one piece per (tile, segment), cut at whole chunks
    k.G = a.defer > 0 ? n_nt * a.defer : (int)std::min<long>(kNumSMs, k.P);
    if (a.defer > 0 && (k.chunks % a.defer || a.defer > kResidSlots || !a.rpart)) return cudaErrorInvalidValue;
    const size_t smem = gemm_tc_smem_bytes(tm);
    if (a.pair > 1) {   // a.pair k segments per n tile, one cluster of a.pair CTAs per tile
        if (a.epi != EPI_QKV || a.defer > 0 || a.pair > 3 || k.chunks < a.pair) return cudaErrorInvalidValue;
        k.G = a.pair * n_nt;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(k.G);
        cfg.blockDim = dim3(kTcThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = a.pair;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        c.launches += 1;
        if (tm == kTileM) return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI_QKV, kTileM>, maps, a, k);
        return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI_QKV, 0>, maps, a, k);
    }
    c.launches += 1;
    switch (a.epi) {
    case EPI_QKV: return launch_tc_e<EPI_QKV>(k.G, smem, s, maps, a, k);
    case EPI_RESID: return launch_tc_e<EPI_RESID>(k.G, smem, s, maps, a, k);
    case EPI_SWIGLU: return launch_tc_e<EPI_SWIGLU>(k.G, smem, s, maps, a, k);
    case EPI_LMHEAD: return launch_tc_e<EPI_LMHEAD>(k.G, smem, s, maps, a, k);
    case EPI_RESAMPLE: return launch_tc_e<EPI_RESAMPLE>(k.G, smem, s, maps, a, k);
    case EPI_LOGITS: return launch_tc_e<EPI_LOGITS>(k.G, smem, s, maps, a, k);
    case EPI_KL: return launch_tc_e<EPI_KL>(k.G, smem, s, maps, a, k);
    default: return cudaErrorNotSupported;
    }
}

}  // namespace orthrus
