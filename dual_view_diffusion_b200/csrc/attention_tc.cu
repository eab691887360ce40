// Dual-view attention on the tcgen05 tensor cores (bf16, head_dim 128).
//
// Z clusters of C CTAs per (KV head, sequence x row group) — one cluster
// normally, four 4-CTA clusters for long contexts at small batch.  Its M =
// 128 query rows are the block rows x the GQA group sharing the KV head, so
// every K/V tile staged in shared memory serves all of them (paper notes
// §2.2-2.3: both views read the one AR cache).  The keys are cut into splits
// aligned to absolute positions; CTA i of the Z * C takes splits i, i + ZC,
// ... and, per 128-key tile:
//
//   S = Q K^T       tcgen05.mma, M 128 x N 128 x K 128 (A = Q, kept in TMEM
//                   for the whole kernel), into TMEM
//   softmax         each softmax thread owns one query row (= TMEM lane): it
//                   reads its 128 scores with tcgen05.ld (which frees S for
//                   the next tile), applies the view's mask, updates its
//                   running max / sum in log2 units, and writes the bf16
//                   probabilities P back to TMEM
//   O += P V        tcgen05.mma, M 128 x N 128 x K 128 (A = P from TMEM), into
//                   a TMEM accumulator
//
// A tcgen05.mma instruction costs the tensor pipe about the same time for any
// N up to 128 (measured on B200: ~130 SM cycles each for M 128, K 16), so the
// tile is as wide as TMEM allows: 16 instructions per 128 keys, against 24
// for two 64-key tiles.
//
// O is rescaled in TMEM only when a warp's running max moved (a factor of
// exactly 1 elsewhere, so skipping it changes no bit).  K tiles come from
// pages laid out [slot][dim], V tiles from pages laid out [dim][slot] (both
// operands K-major), both by TMA with an L2 evict-first hint (a cache tile is
// read once per view).  For the diffusion view the block's own K/V form one
// extra split read from the transient buffer.  A cluster's C partial states
// are merged through distributed shared memory (fp16 rows scaled per half
// row); with Z > 1 each cluster leaves its merged rows in L2 and the last
// cluster to finish (an atomic ticket) merges all Z in cluster order.  A lone
// CTA (C = Z = 1) writes its rows straight from registers.
//
// Roles: warp 0 K producer and warp 2 V producer (TMA, one issuing thread
// each, separate rings: a K tile is free once S is computed, a V tile only
// after its P.V), warp 1 MMA issuer (one thread), warps 4..11 softmax (two
// warpgroups taking alternate tiles) and combine.  A tile's keys are two
// 64-key subtiles, each from its own page.  All mbarrier waits are
// bounded.
#include <cuda.h>
#include <cuda_fp16.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace orthrus {

constexpr int kAtKStages = 2;   // K tiles are released as soon as S = Q K^T is done
constexpr int kAtVStages = 2;   // V tiles live until their P.V
constexpr float kRescaleSlack = 8.0f;   // log2 units a row's max may grow before O is rescaled
constexpr int kAtMaxCluster = 8;        // portable cluster size
constexpr int kAtMaxZ = 4;              // clusters per row group (long contexts)
constexpr int kAtZCluster = 4;          // their size
constexpr int kAtPreWait = 2;           // cache tiles requested before waiting for the predecessor
constexpr int kAtThreads = 384;   // producer warpgroup (K, MMA, V, spare), two softmax warpgroups
constexpr int kAtVWarp = 2;       // the V producer warp
constexpr int kAtSoftWarp0 = 4;   // first softmax warp
constexpr int kAtRows = 128;
constexpr int kAtKeys = 128;      // keys per tile
constexpr int kAtSub = 64;        // keys per subtile (one page box)
constexpr long long kAtSpinCycles = 4000000000LL;   // ~2 s at the B200 SM clock

struct AtSmem {
    alignas(1024) unsigned char k[kAtKStages][2][kAtKeys * 128];  // K tile [128 keys] x dims 0-63 / 64-127, 16 KiB each
    alignas(1024) unsigned char v[kAtVStages][2][128 * 128];      // V^T subtiles [128 dims][64 keys], 16 KiB each
    alignas(8) uint64_t q_ready, kfull[kAtKStages], kempty[kAtKStages], vfull[kAtVStages], vempty[kAtVStages];
    uint64_t s_full[2], s_free, p_full[2], o_done[2];
    float2 xml[2][kAtRows];   // (m, l) of each accumulator, per row
    uint32_t tmem_base;
    int abort;
    int xticket;   // this cluster's arrival order at the cross-cluster combine
};
// Once the last P.V is done, k..v (192 KiB) is reused for the combine: the
// CTA's normalised rows [128][128] as fp16 scaled per half row (16-byte chunk
// ch of row r at ch ^ (r & 15)) and (m, l, scale, scale) per row, read by the
// other CTAs of the cluster.
constexpr uint32_t kStageO = 0, kStageMl = 32 * 1024;
static_assert(kStageMl + kAtRows * 16 <= kAtKStages * 32768 + kAtVStages * 32768, "combine area");

// TMEM columns: two O accumulators (even / odd tiles) [0, 256), S [256, 384)
// (one buffer: the softmax frees it as soon as it has read its scores), P
// [384, 448) and Q [448, 512) (bf16 pairs: the A operands of P.V and of
// Q K^T read straight from TMEM).  One P buffer suffices: P of tile i is
// written once the P.V of tile i-1 is done, which is no later than the
// softmax of tile i needs it.
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemP = 384, kTmemQ = 448, kTmemCols = 512;

__device__ __forceinline__ void at_mbar_init(uint64_t *b, uint32_t n)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(b)), "r"(n));
}
__device__ __forceinline__ void at_expect(uint64_t *b, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void at_arrive(uint64_t *b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(b)) : "memory");
}
// Bounded wait (about two seconds of SM clock); false on timeout, or when
// another role of the CTA already gave up.
__device__ __forceinline__ bool at_wait(uint64_t *b, uint32_t parity, volatile int *abort)
{
    const long long t0 = clock64();
    for (long i = 0;; ++i) {
        uint32_t ok;
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
                     : "=r"(ok) : "r"(smem_u32(b)), "r"(parity) : "memory");
        if (ok) return true;
        if ((i & 255) == 255) {
            if (*abort) return false;
            if (clock64() - t0 > kAtSpinCycles) break;
        }
    }
    *abort = 1;
    return false;
}
__device__ __forceinline__ void at_tma2(void *dst, const CUtensorMap *m, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n"
        ::"r"(smem_u32(dst)), "l"((uint64_t)m), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}
// cache tiles are read once per view: loaded evict-first, they leave the
// rest of L2 (activations, code, block tables) in place
__device__ __forceinline__ void at_tma2_ef(void *dst, const CUtensorMap *m, int x, int y, uint64_t *bar, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;\n"
        ::"r"(smem_u32(dst)), "l"((uint64_t)m), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(pol) : "memory");
}
__device__ __forceinline__ uint64_t at_desc(const void *p)
{
    const uint32_t a = smem_u32(p);
    return (uint64_t)((a & 0x3FFFF) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// kind::f16, fp32 accumulate, bf16 A/B, K-major, M = 128
__host__ __device__ constexpr uint32_t idesc_n(int n) { return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | (8u << 24); }

__device__ __forceinline__ void at_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
                 ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
// D (TMEM) += A (TMEM) * B (shared memory descriptor)
__device__ __forceinline__ void at_mma_ta(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n"
                 ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc) : "memory");
}
__device__ __forceinline__ void at_commit(uint64_t *b)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void at_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void at_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

#define AT_LD32(taddr, r)                                                                                         \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15," \
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"                     \
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), \
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),        \
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),      \
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),      \
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])                                                            \
                 : "r"(taddr))
#define AT_ST32(taddr, r)                                                                                         \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15," \
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"                          \
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),        \
                   "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),    \
                   "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), \
                   "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), \
                   "r"(r[31]) : "memory")
#define AT_ST16(taddr, r)                                                                                         \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15," \
                 "%16};\n"                                                                                          \
                 ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),        \
                   "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),    \
                   "r"(r[15]) : "memory")
__device__ __forceinline__ void at_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void at_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }


// Key range of split s for sequence b: cache splits [s*S, ...) of the cache
// part; in the diffusion view split n_split_grid is the block's own keys.
struct AtSplit {
    int key0, key1, slot, ntiles;
    bool block;
};
__device__ __forceinline__ AtSplit at_split(const AttnArgs &a, int s, int n_split_grid, int t)
{
    AtSplit r;
    r.block = a.mode == 1 && s == n_split_grid;
    if (r.block) {
        r.key0 = t; r.key1 = t + a.K; r.slot = a.n_splits - 1;
    } else {
        r.key0 = s * a.split_tokens;
        r.key1 = min(r.key0 + a.split_tokens, a.mode == 0 ? t + a.K : t);
        r.slot = s;
    }
    r.ntiles = r.key1 > r.key0 ? (r.key1 - r.key0 + kAtKeys - 1) / kAtKeys : 0;
    return r;
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t map_peer_addr(uint32_t local, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory"); }
__device__ __forceinline__ float4 ld_peer4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];\n" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint4 ld_peer4u(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
// Tree verify: 32 visibility bits of block indices j0 .. j0+31 for one query
// row (bit b <-> block index j0 + b): a negative index is a cache key
// (visible), 0 .. 127 the row's ancestor bits m, beyond the block nothing.
__device__ __forceinline__ uint32_t tree_window(const uint32_t (&m)[4], int j0)
{
    const int w = j0 >> 5, sh = j0 & 31;   // floor division: j0 may be negative
    auto word = [&](int i) -> uint32_t {
        return i < 0 ? 0xffffffffu : i == 0 ? m[0] : i == 1 ? m[1] : i == 2 ? m[2] : i == 3 ? m[3] : 0u;
    };
    const uint32_t lo = word(w), hi = word(w + 1);
    return sh ? (lo >> sh) | (hi << (32 - sh)) : lo;
}

__device__ __forceinline__ float ex2(float x)   // 2^x, MUFU; subnormal results flush to zero
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// grid (kv head, sequence x row group, C) with clusters of C CTAs along z:
// cluster = one (sequence, KV head, row group).  CTA r of the cluster loads
// its Q rows once and runs the online softmax over all keys of splits r,
// r + C, r + 2C, ... (a split's keys never depend on which block is being
// decoded, and keys outside a row's window are exact no-ops).  Even and odd
// tiles go to two independent accumulators (O, m, l), so the softmax of one
// tile never waits for the P.V of the tile just before it; the two are merged
// at the end.  The C partial states are then combined on chip: every CTA
// stages its merged rows in its own shared memory, and CTA q reads rows
// [q*128/C, (q+1)*128/C) from all C CTAs (all loads in flight at once) and
// sums them in rank order.
template <int C>
__global__ void __launch_bounds__(kAtThreads, 1) attn_tc_kernel(const __grid_constant__ AtMaps maps, AttnArgs a,
                                                                int n_split_grid)
{
    extern __shared__ __align__(1024) unsigned char at_raw[];
    AtSmem &sm = *(AtSmem *)(((uintptr_t)at_raw + 1023) & ~(uintptr_t)1023);
    pdl_trigger();
    const int kvh = blockIdx.x;
    const int rgroups = gridDim.y / a.B, b = blockIdx.y / rgroups, rg = blockIdx.y % rgroups;
    const int g = a.n_q / a.n_kv, ksub = kAtRows / g;          // block rows per row group
    const int k_lo = rg * ksub, k_hi = min(a.K, k_lo + ksub);
    if (k_lo >= a.K) {   // the whole cluster shares rg
        pdl_wait();
        return;
    }
    constexpr int rpc = kAtRows / C;   // rows owned per CTA
    const int r = (int)cluster_rank();
    // Z clusters of C CTAs share the (sequence, KV head, row group): CTA ci
    // of the Ctot takes splits ci, ci + Ctot, ...
    const int Z = a.xz, zc = (int)blockIdx.z / C, ci = zc * C + r, Ctot = C * Z;
    const int n_total = n_split_grid + (a.mode == 1 ? 1 : 0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;
    // t, the block table and its row are written only by kernels that do not
    // trigger their dependents early (commit, set-length, row-map kernels),
    // so every kernel after them in the stream starts after they completed:
    // they may be read before griddepcontrol.wait
    if (threadIdx.x == 0) {   // the first TMA of each map need not wait for its descriptor
        asm volatile("prefetch.tensormap [%0];\n" ::"l"((uint64_t)&maps.kc) : "memory");
        asm volatile("prefetch.tensormap [%0];\n" ::"l"((uint64_t)&maps.vc) : "memory");
        if (a.mode == 1) {
            asm volatile("prefetch.tensormap [%0];\n" ::"l"((uint64_t)&maps.kb) : "memory");
            asm volatile("prefetch.tensormap [%0];\n" ::"l"((uint64_t)&maps.vb) : "memory");
        }
    }
    const int t = a.seq_lens[b];
    const int bt_row = a.bt_rows[b];
    // Flat subtile f of this CTA is subtile f % tps of split ci + Ctot * (f / tps)
    // for every cache subtile (only the last cache split can be short, and
    // only block tiles follow it).  Each producer warp looks up the pages of
    // 32 flat subtiles at a time, one per lane.
    const int tps = a.split_tokens / kAtSub;
    const int cache_lim = a.mode == 0 ? t + a.K : t;
    // (row = the sequence's block-table row; `got` = that row's entry when
    // already fetched)
    auto page_of = [&](int f, int row, bool have, int got) {
        const int sl = ci + Ctot * (f / tps);
        const int key = sl * a.split_tokens + (f % tps) * kAtSub;
        if (sl >= n_split_grid || key >= cache_lim) return 0;
        const int pidx = key / a.kv.page_size;
        int page = pidx < a.kv.max_pages ? (have ? got : a.kv.block_table[(size_t)row * a.kv.max_pages + pidx]) : -1;
        if (page < 0 || page >= a.kv.num_pages) { raise_err(a.err, ORTHRUS_DEVERR_CAPACITY); page = 0; }
        return page;
    };
    auto lookup = [&](int f) { return page_of(f, bt_row, false, 0); };
    int pg = 0;
    if (warp == 0 || warp == kAtVWarp) {
        // the first pages are read from row b, the usual row map, together
        // with t and the map itself (one round trip instead of two); only a
        // sequence mapped elsewhere reads its own row afterwards
        const int sl = ci + Ctot * (lane / tps);
        const int pidx = (sl * a.split_tokens + (lane % tps) * kAtSub) / a.kv.page_size;
        const int guess = (sl < n_split_grid && pidx < a.kv.max_pages)
                              ? a.kv.block_table[(size_t)b * a.kv.max_pages + pidx] : 0;
        pg = page_of(lane, bt_row, bt_row == b, guess);
    }

    if (threadIdx.x == 0) {
        at_mbar_init(&sm.q_ready, 128);
        for (int i = 0; i < kAtKStages; ++i) { at_mbar_init(&sm.kfull[i], 1); at_mbar_init(&sm.kempty[i], 1); }
        for (int i = 0; i < kAtVStages; ++i) { at_mbar_init(&sm.vfull[i], 1); at_mbar_init(&sm.vempty[i], 1); }
        at_mbar_init(&sm.s_free, 128);
        for (int i = 0; i < 2; ++i) {
            at_mbar_init(&sm.s_full[i], 1);
            at_mbar_init(&sm.p_full[i], 128);
            at_mbar_init(&sm.o_done[i], 1);
        }
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&sm.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    at_fence_before();
    __syncthreads();
    at_fence_after();
    const uint32_t tmem = sm.tmem_base;
    int my_tiles = 0;
    for (int s = ci; s < n_total; s += Ctot) my_tiles += at_split(a, s, n_split_grid, t).ntiles;

    uint32_t jj = 0;
    bool ok = true;
    const int q4 = warp & 3, row = q4 * 32 + lane;   // softmax threads: query row = TMEM lane
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;

    if (warp == 0 || warp == kAtVWarp) {   // ------------------------ K / V producers
        // Two producer warps, one per ring, so V tiles run as far ahead as
        // their deeper ring allows instead of trailing the K issue.  All 32
        // lanes of a producer walk the subtiles together (page lookups); lane
        // 0 issues.  A tile is two 64-key subtiles; where the second lies past
        // the split's end the first is loaded again in its place (finite data,
        // masked out by the softmax).  Up to kAtPreWait cache tiles below t
        // (which the predecessor cannot be writing) are requested before
        // waiting for it.
        const bool kprod = warp == 0;
        uint64_t pol;
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
        uint32_t ks = 0, kph = 0, vs = 0, vph = 0;
        bool waited = false, stop = false;
        auto ensure_wait = [&]() {
            if (waited) return;
            pdl_wait();
            waited = true;
        };
        int f = 0, ft = 0;   // cache subtiles, tiles walked so far
        for (int s = ci; s < n_total && !stop; s += Ctot) {
            const AtSplit sp = at_split(a, s, n_split_grid, t);
            for (int j = 0; j < sp.ntiles; ++j, ++ft) {
                const int p0 = sp.key0 + j * kAtKeys;
                const bool two = p0 + kAtSub < sp.key1;
                int page[2] = {0, 0};
                if (!sp.block) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        if (u == 1 && !two) break;
                        if (f > 0 && (f & 31) == 0) pg = lookup(f + lane);
                        page[u] = __shfl_sync(0xffffffffu, pg, f & 31);
                        ++f;
                    }
                }
                int go = 1;
                if (lane == 0) {
                    if (sp.block || min(p0 + kAtKeys, sp.key1) > t || ft >= kAtPreWait) ensure_wait();
                    const int krow = (a.blk_layer * a.bmax + b) * a.n_kv + kvh;
                    int off[2], hrow[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int uu = (u == 1 && two) ? 1 : 0;
                        off[u] = (p0 + uu * kAtSub) % a.kv.page_size;
                        hrow[u] = (a.layer * a.kv.num_pages + page[uu]) * a.n_kv + kvh;
                    }
                    const int brow0 = j * kAtKeys, brow1 = two ? brow0 + kAtSub : brow0;
                    if (kprod) {
                        if (!at_wait(&sm.kempty[ks], kph ^ 1, abort)) {
                            go = 0;
                        } else {
                            at_expect(&sm.kfull[ks], 4u * 8192u);
#pragma unroll
                            for (int u = 0; u < 2; ++u)
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    if (sp.block)
                                        at_tma2(sm.k[ks][hh] + u * 8192, &maps.kb, hh * 64, krow * a.kp + (u ? brow1 : brow0),
                                                &sm.kfull[ks]);
                                    else
                                        at_tma2_ef(sm.k[ks][hh] + u * 8192, &maps.kc, hh * 64, hrow[u] * a.kv.page_size + off[u],
                                                &sm.kfull[ks], pol);
                                }
                            if (++ks == kAtKStages) { ks = 0; kph ^= 1; }
                        }
                    } else {
                        if (!at_wait(&sm.vempty[vs], vph ^ 1, abort)) {
                            go = 0;
                        } else {
                            at_expect(&sm.vfull[vs], 2u * 16384u);
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                if (sp.block) at_tma2(sm.v[vs][u], &maps.vb, u ? brow1 : brow0, krow * 128, &sm.vfull[vs]);
                                else at_tma2_ef(sm.v[vs][u], &maps.vc, off[u], hrow[u] * 128, &sm.vfull[vs], pol);
                            }
                            if (++vs == kAtVStages) { vs = 0; vph ^= 1; }
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, go, 0)) { stop = true; break; }
            }
        }
        if (lane == 0) ensure_wait();
        __syncwarp();
    } else if (warp == 1) {
        pdl_wait();
        if (lane == 0 && my_tiles > 0) {   // ---------------------------------- MMA issuer
            // S of tile i is issued (once the softmax has read S of tile i-1)
            // before P.V of tile i-1; tile i accumulates into O_(i & 1)
            bool good = at_wait(&sm.q_ready, 0, abort);
            uint32_t ks = 0, kph = 0, vs = 0, vph = 0, i = 0;
            bool pv_pending = false;
            const uint32_t id = idesc_n(128);
            auto issue_pv = [&](uint32_t pi) {   // P.V of tile pi (waits for its P and its V tile)
                const uint32_t h = pi & 1;
                if (!at_wait(&sm.p_full[h], (pi >> 1) & 1, abort)) return false;
                if (!at_wait(&sm.vfull[vs], vph, abort)) return false;
                at_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)   // A = P_h in TMEM, 16 keys (8 columns) per step
                    at_mma_ta(tmem + kTmemO + h * 128, tmem + kTmemP + kk * 8,
                              at_desc(sm.v[vs][kk >> 2]) + 2 * (kk & 3), id, (pi >= 2 || kk > 0) ? 1u : 0u);
                at_commit(&sm.o_done[h]);
                at_commit(&sm.vempty[vs]);
                if (++vs == kAtVStages) { vs = 0; vph ^= 1; }
                return true;
            };
            for (int s = ci; s < n_total && good; s += Ctot) {
                const AtSplit sp = at_split(a, s, n_split_grid, t);
                for (int j = 0; j < sp.ntiles && good; ++j, ++i) {
                    if (!at_wait(&sm.kfull[ks], kph, abort)) { good = false; break; }
                    if (i > 0 && !at_wait(&sm.s_free, (i - 1) & 1, abort)) { good = false; break; }
                    at_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)   // A = Q in TMEM, 16 dims (8 columns) per step
                        at_mma_ta(tmem + kTmemS, tmem + kTmemQ + kk * 8, at_desc(sm.k[ks][kk >> 2]) + 2 * (kk & 3), id,
                                  kk > 0 ? 1u : 0u);
                    at_commit(&sm.s_full[i & 1]);
                    at_commit(&sm.kempty[ks]);
                    if (++ks == kAtKStages) { ks = 0; kph ^= 1; }
                    if (pv_pending && !issue_pv(i - 1)) { good = false; break; }
                    pv_pending = true;
                }
            }
            if (good && pv_pending) issue_pv(i - 1);
        }
        __syncwarp();
    } else if (warp >= kAtSoftWarp0) {   // ---------------------------- softmax, warpgroup h: tiles jj with jj & 1 == h
        pdl_wait();
        const int h = (warp - kAtSoftWarp0) >> 2;
        const int rr = k_lo * g + row;                            // row within the sequence's K*g rows
        const int kblk = rr / g;
        const float scale = 1.4426950408889634f / sqrtf(128.f);
        // exponents are taken relative to m_use, a running max that is only
        // raised (and O rescaled) when a score exceeds it by more than
        // kRescaleSlack: the result is the same softmax, P stays <= 2^slack
        float m_use = -INFINITY, l_run = 0.f;
        int last = -1;   // this warpgroup's last tile
        // tree verify: this row's ancestor bits (rows past the block see nothing
        // of it; they are never written)
        const bool tree = a.mode == 0 && a.tree_mask != nullptr;
        uint32_t tm[4] = {0u, 0u, 0u, 0u};
        if (tree && kblk < k_hi) {
            const uint4 v = *(const uint4 *)(a.tree_mask + (size_t)(b * a.K + kblk) * 4);
            tm[0] = v.x; tm[1] = v.y; tm[2] = v.z; tm[3] = v.w;
        }
        if (h == 0) {   // Q row -> TMEM lane row (bf16 pairs); rows past the block are zero
            uint32_t qr[64];
            if (kblk < k_hi) {
                const uint4 *src = (const uint4 *)((const bf16 *)a.q +
                                                   ((size_t)(b * a.K + kblk) * a.n_q + kvh * g + rr % g) * 128);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint4 v = src[c];
                    qr[4 * c] = v.x; qr[4 * c + 1] = v.y; qr[4 * c + 2] = v.z; qr[4 * c + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) qr[c] = 0u;
            }
            AT_ST32(tmem + lane_off + kTmemQ, qr);
            AT_ST32(tmem + lane_off + kTmemQ + 32, (qr + 32));
            at_wait_st();
            at_fence_before();
            at_arrive(&sm.q_ready);
        }
        for (int s = ci; s < n_total && ok; s += Ctot) {
            const AtSplit sp = at_split(a, s, n_split_grid, t);
            const int lim = min(sp.key1, (sp.block || tree) ? sp.key1 : (a.mode == 0 ? t + kblk + 1 : sp.key1));
            for (int j = 0; j < sp.ntiles; ++j, ++jj) {
                if ((int)(jj & 1) != h) continue;
                last = (int)jj;
                ok = at_wait(&sm.s_full[h], (jj >> 1) & 1, abort);
                if (!ok) break;
                at_fence_after();
                uint32_t sr[128];
#pragma unroll
                for (int q = 0; q < 4; ++q) AT_LD32(tmem + lane_off + kTmemS + q * 32, (sr + q * 32));
                at_wait_ld();
                at_fence_before();
                at_arrive(&sm.s_free);   // S may be overwritten by the next tile
                const int vis = lim - (sp.key0 + j * kAtKeys);   // keys of this tile the row sees
                if (vis < kAtKeys) {
#pragma unroll
                    for (int c = 0; c < kAtKeys; ++c)
                        if (c >= vis) sr[c] = __float_as_uint(-INFINITY);
                }
                const int j0 = sp.key0 + j * kAtKeys - t;          // block index of this tile's first key
                if (tree && j0 + kAtKeys > 0) {                    // the tile reaches the block
                    uint32_t wv[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) wv[i] = tree_window(tm, j0 + 32 * i);
#pragma unroll
                    for (int c = 0; c < kAtKeys; ++c)
                        if (!((wv[c >> 5] >> (c & 31)) & 1u)) sr[c] = __float_as_uint(-INFINITY);
                }
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < kAtKeys; ++c) mx[c & 3] = fmaxf(mx[c & 3], __uint_as_float(sr[c]));
                const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale;
                float alpha = 1.0f;
                if (tmax > m_use + kRescaleSlack || (m_use == -INFINITY && tmax > -INFINITY)) {
                    alpha = m_use == -INFINITY ? 0.f : ex2(m_use - tmax);
                    m_use = tmax;
                }
                const float nmu = m_use == -INFINITY ? 0.f : -m_use;
                // P row: 64 bf16 pairs (the P.V A operand), computed while the
                // P.V of tile jj-1 may still be reading P
                float rs[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t pk[kAtKeys / 2];
#pragma unroll
                for (int c = 0; c < kAtKeys / 2; ++c) {
                    const float p0v = ex2(fmaf(__uint_as_float(sr[2 * c]), scale, nmu));
                    const float p1v = ex2(fmaf(__uint_as_float(sr[2 * c + 1]), scale, nmu));
                    rs[c & 3] += p0v + p1v;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0v, p1v);
                    pk[c] = *(const uint32_t *)&h2;
                }
                if (jj >= 1) {   // P.V of tile jj-1 done (so that of tile jj-2 too): P and O_h are free
                    ok = at_wait(&sm.o_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, abort);
                    if (!ok) break;
                    at_fence_after();
                }
                // P row -> TMEM lane row
#pragma unroll
                for (int q = 0; q < 4; ++q) AT_ST16(tmem + lane_off + kTmemP + q * 16, (pk + 16 * q));
                if (jj >= 2 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t orr[32];
                        AT_LD32(tmem + lane_off + kTmemO + h * 128 + q * 32, orr);
                        at_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
                        AT_ST32(tmem + lane_off + kTmemO + h * 128 + q * 32, orr);
                    }
                }
                at_wait_st();
                at_fence_before();
                at_arrive(&sm.p_full[h]);
                l_run = l_run * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
            }
        }
        // this warpgroup's last P.V (tcgen05 operations complete in issue order)
        if (ok && last >= 0) ok = at_wait(&sm.o_done[h], (last >> 1) & 1, abort);
        sm.xml[h][row] = (ok && last >= 0) ? make_float2(m_use, l_run) : make_float2(-INFINITY, 0.f);
        at_fence_after();
        __syncwarp();
    }

    // ------------------------------------------------------------------ combine
    unsigned char *area = sm.k[0][0];
    const uint32_t area_u = smem_u32(area);
    if (warp >= kAtSoftWarp0) {
        const int h = (warp - kAtSoftWarp0) >> 2;
        asm volatile("bar.sync 1, 256;\n" ::: "memory");   // both warpgroups: every P.V is done
        // merge the two accumulators into the normalised row o = O / l and
        // stage it (the K/V ring is no longer read) as fp16 scaled by the
        // largest |o| of each half row, so every staged value lies in
        // [-1, 1]; warpgroup h takes dims [64h, 64h + 64)
        const float2 x0 = sm.xml[0][row], x1 = sm.xml[1][row];
        const float M = fmaxf(x0.x, x1.x);
        const float w0 = x0.y > 0.f ? ex2(x0.x - M) : 0.f, w1 = x1.y > 0.f ? ex2(x1.x - M) : 0.f;
        const float l = w0 * x0.y + w1 * x1.y;
        float y[64];
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
            uint32_t o0[32], o1[32];
            AT_LD32(tmem + lane_off + kTmemO + (2 * h + qq) * 32, o0);
            AT_LD32(tmem + lane_off + kTmemO + 128 + (2 * h + qq) * 32, o1);
            at_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float y0 = w0 != 0.f ? w0 * __uint_as_float(o0[e]) : 0.f;
                const float y1 = w1 != 0.f ? w1 * __uint_as_float(o1[e]) : 0.f;
                y[32 * qq + e] = y0 + y1;
            }
        }
        if (C == 1 && Z == 1) {   // a lone CTA: this row is final, write it from registers
            const int rr1 = k_lo * g + row, k1 = rr1 / g;
            if (!*abort && k1 < k_hi && l > 0.f) {
                const float inv = 1.0f / l;
                bf16 *o = (bf16 *)a.out + ((size_t)(b * a.K + k1) * a.n_q + kvh * g + rr1 % g) * 128 + 64 * h;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    uint32_t u[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(y[8 * c + 2 * e] * inv, y[8 * c + 2 * e + 1] * inv);
                        u[e] = *(const uint32_t *)&b2;
                    }
                    *(uint4 *)(o + 8 * c) = make_uint4(u[0], u[1], u[2], u[3]);
                }
            }
        } else {
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 64; ++e) amax = fmaxf(amax, fabsf(y[e]));
        const float sc = l > 0.f ? amax / l : 0.f;             // max |o| over the half row
        const float r = amax > 0.f ? 1.0f / amax : 0.f;        // o / sc = y / amax
        unsigned char *so = area + kStageO + row * 256;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __half2 h2 = __floats2half2_rn(y[8 * c + 2 * e] * r, y[8 * c + 2 * e + 1] * r);
                u[e] = *(const uint32_t *)&h2;
            }
            *(uint4 *)(so + (((8 * h + c) ^ (row & 15)) << 4)) = make_uint4(u[0], u[1], u[2], u[3]);
        }
        float *ml = (float *)(area + kStageMl) + row * 4;   // (m, l, scale of dims 0-63, scale of dims 64-127)
        if (h == 0) { ml[0] = l > 0.f ? M : -INFINITY; ml[1] = l > 0.f ? l : 0.f; }
        ml[2 + h] = sc;
        at_fence_before();
        }
        __syncwarp();
    }
    // every CTA's merged rows are in its shared memory (release / acquire)
    cluster_arrive();
    cluster_wait();
    if (warp >= kAtSoftWarp0 && !(C == 1 && Z == 1)) {   // ------- owner: rows [r*rpc, (r+1)*rpc), pulled from every CTA
        constexpr int tpr = 256 / rpc;            // threads per owned row: chunks cc, cc + tpr, ...
        constexpr int cpt = 16 / tpr;             // 8-dim chunks per thread
        static_assert(cpt >= 1, "cluster too large for the owner split");
        const int et = threadIdx.x - 32 * kAtSoftWarp0;
        const int rl = et / tpr, cc = et % tpr;
        const int orow = r * rpc + rl;
        uint32_t peer[C];
#pragma unroll
        for (int c = 0; c < C; ++c) peer[c] = map_peer_addr(area_u, c);
        float4 mls[C];
        uint4 hv[cpt][C];
#pragma unroll
        for (int c = 0; c < C; ++c) mls[c] = ld_peer4(peer[c] + kStageMl + orow * 16);
#pragma unroll
        for (int i = 0; i < cpt; ++i) {
            const int ch = cc + i * tpr;
#pragma unroll
            for (int c = 0; c < C; ++c) hv[i][c] = ld_peer4u(peer[c] + kStageO + orow * 256 + ((ch ^ (orow & 15)) << 4));
        }
        float Mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < C; ++c)
            if (mls[c].y > 0.f) Mx = fmaxf(Mx, mls[c].x);
        float wc[C], L = 0.f;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            wc[c] = mls[c].y > 0.f ? ex2(mls[c].x - Mx) * mls[c].y : 0.f;   // weight x row sum
            L += wc[c];
        }
        const float invL = L > 0.f ? 1.0f / L : 0.f;
        const int rrow = k_lo * g + orow, k = rrow / g, jh = rrow % g;
        const bool vrow = orow < (k_hi - k_lo) * g;
        float yo[cpt][8];   // the cluster's normalised row, dims 8 ch .. 8 ch + 7, CTAs in rank order
#pragma unroll
        for (int i = 0; i < cpt; ++i) {
            const int ch = cc + i * tpr;
#pragma unroll
            for (int e = 0; e < 8; ++e) yo[i][e] = 0.f;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                if (wc[c] == 0.f) continue;
                const float f = wc[c] * invL * (ch < 8 ? mls[c].z : mls[c].w);
                const __half2 *h2 = (const __half2 *)&hv[i][c];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 v = __half22float2(h2[e]);
                    yo[i][2 * e] = fmaf(f, v.x, yo[i][2 * e]);
                    yo[i][2 * e + 1] = fmaf(f, v.y, yo[i][2 * e + 1]);
                }
            }
        }
        const size_t orow_g = (size_t)(b * a.K + k) * a.n_q + kvh * g + jh;   // (token, query head) of the row
        bf16 *o = (bf16 *)a.out + orow_g * 128;
        auto store = [&](int i, const float *v) {
            uint32_t u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                u[e] = *(const uint32_t *)&b2;
            }
            *(uint4 *)(o + (cc + i * tpr) * 8) = make_uint4(u[0], u[1], u[2], u[3]);
        };
        if (Z == 1) {
            if (!*abort && vrow && L > 0.f) {
#pragma unroll
                for (int i = 0; i < cpt; ++i) store(i, yo[i]);
            }
        } else if constexpr (C >= kAtZCluster) {   // (the host picks Z > 1 only with C >= 4)
            // Z clusters: each leaves its normalised row and (Mx, L) in global
            // memory; the last of them (an atomic ticket) merges all Z in
            // cluster order, so the result does not depend on the order they
            // finished in
            const size_t xs = (size_t)a.xrows;
            if (vrow) {
                float4 *xo = (float4 *)(a.xo + ((size_t)zc * xs + orow_g) * 128);
#pragma unroll
                for (int i = 0; i < cpt; ++i) {
                    const int ch = cc + i * tpr;
                    __stcg(xo + 2 * ch, make_float4(yo[i][0], yo[i][1], yo[i][2], yo[i][3]));
                    __stcg(xo + 2 * ch + 1, make_float4(yo[i][4], yo[i][5], yo[i][6], yo[i][7]));
                }
                if (cc == 0) __stcg(a.xml + (size_t)zc * xs + orow_g, make_float2(Mx, L));
            }
            asm volatile("bar.sync 1, 256;\n" ::: "memory");
            const int cidx = ((b * rgroups + rg) * a.n_kv + kvh) * C + r;
            if (et == 0) {
                __threadfence();
                sm.xticket = atomicAdd(a.xcnt + cidx, 1);
            }
            asm volatile("bar.sync 1, 256;\n" ::: "memory");
            if (sm.xticket == Z - 1) {
                __threadfence();
                if (vrow) {
                    // every other cluster's row, all loads in flight at once
                    float2 mlz[kAtMaxZ];
                    float4 az[kAtMaxZ][cpt][2];
#pragma unroll
                    for (int z = 0; z < kAtMaxZ; ++z) {
                        if (z < Z && z != zc) {
                            mlz[z] = __ldcg(a.xml + (size_t)z * xs + orow_g);
                            const float4 *xq = (const float4 *)(a.xo + ((size_t)z * xs + orow_g) * 128);
#pragma unroll
                            for (int i = 0; i < cpt; ++i) {
                                const int ch = cc + i * tpr;
                                az[z][i][0] = __ldcg(xq + 2 * ch);
                                az[z][i][1] = __ldcg(xq + 2 * ch + 1);
                            }
                        } else {
                            mlz[z] = make_float2(Mx, L);
#pragma unroll
                            for (int i = 0; i < cpt; ++i) {
                                az[z][i][0] = make_float4(yo[i][0], yo[i][1], yo[i][2], yo[i][3]);
                                az[z][i][1] = make_float4(yo[i][4], yo[i][5], yo[i][6], yo[i][7]);
                            }
                        }
                    }
                    float Mf = -INFINITY;
#pragma unroll
                    for (int z = 0; z < kAtMaxZ; ++z)
                        if (z < Z && mlz[z].y > 0.f) Mf = fmaxf(Mf, mlz[z].x);
                    float wz[kAtMaxZ], Lf = 0.f;
#pragma unroll
                    for (int z = 0; z < kAtMaxZ; ++z) {
                        wz[z] = (z < Z && mlz[z].y > 0.f) ? ex2(mlz[z].x - Mf) * mlz[z].y : 0.f;
                        Lf += wz[z];
                    }
                    if (!*abort && Lf > 0.f) {
                        const float inv = 1.0f / Lf;
#pragma unroll
                        for (int i = 0; i < cpt; ++i) {
                            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                            for (int z = 0; z < kAtMaxZ; ++z) {
                                if (wz[z] == 0.f) continue;
                                const float f = wz[z] * inv;
                                const float *s0 = &az[z][i][0].x, *s1 = &az[z][i][1].x;
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    v[e] = fmaf(f, s0[e], v[e]);
                                    v[4 + e] = fmaf(f, s1[e], v[4 + e]);
                                }
                            }
                            store(i, v);
                        }
                    }
                }
                if (et == 0) a.xcnt[cidx] = 0;   // ready for the next call
            }
        }
        __syncwarp();
    }
    // no CTA leaves while another may still be reading its shared memory
    cluster_arrive_relaxed();
    cluster_wait();

    if (sm.abort && threadIdx.x == 0) raise_err(a.err, ORTHRUS_DEVERR_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        at_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
    }
}

// ---------------------------------------------------------------- host
bool make_tmap(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool make_tmap_box(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_cols, uint32_t box_rows);

size_t attn_tc_smem_bytes() { return sizeof(AtSmem) + 1024; }

// CTAs of this kernel in C-CTA clusters that the GPU holds at once (one CTA
// per SM), for C = 1, 2, 4, 8: measured by attn_tc_init_attributes; the
// defaults are B200's (148 SMs, clusters confined to a GPC).
static int g_cluster_ctas[4] = {148, 148, 132, 120};
static int cluster_ctas(int C) { return g_cluster_ctas[C >= 8 ? 3 : C >= 4 ? 2 : C >= 2 ? 1 : 0]; }

// CTAs per (sequence, KV head, row group): the largest power of two up to 8
// (the portable cluster size; 16-CTA clusters measured slower on B200: fewer
// than eight of them fit on the GPU at once) that keeps one row group of the
// whole batch within one wave.  A function of the batch and model shape only
// (not of the block size), so a row is reduced in the same order whatever
// block it is in.
int attn_cluster_size(int n_kv, int B)
{
    const int others = n_kv * B;
    int C = 1;
    while (C < kAtMaxCluster && (2 * C) * others <= cluster_ctas(2 * C)) C *= 2;
    return C;
}

template <int C> static cudaError_t at_prepare(int bytes, int *ctas)
{
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, C);
    cfg.blockDim = dim3(kAtThreads);
    cfg.dynamicSmemBytes = bytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = C;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel<C>, &cfg);
    if (e == cudaSuccess && n > 0) *ctas = std::min(n * C, kNumSMs);
    return e;
}

cudaError_t attn_tc_init_attributes()
{
    const int bytes = (int)attn_tc_smem_bytes();
    cudaError_t e = at_prepare<1>(bytes, &g_cluster_ctas[0]);
    if (e == cudaSuccess) e = at_prepare<2>(bytes, &g_cluster_ctas[1]);
    if (e == cudaSuccess) e = at_prepare<4>(bytes, &g_cluster_ctas[2]);
    if (e == cudaSuccess) e = at_prepare<8>(bytes, &g_cluster_ctas[3]);
    return e;
}

// Tensor maps for one call (Q rows are read with plain 16-byte loads).
bool attn_tc_maps(const AttnArgs &a, int n_layers, AtMaps *m)
{
    memset(m, 0, sizeof(*m));
    const int g = a.n_q / a.n_kv;
    if (a.hd != 128 || kAtRows % g || a.kv.page_size % 64 || ((uintptr_t)a.q & 15)) return false;
    const uint64_t heads = (uint64_t)n_layers * a.kv.num_pages * a.n_kv;
    if (!make_tmap_box(&m->kc, a.kv.k_pages, heads * a.kv.page_size, 128, 64, 64)) return false;
    if (!make_tmap_box(&m->vc, a.kv.v_pages, heads * 128, a.kv.page_size, 64, 128)) return false;
    if (a.mode == 1) {
        const uint64_t bh = (uint64_t)a.blk_layers * a.bmax * a.n_kv;
        if (!make_tmap_box(&m->kb, a.k_blk, bh * a.kp, 128, 64, 64)) return false;
        if (!make_tmap_box(&m->vb, a.v_blk, bh * 128, a.kp, 64, 128)) return false;
    } else {
        m->kb = m->kc;
        m->vb = m->vc;
    }
    return true;
}

// Maps for the call, built once per distinct (buffers, shape) and kept in
// the context.
cudaError_t launch_attn_tc_cached(const Ctx &c, const AttnArgs &a, int n_split_grid, int q_rows, cudaStream_t s)
{
    if (!attn_tc_shape_ok(c.cfg.dtype, a.hd, a.n_q, a.n_kv, a.kv.page_size)) return cudaErrorNotSupported;
    AttnMapKey key{a.q, a.kv.k_pages, a.kv.v_pages, a.k_blk, a.kv.num_pages, a.kv.page_size, a.K, a.mode, q_rows};
    auto it = c.amaps.find(key);
    if (it == c.amaps.end()) {
        AtMaps m;
        if (!attn_tc_maps(a, c.cfg.n_layers, &m)) return cudaErrorNotSupported;
        it = c.amaps.emplace(key, std::vector<unsigned char>((unsigned char *)&m, (unsigned char *)&m + sizeof(m))).first;
    }
    c.launches += 1;
    return launch_attn_tc(a, *(const AtMaps *)it->second.data(), n_split_grid, s);
}

cudaError_t launch_attn_tc(const AttnArgs &a, const AtMaps &maps, int n_split_grid, cudaStream_t s)
{
    const int g = a.n_q / a.n_kv;
    const int ksub = kAtRows / g;
    const int rgroups = (a.K + ksub - 1) / ksub;
    int C = attn_cluster_size(a.n_kv, a.B);
    AttnArgs x = a;
    x.xz = 1;
    if (a.xz > 1 && a.xo && a.xml && a.xcnt) {
        // long contexts: Z clusters of 4 per row group, all of them within
        // one wave of four-CTA clusters
        const int Cz = std::min(C, kAtZCluster);
        int Z = 1;
        // (clusters smaller than 4 mean a batch too wide for two of them)
        while (Cz == kAtZCluster && Z < std::min(a.xz, kAtMaxZ) && 2 * Z * Cz * a.n_kv * a.B <= cluster_ctas(Cz)) Z *= 2;
        if (Z > 1) { C = Cz; x.xz = Z; }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.n_kv, a.B * rgroups, C * x.xz);
    cfg.blockDim = dim3(kAtThreads);
    cfg.dynamicSmemBytes = attn_tc_smem_bytes();
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = C;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    switch (C) {
    case 1: return cudaLaunchKernelEx(&cfg, attn_tc_kernel<1>, maps, x, n_split_grid);
    case 2: return cudaLaunchKernelEx(&cfg, attn_tc_kernel<2>, maps, x, n_split_grid);
    case 4: return cudaLaunchKernelEx(&cfg, attn_tc_kernel<4>, maps, x, n_split_grid);
    default: return cudaLaunchKernelEx(&cfg, attn_tc_kernel<8>, maps, x, n_split_grid);
    }
}

}  // namespace orthrus
