// Dual-view attention for callers that cannot allocate device memory.
//
// orthrus_dual_view_attention needs a context, and a context needs a
// workspace that the caller allocates.  Some callers cannot do that: a
// serving runtime that reserves the whole HBM pool for its own allocator at
// start-up (a cudaMalloc from a plugin then fails, or steals memory the pool
// was promised), or a caller on a latency-critical path where cudaMalloc /
// cudaFree would synchronise the device and stall every other stream.  This
// variant runs the same kernels, with the same launch shapes as the workspace
// entry point for the same config, and keeps their scratch in a fixed array
// that the library itself holds on every GPU it is loaded on.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace orthrus {

// Size of the fixed scratch array; every GPU that loads the library holds it
// until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_attn_scratch[kNoAllocScratchBytes];

// Device address of g_attn_scratch per device (host code may not use the
// symbol itself as an address: on the host it names a stand-in object).
static unsigned char *g_scratch_dev[kNoAllocMaxDevices];
static std::mutex g_scratch_mu;

__global__ void noalloc_identity_rows(int32_t *rows, int n)
{
    // no early pdl_trigger: the attention reads these rows before its
    // griddepcontrol.wait, so it may not be scheduled until this kernel exits
    pdl_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) rows[i] = i;
}

static size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace orthrus

using namespace orthrus;

extern "C" orthrus_status_t orthrus_dual_view_attention_noalloc(const orthrus_config_t *cfg, const orthrus_kv_t *kv,
                                                                int32_t layer, int32_t mode, const void *q,
                                                                const void *k_blk, const void *v_blk, int32_t batch,
                                                                int32_t K, void *out, uint32_t *dev_err, void *stream)
{
    if (!cfg || !kv || !q || !out || batch < 1 || K < 1 || (mode != 0 && mode != 1) ||
        (mode == 1 && (!k_blk || !v_blk)))
        return ORTHRUS_ERR_INVALID_ARG;
    if (!kv->k_pages || !kv->v_pages || !kv->block_table || !kv->seq_lens || kv->num_pages < 1 ||
        kv->max_pages_per_seq < 1 || kv->page_size < 16 || kv->page_size % 16 || (uintptr_t)kv->k_pages % 16 ||
        (uintptr_t)kv->v_pages % 16)
        return ORTHRUS_ERR_INVALID_ARG;
    if (cfg->n_q_heads < 1 || cfg->n_kv_heads < 1 || cfg->n_q_heads % cfg->n_kv_heads || layer < 0 ||
        layer >= cfg->n_layers || (cfg->dtype != ORTHRUS_BF16 && cfg->dtype != ORTHRUS_FP32) ||
        cfg->split_tokens < 64 || cfg->split_tokens % 64 || cfg->max_seq < K + 1)
        return ORTHRUS_ERR_INVALID_ARG;
    if (cfg->head_dim != 16 && cfg->head_dim != 32 && cfg->head_dim != 64 && cfg->head_dim != 128)
        return ORTHRUS_ERR_INVALID_ARG;
    if (cfg->dtype == ORTHRUS_BF16 && cfg->head_dim == 128 && kv->page_size % 64) return ORTHRUS_ERR_INVALID_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ORTHRUS_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return ORTHRUS_ERR_UNSUPPORTED;
    unsigned char *base;
    {
        std::lock_guard<std::mutex> lk(g_scratch_mu);
        if (!g_scratch_dev[dev]) {   // first call on this device: its set-up
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) return ORTHRUS_ERR_CUDA;
            if (attention_init_attributes() != cudaSuccess) return ORTHRUS_ERR_CUDA;
            g_scratch_dev[dev] = (unsigned char *)p;
        }
        base = g_scratch_dev[dev];
    }

    // carve, in order: [error word][block-table rows][block K][block V
    // transposed] and then the chosen kernel's own scratch — the
    // cross-cluster merge rows, (m, l) and tickets of the tensor-core kernel
    // on long contexts, or the split partials of the SIMT kernel
    const size_t rows = (size_t)batch * K, nq = cfg->n_q_heads, hd = cfg->head_dim;
    const size_t es = cfg->dtype == ORTHRUS_BF16 ? 2 : 4;
    const size_t kp = ((size_t)K + 63) / 64 * 64;
    const size_t n_splits = ((size_t)cfg->max_seq + cfg->split_tokens - 1) / cfg->split_tokens + 1;
    const size_t blk = (size_t)batch * cfg->n_kv_heads * kp * hd * es;
    const size_t off_rows = 256;
    const size_t off_kb = off_rows + up256((size_t)batch * 4);
    const size_t off_vb = off_kb + up256(mode == 1 ? blk : 0);
    const size_t off_x = off_vb + up256(mode == 1 ? blk : 0);
    if (off_x > kNoAllocScratchBytes) return ORTHRUS_ERR_CAPACITY;

    cudaStream_t s = (cudaStream_t)stream;
    unsigned *err = dev_err ? (unsigned *)dev_err : (unsigned *)base;
    int32_t *bt_rows = (int32_t *)(base + off_rows);
    AttnArgs at{};
    if (mode == 1) { at.k_blk = base + off_kb; at.v_blk = base + off_vb; }
    at.kp = (int)kp; at.bmax = batch; at.blk_layer = 0; at.blk_layers = 1;
    at.q = q; at.out = out;
    at.kv = KvView{kv->k_pages, kv->v_pages, kv->block_table, kv->num_pages, kv->page_size, kv->max_pages_per_seq};
    at.layer = layer; at.seq_lens = kv->seq_lens; at.bt_rows = bt_rows;
    at.B = batch; at.K = K; at.n_q = cfg->n_q_heads; at.n_kv = cfg->n_kv_heads; at.hd = cfg->head_dim;
    at.mode = mode; at.split_tokens = cfg->split_tokens; at.n_splits = (int)n_splits; at.err = err;

    // The path is decided here, before anything is counted or launched, by
    // the same test the workspace entry point applies (shape, then tensor
    // maps over these very buffers), so the scratch counted is the scratch
    // the launched kernels write.
    AtMaps maps;
    const bool tc = attn_tc_shape_ok(cfg->dtype, cfg->head_dim, cfg->n_q_heads, cfg->n_kv_heads, kv->page_size) &&
                    attn_tc_maps(at, cfg->n_layers, &maps);
    size_t need = off_x, off_a = off_x, off_b = off_x, off_c = off_x;
    if (tc) {
        // contexts this long take up to kAttnMaxClusters clusters per row
        // group, merged through rows left in memory, as the workspace entry
        // point does for the same config
        if (cfg->max_seq >= kAttnTwoClusterSeq) {
            off_b = off_a + up256(kAttnMaxClusters * rows * nq * hd * 4);
            off_c = off_b + up256(kAttnMaxClusters * rows * nq * 8);
            need = off_c + rows * cfg->n_kv_heads * 8 * 4;
            at.xo = (float *)(base + off_a); at.xml = (float2 *)(base + off_b); at.xcnt = (int *)(base + off_c);
            at.xrows = (int)(rows * nq); at.xz = kAttnMaxClusters;
        } else {
            at.xz = 1;
        }
    } else {
        off_b = off_a + up256(rows * nq * n_splits * sizeof(float2));
        need = off_b + rows * nq * n_splits * hd * sizeof(float);
        at.ml = (float2 *)(base + off_a); at.part = (float *)(base + off_b);
    }
    if (need > kNoAllocScratchBytes) return ORTHRUS_ERR_CAPACITY;

    if (cudaMemsetAsync(err, 0, sizeof(unsigned), s) != cudaSuccess) return ORTHRUS_ERR_CUDA;
    // the merge tickets must start at zero; earlier calls may have left other
    // data at this offset
    if (at.xcnt && cudaMemsetAsync(at.xcnt, 0, rows * cfg->n_kv_heads * 8 * 4, s) != cudaSuccess)
        return ORTHRUS_ERR_CUDA;
    if (launch_k(noalloc_identity_rows, (batch + 127) / 128, 128, 0, s, bt_rows, (int)batch) != cudaSuccess)
        return ORTHRUS_ERR_CUDA;
    Ctx tmp;                      // only cfg is read by the launchers below
    tmp.cfg = *cfg;
    if (mode == 1 && launch_pack_block(tmp, k_blk, v_blk, base + off_kb, base + off_vb, batch, K, (int)kp, s) !=
                         cudaSuccess)
        return ORTHRUS_ERR_CUDA;
    const int n_split_grid = (cfg->max_seq + cfg->split_tokens - 1) / cfg->split_tokens;
    const cudaError_t e = tc ? launch_attn_tc(at, maps, n_split_grid, s) : launch_attention_simt(tmp, at, s);
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_CUDA;
}
