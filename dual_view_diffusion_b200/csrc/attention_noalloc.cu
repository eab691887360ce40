// Dual-view attention for callers that cannot allocate device memory.
//
// orthrus_dual_view_attention needs a context, and a context needs a
// workspace that the caller allocates.  Some callers cannot do that: a
// serving runtime that reserves the whole HBM pool for its own allocator at
// start-up (a cudaMalloc from a plugin then fails, or steals memory the pool
// was promised), or a caller on a latency-critical path where cudaMalloc /
// cudaFree would synchronise the device and stall every other stream.  This
// variant runs the same kernels with their split partials in a fixed array
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
        kv->max_pages_per_seq < 1 || kv->page_size < 16 || kv->page_size % 16)
        return ORTHRUS_ERR_INVALID_ARG;
    if (cfg->n_q_heads < 1 || cfg->n_kv_heads < 1 || cfg->n_q_heads % cfg->n_kv_heads || layer < 0 ||
        layer >= cfg->n_layers || (cfg->dtype != ORTHRUS_BF16 && cfg->dtype != ORTHRUS_FP32) ||
        cfg->split_tokens < 64 || cfg->split_tokens % 64 || cfg->max_seq < K + 1)
        return ORTHRUS_ERR_INVALID_ARG;
    if (cfg->head_dim != 16 && cfg->head_dim != 32 && cfg->head_dim != 64 && cfg->head_dim != 128)
        return ORTHRUS_ERR_INVALID_ARG;
    if (cfg->dtype == ORTHRUS_BF16 && cfg->head_dim == 128 && kv->page_size % 64) return ORTHRUS_ERR_INVALID_ARG;

    // carve: [error word][block-table rows][block K][block V][(m, l) per
    // split][O partial per split]
    const size_t rows = (size_t)batch * K;
    const size_t es = cfg->dtype == ORTHRUS_BF16 ? 2 : 4;
    const size_t kp = ((size_t)K + 63) / 64 * 64;
    const size_t n_splits = ((size_t)cfg->max_seq + cfg->split_tokens - 1) / cfg->split_tokens + 1;
    const size_t blk = (size_t)batch * cfg->n_kv_heads * kp * cfg->head_dim * es;
    const size_t off_rows = 256;
    const size_t off_kb = off_rows + up256((size_t)batch * 4);
    const size_t off_vb = off_kb + up256(mode == 1 ? blk : 0);
    const size_t off_ml = off_vb + up256(mode == 1 ? blk : 0);
    // split partials: SIMT attention only (the tensor-core path combines on chip)
    const bool simt_attn = !(cfg->dtype == ORTHRUS_BF16 && cfg->head_dim == 128);
    const size_t off_part = off_ml + up256(simt_attn ? rows * cfg->n_q_heads * n_splits * sizeof(float2) : 0);
    const size_t need = off_part + (simt_attn ? rows * cfg->n_q_heads * n_splits * cfg->head_dim * sizeof(float) : 0);
    if (need > kNoAllocScratchBytes) return ORTHRUS_ERR_CAPACITY;

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
    cudaStream_t s = (cudaStream_t)stream;
    unsigned *err = dev_err ? (unsigned *)dev_err : (unsigned *)base;
    int32_t *bt_rows = (int32_t *)(base + off_rows);
    if (cudaMemsetAsync(err, 0, sizeof(unsigned), s) != cudaSuccess) return ORTHRUS_ERR_CUDA;
    if (launch_k(noalloc_identity_rows, (batch + 127) / 128, 128, 0, s, bt_rows, (int)batch) != cudaSuccess)
        return ORTHRUS_ERR_CUDA;

    Ctx tmp;                      // only cfg (and a tensor-map cache) is used by the launchers
    tmp.cfg = *cfg;
    AttnArgs at{};
    if (mode == 1) {
        if (launch_pack_block(tmp, k_blk, v_blk, base + off_kb, base + off_vb, batch, K, (int)kp, s) != cudaSuccess)
            return ORTHRUS_ERR_CUDA;
        at.k_blk = base + off_kb; at.v_blk = base + off_vb;
    }
    at.kp = (int)kp; at.bmax = batch; at.blk_layer = 0; at.blk_layers = 1;
    at.q = q; at.out = out;
    at.kv = KvView{kv->k_pages, kv->v_pages, kv->block_table, kv->num_pages, kv->page_size, kv->max_pages_per_seq};
    at.layer = layer; at.seq_lens = kv->seq_lens; at.bt_rows = bt_rows;
    at.B = batch; at.K = K; at.n_q = cfg->n_q_heads; at.n_kv = cfg->n_kv_heads; at.hd = cfg->head_dim;
    at.mode = mode; at.split_tokens = cfg->split_tokens; at.n_splits = (int)n_splits;
    at.part = (float *)(base + off_part); at.ml = (float2 *)(base + off_ml); at.err = err;
    if (launch_attention(tmp, at, s, batch * K) != cudaSuccess) return ORTHRUS_ERR_CUDA;
    return ORTHRUS_OK;
}
