// Device helpers shared by the kernels of the dual-view decode library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <limits.h>
#include <stdint.h>

#include "../../include/orthrus.h"

namespace orthrus {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------- dtype
template <class T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 x) { return __bfloat162float(x); }

template <class T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// ---------------------------------------------------------------- errors
__device__ __forceinline__ void raise_err(unsigned *err, unsigned bit) { atomicOr(err, bit); }

// ---------------------------------------------------------------- RNG
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of two
// 32x32->64 multiplies, key bumped by the Weyl constants between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k)
{
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
        c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
        k.x += 0x9E3779B9u;
        k.y += 0xBB67AE85u;
    }
    return c;
}

enum Purpose : uint32_t { PURPOSE_DRAFT = 1, PURPOSE_ACCEPT = 2, PURPOSE_RESIDUAL = 3, PURPOSE_AR = 4 };

// The uniform u = (k + 1/2) / 2^24 in (0, 1), k = the top 24 bits of the
// first output word of Philox4x32-10 at counter (id, row, step, purpose) and
// key = seed, is only ever used through -log(u), returned here.  u itself is
// not an fp32 number once k >= 2^23 (k + 1/2 then needs 25 bits), and
// rounding it would move -log(u) by up to 2^-25 / (1 - u) relative: for the
// draws nearest 1, which decide Gumbel-max winners, that is ~1e-3.  So for
// u > 1/2 the exact complement 1 - u = (2^24 - 1 - k + 1/2) / 2^24 (fewer
// than 24 significant bits) goes through log1p.
__device__ __forceinline__ float neg_log_uniform(uint64_t seed, uint32_t step, uint32_t row, uint32_t id,
                                                 uint32_t purpose)
{
    const uint4 o = philox4x32_10(make_uint4(id, row, step, purpose),
                                  make_uint2((uint32_t)seed, (uint32_t)(seed >> 32)));
    const uint32_t k = o.x >> 8;
    constexpr float kInv24 = 1.0f / 16777216.0f;
    if (k < (1u << 23)) return -logf(((float)k + 0.5f) * kInv24);
    return -log1pf(-(((float)((1u << 24) - 1u - k) + 0.5f) * kInv24));
}

// Gumbel noise -log(-log u) of the same uniform.
__device__ __forceinline__ float gumbel(uint64_t seed, uint32_t step, uint32_t row, uint32_t id, uint32_t purpose)
{
    return -logf(neg_log_uniform(seed, step, row, id, purpose));
}

// Row id used in the RNG counter: sequence b, block row k.
__device__ __forceinline__ uint32_t rng_row(int b, int k) { return ((uint32_t)b << 16) | (uint32_t)k; }

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// (value, index) max with the lowest index winning ties; NaN never wins.
__device__ __forceinline__ void argmax_merge(float &v, int &i, float v2, int i2)
{
    if (v2 > v || (v2 == v && i2 < i)) { v = v2; i = i2; }
}

__device__ __forceinline__ void warp_argmax(float &v, int &i)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
        argmax_merge(v, i, v2, i2);
    }
}

// ---------------------------------------------------------------- top-W lists
// Sorted (best first) lists of the kTopWMax largest (value, id) pairs; ties
// go to the lowest id.  Unused entries hold (-inf, INT_MAX).
constexpr int kTopWMax = 8;

__device__ __forceinline__ bool tw_better(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

// One lane's sorted list (best first) gives up its head.
__device__ __forceinline__ void tw_pop(float (&v)[kTopWMax], int (&i)[kTopWMax])
{
#pragma unroll
    for (int j = 0; j + 1 < kTopWMax; ++j) { v[j] = v[j + 1]; i[j] = i[j + 1]; }
    v[kTopWMax - 1] = -INFINITY;
    i[kTopWMax - 1] = INT_MAX;
}

// The warp's kTopWMax best entries over all lanes' sorted lists, best
// first, into ov/oi (every lane gets the same result).  Ids are distinct
// across lanes, so the winner of a round is one lane.
__device__ __forceinline__ void tw_warp_merge(float (&v)[kTopWMax], int (&i)[kTopWMax], float *ov, int *oi)
{
#pragma unroll 1
    for (int r = 0; r < kTopWMax; ++r) {
        float bv = v[0];
        int bi = i[0];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov2 = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi2 = __shfl_xor_sync(0xffffffffu, bi, off);
            if (tw_better(ov2, oi2, bv, bi)) { bv = ov2; bi = oi2; }
        }
        if (i[0] == bi && bi != INT_MAX) tw_pop(v, i);
        ov[r] = bv;
        oi[r] = bi;
    }
}

// A logit into a thread's sorted top list (the common case is one compare).
__device__ __forceinline__ void tw_insert(float x, int v, float (&tv)[kTopWMax], int (&ti)[kTopWMax])
{
    if (tw_better(x, v, tv[kTopWMax - 1], ti[kTopWMax - 1])) {
        tv[kTopWMax - 1] = x;
        ti[kTopWMax - 1] = v;
#pragma unroll
        for (int j = kTopWMax - 1; j > 0; --j)
            if (tw_better(tv[j], ti[j], tv[j - 1], ti[j - 1])) {
                const float a = tv[j]; tv[j] = tv[j - 1]; tv[j - 1] = a;
                const int b = ti[j]; ti[j] = ti[j - 1]; ti[j - 1] = b;
            }
    }
}

// ---------------------------------------------------------------- async copy
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

// 16-byte cp.async; bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// ---------------------------------------------------------------- PDL
// Every kernel of the library is launched with programmatic stream
// serialisation: it may be scheduled while its predecessor is finishing, and
// it waits (griddepcontrol.wait) before touching anything a predecessor
// wrote.  Both instructions are no-ops for a kernel launched without it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, ((KArgs)args)...);
}

}  // namespace orthrus
