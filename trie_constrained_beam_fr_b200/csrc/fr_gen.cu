// fr_gen.cu -- libfr_gen: the workload's seeded hash logits on the GPU.
//
// Makes INPUTS only (see fr_gen.h for the definition of the values); holds
// none of the beam-search arithmetic.  SplitMix64 is the public generator of
// Steele, Lea & Flood (OOPSLA 2014).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fr_gen.h"

namespace {

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float hash_value(uint64_t row_seed, int64_t v) {
    const uint64_t u = splitmix64(row_seed ^ (uint64_t)v);
    return (float)(uint32_t)(u >> 40) * 0x1p-21f - 4.0f;
}

// grid.y = row (b*K + k), grid.x strides the columns; 8 values per thread.
template <bool BF16>
__global__ void k_gen(uint64_t seed, int64_t b_offset, int32_t K, int32_t V, int64_t ld,
                      const int32_t* __restrict__ prefix, int32_t pstride, int32_t t, const int32_t* __restrict__ live,
                      void* __restrict__ out) {
    const int64_t row = blockIdx.y;
    const int32_t b = (int32_t)(row / K), k = (int32_t)(row % K);
    if (live && k >= live[b]) return;
    uint64_t h = 0x243F6A8885A308D3ull;
    for (int i = 0; i < t; ++i) h = splitmix64(h ^ (uint64_t)(int64_t)prefix[row * pstride + i]);
    const uint64_t rs = splitmix64(splitmix64(splitmix64(seed) ^ (uint64_t)(b + b_offset)) ^ h);
    char* base = static_cast<char*>(out) + row * ld * (BF16 ? 2 : 4);
    const bool vec_ok = ((reinterpret_cast<uintptr_t>(base) & 15u) == 0);
    for (int64_t v0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; v0 < V;
         v0 += (int64_t)gridDim.x * blockDim.x * 8) {
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = hash_value(rs, v0 + i);
        if (BF16) {
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(base);
            if (vec_ok && v0 + 8 <= V) {
                __align__(16) __nv_bfloat16 tmp[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) tmp[i] = __float2bfloat16_rn(x[i]);
                *reinterpret_cast<uint4*>(o + v0) = *reinterpret_cast<const uint4*>(tmp);
            } else {
                for (int i = 0; i < 8 && v0 + i < V; ++i) o[v0 + i] = __float2bfloat16_rn(x[i]);
            }
        } else {
            float* o = reinterpret_cast<float*>(base);
            if (vec_ok && v0 + 8 <= V) {
                *reinterpret_cast<float4*>(o + v0) = make_float4(x[0], x[1], x[2], x[3]);
                *reinterpret_cast<float4*>(o + v0 + 4) = make_float4(x[4], x[5], x[6], x[7]);
            } else {
                for (int i = 0; i < 8 && v0 + i < V; ++i) o[v0 + i] = x[i];
            }
        }
    }
}

__global__ void k_flush(uint4* buf, int64_t n16, uint32_t salt) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x)
        buf[i] = make_uint4(salt, (uint32_t)i, salt, (uint32_t)(i >> 32));
}

}  // namespace

extern "C" fr_status fr_gen_hash_logits(uint64_t seed, int64_t b_offset, int32_t B, int32_t K, int32_t V, int64_t ld,
                                        fr_dtype dtype, const int32_t* prefix, int32_t pstride, int32_t t,
                                        const int32_t* live, void* out, fr_stream stream) {
    if (!out || B < 1 || K < 1 || K > 65535 || V < 1 || ld < V || t < 0 || (t > 0 && (!prefix || pstride < t)) ||
        (dtype != FR_F32 && dtype != FR_BF16))
        return FR_ERR_INVALID_ARG;
    const int64_t elt = dtype == FR_BF16 ? 2 : 4;
    if (reinterpret_cast<uintptr_t>(out) % (uintptr_t)elt) return FR_ERR_INVALID_ARG;
    const int threads = 256;
    int64_t gx = (V + threads * 8 - 1) / (threads * 8);
    if (gx > 64) gx = 64;
    // grid.y holds at most 65535 rows: launch whole requests per slab
    const int64_t req_per_slab = 65535 / K;
    for (int64_t b0 = 0; b0 < B; b0 += req_per_slab) {
        const int64_t nb = (B - b0) < req_per_slab ? (B - b0) : req_per_slab;
        const int64_t r0 = b0 * K;
        char* o = static_cast<char*>(out) + r0 * ld * elt;
        const int32_t* p = prefix ? prefix + r0 * pstride : nullptr;
        const int32_t* lv = live ? live + b0 : nullptr;
        dim3 grid((unsigned)gx, (unsigned)(nb * K));
        if (dtype == FR_BF16)
            k_gen<true><<<grid, threads, 0, (cudaStream_t)stream>>>(seed, b_offset + b0, K, V, ld, p, pstride, t, lv, o);
        else
            k_gen<false><<<grid, threads, 0, (cudaStream_t)stream>>>(seed, b_offset + b0, K, V, ld, p, pstride, t, lv, o);
        if (cudaGetLastError() != cudaSuccess) return FR_ERR_CUDA;
    }
    return FR_OK;
}

extern "C" fr_status fr_gen_flush(void* buf, int64_t bytes, fr_stream stream) {
    if (!buf || bytes < 16 || (reinterpret_cast<uintptr_t>(buf) & 15u)) return FR_ERR_INVALID_ARG;
    static uint32_t salt = 0x9E3779B9u;
    salt = salt * 1664525u + 1013904223u;
    k_flush<<<148 * 8, 256, 0, (cudaStream_t)stream>>>(static_cast<uint4*>(buf), bytes / 16, salt);
    return cudaGetLastError() == cudaSuccess ? FR_OK : FR_ERR_CUDA;
}
