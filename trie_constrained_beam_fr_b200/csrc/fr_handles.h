// fr_handles.h -- host-side definitions of the opaque libfr handles.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fr.h"
#include "fr_internal.cuh"

struct fr_trie {
    int32_t depth = 0;
    int32_t sid_base = 0;
    int32_t codebook[FR_MAX_DEPTH] = {};
    int64_t nodes[FR_MAX_DEPTH + 1] = {};
    int32_t max_fanout = 0;
    int32_t level_fanout[FR_MAX_DEPTH] = {};  // largest child count of a level-l node
    int32_t dense[FR_MAX_DEPTH] = {};         // level l is full: every node has all C_l children
    int32_t device = 0;
    int32_t* child_off[FR_MAX_DEPTH] = {};
    int32_t* code[FR_MAX_DEPTH + 1] = {};
    int32_t* leaf_row = nullptr;
    fr::TrieDev dev{};
};

namespace fr {

// Queues the exclusive prefix sum of in[0..n) into out (in-place allowed).
// temp must hold scan_temp_elems(n) int32; total (device, may be null)
// receives the sum of all elements.
int64_t scan_temp_elems(int64_t n);
cudaError_t scan_exclusive_i32(const int32_t* in, int32_t* out, int64_t n, int32_t* temp,
                               int32_t* total, cudaStream_t stream);

}  // namespace fr

#define FR_CUDA_TRY(expr)                                                   \
    do {                                                                    \
        cudaError_t e__ = (expr);                                           \
        if (e__ != cudaSuccess) {                                           \
            (void)cudaGetLastError();                                       \
            return e__ == cudaErrorMemoryAllocation ? FR_ERR_OOM : FR_ERR_CUDA; \
        }                                                                   \
    } while (0)
