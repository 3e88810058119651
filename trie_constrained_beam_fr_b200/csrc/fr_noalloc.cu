// fr_noalloc.cu -- fr_row_logsumexp_noalloc: the streaming log-sum-exp of
// the beam step for callers that must not allocate device memory.
//
// Some callers cannot call cudaMalloc: a plugin running inside a framework
// whose allocator owns every byte of device memory (a second allocator would
// fragment the pool and escape its accounting), or a latency-critical serving
// path where cudaMalloc's implicit device-wide synchronisation would stall the
// other streams.  This entry point takes the rows' log-sum-exp (the
// normaliser of the full-vocabulary log-softmax) with the same streaming
// kernel as fr_beam_step, but its scratch -- the per-CTA partial sums of rows
// split across CTAs, the per-row arrival counters and a status word -- lives
// in one file-scope __device__ array loaded with the library, so the call
// itself allocates nothing.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "fr_handles.h"
#include "fr_step.cuh"

namespace {

// Fixed capacity of the shared scratch.
constexpr int32_t NOALLOC_MAX_ROWS = 65536;
constexpr int32_t NOALLOC_MAX_CTAS = 1024;

struct NoallocScratch {
    int32_t row_cnt[NOALLOC_MAX_ROWS];   // arrival counters of rows split across CTAs
    float2 partial[2 * NOALLOC_MAX_CTAS];  // (max, scaled sum) per CTA and row side
    int32_t live;                        // the row count, read by the kernel
    int32_t err;                         // device status word
};

// Every GPU that loads the library holds this array (about 280 KB) until the
// process exits.  All calls share it.
static __device__ __align__(256) NoallocScratch g_noalloc_scratch;

constexpr int MAX_DEVICES = 64;
std::mutex g_setup_mutex;
NoallocScratch* g_scratch_addr[MAX_DEVICES] = {};
int32_t g_sm_count[MAX_DEVICES] = {};

__global__ void k_noalloc_prepare(NoallocScratch* s, int32_t rows, float* lse_out) {
    // counters of the rows this call uses start at zero (the rest is unused);
    // every output starts as NaN, so a row the streaming kernel never finishes
    // (a bounded wait that ran out) reads as non-finite, not as stale data
    for (int32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += gridDim.x * blockDim.x) {
        s->row_cnt[i] = 0;
        lse_out[i] = __int_as_float(0x7FC00000);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        s->live = rows;
        s->err = 0;
    }
}

// Device address of the scratch for the current device, looked up once per
// device (cudaGetSymbolAddress must run with that device current; in host
// code the array's name is only a host-side stand-in), together with the
// device's SM count and the streaming kernel's shared-memory attribute.  The
// cache is per device ordinal: after cudaDeviceReset the module may load at
// another address, so the entry point is not for use across a device reset.
fr_status scratch_for_current_device(NoallocScratch** out, int32_t* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
        (void)cudaGetLastError();
        return FR_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return FR_ERR_CUDA;
        }
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
            (void)cudaGetLastError();
            return FR_ERR_CUDA;
        }
        // the streaming kernel's shared-memory limit, raised once per device
        if (fr::row_lse_kernel_setup() != cudaSuccess) {
            (void)cudaGetLastError();
            return FR_ERR_CUDA;
        }
        g_scratch_addr[dev] = static_cast<NoallocScratch*>(p);
        g_sm_count[dev] = n;
    }
    *out = g_scratch_addr[dev];
    *sms = g_sm_count[dev];
    return FR_OK;
}

}  // namespace

extern "C" fr_status fr_row_logsumexp_noalloc(const void* logits_dev, int64_t ld, fr_dtype dtype, int32_t rows,
                                              int32_t V, float* lse_dev, fr_stream stream) {
    if (!logits_dev || !lse_dev || rows < 1 || V < 1 || ld < V || (dtype != FR_F32 && dtype != FR_BF16))
        return FR_ERR_INVALID_ARG;
    if (rows > NOALLOC_MAX_ROWS) return FR_ERR_INVALID_ARG;  // beyond the fixed scratch
    const int64_t elt = dtype == FR_BF16 ? 2 : 4;
    if (reinterpret_cast<uintptr_t>(logits_dev) % (uintptr_t)elt != 0) return FR_ERR_INVALID_ARG;
    NoallocScratch* s = nullptr;
    int32_t sms = 0;
    fr_status st = scratch_for_current_device(&s, &sms);
    if (st != FR_OK) return st;
    const int32_t grid = sms < NOALLOC_MAX_CTAS ? sms : NOALLOC_MAX_CTAS;
    const cudaStream_t cs = (cudaStream_t)stream;
    k_noalloc_prepare<<<(rows + 255) / 256 < sms ? (rows + 255) / 256 : sms, 256, 0, cs>>>(s, rows, lse_dev);
    FR_CUDA_TRY(cudaGetLastError());
    FR_CUDA_TRY(fr::launch_row_lse(logits_dev, ld, (int32_t)dtype, rows, V, grid, &s->live, s->partial, s->row_cnt,
                                   &s->err, lse_dev, cs));
    return FR_OK;
}
