// fr_step.cuh -- kernel launchers of the beam step (internal to libfr).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fr_internal.cuh"

namespace fr {

struct StepBuffers {
    StateDev st[2];
    int32_t* parent;      // [B*K] latest step
    int32_t* token;       // [B*K]
    float* cand;          // [B * cand_stride] candidate scores
    float* cand_key;      // [B * cand_stride] perturbed keys (sampling above temperature 0)
    int64_t cand_stride;  // K * max_fanout rounded up to a multiple of 4
    float2* partial;      // [stream_max_pieces(grid) * 2] (max, scaled sum) per piece and row side
    int32_t* piece_ctr;   // [2] the streaming kernel's dynamic-piece counters (zero between launches)
    int32_t* row_cnt;     // [B*K] arrival counters of shared rows
    int32_t* err;         // sticky device status word
};

struct StepShape {
    int32_t B, K, V, D;
    int32_t dtype;  // fr_dtype
    int32_t grid;   // CTAs of the streaming kernel
    int32_t norm;      // fr_norm: the set each row's log-softmax runs over
    int32_t sid_span;  // C_0 + ... + C_{D-1}: width of the SID token range
    int32_t sel_cluster[FR_MAX_DEPTH];  // per step: CTAs per request of the cluster select (0: one CTA)
    int64_t sel_bound[FR_MAX_DEPTH];    // per step: most candidates a request can have
    float inv_temp;      // 1 / temperature; 0 = deterministic top-K
    uint64_t gseed;      // Gumbel stream seed
    int64_t req_offset;  // index of local request 0 in the Gumbel stream
    uint64_t wait_ns;    // limit of the streaming kernel's bounded waits
    int32_t starve;      // test setting: the streaming kernel's producer issues no copies
};

// Launch configuration of a step kernel: programmatic stream serialization
// (see griddep_wait), and optionally a cluster size.  Used in place (cfg
// points into the object).
struct StepLaunch {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[2];
    StepLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t s, unsigned cluster = 0) {
        cfg.gridDim = grid;
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        int n = 1;
        if (cluster) {
            attr[1].id = cudaLaunchAttributeClusterDimension;
            attr[1].val.clusterDim.x = cluster;
            attr[1].val.clusterDim.y = 1;
            attr[1].val.clusterDim.z = 1;
            n = 2;
        }
        cfg.attrs = attr;
        cfg.numAttrs = n;
    }
    StepLaunch(const StepLaunch&) = delete;
    StepLaunch& operator=(const StepLaunch&) = delete;
};

// Blocks of 256 threads covering n items (grid-stride beyond 4096 blocks).
inline int small_grid(int64_t n) {
    const int64_t g = (n + 255) / 256;
    return (int)(g < 1 ? 1 : (g > 4096 ? 4096 : g));
}

// Cluster size of the selection for a step whose requests have at most
// `bound` candidates (0 = the single-CTA kernel).
int select_cluster_size(int32_t B, int32_t K, int64_t bound, int32_t sms);
cudaError_t select_kernel_setup();  // raises the one-CTA selection's shared-memory limit

// Streaming kernel: dynamic shared memory it needs for B requests (bf16 or
// fp32 rows: the ring differs).
size_t stream_smem_bytes(int32_t B, bool bf16);
cudaError_t stream_kernel_setup();  // raises the kernel's shared-memory limit
// Most pieces the streaming kernel cuts a launch into on `grid` CTAs (its
// partial buffer holds two entries per piece).
int64_t stream_max_pieces(int32_t grid);

cudaError_t launch_stream(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t,
                          const void* logits, int64_t ld, cudaStream_t s);
// Step 0 as one kernel (root rows + selection) instead of launch_stream +
// launch_select: used when root_step_fused() holds (temperature 0, at most
// 8,192 root children, no wait test setting).  root_step_setup raises its shared-memory
// limit (once per device).
bool root_step_fused(const StepShape& sh, const TrieDev& trie);
cudaError_t root_step_setup();
cudaError_t launch_root_step(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, const void* logits,
                             int64_t ld, cudaStream_t s);
// Log-sum-exp of `rows` rows (row k at logits + k*ld elements) into lse_out,
// with caller-provided scratch: partial [2*grid], row_cnt [rows] (zero on
// entry, zero again on exit), err [1]; live_dev [1] must hold `rows`.
// row_lse_kernel_setup raises the kernel's shared-memory limit on the current
// device; it must have run there once before launch_row_lse.
cudaError_t row_lse_kernel_setup();
cudaError_t launch_row_lse(const void* logits, int64_t ld, int32_t dtype, int32_t rows, int32_t V, int32_t grid,
                           const int32_t* live_dev, float2* partial, int32_t* row_cnt, int32_t* err, float* lse_out,
                           cudaStream_t s);
// The row phase of a step from given rows: slot (b, k) has the log-sum-exp
// lse[b * row_stride_b + k] over the vocabulary and the SID-range logits
// slice[(b * row_stride_b + k) * sid_span + (v - sid_base)].
cudaError_t launch_step_lse(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t,
                            const float* lse, const float* slice, int64_t row_stride_b, cudaStream_t s);
cudaError_t launch_select(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t, cudaStream_t s);
cudaError_t launch_reset(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, cudaStream_t s);
cudaError_t launch_set_state(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t,
                             const int32_t* prefix_codes, const int32_t* kv_given, cudaStream_t s);
cudaError_t launch_finalize(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t, int32_t* sids,
                            float* scores, int32_t* items, cudaStream_t s);

}  // namespace fr
