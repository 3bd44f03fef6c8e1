// mla_decode_params.cuh -- argument block passed from the host entry point to the
// decode kernels.
#pragma once

#include "mla_common.cuh"

namespace mla {

struct DecodeParams {
    const void* q;              // bf16 [B, s_q, H, 576]
    const void* kv;             // bf16 / e4m3 [num_pages, 64, 576]
    const int32_t* block_table; // [B, max_pages]
    const int32_t* seq_lens;    // [B]
    void* ws;                   // workspace (plan + partials)
    void* out;                  // bf16 [B, s_q, H, 512]
    float* lse;                 // fp32 [B, s_q, H]
    int64_t num_pages;
    int max_pages;
    int B, s_q, H, M;
    int causal;
    int groups_launched;        // groups the grid covers (>= the plan's)
    float score_scale_log2;     // scale * kv_scale * log2(e): scores in base 2
    float out_scale;            // kv_scale for e4m3 (values are e4m3 * kv_scale), 1 for bf16
};

// Dynamic shared memory of the plan kernel (one CTA) for B requests and G groups, and
// the most the planner takes: shapes beyond it are unsupported.
inline size_t plan_shared_bytes(int B, int G) {
    const size_t b = (size_t)B, g = (size_t)G;
    // int64: prefix over requests [B + 1], cuts [G + 1], flags [G + 2], scan scratch [8];
    // int32: the request each cut falls inside [G + 1], segment starts 2 x [B + G], first
    // segment of each group [G + 1]
    return sizeof(int64_t) * ((b + 1) + (g + 1) + (g + 2) + 8) + sizeof(int32_t) * (2 * (g + 1) + 2 * (b + g));
}
constexpr size_t kPlanMaxSharedBytes = 200 * 1024;

mla_status launch_decode_sm100(const DecodeParams& p, int kv_dtype, cudaStream_t stream);
// One CTA that runs the scan kernel's bounded wait on a barrier nothing arrives at (20 ms
// limit) and so sets the timeout status in the workspace header.
mla_status launch_wait_timeout_probe(void* ws, cudaStream_t stream);
// CTAs of the tensor-core scan kernel that the current device runs at once (one per
// SM); the split plan is made for this many by default.
int sm100_cta_slots();
int effective_sms();
mla_status launch_combine(const void* ws, int B, int s_q, int H, void* out, float* lse, cudaStream_t stream);
int device_sm_count();

}  // namespace mla
