// mla_decode_api.cu -- host entry point mla_decode: argument checks, then the decode
// kernel and the split-KV combine on the caller's stream.  Nothing here allocates or
// synchronises.
#include <math.h>

#include "mla_decode_params.cuh"

using namespace mla;

extern "C" mla_status mla_decode_scan(const void* q, const void* kv_pages, int kv_dtype, float kv_scale,
                                 const int32_t* block_table, int max_pages_per_req, const int32_t* seq_lens,
                                 int B, int s_q, int H, int64_t num_pages, float scale, int causal,
                                 void* workspace, size_t ws_bytes, void* out, float* lse, void* stream) {
    if (!q || !kv_pages || !block_table || !seq_lens || !workspace || !out || !lse) return MLA_ERR_INVALID_ARG;
    if (B <= 0 || s_q <= 0 || H <= 0 || max_pages_per_req <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return MLA_ERR_INVALID_ARG;
    if (kv_dtype != MLA_KV_BF16 && kv_dtype != MLA_KV_E4M3) return MLA_ERR_UNSUPPORTED;
    if (kv_dtype == MLA_KV_E4M3 && !(isfinite(kv_scale) && kv_scale > 0.f)) return MLA_ERR_INVALID_ARG;
    if ((int64_t)s_q * H > kMaxRows) return MLA_ERR_UNSUPPORTED;
    if ((((uintptr_t)q) & 15) || (((uintptr_t)kv_pages) & 15) || (((uintptr_t)out) & 15) ||
        (((uintptr_t)workspace) & 255) || (((uintptr_t)lse) & 3) || (((uintptr_t)block_table) & 3))
        return MLA_ERR_INVALID_ARG;
    if ((int64_t)ws_bytes < make_layout(B, s_q, H, 1).total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    const int sms = effective_sms();
    if (sms <= 0) return MLA_ERR_CUDA;

    DecodeParams p;
    p.q = q;
    p.kv = kv_pages;
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.ws = workspace;
    p.out = out;
    p.lse = lse;
    p.num_pages = num_pages;
    p.max_pages = max_pages_per_req;
    p.B = B;
    p.s_q = s_q;
    p.H = H;
    p.M = s_q * H;
    p.causal = causal != 0;
    p.groups_launched = num_groups_for(sms, num_row_blocks(s_q, H));
    // the scan reads its group's head record before it checks the plan (always true for a
    // workspace of at least one group's layout; kept explicit)
    if ((int64_t)ws_bytes < kOffHeads + (int64_t)sizeof(GroupHead) * p.groups_launched)
        return MLA_ERR_WORKSPACE_TOO_SMALL;
    const float ks = kv_dtype == MLA_KV_E4M3 ? kv_scale : 1.f;
    p.score_scale_log2 = scale * ks * kLog2e;
    p.out_scale = ks;
    return launch_decode_sm100(p, kv_dtype, (cudaStream_t)stream);
}

extern "C" mla_status mla_decode(const void* q, const void* kv_pages, int kv_dtype, float kv_scale,
                                 const int32_t* block_table, int max_pages_per_req, const int32_t* seq_lens,
                                 int B, int s_q, int H, int64_t num_pages, float scale, int causal,
                                 void* workspace, size_t ws_bytes, void* out, float* lse, void* stream) {
    mla_status st = mla_decode_scan(q, kv_pages, kv_dtype, kv_scale, block_table, max_pages_per_req, seq_lens, B,
                                    s_q, H, num_pages, scale, causal, workspace, ws_bytes, out, lse, stream);
    if (st != MLA_OK) return st;
    return launch_combine(workspace, B, s_q, H, out, lse, (cudaStream_t)stream);
}
