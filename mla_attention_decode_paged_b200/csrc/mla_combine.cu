// mla_combine.cu -- LSE-weighted merge of split-KV partials.
//
// Each split j of a request leaves, per folded query row, its normalised partial output
// o_j (fp32, 512 wide) and its log-sum-exp in base 2, lse2_j = m_j + log2(l_j).  The
// merged row is
//     L = log2 sum_j 2^lse2_j,   out = sum_j 2^(lse2_j - L) * o_j,   lse = L * ln 2,
// the reduction pass of split-KV decoding ["Faster kernels, slower engine", 7.1 Gluon
// MLA decode].  A split in which a row sees no token has lse2_j = -inf and o_j = 0, so
// it drops out.  The kernel reads every partial once; it is bound by that read.
#include "mla_common.cuh"

namespace mla {

// grid (B, nqb, 128 / 4), block 128: one warp per folded row, 16 columns per lane.
__global__ void __launch_bounds__(128) combine_kernel(const void* __restrict__ ws, int B, int s_q, int H,
                                                      __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    const PlanHeader* h = reinterpret_cast<const PlanHeader*>(ws);
    if (h->magic != kPlanMagic || h->B != B || h->s_q != s_q || h->H != H) return;
    const int b = blockIdx.x, qb = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.z * 4 + warp;
    const int M = s_q * H;
    const int row = qb * kRowsPerBlock + r;
    if (row >= M) return;
    const int32_t* req_seg = ws_ptr<int32_t>(ws, h->off_req_seg);
    const int s0 = req_seg[b], s1 = req_seg[b + 1];
    if (s1 - s0 <= 1) return;  // written directly by the decode kernel
    const int nqb = h->nqb;
    const float* plse = ws_ptr<float>(ws, h->off_plse);
    const float* po = ws_ptr<float>(ws, h->off_po);

    float mx = -INFINITY;
    for (int s = s0; s < s1; ++s) mx = fmaxf(mx, plse[((int64_t)s * nqb + qb) * kRowsPerBlock + r]);
    float sum = 0.f;
    if (mx != -INFINITY)
        for (int s = s0; s < s1; ++s) sum += fast_exp2(plse[((int64_t)s * nqb + qb) * kRowsPerBlock + r] - mx);
    const float L = mx + __log2f(sum);

    float4 acc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = s0; s < s1; ++s) {
        const int64_t prow = ((int64_t)s * nqb + qb) * kRowsPerBlock + r;
        const float l2 = plse[prow];
        if (l2 == -INFINITY) continue;
        const float w = fast_exp2(l2 - L);
        const float4* src = reinterpret_cast<const float4*>(po + prow * kDv);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float4 v = src[lane + 32 * k];
            acc[k].x += w * v.x; acc[k].y += w * v.y; acc[k].z += w * v.z; acc[k].w += w * v.w;
        }
    }
    __nv_bfloat16* dst = out + ((int64_t)b * M + row) * kDv;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[k].x, acc[k].y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[k].z, acc[k].w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(dst + 4 * (lane + 32 * k)) = pk;
    }
    if (lane == 0) lse[(int64_t)b * M + row] = (mx == -INFINITY) ? -INFINITY : L * kLn2;
}

mla_status launch_combine(const void* ws, int B, int s_q, int H, void* out, float* lse, cudaStream_t stream) {
    dim3 grid(B, num_row_blocks(s_q, H), kRowsPerBlock / 4);
    combine_kernel<<<grid, 128, 0, stream>>>(ws, B, s_q, H, reinterpret_cast<__nv_bfloat16*>(out), lse);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla

extern "C" mla_status mla_split_kv_combine(const void* workspace, size_t ws_bytes, int B, int s_q, int H,
                                           void* out, float* lse, void* stream) {
    if (!workspace || !out || !lse || B <= 0 || s_q <= 0 || H <= 0) return MLA_ERR_INVALID_ARG;
    if ((int64_t)s_q * H > mla::kMaxRows) return MLA_ERR_UNSUPPORTED;
    if ((((uintptr_t)out) & 15) != 0) return MLA_ERR_INVALID_ARG;
    mla::WsLayout L = mla::make_layout(B, s_q, H, 1);
    if ((int64_t)ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    return mla::launch_combine(workspace, B, s_q, H, out, lse, (cudaStream_t)stream);
}
