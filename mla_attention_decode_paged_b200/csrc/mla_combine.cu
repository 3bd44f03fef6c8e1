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

constexpr int kCombineThreads = 512;  // 4 groups of 128 threads; a thread owns one float4 column
constexpr int kCombineMaxSplits = kMaxGroups + 1;

// grid (B, nqb, 64): one folded row per CTA.  The row's split weights are computed once
// into shared memory; group j of the CTA accumulates the splits j, j+4, j+8, ... for its
// float4 column (several independent loads in flight per thread), and the four group
// sums are added through shared memory.
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const void* __restrict__ ws, int B, int s_q, int H,
                                                                  __nv_bfloat16* __restrict__ out,
                                                                  float* __restrict__ lse) {
    __shared__ float wsh[kCombineMaxSplits];
    __shared__ float4 part[3][128];
    __shared__ float red[2];
    const PlanHeader* h = reinterpret_cast<const PlanHeader*>(ws);
    if (h->magic != kPlanMagic || h->B != B || h->s_q != s_q || h->H != H) return;
    const int b = blockIdx.x, qb = blockIdx.y, r = blockIdx.z;
    const int M = s_q * H;
    const int row = qb * kRowsPerBlock + r;
    if (row >= M) return;
    const int32_t* req_seg = ws_ptr<int32_t>(ws, h->off_req_seg);
    const int s0 = req_seg[b], ns = req_seg[b + 1] - s0;
    if (ns <= 1) return;  // written directly by the decode kernel
    const int nqb = h->nqb;
    const float* plse = ws_ptr<float>(ws, h->off_plse);
    const float* po = ws_ptr<float>(ws, h->off_po);
    const int64_t stride = (int64_t)nqb * kRowsPerBlock;  // rows between consecutive segments
    const int64_t prow0 = ((int64_t)s0 * nqb + qb) * kRowsPerBlock + r;
    const int tid = threadIdx.x, grp = tid >> 7, c4 = tid & 127;

    // L = log2 sum_j 2^lse2_j and the weights 2^(lse2_j - L), by warp 0
    if (tid < 32) {
        float mx = -INFINITY;
        for (int j = tid; j < ns; j += 32) mx = fmaxf(mx, plse[prow0 + j * stride]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        if (mx != -INFINITY)
            for (int j = tid; j < ns; j += 32) sum += fast_exp2(plse[prow0 + j * stride] - mx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float L = mx + __log2f(sum);
        for (int j = tid; j < ns && j < kCombineMaxSplits; j += 32) {
            const float l2 = plse[prow0 + j * stride];
            wsh[j] = (l2 == -INFINITY) ? 0.f : fast_exp2(l2 - L);  // an empty split drops out
        }
        if (tid == 0) {
            red[0] = L;
            red[1] = mx;
        }
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int j = grp;
    for (; j + 12 < ns; j += 16) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = reinterpret_cast<const float4*>(po + (prow0 + (int64_t)(j + 4 * u) * stride) * kDv)[c4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float w = wsh[j + 4 * u];
            acc.x += w * v[u].x; acc.y += w * v[u].y; acc.z += w * v[u].z; acc.w += w * v[u].w;
        }
    }
    for (; j < ns; j += 4) {
        const float4 v = reinterpret_cast<const float4*>(po + (prow0 + (int64_t)j * stride) * kDv)[c4];
        const float w = wsh[j];
        acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
    }
    if (grp > 0) part[grp - 1][c4] = acc;
    __syncthreads();
    if (grp == 0) {
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const float4 v = part[k][c4];
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(out + ((int64_t)b * M + row) * kDv + 4 * c4) = pk;
        if (c4 == 0) lse[(int64_t)b * M + row] = (red[1] == -INFINITY) ? -INFINITY : red[0] * kLn2;
    }
}

mla_status launch_combine(const void* ws, int B, int s_q, int H, void* out, float* lse, cudaStream_t stream) {
    dim3 grid(B, num_row_blocks(s_q, H), kRowsPerBlock);
    combine_kernel<<<grid, kCombineThreads, 0, stream>>>(ws, B, s_q, H, reinterpret_cast<__nv_bfloat16*>(out), lse);
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
