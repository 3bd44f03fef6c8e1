// mla_combine.cu -- LSE-weighted merge of split-KV partials.
//
// Each split j of a request leaves, per folded query row, its normalised partial output
// o_j (fp32, 512 wide) and its log-sum-exp in base 2, lse2_j = m_j + log2(l_j).  The
// merged row is
//     L = log2 sum_j 2^lse2_j,   out = sum_j 2^(lse2_j - L) * o_j,   lse = L * ln 2,
// the reduction pass of split-KV decoding ["Faster kernels, slower engine", 7.1 Gluon
// MLA decode].  A split in which a row sees no token has lse2_j = -inf and o_j = 0, so
// it drops out.  The kernel reads every partial once; it is bound by that read.  A
// request without tokens has no split at all; its rows are written here, as NaN.
#include <string.h>

#include "mla_decode_params.cuh"

namespace mla {

constexpr int kTileThreads = 256;     // 16 rows x 16 column quads
constexpr int kWChunk = 64;           // splits whose weights are in shared memory at once
constexpr int kPre = 6;               // partials per thread loaded before the weights are known

// What a combine CTA takes from the plan: where the partials are and request b's splits.
// It is read before the grid-dependency wait, while the scan's last CTAs still run: the
// scan releases its dependents only after its own wait for the planner, so the plan is
// complete when this grid starts.  One thread reads it through L2 (.cg: never a line an
// earlier kernel left in this SM's L1; one reader, not every thread of every CTA on the
// same lines) and hands it to the CTA in shared memory.  The partials are read only
// after the wait.
struct CombinePlan {
    bool ok;
    int nqb, s0, ns;
    int64_t off_plse, off_po;
};

__device__ __forceinline__ CombinePlan read_combine_plan(const void* ws, int B, int s_q, int H, int b) {
    __shared__ CombinePlan sh;
    if (threadIdx.x == 0) {
        const PlanHeader* h = reinterpret_cast<const PlanHeader*>(ws);
        CombinePlan c;
        const bool match = __ldcg(&h->magic) == kPlanMagic && __ldcg(&h->B) == B && __ldcg(&h->s_q) == s_q &&
                           __ldcg(&h->H) == H;
        c.nqb = __ldcg(&h->nqb);
        const int max_segments = __ldcg(&h->max_segments);
        const int64_t off_req_seg = __ldcg(reinterpret_cast<const long long*>(&h->off_req_seg));
        c.off_plse = __ldcg(reinterpret_cast<const long long*>(&h->off_plse));
        c.off_po = __ldcg(reinterpret_cast<const long long*>(&h->off_po));
        c.ok = false;
        c.s0 = c.ns = 0;
        if (match) {
            const int32_t* req_seg = ws_ptr<int32_t>(ws, off_req_seg);
            const int s0 = __ldcg(req_seg + b), s1 = __ldcg(req_seg + b + 1);
            // a plan the host accepted always passes; the check keeps every index in bounds
            c.ok = 0 <= s0 && s0 <= s1 && s1 <= max_segments;
            c.s0 = s0;
            c.ns = s1 - s0;
        }
        sh = c;
    }
    __syncthreads();
    return sh;
}

// Requests with many splits (few long requests): one CTA per (request, 16-row group,
// 64-column chunk).  Within a group of 256 threads, thread t owns row t % 16 and column
// quad t / 16 of the 16 x 64 tile; in the workspace's quad-interleaved partial layout the
// tile of one split is 4 KB contiguous, read by the 256 threads with one 16-byte load
// each.  kSplitGroups groups take the splits j = group, group + kSplitGroups, ... so that
// kSplitGroups x kPre partials are in flight before the weights are known; the group sums
// meet in shared memory at the end.
template <int kSplitGroups>
__global__ void __launch_bounds__(kTileThreads * kSplitGroups, 4 / kSplitGroups) combine_many_kernel(
    const void* __restrict__ ws, int B, int s_q, int H, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    constexpr int kCombineThreads = kTileThreads * kSplitGroups;
    __shared__ float wsh[kWChunk][16];
    __shared__ float Lsh[16], Msh[16];
    __shared__ float4 part[kSplitGroups > 1 ? kSplitGroups - 1 : 1][kTileThreads];
    const int b = blockIdx.x, qb = blockIdx.y >> 2, g = blockIdx.y & 3, c64 = blockIdx.z;
    const CombinePlan cp = read_combine_plan(ws, B, s_q, H, b);
    // launched as a programmatic dependent of the scan: no partial is read, and nothing is
    // written, before it completes
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!cp.ok) return;
    const int M = s_q * H;
    const int row0 = qb * kRowsPerBlock + g * 16;
    if (row0 >= M) return;
    const int s0 = cp.s0, ns = cp.ns;
    const int tid = threadIdx.x, t = tid & (kTileThreads - 1), grp = tid / kTileThreads;
    const int r16 = t & 15, cq = t >> 4;
    const int m = row0 + r16;
    if (ns == 0) {
        // a request without tokens (T_b <= 0) has no split: the planner set the status word,
        // and its rows are written here as NaN
        if (grp == 0 && m < M) {
            *reinterpret_cast<uint2*>(out + ((int64_t)b * M + m) * kDv + 64 * c64 + 4 * cq) =
                make_uint2(0x7fc07fc0u, 0x7fc07fc0u);
            if (c64 == 0 && cq == 0) lse[(int64_t)b * M + m] = __int_as_float(0x7fc00000);
        }
        return;
    }
    if (ns == 1) return;  // written directly by the decode kernel
    const int nqb = cp.nqb;
    // split j: partial tile at pc + j * jstride (float4); lse2 of row r at lbase[j * lstride + r]
    const float4* pc = reinterpret_cast<const float4*>(ws_ptr<float>(ws, cp.off_po)) +
                       ((int64_t)s0 * nqb + qb) * (kRowsPerBlock * kDv / 4) + g * 2048 + (int64_t)c64 * 256 +
                       cq * 16 + r16;
    const int64_t jstride = (int64_t)nqb * (kRowsPerBlock * kDv / 4);
    const float* lbase = ws_ptr<float>(ws, cp.off_plse) + ((int64_t)s0 * nqb + qb) * kRowsPerBlock + g * 16;
    const int64_t lstride = (int64_t)nqb * kRowsPerBlock;

    // the first partials, in flight while the weights are computed
    float4 v[kPre];
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
        const int j = grp + kSplitGroups * u;
        v[u] = j < ns ? pc[j * jstride] : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // L = log2 sum_j 2^lse2_j per row: warp w < 8 takes rows 2w and 2w + 1 (one per half-warp)
    if (tid < kTileThreads) {
        const int lane = tid & 31, r = 2 * (tid >> 5) + (lane >> 4), k = lane & 15;
        // fmaxf drops NaN, so a poisoned split (NaN lse2: a bad page or length) is tracked
        // on its own and turns the merged row into NaN even when every split is poisoned
        float mx = -INFINITY;
        bool poisoned = false;
        for (int j = k; j < ns; j += 16) {
            const float l2 = lbase[j * lstride + r];
            poisoned |= l2 != l2;
            mx = fmaxf(mx, l2);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        poisoned = ((__ballot_sync(0xffffffffu, poisoned) >> (lane & 16)) & 0xffffu) != 0;  // this row's half-warp
        float sum = 0.f;
        if (mx != -INFINITY)
            for (int j = k; j < ns; j += 16) sum += fast_exp2(lbase[j * lstride + r] - mx);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (k == 0) {
            const float nanv = __int_as_float(0x7fc00000);
            Lsh[r] = poisoned ? nanv : mx + __log2f(sum);
            Msh[r] = poisoned ? nanv : mx;
        }
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int j0 = 0; j0 < ns; j0 += kWChunk) {
        const int nj = min(kWChunk, ns - j0);
        // the split weights 2^(lse2_j - L) of the 16 rows, for splits [j0, j0 + nj)
        for (int e = tid; e < nj * 16; e += kCombineThreads) {
            const int jj = e >> 4, r = e & 15;
            const float l2 = lbase[(int64_t)(j0 + jj) * lstride + r];
            wsh[jj][r] = (l2 == -INFINITY) ? 0.f : fast_exp2(l2 - Lsh[r]);  // an empty split drops out
        }
        __syncthreads();
        int jj = grp;  // this group's splits within the weight chunk: grp, grp + kSplitGroups, ...
        if (j0 == 0) {
#pragma unroll
            for (int u = 0; u < kPre; ++u) {
                const int j = grp + kSplitGroups * u;
                const float w = j < nj ? wsh[j][r16] : 0.f;
                acc.x += w * v[u].x; acc.y += w * v[u].y; acc.z += w * v[u].z; acc.w += w * v[u].w;
            }
            jj = grp + kSplitGroups * kPre;
        }
        for (; jj + kSplitGroups < nj; jj += 2 * kSplitGroups) {
            float4 x[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) x[u] = pc[(j0 + jj + kSplitGroups * u) * jstride];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float w = wsh[jj + kSplitGroups * u][r16];
                acc.x += w * x[u].x; acc.y += w * x[u].y; acc.z += w * x[u].z; acc.w += w * x[u].w;
            }
        }
        for (; jj < nj; jj += kSplitGroups) {
            const float4 x = pc[(j0 + jj) * jstride];
            const float w = wsh[jj][r16];
            acc.x += w * x.x; acc.y += w * x.y; acc.z += w * x.z; acc.w += w * x.w;
        }
        __syncthreads();  // before the next weight chunk overwrites wsh
    }
    if (kSplitGroups > 1) {
        // the groups' sums meet, then the other groups leave
        if (grp > 0) part[grp - 1][t] = acc;
        __syncthreads();
        if (grp > 0) return;
#pragma unroll
        for (int k = 0; k < kSplitGroups - 1; ++k) {
            const float4 x = part[k][t];
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
        }
    }
    if (m < M) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(out + ((int64_t)b * M + m) * kDv + 64 * c64 + 4 * cq) = pk;
        if (c64 == 0 && cq == 0) lse[(int64_t)b * M + m] = (Msh[r16] == -INFINITY) ? -INFINITY : Lsh[r16] * kLn2;
    }
}

// Requests with few splits (the common case of batches of many requests): one CTA per
// (request, 16-row group, kChunks column chunks of 64); thread t owns row t % 16 and column
// quad t / 16 of every chunk.  The partials of two splits for all the CTA's chunks are
// loaded at once (the first two while the lse pass runs), so a request with two splits
// costs one round trip to memory after the weights instead of one per column chunk.
template <int kChunks>
__global__ void __launch_bounds__(kTileThreads, 2) combine_few_kernel(
    const void* __restrict__ ws, int B, int s_q, int H, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    __shared__ float wsh[kWChunk][16];
    __shared__ float Lsh[16], Msh[16];
    const int b = blockIdx.x, qb = blockIdx.y >> 2, g = blockIdx.y & 3;
    const CombinePlan cp = read_combine_plan(ws, B, s_q, H, b);
    // launched as a programmatic dependent of the scan: no partial is read, and nothing is
    // written, before it completes
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!cp.ok) return;
    const int M = s_q * H;
    const int row0 = qb * kRowsPerBlock + g * 16;
    if (row0 >= M) return;
    const int s0 = cp.s0, ns = cp.ns;
    const int t = threadIdx.x, r16 = t & 15, cq = t >> 4;
    const int m = row0 + r16;
    const int c0 = blockIdx.z * kChunks;  // the CTA's first 64-column chunk
    if (ns == 0) {
        // a request without tokens (T_b <= 0) has no split: the planner set the status word,
        // and its rows are written here as NaN
        if (m < M) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
                *reinterpret_cast<uint2*>(out + ((int64_t)b * M + m) * kDv + 64 * (c0 + c) + 4 * cq) =
                    make_uint2(0x7fc07fc0u, 0x7fc07fc0u);
            if (c0 == 0 && cq == 0) lse[(int64_t)b * M + m] = __int_as_float(0x7fc00000);
        }
        return;
    }
    if (ns == 1) return;  // written directly by the decode kernel
    const int nqb = cp.nqb;
    // split j, chunk c: partial tile at pbase + c * 256 + j * jstride (float4); lse2 of row r
    // at lbase[j * lstride + r]
    const float4* pbase = reinterpret_cast<const float4*>(ws_ptr<float>(ws, cp.off_po)) +
                          ((int64_t)s0 * nqb + qb) * (kRowsPerBlock * kDv / 4) + g * 2048 + cq * 16 + r16 +
                          (int64_t)c0 * 256;
    const int64_t jstride = (int64_t)nqb * (kRowsPerBlock * kDv / 4);
    const float* lbase = ws_ptr<float>(ws, cp.off_plse) + ((int64_t)s0 * nqb + qb) * kRowsPerBlock + g * 16;
    const int64_t lstride = (int64_t)nqb * kRowsPerBlock;

    float4 x0[kChunks], x1[kChunks];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
        x0[c] = pbase[c * 256];
        x1[c] = pbase[c * 256 + jstride];
    }
    {
        // L = log2 sum_j 2^lse2_j per row: warp w takes rows 2w and 2w + 1 (one per half-warp)
        const int lane = t & 31, r = 2 * (t >> 5) + (lane >> 4), k = lane & 15;
        // fmaxf drops NaN, so a poisoned split (NaN lse2: a bad page or length) is tracked
        // on its own and turns the merged row into NaN even when every split is poisoned
        float mx = -INFINITY;
        bool poisoned = false;
        for (int j = k; j < ns; j += 16) {
            const float l2 = lbase[j * lstride + r];
            poisoned |= l2 != l2;
            mx = fmaxf(mx, l2);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        poisoned = ((__ballot_sync(0xffffffffu, poisoned) >> (lane & 16)) & 0xffffu) != 0;  // this row's half-warp
        float sum = 0.f;
        if (mx != -INFINITY)
            for (int j = k; j < ns; j += 16) sum += fast_exp2(lbase[j * lstride + r] - mx);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (k == 0) {
            const float nanv = __int_as_float(0x7fc00000);
            Lsh[r] = poisoned ? nanv : mx + __log2f(sum);
            Msh[r] = poisoned ? nanv : mx;
        }
    }
    __syncthreads();
    float4 acc[kChunks];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    auto add = [&](const float4(&x)[kChunks], float w) {
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
            acc[c].x += w * x[c].x; acc[c].y += w * x[c].y; acc[c].z += w * x[c].z; acc[c].w += w * x[c].w;
        }
    };
#pragma unroll 1
    for (int j0 = 0; j0 < ns; j0 += kWChunk) {
        const int nj = min(kWChunk, ns - j0);
        // the split weights 2^(lse2_j - L) of the 16 rows, for splits [j0, j0 + nj)
        for (int e = t; e < nj * 16; e += kTileThreads) {
            const int jj = e >> 4, r = e & 15;
            const float l2 = lbase[(int64_t)(j0 + jj) * lstride + r];
            wsh[jj][r] = (l2 == -INFINITY) ? 0.f : fast_exp2(l2 - Lsh[r]);  // an empty split drops out
        }
        __syncthreads();
        int jj = 0;
        if (j0 == 0) {
            add(x0, wsh[0][r16]);
            add(x1, wsh[1][r16]);
            jj = 2;
        }
#pragma unroll 1
        for (; jj + 1 < nj; jj += 2) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                x0[c] = pbase[c * 256 + (j0 + jj) * jstride];
                x1[c] = pbase[c * 256 + (j0 + jj + 1) * jstride];
            }
            add(x0, wsh[jj][r16]);
            add(x1, wsh[jj + 1][r16]);
        }
        if (jj < nj) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) x0[c] = pbase[c * 256 + (j0 + jj) * jstride];
            add(x0, wsh[jj][r16]);
        }
        __syncthreads();  // before the next weight chunk overwrites wsh
    }
    if (m < M) {
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc[c].x, acc[c].y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(acc[c].z, acc[c].w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&lo);
            pk.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(out + ((int64_t)b * M + m) * kDv + 64 * (c0 + c) + 4 * cq) = pk;
        }
        if (c0 == 0 && cq == 0) lse[(int64_t)b * M + m] = (Msh[r16] == -INFINITY) ? -INFINITY : Lsh[r16] * kLn2;
    }
}

mla_status launch_combine(const void* ws, int B, int s_q, int H, void* out, float* lse, cudaStream_t stream) {
    // a performance choice only (either kernel is correct for any plan): requests average
    // (B + G) / B splits under the default plan
    const int sms = effective_sms();
    const int G = num_groups_for(sms > 0 ? sms : 1, num_row_blocks(s_q, H));
    const bool many_splits = (int64_t)B + G >= 8 * (int64_t)B;
    // with few splits a CTA takes all eight column chunks of its 16 rows when that still
    // leaves enough CTAs (the row weights are then computed once, and two splits' loads
    // for every chunk go out together), else two
    const int64_t row_groups = (int64_t)B * 4 * num_row_blocks(s_q, H);
    const int chunks = many_splits ? 1 : (row_groups >= 256 ? 8 : 2);
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(B, 4 * num_row_blocks(s_q, H), (kDv / 64) / chunks);
    cfg.blockDim = dim3(kTileThreads * (many_splits ? 4 : 1));
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
    const cudaError_t e = chunks == 1   ? cudaLaunchKernelEx(&cfg, combine_many_kernel<4>, ws, B, s_q, H, o, lse)
                          : chunks == 8 ? cudaLaunchKernelEx(&cfg, combine_few_kernel<8>, ws, B, s_q, H, o, lse)
                                        : cudaLaunchKernelEx(&cfg, combine_few_kernel<2>, ws, B, s_q, H, o, lse);
    if (e != cudaSuccess) return MLA_ERR_CUDA;
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
