// mla_absorb.cu -- the two per-head projections on either side of the latent attention
// ("absorb + project": the query is absorbed through W_UK before the scan and the
// output projected through W_UV after it; zhaifeiyue "TokenSpeed" notes, DeepSeek-V3
// entry).  Per head h, with W_UK[h] and W_UV[h] the [512 x 128] up-projections of the
// latent row c (k_nope = c W_UK[h], v = c W_UV[h]):
//     q[r, h, 0:512]   = W_UK[h] q_nope[r, h]      (so that q . c = q_nope . k_nope)
//     q[r, h, 512:576] = q_rope[r, h]              (the decoupled rope part, copied)
//     y[r, h, :]       = out[r, h, :] W_UV[h]      (128 wide)
// Both are a batched GEMM over heads, Y_h = X_h B_h with B_h = W_UK[h]^T (K = 128,
// N = 512) or W_UV[h] (K = 512, N = 128), and R = B * s_q rows per head.  At decode
// sizes (R = 16..256) the weights dominate the bytes (128 KB per head and matrix); the
// contraction runs on the CUDA cores in fp32 (16 rows per CTA are too few for a 64- or
// 128-row tensor-core tile) and the result is rounded to bf16 (nearest, ties to even).
#include <math.h>

#include <algorithm>

#include "mla_common.cuh"

namespace mla {
namespace {

constexpr int kBN = 32;              // output columns per CTA
constexpr int kRB = 16;              // query rows per CTA
constexpr int kAbsorbThreads = 256;  // 8 warps, each a slice of the contraction
constexpr int kKWarps = kAbsorbThreads / 32;

// Y[r, h, n] (row stride y_rs, head stride y_hs) = sum_k X[r, h, k] * B_h[k, n], with
// X[r, h, k] at x + r * x_rs + h * K + k and B_h[k, n] at w + h * K * N + (B_T ? n * K + k
// : k * N + n).  A CTA takes 32 output columns of one head and every gridDim.z-th block of
// 16 rows: the weight tile (K x 32, read once with 16-byte loads, all in flight together)
// and each block's rows go to shared memory;
// each warp contracts one eighth of K for the whole 16 x 32 tile (a lane holds a 4 x 4
// block: 16 independent accumulators), and the eight partial tiles are added in shared
// memory.
template <bool B_T, int K, int N>
__global__ void __launch_bounds__(kAbsorbThreads) head_gemm_kernel(const __nv_bfloat16* __restrict__ x, int64_t x_rs,
                                                                  const __nv_bfloat16* __restrict__ w,
                                                                  __nv_bfloat16* __restrict__ y, int64_t y_rs,
                                                                  int64_t y_hs, int R,
                                                                  const __nv_bfloat16* __restrict__ rope) {
    extern __shared__ __align__(16) uint8_t absorb_smem[];
    __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(absorb_smem);                 // [K][kBN]
    float* xs = reinterpret_cast<float*>(absorb_smem + K * kBN * 2);                    // [K][kRB]
    float* red = xs + K * kRB;                                                          // [kKWarps][kRB][kBN]
    const int n0 = blockIdx.x * kBN, h = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const __nv_bfloat16* wh = w + (int64_t)h * K * N;
    if (B_T) {
        // rows n0..n0+31 of W (K contiguous values each), transposed into wt[k][n]
        for (int e = tid; e < kBN * (K / 8); e += kAbsorbThreads) {
            const int nn = e / (K / 8), k8 = e % (K / 8);
            const uint4 v = *reinterpret_cast<const uint4*>(wh + (int64_t)(n0 + nn) * K + 8 * k8);
            const __nv_bfloat16* pv = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
            for (int j = 0; j < 8; ++j) wt[(8 * k8 + j) * kBN + nn] = pv[j];
        }
    } else {
        // columns n0..n0+31 of each of the K rows (64 contiguous bytes per row)
        for (int e = tid; e < K * (kBN / 8); e += kAbsorbThreads) {
            const int kk = e / (kBN / 8), c8 = e % (kBN / 8);
            *reinterpret_cast<uint4*>(wt + kk * kBN + 8 * c8) =
                *reinterpret_cast<const uint4*>(wh + (int64_t)kk * N + n0 + 8 * c8);
        }
    }
    // row blocks blockIdx.z, blockIdx.z + gridDim.z, ...: the weight tile is loaded once
    for (int r0 = blockIdx.z * kRB; r0 < R; r0 += gridDim.z * kRB) {
        __syncthreads();  // the previous block's rows and partial tiles are consumed
        // the block's 16 rows, transposed to xs[k][row] in fp32
        for (int e = tid; e < kRB * (K / 8); e += kAbsorbThreads) {
            const int rr = e / (K / 8), k8 = e % (K / 8);
            const int r = r0 + rr;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r < R) v = *reinterpret_cast<const uint4*>(x + (int64_t)r * x_rs + (int64_t)h * K + 8 * k8);
            const __nv_bfloat16* pv = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
            for (int j = 0; j < 8; ++j) xs[(8 * k8 + j) * kRB + rr] = __bfloat162float(pv[j]);
        }
        if (rope && blockIdx.x == 0) {
            // the query's rope part: y[r, h, 512:576] = rope[r, h, :] for this CTA's rows
            for (int e = tid; e < kRB * 8; e += kAbsorbThreads) {
                const int rr = e >> 3, p8 = e & 7, r = r0 + rr;
                if (r < R)
                    *reinterpret_cast<uint4*>(y + (int64_t)r * y_rs + (int64_t)h * y_hs + kDv + 8 * p8) =
                        *reinterpret_cast<const uint4*>(rope + ((int64_t)r * gridDim.y + h) * 64 + 8 * p8);
            }
        }
        __syncthreads();
        const int rg = lane >> 3, cg = lane & 7;  // rows 4 rg .. 4 rg + 3, columns 4 cg .. 4 cg + 3
        float acc[4][4] = {};
        constexpr int kSlice = K / kKWarps;
#pragma unroll 4
        for (int kk = warp * kSlice; kk < (warp + 1) * kSlice; ++kk) {
            const float4 xv = *reinterpret_cast<const float4*>(xs + kk * kRB + 4 * rg);
            const uint2 wb = *reinterpret_cast<const uint2*>(wt + kk * kBN + 4 * cg);
            const float2 w01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb.x));
            const float2 w23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wb.y));
            const float xr[4] = {xv.x, xv.y, xv.z, xv.w}, wc[4] = {w01.x, w01.y, w23.x, w23.y};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xr[i], wc[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4*>(red + (warp * kRB + 4 * rg + i) * kBN + 4 * cg) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        __syncthreads();
        // the eight partial tiles, added in warp order (a fixed order: deterministic)
        for (int o = tid; o < kRB * kBN / 2; o += kAbsorbThreads) {
            const int rr = o / (kBN / 2), c = 2 * (o % (kBN / 2));
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int q = 0; q < kKWarps; ++q) {
                s0 += red[(q * kRB + rr) * kBN + c];
                s1 += red[(q * kRB + rr) * kBN + c + 1];
            }
            const int r = r0 + rr;
            if (r < R)
                *reinterpret_cast<__nv_bfloat162*>(y + (int64_t)r * y_rs + (int64_t)h * y_hs + n0 + c) =
                    __floats2bfloat162_rn(s0, s1);
        }
    }
}

template <bool B_T, int K, int N>
cudaError_t launch_head_gemm(const __nv_bfloat16* x, int64_t x_rs, const __nv_bfloat16* w, __nv_bfloat16* y,
                             int64_t y_rs, int64_t y_hs, int R, int H, const __nv_bfloat16* rope, cudaStream_t st) {
    constexpr int kSmem = K * kBN * 2 + K * kRB * 4 + kKWarps * kRB * kBN * 4;
    if (kSmem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(head_gemm_kernel<B_T, K, N>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
    }
    // at most four CTAs share a (head, column tile): each reads the weight tile once
    const int zblocks = std::min((R + kRB - 1) / kRB, 4);
    head_gemm_kernel<B_T, K, N><<<dim3(N / kBN, H, zblocks), kAbsorbThreads, kSmem, st>>>(
        x, x_rs, w, y, y_rs, y_hs, R, rope);
    return cudaGetLastError();
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace mla

extern "C" mla_status mla_absorb_q(const void* q_nope, const void* q_rope, const void* w_uk, int R, int H, void* q,
                                   void* stream) {
    using namespace mla;
    if (!q_nope || !q_rope || !w_uk || !q || R <= 0 || H <= 0) return MLA_ERR_INVALID_ARG;
    if (!aligned(q_nope, 16) || !aligned(w_uk, 16) || !aligned(q_rope, 16) || !aligned(q, 16)) return MLA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    // X = q_nope [R, H, 128]; B_h = W_UK[h]^T: W_UK[h] is [512 x 128], contiguous along k
    if (launch_head_gemm<true, 128, kDv>(reinterpret_cast<const __nv_bfloat16*>(q_nope), (int64_t)H * 128,
                                         reinterpret_cast<const __nv_bfloat16*>(w_uk), reinterpret_cast<__nv_bfloat16*>(q),
                                         (int64_t)H * kDqk, kDqk, R, H,
                                         reinterpret_cast<const __nv_bfloat16*>(q_rope), st) != cudaSuccess)
        return MLA_ERR_CUDA;
    return MLA_OK;
}

extern "C" mla_status mla_project_out(const void* out, const void* w_uv, int R, int H, void* y, void* stream) {
    using namespace mla;
    if (!out || !w_uv || !y || R <= 0 || H <= 0) return MLA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(w_uv, 16) || !aligned(y, 4)) return MLA_ERR_INVALID_ARG;
    // X = out [R, H, 512]; B_h = W_UV[h] [512 x 128], contiguous along n
    return launch_head_gemm<false, kDv, 128>(reinterpret_cast<const __nv_bfloat16*>(out), (int64_t)H * kDv,
                                             reinterpret_cast<const __nv_bfloat16*>(w_uv),
                                             reinterpret_cast<__nv_bfloat16*>(y), (int64_t)H * 128, 128, R, H, nullptr,
                                             (cudaStream_t)stream) == cudaSuccess
               ? MLA_OK
               : MLA_ERR_CUDA;
}
