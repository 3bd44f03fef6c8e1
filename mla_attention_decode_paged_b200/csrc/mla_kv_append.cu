// mla_kv_append.cu -- the write side of the paged latent cache: the s_q new rows of each
// request (the draft tokens the decode verifies) go to positions T_b - s_q + i, through
// the block table [llm-atlas "Inference systems", 07 PagedAttention], with the 64-wide
// decoupled rope key rotated by its position [llm-atlas "Inference systems", 22
// DeepSeek V2->V3].
//
// Rotation of adjacent pairs, j < 32:
//     (x[2j], x[2j+1]) -> (x[2j] c - x[2j+1] s, x[2j] s + x[2j+1] c),
// c and s read from the caller's rope table [max_pos][64] (32 cosines, then 32 sines).
// The stored value is a rounding decision, so the arithmetic is pinned: binary32
// products and sums, each rounded (no fused multiply-add), then bf16 round-to-nearest-
// even, or for an e4m3 cache e4m3(value / kv_scale) with a rounded binary32 division and
// round-to-nearest-even saturating conversion.
//
// One warp per new row: each lane moves 32 bytes of the 1,024-byte latent part and one
// rotated pair of the rope part.  The kernel is bound by launch latency at decode sizes.
#include <cuda_fp8.h>
#include <math.h>

#include "mla_common.cuh"

namespace mla {
namespace {

constexpr int kAppendWarps = 8;

__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    const __nv_fp8x2_storage_t v = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)v;
}

template <int KV>
__global__ void __launch_bounds__(32 * kAppendWarps) kv_append_kernel(
    const __nv_bfloat16* __restrict__ ckv, const __nv_bfloat16* __restrict__ kpe, const float* __restrict__ cos_sin,
    int max_pos, uint8_t* __restrict__ pool, float kv_scale, const int32_t* __restrict__ block_table, int max_pages,
    const int32_t* __restrict__ seq_lens, int B, int s_q, int64_t num_pages, int32_t* status) {
    constexpr bool kE4m3 = KV == MLA_KV_E4M3;
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    if (r >= (int64_t)B * s_q) return;
    const int b = (int)(r / s_q), i = (int)(r % s_q);
    // the new row's values do not depend on where it goes: their loads are issued first,
    // beside the length's, so that the dependent loads (page id, rope table) follow in one
    // more round trip
    const uint4* src = reinterpret_cast<const uint4*>(ckv + r * kDv) + 2 * lane;
    const uint4 a = src[0], c = src[1];
    const __nv_bfloat162 x = reinterpret_cast<const __nv_bfloat162*>(kpe + r * 64)[lane];
    const int T = seq_lens[b];
    const int pos = T - s_q + i;
    bool ok = T >= s_q && (int64_t)T <= (int64_t)max_pages * kPage && pos < max_pos;
    int32_t page = -1;
    float cj = 0.f, sj = 0.f;
    if (ok) {
        page = block_table[(int64_t)b * max_pages + pos / kPage];
        cj = cos_sin[(int64_t)pos * 64 + lane];
        sj = cos_sin[(int64_t)pos * 64 + 32 + lane];
        ok = page >= 0 && page < num_pages;
    }
    if (!ok) {
        if (lane == 0 && status) atomicCAS(status, 0, (int32_t)kStatusOob);
        return;
    }
    const int64_t row = (int64_t)page * kPage + pos % kPage;
    // latent part: 16 values per lane
    if (!kE4m3) {
        uint4* dst = reinterpret_cast<uint4*>(pool + row * (kDqk * 2)) + 2 * lane;
        dst[0] = a;
        dst[1] = c;
    } else {
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
        uint32_t q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float f[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&w[2 * k + h]);
                f[2 * h] = __fdiv_rn(__low2float(v2), kv_scale);
                f[2 * h + 1] = __fdiv_rn(__high2float(v2), kv_scale);
            }
            q[k] = e4m3x2(f[0], f[1]) | (e4m3x2(f[2], f[3]) << 16);
        }
        *reinterpret_cast<uint4*>(pool + row * kDqk + 16 * lane) = make_uint4(q[0], q[1], q[2], q[3]);
    }
    // rope part: lane j rotates the pair (2j, 2j + 1)
    const float x0 = __low2float(x), x1 = __high2float(x);
    const float r0 = __fsub_rn(__fmul_rn(x0, cj), __fmul_rn(x1, sj));
    const float r1 = __fadd_rn(__fmul_rn(x0, sj), __fmul_rn(x1, cj));
    if (!kE4m3) {
        reinterpret_cast<__nv_bfloat162*>(pool + row * (kDqk * 2) + kDv * 2)[lane] = __floats2bfloat162_rn(r0, r1);
    } else {
        reinterpret_cast<uint16_t*>(pool + row * kDqk + kDv)[lane] =
            (uint16_t)e4m3x2(__fdiv_rn(r0, kv_scale), __fdiv_rn(r1, kv_scale));
    }
}

}  // namespace
}  // namespace mla

extern "C" mla_status mla_kv_append(const void* ckv_new, const void* kpe_new, const float* rope_cos_sin, int max_pos,
                                    void* kv_pages, int kv_dtype, float kv_scale, const int32_t* block_table,
                                    int max_pages_per_req, const int32_t* seq_lens, int B, int s_q,
                                    int64_t num_pages, int32_t* status, void* stream) {
    using namespace mla;
    if (!ckv_new || !kpe_new || !rope_cos_sin || !kv_pages || !block_table || !seq_lens) return MLA_ERR_INVALID_ARG;
    if (B <= 0 || s_q <= 0 || max_pos <= 0 || max_pages_per_req <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
    if (kv_dtype != MLA_KV_BF16 && kv_dtype != MLA_KV_E4M3) return MLA_ERR_INVALID_ARG;
    if (kv_dtype == MLA_KV_E4M3 && !(kv_scale > 0.f && isfinite(kv_scale))) return MLA_ERR_INVALID_ARG;
    if ((((uintptr_t)ckv_new) & 15) || (((uintptr_t)kv_pages) & 15) || (((uintptr_t)kpe_new) & 3) ||
        (((uintptr_t)rope_cos_sin) & 3) || (((uintptr_t)block_table) & 3) || (((uintptr_t)seq_lens) & 3) ||
        (((uintptr_t)status) & 3))
        return MLA_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * s_q;
    const dim3 grid((unsigned)((rows + kAppendWarps - 1) / kAppendWarps));
    cudaStream_t st = (cudaStream_t)stream;
    const auto* ckv = reinterpret_cast<const __nv_bfloat16*>(ckv_new);
    const auto* kpe = reinterpret_cast<const __nv_bfloat16*>(kpe_new);
    auto* pool = reinterpret_cast<uint8_t*>(kv_pages);
    if (kv_dtype == MLA_KV_E4M3)
        kv_append_kernel<MLA_KV_E4M3><<<grid, 32 * kAppendWarps, 0, st>>>(
            ckv, kpe, rope_cos_sin, max_pos, pool, kv_scale, block_table, max_pages_per_req, seq_lens, B, s_q,
            num_pages, status);
    else
        kv_append_kernel<MLA_KV_BF16><<<grid, 32 * kAppendWarps, 0, st>>>(
            ckv, kpe, rope_cos_sin, max_pos, pool, kv_scale, block_table, max_pages_per_req, seq_lens, B, s_q,
            num_pages, status);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
