// mla_absorb.cu -- the two per-head projections on either side of the latent attention
// ("absorb + project": the query is absorbed through W_UK before the scan and the
// output projected through W_UV after it; zhaifeiyue "TokenSpeed" notes, DeepSeek-V3
// entry).  Per head h, with W_UK[h] and W_UV[h] the [512 x 128] up-projections of the
// latent row c (k_nope = c W_UK[h], v = c W_UV[h]):
//     q[r, h, 0:512]   = W_UK[h] q_nope[r, h]      (so that q . c = q_nope . k_nope)
//     q[r, h, 512:576] = q_rope[r, h]              (the decoupled rope part, copied)
//     y[r, h, :]       = out[r, h, :] W_UV[h]      (128 wide)
//
// Both are batched GEMMs over heads with R = B * s_q rows per head, run on the tcgen05
// tensor cores in the transposed form D_h = A_h X_h^T, so that the MMA's 128-row M side
// is the weight's dimension (a full-rate tile at any R) and the rows r are its N side:
//     project: D[c, r] = sum_d W_UV[h][d][c] out[r, h, d]   M = 128 (c), K = 512 (d)
//              A = W_UV[h] read MN-major (c contiguous in memory)
//     absorb:  D[d, r] = sum_k W_UK[h][d][k] q_nope[r, h, k]   M = 512 (d, four tiles), K = 128
//              A = W_UK[h] read K-major (k contiguous)
// X_h^T is K-major in both (a row's K values are contiguous).  One CTA per (head, M tile,
// N tile of up to 256 rows): TMA brings 64-wide K chunks of A (128 x 64) and X (N x 64)
// into 128B-swizzled shared memory, in up to four stages; one thread issues the MMAs
// (M=128, N, K=16) into a TMEM accumulator of N fp32 columns; then the four warps read it
// back (warp w: lanes 32w..32w+31, i.e. 32 values of the M side) and write bf16 (nearest,
// ties to even).  The X boxes are three-dimensional, [K chunk, 1 head, N rows], so one
// head's rows land as a dense N x 128-byte tile.  Rows past R read as zeros (the box runs
// off the tensor) and are not written.
#include <cudaTypedefs.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "mla_decode_params.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kGemmThreads = 128;
constexpr int kKChunk = 64;                       // K per stage: one 128-byte swizzle row of bf16
constexpr int kMaxStages = 4;
constexpr uint32_t kATile = 128 * kKChunk * 2;    // 16 KB
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct __align__(64) GemmArgs {
    CUtensorMap tm_a;   // the weights: project {128 c, 512 d, H} box {64, 64, 1}; absorb {128 k, 512 d, H} box {64, 128, 1}
    CUtensorMap tm_x;   // the rows: {K, H, R} box {64, 1, N}
    __nv_bfloat16* y;   // output rows: y[r * y_rs + h * y_hs + m]
    int64_t y_rs, y_hs;
    const __nv_bfloat16* rope;  // absorb only: q_rope [R, H, 64], copied to y[..., 512:576]
    int R, H, N;        // rows, heads, N tile (a multiple of 16, <= 256)
    int32_t* status;    // where a bounded wait that gave up is recorded (null: these entry points have
                        // no workspace; a wait that gives up leaves its rows unwritten)
};

// Bounded mbarrier wait (2 s); false if it gave up.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, int32_t* status) {
    uint64_t t0 = 0;
    for (uint32_t n = 1;; ++n) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((n & 255) == 0) {
            const uint64_t now = ptx::globaltimer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kWaitLimitNs) {
                if (status) atomicCAS(status, 0, (int32_t)kStatusTimeout);
                return false;
            }
        }
    }
}

// kK: the contraction length (512 project, 128 absorb); kAMn: A read MN-major (project).
template <int kK, bool kAMn>
__global__ void __launch_bounds__(kGemmThreads, 1) head_gemm_sm100_kernel(const __grid_constant__ GemmArgs g) {
    constexpr int kChunks = kK / kKChunk;
    constexpr int kStages = kChunks < kMaxStages ? kChunks : kMaxStages;
    extern __shared__ uint8_t gsm_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int h = blockIdx.x, mt = blockIdx.y, n0 = blockIdx.z * g.N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t x_tile = (uint32_t)g.N * 128;        // N rows x 64 bf16
    const uint32_t stage_bytes = kATile + x_tile;
    const uint32_t off_bar = kStages * stage_bytes;      // full[kStages], empty[kStages], done
    auto bar = [&](int i) { return sbase + off_bar + 8u * (uint32_t)i; };
    const uint32_t holder = off_bar + 8u * (2 * kStages + 1);
    uint32_t ncols = 32;
    while ((int)ncols < g.N) ncols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar(s), 1);
            ptx::mbar_init(bar(kStages + s), 1);
        }
        ptx::mbar_init(bar(2 * kStages), 1);
        ptx::fence_mbar_init_cluster();
        ptx::prefetch_tmap(&g.tm_a);
        ptx::prefetch_tmap(&g.tm_x);
    }
    if (warp == 1) {
        ptx::tmem_alloc(sbase + holder, ncols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + holder);
    bool ok = true;

    if (warp == 0 && lane == 0) {
        // producer: chunk c into stage c % kStages, once the MMAs of chunk c - kStages are done
        for (int c = 0; c < kChunks && ok; ++c) {
            const int s = c % kStages;
            if (c >= kStages && !wait_bounded(bar(kStages + s), ((c / kStages) - 1) & 1, g.status)) {
                ok = false;
                break;
            }
            const uint32_t a_dst = sbase + s * stage_bytes, x_dst = a_dst + kATile;
            ptx::mbar_arrive_expect_tx(bar(s), stage_bytes);
            if (kAMn) {
                // W_UV[h] rows d in [64 c, +64), columns c in [0, 64) and [64, 128): two 8 KB
                // MN-major atoms (64 columns x 64 rows of 128 bytes)
                ptx::tma_load_3d(a_dst, &g.tm_a, bar(s), 0, kKChunk * c, h);
                ptx::tma_load_3d(a_dst + kATile / 2, &g.tm_a, bar(s), 64, kKChunk * c, h);
            } else {
                // W_UK[h] rows d in [128 mt, +128), columns k in [64 c, +64): K-major 128 x 128 B
                ptx::tma_load_3d(a_dst, &g.tm_a, bar(s), kKChunk * c, 128 * mt, h);
            }
            ptx::tma_load_3d(x_dst, &g.tm_x, bar(s), kKChunk * c, h, n0);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: four K=16 steps per chunk into one accumulator
        const uint32_t idesc = ptx::idesc_bf16_f32(128, g.N, kAMn ? 1 : 0, 0);
        for (int c = 0; c < kChunks && ok; ++c) {
            const int s = c % kStages;
            if (!wait_bounded(bar(s), (c / kStages) & 1, g.status)) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t a_src = sbase + s * stage_bytes, x_src = a_src + kATile;
            // MN-major A: 64-column atoms 8 KB apart (leading), 8 K-rows 1 KB apart (stride);
            // K-major A and X: 8 rows 1 KB apart (stride)
            const uint64_t a0 = kAMn ? ptx::smem_desc(a_src, kATile / 2, 1024, ptx::kSwizzle128)
                                     : ptx::smem_desc(a_src, 16, 1024, ptx::kSwizzle128);
            const uint64_t x0 = ptx::smem_desc(x_src, 16, 1024, ptx::kSwizzle128);
#pragma unroll
            for (int ks = 0; ks < kKChunk / 16; ++ks) {
                // K step: 16 values = 32 bytes along a K-major row, or 16 rows = 2 KB of an
                // MN-major atom
                const uint64_t a = a0 + (uint64_t)(kAMn ? ks * (2048 >> 4) : ks * 2);
                ptx::mma_ss(tmem, a, x0 + (uint64_t)(ks * 2), idesc, (c | ks) ? 1u : 0u);
            }
            ptx::mma_commit(bar(kStages + s));
        }
        ptx::mma_commit(bar(2 * kStages));
    }
    __syncwarp();
    // epilogue: every warp waits for the last MMA, then reads its 32 lanes (M side)
    const bool done = wait_bounded(bar(2 * kStages), 0, g.status);
    ptx::tc_fence_after();
    if (done) {
        const int m = 128 * mt + 32 * warp + lane;  // the output column this thread writes
        const uint32_t t_row = tmem + ((uint32_t)(32 * warp) << 16);
        for (int c0 = 0; c0 < g.N; c0 += 16) {
            uint32_t v[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                "%13, %14, %15}, [%16];"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                  "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                : "r"(t_row + (uint32_t)c0)
                : "memory");
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int r = n0 + c0 + j;
                if (r < g.R) g.y[(int64_t)r * g.y_rs + (int64_t)h * g.y_hs + m] = __float2bfloat16_rn(__uint_as_float(v[j]));
            }
        }
        if (g.rope && mt == 0) {
            // the query's rope part: y[r, h, 512:576] = q_rope[r, h, :] for this CTA's rows
            for (int e = threadIdx.x; e < g.N * 8; e += kGemmThreads) {
                const int r = n0 + (e >> 3), p8 = e & 7;
                if (r < g.R)
                    *reinterpret_cast<uint4*>(g.y + (int64_t)r * g.y_rs + (int64_t)h * g.y_hs + kDv + 8 * p8) =
                        *reinterpret_cast<const uint4*>(g.rope + ((int64_t)r * g.H + h) * 64 + 8 * p8);
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, ncols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// A 3-D bf16 tensor map: dims {d0, d1, d2} (d0 contiguous), byte strides of d1 and d2,
// box {b0, b1, b2}, 128-byte swizzle (b0 * 2 bytes = 128).
bool map_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
            uint32_t b0, uint32_t b1, uint32_t b2) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// N tile: R rounded up to 16, at most 256 (the TMEM columns of one accumulator), halved
// (down to 16) while the grid of (head, M tile, N tile) CTAs has fewer CTAs than the
// device has SMs: a CTA's time is mostly its loads' latency, so more, smaller CTAs finish
// sooner, and the weight tiles they share come from L2.
int n_tile(int R, int H, int m_tiles) {
    int n = std::min(256, (R + 15) / 16 * 16);
    const int sms = effective_sms();  // cached per device
    const int64_t want = sms > 0 ? sms : 148;
    while (n > 16 && (int64_t)H * m_tiles * ((R + n - 1) / n) < want) n = std::max(16, (n / 2 + 15) / 16 * 16);
    return n;
}

template <int kK>
constexpr size_t gemm_smem_bytes(int N) {
    return (size_t)(kK / kKChunk < kMaxStages ? kK / kKChunk : kMaxStages) * (kATile + (size_t)N * 128) +
           8 * (2 * kMaxStages + 1) + 16 + 1024;
}

template <int kK, bool kAMn>
mla_status launch_head_gemm(const GemmArgs& g, int m_tiles, cudaStream_t st) {
    // the shared memory opt-in, set once per device for the largest tile (N = 256)
    static int done[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev >= 64 || !done[dev]) {
        if (cudaFuncSetAttribute(head_gemm_sm100_kernel<kK, kAMn>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm_smem_bytes<kK>(256)) != cudaSuccess)
            return MLA_ERR_CUDA;
        if (dev < 64) done[dev] = 1;
    }
    const size_t smem = gemm_smem_bytes<kK>(g.N);
    const dim3 grid(g.H, m_tiles, (g.R + g.N - 1) / g.N);
    head_gemm_sm100_kernel<kK, kAMn><<<grid, kGemmThreads, smem, st>>>(g);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace mla

extern "C" mla_status mla_absorb_q(const void* q_nope, const void* q_rope, const void* w_uk, int R, int H, void* q,
                                   void* stream) {
    using namespace mla;
    if (!q_nope || !q_rope || !w_uk || !q || R <= 0 || H <= 0) return MLA_ERR_INVALID_ARG;
    if (!aligned(q_nope, 16) || !aligned(w_uk, 16) || !aligned(q_rope, 16) || !aligned(q, 16)) return MLA_ERR_INVALID_ARG;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.N = n_tile(R, H, kDv / 128);
    // A = W_UK [H][512 d][128 k]: box of 64 k x 128 d of one head
    if (!map_3d(&g.tm_a, w_uk, 128, kDv, (uint64_t)H, 128 * 2, (uint64_t)kDv * 128 * 2, 64, 128, 1)) return MLA_ERR_CUDA;
    // X = q_nope [R][H][128 k]: box of 64 k x 1 head x N rows
    if (!map_3d(&g.tm_x, q_nope, 128, (uint64_t)H, (uint64_t)R, 128 * 2, (uint64_t)H * 128 * 2, 64, 1, g.N))
        return MLA_ERR_CUDA;
    g.y = reinterpret_cast<__nv_bfloat16*>(q);
    g.y_rs = (int64_t)H * kDqk;
    g.y_hs = kDqk;
    g.rope = reinterpret_cast<const __nv_bfloat16*>(q_rope);
    g.R = R;
    g.H = H;
    return launch_head_gemm<128, false>(g, kDv / 128, (cudaStream_t)stream);
}

extern "C" mla_status mla_project_out(const void* out, const void* w_uv, int R, int H, void* y, void* stream) {
    using namespace mla;
    if (!out || !w_uv || !y || R <= 0 || H <= 0) return MLA_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(w_uv, 16) || !aligned(y, 4)) return MLA_ERR_INVALID_ARG;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.N = n_tile(R, H, 1);
    // A = W_UV [H][512 d][128 c]: box of 64 c x 64 d of one head (MN-major atoms)
    if (!map_3d(&g.tm_a, w_uv, 128, kDv, (uint64_t)H, 128 * 2, (uint64_t)kDv * 128 * 2, 64, 64, 1)) return MLA_ERR_CUDA;
    // X = out [R][H][512 d]: box of 64 d x 1 head x N rows
    if (!map_3d(&g.tm_x, out, kDv, (uint64_t)H, (uint64_t)R, kDv * 2, (uint64_t)H * kDv * 2, 64, 1, g.N))
        return MLA_ERR_CUDA;
    g.y = reinterpret_cast<__nv_bfloat16*>(y);
    g.y_rs = (int64_t)H * 128;
    g.y_hs = 128;
    g.R = R;
    g.H = H;
    return launch_head_gemm<kDv, true>(g, 1, (cudaStream_t)stream);
}
