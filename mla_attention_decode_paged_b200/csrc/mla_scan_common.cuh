// mla_scan_common.cuh -- pieces shared by the two split-scan kernels (bf16 cache in
// mla_decode_sm100.cu, e4m3 cache in mla_decode_sm100_e4m3.cu): the CTA's barrier
// context and its bounded waits, the per-request checks, the rows written for a request
// the scan must poison, and the epilogue that turns the TMEM accumulator into the bf16
// output or an fp32 split partial.
//
// Both kernels use the same CTA roles: warp 0 TMA producer, warp 1 MMA issuer, warps 2-5
// softmax and epilogue (192 threads; the bf16 scan adds warp 6, a second score issuer),
// one block of 64 folded query rows, 64-row tcgen05 MMAs whose rows occupy 16 lanes of
// each 32-lane TMEM subpartition: O (64 x 512 fp32) in the lanes at offset 0, q and the
// scores in the lanes at offset 16.
#pragma once

#include <cudaTypedefs.h>

#include "mla_decode_params.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace scan {

constexpr int kRows = kRowsPerBlock;  // 64 folded rows per CTA (MMA M)
constexpr int kTok = 64;              // tokens per page
constexpr int kThreads = 192;         // warp 0 TMA, warp 1 MMA, warps 2-5 softmax / epilogue
static_assert(kRows == 64, "the TMEM layout is the 64-row MMA layout");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kLaneHi = 16u << 16;  // second half-subpartition lane set (q and scores)
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kEpiWarpBytes = 16 * 128;  // epilogue staging per softmax warp
constexpr int kMaxSmem = 232448;              // dynamic shared memory per block, opt-in maximum

struct __align__(64) Args {
    CUtensorMap tm_kv;  // the cache viewed as [P * 64 rows, 576 columns]
    DecodeParams p;
};

struct Ctx {
    uint32_t bar0;
    volatile int* abort;
    PlanHeader* h;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
};

// Bounded wait: gives up after kLimitNs (sets the timeout status and the CTA abort flag),
// or at once once the CTA is aborting.
template <uint64_t kLimitNs>
__device__ __noinline__ bool wait_bar_for(const Ctx& c, uint32_t bar, uint32_t parity) {
    if (*c.abort) return false;
    uint64_t t0 = 0;
    for (uint32_t n = 1;; ++n) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((n & 255) == 0) {
            if (*c.abort) return false;
            const uint64_t now = ptx::globaltimer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kLimitNs) {
                *c.abort = 1;
                set_status(c.h, kStatusTimeout, (int)blockIdx.x);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar(const Ctx& c, uint32_t bar, uint32_t parity) {
    return wait_bar_for<kWaitLimitNs>(c, bar, parity);
}

// Wait that ignores the abort flag, used only on the way out for work already in flight.
static __device__ __noinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > 200000000ull) return;
    }
}

// The MMA issuer's own bounded poll: progress resets the clock; after kWaitLimitNs without
// progress the CTA aborts with the timeout status.  Returns false to stop issuing.
struct PollClock {
    uint64_t t0 = 0;
    uint32_t spins = 0;
    __device__ bool step(const Ctx& c, bool progressed) {
        if (progressed) {
            t0 = 0;
            spins = 0;
            return true;
        }
        if ((++spins & 255) != 0) return true;
        if (*c.abort) return false;
        const uint64_t now = ptx::globaltimer_ns();
        if (t0 == 0) {
            t0 = now;
        } else if (now - t0 > kWaitLimitNs) {
            *c.abort = 1;
            set_status(c.h, kStatusTimeout, (int)blockIdx.x);
            return false;
        }
        return true;
    }
};

__device__ __forceinline__ bool request_ok(const DecodeParams& p, int T) {
    return T >= 1 && (int64_t)T <= (int64_t)p.max_pages * kPage && !(p.causal && T < p.s_q);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Four floats -> (e4m3 word of x, e4m3 word of the residual x - e4m3(x)), bytes in order.
__device__ __forceinline__ void split_e4m3x4(float x0, float x1, float x2, float x3, uint32_t& hi, uint32_t& lo) {
    const uint16_t h01 = ptx::f32x2_to_e4m3x2(x0, x1), h23 = ptx::f32x2_to_e4m3x2(x2, x3);
    const float2 f01 = e4m3x2_to_float2(h01), f23 = e4m3x2_to_float2(h23);
    hi = (uint32_t)h01 | ((uint32_t)h23 << 16);
    lo = (uint32_t)ptx::f32x2_to_e4m3x2(x0 - f01.x, x1 - f01.y) |
         ((uint32_t)ptx::f32x2_to_e4m3x2(x2 - f23.x, x3 - f23.y) << 16);
}

// Where one softmax thread's results go: thread (row, half) of warp quadrant `quad` owns
// folded row qb * 64 + row and, in the epilogue, the columns [64 q + 32 half, +32).
struct RowSlot {
    int quad, half, r16, lane, row, qb, nqb;
    int m_glob;
    bool row_valid;
};

// A request the scan cannot process (bad length): its rows become NaN, in the output if
// the split holds the request whole, else in its partial (the combine then spreads them).
__device__ __forceinline__ void poison_rows(const DecodeParams& p, const Segment& S, int si, const RowSlot& r,
                                            float* po, float* plse) {
    if (!r.row_valid) return;
    const float nanv = __int_as_float(0x7fc00000);
    const int64_t orow = (int64_t)S.b * p.M + r.m_glob;
    if (!S.split) {
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + orow * kDv + 256 * r.half;
        for (int k = 0; k < 256; ++k) dst[k] = __float2bfloat16_rn(nanv);
        if (r.half == 0) p.lse[orow] = nanv;
    } else {
        // the row's columns [256 half, +256) in the quad-interleaved partial layout
        float* blk = po + ((int64_t)si * r.nqb + r.qb) * kRows * kDv + (r.row >> 4) * 8192 + (r.row & 15) * 4;
        for (int k = 0; k < 256; ++k) {
            const int col = 256 * r.half + k;
            blk[(col >> 2) * 64 + (col & 3)] = nanv;
        }
        if (r.half == 0) plse[((int64_t)si * r.nqb + r.qb) * kRows + r.row] = nanv;
    }
}

// Epilogue of one split: O * inv from TMEM (t_lo: this warp's O lanes) and lse2 (base 2).
// A split writes its fp32 partial in the workspace's quad-interleaved layout (column quads
// outermost, then the warp's 16 rows): each store instruction of the warp covers two whole
// 256-byte runs.  A request held whole goes to the bf16 output, row-major, through a 2 KB
// staging tile per warp (16 rows x 128 bytes, 16-byte pieces XOR-swizzled by row) so that
// every store writes whole row segments.  Two register sets: the next chunk's TMEM load is
// in flight while one is stored.  The loop is not unrolled: this code runs once per split,
// from a cold instruction cache, so its size costs more than its loop overhead.
__device__ __forceinline__ void store_split(const DecodeParams& p, const Segment& S, int si, const RowSlot& r,
                                            uint32_t t_lo, uint8_t* stg, float inv, float lse2, float* po,
                                            float* plse) {
    const int rows_ok = min(16, p.M - (r.qb * kRows + r.quad * 16));  // valid rows of this warp
    const int64_t out_row0 = (int64_t)S.b * p.M + r.qb * kRows + r.quad * 16;
    float4* pq = reinterpret_cast<float4*>(po + ((int64_t)si * r.nqb + r.qb) * kRows * kDv) + r.quad * 2048 +
                 8 * r.half * 16 + r.r16;  // + (16 q + v) * 16 for columns 64 q + 32 half + 4 v
    auto store_chunk = [&](int q, const uint32_t(&oq)[32]) {
        if (!S.split) {
            // bf16: the row's 64 columns are 8 pieces; this thread holds pieces 4 half + w
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint4 v;
                v.x = pack_bf16(__uint_as_float(oq[8 * w + 0]) * inv, __uint_as_float(oq[8 * w + 1]) * inv);
                v.y = pack_bf16(__uint_as_float(oq[8 * w + 2]) * inv, __uint_as_float(oq[8 * w + 3]) * inv);
                v.z = pack_bf16(__uint_as_float(oq[8 * w + 4]) * inv, __uint_as_float(oq[8 * w + 5]) * inv);
                v.w = pack_bf16(__uint_as_float(oq[8 * w + 6]) * inv, __uint_as_float(oq[8 * w + 7]) * inv);
                *reinterpret_cast<uint4*>(stg + r.r16 * 128 + (((4 * r.half + w) ^ (r.r16 & 7)) << 4)) = v;
            }
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int idx = r.lane + 32 * j, rr = idx >> 3, w = idx & 7;
                const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((w ^ (rr & 7)) << 4));
                if (rr < rows_ok)
                    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + (out_row0 + rr) * kDv +
                                              64 * q + 8 * w) = v;
            }
            __syncwarp();
        } else if (r.row_valid) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
                pq[(16 * q + v) * 16] =
                    make_float4(__uint_as_float(oq[4 * v]) * inv, __uint_as_float(oq[4 * v + 1]) * inv,
                                __uint_as_float(oq[4 * v + 2]) * inv, __uint_as_float(oq[4 * v + 3]) * inv);
        }
    };
    uint32_t oa[32], ob[32];
    ptx::tmem_ld16x32<32>(t_lo, oa);
#pragma unroll 1
    for (int q = 0; q < 8; q += 2) {
        ptx::tmem_wait_ld();
        ptx::tmem_ld16x32<32>(t_lo + 64u * (q + 1), ob);
        store_chunk(q, oa);
        ptx::tmem_wait_ld();
        if (q + 2 < 8) ptx::tmem_ld16x32<32>(t_lo + 64u * (q + 2), oa);
        store_chunk(q + 1, ob);
    }
    if (r.row_valid && r.half == 0) {
        if (!S.split)
            p.lse[(int64_t)S.b * p.M + r.m_glob] = lse2 * kLn2;
        else
            plse[((int64_t)si * r.nqb + r.qb) * kRows + r.row] = lse2;
    }
}

// Rescale this thread's half of O (columns [32 half + 64 q, +32), q = 0..7) by f.
__device__ __forceinline__ void rescale_o(uint32_t t_lo, float f) {
#pragma unroll 1
    for (int q = 0; q < 8; ++q) {
        uint32_t o[32];
        ptx::tmem_ld16x32<32>(t_lo + 64u * q, o);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
        ptx::tmem_st16x32<32>(t_lo + 64u * q, o);
    }
    ptx::tmem_wait_st();
}

}  // namespace scan

// Host: a 2-D tiled tensor map over the cache (defined in mla_decode_sm100.cu).
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
                 uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw);
mla_status launch_decode_e4m3(const DecodeParams& p, cudaStream_t stream);

}  // namespace mla
