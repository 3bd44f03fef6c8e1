// mla_common.cuh -- internal definitions shared by the planner, the decode kernels
// and the combine kernel of libmla_decode.so: workspace layout, plan records,
// status words and small device helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mla_decode.h"

namespace mla {

constexpr int kDqk = MLA_HEAD_DIM_QK;  // 512 latent + 64 rope
constexpr int kDv = MLA_HEAD_DIM_V;
constexpr int kPage = MLA_PAGE_SIZE;
constexpr int kRowsPerBlock = 64;      // folded query rows per row block (one CTA, MMA M = 64)
constexpr int kMaxRows = 256;          // s_q * H supported per request
constexpr int kMaxGroups = 1023;       // plan groups (a request has at most groups + 1 splits)
constexpr int32_t kPlanMagic = 0x4d4c4131;  // "MLA1"

// Device-side error codes (mirror mla_status values).
enum : int32_t { kStatusOk = 0, kStatusOob = MLA_ERR_DEVICE_OOB, kStatusTimeout = MLA_ERR_DEVICE_TIMEOUT,
                 kStatusPlanMismatch = MLA_ERR_PLAN_MISMATCH };

// One split of one request: pages [tile_begin, tile_end) of request b.
struct __align__(16) Segment {
    int32_t b;
    int32_t tile_begin;
    int32_t tile_end;
    int32_t split;  // 1 if the request is cut into several segments (partials + combine)
};

// Workspace header, written by the plan kernel, read by decode and combine.
struct __align__(16) PlanHeader {
    int32_t status;       // first device error code (0 = none)
    int32_t status_info;  // request index of the first error
    int32_t magic;
    int32_t B, s_q, H;
    int32_t nqb;          // row blocks per request: ceil(s_q*H / 128)
    int32_t num_groups;   // groups of CTAs; all CTAs of a group scan the same pages
    int32_t num_segments;
    int32_t max_segments;
    int32_t total_tiles;
    int32_t pad0;
    int64_t off_group_begin;  // int32 [num_groups + 1]
    int64_t off_req_seg;      // int32 [B + 1]
    int64_t off_segs;         // Segment [max_segments]
    int64_t off_plse;         // float [max_segments][nqb][64]   (log2 domain)
    int64_t off_po;           // float [max_segments][nqb][4][128][16][4]: per 16-row group of a
                              // 64-row block, column quads outermost, the group's 16 rows next,
                              // the quad's 4 columns innermost (row r, column c of the block at
                              // (r / 16) * 8192 + (c / 4) * 64 + (r % 16) * 4 + c % 4)
    int64_t total_bytes;
};

// A group's segment range and its first segment, at a fixed place in the workspace
// (kOffHeads + 32 g): a scan CTA reads it together with the plan header, so that its first
// page loads wait for one round trip to memory instead of three.
struct __align__(16) GroupHead {
    int32_t seg_lo, seg_hi;  // the group's segments [seg_lo, seg_hi)
    int32_t pad0, pad1;
    Segment first;           // segment seg_lo (zeros for a group without pages)
};
constexpr int64_t kOffHeads = 256;
static_assert(sizeof(PlanHeader) <= kOffHeads, "the head table follows the header");

struct WsLayout {
    int64_t off_heads, off_group_begin, off_req_seg, off_segs, off_plse, off_po, total;
    int nqb, num_groups, max_segments;
};

__host__ __device__ inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline int num_row_blocks(int s_q, int H) {
    return (s_q * H + kRowsPerBlock - 1) / kRowsPerBlock;
}

// Groups of CTAs for a device with num_sms SMs (one scan CTA per SM): every group holds
// nqb CTAs (one per row block) so that the CTAs of a group read the same pages at the
// same time and share them through L2.
__host__ __device__ inline int num_groups_for(int num_sms, int nqb) {
    int g = num_sms / nqb;
    return g < 1 ? 1 : g;
}

__host__ __device__ inline WsLayout make_layout(int B, int s_q, int H, int num_groups) {
    WsLayout L;
    L.nqb = num_row_blocks(s_q, H);
    L.num_groups = num_groups;
    L.max_segments = B + num_groups;
    int64_t o = kOffHeads;
    L.off_heads = o;
    o = align_up(o + (int64_t)sizeof(GroupHead) * num_groups, 256);
    L.off_group_begin = o;
    o = align_up(o + 4 * (int64_t)(num_groups + 1), 256);
    L.off_req_seg = o;
    o = align_up(o + 4 * (int64_t)(B + 1), 256);
    L.off_segs = o;
    o = align_up(o + (int64_t)sizeof(Segment) * L.max_segments, 256);
    L.off_plse = o;
    o = align_up(o + 4 * (int64_t)L.max_segments * L.nqb * kRowsPerBlock, 256);
    L.off_po = o;
    o = align_up(o + 4 * (int64_t)L.max_segments * L.nqb * kRowsPerBlock * kDv, 256);
    L.total = o;
    return L;
}

template <typename T>
__device__ __forceinline__ T* ws_ptr(void* ws, int64_t off) {
    return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off);
}
template <typename T>
__device__ __forceinline__ const T* ws_ptr(const void* ws, int64_t off) {
    return reinterpret_cast<const T*>(reinterpret_cast<const char*>(ws) + off);
}

// Record the first device-detected error of a launch sequence.
__device__ __forceinline__ void set_status(PlanHeader* h, int32_t code, int32_t info) {
    if (atomicCAS(&h->status, 0, code) == 0) h->status_info = info;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two e4m3 bytes (low byte first) -> two floats, exact (every e4m3 value is an fp16 value).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
    __half2 h = *reinterpret_cast<__half2*>(&h2);
    return __half22float2(h);
}

}  // namespace mla
