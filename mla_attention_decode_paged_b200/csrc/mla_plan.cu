// mla_plan.cu -- split-KV planner: workspace sizing and the device-side plan kernel.
//
// Split-KV ("flash-decoding") scans each request's cache in contiguous pieces whose
// partial results are merged afterwards ["Faster kernels, slower engine", 7.1 Gluon MLA
// decode: split scan plus a reduction pass].  The plan here balances the whole batch:
// the pages of all requests, laid end to end in request order, are cut into
// num_groups equal contiguous shares.  A share that ends inside a request splits it;
// a request that one share holds whole is written out directly, with no partials.
// Every group holds one CTA per 64-row block of the folded query (s_q * H rows), and
// all CTAs of a group scan the same pages, so a page read from HBM by one CTA is found
// in L2 by the others.
#include <math.h>

#include "mla_decode_params.cuh"

namespace mla {

constexpr int kPlanThreads = 256;

// In-place exclusive prefix sum of a[0..n) by the whole block (n + 1 entries are written:
// a[n] receives the total).  Each thread scans a contiguous chunk; the chunk totals are
// scanned with warp shuffles (one warp per 32 chunks, then one warp over the 8 warp sums).
// The caller synchronises the block before the call; the call ends with a barrier.  Not
// inlined: the plan runs once per launch on a cold SM, so one shared copy of the code
// costs fewer instruction fetches than three inlined ones.
__device__ __noinline__ void block_exclusive_scan(int64_t* a, int n, int64_t* partial) {
    static_assert(kPlanThreads == 256, "two-level warp scan below assumes 8 warps");
    const int per = (n + kPlanThreads - 1) / kPlanThreads;
    const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t run = 0;
    for (int i = lo; i < hi; ++i) run += a[i];
    // inclusive scan of the chunk totals within the warp
    int64_t v = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) partial[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int64_t w = lane < 8 ? partial[lane] : 0;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            const int64_t u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        if (lane < 8) partial[8 + lane] = w;  // inclusive totals of warps 0..lane
    }
    __syncthreads();
    int64_t acc = (v - run) + (warp > 0 ? partial[8 + warp - 1] : 0);  // exclusive offset of this chunk
    if (threadIdx.x == kPlanThreads - 1) a[n] = partial[15];
    for (int i = lo; i < hi; ++i) {
        const int64_t x = a[i];
        a[i] = acc;
        acc += x;
    }
    __syncthreads();
}

// first index i in [0, n) with a[i] >= x (a non-decreasing), n if none
__device__ __noinline__ int lower_bound64(const int64_t* a, int n, int64_t x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] < x) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// One CTA, everything in shared memory and in parallel:
//   pk[b]    (pages before request b) << 32 | (requests with tokens before b): one scan of
//            (ceil(T_b / 64) << 32 | [T_b > 0]); the low field never carries into the high one;
//   cut(g)   share boundary floor(total * g / G), and the first g whose cut is >= x in
//            closed form, ceil(x * G / total);
//   a cut that falls strictly inside a request, and is the first of its value, starts a new
//   segment ("flagged"); every request with pages starts one;
//   a request's segments are its start plus its flagged cuts; a group's first segment is
//   the number of segment starts below its boundary.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ seq_lens, int B, int s_q,
                                                            int H, WsLayout L, void* ws) {
    const int G = L.num_groups;
    extern __shared__ int64_t plan_sh[];
    int64_t* pk = plan_sh;             // [B + 1]
    int64_t* flag = pk + (B + 1);      // [G + 2] -> flagged cuts before g
    int64_t* nseg = flag + (G + 2);    // [B + 1] -> first segment of request b
    int64_t* part = nseg + (B + 1);    // [16] scan scratch
    __shared__ int bad_first;
    PlanHeader* h = reinterpret_cast<PlanHeader*>(ws);
    int32_t* group_begin = ws_ptr<int32_t>(ws, L.off_group_begin);
    int32_t* req_seg = ws_ptr<int32_t>(ws, L.off_req_seg);
    Segment* segs = ws_ptr<Segment>(ws, L.off_segs);
    const int tid = threadIdx.x;
    // the scan kernel (a programmatic dependent) may start its prologue; it waits for this
    // grid to complete before reading the plan
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (tid == 0) bad_first = B;
    __syncthreads();
    for (int b = tid; b < B; b += kPlanThreads) {
        const int T = seq_lens[b];
        pk[b] = T > 0 ? ((int64_t)((T + kPage - 1) / kPage) << 32) | 1 : 0;
        if (T <= 0) atomicMin(&bad_first, b);
    }
    __syncthreads();
    block_exclusive_scan(pk, B, part);
    const int64_t total = pk[B] >> 32;
    // first g in [0, G] with cut(g) >= x; G + 1 if none
    auto first_cut_ge = [&](int64_t x) -> int {
        if (x <= 0) return 0;
        if (x > total) return G + 1;
        return (int)((x * G + total - 1) / total);
    };
    for (int g = tid; g <= G; g += kPlanThreads) {
        int64_t f = 0;
        if (g > 0 && g < G) {
            const int64_t cg = total * g / G;
            if (cg > 0 && cg < total && cg != total * (g - 1) / G) {
                // a request start? the last request whose start is <= cg starts exactly at cg
                // and has pages
                const int bl = lower_bound64(pk, B + 1, (cg + 1) << 32) - 1;
                const bool is_start = bl < B && (pk[bl] >> 32) == cg && (pk[bl + 1] >> 32) > cg;
                f = is_start ? 0 : 1;
            }
        }
        flag[g] = f;
    }
    __syncthreads();
    block_exclusive_scan(flag, G + 1, part);  // flag[g] = flagged cuts with index < g
    for (int b = tid; b < B; b += kPlanThreads) {
        const int64_t p0 = pk[b] >> 32, p1 = pk[b + 1] >> 32;
        int64_t n = 0;
        if (p1 > p0) {
            const int gl = first_cut_ge(p0 + 1), gh = first_cut_ge(p1);
            n = 1 + (gh > gl ? flag[gh] - flag[gl] : 0);
        }
        nseg[b] = n;
    }
    __syncthreads();
    block_exclusive_scan(nseg, B, part);  // nseg[b] = first segment of request b
    const int nseg_total = (int)nseg[B];
    // segments, in parallel: every request with pages starts its first segment at tile 0,
    // every flagged cut starts the next segment of the request it falls in; a segment ends
    // at the next flagged cut inside its request (found by a search of the scanned flags:
    // cut g is flagged iff flag[g + 1] > flag[g]) or at the request's end
    for (int b = tid; b < B; b += kPlanThreads) {
        req_seg[b] = (int)nseg[b];
        const int64_t p0 = pk[b] >> 32, p1 = pk[b + 1] >> 32;
        if (p1 <= p0) continue;
        const int gl = first_cut_ge(p0 + 1), gh = first_cut_ge(p1);
        const int g1 = lower_bound64(flag, G + 2, flag[gl] + 1) - 1;  // first flagged cut >= gl
        Segment sg;
        sg.b = b;
        sg.tile_begin = 0;
        sg.tile_end = (int32_t)((g1 < gh ? total * g1 / G : p1) - p0);
        sg.split = nseg[b + 1] - nseg[b] > 1;
        segs[nseg[b]] = sg;
    }
    for (int g = tid + 1; g < G; g += kPlanThreads) {
        if (flag[g + 1] == flag[g]) continue;  // not a flagged cut
        const int64_t cg = total * g / G;
        const int b = lower_bound64(pk, B + 1, (cg + 1) << 32) - 1;  // the request cg falls strictly inside
        const int64_t p0 = pk[b] >> 32, p1 = pk[b + 1] >> 32;
        const int gh = first_cut_ge(p1);
        const int g2 = lower_bound64(flag, G + 2, flag[g + 1] + 1) - 1;  // next flagged cut after g
        Segment sg;
        sg.b = b;
        sg.tile_begin = (int32_t)(cg - p0);
        sg.tile_end = (int32_t)((g2 < gh ? total * g2 / G : p1) - p0);
        sg.split = 1;
        segs[nseg[b] + 1 + (flag[g] - flag[first_cut_ge(p0 + 1)])] = sg;
    }
    for (int g = tid; g <= G; g += kPlanThreads) {
        int v;
        if (g == 0) {
            v = 0;
        } else if (g == G) {
            v = nseg_total;
        } else {
            // segment starts below cut(g): request starts below it plus flagged cuts below it
            const int64_t x = total * g / G;
            const int bx = lower_bound64(pk, B, x << 32);  // requests 0..bx-1 start below x
            v = (int)(pk[bx] & 0xffffffff) + (int)flag[first_cut_ge(x)];
        }
        group_begin[g] = v;
    }
    if (tid == 0) {
        req_seg[B] = nseg_total;
        const int bad = bad_first < B ? bad_first : -1;
        h->status = bad >= 0 ? kStatusOob : kStatusOk;
        h->status_info = bad >= 0 ? bad : 0;
        h->B = B;
        h->s_q = s_q;
        h->H = H;
        h->nqb = L.nqb;
        h->num_groups = G;
        h->num_segments = nseg_total;
        h->max_segments = L.max_segments;
        h->total_tiles = (int32_t)total;
        h->off_group_begin = L.off_group_begin;
        h->off_req_seg = L.off_req_seg;
        h->off_segs = L.off_segs;
        h->off_plse = L.off_plse;
        h->off_po = L.off_po;
        h->total_bytes = L.total;
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        h->magic = kPlanMagic;
    }
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
}

// SMs the default plan is made for: the number of scan CTAs the device keeps resident
// at once (one per SM).
int effective_sms() {
    int n = sm100_cta_slots();
    if (n > 0) return n;
    return device_sm_count();
}

bool shape_ok(int B, int s_q, int H) {
    return B > 0 && s_q > 0 && H > 0 && (int64_t)s_q * H <= 65536;
}

}  // namespace mla

using namespace mla;

extern "C" size_t mla_decode_workspace_size(int B, int s_q, int H, int num_sms) {
    if (!shape_ok(B, s_q, H) || num_sms < 0) return 0;
    if (num_sms == 0) {
        num_sms = effective_sms();
        if (num_sms <= 0) return 0;
    }
    WsLayout L = make_layout(B, s_q, H, num_groups_for(num_sms, num_row_blocks(s_q, H)));
    if (L.num_groups > kMaxGroups || plan_shared_bytes(B, L.num_groups) > kPlanMaxSharedBytes) return 0;
    return (size_t)L.total;
}

extern "C" mla_status mla_decode_plan(const int32_t* seq_lens, int B, int s_q, int H, int num_sms,
                                      void* workspace, size_t ws_bytes, void* stream) {
    if (!seq_lens || !workspace || !shape_ok(B, s_q, H) || num_sms < 0) return MLA_ERR_INVALID_ARG;
    if (((uintptr_t)workspace & 255) != 0) return MLA_ERR_INVALID_ARG;
    if (num_sms == 0) {
        num_sms = effective_sms();
        if (num_sms <= 0) return MLA_ERR_CUDA;
    }
    if (num_sms < 1) return MLA_ERR_INVALID_ARG;
    WsLayout L = make_layout(B, s_q, H, num_groups_for(num_sms, num_row_blocks(s_q, H)));
    if (L.num_groups > kMaxGroups) return MLA_ERR_UNSUPPORTED;
    if ((int64_t)ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    const size_t smem = plan_shared_bytes(B, L.num_groups);
    if (smem > kPlanMaxSharedBytes) return MLA_ERR_UNSUPPORTED;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    plan_kernel<<<1, kPlanThreads, smem, (cudaStream_t)stream>>>(seq_lens, B, s_q, H, L, workspace);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

extern "C" mla_status mla_debug_wait_timeout(void* workspace, size_t ws_bytes, void* stream) {
    if (!workspace || ((uintptr_t)workspace & 255) != 0) return MLA_ERR_INVALID_ARG;
    if (ws_bytes < sizeof(PlanHeader)) return MLA_ERR_WORKSPACE_TOO_SMALL;
    return launch_wait_timeout_probe(workspace, (cudaStream_t)stream);
}

extern "C" mla_status mla_get_device_status(void* workspace, int* code, void* stream) {
    if (!workspace || !code) return MLA_ERR_INVALID_ARG;
    int32_t h[2] = {0, 0};
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(h), s) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
    *code = h[0];
    return MLA_OK;
}

extern "C" const char* mla_decode_version(void) { return "mla_decode 0.1 (sm_100a)"; }
