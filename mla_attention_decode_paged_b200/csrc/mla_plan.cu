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
template <typename T>
__device__ void block_exclusive_scan(T* a, int n, T* partial) {
    static_assert(kPlanThreads == 256, "two-level warp scan below assumes 8 warps");
    const int per = (n + kPlanThreads - 1) / kPlanThreads;
    const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    T run = 0;
    for (int i = lo; i < hi; ++i) run += a[i];
    // inclusive scan of the chunk totals within the warp
    T v = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const T u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) partial[warp] = v;
    __syncthreads();
    if (warp == 0) {
        T w = lane < 8 ? partial[lane] : 0;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
            const T u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        if (lane < 8) partial[8 + lane] = w;  // inclusive totals of warps 0..lane
    }
    __syncthreads();
    T acc = (v - run) + (warp > 0 ? partial[8 + warp - 1] : 0);  // exclusive offset of this chunk
    if (threadIdx.x == kPlanThreads - 1) a[n] = partial[15];
    for (int i = lo; i < hi; ++i) {
        const T x = a[i];
        a[i] = acc;
        acc += x;
    }
    __syncthreads();
}

// first index i in [0, n) with a[i] >= x (a non-decreasing), n if none
__device__ __forceinline__ int lower_bound64(const int64_t* a, int n, int64_t x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] < x) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// One CTA, everything in shared memory and in parallel:
//   pre[b]   pages before request b (exclusive scan of ceil(T_b / 64));
//   cuts[g]  share boundaries floor(total * g / G);
//   a cut that falls strictly inside a request, and is the first of its value, starts a new
//   segment ("flagged"); every request with pages starts one;
//   a request's segments are its start plus its flagged cuts; a group's first segment is
//   the number of segment starts below its boundary.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ seq_lens, int B, int s_q,
                                                            int H, WsLayout L, void* ws) {
    const int G = L.num_groups;
    extern __shared__ int64_t plan_sh[];
    int64_t* pre = plan_sh;                                          // [B + 1]
    int64_t* cuts = pre + (B + 1);                                   // [G + 1]
    int64_t* part64 = cuts + (G + 1);                                // [kPlanThreads]
    int32_t* nseg = reinterpret_cast<int32_t*>(part64 + kPlanThreads);  // [B + 1] -> segment base
    int32_t* vcnt = nseg + (B + 1);                                  // [B + 1] valid requests before b
    int32_t* flag = vcnt + (B + 1);                                  // [G + 2] -> flagged cuts before g
    int32_t* part32 = flag + (G + 2);                                // [kPlanThreads]
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
        pre[b] = T > 0 ? (T + kPage - 1) / kPage : 0;
        vcnt[b] = T > 0 ? 1 : 0;
        if (T <= 0) atomicMin(&bad_first, b);
    }
    __syncthreads();
    block_exclusive_scan(pre, B, part64);
    block_exclusive_scan(vcnt, B, part32);
    const int64_t total = pre[B];
    for (int g = tid; g <= G; g += kPlanThreads) cuts[g] = total * (int64_t)g / G;
    __syncthreads();
    for (int g = tid; g <= G; g += kPlanThreads) {
        int f = 0;
        const int64_t cg = cuts[g];
        if (g > 0 && g < G && cg > 0 && cg < total && cg != cuts[g - 1]) {
            // a request start? the last request whose start is <= cg starts exactly at cg and
            // has pages
            const int bl = lower_bound64(pre, B + 1, cg + 1) - 1;
            const bool is_start = bl < B && pre[bl] == cg && pre[bl + 1] > cg;
            f = is_start ? 0 : 1;
        }
        flag[g] = f;
    }
    __syncthreads();
    block_exclusive_scan(flag, G + 1, part32);  // flag[g] = flagged cuts with index < g
    for (int b = tid; b < B; b += kPlanThreads) {
        const int64_t p0 = pre[b], p1 = pre[b + 1];
        int n = 0;
        if (p1 > p0) {
            const int gl = lower_bound64(cuts, G + 1, p0 + 1);  // first cut > p0
            const int gh = lower_bound64(cuts, G + 1, p1);      // first cut >= p1
            n = 1 + (gh > gl ? flag[gh] - flag[gl] : 0);
        }
        nseg[b] = n;
    }
    __syncthreads();
    block_exclusive_scan(nseg, B, part32);  // nseg[b] = first segment of request b
    const int nseg_total = nseg[B];
    for (int b = tid; b < B; b += kPlanThreads) {
        req_seg[b] = nseg[b];
        const int64_t p0 = pre[b], p1 = pre[b + 1];
        if (p1 <= p0) continue;
        const int n = nseg[b + 1] - nseg[b];
        const int gl = lower_bound64(cuts, G + 1, p0 + 1);
        const int gh = lower_bound64(cuts, G + 1, p1);
        int k = nseg[b];
        int64_t start = p0;
        for (int g = gl; g < gh; ++g) {
            if (flag[g + 1] == flag[g]) continue;  // not a flagged cut
            Segment sg;
            sg.b = b;
            sg.tile_begin = (int32_t)(start - p0);
            sg.tile_end = (int32_t)(cuts[g] - p0);
            sg.split = n > 1;
            segs[k++] = sg;
            start = cuts[g];
        }
        Segment sg;
        sg.b = b;
        sg.tile_begin = (int32_t)(start - p0);
        sg.tile_end = (int32_t)(p1 - p0);
        sg.split = n > 1;
        segs[k] = sg;
    }
    for (int g = tid; g <= G; g += kPlanThreads) {
        int v;
        if (g == 0) {
            v = 0;
        } else if (g == G) {
            v = nseg_total;
        } else {
            // segment starts below cuts[g]: request starts below it plus flagged cuts below it
            const int64_t x = cuts[g];
            const int bx = lower_bound64(pre, B, x);           // requests 0..bx-1 start below x
            const int gf = lower_bound64(cuts, G + 1, x);      // first cut of this value
            v = vcnt[bx] + flag[gf];
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
    if (L.num_groups > kMaxGroups) return 0;
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
    const size_t smem = sizeof(int64_t) * ((size_t)B + 1 + (size_t)L.num_groups + 1 + kPlanThreads) +
                        sizeof(int32_t) * (2 * ((size_t)B + 1) + (size_t)L.num_groups + 2 + kPlanThreads);
    if (smem > 200 * 1024) return MLA_ERR_UNSUPPORTED;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MLA_ERR_CUDA;
    plan_kernel<<<1, kPlanThreads, smem, (cudaStream_t)stream>>>(seq_lens, B, s_q, H, L, workspace);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
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
