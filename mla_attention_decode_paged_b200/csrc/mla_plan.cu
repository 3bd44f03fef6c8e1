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
constexpr int kPlanWarps = kPlanThreads / 32;
static_assert(kPlanWarps == 8, "plan_shared_bytes reserves 8 words of scan scratch");

// Thread t's contiguous share [x, y) of n items: the loads, the flag tests and the scans
// below give every thread the same share, so a thread scans only what it wrote itself
// and no barrier is needed between writing an array and scanning it.
__device__ __forceinline__ int2 chunk_of(int n) {
    const int per = (n + kPlanThreads - 1) / kPlanThreads;
    const int lo = min(n, (int)threadIdx.x * per);
    return make_int2(lo, min(n, lo + per));
}

// In-place exclusive prefix sum of a[0..n) by the whole block; a[n] receives the total.
// Each thread scans its own chunk; chunk totals are scanned with warp shuffles and the
// warp totals are added by every thread from shared memory.  Two barriers, the second
// ends the call.
__device__ __forceinline__ void block_exclusive_scan(int64_t* a, int n, int64_t* wsum) {
    const int2 c = chunk_of(n);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t run = 0;
    for (int i = c.x; i < c.y; ++i) run += a[i];
    int64_t v = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    int64_t acc = v - run;  // exclusive offset of this chunk
    for (int w = 0; w < warp; ++w) acc += wsum[w];
    if (threadIdx.x == kPlanThreads - 1) a[n] = acc + run;
    for (int i = c.x; i < c.y; ++i) {
        const int64_t x = a[i];
        a[i] = acc;
        acc += x;
    }
    __syncthreads();
}

// last request index b in [0, B] whose first page is <= x (pk: pages before b in the
// high word, non-decreasing); x >= 0
__device__ __forceinline__ int last_start_le(const int64_t* pk, int B, int64_t x) {
    const int64_t key = (x + 1) << 32;
    int lo = 0, hi = B + 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pk[mid] < key) lo = mid + 1; else hi = mid;
    }
    return lo - 1;
}

// One CTA, everything in shared memory:
//   pk[b]    (pages before request b) << 32 | (requests with pages before b): one scan of
//            (ceil(T_b / 64) << 32 | [T_b > 0]); the low field never carries into the high one;
//   cut[g]   share boundary floor(total * g / G);
//   a cut that falls strictly inside a request, and is the first of its value, starts a new
//   segment ("flagged"); every request with pages starts one.  Segments are numbered in
//   page order, so a segment's index is the number of segment starts below it: requests
//   with pages that start below it plus flagged cuts below it.  Each start is recorded at
//   its index; a segment ends where the next one of its request starts, or at the
//   request's end.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ seq_lens, int B, int s_q,
                                                            int H, WsLayout L, void* ws) {
    const int G = L.num_groups;
    extern __shared__ int64_t plan_sh[];
    int64_t* pk = plan_sh;                                        // [B + 1]
    int64_t* cut = pk + (B + 1);                                  // [G + 1]
    int64_t* fsum = cut + (G + 1);                                // [G + 2] flags, then flagged cuts below g
    int64_t* wsum = fsum + (G + 2);                               // [kPlanWarps] scan scratch
    int32_t* inside = reinterpret_cast<int32_t*>(wsum + kPlanWarps);  // [G + 1] request a flagged cut cuts
    int32_t* rec_b = inside + (G + 1);                            // [B + G] segment starts: request
    int32_t* rec_t = rec_b + (B + G);                             // [B + G] segment starts: first page in it
    int32_t* gb_s = rec_t + (B + G);                              // [G + 1] first segment of each group
    __shared__ int bad_first;
    PlanHeader* h = reinterpret_cast<PlanHeader*>(ws);
    int32_t* group_begin = ws_ptr<int32_t>(ws, L.off_group_begin);
    GroupHead* heads = ws_ptr<GroupHead>(ws, L.off_heads);
    int32_t* req_seg = ws_ptr<int32_t>(ws, L.off_req_seg);
    Segment* segs = ws_ptr<Segment>(ws, L.off_segs);
    const int tid = threadIdx.x;
    // the scan kernel (a programmatic dependent) may start its prologue; it waits for this
    // grid to complete before reading the plan
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (tid == 0) bad_first = -1;
    {
        const int2 c = chunk_of(B);
        for (int b = c.x; b < c.y; ++b) {
            const int64_t T = seq_lens[b];
            pk[b] = T > 0 ? ((T + kPage - 1) / kPage) << 32 | 1 : 0;
        }
    }
    block_exclusive_scan(pk, B, wsum);
    const int64_t total = pk[B] >> 32;
    const int nvalid = (int)(pk[B] & 0xffffffff);
    {
        const int2 c = chunk_of(G + 1);
        for (int g = c.x; g < c.y; ++g) {
            const int64_t cg = total * g / G;
            int64_t f = 0;
            int in = -1;
            if (g > 0 && g < G && cg > 0 && cg < total && cg != total * (g - 1) / G) {
                // the last request starting at or below cg starts exactly there (and has
                // pages), or cg falls strictly inside it
                const int bl = last_start_le(pk, B, cg);
                if ((pk[bl] >> 32) != cg) {
                    f = 1;
                    in = bl;
                }
            }
            cut[g] = cg;
            fsum[g] = f;
            inside[g] = in;
        }
    }
    block_exclusive_scan(fsum, G + 1, wsum);  // fsum[g] = flagged cuts with index < g
    const int nseg_total = nvalid + (int)fsum[G + 1];
    // first g in [0, G] with cut[g] >= x, i.e. ceil(x * G / total); G + 1 if none.  A float
    // estimate, corrected against the exact cuts.
    auto first_cut_ge = [&](int64_t x) -> int {
        if (x <= 0) return 0;
        if (x > total) return G + 1;
        int g = (int)ceilf((float)x * (float)G / (float)total);
        g = min(max(g, 0), G);
        while (g > 0 && cut[g - 1] >= x) --g;
        while (g < G && cut[g] < x) ++g;
        return g;
    };
    for (int b = tid; b < B; b += kPlanThreads) {
        const int64_t p0 = pk[b] >> 32, p1 = pk[b + 1] >> 32;
        const int before = (int)(pk[b] & 0xffffffff);
        const int first = before + (int)fsum[first_cut_ge(p0)];
        req_seg[b] = first;
        if (p1 > p0) {
            rec_b[first] = b;
            rec_t[first] = 0;
        } else if (before == b) {
            bad_first = b;  // the first request without tokens: every one before it has some
        }
    }
    for (int g = tid + 1; g < G; g += kPlanThreads) {
        const int b = inside[g];
        if (b < 0) continue;
        const int idx = (int)(pk[b] & 0xffffffff) + 1 + (int)fsum[g];
        rec_b[idx] = b;
        rec_t[idx] = (int32_t)(cut[g] - (pk[b] >> 32));
    }
    for (int g = tid; g <= G; g += kPlanThreads) {
        int v;
        if (g == 0) {
            v = 0;
        } else if (g == G) {
            v = nseg_total;
        } else {
            // segment starts below cut(g): requests with pages starting below it plus
            // flagged cuts below it
            const int64_t x = cut[g];
            const int bl = last_start_le(pk, B, x);
            const int below = (int)(((pk[bl] >> 32) == x ? pk[bl] : pk[bl + 1]) & 0xffffffff);
            v = below + (int)fsum[first_cut_ge(x)];
        }
        group_begin[g] = v;
        gb_s[g] = v;
    }
    __syncthreads();
    auto segment_at = [&](int i) -> Segment {
        const int b = rec_b[i];
        const bool last = i + 1 == nseg_total || rec_b[i + 1] != b;
        Segment sg;
        sg.b = b;
        sg.tile_begin = rec_t[i];
        sg.tile_end = last ? (int32_t)((pk[b + 1] >> 32) - (pk[b] >> 32)) : rec_t[i + 1];
        sg.split = !(last && rec_t[i] == 0);
        return sg;
    };
    for (int i = tid; i < nseg_total; i += kPlanThreads) segs[i] = segment_at(i);
    for (int g = tid; g < G; g += kPlanThreads) {
        GroupHead gh;
        gh.seg_lo = gb_s[g];
        gh.seg_hi = gb_s[g + 1];
        gh.pad0 = gh.pad1 = 0;
        if (gh.seg_lo < gh.seg_hi) {
            gh.first = segment_at(gh.seg_lo);
        } else {
            gh.first.b = gh.first.tile_begin = gh.first.tile_end = gh.first.split = 0;
        }
        heads[g] = gh;
    }
    if (tid == 0) {
        req_seg[B] = nseg_total;
        const int bad = bad_first;
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
        // every reader of the plan starts after this grid has completed (stream order, or
        // a programmatic dependent's grid-dependency wait): no fence orders the magic last
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
