// mla_plan.cu -- split-KV planner: workspace sizing and the device-side plan kernel.
//
// Split-KV ("flash-decoding") scans each request's cache in contiguous pieces whose
// partial results are merged afterwards ["Faster kernels, slower engine", 7.1 Gluon MLA
// decode: split scan plus a reduction pass].  The plan here balances the whole batch:
// the pages of all requests, laid end to end in request order, are cut into
// num_groups equal contiguous shares.  A share that ends inside a request splits it;
// a request that one share holds whole is written out directly, with no partials.
// Every group holds one SM pair per 128-row block of the folded query (s_q * H rows),
// and all pairs of a group scan the same pages, so a page read from HBM by one pair
// is found in L2 by the others.
#include <math.h>

#include "mla_decode_params.cuh"

namespace mla {

__global__ void plan_kernel(const int32_t* __restrict__ seq_lens, int B, int s_q, int H,
                            WsLayout L, void* ws) {
    if (threadIdx.x != 0) return;
    PlanHeader* h = reinterpret_cast<PlanHeader*>(ws);
    int32_t* group_begin = ws_ptr<int32_t>(ws, L.off_group_begin);
    int32_t* req_seg = ws_ptr<int32_t>(ws, L.off_req_seg);
    Segment* segs = ws_ptr<Segment>(ws, L.off_segs);
    const int G = L.num_groups;

    int64_t total = 0;
    int bad = -1;
    for (int b = 0; b < B; ++b) {
        int T = seq_lens[b];
        if (T <= 0) { if (bad < 0) bad = b; continue; }
        total += (T + kPage - 1) / kPage;
    }
    // cut(g) = floor(total * g / G): share g is pages [cut(g), cut(g+1)) of the batch
    auto cut = [&](int g) -> int64_t { return total * (int64_t)g / G; };

    int seg = 0, g = 0;
    int64_t prefix = 0;
    group_begin[0] = 0;
    for (int b = 0; b < B; ++b) {
        req_seg[b] = seg;
        int T = seq_lens[b];
        int64_t tiles = T > 0 ? (T + kPage - 1) / kPage : 0;
        int64_t pos = prefix, end = prefix + tiles;
        while (pos < end) {
            while (g < G && cut(g + 1) <= pos) { ++g; group_begin[g] = seg; }
            int64_t e = cut(g + 1) < end ? cut(g + 1) : end;
            Segment s;
            s.b = b;
            s.tile_begin = (int32_t)(pos - prefix);
            s.tile_end = (int32_t)(e - prefix);
            s.split = 0;
            segs[seg++] = s;
            pos = e;
        }
        if (seg - req_seg[b] > 1)
            for (int k = req_seg[b]; k < seg; ++k) segs[k].split = 1;
        prefix = end;
    }
    req_seg[B] = seg;
    while (g < G) { ++g; group_begin[g] = seg; }

    h->status = bad >= 0 ? kStatusOob : kStatusOk;
    h->status_info = bad >= 0 ? bad : 0;
    h->B = B;
    h->s_q = s_q;
    h->H = H;
    h->nqb = L.nqb;
    h->num_groups = G;
    h->num_segments = seg;
    h->max_segments = L.max_segments;
    h->total_tiles = (int32_t)total;
    h->off_group_begin = L.off_group_begin;
    h->off_req_seg = L.off_req_seg;
    h->off_segs = L.off_segs;
    h->off_plse = L.off_plse;
    h->off_po = L.off_po;
    h->total_bytes = L.total;
    __threadfence();
    h->magic = kPlanMagic;
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
}

// SMs the default plan is made for: twice the number of CTA pairs of the scan kernel that
// the device keeps resident at once (a pair must sit in one GPC, so this can be below the
// SM count).
int effective_sms() {
    int pairs = sm100_pair_slots();
    if (pairs > 0) return 2 * pairs;
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
    if (num_sms < 2) return MLA_ERR_INVALID_ARG;
    WsLayout L = make_layout(B, s_q, H, num_groups_for(num_sms, num_row_blocks(s_q, H)));
    if ((int64_t)ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
    plan_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(seq_lens, B, s_q, H, L, workspace);
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
