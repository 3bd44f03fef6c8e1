// mla_prefill.cu -- long-prefix MLA prefill: a chunk of C new query tokens per request
// attends causally to the request's paged latent cache, whose last C rows are the chunk's
// own (prefill over a cache that already holds a long prefix is one of the two MLA
// workloads of the "TokenSpeed" launch digest (cvshuo.com), MLA kernel paragraphs).
// Token i of the chunk of request b sits at position T_b - C + i and sees cached tokens
// t <= T_b - C + i.
//
// That is the decode's causal rule with s_q = C, so the prefill runs on the decode path.
// The chunk is cut into n = C / d sub-chunks of d tokens, d * H <= 256 rows each; each
// sub-chunk is a request of the decode: sub-chunk j of request b becomes request
// b' = b * n + j with
//     seq_len'[b'] = T_b - C + (j + 1) * d,   block_table'[b'] = block_table[b],
// so its draft k (chunk token i = j d + k) sees t <= seq_len' - d + k = T_b - C + i,
// the chunk's own causal rule.  q [B, C, H, 576], out [B, C, H, 512] and lse [B, C, H]
// are, unchanged, the decode's [B n, d, H, .] arrays.  One small kernel writes seq_len'
// and block_table' into the workspace; the planner, the split scan and the combine then
// run as for a decode of B n requests: all sub-chunks of a request read the same pages,
// which after the first read come from L2 while they fit in it.
#include <limits.h>
#include <math.h>

#include <algorithm>

#include "mla_decode_params.cuh"

namespace mla {
namespace {

constexpr int kExpandThreads = 256;

// seq_len' and block_table' of the B n sub-chunk requests.  A request whose length
// cannot hold its chunk (T_b < C) or exceeds its block table (T_b > max_pages * 64)
// gives all of its sub-chunks length 0: the planner then records MLA_ERR_DEVICE_OOB
// and the combine writes their rows as NaN.
__global__ void __launch_bounds__(kExpandThreads) prefill_expand_kernel(
    const int32_t* __restrict__ seq_lens, const int32_t* __restrict__ block_table, int B, int n, int d, int chunk,
    int max_pages, int32_t* __restrict__ lens_x, int32_t* __restrict__ bt_x) {
    const int64_t stride = (int64_t)gridDim.x * kExpandThreads;
    const int64_t first = (int64_t)blockIdx.x * kExpandThreads + threadIdx.x;
    const int64_t rows = (int64_t)B * n;
    for (int64_t r = first; r < rows; r += stride) {
        const int b = (int)(r / n), j = (int)(r % n);
        const int T = seq_lens[b];
        const bool ok = T >= chunk && T <= (int64_t)max_pages * kPage;
        lens_x[r] = ok ? T - chunk + (j + 1) * d : 0;
    }
    const int64_t total = rows * max_pages;
    for (int64_t e = first; e < total; e += stride) {
        const int64_t r = e / max_pages;
        const int p = (int)(e % max_pages);
        bt_x[e] = block_table[(r / n) * max_pages + p];
    }
}

struct PrefillLayout {
    int d, n, Bx;
    int64_t decode_bytes, off_lens, off_bt, total;
};

// Sub-chunk size and workspace layout; false for an unsupported shape.  The decode's
// workspace comes first (its status header at offset 0, so mla_get_device_status reads a
// prefill workspace as it reads a decode one), then seq_len' and block_table'.
bool prefill_layout(int B, int chunk, int H, int max_pages, int num_sms, PrefillLayout* L) {
    const int d = mla_prefill_sub_chunk(chunk, H);
    if (d <= 0 || B <= 0 || max_pages <= 0 || num_sms <= 0) return false;
    const int n = chunk / d;
    if ((int64_t)B * n > INT_MAX) return false;
    const int Bx = B * n;
    const int G = num_groups_for(num_sms, num_row_blocks(d, H));
    if (G > kMaxGroups || plan_shared_bytes(Bx, G) > kPlanMaxSharedBytes) return false;
    L->d = d;
    L->n = n;
    L->Bx = Bx;
    L->decode_bytes = make_layout(Bx, d, H, G).total;
    L->off_lens = L->decode_bytes;
    L->off_bt = align_up(L->off_lens + 4 * (int64_t)Bx, 256);
    L->total = align_up(L->off_bt + 4 * (int64_t)Bx * max_pages, 256);
    return true;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" int mla_prefill_sub_chunk(int chunk, int H) {
    if (chunk <= 0 || H <= 0 || H > kMaxRows) return 0;
    // the divisor d of the chunk (d * H <= 256 rows) with the fewest 64-row blocks to scan
    // per cached page, (chunk / d) * ceil(d H / 64); ties go to the larger d (fewer
    // requests for the planner and fewer partials for the combine)
    int best = 0;
    int64_t best_cost = 0;
    for (int d = 1; d <= chunk && (int64_t)d * H <= kMaxRows; ++d) {
        if (chunk % d != 0) continue;
        const int64_t cost = (int64_t)(chunk / d) * num_row_blocks(d, H);
        if (best == 0 || cost <= best_cost) {
            best = d;
            best_cost = cost;
        }
    }
    return best;
}

extern "C" size_t mla_prefill_workspace_size(int B, int chunk, int H, int max_pages_per_req, int num_sms) {
    if (num_sms < 0) return 0;
    if (num_sms == 0) {
        num_sms = effective_sms();
        if (num_sms <= 0) return 0;
    }
    PrefillLayout L;
    if (!prefill_layout(B, chunk, H, max_pages_per_req, num_sms, &L)) return 0;
    return (size_t)L.total;
}

extern "C" mla_status mla_prefill(const void* q, const void* kv_pages, int kv_dtype, float kv_scale,
                                  const int32_t* block_table, int max_pages_per_req, const int32_t* seq_lens,
                                  int B, int chunk, int H, int64_t num_pages, float scale, void* workspace,
                                  size_t ws_bytes, void* out, float* lse, void* stream) {
    if (!q || !kv_pages || !block_table || !seq_lens || !workspace || !out || !lse) return MLA_ERR_INVALID_ARG;
    if (B <= 0 || chunk <= 0 || H <= 0 || max_pages_per_req <= 0 || num_pages <= 0) return MLA_ERR_INVALID_ARG;
    if (!isfinite(scale)) return MLA_ERR_INVALID_ARG;
    if (kv_dtype != MLA_KV_BF16 && kv_dtype != MLA_KV_E4M3) return MLA_ERR_UNSUPPORTED;
    if (kv_dtype == MLA_KV_E4M3 && !(isfinite(kv_scale) && kv_scale > 0.f)) return MLA_ERR_INVALID_ARG;
    if (H > kMaxRows) return MLA_ERR_UNSUPPORTED;
    if ((((uintptr_t)q) & 15) || (((uintptr_t)kv_pages) & 15) || (((uintptr_t)out) & 15) ||
        (((uintptr_t)workspace) & 255) || (((uintptr_t)lse) & 3) || (((uintptr_t)block_table) & 3) ||
        (((uintptr_t)seq_lens) & 3))
        return MLA_ERR_INVALID_ARG;
    const int sms = effective_sms();
    if (sms <= 0) return MLA_ERR_CUDA;
    PrefillLayout L;
    if (!prefill_layout(B, chunk, H, max_pages_per_req, sms, &L)) return MLA_ERR_UNSUPPORTED;
    if ((int64_t)ws_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t st = (cudaStream_t)stream;
    int32_t* lens_x = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(workspace) + L.off_lens);
    int32_t* bt_x = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(workspace) + L.off_bt);
    const int64_t elems = (int64_t)L.Bx * max_pages_per_req;
    const int blocks = (int)std::min<int64_t>((elems + kExpandThreads - 1) / kExpandThreads, 8LL * sms);
    prefill_expand_kernel<<<blocks, kExpandThreads, 0, st>>>(seq_lens, block_table, B, L.n, L.d, chunk,
                                                              max_pages_per_req, lens_x, bt_x);
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;
    mla_status s = mla_decode_plan(lens_x, L.Bx, L.d, H, sms, workspace, (size_t)L.decode_bytes, stream);
    if (s != MLA_OK) return s;
    return mla_decode(q, kv_pages, kv_dtype, kv_scale, bt_x, max_pages_per_req, lens_x, L.Bx, L.d, H, num_pages,
                      scale, 1, workspace, (size_t)L.decode_bytes, out, lse, stream);
}
