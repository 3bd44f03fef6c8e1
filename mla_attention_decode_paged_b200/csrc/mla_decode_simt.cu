// mla_decode_simt.cu -- straightforward CUDA-core decode kernel (fp32 FMA).
//
// One CTA handles 32 folded query rows of one row block for every split of its plan
// group: q rows and 32-token cache tiles are staged in shared memory as fp32 (bf16 and
// e4m3 both widen exactly), scores in base 2, online softmax with a running max and
// sum per row, and a probability-weighted sum of the 512 latent columns.  Rows past a
// request's length are zero-filled on load, so the NaN of stale or unwritten rows
// never meets a zero probability.
#include "mla_decode_params.cuh"

namespace mla {
namespace {

constexpr int kSimtRows = 32;
constexpr int kSimtTok = 32;
constexpr int kLd = kDqk + 4;  // padded row stride (floats): conflict-free column reads

template <int KV_DTYPE>
__device__ __forceinline__ void load_kv_row_chunk(const void* kv, int64_t row, int c, float* dst) {
    if (KV_DTYPE == MLA_KV_BF16) {
        // 8 bf16 per 16-byte chunk, 72 chunks per row
        uint4 v = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(kv) + row * kDqk)[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float4 a, bq;
        a.x = __uint_as_float(w[0] << 16); a.y = __uint_as_float(w[0] & 0xffff0000u);
        a.z = __uint_as_float(w[1] << 16); a.w = __uint_as_float(w[1] & 0xffff0000u);
        bq.x = __uint_as_float(w[2] << 16); bq.y = __uint_as_float(w[2] & 0xffff0000u);
        bq.z = __uint_as_float(w[3] << 16); bq.w = __uint_as_float(w[3] & 0xffff0000u);
        reinterpret_cast<float4*>(dst + c * 8)[0] = a;
        reinterpret_cast<float4*>(dst + c * 8)[1] = bq;
    } else {
        // 16 e4m3 per 16-byte chunk, 36 chunks per row
        uint4 v = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(kv) + row * kDqk)[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float2 lo = e4m3x2_to_float2((uint16_t)(w[k] & 0xffff));
            float2 hi = e4m3x2_to_float2((uint16_t)(w[k] >> 16));
            reinterpret_cast<float4*>(dst + c * 16)[k] = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
    }
}

template <int KV_DTYPE>
__global__ void __launch_bounds__(256, 1) decode_simt_kernel(DecodeParams p) {
    extern __shared__ float4 smem4[];
    float* qs = reinterpret_cast<float*>(smem4);          // [32][kLd]
    float* kvs = qs + kSimtRows * kLd;                      // [32][kLd]
    float* ps = kvs + kSimtTok * kLd;                       // [32][33]
    __shared__ int bad_page;

    PlanHeader* h = reinterpret_cast<PlanHeader*>(p.ws);
    if (h->magic != kPlanMagic || h->B != p.B || h->s_q != p.s_q || h->H != p.H ||
        h->num_groups > p.groups_launched) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(h, kStatusPlanMismatch, 0);
        return;
    }
    const int nqb = h->nqb;
    const int sub = blockIdx.x % 4;
    const int qb = (blockIdx.x / 4) % nqb;
    const int g = blockIdx.x / (4 * nqb);
    if (g >= h->num_groups) return;
    const int R0 = qb * kRowsPerBlock + sub * kSimtRows;
    const int nrows = min(kSimtRows, p.M - R0);
    if (nrows <= 0) return;

    const int tid = threadIdx.x;
    const int r = tid >> 3;      // row within the CTA
    const int gi = tid & 7;      // token / column interleave
    const int32_t* group_begin = ws_ptr<int32_t>(p.ws, h->off_group_begin);
    const Segment* segs = ws_ptr<Segment>(p.ws, h->off_segs);
    float* plse = ws_ptr<float>(p.ws, h->off_plse);
    float* po = ws_ptr<float>(p.ws, h->off_po);
    const uint16_t* q = reinterpret_cast<const uint16_t*>(p.q);

    for (int si = group_begin[g]; si < group_begin[g + 1]; ++si) {
        const Segment S = segs[si];
        const int b = S.b;
        const int T = p.seq_lens[b];
        bool bad = T < 1 || T > p.max_pages * kPage || (p.causal && T < p.s_q);
        __syncthreads();  // previous segment finished with qs / kvs
        if (tid == 0) bad_page = 0;
        for (int idx = tid; idx < kSimtRows * kDqk; idx += 256) {
            int rr = idx / kDqk, d = idx % kDqk;
            qs[rr * kLd + d] = rr < nrows ? bf16_bits_to_float(q[((int64_t)b * p.M + R0 + rr) * kDqk + d]) : 0.f;
        }
        const int row_global = R0 + r;
        const int last = p.causal ? T - p.s_q + row_global / p.H : T - 1;  // last visible token
        float m = -INFINITY, l = 0.f;
        float o[64];
#pragma unroll
        for (int k = 0; k < 64; ++k) o[k] = 0.f;
        const int tok_begin = S.tile_begin * kPage;
        const int tok_end = bad ? tok_begin : min(S.tile_end * kPage, T);

        for (int t0 = tok_begin; t0 < tok_end; t0 += kSimtTok) {
            __syncthreads();
            constexpr int kChunks = KV_DTYPE == MLA_KV_BF16 ? 72 : 36;
            for (int idx = tid; idx < kSimtTok * kChunks; idx += 256) {
                int tt = idx / kChunks, c = idx % kChunks;
                int t = t0 + tt;
                float* dst = kvs + tt * kLd;
                bool ok = t < tok_end;
                int64_t page = 0;
                if (ok) {
                    page = p.block_table[(int64_t)b * p.max_pages + t / kPage];
                    if (page < 0 || page >= p.num_pages) { ok = false; bad_page = 1; }
                }
                if (ok) {
                    load_kv_row_chunk<KV_DTYPE>(p.kv, page * kPage + (t % kPage), c, dst);
                } else {
                    constexpr int kw = KV_DTYPE == MLA_KV_BF16 ? 8 : 16;
#pragma unroll
                    for (int k = 0; k < kw; ++k) dst[c * kw + k] = 0.f;
                }
            }
            __syncthreads();
            // scores of row r against tokens gi, gi+8, gi+16, gi+24
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const float4* qr = reinterpret_cast<const float4*>(qs + r * kLd);
            for (int d4 = 0; d4 < kDqk / 4; ++d4) {
                float4 a = qr[d4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float4 kk = reinterpret_cast<const float4*>(kvs + (gi + 8 * j) * kLd)[d4];
                    acc[j] = fmaf(a.x, kk.x, acc[j]);
                    acc[j] = fmaf(a.y, kk.y, acc[j]);
                    acc[j] = fmaf(a.z, kk.z, acc[j]);
                    acc[j] = fmaf(a.w, kk.w, acc[j]);
                }
            }
            float x[4], mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int t = t0 + gi + 8 * j;
                x[j] = (t < tok_end && t <= last) ? acc[j] * p.score_scale_log2 : -INFINITY;
                mx = fmaxf(mx, x[j]);
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            const float m_new = fmaxf(m, mx);
            float pj[4], rs = 0.f;
            float alpha = 1.f;
            if (m_new == -INFINITY) {
#pragma unroll
                for (int j = 0; j < 4; ++j) pj[j] = 0.f;
            } else {
                alpha = fast_exp2(m - m_new);
#pragma unroll
                for (int j = 0; j < 4; ++j) { pj[j] = fast_exp2(x[j] - m_new); rs += pj[j]; }
            }
            rs += __shfl_xor_sync(0xffffffffu, rs, 1);
            rs += __shfl_xor_sync(0xffffffffu, rs, 2);
            rs += __shfl_xor_sync(0xffffffffu, rs, 4);
            l = l * alpha + rs;
            m = m_new;
#pragma unroll
            for (int j = 0; j < 4; ++j) ps[r * 33 + gi + 8 * j] = pj[j];
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 64; ++k) o[k] *= alpha;
            for (int j = 0; j < kSimtTok; ++j) {
                const float pv = ps[r * 33 + j];
                const float* vr = kvs + j * kLd + gi;
#pragma unroll
                for (int k = 0; k < 64; ++k) o[k] = fmaf(pv, vr[8 * k], o[k]);
            }
        }
        __syncthreads();
        bad = bad || bad_page;
        if (bad && tid == 0) set_status(h, kStatusOob, b);
        if (r < nrows) {
            const float inv = l > 0.f ? p.out_scale / l : 0.f;
            const float nanv = __int_as_float(0x7fc00000);
            if (!S.split) {
                __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + ((int64_t)b * p.M + row_global) * kDv;
#pragma unroll
                for (int k = 0; k < 64; ++k) dst[gi + 8 * k] = __float2bfloat16_rn(bad ? nanv : o[k] * inv);
                if (gi == 0)
                    p.lse[(int64_t)b * p.M + row_global] = bad ? nanv : (l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY);
            } else {
                const int64_t prow = ((int64_t)si * nqb + qb) * kRowsPerBlock + sub * kSimtRows + r;
                float* dst = po + prow * kDv;
#pragma unroll
                for (int k = 0; k < 64; ++k) dst[gi + 8 * k] = bad ? nanv : o[k] * inv;
                if (gi == 0) plse[prow] = bad ? nanv : (l > 0.f ? m + __log2f(l) : -INFINITY);
            }
        }
    }
}

}  // namespace

mla_status launch_decode_simt(const DecodeParams& p, int kv_dtype, cudaStream_t stream) {
    const int nqb = num_row_blocks(p.s_q, p.H);
    const size_t smem = sizeof(float) * (2 * kSimtRows * kLd + kSimtRows * 33);
    dim3 grid(p.groups_launched * nqb * 4);
    if (kv_dtype == MLA_KV_BF16) {
        cudaFuncSetAttribute(decode_simt_kernel<MLA_KV_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        decode_simt_kernel<MLA_KV_BF16><<<grid, 256, smem, stream>>>(p);
    } else {
        cudaFuncSetAttribute(decode_simt_kernel<MLA_KV_E4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        decode_simt_kernel<MLA_KV_E4M3><<<grid, 256, smem, stream>>>(p);
    }
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
