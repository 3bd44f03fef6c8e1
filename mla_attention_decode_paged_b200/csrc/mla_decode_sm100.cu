// mla_decode_sm100.cu -- the split scan of paged absorbed-MLA decode on Blackwell
// tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// Work unit.  A cluster of two CTAs (a "pair", one CTA per SM) owns one block of 128
// folded query rows (row m = i * H + h, the query-sequence axis folded into the head
// axis so that the MMA M tile is full: "TokenSpeed" launch digest, MLA kernel
// paragraphs) of one split of one request, and walks the split's 64-token pages.
//
// Column split.  The 576-wide score contraction and the 512-wide output are divided
// between the two CTAs: CTA c holds latent columns [256c, 256c+256) and RoPE columns
// [512+32c, 512+32c+32) of q and of every cached row (288 columns, 72 KB of q), and it
// accumulates out[:, 256c:256c+256] in tensor memory.  Each CTA computes the partial
// score S_c = q[:, cols_c] . KV[:, cols_c]^T of a page, the two CTAs swap partials
// through distributed shared memory, and both add them in the same order, so both hold
// bit-identical scores and take identical softmax decisions.  Every score and output
// FLOP is done once, and each CTA loads only its own 288 columns of each page.
//
// Per CTA and page (64 tokens):
//   TMA (producer warp): 4 latent boxes [64 tok x 64 col] (128-byte swizzle) and one RoPE
//       box [64 x 32] (64-byte swizzle) of the physical page block_table[b][p].
//   MMA (one thread): S = Q_c . K_c^T, M=128 N=64, 18 K-steps of 16, into TMEM;
//       later O += P . V_c, M=128 N=256, 4 K-steps, with P read from TMEM and V the same
//       shared-memory page viewed MN-major.
//   softmax (4 warps, one thread per row): partial S from TMEM, exchange, base-2 online
//       softmax with the causal draft mask, P in bf16 back into TMEM over its S columns.
//       The running maximum is only raised (and O rescaled) when a new score exceeds it
//       by more than 8 in base 2, so P <= 256 and rescales are rare.
//   epilogue: O / l -> bf16 out (request held whole by this split) or fp32 partial + lse2
//       (split request; merged by the combine kernel).
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "mla_decode_params.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kRows = 128;       // folded query rows per pair (MMA M)
constexpr int kTok = 64;         // tokens per page / tile (S MMA N)
constexpr int kStages = 3;       // cache pages in flight per CTA
constexpr int kThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2-5 softmax / epilogue

constexpr uint32_t kQLatChunk = kRows * 128;                  // 128 rows x 64 bf16
constexpr uint32_t kQRope = kRows * 64;                       // 128 rows x 32 bf16
constexpr uint32_t kQBytes = 4 * kQLatChunk + kQRope;         // 73,728
constexpr uint32_t kKvLatChunk = kTok * 128;                  // 64 tokens x 64 bf16
constexpr uint32_t kKvRope = kTok * 64;                       // 64 tokens x 32 bf16
constexpr uint32_t kStageBytes = 4 * kKvLatChunk + kKvRope;   // 36,864
constexpr uint32_t kXchgBytes = kRows * kTok * 4;             // fp32 partial scores
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKv = kOffQ + kQBytes;
constexpr uint32_t kOffXchg = kOffKv + kStages * kStageBytes;
constexpr uint32_t kOffBar = kOffXchg + kXchgBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;         // barriers + alignment slack

// mbarrier slots (8 bytes each)
enum : int {
    B_Q_FULL = 0, B_Q_EMPTY, B_KV_FULL0, B_KV_EMPTY0 = B_KV_FULL0 + kStages, B_S_FULL0 = B_KV_EMPTY0 + kStages,
    B_P_READY0 = B_S_FULL0 + 2, B_PV_DONE0 = B_P_READY0 + 2, B_O_EMPTY = B_PV_DONE0 + 2, B_XFULL, B_XEMPTY,
    B_SMSYNC, B_DRAIN, B_COUNT
};
constexpr uint32_t kOffTmemHolder = kOffBar + 8 * B_COUNT;
constexpr uint32_t kOffAbort = kOffTmemHolder + 4;
static_assert(kOffAbort + 4 <= kOffBar + 256, "barrier area");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;     // 256 columns: out[:, 256c : 256c+256] accumulator
constexpr uint32_t kTmemS = 256;   // 2 x 64 columns: scores, then P (bf16 pairs) in place
constexpr float kRescaleThreshold = 8.0f;  // base-2 headroom before the running max is raised
constexpr uint64_t kWaitLimitNs = 2000000000ull;

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kRows, kTok, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kRows, 256, 0, 1);

struct __align__(64) Sm100Args {
    CUtensorMap tm_q_lat;    // q viewed [B*M rows, 576], box 64 cols x 128 rows, 128B swizzle
    CUtensorMap tm_q_rope;   // box 32 x 128, 64B swizzle
    CUtensorMap tm_kv_lat;   // cache viewed [P*64 rows, 576], box 64 x 64, 128B swizzle
    CUtensorMap tm_kv_rope;  // box 32 x 64, 64B swizzle
    DecodeParams p;
};

struct Ctx {
    uint32_t bar0;            // shared address of barrier 0
    volatile int* abort;
    PlanHeader* h;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
};

// Bounded wait: gives up after kWaitLimitNs (sets the timeout status and the CTA abort
// flag), or at once once the CTA is aborting.
__device__ __noinline__ bool wait_bar(const Ctx& c, uint32_t bar, uint32_t parity, bool cluster_scope) {
    if (*c.abort) return false;
    uint64_t t0 = 0;
    for (uint32_t n = 1;; ++n) {
        bool ok = cluster_scope ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity);
        if (ok) return true;
        if ((n & 255) == 0) {
            if (*c.abort) return false;
            uint64_t now = ptx::globaltimer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kWaitLimitNs) {
                *c.abort = 1;
                set_status(c.h, kStatusTimeout, (int)blockIdx.x);
                return false;
            }
        }
    }
}

// Wait that ignores the abort flag, used only on the way out for work already in flight.
__device__ void drain_wait(uint32_t bar, uint32_t parity) {
    uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > 200000000ull) return;
    }
}

__device__ __forceinline__ bool request_ok(const DecodeParams& p, int T) {
    return T >= 1 && T <= p.max_pages * kPage && !(p.causal && T < p.s_q);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    decode_sm100_kernel(const __grid_constant__ Sm100Args args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const DecodeParams& p = args.p;
    PlanHeader* h = reinterpret_cast<PlanHeader*>(p.ws);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (h->magic != kPlanMagic || h->B != p.B || h->s_q != p.s_q || h->H != p.H ||
        h->num_groups > p.groups_launched) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(h, kStatusPlanMismatch, 0);
        return;  // both CTAs of every pair see the same header
    }
    const int nqb = h->nqb;
    const int pair = blockIdx.x >> 1;
    const int g = pair / nqb, qb = pair % nqb;
    if (g >= h->num_groups) return;
    const uint32_t crank = ptx::cluster_ctarank();
    const uint32_t peer = crank ^ 1u;

    Ctx c;
    c.bar0 = sbase + kOffBar;
    c.abort = reinterpret_cast<volatile int*>(smem + kOffAbort);
    c.h = h;

    if (threadIdx.x == 0) {
        *c.abort = 0;
        ptx::mbar_init(c.bar(B_Q_FULL), 1);
        ptx::mbar_init(c.bar(B_Q_EMPTY), 1);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(c.bar(B_KV_FULL0 + s), 1);
            ptx::mbar_init(c.bar(B_KV_EMPTY0 + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(c.bar(B_S_FULL0 + s), 1);
            ptx::mbar_init(c.bar(B_P_READY0 + s), 128);
            ptx::mbar_init(c.bar(B_PV_DONE0 + s), 1);
        }
        ptx::mbar_init(c.bar(B_O_EMPTY), 128);
        ptx::mbar_init(c.bar(B_XFULL), 1);
        ptx::mbar_init(c.bar(B_XEMPTY), 1);
        ptx::mbar_init(c.bar(B_SMSYNC), 128);
        ptx::mbar_init(c.bar(B_DRAIN), 1);
        ptx::fence_mbar_init_cluster();
        // arm the first exchange phase: the peer's partial scores complete it
        ptx::mbar_arrive_expect_tx(c.bar(B_XFULL), kXchgBytes);
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&args.tm_q_lat);
        ptx::prefetch_tmap(&args.tm_q_rope);
        ptx::prefetch_tmap(&args.tm_kv_lat);
        ptx::prefetch_tmap(&args.tm_kv_rope);
    }
    if (warp == 1) {
        ptx::tmem_alloc(sbase + kOffTmemHolder, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    ptx::cluster_sync();  // the peer's barriers exist before any remote arrive or st.async
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemHolder);

    const int32_t* group_begin = ws_ptr<int32_t>(p.ws, h->off_group_begin);
    const Segment* segs = ws_ptr<Segment>(p.ws, h->off_segs);
    const int seg_lo = group_begin[g], seg_hi = group_begin[g + 1];

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int it = 0, nseg = 0;
            for (int si = seg_lo; si < seg_hi && !*c.abort; ++si) {
                const Segment S = segs[si];
                const int T = p.seq_lens[S.b];
                if (!request_ok(p, T)) continue;
                if (nseg > 0 && !wait_bar(c, c.bar(B_Q_EMPTY), (nseg - 1) & 1, false)) break;
                const int qy = S.b * p.M + qb * kRows;
                ptx::mbar_arrive_expect_tx(c.bar(B_Q_FULL), kQBytes);
                for (int j = 0; j < 4; ++j)
                    ptx::tma_load_2d(sbase + kOffQ + j * kQLatChunk, &args.tm_q_lat, c.bar(B_Q_FULL),
                                     256 * (int)crank + 64 * j, qy);
                ptx::tma_load_2d(sbase + kOffQ + 4 * kQLatChunk, &args.tm_q_rope, c.bar(B_Q_FULL),
                                 512 + 32 * (int)crank, qy);
                for (int t = S.tile_begin; t < S.tile_end; ++t, ++it) {
                    const int st = it % kStages;
                    if (it >= kStages && !wait_bar(c, c.bar(B_KV_EMPTY0 + st), ((it / kStages) - 1) & 1, false))
                        break;
                    const int32_t page = p.block_table[(int64_t)S.b * p.max_pages + t];
                    // an invalid page id becomes a fully out-of-range box (zero fill); the
                    // softmax warps see the same id and poison the rows
                    const int ky = (page >= 0 && page < p.num_pages) ? page * kPage : -kPage;
                    const uint32_t dst = sbase + kOffKv + st * kStageBytes;
                    ptx::mbar_arrive_expect_tx(c.bar(B_KV_FULL0 + st), kStageBytes);
                    for (int j = 0; j < 4; ++j)
                        ptx::tma_load_2d(dst + j * kKvLatChunk, &args.tm_kv_lat, c.bar(B_KV_FULL0 + st),
                                         256 * (int)crank + 64 * j, ky);
                    ptx::tma_load_2d(dst + 4 * kKvLatChunk, &args.tm_kv_rope, c.bar(B_KV_FULL0 + st),
                                     512 + 32 * (int)crank, ky);
                }
                ++nseg;
            }
            if (*c.abort) {
                // let loads already issued land before the CTA goes away
                for (int k = (it > kStages ? it - kStages : 0); k < it; ++k)
                    drain_wait(c.bar(B_KV_FULL0 + k % kStages), (k / kStages) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, nseg = 0;
            bool ok = true;
            for (int si = seg_lo; si < seg_hi && ok; ++si) {
                const Segment S = segs[si];
                const int T = p.seq_lens[S.b];
                if (!request_ok(p, T)) continue;
                if (!wait_bar(c, c.bar(B_Q_FULL), nseg & 1, false)) break;
                ptx::tc_fence_after();
                const int n = S.tile_end - S.tile_begin;
                auto issue_pv = [&](int itp, bool first) -> bool {
                    if (first && nseg > 0 && !wait_bar(c, c.bar(B_O_EMPTY), (nseg - 1) & 1, false)) return false;
                    if (!wait_bar(c, c.bar(B_P_READY0 + (itp & 1)), (itp >> 1) & 1, false)) return false;
                    ptx::tc_fence_after();
                    const uint32_t vbase = sbase + kOffKv + (itp % kStages) * kStageBytes;
                    const uint32_t a_tmem = tmem + kTmemS + 64u * (itp & 1);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        // V = the page's latent columns, MN-major: 64-column blocks 8 KB apart
                        // (leading offset), 8-token groups 1 KB apart (stride offset)
                        const uint64_t bdesc = ptx::smem_desc(vbase + ks * 2048, kKvLatChunk, 1024, ptx::kSwizzle128);
                        ptx::mma_ts(tmem + kTmemO, a_tmem + 8 * ks, bdesc, kIdescPV, (first && ks == 0) ? 0u : 1u);
                    }
                    ptx::mma_commit(c.bar(B_PV_DONE0 + (itp & 1)));
                    ptx::mma_commit(c.bar(B_KV_EMPTY0 + (itp % kStages)));
                    return true;
                };
                for (int jj = 0; jj < n && ok; ++jj, ++it) {
                    const int st = it % kStages;
                    if (!wait_bar(c, c.bar(B_KV_FULL0 + st), (it / kStages) & 1, false)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t kbase = sbase + kOffKv + st * kStageBytes;
                    const uint32_t d = tmem + kTmemS + 64u * (it & 1);
#pragma unroll
                    for (int kc = 0; kc < 4; ++kc) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t a = ptx::smem_desc(sbase + kOffQ + kc * kQLatChunk + ks * 32, 16, 1024,
                                                              ptx::kSwizzle128);
                            const uint64_t b = ptx::smem_desc(kbase + kc * kKvLatChunk + ks * 32, 16, 1024,
                                                              ptx::kSwizzle128);
                            ptx::mma_ss(d, a, b, kIdescS, (kc | ks) ? 1u : 0u);
                        }
                    }
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        const uint64_t a = ptx::smem_desc(sbase + kOffQ + 4 * kQLatChunk + ks * 32, 16, 512,
                                                          ptx::kSwizzle64);
                        const uint64_t b = ptx::smem_desc(kbase + 4 * kKvLatChunk + ks * 32, 16, 512, ptx::kSwizzle64);
                        ptx::mma_ss(d, a, b, kIdescS, 1u);
                    }
                    ptx::mma_commit(c.bar(B_S_FULL0 + (it & 1)));
                    if (jj > 0 && !issue_pv(it - 1, jj == 1)) { ok = false; break; }
                }
                if (!ok) break;
                if (!issue_pv(it - 1, n == 1)) break;
                ptx::mma_commit(c.bar(B_Q_EMPTY));
                ++nseg;
            }
            ptx::mma_commit(c.bar(B_DRAIN));
            drain_wait(c.bar(B_DRAIN), 0);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
        const int row = quad * 32 + lane;          // folded row within the block
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
        const int tid = threadIdx.x - 64;          // 0..127
        const uint32_t xchg_local = sbase + kOffXchg;
        const uint32_t xchg_remote = ptx::mapa(xchg_local, peer);
        const uint32_t xfull_remote = ptx::mapa(c.bar(B_XFULL), peer);
        const uint32_t xempty_remote = ptx::mapa(c.bar(B_XEMPTY), peer);
        const float* xchg_f = reinterpret_cast<const float*>(smem + kOffXchg);
        const int m_glob = qb * kRows + row;
        const bool row_valid = m_glob < p.M;
        float* plse = ws_ptr<float>(p.ws, h->off_plse);
        float* po = ws_ptr<float>(p.ws, h->off_po);
        int it = 0, nseg = 0;

        for (int si = seg_lo; si < seg_hi; ++si) {
            const Segment S = segs[si];
            const int T = p.seq_lens[S.b];
            const int64_t orow = (int64_t)S.b * p.M + m_glob;
            const int64_t prow = ((int64_t)si * nqb + qb) * kRows + row;
            if (!request_ok(p, T)) {
                if (tid == 0) set_status(h, kStatusOob, S.b);
                if (row_valid) {
                    const float nanv = __int_as_float(0x7fc00000);
                    if (!S.split) {
                        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + orow * kDv + 256 * crank;
                        for (int k = 0; k < 256; ++k) dst[k] = __float2bfloat16_rn(nanv);
                        if (crank == 0) p.lse[orow] = nanv;
                    } else {
                        float* dst = po + prow * kDv + 256 * crank;
                        for (int k = 0; k < 256; ++k) dst[k] = nanv;
                        if (crank == 0) plse[prow] = nanv;
                    }
                }
                continue;
            }
            if (*c.abort) break;
            const int last_t = p.causal ? T - p.s_q + m_glob / p.H : T - 1;
            const int ntiles_req = (T + kPage - 1) / kPage;
            const int n = S.tile_end - S.tile_begin;
            float m_run = -INFINITY, l = 0.f;
            bool badpage = false;
            bool alive = true;
            for (int jj = 0; jj < n; ++jj, ++it) {
                const int tile = S.tile_begin + jj;
                const int32_t page = p.block_table[(int64_t)S.b * p.max_pages + tile];
                badpage |= !(page >= 0 && page < p.num_pages);
                const int sb = it & 1;
                alive = wait_bar(c, c.bar(B_S_FULL0 + sb), (it >> 1) & 1, false);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                ptx::tc_fence_after();
                uint32_t sr[64];
                ptx::tmem_ld32(trow + kTmemS + 64u * sb, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                ptx::tmem_ld32(trow + kTmemS + 64u * sb + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                ptx::tmem_wait_ld();
                float s[64];
#pragma unroll
                for (int k = 0; k < 64; ++k) s[k] = __uint_as_float(sr[k]);
                // exchange partial scores with the peer CTA
                if (it > 0) alive = wait_bar(c, c.bar(B_XEMPTY), (it - 1) & 1, true);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
#pragma unroll
                for (int k4 = 0; k4 < 16; ++k4)
                    ptx::st_async_v4(xchg_remote + (uint32_t)(k4 * kRows + row) * 16u,
                                     make_float4(s[4 * k4], s[4 * k4 + 1], s[4 * k4 + 2], s[4 * k4 + 3]), xfull_remote);
                alive = wait_bar(c, c.bar(B_XFULL), it & 1, true);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
#pragma unroll
                for (int k4 = 0; k4 < 16; ++k4) {
                    const float4 v = *reinterpret_cast<const float4*>(xchg_f + (size_t)(k4 * kRows + row) * 4);
                    s[4 * k4] += v.x;
                    s[4 * k4 + 1] += v.y;
                    s[4 * k4 + 2] += v.z;
                    s[4 * k4 + 3] += v.w;
                }
                // all 128 rows have read the peer's data: re-arm and release the buffer
                ptx::mbar_arrive(c.bar(B_SMSYNC));
                alive = wait_bar(c, c.bar(B_SMSYNC), it & 1, false);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                if (tid == 0) {
                    ptx::mbar_arrive_expect_tx(c.bar(B_XFULL), kXchgBytes);
                    ptx::mbar_arrive_remote(xempty_remote);
                }
                // base-2 scores with the visibility mask
                const int tok0 = tile * kPage;
                float mt = -INFINITY;
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    const int t = tok0 + k;
                    s[k] = (t < T && t <= last_t) ? s[k] * p.score_scale_log2 : -INFINITY;
                    mt = fmaxf(mt, s[k]);
                }
                const bool raise = mt > m_run + kRescaleThreshold;
                float alpha = 1.f;
                if (raise) {
                    alpha = fast_exp2(m_run - mt);
                    l *= alpha;
                }
                const bool need_o = raise && jj > 0 && m_run != -INFINITY;
                if (raise) m_run = mt;
                if (__any_sync(0xffffffffu, need_o)) {
                    // O holds earlier pages of this split: wait for the last PV, rescale the rows
                    alive = wait_bar(c, c.bar(B_PV_DONE0 + ((it - 1) & 1)), ((it - 1) >> 1) & 1, false);
                    if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                    ptx::tc_fence_after();
                    const float f = need_o ? alpha : 1.f;
#pragma unroll 1
                    for (int q = 0; q < 8; ++q) {
                        uint32_t o[32];
                        ptx::tmem_ld32(trow + kTmemO + 32 * q, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
                        ptx::tmem_st32(trow + kTmemO + 32 * q, o);
                    }
                    ptx::tmem_wait_st();
                }
                uint32_t pk[32];
                float rs = 0.f;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float p0 = m_run == -INFINITY ? 0.f : fast_exp2(s[2 * k] - m_run);
                    const float p1 = m_run == -INFINITY ? 0.f : fast_exp2(s[2 * k + 1] - m_run);
                    rs += p0 + p1;
                    pk[k] = pack_bf16(p0, p1);
                }
                l += rs;
                if (tile == ntiles_req - 1 && (T % kPage) != 0) {
                    // rows past the request's end hold stale data (maybe NaN): zero their
                    // latent columns before the PV product reads them with P = 0
                    alive = wait_bar(c, c.bar(B_KV_FULL0 + it % kStages), (it / kStages) & 1, false);
                    if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                    const int r0 = T % kPage;
                    uint8_t* vb = smem + kOffKv + (it % kStages) * kStageBytes;
                    const int pieces = (kPage - r0) * 4 * 8;  // rows x chunks x 16-byte pieces
                    for (int q = tid; q < pieces; q += 128) {
                        const int r = r0 + q / 32, j = (q / 8) % 4, w = q % 8;
                        *reinterpret_cast<uint4*>(vb + j * kKvLatChunk + r * 128 + w * 16) = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                ptx::tmem_st32(trow + kTmemS + 64u * sb, pk);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(c.bar(B_P_READY0 + sb));
            }
            if (!alive || *c.abort) break;
            // epilogue: wait for the last PV of the split
            alive = wait_bar(c, c.bar(B_PV_DONE0 + ((it - 1) & 1)), ((it - 1) >> 1) & 1, false);
            if (__any_sync(0xffffffffu, !alive)) break;
            ptx::tc_fence_after();
            if (badpage && tid == 0) set_status(h, kStatusOob, S.b);
            const float nanv = __int_as_float(0x7fc00000);
            const float inv = badpage ? nanv : (l > 0.f ? p.out_scale / l : 0.f);
#pragma unroll 1
            for (int q = 0; q < 8; ++q) {
                uint32_t o[32];
                ptx::tmem_ld32(trow + kTmemO + 32 * q, o);
                ptx::tmem_wait_ld();
                if (!row_valid) continue;
                if (!S.split) {
                    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) + orow * kDv +
                                                          256 * crank + 32 * q);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
                        dst[v] = w;
                    }
                } else {
                    float4* dst = reinterpret_cast<float4*>(po + prow * kDv + 256 * crank + 32 * q);
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                             __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
                }
            }
            if (row_valid && crank == 0) {
                const float lse2 = badpage ? nanv : (l > 0.f ? m_run + __log2f(l) : -INFINITY);
                if (!S.split)
                    p.lse[orow] = lse2 * kLn2;
                else
                    plse[prow] = lse2;
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(c.bar(B_O_EMPTY));
            ++nseg;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
    ptx::cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
}

// ------------------------------------------------------------------ host side

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

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t cols, uint64_t rows,
                 uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int sm100_pair_slots() {
    // How many pairs of this kernel the current device runs at once (1 CTA per SM).
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    if (cudaFuncSetAttribute(decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
        return -1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, decode_sm100_kernel, &cfg) != cudaSuccess || n <= 0) return -1;
    if (dev < 64) cached[dev] = n;
    return n;
}

mla_status launch_decode_sm100(const DecodeParams& p, cudaStream_t stream) {
    Sm100Args a;
    memset(&a, 0, sizeof(a));
    a.p = p;
    const uint64_t qrows = (uint64_t)p.B * p.M;
    const uint64_t kvrows = (uint64_t)p.num_pages * kPage;
    if (!make_map_2d(&a.tm_q_lat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, kDqk, qrows, kDqk * 2, 64, kRows,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&a.tm_q_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.q, kDqk, qrows, kDqk * 2, 32, kRows,
                     CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_2d(&a.tm_kv_lat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.kv, kDqk, kvrows, kDqk * 2, 64, kTok,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&a.tm_kv_rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.kv, kDqk, kvrows, kDqk * 2, 32, kTok,
                     CU_TENSOR_MAP_SWIZZLE_64B))
        return MLA_ERR_CUDA;
    if (cudaFuncSetAttribute(decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
        return MLA_ERR_CUDA;
    const int clusters = p.groups_launched * num_row_blocks(p.s_q, p.H);
    decode_sm100_kernel<<<2 * clusters, kThreads, kSmemBytes, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
