// mla_decode_sm100.cu -- the split scan of paged absorbed-MLA decode on Blackwell
// tensor cores (tcgen05 + TMEM + TMA), sm_100a, for a bf16 cache; the host side of both
// scans (tensor maps, launch, the device's CTA slots).  The e4m3 cache has its own scan
// kernel in mla_decode_sm100_e4m3.cu.
//
// Work unit.  One CTA (one per SM) owns a block of 64 folded query rows (row
// m = i * H + h: the query-sequence axis folded into the head axis, "TokenSpeed" launch
// digest, MLA kernel paragraphs) of one split of one request, and walks the split's
// 64-token pages.  There is no cross-CTA traffic: the CTAs of a plan group read the
// same pages at the same time and share them through L2.
//
// Tensor memory (128 lanes x 512 columns) with 64-row MMAs, whose rows occupy 16 lanes
// of each 32-lane subpartition:
//   lanes at offset 0  : O, the 64 x 512 fp32 output accumulator (all 512 columns)
//   lanes at offset 16 : q's latent part (64 x 512 bf16, 256 columns, loaded once per
//                        split), two 64-column buffers for the first half of each page's
//                        scores and two for the second half.
// q's rope part (64 x 64 bf16, 8 KB) sits in shared memory, in the epilogue's staging tile
// (which the epilogue needs only after the split's last MMA), as the A operand of the
// four rope K-steps.
// Per page:
//   TMA (producer warp): the page's 64 rows x 576 columns as nine 64-column boxes with
//       128-byte swizzle (one 72 KB stage; three stages).
//   MMA (two threads): S = q . K^T (M=64 N=64 K=16, 36 K-steps), its first 18 K-steps
//       issued by one thread (warp 1) and its last 18 by another (warp 6) into a second
//       accumulator: one thread issuing a 64-row MMA takes about as long as the tensor core
//       takes to run it, so one issuer alone leaves the tensor core short of work.  q comes
//       from TMEM, except in the four rope K-steps.  Warp 1 also issues O += P . V with P
//       (bf16) and V (the same page, read MN-major) from shared memory (M=64 N=256 K=16,
//       twice, 4 K-steps each).  P is written over the page's rope chunk, which only the
//       score MMAs read: every stage carries its own P, and the softmax of a page never
//       waits for the previous page's PV.
//   softmax (4 warps, 16 rows each, two threads per row with 32 scores each): adds the
//       two halves of the scores, base-2 online softmax with the causal draft mask; the running max is only raised (and
//       O rescaled) when a score exceeds it by more than 8, so P <= 256.
//   epilogue: O / l -> bf16 out (a request the split holds whole) or an fp32 partial and
//       its base-2 lse (split request; merged by the combine kernel).
#include <math.h>
#include <string.h>

#include <mutex>

#include "mla_scan_common.cuh"

namespace mla {
namespace {

using namespace scan;

constexpr int kStages = 3;
// warp 0 TMA, warp 1 score chain (first half) and PV, warps 2-5 softmax / epilogue, warp 6
// score chain (second half)
constexpr int kThreadsBf16 = kThreads + 32;
constexpr uint32_t kChunk = kTok * 128;              // 64 tokens x 64 columns bf16, 128B-swizzled
constexpr uint32_t kStageBytes = 9 * kChunk;         // 8 latent chunks + 1 rope chunk: 72 KB
constexpr uint32_t kOffKv = 0;
constexpr uint32_t kOffPInStage = 8 * kChunk;        // P (64 rows x 64 tokens bf16) over the rope chunk
constexpr uint32_t kOffEpi = kOffKv + kStages * kStageBytes;  // epilogue staging: 2 KB per softmax warp
constexpr uint32_t kOffBar = kOffEpi + 4 * kEpiWarpBytes;
static_assert(kRows * kTok * 2 == kChunk, "P fills the rope chunk exactly");
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
static_assert(kSmemBytes <= (uint32_t)kMaxSmem, "dynamic shared memory limit per block");

enum : int {
    B_KV_FULL0 = 0, B_KV_EMPTY0 = B_KV_FULL0 + kStages, B_Q_FULL = B_KV_EMPTY0 + kStages, B_S_FULL0,
    B_P_READY0 = B_S_FULL0 + 2, B_PV_DONE0 = B_P_READY0 + 2, B_DRAIN = B_PV_DONE0 + 2,
    B_SB_FULL0, B_SB_FREE0 = B_SB_FULL0 + 2, B_DRAIN_B = B_SB_FREE0 + 2, B_COUNT
};
constexpr uint32_t kOffTmemHolder = kOffBar + 8 * B_COUNT;
constexpr uint32_t kOffAbort = kOffTmemHolder + 4;
static_assert(kOffAbort + 4 <= kOffBar + 256, "barrier area");

constexpr uint32_t kColQ = 0;            // q, dims 0-511: 256 columns (bf16 pairs)
constexpr uint32_t kColS = 256;          // scores, K-steps [0, kHalfSteps): 2 x 64 columns
constexpr uint32_t kColSB = 384;         // scores, K-steps [kHalfSteps, 36): 2 x 64 columns
constexpr int kHalfSteps = 18;
constexpr int kRopeStep = 32;            // K-steps 32-35 read q's rope part from shared memory
static_assert(kHalfSteps <= kRopeStep, "the first issuer reads q from TMEM only");
static_assert(kRows * 128 == 4 * kEpiWarpBytes, "q's rope part fills the epilogue staging tile");
constexpr float kRescaleThreshold = 8.0f;

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kRows, kTok, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kRows, 256, 0, 1);

// Score K-steps [K0, K0 + NK) (of 36) into accumulator d, the first of them overwriting it:
// q from TMEM, the page from shared memory.  K0 is a template constant so that every
// descriptor offset is an immediate.
template <int K0, int NK>
__device__ __forceinline__ void issue_s_steps(uint32_t d, uint32_t a0, uint64_t b0) {
#pragma unroll
    for (int k = 0; k < NK; ++k) {
        constexpr int kChunkUnits = kChunk >> 4;
        const int ks = K0 + k;
        ptx::mma_ts(d, a0 + 8u * ks, b0 + (uint64_t)((ks >> 2) * kChunkUnits + (ks & 3) * 2), kIdescS,
                    k ? 1u : 0u);
    }
}

// The four rope K-steps (32-35), accumulating into d: A = q's rope part from shared memory
// (K-major, 128-byte swizzle, like P), B = the page's rope chunk.
__device__ __forceinline__ void issue_s_rope(uint32_t d, uint64_t aq, uint64_t b0) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
        ptx::mma_ss(d, aq + (uint64_t)(k * 2), b0 + (uint64_t)(8 * (kChunk >> 4) + k * 2), kIdescS, 1u);
}

__global__ void __launch_bounds__(kThreadsBf16, 1) decode_sm100_kernel(const __grid_constant__ Args args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const DecodeParams& p = args.p;
    PlanHeader* h = reinterpret_cast<PlanHeader*>(p.ws);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // prologue that reads no global memory, ahead of the wait for the grid before this one
    Ctx c;
    c.bar0 = sbase + kOffBar;
    c.abort = reinterpret_cast<volatile int*>(smem + kOffAbort);
    c.h = h;
    if (threadIdx.x == 0) {
        *c.abort = 0;
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(c.bar(B_KV_FULL0 + s), 1);
            ptx::mbar_init(c.bar(B_KV_EMPTY0 + s), 1);
        }
        ptx::mbar_init(c.bar(B_Q_FULL), 128);
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(c.bar(B_S_FULL0 + s), 1);
            ptx::mbar_init(c.bar(B_P_READY0 + s), 128);
            ptx::mbar_init(c.bar(B_PV_DONE0 + s), 1);
        }
        ptx::mbar_init(c.bar(B_DRAIN), 1);
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(c.bar(B_SB_FULL0 + s), 1);
            ptx::mbar_init(c.bar(B_SB_FREE0 + s), 128);
        }
        ptx::mbar_init(c.bar(B_DRAIN_B), 1);
        ptx::fence_mbar_init_cluster();
    }
    if (warp == 0 && lane == 0) ptx::prefetch_tmap(&args.tm_kv);
    if (warp == 1) {
        ptx::tmem_alloc(sbase + kOffTmemHolder, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemHolder);

    // the plan (and every earlier write) must be complete before the header is read
    ptx::griddep_wait();
    // Only now may the combine launch: it reads the plan before its own wait for this grid
    // (the plan is complete once the wait above returns), the partials after it.
    ptx::griddep_launch_dependents();
    // The header and this group's head record are read together: the head table sits at a
    // fixed offset, and every workspace the host accepts holds it for any group launched.
    const int nqb = num_row_blocks(p.s_q, p.H);
    const int g = blockIdx.x / nqb, qb = blockIdx.x % nqb;
    const GroupHead gh = ws_ptr<GroupHead>(p.ws, kOffHeads)[g];
    const bool plan_ok = h->magic == kPlanMagic && h->B == p.B && h->s_q == p.s_q && h->H == p.H &&
                         h->num_groups <= p.groups_launched;
    if (!plan_ok || g >= h->num_groups) {
        if (!plan_ok && blockIdx.x == 0 && threadIdx.x == 0) set_status(h, kStatusPlanMismatch, 0);
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
        if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
        return;
    }

    const Segment* segs = ws_ptr<Segment>(p.ws, h->off_segs);
    const int seg_lo = gh.seg_lo, seg_hi = gh.seg_hi;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp walks the tiles; every 32 tiles each lane fetches one block-table
        // entry (one window ahead), so the page ids reach lane 0 (which waits and issues) by
        // shuffles instead of one dependent global load per page.
        int it = 0;
        bool ok = true;
        for (int si = seg_lo; si < seg_hi && ok; ++si) {
            if (__shfl_sync(0xffffffffu, lane == 0 ? *c.abort : 0, 0)) break;
            const Segment S = si == seg_lo ? gh.first : segs[si];
            const int32_t* bt_row = p.block_table + (int64_t)S.b * p.max_pages;
            // the first window of page ids is read beside the length (both wait on the same
            // round trip); a window slot past max_pages is never read
            const int t_first = S.tile_begin + lane;
            const int32_t pg_first = (t_first < S.tile_end && t_first < p.max_pages) ? bt_row[t_first] : 0;
            const int T = p.seq_lens[S.b];
            if (!request_ok(p, T)) continue;
            int32_t pg = 0, pgn = 0;  // page ids of tiles [t0, t0 + 32) and [t0 + 32, t0 + 64)
            for (int t = S.tile_begin; t < S.tile_end; ++t, ++it) {
                const int j = (t - S.tile_begin) & 31;
                if (j == 0) {
                    pg = t == S.tile_begin ? pg_first : pgn;
                    pgn = (t + 32 + lane < S.tile_end) ? bt_row[t + 32 + lane] : 0;
                }
                const int32_t page = __shfl_sync(0xffffffffu, pg, j);
                if (lane == 0) {
                    const int st = it % kStages;
                    if (it >= kStages && !wait_bar(c, c.bar(B_KV_EMPTY0 + st), ((it / kStages) - 1) & 1)) {
                        ok = false;
                    } else {
                        // an invalid page id becomes a box entirely out of range (zero fill);
                        // the softmax warps see the same id and poison the request's rows
                        const int ky = (page >= 0 && page < p.num_pages) ? page * kPage : -kPage;
                        const uint32_t dst = sbase + kOffKv + st * kStageBytes;
                        ptx::mbar_arrive_expect_tx(c.bar(B_KV_FULL0 + st), kStageBytes);
#pragma unroll
                        for (int jb = 0; jb < 9; ++jb)
                            ptx::tma_load_2d(dst + jb * kChunk, &args.tm_kv, c.bar(B_KV_FULL0 + st), 64 * jb, ky);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        if (lane == 0 && *c.abort) {
            for (int k = (it > kStages ? it - kStages : 0); k < it; ++k)
                drain_wait(c.bar(B_KV_FULL0 + k % kStages), (k / kStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // An event loop: the first half of the next page's score MMAs and the PV MMAs of the
        // oldest page whose P is ready are issued in whichever order their inputs arrive.
        // Barriers are polled with test_wait, which never suspends the thread.
        if (lane == 0) {
            int it = 0, nseg = 0;
            bool ok = true;
            for (int si = seg_lo; si < seg_hi && ok; ++si) {
                const Segment S = si == seg_lo ? gh.first : segs[si];
                const int T = p.seq_lens[S.b];
                if (!request_ok(p, T)) continue;
                if (!wait_bar(c, c.bar(B_Q_FULL), nseg & 1)) break;
                ptx::tc_fence_after();
                const int n = S.tile_end - S.tile_begin;
                int ns = 0, npv = 0;  // pages of this split with S issued / PV issued
                PollClock clk;
                while (npv < n) {
                    bool progressed = false;
                    // S(ns) reuses the score buffer of page ns-2, whose PV must be issued first.
                    // The chain's half is issued whole: PV MMAs placed between its K-steps (another
                    // accumulator) slow it down far more than they gain.
                    if (ns < n && ns <= npv + 1) {
                        const int its = it + ns, st = its % kStages;
                        if (ptx::mbar_test_wait(c.bar(B_KV_FULL0 + st), (its / kStages) & 1)) {
                            ptx::tc_fence_after();
                            // descriptors are built once and advanced by constant 16-byte offsets:
                            // the fully unrolled issue loop is a handful of integer adds per MMA
                            const uint64_t b0 = ptx::smem_desc(sbase + kOffKv + st * kStageBytes, 16, 1024,
                                                               ptx::kSwizzle128);
                            const uint32_t d = tmem + kLaneHi + kColS + 64u * (its & 1);
                            const uint32_t a0 = tmem + kLaneHi + kColQ;
                            issue_s_steps<0, kHalfSteps>(d, a0, b0);
                            ptx::mma_commit(c.bar(B_S_FULL0 + (its & 1)));
                            ++ns;
                            progressed = true;
                        }
                    }
                    if (npv < ns) {
                        const int itp = it + npv;
                        if (ptx::mbar_test_wait(c.bar(B_P_READY0 + (itp & 1)), (itp >> 1) & 1)) {
                            ptx::tc_fence_after();
                            const bool first = npv == 0;
                            // A = P (K-major); B = V, MN-major: 64-column blocks 8 KB apart (leading
                            // offset), 8-token groups 1 KB apart (stride offset)
                            const uint32_t stage = sbase + kOffKv + (itp % kStages) * kStageBytes;
                            const uint64_t a0 = ptx::smem_desc(stage + kOffPInStage, 16, 1024, ptx::kSwizzle128);
                            const uint64_t v0 = ptx::smem_desc(stage, kChunk, 1024, ptx::kSwizzle128);
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)
                                    ptx::mma_ss(tmem + 256u * half, a0 + (uint64_t)(ks * 2),
                                                v0 + (uint64_t)(half * 4 * (kChunk >> 4) + ks * (2048 >> 4)), kIdescPV,
                                                (first && ks == 0) ? 0u : 1u);
                            }
                            ptx::mma_commit(c.bar(B_PV_DONE0 + (itp & 1)));
                            ptx::mma_commit(c.bar(B_KV_EMPTY0 + (itp % kStages)));
                            ++npv;
                            progressed = true;
                        }
                    }
                    if (!clk.step(c, progressed)) {
                        ok = false;
                        break;
                    }
                }
                it += n;
                ++nseg;
            }
            ptx::mma_commit(c.bar(B_DRAIN));
            drain_wait(c.bar(B_DRAIN), 0);
        }
    } else if (warp == 6) {
        // ------------------------------------------------------------ second score issuer
        const uint64_t aq = ptx::smem_desc(sbase + kOffEpi, 16, 1024, ptx::kSwizzle128);
        // K-steps [kHalfSteps, 36) of every page's score chain into the second-half buffers.
        // It walks the same pages as the first issuer; a page's half is issued once its
        // stage is full and the softmax warps have loaded the half of the page two before
        // (SB_FREE, the same buffer), so no SB_FULL phase runs ahead of its waiters.
        if (lane == 0) {
            int it = 0, nseg = 0;
            bool ok = true;
            for (int si = seg_lo; si < seg_hi && ok; ++si) {
                const Segment S = si == seg_lo ? gh.first : segs[si];
                const int T = p.seq_lens[S.b];
                if (!request_ok(p, T)) continue;
                if (!wait_bar(c, c.bar(B_Q_FULL), nseg & 1)) break;
                ptx::tc_fence_after();
                const int n = S.tile_end - S.tile_begin;
                for (int j = 0; j < n; ++j) {
                    const int its = it + j, st = its % kStages;
                    if ((its >= 2 && !wait_bar(c, c.bar(B_SB_FREE0 + (its & 1)), ((its - 2) >> 1) & 1)) ||
                        !wait_bar(c, c.bar(B_KV_FULL0 + st), (its / kStages) & 1)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint64_t b0 = ptx::smem_desc(sbase + kOffKv + st * kStageBytes, 16, 1024, ptx::kSwizzle128);
                    const uint32_t d = tmem + kLaneHi + kColSB + 64u * (its & 1);
                    issue_s_steps<kHalfSteps, kRopeStep - kHalfSteps>(d, tmem + kLaneHi + kColQ, b0);
                    issue_s_rope(d, aq, b0);
                    ptx::mma_commit(c.bar(B_SB_FULL0 + (its & 1)));
                }
                it += n;
                ++nseg;
            }
            ptx::mma_commit(c.bar(B_DRAIN_B));
            drain_wait(c.bar(B_DRAIN_B), 0);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        RowSlot r;
        r.quad = warp & 3;                     // TMEM lane quadrant this warp may access
        r.r16 = lane & 15;
        r.half = lane >> 4;                    // score columns [32 half, +32), output columns [32 half + 64 q, +32)
        r.lane = lane;
        r.row = r.quad * 16 + r.r16;           // folded row within the block
        r.qb = qb;
        r.nqb = nqb;
        r.m_glob = qb * kRows + r.row;
        r.row_valid = r.m_glob < p.M;
        const int half = r.half, row = r.row;
        const uint32_t t_hi = tmem + ((uint32_t)(r.quad * 32) << 16) + kLaneHi;  // q and scores
        const uint32_t t_lo = tmem + ((uint32_t)(r.quad * 32) << 16);            // O
        const int tid = threadIdx.x - 64;      // 0..127
        const uint16_t* qsrc = reinterpret_cast<const uint16_t*>(p.q);
        float* plse = ws_ptr<float>(p.ws, h->off_plse);
        float* po = ws_ptr<float>(p.ws, h->off_po);
        int it = 0;
        bool alive = true;

        for (int si = seg_lo; si < seg_hi; ++si) {
            const Segment S = si == seg_lo ? gh.first : segs[si];
            const int T = p.seq_lens[S.b];
            // q rows of this block: dims 0-511 into TMEM (8 x 16 columns per half), the rope
            // part into shared memory.
            // The loads are all issued before the first is used, beside the length's read: at a
            // split's start the memory system is full of the first pages' loads, and every
            // dependent round trip here delays the first score MMA.
            const uint4* src = reinterpret_cast<const uint4*>(qsrc + ((int64_t)S.b * p.M + r.m_glob) * kDqk);
            uint4 x[9][4];
#pragma unroll
            for (int k = 0; k < 9; ++k)
#pragma unroll
                for (int w = 0; w < 4; ++w)  // dims [64 k + 32 half, +32)
                    x[k][w] = r.row_valid ? src[(64 * k + 32 * half) / 8 + w] : make_uint4(0, 0, 0, 0);
            if (!request_ok(p, T)) {
                if (tid == 0) set_status(h, kStatusOob, S.b);
                poison_rows(p, S, si, r, po, plse);
                continue;
            }
            if (*c.abort) break;
            {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    uint32_t v[16];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        v[4 * w] = x[k][w].x;
                        v[4 * w + 1] = x[k][w].y;
                        v[4 * w + 2] = x[k][w].z;
                        v[4 * w + 3] = x[k][w].w;
                    }
                    ptx::tmem_st16x16<16>(t_hi + kColQ + 32u * k, v);
                }
                // the rope part: row `row`, dims [512 + 32 half, +32) as four 16-byte pieces of
                // the row's 128 bytes, 128-byte swizzle; the rows of this warp's quadrant are its
                // own epilogue staging tile, which its previous epilogue has finished with
                uint8_t* qrow = smem + kOffEpi + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    *reinterpret_cast<uint4*>(qrow + (((4 * half + w) ^ (row & 7)) << 4)) = x[8][w];
                ptx::fence_proxy_async_smem();
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(c.bar(B_Q_FULL));
            }
            const int last_t = p.causal ? T - p.s_q + r.m_glob / p.H : T - 1;
            const int full_end = p.causal ? T - p.s_q + 1 : T;  // tokens < full_end are visible to every row
            const int ntiles_req = (T + kPage - 1) / kPage;
            const int n = S.tile_end - S.tile_begin;
            const float sc = p.score_scale_log2;
            float m_run = -INFINITY, l = 0.f;
            bool badpage = false;
            for (int jj = 0; jj < n; ++jj, ++it) {
                const int tile = S.tile_begin + jj;
                const int32_t page = p.block_table[(int64_t)S.b * p.max_pages + tile];
                badpage |= !(page >= 0 && page < p.num_pages);
                alive = wait_bar(c, c.bar(B_S_FULL0 + (it & 1)), (it >> 1) & 1) &&
                        wait_bar(c, c.bar(B_SB_FULL0 + (it & 1)), (it >> 1) & 1);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                ptx::tc_fence_after();
                uint32_t sr[32], sr2[32];
                ptx::tmem_ld16x32<32>(t_hi + kColS + 64u * (it & 1), sr);
                ptx::tmem_ld16x32<32>(t_hi + kColSB + 64u * (it & 1), sr2);
                ptx::tmem_wait_ld();
                // this second-half buffer may take the half of the page two ahead
                ptx::tc_fence_before();
                ptx::mbar_arrive(c.bar(B_SB_FREE0 + (it & 1)));
                float s[32];
                const int tok0 = tile * kPage + 32 * half;
                if (tile * kPage + kPage <= full_end) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) s[k] = (__uint_as_float(sr[k]) + __uint_as_float(sr2[k])) * sc;
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int t = tok0 + k;
                        s[k] = (t < T && t <= last_t) ? (__uint_as_float(sr[k]) + __uint_as_float(sr2[k])) * sc
                                                      : -INFINITY;
                    }
                }
                float mx[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mx[k] = fmaxf(fmaxf(s[4 * k], s[4 * k + 1]), fmaxf(s[4 * k + 2], s[4 * k + 3]));
#pragma unroll
                for (int k = 0; k < 4; ++k) mx[k] = fmaxf(mx[k], mx[k + 4]);
                float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
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
                    alive = wait_bar(c, c.bar(B_PV_DONE0 + ((it - 1) & 1)), ((it - 1) >> 1) & 1);
                    if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                    ptx::tc_fence_after();
                    rescale_o(t_lo, need_o ? alpha : 1.f);
                }
                uint32_t pk[16];
                float rs[4] = {0.f, 0.f, 0.f, 0.f};
                const bool live = m_run != -INFINITY;
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float p0 = live ? fast_exp2(s[2 * k] - m_run) : 0.f;
                    const float p1 = live ? fast_exp2(s[2 * k + 1] - m_run) : 0.f;
                    rs[k & 3] += p0 + p1;
                    pk[k] = pack_bf16(p0, p1);
                }
                l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
                uint8_t* stage_p = smem + kOffKv + (it % kStages) * kStageBytes;
                if (tile == ntiles_req - 1 && (T % kPage) != 0) {
                    // rows past the request's end hold stale data (maybe NaN): zero their
                    // latent columns before the PV product reads them with P = 0
                    alive = wait_bar(c, c.bar(B_KV_FULL0 + it % kStages), (it / kStages) & 1);
                    if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                    const int r0 = T % kPage;
                    const int pieces = (kPage - r0) * 8 * 8;  // rows x latent chunks x 16-byte pieces
                    for (int q = tid; q < pieces; q += 128) {
                        const int rr = r0 + q / 64, j = (q / 8) % 8, w = q % 8;
                        *reinterpret_cast<uint4*>(stage_p + j * kChunk + rr * 128 + w * 16) = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                {
                    // P row `row`, tokens [32 half, 32 half + 32): four 16-byte chunks of the
                    // 128-byte K-major row, 128-byte swizzle, over the page's rope chunk (the
                    // score MMAs that read it have completed: S_FULL was waited above)
                    uint8_t* prow_s = stage_p + kOffPInStage + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int chunk = 4 * half + w;
                        *reinterpret_cast<uint4*>(prow_s + ((chunk ^ (row & 7)) << 4)) =
                            make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
                    }
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();  // the score loads above precede the MMAs that follow P_READY
                ptx::mbar_arrive(c.bar(B_P_READY0 + (it & 1)));
            }
            if (!alive || *c.abort) break;
            // epilogue: wait for the last PV of the split; the row sum is the two halves' sum
            alive = wait_bar(c, c.bar(B_PV_DONE0 + ((it - 1) & 1)), ((it - 1) >> 1) & 1);
            if (__any_sync(0xffffffffu, !alive)) break;
            ptx::tc_fence_after();
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            if (badpage && tid == 0) set_status(h, kStatusOob, S.b);
            const float nanv = __int_as_float(0x7fc00000);
            const float inv = badpage ? nanv : (l > 0.f ? p.out_scale / l : 0.f);
            const float lse2 = badpage ? nanv : (l > 0.f ? m_run + __log2f(l) : -INFINITY);
            // the staging tile of this warp holds its quadrant's rows of q's rope part, which the
            // split's score MMAs (all complete: the last PV is) no longer read
            store_split(p, S, si, r, t_lo, smem + kOffEpi + r.quad * kEpiWarpBytes, inv, lse2, po, plse);
            // the next split's q overwrites TMEM only after this epilogue's reads (same threads)
            ptx::tc_fence_before();
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
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

// The tensor map of the cache depends only on (device, cache pointer, page count); a
// decode step calls the scan once per layer with the same few caches, so the last map
// each host thread encoded is kept and reused while those match.
struct TmapCacheEntry {
    int dev = -1;
    const void* kv = nullptr;
    int64_t num_pages = -1;
    CUtensorMap map;
};

bool cached_kv_map(int dev, const DecodeParams& p, CUtensorMap* out) {
    static thread_local TmapCacheEntry e;
    if (e.dev != dev || e.kv != p.kv || e.num_pages != p.num_pages) {
        const uint64_t kvrows = (uint64_t)p.num_pages * kPage;
        if (!make_map_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.kv, kDqk, kvrows, kDqk * 2, 64, kTok,
                         CU_TENSOR_MAP_SWIZZLE_128B)) {
            e.dev = -1;
            return false;
        }
        e.dev = dev;
        e.kv = p.kv;
        e.num_pages = p.num_pages;
    }
    *out = e.map;
    return true;
}

// The dynamic shared memory opt-in is a per-device property of the kernel: set once.
bool smem_attribute_set(int dev) {
    static int done[64] = {};
    if (dev < 64 && done[dev]) return true;
    if (cudaFuncSetAttribute(decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
        return false;
    if (dev < 64) done[dev] = 1;
    return true;
}

mla_status launch_bf16(const DecodeParams& p, cudaStream_t stream) {
    Args a;
    memset(&a, 0, sizeof(a));
    a.p = p;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (!cached_kv_map(dev, p, &a.tm_kv)) return MLA_ERR_CUDA;
    if (!smem_attribute_set(dev)) return MLA_ERR_CUDA;
    const int ctas = p.groups_launched * num_row_blocks(p.s_q, p.H);
    // programmatic dependent launch: the prologue (barriers, TMEM, tensor map) overlaps the
    // tail of the previous grid in the stream; the kernel waits for it before any global access
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(kThreadsBf16);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_sm100_kernel, a) != cudaSuccess) return MLA_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// The bounded wait of the scan kernel, on a barrier that nothing arrives at, with a 20 ms
// limit: it gives up, sets the timeout status and returns.  A test of that mechanism
// that needs no fault and no hang.
__global__ void wait_timeout_probe_kernel(void* ws) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    const uint32_t b = ptx::smem_u32(&bar);
    ptx::mbar_init(b, 1);
    ptx::fence_mbar_init_cluster();
    Ctx c;
    c.bar0 = b;
    c.abort = &abort_flag;
    c.h = reinterpret_cast<PlanHeader*>(ws);
    wait_bar_for<20000000ull>(c, b, 0);
}

}  // namespace

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

int sm100_cta_slots() {
    // CTAs of the scan kernel the current device keeps resident at once (one per SM; the
    // e4m3 scan has the same block size and shared memory).
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    if (!smem_attribute_set(dev)) return -1;
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_sm100_kernel, kThreadsBf16, kSmemBytes) !=
            cudaSuccess ||
        per_sm <= 0)
        return -1;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    const int n = per_sm * sms;
    if (dev < 64) cached[dev] = n;
    return n;
}

mla_status launch_wait_timeout_probe(void* ws, cudaStream_t stream) {
    wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(ws);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status launch_decode_sm100(const DecodeParams& p, int kv_dtype, cudaStream_t stream) {
    return kv_dtype == MLA_KV_E4M3 ? launch_decode_e4m3(p, stream) : launch_bf16(p, stream);
}

}  // namespace mla
