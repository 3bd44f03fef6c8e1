// mla_decode_sm100_e4m3.cu -- the split scan of paged absorbed-MLA decode for an fp8
// (e4m3) cache on Blackwell tensor cores, sm_100a: e4m3 x e4m3 MMAs (tcgen05
// kind::f8f6f4) that read the cache bytes as they are ("Faster kernels, slower
// engine", setup note on the fp8 KV cache: half the bytes per cached token).  kv_scale
// is folded into the score and output scales.
//
// The CTA, its warp roles, the folded 64-row block, the split plan and the epilogue are
// those of the bf16 scan (mla_decode_sm100.cu, shared pieces in mla_scan_common.cuh).
// What differs:
//
// Operands.  Both MMA operands must be fp8, so q and P are each cut into two e4m3 terms:
//   q_hi = e4m3(q / s_r), q_lo = e4m3(q / s_r - q_hi), where s_r is the smallest power of
//     two with max|q_r| / s_r <= 448: q / s_r is still a bf16 value, whose 8 significant
//     bits the two 4-bit terms hold exactly (bar e4m3's subnormal range), so the scores
//     are those of the bf16 q; s_r multiplies the row's scores.
//   P = 2^(x - m + 4), P_hi = e4m3(P), P_lo = e4m3(P - P_hi): P to 8 significant bits,
//     as a bf16 P would be; the running max is raised (and O rescaled) when a score
//     exceeds it by more than 4, so P <= 256 < 448 and the bulk of a long near-uniform row
//     stays far above e4m3's subnormal floor.  The row sum uses the unrounded P.
//
// Page pairs.  A page is 36 KB in e4m3, so two pages form one work unit: the score MMAs
// run with N = 128 tokens (half the instructions per page of N = 64; a score MMA's cost
// barely grows from N = 64 to 128).  A split's pages are taken in pairs from its start;
// an odd last page is a unit of its own (N = 64).
//
// Shared memory: three pair slots of 72 KB and an 8 KB buffer.  In a slot, chunk j (64
// tokens x 64 bytes, 64-byte swizzle) of the unit's page w sits at j * 8 KB + w * 4 KB, so
// the K-major score operand of chunk j is 128 rows at one 512-byte stride across both
// pages, and the MN-major V operand of a page is its chunks at an 8 KB stride.  P_hi
// (64 rows x 128 tokens) is written over the pair's two rope chunks (which only the score
// MMAs read), P_lo into the 8 KB buffer: a unit's P is written only after the previous
// unit's PV is done, so one buffer suffices, and the epilogue stages its bf16 output there
// too (it runs after the split's last PV).
//
// Tensor memory, lanes at offset 16 (the 64-row layout; O fills the lanes at offset 0):
//   columns   0..143  q_hi (4 e4m3 per column)      144..287  q_lo
//   columns 288..415  the unit's scores (one 128-column buffer, freed as soon as the
//                     softmax warps have loaded it)
// Per unit:
//   TMA: nine 64 x 64-byte boxes per page into the unit's slot.
//   MMA: S = (q_hi + q_lo) . K^T: 2 terms x 18 K-steps of M=64 N=128 (or 64) K=32 into
//        one accumulator; O += (P_hi + P_lo) . V: 2 terms x 2 output halves x 2 K-steps
//        per page of M=64 N=256 K=32, P and V from shared memory.
#include <math.h>
#include <string.h>

#include "mla_scan_common.cuh"

namespace mla {
namespace {

using namespace scan;

constexpr int kSlots = 3;                         // pair slots
constexpr uint32_t kChunk = kTok * 64;            // one page's chunk: 64 tokens x 64 bytes
constexpr uint32_t kPageBytes = 9 * kChunk;       // 36 KB
constexpr uint32_t kChunkPair = 2 * kChunk;       // chunk j of both pages of a slot
constexpr uint32_t kSlotBytes = 9 * kChunkPair;   // 72 KB
constexpr uint32_t kOffKv = 0;
constexpr uint32_t kOffPInSlot = 8 * kChunkPair;             // P_hi over the two rope chunks
// P_lo (two 4 KB halves: the unit's pages), also the epilogue staging (2 KB per softmax warp)
constexpr uint32_t kOffScratch = kOffKv + kSlots * kSlotBytes;
static_assert(4 * kEpiWarpBytes == 2 * kChunk, "P_lo and the epilogue staging share the buffer");
constexpr uint32_t kOffBar = kOffScratch + 2 * kChunk;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;        // barriers + alignment slack
static_assert(kSmemBytes <= (uint32_t)kMaxSmem, "dynamic shared memory limit per block");

enum : int {
    B_KV_FULL0 = 0, B_KV_EMPTY0 = B_KV_FULL0 + kSlots, B_Q_FULL = B_KV_EMPTY0 + kSlots, B_S_FULL, B_S_FREE,
    B_P_READY, B_PV_DONE, B_DRAIN, B_COUNT
};
constexpr uint32_t kOffTmemHolder = kOffBar + 8 * B_COUNT;
constexpr uint32_t kOffAbort = kOffTmemHolder + 4;
static_assert(kOffAbort + 4 <= kOffBar + 256, "barrier area");

constexpr uint32_t kColQhi = 0, kColQlo = 144, kColS = 288;
static_assert(kColS + 2 * kTok <= kTmemCols, "tensor memory columns");
constexpr float kRescaleThreshold = 4.0f;
constexpr float kPOffset = 4.0f;  // P = 2^(x - m + 4)

constexpr uint32_t kIdescS128 = ptx::idesc_e4m3_f32(kRows, 2 * kTok, 0, 0);
constexpr uint32_t kIdescS64 = ptx::idesc_e4m3_f32(kRows, kTok, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_e4m3_f32(kRows, 256, 0, 1);

// Twelve of the 36 score MMAs, starting at U0: term u / 18 (q_hi, q_lo), K-step
// v = u % 18 covering dims [32 v, 32 v + 32): chunk v / 2, 32-byte step v % 2 in the
// 64-byte row.  U0 is a template constant so that every descriptor offset is an immediate.
template <int U0>
__device__ __forceinline__ void issue_s_chunk(uint32_t d, uint32_t a0, uint64_t b0, uint32_t idesc) {
    constexpr uint32_t kPairUnits = kChunkPair >> 4;
#pragma unroll
    for (int k = 0; k < 12; ++k) {
        const int u = U0 + k, v = u % 18;
        ptx::mma_ts_f8(d, a0 + kColQlo * (uint32_t)(u / 18) + 8u * v,
                       b0 + (uint64_t)((v >> 1) * kPairUnits + (v & 1) * 2), idesc, u ? 1u : 0u);
    }
}

// Pages of unit v of a split of n pages: 2, or 1 for an odd last page.
__device__ __forceinline__ int unit_pages(int v, int n) { return min(2, n - 2 * v); }

__global__ void __launch_bounds__(kThreads, 1) decode_e4m3_kernel(const __grid_constant__ Args args) {
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
        for (int s = 0; s < kSlots; ++s) {
            ptx::mbar_init(c.bar(B_KV_FULL0 + s), 1);
            ptx::mbar_init(c.bar(B_KV_EMPTY0 + s), 1);
        }
        ptx::mbar_init(c.bar(B_Q_FULL), 128);
        ptx::mbar_init(c.bar(B_S_FULL), 1);
        ptx::mbar_init(c.bar(B_S_FREE), 128);
        ptx::mbar_init(c.bar(B_P_READY), 128);
        ptx::mbar_init(c.bar(B_PV_DONE), 1);
        ptx::mbar_init(c.bar(B_DRAIN), 1);
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
        // As in the bf16 scan, the warp fetches the block-table entries 32 at a time (one
        // window ahead) and lane 0 issues; here each unit's pages go to one pair slot, whose
        // barrier expects the bytes of all the unit's pages.
        int un = 0;  // units issued by this CTA
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
            const int n = S.tile_end - S.tile_begin;
            int32_t pg = 0, pgn = 0;  // page ids of tiles [t0, t0 + 32) and [t0 + 32, t0 + 64)
            for (int t = S.tile_begin; t < S.tile_end; ++t) {
                const int jt = t - S.tile_begin, j = jt & 31, w = jt & 1;
                if (j == 0) {
                    pg = t == S.tile_begin ? pg_first : pgn;
                    pgn = (t + 32 + lane < S.tile_end) ? bt_row[t + 32 + lane] : 0;
                }
                const int32_t page = __shfl_sync(0xffffffffu, pg, j);
                if (lane == 0) {
                    const int slot = un % kSlots;
                    if (w == 0) {
                        if (un >= kSlots && !wait_bar(c, c.bar(B_KV_EMPTY0 + slot), ((un / kSlots) - 1) & 1))
                            ok = false;
                        else
                            ptx::mbar_arrive_expect_tx(c.bar(B_KV_FULL0 + slot), kPageBytes * unit_pages(jt >> 1, n));
                    }
                    if (ok) {
                        // an invalid page id becomes a box entirely out of range (zero fill);
                        // the softmax warps see the same id and poison the request's rows
                        const int ky = (page >= 0 && page < p.num_pages) ? page * kPage : -kPage;
                        const uint32_t dst = sbase + kOffKv + slot * kSlotBytes + w * kChunk;
#pragma unroll
                        for (int jb = 0; jb < 9; ++jb)
                            ptx::tma_load_2d(dst + jb * kChunkPair, &args.tm_kv, c.bar(B_KV_FULL0 + slot), 64 * jb, ky);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (w == 1 || t == S.tile_end - 1) ++un;
            }
        }
        if (lane == 0 && *c.abort) {
            for (int k = (un > kSlots ? un - kSlots : 0); k < un; ++k)
                drain_wait(c.bar(B_KV_FULL0 + k % kSlots), (k / kSlots) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The score MMAs of the next unit (once its slot is full and the softmax warps have
        // loaded the previous unit's scores) and the PV MMAs of the oldest unit whose P is in
        // TMEM, in whichever order their inputs arrive; the tensor core runs them in issue
        // order.  Barriers are polled with test_wait, which never suspends the thread.
        if (lane == 0) {
            int un = 0, nseg = 0;
            bool ok = true;
            for (int si = seg_lo; si < seg_hi && ok; ++si) {
                const Segment S = si == seg_lo ? gh.first : segs[si];
                const int T = p.seq_lens[S.b];
                if (!request_ok(p, T)) continue;
                if (!wait_bar(c, c.bar(B_Q_FULL), nseg & 1)) break;
                ptx::tc_fence_after();
                const int n = S.tile_end - S.tile_begin, nu = (n + 1) >> 1;
                int ns = 0, npv = 0;  // units of this split with S issued / PV issued
                PollClock clk;
                while (npv < nu) {
                    bool progressed = false;
                    if (ns < nu) {
                        const int us = un + ns, slot = us % kSlots;
                        if (ptx::mbar_test_wait(c.bar(B_KV_FULL0 + slot), (us / kSlots) & 1) &&
                            (us == 0 || ptx::mbar_test_wait(c.bar(B_S_FREE), (us - 1) & 1))) {
                            ptx::tc_fence_after();
                            // descriptors built once and advanced by constant 16-byte offsets
                            const uint64_t b0 = ptx::smem_desc(sbase + kOffKv + slot * kSlotBytes, 16, 512,
                                                               ptx::kSwizzle64);
                            const uint32_t d = tmem + kLaneHi + kColS;
                            const uint32_t a0 = tmem + kLaneHi + kColQhi;
                            const uint32_t idesc = unit_pages(ns, n) == 2 ? kIdescS128 : kIdescS64;
                            issue_s_chunk<0>(d, a0, b0, idesc);
                            issue_s_chunk<12>(d, a0, b0, idesc);
                            issue_s_chunk<24>(d, a0, b0, idesc);
                            ptx::mma_commit(c.bar(B_S_FULL));
                            ++ns;
                            progressed = true;
                        }
                    }
                    if (npv < ns) {
                        const int up = un + npv, slot = up % kSlots;
                        if (ptx::mbar_test_wait(c.bar(B_P_READY), up & 1)) {
                            ptx::tc_fence_after();
                            const bool first = npv == 0;
                            // A = P of page ks / 2 (K-major, 32 tokens = 32 bytes of each 64-byte
                            // row); B = V of page ks / 2, MN-major: 64-column chunks 8 KB apart
                            // (leading offset), 8-token groups 512 bytes apart (stride offset),
                            // 2 KB per 32 tokens
                            const uint32_t slot_a = sbase + kOffKv + slot * kSlotBytes;
                            const uint64_t ph = ptx::smem_desc(slot_a + kOffPInSlot, 16, 512, ptx::kSwizzle64);
                            const uint64_t pl = ptx::smem_desc(sbase + kOffScratch, 16, 512, ptx::kSwizzle64);
                            const uint64_t v0 = ptx::smem_desc(slot_a, kChunkPair, 512, ptx::kSwizzle64);
                            const int nks = 2 * unit_pages(npv, n);
#pragma unroll
                            for (int term = 0; term < 2; ++term)
#pragma unroll
                                for (int half = 0; half < 2; ++half)
#pragma unroll
                                    for (int ks = 0; ks < 4; ++ks)
                                        if (ks < nks)
                                            ptx::mma_ss_f8(tmem + 256u * half,
                                                           (term ? pl : ph) +
                                                               (uint64_t)((ks >> 1) * (kChunk >> 4) + (ks & 1) * 2),
                                                           v0 + (uint64_t)((ks >> 1) * (kChunk >> 4) +
                                                                           half * 4 * (kChunkPair >> 4) +
                                                                           (ks & 1) * (2048 >> 4)),
                                                           kIdescPV, (first && term == 0 && ks == 0) ? 0u : 1u);
                            ptx::mma_commit(c.bar(B_PV_DONE));
                            ptx::mma_commit(c.bar(B_KV_EMPTY0 + slot));
                            ++npv;
                            progressed = true;
                        }
                    }
                    if (!clk.step(c, progressed)) {
                        ok = false;
                        break;
                    }
                }
                un += nu;
                ++nseg;
            }
            ptx::mma_commit(c.bar(B_DRAIN));
            drain_wait(c.bar(B_DRAIN), 0);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        RowSlot r;
        r.quad = warp & 3;   // TMEM lane quadrant this warp may access
        r.r16 = lane & 15;
        r.half = lane >> 4;  // tokens [32 half, +32) of each page of the unit; output columns [32 half + 64 q, +32)
        r.lane = lane;
        r.row = r.quad * 16 + r.r16;
        r.qb = qb;
        r.nqb = nqb;
        r.m_glob = qb * kRows + r.row;
        r.row_valid = r.m_glob < p.M;
        const int half = r.half;
        const uint32_t t_hi = tmem + ((uint32_t)(r.quad * 32) << 16) + kLaneHi;  // q, scores, P
        const uint32_t t_lo = tmem + ((uint32_t)(r.quad * 32) << 16);            // O
        const int tid = threadIdx.x - 64;  // 0..127
        const uint16_t* qsrc = reinterpret_cast<const uint16_t*>(p.q);
        float* plse = ws_ptr<float>(p.ws, h->off_plse);
        float* po = ws_ptr<float>(p.ws, h->off_po);
        int un = 0;
        bool alive = true;

        for (int si = seg_lo; si < seg_hi; ++si) {
            const Segment S = si == seg_lo ? gh.first : segs[si];
            const int T = p.seq_lens[S.b];
            if (!request_ok(p, T)) {
                if (tid == 0) set_status(h, kStatusOob, S.b);
                poison_rows(p, S, si, r, po, plse);
                continue;
            }
            if (*c.abort) break;
            // q: thread (row, half) holds dims [64 k + 32 half, +32), k = 0..8.  First pass: the
            // row's max |q| (both halves) from one batch of 36 16-byte loads; second pass: each
            // 32-dim block loaded again (an L1 hit) and cut into its two e4m3 terms, so that the
            // loaded row and its terms are never live together.
            float row_scale = 0.f;
            {
                const uint4* src = reinterpret_cast<const uint4*>(qsrc + ((int64_t)S.b * p.M + r.m_glob) * kDqk);
                float amax = 0.f;
                {
                    uint4 x[9][4];
#pragma unroll
                    for (int k = 0; k < 9; ++k)
#pragma unroll
                        for (int w = 0; w < 4; ++w)
                            x[k][w] = r.row_valid ? src[(64 * k + 32 * half) / 8 + w] : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int k = 0; k < 9; ++k)
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const uint32_t v4[4] = {x[k][w].x, x[k][w].y, x[k][w].z, x[k][w].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(v4[e] << 16)),
                                                         fabsf(__uint_as_float(v4[e] & 0xffff0000u))));
                        }
                }
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
                float inv = 0.f;
                if (amax > 0.f) {
                    int e;
                    const float f = frexpf(amax, &e);  // amax = f 2^e, f in [0.5, 1)
                    const int k = min(127, max(-126, (f <= 0.875f ? 9 : 8) - e));  // max|q| 2^k <= 448
                    inv = ldexpf(1.f, k);
                    row_scale = ldexpf(1.f, -k);
                }
#pragma unroll 1
                for (int k = 0; k < 9; ++k) {
                    uint4 y[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        y[w] = r.row_valid ? src[(64 * k + 32 * half) / 8 + w] : make_uint4(0, 0, 0, 0);
                    uint32_t hi[8], lo[8];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t v4[4] = {y[w].x, y[w].y, y[w].z, y[w].w};
#pragma unroll
                        for (int e = 0; e < 4; e += 2)
                            split_e4m3x4(__uint_as_float(v4[e] << 16) * inv, __uint_as_float(v4[e] & 0xffff0000u) * inv,
                                         __uint_as_float(v4[e + 1] << 16) * inv,
                                         __uint_as_float(v4[e + 1] & 0xffff0000u) * inv, hi[2 * w + e / 2],
                                         lo[2 * w + e / 2]);
                    }
                    ptx::tmem_st16x8<8>(t_hi + kColQhi + 16u * k, hi);
                    ptx::tmem_st16x8<8>(t_hi + kColQlo + 16u * k, lo);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(c.bar(B_Q_FULL));
            }
            const int last_t = p.causal ? T - p.s_q + r.m_glob / p.H : T - 1;
            const int full_end = p.causal ? T - p.s_q + 1 : T;  // tokens < full_end are visible to every row
            const int ntiles_req = (T + kPage - 1) / kPage;
            const int n = S.tile_end - S.tile_begin, nu = (n + 1) >> 1;
            const float sc = p.score_scale_log2 * row_scale;
            float m_run = -INFINITY, l = 0.f;
            bool badpage = false;
            for (int v = 0; v < nu; ++v, ++un) {
                const int t0 = S.tile_begin + 2 * v, npg = unit_pages(v, n);
                const int32_t* bt = p.block_table + (int64_t)S.b * p.max_pages + t0;
                for (int w = 0; w < npg; ++w) badpage |= !(bt[w] >= 0 && bt[w] < p.num_pages);
                alive = wait_bar(c, c.bar(B_S_FULL), un & 1);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                ptx::tc_fence_after();
                // thread half h: tokens [32 h, +32) of the unit's page 0 (sa) and of page 1 (sb)
                uint32_t sa[32], sb[32];
                ptx::tmem_ld16x32<32>(t_hi + kColS, sa);
                ptx::tmem_ld16x32<32>(t_hi + kColS + kTok, sb);
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                ptx::mbar_arrive(c.bar(B_S_FREE));  // the next unit's scores may overwrite the buffer
                float s[64];
                const int tok0 = t0 * kPage + 32 * half;  // s[k]: token tok0 + k (k < 32), tok0 + 32 + k (k >= 32)
                if ((t0 + npg) * kPage <= full_end) {
#pragma unroll
                    for (int k = 0; k < 64; ++k)
                        s[k] = (k < 32 || npg == 2) ? __uint_as_float(k < 32 ? sa[k] : sb[k - 32]) * sc : -INFINITY;
                } else {
#pragma unroll
                    for (int k = 0; k < 64; ++k) {
                        const int t = tok0 + k + (k < 32 ? 0 : 32);
                        s[k] = ((k < 32 || npg == 2) && t < T && t <= last_t)
                                   ? __uint_as_float(k < 32 ? sa[k] : sb[k - 32]) * sc
                                   : -INFINITY;
                    }
                }
                float mx[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    mx[k] = fmaxf(fmaxf(s[8 * k], s[8 * k + 1]), fmaxf(s[8 * k + 2], s[8 * k + 3]));
                    mx[k] = fmaxf(mx[k], fmaxf(fmaxf(s[8 * k + 4], s[8 * k + 5]), fmaxf(s[8 * k + 6], s[8 * k + 7])));
                }
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
                const bool need_o = raise && v > 0 && m_run != -INFINITY;
                if (raise) m_run = mt;
                // The previous unit's PV must be done before O is rescaled or P_lo overwritten
                // (the first unit of a split follows the previous split's epilogue, which waited
                // for its last PV).
                if (v > 0) {
                    alive = wait_bar(c, c.bar(B_PV_DONE), (un - 1) & 1);
                    if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                    ptx::tc_fence_after();
                }
                if (__any_sync(0xffffffffu, need_o)) rescale_o(t_lo, need_o ? alpha : 1.f);
                const bool live = m_run != -INFINITY;
                const float mo = m_run - kPOffset;
                float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    s[k] = live ? fast_exp2(s[k] - mo) : 0.f;  // P
                    rs[k & 3] += s[k];
                }
                l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
                const int tl = t0 + npg - 1;  // the unit's last page
                if (tl == ntiles_req - 1 && (T % kPage) != 0) {
                    // rows past the request's end hold stale data (maybe NaN): zero their latent
                    // columns before the PV product reads them with P = 0
                    const int slot = un % kSlots;
                    alive = wait_bar(c, c.bar(B_KV_FULL0 + slot), (un / kSlots) & 1);
                    if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                    uint8_t* pg = smem + kOffKv + slot * kSlotBytes + (npg - 1) * kChunk;
                    const int r0 = T % kPage;
                    const int pieces = (kPage - r0) * 8 * 4;  // rows x latent chunks x 16-byte pieces
                    for (int q = tid; q < pieces; q += 128) {
                        const int rr = r0 + q / 32, j = (q / 4) % 8, w = q % 4;
                        *reinterpret_cast<uint4*>(pg + j * kChunkPair + rr * 64 + w * 16) = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                {
                    // P_hi over the slot's rope chunks, P_lo into the buffer: row `row`, tokens
                    // [32 half, +32) of each page, two 16-byte pieces of the 64-byte K-major row,
                    // 64-byte swizzle (piece c of row r at (c ^ ((r >> 1) & 3)) * 16)
                    uint8_t* ph = smem + kOffKv + (un % kSlots) * kSlotBytes + kOffPInSlot + r.row * 64;
                    uint8_t* pl = smem + kOffScratch + r.row * 64;
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        uint32_t hi[8], lo[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            split_e4m3x4(s[32 * w + 4 * k], s[32 * w + 4 * k + 1], s[32 * w + 4 * k + 2],
                                         s[32 * w + 4 * k + 3], hi[k], lo[k]);
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const int off = w * kChunk + (((2 * half + i) ^ ((r.row >> 1) & 3)) << 4);
                            *reinterpret_cast<uint4*>(ph + off) = make_uint4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
                            *reinterpret_cast<uint4*>(pl + off) = make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]);
                        }
                    }
                }
                ptx::fence_proxy_async_smem();  // P and the zeroed rows above, for the PV MMAs
                ptx::tc_fence_before();
                ptx::mbar_arrive(c.bar(B_P_READY));
            }
            if (!alive || *c.abort) break;
            // epilogue: wait for the last PV of the split; the row sum is the two halves' sum
            alive = wait_bar(c, c.bar(B_PV_DONE), (un - 1) & 1);
            if (__any_sync(0xffffffffu, !alive)) break;
            ptx::tc_fence_after();
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            if (badpage && tid == 0) set_status(h, kStatusOob, S.b);
            const float nanv = __int_as_float(0x7fc00000);
            const float inv = badpage ? nanv : (l > 0.f ? p.out_scale / l : 0.f);
            const float lse2 = badpage ? nanv : (l > 0.f ? m_run - kPOffset + __log2f(l) : -INFINITY);
            store_split(p, S, si, r, t_lo, smem + kOffScratch + (warp - 2) * kEpiWarpBytes, inv, lse2, po, plse);
            // the next split's q overwrites TMEM only after this epilogue's reads (same threads)
            ptx::tc_fence_before();
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
}

struct TmapCacheEntry {
    int dev = -1;
    const void* kv = nullptr;
    int64_t num_pages = -1;
    CUtensorMap map;
};

// As for the bf16 scan: the last tensor map each host thread encoded is reused while the
// device, cache pointer and page count match.
bool cached_kv_map(int dev, const DecodeParams& p, CUtensorMap* out) {
    static thread_local TmapCacheEntry e;
    if (e.dev != dev || e.kv != p.kv || e.num_pages != p.num_pages) {
        const uint64_t kvrows = (uint64_t)p.num_pages * kPage;
        if (!make_map_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.kv, kDqk, kvrows, kDqk, 64, kTok,
                         CU_TENSOR_MAP_SWIZZLE_64B)) {
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

bool smem_attribute_set(int dev) {
    static int done[64] = {};
    if (dev < 64 && done[dev]) return true;
    if (cudaFuncSetAttribute(decode_e4m3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
        return false;
    if (dev < 64) done[dev] = 1;
    return true;
}

}  // namespace

mla_status launch_decode_e4m3(const DecodeParams& p, cudaStream_t stream) {
    Args a;
    memset(&a, 0, sizeof(a));
    a.p = p;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (!cached_kv_map(dev, p, &a.tm_kv)) return MLA_ERR_CUDA;
    if (!smem_attribute_set(dev)) return MLA_ERR_CUDA;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(p.groups_launched * num_row_blocks(p.s_q, p.H));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_e4m3_kernel, a) != cudaSuccess) return MLA_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla
