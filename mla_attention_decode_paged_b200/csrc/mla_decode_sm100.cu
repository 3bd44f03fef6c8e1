// mla_decode_sm100.cu -- the split scan of paged absorbed-MLA decode on Blackwell
// tensor cores (tcgen05 + TMEM + TMA), sm_100a.
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
//   lanes at offset 16 : q (loaded once per split: 64 x 576 bf16, or for an e4m3 cache
//                        two e4m3 terms of 64 x 576; 288 columns either way) and two
//                        64-column score buffers.
// Per page, bf16 cache (kind::f16 MMAs):
//   TMA (producer warp): the page's 64 rows x 576 columns as nine 64-column boxes with
//       128-byte swizzle (one 72 KB stage; three stages).
//   MMA (one thread): S = q . K^T with q read from TMEM (M=64 N=64 K=16, 36 K-steps),
//       then O += P . V with P (bf16) and V (the same page, read MN-major) from shared
//       memory (M=64 N=256 K=16, twice, 4 K-steps each).
// Per page, e4m3 cache (kind::f8f6f4 MMAs, both operands e4m3: the cache bytes are read
//   by the tensor cores as they are, with kv_scale folded into the score and output
//   scales):
//   TMA: nine 64 x 64-byte boxes with 64-byte swizzle (one 36 KB stage; six stages).
//   MMA: S = (q_hi + q_lo) . K^T, two chains of 18 K-steps (M=64 N=64 K=32) into one
//       accumulator, where per row q_hi = e4m3(q / s_r), q_lo = e4m3(q / s_r - q_hi) and
//       s_r is the smallest power of two with max|q_r| / s_r <= 448: q / s_r is then still
//       a bf16 value, whose 8 significant bits the two 4-bit terms hold exactly (bar
//       e4m3's subnormal range), so the scores are those of the bf16 q.  Then
//       O += (P_hi + P_lo) . V with P_hi = e4m3(P), P_lo = e4m3(P - P_hi) (M=64 N=256 K=32:
//       2 terms x 2 halves x 2 K-steps), P to 8 significant bits as a bf16 P would be.
//       One e4m3 term of q moves lse past 1e-3, and one of P moves short rows past the
//       relative L2 bound.
// Either way P is written over the page's rope chunk (the e4m3 P_lo into a two-entry
// ring), which only the score MMAs read: every stage carries its own P, and the softmax
// of a page never waits for the previous page's PV.
//   softmax (4 warps, 16 rows each, two threads per row with 32 scores each): base-2
//       online softmax with the causal draft mask; the running max is only raised (and
//       O rescaled) when a score exceeds it by more than 8 (bf16) or 4 (e4m3), and the
//       e4m3 P is 2^(x - m + 4): P <= 256 < 448, with the bulk of a long near-uniform row
//       far above e4m3's subnormal floor.
//   epilogue: O / l -> bf16 out (a request the split holds whole) or an fp32 partial and
//       its base-2 lse (split request; merged by the combine kernel).
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "mla_decode_params.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr int kRows = kRowsPerBlock;  // 64 folded rows per CTA (MMA M)
constexpr int kTok = 64;              // tokens per page (S MMA N)
// warp 0 TMA, warp 1 MMA, warps 2-5 softmax / epilogue
constexpr int kThreads = 192;
static_assert(kRows == 64, "the TMEM layout below is the 64-row MMA layout");

// Shared-memory geometry per cache type.  A chunk is 64 tokens x 64 columns of one page,
// 8-row swizzle atoms; a stage holds one page (8 latent chunks + the rope chunk).
template <int KV>
struct Geo;
template <>
struct Geo<MLA_KV_BF16> {
    static constexpr int kStages = 3;
    static constexpr uint32_t kChunk = kTok * 128;   // 128-byte rows, 128-byte swizzle
    static constexpr uint32_t kSbo = 8 * 128;
    static constexpr uint32_t kSwizzle = ptx::kSwizzle128;
    static constexpr float kRescale = 8.f;           // raise the running max past this margin
    static constexpr float kPOffset = 0.f;           // P = 2^(x - m + offset)
};
template <>
struct Geo<MLA_KV_E4M3> {
    static constexpr int kStages = 6;
    static constexpr uint32_t kChunk = kTok * 64;    // 64-byte rows, 64-byte swizzle
    static constexpr uint32_t kSbo = 8 * 64;
    static constexpr uint32_t kSwizzle = ptx::kSwizzle64;
    static constexpr float kRescale = 4.f;
    static constexpr float kPOffset = 4.f;
};
constexpr int kMaxStages = 6;
template <int KV>
constexpr uint32_t stage_bytes() { return 9 * Geo<KV>::kChunk; }

constexpr uint32_t kOffKv = 0;
// after the stages (221,184 B for either cache type): 8 KB of scratch, the epilogue
// staging (2 KB per softmax warp) and, for e4m3, the two-entry P_lo ring (4 KB each),
// which is never in use while a warp stages its epilogue (that waits for the split's
// last PV; the next split's P is written by the same threads afterwards)
constexpr uint32_t kOffScratch = 3 * 9 * 8192;
static_assert(Geo<MLA_KV_BF16>::kStages * stage_bytes<MLA_KV_BF16>() == kOffScratch, "bf16 stages");
static_assert(Geo<MLA_KV_E4M3>::kStages * stage_bytes<MLA_KV_E4M3>() == kOffScratch, "e4m3 stages");
constexpr uint32_t kEpiWarpBytes = 16 * 128;
constexpr uint32_t kOffBar = kOffScratch + 8192;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
static_assert(kSmemBytes <= 232448, "dynamic shared memory limit per block");
static_assert(kRows * kTok * 2 == Geo<MLA_KV_BF16>::kChunk, "bf16 P fills the rope chunk exactly");
static_assert(kRows * kTok == Geo<MLA_KV_E4M3>::kChunk, "e4m3 P_hi fills the rope chunk exactly");

enum : int {
    B_KV_FULL0 = 0, B_KV_EMPTY0 = B_KV_FULL0 + kMaxStages, B_Q_FULL = B_KV_EMPTY0 + kMaxStages, B_S_FULL0,
    B_P_READY0 = B_S_FULL0 + 2, B_PV_DONE0 = B_P_READY0 + 2, B_DRAIN = B_PV_DONE0 + 2, B_COUNT
};
constexpr uint32_t kOffTmemHolder = kOffBar + 8 * B_COUNT;
constexpr uint32_t kOffAbort = kOffTmemHolder + 4;
static_assert(kOffAbort + 4 <= kOffBar + 256, "barrier area");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kLaneHi = 16u << 16;  // second half-subpartition set (q and scores)
constexpr uint32_t kColQ = 0;            // q: 288 columns (bf16 pairs, or e4m3 q_hi | q_lo quads)
constexpr uint32_t kColQlo = 144;        // e4m3 q_lo
constexpr uint32_t kColS = 288;          // scores: 2 x 64 columns
constexpr uint64_t kWaitLimitNs = 2000000000ull;

template <int KV>
constexpr uint32_t idesc_s() {
    return KV == MLA_KV_E4M3 ? ptx::idesc_e4m3_f32(kRows, kTok, 0, 0) : ptx::idesc_bf16_f32(kRows, kTok, 0, 0);
}
template <int KV>
constexpr uint32_t idesc_pv() {
    return KV == MLA_KV_E4M3 ? ptx::idesc_e4m3_f32(kRows, 256, 0, 1) : ptx::idesc_bf16_f32(kRows, 256, 0, 1);
}

struct __align__(64) Sm100Args {
    CUtensorMap tm_kv;  // cache viewed [P*64 rows, 576 cols]: bf16 box 64 x 64 with 128B swizzle, or
                        // e4m3 box 64 x 64 bytes with 64B swizzle
    DecodeParams p;
};

struct Ctx {
    uint32_t bar0;
    volatile int* abort;
    PlanHeader* h;
    __device__ uint32_t bar(int i) const { return bar0 + 8u * (uint32_t)i; }
};

// Bounded wait: gives up after kWaitLimitNs (sets the timeout status and the CTA abort
// flag), or at once once the CTA is aborting.
template <uint64_t kLimitNs>
__device__ __noinline__ bool wait_bar_for(const Ctx& c, uint32_t bar, uint32_t parity) {
    if (*c.abort) return false;
    uint64_t t0 = 0;
    for (uint32_t n = 1;; ++n) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((n & 255) == 0) {
            if (*c.abort) return false;
            const uint64_t now = ptx::globaltimer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kLimitNs) {
                *c.abort = 1;
                set_status(c.h, kStatusTimeout, (int)blockIdx.x);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar(const Ctx& c, uint32_t bar, uint32_t parity) {
    return wait_bar_for<kWaitLimitNs>(c, bar, parity);
}

// Wait that ignores the abort flag, used only on the way out for work already in flight.
__device__ void drain_wait(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > 200000000ull) return;
    }
}

__device__ __forceinline__ bool request_ok(const DecodeParams& p, int T) {
    return T >= 1 && (int64_t)T <= (int64_t)p.max_pages * kPage && !(p.causal && T < p.s_q);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Four floats -> (e4m3 word of x, e4m3 word of the residual x - e4m3(x)), bytes in order.
__device__ __forceinline__ void split_e4m3x4(float x0, float x1, float x2, float x3, uint32_t& hi, uint32_t& lo) {
    const uint16_t h01 = ptx::f32x2_to_e4m3x2(x0, x1), h23 = ptx::f32x2_to_e4m3x2(x2, x3);
    const float2 f01 = e4m3x2_to_float2(h01), f23 = e4m3x2_to_float2(h23);
    hi = (uint32_t)h01 | ((uint32_t)h23 << 16);
    lo = (uint32_t)ptx::f32x2_to_e4m3x2(x0 - f01.x, x1 - f01.y) |
         ((uint32_t)ptx::f32x2_to_e4m3x2(x2 - f23.x, x3 - f23.y) << 16);
}

// Twelve of the 36 score MMAs, starting at U0: q from TMEM, the page from shared memory.
// U0 is a template constant so that every descriptor offset is an immediate.
//   bf16: K-step u covers dims [16u, 16u + 16): chunk u / 4, 32-byte step u % 4 in the row.
//   e4m3: term u / 18 (q_hi, q_lo), K-step v = u % 18 covers dims [32v, 32v + 32): chunk
//         v / 2, 32-byte step v % 2 in the 64-byte row; q_lo starts 144 columns on.
template <int KV, int U0>
__device__ __forceinline__ void issue_s_chunk(uint32_t d, uint32_t a0, uint64_t b0) {
    constexpr uint32_t kChunkUnits = Geo<KV>::kChunk >> 4;
#pragma unroll
    for (int k = 0; k < 12; ++k) {
        const int u = U0 + k;
        if constexpr (KV == MLA_KV_E4M3) {
            const int v = u % 18;
            ptx::mma_ts_f8(d, a0 + kColQlo * (uint32_t)(u / 18) + 8u * v,
                           b0 + (uint64_t)((v >> 1) * kChunkUnits + (v & 1) * 2), idesc_s<KV>(), u ? 1u : 0u);
        } else {
            ptx::mma_ts(d, a0 + 8u * u, b0 + (uint64_t)((u >> 2) * kChunkUnits + (u & 3) * 2), idesc_s<KV>(),
                        u ? 1u : 0u);
        }
    }
}

template <int KV>
__global__ void __launch_bounds__(kThreads, 1) decode_sm100_kernel(const __grid_constant__ Sm100Args args) {
    constexpr bool kE4m3 = KV == MLA_KV_E4M3;
    constexpr int kStages = Geo<KV>::kStages;
    constexpr uint32_t kChunk = Geo<KV>::kChunk;
    constexpr uint32_t kStageBytes = stage_bytes<KV>();
    constexpr uint32_t kOffPInStage = 8 * kChunk;  // P (or P_hi) over the rope chunk
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const DecodeParams& p = args.p;
    PlanHeader* h = reinterpret_cast<PlanHeader*>(p.ws);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the combine may start its prologue now; it waits for this grid before reading
    ptx::griddep_launch_dependents();

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
    const bool plan_ok = h->magic == kPlanMagic && h->B == p.B && h->s_q == p.s_q && h->H == p.H &&
                         h->num_groups <= p.groups_launched;
    const int nqb = plan_ok ? h->nqb : 1;
    const int g = blockIdx.x / nqb, qb = blockIdx.x % nqb;
    if (!plan_ok || g >= h->num_groups) {
        if (!plan_ok && blockIdx.x == 0 && threadIdx.x == 0) set_status(h, kStatusPlanMismatch, 0);
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
        if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
        return;
    }

    const int32_t* group_begin = ws_ptr<int32_t>(p.ws, h->off_group_begin);
    const Segment* segs = ws_ptr<Segment>(p.ws, h->off_segs);
    const int seg_lo = group_begin[g], seg_hi = group_begin[g + 1];

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp walks the tiles; every 32 tiles each lane fetches one block-table
        // entry (one window ahead), so the page ids reach lane 0 (which waits and issues) by
        // shuffles instead of one dependent global load per page.
        int it = 0;
        bool ok = true;
        for (int si = seg_lo; si < seg_hi && ok; ++si) {
            if (__shfl_sync(0xffffffffu, lane == 0 ? *c.abort : 0, 0)) break;
            const Segment S = segs[si];
            const int T = p.seq_lens[S.b];
            if (!request_ok(p, T)) continue;
            const int32_t* bt_row = p.block_table + (int64_t)S.b * p.max_pages;
            int32_t pg = 0, pgn = 0;  // page ids of tiles [t0, t0 + 32) and [t0 + 32, t0 + 64)
            for (int t = S.tile_begin; t < S.tile_end; ++t, ++it) {
                const int j = (t - S.tile_begin) & 31;
                if (j == 0) {
                    pg = t == S.tile_begin ? ((t + lane < S.tile_end) ? bt_row[t + lane] : 0) : pgn;
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
        // An event loop: the score MMAs of the next page and the PV MMAs of the oldest
        // page whose P is ready are issued in whichever order their inputs arrive.  The
        // tensor core runs them in issue order.  Barriers are polled with test_wait, which
        // never suspends the thread.
        if (lane == 0) {
            int it = 0, nseg = 0;
            bool ok = true;
            for (int si = seg_lo; si < seg_hi && ok; ++si) {
                const Segment S = segs[si];
                const int T = p.seq_lens[S.b];
                if (!request_ok(p, T)) continue;
                if (!wait_bar(c, c.bar(B_Q_FULL), nseg & 1)) break;
                ptx::tc_fence_after();
                const int n = S.tile_end - S.tile_begin;
                int ns = 0, npv = 0;  // pages of this split with S issued / PV issued
                uint64_t t0 = 0;
                uint32_t spins = 0;
                while (npv < n) {
                    bool progressed = false;
                    // S(ns) reuses the score buffer of page ns-2, whose PV must be issued first.
                    // A score chain is issued whole: PV MMAs placed between its K-steps (another
                    // accumulator) slow the chain down far more than they gain.
                    if (ns < n && ns <= npv + 1) {
                        const int its = it + ns, st = its % kStages;
                        if (ptx::mbar_test_wait(c.bar(B_KV_FULL0 + st), (its / kStages) & 1)) {
                            ptx::tc_fence_after();
                            // descriptors are built once and advanced by constant 16-byte offsets:
                            // the fully unrolled issue loop is a handful of integer adds per MMA
                            const uint64_t b0 = ptx::smem_desc(sbase + kOffKv + st * kStageBytes, 16, Geo<KV>::kSbo,
                                                               Geo<KV>::kSwizzle);
                            const uint32_t d = tmem + kLaneHi + kColS + 64u * (its & 1);
                            const uint32_t a0 = tmem + kLaneHi + kColQ;
                            issue_s_chunk<KV, 0>(d, a0, b0);
                            issue_s_chunk<KV, 12>(d, a0, b0);
                            issue_s_chunk<KV, 24>(d, a0, b0);
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
                            // A = P (K-major); B = V, MN-major: 64-column chunks one chunk apart
                            // (leading offset), 8-token groups one swizzle atom apart (stride offset)
                            const uint32_t stage = sbase + kOffKv + (itp % kStages) * kStageBytes;
                            const uint64_t v0 = ptx::smem_desc(stage, kChunk, Geo<KV>::kSbo, Geo<KV>::kSwizzle);
                            if constexpr (kE4m3) {
                                const uint64_t ph = ptx::smem_desc(stage + kOffPInStage, 16, 512, ptx::kSwizzle64);
                                const uint64_t pl =
                                    ptx::smem_desc(sbase + kOffScratch + 4096u * (itp & 1), 16, 512, ptx::kSwizzle64);
#pragma unroll
                                for (int term = 0; term < 2; ++term)
#pragma unroll
                                    for (int half = 0; half < 2; ++half)
#pragma unroll
                                        for (int ks = 0; ks < 2; ++ks)  // 32 tokens: 32 bytes of P, 2 KB of V
                                            ptx::mma_ss_f8(tmem + 256u * half, (term ? pl : ph) + (uint64_t)(ks * 2),
                                                           v0 + (uint64_t)(half * 4 * (kChunk >> 4) + ks * (2048 >> 4)),
                                                           idesc_pv<KV>(), (first && term == 0 && ks == 0) ? 0u : 1u);
                            } else {
                                const uint64_t a0 = ptx::smem_desc(stage + kOffPInStage, 16, 1024, ptx::kSwizzle128);
#pragma unroll
                                for (int half = 0; half < 2; ++half) {
#pragma unroll
                                    for (int ks = 0; ks < 4; ++ks)  // 16 tokens: 32 bytes of P, 2 KB of V
                                        ptx::mma_ss(tmem + 256u * half, a0 + (uint64_t)(ks * 2),
                                                    v0 + (uint64_t)(half * 4 * (kChunk >> 4) + ks * (2048 >> 4)),
                                                    idesc_pv<KV>(), (first && ks == 0) ? 0u : 1u);
                                }
                            }
                            ptx::mma_commit(c.bar(B_PV_DONE0 + (itp & 1)));
                            ptx::mma_commit(c.bar(B_KV_EMPTY0 + (itp % kStages)));
                            ++npv;
                            progressed = true;
                        }
                    }
                    if (progressed) {
                        t0 = 0;
                        spins = 0;
                    } else if ((++spins & 255) == 0) {
                        // same bound as every other wait in this kernel
                        if (*c.abort) { ok = false; break; }
                        const uint64_t now = ptx::globaltimer_ns();
                        if (t0 == 0) {
                            t0 = now;
                        } else if (now - t0 > kWaitLimitNs) {
                            *c.abort = 1;
                            set_status(h, kStatusTimeout, (int)blockIdx.x);
                            ok = false;
                            break;
                        }
                    }
                }
                it += n;
                ++nseg;
            }
            ptx::mma_commit(c.bar(B_DRAIN));
            drain_wait(c.bar(B_DRAIN), 0);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quad = warp & 3;             // TMEM lane quadrant this warp may access
        const int r16 = lane & 15;
        const int half = lane >> 4;            // score columns [32 half, +32), output columns [32 half + 64 q, +32)
        const int row = quad * 16 + r16;       // folded row within the block
        const uint32_t t_hi = tmem + ((uint32_t)(quad * 32) << 16) + kLaneHi;  // q and scores
        const uint32_t t_lo = tmem + ((uint32_t)(quad * 32) << 16);            // O
        const int tid = threadIdx.x - 64;      // 0..127
        const int m_glob = qb * kRows + row;
        const bool row_valid = m_glob < p.M;
        const uint16_t* qsrc = reinterpret_cast<const uint16_t*>(p.q);
        float* plse = ws_ptr<float>(p.ws, h->off_plse);
        float* po = ws_ptr<float>(p.ws, h->off_po);
        int it = 0;
        bool alive = true;

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
                        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + orow * kDv + 256 * half;
                        for (int k = 0; k < 256; ++k) dst[k] = __float2bfloat16_rn(nanv);
                        if (half == 0) p.lse[orow] = nanv;
                    } else {
                        // the row's columns [256 half, +256) in the quad-interleaved partial layout
                        float* blk = po + ((int64_t)si * nqb + qb) * kRows * kDv + (row >> 4) * 8192 + (row & 15) * 4;
                        for (int k = 0; k < 256; ++k) {
                            const int col = 256 * half + k;
                            blk[(col >> 2) * 64 + (col & 3)] = nanv;
                        }
                        if (half == 0) plse[prow] = nanv;
                    }
                }
                continue;
            }
            if (*c.abort) break;
            // q rows of this block into TMEM.  Thread (row, half) holds dims [64 k + 32 half,
            // +32) for k = 0..8, loaded in one batch of 36 16-byte loads (all issued before the
            // first is used: at a split's start the memory system is full of the first pages'
            // loads, and every dependent round trip here delays the first score MMA).
            // For an e4m3 cache the row is cut into two e4m3 terms at one per-row scale
            // s_r = max|q_r| / 448, which multiplies the row's scores.
            float row_scale = 1.f;
            {
                const uint4* src = reinterpret_cast<const uint4*>(qsrc + ((int64_t)S.b * p.M + m_glob) * kDqk);
                uint4 x[9][4];
#pragma unroll
                for (int k = 0; k < 9; ++k)
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        x[k][w] = row_valid ? src[(64 * k + 32 * half) / 8 + w] : make_uint4(0, 0, 0, 0);
                if constexpr (kE4m3) {
                    // first pass: the row's max |q| (both halves); second pass: each 32-dim
                    // block loaded again (an L1 hit) and split into its two e4m3 terms, so that
                    // the loaded row and its terms are never live together
                    float amax = 0.f;
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
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
                    // the largest power of two 2^k with max|q| 2^k <= 448: q 2^k is still a
                    // bf16 value (8 significant bits), which the two e4m3 terms (4 + 4 bits)
                    // hold exactly unless it is small enough for e4m3's subnormal range
                    float inv = 0.f;
                    row_scale = 0.f;
                    if (amax > 0.f) {
                        int e;
                        const float f = frexpf(amax, &e);  // amax = f 2^e, f in [0.5, 1)
                        const int k = min(127, max(-126, (f <= 0.875f ? 9 : 8) - e));
                        inv = ldexpf(1.f, k);
                        row_scale = ldexpf(1.f, -k);
                    }
#pragma unroll 1
                    for (int k = 0; k < 9; ++k) {
                        uint4 y[4];
#pragma unroll
                        for (int w = 0; w < 4; ++w)
                            y[w] = row_valid ? src[(64 * k + 32 * half) / 8 + w] : make_uint4(0, 0, 0, 0);
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
                        ptx::tmem_st16x8<8>(t_hi + kColQ + 16u * k, hi);
                        ptx::tmem_st16x8<8>(t_hi + kColQlo + 16u * k, lo);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 9; ++k) {
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
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(c.bar(B_Q_FULL));
            }
            const int last_t = p.causal ? T - p.s_q + m_glob / p.H : T - 1;
            const int full_end = p.causal ? T - p.s_q + 1 : T;  // tokens < full_end are visible to every row
            const int ntiles_req = (T + kPage - 1) / kPage;
            const int n = S.tile_end - S.tile_begin;
            const float sc = p.score_scale_log2 * row_scale;
            float m_run = -INFINITY, l = 0.f;
            bool badpage = false;
            for (int jj = 0; jj < n; ++jj, ++it) {
                const int tile = S.tile_begin + jj;
                const int32_t page = p.block_table[(int64_t)S.b * p.max_pages + tile];
                badpage |= !(page >= 0 && page < p.num_pages);
                alive = wait_bar(c, c.bar(B_S_FULL0 + (it & 1)), (it >> 1) & 1);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                ptx::tc_fence_after();
                uint32_t sr[32];
                ptx::tmem_ld16x32<32>(t_hi + kColS + 64u * (it & 1), sr);
                ptx::tmem_wait_ld();
                float s[32];
                const int tok0 = tile * kPage + 32 * half;
                if (tile * kPage + kPage <= full_end) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(sr[k]) * sc;
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int t = tok0 + k;
                        s[k] = (t < T && t <= last_t) ? __uint_as_float(sr[k]) * sc : -INFINITY;
                    }
                }
                float mx[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mx[k] = fmaxf(fmaxf(s[4 * k], s[4 * k + 1]), fmaxf(s[4 * k + 2], s[4 * k + 3]));
#pragma unroll
                for (int k = 0; k < 4; ++k) mx[k] = fmaxf(mx[k], mx[k + 4]);
                float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                const bool raise = mt > m_run + Geo<KV>::kRescale;
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
                    const float f = need_o ? alpha : 1.f;
#pragma unroll 1
                    for (int q = 0; q < 8; ++q) {
                        uint32_t o[32];
                        ptx::tmem_ld16x32<32>(t_lo + 64u * q, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
                        ptx::tmem_st16x32<32>(t_lo + 64u * q, o);
                    }
                    ptx::tmem_wait_st();
                }
                const bool live = m_run != -INFINITY;
                const float mo = m_run - Geo<KV>::kPOffset;  // P = 2^(x - m + offset)
                float pv[32];
                float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    pv[k] = live ? fast_exp2(s[k] - mo) : 0.f;
                    rs[(k >> 1) & 3] += pv[k];
                }
                l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
                uint8_t* stage_p = smem + kOffKv + (it % kStages) * kStageBytes;
                if (tile == ntiles_req - 1 && (T % kPage) != 0) {
                    // rows past the request's end hold stale data (maybe NaN): zero their
                    // latent columns before the PV product reads them with P = 0
                    alive = wait_bar(c, c.bar(B_KV_FULL0 + it % kStages), (it / kStages) & 1);
                    if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                    const int r0 = T % kPage;
                    constexpr int kPieces = (int)(kChunk / kTok / 16);  // 16-byte pieces per chunk row
                    const int pieces = (kPage - r0) * 8 * kPieces;      // rows x latent chunks x pieces
                    for (int q = tid; q < pieces; q += 128) {
                        const int r = r0 + q / (8 * kPieces), j = (q / kPieces) % 8, w = q % kPieces;
                        *reinterpret_cast<uint4*>(stage_p + j * kChunk + r * (kChunk / kTok) + w * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                if constexpr (kE4m3) {
                    // P_hi over the rope chunk, P_lo into the ring: row `row`, tokens [32 half,
                    // +32): two 16-byte pieces of the 64-byte K-major row, 64-byte swizzle
                    // (piece c of row r at (c ^ ((r >> 1) & 3)) * 16)
                    uint32_t hi[8], lo[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        split_e4m3x4(pv[4 * k], pv[4 * k + 1], pv[4 * k + 2], pv[4 * k + 3], hi[k], lo[k]);
                    uint8_t* ph = stage_p + kOffPInStage + row * 64;
                    uint8_t* pl = smem + kOffScratch + 4096 * (it & 1) + row * 64;
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        const int off = ((2 * half + w) ^ ((row >> 1) & 3)) << 4;
                        *reinterpret_cast<uint4*>(ph + off) = make_uint4(hi[4 * w], hi[4 * w + 1], hi[4 * w + 2], hi[4 * w + 3]);
                        *reinterpret_cast<uint4*>(pl + off) = make_uint4(lo[4 * w], lo[4 * w + 1], lo[4 * w + 2], lo[4 * w + 3]);
                    }
                } else {
                    // P row `row`, tokens [32 half, 32 half + 32): four 16-byte chunks of the
                    // 128-byte K-major row, 128-byte swizzle, over the page's rope chunk (the
                    // score MMAs that read it have completed: S_FULL was waited above)
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) pk[k] = pack_bf16(pv[2 * k], pv[2 * k + 1]);
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
            // O / l.  A split writes its fp32 partial in the workspace's quad-interleaved layout
            // (column quads outermost, then the warp's 16 rows): each store instruction of the
            // warp covers two whole 256-byte runs.  A request held whole goes to the bf16
            // output, row-major, through a 2 KB staging tile per warp (16 rows x 128 bytes,
            // 16-byte pieces XOR-swizzled by row) so that every store writes whole row segments.
            uint8_t* stg = smem + kOffScratch + (warp - 2) * kEpiWarpBytes;
            const int rows_ok = min(16, p.M - (qb * kRows + quad * 16));  // valid rows of this warp
            const int64_t out_row0 = (int64_t)S.b * p.M + qb * kRows + quad * 16;
            float4* pq = reinterpret_cast<float4*>(po + ((int64_t)si * nqb + qb) * kRows * kDv) + quad * 2048 +
                         8 * half * 16 + r16;  // + (16 q + v) * 16 for columns 64 q + 32 half + 4 v
            // one column chunk (64 columns) of O / l from registers to memory
            auto store_chunk = [&](int q, const uint32_t(&oq)[32]) {
                if (!S.split) {
                    // bf16: the row's 64 columns are 8 pieces; this thread holds pieces 4 half + w
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(oq[8 * w + 0]) * inv, __uint_as_float(oq[8 * w + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(oq[8 * w + 2]) * inv, __uint_as_float(oq[8 * w + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(oq[8 * w + 4]) * inv, __uint_as_float(oq[8 * w + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(oq[8 * w + 6]) * inv, __uint_as_float(oq[8 * w + 7]) * inv);
                        *reinterpret_cast<uint4*>(stg + r16 * 128 + (((4 * half + w) ^ (r16 & 7)) << 4)) = v;
                    }
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int idx = lane + 32 * j, rr = idx >> 3, w = idx & 7;
                        const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((w ^ (rr & 7)) << 4));
                        if (rr < rows_ok)
                            *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.out) +
                                                      (out_row0 + rr) * kDv + 64 * q + 8 * w) = v;
                    }
                    __syncwarp();
                } else if (row_valid) {
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        pq[(16 * q + v) * 16] =
                            make_float4(__uint_as_float(oq[4 * v]) * inv, __uint_as_float(oq[4 * v + 1]) * inv,
                                        __uint_as_float(oq[4 * v + 2]) * inv, __uint_as_float(oq[4 * v + 3]) * inv);
                }
            };
            // two register sets: the next chunk's TMEM load is in flight while one is stored.
            // The loop is not unrolled: this code runs once per split, from a cold
            // instruction cache, so its size costs more than its loop overhead.
            uint32_t oa[32], ob[32];
            ptx::tmem_ld16x32<32>(t_lo, oa);
#pragma unroll 1
            for (int q = 0; q < 8; q += 2) {
                ptx::tmem_wait_ld();
                ptx::tmem_ld16x32<32>(t_lo + 64u * (q + 1), ob);
                store_chunk(q, oa);
                ptx::tmem_wait_ld();
                if (q + 2 < 8) ptx::tmem_ld16x32<32>(t_lo + 64u * (q + 2), oa);
                store_chunk(q + 1, ob);
            }
            if (row_valid && half == 0) {
                const float lse2 =
                    badpage ? nanv : (l > 0.f ? m_run - Geo<KV>::kPOffset + __log2f(l) : -INFINITY);
                if (!S.split)
                    p.lse[orow] = lse2 * kLn2;
                else
                    plse[prow] = lse2;
            }
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

int sm100_cta_slots() {
    // CTAs of the scan kernel the current device keeps resident at once (one per SM).
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    if (cudaFuncSetAttribute(decode_sm100_kernel<MLA_KV_E4M3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return -1;
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_sm100_kernel<MLA_KV_E4M3>, kThreads,
                                                      kSmemBytes) !=
            cudaSuccess ||
        per_sm <= 0)
        return -1;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    const int n = per_sm * sms;
    if (dev < 64) cached[dev] = n;
    return n;
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

template <int KV>
bool cached_kv_map(int dev, const DecodeParams& p, CUtensorMap* out) {
    static thread_local TmapCacheEntry e;
    if (e.dev != dev || e.kv != p.kv || e.num_pages != p.num_pages) {
        const uint64_t kvrows = (uint64_t)p.num_pages * kPage;
        const bool ok = KV == MLA_KV_E4M3
                            ? make_map_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.kv, kDqk, kvrows, kDqk, 64, kTok,
                                          CU_TENSOR_MAP_SWIZZLE_64B)
                            : make_map_2d(&e.map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.kv, kDqk, kvrows, kDqk * 2, 64,
                                          kTok, CU_TENSOR_MAP_SWIZZLE_128B);
        if (!ok) {
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
template <int KV>
bool smem_attribute_set(int dev) {
    static int done[64] = {};
    if (dev < 64 && done[dev]) return true;
    if (cudaFuncSetAttribute(decode_sm100_kernel<KV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
        return false;
    if (dev < 64) done[dev] = 1;
    return true;
}

template <int KV>
mla_status launch_typed(const DecodeParams& p, cudaStream_t stream) {
    Sm100Args a;
    memset(&a, 0, sizeof(a));
    a.p = p;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (!cached_kv_map<KV>(dev, p, &a.tm_kv)) return MLA_ERR_CUDA;
    if (!smem_attribute_set<KV>(dev)) return MLA_ERR_CUDA;
    const int ctas = p.groups_launched * num_row_blocks(p.s_q, p.H);
    // programmatic dependent launch: the prologue (barriers, TMEM, tensor map) overlaps the
    // tail of the previous grid in the stream; the kernel waits for it before any global access
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_sm100_kernel<KV>, a) != cudaSuccess) return MLA_ERR_CUDA;
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

mla_status launch_wait_timeout_probe(void* ws, cudaStream_t stream) {
    wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(ws);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status launch_decode_sm100(const DecodeParams& p, int kv_dtype, cudaStream_t stream) {
    return kv_dtype == MLA_KV_E4M3 ? launch_typed<MLA_KV_E4M3>(p, stream) : launch_typed<MLA_KV_BF16>(p, stream);
}

}  // namespace mla
