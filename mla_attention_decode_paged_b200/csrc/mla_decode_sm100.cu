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
//   lanes at offset 16 : q (64 x 576 bf16, 288 columns, loaded once per split) and two
//                        64-column score buffers.
// Per page:
//   TMA (producer warp): the page's 64 rows x 576 columns as nine 64-column boxes with
//       128-byte swizzle (one 72 KB stage; three stages).  An e4m3 page lands as nine
//       unswizzled 64 x 64-byte boxes in the upper half of each bf16 slot, and four more
//       warps widen it to bf16 in place (exact); kv_scale is folded into the score and
//       output scales.
//   MMA (one thread): S = q . K^T with q read from TMEM (M=64 N=64, 36 K-steps), then
//       O += P . V with P (bf16) and V (the same page, read MN-major) from shared memory
//       (M=64 N=256, twice, 4 K-steps each).  P is written over the page's rope chunk,
//       which only the score MMAs read: every stage carries its own P, and the softmax
//       of a page never waits for the previous page's PV.
//   softmax (4 warps, 16 rows each, two threads per row with 32 scores each): base-2
//       online softmax with the causal draft mask; the running max is only raised (and
//       O rescaled) when a score exceeds it by more than 8, so P <= 256.
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
constexpr int kStages = 3;
// warp 0 TMA, warp 1 MMA, warps 2-5 softmax / epilogue, and for an e4m3 cache warps 6-9
// widen each landed page to bf16 in place
constexpr int kThreadsBf16 = 192;
constexpr int kThreadsE4m3 = 320;
template <int KV>
constexpr int threads_for() { return KV == MLA_KV_E4M3 ? kThreadsE4m3 : kThreadsBf16; }
static_assert(kRows == 64, "the TMEM layout below is the 64-row MMA layout");

constexpr uint32_t kChunk = kTok * 128;              // 64 tokens x 64 columns bf16, 128B-swizzled
constexpr uint32_t kStageBytes = 9 * kChunk;         // 8 latent chunks + 1 rope chunk: 72 KB
constexpr uint32_t kRawChunk = kTok * 64;            // e4m3: 64 tokens x 64 columns, in the upper half
constexpr uint32_t kRawStageBytes = 9 * kRawChunk;   //        of each bf16 chunk slot
constexpr uint32_t kOffKv = 0;
constexpr uint32_t kOffPInStage = 8 * kChunk;        // P (64 rows x 64 tokens bf16) over the rope chunk
constexpr uint32_t kOffEpi = kOffKv + kStages * kStageBytes;  // epilogue staging: 2 KB per softmax warp
constexpr uint32_t kEpiWarpBytes = 16 * 128;
constexpr uint32_t kOffBar = kOffEpi + 4 * kEpiWarpBytes;
static_assert(kRows * kTok * 2 == kChunk, "P fills the rope chunk exactly");
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // barriers + alignment slack
static_assert(kSmemBytes <= 232448, "dynamic shared memory limit per block");

enum : int {
    B_KV_FULL0 = 0, B_KV_EMPTY0 = B_KV_FULL0 + kStages, B_Q_FULL = B_KV_EMPTY0 + kStages, B_S_FULL0,
    B_P_READY0 = B_S_FULL0 + 2, B_PV_DONE0 = B_P_READY0 + 2, B_DRAIN = B_PV_DONE0 + 2, B_RAW0,
    B_CONV = B_RAW0 + kStages, B_COUNT
};
constexpr uint32_t kOffTmemHolder = kOffBar + 8 * B_COUNT;
constexpr uint32_t kOffAbort = kOffTmemHolder + 4;
static_assert(kOffAbort + 4 <= kOffBar + 256, "barrier area");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kLaneHi = 16u << 16;  // second half-subpartition set (q and scores)
constexpr uint32_t kColQ = 0;            // q: 288 columns (bf16 pairs)
constexpr uint32_t kColS = 288;          // scores: 2 x 64 columns
constexpr float kRescaleThreshold = 8.0f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kRows, kTok, 0, 0);
constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kRows, 256, 0, 1);

struct __align__(64) Sm100Args {
    CUtensorMap tm_kv;  // cache viewed [P*64 rows, 576 cols]: bf16 box 64 x 64 with 128B swizzle, or
                        // e4m3 box 64 x 64 bytes without swizzle
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

// Twelve score K-steps starting at K0 (of 36): q from TMEM, the page from shared memory.
// K0 is a template constant so that every descriptor offset is an immediate.
template <int K0>
__device__ __forceinline__ void issue_s_chunk(uint32_t d, uint32_t a0, uint64_t b0) {
#pragma unroll
    for (int k = 0; k < 12; ++k) {
        constexpr int kChunkUnits = kChunk >> 4;
        const int ks = K0 + k;
        ptx::mma_ts(d, a0 + 8u * ks, b0 + (uint64_t)((ks >> 2) * kChunkUnits + (ks & 3) * 2), kIdescS,
                    ks ? 1u : 0u);
    }
}

// e4m3 -> bf16 for 32 consecutive bytes (exact: every e4m3 value is a bf16 value)
__device__ __forceinline__ void widen_e4m3x32(const uint4 (&in)[2], uint32_t (&out)[16]) {
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        const uint32_t word = (w < 4) ? (&in[0].x)[w] : (&in[1].x)[w - 4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const float2 f = e4m3x2_to_float2((uint16_t)(word >> (16 * hh)));
            __nv_bfloat162 v = __floats2bfloat162_rn(f.x, f.y);
            out[2 * w + hh] = *reinterpret_cast<uint32_t*>(&v);
        }
    }
}

template <int KV>
__global__ void __launch_bounds__(threads_for<KV>(), 1) decode_sm100_kernel(const __grid_constant__ Sm100Args args) {
    constexpr bool kE4m3 = KV == MLA_KV_E4M3;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const DecodeParams& p = args.p;
    PlanHeader* h = reinterpret_cast<PlanHeader*>(p.ws);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the combine may start its prologue now; it waits for this grid before reading
    ptx::griddep_launch_dependents();
    if (warp == 0 && lane == 0) ptx::prefetch_tmap(&args.tm_kv);
    // the plan (and every earlier write) must be complete before the header is read
    ptx::griddep_wait();

    if (h->magic != kPlanMagic || h->B != p.B || h->s_q != p.s_q || h->H != p.H ||
        h->num_groups > p.groups_launched) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(h, kStatusPlanMismatch, 0);
        return;
    }
    const int nqb = h->nqb;
    const int g = blockIdx.x / nqb, qb = blockIdx.x % nqb;
    if (g >= h->num_groups) return;

    Ctx c;
    c.bar0 = sbase + kOffBar;
    c.abort = reinterpret_cast<volatile int*>(smem + kOffAbort);
    c.h = h;
    if (threadIdx.x == 0) {
        *c.abort = 0;
        for (int s = 0; s < kStages; ++s) {
            // bf16: the TMA completes the stage; e4m3: the 128 converter threads do
            ptx::mbar_init(c.bar(B_KV_FULL0 + s), kE4m3 ? 128 : 1);
            ptx::mbar_init(c.bar(B_KV_EMPTY0 + s), 1);
            ptx::mbar_init(c.bar(B_RAW0 + s), 1);
        }
        ptx::mbar_init(c.bar(B_CONV), 128);
        ptx::mbar_init(c.bar(B_Q_FULL), 128);
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(c.bar(B_S_FULL0 + s), 1);
            ptx::mbar_init(c.bar(B_P_READY0 + s), 128);
            ptx::mbar_init(c.bar(B_PV_DONE0 + s), 1);
        }
        ptx::mbar_init(c.bar(B_DRAIN), 1);
        ptx::fence_mbar_init_cluster();
    }
    if (warp == 1) {
        ptx::tmem_alloc(sbase + kOffTmemHolder, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemHolder);

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
                        if (kE4m3) {
                            ptx::mbar_arrive_expect_tx(c.bar(B_RAW0 + st), kRawStageBytes);
#pragma unroll
                            for (int jb = 0; jb < 9; ++jb)
                                ptx::tma_load_2d(dst + jb * kChunk + kRawChunk, &args.tm_kv, c.bar(B_RAW0 + st),
                                                 64 * jb, ky);
                        } else {
                            ptx::mbar_arrive_expect_tx(c.bar(B_KV_FULL0 + st), kStageBytes);
#pragma unroll
                            for (int jb = 0; jb < 9; ++jb)
                                ptx::tma_load_2d(dst + jb * kChunk, &args.tm_kv, c.bar(B_KV_FULL0 + st), 64 * jb,
                                                 ky);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        if (lane == 0 && *c.abort) {
            for (int k = (it > kStages ? it - kStages : 0); k < it; ++k)
                drain_wait(c.bar((kE4m3 ? B_RAW0 : B_KV_FULL0) + k % kStages), (k / kStages) & 1);
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
                            const uint64_t b0 = ptx::smem_desc(sbase + kOffKv + st * kStageBytes, 16, 1024,
                                                               ptx::kSwizzle128);
                            const uint32_t d = tmem + kLaneHi + kColS + 64u * (its & 1);
                            const uint32_t a0 = tmem + kLaneHi + kColQ;
                            issue_s_chunk<0>(d, a0, b0);
                            issue_s_chunk<12>(d, a0, b0);
                            issue_s_chunk<24>(d, a0, b0);
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
    } else if (kE4m3 && warp >= 6) {
        // ------------------------------------------------------------ e4m3 -> bf16 (warps 6-9)
        // Every thread takes one half-row (32 bytes) of each of the nine chunks: all reads
        // first, a bounded barrier among the converters, then the writes, because each bf16
        // chunk overwrites its own e4m3 bytes in the upper half of its slot.
        const int ct = threadIdx.x - 192;  // 0..127
        const int r = ct >> 1, hf = ct & 1;
        int it = 0;
        bool alive = true;
        for (int si = seg_lo; si < seg_hi && alive; ++si) {
            const Segment S = segs[si];
            const int T = p.seq_lens[S.b];
            if (!request_ok(p, T)) continue;
            for (int t = S.tile_begin; t < S.tile_end; ++t, ++it) {
                const int st = it % kStages;
                alive = wait_bar(c, c.bar(B_RAW0 + st), (it / kStages) & 1);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                uint8_t* stage = smem + kOffKv + st * kStageBytes;
                uint4 raw[9][2];
#pragma unroll
                for (int j = 0; j < 9; ++j) {
                    const uint4* src = reinterpret_cast<const uint4*>(stage + j * kChunk + kRawChunk + r * 64 + hf * 32);
                    raw[j][0] = src[0];
                    raw[j][1] = src[1];
                }
                ptx::mbar_arrive(c.bar(B_CONV));
                alive = wait_bar(c, c.bar(B_CONV), it & 1);
                if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
#pragma unroll
                for (int j = 0; j < 9; ++j) {
                    uint32_t o[16];
                    widen_e4m3x32(raw[j], o);
                    uint8_t* rowp = stage + j * kChunk + r * 128;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int piece = 4 * hf + w;  // 16-byte piece of the 128-byte row, swizzled
                        *reinterpret_cast<uint4*>(rowp + ((piece ^ (r & 7)) << 4)) =
                            make_uint4(o[4 * w], o[4 * w + 1], o[4 * w + 2], o[4 * w + 3]);
                    }
                }
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(c.bar(B_KV_FULL0 + st));
            }
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
            // q rows of this block into TMEM: 9 x (16 columns per half) = 576 bf16 per row.
            // The loads of a batch are all issued before the first is used: at a split's start
            // the memory system is full of the first pages' loads, and every dependent round
            // trip here delays the first score MMA.  One batch of 36 loads per thread; three
            // for an e4m3 cache, whose kernel has fewer registers per thread.
            {
                constexpr int kQBatch = kE4m3 ? 3 : 9;  // column blocks per batch
                const uint4* src = reinterpret_cast<const uint4*>(qsrc + ((int64_t)S.b * p.M + m_glob) * kDqk);
#pragma unroll 1
                for (int kb = 0; kb < 9; kb += kQBatch) {
                    uint4 x[kQBatch][4];
#pragma unroll
                    for (int k = 0; k < kQBatch; ++k)
#pragma unroll
                        for (int w = 0; w < 4; ++w)  // dims [64 (kb + k) + 32 half, +32)
                            x[k][w] = row_valid ? src[(64 * (kb + k) + 32 * half) / 8 + w] : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int k = 0; k < kQBatch; ++k) {
                        uint32_t v[16];
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            v[4 * w] = x[k][w].x;
                            v[4 * w + 1] = x[k][w].y;
                            v[4 * w + 2] = x[k][w].z;
                            v[4 * w + 3] = x[k][w].w;
                        }
                        ptx::tmem_st16x16<16>(t_hi + kColQ + 32u * (kb + k), v);
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
                const float sc = p.score_scale_log2;
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
                if (tile == ntiles_req - 1 && (T % kPage) != 0) {
                    // rows past the request's end hold stale data (maybe NaN): zero their
                    // latent columns before the PV product reads them with P = 0
                    alive = wait_bar(c, c.bar(B_KV_FULL0 + it % kStages), (it / kStages) & 1);
                    if (__any_sync(0xffffffffu, !alive)) { alive = false; break; }
                    const int r0 = T % kPage;
                    uint8_t* vb = smem + kOffKv + (it % kStages) * kStageBytes;
                    const int pieces = (kPage - r0) * 8 * 8;  // rows x latent chunks x 16-byte pieces
                    for (int q = tid; q < pieces; q += 128) {
                        const int r = r0 + q / 64, j = (q / 8) % 8, w = q % 8;
                        *reinterpret_cast<uint4*>(vb + j * kChunk + r * 128 + w * 16) = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                {
                    // P row `row`, tokens [32 half, 32 half + 32): four 16-byte chunks of the
                    // 128-byte K-major row, 128-byte swizzle, over the page's rope chunk (the
                    // score MMAs that read it have completed: S_FULL was waited above)
                    uint8_t* pbuf = smem + kOffKv + (it % kStages) * kStageBytes + kOffPInStage;
                    uint8_t* prow_s = pbuf + (row >> 3) * 1024 + (row & 7) * 128;
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
            uint8_t* stg = smem + kOffEpi + (warp - 2) * kEpiWarpBytes;
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
                const float lse2 = badpage ? nanv : (l > 0.f ? m_run + __log2f(l) : -INFINITY);
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
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_sm100_kernel<MLA_KV_E4M3>, kThreadsE4m3,
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
                                          CU_TENSOR_MAP_SWIZZLE_NONE)
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
    cfg.blockDim = dim3(threads_for<KV>());
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
