/*
 * mla_decode.h -- C ABI of the paged, weight-absorbed MLA decode library
 * (libmla_decode.so, CUDA for sm_100a).
 *
 * The operation.  Multi-head Latent Attention keeps one shared latent row per cached
 * token: a 512-wide c_kv plus a decoupled 64-wide RoPE key, 576 values in all
 * ["TokenSpeed" related-work notes (zhaifeiyue.github.io), DeepSeek-V3 entry: 512-dim
 * latent KV; llm-atlas "Inference systems", 22 DeepSeek V2->V3: RoPE part decoupled].
 * Decode runs in that latent space ("absorb + project", same entry): the no-RoPE query
 * is multiplied through W_UK first, so q is 576 wide, and the 512-wide output through
 * W_UV afterwards (mla_absorb_q and mla_project_out below, or the caller's own GEMMs).  The s_q speculative query tokens of a
 * request and its H heads are folded into one row axis of M = s_q * H rows, row
 * m = i * H + h, all attending to the same cached rows ("TokenSpeed" launch digest
 * (cvshuo.com), MLA kernel paragraphs: the query-sequence axis is folded into the
 * head axis to fill the M tile; zhaifeiyue notes, Attack 1: H_eff = num_heads x F).
 * The cache is paged: logical block p of request b lives in physical page
 * block_table[b][p] [llm-atlas "Inference systems", 07 PagedAttention].  Draft token
 * i of request b sees cached tokens t <= T_b - s_q + i (causal) or t < T_b, i.e.
 * seq_lens counts the drafts, whose rows are the last s_q rows of the cache
 * [llm-atlas "Inference systems", 16 Speculative decoding: candidates verified in
 * parallel].  For each row:
 *     s_t = scale * q . KV_t,   out = sum_t softmax(s)_t * KV_t[0:512],
 *     lse = ln sum_t exp(s_t).
 * Long caches are scanned in splits whose partial (out, lse) are merged by an
 * LSE-weighted combine ["Faster kernels, slower engine" (jinnpan.com), 7.1 Gluon MLA
 * decode: split-KV scan and reduction].  An fp8 cache stores e4m3 bytes with one
 * fp32 scale per tensor, value = e4m3(byte) * kv_scale ["Faster kernels, slower
 * engine", setup note on the fp8 KV cache: half the bytes per cached token].
 *
 * Conventions for every entry point.
 *  - Pointers are DEVICE pointers unless marked host.  All arrays are dense,
 *    row-major, and start on a 16-byte boundary (the cache and q on 128 bytes).
 *  - The caller owns every buffer, including the workspace; nothing is retained after
 *    a call returns.  mla_decode_plan / mla_decode / mla_split_kv_combine and the other
 *    compute entry points (mla_prefill, mla_kv_append, mla_absorb_q, mla_project_out)
 *    never allocate, free or synchronise: they enqueue work on `stream` (a
 *    cudaStream_t, 0 = legacy default stream) and return.
 *  - Errors are return codes; nothing is thrown across the ABI.  Arguments are
 *    checked on the host before anything is enqueued.  Conditions only the device can
 *    see (a page id outside [0, num_pages), seq_len outside [1, max_pages * 64], or
 *    seq_len < s_q under the causal rule) set a status word in the workspace and turn
 *    the affected rows into NaN; read it with mla_get_device_status.
 */
#ifndef MLA_DECODE_H_
#define MLA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,         /* null pointer, non-positive size, non-finite scale */
    MLA_ERR_UNSUPPORTED = 2,         /* shape or dtype the kernels do not handle */
    MLA_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < mla_decode_workspace_size(...) */
    MLA_ERR_CUDA = 4,                /* a CUDA runtime/driver call failed */
    MLA_ERR_DEVICE_OOB = 5,          /* device status: bad page id or sequence length */
    MLA_ERR_DEVICE_TIMEOUT = 6,      /* device status: a bounded wait gave up */
    MLA_ERR_PLAN_MISMATCH = 7        /* device status: workspace plan made for other B/s_q/H */
} mla_status;

typedef enum { MLA_KV_BF16 = 0, MLA_KV_E4M3 = 1 } mla_kv_dtype;

/* Fixed geometry of the latent row and the page. */
#define MLA_HEAD_DIM_QK 576
#define MLA_HEAD_DIM_V 512
#define MLA_PAGE_SIZE 64

/*
 * Bytes of workspace a plan + decode of this shape needs (host, pure).
 * num_sms: SM count the split plan is made for; 0 = the current device's.
 * Returns 0 for an unsupported shape (B, s_q, H <= 0, or s_q * H > 65536), for a
 * num_sms that would make more than 1023 groups, or for a batch too large for the
 * planner's shared memory (more than about 12,000 requests).
 */
size_t mla_decode_workspace_size(int B, int s_q, int H, int num_sms);

/*
 * Split planner (one small kernel on `stream`).  From seq_lens[B] (device int32) it
 * partitions the pages of all requests, laid end to end, into G equal contiguous shares
 * (G = num_sms / row blocks, a row block being 64 folded query rows), one share per
 * group of scan CTAs (one CTA per row block), cutting requests into splits where a
 * share ends.  The plan is written into `workspace` and is valid for every later
 * mla_decode of the same seq_lens, B, s_q and H (e.g. all layers of one decode step).
 * num_sms as above; a smaller value gives fewer, longer splits (1 = no splits at all);
 * a plan made for more groups than the device runs at once is refused by the decode
 * (device status MLA_ERR_PLAN_MISMATCH).
 */
mla_status mla_decode_plan(const int32_t* seq_lens, int B, int s_q, int H, int num_sms,
                           void* workspace, size_t ws_bytes, void* stream);

/*
 * Paged absorbed-MLA decode: split scan over the plan in `workspace`, then the
 * split-KV combine.
 *   q           bf16 [B, s_q, H, 576]
 *   kv_pages    bf16 or e4m3 [num_pages, 64, 576]
 *   kv_dtype    MLA_KV_BF16 or MLA_KV_E4M3; kv_scale multiplies e4m3 values (ignored
 *               for bf16; must be finite and > 0 for e4m3)
 *   block_table int32 [B, max_pages_per_req]; entries past ceil(T_b / 64) are never
 *               read
 *   seq_lens    int32 [B], T_b >= 1, T_b <= max_pages_per_req * 64, and T_b >= s_q
 *               when causal != 0 (the same array the plan was made from)
 *   scale       softmax scale applied to the full 576-wide dot product
 *   causal      != 0: draft i sees t <= T_b - s_q + i; 0: every t < T_b
 *   out         bf16 [B, s_q, H, 512];  lse  fp32 [B, s_q, H], natural log
 * Supported: s_q * H <= 256 per request.
 * An e4m3 cache is read as it is by e4m3 x e4m3 tensor-core MMAs: q and the softmax
 * weights P are each cut into two e4m3 terms (q at a per-row power-of-two scale, which
 * holds a bf16 q exactly; P to 8 significant bits, as a bf16 P), so the results stay
 * within the rounding of the bf16 path.
 */
mla_status mla_decode(const void* q, const void* kv_pages, int kv_dtype, float kv_scale,
                      const int32_t* block_table, int max_pages_per_req,
                      const int32_t* seq_lens, int B, int s_q, int H, int64_t num_pages,
                      float scale, int causal, void* workspace, size_t ws_bytes, void* out,
                      float* lse, void* stream);

/*
 * The split scan of mla_decode alone (same arguments): rows of unsplit requests get
 * their final out / lse, split requests leave per-split partials in `workspace` for
 * mla_split_kv_combine.  mla_decode == mla_decode_scan followed by
 * mla_split_kv_combine; the two halves are exported so that each can be run and timed
 * on its own.
 */
mla_status mla_decode_scan(const void* q, const void* kv_pages, int kv_dtype, float kv_scale,
                           const int32_t* block_table, int max_pages_per_req,
                           const int32_t* seq_lens, int B, int s_q, int H, int64_t num_pages,
                           float scale, int causal, void* workspace, size_t ws_bytes, void* out,
                           float* lse, void* stream);

/*
 * The LSE-weighted combine of the split partials held in `workspace`: for every row of
 * a request that the plan split, lse = ln sum_j exp(lse_j) and
 * out = sum_j exp(lse_j - lse) * out_j (bf16); empty splits (lse_j = -inf) drop out.
 * Rows of unsplit requests are left untouched, and the rows of a request with
 * seq_len <= 0 (which the plan gives no split) are written as NaN here, not by the scan.
 * mla_decode calls it; it is exported so that it can be run (and timed) on its own.
 */
mla_status mla_split_kv_combine(const void* workspace, size_t ws_bytes, int B, int s_q, int H,
                                void* out, float* lse, void* stream);

/*
 * The projections on either side of the latent attention ("absorb + project":
 * zhaifeiyue "TokenSpeed" notes, DeepSeek-V3 entry).  Per head h, W_UK[h] and W_UV[h]
 * are the [512 x 128] up-projections of a latent row c (k_nope = c W_UK[h],
 * v = c W_UV[h]), bf16, stored [H, 512, 128] row-major.  R = B * s_q query rows.
 *
 * mla_absorb_q builds the decode's query: q[r, h, 0:512] = W_UK[h] q_nope[r, h] (so that
 * q . c = q_nope . k_nope), q[r, h, 512:576] = q_rope[r, h] (copied).
 *   q_nope bf16 [R, H, 128] (16-byte aligned); q_rope bf16 [R, H, 64] (16-byte aligned);
 *   w_uk bf16 [H, 512, 128] (16-byte aligned); q bf16 [R, H, 576] (16-byte aligned), the
 *   layout mla_decode reads.
 * mla_project_out maps the decode's output to the heads' value space:
 *   y[r, h, :] = out[r, h, :] W_UV[h];  out bf16 [R, H, 512] and w_uv bf16 [H, 512, 128]
 *   (16-byte aligned), y bf16 [R, H, 128] (4-byte aligned).
 * Both run on the tcgen05 tensor cores, accumulate in fp32 and round to bf16 (nearest,
 * ties to even).  Argument errors return before any launch.  Every wait inside the kernel
 * is bounded (2 s); these calls have no workspace and so no device status word: a wait
 * that gave up (never expected) leaves its rows unwritten.
 */
mla_status mla_absorb_q(const void* q_nope, const void* q_rope, const void* w_uk, int R, int H, void* q,
                        void* stream);
mla_status mla_project_out(const void* out, const void* w_uv, int R, int H, void* y, void* stream);

/*
 * Paged KV append: the write side of the same cache (the step after the decode in the
 * scope table).  The s_q new latent rows of request b -- the draft tokens the decode
 * verifies, counted in seq_lens -- are stored at positions T_b - s_q + i, row
 * pool[block_table[b][pos / 64]][pos % 64] (paging: llm-atlas "Inference systems", 07
 * PagedAttention), with the 64-wide decoupled rope key rotated by its position (22
 * DeepSeek V2->V3):
 *   ckv_new       bf16 [B, s_q, 512], 16-byte aligned: the latent c_kv rows, stored as
 *                 given (an e4m3 cache stores e4m3(value / kv_scale));
 *   kpe_new       bf16 [B, s_q, 64]: the rope key before rotation; pairs (2j, 2j+1) are
 *                 rotated: (x0 c_j - x1 s_j, x0 s_j + x1 c_j);
 *   rope_cos_sin  float [max_pos, 64]: for each position the 32 cosines, then the 32
 *                 sines (the caller's precomputed rope cache); positions >= max_pos are
 *                 an error;
 *   kv_pages, kv_dtype, kv_scale, block_table, max_pages_per_req, num_pages: the cache,
 *                 as for mla_decode (kv_scale > 0 for e4m3, ignored for bf16);
 *   status        optional device int32: set to MLA_ERR_DEVICE_OOB (if it was 0) for a
 *                 request whose length (T_b < s_q or > max_pages * 64), position or page
 *                 id is out of range; its rows are not written.  May be NULL.
 * Arithmetic: binary32 products and sums each rounded (no fused multiply-add), then
 * bf16 round-to-nearest-even, or e4m3 of a rounded binary32 division, round-to-nearest-
 * even, saturating at +-448.  Argument errors return before any launch.
 */
mla_status mla_kv_append(const void* ckv_new, const void* kpe_new, const float* rope_cos_sin, int max_pos,
                         void* kv_pages, int kv_dtype, float kv_scale, const int32_t* block_table,
                         int max_pages_per_req, const int32_t* seq_lens, int B, int s_q, int64_t num_pages,
                         int32_t* status, void* stream);

/*
 * Long-prefix MLA prefill: the second workload shape on the same cache (prefill over a
 * cache that already holds a long prefix is the other MLA workload of the "TokenSpeed"
 * launch digest (cvshuo.com), MLA kernel paragraphs).  Request b adds a chunk of `chunk` query tokens
 * whose latent rows are already its last `chunk` cache rows (seq_lens counts them, as it
 * counts the drafts of a decode): chunk token i sees cached tokens t <= T_b - chunk + i.
 * Each row's result is the decode's: out = softmax_t(scale q . KV_t) KV_t[0:512] and
 * lse = ln sum_t exp(scale q . KV_t).
 *   q           bf16 [B, chunk, H, 576], absorbed as for mla_decode
 *   kv_pages, kv_dtype, kv_scale, block_table, max_pages_per_req, num_pages, scale:
 *               as for mla_decode
 *   seq_lens    int32 [B] (4-byte aligned), chunk <= T_b <= max_pages_per_req * 64
 *   workspace   at least mla_prefill_workspace_size(B, chunk, H, max_pages_per_req, 0)
 *               bytes, 256-byte aligned, owned by the caller
 *   out         bf16 [B, chunk, H, 512];  lse  fp32 [B, chunk, H], natural log
 * The chunk runs on the decode path.  It is cut into sub-chunks of
 * d = mla_prefill_sub_chunk(chunk, H) tokens (d divides chunk, d * H <= 256 rows), and
 * sub-chunk j of request b is scanned as a decode request with seq_len
 * T_b - chunk + (j + 1) d and b's block-table row: its draft k is chunk token j d + k and
 * sees exactly the chunk's causal prefix.  q, out and lse need no copy (they are the
 * decode's arrays for B * chunk / d requests of d drafts).  A small kernel writes those
 * lengths and block-table rows into the workspace, then the planner, the split scan and
 * the combine run, all on `stream`; nothing is allocated or synchronised.  A request with
 * T_b < chunk or T_b > max_pages_per_req * 64 sets the device status MLA_ERR_DEVICE_OOB
 * and its rows come out NaN.
 * mla_prefill_sub_chunk (host, pure) returns d: the divisor of `chunk` with d * H <= 256
 * that needs the fewest 64-row blocks, (chunk / d) * ceil(d H / 64), ties to the larger;
 * 0 if chunk <= 0, H <= 0 or H > 256.  mla_prefill_workspace_size returns 0 for an
 * unsupported shape (as mla_decode_workspace_size, for B * chunk / d requests).
 */
int mla_prefill_sub_chunk(int chunk, int H);
size_t mla_prefill_workspace_size(int B, int chunk, int H, int max_pages_per_req, int num_sms);
mla_status mla_prefill(const void* q, const void* kv_pages, int kv_dtype, float kv_scale,
                       const int32_t* block_table, int max_pages_per_req, const int32_t* seq_lens,
                       int B, int chunk, int H, int64_t num_pages, float scale, void* workspace,
                       size_t ws_bytes, void* out, float* lse, void* stream);

/*
 * Test and debugging aid for the device-side failure detection (no counterpart on the
 * pages).  Every wait of the scan kernel on an mbarrier is bounded: after its limit (2 s)
 * the CTA gives up, records MLA_ERR_DEVICE_TIMEOUT in the workspace status word and
 * returns, so that a lost arrival never hangs the GPU.  This call runs that same wait
 * code in one thread on a barrier that nothing arrives at, with a 20 ms limit; afterwards
 * mla_get_device_status reports MLA_ERR_DEVICE_TIMEOUT and the context stays usable.
 * `workspace` needs only the 96-byte status header (256-byte aligned); a plan stored in
 * it is left intact.  Returns MLA_ERR_INVALID_ARG / MLA_ERR_WORKSPACE_TOO_SMALL / MLA_OK.
 */
mla_status mla_debug_wait_timeout(void* workspace, size_t ws_bytes, void* stream);

/*
 * Reads and clears the device status word of `workspace` (host out: *code, one of
 * MLA_OK, MLA_ERR_DEVICE_OOB, MLA_ERR_DEVICE_TIMEOUT, MLA_ERR_PLAN_MISMATCH).  This
 * call synchronises `stream`; it is meant for tests and debugging.
 */
mla_status mla_get_device_status(void* workspace, int* code, void* stream);

/*
 * mla_decode without a caller-provided workspace, for callers that cannot allocate
 * device memory: a plugin inside another runtime that owns all device memory and
 * forbids allocation on its execution path, or a latency-critical path that cannot
 * afford cudaMalloc's implicit device-wide synchronisation.  (The TokenSpeed pages
 * have no counterpart of this entry point; it is a property of this library.)
 *
 * Same arguments and results as mla_decode minus the workspace; it runs the planner,
 * the split scan and the combine.  The workspace is a scratch array compiled into the
 * library, MLA_NOALLOC_SCRATCH_BYTES (48 MiB) of device memory that every GPU which
 * loads the library holds until the process exits.  Nothing is allocated or freed by
 * the call.  Shapes whose plan needs more scratch than that return
 * MLA_ERR_WORKSPACE_TOO_SMALL (use mla_decode with your own workspace instead); the
 * five reference workloads, up to B = 32 requests of s_q * H = 256 rows, fit.
 *
 * Every call made outside stream capture looks up the scratch array's device address on
 * the current device (cudaGetSymbolAddress, which allocates nothing), so a device reset
 * that reloads the library's module is harmless; a call made while `stream` is being
 * captured uses the address found by the last uncaptured call on that device instead,
 * so make one uncaptured call first (and again after a device reset).
 * Every call shares the one array and the array keeps the last call's contents: the
 * planner rewrites everything that a call reads before reading it, but calls whose
 * work overlaps on the GPU (several streams, or several host threads on one device)
 * race on the scratch and give wrong results.  Serialise them.  Device-side errors
 * (bad page id or length) show only as NaN rows here: there is no workspace whose
 * status word the caller could read.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (48u << 20)
mla_status mla_decode_noalloc(const void* q, const void* kv_pages, int kv_dtype, float kv_scale,
                              const int32_t* block_table, int max_pages_per_req,
                              const int32_t* seq_lens, int B, int s_q, int H, int64_t num_pages,
                              float scale, int causal, void* out, float* lse, void* stream);

/* Library version string (host, static storage). */
const char* mla_decode_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H_ */
