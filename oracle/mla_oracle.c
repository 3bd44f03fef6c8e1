/*
 * mla_oracle.c -- plain, slow, float64 CPU oracle for weight-absorbed MLA decode
 * over a paged latent KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU
 * baseline leg may load this library.  It shares no code, header, table or helper
 * with the CUDA library; it is written from the definitions below, not from any
 * kernel.
 *
 * What it computes (one query row = one draft token i of request b, head h):
 *
 *   Latent cache row of token t of request b:
 *       KV_t = pool[ block_table[b][t / page] ][ t % page ][ 0 .. 575 ]
 *     Paging maps a logical block to a non-contiguous physical page
 *     [llm-atlas "Inference systems", 07 PagedAttention].
 *     Columns 0..511 are the shared 512-dim latent c_kv, 512..575 the decoupled
 *     RoPE key [zhaifeiyue "TokenSpeed" notes, DeepSeek-V3 entry (512-dim latent);
 *     llm-atlas "Inference systems", 22 DeepSeek V2->V3 (RoPE part decoupled)].
 *     For an fp8 cache the value is e4m3(byte) * kv_scale [Faster kernels, slower
 *     engine, two-stacks setup note on the fp8 KV cache].
 *
 *   Visible tokens (speculative verification: the s_q draft rows are the last s_q
 *   cache rows and are checked in parallel, each seeing its own prefix)
 *   [llm-atlas "Inference systems", 16 Speculative decoding]:
 *       causal:      t <= T_b - s_q + i
 *       non-causal:  t <  T_b
 *
 *   Absorbed attention (the query is already absorbed through W_UK, the output is
 *   projected through W_UV by the caller: "absorb + project")
 *   [zhaifeiyue "TokenSpeed" notes, DeepSeek-V3 entry]:
 *       s_t  = scale * sum_{d<576} q[b,i,h,d] * KV_t[d]
 *       m    = max_t s_t,   Z = sum_t exp(s_t - m)
 *       out  = sum_t exp(s_t - m) / Z * KV_t[0..511]
 *       lse  = m + ln Z                                  (natural log)
 *
 *   Split-KV partials and their LSE-weighted combination
 *   [Faster kernels, slower engine, 7.1 Gluon MLA decode (split scan + reduce)]:
 *       lse = ln sum_j exp(lse_j),  out = sum_j exp(lse_j - lse) * out_j
 *     An empty split has lse_j = -inf and contributes nothing.
 *
 * Everything is float64 from the exact bf16 / e4m3 input values.  Straight two-pass
 * softmax, no tiling, no online rescaling.  OpenMP over (request, row block).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_DQK 576
#define ORACLE_DV 512

enum { ORACLE_KV_BF16 = 0, ORACLE_KV_E4M3 = 1 };

/* bfloat16 is the upper half of an IEEE binary32: widen and reinterpret. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3 ("fn" flavour): 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite 448.
 * Exponent field 0 encodes subnormals m/8 * 2^-6. */
double oracle_e4m3_to_double(uint8_t byte) {
    int sign = (byte >> 7) & 1;
    int e = (byte >> 3) & 0xF;
    int m = byte & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

double oracle_bf16_to_double(uint16_t bits) { return bf16_bits_to_double(bits); }

/* Decode one 576-wide cache row of (physical page, slot) into doubles. */
static void load_row(const void* pool, int kv_dtype, double kv_scale, int64_t page,
                     int slot, int page_size, double* dst) {
    int64_t row = page * (int64_t)page_size + slot;
    if (kv_dtype == ORACLE_KV_BF16) {
        const uint16_t* p = (const uint16_t*)pool + row * ORACLE_DQK;
        for (int d = 0; d < ORACLE_DQK; ++d) dst[d] = bf16_bits_to_double(p[d]);
    } else {
        const uint8_t* p = (const uint8_t*)pool + row * ORACLE_DQK;
        for (int d = 0; d < ORACLE_DQK; ++d) dst[d] = oracle_e4m3_to_double(p[d]) * kv_scale;
    }
}

/*
 * Attention of every query row over the visible tokens t in [tok_lo, tok_hi) of its
 * request (tok_lo = 0, tok_hi = T_b for the unsplit result).  Returns 0 on success,
 * a negative value on an argument the definition does not cover (T_b < s_q under the
 * causal rule, T_b <= 0, a page id outside [0, P), T_b beyond the block table).
 *
 * q:        bf16 bits [B, s_q, H, 576]
 * pool:     bf16 bits or e4m3 bytes [P, page, 576]
 * out:      float64 [B, s_q, H, 512]   (0 where no token is visible)
 * lse:      float64 [B, s_q, H]        (-inf where no token is visible)
 */
int oracle_mla_decode_range(const uint16_t* q, const void* pool, int kv_dtype,
                            double kv_scale, const int32_t* block_table,
                            int max_pages, const int32_t* seq_lens, int B, int s_q,
                            int H, int64_t num_pages, int page_size, double scale,
                            int causal, const int32_t* tok_lo, const int32_t* tok_hi,
                            double* out, double* lse) {
    const int M = s_q * H;
    int bad = 0;
    for (int b = 0; b < B; ++b) {
        int T = seq_lens[b];
        if (T <= 0 || T > max_pages * page_size || (causal && T < s_q)) return -1;
        for (int p = 0; p < (T + page_size - 1) / page_size; ++p) {
            int32_t pg = block_table[(int64_t)b * max_pages + p];
            if (pg < 0 || pg >= num_pages) return -2;
        }
    }
    const int RB = 16; /* rows per block: keeps the score buffer per thread small */
    const int nrb = (M + RB - 1) / RB;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t job = 0; job < (int64_t)B * nrb; ++job) {
        int b = (int)(job / nrb);
        int r0 = (int)(job % nrb) * RB;
        int r1 = r0 + RB < M ? r0 + RB : M;
        int nr = r1 - r0;
        int T = seq_lens[b];
        int lo = tok_lo ? tok_lo[b] : 0;
        int hi = tok_hi ? tok_hi[b] : T;
        if (lo < 0) lo = 0;
        if (hi > T) hi = T;
        double* qd = (double*)malloc(sizeof(double) * RB * ORACLE_DQK);
        double* kv = (double*)malloc(sizeof(double) * ORACLE_DQK);
        int n = hi > lo ? hi - lo : 0;
        double* s = (double*)malloc(sizeof(double) * RB * (n > 0 ? n : 1));
        int last[16];
        double mx[16], Z[16];
        if (!qd || !kv || !s) { bad = 1; free(qd); free(kv); free(s); continue; }

        for (int r = 0; r < nr; ++r) {
            int row = r0 + r; /* folded row index = i * H + h */
            int i = row / H;
            const uint16_t* qr = q + ((int64_t)b * M + row) * ORACLE_DQK;
            for (int d = 0; d < ORACLE_DQK; ++d) qd[r * ORACLE_DQK + d] = bf16_bits_to_double(qr[d]);
            last[r] = causal ? (T - s_q + i) : (T - 1); /* last visible token */
            mx[r] = -INFINITY;
            Z[r] = 0.0;
        }
        /* pass 1: scores and row maxima */
        for (int t = lo; t < hi; ++t) {
            load_row(pool, kv_dtype, kv_scale, block_table[(int64_t)b * max_pages + t / page_size],
                     t % page_size, page_size, kv);
            for (int r = 0; r < nr; ++r) {
                if (t > last[r]) { s[(int64_t)r * n + (t - lo)] = -INFINITY; continue; }
                double acc = 0.0;
                const double* qr = qd + r * ORACLE_DQK;
                for (int d = 0; d < ORACLE_DQK; ++d) acc += qr[d] * kv[d];
                acc *= scale;
                s[(int64_t)r * n + (t - lo)] = acc;
                if (acc > mx[r]) mx[r] = acc;
            }
        }
        /* normaliser */
        for (int r = 0; r < nr; ++r) {
            if (mx[r] == -INFINITY) continue;
            double z = 0.0;
            for (int t = 0; t < n; ++t) {
                double v = s[(int64_t)r * n + t];
                if (v != -INFINITY) z += exp(v - mx[r]);
            }
            Z[r] = z;
        }
        /* pass 2: probability-weighted sum of the latent rows */
        for (int r = 0; r < nr; ++r) {
            double* o = out + ((int64_t)b * M + r0 + r) * ORACLE_DV;
            for (int d = 0; d < ORACLE_DV; ++d) o[d] = 0.0;
        }
        for (int t = lo; t < hi; ++t) {
            int any = 0;
            for (int r = 0; r < nr; ++r) any |= (t <= last[r]);
            if (!any) continue;
            load_row(pool, kv_dtype, kv_scale, block_table[(int64_t)b * max_pages + t / page_size],
                     t % page_size, page_size, kv);
            for (int r = 0; r < nr; ++r) {
                if (t > last[r]) continue;
                double p = exp(s[(int64_t)r * n + (t - lo)] - mx[r]) / Z[r];
                double* o = out + ((int64_t)b * M + r0 + r) * ORACLE_DV;
                for (int d = 0; d < ORACLE_DV; ++d) o[d] += p * kv[d];
            }
        }
        for (int r = 0; r < nr; ++r)
            lse[(int64_t)b * M + r0 + r] = (mx[r] == -INFINITY) ? -INFINITY : mx[r] + log(Z[r]);
        free(qd);
        free(kv);
        free(s);
    }
    return bad ? -3 : 0;
}

/* The unsplit result: every visible token of every request. */
int oracle_mla_decode(const uint16_t* q, const void* pool, int kv_dtype, double kv_scale,
                      const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                      int B, int s_q, int H, int64_t num_pages, int page_size, double scale,
                      int causal, double* out, double* lse) {
    return oracle_mla_decode_range(q, pool, kv_dtype, kv_scale, block_table, max_pages,
                                   seq_lens, B, s_q, H, num_pages, page_size, scale, causal,
                                   NULL, NULL, out, lse);
}

/*
 * LSE-weighted combination of n partial results of the same rows.
 * outs: float64 [n, rows, 512], lses: float64 [n, rows] (natural log, -inf = empty).
 */
void oracle_combine(const double* outs, const double* lses, int n, int64_t rows,
                    double* out, double* lse) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double mx = -INFINITY;
        for (int j = 0; j < n; ++j)
            if (lses[(int64_t)j * rows + r] > mx) mx = lses[(int64_t)j * rows + r];
        double* o = out + r * ORACLE_DV;
        for (int d = 0; d < ORACLE_DV; ++d) o[d] = 0.0;
        if (mx == -INFINITY) { lse[r] = -INFINITY; continue; }
        double z = 0.0;
        for (int j = 0; j < n; ++j) {
            double l = lses[(int64_t)j * rows + r];
            if (l != -INFINITY) z += exp(l - mx);
        }
        double L = mx + log(z);
        for (int j = 0; j < n; ++j) {
            double l = lses[(int64_t)j * rows + r];
            if (l == -INFINITY) continue;
            double w = exp(l - L);
            const double* oj = outs + ((int64_t)j * rows + r) * ORACLE_DV;
            for (int d = 0; d < ORACLE_DV; ++d) o[d] += w * oj[d];
        }
        lse[r] = L;
    }
}

/* ------------------------------------------------------------------ paged KV append
 *
 * The write side of the same cache.  The s_q new latent rows of request b (the draft
 * tokens under verification) take the positions
 *     pos_i = T_b - s_q + i          (seq_lens counts them, as in the decode above)
 * and row pos of request b is pool[ block_table[b][pos / page] ][ pos % page ]
 * [llm-atlas "Inference systems", 07 PagedAttention].
 *   columns 0..511   = c_kv of the new token, stored as given (an e4m3 cache stores its
 *                      quantised value);
 *   columns 512..575 = the decoupled rope key rotated by its position
 *                      [llm-atlas "Inference systems", 22 DeepSeek V2->V3].
 * Rotation (reading: adjacent pairs, as in the RoFormer formulation): for j < 32
 *     (x[2j], x[2j+1]) -> (x[2j] c_j - x[2j+1] s_j,  x[2j] s_j + x[2j+1] c_j),
 *     c_j = cos(pos * theta_j), s_j = sin(pos * theta_j), theta_j = base^(-2j/64).
 * The caller passes c and s as a float table [max_pos][64] (the 32 cosines, then the 32
 * sines), the precomputed rope cache serving engines carry; oracle_rope_table builds it
 * from the formula in float64 and rounds each entry to float.
 * The stored value is a rounding decision, so it is taken in one stated precision:
 * every product and sum in IEEE binary32, round to nearest, no fused multiply-add; then
 * bf16 (nearest, ties to even) or, for an e4m3 cache, e4m3 of (value / kv_scale) with
 * the division in binary32 (nearest, ties to the even code, saturating at +-448, NaN
 * kept).
 */

void oracle_rope_table(int max_pos, double base, float* table) {
    for (int pos = 0; pos < max_pos; ++pos)
        for (int j = 0; j < 32; ++j) {
            const double theta = pow(base, -2.0 * j / 64.0);
            table[(int64_t)pos * 64 + j] = (float)cos(pos * theta);
            table[(int64_t)pos * 64 + 32 + j] = (float)sin(pos * theta);
        }
}

/* binary32 -> bfloat16 bits, round to nearest, ties to even; NaN stays NaN. */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
    const uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* binary32 -> e4m3 byte: the nearest finite e4m3 value (ties to the even code, i.e. the
 * one whose mantissa's last bit is 0), magnitudes past 448 saturate to 448, NaN -> NaN.
 * Written as a search over the 127 non-negative finite codes. */
uint8_t oracle_f32_to_e4m3(float f) {
    if (f != f) return 0x7F;
    const uint8_t sign = signbit(f) ? 0x80 : 0x00;
    const double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    double best_err = INFINITY;
    for (int code = 0; code <= 0x7E; ++code) {
        const double err = fabs(oracle_e4m3_to_double((uint8_t)code) - a);
        if (err < best_err || (err == best_err && (code & 1) == 0)) {
            best = code;
            best_err = err;
        }
    }
    return sign | (uint8_t)best;
}

/* Returns 0, or -1 if some request was skipped (length or page id out of range). */
int oracle_kv_append(const uint16_t* ckv, const uint16_t* kpe, const float* cos_sin, int max_pos, void* pool,
                     int kv_dtype, float kv_scale, const int32_t* block_table, int max_pages,
                     const int32_t* seq_lens, int B, int s_q, int64_t num_pages, int page) {
    int rc = 0;
    for (int b = 0; b < B; ++b) {
        const int T = seq_lens[b];
        if (T < s_q || T > (int64_t)max_pages * page) { rc = -1; continue; }
        for (int i = 0; i < s_q; ++i) {
            const int pos = T - s_q + i;
            const int32_t pg = block_table[(int64_t)b * max_pages + pos / page];
            if (pg < 0 || pg >= num_pages || pos >= max_pos) { rc = -1; continue; }
            const int64_t row = (int64_t)pg * page + pos % page;
            const uint16_t* src = ckv + ((int64_t)b * s_q + i) * ORACLE_DV;
            const uint16_t* rk = kpe + ((int64_t)b * s_q + i) * 64;
            const float* cs = cos_sin + (int64_t)pos * 64;
            float vals[ORACLE_DQK];
            for (int d = 0; d < ORACLE_DV; ++d) vals[d] = (float)bf16_bits_to_double(src[d]);
            for (int j = 0; j < 32; ++j) {
                const float x0 = (float)bf16_bits_to_double(rk[2 * j]);
                const float x1 = (float)bf16_bits_to_double(rk[2 * j + 1]);
                const float c = cs[j], s = cs[32 + j];
                const float p00 = x0 * c, p11 = x1 * s, p01 = x0 * s, p10 = x1 * c;
                vals[ORACLE_DV + 2 * j] = p00 - p11;
                vals[ORACLE_DV + 2 * j + 1] = p01 + p10;
            }
            if (kv_dtype == ORACLE_KV_BF16) {
                uint16_t* dst = (uint16_t*)pool + row * ORACLE_DQK;
                for (int d = 0; d < ORACLE_DV; ++d) dst[d] = src[d];
                for (int d = ORACLE_DV; d < ORACLE_DQK; ++d) dst[d] = oracle_f32_to_bf16(vals[d]);
            } else {
                uint8_t* dst = (uint8_t*)pool + row * ORACLE_DQK;
                for (int d = 0; d < ORACLE_DQK; ++d) dst[d] = oracle_f32_to_e4m3(vals[d] / kv_scale);
            }
        }
    }
    return rc;
}
