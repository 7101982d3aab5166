/*
 * attn_oracle.c -- plain fp64 CPU reference for exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or table with the CUDA
 * library.
 *
 * Every function below is the plain definition of what the GPU kernels
 * compute, written for a reader to check by eye:
 *   - the score row is materialised in full, masked entries set to -inf;
 *   - softmax is the three-pass form (max, sum of exponentials, normalise);
 *   - all arithmetic is IEEE double, exp/log from libm.
 * Inputs arrive as float32 arrays (every bf16 or fp32 value the kernels read
 * is exact in float32) and are widened to double before any arithmetic.
 *
 * Sources (docs.rs source pages):
 *   [P1] scirs2-neural 0.4.3, src/layers/flash_attention.rs
 *   [P2] scirs2-neural 0.4.4, src/layers/grouped_query_attention.rs
 *   [P3] whisper-apr 0.3.1, src/model/attention_generated.rs
 *   [P4] oxibonsai-model 0.1.4, src/layers/flash_decode.rs
 *   [P5] whisper-apr 0.3.1, src/model/lfm2/gqa.rs
 *
 * Readings where the pages disagree or are silent:
 *   causal alignment  bottom-right: key j is masked for query row i when
 *                     j > i + (Skv - Sq)   ([P2] forward_with_cache mask with
 *                     a cache offset; [P3] streaming attention max_attend).
 *   fully masked row  output 0, LSE -inf   ([P1] final rescale skips l == 0;
 *                     [P4] flash_decode_tile all -inf tile).
 *   LSE               natural log of the sum of exp of the *scaled* scores
 *                     ([P4] flash_decode_tile: lse = m + ln(sum)).
 *   RoPE pairs        interleaved (2i, 2i+1), theta_i = pos * base^(-2i/D),
 *                     angles in double ([P2] RotaryPositionEmbedding::apply).
 *   GQA               q head h reads kv head h / (Hq/Hkv) ([P2]
 *                     forward_with_cache head grouping; [P5] attention_cached).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_INVALID_ARG 1
#define ORACLE_ERR_DIM_MISMATCH 2
#define ORACLE_ERR_EMPTY_KV 3
#define ORACLE_ERR_NOMEM 9

/* ------------------------------------------------------------------------------------------ */
/* RoPE                                                                                        */
/* ------------------------------------------------------------------------------------------ */

/* Rotate one head vector x[0..D) for position pos, in place.
 * [P2] RotaryPositionEmbedding::apply: for each pair i,
 *   theta = pos / base^(2i/D)
 *   x'_{2i}   = x_{2i} cos(theta) - x_{2i+1} sin(theta)
 *   x'_{2i+1} = x_{2i} sin(theta) + x_{2i+1} cos(theta)                                      */
static void rope_vec(double* x, double pos, int D, double base) {
    for (int i = 0; i < D / 2; ++i) {
        double theta = pos / pow(base, 2.0 * (double)i / (double)D);
        double c = cos(theta), s = sin(theta);
        double x0 = x[2 * i], x1 = x[2 * i + 1];
        x[2 * i] = x0 * c - x1 * s;
        x[2 * i + 1] = x0 * s + x1 * c;
    }
}

/* x [T, H, D] (float32 values) -> out [T, H, D] double, rotated at pos[t].                   */
int oracle_rope_f64(const float* x, const int32_t* pos, double* out, int T, int H, int D,
                    double base) {
    if (T < 0 || H <= 0 || D <= 0) return ORACLE_ERR_INVALID_ARG;
    if (D % 2 != 0) return ORACLE_ERR_INVALID_ARG; /* [P2] "RoPE head_dim must be even" */
    if (!(base > 0.0)) return ORACLE_ERR_INVALID_ARG;
    for (long t = 0; t < T; ++t)
        for (long h = 0; h < H; ++h) {
            double* o = out + (t * H + h) * D;
            const float* xi = x + (t * H + h) * D;
            for (int d = 0; d < D; ++d) o[d] = (double)xi[d];
            rope_vec(o, (double)pos[t], D, base);
        }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* One query row against keys [0, Skv): the definition                                         */
/* ------------------------------------------------------------------------------------------ */

/* q: D doubles.  K, V: Skv rows of D doubles (contiguous).  Keys j >= n_visible are masked.
 * s: scratch of Skv doubles.  Writes o[0..D) and *lse.
 *   s_j   = scale * sum_d q_d K_jd           (masked: -inf)
 *   m     = max_j s_j
 *   l     = sum_j exp(s_j - m)
 *   p_j   = exp(s_j - m) / l
 *   o_d   = sum_j p_j V_jd
 *   lse   = m + ln l
 * A row with every key masked returns o = 0, lse = -inf, before any softmax arithmetic.
 * [P3] scaled_dot_product_attention / apply_row_softmax (materialised scores, three-pass
 * softmax); [P4] flash_decode_tile (lse = m + ln(sum)); [P1] flash_attention_forward
 * (rows with zero sum stay zero).                                                            */
static void attn_row(const double* q, const double* K, const double* V, int Skv, int D,
                     int n_visible, double scale, double* s, double* o, double* lse) {
    if (n_visible <= 0) {
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    for (int j = 0; j < Skv; ++j) {
        if (j >= n_visible) {
            s[j] = -INFINITY;
            continue;
        }
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * K[(long)j * D + d];
        s[j] = scale * dot;
    }
    double m = -INFINITY;
    for (int j = 0; j < Skv; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int j = 0; j < Skv; ++j) l += exp(s[j] - m);
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int j = 0; j < Skv; ++j) {
        double p = exp(s[j] - m) / l;
        if (p == 0.0) continue;
        for (int d = 0; d < D; ++d) o[d] += p * V[(long)j * D + d];
    }
    *lse = m + log(l);
}

/* Number of keys query row i may see (bottom-right causal alignment).                        */
static int visible_keys(int i, int Sq, int Skv, int causal) {
    if (!causal) return Skv;
    long n = (long)i + (long)(Skv - Sq) + 1;
    if (n < 0) n = 0;
    if (n > Skv) n = Skv;
    return (int)n;
}

/* Gather K or V of (b, kvh) from [B, S, Hkv, D] float32 into contiguous double [S][D],
 * optionally rotated at positions 0..S-1.                                                    */
static void gather_head(const float* x, int b, int kvh, int S, int Hkv, int D, double rope_base,
                        double* out) {
    for (long j = 0; j < S; ++j) {
        const float* src = x + (((long)b * S + j) * Hkv + kvh) * D;
        double* dst = out + j * D;
        for (int d = 0; d < D; ++d) dst[d] = (double)src[d];
        if (rope_base > 0.0) rope_vec(dst, (double)j, D, rope_base);
    }
}

static int check_dims(int B, int Hq, int Hkv, int Sq, int Skv, int D) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || D <= 0) return ORACLE_ERR_INVALID_ARG;
    if (Skv <= 0) return ORACLE_ERR_EMPTY_KV;           /* [P4] FlashDecodeError::EmptyKv */
    if (Hq % Hkv != 0) return ORACLE_ERR_DIM_MISMATCH;  /* [P2] num_heads % num_kv_heads */
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Prefill / forward                                                                           */
/* ------------------------------------------------------------------------------------------ */

/* q [B,Sq,Hq,D], k/v [B,Skv,Hkv,D] float32 values.
 * If rows == NULL: o [B,Sq,Hq,D], lse [B,Hq,Sq] (double) for every row.
 * Else rows[r] = (b*Hq + hq)*Sq + i selects nrows rows; o [nrows,D], lse [nrows].
 * rope_base > 0: q row i is rotated at q_pos0 + i and key j at j before the scores.          */
int oracle_attn_fwd_f64(const float* q, const float* k, const float* v, double* o, double* lse,
                        int B, int Hq, int Hkv, int Sq, int Skv, int D, double scale, int causal,
                        double rope_base, int q_pos0, const int64_t* rows, int64_t nrows) {
    int st = check_dims(B, Hq, Hkv, Sq, Skv, D);
    if (st) return st;
    if (rope_base > 0.0 && D % 2) return ORACLE_ERR_INVALID_ARG;
    const int g = Hq / Hkv;
    double* Kd = (double*)malloc(sizeof(double) * (size_t)Skv * D);
    double* Vd = (double*)malloc(sizeof(double) * (size_t)Skv * D);
    if (!Kd || !Vd) {
        free(Kd);
        free(Vd);
        return ORACLE_ERR_NOMEM;
    }
    for (int b = 0; b < B; ++b) {
        for (int kvh = 0; kvh < Hkv; ++kvh) {
            /* which output rows belong to this (b, kvh)? */
            int64_t lo_row = ((int64_t)b * Hq + (int64_t)kvh * g) * Sq;
            int64_t hi_row = lo_row + (int64_t)g * Sq;
            int any = 0;
            if (rows) {
                for (int64_t r = 0; r < nrows && !any; ++r) any = rows[r] >= lo_row && rows[r] < hi_row;
                if (!any) continue;
            }
            gather_head(k, b, kvh, Skv, Hkv, D, rope_base, Kd);
            gather_head(v, b, kvh, Skv, Hkv, D, 0.0, Vd);
            int64_t n_work = rows ? nrows : (int64_t)g * Sq;
#pragma omp parallel
            {
                double* s = (double*)malloc(sizeof(double) * (size_t)Skv);
                double* qd = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 4)
                for (int64_t w = 0; w < n_work; ++w) {
                    int64_t row;
                    if (rows) {
                        row = rows[w];
                        if (row < lo_row || row >= hi_row) continue;
                    } else {
                        row = lo_row + w;
                    }
                    int hq = (int)((row / Sq) % Hq);
                    int i = (int)(row % Sq);
                    const float* qs = q + (((int64_t)b * Sq + i) * Hq + hq) * D;
                    for (int d = 0; d < D; ++d) qd[d] = (double)qs[d];
                    if (rope_base > 0.0) rope_vec(qd, (double)q_pos0 + (double)i, D, rope_base);
                    double* orow;
                    double* lrow;
                    if (rows) {
                        orow = o + w * D;
                        lrow = lse + w;
                    } else {
                        orow = o + (((int64_t)b * Sq + i) * Hq + hq) * D;
                        lrow = lse + ((int64_t)b * Hq + hq) * Sq + i;
                    }
                    attn_row(qd, Kd, Vd, Skv, D, visible_keys(i, Sq, Skv, causal), scale, s, orow,
                             lrow);
                }
                free(s);
                free(qd);
            }
        }
    }
    free(Kd);
    free(Vd);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Tiled forward with the online softmax (the method's own recurrence, in double)              */
/* ------------------------------------------------------------------------------------------ */

/* [P1] flash_attention_forward + online_softmax_update, per (b, hq), with query blocks of bq
 * rows and key blocks of bkv keys.  For each row, per key block:
 *   m' = max(m, max_j s_j);  c = (m == -inf) ? 0 : exp(m - m')
 *   l' = c l + sum_j exp(s_j - m');  O' = c O + sum_j exp(s_j - m') v_j
 * masked entries (-inf) contribute nothing; key blocks wholly above the causal diagonal are
 * skipped; at the end O /= l when l > 0 and lse = m + ln l (-inf when l == 0).
 * Used to pin the recurrence the kernels implement against the three-pass definition.        */
int oracle_attn_fwd_tiled_f64(const float* q, const float* k, const float* v, double* o,
                              double* lse, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                              double scale, int causal, int bq, int bkv) {
    int st = check_dims(B, Hq, Hkv, Sq, Skv, D);
    if (st) return st;
    if (bq <= 0 || bkv <= 0) return ORACLE_ERR_INVALID_ARG;
    const int g = Hq / Hkv;
    const long off = (long)Skv - (long)Sq;
    double* m = (double*)malloc(sizeof(double) * (size_t)Sq);
    double* l = (double*)malloc(sizeof(double) * (size_t)Sq);
    double* acc = (double*)malloc(sizeof(double) * (size_t)Sq * D);
    double* sblk = (double*)malloc(sizeof(double) * (size_t)bkv);
    if (!m || !l || !acc || !sblk) {
        free(m), free(l), free(acc), free(sblk);
        return ORACLE_ERR_NOMEM;
    }
    for (int b = 0; b < B; ++b)
        for (int hq = 0; hq < Hq; ++hq) {
            int kvh = hq / g;
            for (int i = 0; i < Sq; ++i) {
                m[i] = -INFINITY;
                l[i] = 0.0;
                for (int d = 0; d < D; ++d) acc[(long)i * D + d] = 0.0;
            }
            for (int q0 = 0; q0 < Sq; q0 += bq) {
                int q1 = q0 + bq < Sq ? q0 + bq : Sq;
                for (int k0 = 0; k0 < Skv; k0 += bkv) {
                    int k1 = k0 + bkv < Skv ? k0 + bkv : Skv;
                    if (causal && (long)k0 > (long)(q1 - 1) + off) continue; /* whole block masked */
                    for (int i = q0; i < q1; ++i) {
                        const float* qi = q + (((long)b * Sq + i) * Hq + hq) * D;
                        double bmax = -INFINITY;
                        for (int j = k0; j < k1; ++j) {
                            double sc;
                            if (causal && (long)j > (long)i + off) {
                                sc = -INFINITY;
                            } else {
                                const float* kj = k + (((long)b * Skv + j) * Hkv + kvh) * D;
                                double dot = 0.0;
                                for (int d = 0; d < D; ++d) dot += (double)qi[d] * (double)kj[d];
                                sc = scale * dot;
                            }
                            sblk[j - k0] = sc;
                            if (sc > bmax) bmax = sc;
                        }
                        double mnew = m[i] > bmax ? m[i] : bmax;
                        double c = (m[i] == -INFINITY) ? 0.0 : exp(m[i] - mnew);
                        l[i] *= c;
                        for (int d = 0; d < D; ++d) acc[(long)i * D + d] *= c;
                        for (int j = k0; j < k1; ++j) {
                            double sc = sblk[j - k0];
                            if (!(sc > -INFINITY)) continue;
                            double e = exp(sc - mnew);
                            l[i] += e;
                            const float* vj = v + (((long)b * Skv + j) * Hkv + kvh) * D;
                            for (int d = 0; d < D; ++d) acc[(long)i * D + d] += e * (double)vj[d];
                        }
                        m[i] = mnew;
                    }
                }
            }
            for (int i = 0; i < Sq; ++i) {
                double* orow = o + (((long)b * Sq + i) * Hq + hq) * D;
                for (int d = 0; d < D; ++d) orow[d] = l[i] > 0.0 ? acc[(long)i * D + d] / l[i] : 0.0;
                lse[((long)b * Hq + hq) * Sq + i] = l[i] > 0.0 ? m[i] + log(l[i]) : -INFINITY;
            }
        }
    free(m), free(l), free(acc), free(sblk);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Decode                                                                                      */
/* ------------------------------------------------------------------------------------------ */

/* One query token per (b, hq) against the first seqlens[b] cache rows; no mask
 * ([P5] attention_cached: a single new token sees the whole cache).
 * q [B,Hq,D]; kc/vc [B,Smax,Hkv,D] float32 values; o [B,Hq,D], lse [B,Hq] double.
 * The unsplit definition: the number of KV splits a kernel uses does not enter.              */
int oracle_decode_f64(const float* q, const float* kc, const float* vc, const int32_t* seqlens,
                      double* o, double* lse, int B, int Hq, int Hkv, int Smax, int D,
                      double scale) {
    int st = check_dims(B, Hq, Hkv, 1, Smax, D);
    if (st) return st;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 1 || seqlens[b] > Smax) return ORACLE_ERR_INVALID_ARG;
    const int g = Hq / Hkv;
    double* Kd = (double*)malloc(sizeof(double) * (size_t)Smax * D);
    double* Vd = (double*)malloc(sizeof(double) * (size_t)Smax * D);
    if (!Kd || !Vd) {
        free(Kd), free(Vd);
        return ORACLE_ERR_NOMEM;
    }
    for (int b = 0; b < B; ++b) {
        int L = seqlens[b];
        for (int kvh = 0; kvh < Hkv; ++kvh) {
            for (long j = 0; j < L; ++j)
                for (int d = 0; d < D; ++d) {
                    Kd[j * D + d] = (double)kc[(((long)b * Smax + j) * Hkv + kvh) * D + d];
                    Vd[j * D + d] = (double)vc[(((long)b * Smax + j) * Hkv + kvh) * D + d];
                }
#pragma omp parallel for schedule(static)
            for (int hq = kvh * g; hq < (kvh + 1) * g; ++hq) {
                double* s = (double*)malloc(sizeof(double) * (size_t)L);
                double qd[1024];
                double* qq = D <= 1024 ? qd : (double*)malloc(sizeof(double) * D);
                for (int d = 0; d < D; ++d) qq[d] = (double)q[((long)b * Hq + hq) * D + d];
                attn_row(qq, Kd, Vd, L, D, L, scale, s, o + ((long)b * Hq + hq) * D,
                         lse + (long)b * Hq + hq);
                if (qq != qd) free(qq);
                free(s);
            }
        }
    }
    free(Kd), free(Vd);
    return ORACLE_OK;
}

/* [P4] flash_decode_tile: softmax partial of one query over one contiguous key tile.
 * Returns the tile's normalised output and lse = m + ln(sum exp(s - m)); a tile whose scores
 * are all -inf (or that is empty) gives output 0 and lse -inf.                               */
static void decode_tile(const double* q, const double* K, const double* V, int n, int D,
                        double scale, double* s, double* out, double* lse) {
    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q[d] * K[(long)t * D + d];
        s[t] = scale * dot;
        if (s[t] > m) m = s[t];
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (!isfinite(m)) {
        *lse = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int t = 0; t < n; ++t) {
        s[t] = exp(s[t] - m);
        sum += s[t];
    }
    for (int t = 0; t < n; ++t)
        for (int d = 0; d < D; ++d) out[d] += s[t] * V[(long)t * D + d];
    for (int d = 0; d < D; ++d) out[d] /= sum;
    *lse = m + log(sum);
}

/* [P4] combine_tile_outputs: tiles with non-finite lse are dropped; with the global
 * L = max_i lse_i + ln(sum_i exp(lse_i - max_i lse_i)), out = sum_i exp(lse_i - L) out_i.
 * Also returns L (-inf and out = 0 when no tile is valid).                                   */
static void combine_tiles(int n, const double* outs, const double* lses, int D, double* out,
                          double* lse) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    double gmax = -INFINITY;
    for (int t = 0; t < n; ++t)
        if (isfinite(lses[t]) && lses[t] > gmax) gmax = lses[t];
    if (!isfinite(gmax)) {
        *lse = -INFINITY;
        return;
    }
    double gsum = 0.0;
    for (int t = 0; t < n; ++t)
        if (isfinite(lses[t])) gsum += exp(lses[t] - gmax);
    double L = gmax + log(gsum);
    for (int t = 0; t < n; ++t) {
        if (!isfinite(lses[t])) continue;
        double w = exp(lses[t] - L);
        for (int d = 0; d < D; ++d) out[d] += w * outs[(long)t * D + d];
    }
    *lse = L;
}

/* Split-KV decode exactly as [P4] flash_decode_single_head: num_tiles clamped to [1, L];
 * tile lengths L / n, the first L % n tiles one longer; per-tile partials combined by LSE.
 * Same layouts as oracle_decode_f64.  Any tile count gives the unsplit result up to rounding. */
int oracle_decode_split_f64(const float* q, const float* kc, const float* vc,
                            const int32_t* seqlens, double* o, double* lse, int B, int Hq, int Hkv,
                            int Smax, int D, double scale, int num_tiles) {
    int st = check_dims(B, Hq, Hkv, 1, Smax, D);
    if (st) return st;
    if (num_tiles < 1) return ORACLE_ERR_INVALID_ARG;
    const int g = Hq / Hkv;
    for (int b = 0; b < B; ++b) {
        int L = seqlens[b];
        if (L < 1 || L > Smax) return ORACLE_ERR_INVALID_ARG;
        int n = num_tiles < L ? num_tiles : L;
        int base = L / n, rem = L % n;
        for (int hq = 0; hq < Hq; ++hq) {
            int kvh = hq / g;
            double* qd = (double*)malloc(sizeof(double) * D);
            double* Kt = (double*)malloc(sizeof(double) * (size_t)(base + 1) * D);
            double* Vt = (double*)malloc(sizeof(double) * (size_t)(base + 1) * D);
            double* s = (double*)malloc(sizeof(double) * (size_t)(base + 1));
            double* outs = (double*)malloc(sizeof(double) * (size_t)n * D);
            double* lses = (double*)malloc(sizeof(double) * (size_t)n);
            for (int d = 0; d < D; ++d) qd[d] = (double)q[((long)b * Hq + hq) * D + d];
            int start = 0;
            for (int t = 0; t < n; ++t) {
                int len = base + (t < rem ? 1 : 0);
                for (int r = 0; r < len; ++r)
                    for (int d = 0; d < D; ++d) {
                        long src = (((long)b * Smax + start + r) * Hkv + kvh) * D + d;
                        Kt[(long)r * D + d] = (double)kc[src];
                        Vt[(long)r * D + d] = (double)vc[src];
                    }
                decode_tile(qd, Kt, Vt, len, D, scale, s, outs + (long)t * D, lses + t);
                start += len;
            }
            combine_tiles(n, outs, lses, D, o + ((long)b * Hq + hq) * D, lse + (long)b * Hq + hq);
            free(qd), free(Kt), free(Vt), free(s), free(outs), free(lses);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Backward                                                                                    */
/* ------------------------------------------------------------------------------------------ */

/* Gradients of the forward above with respect to q, k and v for an upstream gradient dout of o,
 * written from the definition (the backward of [P1] flash_backward_head, FA-2's Algorithm 4,
 * without its blocking; [P2] GQA backward: a kv head's gradients are summed over the q heads of
 * its group and the RoPE rotation is undone on dq and dk).  For every (b, q head, row i), with
 * s_j and p_j the scores and probabilities of attn_row (p_j = 0 for masked keys):
 *   dP_j  = sum_d dout_d V_jd
 *   Dsum  = sum_j p_j dP_j
 *   dS_j  = p_j (dP_j - Dsum)
 *   dq_r  = scale * sum_j dS_j K_j          (K, q as rotated in the forward)
 *   dk_r[j] += scale * dS_j q_r,   dv[j] += p_j dout
 * and finally dq = R(-theta) dq_r, dk = R(-theta) dk_r: the transpose of a rotation is the
 * rotation by the negated angle.  A row with no visible key contributes nothing.
 * q, dout [B,Sq,Hq,D]; k, v [B,Skv,Hkv,D] (float32 values); dq [B,Sq,Hq,D], dk, dv [B,Skv,Hkv,D]
 * (double).                                                                                  */
static int attn_bwd_core(const float* q, const float* k, const float* v, const float* dout,
                         const float* mask, int64_t mask_bstride, int64_t mask_hstride, double* dq, double* dk,
                         double* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, double scale, int causal,
                         double rope_base, int q_pos0) {
    int st = check_dims(B, Hq, Hkv, Sq, Skv, D);
    if (st) return st;
    if (rope_base > 0.0 && D % 2) return ORACLE_ERR_INVALID_ARG;
    const int g = Hq / Hkv;
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int b = 0; b < B; ++b) {
        for (int kvh = 0; kvh < Hkv; ++kvh) {
            double* Kd = (double*)malloc(sizeof(double) * (size_t)Skv * D);
            double* Vd = (double*)malloc(sizeof(double) * (size_t)Skv * D);
            double* dKr = (double*)calloc((size_t)Skv * D, sizeof(double));
            double* dVa = (double*)calloc((size_t)Skv * D, sizeof(double));
            double* s = (double*)malloc(sizeof(double) * (size_t)Skv);
            double* p = (double*)malloc(sizeof(double) * (size_t)Skv);
            double* dP = (double*)malloc(sizeof(double) * (size_t)Skv);
            double* qd = (double*)malloc(sizeof(double) * (size_t)D);
            double* go = (double*)malloc(sizeof(double) * (size_t)D);
            double* dqr = (double*)malloc(sizeof(double) * (size_t)D);
            if (!Kd || !Vd || !dKr || !dVa || !s || !p || !dP || !qd || !go || !dqr) {
#pragma omp atomic write
                fail = 1;
            } else {
                gather_head(k, b, kvh, Skv, Hkv, D, rope_base, Kd);
                gather_head(v, b, kvh, Skv, Hkv, D, 0.0, Vd);
                for (int hg = 0; hg < g; ++hg) {
                    const int hq = kvh * g + hg;
                    for (int i = 0; i < Sq; ++i) {
                        const long qoff = (((long)b * Sq + i) * Hq + hq) * D;
                        double* dqo = dq + qoff;
                        const int nvis = visible_keys(i, Sq, Skv, causal);
                        if (nvis <= 0) {
                            for (int d = 0; d < D; ++d) dqo[d] = 0.0;
                            continue;
                        }
                        for (int d = 0; d < D; ++d) qd[d] = (double)q[qoff + d];
                        if (rope_base > 0.0) rope_vec(qd, (double)q_pos0 + (double)i, D, rope_base);
                        for (int d = 0; d < D; ++d) go[d] = (double)dout[qoff + d];
                        /* scores (with the additive mask, if any) and the three-pass softmax */
                        const float* mrow =
                            mask ? mask + (long)b * mask_bstride + (long)hq * mask_hstride + (long)i * Skv : NULL;
                        double m = -INFINITY;
                        for (int j = 0; j < nvis; ++j) {
                            double dot = 0.0;
                            for (int d = 0; d < D; ++d) dot += qd[d] * Kd[(long)j * D + d];
                            s[j] = scale * dot + (mrow ? (double)mrow[j] : 0.0);
                            if (s[j] > m) m = s[j];
                        }
                        if (m == -INFINITY) { /* every key masked: no gradient through this row */
                            for (int d = 0; d < D; ++d) dqo[d] = 0.0;
                            continue;
                        }
                        double l = 0.0;
                        for (int j = 0; j < nvis; ++j) l += exp(s[j] - m);
                        double Dsum = 0.0;
                        for (int j = 0; j < nvis; ++j) {
                            p[j] = exp(s[j] - m) / l;
                            double dot = 0.0;
                            for (int d = 0; d < D; ++d) dot += go[d] * Vd[(long)j * D + d];
                            dP[j] = dot;
                            Dsum += p[j] * dP[j];
                        }
                        for (int d = 0; d < D; ++d) dqr[d] = 0.0;
                        for (int j = 0; j < nvis; ++j) {
                            const double dS = p[j] * (dP[j] - Dsum);
                            for (int d = 0; d < D; ++d) {
                                dqr[d] += scale * dS * Kd[(long)j * D + d];
                                dKr[(long)j * D + d] += scale * dS * qd[d];
                                dVa[(long)j * D + d] += p[j] * go[d];
                            }
                        }
                        if (rope_base > 0.0) rope_vec(dqr, -((double)q_pos0 + (double)i), D, rope_base);
                        for (int d = 0; d < D; ++d) dqo[d] = dqr[d];
                    }
                }
                for (int j = 0; j < Skv; ++j) {
                    double* dkr = dKr + (long)j * D;
                    if (rope_base > 0.0) rope_vec(dkr, -(double)j, D, rope_base);
                    const long koff = (((long)b * Skv + j) * Hkv + kvh) * D;
                    for (int d = 0; d < D; ++d) {
                        dk[koff + d] = dkr[d];
                        dv[koff + d] = dVa[(long)j * D + d];
                    }
                }
            }
            free(Kd);
            free(Vd);
            free(dKr);
            free(dVa);
            free(s);
            free(p);
            free(dP);
            free(qd);
            free(go);
            free(dqr);
        }
    }
    return fail ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

int oracle_attn_bwd_f64(const float* q, const float* k, const float* v, const float* dout,
                        double* dq, double* dk, double* dv, int B, int Hq, int Hkv, int Sq, int Skv,
                        int D, double scale, int causal, double rope_base, int q_pos0) {
    return attn_bwd_core(q, k, v, dout, NULL, 0, 0, dq, dk, dv, B, Hq, Hkv, Sq, Skv, D, scale, causal,
                         rope_base, q_pos0);
}

/* The backward of oracle_attn_fwd_mask_f64: the same definition with s_j including the mask.   */
int oracle_attn_bwd_mask_f64(const float* q, const float* k, const float* v, const float* dout,
                             const float* mask, int64_t mask_bstride, int64_t mask_hstride, double* dq,
                             double* dk, double* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                             double scale, int causal, double rope_base, int q_pos0) {
    if (!mask) return ORACLE_ERR_INVALID_ARG;
    return attn_bwd_core(q, k, v, dout, mask, mask_bstride, mask_hstride, dq, dk, dv, B, Hq, Hkv, Sq, Skv, D,
                         scale, causal, rope_base, q_pos0);
}

/* ------------------------------------------------------------------------------------------ */
/* Forward with an additive mask                                                               */
/* ------------------------------------------------------------------------------------------ */

/* As oracle_attn_fwd_f64 (full rows, no row subset), with an additive mask on the scaled scores
 * ([P3] compute_block_scores: score = dot * scale, then score += mask[q, k]; [P3]
 * scaled_dot_product_attention adds the mask before the row softmax):
 *   s_j = scale * q . k_j + mask[b, h, i, j]     (then the causal mask, if any: -inf)
 * mask element (b, h, i, j) sits at mask[b * mask_bstride + h * mask_hstride + i * Skv + j]
 * (a stride of 0 broadcasts).  A row whose scores are all -inf gets o = 0, lse = -inf.        */
int oracle_attn_fwd_mask_f64(const float* q, const float* k, const float* v, const float* mask,
                             int64_t mask_bstride, int64_t mask_hstride, double* o, double* lse, int B,
                             int Hq, int Hkv, int Sq, int Skv, int D, double scale, int causal,
                             double rope_base, int q_pos0) {
    int st = check_dims(B, Hq, Hkv, Sq, Skv, D);
    if (st) return st;
    if (!mask) return ORACLE_ERR_INVALID_ARG;
    if (rope_base > 0.0 && D % 2) return ORACLE_ERR_INVALID_ARG;
    const int g = Hq / Hkv;
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int b = 0; b < B; ++b) {
        for (int kvh = 0; kvh < Hkv; ++kvh) {
            double* Kd = (double*)malloc(sizeof(double) * (size_t)Skv * D);
            double* Vd = (double*)malloc(sizeof(double) * (size_t)Skv * D);
            double* s = (double*)malloc(sizeof(double) * (size_t)Skv);
            double* qd = (double*)malloc(sizeof(double) * (size_t)D);
            if (!Kd || !Vd || !s || !qd) {
#pragma omp atomic write
                fail = 1;
            } else {
                gather_head(k, b, kvh, Skv, Hkv, D, rope_base, Kd);
                gather_head(v, b, kvh, Skv, Hkv, D, 0.0, Vd);
                for (int hg = 0; hg < g; ++hg) {
                    const int hq = kvh * g + hg;
                    for (int i = 0; i < Sq; ++i) {
                        const long qoff = (((long)b * Sq + i) * Hq + hq) * D;
                        double* orow = o + qoff;
                        double* lrow = lse + ((long)b * Hq + hq) * Sq + i;
                        for (int d = 0; d < D; ++d) qd[d] = (double)q[qoff + d];
                        if (rope_base > 0.0) rope_vec(qd, (double)q_pos0 + (double)i, D, rope_base);
                        const float* mrow = mask + (long)b * mask_bstride + (long)hq * mask_hstride + (long)i * Skv;
                        const int nvis = visible_keys(i, Sq, Skv, causal);
                        double m = -INFINITY;
                        for (int j = 0; j < Skv; ++j) {
                            if (j >= nvis) {
                                s[j] = -INFINITY;
                                continue;
                            }
                            double dot = 0.0;
                            for (int d = 0; d < D; ++d) dot += qd[d] * Kd[(long)j * D + d];
                            s[j] = scale * dot + (double)mrow[j];
                            if (s[j] > m) m = s[j];
                        }
                        for (int d = 0; d < D; ++d) orow[d] = 0.0;
                        if (m == -INFINITY) {
                            *lrow = -INFINITY;
                            continue;
                        }
                        double l = 0.0;
                        for (int j = 0; j < Skv; ++j) l += exp(s[j] - m);
                        for (int j = 0; j < Skv; ++j) {
                            const double p = exp(s[j] - m) / l;
                            if (p == 0.0) continue;
                            for (int d = 0; d < D; ++d) orow[d] += p * Vd[(long)j * D + d];
                        }
                        *lrow = m + log(l);
                    }
                }
            }
            free(Kd);
            free(Vd);
            free(s);
            free(qd);
        }
    }
    return fail ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Backward at sampled rows and keys of one (batch, kv head) group                             */
/* ------------------------------------------------------------------------------------------ */

/* The same definition as oracle_attn_bwd_f64 ([P1] flash_backward_head: P from the full score row,
 * dP = dO . v_j, D = sum_j p_j dP_j, dS = p (dP - D); dQ = scale sum_j dS_j k_j, dK_j = scale
 * sum_i dS_ij q_i, dV_j = sum_i p_ij dO_i; [P2] the kv head's gradients summed over its q heads
 * and RoPE undone by the negated angle), evaluated only where a full-size problem is checked:
 *   dq_s [g][nrows][D]  dq of every q head of kv head `kvh` of batch `b` at query rows rows[]
 *   dk_s, dv_s [nkeys][D]  dk, dv of that kv head at keys keys[]
 * Every query row of the group is still evaluated in full (its P and D need the whole row); only
 * the sums that are not asked for are skipped.  Rows are split among threads, each with its own
 * partial sums for the sampled keys, added up in thread order at the end.                     */
int oracle_attn_bwd_sampled_f64(const float* q, const float* k, const float* v, const float* dout, int B, int Hq,
                                int Hkv, int Sq, int Skv, int D, double scale, int causal, double rope_base,
                                int q_pos0, int b, int kvh, const int64_t* rows, int nrows, const int64_t* keys,
                                int nkeys, double* dq_s, double* dk_s, double* dv_s) {
    int st = check_dims(B, Hq, Hkv, Sq, Skv, D);
    if (st) return st;
    if (rope_base > 0.0 && D % 2) return ORACLE_ERR_INVALID_ARG;
    if (b < 0 || b >= B || kvh < 0 || kvh >= Hkv || nrows < 0 || nkeys < 0) return ORACLE_ERR_INVALID_ARG;
    for (int r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= Sq) return ORACLE_ERR_INVALID_ARG;
    for (int t = 0; t < nkeys; ++t)
        if (keys[t] < 0 || keys[t] >= Skv) return ORACLE_ERR_INVALID_ARG;
    const int g = Hq / Hkv;
    double* Kd = (double*)malloc(sizeof(double) * (size_t)Skv * D);
    double* Vd = (double*)malloc(sizeof(double) * (size_t)Skv * D);
    int nthr = 1;
#ifdef _OPENMP
    nthr = omp_get_max_threads();
#endif
    double* part = (double*)calloc((size_t)nthr * 2 * (nkeys > 0 ? nkeys : 1) * D, sizeof(double));
    int* slot = (int*)malloc(sizeof(int) * (size_t)(Sq > 0 ? Sq : 1));   /* row -> index in rows[], or -1 */
    if (!Kd || !Vd || !part || !slot) {
        free(Kd), free(Vd), free(part), free(slot);
        return ORACLE_ERR_NOMEM;
    }
    gather_head(k, b, kvh, Skv, Hkv, D, rope_base, Kd);
    gather_head(v, b, kvh, Skv, Hkv, D, 0.0, Vd);
    for (int i = 0; i < Sq; ++i) slot[i] = -1;
    for (int r = 0; r < nrows; ++r) slot[rows[r]] = r;
    for (long e = 0; e < (long)g * nrows * D; ++e) dq_s[e] = 0.0;
    int fail = 0;
#pragma omp parallel
    {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        double* dKp = part + (size_t)tid * 2 * (nkeys > 0 ? nkeys : 1) * D;
        double* dVp = dKp + (size_t)(nkeys > 0 ? nkeys : 1) * D;
        double* s = (double*)malloc(sizeof(double) * (size_t)Skv);
        double* dP = (double*)malloc(sizeof(double) * (size_t)Skv);
        double* qd = (double*)malloc(sizeof(double) * (size_t)D);
        double* go = (double*)malloc(sizeof(double) * (size_t)D);
        double* dqr = (double*)malloc(sizeof(double) * (size_t)D);
        if (!s || !dP || !qd || !go || !dqr) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 4) collapse(2)
            for (int hg = 0; hg < g; ++hg) {
                for (int i = 0; i < Sq; ++i) {
                    const int hq = kvh * g + hg;
                    const long qoff = (((long)b * Sq + i) * Hq + hq) * D;
                    const int nvis = visible_keys(i, Sq, Skv, causal);
                    if (nvis <= 0) continue; /* no gradient through this row; dq stays 0 */
                    for (int d = 0; d < D; ++d) qd[d] = (double)q[qoff + d];
                    if (rope_base > 0.0) rope_vec(qd, (double)q_pos0 + (double)i, D, rope_base);
                    for (int d = 0; d < D; ++d) go[d] = (double)dout[qoff + d];
                    double m = -INFINITY;
                    for (int j = 0; j < nvis; ++j) {
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d) dot += qd[d] * Kd[(long)j * D + d];
                        s[j] = scale * dot;
                        if (s[j] > m) m = s[j];
                    }
                    double l = 0.0;
                    for (int j = 0; j < nvis; ++j) l += exp(s[j] - m);
                    double Dsum = 0.0;
                    for (int j = 0; j < nvis; ++j) {
                        const double p = exp(s[j] - m) / l;
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d) dot += go[d] * Vd[(long)j * D + d];
                        dP[j] = dot;
                        Dsum += p * dot;
                    }
                    if (slot[i] >= 0) {
                        for (int d = 0; d < D; ++d) dqr[d] = 0.0;
                        for (int j = 0; j < nvis; ++j) {
                            const double p = exp(s[j] - m) / l;
                            const double dS = p * (dP[j] - Dsum);
                            for (int d = 0; d < D; ++d) dqr[d] += scale * dS * Kd[(long)j * D + d];
                        }
                        if (rope_base > 0.0) rope_vec(dqr, -((double)q_pos0 + (double)i), D, rope_base);
                        double* dst = dq_s + ((long)hg * nrows + slot[i]) * D;
                        for (int d = 0; d < D; ++d) dst[d] = dqr[d];
                    }
                    for (int t = 0; t < nkeys; ++t) {
                        const long j = keys[t];
                        if (j >= nvis) continue;
                        const double p = exp(s[j] - m) / l;
                        const double dS = p * (dP[j] - Dsum);
                        for (int d = 0; d < D; ++d) {
                            dKp[(long)t * D + d] += scale * dS * qd[d];
                            dVp[(long)t * D + d] += p * go[d];
                        }
                    }
                }
            }
        }
        free(s), free(dP), free(qd), free(go), free(dqr);
    }
    if (!fail) {
        for (int t = 0; t < nkeys; ++t) {
            double* dkr = dk_s + (long)t * D;
            double* dvr = dv_s + (long)t * D;
            for (int d = 0; d < D; ++d) dkr[d] = dvr[d] = 0.0;
            for (int th = 0; th < nthr; ++th) {
                const double* dKp = part + (size_t)th * 2 * nkeys * D;
                const double* dVp = dKp + (size_t)nkeys * D;
                for (int d = 0; d < D; ++d) {
                    dkr[d] += dKp[(long)t * D + d];
                    dvr[d] += dVp[(long)t * D + d];
                }
            }
            if (rope_base > 0.0) rope_vec(dkr, -(double)keys[t], D, rope_base);
        }
    }
    free(Kd), free(Vd), free(part), free(slot);
    return fail ? ORACLE_ERR_NOMEM : ORACLE_OK;
}
