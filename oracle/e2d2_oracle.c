/*
 * e2d2_oracle.c -- plain CPU oracle for the E2D2 fused block-diffusion attention.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code, header,
 * table or constant with the CUDA path.
 *
 * Sources (page title, section):
 *   [E2D2 notes]  "Encoder-Decoder Diffusion Language Models for Efficient Training and
 *                 Inference" (paper notes), sec. 2 "two connection variants",
 *                 sec. 3 "sampling algorithm", sec. 4 "training algorithm" (+ FLOPs table).
 *   [BD3LM blog]  "Block Diffusion: Interpolating Between Autoregressive and Diffusion
 *                 Language Models", sec. 2 "core insight", sec. 3 "block decomposition".
 *
 * What is computed (the plain definition, in fp64, from the exact bf16 input values that
 * the caller passes as float32):
 *   for every batch b and query head h (kv head g = h / (Hq/Hkv)):
 *     s_ij   = scale * sum_k q_ik k_jk            for every key j the mask allows
 *     m_i    = max_j s_ij
 *     l_i    = sum_j exp(s_ij - m_i)
 *     out_i  = sum_j exp(s_ij - m_i) v_j / l_i
 *     lse_i  = m_i + ln(l_i)                      (natural log of the scaled scores)
 *
 * The masks are explicit boolean matrices built from the words of [E2D2 notes, sec. 4]:
 *   encoder:  a clean token attends to the tokens of its own block and of earlier blocks;
 *   decoder:  the key set spans 2L positions -- the L encoder (clean) representations
 *             followed by the L decoder (noised) positions; a noised token attends to its
 *             own block of noised tokens and to the encoder representations of the clean
 *             blocks strictly before its own;
 *   sampling: [E2D2 notes, sec. 3] the S noised queries of the block being denoised see
 *             the whole cached clean prefix (P keys) and their own block (S keys).
 * Block index of position i is floor(i / S) ([BD3LM blog, sec. 3]: the sequence is cut
 * into consecutive blocks of S tokens).
 *
 * No tiling, no online softmax, no reordering: one query at a time, keys in mask order.
 * Layouts (all row-major, head_dim innermost):
 *   q, k, v, out  [B][H][len][d];  lse [B][Hq][len];  KV cache [B][Hkv][capacity][d].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Block index of a position: consecutive blocks of S tokens ([BD3LM blog, sec. 3]). */
static int block_of(int pos, int S) { return pos / S; }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of the parallel loops that follow on the calling thread (n >= 1; ignored without
 * OpenMP).  Lets a caller that was started with OMP_NUM_THREADS=1 use every host core. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Encoder block-causal mask [L][L] ([E2D2 notes, sec. 4]): allowed(i, j) iff the block of
 * key j is the block of query i or an earlier one. */
void oracle_mask_encoder(int L, int S, uint8_t* mask) {
    for (int i = 0; i < L; ++i)
        for (int j = 0; j < L; ++j)
            mask[(size_t)i * L + j] = (uint8_t)(block_of(j, S) <= block_of(i, S));
}

/* Decoder training mask [L][2L] ([E2D2 notes, sec. 4]).  Columns 0..L-1 are the encoder
 * (clean) representations, columns L..2L-1 the decoder (noised) positions. */
void oracle_mask_decoder(int L, int S, uint8_t* mask) {
    const size_t W = (size_t)2 * L;
    for (int i = 0; i < L; ++i) {
        for (int j = 0; j < L; ++j)  /* earlier clean blocks only */
            mask[i * W + j] = (uint8_t)(block_of(j, S) < block_of(i, S));
        for (int j = 0; j < L; ++j)  /* own noised block only */
            mask[i * W + L + j] = (uint8_t)(block_of(j, S) == block_of(i, S));
    }
}

/* Sampling-step mask [S][P+S] ([E2D2 notes, sec. 3]): every noised query of the block
 * sees the whole cached prefix and its whole own block. */
void oracle_mask_sample(int S, int P, uint8_t* mask) {
    for (int i = 0; i < S; ++i)
        for (int j = 0; j < P + S; ++j)
            mask[(size_t)i * (P + S) + j] = 1;
}

/* Masked softmax attention of nq queries over nk keys, all in fp64.
 * q: [nq][d] (float), keys/vals: [nk][d] (double), mask: [nq][nk].
 * Returns 0, or -1 if some query row has no allowed key. */
static int attend(const float* q, const double* keys, const double* vals, const uint8_t* mask,
                  int nq, int nk, int d, double scale, double* out, double* lse) {
    double* s = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    if (!s) return -2;
    int rc = 0;
    for (int i = 0; i < nq; ++i) {
        const uint8_t* mrow = mask + (size_t)i * nk;
        double m = -INFINITY;
        int any = 0;
        for (int j = 0; j < nk; ++j) {
            if (!mrow[j]) continue;
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += (double)q[(size_t)i * d + c] * keys[(size_t)j * d + c];
            s[j] = scale * acc;
            if (!any || s[j] > m) m = s[j];
            any = 1;
        }
        double* o = out + (size_t)i * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (!any) {
            lse[i] = -INFINITY;
            rc = -1;
            continue;
        }
        double l = 0.0;
        for (int j = 0; j < nk; ++j) {
            if (!mrow[j]) continue;
            double p = exp(s[j] - m);
            l += p;
            for (int c = 0; c < d; ++c) o[c] += p * vals[(size_t)j * d + c];
        }
        for (int c = 0; c < d; ++c) o[c] /= l;
        lse[i] = m + log(l);
    }
    free(s);
    return rc;
}

static double resolve_scale(double scale, int d) { return scale > 0.0 ? scale : 1.0 / sqrt((double)d); }

/* Copy n rows of d floats into a double buffer. */
static void rows_to_double(const float* src, int n, int d, double* dst) {
    for (size_t t = 0; t < (size_t)n * d; ++t) dst[t] = (double)src[t];
}

/* Encoder block-causal self-attention over clean tokens ([E2D2 notes, sec. 4]).
 * q: [B][Hq][L][d]; k, v: [B][Hkv][L][d]; out: [B][Hq][L][d]; lse: [B][Hq][L]. */
int oracle_encoder(const float* q, const float* k, const float* v, int B, int Hq, int Hkv,
                   int L, int S, int d, double scale, double* out, double* lse) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L < 0 || S <= 0 || d <= 0) return -3;
    const int G = Hq / Hkv;
    scale = resolve_scale(scale, d);
    uint8_t* mask = (uint8_t*)malloc((size_t)L * L + 1);
    if (!mask) return -2;
    oracle_mask_encoder(L, S, mask);
    int rc = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : rc)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            double* kd = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));
            double* vd = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));
            if (!kd || !vd) { rc |= 2; free(kd); free(vd); continue; }
            rows_to_double(k + ((size_t)b * Hkv + g) * L * d, L, d, kd);
            rows_to_double(v + ((size_t)b * Hkv + g) * L * d, L, d, vd);
            const size_t qo = ((size_t)b * Hq + h) * L;
            if (attend(q + qo * d, kd, vd, mask, L, L, d, scale, out + qo * d, lse + qo)) rc |= 1;
            free(kd);
            free(vd);
        }
    }
    free(mask);
    return rc ? -1 : 0;
}

/* Decoder fused self+cross attention, training mode ([E2D2 notes, sec. 2 and 4]).
 * q: [B][Hq][L][d] (noised queries); k_enc, v_enc: [B][Hkv][L][d] (encoder side);
 * k_dec, v_dec: [B][Hkv][L][d] (decoder side).  The 2L-key set is k_enc rows then k_dec rows. */
int oracle_decoder_train(const float* q, const float* k_enc, const float* v_enc,
                         const float* k_dec, const float* v_dec, int B, int Hq, int Hkv,
                         int L, int S, int d, double scale, double* out, double* lse) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L < 0 || S <= 0 || d <= 0) return -3;
    const int G = Hq / Hkv;
    scale = resolve_scale(scale, d);
    const size_t W = (size_t)2 * L;
    uint8_t* mask = (uint8_t*)malloc((size_t)L * W + 1);
    if (!mask) return -2;
    oracle_mask_decoder(L, S, mask);
    int rc = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : rc)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            double* kd = (double*)malloc(sizeof(double) * (W * d + 1));
            double* vd = (double*)malloc(sizeof(double) * (W * d + 1));
            if (!kd || !vd) { rc |= 2; free(kd); free(vd); continue; }
            const size_t ko = ((size_t)b * Hkv + g) * L * d;
            rows_to_double(k_enc + ko, L, d, kd);
            rows_to_double(k_dec + ko, L, d, kd + (size_t)L * d);
            rows_to_double(v_enc + ko, L, d, vd);
            rows_to_double(v_dec + ko, L, d, vd + (size_t)L * d);
            const size_t qo = ((size_t)b * Hq + h) * L;
            if (attend(q + qo * d, kd, vd, mask, L, (int)W, d, scale, out + qo * d, lse + qo)) rc |= 1;
            free(kd);
            free(vd);
        }
    }
    free(mask);
    return rc ? -1 : 0;
}

/* BD3LM's training attention over 2L tokens, the comparison point of [E2D2 notes, sec. 1 and 4]:
 * a decoder-only block diffusion model whose training forward takes the noised and the clean copy
 * of the sequence together (2L tokens; attention cost 4ND(L^2 + LS) in the FLOPs table).
 * Positions 0..L-1 hold the noised copy, L..2L-1 the clean copy.  The pages give the cost, not the
 * mask; the reading taken: a noised token sees the noised tokens of its own block and the clean
 * tokens of the blocks strictly before its own, a clean token the clean tokens of its own and
 * earlier blocks; no clean token sees a noised one.  mask: [2L][2L]. */
void oracle_mask_bd3lm(int L, int S, uint8_t* mask) {
    const size_t W = (size_t)2 * L;
    for (int i = 0; i < 2 * L; ++i) {
        const int noised_row = i < L;
        const int bi = block_of(noised_row ? i : i - L, S);
        for (int j = 0; j < 2 * L; ++j) {
            const int noised_col = j < L;
            const int bj = block_of(noised_col ? j : j - L, S);
            uint8_t a;
            if (noised_row) a = noised_col ? (bj == bi) : (bj < bi);
            else a = noised_col ? 0 : (bj <= bi);
            mask[(size_t)i * W + j] = a;
        }
    }
}

/* q, k, v: [B][H][2L][d] (noised rows first); out [B][Hq][2L][d]; lse [B][Hq][2L]. */
int oracle_bd3lm_train(const float* q, const float* k, const float* v, int B, int Hq, int Hkv, int L, int S,
                       int d, double scale, double* out, double* lse) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L < 0 || S <= 0 || d <= 0) return -3;
    const int G = Hq / Hkv;
    scale = resolve_scale(scale, d);
    const size_t W = (size_t)2 * L;
    uint8_t* mask = (uint8_t*)malloc(W * W + 1);
    if (!mask) return -2;
    oracle_mask_bd3lm(L, S, mask);
    int rc = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : rc)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            double* kd = (double*)malloc(sizeof(double) * (W * d + 1));
            double* vd = (double*)malloc(sizeof(double) * (W * d + 1));
            if (!kd || !vd) { rc |= 2; free(kd); free(vd); continue; }
            rows_to_double(k + ((size_t)b * Hkv + g) * W * d, (int)W, d, kd);
            rows_to_double(v + ((size_t)b * Hkv + g) * W * d, (int)W, d, vd);
            const size_t qo = ((size_t)b * Hq + h) * W;
            if (attend(q + qo * d, kd, vd, mask, (int)W, (int)W, d, scale, out + qo * d, lse + qo)) rc |= 1;
            free(kd);
            free(vd);
        }
    }
    free(mask);
    return rc ? -1 : 0;
}

/* Decoder sampling step ([E2D2 notes, sec. 3]): the S noised queries of the current block
 * attend to the cached clean prefix (first P rows of the cache) and to their own block.
 * q: [B][Hq][S][d]; k_cache, v_cache: [B][Hkv][capacity][d]; k_blk, v_blk: [B][Hkv][S][d]. */
int oracle_decoder_sample(const float* q, const float* k_cache, const float* v_cache, int capacity,
                          int P, const float* k_blk, const float* v_blk, int B, int Hq, int Hkv,
                          int S, int d, double scale, double* out, double* lse) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || S <= 0 || d <= 0 || P < 0 || P > capacity)
        return -3;
    const int G = Hq / Hkv;
    scale = resolve_scale(scale, d);
    const int nk = P + S;
    uint8_t* mask = (uint8_t*)malloc((size_t)S * nk + 1);
    if (!mask) return -2;
    oracle_mask_sample(S, P, mask);
    int rc = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : rc)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            double* kd = (double*)malloc(sizeof(double) * ((size_t)nk * d + 1));
            double* vd = (double*)malloc(sizeof(double) * ((size_t)nk * d + 1));
            if (!kd || !vd) { rc |= 2; free(kd); free(vd); continue; }
            const size_t co = ((size_t)b * Hkv + g) * (size_t)capacity * d;
            const size_t bo = ((size_t)b * Hkv + g) * (size_t)S * d;
            rows_to_double(k_cache + co, P, d, kd);
            rows_to_double(k_blk + bo, S, d, kd + (size_t)P * d);
            rows_to_double(v_cache + co, P, d, vd);
            rows_to_double(v_blk + bo, S, d, vd + (size_t)P * d);
            const size_t qo = ((size_t)b * Hq + h) * S;
            if (attend(q + qo * d, kd, vd, mask, S, nk, d, scale, out + qo * d, lse + qo)) rc |= 1;
            free(kd);
            free(vd);
        }
    }
    free(mask);
    return rc ? -1 : 0;
}

/* Sampling step over a batch whose sequences have decoded different numbers of clean tokens
 * (ragged prefixes): the plainest extension of [E2D2 notes, sec. 3] to such a batch -- batch
 * entry b's S noised queries see the first P[b] rows of its own cache and its own block, exactly
 * the single-prefix step with P = P[b].  Each P[b] lies in [0, capacity].  Layouts as for
 * oracle_decoder_sample. */
int oracle_decoder_sample_ragged(const float* q, const float* k_cache, const float* v_cache, int capacity,
                                 const int* P, const float* k_blk, const float* v_blk, int B, int Hq,
                                 int Hkv, int S, int d, double scale, double* out, double* lse) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || S <= 0 || d <= 0 || capacity < 0 || (B > 0 && !P))
        return -3;
    for (int b = 0; b < B; ++b)
        if (P[b] < 0 || P[b] > capacity) return -3;
    const int G = Hq / Hkv;
    scale = resolve_scale(scale, d);
    int rc = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : rc)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < Hq; ++h) {
            const int g = h / G;
            const int Pb = P[b];
            const int nk = Pb + S;
            uint8_t* mask = (uint8_t*)malloc((size_t)S * nk + 1);
            double* kd = (double*)malloc(sizeof(double) * ((size_t)nk * d + 1));
            double* vd = (double*)malloc(sizeof(double) * ((size_t)nk * d + 1));
            if (!mask || !kd || !vd) { rc |= 2; free(mask); free(kd); free(vd); continue; }
            oracle_mask_sample(S, Pb, mask);
            const size_t co = ((size_t)b * Hkv + g) * (size_t)capacity * d;
            const size_t bo = ((size_t)b * Hkv + g) * (size_t)S * d;
            rows_to_double(k_cache + co, Pb, d, kd);
            rows_to_double(k_blk + bo, S, d, kd + (size_t)Pb * d);
            rows_to_double(v_cache + co, Pb, d, vd);
            rows_to_double(v_blk + bo, S, d, vd + (size_t)Pb * d);
            const size_t qo = ((size_t)b * Hq + h) * S;
            if (attend(q + qo * d, kd, vd, mask, S, nk, d, scale, out + qo * d, lse + qo)) rc |= 1;
            free(mask);
            free(kd);
            free(vd);
        }
    }
    return rc ? -1 : 0;
}

/* KV-cache append ([E2D2 notes, sec. 3]: once a block is decoded the encoder absorbs it and
 * the cache grows by that block): rows P..P+S_new-1 of every (b, kv head) cache become the
 * new rows.  Caches are [B][Hkv][capacity][d]; new rows [B][Hkv][S_new][d].  Values are
 * copied bit for bit (they are bf16 payloads carried as uint16). */
int oracle_kv_append(uint16_t* k_cache, uint16_t* v_cache, int capacity, int P,
                     const uint16_t* k_new, const uint16_t* v_new, int S_new, int B, int Hkv, int d) {
    if (P < 0 || S_new < 0 || P + S_new > capacity || B < 0 || Hkv <= 0 || d <= 0) return -3;
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < Hkv; ++g)
            for (int r = 0; r < S_new; ++r) {
                const size_t dst = (((size_t)b * Hkv + g) * capacity + P + r) * d;
                const size_t src = (((size_t)b * Hkv + g) * S_new + r) * d;
                memcpy(k_cache + dst, k_new + src, sizeof(uint16_t) * d);
                memcpy(v_cache + dst, v_new + src, sizeof(uint16_t) * d);
            }
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * Backward of the train calls ([E2D2 notes, sec. 4]: one encoder pass and one decoder pass
 * with custom masks train all blocks; the page gives no backward, so this is the plain
 * derivative of those passes that a gradient step needs).  From the chain
 * rule applied to the definition at the top of this file, with p_ij = exp(s_ij - lse_i) over
 * the allowed keys of row i and dout the gradient of the loss with respect to out:
 *   dv_j   += sum_i p_ij dout_i
 *   dp_ij   = dout_i . v_j
 *   ds_ij   = p_ij (dp_ij - sum_j' p_ij' dp_ij')
 *   dq_i    = scale sum_j ds_ij k_j
 *   dk_j   += scale sum_i ds_ij q_i
 * The forward quantities are recomputed here (no reuse of the kernel's LSE).  dk, dv of a kv
 * head collect the contributions of all G query heads that share it.
 * --------------------------------------------------------------------------------------- */

/* One query head: nq queries over nk keys.  Writes dq [nq][d], adds into dk, dv [nk][d]. */
static int attend_backward(const float* q, const double* keys, const double* vals, const uint8_t* mask,
                           const float* dout, int nq, int nk, int d, double scale, double* dq,
                           double* dk, double* dv) {
    double* s = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    double* dp = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    if (!s || !dp) { free(s); free(dp); return -2; }
    int rc = 0;
    for (int i = 0; i < nq; ++i) {
        const uint8_t* mrow = mask + (size_t)i * nk;
        const float* qi = q + (size_t)i * d;
        const float* gi = dout + (size_t)i * d;
        double* dqi = dq + (size_t)i * d;
        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
        double m = -INFINITY;
        int any = 0;
        for (int j = 0; j < nk; ++j) {
            if (!mrow[j]) continue;
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += (double)qi[c] * keys[(size_t)j * d + c];
            s[j] = scale * acc;
            if (!any || s[j] > m) m = s[j];
            any = 1;
        }
        if (!any) { rc = -1; continue; }
        double l = 0.0;
        for (int j = 0; j < nk; ++j)
            if (mrow[j]) l += exp(s[j] - m);
        const double lse = m + log(l);
        double dsum = 0.0;  /* sum_j p_ij dp_ij */
        for (int j = 0; j < nk; ++j) {
            if (!mrow[j]) continue;
            const double p = exp(s[j] - lse);
            double acc = 0.0;
            for (int c = 0; c < d; ++c) {
                acc += (double)gi[c] * vals[(size_t)j * d + c];
                dv[(size_t)j * d + c] += p * (double)gi[c];
            }
            dp[j] = acc;
            dsum += p * acc;
        }
        for (int j = 0; j < nk; ++j) {
            if (!mrow[j]) continue;
            const double ds = exp(s[j] - lse) * (dp[j] - dsum);
            for (int c = 0; c < d; ++c) {
                dqi[c] += scale * ds * keys[(size_t)j * d + c];
                dk[(size_t)j * d + c] += scale * ds * (double)qi[c];
            }
        }
    }
    free(s);
    free(dp);
    return rc;
}

/* Encoder backward.  q, dout: [B][Hq][L][d]; k, v: [B][Hkv][L][d];
 * dq: [B][Hq][L][d]; dk, dv: [B][Hkv][L][d] (fp64, overwritten). */
int oracle_encoder_backward(const float* q, const float* k, const float* v, const float* dout, int B, int Hq,
                            int Hkv, int L, int S, int d, double scale, double* dq, double* dk, double* dv) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L < 0 || S <= 0 || d <= 0) return -3;
    const int G = Hq / Hkv;
    scale = resolve_scale(scale, d);
    uint8_t* mask = (uint8_t*)malloc((size_t)L * L + 1);
    if (!mask) return -2;
    oracle_mask_encoder(L, S, mask);
    int rc = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : rc)
    for (int b = 0; b < B; ++b) {
        for (int g = 0; g < Hkv; ++g) {
            const size_t ko = ((size_t)b * Hkv + g) * L * d;
            double* kd = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));
            double* vd = (double*)malloc(sizeof(double) * ((size_t)L * d + 1));
            if (!kd || !vd) { rc |= 2; free(kd); free(vd); continue; }
            rows_to_double(k + ko, L, d, kd);
            rows_to_double(v + ko, L, d, vd);
            for (size_t t = 0; t < (size_t)L * d; ++t) { dk[ko + t] = 0.0; dv[ko + t] = 0.0; }
            for (int h = g * G; h < (g + 1) * G; ++h) {
                const size_t qo = ((size_t)b * Hq + h) * L * d;
                if (attend_backward(q + qo, kd, vd, mask, dout + qo, L, L, d, scale, dq + qo, dk + ko, dv + ko))
                    rc |= 1;
            }
            free(kd);
            free(vd);
        }
    }
    free(mask);
    return rc ? -1 : 0;
}

/* Decoder-train backward over the 2L keys (k_enc rows, then k_dec rows).  q, dout:
 * [B][Hq][L][d]; k_*, v_*: [B][Hkv][L][d]; dq: [B][Hq][L][d]; dk_enc, dv_enc, dk_dec,
 * dv_dec: [B][Hkv][L][d] (fp64, overwritten). */
int oracle_decoder_train_backward(const float* q, const float* k_enc, const float* v_enc, const float* k_dec,
                                  const float* v_dec, const float* dout, int B, int Hq, int Hkv, int L, int S,
                                  int d, double scale, double* dq, double* dk_enc, double* dv_enc,
                                  double* dk_dec, double* dv_dec) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || L < 0 || S <= 0 || d <= 0) return -3;
    const int G = Hq / Hkv;
    scale = resolve_scale(scale, d);
    const size_t W = (size_t)2 * L;
    uint8_t* mask = (uint8_t*)malloc((size_t)L * W + 1);
    if (!mask) return -2;
    oracle_mask_decoder(L, S, mask);
    int rc = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : rc)
    for (int b = 0; b < B; ++b) {
        for (int g = 0; g < Hkv; ++g) {
            const size_t ko = ((size_t)b * Hkv + g) * L * d;
            double* kd = (double*)malloc(sizeof(double) * (W * d + 1));
            double* vd = (double*)malloc(sizeof(double) * (W * d + 1));
            double* dkd = (double*)calloc(W * d + 1, sizeof(double));
            double* dvd = (double*)calloc(W * d + 1, sizeof(double));
            if (!kd || !vd || !dkd || !dvd) { rc |= 2; free(kd); free(vd); free(dkd); free(dvd); continue; }
            rows_to_double(k_enc + ko, L, d, kd);
            rows_to_double(k_dec + ko, L, d, kd + (size_t)L * d);
            rows_to_double(v_enc + ko, L, d, vd);
            rows_to_double(v_dec + ko, L, d, vd + (size_t)L * d);
            for (int h = g * G; h < (g + 1) * G; ++h) {
                const size_t qo = ((size_t)b * Hq + h) * L * d;
                if (attend_backward(q + qo, kd, vd, mask, dout + qo, L, (int)W, d, scale, dq + qo, dkd, dvd))
                    rc |= 1;
            }
            memcpy(dk_enc + ko, dkd, sizeof(double) * (size_t)L * d);
            memcpy(dk_dec + ko, dkd + (size_t)L * d, sizeof(double) * (size_t)L * d);
            memcpy(dv_enc + ko, dvd, sizeof(double) * (size_t)L * d);
            memcpy(dv_dec + ko, dvd + (size_t)L * d, sizeof(double) * (size_t)L * d);
            free(kd);
            free(vd);
            free(dkd);
            free(dvd);
        }
    }
    free(mask);
    return rc ? -1 : 0;
}
