/*
 * pa_oracle.c -- float64 CPU oracle for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow statement of what the
 * GPU library computes.  Only the test suite, the smoke entry and the bench's
 * CPU-baseline leg may load it; the product path never does.  It shares no
 * code, header or table with the CUDA library.
 *
 * What is computed (one query token per sequence, one output row per query head):
 *
 *   Attention itself.  Every query vector is scored against every key of its
 *   sequence and the values are then mixed with the softmax of those scores
 *   (page "wenku.it search: paged attention", Transformer-introduction snippet on
 *   per-word attention: each Q scores every K, features are then redistributed by
 *   the scores; page "wenku.it search: Multi-head Latent Attention (MLA)",
 *   Transformer encoder snippet: multi-head attention is h independent
 *   self-attentions, its formula is cut off after its arguments, so the standard
 *   softmax(q K^T * scale) V is taken; page "bjpcjp.github.io: llms-attention",
 *   softmax-attention abstract: outputs are convex combinations of the values,
 *   obtained by a row-wise reduction along the sequence).
 *
 *   Paging.  Keys and values live in fixed-size physical blocks; a per-sequence
 *   block table maps logical block j to a physical block id (page "wenku.it
 *   search: paged attention", vLLM PagedAttention snippet on managing attention
 *   key/value memory).  Logical token t of sequence b is row t % bs of physical
 *   block block_table[b][t / bs].
 *
 *   Split + log-sum-exp merge.  Flash-Decoding splits keys/values into blocks
 *   along the sequence, attends to each block separately while recording the
 *   log-sum-exp of each softmax row, then rescales and reduces the per-block
 *   outputs (page "cidian.kuaisou.com: flash decoding ++", snippets describing
 *   the three Flash-Decoding steps and the rescale-and-combine idea).  The
 *   unsplit definition is the reference result; the split form is kept here,
 *   separately written, only so that the tests can check that the two agree.
 *
 *   MLA.  One compressed latent vector per token is shared by all heads (page
 *   "wenku.it search: Multi-head Latent Attention (MLA)", DeepSeek-V2 abstract on
 *   compressing the KV cache into a latent vector).  The pages print no MLA
 *   formula; the absorbed-decode form used here scores q (Dk wide) against the
 *   whole latent row and takes the first Dv latent dims as the value.
 *
 * Readings where the pages are silent (each is a parameter or documented choice):
 *   - K/V cache layout: [num_blocks][num_kv_heads][block_size][head_dim] (HND).
 *   - MLA latent layout: [num_blocks][block_size][Dk].
 *   - GQA head map: query head h reads kv head h / (Hq / Hkv).
 *   - natural exp with max subtraction; a sequence with context length 0 gives
 *     an all-zero output row.
 *
 * All arithmetic is IEEE double.  Inputs are raw 16-bit patterns (binary16 or
 * bfloat16) or, for a float8 KV cache, E4M3 bytes, decoded exactly to double by
 * the routines below.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { PA_ORACLE_F16 = 0, PA_ORACLE_BF16 = 1 };

enum {
  PA_ORACLE_OK = 0,
  PA_ORACLE_BAD_ARG = 1,
  PA_ORACLE_BAD_BLOCK = 2,
  PA_ORACLE_NO_MEMORY = 3
};

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double pa_oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double mag;
  if (e == 0) {
    mag = ldexp((double)f, -24);               /* subnormal: f * 2^-14 * 2^-10 */
  } else if (e == 31) {
    mag = f ? NAN : INFINITY;
  } else {
    mag = ldexp((double)(1024 + f), e - 25);   /* (1 + f/1024) * 2^(e-15) */
  }
  return sign ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE binary32 pattern. */
double pa_oracle_bf16_to_f64(uint16_t h) {
  uint32_t bits = (uint32_t)h << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Record a failure code from inside a parallel loop (any non-zero code wins). */
/*
 * 8-bit float E4M3 (the OCP 8-bit floating point format's E4M3 encoding): 1 sign
 * bit, 4 exponent bits (bias 7), 3 fraction bits; exponent 0 holds subnormals
 * m x 2^-9; there is no infinity, and the one pattern with exponent 15 and
 * fraction 7 is NaN (so the largest finite magnitude is 1.75 x 2^8 = 448).
 * The pages only name FP8 as a Hopper capability (page "bjpcjp.github.io:
 * llms-attention", FlashAttention-3 teaser: FP8 low precision); this standard
 * encoding with one scale per tensor is the plainest reading of an FP8 KV cache.
 */
double pa_oracle_e4m3_to_f64(uint8_t c) {
  const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);
  else v = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -v : v;
}

static void set_status(int *status, int code) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
  *status = code;
}

static double decode16(uint16_t v, int dtype) {
  return dtype == PA_ORACLE_BF16 ? pa_oracle_bf16_to_f64(v) : pa_oracle_f16_to_f64(v);
}

/* Physical block of logical token t of sequence b, or -1 when out of range. */
static long block_of(const int32_t *block_table, int mbs, int nb, int bs, int b, int t) {
  int j = t / bs;
  if (j >= mbs) return -1;
  long blk = block_table[(long)b * mbs + j];
  if (blk < 0 || blk >= nb) return -1;
  return blk;
}

/*
 * Softmax-weighted sum over n gathered rows: out[dv] = sum_t p_t V[t][dv] / sum_t p_t
 * with p_t = exp(s_t - max s).  s has n entries, V is n x dv (row-major).
 */
static void softmax_mix(int n, const double *s, const double *V, int dv, double *out) {
  double m = -INFINITY;
  for (int t = 0; t < n; ++t) if (s[t] > m) m = s[t];
  double Z = 0.0;
  for (int d = 0; d < dv; ++d) out[d] = 0.0;
  for (int t = 0; t < n; ++t) {
    double p = exp(s[t] - m);
    Z += p;
    for (int d = 0; d < dv; ++d) out[d] += p * V[(long)t * dv + d];
  }
  for (int d = 0; d < dv; ++d) out[d] /= Z;
}

/*
 * GQA / MHA / MQA paged decode, the definition written out.
 *
 * q            [B][Hq][D]            raw 16-bit
 * k_cache      [NB][Hkv][bs][D]      raw 16-bit
 * v_cache      [NB][Hkv][bs][D]      raw 16-bit
 * block_table  [B][mbs]              int32 (entries past ceil(ctx/bs) are never read)
 * context_lens [B]                   int32
 * pairs        optional list of npairs (b, h) pairs (2*npairs ints); NULL = all B*Hq
 * out          [npairs or B*Hq][D]   double
 */
int pa_oracle_decode(int B, int Hq, int Hkv, int D, int bs, int mbs, int nb, int dtype,
                     const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                     const int32_t *block_table, const int32_t *context_lens, double scale,
                     const int32_t *pairs, int npairs, double *out, int nthreads) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0 || mbs < 0 || nb < 0)
    return PA_ORACLE_BAD_ARG;
  const int G = Hq / Hkv;
  const long n_out = pairs ? (long)npairs : (long)B * Hq;
  int status = PA_ORACLE_OK;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (long i = 0; i < n_out; ++i) {
    int b = pairs ? pairs[2 * i] : (int)(i / Hq);
    int h = pairs ? pairs[2 * i + 1] : (int)(i % Hq);
    double *o = out + i * D;
    if (b < 0 || b >= B || h < 0 || h >= Hq) { set_status(&status, PA_ORACLE_BAD_ARG); continue; }
    int n = context_lens[b];
    if (n < 0 || (long)n > (long)mbs * bs) { set_status(&status, PA_ORACLE_BAD_ARG); continue; }
    if (n == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
    int g = h / G;
    double *qd = malloc(sizeof(double) * D);
    double *s = malloc(sizeof(double) * n);
    double *V = malloc(sizeof(double) * (size_t)n * D);
    if (!qd || !s || !V) { free(qd); free(s); free(V); set_status(&status, PA_ORACLE_NO_MEMORY); continue; }
    for (int d = 0; d < D; ++d) qd[d] = decode16(q[((long)b * Hq + h) * D + d], dtype);
    int bad = 0;
    for (int t = 0; t < n; ++t) {
      long blk = block_of(block_table, mbs, nb, bs, b, t);
      if (blk < 0) { bad = 1; break; }
      long row = ((blk * Hkv + g) * bs + t % bs) * (long)D;
      double acc = 0.0;
      for (int d = 0; d < D; ++d) {
        acc += qd[d] * decode16(k_cache[row + d], dtype);
        V[(long)t * D + d] = decode16(v_cache[row + d], dtype);
      }
      s[t] = scale * acc;
    }
    if (bad) set_status(&status, PA_ORACLE_BAD_BLOCK);
    else softmax_mix(n, s, V, D, o);
    free(qd); free(s); free(V);
  }
  return status;
}

/*
 * GQA / MHA / MQA paged decode over a float8 KV cache: k_cache / v_cache hold E4M3
 * codes (one byte each, layout as pa_oracle_decode) and the key / value is the
 * decoded code times k_scale / v_scale; q is raw 16-bit of q_dtype.  Otherwise the
 * same definition as pa_oracle_decode (output [npairs or B*Hq][D] double).
 */
int pa_oracle_decode_kv8(int B, int Hq, int Hkv, int D, int bs, int mbs, int nb, int q_dtype,
                         const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                         double k_scale, double v_scale, const int32_t *block_table,
                         const int32_t *context_lens, double scale, const int32_t *pairs,
                         int npairs, double *out, int nthreads) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0 || mbs < 0 || nb < 0)
    return PA_ORACLE_BAD_ARG;
  const int G = Hq / Hkv;
  const long n_out = pairs ? (long)npairs : (long)B * Hq;
  int status = PA_ORACLE_OK;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (long i = 0; i < n_out; ++i) {
    int b = pairs ? pairs[2 * i] : (int)(i / Hq);
    int h = pairs ? pairs[2 * i + 1] : (int)(i % Hq);
    double *o = out + i * D;
    if (b < 0 || b >= B || h < 0 || h >= Hq) { set_status(&status, PA_ORACLE_BAD_ARG); continue; }
    int n = context_lens[b];
    if (n < 0 || (long)n > (long)mbs * bs) { set_status(&status, PA_ORACLE_BAD_ARG); continue; }
    if (n == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
    int g = h / G;
    double *qd = malloc(sizeof(double) * D);
    double *s = malloc(sizeof(double) * n);
    double *V = malloc(sizeof(double) * (size_t)n * D);
    if (!qd || !s || !V) { free(qd); free(s); free(V); set_status(&status, PA_ORACLE_NO_MEMORY); continue; }
    for (int d = 0; d < D; ++d) qd[d] = decode16(q[((long)b * Hq + h) * D + d], q_dtype);
    int bad = 0;
    for (int t = 0; t < n; ++t) {
      long blk = block_of(block_table, mbs, nb, bs, b, t);
      if (blk < 0) { bad = 1; break; }
      long row = ((blk * Hkv + g) * bs + t % bs) * (long)D;
      double acc = 0.0;
      for (int d = 0; d < D; ++d) {
        acc += qd[d] * (pa_oracle_e4m3_to_f64(k_cache[row + d]) * k_scale);
        V[(long)t * D + d] = pa_oracle_e4m3_to_f64(v_cache[row + d]) * v_scale;
      }
      s[t] = scale * acc;
    }
    if (bad) set_status(&status, PA_ORACLE_BAD_BLOCK);
    else softmax_mix(n, s, V, D, o);
    free(qd); free(s); free(V);
  }
  return status;
}

/*
 * Index-list paged decode: each sequence attends over a given list of its token
 * positions instead of [0, context length) -- the dense kernel behind sparse
 * attention that keeps only selected entries (page "bjpcjp.github.io:
 * llms-attention", DeepSeek-V4 explainer: a top-k indexer keeps the top 1024
 * entries per query, and HCA attends densely over all kept entries).  The
 * selection itself is an input.
 *
 * token_index  [B][max_sel] int32: positions, each < mbs * bs (a position's block
 *              is block_table[b][pos / bs], row pos % bs); entries past n_sel[b]
 *              are never read.  A position listed twice counts twice.
 * n_sel        [B] int32: number of selected positions (0 = all-zero output row).
 * Everything else as pa_oracle_decode.
 */
int pa_oracle_decode_indexed(int B, int Hq, int Hkv, int D, int bs, int mbs, int nb, int dtype,
                             const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                             const int32_t *block_table, const int32_t *token_index,
                             int max_sel, const int32_t *n_sel, double scale,
                             const int32_t *pairs, int npairs, double *out, int nthreads) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0 || mbs < 0 || nb < 0 ||
      max_sel < 0)
    return PA_ORACLE_BAD_ARG;
  const int G = Hq / Hkv;
  const long n_out = pairs ? (long)npairs : (long)B * Hq;
  int status = PA_ORACLE_OK;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (long i = 0; i < n_out; ++i) {
    int b = pairs ? pairs[2 * i] : (int)(i / Hq);
    int h = pairs ? pairs[2 * i + 1] : (int)(i % Hq);
    double *o = out + i * D;
    if (b < 0 || b >= B || h < 0 || h >= Hq) { set_status(&status, PA_ORACLE_BAD_ARG); continue; }
    int n = n_sel[b];
    if (n < 0 || n > max_sel) { set_status(&status, PA_ORACLE_BAD_ARG); continue; }
    if (n == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
    int g = h / G;
    double *qd = malloc(sizeof(double) * D);
    double *s = malloc(sizeof(double) * n);
    double *V = malloc(sizeof(double) * (size_t)n * D);
    if (!qd || !s || !V) { free(qd); free(s); free(V); set_status(&status, PA_ORACLE_NO_MEMORY); continue; }
    for (int d = 0; d < D; ++d) qd[d] = decode16(q[((long)b * Hq + h) * D + d], dtype);
    int bad = 0;
    for (int t = 0; t < n; ++t) {
      int pos = token_index[(long)b * max_sel + t];
      long blk = pos < 0 ? -1 : block_of(block_table, mbs, nb, bs, b, pos);
      if (blk < 0) { bad = 1; break; }
      long row = ((blk * Hkv + g) * bs + pos % bs) * (long)D;
      double acc = 0.0;
      for (int d = 0; d < D; ++d) {
        acc += qd[d] * decode16(k_cache[row + d], dtype);
        V[(long)t * D + d] = decode16(v_cache[row + d], dtype);
      }
      s[t] = scale * acc;
    }
    if (bad) set_status(&status, PA_ORACLE_BAD_BLOCK);
    else softmax_mix(n, s, V, D, o);
    free(qd); free(s); free(V);
  }
  return status;
}

/*
 * The same GQA operation computed the Flash-Decoding way, as an independent
 * statement for the split-then-merge property: tokens [0, n) are cut into splits
 * of split_len tokens; each split yields o_s (normalised) and
 * lse_s = m_s + log Z_s; the final row is sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M)
 * with M = max_s lse_s.  Argument layout as pa_oracle_decode.
 */
int pa_oracle_decode_split(int B, int Hq, int Hkv, int D, int bs, int mbs, int nb, int dtype,
                           const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                           const int32_t *block_table, const int32_t *context_lens,
                           double scale, int split_len, double *out, int nthreads) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || bs <= 0 || split_len <= 0)
    return PA_ORACLE_BAD_ARG;
  const int G = Hq / Hkv;
  int status = PA_ORACLE_OK;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (long i = 0; i < (long)B * Hq; ++i) {
    int b = (int)(i / Hq), h = (int)(i % Hq), g = h / G;
    double *o = out + i * D;
    int n = context_lens[b];
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (n <= 0) continue;
    int S = (n + split_len - 1) / split_len;
    double *qd = malloc(sizeof(double) * D);
    double *os = malloc(sizeof(double) * (size_t)S * D);
    double *lse = malloc(sizeof(double) * S);
    if (!qd || !os || !lse) { free(qd); free(os); free(lse); set_status(&status, PA_ORACLE_NO_MEMORY); continue; }
    for (int d = 0; d < D; ++d) qd[d] = decode16(q[((long)b * Hq + h) * D + d], dtype);
    int bad = 0;
    for (int sp = 0; sp < S && !bad; ++sp) {
      int t0 = sp * split_len, t1 = t0 + split_len < n ? t0 + split_len : n;
      /* per-split softmax with its own running max, then its log-sum-exp */
      double m = -INFINITY;
      for (int pass = 0; pass < 2 && !bad; ++pass) {
        double Z = 0.0;
        double *os_sp = os + (long)sp * D;
        if (pass == 1) for (int d = 0; d < D; ++d) os_sp[d] = 0.0;
        for (int t = t0; t < t1; ++t) {
          long blk = block_of(block_table, mbs, nb, bs, b, t);
          if (blk < 0) { bad = 1; break; }
          long row = ((blk * Hkv + g) * bs + t % bs) * (long)D;
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += qd[d] * decode16(k_cache[row + d], dtype);
          double sc = scale * acc;
          if (pass == 0) { if (sc > m) m = sc; continue; }
          double p = exp(sc - m);
          Z += p;
          for (int d = 0; d < D; ++d) os_sp[d] += p * decode16(v_cache[row + d], dtype);
        }
        if (pass == 1 && !bad) {
          for (int d = 0; d < D; ++d) os_sp[d] /= Z;
          lse[sp] = m + log(Z);
        }
      }
    }
    if (bad) { set_status(&status, PA_ORACLE_BAD_BLOCK); free(qd); free(os); free(lse); continue; }
    double M = -INFINITY;
    for (int sp = 0; sp < S; ++sp) if (lse[sp] > M) M = lse[sp];
    double W = 0.0;
    for (int sp = 0; sp < S; ++sp) {
      double w = exp(lse[sp] - M);
      W += w;
      for (int d = 0; d < D; ++d) o[d] += w * os[(long)sp * D + d];
    }
    for (int d = 0; d < D; ++d) o[d] /= W;
    free(qd); free(os); free(lse);
  }
  return status;
}

/*
 * MLA absorbed decode.  All H heads of a sequence read the same latent row per
 * token: the key is the whole Dk-wide latent row and the value is its first Dv
 * dims.
 *
 * q            [B][H][Dk]       raw 16-bit
 * latent_cache [NB][bs][Dk]     raw 16-bit
 * block_table  [B][mbs], context_lens [B] as for pa_oracle_decode
 * pairs        optional (b, h) list, NULL = all B*H
 * out          [npairs or B*H][Dv] double
 */
int pa_oracle_decode_mla(int B, int H, int Dk, int Dv, int bs, int mbs, int nb, int dtype,
                         const uint16_t *q, const uint16_t *latent_cache,
                         const int32_t *block_table, const int32_t *context_lens, double scale,
                         const int32_t *pairs, int npairs, double *out, int nthreads) {
  if (B < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || Dv > Dk || bs <= 0 || mbs < 0 || nb < 0)
    return PA_ORACLE_BAD_ARG;
  const long n_out = pairs ? (long)npairs : (long)B * H;
  int status = PA_ORACLE_OK;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (long i = 0; i < n_out; ++i) {
    int b = pairs ? pairs[2 * i] : (int)(i / H);
    int h = pairs ? pairs[2 * i + 1] : (int)(i % H);
    double *o = out + i * Dv;
    if (b < 0 || b >= B || h < 0 || h >= H) { set_status(&status, PA_ORACLE_BAD_ARG); continue; }
    int n = context_lens[b];
    if (n < 0 || (long)n > (long)mbs * bs) { set_status(&status, PA_ORACLE_BAD_ARG); continue; }
    if (n == 0) { for (int d = 0; d < Dv; ++d) o[d] = 0.0; continue; }
    double *qd = malloc(sizeof(double) * Dk);
    double *s = malloc(sizeof(double) * n);
    double *V = malloc(sizeof(double) * (size_t)n * Dv);
    if (!qd || !s || !V) { free(qd); free(s); free(V); set_status(&status, PA_ORACLE_NO_MEMORY); continue; }
    for (int d = 0; d < Dk; ++d) qd[d] = decode16(q[((long)b * H + h) * Dk + d], dtype);
    int bad = 0;
    for (int t = 0; t < n; ++t) {
      long blk = block_of(block_table, mbs, nb, bs, b, t);
      if (blk < 0) { bad = 1; break; }
      const uint16_t *row = latent_cache + (blk * bs + t % bs) * (long)Dk;
      double acc = 0.0;
      for (int d = 0; d < Dk; ++d) acc += qd[d] * decode16(row[d], dtype);
      s[t] = scale * acc;
      for (int d = 0; d < Dv; ++d) V[(long)t * Dv + d] = decode16(row[d], dtype);
    }
    if (bad) set_status(&status, PA_ORACLE_BAD_BLOCK);
    else softmax_mix(n, s, V, Dv, o);
    free(qd); free(s); free(V);
  }
  return status;
}

int pa_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
