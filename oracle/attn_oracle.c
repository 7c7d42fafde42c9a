/*
 * attn_oracle.c -- plain, slow, fp64 scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this
 * file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark load it.  It shares no code with the CUDA kernels.
 *
 * What it computes is the plain definition, written out row by row with the
 * full score row materialised (no tiling, no online softmax):
 *
 *   For query token t of sequence b (local index i), query head h:
 *     kv head       g = h / (Hq / Hkv)
 *         (oxillama-runtime 0.1.0 flash_attention.rs, flash_attention_gqa:
 *          q head kv_h*G + r reads kv head kv_h; mxflashattn 1.4.0
 *          prefill.py, repeat_interleave of K/V by the group size)
 *     visible keys  V(i) = { j : 0 <= j < Sk_b and
 *                            (!causal or j <= i + Sk_b - Sq_b) }
 *         (bottom-right causal alignment: mxflashattn 1.4.0 prefill.py,
 *          query_positions = arange(Sq) + (Sk - Sq))
 *     s_j   = scale * sum_d q[t,h,d] * k[j,g,d]      (j in V(i)), -inf else
 *         (lattice-inference 0.7.1 standard.rs: masked scores are -inf,
 *          never a finite sentinel)
 *     m     = max_j s_j;  l = sum_j exp(s_j - m);  P_j = exp(s_j - m) / l
 *     O     = sum_j P_j * v[j,g,0:Dv]
 *     LSE   = m + ln(l)
 *     V(i) empty:  O = 0, LSE = -inf
 *         (mxflashattn prefill.py and oxillama flash_attention both return
 *          O = 0 for a row with nothing to attend to; LSE = ln 0 = -inf is
 *          this library's reading, the pages return no LSE)
 *
 * MLA decode (kernelbot-amd-mixed-mla submission 588924, _flash_fused):
 * k = kv[:, 0:576] and v = kv[:, 0:512] of one shared kv head; the caller
 * expresses that with pointers and row strides, nothing here is special.
 *
 * Arithmetic is IEEE fp64 (built with -O2, no fast-math): inputs of any of
 * the supported storage types are upcast exactly to double first.
 *
 * Build with -DORACLE_MUTANT=n to plant one deliberate mistake (used only
 * by the test that proves the oracle's pins catch such mistakes).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

enum { ORC_F64 = 0, ORC_F32 = 1, ORC_F16 = 2, ORC_BF16 = 3 };

/* Exact upcast of one stored element to double. */
static double load_elem(const void *base, int dtype, int64_t idx) {
  switch (dtype) {
    case ORC_F64: return ((const double *)base)[idx];
    case ORC_F32: return (double)((const float *)base)[idx];
    case ORC_BF16: {
      uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
      float f;
      memcpy(&f, &bits, sizeof f);
      return (double)f;
    }
    case ORC_F16: {
      /* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
      uint16_t hbits = ((const uint16_t *)base)[idx];
      int sign = (hbits >> 15) & 1;
      int ex = (hbits >> 10) & 0x1f;
      int fr = hbits & 0x3ff;
      double val;
      if (ex == 0) val = ldexp((double)fr, -24);               /* subnormal */
      else if (ex == 31) val = fr ? NAN : INFINITY;
      else val = ldexp((double)(fr | 0x400), ex - 25);         /* 1.f * 2^(ex-15) */
      return sign ? -val : val;
    }
  }
  return NAN;
}

typedef struct {
  const void *q, *k, *v;
  int dtype;
  int64_t q_rs, q_hs, k_rs, k_hs, v_rs, v_hs; /* element strides: token, head */
  const int64_t *cu_q, *cu_k;
  int batch, hq, hkv, dqk, dv;
  double scale;
  int causal;
  const int64_t *pairs; /* npairs x 2: (token, head) */
  int64_t npairs;
  double *o;    /* npairs x dv */
  double *lse;  /* npairs */
  double *psum; /* npairs: sum of the materialised probabilities */
  int nthreads;
  int tid;
} oracle_job;

/* Sequence b that holds query token t: the largest b with cu_q[b] <= t. */
static int find_seq(const int64_t *cu, int batch, int64_t t) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
#if ORACLE_MUTANT == 8
  if (lo > 0) lo -= 1; /* planted: wrong sequence lookup */
#endif
  return lo;
}

static void one_row(const oracle_job *J, int64_t p, double *s) {
  const int64_t t = J->pairs[2 * p], h = J->pairs[2 * p + 1];
  const int b = find_seq(J->cu_q, J->batch, t);
  const int64_t i = t - J->cu_q[b];
  const int64_t sq = J->cu_q[b + 1] - J->cu_q[b];
  const int64_t sk = J->cu_k[b + 1] - J->cu_k[b];
  const int64_t k0 = J->cu_k[b];
  const int group = J->hq / J->hkv;
#if ORACLE_MUTANT == 2
  const int64_t g = h % J->hkv; /* planted: interleaved instead of grouped heads */
#else
  const int64_t g = h / group;
#endif
  double *o = J->o + p * J->dv;
  double m = -INFINITY;

  for (int64_t j = 0; j < sk; ++j) {
#if ORACLE_MUTANT == 3
    int visible = !J->causal || j < i + sk - sq;      /* planted: diagonal masked */
#elif ORACLE_MUTANT == 4
    int visible = !J->causal || j <= i;               /* planted: top-left alignment */
#else
    int visible = !J->causal || j <= i + sk - sq;
#endif
    if (!visible) { s[j] = -INFINITY; continue; }
    double acc = 0.0;
    for (int d = 0; d < J->dqk; ++d) {
      double qd = load_elem(J->q, J->dtype, t * J->q_rs + h * J->q_hs + d);
#if ORACLE_MUTANT == 5
      double kd = load_elem(J->k, J->dtype, (k0 + j) * J->k_rs + g * J->k_hs + (J->dqk - 1 - d)); /* planted: reversed k */
#else
      double kd = load_elem(J->k, J->dtype, (k0 + j) * J->k_rs + g * J->k_hs + d);
#endif
      acc += qd * kd;
    }
#if ORACLE_MUTANT == 1
    s[j] = acc; /* planted: scale dropped */
#elif ORACLE_MUTANT == 6
    s[j] = -J->scale * acc; /* planted: sign flipped */
#else
    s[j] = J->scale * acc;
#endif
    if (s[j] > m) m = s[j];
  }

  for (int d = 0; d < J->dv; ++d) o[d] = 0.0;
  if (m == -INFINITY) { /* nothing visible */
    J->lse[p] = -INFINITY;
    J->psum[p] = 0.0;
    return;
  }
  double l = 0.0;
  for (int64_t j = 0; j < sk; ++j) {
    s[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
    l += s[j];
  }
  double ps = 0.0;
  for (int64_t j = 0; j < sk; ++j) {
#if ORACLE_MUTANT == 7
    double pj = s[j]; /* planted: normalisation dropped */
#else
    double pj = s[j] / l;
#endif
    ps += pj;
    if (pj == 0.0) continue;
    for (int d = 0; d < J->dv; ++d) {
#if ORACLE_MUTANT == 9
      o[d] += pj * load_elem(J->k, J->dtype, (k0 + j) * J->k_rs + g * J->k_hs + d); /* planted: k in place of v */
#else
      o[d] += pj * load_elem(J->v, J->dtype, (k0 + j) * J->v_rs + g * J->v_hs + d);
#endif
    }
  }
  J->psum[p] = ps;
#if ORACLE_MUTANT == 10
  J->lse[p] = m + l; /* planted: log dropped */
#else
  J->lse[p] = m + log(l);
#endif
}

static void *worker(void *arg) {
  oracle_job *J = (oracle_job *)arg;
  int64_t max_sk = 0;
  for (int b = 0; b < J->batch; ++b) {
    int64_t n = J->cu_k[b + 1] - J->cu_k[b];
    if (n > max_sk) max_sk = n;
  }
  double *s = (double *)malloc(sizeof(double) * (size_t)(max_sk > 0 ? max_sk : 1));
  if (!s) return (void *)1;
  for (int64_t p = J->tid; p < J->npairs; p += J->nthreads) one_row(J, p, s);
  free(s);
  return NULL;
}

/*
 * oracle_attention: evaluate O and LSE for the listed (token, head) pairs.
 * Returns 0 on success, nonzero on a bad argument or a failed allocation.
 * Strides are in elements; the last dimension of q, k, v is contiguous.
 */
int oracle_attention(const void *q, const void *k, const void *v, int dtype,
                     int64_t q_rs, int64_t q_hs, int64_t k_rs, int64_t k_hs,
                     int64_t v_rs, int64_t v_hs,
                     const int64_t *cu_q, const int64_t *cu_k, int batch,
                     int hq, int hkv, int dqk, int dv, double scale, int causal,
                     const int64_t *pairs, int64_t npairs,
                     double *o, double *lse, double *psum, int nthreads) {
  if (!q || !k || !v || !cu_q || !cu_k || !o || !lse || !psum) return 1;
  if (batch <= 0 || hq <= 0 || hkv <= 0 || hq % hkv || dqk <= 0 || dv <= 0) return 1;
  if (npairs < 0 || (npairs > 0 && !pairs)) return 1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  oracle_job base = {q, k, v, dtype, q_rs, q_hs, k_rs, k_hs, v_rs, v_hs, cu_q, cu_k,
                     batch, hq, hkv, dqk, dv, scale, causal, pairs, npairs, o, lse, psum,
                     nthreads, 0};
  oracle_job jobs[512];
  pthread_t th[512];
  int rc = 0;
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = base;
    jobs[i].tid = i;
    if (pthread_create(&th[i], NULL, worker, &jobs[i]) != 0) { nthreads = i; rc = 1; break; }
  }
  for (int i = 0; i < nthreads; ++i) {
    void *ret = NULL;
    pthread_join(th[i], &ret);
    if (ret) rc = 1;
  }
  return rc;
}
