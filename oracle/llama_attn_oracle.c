/*
 * Plain, slow fp64 CPU oracle for LLaMA self-attention (RoPE -> GQA -> scaled
 * QK^T + mask -> softmax -> weighted sum with V), prefill and KV-cache decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; it is used by the tests, by the package smoke check and by
 * the CPU-baseline leg of the benchmark.  It shares no code with the CUDA path.
 *
 * Sources (page titles as printed on each page):
 *  [HF]   "[HuggingFace Transformers] LlamaAttention source walkthrough"
 *         (blog.csdn.net), section 1.2 "attention computation" steps 2-5, and
 *         section 2 forward() steps 2 (head reshape), 3 (RoPE), 4 (repeat_kv),
 *         5.1 (scaled QK^T + mask), 5.2 (fp32 softmax), 5.3 (weights x V),
 *         6 (transpose/concat of heads).
 *  [L2]   "LLaMA2 large language model architecture analysis"
 *         (obsidian-quartz-blog), sections "Rotary Position Encoding" (RoPE on
 *         Q and K only, after projection; RoFormer), "KV cache" (one query row
 *         against all cached keys) and "GQA" (query heads share K/V heads).
 *  [P5]   "Llama2 Transformer architecture and optimisation practice"
 *         (lpqz.cn), section 2.1 (q*cos + rotate(q)*sin; 8 query heads share one
 *         K/V head) and section 6.1 (linear RoPE scaling, factor 2.0).
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes): inverse frequency theta^(-2i/D) from the RoFormer paper the [L2]
 * RoPE section cites; rotate-half pairing (i, i + D/2) as in the HF
 * apply_rotary_pos_emb that [HF] step 3 calls; linear scaling divides the
 * position by the factor; query head h uses K/V head h / (H/Hkv) (contiguous
 * groups, the repeat_kv expansion of [HF] step 4); a row whose every key is
 * masked out yields an all-zero output row.
 *
 * Everything is computed in double.  Inputs arrive as float arrays: bf16 and
 * fp32 tensors are both exactly representable in float, so the oracle sees the
 * very same values the GPU sees.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* cos/sin of the RoPE angle for each position; layout [n, D], the angle of
 * pair i (i < D/2) is duplicated into columns i and i + D/2, as the HF rotary
 * embedding concatenates its frequencies twice ([HF] step 3). */
void oracle_rope_cos_sin(const long long* pos, long n, int D, double theta,
                         double factor, double* cos_out, double* sin_out) {
  const int half = D / 2;
  for (long r = 0; r < n; ++r) {
    const double p = (double)pos[r] / factor;     /* linear scaling: [P5] 6.1 */
    for (int i = 0; i < half; ++i) {
      const double inv_freq = pow(theta, -2.0 * (double)i / (double)D);
      const double angle = p * inv_freq;
      cos_out[r * D + i] = cos(angle);
      cos_out[r * D + i + half] = cos(angle);
      sin_out[r * D + i] = sin(angle);
      sin_out[r * D + i + half] = sin(angle);
    }
  }
}

/* NTK-aware RoPE scaling: the base is raised to theta * alpha^(D / (D - 2)),
 * so the highest frequency (i = 0) is kept and the lowest (i = D/2 - 1) is
 * divided by exactly alpha.  [P5] 6.1 names "adjusting the base frequency" for
 * length extrapolation without a formula; this is the published NTK-aware
 * rule, taken as the reading.  The table is then oracle_rope_cos_sin with
 * this base and no position scaling. */
double oracle_rope_ntk_theta(double theta, double alpha, int D) {
  return theta * pow(alpha, (double)D / (double)(D - 2));
}

/* y = x * cos + rotate_half(x) * sin, with rotate_half(x) = [-x[D/2:], x[:D/2]]
 * (rotate-half form of [P5] 2.1 / the apply_rotary_pos_emb of [HF] step 3). */
void oracle_rope_rotate(const double* x, long n, int D, const double* cos_t,
                        const double* sin_t, double* y) {
  const int half = D / 2;
  for (long r = 0; r < n; ++r) {
    const double* xr = x + r * D;
    const double* c = cos_t + r * D;
    const double* s = sin_t + r * D;
    double* yr = y + r * D;
    for (int d = 0; d < D; ++d) {
      const double rot = (d < half) ? -xr[d + half] : xr[d - half];
      yr[d] = xr[d] * c[d] + rot * s[d];
    }
  }
}

/* Rotate one row of length D given as float, at position p, into out (double).
 * Builds the row's cos/sin through oracle_rope_cos_sin so there is one
 * definition of the angle. */
static void rotate_row_f(const float* x, int D, long long p, double theta,
                         double factor, double* tmp_cs, double* out) {
  double* c = tmp_cs;
  double* s = tmp_cs + D;
  double* xd = tmp_cs + 2 * D;
  oracle_rope_cos_sin(&p, 1, D, theta, factor, c, s);
  for (int d = 0; d < D; ++d) xd[d] = (double)x[d];
  oracle_rope_rotate(xd, 1, D, c, s, out);
}

/* Softmax-weighted sum for one query row given its scores.
 * scores[j] = -INFINITY marks an excluded key.  Writes o[D] and, when probs
 * is non-NULL, the normalised weights.  [HF] 1.2 steps 3-4, section 2 5.2-5.3. */
static void softmax_weighted_sum(const double* scores, int n_keys,
                                 const float* v_base, long v_row_stride, int D,
                                 double* p_work, double* o, double* probs) {
  double mx = -INFINITY;
  for (int j = 0; j < n_keys; ++j)
    if (scores[j] > mx) mx = scores[j];
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (mx == -INFINITY) { /* every key masked: zero row (documented reading) */
    if (probs)
      for (int j = 0; j < n_keys; ++j) probs[j] = 0.0;
    return;
  }
  double denom = 0.0;
  for (int j = 0; j < n_keys; ++j) {
    p_work[j] = (scores[j] == -INFINITY) ? 0.0 : exp(scores[j] - mx);
    denom += p_work[j];
  }
  for (int j = 0; j < n_keys; ++j) {
    const double w = p_work[j] / denom;
    if (probs) probs[j] = w;
    if (w == 0.0) continue;
    const float* vr = v_base + (long)j * v_row_stride;
    for (int d = 0; d < D; ++d) o[d] += w * (double)vr[d];
  }
}

/*
 * Prefill.  q [bsz, S, H, D], k and v [bsz, S, Hkv, D] (the projection outputs
 * viewed per head without the transpose, [HF] step 2), pos [bsz, S] RoPE
 * position ids or NULL for no RoPE, mask [bsz, 1, S, S] additive or NULL.
 * Computes out[b, i, h*D + d] (heads concatenated in order 0..H-1 on the last
 * dim, [HF] step 6) for heads h in [h_lo, h_hi) and query rows i in
 * [i_lo, i_hi); other entries of out are left untouched.  probs, when not
 * NULL, receives the softmax weights [bsz, H, S, S] of the computed rows.
 * Returns 0, or -1 on invalid arguments.
 */
int oracle_prefill(const float* q, const float* k, const float* v,
                   const long long* pos, int bsz, int H, int Hkv, int S, int D,
                   double theta, double factor, double scale, int causal,
                   const float* mask, int h_lo, int h_hi, int i_lo, int i_hi,
                   double* out, double* probs, int nthreads) {
  if (bsz < 1 || H < 1 || Hkv < 1 || S < 1 || D < 2 || (D % 2) || (H % Hkv))
    return -1;
  if (h_lo < 0 || h_hi > H || h_lo >= h_hi || i_lo < 0 || i_hi > S || i_lo >= i_hi)
    return -1;
  const int group = H / Hkv; /* num_key_value_groups, [HF] __init__ */

  /* Rotated keys, one copy per (b, kv head) used by the selected heads. */
  double* krot = (double*)malloc(sizeof(double) * (size_t)bsz * Hkv * S * D);
  if (!krot) return -1;
  int kv_lo = h_lo / group, kv_hi = (h_hi - 1) / group + 1;

#ifdef _OPENMP
  /* thread count for this call only (nthreads <= 0: the process default) */
  const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel for collapse(2) schedule(dynamic) num_threads(nt)
#endif
  for (int b = 0; b < bsz; ++b)
    for (int j = 0; j < S; ++j) {
      double tmp[3 * 512];
      for (int kh = kv_lo; kh < kv_hi; ++kh) {
        const float* kr = k + (((long)b * S + j) * Hkv + kh) * D;
        double* dst = krot + (((long)b * Hkv + kh) * S + j) * D;
        if (pos) {
          rotate_row_f(kr, D, pos[(long)b * S + j], theta, factor, tmp, dst);
        } else {
          for (int d = 0; d < D; ++d) dst[d] = (double)kr[d];
        }
      }
    }

  const long n_rows = (long)bsz * (h_hi - h_lo) * (i_hi - i_lo);
#ifdef _OPENMP
#pragma omp parallel num_threads(nt)
#endif
  {
    double* scores = (double*)malloc(sizeof(double) * S);
    double* pw = (double*)malloc(sizeof(double) * S);
    double* qd = (double*)malloc(sizeof(double) * D);
    double* o = (double*)malloc(sizeof(double) * D);
    double tmp[3 * 512];
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
    for (long r = 0; r < n_rows; ++r) {
      const int i = i_lo + (int)(r % (i_hi - i_lo));
      const int h = h_lo + (int)((r / (i_hi - i_lo)) % (h_hi - h_lo));
      const int b = (int)(r / ((long)(i_hi - i_lo) * (h_hi - h_lo)));
      const int kh = h / group; /* repeat_kv: query head h reads K/V head h/group */
      const float* qr = q + (((long)b * S + i) * H + h) * D;
      if (pos) {
        rotate_row_f(qr, D, pos[(long)b * S + i], theta, factor, tmp, qd);
      } else {
        for (int d = 0; d < D; ++d) qd[d] = (double)qr[d];
      }
      for (int j = 0; j < S; ++j) {
        if (causal && j > i) { scores[j] = -INFINITY; continue; }
        const double* kr = krot + (((long)b * Hkv + kh) * S + j) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qd[d] * kr[d];
        double s = dot * scale;
        if (mask) s += (double)mask[((long)b * S + i) * S + j];
        scores[j] = s;
      }
      double* prow = probs ? probs + (((long)b * H + h) * S + i) * S : NULL;
      softmax_weighted_sum(scores, S, v + ((long)b * S * Hkv + kh) * D,
                           (long)Hkv * D, D, pw, o, prow);
      double* orow = out + ((long)b * S + i) * ((long)H * D) + (long)h * D;
      for (int d = 0; d < D; ++d) orow[d] = o[d];
    }
    free(scores); free(pw); free(qd); free(o);
  }
  free(krot);
  return 0;
}

/*
 * Single-token decode against a KV cache ([L2] "KV cache": one query row,
 * keys/values already cached).  q [bsz, H, D] un-rotated; it is rotated at
 * qpos[b] (NULL: no RoPE).  k_cache/v_cache [bsz, Hkv, L, D] hold keys that are
 * already rotated; the first lens[b] rows are attended, none masked.
 * out [bsz, H*D].  probs, when not NULL, receives [bsz, H, L] weights (zero
 * past lens[b]).  Returns 0, or -1 on invalid arguments.
 */
int oracle_decode(const float* q, const float* k_cache, const float* v_cache,
                  const int* lens, const long long* qpos, int bsz, int H,
                  int Hkv, int L, int D, double theta, double factor,
                  double scale, double* out, double* probs, int nthreads) {
  if (bsz < 1 || H < 1 || Hkv < 1 || L < 1 || D < 2 || (D % 2) || (H % Hkv))
    return -1;
  for (int b = 0; b < bsz; ++b)
    if (lens[b] < 0 || lens[b] > L) return -1;
  const int group = H / Hkv;
#ifdef _OPENMP
  /* thread count for this call only (nthreads <= 0: the process default) */
  const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#pragma omp parallel num_threads(nt)
#endif
  {
    double* scores = (double*)malloc(sizeof(double) * L);
    double* pw = (double*)malloc(sizeof(double) * L);
    double* qd = (double*)malloc(sizeof(double) * D);
    double* o = (double*)malloc(sizeof(double) * D);
    double tmp[3 * 512];
#ifdef _OPENMP
#pragma omp for collapse(2) schedule(dynamic)
#endif
    for (int b = 0; b < bsz; ++b)
      for (int h = 0; h < H; ++h) {
        const int kh = h / group;
        const float* qr = q + ((long)b * H + h) * D;
        if (qpos) {
          rotate_row_f(qr, D, qpos[b], theta, factor, tmp, qd);
        } else {
          for (int d = 0; d < D; ++d) qd[d] = (double)qr[d];
        }
        const int n = lens[b];
        const float* kb = k_cache + ((long)b * Hkv + kh) * (long)L * D;
        for (int j = 0; j < n; ++j) {
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += qd[d] * (double)kb[(long)j * D + d];
          scores[j] = dot * scale;
        }
        double* prow = probs ? probs + ((long)b * H + h) * L : NULL;
        if (prow)
          for (int j = n; j < L; ++j) prow[j] = 0.0;
        if (n == 0) {
          for (int d = 0; d < D; ++d) o[d] = 0.0;
        } else {
          softmax_weighted_sum(scores, n,
                               v_cache + ((long)b * Hkv + kh) * (long)L * D,
                               D, D, pw, o, prow);
        }
        double* orow = out + (long)b * H * D + (long)h * D;
        for (int d = 0; d < D; ++d) orow[d] = o[d];
      }
    free(scores); free(pw); free(qd); free(o);
  }
  return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
