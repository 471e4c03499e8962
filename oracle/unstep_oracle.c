/*
 * unstep_oracle.c -- plain fp64 CPU oracle for the UnStep chunk-causal attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file;
 * only the test-suite, the smoke check and the bench's CPU-baseline leg use it.  It shares no
 * code, header, table or helper with the CUDA library.
 *
 * Source: "UnStep: Training-Free Acceleration of Causal Video Diffusion with Fewer Steps Than
 * Distillation" (arXiv 2609.32518), abstract: the DiT runtime stack applies RoPE from cached
 * coefficients, indexes a KV cache, and limits the temporal window that the attention KV cache
 * retains; Table 1 row C4 (the attention window limit added).  The pages give no formulas for these
 * steps, so this file writes out the textbook definitions they name:
 *
 *   3D RoPE: the head dimension D is split into a temporal, a height and a width block
 *   (d_t + d_h + d_w = D, channel order t, h, w).  Channel pair p = (2p, 2p+1) of block a with
 *   in-block pair index j is rotated by the angle pos_a * theta^(-2j/d_a), where pos_t is the
 *   absolute latent frame index, pos_h the token row and pos_w the token column:
 *       (x0, x1) -> (x0 cos(ang) - x1 sin(ang),  x0 sin(ang) + x1 cos(ang)).
 *
 *   Attention of one query row: s_j = scale * <q, k_j> over the window keys, o = sum_j
 *   softmax(s)_j v_j, written as the two-pass definition (max, exponentials, sum, weighted sum).
 *
 * Everything is computed in double precision from the bf16 inputs.  OpenMP splits independent
 * rows; it does not change any arithmetic order inside a row.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EARG -1
#define ORC_ENOMEM -2

/* bf16 -> double: a bf16 is the top half of an IEEE binary32, so the conversion is exact. */
double orc_bf16_to_f64(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* double -> bf16, round to nearest, ties to even, taken directly from the double (no detour
 * through binary32, which could round twice).  NaN maps to a quiet NaN; overflow to +-inf. */
uint16_t orc_f64_to_bf16_rne(double x) {
  if (x != x) return (uint16_t)0x7FC0;
  uint16_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7F80);
  /* bf16 has an 8-bit significand (7 stored bits) and binary32's exponent range.
   * The smallest normal is 2^-126; subnormals have spacing 2^-133. */
  int e;
  frexp(a, &e);          /* a = m * 2^e, m in [0.5, 1) -> a in [2^(e-1), 2^e) */
  int ulp_exp = e - 8;   /* spacing of 8-bit significands in this binade */
  if (ulp_exp < -133) ulp_exp = -133;
  double q = ldexp(a, -ulp_exp);     /* exact: scaling by a power of two */
  double r = floor(q);
  double frac = q - r;                /* exact */
  if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
  double y = ldexp(r, ulp_exp);       /* the rounded magnitude, exactly representable */
  if (y > 3.3895313892515355e38) {    /* beyond the largest finite bf16, (2 - 2^-7) * 2^127 */
    return (uint16_t)(sign | 0x7F80);
  }
  float f = (float)y;                 /* exact: y has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

/* Which block a channel pair belongs to, its index inside the block and the block width. */
static void pair_axis(int p, int d_t, int d_h, int *axis, int *j, int *d_a, int d_w) {
  int c = 2 * p;
  if (c < d_t) {
    *axis = 0; *j = p; *d_a = d_t;
  } else if (c < d_t + d_h) {
    *axis = 1; *j = p - d_t / 2; *d_a = d_h;
  } else {
    *axis = 2; *j = p - (d_t + d_h) / 2; *d_a = d_w;
  }
}

/* Rotation angle of pair j of a block of width d_a at position pos: pos * theta^(-2j/d_a). */
double orc_rope_angle(int pos, int j, int d_a, double theta) {
  return (double)pos * pow(theta, -2.0 * (double)j / (double)d_a);
}

/*
 * 3D RoPE of one chunk.
 *   x    : bf16 bits, [B][L][H][D], L = frames*Hg*Wg; token l -> (i, y, x) with
 *          l = i*Hg*Wg + y*Wg + x and absolute frame f = frame_idx + i.
 *   out  : double, same layout, the exact rotation of the bf16 inputs.
 */
int orc_rope3d(const uint16_t *x, int B, int L, int H, int D, int frame_idx, int frames, int Hg,
               int Wg, int d_t, int d_h, int d_w, double theta, double *out) {
  if (!x || !out || B < 1 || H < 1 || D < 2 || (D & 1) || Hg < 1 || Wg < 1 || frames < 1)
    return ORC_EARG;
  if (d_t + d_h + d_w != D || (d_t & 1) || (d_h & 1) || (d_w & 1) || d_t < 0 || d_h < 0 || d_w < 0)
    return ORC_EARG;
  if ((long)frames * Hg * Wg != (long)L || frame_idx < 0) return ORC_EARG;
  const int Tf = Hg * Wg;
  const long rows = (long)B * L;
#pragma omp parallel for schedule(static)
  for (long r = 0; r < rows; ++r) {
    int l = (int)(r % L);
    int i = l / Tf;
    int tok = l % Tf;
    int pos[3];
    pos[0] = frame_idx + i;
    pos[1] = tok / Wg;
    pos[2] = tok % Wg;
    for (int h = 0; h < H; ++h) {
      const uint16_t *src = x + (r * H + h) * (long)D;
      double *dst = out + (r * H + h) * (long)D;
      for (int p = 0; p < D / 2; ++p) {
        int axis, j, d_a;
        pair_axis(p, d_t, d_h, &axis, &j, &d_a, d_w);
        double ang = orc_rope_angle(pos[axis], j, d_a, theta);
        double c = cos(ang), s = sin(ang);
        double a = orc_bf16_to_f64(src[2 * p]);
        double b = orc_bf16_to_f64(src[2 * p + 1]);
        dst[2 * p] = a * c - b * s;
        dst[2 * p + 1] = a * s + b * c;
      }
    }
  }
  return ORC_OK;
}

/* Element-wise bf16 -> double and double -> bf16 (RNE) over n values. */
int orc_bf16_array_to_f64(const uint16_t *x, long n, double *out) {
  if (!x || !out || n < 0) return ORC_EARG;
#pragma omp parallel for schedule(static)
  for (long i = 0; i < n; ++i) out[i] = orc_bf16_to_f64(x[i]);
  return ORC_OK;
}

int orc_f64_array_to_bf16(const double *x, long n, uint16_t *out) {
  if (!x || !out || n < 0) return ORC_EARG;
#pragma omp parallel for schedule(static)
  for (long i = 0; i < n; ++i) out[i] = orc_f64_to_bf16_rne(x[i]);
  return ORC_OK;
}

/*
 * Softmax attention of selected query rows over one key set per (b, h).
 *   q     : double [B][L][H][D]
 *   K, V  : double [B][H][Nk][D]   (the window keys, any order)
 *   rows  : nrows triples (b, l, h)
 *   out   : double [nrows][D]
 * For each row: s_j = scale * sum_d q_d K_jd; m = max_j s_j; e_j = exp(s_j - m);
 * o_d = (sum_j e_j V_jd) / (sum_j e_j).
 */
int orc_attention_rows(const double *q, int B, int L, int H, int D, const double *K,
                       const double *V, int Nk, const int *rows_b, const int *rows_l,
                       const int *rows_h, int nrows, double scale, double *out) {
  if (!q || !K || !V || !rows_b || !rows_l || !rows_h || !out) return ORC_EARG;
  if (B < 1 || L < 1 || H < 1 || D < 1 || Nk < 1 || nrows < 0) return ORC_EARG;
  for (int r = 0; r < nrows; ++r) {
    if (rows_b[r] < 0 || rows_b[r] >= B || rows_l[r] < 0 || rows_l[r] >= L || rows_h[r] < 0 ||
        rows_h[r] >= H)
      return ORC_EARG;
  }
  int err = ORC_OK;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
    double *acc = (double *)malloc(sizeof(double) * (size_t)D);
    if (!s || !acc) {
#pragma omp atomic write
      err = ORC_ENOMEM;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int r = 0; r < nrows; ++r) {
        const int b = rows_b[r], l = rows_l[r], h = rows_h[r];
        const double *qr = q + (((long)b * L + l) * H + h) * (long)D;
        const double *Kbh = K + ((long)b * H + h) * (long)Nk * D;
        const double *Vbh = V + ((long)b * H + h) * (long)Nk * D;
        double m = -INFINITY;
        for (int j = 0; j < Nk; ++j) {
          double dot = 0.0;
          const double *kj = Kbh + (long)j * D;
          for (int d = 0; d < D; ++d) dot += qr[d] * kj[d];
          s[j] = scale * dot;
          if (s[j] > m) m = s[j];
        }
        double sum = 0.0;
        for (int j = 0; j < Nk; ++j) {
          s[j] = exp(s[j] - m);
          sum += s[j];
        }
        for (int d = 0; d < D; ++d) acc[d] = 0.0;
        for (int j = 0; j < Nk; ++j) {
          const double *vj = Vbh + (long)j * D;
          for (int d = 0; d < D; ++d) acc[d] += s[j] * vj[d];
        }
        double *o = out + (long)r * D;
        for (int d = 0; d < D; ++d) o[d] = acc[d] / sum;
      }
    }
    free(s);
    free(acc);
  }
  return err;
}

/* Number of OpenMP threads a parallel region of this library uses. */
int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
