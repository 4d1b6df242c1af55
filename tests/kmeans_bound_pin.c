/* kmeans_bound_pin.c - numerical check of the error bound behind the
 * k-means label certificate (test infrastructure, CPU only).
 *
 * Page "VC-Attention acelera atenção em modelos de vídeo de IA em até 3,58×
 * sem retreinamento", section "V-Smooth: corrigindo outliers de valor", item
 * Group. The pinned label of a token is the argmin over clusters of the fp32
 * chain d~_j = fmaf(x, x, d) over channels in order, x = fl(v - c_j). The
 * kernel decides it from e_j = fl(fl(|v|^2 + |c_j|^2) - 2 fl(v.hi_j + v.lo_j))
 * with hi_j = bf16(c_j), lo_j = bf16(c_j - hi_j), the two dot products
 * accumulated by the tensor cores in fp32, and trusts the estimate when every
 * other cluster's estimate exceeds the smallest by more than E_b + E_j,
 * E_j = 2^-13 fl(|v|^2 + |c_j|^2). That is sound if |e_j - d~_j| <= E_j.
 *
 * The tensor cores' fp32 accumulation order is not specified, so every dot
 * product is taken under four models: the exact sum rounded once, a
 * sequential fp32 sum, a pairwise fp32 tree, and exact sums of 16 products
 * truncated toward zero before a sequential fp32 sum of the groups (a
 * pessimistic model of blocked accumulation). |v|^2 is summed as the kernel
 * does: eight fp32 partial sums (chunk q of 8 channels into sum q % 8) added
 * pairwise; |c_j|^2 in fp64, rounded to fp32.
 *
 * pin_kmeans_bound returns, over all tokens, clusters and models, the largest
 * |e_j - d~_j| / E_j (must be below 1), and counts the tokens whose
 * certificate accepts a cluster other than the chain's argmin (must be 0).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float bf16_value(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* round-to-nearest-even binary32 -> bf16 (finite inputs) */
static uint16_t bf16_rn(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static float chain(const float *v, const float *c, int d) {
  float a = 0.0f;
  for (int i = 0; i < d; ++i) {
    const float x = v[i] - c[i];
    a = fmaf(x, x, a);
  }
  return a;
}

/* fp32 value nearest to s, toward zero */
static float trunc_f32(double s) {
  float r = (float)s;
  if (fabs((double)r) > fabs(s)) r = nextafterf(r, 0.0f);
  return r;
}

static float dot_model(const float *v, const float *w, int d, int model) {
  if (model == 0) {
    double s = 0.0; /* products are exact in fp32 (8 x 8 significant bits); their sum in fp64 */
    for (int i = 0; i < d; ++i) s += (double)(v[i] * w[i]);
    return (float)s;
  }
  if (model == 1) {
    float s = 0.0f;
    for (int i = 0; i < d; ++i) s += v[i] * w[i];
    return s;
  }
  if (model == 2) {
    float t[128];
    int n = d;
    for (int i = 0; i < d; ++i) t[i] = v[i] * w[i];
    while (n > 1) {
      for (int i = 0; i < n / 2; ++i) t[i] = t[2 * i] + t[2 * i + 1];
      if (n & 1) t[n / 2] = t[n - 1];
      n = (n + 1) / 2;
    }
    return t[0];
  }
  float s = 0.0f;
  for (int g = 0; g < d; g += 16) {
    double gs = 0.0;
    for (int i = g; i < g + 16 && i < d; ++i) gs += (double)(v[i] * w[i]);
    s += trunc_f32(gs);
  }
  return s;
}

static float vsq_kernel_order(const float *v, int d) {
  float p[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int q = 0; q < d / 8; ++q)
    for (int e = 0; e < 8; ++e) p[q & 7] = fmaf(v[8 * q + e], v[8 * q + e], p[q & 7]);
  return ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
}

/* V: n tokens x d bf16 (d a multiple of 8, d <= 128); C: k x d fp32 centroids. */
/* bscale multiplies E_j in the acceptance test only (1 = the kernel's rule; a
 * test plants a smaller margin to show that the margin is what keeps wrong
 * labels out). */
int pin_kmeans_bound(const uint16_t *V, int n, const float *C, int k, int d, float bscale, double *worst_ratio,
                     long long *wrong_accept, long long *accepted) {
  float hi[8][128], lo[8][128], cc[8];
  if (k > 8 || d > 128 || d % 8) return 1;
  for (int j = 0; j < k; ++j) {
    double s2 = 0.0;
    for (int i = 0; i < d; ++i) {
      const float c = C[j * d + i];
      hi[j][i] = bf16_value(bf16_rn(c));
      lo[j][i] = bf16_value(bf16_rn(c - hi[j][i]));
      s2 += (double)c * (double)c;
    }
    cc[j] = (float)s2;
  }
  double worst = 0.0;
  long long wrong = 0, acc = 0;
  for (int t = 0; t < n; ++t) {
    float v[128], dt[8];
    for (int i = 0; i < d; ++i) v[i] = bf16_value(V[(long long)t * d + i]);
    int jmin = 0;
    for (int j = 0; j < k; ++j) {
      dt[j] = chain(v, C + j * d, d);
      if (dt[j] < dt[jmin]) jmin = j;
    }
    const float vv = vsq_kernel_order(v, d);
    for (int model = 0; model < 4; ++model) {
      float e[8], E[8];
      int b = 0;
      for (int j = 0; j < k; ++j) {
        const float dot = dot_model(v, hi[j], d, model) + dot_model(v, lo[j], d, model);
        const float s = vv + cc[j];
        e[j] = s - 2.0f * dot;
        E[j] = 0x1p-13f * s;
        const double r = fabs((double)e[j] - (double)dt[j]) / (double)E[j];
        if (E[j] > 0.0f && r > worst) worst = r;
        if (e[j] < e[b]) b = j;
      }
      int certain = 1;
      for (int j = 0; j < k; ++j)
        if (j != b && !(e[j] - e[b] > bscale * (E[b] + E[j]))) certain = 0;
      if (certain) {
        ++acc;
        if (b != jmin) ++wrong;
      }
    }
  }
  *worst_ratio = worst;
  *wrong_accept = wrong;
  *accepted = acc;
  return 0;
}
