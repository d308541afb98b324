/*
 * Wan2.2 DiT self-attention oracle: plain, slow, fp64 CPU code.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links or calls this
 * file; only the tests, the package's smoke check and the bench's CPU-baseline
 * leg do. It shares no code, header or table with the CUDA kernels.
 *
 * What it computes, step by step, in the order the pages give:
 *
 *  1. Q/K RMSNorm over the full hidden width D = heads*128 of each token
 *     (review comments on TensorRT-LLM PR "[visual_gen] Optimize Wan2.2
 *     Dataflow": the norm spans num_heads*head_dim, and the weight of channel
 *     (head, dim) is gamma[head*head_dim + dim]).
 *        r = 1 / sqrt(mean_c x_c^2 + eps),  y_c = x_c * r * gamma_c      (fp64)
 *  2. Round y to bf16, round-to-nearest-even (same PR, "Fused Q/K Norm and
 *     RoPE": the BF16 rounding point sits between the norm and RoPE).
 *  3. 3D RoPE on adjacent pairs (2i, 2i+1) of each head: pairs [0,22) rotate
 *     by the frame index, [22,43) by the row index, [43,64) by the column
 *     index; within an axis of width d_a the j-th pair has frequency
 *     theta^(-2j/d_a). Angle = position * frequency; rotation
 *        (u, v) -> (u cos a - v sin a, u sin a + v cos a)          (fp64)
 *     then round to bf16. V is copied unchanged. Token s sits at frame
 *     s / (H*W), row (s / W) % H, column s % W.
 *  4. Full bidirectional softmax attention per (batch, head):
 *        o_i = sum_j softmax_j(scale * q_i . k_j) v_j                 (fp64)
 *     evaluated as the plain definition (max-subtracted exponentials).
 *
 * The pair layout, axis order, frequency exponent, eps placement and rounding
 * mode are readings of pages that leave them open; each is a parameter or a
 * named constant here so that a test can flip it.
 *
 * bf16 values travel as their 16-bit patterns (uint16_t).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define HEAD_DIM 128

static double bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bf16 value (8 significant bits), ties to even.
 * Written from the definition of the format: frexp gives x = m * 2^e with
 * 0.5 <= |m| < 1, so m * 2^8 has exactly the 8 kept bits above the point. */
double wan_oracle_round_bf16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  double m = frexp(x, &e);
  double r = nearbyint(ldexp(m, 8)); /* default rounding mode: nearest-even */
  return ldexp(r, e - 8);
}

static uint16_t f64_to_bf16_bits(double x) {
  /* x is already a bf16 value: the float conversion is exact. */
  float f = (float)wan_oracle_round_bf16(x);
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

void wan_oracle_bf16_to_f64(const uint16_t* in, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_f64(in[i]);
}

void wan_oracle_f64_to_bf16(const double* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = f64_to_bf16_bits(in[i]);
}

/* Step 1 alone: y = x * r * gamma (fp64, not rounded) for n rows of width d.
 * x: bf16 rows with a row stride of x_stride elements. */
void wan_oracle_rmsnorm(const uint16_t* x, int64_t n, int64_t d, int64_t x_stride,
                        const uint16_t* gamma, double eps, double* y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t) {
    const uint16_t* row = x + t * x_stride;
    double ss = 0.0;
    for (int64_t c = 0; c < d; ++c) {
      double v = bf16_to_f64(row[c]);
      ss += v * v;
    }
    double r = 1.0 / sqrt(ss / (double)d + eps);
    for (int64_t c = 0; c < d; ++c) y[t * d + c] = bf16_to_f64(row[c]) * r * bf16_to_f64(gamma[c]);
  }
}

/* Which axis (0 frame, 1 row, 2 column) and which index within it a pair of
 * a 128-wide head belongs to, for the split (d0, d1, d2) of head dims. */
static void pair_axis(int pair, const int32_t split[3], int* axis, int* j) {
  int p0 = split[0] / 2, p1 = split[1] / 2;
  if (pair < p0) { *axis = 0; *j = pair; }
  else if (pair < p0 + p1) { *axis = 1; *j = pair - p0; }
  else { *axis = 2; *j = pair - p0 - p1; }
}

/* Rotate the pairs of one token's heads (heads x 128 doubles) for sequence
 * index s of an F x H x W grid. half_split=0: adjacent pairs (2i, 2i+1), the
 * reading taken; 1: pairs (i, i+64), kept only so a test can show the choice
 * is observable. */
static void rope_token(double* y, int64_t s, int32_t heads, int32_t H, int32_t W, double theta,
                       const int32_t split[3], int32_t half_split) {
  int64_t pos[3] = {s / ((int64_t)H * W), (s / W) % H, s % W};
  for (int32_t h = 0; h < heads; ++h) {
    double* head = y + (int64_t)h * HEAD_DIM;
    for (int pair = 0; pair < HEAD_DIM / 2; ++pair) {
      int axis, j;
      pair_axis(pair, split, &axis, &j);
      double freq = pow(theta, -2.0 * (double)j / (double)split[axis]);
      double a = (double)pos[axis] * freq;
      double c = cos(a), sn = sin(a);
      int i0 = half_split ? pair : 2 * pair;
      int i1 = half_split ? pair + HEAD_DIM / 2 : 2 * pair + 1;
      double u = head[i0], v = head[i1];
      head[i0] = u * c - v * sn;
      head[i1] = u * sn + v * c;
    }
  }
}

/* Step 3 alone: rotate y (n tokens x heads x 128, fp64) in place, token t at
 * sequence index seq0 + t; not rounded. */
void wan_oracle_rope(double* y, int64_t n, int64_t seq0, int32_t heads, int32_t H, int32_t W,
                     double theta, const int32_t split[3], int32_t half_split) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < n; ++t)
    rope_token(y + t * heads * HEAD_DIM, seq0 + t, heads, H, W, theta, split, half_split);
}

/* Steps 1-3 for one token: x (bf16 Q or K row of width heads*128) at
 * sequence index s -> o (bf16). y is a scratch row of heads*128 doubles. */
static void norm_rope_row(const uint16_t* x, uint16_t* o, double* y, int64_t s, int32_t heads,
                          int32_t H, int32_t W, const uint16_t* gamma, double eps, double theta) {
  const int32_t split[3] = {44, 42, 42};
  const int64_t D = (int64_t)heads * HEAD_DIM;
  wan_oracle_rmsnorm(x, 1, D, D, gamma, eps, y);                           /* step 1 */
  for (int64_t c = 0; c < D; ++c) y[c] = wan_oracle_round_bf16(y[c]);  /* step 2 */
  rope_token(y, s, heads, H, W, theta, split, 0);                      /* step 3 */
  for (int64_t c = 0; c < D; ++c) o[c] = f64_to_bf16_bits(y[c]);
}

/* Steps 1-3 for the packed buffer [B, S, 3, heads, 128] (bf16 bits):
 * qkv_out gets normalised+rotated Q and K and a copy of V. */
void wan_oracle_qk_norm_rope(const uint16_t* qkv_in, uint16_t* qkv_out, int64_t batch,
                             int32_t F, int32_t H, int32_t W, int32_t heads,
                             const uint16_t* gamma_q, const uint16_t* gamma_k, double eps,
                             double theta) {
  const int64_t S = (int64_t)F * H * W, D = (int64_t)heads * HEAD_DIM, D3 = 3 * D;
  memcpy(qkv_out, qkv_in, (size_t)(batch * S * D3) * sizeof(uint16_t));
#pragma omp parallel
  {
    double* y = (double*)malloc((size_t)D * sizeof(double));
#pragma omp for schedule(static)
    for (int64_t bt = 0; bt < batch * S; ++bt) {
      norm_rope_row(qkv_in + bt * D3, qkv_out + bt * D3, y, bt % S, heads, H, W, gamma_q, eps, theta);
      norm_rope_row(qkv_in + bt * D3 + D, qkv_out + bt * D3 + D, y, bt % S, heads, H, W, gamma_k,
                    eps, theta);
    }
    free(y);
  }
}

/* Steps 1-3 for listed tokens only: tokens holds n pairs (b, s); out gets n
 * rows of [Q | K] (2 * heads * 128 bf16 each). */
void wan_oracle_qk_norm_rope_tokens(const uint16_t* qkv_in, int64_t batch, int32_t F, int32_t H,
                                    int32_t W, int32_t heads, const uint16_t* gamma_q,
                                    const uint16_t* gamma_k, double eps, double theta,
                                    const int64_t* tokens, int64_t n, uint16_t* out) {
  (void)batch;
  const int64_t S = (int64_t)F * H * W, D = (int64_t)heads * HEAD_DIM, D3 = 3 * D;
#pragma omp parallel
  {
    double* y = (double*)malloc((size_t)D * sizeof(double));
#pragma omp for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
      const int64_t bt = tokens[2 * r] * S + tokens[2 * r + 1];
      norm_rope_row(qkv_in + bt * D3, out + r * 2 * D, y, tokens[2 * r + 1], heads, H, W, gamma_q,
                    eps, theta);
      norm_rope_row(qkv_in + bt * D3 + D, out + r * 2 * D + D, y, tokens[2 * r + 1], heads, H, W,
                    gamma_k, eps, theta);
    }
    free(y);
  }
}

/* Step 4 on listed query rows. qkv: packed bf16 [B, S, 3, heads, 128] holding
 * the (already normalised and rotated) Q and K and V. rows: n triplets
 * (b, h, i). out: n x 128 fp64, unrounded. */
void wan_oracle_attention_rows(const uint16_t* qkv, int64_t batch, int64_t S, int32_t heads,
                               double scale, const int64_t* rows, int64_t n, double* out) {
  (void)batch;
  const int64_t D = (int64_t)heads * HEAD_DIM, D3 = 3 * D;
#pragma omp parallel
  {
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
      const uint16_t* base = qkv + b * S * D3;
      double q[HEAD_DIM];
      for (int d = 0; d < HEAD_DIM; ++d) q[d] = bf16_to_f64(base[i * D3 + h * HEAD_DIM + d]);
      /* pass 1: the largest logit */
      double m = -INFINITY;
      for (int64_t j = 0; j < S; ++j) {
        const uint16_t* k = base + j * D3 + D + h * HEAD_DIM;
        double dot = 0.0;
        for (int d = 0; d < HEAD_DIM; ++d) dot += q[d] * bf16_to_f64(k[d]);
        double l = dot * scale;
        if (l > m) m = l;
      }
      /* pass 2: exponentials, their sum and the weighted sum of V */
      double acc[HEAD_DIM];
      for (int d = 0; d < HEAD_DIM; ++d) acc[d] = 0.0;
      double sum = 0.0;
      for (int64_t j = 0; j < S; ++j) {
        const uint16_t* k = base + j * D3 + D + h * HEAD_DIM;
        const uint16_t* v = base + j * D3 + 2 * D + h * HEAD_DIM;
        double dot = 0.0;
        for (int d = 0; d < HEAD_DIM; ++d) dot += q[d] * bf16_to_f64(k[d]);
        double w = exp(dot * scale - m);
        sum += w;
        for (int d = 0; d < HEAD_DIM; ++d) acc[d] += w * bf16_to_f64(v[d]);
      }
      for (int d = 0; d < HEAD_DIM; ++d) out[r * HEAD_DIM + d] = acc[d] / sum;
    }
  }
}

/* Step 4 for one key range, as one round of ring context parallelism
 * (AWS Neuron "Optimizing High-Quality Offline Video Generation", "Context
 * parallelism": each rank's queries meet the K/V chunks one at a time, and
 * the rounds' results are combined). For each listed query row (b, h, i) of
 * q_qkv (packed [B, Sq, 3, heads, 128]) and the keys [k_row0, k_row0 + k_rows)
 * of kv ([B, kv_rows, kv_pitch], K then V in the last 2*heads*128 columns):
 *     a_j = scale * q_i . k_j,  m = max_j a_j,
 *     l = sum_j exp(a_j - m),    o = sum_j exp(a_j - m) v_j        (fp64)
 * o: n x 128, ml: n x 2 (m, l), natural-log units. The softmax of the range
 * is o / l; two ranges' states merge as in oracle.merge_partial. */
void wan_oracle_attention_partial_rows(const uint16_t* q_qkv, int64_t Sq, const uint16_t* kv, int64_t kv_rows,
                                       int64_t kv_pitch, int64_t k_row0, int64_t k_rows, int32_t heads,
                                       double scale, const int64_t* rows, int64_t n, double* o, double* ml) {
  const int64_t D = (int64_t)heads * HEAD_DIM, D3 = 3 * D;
  const int64_t k_col = kv_pitch - 2 * D, v_col = kv_pitch - D;
#pragma omp parallel
  {
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
      const uint16_t* qrow = q_qkv + (b * Sq + i) * D3 + h * HEAD_DIM;
      const uint16_t* kvb = kv + b * kv_rows * kv_pitch;
      double q[HEAD_DIM];
      for (int d = 0; d < HEAD_DIM; ++d) q[d] = bf16_to_f64(qrow[d]);
      /* pass 1: the largest logit of the range */
      double m = -INFINITY;
      for (int64_t j = k_row0; j < k_row0 + k_rows; ++j) {
        const uint16_t* k = kvb + j * kv_pitch + k_col + h * HEAD_DIM;
        double dot = 0.0;
        for (int d = 0; d < HEAD_DIM; ++d) dot += q[d] * bf16_to_f64(k[d]);
        if (dot * scale > m) m = dot * scale;
      }
      /* pass 2: exponentials, their sum and the weighted sum of V */
      double acc[HEAD_DIM];
      for (int d = 0; d < HEAD_DIM; ++d) acc[d] = 0.0;
      double sum = 0.0;
      for (int64_t j = k_row0; j < k_row0 + k_rows; ++j) {
        const uint16_t* k = kvb + j * kv_pitch + k_col + h * HEAD_DIM;
        const uint16_t* v = kvb + j * kv_pitch + v_col + h * HEAD_DIM;
        double dot = 0.0;
        for (int d = 0; d < HEAD_DIM; ++d) dot += q[d] * bf16_to_f64(k[d]);
        double w = exp(dot * scale - m);
        sum += w;
        for (int d = 0; d < HEAD_DIM; ++d) acc[d] += w * bf16_to_f64(v[d]);
      }
      for (int d = 0; d < HEAD_DIM; ++d) o[r * HEAD_DIM + d] = acc[d];
      ml[2 * r] = m;
      ml[2 * r + 1] = sum;
    }
  }
}

/* Step 4 with Skip-Softmax in threshold mode (vLLM-Omni "Wan2.2 Text-to-Video"
 * recipe, "Accelerating with TRTLLM_ATTN + Skip-Softmax": a direct skip
 * threshold, no calibration). The pages name the threshold but not the rule;
 * the reading implemented here:
 *   - keys come in tiles of 128 (tile j = keys [128j, 128j+128) below S);
 *     query rows in groups of 32 (group g = rows [32g, 32g+32));
 *   - in base-2 units, a_ik = (q_i . k_k) * scale * log2(e); t_ij is row i's
 *     largest a_ik over tile j, M_i(j) its largest a_ik over tiles < j;
 *   - tile j >= 1 is skipped for the group when every row i of the group has
 *     t_ij < M_i(j) + log2(threshold), i.e. every weight of the tile is below
 *     `threshold` times the row's running maximum weight. A skipped tile
 *     contributes neither to the row sum nor to the weighted sum of V. Tile 0
 *     is never skipped; threshold 0 means dense. A group with a row at or past
 *     S (a zero query: all its a_ik are 0) never skips.
 *   - o_i = sum over kept keys of exp(a_ik ln2 - m) v_k / sum of the same
 *     weights, m the row's largest a over kept keys (fp64, two passes).
 * groups: n triplets (b, h, g). out: n x 32 x 128 fp64 (rows past S: NaN).
 * skipped: n x n_tiles bytes (1 = skipped). margin: per group, the smallest
 * |max_i (t_ij - M_i(j)) - log2(threshold)| over its tiles j >= 1 (+inf when
 * none), so that a test can tell decisions that rounding could flip. */
void wan_oracle_attention_skip_groups(const uint16_t* qkv, int64_t batch, int64_t S, int32_t heads,
                                      double scale, double threshold, const int64_t* groups,
                                      int64_t n, double* out, uint8_t* skipped, double* margin) {
  (void)batch;
  const int64_t D = (int64_t)heads * HEAD_DIM, D3 = 3 * D;
  const int64_t n_tiles = (S + 127) / 128;
  const double lg = threshold > 0.0 ? log2(threshold) : -INFINITY;
  const double to_base2 = scale * 1.4426950408889634074;  /* log2(e) */
#pragma omp parallel
  {
    double* a = (double*)malloc((size_t)(32 * S) * sizeof(double));
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      const int64_t b = groups[3 * r], h = groups[3 * r + 1], g = groups[3 * r + 2];
      const uint16_t* base = qkv + b * S * D3;
      const int64_t i0 = 32 * g;
      int has_pad = 0;
      for (int64_t ii = 0; ii < 32; ++ii) {
        const int64_t i = i0 + ii;
        if (i >= S) {
          has_pad = 1;
          for (int64_t k = 0; k < S; ++k) a[ii * S + k] = 0.0;
          continue;
        }
        double q[HEAD_DIM];
        for (int d = 0; d < HEAD_DIM; ++d) q[d] = bf16_to_f64(base[i * D3 + h * HEAD_DIM + d]);
        for (int64_t k = 0; k < S; ++k) {
          const uint16_t* kk = base + k * D3 + D + h * HEAD_DIM;
          double dot = 0.0;
          for (int d = 0; d < HEAD_DIM; ++d) dot += q[d] * bf16_to_f64(kk[d]);
          a[ii * S + k] = dot * to_base2;
        }
      }
      /* the decisions */
      uint8_t* sk = skipped + r * n_tiles;
      double mg = INFINITY;
      sk[0] = 0;
      for (int64_t j = 1; j < n_tiles; ++j) {
        const int64_t k0 = 128 * j, k1 = (k0 + 128 < S) ? k0 + 128 : S;
        double worst = -INFINITY; /* max over rows of t_ij - M_i(j) */
        for (int64_t ii = 0; ii < 32; ++ii) {
          double M = -INFINITY, t = -INFINITY;
          for (int64_t k = 0; k < k0; ++k) M = fmax(M, a[ii * S + k]);
          for (int64_t k = k0; k < k1; ++k) t = fmax(t, a[ii * S + k]);
          worst = fmax(worst, t - M);
        }
        sk[j] = (!has_pad && worst < lg) ? 1 : 0;
        if (isfinite(lg)) mg = fmin(mg, fabs(worst - lg));
      }
      margin[r] = mg;
      /* the weighted sums over kept tiles */
      for (int64_t ii = 0; ii < 32; ++ii) {
        double* o = out + (r * 32 + ii) * HEAD_DIM;
        if (i0 + ii >= S) {
          for (int d = 0; d < HEAD_DIM; ++d) o[d] = NAN;
          continue;
        }
        double m = -INFINITY;
        for (int64_t k = 0; k < S; ++k)
          if (!sk[k / 128]) m = fmax(m, a[ii * S + k]);
        double acc[HEAD_DIM];
        for (int d = 0; d < HEAD_DIM; ++d) acc[d] = 0.0;
        double sum = 0.0;
        for (int64_t k = 0; k < S; ++k) {
          if (sk[k / 128]) continue;
          const uint16_t* v = base + k * D3 + 2 * D + h * HEAD_DIM;
          const double w = exp2(a[ii * S + k] - m);
          sum += w;
          for (int d = 0; d < HEAD_DIM; ++d) acc[d] += w * bf16_to_f64(v[d]);
        }
        for (int d = 0; d < HEAD_DIM; ++d) o[d] = acc[d] / sum;
      }
    }
    free(a);
  }
}

/* ---- FP8 (e4m3) attention variant ------------------------------------------
 * The path the pages time is FP8 attention (Neuron "Optimizing High-Quality
 * Offline Video Generation" and the TensorRT-LLM PR's profiling of TE FP8
 * attention) with per-tensor scales. Reading: a tensor X with scale s is
 * stored as codes c = e4m3(fl32(x * (1/s))) -- the product rounded to fp32
 * (the precision the kernel decides the code in), then round to nearest even
 * onto the e4m3 grid (3 mantissa bits, exponent bias 7, subnormals down to
 * 2^-9), saturating at +-448 -- and stands for c * s. Attention then runs on
 * the dequantised Q, K and V (fp64 here). */

/* e4m3 code (sign bit 7) of a finite double, round to nearest even, saturating. */
uint8_t wan_oracle_e4m3_encode(double v) {
  const uint8_t sign = (v < 0.0 || (v == 0.0 && signbit(v))) ? 0x80 : 0x00;
  double a = fabs(v);
  if (a == 0.0) return sign;
  int e;
  (void)frexp(a, &e); /* a = f * 2^e, f in [0.5, 1): the binade's exponent is e - 1 */
  int eb = e - 1;
  if (eb < -6) eb = -6; /* below 2^-6 the grid is the subnormal one, step 2^-9 */
  const double q = ldexp(1.0, eb - 3);
  double r = nearbyint(a / q) * q; /* exact: a / q is a power-of-two scaling */
  if (r > 448.0) r = 448.0;
  if (r == 0.0) return sign;
  int er;
  (void)frexp(r, &er);
  er -= 1;
  if (er < -6) return (uint8_t)(sign | (uint8_t)(r / ldexp(1.0, -9))); /* subnormal: m * 2^-9 */
  const int mant = (int)((r / ldexp(1.0, er) - 1.0) * 8.0);
  return (uint8_t)(sign | (uint8_t)((er + 7) << 3) | (uint8_t)mant);
}

double wan_oracle_e4m3_decode(uint8_t c) {
  const double s = (c & 0x80) ? -1.0 : 1.0;
  const int ef = (c >> 3) & 0xF, m = c & 7;
  if (ef == 0xF && m == 7) return NAN;
  if (ef == 0) return s * ldexp((double)m, -9);
  return s * ldexp(1.0 + m / 8.0, ef - 7);
}

/* codes of n bf16 values: e4m3(fl32(x * inv_scale)). */
void wan_oracle_quantize_e4m3(const uint16_t* x, int64_t n, float inv_scale, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    const float xf = (float)bf16_to_f64(x[i]);
    const float prod = xf * inv_scale; /* one fp32 rounding (contraction is off) */
    out[i] = wan_oracle_e4m3_encode((double)prod);
  }
}

/* Step 4 on e4m3 codes. qk8: [B, S, 2, heads, 128] codes of Q then K;
 * v8t: [B, heads, 128, s_pitch] codes of V transposed (dimension-major);
 * sq, sk, sv: the tensors' scales. rows: n triplets (b, h, i). out: n x 128
 * fp64, the attention of the dequantised values (unrounded). */
void wan_oracle_attention_fp8_rows(const uint8_t* qk8, const uint8_t* v8t, int64_t batch, int64_t S,
                                   int64_t s_pitch, int32_t heads, double scale, double sq, double sk,
                                   double sv, const int64_t* rows, int64_t n, double* out) {
  (void)batch;
  const int64_t D = (int64_t)heads * HEAD_DIM, D2 = 2 * D;
#pragma omp parallel
  {
    double* w = (double*)malloc((size_t)S * sizeof(double));
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n; ++r) {
      const int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
      const uint8_t* base = qk8 + b * S * D2;
      double q[HEAD_DIM];
      for (int d = 0; d < HEAD_DIM; ++d) q[d] = wan_oracle_e4m3_decode(base[i * D2 + h * HEAD_DIM + d]) * sq;
      double m = -INFINITY;
      for (int64_t j = 0; j < S; ++j) {
        const uint8_t* k = base + j * D2 + D + h * HEAD_DIM;
        double dot = 0.0;
        for (int d = 0; d < HEAD_DIM; ++d) dot += q[d] * (wan_oracle_e4m3_decode(k[d]) * sk);
        w[j] = dot * scale;
        if (w[j] > m) m = w[j];
      }
      double sum = 0.0;
      for (int64_t j = 0; j < S; ++j) {
        w[j] = exp(w[j] - m);
        sum += w[j];
      }
      const uint8_t* vt = v8t + (b * heads + h) * (int64_t)HEAD_DIM * s_pitch;
      for (int d = 0; d < HEAD_DIM; ++d) {
        double acc = 0.0;
        for (int64_t j = 0; j < S; ++j) acc += w[j] * (wan_oracle_e4m3_decode(vt[d * s_pitch + j]) * sv);
        out[r * HEAD_DIM + d] = acc / sum;
      }
    }
    free(w);
  }
}
