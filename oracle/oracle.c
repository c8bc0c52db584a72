/*
 * CPU oracle for the variable-precision weight read path.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, plain, obviously-correct
 * reference that the CUDA library is checked against. Only the test suite,
 * the package's smoke check and the timed CPU baseline of the benchmark may
 * load it. Nothing in the product path links, imports or calls it, and it
 * shares no code, header, table or constant generator with the CUDA sources.
 *
 * Every floating-point result that has a plain definition is computed from
 * that definition in double precision; the lens rule, which decides integer
 * levels from fp32 arithmetic, is evaluated in fp32 with one fixed order of
 * IEEE-rounded operations (compile with -ffp-contract=off).
 *
 * Sources (page title, section):
 *  [FoQLens landing] "FoQLens" landing page, progress table, "A format of our
 *      own": one stored stack read at 2, 4, 6 or 8 bits without repacking;
 *      "The card reads a layout inside the pass": every block of rows read at
 *      its own depth; FoQZones mechanism, rule list 1-7.
 *  [FoQLens lens] "Precision where the question is, not everywhere", section
 *      "The mechanism": rules 1-7 (R_i = r_i f/(1-f), kappa, stops, lift,
 *      combine, level, memory bits), ladder ZERO < D2 < D4 < D6 < D8.
 *  [Precision on Demand] "Precision on Demand: Escalating Weight Bits at
 *      Uncertain Decoding Steps in a Small Local Model", abstract: store
 *      8-bit weights, decode with their top 4 bits, redo at 8 bits when the
 *      entropy is above a threshold or the top-two margin is small.
 *  [Ember v0.3] "v0.3, quantized on disk, quantized in memory", sections on
 *      GGUF layouts (Q4_K: 8 blocks per super-block with scales and offsets;
 *      Q6_K: 16 blocks with int8 scales) and the design constraint
 *      (dequantize only at block granularity inside the matmul).
 *
 * Readings where the pages are silent are listed at each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Scalar helpers                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 bit pattern -> float: a bf16 value is the top half of an fp32. */
static double bf16_to_double(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* IEEE binary16 bit pattern -> double (exact; handles subnormals, inf, nan). */
static double fp16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 31;
  int mant = h & 1023;
  double v;
  if (expo == 0)
    v = ldexp((double)mant, -24);
  else if (expo == 31)
    v = mant ? NAN : INFINITY;
  else
    v = ldexp((double)(mant + 1024), expo - 25);
  return sign ? -v : v;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

ORC_API int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Int8 absmax quantizer (test data).                                        */
/* The pages store "8-bit weights" and read a stack of them; the scale shape */
/* (fp32 absmax per row per 128 columns) and the rounding (half to even,     */
/* clamp to +-127, zero group -> zero codes) are the readings we take.       */
/* ------------------------------------------------------------------------ */
ORC_API void orc_quantize_int8(const float* w, int out, int in, int8_t* q, float* s) {
  const int G = in / 128;
  for (int r = 0; r < out; ++r) {
    for (int g = 0; g < G; ++g) {
      float amax = 0.0f;
      for (int c = 0; c < 128; ++c) {
        float a = fabsf(w[(size_t)r * in + 128 * g + c]);
        if (a > amax) amax = a;
      }
      float sc = amax / 127.0f;
      s[(size_t)r * G + g] = sc;
      for (int c = 0; c < 128; ++c) {
        size_t i = (size_t)r * in + 128 * g + c;
        int v = 0;
        if (sc > 0.0f) {
          float t = rintf(w[i] / sc);
          if (t > 127.0f) t = 127.0f;
          if (t < -127.0f) t = -127.0f;
          v = (int)t;
        }
        q[i] = (int8_t)v;
      }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Depth reconstruction ([FoQLens landing] "a format of our own";           */
/* [Precision on Demand] "top 4 bits of 8-bit weights").                    */
/*                                                                           */
/* Reading taken: the stored code is u = q + 128 in [1, 255]; a read at      */
/* depth d keeps the top d bits of u (plane k = bits 7-2k and 6-2k, k = 0 is  */
/* the top) and reconstructs at the centre of the bucket the dropped bits    */
/* span:  w_d = s * (u_d - 128 + c_d),  u_d = u with its low 8-d bits zero,  */
/* c_d = (2^(8-d) - 1) / 2.  Depth 0 (ZERO) contributes nothing.             */
/* ------------------------------------------------------------------------ */
static double recon_code(int8_t q, int depth) {
  if (depth <= 0) return 0.0;
  int u = (int)q + 128;
  int drop = 8 - depth;
  int ud = (u >> drop) << drop;
  double cd = ((double)(1 << drop) - 1.0) / 2.0;
  return (double)ud - 128.0 + cd;
}

/* w_d for one code and scale (exposed for the error-bound pins). */
ORC_API double orc_dequant_depth(int8_t q, float s, int depth) {
  return (double)s * recon_code(q, depth);
}

/* Ladder: level l in {0..4} reads 2*l bits (ZERO, D2, D4, D6, D8); a level
 * above 4 is read as 4 (library convention for out-of-range map entries). */
static int level_bits(uint8_t level) { return 2 * (level > 4 ? 4 : (int)level); }

/* y[t][r] = sum_c w_d(b(r))[r][c] * x[t][c], d = bits of levels[r / 64].    */
/* mass (optional) receives sum_c |w_d[r][c]| |x[t][c]|, the scale of the    */
/* tolerance the GPU result is held to.                                      */
ORC_API void orc_gemv_depth(const int8_t* q, const float* s, int out, int in, const uint8_t* levels,
                            const uint16_t* x, int batch, double* y, double* mass, int nthreads) {
  const int G = in / 128;
  set_threads(nthreads);
#pragma omp parallel for schedule(static)
  for (int r = 0; r < out; ++r) {
    int d = level_bits(levels[r / 64]);
    for (int t = 0; t < batch; ++t) {
      double acc = 0.0, am = 0.0;
      if (d > 0) {
        for (int c = 0; c < in; ++c) {
          double w = (double)s[(size_t)r * G + c / 128] * recon_code(q[(size_t)r * in + c], d);
          double xv = bf16_to_double(x[(size_t)t * in + c]);
          acc += w * xv;
          am += fabs(w) * fabs(xv);
        }
      }
      y[(size_t)t * out + r] = acc;
      if (mass) mass[(size_t)t * out + r] = am;
    }
  }
}

/* Escalation residual: dy[t][r] = sum_c (w_b - w_a)[r][c] x[t][c] with      */
/* a = bits(from_levels[blk]), b = bits(to_levels[blk]), w_0 = 0.            */
/* ([Precision on Demand]: the redo at 8 bits written as an addition to the  */
/* low pass.) Escalation only raises depth: a block with b <= a adds 0.      */
ORC_API void orc_gemv_residual(const int8_t* q, const float* s, int out, int in, const uint8_t* from_levels,
                               const uint8_t* to_levels, const uint16_t* x, int batch, double* dy, double* mass,
                               int nthreads) {
  const int G = in / 128;
  set_threads(nthreads);
#pragma omp parallel for schedule(static)
  for (int r = 0; r < out; ++r) {
    int a = level_bits(from_levels[r / 64]);
    int b = level_bits(to_levels[r / 64]);
    for (int t = 0; t < batch; ++t) {
      double acc = 0.0, am = 0.0;
      for (int c = 0; c < in && b > a; ++c) {
        int8_t qq = q[(size_t)r * in + c];
        double sc = (double)s[(size_t)r * G + c / 128];
        double dw = sc * recon_code(qq, b) - sc * recon_code(qq, a);
        double xv = bf16_to_double(x[(size_t)t * in + c]);
        acc += dw * xv;
        am += fabs(dw) * fabs(xv);
      }
      dy[(size_t)t * out + r] = acc;
      if (mass) mass[(size_t)t * out + r] = am;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Plane store (our storage layout of the one stored copy).                 */
/*                                                                           */
/* Block b (64 rows) occupies 8448 * G bytes, G = in / 128:                  */
/*   [0, 256 G)            fp32 scales, scale of (group g, row r) at 4(64g+r)*/
/*   [256 G + 2048 (G k + g) + 32 r + byte]   plane k in 0..3, group g, row r*/
/* so a block read at depth d is the contiguous prefix of 256 G + 1024 G d    */
/* bytes.  Inside the 32 bytes of (k, g, r) the 128 columns of the group are  */
/* four little-endian 32-bit words of 16 columns; column j of word w (j in    */
/* 0..15, column 16 w + j of the group) sits at bit                           */
/*      (8 (j % 4) + 6 - 2 k + 2 (j / 4)) mod 32                              */
/* and holds the 2-bit field p_k = (u >> (6 - 2k)) & 3 of u = q + 128.        */
/* ------------------------------------------------------------------------ */
ORC_API size_t orc_store_bytes(int out, int in) {
  return (size_t)(out / 64) * (size_t)(in / 128) * 8448u;
}

static size_t field_byte_and_shift(int G, int blk, int k, int g, int r, int col, int* shift) {
  int w = col / 16, j = col % 16;
  int bit = (8 * (j % 4) + 6 - 2 * k + 2 * (j / 4)) & 31;
  *shift = bit % 8;
  return (size_t)blk * 8448u * G + 256u * G + 2048u * ((size_t)G * k + g) + 32u * r + 4u * w + bit / 8;
}

ORC_API void orc_pack_planes(const int8_t* q, const float* s, int out, int in, uint8_t* store) {
  const int G = in / 128;
  memset(store, 0, orc_store_bytes(out, in));
  for (int r = 0; r < out; ++r) {
    int blk = r / 64, rr = r % 64;
    for (int g = 0; g < G; ++g) {
      float sc = s[(size_t)r * G + g];
      memcpy(store + (size_t)blk * 8448u * G + 4u * (64u * g + rr), &sc, 4);
      for (int col = 0; col < 128; ++col) {
        int u = (int)q[(size_t)r * in + 128 * g + col] + 128;
        for (int k = 0; k < 4; ++k) {
          int sh;
          size_t off = field_byte_and_shift(G, blk, k, g, rr, col, &sh);
          store[off] |= (uint8_t)(((u >> (6 - 2 * k)) & 3) << sh);
        }
      }
    }
  }
}

/* Inverse of orc_pack_planes: codes and scales back from the store. */
ORC_API void orc_unpack_planes(const uint8_t* store, int out, int in, int8_t* q, float* s) {
  const int G = in / 128;
  for (int r = 0; r < out; ++r) {
    int blk = r / 64, rr = r % 64;
    for (int g = 0; g < G; ++g) {
      memcpy(&s[(size_t)r * G + g], store + (size_t)blk * 8448u * G + 4u * (64u * g + rr), 4);
      for (int col = 0; col < 128; ++col) {
        int u = 0;
        for (int k = 0; k < 4; ++k) {
          int sh;
          size_t off = field_byte_and_shift(G, blk, k, g, rr, col, &sh);
          u |= ((store[off] >> sh) & 3) << (6 - 2 * k);
        }
        q[(size_t)r * in + 128 * g + col] = (int8_t)(u - 128);
      }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Lens rule ([FoQLens lens], "The mechanism", rules 1-6).                   */
/*                                                                           */
/*  1 R_i = r_i f / (1 - f)                                                  */
/*  2 kappa = gamma + floor(g (m - gamma))                                   */
/*  3 stops s_kappa < ... < s_(gamma+1), given ascending; s_last = s_(gamma+1)*/
/*  4 rho_i = d(b, c_i) / R_i;  L_i = max(0, 1 - rho_i / s_last)             */
/*  5 L = min(1, sum_i L_i)  (combine 0)  or  max_i L_i  (combine 1)          */
/*  6 rho* = s_last (1 - L); the ring rho* falls into; outside every lens: G  */
/*                                                                           */
/* Readings: distance is Euclidean in the plane; ring j (level j) covers      */
/* rho* in [s_(j+1), s_j) with s_(kappa+1) = 0, so level = gamma + #{stops     */
/* strictly above rho*}; R = 0 gives rho = 0 at distance 0 and +inf          */
/* elsewhere; kappa = gamma means no rings and every block sits at gamma.     */
/* All arithmetic is fp32 in this exact order, each operation rounded.        */
/* ------------------------------------------------------------------------ */
ORC_API int orc_lens_kappa(float g, int gamma, int m) {
  float t = g * (float)(m - gamma);
  return gamma + (int)floorf(t);
}

ORC_API void orc_level_map(const float* xy, int nblocks, const float* cxy, const float* r, int nlenses, float f,
                           float g, int gamma, int m, int nstops, const float* stops, int combine,
                           uint8_t* levels) {
  int kappa = orc_lens_kappa(g, gamma, m);
  (void)nstops;
  for (int b = 0; b < nblocks; ++b) {
    if (kappa <= gamma || nlenses == 0) {
      levels[b] = (uint8_t)gamma;
      continue;
    }
    float s_last = stops[kappa - gamma - 1];
    float L = 0.0f;
    for (int i = 0; i < nlenses; ++i) {
      float num = r[i] * f;
      float den = 1.0f - f;
      float R = num / den;
      float dx = xy[2 * b] - cxy[2 * i];
      float dy = xy[2 * b + 1] - cxy[2 * i + 1];
      float dx2 = dx * dx;
      float dy2 = dy * dy;
      float d = sqrtf(dx2 + dy2);
      float rho;
      if (R > 0.0f)
        rho = d / R;
      else
        rho = (d == 0.0f) ? 0.0f : INFINITY;
      float li = 1.0f - rho / s_last;
      if (!(li > 0.0f)) li = 0.0f;
      if (combine == 0)
        L = L + li;
      else if (li > L)
        L = li;
    }
    if (L > 1.0f) L = 1.0f;
    float rho_star = s_last * (1.0f - L);
    int lev = gamma;
    for (int j = 0; j < kappa - gamma; ++j)
      if (rho_star < stops[j]) lev += 1;
    levels[b] = (uint8_t)lev;
  }
}

/* Rule 7: memory bits = sum_b w_b bits(b) / sum_b w_b. */
ORC_API double orc_memory_bits(const uint8_t* levels, int nblocks, const double* wb, const double* bits_of_level) {
  double num = 0.0, den = 0.0;
  for (int b = 0; b < nblocks; ++b) {
    num += wb[b] * bits_of_level[levels[b]];
    den += wb[b];
  }
  return den > 0.0 ? num / den : 0.0;
}

/* ------------------------------------------------------------------------ */
/* In-pass level decision ([FoQLens landing], FoQZones mechanism: the layer  */
/* decides for itself from what entered it; score, reduced score, ladder     */
/* level capped at kappa, or the top share f by reduced score).              */
/*                                                                           */
/* Of the three scores the page tries, this is the draft one: the layer read */
/* at the base shows which units carry the step.                             */
/*   unit c        one 64-row block of the layer (the unit the store reads   */
/*                 at one depth)                                              */
/*   s_c           = ||y_c(base)||^2 * D_c^2: squares of the block's base-    */
/*                 level outputs, summed over its 64 rows and every row of    */
/*                 the batch                                                  */
/*   D_c^2         the block's squared quantization step at the base level,   */
/*                 (s[r][g] 2^(8 - bits(gamma)))^2 averaged over its rows r    */
/*                 and column groups g                                        */
/*   reduced       r_c = s_c * D_c^2 / w_c, w_c = 64 * in weights             */
/*   rule 0 ladder level = gamma + #{ j >= 1 : r_c >= lambda 16^j }, at most  */
/*                 kappa                                                      */
/*   rule 1 share  the floor(f * nblocks) blocks of largest r_c rise to       */
/*                 kappa (equal scores: the lower block index first); the     */
/*                 rest stay at gamma                                         */
/* Readings: the page leaves the score open; the draft variant is the one    */
/* that needs only the pass itself. The formula is taken as printed (D_c^2   */
/* enters the score and again the reduction). A "rise" in the share rule     */
/* goes to the cap kappa. 1 <= gamma <= kappa <= 4 (a ZERO base has no        */
/* draft). Everything in double.                                              */
/* ------------------------------------------------------------------------ */
typedef struct {
  double r;
  int idx;
} orc_scored;

static int orc_scored_desc(const void* a, const void* b) {
  const orc_scored* x = (const orc_scored*)a;
  const orc_scored* y = (const orc_scored*)b;
  if (x->r > y->r) return -1;
  if (x->r < y->r) return 1;
  return (x->idx > y->idx) - (x->idx < y->idx);
}

ORC_API int orc_level_decide(const float* y, int batch, int out, const float* s, int in, int gamma, int kappa,
                             int rule, double lambda, double f, uint8_t* levels, double* reduced) {
  if (gamma < 1 || kappa < gamma || kappa > 4 || out % 64 || in % 128 || (rule != 0 && rule != 1)) return -1;
  const int nb = out / 64, G = in / 128;
  const double step = ldexp(1.0, 8 - level_bits((uint8_t)gamma));
  orc_scored* order = (orc_scored*)malloc(sizeof(orc_scored) * (size_t)(nb > 0 ? nb : 1));
  if (!order) return -2;
  for (int c = 0; c < nb; ++c) {
    double yy = 0.0;
    for (int t = 0; t < batch; ++t)
      for (int r = 64 * c; r < 64 * c + 64; ++r) yy += (double)y[(size_t)t * out + r] * (double)y[(size_t)t * out + r];
    double d2 = 0.0;
    for (int r = 64 * c; r < 64 * c + 64; ++r)
      for (int g = 0; g < G; ++g) {
        double dl = (double)s[(size_t)r * G + g] * step;
        d2 += dl * dl;
      }
    d2 /= 64.0 * G;
    const double score = yy * d2;
    const double red = score * d2 / (64.0 * in);
    if (reduced) reduced[c] = red;
    order[c].r = red;
    order[c].idx = c;
    int lev = gamma;
    if (rule == 0) {
      for (int j = 1; j <= kappa - gamma; ++j)
        if (red >= lambda * ldexp(1.0, 4 * j)) lev += 1;
    }
    levels[c] = (uint8_t)lev;
  }
  if (rule == 1) {
    int n_up = (int)floor(f * (double)nb);
    if (n_up > nb) n_up = nb;
    if (n_up < 0) n_up = 0;
    qsort(order, (size_t)nb, sizeof(orc_scored), orc_scored_desc);
    for (int k = 0; k < n_up; ++k) levels[order[k].idx] = (uint8_t)kappa;
  }
  free(order);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Uncertainty gate ([Precision on Demand]: entropy above a threshold or a   */
/* small top-two margin). Readings: entropy of softmax(z) in nats; margin is  */
/* the probability gap p1 - p2 of the two largest logits; ties go to the     */
/* lower index; escalate = (H > tau_H) or (margin < tau_m).                  */
/* ------------------------------------------------------------------------ */
ORC_API void orc_logit_gate(const float* logits, int vocab, int batch, double tau_h, double tau_m, double* entropy,
                            double* margin, int32_t* top2, uint8_t* escalate) {
  for (int t = 0; t < batch; ++t) {
    const float* z = logits + (size_t)t * vocab;
    int i1 = 0;
    for (int v = 1; v < vocab; ++v)
      if (z[v] > z[i1]) i1 = v;
    int i2 = (i1 == 0) ? 1 : 0;
    for (int v = 0; v < vocab; ++v)
      if (v != i1 && z[v] > z[i2]) i2 = v;
    /* i2 must be the lowest index among the second-largest values. */
    for (int v = 0; v < vocab; ++v)
      if (v != i1 && z[v] == z[i2] && v < i2) i2 = v;
    double mx = (double)z[i1];
    double S = 0.0, T = 0.0;
    for (int v = 0; v < vocab; ++v) {
      double e = exp((double)z[v] - mx);
      S += e;
      T += ((double)z[v] - mx) * e;
    }
    double H = log(S) - T / S;
    double p1 = 1.0 / S;
    double p2 = exp((double)z[i2] - mx) / S;
    entropy[t] = H;
    margin[t] = p1 - p2;
    top2[2 * t] = i1;
    top2[2 * t + 1] = i2;
    escalate[t] = (uint8_t)((H > tau_h) || (p1 - p2 < tau_m));
  }
}

/* ------------------------------------------------------------------------ */
/* Verified speculation ([Precision on Demand], abstract: a low-precision     */
/* draft verified at 8 bits, counted in the same weight-byte cost model).     */
/* Readings: greedy speculation over a window of k steps. The draft token of  */
/* step t is the argmax of its D4 logits, the verified token the argmax of    */
/* its D8 logits (ties to the lower index, as the gate's top-2). The window   */
/* accepts the longest prefix of steps whose draft token equals the verified  */
/* one: accepted = a. It emits the verified tokens of steps 0..a (the a       */
/* accepted drafts and, when a < k, the correction at step a), so emitted =   */
/* min(a + 1, k) and the emitted sequence is the D8 model's own greedy one.   */
/* ------------------------------------------------------------------------ */
ORC_API void orc_spec_accept(const int32_t* draft, const int32_t* verified, int k, int32_t* accepted,
                             int32_t* emitted) {
  int a = 0;
  while (a < k && draft[a] == verified[a]) ++a;
  *accepted = a;
  *emitted = a < k ? a + 1 : k;
}

/* ------------------------------------------------------------------------ */
/* K-quant super-blocks ([Ember v0.3], GGUF layouts; dequantized per block    */
/* inside the product). The value rules are GGUF's; the byte layout is our    */
/* own with the GGUF byte counts (144 and 210 bytes per 256 weights).        */
/*                                                                           */
/* Q4_K, 144 bytes, 8 sub-blocks j of 32 weights:                            */
/*   [0,2) d fp16   [2,4) dmin fp16                                          */
/*   [4,12)  byte 4 + j  = sc_j | (mn_j & 3) << 6                            */
/*   [12,16) nibble j of the little-endian word (bits 4j..4j+3) = mn_j >> 2   */
/*   [16,144) byte 16 + 16 j + b (b = 0..15): low nibble = q of weight        */
/*            32 j + b, high nibble = q of weight 32 j + 16 + b              */
/*   w = d * sc_j * q - dmin * mn_j                                          */
/* Q6_K, 210 bytes, 16 sub-blocks j of 16 weights, 6-bit q (0..63).          */
/*   The parity of the record's row decides where the 192-byte q area sits:   */
/*   even row: [0,192) q, [192,208) sc_j int8, [208,210) d fp16              */
/*   odd row:  [0,2) d fp16, [2,194) q, [194,210) sc_j int8                  */
/*   q area: chunk t (0..3) = bytes [48 t, 48 t + 48), group m (0..3) =       */
/*   12 bytes at 48 t + 12 m = words A, B, C; with W(j, L) = 16 j + 4 t + L:  */
/*     A byte L = lo4 q[W(4m, L)]   | lo4 q[W(4m+1, L)] << 4                  */
/*     B byte L = lo4 q[W(4m+2, L)] | lo4 q[W(4m+3, L)] << 4                  */
/*     C byte L = hi2 q[W(4m+2, L)] | hi2 q[W(4m+3, L)] << 2                  */
/*              | hi2 q[W(4m, L)] << 4 | hi2 q[W(4m+1, L)] << 6               */
/*   w = d * sc_j * (q - 32)                                                 */
/* ------------------------------------------------------------------------ */
static uint16_t rd16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

ORC_API void orc_dequant_q4k(const uint8_t* blk, double* w) {
  double d = fp16_to_double(rd16(blk));
  double dmin = fp16_to_double(rd16(blk + 2));
  for (int j = 0; j < 8; ++j) {
    int sc = blk[4 + j] & 63;
    int mnlo = blk[4 + j] >> 6;
    int nib = (j % 2 == 0) ? (blk[12 + j / 2] & 15) : (blk[12 + j / 2] >> 4);
    int mn = mnlo | (nib << 2);
    for (int b = 0; b < 16; ++b) {
      uint8_t byte = blk[16 + 16 * j + b];
      w[32 * j + b] = d * (double)sc * (double)(byte & 15) - dmin * (double)mn;
      w[32 * j + 16 + b] = d * (double)sc * (double)(byte >> 4) - dmin * (double)mn;
    }
  }
}

ORC_API void orc_dequant_q6k(const uint8_t* blk, int odd, double* w) {
  const uint8_t* q = blk + (odd ? 2 : 0);
  const uint8_t* sc = blk + (odd ? 194 : 192);
  double d = fp16_to_double(rd16(blk + (odd ? 0 : 208)));
  int code[256];
  for (int t = 0; t < 4; ++t) {
    for (int m = 0; m < 4; ++m) {
      const uint8_t* A = q + 48 * t + 12 * m;
      const uint8_t* B = A + 4;
      const uint8_t* C = A + 8;
      for (int L = 0; L < 4; ++L) {
        int j0 = 4 * m, j1 = 4 * m + 1, j2 = 4 * m + 2, j3 = 4 * m + 3;
        code[16 * j0 + 4 * t + L] = (A[L] & 15) | (((C[L] >> 4) & 3) << 4);
        code[16 * j1 + 4 * t + L] = (A[L] >> 4) | (((C[L] >> 6) & 3) << 4);
        code[16 * j2 + 4 * t + L] = (B[L] & 15) | ((C[L] & 3) << 4);
        code[16 * j3 + 4 * t + L] = (B[L] >> 4) | (((C[L] >> 2) & 3) << 4);
      }
    }
  }
  for (int i = 0; i < 256; ++i) w[i] = d * (double)(int8_t)sc[i / 16] * (double)(code[i] - 32);
}

/* GGUF type ids for the two formats on the fast path. */
#define ORC_Q4_K 12
#define ORC_Q6_K 14

/* Storage order of a tensor's records (ours; the pages fix only a record's   */
/* content): 64-row blocks, then super-blocks, then the block's 64 rows, so   */
/* the record of (row r, super-block sb) is number                            */
/*   ((r / 64) * nsb + sb) * 64 + r % 64.                                     */
/* y[t][r] = sum_c w[r][c] x[t][c], each super-block dequantized then dotted.*/
ORC_API int orc_gemv_kquant(const uint8_t* blocks, int type, int out, int in, const uint16_t* x, int batch,
                            double* y, double* mass, int nthreads) {
  int rec;
  if (type == ORC_Q4_K)
    rec = 144;
  else if (type == ORC_Q6_K)
    rec = 210;
  else
    return -3;
  const int nsb = in / 256;
  set_threads(nthreads);
#pragma omp parallel for schedule(static)
  for (int r = 0; r < out; ++r) {
    double w[256];
    double acc[16], am[16];
    for (int t = 0; t < batch; ++t) acc[t] = am[t] = 0.0;
    for (int sb = 0; sb < nsb; ++sb) {
      const uint8_t* blk = blocks + (((size_t)(r / 64) * nsb + sb) * 64 + r % 64) * rec;
      if (type == ORC_Q4_K)
        orc_dequant_q4k(blk, w);
      else
        orc_dequant_q6k(blk, r & 1, w);
      for (int t = 0; t < batch; ++t)
        for (int i = 0; i < 256; ++i) {
          double xv = bf16_to_double(x[(size_t)t * in + 256 * sb + i]);
          acc[t] += w[i] * xv;
          am[t] += fabs(w[i]) * fabs(xv);
        }
    }
    for (int t = 0; t < batch; ++t) {
      y[(size_t)t * out + r] = acc[t];
      if (mass) mass[(size_t)t * out + r] = am[t];
    }
  }
  return 0;
}
