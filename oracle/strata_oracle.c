/*
 * strata_oracle.c -- plain, slow CPU oracle for the routed-expert FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; its format decoder, number conversions and arithmetic are
 * written here from the layer's definition.
 *
 * What the layer computes (sources):
 *   - Strata walk-through, blog.5616760.com/0039, section 5 ("MoE 的本质"),
 *     flowchart: a router scores each token, the top-10 experts are chosen,
 *     their outputs are merged with softmax weights into the layer output.
 *   - Same page, section 4 and lcz.me/topic/2153 section 3.2: hidden 2560,
 *     512 experts per layer, expert width 640 (ModelGeometry literals).
 *   - ai-coding.wiselychen.com (Strata two-weeks review), "success idea one",
 *     step 1: the GPU runs the router, then the chosen experts; step 4: the
 *     expert results are summed.
 * The arithmetic the pages leave open is fixed by the workload definition
 * this library implements and is restated here:
 *   logits  = fp32( sum_h hidden[t,h] * W_r[h,e] ) + bias[e]     (exact sum, one rounding)
 *   p       = softmax over ALL E logits (double)
 *   top-k   = k largest logits, ties to the lower expert index, listed in
 *             descending-logit order
 *   w_j     = p_j / sum_{chosen} p                                  (fp32)
 *   expert  = SwiGLU MLP: g = x.W_gate, u = x.W_up, h = silu(g)*u, y = h.W_down
 *             with fp32 accumulation (an fp64 variant is kept as a cross-check)
 *   out[t]  = sum_j w_j * y_j (j = 0..k-1, in order) [+ shared expert y] in
 *             fp32, then rounded to bf16 (round to nearest even)
 *
 * Weight formats (blocks of 32 consecutive K elements of one output row, one
 * fp16 scale d per block; matrices are stored output-feature rows, K contiguous):
 *   fmt 1, Q2_32  : 2-bit code c, element k at byte k/4, bits 2*(k%4)..+1;
 *                   w = d * (c - 1.5)
 *   fmt 2, Q4CB_32: 4-bit code c, element k at byte k/2, low nibble for even
 *                   k, high nibble for odd k; w = d * KV[c] with the 16-entry
 *                   non-linear codebook below (the IQ4_NL table named by the
 *                   Strata walk-through, section 13)
 *   fmt 3, MXFP4_32: the OCP Microscaling (MX) v1.0 MXFP4 format, the
 *                   experts of the native-MXFP4 model tier (lcz.me/topic/2153,
 *                   model tier list, "ds4f-mxfp4"; the llama.cpp MXFP4 GGUF
 *                   line on the same page).  Element codes as in fmt 2 (one
 *                   nibble per element, low nibble for even k), each an FP4
 *                   E2M1 number: bit 3 sign, bits 2-1 exponent (bias 1),
 *                   bit 0 mantissa, exponent 0 subnormal; the block scale is
 *                   one E8M0 byte e (no sign, no mantissa): 2^(e-127), e = 255
 *                   is NaN.  w = e2m1(c) * 2^(e-127).  The scales plane holds
 *                   one byte per block instead of two.
 *   Expert blob: gate codes | gate scales | up codes | up scales | down codes |
 *   down scales, each plane starting on a 256-byte boundary.  gate and up are
 *   [I rows x H], down is [H rows x I].
 * Dequantisation is exact in fp32 for fmt 1 and 2: d has 11 significant bits
 * and the code value at most 8, so the product fits in 24 bits.  For fmt 3
 * the product is formed in double (exact: two significant bits times a power
 * of two) and rounded once to fp32, which is exact unless it leaves fp32's
 * range (e >= 253).
 *
 * Pins (tests/test_oracle_pins.py): hand-built blocks with known values,
 * brute-force top-k on tiny inputs, the k = E identical-expert identity with a
 * dense SwiGLU MLP, E = 1 against a float64 textbook MLP, exact scaling and
 * permutation invariants, bucket invariants, and closed-form sizes.  Output
 * values at full size have no printed worked example on the pages; beyond these
 * invariants they are pinned only through the pinned parts.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_VERSION 1

/* ------------------------------------------------------------------ numbers */

/* IEEE binary16 -> float, written from the format definition. */
static float half_to_float(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 31;
  int mant = h & 1023;
  double v;
  if (expo == 0) {
    v = ldexp((double)mant, -24); /* subnormal: mant * 2^-24 */
  } else if (expo == 31) {
    v = mant ? NAN : INFINITY;
  } else {
    v = ldexp((double)(mant + 1024), expo - 25); /* (1 + mant/1024) * 2^(expo-15) */
  }
  return (float)(sign ? -v : v);
}

/* bfloat16 -> float: the bf16 bits are the top half of an fp32. */
static float bf16_to_float(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round a double to the nearest bf16 (ties to even), for finite normal values
 * in bf16's range; zero keeps its sign. */
static uint16_t double_to_bf16(double v) {
  if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
  if (isnan(v)) return 0x7fc0;
  int e;
  double m = frexp(fabs(v), &e);      /* fabs(v) = m * 2^e, m in [0.5, 1) */
  double scaled = m * 256.0;          /* 8 significant bits -> [128, 256) */
  double r = nearbyint(scaled);       /* nearest, ties to even */
  float f = (float)ldexp(r, e - 8);   /* exact: r has at most 9 bits */
  if (v < 0) f = -f;
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ format */

static const int KV4[16] = {-127, -104, -83, -65, -49, -35, -22, -10,
                            1,    13,   25,  38,  53,  69,  89,  113};

static size_t round_up_256(size_t x) { return (x + 255) & ~(size_t)255; }

static size_t codes_plane_bytes(int fmt, int rows, int K) {
  return fmt == 1 ? (size_t)rows * (size_t)(K / 4) : (size_t)rows * (size_t)(K / 2);
}
/* fp16 scales for fmt 1 and 2, one E8M0 byte for fmt 3 */
static size_t scales_plane_bytes(int fmt, int rows, int K) {
  return (size_t)rows * (size_t)(K / 32) * (fmt == 3 ? 1 : 2);
}

/* OCP MX v1.0 FP4 (E2M1) element value, from the field definition. */
static double e2m1_value(int c) {
  const int sign = (c >> 3) & 1, ex = (c >> 1) & 3, man = c & 1;
  const double mag = ex == 0 ? 0.5 * man                    /* subnormal: m * 2^(1-bias) / 2 */
                             : ldexp(1.0 + 0.5 * man, ex - 1); /* (1 + m/2) * 2^(ex-bias) */
  return sign ? -mag : mag;
}

/* OCP MX v1.0 E8M0 scale value: 2^(e-127); 255 encodes NaN. */
static double e8m0_value(int e) { return e == 255 ? NAN : ldexp(1.0, e - 127); }

/* Offsets of the six planes of one expert blob.  which: 0 gate, 1 up, 2 down. */
static void plane_offsets(int fmt, int H, int I, int which, size_t* codes_off,
                          size_t* scales_off, int* rows, int* K) {
  size_t off = 0;
  for (int m = 0; m < 3; ++m) {
    int r = (m == 2) ? H : I;
    int k = (m == 2) ? I : H;
    size_t c = off;
    off = round_up_256(off + codes_plane_bytes(fmt, r, k));
    size_t s = off;
    off = round_up_256(off + scales_plane_bytes(fmt, r, k));
    if (m == which) {
      *codes_off = c;
      *scales_off = s;
      *rows = r;
      *K = k;
    }
  }
}

size_t oracle_expert_bytes(int fmt, int H, int I) {
  size_t off = 0;
  for (int m = 0; m < 3; ++m) {
    int r = (m == 2) ? H : I;
    int k = (m == 2) ? I : H;
    off = round_up_256(off + codes_plane_bytes(fmt, r, k));
    off = round_up_256(off + scales_plane_bytes(fmt, r, k));
  }
  return off;
}

int oracle_version(void) { return ORACLE_VERSION; }

/* Dequantise row `row` of matrix `which` (0 gate, 1 up, 2 down) of one expert
 * blob into K floats.  Returns 0, or -1 on a bad argument. */
int oracle_dequant_row(int fmt, const uint8_t* blob, int H, int I, int which,
                       int row, float* out) {
  if (fmt < 1 || fmt > 3 || which < 0 || which > 2 || H % 32 || I % 32) return -1;
  size_t co = 0, so = 0;
  int rows = 0, K = 0;
  plane_offsets(fmt, H, I, which, &co, &so, &rows, &K);
  if (row < 0 || row >= rows) return -1;
  const uint8_t* codes = blob + co + codes_plane_bytes(fmt, 1, K) * (size_t)row;
  const uint8_t* scales = blob + so + scales_plane_bytes(fmt, 1, K) * (size_t)row;
  for (int k = 0; k < K; ++k) {
    float w;
    if (fmt == 3) {
      int c = (codes[k / 2] >> (4 * (k % 2))) & 15;
      out[k] = (float)(e2m1_value(c) * e8m0_value(scales[k / 32]));
      continue;
    }
    uint16_t dbits = (uint16_t)(scales[2 * (k / 32)] | (scales[2 * (k / 32) + 1] << 8));
    float d = half_to_float(dbits);
    if (fmt == 1) {
      int c = (codes[k / 4] >> (2 * (k % 4))) & 3;
      w = d * ((float)c - 1.5f);
    } else {
      int byte = codes[k / 2];
      int c = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
      w = d * (float)KV4[c];
    }
    out[k] = w;
  }
  return 0;
}

/* ------------------------------------------------------------------ steps */

/* RMSNorm with unit gain: xhat = x / sqrt(mean(x^2) + eps), bf16 output. */
void oracle_rmsnorm(const float* x, int T, int H, double eps, uint16_t* out) {
  for (int t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int h = 0; h < H; ++h) ss += (double)x[(size_t)t * H + h] * (double)x[(size_t)t * H + h];
    double inv = 1.0 / sqrt(ss / (double)H + eps);
    for (int h = 0; h < H; ++h)
      out[(size_t)t * H + h] = double_to_bf16((double)x[(size_t)t * H + h] * inv);
  }
}

/* Router logits: fp32 of the exact dot product (accumulated in double; every
 * bf16 x bf16 product is exact in double), then + bias[e] in fp32.
 * W_r is [H, E] row-major. */
void oracle_router_logits(const uint16_t* hidden, const uint16_t* wr,
                          const float* bias, int T, int H, int E, float* logits) {
  for (int t = 0; t < T; ++t) {
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += (double)bf16_to_float(hidden[(size_t)t * H + h]) *
               (double)bf16_to_float(wr[(size_t)h * E + e]);
      float l = (float)acc;
      if (bias) l = l + bias[e];
      logits[(size_t)t * E + e] = l;
    }
  }
}

typedef struct {
  float v;
  int i;
} scored;

static int by_logit_desc_index_asc(const void* a, const void* b) {
  const scored* x = (const scored*)a;
  const scored* y = (const scored*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->i < y->i) ? -1 : (x->i > y->i);
}

/* Softmax over all E (double), top-k by (logit descending, index ascending),
 * weights renormalised over the chosen k, stored as fp32. */
int oracle_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w) {
  if (k < 1 || k > E) return -1;
  scored* s = (scored*)malloc(sizeof(scored) * (size_t)E);
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  if (!s || !p) {
    free(s);
    free(p);
    return -1;
  }
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e) mx = fmax(mx, (double)l[e]);
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp((double)l[e] - mx);
      z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= z;
    for (int e = 0; e < E; ++e) {
      s[e].v = l[e];
      s[e].i = e;
    }
    qsort(s, (size_t)E, sizeof(scored), by_logit_desc_index_asc);
    double chosen = 0.0;
    for (int j = 0; j < k; ++j) chosen += p[s[j].i];
    for (int j = 0; j < k; ++j) {
      ids[(size_t)t * k + j] = s[j].i;
      w[(size_t)t * k + j] = (float)(p[s[j].i] / chosen);
    }
  }
  free(s);
  free(p);
  return 0;
}

/* Counting sort of the P = T*k (token, slot) pairs by expert, stable in pair
 * order p = t*k + j.  perm[sorted position] = p, inv[p] = sorted position. */
int oracle_bucket(const int32_t* ids, int T, int k, int E, int32_t* counts,
                  int32_t* offsets, int32_t* perm, int32_t* inv) {
  if (T < 0 || k < 1 || E < 1) return -1;
  int P = T * k;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int p = 0; p < P; ++p) {
    if (ids[p] < 0 || ids[p] >= E) return -1;
    counts[ids[p]]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  if (!fill) return -1;
  for (int p = 0; p < P; ++p) {
    int e = ids[p];
    int pos = offsets[e] + fill[e]++;
    perm[pos] = p;
    inv[p] = pos;
  }
  free(fill);
  return 0;
}

/* One expert on one token.  x is the token's bf16 hidden row [H]; y gets [H]
 * fp32.  acc64 = 0: fp32 accumulation in k order; acc64 = 1: fp64 throughout,
 * y rounded once.  h = silu(g) * u is formed in double from the accumulated
 * g and u and rounded to fp32 (acc64 = 0). */
int oracle_expert_ffn(int fmt, const uint8_t* blob, int H, int I,
                      const uint16_t* x, float* y, int acc64) {
  float* wrow = (float*)malloc(sizeof(float) * (size_t)(H > I ? H : I));
  float* hf = (float*)malloc(sizeof(float) * (size_t)I);
  double* hd = (double*)malloc(sizeof(double) * (size_t)I);
  if (!wrow || !hf || !hd) {
    free(wrow);
    free(hf);
    free(hd);
    return -1;
  }
  for (int i = 0; i < I; ++i) {
    double g, u;
    if (oracle_dequant_row(fmt, blob, H, I, 0, i, wrow)) goto fail;
    if (acc64) {
      double a = 0.0;
      for (int h = 0; h < H; ++h) a += (double)bf16_to_float(x[h]) * (double)wrow[h];
      g = a;
    } else {
      float a = 0.0f;
      for (int h = 0; h < H; ++h) a += bf16_to_float(x[h]) * wrow[h];
      g = a;
    }
    if (oracle_dequant_row(fmt, blob, H, I, 1, i, wrow)) goto fail;
    if (acc64) {
      double a = 0.0;
      for (int h = 0; h < H; ++h) a += (double)bf16_to_float(x[h]) * (double)wrow[h];
      u = a;
    } else {
      float a = 0.0f;
      for (int h = 0; h < H; ++h) a += bf16_to_float(x[h]) * wrow[h];
      u = a;
    }
    double silu = g / (1.0 + exp(-g));
    hd[i] = silu * u;
    hf[i] = (float)(silu * u);
  }
  for (int n = 0; n < H; ++n) {
    if (oracle_dequant_row(fmt, blob, H, I, 2, n, wrow)) goto fail;
    if (acc64) {
      double a = 0.0;
      for (int i = 0; i < I; ++i) a += hd[i] * (double)wrow[i];
      y[n] = (float)a;
    } else {
      float a = 0.0f;
      for (int i = 0; i < I; ++i) a += hf[i] * wrow[i];
      y[n] = a;
    }
  }
  free(wrow);
  free(hf);
  free(hd);
  return 0;
fail:
  free(wrow);
  free(hf);
  free(hd);
  return -1;
}

/* Weighted combine for one token: acc = sum_j w_j * y_j in j order (fp32),
 * then + shared y (fp32).  out_f32 gets acc, out_bf16 its bf16 rounding,
 * residual_out (if given) residual + acc. */
static void combine_token(const float* const* yj, const float* w, int k, int H,
                          const float* shared, const float* residual,
                          float* out_f32, uint16_t* out_bf16, float* residual_out) {
  for (int h = 0; h < H; ++h) {
    float acc = 0.0f;
    for (int j = 0; j < k; ++j) {
      float prod = w[j] * yj[j][h];
      acc = acc + prod;
    }
    if (shared) acc = acc + shared[h];
    if (out_f32) out_f32[h] = acc;
    if (out_bf16) out_bf16[h] = double_to_bf16((double)acc);
    if (residual_out) residual_out[h] = residual[h] + acc;
  }
}

/* Combine from per-pair expert outputs y_pairs [T*k, H] in pair order. */
void oracle_combine(const float* y_pairs, const float* w, const float* shared,
                    const float* residual, int T, int k, int H, float* out_f32,
                    uint16_t* out_bf16, float* residual_out) {
  const float** yj = (const float**)malloc(sizeof(float*) * (size_t)k);
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) yj[j] = y_pairs + ((size_t)t * k + j) * H;
    combine_token(yj, w + (size_t)t * k, k, H, shared ? shared + (size_t)t * H : NULL,
                  residual ? residual + (size_t)t * H : NULL,
                  out_f32 ? out_f32 + (size_t)t * H : NULL,
                  out_bf16 ? out_bf16 + (size_t)t * H : NULL,
                  residual_out ? residual_out + (size_t)t * H : NULL);
  }
  free(yj);
}

/* The whole layer on T tokens (tokens are independent; OpenMP over tokens).
 *   hidden      bf16 [T, H] (the RMSNorm output the GPU received)
 *   wr          bf16 [H, E];  bias fp32 [E] or NULL
 *   blobs       E pointers to expert blobs of format fmt (a NULL entry is an
 *               error only if that expert is routed)
 *   shared_blob NULL, or one blob of format shared_fmt added with weight 1
 *   forced_ids  NULL, or [T, k] expert ids to use instead of the router's
 *   residual    NULL, or fp32 [T, H]
 * Outputs (any may be NULL): logits [T,E], ids [T,k], w [T,k],
 *   out_f32 [T,H], out_bf16 [T,H], residual_out [T,H].
 * Returns 0, or -1 on a bad argument or missing blob. */
int oracle_moe_layer(const uint16_t* hidden, int T, int H, const uint16_t* wr,
                     const float* bias, int E, int k, int fmt, int I,
                     const uint8_t* const* blobs, int shared_fmt,
                     const uint8_t* shared_blob, const int32_t* forced_ids,
                     const float* residual, float* logits, int32_t* ids, float* w,
                     float* out_f32, uint16_t* out_bf16, float* residual_out,
                     int acc64) {
  if (T < 0 || H <= 0 || E <= 0 || k < 1 || k > E || I <= 0) return -1;
  if (H % 32 || I % 32) return -1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int t = 0; t < T; ++t) {
    const uint16_t* x = hidden + (size_t)t * H;
    float* lg = (float*)malloc(sizeof(float) * (size_t)E);
    int32_t* tid = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    float* tw = (float*)malloc(sizeof(float) * (size_t)k);
    float* ybuf = (float*)malloc(sizeof(float) * (size_t)k * H);
    float* sh = shared_blob ? (float*)malloc(sizeof(float) * (size_t)H) : NULL;
    const float** yj = (const float**)malloc(sizeof(float*) * (size_t)k);
    if (!lg || !tid || !tw || !ybuf || !yj || (shared_blob && !sh)) {
      bad = 1;
    } else {
      oracle_router_logits(x, wr, bias, 1, H, E, lg);
      if (oracle_topk(lg, 1, E, k, tid, tw)) bad = 1;
      if (forced_ids) {
        /* forced routing: weights of the forced experts, renormalised */
        double mx = -INFINITY, z = 0.0, chosen = 0.0;
        for (int e = 0; e < E; ++e) mx = fmax(mx, (double)lg[e]);
        for (int e = 0; e < E; ++e) z += exp((double)lg[e] - mx);
        for (int j = 0; j < k; ++j) {
          int e = forced_ids[(size_t)t * k + j];
          if (e < 0 || e >= E) bad = 1;
          else chosen += exp((double)lg[e] - mx) / z;
        }
        for (int j = 0; j < k && !bad; ++j) {
          int e = forced_ids[(size_t)t * k + j];
          tid[j] = e;
          tw[j] = (float)((exp((double)lg[e] - mx) / z) / chosen);
        }
      }
      for (int j = 0; j < k && !bad; ++j) {
        const uint8_t* b = blobs[tid[j]];
        if (!b || oracle_expert_ffn(fmt, b, H, I, x, ybuf + (size_t)j * H, acc64)) bad = 1;
        yj[j] = ybuf + (size_t)j * H;
      }
      if (!bad && shared_blob && oracle_expert_ffn(shared_fmt, shared_blob, H, I, x, sh, acc64))
        bad = 1;
      if (!bad) {
        combine_token(yj, tw, k, H, sh, residual ? residual + (size_t)t * H : NULL,
                      out_f32 ? out_f32 + (size_t)t * H : NULL,
                      out_bf16 ? out_bf16 + (size_t)t * H : NULL,
                      residual_out ? residual_out + (size_t)t * H : NULL);
        if (logits) memcpy(logits + (size_t)t * E, lg, sizeof(float) * (size_t)E);
        if (ids) memcpy(ids + (size_t)t * k, tid, sizeof(int32_t) * (size_t)k);
        if (w) memcpy(w + (size_t)t * k, tw, sizeof(float) * (size_t)k);
      }
    }
    free(lg);
    free(tid);
    free(tw);
    free(ybuf);
    free(sh);
    free(yj);
  }
  return bad ? -1 : 0;
}

/* Number of OpenMP threads the layer function will use. */
int oracle_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    n =
#ifdef _OPENMP
        omp_get_num_threads();
#else
        1;
#endif
  }
  return n;
}
