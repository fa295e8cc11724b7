/*
 * CPU oracle for MoE token dispatch and combine.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, single-threaded
 * statement of what the GPU path computes.  Only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg load it.  It shares no code,
 * header, table or constant with the CUDA library and includes none of it.
 *
 * Sources (web pages; the section named is where each definition is stated):
 *  [ASC]   Huawei torch_npu "npu_moe_distribute_combine" API reference:
 *          the function description (combine = weighted sum of the expert
 *          outputs returned along the dispatch path, plus the shared expert),
 *          and the parameter list (expert_ids, expand_idx, ep_send_counts,
 *          expert_scales, shared_expert_x, moe_expert_num, H, BS, K, A).
 *  [DEP]   DeepEP pull request "Intra-node compute compensation + overlap
 *          robustness (CUDA719 fix)", section "Kernel / host": fused unzip,
 *          chunk-completion counters, bounds guards.
 *  [TEMPO] TEMPO summary (makespan-aware expert load balancing), section 1:
 *          grouped GEMMs round each expert's tokens up to 128-token M-tiles.
 *
 * Floating point: arithmetic that the method defines exactly (sums, products)
 * is done in double and rounded once to the output type.  The FP8 quantiser
 * decides integer codes, so it works in float (fp32), the precision its
 * scale is stored in.
 *
 * Readings where the pages are silent (each repeated at its function):
 *  - expert e belongs to logical rank e / (E/R) (contiguous blocks);
 *  - rows of one expert are ordered by ascending token index;
 *  - each expert's rows are padded up to a multiple of 128; empty experts
 *    take no rows;
 *  - offsets are exclusive prefix sums with one extra entry (the total);
 *  - the shared-expert term is added without a weight.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_TILE 128

enum {
  OR_OK = 0,
  OR_ERR_INVALID_ARG = 1,
  OR_ERR_EXPERT_RANGE = 2,
  OR_ERR_DUPLICATE_EXPERT = 3,
  OR_ERR_CAPACITY = 4
};

/* ------------------------------------------------------------------------ */
/* Number formats                                                            */
/* ------------------------------------------------------------------------ */

/* bfloat16 = the upper 16 bits of an IEEE-754 binary32. */
double oracle_bf16_decode(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bfloat16, ties to even (IEEE-754 default
 * rounding), in one step.  bfloat16 keeps 8 significant bits (1 implicit +
 * 7 stored) and the binary32 exponent range, so in the binade [2^ex, 2^(ex+1))
 * the spacing is 2^(ex-7); below 2^-126 the spacing stays 2^-133 (subnormals). */
uint16_t oracle_bf16_encode(double v) {
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  if (isnan(v)) return (uint16_t)(sign | 0x7FC0u);
  double a = fabs(v);
  if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
  int ex = e - 1;
  if (ex < -126) ex = -126;
  double q = ldexp(1.0, ex - 7);
  double r = nearbyint(a / q) * q; /* a/q is exact: q is a power of two */
  const double max_finite = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
  if (r > max_finite) return (uint16_t)(sign | 0x7F80u);
  float f = (float)r; /* exact: r is a bfloat16 value */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(sign | (u >> 16));
}

/* OCP 8-bit floating point, E4M3 variant: 1 sign, 4 exponent (bias 7),
 * 3 mantissa bits; no infinities; S.1111.111 is NaN; largest finite 448;
 * exponent field 0 holds subnormals m/8 * 2^-6. */
double oracle_e4m3_decode(uint8_t c) {
  int s = c >> 7, E = (c >> 3) & 0xF, m = c & 7;
  if (E == 15 && m == 7) return NAN;
  double mag = (E == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), E - 10);
  return s ? -mag : mag;
}

/* Round to the nearest E4M3 value, ties to even, saturating: magnitudes that
 * round above 448 (and infinities) become 448.  NaN stays NaN (0x7F/0xFF). */
uint8_t oracle_e4m3_encode(double v) {
  uint8_t sign = signbit(v) ? 0x80u : 0u;
  if (isnan(v)) return (uint8_t)(sign | 0x7Fu);
  double a = fabs(v);
  double r;
  if (isinf(a)) {
    r = 448.0;
  } else if (a == 0.0) {
    return sign;
  } else {
    int e;
    frexp(a, &e);
    int ex = e - 1;
    if (ex < -6) ex = -6; /* subnormal spacing 2^-9 below 2^-6 */
    double q = ldexp(1.0, ex - 3);
    r = nearbyint(a / q) * q;
    if (r > 448.0) r = 448.0;
  }
  if (r == 0.0) return sign;
  if (r < ldexp(1.0, -6)) { /* subnormal: E = 0 */
    int m = (int)(r / ldexp(1.0, -9));
    return (uint8_t)(sign | m);
  }
  int e2;
  frexp(r, &e2);
  int ex2 = e2 - 1;                 /* r in [2^ex2, 2^(ex2+1)) */
  int E = ex2 + 7;
  int m = (int)((r / ldexp(1.0, ex2) - 1.0) * 8.0);
  return (uint8_t)(sign | (E << 3) | m);
}

/* ------------------------------------------------------------------------ */
/* Sizes                                                                     */
/* ------------------------------------------------------------------------ */

/* Padded row capacity.  Every non-empty expert adds at most 127 padding rows
 * to its c_e rows ([TEMPO] 128-token M-tiles), and at most min(E, T*K)
 * experts are non-empty, so P <= T*K + 127*min(E, T*K). */
int64_t oracle_padded_capacity(int64_t T, int K, int E) {
  int64_t n = T * (int64_t)K;
  int64_t ne = n < (int64_t)E ? n : (int64_t)E;
  int64_t cap = n + 127 * ne;
  return (cap + ORACLE_TILE - 1) / ORACLE_TILE * ORACLE_TILE;
}

/* ------------------------------------------------------------------------ */
/* Dispatch layout  ([ASC] expert_ids, expand_idx, ep_send_counts;          */
/*                   [TEMPO] 128-token M-tiles; [DEP] fused unzip mapping)  */
/* ------------------------------------------------------------------------ */

/*
 * ids       int32 [T, K]   top-K expert ids of each token
 * counts    int32 [E]      c_e = number of (t, k) with ids[t,k] == e
 * offsets   int32 [E + 1]  exclusive prefix sum of 128 * ceil(c_e / 128);
 *                          offsets[E] = P, the padded total
 * rank_counts  int32 [R]   sum of c_e over the experts of logical rank r
 * rank_offsets int32 [R+1] offsets[r * E/R]; rank_offsets[R] = P
 * dst_row   int32 [T * K]  row of slot (t, k) in the expert-major buffer:
 *                          offsets[e] + #{t' < t : e in ids[t']}; -1 if the
 *                          id is out of range
 * row_src   int32 [P_cap]  inverse map: slot index t*K + k, or -1 for padding
 *                          rows and for every row at or beyond P
 *
 * Validation ([ASC] expert_ids): ids in [0, E) and no repeats in a row.
 * Out-of-range ids take no row (they are not counted); repeated ids are
 * reported but still placed.  Returns the first error found in slot order
 * (OR_ERR_EXPERT_RANGE or OR_ERR_DUPLICATE_EXPERT), else OR_OK.
 */
int oracle_layout(const int32_t* ids, int64_t T, int K, int E, int R,
                  int32_t* counts, int32_t* offsets, int32_t* rank_counts,
                  int32_t* rank_offsets, int32_t* dst_row, int32_t* row_src,
                  int64_t P_cap) {
  if (T < 0 || K <= 0 || E <= 0 || R <= 0 || E % R != 0) return OR_ERR_INVALID_ARG;
  if (P_cap < oracle_padded_capacity(T, K, E)) return OR_ERR_CAPACITY;
  int status = OR_OK;

  /* validate, and count tokens per expert */
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t t = 0; t < T; ++t) {
    for (int k = 0; k < K; ++k) {
      int32_t e = ids[t * K + k];
      if (e < 0 || e >= E) {
        if (status == OR_OK) status = OR_ERR_EXPERT_RANGE;
        continue;
      }
      for (int j = 0; j < k; ++j)
        if (ids[t * K + j] == e && status == OR_OK) status = OR_ERR_DUPLICATE_EXPERT;
      counts[e] += 1;
    }
  }

  /* padded exclusive prefix sums over experts */
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) {
    int32_t padded = (counts[e] + ORACLE_TILE - 1) / ORACLE_TILE * ORACLE_TILE;
    offsets[e + 1] = offsets[e] + padded;
  }

  /* logical EP ranks own contiguous blocks of E/R experts */
  int El = E / R;
  for (int r = 0; r < R; ++r) {
    int32_t s = 0;
    for (int e = r * El; e < (r + 1) * El; ++e) s += counts[e];
    rank_counts[r] = s;
    rank_offsets[r] = offsets[r * El];
  }
  rank_offsets[R] = offsets[E];

  /* stable placement: tokens in ascending order inside each expert */
  for (int64_t p = 0; p < P_cap; ++p) row_src[p] = -1;
  int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  for (int64_t t = 0; t < T; ++t) {
    for (int k = 0; k < K; ++k) {
      int64_t slot = t * K + k;
      int32_t e = ids[slot];
      if (e < 0 || e >= E) {
        dst_row[slot] = -1;
        continue;
      }
      int32_t row = offsets[e] + fill[e]++;
      dst_row[slot] = row;
      row_src[row] = (int32_t)slot;
    }
  }
  free(fill);
  return status;
}

/* ------------------------------------------------------------------------ */
/* Dispatch permute ([DEP] fused unzip; [ASC] expand_x)                      */
/* ------------------------------------------------------------------------ */

/*
 * Byte-exact row scatter: xp[dst_row[t,k]] = x[t] for every placed slot,
 * padding rows [offsets[e] + counts[e], offsets[e+1]) all-zero bytes, rows
 * at or beyond P untouched.  Works on raw bytes, so the same routine serves
 * bf16 rows, E4M3 code rows and fp32 scale rows (a zero scale is 0.0f).
 */
void oracle_permute_rows(const uint8_t* x, int64_t T, int64_t row_bytes,
                         int64_t x_stride_bytes, const int32_t* dst_row, int K,
                         const int32_t* counts, const int32_t* offsets, int E,
                         uint8_t* xp) {
  for (int64_t t = 0; t < T; ++t)
    for (int k = 0; k < K; ++k) {
      int32_t row = dst_row[t * K + k];
      if (row < 0) continue;
      memcpy(xp + (int64_t)row * row_bytes, x + t * x_stride_bytes, (size_t)row_bytes);
    }
  for (int e = 0; e < E; ++e)
    for (int64_t p = (int64_t)offsets[e] + counts[e]; p < offsets[e + 1]; ++p)
      memset(xp + p * row_bytes, 0, (size_t)row_bytes);
}

/* ------------------------------------------------------------------------ */
/* Combine ([ASC] function description and expert_scales, shared_expert_x)  */
/* ------------------------------------------------------------------------ */

/*
 * out[t] = sum_k scales[t,k] * y[dst_row[t,k]]  +  shared[t]
 * y: bf16 [*, H]; scales: fp32 [T, K]; shared: bf16 [T, H] or NULL (no
 * shared expert); out: bf16 [T, H].  The sum is formed in double and rounded
 * once to bf16.  The shared term carries no weight.  Slots with
 * dst_row < 0 contribute nothing.
 */
void oracle_combine(const uint16_t* y, int64_t H, const int32_t* dst_row,
                    const float* scales, const uint16_t* shared, int64_t T, int K,
                    uint16_t* out) {
  double* acc = (double*)malloc((size_t)H * sizeof(double));
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t h = 0; h < H; ++h) acc[h] = 0.0;
    for (int k = 0; k < K; ++k) {
      int32_t row = dst_row[t * K + k];
      if (row < 0) continue;
      double s = (double)scales[t * K + k];
      const uint16_t* yr = y + (int64_t)row * H;
      for (int64_t h = 0; h < H; ++h) acc[h] += s * oracle_bf16_decode(yr[h]);
    }
    if (shared)
      for (int64_t h = 0; h < H; ++h) acc[h] += oracle_bf16_decode(shared[t * H + h]);
    for (int64_t h = 0; h < H; ++h) out[t * H + h] = oracle_bf16_encode(acc[h]);
  }
  free(acc);
}

/*
 * Backward of combine (out is linear in y and in scales):
 *   grad_y[dst_row[t,k]] = bf16(scales[t,k] * g[t])
 *   grad_scales[t,k]     = <g[t], y[dst_row[t,k]]>   (double, rounded to fp32)
 * Padding rows of grad_y (below P) are zero; rows at or beyond P untouched.
 */
void oracle_combine_bwd(const uint16_t* g, const uint16_t* y, int64_t H,
                        const float* scales, const int32_t* dst_row,
                        const int32_t* counts, const int32_t* offsets, int E,
                        int64_t T, int K, uint16_t* grad_y, float* grad_scales) {
  for (int64_t t = 0; t < T; ++t)
    for (int k = 0; k < K; ++k) {
      int32_t row = dst_row[t * K + k];
      if (row < 0) {
        grad_scales[t * K + k] = 0.0f;
        continue;
      }
      double s = (double)scales[t * K + k];
      const uint16_t* gr = g + t * H;
      const uint16_t* yr = y + (int64_t)row * H;
      uint16_t* gy = grad_y + (int64_t)row * H;
      double dot = 0.0;
      for (int64_t h = 0; h < H; ++h) {
        double gv = oracle_bf16_decode(gr[h]);
        gy[h] = oracle_bf16_encode(s * gv);
        dot += gv * oracle_bf16_decode(yr[h]);
      }
      grad_scales[t * K + k] = (float)dot;
    }
  for (int e = 0; e < E; ++e)
    for (int64_t p = (int64_t)offsets[e] + counts[e]; p < offsets[e + 1]; ++p)
      memset(grad_y + p * H, 0, (size_t)H * sizeof(uint16_t));
}

/*
 * Backward of dispatch (the permute copies x[t] to K rows, so its adjoint
 * sums those rows back):  grad_x[t] = bf16( sum_k grad_xp[dst_row[t,k]] ).
 */
void oracle_dispatch_bwd(const uint16_t* grad_xp, int64_t H, const int32_t* dst_row,
                         int64_t T, int K, uint16_t* grad_x) {
  double* acc = (double*)malloc((size_t)H * sizeof(double));
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t h = 0; h < H; ++h) acc[h] = 0.0;
    for (int k = 0; k < K; ++k) {
      int32_t row = dst_row[t * K + k];
      if (row < 0) continue;
      const uint16_t* r = grad_xp + (int64_t)row * H;
      for (int64_t h = 0; h < H; ++h) acc[h] += oracle_bf16_decode(r[h]);
    }
    for (int64_t h = 0; h < H; ++h) grad_x[t * H + h] = oracle_bf16_encode(acc[h]);
  }
  free(acc);
}

/* ------------------------------------------------------------------------ */
/* FP8 (E4M3) quantisation with one fp32 scale per 128 channels              */
/* ------------------------------------------------------------------------ */

/*
 * For each token t and channel block b of 128:
 *   amax = max |x|;  s = amax / 448 (fp32), or 1 when amax == 0;
 *   q    = E4M3(x / s) rounded to nearest even, saturating at 448.
 * x: bf16 [T, H] with row stride x_stride (elements); q: uint8 [T, H];
 * s: fp32 [T, H/128].  The divisions are fp32 (the type the scale is kept
 * in), so the code each element gets is decided in that precision.
 */
int oracle_quantize_e4m3(const uint16_t* x, int64_t T, int64_t H, int64_t x_stride,
                         uint8_t* q, float* s) {
  if (H % 128 != 0) return OR_ERR_INVALID_ARG;
  int64_t nb = H / 128;
  for (int64_t t = 0; t < T; ++t)
    for (int64_t b = 0; b < nb; ++b) {
      const uint16_t* xb = x + t * x_stride + b * 128;
      float amax = 0.0f;
      for (int c = 0; c < 128; ++c) {
        float a = fabsf((float)oracle_bf16_decode(xb[c]));
        if (a > amax) amax = a;
      }
      float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
      s[t * nb + b] = sc;
      for (int c = 0; c < 128; ++c) {
        float r = (float)oracle_bf16_decode(xb[c]) / sc;
        q[t * H + b * 128 + c] = oracle_e4m3_encode((double)r);
      }
    }
  return OR_OK;
}

/* deq = float(code) * scale, in fp32.  out: fp32 [T, H]. */
void oracle_dequantize_e4m3(const uint8_t* q, const float* s, int64_t T, int64_t H,
                            float* out) {
  int64_t nb = H / 128;
  for (int64_t t = 0; t < T; ++t)
    for (int64_t h = 0; h < H; ++h)
      out[t * H + h] = (float)oracle_e4m3_decode(q[t * H + h]) * s[t * nb + h / 128];
}

/* ------------------------------------------------------------------------ */
/* Chunk-completion check ([DEP] one acquire per chunk)                      */
/* ------------------------------------------------------------------------ */

/*
 * Content checksum of each complete 128-row tile j < P/128 of an
 * expert-major buffer: sum over the tile's 32-bit little-endian words w_i
 * (i counted from the tile's first byte, data rows then, if present, scale
 * rows) of w_i * (2i + 1), modulo 2^32.  The odd weights make a swap of
 * two unequal words inside a tile change the sum.
 */
void oracle_tile_checksums(const uint8_t* xp, int64_t row_bytes, const uint8_t* xs,
                           int64_t scale_row_bytes, int64_t n_tiles, uint32_t* out) {
  for (int64_t j = 0; j < n_tiles; ++j) {
    uint32_t acc = 0;
    uint32_t i = 0;
    const uint8_t* base = xp + j * ORACLE_TILE * row_bytes;
    for (int64_t b = 0; b < ORACLE_TILE * row_bytes; b += 4, ++i) {
      uint32_t w;
      memcpy(&w, base + b, 4);
      acc += w * (2u * i + 1u);
    }
    if (xs) {
      const uint8_t* sb = xs + j * ORACLE_TILE * scale_row_bytes;
      for (int64_t b = 0; b < ORACLE_TILE * scale_row_bytes; b += 4, ++i) {
        uint32_t w;
        memcpy(&w, sb + b, 4);
        acc += w * (2u * i + 1u);
      }
    }
    out[j] = acc;
  }
}
