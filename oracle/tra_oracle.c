/*
 * tra_oracle.c -- plain, slow, obviously-correct CPU oracle for tile-routed
 * mixed-precision causal attention (prefill and compressed-KV decode).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library; neither side includes the other.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 *        (no -ffast-math: the quantiser relies on IEEE fp32 divide and
 *         round-half-even under the default rounding mode).  OpenMP only
 *         spreads independent traversal rows over threads; every row is
 *         computed by one thread in the same order, so results do not depend
 *         on the thread count.
 *
 * Sources followed (page titles; the pages print no formulas, so each rule
 * below is the plainest reading of the cited sentence):
 *  [TRI]  "TriAttention: Unified Sparse Mixed-Precision Attention for
 *          Long-Context LLM Inference", abstract: QK tiles go to skip, 4-bit or
 *          8-bit computation; each head's regions are encoded by two
 *          diagonal-distance boundaries; boundaries generate precision-grouped
 *          traversals; one fused kernel combines both precisions into one
 *          normalised output; the quantised K/V are reused as a compressed KV
 *          cache for decoding.
 *  [TMX]  "TileMix: Tile-Centric Mixed-Precision Attention for LLM Inference
 *          Acceleration", abstract: hardware-aligned score tiles, routing
 *          decisions packed into bitmasks, one bit per group of adjacent key
 *          tiles, FP16 (here BF16) or INT8 score paths sharing one online
 *          softmax state, GQA, variable-length batches, INT8 K/V caches.
 *  [HYQ]  "HyQuant Uses Hybrid Precision to Compress LLM Attention",
 *          "How HyQuant works": dequantisation fused with decode attention.
 *
 * Conventions this library adopts where the pages are silent:
 *  - tiles are 64 tokens; a sequence of T tokens has nt = ceil(T/64) tiles and
 *    tile numbering restarts at every sequence start;
 *  - one symmetric scale per (head, tile) over all 64*d values of the tile:
 *    s8 = fl32(amax/127), s4 = fl32(amax/7); code = clamp(rne(fl32(x/s)));
 *    amax == 0 gives s = 0 and all codes 0; rows past the sequence end are
 *    excluded from amax and get code 0;
 *  - INT4 codes are packed two per byte, even channel in the low nibble;
 *  - boundary rule on dist = qt - kt: dist < b1 -> INT8, b1 <= dist < b2 ->
 *    INT4, dist >= b2 -> skip (1 <= b1 <= b2, so the diagonal is INT8);
 *  - bitmask rule: bit g of row (h, q-tile) covers k-tiles [gG, gG+G);
 *    1 -> BF16, 0 -> INT8; no skip state; LSB-first words;
 *  - a traversal row lists the INT4 k-tiles ascending, then INT8 ascending,
 *    then BF16 ascending; entry = (precision << 28) | kt with
 *    precision 1 = INT4, 2 = INT8, 3 = BF16;
 *  - prefill P*V uses the original bf16 V (precision is assigned to QK tiles);
 *  - decode cache precision of a k-tile is the highest precision any query
 *    head of the GQA group gives it at dist = (last prefill tile) - kt; in
 *    bitmask mode every cached tile is INT8.
 *  - FP8 middle band (an extension the pages do not describe: an FP8 score
 *    tier between INT8 and INT4): a third boundary b8 with b1 <= b8 <= b2;
 *    b1 <= dist < b8 -> FP8 (E4M3) instead of INT4; per (head, tile) scale
 *    sf = fl32(amax/448) and code = E4M3 round-to-nearest-even of fl32(x/sf),
 *    saturating at +-448; precision code 4, listed after the other groups;
 *    the decode cache keeps an FP8-band tile as INT8.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_TILE 64
#define ORC_SKIP 0
#define ORC_INT4 1
#define ORC_INT8 2
#define ORC_BF16 3
#define ORC_FP8 4

/* bf16 bit pattern -> double; exact (bf16 is the top half of an fp32). */
static double bf16_val(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static float bf16_f32(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

static int ceil_tiles(int T) { return (T + ORC_TILE - 1) / ORC_TILE; }

/* Tile offset of every sequence (tiles restart at each sequence start). */
static int64_t tile_offsets(const int32_t* cu, int B, int64_t* off /* [B+1] */) {
  off[0] = 0;
  for (int b = 0; b < B; ++b) off[b + 1] = off[b] + ceil_tiles(cu[b + 1] - cu[b]);
  return off[B];
}

/* Threads used by orc_prefill_rows (independent rows); n < 1 selects all cores. */
int orc_set_threads(int n) {
  if (n < 1) n = omp_get_num_procs();
  omp_set_num_threads(n);
  return n;
}

int64_t orc_num_tiles(const int32_t* cu, int B) {
  int64_t t = 0;
  for (int b = 0; b < B; ++b) t += ceil_tiles(cu[b + 1] - cu[b]);
  return t;
}

/* ---------------------------------------------------------------------------
 * Tile quantisation (per (head, 64-token tile) symmetric INT8 and INT4).
 * x: bf16 bits [ntok][H][d].  Outputs are tile-major per head:
 *   x8 [H][ntiles][64][d] int8, x4 [H][ntiles][64][d/2] packed, s8/s4 [H][ntiles].
 * Either of (x8,s8) or (x4,s4) may be NULL to skip that format.
 * ------------------------------------------------------------------------- */
static int8_t quant_code(float x, float s, int qmax) {
  if (s == 0.0f) return 0;
  float r = x / s;              /* IEEE fp32 divide, round-to-nearest-even */
  float c = nearbyintf(r);      /* round half to even (default FE_TONEAREST) */
  if (c > (float)qmax) c = (float)qmax;
  if (c < (float)-qmax) c = (float)-qmax;
  return (int8_t)c;
}

int orc_quantize(const uint16_t* x, const int32_t* cu, int B, int H, int d,
                 int8_t* x8, uint8_t* x4, float* s8, float* s4) {
  if (d % 2) return -1;
  int64_t* off = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  int64_t ntiles = tile_offsets(cu, B, off);
  for (int h = 0; h < H; ++h) {
    for (int b = 0; b < B; ++b) {
      int T = cu[b + 1] - cu[b];
      int nt = ceil_tiles(T);
      for (int t = 0; t < nt; ++t) {
        int64_t gt = off[b] + t;
        /* amax over the valid rows of this tile */
        float amax = 0.0f;
        for (int r = 0; r < ORC_TILE; ++r) {
          int tok = t * ORC_TILE + r;
          if (tok >= T) break;
          const uint16_t* row = x + ((int64_t)(cu[b] + tok) * H + h) * d;
          for (int c = 0; c < d; ++c) {
            float a = fabsf(bf16_f32(row[c]));
            if (a > amax) amax = a;
          }
        }
        float sc8 = amax / 127.0f;
        float sc4 = amax / 7.0f;
        if (s8) s8[(int64_t)h * ntiles + gt] = sc8;
        if (s4) s4[(int64_t)h * ntiles + gt] = sc4;
        for (int r = 0; r < ORC_TILE; ++r) {
          int tok = t * ORC_TILE + r;
          int valid = tok < T;
          const uint16_t* row = valid ? x + ((int64_t)(cu[b] + tok) * H + h) * d : NULL;
          int8_t* o8 = x8 ? x8 + (((int64_t)h * ntiles + gt) * ORC_TILE + r) * d : NULL;
          uint8_t* o4 = x4 ? x4 + (((int64_t)h * ntiles + gt) * ORC_TILE + r) * (d / 2) : NULL;
          for (int c = 0; c < d; ++c) {
            float xv = valid ? bf16_f32(row[c]) : 0.0f;
            if (o8) o8[c] = valid ? quant_code(xv, sc8, 127) : 0;
          }
          if (o4) {
            for (int c = 0; c < d; c += 2) {
              int8_t lo = valid ? quant_code(bf16_f32(row[c]), sc4, 7) : 0;
              int8_t hi = valid ? quant_code(bf16_f32(row[c + 1]), sc4, 7) : 0;
              o4[c / 2] = (uint8_t)(((uint8_t)lo & 0x0F) | (((uint8_t)hi & 0x0F) << 4));
            }
          }
        }
      }
    }
  }
  free(off);
  return 0;
}

/* Signed INT4 code of channel c from a packed row. */
static int int4_code(const uint8_t* row, int c) {
  int nib = (row[c / 2] >> ((c & 1) * 4)) & 0x0F;
  return nib >= 8 ? nib - 16 : nib;
}

/* ---------------------------------------------------------------------------
 * FP8 E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; code 0x7F / 0xFF is NaN, so the largest finite magnitude is
 * 1.75 * 2^8 = 448).  Magnitude code c = (e << 3) | m:
 *   e = 0: m/8 * 2^-6 (subnormal);  e >= 1: (1 + m/8) * 2^(e - 7).
 * ------------------------------------------------------------------------- */
double orc_e4m3_value(int code) {
  int e = (code >> 3) & 0xF, m = code & 7;
  double mag = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return (code & 0x80) ? -mag : mag;
}

/* Round-to-nearest-even of r onto the finite E4M3 values, saturating at +-448:
 * the nearest of the 127 non-negative finite magnitudes (a sorted table, binary
 * search, then the closer neighbour), a tie going to the even code (mantissa LSB
 * 0); the sign bit is r's own (so -0 and small negatives give 0x80). */
int orc_e4m3_encode(float r) {
  double a = fabs((double)r);
  int lo = 0, hi = 126;                       /* magnitude codes 0x00 .. 0x7E */
  if (a >= orc_e4m3_value(126)) {
    lo = 126;
  } else {
    while (hi - lo > 1) {                     /* value(lo) <= a < value(hi) */
      int mid = (lo + hi) / 2;
      if (orc_e4m3_value(mid) <= a) lo = mid; else hi = mid;
    }
    double dl = a - orc_e4m3_value(lo), dh = orc_e4m3_value(hi) - a;
    if (dh < dl || (dh == dl && (hi & 1) == 0)) lo = hi;
  }
  return (signbit(r) ? 0x80 : 0) | lo;
}

/* FP8 quantisation of one tensor: xf [H][ntiles][64][d] E4M3 codes, sf [H][ntiles]. */
int orc_quantize_f8(const uint16_t* x, const int32_t* cu, int B, int H, int d, uint8_t* xf,
                    float* sf) {
  int64_t* off = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  int64_t ntiles = tile_offsets(cu, B, off);
  for (int h = 0; h < H; ++h)
    for (int b = 0; b < B; ++b) {
      int T = cu[b + 1] - cu[b];
      int nt = ceil_tiles(T);
      for (int t = 0; t < nt; ++t) {
        int64_t gt = off[b] + t;
        float amax = 0.0f;
        for (int r = 0; r < ORC_TILE && t * ORC_TILE + r < T; ++r) {
          const uint16_t* row = x + ((int64_t)(cu[b] + t * ORC_TILE + r) * H + h) * d;
          for (int c = 0; c < d; ++c) {
            float a = fabsf(bf16_f32(row[c]));
            if (a > amax) amax = a;
          }
        }
        float s = amax / 448.0f;              /* IEEE fp32 divide */
        sf[(int64_t)h * ntiles + gt] = s;
        for (int r = 0; r < ORC_TILE; ++r) {
          int tok = t * ORC_TILE + r;
          uint8_t* o = xf + (((int64_t)h * ntiles + gt) * ORC_TILE + r) * d;
          for (int c = 0; c < d; ++c) {
            if (tok >= T || s == 0.0f) { o[c] = 0; continue; }
            float xv = bf16_f32(x[((int64_t)(cu[b] + tok) * H + h) * d + c]);
            o[c] = (uint8_t)orc_e4m3_encode(xv / s);
          }
        }
      }
    }
  free(off);
  return 0;
}

/* ---------------------------------------------------------------------------
 * Traversal lists.  Rows: prefill rows are (h, global q-tile) in h-major order;
 * decode-cache rows are (b, kv-head) in b-major order.
 * Pass row_ptr/entries NULL to only count; returns nnz (or -1 on error).
 * ------------------------------------------------------------------------- */
static int boundary_prec(int dist, int b1, int b2) {
  if (dist < b1) return ORC_INT8;
  if (dist < b2) return ORC_INT4;
  return ORC_SKIP;
}

/* with the FP8 middle band [b1, b8) */
static int boundary_prec3(int dist, int b1, int b8, int b2) {
  if (dist < b1) return ORC_INT8;
  if (dist < b8) return ORC_FP8;
  if (dist < b2) return ORC_INT4;
  return ORC_SKIP;
}

/* Emit one row's entries from a per-k-tile precision array, grouped. */
static int64_t emit_row(const int* prec, int n, uint32_t* entries, int64_t pos) {
  static const int order[4] = {ORC_INT4, ORC_INT8, ORC_BF16, ORC_FP8};
  for (int g = 0; g < 4; ++g)
    for (int kt = 0; kt < n; ++kt)
      if (prec[kt] == order[g]) {
        if (entries) entries[pos] = ((uint32_t)order[g] << 28) | (uint32_t)kt;
        ++pos;
      }
  return pos;
}

/* b8 may be NULL (no FP8 band, b8 = b1). */
int64_t orc_lists_boundary(const int32_t* cu, int B, int Hq, const int32_t* b1,
                           const int32_t* b8, const int32_t* b2, int32_t* row_ptr,
                           uint32_t* entries) {
  int64_t ntiles = orc_num_tiles(cu, B);
  int64_t pos = 0, row = 0;
  int nt_max = 0;
  for (int b = 0; b < B; ++b) if (ceil_tiles(cu[b + 1] - cu[b]) > nt_max) nt_max = ceil_tiles(cu[b + 1] - cu[b]);
  int* prec = (int*)malloc(sizeof(int) * (size_t)(nt_max + 1));
  for (int h = 0; h < Hq; ++h) {
    const int bm = b8 ? b8[h] : b1[h];
    if (b1[h] < 1 || bm < b1[h] || b2[h] < bm) { free(prec); return -1; }
    for (int b = 0; b < B; ++b) {
      int nt = ceil_tiles(cu[b + 1] - cu[b]);
      for (int qt = 0; qt < nt; ++qt, ++row) {
        if (row_ptr) row_ptr[row] = (int32_t)pos;
        for (int kt = 0; kt <= qt; ++kt) prec[kt] = boundary_prec3(qt - kt, b1[h], bm, b2[h]);
        pos = emit_row(prec, qt + 1, entries, pos);
      }
    }
  }
  if (row_ptr) row_ptr[row] = (int32_t)pos;
  (void)ntiles;
  free(prec);
  return pos;
}

/* bitmask: [Hq][ntiles][W] uint32; bit g of a row covers k-tiles [gG, gG+G). */
int64_t orc_lists_bitmask(const int32_t* cu, int B, int Hq, const uint32_t* bitmask,
                          int G, int W, int32_t* row_ptr, uint32_t* entries) {
  if (G < 1) return -1;
  int64_t ntiles = orc_num_tiles(cu, B);
  int64_t pos = 0, row = 0;
  int nt_max = 0;
  for (int b = 0; b < B; ++b) if (ceil_tiles(cu[b + 1] - cu[b]) > nt_max) nt_max = ceil_tiles(cu[b + 1] - cu[b]);
  if ((int64_t)W * 32 < (nt_max + G - 1) / G) return -1;
  int* prec = (int*)malloc(sizeof(int) * (size_t)(nt_max + 1));
  int64_t gt0 = 0;
  for (int h = 0; h < Hq; ++h) {
    gt0 = 0;
    for (int b = 0; b < B; ++b) {
      int nt = ceil_tiles(cu[b + 1] - cu[b]);
      for (int qt = 0; qt < nt; ++qt, ++row) {
        const uint32_t* words = bitmask + ((int64_t)h * ntiles + gt0 + qt) * W;
        if (row_ptr) row_ptr[row] = (int32_t)pos;
        for (int kt = 0; kt <= qt; ++kt) {
          int g = kt / G;
          int bit = (int)((words[g / 32] >> (g % 32)) & 1u);
          prec[kt] = bit ? ORC_BF16 : ORC_INT8;
        }
        pos = emit_row(prec, qt + 1, entries, pos);
      }
      gt0 += nt;
    }
  }
  if (row_ptr) row_ptr[row] = (int32_t)pos;
  free(prec);
  return pos;
}

/* mixed: the boundary rule decides skip / INT4 / INT8 by distance, and the
 * bitmask bit of a kept tile's group (bit g covers k-tiles [gG, gG+G), as in
 * orc_lists_bitmask) promotes it to BF16.  This combination of the two pages'
 * policies is a reading; neither page describes it. */
int64_t orc_lists_mixed(const int32_t* cu, int B, int Hq, const int32_t* b1, const int32_t* b2,
                        const uint32_t* bitmask, int G, int W, int32_t* row_ptr,
                        uint32_t* entries) {
  if (G < 1) return -1;
  int64_t ntiles = orc_num_tiles(cu, B);
  int64_t pos = 0, row = 0;
  int nt_max = 0;
  for (int b = 0; b < B; ++b) if (ceil_tiles(cu[b + 1] - cu[b]) > nt_max) nt_max = ceil_tiles(cu[b + 1] - cu[b]);
  if ((int64_t)W * 32 < (nt_max + G - 1) / G) return -1;
  int* prec = (int*)malloc(sizeof(int) * (size_t)(nt_max + 1));
  for (int h = 0; h < Hq; ++h) {
    if (b1[h] < 1 || b2[h] < b1[h]) { free(prec); return -1; }
    int64_t gt0 = 0;
    for (int b = 0; b < B; ++b) {
      int nt = ceil_tiles(cu[b + 1] - cu[b]);
      for (int qt = 0; qt < nt; ++qt, ++row) {
        const uint32_t* words = bitmask + ((int64_t)h * ntiles + gt0 + qt) * W;
        if (row_ptr) row_ptr[row] = (int32_t)pos;
        for (int kt = 0; kt <= qt; ++kt) {
          int pr = boundary_prec(qt - kt, b1[h], b2[h]);
          int g = kt / G;
          if (pr != ORC_SKIP && ((words[g / 32] >> (g % 32)) & 1u)) pr = ORC_BF16;
          prec[kt] = pr;
        }
        pos = emit_row(prec, qt + 1, entries, pos);
      }
      gt0 += nt;
    }
  }
  if (row_ptr) row_ptr[row] = (int32_t)pos;
  free(prec);
  return pos;
}

/* Decode-cache lists: rows (b, kvh).  mode 0 = boundary (b1,b2 per q head),
 * mode 1 = bitmask (every prefill tile cached as INT8). */
int64_t orc_lists_decode(const int32_t* cu, int B, int Hq, int Hkv, int mode,
                         const int32_t* b1, const int32_t* b8, const int32_t* b2,
                         int32_t* row_ptr, uint32_t* entries) {
  if (Hkv <= 0 || Hq % Hkv) return -1;
  int grp = Hq / Hkv;
  int64_t pos = 0, row = 0;
  int nt_max = 0;
  for (int b = 0; b < B; ++b) if (ceil_tiles(cu[b + 1] - cu[b]) > nt_max) nt_max = ceil_tiles(cu[b + 1] - cu[b]);
  int* prec = (int*)malloc(sizeof(int) * (size_t)(nt_max + 1));
  for (int b = 0; b < B; ++b) {
    int nt = ceil_tiles(cu[b + 1] - cu[b]);
    for (int kvh = 0; kvh < Hkv; ++kvh, ++row) {
      if (row_ptr) row_ptr[row] = (int32_t)pos;
      for (int kt = 0; kt < nt; ++kt) {
        int best = ORC_SKIP;
        if (mode == 1) {
          best = ORC_INT8;
        } else {
          for (int j = 0; j < grp; ++j) {
            int h = kvh * grp + j;
            /* an FP8-band tile is cached as INT8 */
            int p = boundary_prec3((nt - 1) - kt, b1[h], b8 ? b8[h] : b1[h], b2[h]);
            if (p == ORC_FP8) p = ORC_INT8;
            if (p > best) best = p;
          }
        }
        prec[kt] = best;
      }
      pos = emit_row(prec, nt, entries, pos);
    }
  }
  if (row_ptr) row_ptr[row] = (int32_t)pos;
  free(prec);
  return pos;
}

/* ---------------------------------------------------------------------------
 * Integer score tile: S_int[r][c] = sum_ch qcode[r][ch] * kcode[c][ch] over the
 * codes of the given precision (INT4 unpacked), no masking.  int64 arithmetic.
 * ------------------------------------------------------------------------- */
int orc_int_tile(int prec, int d, const int8_t* q8t, const uint8_t* q4t,
                 const int8_t* k8t, const uint8_t* k4t, int32_t* out /* [64][64] */) {
  for (int r = 0; r < ORC_TILE; ++r)
    for (int c = 0; c < ORC_TILE; ++c) {
      int64_t acc = 0;
      for (int ch = 0; ch < d; ++ch) {
        int a, bq;
        if (prec == ORC_INT8) {
          a = q8t[r * d + ch];
          bq = k8t[c * d + ch];
        } else if (prec == ORC_INT4) {
          a = int4_code(q4t + r * (d / 2), ch);
          bq = int4_code(k4t + c * (d / 2), ch);
        } else {
          return -1;
        }
        acc += (int64_t)a * bq;
      }
      out[r * ORC_TILE + c] = (int32_t)acc;
    }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Prefill for selected traversal rows.  rows[i] = h * ntiles + (global q-tile).
 * For every query token of the row's q-tile and every listed (kt, precision),
 * every causal key of that k-tile contributes one score; softmax and P*V in
 * fp64 over all kept keys (one normalised output per query).
 * out: [nrows][64][d] (rows past the sequence end are left 0);
 * lse: [nrows][64] natural-log logsumexp of the scaled scores (or NULL).
 * ------------------------------------------------------------------------- */
int orc_prefill_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     const int32_t* cu, int B, int Hq, int Hkv, int d,
                     const int8_t* q8, const uint8_t* q4, const float* sq8, const float* sq4,
                     const int8_t* k8, const uint8_t* k4, const float* sk8, const float* sk4,
                     const uint8_t* qf, const float* sqf, const uint8_t* kf, const float* skf,
                     const int32_t* row_ptr, const uint32_t* entries, double scale,
                     int nrows, const int64_t* rows, double* out, double* lse) {
  if (Hkv <= 0 || Hq % Hkv) return -1;
  int grp = Hq / Hkv;
  int64_t* off = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  int64_t ntiles = tile_offsets(cu, B, off);
  int nt_max = 0;
  for (int b = 0; b < B; ++b) if (ceil_tiles(cu[b + 1] - cu[b]) > nt_max) nt_max = ceil_tiles(cu[b + 1] - cu[b]);
  int bad = 0;
#pragma omp parallel
  {
  /* per-thread score and key buffers; each row is handled by one thread */
  double* s = (double*)malloc(sizeof(double) * (size_t)(nt_max + 1) * 2 * ORC_TILE);
  int64_t* key = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nt_max + 1) * 2 * ORC_TILE);
#pragma omp for schedule(dynamic, 1)
  for (int i = 0; i < nrows; ++i) {
    int64_t row = rows[i];
    int h = (int)(row / ntiles);
    int64_t gq = row % ntiles;
    int b = 0;
    while (!(gq >= off[b] && gq < off[b + 1])) ++b;
    int qt = (int)(gq - off[b]);
    int T = cu[b + 1] - cu[b];
    int kvh = h / grp;
    memset(out + (int64_t)i * ORC_TILE * d, 0, sizeof(double) * ORC_TILE * d);
    for (int r = 0; r < ORC_TILE; ++r) {
      int tq = qt * ORC_TILE + r;
      if (lse) lse[(int64_t)i * ORC_TILE + r] = 0.0;
      if (tq >= T) continue;
      int ns = 0;
      for (int32_t e = row_ptr[row]; e < row_ptr[row + 1]; ++e) {
        int prec = (int)(entries[e] >> 28);
        int kt = (int)(entries[e] & 0x0FFFFFFFu);
        int64_t gk = off[b] + kt;
        for (int c = 0; c < ORC_TILE; ++c) {
          int tk = kt * ORC_TILE + c;
          if (tk > tq || tk >= T) continue; /* causal and sequence-end mask */
          double sc;
          if (prec == ORC_BF16) {
            const uint16_t* qr = q + ((int64_t)(cu[b] + tq) * Hq + h) * d;
            const uint16_t* kr = k + ((int64_t)(cu[b] + tk) * Hkv + kvh) * d;
            double acc = 0.0;
            for (int ch = 0; ch < d; ++ch) acc += bf16_val(qr[ch]) * bf16_val(kr[ch]);
            sc = acc * scale;
          } else if (prec == ORC_FP8) {
            /* E4M3 values are exact in double, and so is the sum of their products */
            const uint8_t* qr = qf + (((int64_t)h * ntiles + gq) * ORC_TILE + r) * d;
            const uint8_t* kr = kf + (((int64_t)kvh * ntiles + gk) * ORC_TILE + c) * d;
            double acc = 0.0;
            for (int ch = 0; ch < d; ++ch) acc += orc_e4m3_value(qr[ch]) * orc_e4m3_value(kr[ch]);
            sc = acc * (double)sqf[(int64_t)h * ntiles + gq] * (double)skf[(int64_t)kvh * ntiles + gk] *
                 scale;
          } else {
            int64_t acc = 0;
            if (prec == ORC_INT8) {
              const int8_t* qr = q8 + (((int64_t)h * ntiles + gq) * ORC_TILE + r) * d;
              const int8_t* kr = k8 + (((int64_t)kvh * ntiles + gk) * ORC_TILE + c) * d;
              for (int ch = 0; ch < d; ++ch) acc += (int64_t)qr[ch] * kr[ch];
              sc = (double)acc * (double)sq8[(int64_t)h * ntiles + gq] *
                   (double)sk8[(int64_t)kvh * ntiles + gk] * scale;
            } else if (prec == ORC_INT4) {
              const uint8_t* qr = q4 + (((int64_t)h * ntiles + gq) * ORC_TILE + r) * (d / 2);
              const uint8_t* kr = k4 + (((int64_t)kvh * ntiles + gk) * ORC_TILE + c) * (d / 2);
              for (int ch = 0; ch < d; ++ch) acc += (int64_t)int4_code(qr, ch) * int4_code(kr, ch);
              sc = (double)acc * (double)sq4[(int64_t)h * ntiles + gq] *
                   (double)sk4[(int64_t)kvh * ntiles + gk] * scale;
            } else {
#pragma omp atomic write
              bad = 1;
              sc = 0.0;
            }
          }
          s[ns] = sc;
          key[ns] = tk;
          ++ns;
        }
      }
      /* softmax over the kept keys, then P*V with the original bf16 V */
      double m = -INFINITY;
      for (int j = 0; j < ns; ++j) if (s[j] > m) m = s[j];
      double l = 0.0;
      for (int j = 0; j < ns; ++j) l += exp(s[j] - m);
      double* o = out + ((int64_t)i * ORC_TILE + r) * d;
      for (int j = 0; j < ns; ++j) {
        double p = exp(s[j] - m) / l;
        const uint16_t* vr = v + ((int64_t)(cu[b] + key[j]) * Hkv + kvh) * d;
        for (int ch = 0; ch < d; ++ch) o[ch] += p * bf16_val(vr[ch]);
      }
      if (lse) lse[(int64_t)i * ORC_TILE + r] = m + log(l);
    }
  }
  free(s); free(key);
  }
  free(off);
  return bad ? -2 : 0;
}

/* ---------------------------------------------------------------------------
 * One decode step.  For every sequence b and query head h: scores against the
 * cached k-tiles listed for (b, kvh) (dequantised: k = sK * code) plus the bf16
 * tail tokens [0, tail_len[b]) (the new token already appended), softmax in
 * fp64, o = sum p * v with v = sV * code (cache) or the bf16 tail value.
 * qd: [B][Hq][d] bf16; tails: [B][Hkv][cap][d] bf16; out: [B][Hq][d] double.
 * ------------------------------------------------------------------------- */
int orc_decode_step(const uint16_t* qd, const int32_t* cu, int B, int Hq, int Hkv, int d,
                    const int8_t* k8, const uint8_t* k4, const float* sk8, const float* sk4,
                    const int8_t* v8, const uint8_t* v4, const float* sv8, const float* sv4,
                    const int32_t* row_ptr, const uint32_t* entries,
                    const uint16_t* k_tail, const uint16_t* v_tail, const int32_t* tail_len,
                    int cap, double scale, double* out) {
  if (Hkv <= 0 || Hq % Hkv) return -1;
  int grp = Hq / Hkv;
  int64_t* off = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  int64_t ntiles = tile_offsets(cu, B, off);
  int nt_max = 0;
  for (int b = 0; b < B; ++b) if (ceil_tiles(cu[b + 1] - cu[b]) > nt_max) nt_max = ceil_tiles(cu[b + 1] - cu[b]);
  int64_t maxkeys = (int64_t)nt_max * ORC_TILE + cap;
  double* s = (double*)malloc(sizeof(double) * (size_t)maxkeys);
  double* kv = (double*)malloc(sizeof(double) * (size_t)d);
  for (int b = 0; b < B; ++b) {
    int T = cu[b + 1] - cu[b];
    for (int h = 0; h < Hq; ++h) {
      int kvh = h / grp;
      int64_t row = (int64_t)b * Hkv + kvh;
      const uint16_t* qr = qd + ((int64_t)b * Hq + h) * d;
      int ns = 0;
      /* pass 1: scores */
      for (int32_t e = row_ptr[row]; e < row_ptr[row + 1]; ++e) {
        int prec = (int)(entries[e] >> 28);
        int kt = (int)(entries[e] & 0x0FFFFFFFu);
        int64_t gk = off[b] + kt;
        for (int c = 0; c < ORC_TILE; ++c) {
          if (kt * ORC_TILE + c >= T) { continue; }
          double acc = 0.0;
          for (int ch = 0; ch < d; ++ch) {
            double kval;
            if (prec == ORC_INT8)
              kval = (double)sk8[(int64_t)kvh * ntiles + gk] *
                     k8[(((int64_t)kvh * ntiles + gk) * ORC_TILE + c) * d + ch];
            else
              kval = (double)sk4[(int64_t)kvh * ntiles + gk] *
                     int4_code(k4 + (((int64_t)kvh * ntiles + gk) * ORC_TILE + c) * (d / 2), ch);
            acc += bf16_val(qr[ch]) * kval;
          }
          s[ns++] = acc * scale;
        }
      }
      for (int t = 0; t < tail_len[b]; ++t) {
        const uint16_t* kr = k_tail + (((int64_t)b * Hkv + kvh) * cap + t) * d;
        double acc = 0.0;
        for (int ch = 0; ch < d; ++ch) acc += bf16_val(qr[ch]) * bf16_val(kr[ch]);
        s[ns++] = acc * scale;
      }
      double m = -INFINITY;
      for (int j = 0; j < ns; ++j) if (s[j] > m) m = s[j];
      double l = 0.0;
      for (int j = 0; j < ns; ++j) l += exp(s[j] - m);
      double* o = out + ((int64_t)b * Hq + h) * d;
      for (int ch = 0; ch < d; ++ch) o[ch] = 0.0;
      /* pass 2: P*V in the same key order */
      int j = 0;
      for (int32_t e = row_ptr[row]; e < row_ptr[row + 1]; ++e) {
        int prec = (int)(entries[e] >> 28);
        int kt = (int)(entries[e] & 0x0FFFFFFFu);
        int64_t gk = off[b] + kt;
        for (int c = 0; c < ORC_TILE; ++c) {
          if (kt * ORC_TILE + c >= T) { continue; }
          double p = exp(s[j++] - m) / l;
          for (int ch = 0; ch < d; ++ch) {
            if (prec == ORC_INT8)
              kv[ch] = (double)sv8[(int64_t)kvh * ntiles + gk] *
                       v8[(((int64_t)kvh * ntiles + gk) * ORC_TILE + c) * d + ch];
            else
              kv[ch] = (double)sv4[(int64_t)kvh * ntiles + gk] *
                       int4_code(v4 + (((int64_t)kvh * ntiles + gk) * ORC_TILE + c) * (d / 2), ch);
            o[ch] += p * kv[ch];
          }
        }
      }
      for (int t = 0; t < tail_len[b]; ++t) {
        const uint16_t* vr = v_tail + (((int64_t)b * Hkv + kvh) * cap + t) * d;
        double p = exp(s[j++] - m) / l;
        for (int ch = 0; ch < d; ++ch) o[ch] += p * bf16_val(vr[ch]);
      }
    }
  }
  free(off); free(s); free(kv);
  return 0;
}
