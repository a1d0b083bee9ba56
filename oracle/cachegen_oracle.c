/*
 * cachegen_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU restatement of the CacheGen KV-cache
 * codec, used to check the CUDA library bit for bit.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg may load it; the
 * library never does, and this file shares no code, header, table or helper
 * with the CUDA sources.
 *
 * Pages followed (cited by title and section):
 *   [Practice] "CacheGen实战：KV缓存压缩与流式传输在大型语言模型服务中的高效应用"
 *              sections 1, 2.1, 2.3, 3.1;
 *   [Overview] "CacheGen：大语言模型推理加速的KV缓存压缩与流式传输技术解析"
 *              sections "KV缓存的量化压缩机制", "量化编码器设计".
 * The pages give the method's shape (per-channel scale and zero point, deltas
 * between nearby tokens, layer-dependent steps, three levels, grouped entropy
 * coding, 1.5K-token chunks).  The exact codec -- anchors every 10 tokens,
 * 8-bit anchors, half-away-from-zero rounding, the [-127, 127] clamp, static
 * rANS with 12-bit tables per (layer, K/V, kv_head), one 32-bit stream per
 * (layer, K/V, token) and an offsets array -- is the reading this project
 * fixes where the pages are silent.  Every step below is written in the
 * order the method applies it, with no blocking or fusion.
 *
 * Two container formats: format 1 codes every token of a group as a delta to
 * the group's reconstructed anchor; format 2 reads [Practice] 1 literally
 * ("the difference between adjacent tokens") and codes token t as a delta to
 * the reconstruction of token t - 1, restarting at every anchor.  The formats
 * differ only in that reference and in the header's version field.
 *
 * Compiled with -O2 -ffp-contract=off and without -ffast-math, so every
 * float expression is one IEEE round-to-nearest operation per operator.
 *
 * Pins: every public function here is checked by tests against values that
 * come from outside this file (the step table as printed, brute-force
 * argmin, exact rational arithmetic, numpy's float16 conversion, a rANS
 * closed form, entropy bounds); see tests/test_oracle_*.py.
 */
#include "cachegen_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Status codes (same numbering as the library's public status enum).        */
enum {
  ORC_OK = 0,
  ORC_INVALID = 1,
  ORC_CAPACITY = 2,
  ORC_CORRUPT = 3,
  ORC_MISMATCH = 4,
  ORC_NONFINITE = 5
};

#define ORC_GROUP 10
#define ORC_M 4096u           /* 2^12: total of every frequency table */
#define ORC_RANS_L 32768u     /* 2^15: lower bound of the rANS state */
#define ORC_HEADER 64u
#define ORC_MAGIC 0x314B4743u /* "CGK1" little-endian */

/* ------------------------------------------------------------------------ */
/* fp16 <-> fp32, written from the IEEE 754 binary16 definition.             */

float orc_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  float v;
  if (e == 0) {
    v = ldexpf((float)m, -24); /* subnormal: m * 2^-24 (exact) */
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexpf((float)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* Round an fp32 value to the nearest binary16 value, ties to even. */
uint16_t orc_f32_to_f16(float x) {
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  if (isnan(x)) return (uint16_t)(sign | 0x7E00);
  float a = fabsf(x);
  if (isinf(a)) return (uint16_t)(sign | 0x7C00);
  if (a == 0.0f) return sign;
  /* The binary16 grid spacing in a's binade: 2^(e-11) for a in [2^(e-1), 2^e),
   * never finer than the subnormal spacing 2^-24. */
  int e;
  frexpf(a, &e); /* a = fr * 2^e, fr in [0.5, 1) */
  int qexp = e - 11;
  if (qexp < -24) qexp = -24;
  double units = ldexp((double)a, -qexp); /* a / spacing, exact */
  double r = rint(units);                 /* nearest, ties to even (default mode) */
  double v = ldexp(r, qexp);              /* the rounded magnitude, exact */
  if (v >= 65536.0) return (uint16_t)(sign | 0x7C00); /* rounds past 65504 */
  if (v < 6.103515625e-05) {               /* below 2^-14: subnormal */
    return (uint16_t)(sign | (uint16_t)ldexp(v, 24));
  }
  int ve;
  double vf = frexp(v, &ve); /* v = vf * 2^ve, vf in [0.5, 1) */
  int biased = ve - 1 + 15;
  int mant = (int)ldexp(vf, 11) - 1024;
  return (uint16_t)(sign | (biased << 10) | mant);
}

/* ------------------------------------------------------------------------ */
/* Layer-dependent steps: [Practice] 3.1 prints the three levels' steps for
 * the first / middle / last layers; [Practice] 1 says shallow layers are more
 * sensitive, so the first third takes the finest step.  Thirds: floor(3l/L). */

int orc_layer_third(int l, int L) { return (3 * l) / L; }

float orc_step(int level, int l, int L) {
  static const float steps[3][3] = {
      {0.3f, 0.8f, 1.2f}, /* high quality */
      {0.5f, 1.0f, 1.5f}, /* balanced */
      {0.8f, 1.5f, 2.0f}, /* fast */
  };
  return steps[level][orc_layer_third(l, L)];
}

/* ------------------------------------------------------------------------ */
/* Quantiser ([Overview] KV-cache quantisation mechanism: per-channel scale and
 * zero point; [Practice] 1: deltas between nearby tokens, uniform steps). */

void orc_anchor_params(const float* anchors, int m, float* zp, float* scale) {
  float lo = anchors[0], hi = anchors[0];
  for (int i = 1; i < m; i++) {
    if (anchors[i] < lo) lo = anchors[i];
    if (anchors[i] > hi) hi = anchors[i];
  }
  float sum = lo + hi;
  *zp = sum * 0.5f;
  float width = hi - lo;
  *scale = width / 254.0f;
}

static int clamp_round(float y) {
  float r = roundf(y); /* half away from zero */
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return (int)r;
}

int orc_anchor_code(float x, float zp, float scale) {
  if (scale == 0.0f) return 0;
  float d = x - zp;
  float y = d / scale;
  return clamp_round(y);
}

float orc_anchor_value(int c, float zp, float scale) {
  float prod = (float)c * scale;
  return zp + prod;
}

int orc_delta_code(float x, float ahat, float step) {
  float d = x - ahat;
  float y = d / step;
  return clamp_round(y);
}

float orc_delta_value(int q, float ahat, float step) {
  float prod = (float)q * step;
  return ahat + prod;
}

/* ------------------------------------------------------------------------ */
/* Frequency table normalisation to a total of 4096. */

void orc_normalize(const uint32_t counts[255], uint64_t total, uint16_t f[256]) {
  uint32_t g[256];
  uint64_t sum = 0;
  for (int u = 0; u < 256; u++) g[u] = 0;
  for (int u = 0; u < 255; u++) {
    if (counts[u] == 0) continue;
    uint64_t v = ((uint64_t)counts[u] * ORC_M) / total;
    if (v < 1) v = 1;
    g[u] = (uint32_t)v;
    sum += v;
  }
  if (sum < ORC_M) {
    int best = -1;
    for (int u = 0; u < 255; u++)
      if (counts[u] > 0 && (best < 0 || counts[u] > counts[best])) best = u;
    g[best] += (uint32_t)(ORC_M - sum);
    sum = ORC_M;
  }
  while (sum > ORC_M) {
    int best = -1;
    for (int u = 0; u < 255; u++)
      if (g[u] > 1 && (best < 0 || g[u] > g[best])) best = u;
    g[best] -= 1;
    sum -= 1;
  }
  for (int u = 0; u < 256; u++) f[u] = (uint16_t)g[u];
}

static void cum_of(const uint16_t f[256], uint32_t cum[257]) {
  cum[0] = 0;
  for (int u = 0; u < 256; u++) cum[u + 1] = cum[u] + f[u];
}

/* The symbol owning each of the 4096 slots: slot s belongs to the u with
 * cum[u] <= s < cum[u+1].  Slots no symbol covers (a table whose total is not
 * 4096) are marked 255, which no valid table can own. */
static void slots_of(const uint32_t cum[257], uint8_t slot_sym[4096]) {
  for (int s = 0; s < 4096; s++) slot_sym[s] = 255;
  for (int u = 0; u < 255; u++)
    for (uint32_t s = cum[u]; s < cum[u + 1] && s < 4096; s++) slot_sym[s] = (uint8_t)u;
}

/* ------------------------------------------------------------------------ */
/* rANS, one stream.  Symbol j (0-based) uses table number j / per_table;
 * table k's frequencies are freq[k*256 .. k*256+255] and its cumulative
 * frequencies cums[k*257 .. k*257+256]. */

static int64_t rans_encode_tabs(const uint8_t* sym, int nsym, int per_table, const uint16_t* freq,
                                const uint32_t* cums, uint16_t* words, int64_t cap,
                                uint16_t* tmp) {
  int64_t m = 0;
  uint32_t x = ORC_RANS_L;
  for (int j = nsym - 1; j >= 0; j--) {
    int k = j / per_table;
    uint32_t fs = freq[(size_t)k * 256 + sym[j]];
    uint32_t cum = cums[(size_t)k * 257 + sym[j]];
    if (fs == 0) return -2;
    /* renormalise: push 16 bits out when the step would leave [L, 2^16 L) */
    if ((uint64_t)x >= (((uint64_t)ORC_RANS_L >> 12) << 16) * fs) {
      tmp[m++] = (uint16_t)(x & 0xFFFF);
      x >>= 16;
    }
    x = (x / fs) * ORC_M + (x % fs) + cum;
  }
  tmp[m++] = (uint16_t)(x & 0xFFFF); /* flush the final state, low half first */
  tmp[m++] = (uint16_t)(x >> 16);
  if (m > cap) return -3;
  for (int64_t i = 0; i < m; i++) words[i] = tmp[m - 1 - i]; /* decoder reads in reverse */
  return m;
}

static int rans_decode_tabs(const uint16_t* words, int64_t nwords, int nsym, int per_table,
                            const uint16_t* freq, const uint32_t* cums, const uint8_t* slots,
                            uint8_t* sym) {
  if (nwords < 2) return ORC_CORRUPT;
  uint32_t x = ((uint32_t)words[0] << 16) | words[1];
  int64_t p = 2;
  for (int j = 0; j < nsym; j++) {
    int k = j / per_table;
    uint32_t slot = x & (ORC_M - 1);
    int u = slots[(size_t)k * 4096 + slot];
    if (u == 255) return ORC_CORRUPT;
    sym[j] = (uint8_t)u;
    x = freq[(size_t)k * 256 + u] * (x >> 12) + slot - cums[(size_t)k * 257 + u];
    if (x < ORC_RANS_L) { /* renormalise: pull the next 16 bits in */
      if (p >= nwords) return ORC_CORRUPT;
      x = (x << 16) | words[p++];
    }
  }
  if (x != ORC_RANS_L || p != nwords) return ORC_CORRUPT;
  return ORC_OK;
}

int64_t orc_rans_encode(const uint8_t* sym, int nsym, int per_table, const uint16_t* freq,
                        uint16_t* words, int64_t cap) {
  int ntab = (nsym + per_table - 1) / per_table;
  uint32_t* cums = (uint32_t*)malloc(sizeof(uint32_t) * 257 * (size_t)(ntab > 0 ? ntab : 1));
  uint16_t* tmp = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)nsym + 2));
  int64_t m = -1;
  if (cums && tmp) {
    for (int k = 0; k < ntab; k++) cum_of(freq + (size_t)k * 256, cums + (size_t)k * 257);
    m = rans_encode_tabs(sym, nsym, per_table, freq, cums, words, cap, tmp);
  }
  free(cums);
  free(tmp);
  return m;
}

int orc_rans_decode(const uint16_t* words, int64_t nwords, int nsym, int per_table,
                    const uint16_t* freq, uint8_t* sym) {
  int ntab = (nsym + per_table - 1) / per_table;
  if (ntab < 1) ntab = 1;
  uint32_t* cums = (uint32_t*)malloc(sizeof(uint32_t) * 257 * (size_t)ntab);
  uint8_t* slots = (uint8_t*)malloc((size_t)4096 * ntab);
  int rc = ORC_INVALID;
  if (cums && slots) {
    for (int k = 0; k < ntab; k++) {
      cum_of(freq + (size_t)k * 256, cums + (size_t)k * 257);
      slots_of(cums + (size_t)k * 257, slots + (size_t)k * 4096);
    }
    rc = rans_decode_tabs(words, nwords, nsym, per_table, freq, cums, slots, sym);
  }
  free(cums);
  free(slots);
  return rc;
}

/* ------------------------------------------------------------------------ */
/* Container layout. */

static uint64_t up16(uint64_t v) { return (v + 15) & ~(uint64_t)15; }

void orc_sections(int L, int H, int D, int64_t n, uint64_t offs[5]) {
  uint64_t chans = (uint64_t)L * 2 * H * D;
  offs[0] = ORC_HEADER;
  offs[1] = up16(offs[0] + 4 * chans);
  offs[2] = up16(offs[1] + 4 * chans);
  offs[3] = up16(offs[2] + (uint64_t)L * 2 * H * 256 * 2);
  offs[4] = up16(offs[3] + 4 * ((uint64_t)L * 2 * n + 1));
}

uint64_t orc_encoded_bound(int L, int H, int D, int C) {
  uint64_t offs[5];
  orc_sections(L, H, D, C, offs);
  uint64_t per_stream = 2 * ((uint64_t)H * D + 2);
  return up16(offs[4] + (uint64_t)L * 2 * C * per_stream);
}

static void put16(uint8_t* p, uint16_t v) {
  p[0] = (uint8_t)v;
  p[1] = (uint8_t)(v >> 8);
}
static void put32(uint8_t* p, uint32_t v) {
  for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put64(uint8_t* p, uint64_t v) {
  for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint16_t get16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t get32(const uint8_t* p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
  return v;
}
static uint64_t get64(const uint8_t* p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
  return v;
}
static void putf32(uint8_t* p, float v) {
  uint32_t b;
  memcpy(&b, &v, 4);
  put32(p, b);
}
static float getf32(const uint8_t* p) {
  uint32_t b = get32(p);
  float v;
  memcpy(&v, &b, 4);
  return v;
}

/* ------------------------------------------------------------------------ */
/* Quantise one chunk: symbols u = v + 127, laid out [L][2][n][H][D], plus the
 * per-channel zp and scale [L][2][H][D]. */

static size_t kv_index(int64_t T, int H, int D, int l, int kv, int64_t t, int h, int d) {
  return ((((size_t)l * 2 + kv) * (size_t)T + (size_t)t) * H + h) * (size_t)D + d;
}

/* adjacent == 0 (format 1): every token of a group is a delta to the group's
 * reconstructed anchor.  adjacent == 1 (format 2, [Practice] 1 read
 * literally: "the difference between adjacent tokens"): every token is a
 * delta to the reconstruction of the token just before it, x^_t =
 * x^_(t-1) + q_t * step, and the chain restarts at each group's anchor. */
int orc_quantize_chunk_v(int L, int H, int D, const uint16_t* kv, int64_t T, int64_t token_start,
                         int C, int level, int adjacent, uint8_t* sym, float* zp, float* scale) {
  if (L < 1 || H < 1 || D < 1 || C < 1 || level < 0 || level > 2) return ORC_INVALID;
  if (adjacent != 0 && adjacent != 1) return ORC_INVALID;
  if (token_start < 0 || token_start >= T) return ORC_INVALID;
  int64_t n = T - token_start;
  if (n > C) n = C;
  int64_t groups = (n + ORC_GROUP - 1) / ORC_GROUP;
  float* anchors = (float*)malloc(sizeof(float) * (size_t)groups);
  if (!anchors) return ORC_INVALID;
  for (int l = 0; l < L; l++) {
    float step = orc_step(level, l, L);
    for (int kvi = 0; kvi < 2; kvi++) {
      for (int h = 0; h < H; h++) {
        for (int d = 0; d < D; d++) {
          /* non-finite check over the whole channel of this chunk */
          for (int64_t t = 0; t < n; t++) {
            float x = orc_f16_to_f32(kv[kv_index(T, H, D, l, kvi, token_start + t, h, d)]);
            if (!isfinite(x)) {
              free(anchors);
              return ORC_NONFINITE;
            }
          }
          for (int64_t g = 0; g < groups; g++)
            anchors[g] = orc_f16_to_f32(
                kv[kv_index(T, H, D, l, kvi, token_start + g * ORC_GROUP, h, d)]);
          size_t ch = (((size_t)l * 2 + kvi) * H + h) * D + d;
          orc_anchor_params(anchors, (int)groups, &zp[ch], &scale[ch]);
          for (int64_t g = 0; g < groups; g++) {
            int c = orc_anchor_code(anchors[g], zp[ch], scale[ch]);
            float ahat = orc_anchor_value(c, zp[ch], scale[ch]);
            int64_t t0 = g * ORC_GROUP;
            sym[kv_index(n, H, D, l, kvi, t0, h, d)] = (uint8_t)(c + 127);
            float ref = ahat; /* what the next delta is taken against */
            for (int64_t t = t0 + 1; t < t0 + ORC_GROUP && t < n; t++) {
              float x = orc_f16_to_f32(kv[kv_index(T, H, D, l, kvi, token_start + t, h, d)]);
              int q = orc_delta_code(x, ref, step);
              sym[kv_index(n, H, D, l, kvi, t, h, d)] = (uint8_t)(q + 127);
              if (adjacent) ref = orc_delta_value(q, ref, step);
            }
          }
        }
      }
    }
  }
  free(anchors);
  return ORC_OK;
}

int orc_quantize_chunk(int L, int H, int D, const uint16_t* kv, int64_t T, int64_t token_start,
                       int C, int level, uint8_t* sym, float* zp, float* scale) {
  return orc_quantize_chunk_v(L, H, D, kv, T, token_start, C, level, 0, sym, zp, scale);
}

/* Frequency tables [L][2][H][256] of a quantised chunk. */
void orc_tables_of(int L, int H, int D, int64_t n, const uint8_t* sym, uint16_t* freq) {
  for (int l = 0; l < L; l++)
    for (int kvi = 0; kvi < 2; kvi++)
      for (int h = 0; h < H; h++) {
        uint32_t counts[255];
        memset(counts, 0, sizeof(counts));
        for (int64_t t = 0; t < n; t++)
          for (int d = 0; d < D; d++) counts[sym[kv_index(n, H, D, l, kvi, t, h, d)]]++;
        orc_normalize(counts, (uint64_t)n * D, freq + (((size_t)l * 2 + kvi) * H + h) * 256);
      }
}

/* ------------------------------------------------------------------------ */
/* Encode one chunk into a container ([Practice] 2.1: each chunk is encoded on
 * its own; [Practice] 1: quantise, then entropy-code). */

int orc_encode_chunk_v(int L, int H, int D, const uint16_t* kv, int64_t T, int64_t token_start,
                       int C, int level, int adjacent, uint8_t* out, uint64_t cap,
                       uint64_t* out_size) {
  if (L < 1 || H < 1 || D < 1 || C < 1 || level < 0 || level > 2) return ORC_INVALID;
  if (adjacent != 0 && adjacent != 1) return ORC_INVALID;
  if (token_start < 0 || token_start >= T) return ORC_INVALID;
  int64_t n = T - token_start;
  if (n > C) n = C;
  size_t chans = (size_t)L * 2 * H * D;
  size_t nsym_chunk = (size_t)L * 2 * n * H * D;
  uint8_t* sym = (uint8_t*)malloc(nsym_chunk);
  float* zp = (float*)malloc(sizeof(float) * chans);
  float* scale = (float*)malloc(sizeof(float) * chans);
  uint16_t* freq = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)L * 2 * H * 256);
  uint16_t* words = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)H * D + 2));
  uint16_t* tmp = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)H * D + 2));
  uint32_t* cums = (uint32_t*)malloc(sizeof(uint32_t) * 257 * (size_t)H);
  int rc = ORC_OK;
  if (!sym || !zp || !scale || !freq || !words || !tmp || !cums) {
    rc = ORC_INVALID;
    goto done;
  }
  rc = orc_quantize_chunk_v(L, H, D, kv, T, token_start, C, level, adjacent, sym, zp, scale);
  if (rc != ORC_OK) goto done;
  orc_tables_of(L, H, D, n, sym, freq);

  uint64_t offs[5];
  orc_sections(L, H, D, n, offs);
  if (cap < offs[4]) {
    rc = ORC_CAPACITY;
    goto done;
  }
  memset(out, 0, offs[4]);
  for (size_t i = 0; i < chans; i++) {
    putf32(out + offs[0] + 4 * i, zp[i]);
    putf32(out + offs[1] + 4 * i, scale[i]);
  }
  for (size_t i = 0; i < (size_t)L * 2 * H * 256; i++) put16(out + offs[2] + 2 * i, freq[i]);

  uint64_t pos = 0; /* payload bytes written so far */
  int64_t nstreams = (int64_t)L * 2 * n;
  for (int l = 0; l < L; l++)
    for (int kvi = 0; kvi < 2; kvi++) {
      const uint16_t* ftab = freq + ((size_t)l * 2 + kvi) * H * 256;
      for (int h = 0; h < H; h++) cum_of(ftab + (size_t)h * 256, cums + (size_t)h * 257);
      for (int64_t t = 0; t < n; t++) {
        int64_t s = ((int64_t)l * 2 + kvi) * n + t;
        put32(out + offs[3] + 4 * (uint64_t)s, (uint32_t)pos);
        const uint8_t* ss = sym + kv_index(n, H, D, l, kvi, t, 0, 0);
        int64_t m = rans_encode_tabs(ss, H * D, D, ftab, cums, words, (int64_t)H * D + 2, tmp);
        if (m < 0) {
          rc = ORC_INVALID;
          goto done;
        }
        if (offs[4] + pos + 2 * (uint64_t)m > cap) {
          rc = ORC_CAPACITY;
          goto done;
        }
        for (int64_t i = 0; i < m; i++) put16(out + offs[4] + pos + 2 * i, words[i]);
        pos += 2 * (uint64_t)m;
      }
    }
  put32(out + offs[3] + 4 * (uint64_t)nstreams, (uint32_t)pos);
  uint64_t total = up16(offs[4] + pos);
  if (total > cap) {
    rc = ORC_CAPACITY;
    goto done;
  }
  for (uint64_t i = offs[4] + pos; i < total; i++) out[i] = 0;

  memset(out, 0, ORC_HEADER);
  put32(out + 0, ORC_MAGIC);
  put16(out + 4, (uint16_t)(1 + adjacent)); /* format 1: anchor deltas; 2: adjacent */
  out[6] = (uint8_t)level;
  out[7] = ORC_GROUP;
  put32(out + 8, (uint32_t)L);
  put32(out + 12, (uint32_t)H);
  put32(out + 16, (uint32_t)D);
  put32(out + 20, (uint32_t)C);
  put32(out + 24, (uint32_t)n);
  put32(out + 28, 12);
  put64(out + 32, (uint64_t)token_start);
  put64(out + 40, pos);
  put64(out + 48, total);
  put64(out + 56, 0);
  *out_size = total;
done:
  free(sym);
  free(zp);
  free(scale);
  free(freq);
  free(words);
  free(tmp);
  free(cums);
  return rc;
}

int orc_encode_chunk(int L, int H, int D, const uint16_t* kv, int64_t T, int64_t token_start,
                     int C, int level, uint8_t* out, uint64_t cap, uint64_t* out_size) {
  return orc_encode_chunk_v(L, H, D, kv, T, token_start, C, level, 0, out, cap, out_size);
}

/* ------------------------------------------------------------------------ */
/* Decode one container ([Practice] 2.3: decode, then fill the model's KV).
 * Values go to out[L][2][n][H][D] (out_elems must hold them). */

int orc_decode_chunk_v(const uint8_t* in, uint64_t in_bytes, int L, int H, int D, int C,
                       int level, int adjacent, uint16_t* out, uint64_t out_elems,
                       int64_t* n_out, int64_t* start_out) {
  if (adjacent != 0 && adjacent != 1) return ORC_INVALID;
  if (in_bytes < ORC_HEADER) return ORC_CORRUPT;
  int version = get16(in + 4);
  if (get32(in) != ORC_MAGIC || (version != 1 && version != 2) || in[7] != ORC_GROUP ||
      get32(in + 28) != 12)
    return ORC_CORRUPT;
  if (version != 1 + adjacent) return ORC_MISMATCH; /* the other delta format */
  if (in[6] != level || get32(in + 8) != (uint32_t)L || get32(in + 12) != (uint32_t)H ||
      get32(in + 16) != (uint32_t)D || get32(in + 20) != (uint32_t)C)
    return ORC_MISMATCH;
  int64_t n = get32(in + 24);
  if (n < 1 || n > C) return ORC_CORRUPT;
  uint64_t offs[5];
  orc_sections(L, H, D, n, offs);
  uint64_t payload = get64(in + 40);
  uint64_t total = get64(in + 48);
  if (total > in_bytes || offs[4] + payload > total) return ORC_CORRUPT;
  if ((uint64_t)L * 2 * n * H * D > out_elems) return ORC_INVALID;
  *n_out = n;
  *start_out = (int64_t)get64(in + 32);

  size_t chans = (size_t)L * 2 * H * D;
  uint16_t* freq = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)L * 2 * H * 256);
  uint8_t* sym = (uint8_t*)malloc((size_t)n * H * D);
  uint32_t* cums = (uint32_t*)malloc(sizeof(uint32_t) * 257 * (size_t)H);
  uint8_t* slots = (uint8_t*)malloc((size_t)4096 * H);
  uint16_t* words = NULL;
  int rc = ORC_OK;
  if (!freq || !sym || !cums || !slots) {
    rc = ORC_INVALID;
    goto done;
  }
  for (size_t i = 0; i < (size_t)L * 2 * H * 256; i++) freq[i] = get16(in + offs[2] + 2 * i);
  for (size_t tb = 0; tb < (size_t)L * 2 * H; tb++) {
    uint32_t sum = 0;
    for (int u = 0; u < 256; u++) sum += freq[tb * 256 + u];
    if (sum != ORC_M || freq[tb * 256 + 255] != 0) {
      rc = ORC_CORRUPT;
      goto done;
    }
  }
  for (int l = 0; l < L; l++) {
    float step = orc_step(level, l, L);
    for (int kvi = 0; kvi < 2; kvi++) {
      const uint16_t* ftab = freq + ((size_t)l * 2 + kvi) * H * 256;
      for (int h = 0; h < H; h++) {
        cum_of(ftab + (size_t)h * 256, cums + (size_t)h * 257);
        slots_of(cums + (size_t)h * 257, slots + (size_t)h * 4096);
      }
      /* 1. every stream of this (l, kv) back to symbols */
      for (int64_t t = 0; t < n; t++) {
        int64_t s = ((int64_t)l * 2 + kvi) * n + t;
        uint64_t o0 = get32(in + offs[3] + 4 * (uint64_t)s);
        uint64_t o1 = get32(in + offs[3] + 4 * (uint64_t)(s + 1));
        if (o1 < o0 || o1 > payload || ((o1 - o0) & 1)) {
          rc = ORC_CORRUPT;
          goto done;
        }
        int64_t nw = (int64_t)((o1 - o0) / 2);
        uint16_t* w2 = (uint16_t*)realloc(words, sizeof(uint16_t) * (size_t)(nw + 1));
        if (!w2) {
          rc = ORC_INVALID;
          goto done;
        }
        words = w2;
        for (int64_t i = 0; i < nw; i++) words[i] = get16(in + offs[4] + o0 + 2 * (uint64_t)i);
        rc = rans_decode_tabs(words, nw, H * D, D, ftab, cums, slots, sym + (size_t)t * H * D);
        if (rc != ORC_OK) goto done;
      }
      /* 2. symbols back to values: anchors first, then their group's deltas */
      for (int h = 0; h < H; h++)
        for (int d = 0; d < D; d++) {
          size_t ch = (((size_t)l * 2 + kvi) * H + h) * D + d;
          float zp = getf32(in + offs[0] + 4 * ch);
          float scale = getf32(in + offs[1] + 4 * ch);
          for (int64_t t0 = 0; t0 < n; t0 += ORC_GROUP) {
            int c = (int)sym[((size_t)t0 * H + h) * D + d] - 127;
            float ahat = orc_anchor_value(c, zp, scale);
            out[kv_index(n, H, D, l, kvi, t0, h, d)] = orc_f32_to_f16(ahat);
            float ref = ahat;
            for (int64_t t = t0 + 1; t < t0 + ORC_GROUP && t < n; t++) {
              int q = (int)sym[((size_t)t * H + h) * D + d] - 127;
              float v = orc_delta_value(q, ref, step);
              out[kv_index(n, H, D, l, kvi, t, h, d)] = orc_f32_to_f16(v);
              if (adjacent) ref = v; /* format 2: the next delta builds on this token */
            }
          }
        }
    }
  }
  (void)chans;
done:
  free(freq);
  free(sym);
  free(cums);
  free(slots);
  free(words);
  return rc;
}

int orc_decode_chunk(const uint8_t* in, uint64_t in_bytes, int L, int H, int D, int C, int level,
                     uint16_t* out, uint64_t out_elems, int64_t* n_out, int64_t* start_out) {
  return orc_decode_chunk_v(in, in_bytes, L, H, D, C, level, 0, out, out_elems, n_out, start_out);
}

/* ------------------------------------------------------------------------ */
/* Array forms of the fp16 conversions (plain loops, for the tests). */

void orc_f32_to_f16_array(const float* x, uint16_t* h, int64_t n) {
  for (int64_t i = 0; i < n; i++) h[i] = orc_f32_to_f16(x[i]);
}

void orc_f16_to_f32_array(const uint16_t* h, float* x, int64_t n) {
  for (int64_t i = 0; i < n; i++) x[i] = orc_f16_to_f32(h[i]);
}
