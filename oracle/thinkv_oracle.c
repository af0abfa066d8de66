/*
 * thinkv_oracle.c -- plain, slow CPU oracle for the ThinKV decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY (see thinkv_oracle.h).  Build:
 *   gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fexcess-precision=standard
 *       -fno-fast-math [-fopenmp] thinkv_oracle.c -o libthinkv_oracle.so -lm
 *
 * Sources followed ("ThinKV: Thought-Adaptive KV Cache Compression for
 * Efficient Reasoning Models"):
 *   [TBQ]  explainer, Resume Technique > Methodologie > "Quantification
 *          Adaptative a la Pensee (TBQ)": each token's precision follows its
 *          thought type, R > E > T, by group quantisation.
 *   [TBE]  explainer, Methodologie > "Eviction Adaptative a la Pensee (TBE)":
 *          tokens of less important thoughts are evicted.
 *   [CT]   explainer, Methodologie > "Implementation Systeme: Pensee Continue
 *          (CT)" and the arXiv abstract: paged attention memory whose
 *          block table also records each slot's thought type, start index
 *          and eviction state; an evicted slot is refilled in place by a
 *          later token of the same type, so nothing is ever compacted.
 * Readings where the pages are silent (code format, rounding of the fp16
 * scale/zero, free-list discipline, eviction order, ...) are listed with the
 * design notes; each is marked "reading" below where it is used.
 */
#include "thinkv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ====================================================================== */
/* fp16 <-> fp32, written from the IEEE 754 binary16 definition           */
/* ====================================================================== */
float or_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  float v;
  if (e == 0) v = ldexpf((float)m, -24);                 /* subnormal: m * 2^-24 */
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexpf((float)(1024 + m), e - 25);            /* (1.m) * 2^(e-15) */
  return sign ? -v : v;
}

/* Magnitude of a (a >= 0, finite) truncated toward zero onto the binary16
 * grid, as a bit pattern; *inexact tells whether a was not on the grid.
 * Incrementing the bit pattern by one gives the next larger magnitude
 * (0x7BFF + 1 = 0x7C00 = infinity). */
static uint16_t f16_trunc_mag(float a, int* inexact) {
  if (a >= 65536.0f) { *inexact = 1; return 0x7BFF; }   /* above the largest finite */
  uint32_t u;
  memcpy(&u, &a, 4);
  uint32_t E = (u >> 23) & 0xFF, M = u & 0x7FFFFF;
  if (E >= 113) {                                       /* a >= 2^-14: binary16 normal */
    *inexact = (M & 0x1FFF) != 0;
    return (uint16_t)(((E - 112) << 10) | (M >> 13));
  }
  float y = a * 16777216.0f;                            /* a / 2^-24, exact */
  float n = floorf(y);                                  /* y < 1024 */
  *inexact = (n != y);
  return (uint16_t)n;
}

uint16_t or_f16_round_down(float x) {                   /* toward -infinity */
  if (isnan(x)) return 0x7E00;
  if (isinf(x)) return x > 0 ? 0x7C00 : 0xFC00;
  int inexact;
  if (!signbit(x)) return f16_trunc_mag(x, &inexact);
  uint16_t m = f16_trunc_mag(-x, &inexact);
  return (uint16_t)(0x8000 | (m + (inexact ? 1 : 0)));
}

uint16_t or_f16_round_up(float x) {                     /* toward +infinity */
  if (isnan(x)) return 0x7E00;
  if (isinf(x)) return x > 0 ? 0x7C00 : 0xFC00;
  int inexact;
  if (signbit(x)) return (uint16_t)(0x8000 | f16_trunc_mag(-x, &inexact));
  uint16_t m = f16_trunc_mag(x, &inexact);
  return (uint16_t)(m + (inexact ? 1 : 0));
}

uint16_t or_f16_round_nearest(float x) {                /* ties to even */
  if (isnan(x)) return 0x7E00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  float a = fabsf(x);
  if (isinf(a) || a >= 65520.0f) return (uint16_t)(sign | 0x7C00);
  uint32_t u;
  memcpy(&u, &a, 4);
  uint32_t E = (u >> 23) & 0xFF, M = u & 0x7FFFFF;
  uint16_t bits;
  if (E >= 113) {
    bits = (uint16_t)(((E - 112) << 10) | (M >> 13));
    uint32_t rest = M & 0x1FFF;
    if (rest > 0x1000 || (rest == 0x1000 && (bits & 1))) bits++;
  } else {
    float y = a * 16777216.0f, n = floorf(y), frac = y - n;
    bits = (uint16_t)n;
    if (frac > 0.5f || (frac == 0.5f && (bits & 1))) bits++;
  }
  return (uint16_t)(sign | bits);
}

/* element-wise rounding of an array (mode 0 = down, 1 = up, 2 = nearest) */
void or_f16_round_array(const float* x, int64_t n, int32_t mode, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i)
    out[i] = mode == 0 ? or_f16_round_down(x[i])
           : mode == 1 ? or_f16_round_up(x[i]) : or_f16_round_nearest(x[i]);
}

/* ====================================================================== */
/* [TBQ] group quantiser                                                   */
/* ====================================================================== */
/* One group of G consecutive channels of one token, b in {2,4,8}.
 * Reading: asymmetric integer codes; zero = the group minimum rounded DOWN to
 * fp16, scale = (max - zero)/(2^b - 1) in fp32 rounded UP to fp16, so every x
 * lies in [zero, zero + (2^b-1)*scale]; codes = round-half-even((x-zero)/scale)
 * with both fp32 operations rounded to nearest; a constant group has scale 0
 * and all codes 0.  Dequantised value: zero + code*scale (exact in fp64). */
void or_quantize_group(const uint16_t* x, int32_t G, int32_t bits,
                       uint8_t* codes, uint16_t* scale, uint16_t* zero) {
  float mn = INFINITY, mx = -INFINITY;
  for (int j = 0; j < G; ++j) {
    float v = or_f16_to_f32(x[j]);
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  uint16_t z = or_f16_round_down(mn);
  float zf = or_f16_to_f32(z);
  float levels = (float)((1 << bits) - 1);
  float diff = mx - zf;                                 /* fp32, rounded to nearest */
  float s32 = diff / levels;                            /* fp32, rounded to nearest */
  uint16_t s = or_f16_round_up(s32);
  float sf = or_f16_to_f32(s);
  for (int j = 0; j < G; ++j) {
    if (sf == 0.0f) { codes[j] = 0; continue; }
    float v = or_f16_to_f32(x[j]);
    float t = (v - zf) / sf;                            /* two fp32 RN operations */
    float c = rintf(t);                                 /* ties to even */
    if (c < 0.0f) c = 0.0f;
    if (c > levels) c = levels;
    codes[j] = (uint8_t)c;
  }
  *scale = s;
  *zero = z;
}

/* ====================================================================== */
/* [TBQ] the pages' float formats: FP8 E4M3, FP4 E2M1, ternary             */
/* ====================================================================== */
/* The explainer's TBQ names 8-bit FP8 or 4-bit NVFP4 for Reasoning tokens
 * and 2-bit ternary for Transition tokens.  Formats, from their definitions:
 *   E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
 *         subnormal (m/8 * 2^-6); S.1111.111 is NaN, so the largest finite
 *         value is 1.75 * 2^8 = 448; no infinities.
 *   E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit: 0, 0.5, 1, 1.5, 2,
 *         3, 4, 6 and their negatives.
 * Rounding from fp32: to the nearest value, ties to the even mantissa, and
 * magnitudes beyond the largest finite value saturate to it. */
double or_e4m3_value(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);                  /* m/8 * 2^-6 */
  else v = ldexp(8.0 + m, e - 10);                       /* (1 + m/8) * 2^(e-7) */
  return s ? -v : v;
}

double or_e2m1_value(uint8_t c) {
  int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
  double v = e == 0 ? 0.5 * m : ldexp(2.0 + m, e - 2);   /* (1 + m/2) * 2^(e-1) */
  return s ? -v : v;
}

/* nearest code of |x| among the finite non-negative codes 0..last of a
 * format whose values grow with the code; ties go to the even code (the even
 * mantissa bit) */
static uint8_t nearest_code(double a, double (*val)(uint8_t), int last) {
  if (a >= val((uint8_t)last)) return (uint8_t)last;      /* saturate */
  int lo = 0;
  while (lo < last && val((uint8_t)(lo + 1)) <= a) ++lo;  /* val(lo) <= a < val(lo + 1) */
  double below = val((uint8_t)lo), above = val((uint8_t)(lo + 1));
  if (a - below < above - a) return (uint8_t)lo;
  if (a - below > above - a) return (uint8_t)(lo + 1);
  return (uint8_t)((lo & 1) ? lo + 1 : lo);
}

uint8_t or_e4m3_from_f32(float x) {
  if (isnan(x)) return 0x7F;
  uint8_t c = nearest_code(fabs((double)x), or_e4m3_value, 0x7E);
  return (uint8_t)(signbit(x) ? (c | 0x80) : c);
}

uint8_t or_e2m1_from_f32(float x) {
  if (isnan(x)) return 0x7;                               /* no NaN in E2M1: saturate */
  uint8_t c = nearest_code(fabs((double)x), or_e2m1_value, 0x7);
  return (uint8_t)(signbit(x) ? (c | 0x8) : c);
}

/* One group in a float format (reading of TBQ's formats for the cache's
 * per-group params):
 *   FP8 (b = 8): scale = fp16 rounded UP of fp32(amax / 448), zero = 0,
 *                code = E4M3 of fp32(x / scale);
 *   FP4 (b = 4): scale = fp16 rounded UP of fp32(amax / 6), zero = 0,
 *                code = E2M1 of fp32(x / scale) (NVFP4's element format; the
 *                cache's group of G channels with an fp16 scale takes the
 *                place of NVFP4's 16-element E4M3 micro-scales);
 *   ternary (b = 2): scale = fp16 rounded UP of amax, zero = -scale,
 *                code = clamp(rint_even(fp32(x / scale)), -1, 1) + 1,
 *                so that zero + code * scale = scale * {-1, 0, +1}.
 * amax = the largest |x| of the group (fp32).  A zero scale gives the code of
 * 0 (E4M3/E2M1: 0; ternary: 1) for every element. */
void or_quantize_group_fmt(const uint16_t* x, int32_t G, int32_t bits, int32_t fmt,
                           uint8_t* codes, uint16_t* scale, uint16_t* zero) {
  if (fmt == 0) { or_quantize_group(x, G, bits, codes, scale, zero); return; }
  float amax = 0.0f;
  for (int j = 0; j < G; ++j) {
    float a = fabsf(or_f16_to_f32(x[j]));
    if (a > amax) amax = a;
  }
  float top = bits == 8 ? 448.0f : (bits == 4 ? 6.0f : 1.0f);
  uint16_t s = or_f16_round_up(amax / top);
  float sf = or_f16_to_f32(s);
  for (int j = 0; j < G; ++j) {
    float v = or_f16_to_f32(x[j]);
    if (bits == 2) {
      float c = sf == 0.0f ? 0.0f : rintf(v / sf);
      if (c < -1.0f) c = -1.0f;
      if (c > 1.0f) c = 1.0f;
      codes[j] = (uint8_t)((int)c + 1);
    } else {
      float t = sf == 0.0f ? 0.0f : v / sf;
      codes[j] = bits == 8 ? or_e4m3_from_f32(t) : or_e2m1_from_f32(t);
    }
  }
  *scale = s;
  *zero = bits == 2 ? (uint16_t)(s ^ 0x8000) : 0;         /* -scale: exact in fp16 */
}

/* ====================================================================== */
/* state                                                                   */
/* ====================================================================== */
struct or_state {
  or_layout L;
  int32_t cap;                 /* max_blocks * 16: slots one (seq, class) can own */
  void* codes[3];              /* uint8 (bits<=8) or uint16 raw fp16 (bits==16) */
  uint16_t* params[3];
  int32_t* slot_pos[3];
  uint64_t* table;
  int32_t* num_blocks;
  int32_t* free_slots;
  int32_t* free_top;
  int32_t* fifo;
  int32_t* fifo_head;
  int32_t* fifo_tail;
  int32_t* live_count;
  uint64_t* live_list;
  int32_t* live_index;
  int32_t* num_live;
  int32_t page_bump[3];
  /* TBE segments: per sequence, up to cap records of SEG_FIELDS ints */
  int32_t* seg;
  int32_t* nseg;
};

/* fields of one TBE segment record */
enum { SEG_CLS = 0, SEG_LEVEL = 1, SEG_LO = 2, SEG_LEN = 3, SEG_TRIM = 4, SEG_FIELDS = 5 };

#define ENTRY_PAGE(e) ((int32_t)((e) & 0xFFFFFFFFull))
#define ENTRY_CLASS(e) ((int32_t)(((e) >> 32) & 0xFF))
#define ENTRY_MASK(e) ((uint32_t)(((e) >> 48) & 0xFFFF))
/* live-list descriptor of a table entry: page | class << 32 | entry << 40 */
#define LIVE_ENTRY(x) ((int32_t)((x) >> 40))
static uint64_t live_desc(int32_t page, int c, int32_t e) {
  return (uint64_t)(uint32_t)page | ((uint64_t)c << 32) | ((uint64_t)e << 40);
}

static size_t code_elem_size(const or_layout* L, int c) { return L->bits[c] == 16 ? 2 : 1; }
static size_t codes_per_page(const or_layout* L) {
  return (size_t)L->num_kv_heads * 2 * OR_PAGE * L->head_dim;
}
static size_t params_per_page(const or_layout* L) {
  return (size_t)L->num_kv_heads * 2 * OR_PAGE * (L->head_dim / L->group_size) * 2;
}

static int layout_ok(const or_layout* L) {
  if (!L) return 0;
  if (L->page_size != OR_PAGE) return 0;
  if (L->num_kv_heads <= 0 || L->num_q_heads <= 0 || L->num_q_heads % L->num_kv_heads) return 0;
  if (L->head_dim <= 0 || L->group_size <= 0 || L->head_dim % L->group_size) return 0;
  for (int c = 0; c < 3; ++c) {
    int b = L->bits[c];
    if (b != 2 && b != 4 && b != 8 && b != 16) return 0;
    if (L->pool_pages[c] < 0) return 0;
    if (L->fmt[c] != 0 && !(L->fmt[c] == 1 && b != 16)) return 0;
  }
  if (L->max_seqs <= 0 || L->max_blocks_per_seq <= 0) return 0;
  return 1;
}

or_state* or_create(const or_layout* L) {
  if (!layout_ok(L)) return NULL;
  or_state* S = (or_state*)calloc(1, sizeof(or_state));
  if (!S) return NULL;
  S->L = *L;
  S->cap = L->max_blocks_per_seq * OR_PAGE;
  size_t ns = (size_t)L->max_seqs, nb = (size_t)L->max_blocks_per_seq;
  int fail = 0;
  for (int c = 0; c < 3; ++c) {
    size_t pages = (size_t)L->pool_pages[c];
    S->codes[c] = calloc(pages * codes_per_page(L) + 1, code_elem_size(L, c));
    S->params[c] = L->bits[c] == 16 ? NULL
                 : (uint16_t*)calloc(pages * params_per_page(L) + 1, sizeof(uint16_t));
    S->slot_pos[c] = (int32_t*)malloc((pages * OR_PAGE + 1) * sizeof(int32_t));
    if (!S->codes[c] || (L->bits[c] != 16 && !S->params[c]) || !S->slot_pos[c]) fail = 1;
    else for (size_t i = 0; i < pages * OR_PAGE; ++i) S->slot_pos[c][i] = -1;
  }
  S->table = (uint64_t*)calloc(ns * nb, sizeof(uint64_t));
  S->num_blocks = (int32_t*)calloc(ns, sizeof(int32_t));
  S->free_slots = (int32_t*)calloc(ns * 3 * (size_t)S->cap, sizeof(int32_t));
  S->free_top = (int32_t*)calloc(ns * 3, sizeof(int32_t));
  S->fifo = (int32_t*)calloc(ns * 3 * (size_t)S->cap, sizeof(int32_t));
  S->fifo_head = (int32_t*)calloc(ns * 3, sizeof(int32_t));
  S->fifo_tail = (int32_t*)calloc(ns * 3, sizeof(int32_t));
  S->live_count = (int32_t*)calloc(ns, sizeof(int32_t));
  S->live_list = (uint64_t*)calloc(ns * nb, sizeof(uint64_t));
  S->live_index = (int32_t*)malloc(ns * nb * sizeof(int32_t));
  S->num_live = (int32_t*)calloc(ns, sizeof(int32_t));
  S->seg = (int32_t*)calloc(ns * (size_t)S->cap * SEG_FIELDS + 1, sizeof(int32_t));
  S->nseg = (int32_t*)calloc(ns, sizeof(int32_t));
  if (!S->seg || !S->nseg) fail = 1;
  if (!S->table || !S->num_blocks || !S->free_slots || !S->free_top || !S->fifo ||
      !S->fifo_head || !S->fifo_tail || !S->live_count || !S->live_list ||
      !S->live_index || !S->num_live)
    fail = 1;
  if (fail) { or_destroy(S); return NULL; }
  for (size_t i = 0; i < ns * nb; ++i) S->live_index[i] = -1;
  return S;
}

void or_destroy(or_state* S) {
  if (!S) return;
  for (int c = 0; c < 3; ++c) { free(S->codes[c]); free(S->params[c]); free(S->slot_pos[c]); }
  free(S->table); free(S->num_blocks); free(S->free_slots); free(S->free_top);
  free(S->fifo); free(S->fifo_head); free(S->fifo_tail); free(S->live_count);
  free(S->live_list); free(S->live_index); free(S->num_live);
  free(S->seg); free(S->nseg);
  free(S);
}

const or_layout* or_get_layout(const or_state* S) { return &S->L; }

/* index helpers */
static int32_t* free_stack(or_state* S, int s, int c) {
  return S->free_slots + ((size_t)s * 3 + c) * S->cap;
}
static int32_t* fifo_ring(or_state* S, int s, int c) {
  return S->fifo + ((size_t)s * 3 + c) * S->cap;
}
static uint64_t* table_row(const or_state* S, int s) {
  return S->table + (size_t)s * S->L.max_blocks_per_seq;
}

/* ====================================================================== */
/* append: quantise on append into a free slot of the token's class [CT]   */
/* ====================================================================== */
static void write_token(or_state* S, int c, int32_t page, int slot,
                        const uint16_t* k, const uint16_t* v) {
  const or_layout* L = &S->L;
  int H = L->num_kv_heads, d = L->head_dim, G = L->group_size, ng = d / G, b = L->bits[c];
  for (int h = 0; h < H; ++h) {
    for (int kv = 0; kv < 2; ++kv) {
      const uint16_t* x = (kv == 0 ? k : v) + (size_t)h * d;
      size_t row = ((((size_t)page * H + h) * 2 + kv) * OR_PAGE + slot);
      if (b == 16) {                                     /* 16-bit pass-through */
        uint16_t* dst = (uint16_t*)S->codes[c] + row * d;
        memcpy(dst, x, (size_t)d * 2);
        continue;
      }
      uint8_t* dst = (uint8_t*)S->codes[c] + row * d;
      uint16_t* prm = S->params[c] + row * ng * 2;
      for (int g = 0; g < ng; ++g)
        or_quantize_group_fmt(x + g * G, G, b, L->fmt[c], dst + g * G, &prm[2 * g], &prm[2 * g + 1]);
    }
  }
}

int or_append(or_state* S, int32_t n, const int32_t* seq, const int32_t* pos,
              const uint8_t* tag, const uint16_t* k, const uint16_t* v) {
  const or_layout* L = &S->L;
  if (n < 0) return OR_ERR_INVALID;
  if (n == 0) return OR_OK;
  int ns = L->max_seqs;
  /* -- validation (all-or-nothing) ---------------------------------- */
  /* Tokens come grouped by sequence (one contiguous run per sequence),
   * positions strictly ascending inside a run. */
  char* seen = (char*)calloc((size_t)ns, 1);
  int64_t* cnt = (int64_t*)calloc((size_t)ns * 3, sizeof(int64_t));
  int bad = 0;
  for (int32_t i = 0; i < n && !bad; ++i) {
    int s = seq[i];
    if (s < 0 || s >= ns || tag[i] > 2 || pos[i] < 0) { bad = 1; break; }
    int new_run = (i == 0 || seq[i - 1] != s);
    if (new_run) {
      if (seen[s]) bad = 1;
      seen[s] = 1;
    } else if (pos[i] <= pos[i - 1]) bad = 1;
    cnt[(size_t)s * 3 + tag[i]]++;
  }
  if (bad) { free(seen); free(cnt); return OR_ERR_INVALID; }
  int64_t grants_c[3] = {0, 0, 0};
  int status = OR_OK;
  for (int s = 0; s < ns && status == OR_OK; ++s) {
    int64_t gs = 0;
    for (int c = 0; c < 3; ++c) {
      int64_t need = cnt[(size_t)s * 3 + c] - S->free_top[s * 3 + c];
      int64_t g = need > 0 ? (need + OR_PAGE - 1) / OR_PAGE : 0;
      grants_c[c] += g;
      gs += g;
    }
    if (gs > (int64_t)L->max_blocks_per_seq - S->num_blocks[s]) status = OR_ERR_OUT_OF_BLOCKS;
  }
  for (int c = 0; c < 3; ++c)
    if (grants_c[c] > (int64_t)L->pool_pages[c] - S->page_bump[c]) status = OR_ERR_OUT_OF_PAGES;
  free(seen);
  free(cnt);
  if (status != OR_OK) return status;

  /* -- tokens in call order ------------------------------------------ */
  size_t tok = (size_t)L->num_kv_heads * L->head_dim;
  for (int32_t i = 0; i < n; ++i) {
    int s = seq[i], c = tag[i];
    int32_t* top = &S->free_top[s * 3 + c];
    int32_t* stack = free_stack(S, s, c);
    int32_t ts;                                  /* table slot: entry*16 + slot */
    if (*top > 0) {
      ts = stack[--(*top)];                      /* reuse the most recently freed slot */
    } else {
      /* reading: a class with no free slot opens a new page of that class;
       * its slots 15..1 go onto the free stack (slot 1 on top), slot 0 is used */
      int32_t page = S->page_bump[c]++;
      int32_t e = S->num_blocks[s]++;
      table_row(S, s)[e] = (uint64_t)(uint32_t)page | ((uint64_t)c << 32);
      for (int sl = 0; sl < OR_PAGE; ++sl) S->slot_pos[c][(size_t)page * OR_PAGE + sl] = -1;
      for (int sl = OR_PAGE - 1; sl >= 1; --sl) stack[(*top)++] = e * OR_PAGE + sl;
      ts = e * OR_PAGE;
    }
    int32_t e = ts / OR_PAGE, slot = ts % OR_PAGE;
    uint64_t* ent = &table_row(S, s)[e];
    int32_t page = ENTRY_PAGE(*ent);
    write_token(S, c, page, slot, k + i * tok, v + i * tok);
    uint32_t before = ENTRY_MASK(*ent);
    *ent |= (uint64_t)1 << (48 + slot);          /* eviction mask bit: live */
    if (before == 0) {                           /* the page became non-empty */
      int32_t at = S->num_live[s]++;
      S->live_list[(size_t)s * L->max_blocks_per_seq + at] = live_desc(page, c, e);
      S->live_index[(size_t)s * L->max_blocks_per_seq + e] = at;
    }
    S->slot_pos[c][(size_t)page * OR_PAGE + slot] = pos[i];  /* start index */
    int32_t* tail = &S->fifo_tail[s * 3 + c];
    fifo_ring(S, s, c)[(*tail) % S->cap] = ts;
    (*tail)++;
    S->live_count[s]++;
  }
  return OR_OK;
}

/* ====================================================================== */
/* evict to budget [TBE][CT]                                               */
/* ====================================================================== */
/* One victim: table slot ts (entry*16 + slot) of class c in sequence s.  Its
 * mask bit is cleared (an entry left with no live token leaves the live-page
 * list by swap-with-last), its start index set to -1, its slot pushed onto
 * its class's free stack, and the live count drops.  Nothing is moved. */
static void evict_token(or_state* S, int s, int c, int32_t ts) {
  const or_layout* L = &S->L;
  int32_t e = ts / OR_PAGE, slot = ts % OR_PAGE;
  uint64_t* ent = &table_row(S, s)[e];
  *ent &= ~((uint64_t)1 << (48 + slot));
  if (ENTRY_MASK(*ent) == 0) {                 /* page emptied: swap-remove */
    uint64_t* list = S->live_list + (size_t)s * L->max_blocks_per_seq;
    int32_t* index = S->live_index + (size_t)s * L->max_blocks_per_seq;
    int32_t at = index[e], last = --S->num_live[s];
    uint64_t moved = list[last];
    list[at] = moved;
    index[LIVE_ENTRY(moved)] = at;
    index[e] = -1;
  }
  S->slot_pos[c][(size_t)ENTRY_PAGE(*ent) * OR_PAGE + slot] = -1;
  int32_t* top = &S->free_top[s * 3 + c];
  free_stack(S, s, c)[(*top)++] = ts;
  S->live_count[s]--;
}

/* Reading: n = max(0, live - budget) victims, taken oldest first from the
 * class FIFOs in the given class order (default T, then E, then R).  Each
 * victim's mask bit is cleared, its start index set to -1 and its slot pushed
 * onto its class's free stack, in victim order.  Pages are never released.
 * A FIFO entry of -1 is a tombstone (a token TBE already evicted): taking a
 * victim from a class first steps its head over the tombstones there. */
int or_evict(or_state* S, int32_t n, const int32_t* seq, const int32_t* budget,
             const uint8_t* order) {
  const or_layout* L = &S->L;
  static const uint8_t default_order[3] = {OR_T, OR_E, OR_R};
  if (!order) order = default_order;
  if (n < 0) return OR_ERR_INVALID;
  if (order[0] > 2 || order[1] > 2 || order[2] > 2 || order[0] == order[1] ||
      order[0] == order[2] || order[1] == order[2])
    return OR_ERR_INVALID;
  char* seen = (char*)calloc((size_t)L->max_seqs, 1);
  for (int32_t i = 0; i < n; ++i) {
    int s = seq[i];
    if (s < 0 || s >= L->max_seqs || budget[i] < 0 || seen[s]) { free(seen); return OR_ERR_INVALID; }
    seen[s] = 1;
  }
  free(seen);
  for (int32_t i = 0; i < n; ++i) {
    int s = seq[i];
    int32_t nv = S->live_count[s] - budget[i];
    for (int32_t k = 0; k < nv; ++k) {
      int c = -1;
      for (int o = 0; o < 3; ++o) {
        int cc = order[o];
        int32_t* head = &S->fifo_head[s * 3 + cc];
        while (*head < S->fifo_tail[s * 3 + cc] && fifo_ring(S, s, cc)[(*head) % S->cap] < 0)
          (*head)++;                             /* tombstone */
        if (*head < S->fifo_tail[s * 3 + cc]) { c = cc; break; }
      }
      if (c < 0) break;                          /* unreachable: live > budget >= 0 */
      int32_t* head = &S->fifo_head[s * 3 + c];
      int32_t ts = fifo_ring(S, s, c)[(*head) % S->cap];
      (*head)++;
      evict_token(S, s, c, ts);
    }
  }
  return OR_OK;
}

/* ====================================================================== */
/* explicit victims                                                        */
/* ====================================================================== */
/* The eviction step a policy drives directly (the explicit-victim call TBE
 * needs when the policy runs on the host).  Victim i is the token at FIFO
 * counter idx[i] of the class cls[i] FIFO of sequence seq[i]
 * (head <= idx < tail).  Victims go in call order, each like a TBE victim:
 * mask bit cleared, start index -1, slot pushed onto its class's free stack,
 * FIFO entry made a tombstone (-1).  A victim whose entry is already a
 * tombstone (evicted before, or named earlier in the call) is skipped.  The
 * call is all-or-nothing on its arguments: a sequence out of range, a class
 * above 2, a counter outside its FIFO window, or a sequence whose victims are
 * not contiguous in the call make it invalid, and nothing changes. */
int or_evict_slots(or_state* S, int32_t n, const int32_t* seq, const uint8_t* cls,
                   const int32_t* idx) {
  const or_layout* L = &S->L;
  if (n < 0) return OR_ERR_INVALID;
  char* seen = (char*)calloc((size_t)L->max_seqs, 1);
  for (int32_t i = 0; i < n; ++i) {
    int s = seq[i];
    if (s < 0 || s >= L->max_seqs || cls[i] > 2) { free(seen); return OR_ERR_INVALID; }
    int c = cls[i];
    if (idx[i] < S->fifo_head[s * 3 + c] || idx[i] >= S->fifo_tail[s * 3 + c]) {
      free(seen);
      return OR_ERR_INVALID;
    }
    if (i == 0 || seq[i - 1] != s) {             /* a new run of victims */
      if (seen[s]) { free(seen); return OR_ERR_INVALID; }
      seen[s] = 1;
    }
  }
  free(seen);
  for (int32_t i = 0; i < n; ++i) {
    int s = seq[i], c = cls[i];
    int32_t* entry = &fifo_ring(S, s, c)[idx[i] % S->cap];
    if (*entry < 0) continue;                    /* already a tombstone */
    evict_token(S, s, c, *entry);
    *entry = -1;
  }
  return OR_OK;
}

/* ====================================================================== */
/* TBE: segment-level eviction on Transition thoughts                      */
/* ====================================================================== */
/* Explainer, Methodologie, "Eviction Adaptative a la Pensee (TBE)": when a
 * Transition thought appears, tokens of the earlier, less critical Reasoning
 * and Execution segments are evicted progressively along an annealing
 * schedule (retention 64, then 32, then 16), a segment at a time rather than
 * token by token; and (the explainer's "Astuce B") a small safety net of
 * Transition tokens is always kept.  Readings:
 *   - a segment is a maximal run of consecutive tokens of one sequence with
 *     the same tag, in append order; a T event is the first token of a new T
 *     segment;
 *   - at a T event each earlier R or E segment takes the next step of the
 *     schedule (its k-th event keeps at most schedule[min(k,3)-1] tokens) and
 *     each earlier T segment keeps only its share of the t_min most recent
 *     live tokens of all earlier T segments;
 *   - a segment gives up its oldest live tokens first (the segment's live
 *     tokens are always a suffix of it); victims go in segment order, then
 *     token order;
 *   - an evicted token's FIFO entry becomes a tombstone (-1), since it need
 *     not be at the FIFO head.
 * A segment record holds its class, schedule level, the FIFO counter of its
 * first token (lo), its length, and trim: how far from lo TBE has passed.
 * Its live tokens are the FIFO entries [max(lo + trim, head), lo + len). */
static int32_t* seg_rec(or_state* S, int s, int32_t j) {
  return S->seg + (((size_t)s * S->cap) + (size_t)j) * SEG_FIELDS;
}

static int32_t seg_first_live(const or_state* S, int s, const int32_t* g) {
  int32_t a = g[SEG_LO] + g[SEG_TRIM], head = S->fifo_head[s * 3 + g[SEG_CLS]];
  return a > head ? a : head;
}

static int32_t seg_live(const or_state* S, int s, const int32_t* g) {
  int32_t live = g[SEG_LO] + g[SEG_LEN] - seg_first_live(S, s, g);
  return live > 0 ? live : 0;
}

/* the x oldest live tokens of segment g, tombstoned in the FIFO */
static void trim_segment(or_state* S, int s, int32_t* g, int32_t x) {
  int c = g[SEG_CLS];
  int32_t first = seg_first_live(S, s, g);
  for (int32_t k = 0; k < x; ++k) {
    int32_t* entry = &fifo_ring(S, s, c)[(first + k) % S->cap];
    evict_token(S, s, c, *entry);
    *entry = -1;
  }
  g[SEG_TRIM] = first + x - g[SEG_LO];
}

/* the T event that opens segment e of sequence s */
static void tbe_event(or_state* S, int s, int32_t e, int32_t t_min, const int32_t* schedule) {
  int32_t* keep_t = (int32_t*)calloc((size_t)e + 1, sizeof(int32_t));
  int32_t net = t_min;                           /* safety net, newest T tokens first */
  for (int32_t j = e - 1; j >= 0; --j) {
    int32_t* g = seg_rec(S, s, j);
    if (g[SEG_CLS] != OR_T) continue;
    int32_t live = seg_live(S, s, g), k = live < net ? live : net;
    keep_t[j] = k;
    net -= k;
  }
  for (int32_t j = 0; j < e; ++j) {
    int32_t* g = seg_rec(S, s, j);
    int32_t live = seg_live(S, s, g), x;
    if (g[SEG_CLS] == OR_T) {
      x = live - keep_t[j];
    } else {
      if (g[SEG_LEVEL] < 3) g[SEG_LEVEL]++;
      x = live - schedule[g[SEG_LEVEL] - 1];
    }
    if (x > 0) trim_segment(S, s, g, x);
  }
  free(keep_t);
}

int or_tbe(or_state* S, int32_t n, const int32_t* seq, const int32_t* pos, const uint8_t* tag,
           int32_t t_min, const int32_t* schedule) {
  const or_layout* L = &S->L;
  static const int32_t default_schedule[3] = {64, 32, 16};
  if (!schedule) schedule = default_schedule;
  if (n < 0 || t_min < 0 || schedule[0] < 0 || schedule[1] < 0 || schedule[2] < 0)
    return OR_ERR_INVALID;
  if (n == 0) return OR_OK;
  int ns = L->max_seqs;
  /* the same token runs as the append that has just stored them */
  char* seen = (char*)calloc((size_t)ns, 1);
  int64_t* cnt = (int64_t*)calloc((size_t)ns * 3, sizeof(int64_t));
  int32_t* newseg = (int32_t*)calloc((size_t)ns, sizeof(int32_t));
  int bad = 0;
  for (int32_t i = 0; i < n && !bad; ++i) {
    int s = seq[i];
    if (s < 0 || s >= ns || tag[i] > 2 || pos[i] < 0) { bad = 1; break; }
    int new_run = (i == 0 || seq[i - 1] != s);
    if (new_run) {
      if (seen[s]) bad = 1;
      seen[s] = 1;
    } else if (pos[i] <= pos[i - 1]) bad = 1;
    cnt[(size_t)s * 3 + tag[i]]++;
    int32_t last_cls = new_run ? (S->nseg[s] > 0 ? seg_rec(S, s, S->nseg[s] - 1)[SEG_CLS] : -1)
                               : tag[i - 1];
    if (tag[i] != last_cls) newseg[s]++;
  }
  for (int s = 0; s < ns && !bad; ++s) {
    if ((int64_t)S->nseg[s] + newseg[s] > S->cap) bad = 1;
    /* the tokens must be the newest of their class FIFOs: the append that
     * precedes this call put them there */
    for (int c = 0; c < 3; ++c)
      if (cnt[(size_t)s * 3 + c] > S->fifo_tail[s * 3 + c] - S->fifo_head[s * 3 + c]) bad = 1;
  }
  free(seen);
  free(newseg);
  if (bad) { free(cnt); return OR_ERR_INVALID; }
  /* the append pushed sequence s's class-c tokens of the call, in call order,
   * onto FIFO counters tail - cnt .. tail - 1 */
  int32_t* next = (int32_t*)calloc((size_t)ns * 3, sizeof(int32_t));
  for (int s = 0; s < ns; ++s)
    for (int c = 0; c < 3; ++c)
      next[s * 3 + c] = S->fifo_tail[s * 3 + c] - (int32_t)cnt[(size_t)s * 3 + c];
  for (int32_t i = 0; i < n; ++i) {
    int s = seq[i], c = tag[i];
    int32_t idx = next[s * 3 + c]++;
    int32_t ns_s = S->nseg[s];
    if (ns_s > 0 && seg_rec(S, s, ns_s - 1)[SEG_CLS] == c) {
      seg_rec(S, s, ns_s - 1)[SEG_LEN]++;
      continue;
    }
    int32_t* g = seg_rec(S, s, ns_s);
    g[SEG_CLS] = c;
    g[SEG_LEVEL] = 0;
    g[SEG_LO] = idx;
    g[SEG_LEN] = 1;
    g[SEG_TRIM] = 0;
    S->nseg[s] = ns_s + 1;
    if (c == OR_T) tbe_event(S, s, ns_s, t_min, schedule);
  }
  free(next);
  free(cnt);
  return OR_OK;
}

/* ====================================================================== */
/* gather compaction: the step CT avoids                                   */
/* ====================================================================== */
/* Explainer, Methodologie, "Implementation Systeme: Pensee Continue (CT)":
 * without CT, evicting scattered tokens leaves holes that a gather-based
 * compaction closes by moving the survivors together (at a cost in time and
 * HBM bandwidth); CT instead refills the holes in place.  Reading of the
 * compaction the pages compare against: each listed sequence's live tokens
 * are gathered into fresh, hole-free pages of an empty cache dst of the same
 * geometry -- class by class (R, E, T), in FIFO (arrival) order within a
 * class, 16 to a page -- as if they were appended there in that order with
 * their codes copied, not requantised.  The last page of a class keeps its
 * unused slots on the free stack, as an append leaves them.  Tombstones and
 * free slots are not carried over.  A token keeps its sequence id and
 * position; dst's pages are granted in call order. */
static void copy_token(const or_state* src, int c, int32_t sp, int ss, or_state* dst,
                       int32_t dp, int ds) {
  const or_layout* L = &src->L;
  size_t rows = (size_t)L->num_kv_heads * 2, d = (size_t)L->head_dim;
  size_t ng = (size_t)(L->head_dim / L->group_size);
  for (size_t hk = 0; hk < rows; ++hk) {           /* (head, K|V) rows */
    size_t a = (((size_t)sp * rows + hk) * OR_PAGE + ss), b = (((size_t)dp * rows + hk) * OR_PAGE + ds);
    if (L->bits[c] == 16) {
      memcpy((uint16_t*)dst->codes[c] + b * d, (const uint16_t*)src->codes[c] + a * d, d * 2);
    } else {
      memcpy((uint8_t*)dst->codes[c] + b * d, (const uint8_t*)src->codes[c] + a * d, d);
      memcpy(dst->params[c] + b * ng * 2, src->params[c] + a * ng * 2, ng * 4);
    }
  }
}

int or_compact(const or_state* src, or_state* dst, int32_t n, const int32_t* seq) {
  const or_layout* A = &src->L;
  const or_layout* B = &dst->L;
  if (n < 0) return OR_ERR_INVALID;
  if (A->num_q_heads != B->num_q_heads || A->num_kv_heads != B->num_kv_heads ||
      A->head_dim != B->head_dim || A->group_size != B->group_size ||
      A->bits[0] != B->bits[0] || A->bits[1] != B->bits[1] || A->bits[2] != B->bits[2] ||
      A->fmt[0] != B->fmt[0] || A->fmt[1] != B->fmt[1] || A->fmt[2] != B->fmt[2] ||
      A->max_seqs != B->max_seqs || A->max_blocks_per_seq != B->max_blocks_per_seq)
    return OR_ERR_INVALID;
  char* seen = (char*)calloc((size_t)A->max_seqs, 1);
  int64_t need[3] = {0, 0, 0};
  int bad = 0;
  for (int32_t i = 0; i < n && !bad; ++i) {
    int s = seq[i];
    if (s < 0 || s >= A->max_seqs || seen[s]) { bad = 1; break; }
    seen[s] = 1;
    if (dst->num_blocks[s] != 0) bad = 1;        /* dst must be empty for s */
    for (int c = 0; c < 3; ++c) {
      int64_t live = 0;
      for (int32_t k = src->fifo_head[s * 3 + c]; k < src->fifo_tail[s * 3 + c]; ++k)
        if (src->fifo[((size_t)s * 3 + c) * src->cap + (size_t)(k % src->cap)] >= 0) ++live;
      need[c] += (live + OR_PAGE - 1) / OR_PAGE;
    }
  }
  free(seen);
  for (int c = 0; c < 3 && !bad; ++c)
    if (need[c] > (int64_t)B->pool_pages[c] - dst->page_bump[c]) return OR_ERR_OUT_OF_PAGES;
  if (bad) return OR_ERR_INVALID;
  for (int32_t i = 0; i < n; ++i) {
    int s = seq[i];
    for (int c = 0; c < 3; ++c) {
      int32_t used = OR_PAGE, e = -1, page = -1;
      for (int32_t k = src->fifo_head[s * 3 + c]; k < src->fifo_tail[s * 3 + c]; ++k) {
        int32_t ts = src->fifo[((size_t)s * 3 + c) * src->cap + (size_t)(k % src->cap)];
        if (ts < 0) continue;                    /* tombstone */
        int32_t se = ts / OR_PAGE, ss = ts % OR_PAGE;
        int32_t sp = ENTRY_PAGE(table_row(src, s)[se]);
        if (used == OR_PAGE) {                   /* a fresh page of class c */
          page = dst->page_bump[c]++;
          e = dst->num_blocks[s]++;
          table_row(dst, s)[e] = (uint64_t)(uint32_t)page | ((uint64_t)c << 32);
          for (int sl = 0; sl < OR_PAGE; ++sl) dst->slot_pos[c][(size_t)page * OR_PAGE + sl] = -1;
          int32_t at = dst->num_live[s]++;
          dst->live_list[(size_t)s * B->max_blocks_per_seq + at] = live_desc(page, c, e);
          dst->live_index[(size_t)s * B->max_blocks_per_seq + e] = at;
          used = 0;
        }
        int32_t slot = used++;
        copy_token(src, c, sp, ss, dst, page, slot);
        table_row(dst, s)[e] |= (uint64_t)1 << (48 + slot);
        dst->slot_pos[c][(size_t)page * OR_PAGE + slot] =
            src->slot_pos[c][(size_t)sp * OR_PAGE + ss];
        int32_t* tail = &dst->fifo_tail[s * 3 + c];
        fifo_ring(dst, s, c)[(*tail) % dst->cap] = e * OR_PAGE + slot;
        (*tail)++;
        dst->live_count[s]++;
      }
      /* the unused slots of the last page go on the free stack, the lowest on top */
      if (page >= 0)
        for (int sl = OR_PAGE - 1; sl >= used; --sl)
          free_stack(dst, s, c)[dst->free_top[s * 3 + c]++] = e * OR_PAGE + sl;
    }
  }
  return OR_OK;
}

/* ====================================================================== */
/* decode attention over the mixed-precision pages                         */
/* ====================================================================== */
typedef struct { int32_t pos, cls, page, slot; } live_tok;

static int cmp_pos(const void* a, const void* b) {
  int32_t pa = ((const live_tok*)a)->pos, pb = ((const live_tok*)b)->pos;
  return (pa > pb) - (pa < pb);
}
static int cmp_desc(const void* a, const void* b) {
  double x = *(const double*)a, y = *(const double*)b;
  return (x < y) - (x > y);
}

/* dequantised value of channel j of (page, head, K|V, slot): zero + code*scale */
static double deq(const or_state* S, int c, int32_t page, int h, int kv, int slot, int j) {
  const or_layout* L = &S->L;
  size_t row = ((((size_t)page * L->num_kv_heads + h) * 2 + kv) * OR_PAGE + slot);
  if (L->bits[c] == 16)
    return (double)or_f16_to_f32(((const uint16_t*)S->codes[c])[row * L->head_dim + j]);
  int ng = L->head_dim / L->group_size, g = j / L->group_size;
  const uint16_t* prm = S->params[c] + row * ng * 2 + 2 * g;
  double scale = or_f16_to_f32(prm[0]), zero = or_f16_to_f32(prm[1]);
  uint8_t code = ((const uint8_t*)S->codes[c])[row * L->head_dim + j];
  if (L->fmt[c] == 1 && L->bits[c] == 8) return scale * or_e4m3_value(code);
  if (L->fmt[c] == 1 && L->bits[c] == 4) return scale * or_e2m1_value(code);
  return zero + (double)code * scale;                    /* integer codes; ternary */
}

static void decode_one(const or_state* S, int s, const uint16_t* q, double scale,
                       int32_t topk, double* out, double* mass) {
  const or_layout* L = &S->L;
  int H = L->num_kv_heads, Hq = L->num_q_heads, d = L->head_dim, gq = Hq / H;
  /* the live set of the sequence: every slot whose mask bit is set */
  int32_t nb = S->num_blocks[s];
  live_tok* t = (live_tok*)malloc(((size_t)nb * OR_PAGE + 1) * sizeof(live_tok));
  int32_t n = 0;
  for (int32_t e = 0; e < nb; ++e) {
    uint64_t ent = table_row(S, s)[e];
    for (int sl = 0; sl < OR_PAGE; ++sl) {
      if (!((ENTRY_MASK(ent) >> sl) & 1)) continue;
      live_tok x;
      x.cls = ENTRY_CLASS(ent);
      x.page = ENTRY_PAGE(ent);
      x.slot = sl;
      x.pos = S->slot_pos[x.cls][(size_t)x.page * OR_PAGE + sl];
      t[n++] = x;
    }
  }
  /* sort by position so the fp64 sums do not depend on slot placement */
  qsort(t, (size_t)n, sizeof(live_tok), cmp_pos);
  double* kh = (double*)malloc(((size_t)n * d + 1) * sizeof(double));
  double* vh = (double*)malloc(((size_t)n * d + 1) * sizeof(double));
  double* lg = (double*)malloc(((size_t)n + 1) * sizeof(double));
  for (int h = 0; h < H; ++h) {
    for (int32_t i = 0; i < n; ++i)
      for (int j = 0; j < d; ++j) {
        kh[(size_t)i * d + j] = deq(S, t[i].cls, t[i].page, h, 0, t[i].slot, j);
        vh[(size_t)i * d + j] = deq(S, t[i].cls, t[i].page, h, 1, t[i].slot, j);
      }
    for (int r = 0; r < gq; ++r) {
      int hq = h * gq + r;                       /* q-heads map contiguously to kv-heads */
      const uint16_t* qv = q + (size_t)hq * d;
      double* o = out + (size_t)hq * d;
      for (int j = 0; j < d; ++j) o[j] = 0.0;
      if (n == 0) { if (mass) mass[hq] = 0.0; continue; }
      double m = -INFINITY;
      for (int32_t i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += (double)or_f16_to_f32(qv[j]) * kh[(size_t)i * d + j];
        lg[i] = scale * acc;
        if (lg[i] > m) m = lg[i];
      }
      double sum = 0.0;
      for (int32_t i = 0; i < n; ++i) { lg[i] = exp(lg[i] - m); sum += lg[i]; }
      for (int32_t i = 0; i < n; ++i) {
        double p = lg[i] / sum;
        lg[i] = p;
        for (int j = 0; j < d; ++j) o[j] += p * vh[(size_t)i * d + j];
      }
      if (mass) {
        /* share of probability mass held by the top-k live slots */
        qsort(lg, (size_t)n, sizeof(double), cmp_desc);
        double acc = 0.0;
        int32_t kk = topk < n ? topk : n;
        for (int32_t i = 0; i < kk; ++i) acc += lg[i];
        mass[hq] = kk == n ? 1.0 : acc;
      }
    }
  }
  free(t); free(kh); free(vh); free(lg);
}

int or_decode(const or_state* S, int32_t n, const int32_t* seq, const uint16_t* q,
              double softmax_scale, int32_t topk, double* out, double* mass, int32_t threads) {
  const or_layout* L = &S->L;
  if (n < 0) return OR_ERR_INVALID;
  if (mass && (topk < 1)) return OR_ERR_INVALID;
  for (int32_t i = 0; i < n; ++i)
    if (seq[i] < 0 || seq[i] >= L->max_seqs) return OR_ERR_INVALID;
  double scale = softmax_scale > 0 ? softmax_scale : 1.0 / sqrt((double)L->head_dim);
  size_t qstride = (size_t)L->num_q_heads * L->head_dim;
  (void)threads;
#ifdef _OPENMP
  int nt = threads > 0 ? threads : 1;
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
#endif
  for (int32_t i = 0; i < n; ++i)
    decode_one(S, seq[i], q + i * qstride, scale, topk, out + i * qstride,
               mass ? mass + (size_t)i * L->num_q_heads : NULL);
  return OR_OK;
}

/* ====================================================================== */
/* thought decomposition from attention sparsity (mechanism only)          */
/* ====================================================================== */
/* Explainer, Methodologie, "Decomposition de la Pensee via la Parcimonie de
 * l'Attention": thoughts are told apart by how sparse their attention is --
 * Transition the sparsest, then Reasoning, Execution the least sparse.
 * Reading: the sparsity of one decode step of sequence i is the mean over
 * query heads of the top-k attention mass (a head whose probability sits on a
 * few tokens has a mass near 1).  The mean is an fp32 sum in head order
 * divided by the head count (both rounded to nearest), so that the tag -- an
 * integer decided by floating point -- is reproducible exactly.  The two
 * thresholds are the calibration the pages leave to a real model. */
void or_classify(int32_t n, int32_t hq, const float* mass, float theta_t, float theta_r,
                 uint8_t* tags) {
  for (int32_t i = 0; i < n; ++i) {
    float sum = 0.0f;
    for (int32_t h = 0; h < hq; ++h) sum = sum + mass[(size_t)i * hq + h];
    float score = sum / (float)hq;
    tags[i] = score >= theta_t ? OR_T : (score >= theta_r ? OR_R : OR_E);
  }
}

/* ====================================================================== */
/* state export                                                            */
/* ====================================================================== */
const void* or_codes(const or_state* S, int c) { return S->codes[c]; }
const uint16_t* or_params(const or_state* S, int c) { return S->params[c]; }
const int32_t* or_slot_pos(const or_state* S, int c) { return S->slot_pos[c]; }
const uint64_t* or_table(const or_state* S) { return S->table; }
const int32_t* or_num_blocks(const or_state* S) { return S->num_blocks; }
const int32_t* or_free_slots(const or_state* S) { return S->free_slots; }
const int32_t* or_free_top(const or_state* S) { return S->free_top; }
const int32_t* or_fifo(const or_state* S) { return S->fifo; }
const int32_t* or_fifo_head(const or_state* S) { return S->fifo_head; }
const int32_t* or_fifo_tail(const or_state* S) { return S->fifo_tail; }
const int32_t* or_live_count(const or_state* S) { return S->live_count; }
const uint64_t* or_live_list(const or_state* S) { return S->live_list; }
const int32_t* or_live_index(const or_state* S) { return S->live_index; }
const int32_t* or_num_live(const or_state* S) { return S->num_live; }
const int32_t* or_page_bump(const or_state* S) { return S->page_bump; }
const int32_t* or_seg(const or_state* S) { return S->seg; }
const int32_t* or_nseg(const or_state* S) { return S->nseg; }
