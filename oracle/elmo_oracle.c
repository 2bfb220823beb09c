/*
 * elmo_oracle.c -- plain, slow CPU oracle for the ELMO classifier-head step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares
 * no code, header, table or constant with the CUDA path.
 *
 * Source: "ELMO: Efficiency via Low-precision and Peak Memory Optimization in
 * Large Output Spaces" (Zhang, Ullah, Schultheis, Babbar; arXiv 2510.11168),
 * as summarised on its pages: Approach (pure BF16/FP8 classifier without FP32
 * master weights or tensor scaling, stochastic rounding, momentum-free SGD,
 * classifier gradient fused with the SGD update, label chunking) and
 * "Surprising findings" (E4M3 native range suffices, momentum dropped).
 * The update rule W_c <- SR(W_c - lr * G_c^T X) with G = sigmoid(Z) - Y and
 * the input gradient dX = G W (old W) are the step those passages describe.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   - summed BCE, no 1/B, no bias, no weight decay; lr is a per-call scalar;
 *   - dX uses the OLD weights;
 *   - fp8 mode: X is quantised to E4M3 with a per-step power-of-two scale
 *     s_X = 2^floor(log2(448/max|X|)); G is quantised as E4M3(2^8 * g); both
 *     scales are undone exactly in fp32;  bf16 mode: X as is, G -> RNE bf16;
 *   - E4M3 is OCP E4M3FN (max 448, no infinities), saturating;
 *   - SR uses a 16-bit uniform draw k taken from Philox4x32-10
 *     (Salmon et al., SC'11, "Parallel Random Numbers: As Easy as 1, 2, 3")
 *     keyed by the seed, with counter (idx >> 3, step): 8 elements share one
 *     Philox block, element idx uses 16-bit half (idx & 1) of word
 *     ((idx >> 1) & 3), low half first;
 *   - SR(v): v on the grid stays; otherwise with grid neighbours lo < v < hi
 *     and f = (v - lo) / (hi - lo), return hi iff k < floor(2^16 f): the draw
 *     is added to the first 16 bits of the discarded fraction and the sum
 *     truncated; equivalently hi iff u <= f for u = (k + 1) / 2^16 on the
 *     16-bit grid of (0, 1] (exactly unbiased on bf16, whose fraction has 16
 *     bits; on the 8-bit grids P(hi) = floor(2^16 f) / 2^16), on magnitudes
 *     (sign restored);
 *     NaN -> canonical NaN (bf16 0x7FC0, E4M3 0x7F); E4M3: |v| >= 448 and
 *     +-inf -> +-448; bf16: finite |v| above the largest finite -> largest
 *     finite, +-inf stays +-inf;
 *   - top-k scores are the fp32 fma chain over j = 0..d-1 in order, ranked by
 *     score descending, ties to the lower label index, NaN last;
 *   - the adjacent FP8 choices: an E5M2 gradient operand (E5M2 of 2^8 g, W and
 *     X E4M3), and an E5M2 head (W stored and rounded on the E5M2 grid, which
 *     has infinities: +-inf stays, finite values above 57344 saturate; X and
 *     G E4M3);
 *   - the encoder side: Kahan-compensated SGD of bf16 parameters with a bf16
 *     compensation, one IEEE fp32 operation per step, RNE at the stores.
 *
 * Everything here is written for a reader checking it against those
 * definitions: no blocking, no fusion, no reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_EDATA 6

#define DT_BF16 0
#define DT_E4M3 1
#define DT_E4M3_GE5M2 2   /* E4M3 weights and X, E5M2 gradient operand */
#define DT_E5M2 3         /* E5M2 values; as a head: E5M2 weights, E4M3 X and gradient operand */
#define IS_FP8(dt) ((dt) == DT_E4M3 || (dt) == DT_E4M3_GE5M2 || (dt) == DT_E5M2)

/* ------------------------------------------------------------------------ */
/* Philox-4xW-10 (Salmon et al. 2011).  One round maps the counter words     */
/* (c0, c1, c2, c3) with key (k0, k1) to                                     */
/*   (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0));      */
/* the key is bumped by the Weyl constants between rounds.                   */
/* ------------------------------------------------------------------------ */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; r++) {
    if (r > 0) { k0 += W0; k1 += W1; }
    uint64_t p0 = (uint64_t)M0 * (uint64_t)c0;
    uint64_t p1 = (uint64_t)M1 * (uint64_t)c2;
    uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    uint32_t n1 = (uint32_t)p1;
    uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    uint32_t n3 = (uint32_t)p0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 64-bit-word member of the same family; only used to pin the round
 * structure against an independent library implementation. */
void orc_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
  const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
  uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint64_t k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; r++) {
    if (r > 0) { k0 += W0; k1 += W1; }
    unsigned __int128 p0 = (unsigned __int128)M0 * c0;
    unsigned __int128 p1 = (unsigned __int128)M1 * c2;
    uint64_t n0 = (uint64_t)(p1 >> 64) ^ c1 ^ k0;
    uint64_t n1 = (uint64_t)p1;
    uint64_t n2 = (uint64_t)(p0 >> 64) ^ c3 ^ k1;
    uint64_t n3 = (uint64_t)p0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 16-bit draw k for element idx of SR call (seed, step). */
uint32_t orc_draw16(uint64_t seed, uint64_t step, uint64_t idx) {
  uint64_t blk = idx >> 3;
  uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), (uint32_t)step, (uint32_t)(step >> 32)};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  orc_philox4x32_10(ctr, key, out);
  uint32_t word = out[(idx >> 1) & 3];
  return (idx & 1) ? (word >> 16) : (word & 0xFFFFu);
}

/* ------------------------------------------------------------------------ */
/* Number grids                                                              */
/* ------------------------------------------------------------------------ */
static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float orc_bf16_value(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* OCP E4M3FN: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent
 * field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; no infinities. */
float orc_e4m3_value(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  float mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexpf((float)m, -9);
  else mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return s ? -mag : mag;
}

/* Non-negative finite E4M3 magnitudes, ascending, indexed by code 0..126. */
static double e4m3_pos[127];
static int e4m3_ready = 0;
/* filled once when the library loads, before any parallel region */
__attribute__((constructor)) static void e4m3_fill(void) {
  for (int c = 0; c < 127; c++) e4m3_pos[c] = (double)orc_e4m3_value((uint8_t)c);
  e4m3_ready = 1;
}
static void e4m3_table(void) {
  if (!e4m3_ready) e4m3_fill();
}

/* Round-to-nearest-even onto the bf16 grid (standard conversion). */
uint16_t orc_rne_bf16(float v) {
  uint32_t b = bits_from_f32(v);
  if (isnan(v)) return 0x7FC0;
  uint32_t sign = b & 0x80000000u, mag = b & 0x7FFFFFFFu;
  uint32_t lo = mag >> 16;                 /* bf16 magnitude pattern just below */
  double a = fabs((double)v);
  double vlo = (double)orc_bf16_value((uint16_t)lo);
  /* the value above the largest finite is 2^128 (unbounded-exponent rounding; picking it overflows to inf) */
  double vhi = (lo + 1 == 0x7F80) ? ldexp(1.0, 128) : (double)orc_bf16_value((uint16_t)(lo + 1));
  uint32_t pick;
  if (a == vlo) pick = lo;
  else {
    double dlo = a - vlo, dhi = vhi - a;
    if (dlo < dhi) pick = lo;
    else if (dhi < dlo) pick = lo + 1;
    else pick = (lo & 1) ? lo + 1 : lo;    /* tie: even pattern */
  }
  return (uint16_t)((sign >> 16) | pick);
}

/* OCP E5M2: 1 sign, 5 exponent bits (bias 15), 2 mantissa bits; exponent
 * field 0 is subnormal (m * 2^-16); field 31 is infinity (m = 0) or NaN. */
float orc_e5m2_value(uint8_t c) {
  int s = c >> 7, e = (c >> 2) & 31, m = c & 3;
  float mag;
  if (e == 31) mag = m ? NAN : INFINITY;
  else if (e == 0) mag = ldexpf((float)m, -16);
  else mag = ldexpf(1.0f + (float)m / 4.0f, e - 15);
  return s ? -mag : mag;
}

/* Round-to-nearest-even onto the finite E5M2 grid, saturating to +-57344
 * (the largest finite value; infinities saturate too); NaN -> 0x7F. */
uint8_t orc_rne_e5m2(float v) {
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0;
  double a = fabs((double)v);
  if (a >= 57344.0) return sign | 0x7B;   /* codes 0x00 .. 0x7B are the finite magnitudes */
  int lo = 0;
  while (lo + 1 <= 0x7B && (double)orc_e5m2_value((uint8_t)(lo + 1)) <= a) lo++;
  double vlo = (double)orc_e5m2_value((uint8_t)lo);
  if (vlo == a) return sign | (uint8_t)lo;
  double vhi = (double)orc_e5m2_value((uint8_t)(lo + 1));
  double dlo = a - vlo, dhi = vhi - a;
  int pick;
  if (dlo < dhi) pick = lo;
  else if (dhi < dlo) pick = lo + 1;
  else pick = (lo & 1) ? lo + 1 : lo;      /* tie: even code */
  return sign | (uint8_t)pick;
}

/* Round-to-nearest-even onto the E4M3 grid, saturating to +-448. */
uint8_t orc_rne_e4m3(float v) {
  e4m3_table();
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0;
  double a = fabs((double)v);
  if (a >= 448.0) return sign | 126;
  int lo = 0;
  while (lo + 1 < 127 && e4m3_pos[lo + 1] <= a) lo++;
  if (e4m3_pos[lo] == a) return sign | (uint8_t)lo;
  int hi = lo + 1;
  double dlo = a - e4m3_pos[lo], dhi = e4m3_pos[hi] - a;
  int pick;
  if (dlo < dhi) pick = lo;
  else if (dhi < dlo) pick = hi;
  else pick = (lo & 1) ? hi : lo;          /* tie: even code */
  return sign | (uint8_t)pick;
}

/* ------------------------------------------------------------------------ */
/* Stochastic rounding, written from its definition: neighbours lo < v < hi */
/* on the target grid, f = (v - lo) / (hi - lo), and the element's 16-bit   */
/* draw k: round to hi iff k < floor(2^16 f), i.e. iff adding 2^16 - 1 - k  */
/* to the first 16 bits of the discarded fraction carries.  All in double,  */
/* where these quantities are exact for fp32 inputs.  On bf16 the fraction  */
/* has exactly 16 bits (floor(2^16 f) = 2^16 f): unbiased; on the 8-bit     */
/* grids the probability of hi is f less at most 2^-16.                     */
/* ------------------------------------------------------------------------ */
static int sr_up(double f, uint32_t k16) { return (double)k16 < floor(f * 65536.0); }

uint16_t orc_sr_bf16(float v, uint32_t k16) {
  if (isnan(v)) return 0x7FC0;
  uint32_t b = bits_from_f32(v);
  uint16_t sign = (uint16_t)((b >> 16) & 0x8000u);
  if (isinf(v)) return sign | 0x7F80;
  double a = fabs((double)v);
  uint32_t lo = (b & 0x7FFFFFFFu) >> 16;    /* largest bf16 magnitude <= a */
  double vlo = (double)orc_bf16_value((uint16_t)lo);
  if (vlo == a) return sign | (uint16_t)lo; /* on the grid: fixed point */
  if (lo + 1 >= 0x7F80) return sign | 0x7F7F;  /* above the largest finite */
  double vhi = (double)orc_bf16_value((uint16_t)(lo + 1));
  double f = (a - vlo) / (vhi - vlo);
  return sign | (uint16_t)(sr_up(f, k16) ? lo + 1 : lo);
}

uint8_t orc_sr_e4m3(float v, uint32_t k16) {
  e4m3_table();
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0;
  double a = fabs((double)v);
  if (a >= 448.0) return sign | 126;       /* saturate, inf included */
  int lo = 0;
  while (lo + 1 < 127 && e4m3_pos[lo + 1] <= a) lo++;
  if (e4m3_pos[lo] == a) return sign | (uint8_t)lo;
  int hi = lo + 1;
  double f = (a - e4m3_pos[lo]) / (e4m3_pos[hi] - e4m3_pos[lo]);
  return sign | (uint8_t)(sr_up(f, k16) ? hi : lo);
}

/* E5M2 has infinities, like bf16: +-inf stays +-inf, a finite |v| above the
 * largest finite value (57344) saturates to it, NaN -> 0x7F. */
uint8_t orc_sr_e5m2(float v, uint32_t k16) {
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0;
  if (isinf(v)) return sign | 0x7C;
  double a = fabs((double)v);
  if (a >= 57344.0) return sign | 0x7B;
  int lo = 0;                               /* codes 0 .. 0x7B: the finite magnitudes, ascending */
  while (lo + 1 <= 0x7B && (double)orc_e5m2_value((uint8_t)(lo + 1)) <= a) lo++;
  double vlo = (double)orc_e5m2_value((uint8_t)lo);
  if (vlo == a) return sign | (uint8_t)lo;
  double vhi = (double)orc_e5m2_value((uint8_t)(lo + 1));
  double f = (a - vlo) / (vhi - vlo);
  return sign | (uint8_t)(sr_up(f, k16) ? lo + 1 : lo);
}

/* out[i] = SR(in[i]) with the draw of element index_base + i. */
int orc_sr_round(const float* in, void* out, int64_t n, int dt, uint64_t seed,
                 uint64_t step, uint64_t index_base) {
  if (n < 0 || (n > 0 && (!in || !out))) return ORC_EINVAL;
  for (int64_t i = 0; i < n; i++) {
    uint32_t k = orc_draw16(seed, step, index_base + (uint64_t)i);
    if (dt == DT_BF16) ((uint16_t*)out)[i] = orc_sr_bf16(in[i], k);
    else if (dt == DT_E4M3) ((uint8_t*)out)[i] = orc_sr_e4m3(in[i], k);
    else if (dt == DT_E5M2) ((uint8_t*)out)[i] = orc_sr_e5m2(in[i], k);
    else return ORC_EINVAL;
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Operand preparation                                                       */
/* ------------------------------------------------------------------------ */
static float w_value(const void* W, int dt, int64_t i) {
  if (dt == DT_BF16) return orc_bf16_value(((const uint16_t*)W)[i]);
  if (dt == DT_E5M2) return orc_e5m2_value(((const uint8_t*)W)[i]);
  return orc_e4m3_value(((const uint8_t*)W)[i]);
}

/* s_X = 2^e with e the largest integer such that 2^e * max|X| <= 448,
 * clamped to [-126, 126]; max|X| == 0 or non-finite gives s_X = 1. */
float orc_fp8_x_scale(const uint16_t* X, int64_t n) {
  double amax = 0.0;
  int finite = 1;
  for (int64_t i = 0; i < n; i++) {
    double a = fabs((double)orc_bf16_value(X[i]));
    if (!isfinite(a)) finite = 0;
    else if (a > amax) amax = a;
  }
  if (!finite || amax == 0.0) return 1.0f;
  int e = 0;
  while (e < 126 && ldexp(amax, e + 1) <= 448.0) e++;
  while (e > -126 && ldexp(amax, e) > 448.0) e--;
  return ldexpf(1.0f, e);
}

/* The x operand values the step multiplies with, as fp32: bf16 mode the
 * values of X; fp8 mode E4M3(x * s_X) / s_X. */
static float* make_xv(const uint16_t* X, int32_t B, int32_t d, int dt, float* sx_out) {
  float* xv = (float*)malloc(sizeof(float) * (size_t)B * (size_t)d);
  float sx = 1.0f;
  if (IS_FP8(dt)) sx = orc_fp8_x_scale(X, (int64_t)B * d);
  for (int64_t i = 0; i < (int64_t)B * d; i++) {
    float x = orc_bf16_value(X[i]);
    if (IS_FP8(dt)) xv[i] = orc_e4m3_value(orc_rne_e4m3(x * sx)) / sx;
    else xv[i] = x;
  }
  if (sx_out) *sx_out = sx;
  return xv;
}

/* Sorted copy of every sample's positive labels (duplicates allowed). */
typedef struct { int32_t* lab; int64_t* off; } pos_t;
static int make_pos(const int32_t* rowptr, const int32_t* cols, int32_t B, int64_t L, pos_t* p) {
  if (rowptr[0] != 0) return ORC_EDATA;
  for (int b = 0; b < B; b++) if (rowptr[b + 1] < rowptr[b]) return ORC_EDATA;
  int64_t nnz = rowptr[B];
  for (int64_t i = 0; i < nnz; i++) if (cols[i] < 0 || (int64_t)cols[i] >= L) return ORC_EDATA;
  p->lab = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nnz > 0 ? nnz : 1));
  p->off = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  memcpy(p->lab, cols, sizeof(int32_t) * (size_t)nnz);
  for (int b = 0; b <= B; b++) p->off[b] = rowptr[b];
  for (int b = 0; b < B; b++) {           /* insertion sort: rows are short */
    int32_t* r = p->lab + p->off[b];
    int64_t n = p->off[b + 1] - p->off[b];
    for (int64_t i = 1; i < n; i++) {
      int32_t key = r[i]; int64_t j = i - 1;
      while (j >= 0 && r[j] > key) { r[j + 1] = r[j]; j--; }
      r[j + 1] = key;
    }
  }
  return ORC_OK;
}
static void free_pos(pos_t* p) { free(p->lab); free(p->off); }
static int is_positive(const pos_t* p, int b, int64_t l) {
  int64_t lo = p->off[b], hi = p->off[b + 1];
  while (lo < hi) {
    int64_t mid = (lo + hi) / 2;
    if (p->lab[mid] < l) lo = mid + 1; else hi = mid;
  }
  return lo < p->off[b + 1] && p->lab[lo] == l;
}

/* z = sum_j x[b,j] * w[l,j], fp32 accumulation in order j = 0..d-1; in fp8
 * mode the x operand is E4M3(x s_X) and the sum is divided by s_X. */
static float logit(const float* xq_row, const void* W, int dt, int64_t l, int32_t d, float inv_sx) {
  float acc = 0.0f;
  for (int j = 0; j < d; j++) {
    float prod = xq_row[j] * w_value(W, dt, l * d + j);
    acc = acc + prod;
  }
  return acc * inv_sx;
}

/* g = sigmoid(z) - y in fp32, then rounded to the operand grid: bf16, or
 * E4M3 / E5M2 of 2^8 g (the same fixed scale for both FP8 gradient grids). */
static float grad_operand(float z, int y, int dt) {
  float s = (float)(1.0 / (1.0 + exp(-(double)z)));
  float g = s - (y ? 1.0f : 0.0f);
  if (dt == DT_BF16) return orc_bf16_value(orc_rne_bf16(g));
  if (dt == DT_E4M3_GE5M2) return orc_e5m2_value(orc_rne_e5m2(g * 256.0f)) / 256.0f;
  return orc_e4m3_value(orc_rne_e4m3(g * 256.0f)) / 256.0f;
}

static int nthreads_or_default(int n) {
#ifdef _OPENMP
  return n > 0 ? n : omp_get_max_threads();
#else
  (void)n; return 1;
#endif
}

/*
 * One training step over labels [l0, l1).
 *   W      : [L, d] stored weights (bf16 bits or E4M3 codes), read only
 *   W_out  : [(l1-l0), d] updated weights of those labels
 *   dX     : [B, d] fp32 or NULL; receives sum over l in [l0,l1) of g_hat[b,l] * w[l,:]
 *   Z, G   : [(l1-l0), B] fp32 or NULL; logits and rounded gradient operand values
 * Returns ORC_EDATA on a malformed CSR.
 */
int orc_train_step(const void* W, void* W_out, int64_t L, int32_t d, int dt,
                   const uint16_t* X, int32_t B, const int32_t* rowptr, const int32_t* cols,
                   float lr, uint64_t seed, uint64_t step, int64_t l0, int64_t l1,
                   float* dX, float* Z, float* G, int nthreads) {
  if (!W || !X || !rowptr || B < 0 || d <= 0 || L < 0 || l0 < 0 || l1 > L || l0 > l1) return ORC_EINVAL;
  if (dt != DT_BF16 && !IS_FP8(dt)) return ORC_EINVAL;
  pos_t pos;
  int rc = make_pos(rowptr, cols, B, L, &pos);
  if (rc) return rc;
  float sx;
  float* xv = make_xv(X, B, d, dt, &sx);
  float* xq = (float*)malloc(sizeof(float) * (size_t)B * (size_t)d);  /* x operand before 1/s_X */
  for (int64_t i = 0; i < (int64_t)B * d; i++) xq[i] = xv[i] * sx;
  const float inv_sx = 1.0f / sx;
  int nt = nthreads_or_default(nthreads);
  int64_t nl = l1 - l0;
  float* part = NULL;
  if (dX) part = (float*)calloc((size_t)nt * (size_t)B * (size_t)d, sizeof(float));

#pragma omp parallel num_threads(nt)
  {
    int t = 0;
#ifdef _OPENMP
    t = omp_get_thread_num();
#endif
    float* gl = (float*)malloc(sizeof(float) * (size_t)(B > 0 ? B : 1));
    float* dxp = part ? part + (size_t)t * B * d : NULL;
    int64_t a = l0 + nl * t / nt, e = l0 + nl * (t + 1) / nt;   /* contiguous label range */
    for (int64_t l = a; l < e; l++) {
      for (int b = 0; b < B; b++) {
        float z = logit(xq + (size_t)b * d, W, dt, l, d, inv_sx);
        int y = is_positive(&pos, b, l);
        gl[b] = grad_operand(z, y, dt);
        if (Z) Z[(l - l0) * B + b] = z;
        if (G) G[(l - l0) * B + b] = gl[b];
      }
      for (int j = 0; j < d; j++) {
        float w = w_value(W, dt, l * d + j);
        float dw = 0.0f;
        for (int b = 0; b < B; b++) dw = dw + gl[b] * xv[(size_t)b * d + j];
        float step_ = lr * dw;
        float v = w - step_;
        uint32_t k = orc_draw16(seed, step, (uint64_t)l * (uint64_t)d + (uint64_t)j);
        if (W_out) {
          if (dt == DT_BF16) ((uint16_t*)W_out)[(l - l0) * d + j] = orc_sr_bf16(v, k);
          else if (dt == DT_E5M2) ((uint8_t*)W_out)[(l - l0) * d + j] = orc_sr_e5m2(v, k);
          else ((uint8_t*)W_out)[(l - l0) * d + j] = orc_sr_e4m3(v, k);
        }
        if (dxp) for (int b = 0; b < B; b++) dxp[(size_t)b * d + j] = dxp[(size_t)b * d + j] + gl[b] * w;
      }
    }
    free(gl);
  }
  if (dX) {
    for (int64_t i = 0; i < (int64_t)B * d; i++) {
      float s = 0.0f;
      for (int t = 0; t < nt; t++) s = s + part[(size_t)t * B * d + i];
      dX[i] = s;
    }
    free(part);
  }
  free(xv); free(xq); free_pos(&pos);
  return ORC_OK;
}

/*
 * Rows of dX for selected samples, over ALL labels: dX[b, :] = sum_l g_hat[b,l] w[l,:].
 * Each row depends only on its own sample, so full-size runs can be sampled.
 * Z_rows, G_rows ([ns, L] fp32, or NULL): the logits and rounded gradient
 * operand values of those samples.
 */
int orc_dx_rows(const void* W, int64_t L, int32_t d, int dt, const uint16_t* X, int32_t B,
                const int32_t* rowptr, const int32_t* cols, const int32_t* samples, int32_t ns,
                float* dX_rows, float* Z_rows, float* G_rows, int nthreads) {
  if (!W || !X || !rowptr || !samples || !dX_rows || d <= 0) return ORC_EINVAL;
  pos_t pos;
  int rc = make_pos(rowptr, cols, B, L, &pos);
  if (rc) return rc;
  for (int s = 0; s < ns; s++) if (samples[s] < 0 || samples[s] >= B) { free_pos(&pos); return ORC_EINVAL; }
  float sx;
  float* xv = make_xv(X, B, d, dt, &sx);
  const float inv_sx = 1.0f / sx;
  int nt = nthreads_or_default(nthreads);
  float* part = (float*)calloc((size_t)nt * (size_t)ns * (size_t)d, sizeof(float));
  float* xq = (float*)malloc(sizeof(float) * (size_t)ns * (size_t)d);
  for (int s = 0; s < ns; s++)
    for (int j = 0; j < d; j++) xq[(size_t)s * d + j] = xv[(size_t)samples[s] * d + j] * sx;
#pragma omp parallel num_threads(nt)
  {
    int t = 0;
#ifdef _OPENMP
    t = omp_get_thread_num();
#endif
    float* p = part + (size_t)t * ns * d;
    int64_t a = L * t / nt, e = L * (t + 1) / nt;
    for (int64_t l = a; l < e; l++) {
      for (int s = 0; s < ns; s++) {
        float z = logit(xq + (size_t)s * d, W, dt, l, d, inv_sx);
        float g = grad_operand(z, is_positive(&pos, samples[s], l), dt);
        if (Z_rows) Z_rows[(size_t)s * L + l] = z;
        if (G_rows) G_rows[(size_t)s * L + l] = g;
        for (int j = 0; j < d; j++) p[(size_t)s * d + j] = p[(size_t)s * d + j] + g * w_value(W, dt, l * d + j);
      }
    }
  }
  for (int64_t i = 0; i < (int64_t)ns * d; i++) {
    float acc = 0.0f;
    for (int t = 0; t < nt; t++) acc = acc + part[(size_t)t * ns * d + i];
    dX_rows[i] = acc;
  }
  free(part); free(xq); free(xv); free_pos(&pos);
  return ORC_OK;
}

/* Ranking order of the top-k: higher score first, NaN after every number,
 * equal scores (and NaNs among themselves) by lower label index. */
static int ranks_before(float sa, int64_t ia, float sb, int64_t ib) {
  int na = isnan(sa), nb = isnan(sb);
  if (na != nb) return nb;                 /* the number goes first */
  if (!na && sa != sb) return sa > sb;
  return ia < ib;
}

/* Exact score of (b, l): s = fma(x[b,j], w[l,j], s) for j = 0..d-1 from 0. */
float orc_score(const void* W, int dt, int64_t l, const uint16_t* X, int32_t b, int32_t d) {
  float s = 0.0f;
  for (int j = 0; j < d; j++) s = fmaf(orc_bf16_value(X[(size_t)b * d + j]), w_value(W, dt, l * d + j), s);
  return s;
}

/* Exact scores of the listed rows of X against labels [l0, l1): out[r, l - l0]. */
int orc_scores(const void* W, int64_t L, int32_t d, int dt, const uint16_t* X, int32_t B, const int32_t* rows,
               int32_t nrows, int64_t l0, int64_t l1, float* out, int nthreads) {
  if (!W || !X || !rows || !out || l0 < 0 || l1 > L || l0 > l1 || d <= 0) return ORC_EINVAL;
  for (int r = 0; r < nrows; r++) if (rows[r] < 0 || rows[r] >= B) return ORC_EINVAL;
  int nt = nthreads_or_default(nthreads);
#pragma omp parallel for num_threads(nt) schedule(static)
  for (int64_t l = l0; l < l1; l++)
    for (int r = 0; r < nrows; r++) out[(size_t)r * (l1 - l0) + (l - l0)] = orc_score(W, dt, l, X, rows[r], d);
  return ORC_OK;
}

/*
 * Top-k over all L labels for the listed rows (rows == NULL: rows 0..nrows-1).
 * X is used unquantised (bf16 values) in both modes.  Outputs [nrows, k].
 */
int orc_topk(const void* W, int64_t L, int32_t d, int dt, const uint16_t* X, int32_t B, int32_t k,
             const int32_t* rows, int32_t nrows, int32_t* idx_out, float* score_out, int nthreads) {
  if (!W || !X || !idx_out || !score_out || k <= 0 || k > L || d <= 0) return ORC_EINVAL;
  int nt = nthreads_or_default(nthreads);
  for (int r = 0; r < nrows; r++) {
    int32_t b = rows ? rows[r] : r;
    if (b < 0 || b >= B) return ORC_EINVAL;
    /* every thread keeps its own sorted top-k of a label range; then merge */
    int32_t* ti = (int32_t*)malloc(sizeof(int32_t) * (size_t)nt * k);
    float* ts = (float*)malloc(sizeof(float) * (size_t)nt * k);
    int* tn = (int*)calloc((size_t)nt, sizeof(int));
#pragma omp parallel num_threads(nt)
    {
      int t = 0;
#ifdef _OPENMP
      t = omp_get_thread_num();
#endif
      int32_t* mi = ti + (size_t)t * k; float* ms = ts + (size_t)t * k; int n = 0;
      int64_t a = L * t / nt, e = L * (t + 1) / nt;
      for (int64_t l = a; l < e; l++) {
        float s = orc_score(W, dt, l, X, b, d);
        if (n == k && !ranks_before(s, l, ms[k - 1], mi[k - 1])) continue;
        int pos = (n < k) ? n++ : k - 1;
        while (pos > 0 && ranks_before(s, l, ms[pos - 1], mi[pos - 1])) {
          ms[pos] = ms[pos - 1]; mi[pos] = mi[pos - 1]; pos--;
        }
        ms[pos] = s; mi[pos] = (int32_t)l;
      }
      tn[t] = n;
    }
    int32_t* oi = idx_out + (size_t)r * k; float* os = score_out + (size_t)r * k; int n = 0;
    for (int t = 0; t < nt; t++) {
      for (int q = 0; q < tn[t]; q++) {
        float s = ts[(size_t)t * k + q]; int64_t l = ti[(size_t)t * k + q];
        if (n == k && !ranks_before(s, l, os[k - 1], oi[k - 1])) continue;
        int pos = (n < k) ? n++ : k - 1;
        while (pos > 0 && ranks_before(s, l, os[pos - 1], oi[pos - 1])) {
          os[pos] = os[pos - 1]; oi[pos] = oi[pos - 1]; pos--;
        }
        os[pos] = s; oi[pos] = (int32_t)l;
      }
    }
    free(ti); free(ts); free(tn);
  }
  return ORC_OK;
}

/*
 * P@j for j = 1..k ("ELMO: Efficiency via Low-precision and Peak Memory
 * Optimization in Large Output Spaces", atlas summary, metrics P@1/3/5): the
 * mean over the B rows of |{first j predicted labels of the row} ∩ Y_b| / j,
 * with Y_b the row's positive labels cols[rowptr[b] .. rowptr[b+1]).  idx is
 * [B, k] (each row's predictions in rank order).  p[j-1] = P@j, computed as an
 * exact integer hit count over j*B in double.
 */
int orc_precision_at_k(const int32_t* idx, int32_t B, int32_t k, const int32_t* rowptr, const int32_t* cols,
                       double* p) {
  if (!idx || !rowptr || !p || B < 1 || k < 1) return ORC_EINVAL;
  for (int j = 0; j < k; j++) p[j] = 0.0;
  int64_t* hits = (int64_t*)calloc((size_t)k, sizeof(int64_t));
  for (int32_t b = 0; b < B; b++) {
    int64_t h = 0;
    for (int32_t i = 0; i < k; i++) {
      int32_t lab = idx[(size_t)b * k + i];
      int hit = 0;
      for (int32_t q = rowptr[b]; q < rowptr[b + 1] && !hit; q++) hit = (cols[q] == lab);
      h += hit;
      hits[i] += h;                 /* hits among the first i + 1 predictions */
    }
  }
  for (int j = 0; j < k; j++) p[j] = (double)hits[j] / ((double)(j + 1) * (double)B);
  free(hits);
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Kahan-compensated SGD of a dense BF16 layer (the encoder side).           */
/* The pages train the encoder in pure BF16 with Kahan summation in place of */
/* FP32 master weights (atlas summary "Approach"; abstract).  Reading: the   */
/* parameters p and the compensation c are stored in bf16, the gradient g   */
/* arrives in bf16; every operation below is one IEEE fp32 operation and    */
/* the two stored results are rounded to bf16 to nearest-even:              */
/*   u  = -(lr * g)               the plain SGD increment                   */
/*   y  = u + c                   plus what earlier steps could not store   */
/*   p' = bf16(p + y)             the new parameter                         */
/*   c' = bf16(y - (p' - p))      what this step could not store            */
/* Kahan's compensated summation (Kahan 1965) applied to p + sum of u.      */
/* ------------------------------------------------------------------------ */
void orc_kahan_sgd(uint16_t* p, uint16_t* c, const uint16_t* g, int64_t n, float lr) {
  for (int64_t i = 0; i < n; i++) {
    const float pv = orc_bf16_value(p[i]);
    const float cv = orc_bf16_value(c[i]);
    const float gv = orc_bf16_value(g[i]);
    const float prod = lr * gv;
    const float u = -prod;
    const float y = u + cv;
    const float sum = pv + y;
    const uint16_t pn = orc_rne_bf16(sum);
    const float moved = orc_bf16_value(pn) - pv;
    const float lost = y - moved;
    c[i] = orc_rne_bf16(lost);
    p[i] = pn;
  }
}

/* ------------------------------------------------------------------------ */
/* Array helpers for the Python side (loops over the scalar definitions).   */
/* ------------------------------------------------------------------------ */
void orc_draw16_array(uint64_t seed, uint64_t step, uint64_t base, int64_t n, uint32_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_draw16(seed, step, base + (uint64_t)i);
}
void orc_sr_bf16_array(const float* v, const uint32_t* k, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_sr_bf16(v[i], k[i]);
}
void orc_sr_e5m2_array(const float* v, const uint32_t* k, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_sr_e5m2(v[i], k[i]);
}
void orc_sr_e4m3_array(const float* v, const uint32_t* k, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_sr_e4m3(v[i], k[i]);
}
void orc_rne_bf16_array(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_rne_bf16(v[i]);
}
void orc_rne_e5m2_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_rne_e5m2(v[i]);
}
void orc_e5m2_value_array(const uint8_t* c, int64_t n, float* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_e5m2_value(c[i]);
}
void orc_rne_e4m3_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_rne_e4m3(v[i]);
}
void orc_e4m3_value_array(const uint8_t* c, int64_t n, float* out) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_e4m3_value(c[i]);
}
