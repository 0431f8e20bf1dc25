/*
 * mla_oracle.c -- plain, slow, fp64 CPU oracle for MLA decoding over a paged
 * latent KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or helper with
 * the CUDA library: every conversion below (bf16, E4M3, the 656-byte cache
 * row, RoPE angles) is written out here from the format or the formula.
 *
 * What it computes (sources, by page title and section):
 *  - Attention of every query head against ONE shared 576-dim latent KV head
 *    (512 "nope" dims + 64 decoupled-RoPE dims), V being the first d_v dims
 *    of the same latent row; exact softmax attention in the FlashAttention
 *    sense, returning the output and its log-sum-exp.
 *      [FlashMLA (AI Wiki), "How does MLA differ from MHA and GQA?"]
 *      [FlashMLA (AI Wiki), "How is FlashMLA designed?"]
 *      [FlashMLA (AI Wiki), "Interfaces"]  (output AND log-sum-exp)
 *  - Paged cache with 64-token blocks reached through a block table, and
 *    variable per-sequence lengths.
 *      [FlashMLA (AI Wiki), "What is FlashMLA?" day-one description]
 *      [FlashMLA Ampere port README, "Usage"]  (metadata / with_kvcache call)
 *  - The fused step order: Q RMSNorm, Q-RoPE, attention, conjugate O-RoPE,
 *    FP8 cast.
 *      [FlashMLA fused norm-RoPE-attention-RoPE-cast kernel card, "Arithmetic
 *       intensity"] and [deepseek-ai/FlashMLA README, "News", 2026.09.10]
 *  - Token-level sparse decode: indices (b, s_q, topk) hold physical slots
 *    (block*64 + offset), -1 marks an invalid slot, block table ignored.
 *    Sparse prefill has no batch dimension and optional attention-sink and
 *    per-token top-k-length arguments.
 *      [FlashMLA (AI Wiki), "Interfaces"]
 *  - The fused kernel is recommended over the standalone sparse kernels, so
 *    its steps also run over a sparse selection of slots.
 *      [FlashMLA fused norm-RoPE-attention-RoPE-cast kernel card,
 *       "Workarounds"]
 *  - The 656-byte FP8 cache row: 512 E4M3 codes, 4 fp32 tile scales (one per
 *    128 values), 64 bf16 RoPE dims.
 *      [FlashMLA (AI Wiki), "The FP8 and FP4 KV cache"]
 *  - The 528-byte V4.1 FP8 cache row: 512 E4M3 codes covering every dim of a
 *    512-dim latent (RoPE dims included), then 16 E8M0 scales, one per 32
 *    consecutive codes.
 *  - The 288-byte V4.1 FP4 cache row: 512 E2M1 codes packed two per byte
 *    into 256 bytes, then 32 E4M3 scales, one per 16 consecutive codes.
 *      [FlashMLA (AI Wiki), "The FP8 and FP4 KV cache", layout table]
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - LSE is the natural log; an empty row gives O = 0 and LSE = -inf.
 *  - Causal alignment is bottom-right: query i of s_q sees L - s_q + 1 + i
 *    tokens.
 *  - Row byte order of the 656-byte cache: [512 x e4m3][4 x fp32][64 x bf16].
 *  - RoPE pairs are interleaved (2k, 2k+1), theta_k = pos * base^(-2k/64);
 *    conjugate RoPE rotates by -theta_k.
 *  - Fused path: the normalised, rotated query enters the attention in bf16
 *    (the tensor-core operand precision); the pages leave this precision
 *    open, and fixing it makes the FP8 code decisions comparable.
 *  - Sparse prefill: a sink is one logit per head that joins the softmax
 *    normaliser without a value row (the returned LSE includes it); a
 *    top-k length counts only the first entries of a token's indices.
 *  - Fused sparse mode: the query position is an input.
 *  - Sparse paths: the dequantised rows enter the attention rounded to bf16
 *    (round to nearest even), as the quantised decoding kernels convert them.
 *  - V4.1 rows: the latent is 512 wide, q . K runs over all 512 dims and V is
 *    the whole latent (d_v = 512).  An E8M0 byte e is the power of two
 *    2^(e - 127); 0xFF is NaN.  In the FP4 row, code 2i sits in the low
 *    nibble of byte i and code 2i + 1 in the high nibble.
 *  - FP8 output: scale = absmax/448 (scale := 1 when absmax == 0), code =
 *    E4M3 round-to-nearest-even with saturation to +-448 of (o / scale),
 *    where the ratio is rounded to fp32 before encoding (the kernel takes
 *    the same decision in fp32).
 *
 * Everything is fp64 (inputs are decoded exactly from bf16 / e4m3 / fp32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_D 576
#define ORACLE_NOPE 512
#define ORACLE_ROPE 64
#define ORACLE_ROW656 656
#define ORACLE_D41 512
#define ORACLE_ROW528 528
#define ORACLE_ROW288 288

/* ---------------------------------------------------------------- formats */

/* bf16 is the top half of an IEEE binary32 word: decoding is exact. */
static double bf16_bits_to_f64(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static double f32_bytes_to_f64(const uint8_t* p) {
  float f;
  memcpy(&f, p, 4); /* little-endian host, as the cache format is written */
  return (double)f;
}

/* OCP 8-bit floating point, E4M3 ("fn": no infinities, one NaN pattern per
 * sign, S.1111.111).  Exponent bias 7, three mantissa bits. */
double oracle_e4m3_decode(uint8_t c) {
  int sign = c >> 7;
  int e = (c >> 3) & 0xF;
  int m = c & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9); /* subnormal: m/8 * 2^(1-7) */
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Round-half-to-even of a non-negative double to an integer value. */
static double rne(double x) {
  double f = floor(x);
  double r = x - f;
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* E4M3 encoder: round to nearest even, saturate finite values to +-448,
 * NaN -> 0x7F.  Written from the format: normal numbers (1+m/8)*2^(e-7) for
 * e in 1..15 (excluding the NaN slot), subnormals m*2^-9. */
uint8_t oracle_e4m3_encode(double x) {
  uint8_t sign;
  double a;
  if (isnan(x)) return 0x7F;
  sign = signbit(x) ? 0x80 : 0x00;
  a = fabs(x);
  if (a >= 448.0) return sign | 0x7E;
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: quantum 2^-9; m == 8 is exactly the smallest normal,
     * whose code (e=1, m=0) is 0x08, so the code is m itself. */
    double m = rne(a * 512.0);
    return sign | (uint8_t)m;
  } else {
    int e2;
    double fr = frexp(a, &e2); /* a = fr * 2^e2, fr in [0.5, 1) */
    int e = e2 - 1;            /* a = (2 fr) * 2^e, 2fr in [1, 2) */
    double m = rne((2.0 * fr - 1.0) * 8.0);
    if (m >= 8.0) {
      m = 0.0;
      e += 1;
    }
    {
      int be = e + 7;
      if (be > 15 || (be == 15 && m > 6.0)) return sign | 0x7E;
      return sign | (uint8_t)((be << 3) | (int)m);
    }
  }
}

/* Round to the nearest bf16 value (8 significant bits, ties to even); bf16
 * shares fp32's exponent range, and the values rounded here are normal. */
double oracle_round_bf16(double v) {
  int e;
  double m, r;
  if (v == 0.0 || !isfinite(v)) return v;
  m = frexp(fabs(v), &e); /* |v| = m * 2^e, m in [0.5, 1) */
  r = rne(ldexp(m, 8));   /* 8 significant bits */
  r = ldexp(r, e - 8);
  return v < 0 ? -r : r;
}

/* ---------------------------------------------------------------- RMSNorm */

/* y = x / sqrt(mean(x^2) + eps) * g over n dims.
 * [FlashMLA fused norm-RoPE-attention-RoPE-cast kernel card] names Q-norm;
 * RMSNorm over the 576 latent dims with one gain vector is the reading. */
void oracle_rmsnorm(const double* x, const double* g, int n, double eps, double* y) {
  double ss = 0.0;
  int i;
  for (i = 0; i < n; ++i) ss += x[i] * x[i];
  {
    double inv = 1.0 / sqrt(ss / n + eps);
    for (i = 0; i < n; ++i) y[i] = x[i] * inv * g[i];
  }
}

/* ------------------------------------------------------------------- RoPE */

/* Rotary embedding on a 64-dim vector, interleaved pairs (2k, 2k+1):
 *   theta_k = pos * base^(-2k/64)
 *   (a, b) -> (a cos - b sin, a sin + b cos)          (sign = +1)
 * The conjugate rotation (sign = -1) rotates by -theta_k.
 * [FlashMLA (AI Wiki), "How does MLA differ from MHA and GQA?"] (decoupled
 * RoPE dims) and the fused kernel card (Q-RoPE, conjugate O-RoPE). */
void oracle_rope64(const double* x, double pos, double base, int sign, double* y) {
  int k;
  for (k = 0; k < ORACLE_ROPE / 2; ++k) {
    double theta = pos * pow(base, -2.0 * k / (double)ORACLE_ROPE);
    double c = cos(theta), s = sin(theta) * (sign < 0 ? -1.0 : 1.0);
    double a = x[2 * k], b = x[2 * k + 1];
    y[2 * k] = a * c - b * s;
    y[2 * k + 1] = a * s + b * c;
  }
}

/* -------------------------------------------------------- attention core */

/* A key row source: fetch(ctx, j, out) writes the fp64 latent row of the
 * j-th attended token into out[576]. */
typedef void (*row_fetch_fn)(const void* ctx, int j, double* out);

/* Exact attention of one query row q[d_qk] over n tokens, with an optional
 * attention-sink logit (-inf = none) that joins the normaliser without a
 * value row:
 *   s_t = scale * q . K_t ;  m = max(max_t s_t, sink) ;
 *   LSE = m + ln (sum_t exp(s_t - m) + exp(sink - m)) ;
 *   O   = sum_t exp(s_t - LSE) * K_t[0:d_v]
 * Two passes over the rows (scores, then the weighted sum); n == 0 gives
 * O = 0, LSE = sink. */
static void attend_rows_ds(const double* q, int d_qk, row_fetch_fn fetch, const void* ctx, int n,
                           int d_v, double scale, double sink, double* o, double* lse) {
  int t, d;
  double m = sink, sum = 0.0, l;
  double k[ORACLE_D];
  double* s;
  for (d = 0; d < d_v; ++d) o[d] = 0.0;
  if (n == 0) {
    *lse = sink;
    return;
  }
  s = (double*)malloc(sizeof(double) * (size_t)n);
  for (t = 0; t < n; ++t) {
    double acc = 0.0;
    fetch(ctx, t, k);
    for (d = 0; d < d_qk; ++d) acc += q[d] * k[d];
    s[t] = scale * acc;
    if (s[t] > m) m = s[t];
  }
  for (t = 0; t < n; ++t) sum += exp(s[t] - m);
  if (sink != -INFINITY) sum += exp(sink - m);
  l = m + log(sum);
  for (t = 0; t < n; ++t) {
    double p = exp(s[t] - l);
    fetch(ctx, t, k);
    for (d = 0; d < d_v; ++d) o[d] += p * k[d];
  }
  *lse = l;
  free(s);
}

static void attend_rows_d(const double* q, int d_qk, row_fetch_fn fetch, const void* ctx, int n,
                          int d_v, double scale, double* o, double* lse) {
  attend_rows_ds(q, d_qk, fetch, ctx, n, d_v, scale, -INFINITY, o, lse);
}

static void attend_rows(const double* q, row_fetch_fn fetch, const void* ctx, int n, int d_v,
                        double scale, double* o, double* lse) {
  attend_rows_d(q, ORACLE_D, fetch, ctx, n, d_v, scale, o, lse);
}

/* Paged bf16 cache source: token j of the window is logical token lo + j of
 * sequence b, found through the block table. */
typedef struct {
  const uint16_t* kcache;
  const int32_t* block_table;
  int num_blocks, max_pages, b, lo, page;
} paged_ctx;

/* A block id outside [0, num_blocks) names no page of the cache; it is read
 * as block 0 (reading: a stand-in that keeps every read inside the cache,
 * with the fault reported to the caller). */
static int paged_block(const paged_ctx* c, int page_idx) {
  int blk = c->block_table[(size_t)c->b * c->max_pages + page_idx];
  return (blk < 0 || blk >= c->num_blocks) ? 0 : blk;
}

/* Tokens of sequence b that the block table can reach: a length beyond
 * max_pages * page is read as that many (reading: the table names no
 * further page). */
static int paged_length(int L, int max_pages, int page) {
  long long cap = (long long)max_pages * page;
  return (long long)L > cap ? (int)cap : L;
}

/* 1 when sequence c->b's table has an out-of-range id among its first
 * ceil(L / page) entries, or its raw length L_raw exceeds the table. */
static int paged_faults(const paged_ctx* c, int L_raw, int L) {
  int p, blk;
  if (L_raw != L) return 1;
  for (p = 0; p < (L + c->page - 1) / c->page; ++p) {
    blk = c->block_table[(size_t)c->b * c->max_pages + p];
    if (blk < 0 || blk >= c->num_blocks) return 1;
  }
  return 0;
}

static void fetch_paged_bf16(const void* vctx, int j, double* out) {
  const paged_ctx* c = (const paged_ctx*)vctx;
  int t = c->lo + j;
  int blk = paged_block(c, t / c->page);
  const uint16_t* row = c->kcache + ((size_t)blk * c->page + (size_t)(t % c->page)) * ORACLE_D;
  int d;
  for (d = 0; d < ORACLE_D; ++d) out[d] = bf16_bits_to_f64(row[d]);
}

/* Decode one 656-byte FP8 cache row: [512 e4m3][4 fp32 scales][64 bf16]. */
void oracle_decode_row656(const uint8_t* row, double* out) {
  int d;
  for (d = 0; d < ORACLE_NOPE; ++d)
    out[d] = oracle_e4m3_decode(row[d]) * f32_bytes_to_f64(row + ORACLE_NOPE + 4 * (d / 128));
  for (d = 0; d < ORACLE_ROPE; ++d) {
    uint16_t h;
    memcpy(&h, row + ORACLE_NOPE + 16 + 2 * d, 2);
    out[ORACLE_NOPE + d] = bf16_bits_to_f64(h);
  }
}

/* FP8 cache source: the j-th entry of a list of physical slots. */
typedef struct {
  const uint8_t* cache;
  const int32_t* slots;
} fp8_ctx;

/* The attention sees a dequantised row rounded to bf16 (RNE): the quantised
 * decoding kernels convert their dequantised values with round-to-nearest to
 * bf16 pairs for the tensor cores [FlashMLA (AI Wiki), "Requirements and
 * build", NVIDIA toolchain row].  Exact for the V4.1 rows, whose values are
 * bf16 numbers already. */
static void round_row_bf16(double* out, int n) {
  int d;
  for (d = 0; d < n; ++d) out[d] = oracle_round_bf16(out[d]);
}

static void fetch_fp8(const void* vctx, int j, double* out) {
  const fp8_ctx* c = (const fp8_ctx*)vctx;
  oracle_decode_row656(c->cache + (size_t)c->slots[j] * ORACLE_ROW656, out);
  round_row_bf16(out, ORACLE_D);
}

/* Number of tokens query i (of s_q) of a sequence of length L may see. */
static int visible_tokens(int L, int s_q, int i, int causal) {
  int v = causal ? L - s_q + 1 + i : L;
  if (v < 0) v = 0;
  if (v > L) v = L;
  return v;
}

/* ------------------------------------------------------------ dense path */

/* Dense paged MLA decode.
 *  q           [b, s_q, h_q, 576] bf16 bits
 *  kcache      [num_blocks, page, 1, 576] bf16 bits
 *  block_table [b, max_pages] int32; an id outside [0, num_blocks) reads
 *              block 0, and a length above max_pages * page is read as
 *              max_pages * page (both are input faults: the return is 1)
 *  seqlens     [b] int32
 *  rows        optional list of n_rows flat row ids (b*s_q + i)*h_q + h;
 *              NULL computes every row.  Outputs are indexed by the flat row
 *              id when rows == NULL, else by position in `rows`.
 *  out         [.., d_v] fp64;  lse [..] fp64 (natural log)
 *  token_lo/hi optional per-batch half-open logical token window [lo, hi)
 *              intersected with the visible range (used to form split
 *              partials); NULL = whole range.
 * Returns 0. */
int oracle_dense_decode(const uint16_t* q, const uint16_t* kcache, int num_blocks,
                        const int32_t* block_table, int max_pages, const int32_t* seqlens,
                        int batch, int s_q, int h_q, int d_v, int page, double scale, int causal,
                        const int64_t* rows, int64_t n_rows, const int32_t* token_lo,
                        const int32_t* token_hi, double* out, double* lse) {
  int64_t total = (int64_t)batch * s_q * h_q;
  int64_t n = rows ? n_rows : total;
  int64_t r;
  int fault = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : fault)
  for (r = 0; r < n; ++r) {
    int64_t flat = rows ? rows[r] : r;
    int i = (int)((flat / h_q) % s_q);
    int b = (int)(flat / ((int64_t)h_q * s_q));
    int L = paged_length(seqlens[b], max_pages, page);
    int vis = visible_tokens(L, s_q, i, causal);
    int lo = token_lo ? token_lo[b] : 0;
    int hi = token_hi ? token_hi[b] : vis;
    int d, cnt;
    double qv[ORACLE_D];
    paged_ctx ctx;
    const uint16_t* qr = q + (size_t)flat * ORACLE_D;
    if (hi > vis) hi = vis;
    if (lo < 0) lo = 0;
    cnt = hi > lo ? hi - lo : 0;
    for (d = 0; d < ORACLE_D; ++d) qv[d] = bf16_bits_to_f64(qr[d]);
    ctx.kcache = kcache;
    ctx.block_table = block_table;
    ctx.num_blocks = num_blocks;
    ctx.max_pages = max_pages;
    ctx.b = b;
    ctx.lo = lo;
    ctx.page = page;
    fault |= paged_faults(&ctx, seqlens[b], L);
    attend_rows(qv, fetch_paged_bf16, &ctx, cnt, d_v, scale, out + (size_t)r * d_v, lse + r);
  }
  return fault;
}

/* LSE-weighted merge of n_splits partial results of one row:
 *   LSE = log sum_i exp(LSE_i)   (max-subtracted)
 *   O   = sum_i exp(LSE_i - LSE) * O_i
 * Splits with LSE_i = -inf contribute nothing; all empty -> O = 0, -inf. */
void oracle_combine(int n_splits, const double* lse_i, const double* o_i, int d_v, double* o,
                    double* lse) {
  int s, d;
  double m = -INFINITY, sum = 0.0, l;
  for (d = 0; d < d_v; ++d) o[d] = 0.0;
  for (s = 0; s < n_splits; ++s)
    if (lse_i[s] > m) m = lse_i[s];
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  for (s = 0; s < n_splits; ++s) sum += exp(lse_i[s] - m);
  l = m + log(sum);
  for (s = 0; s < n_splits; ++s) {
    double w = exp(lse_i[s] - l);
    if (lse_i[s] == -INFINITY) continue;
    for (d = 0; d < d_v; ++d) o[d] += w * o_i[(size_t)s * d_v + d];
  }
  *lse = l;
}

/* ------------------------------------------------------------ fused path */

/* Fused norm -> Q-RoPE -> attention -> conjugate O-RoPE -> FP8 cast, s_q = 1.
 *  q_raw   [b, 1, h_q, 576] bf16 bits
 *  gain    [576] fp64 (the fp32 gain, widened)
 *  positions optional [b]; NULL means position = seqlen - 1
 *  The cache's last 64 dims are taken as already rotated at their own
 *  positions (the cache writer's job); attention uses d_v = 576.
 *  codes   [.., 576] e4m3;  out_scale [..];  lse [..];
 *  o_pre   optional [.., 576]: the fp64 row after conjugate RoPE, before the
 *          cast (lets tests compare the pre-cast values).
 * Step order: [FlashMLA fused norm-RoPE-attention-RoPE-cast kernel card]. */
/* The fused steps for one query row over n tokens given by `fetch`: RMSNorm
 * of the raw query, RoPE of its dims 512..575 at `pos`, one bf16 rounding,
 * attention with d_v = 576, conjugate RoPE of O's dims 512..575, then the
 * per-row FP8 cast (scale = absmax/448). */
static void fused_row(const uint16_t* qr, const double* gain, double eps, double rope_base,
                      double pos, row_fetch_fn fetch, const void* ctx, int n, double scale,
                      uint8_t* codes, double* out_scale, double* lse, double* o_pre) {
  double x[ORACLE_D], y[ORACLE_D], o[ORACLE_D], orot[ORACLE_ROPE];
  double l, amax = 0.0, sc;
  int d;
  for (d = 0; d < ORACLE_D; ++d) x[d] = bf16_bits_to_f64(qr[d]);
  oracle_rmsnorm(x, gain, ORACLE_D, eps, y);
  oracle_rope64(y + ORACLE_NOPE, pos, rope_base, +1, x + ORACLE_NOPE);
  for (d = 0; d < ORACLE_NOPE; ++d) x[d] = y[d];
  for (d = 0; d < ORACLE_D; ++d) x[d] = oracle_round_bf16(x[d]);
  attend_rows(x, fetch, ctx, n, ORACLE_D, scale, o, &l);
  oracle_rope64(o + ORACLE_NOPE, pos, rope_base, -1, orot);
  for (d = 0; d < ORACLE_ROPE; ++d) o[ORACLE_NOPE + d] = orot[d];
  for (d = 0; d < ORACLE_D; ++d)
    if (fabs(o[d]) > amax) amax = fabs(o[d]);
  sc = amax > 0.0 ? amax / 448.0 : 1.0;
  for (d = 0; d < ORACLE_D; ++d) {
    float ratio = (float)(o[d] / sc);
    codes[d] = oracle_e4m3_encode((double)ratio);
    if (o_pre) o_pre[d] = o[d];
  }
  *out_scale = sc;
  *lse = l;
}

int oracle_fused_decode(const uint16_t* q_raw, const double* gain, double eps, double rope_base,
                        const int32_t* positions, const uint16_t* kcache, int num_blocks,
                        const int32_t* block_table, int max_pages, const int32_t* seqlens,
                        int batch, int h_q, int page, double scale, const int64_t* rows,
                        int64_t n_rows, uint8_t* codes, double* out_scale, double* lse,
                        double* o_pre) {
  int64_t total = (int64_t)batch * h_q;
  int64_t n = rows ? n_rows : total;
  int64_t r;
  int fault = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : fault)
  for (r = 0; r < n; ++r) {
    int64_t flat = rows ? rows[r] : r;
    int b = (int)(flat / h_q);
    /* the default query position follows the length as given; the tokens
     * attended stop where the block table does */
    int L = paged_length(seqlens[b] > 0 ? seqlens[b] : 0, max_pages, page);
    double pos = positions ? (double)positions[b] : (double)(seqlens[b] - 1);
    paged_ctx ctx;
    ctx.kcache = kcache;
    ctx.block_table = block_table;
    ctx.num_blocks = num_blocks;
    ctx.max_pages = max_pages;
    ctx.b = b;
    ctx.lo = 0;
    ctx.page = page;
    fault |= paged_faults(&ctx, seqlens[b], L);
    fused_row(q_raw + (size_t)flat * ORACLE_D, gain, eps, rope_base, pos, fetch_paged_bf16, &ctx,
              L, scale, codes + (size_t)r * ORACLE_D, out_scale + r, lse + r,
              o_pre ? o_pre + (size_t)r * ORACLE_D : 0);
  }
  return fault;
}

/* ----------------------------------------------------------- sparse path */

/* Token-level sparse decode over the 656-byte FP8 cache.
 *  q        [b, s_q, h_q, 576] bf16 bits
 *  cache    [num_slots, 656] bytes (slot = block*64 + offset)
 *  indices  [b, s_q, topk] int32 physical slots, -1 = invalid (skipped)
 *  No causal mask: the indices already name the visible tokens.
 *  rows/out/lse as in the dense path. */
int oracle_sparse_decode(const uint16_t* q, const uint8_t* cache, int64_t num_slots,
                         const int32_t* indices, int batch, int s_q, int h_q, int topk, int d_v,
                         double scale, const int64_t* rows, int64_t n_rows, double* out,
                         double* lse) {
  int64_t total = (int64_t)batch * s_q * h_q;
  int64_t n = rows ? n_rows : total;
  int64_t r;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (r = 0; r < n; ++r) {
    int64_t flat = rows ? rows[r] : r;
    int64_t bi = flat / h_q; /* (b, i) */
    const int32_t* idx = indices + (size_t)bi * topk;
    const uint16_t* qr = q + (size_t)flat * ORACLE_D;
    double qv[ORACLE_D];
    int32_t* slots = (int32_t*)malloc(sizeof(int32_t) * (size_t)(topk > 0 ? topk : 1));
    fp8_ctx ctx;
    int j, d, cnt = 0;
    for (d = 0; d < ORACLE_D; ++d) qv[d] = bf16_bits_to_f64(qr[d]);
    for (j = 0; j < topk; ++j) {
      int32_t s = idx[j];
      if (s < 0) continue;
      if ((int64_t)s >= num_slots) {
        bad = 1;
        continue;
      }
      slots[cnt++] = s;
    }
    ctx.cache = cache;
    ctx.slots = slots;
    attend_rows(qv, fetch_fp8, &ctx, cnt, d_v, scale, out + (size_t)r * d_v, lse + r);
    free(slots);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------- V4.1 FP8 cache (528 B) */

/* E8M0: an 8-bit biased exponent with no sign and no mantissa. */
double oracle_e8m0_decode(uint8_t e) {
  if (e == 0xFF) return NAN;
  return ldexp(1.0, (int)e - 127);
}

/* Decode one 528-byte row: [512 e4m3 codes][16 e8m0 scales, one per 32]. */
void oracle_decode_row528(const uint8_t* row, double* out) {
  int d;
  for (d = 0; d < ORACLE_D41; ++d)
    out[d] = oracle_e4m3_decode(row[d]) * oracle_e8m0_decode(row[ORACLE_D41 + d / 32]);
}

static void fetch_row528(const void* vctx, int j, double* out) {
  const fp8_ctx* c = (const fp8_ctx*)vctx;
  oracle_decode_row528(c->cache + (size_t)c->slots[j] * ORACLE_ROW528, out);
  round_row_bf16(out, ORACLE_D41);
}

/* E2M1 (a 4-bit code): sign, 2 exponent bits with bias 1, 1 mantissa bit;
 * exponent 0 holds the subnormals 0 and 0.5.  No inf or NaN. */
double oracle_e2m1_decode(uint8_t c) {
  int sign = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
  double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return sign ? -mag : mag;
}

/* Decode one 288-byte row: [256 bytes of E2M1 pairs][32 e4m3 scales, one per
 * 16 codes]. */
void oracle_decode_row288(const uint8_t* row, double* out) {
  int d;
  for (d = 0; d < ORACLE_D41; ++d) {
    uint8_t byte = row[d / 2];
    uint8_t code = (d % 2 == 0) ? (uint8_t)(byte & 0x0F) : (uint8_t)(byte >> 4);
    out[d] = oracle_e2m1_decode(code) * oracle_e4m3_decode(row[ORACLE_D41 / 2 + d / 16]);
  }
}

static void fetch_row288(const void* vctx, int j, double* out) {
  const fp8_ctx* c = (const fp8_ctx*)vctx;
  oracle_decode_row288(c->cache + (size_t)c->slots[j] * ORACLE_ROW288, out);
  round_row_bf16(out, ORACLE_D41);
}

/* Token-level sparse decode over a 512-dim V4.1 cache of `row_bytes`-byte
 * rows decoded by `fetch`.
 *  q        [b, s_q, h_q, 512] bf16 bits
 *  cache    [num_slots, row_bytes] (slot = block*64 + offset)
 *  indices  [b, s_q, topk] int32 physical slots, -1 = invalid (skipped)
 *  out      [rows, 512]: V is the whole 512-dim latent.  No causal mask. */
static int sparse_decode_512(row_fetch_fn fetch, const uint16_t* q, const uint8_t* cache,
                             int64_t num_slots, const int32_t* indices, int batch, int s_q,
                             int h_q, int topk, double scale, const int64_t* rows, int64_t n_rows,
                             double* out, double* lse) {
  int64_t total = (int64_t)batch * s_q * h_q;
  int64_t n = rows ? n_rows : total;
  int64_t r;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (r = 0; r < n; ++r) {
    int64_t flat = rows ? rows[r] : r;
    int64_t bi = flat / h_q; /* (b, i) */
    const int32_t* idx = indices + (size_t)bi * topk;
    const uint16_t* qr = q + (size_t)flat * ORACLE_D41;
    double qv[ORACLE_D41];
    int32_t* slots = (int32_t*)malloc(sizeof(int32_t) * (size_t)(topk > 0 ? topk : 1));
    fp8_ctx ctx;
    int j, d, cnt = 0;
    for (d = 0; d < ORACLE_D41; ++d) qv[d] = bf16_bits_to_f64(qr[d]);
    for (j = 0; j < topk; ++j) {
      int32_t s = idx[j];
      if (s < 0) continue;
      if ((int64_t)s >= num_slots) {
        bad = 1;
        continue;
      }
      slots[cnt++] = s;
    }
    ctx.cache = cache;
    ctx.slots = slots;
    attend_rows_d(qv, ORACLE_D41, fetch, &ctx, cnt, ORACLE_D41, scale,
                  out + (size_t)r * ORACLE_D41, lse + r);
    free(slots);
  }
  return bad ? -1 : 0;
}

/* Sparse decode over the 528-byte V4.1 FP8 rows. */
int oracle_sparse_decode_v41(const uint16_t* q, const uint8_t* cache, int64_t num_slots,
                             const int32_t* indices, int batch, int s_q, int h_q, int topk,
                             double scale, const int64_t* rows, int64_t n_rows, double* out,
                             double* lse) {
  return sparse_decode_512(fetch_row528, q, cache, num_slots, indices, batch, s_q, h_q, topk,
                           scale, rows, n_rows, out, lse);
}

/* Sparse decode over the 288-byte V4.1 FP4 rows. */
int oracle_sparse_decode_v41_fp4(const uint16_t* q, const uint8_t* cache, int64_t num_slots,
                                 const int32_t* indices, int batch, int s_q, int h_q, int topk,
                                 double scale, const int64_t* rows, int64_t n_rows, double* out,
                                 double* lse) {
  return sparse_decode_512(fetch_row288, q, cache, num_slots, indices, batch, s_q, h_q, topk,
                           scale, rows, n_rows, out, lse);
}

/* Fused decode in sparse mode: the fused steps of oracle_fused_decode over
 * the valid slots of indices [b, 1, topk] in the 656-byte FP8 cache (decoded
 * to 576 dims; V is the whole row, d_v = 576).  positions [b] is required:
 * the selected tokens say nothing about the query's own position. */
int oracle_fused_sparse_decode(const uint16_t* q_raw, const double* gain, double eps,
                               double rope_base, const int32_t* positions, const uint8_t* cache,
                               int64_t num_slots, const int32_t* indices, int batch, int h_q,
                               int topk, double scale, const int64_t* rows, int64_t n_rows,
                               uint8_t* codes, double* out_scale, double* lse) {
  int64_t total = (int64_t)batch * h_q;
  int64_t n = rows ? n_rows : total;
  int64_t r;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (r = 0; r < n; ++r) {
    int64_t flat = rows ? rows[r] : r;
    int b = (int)(flat / h_q);
    const int32_t* idx = indices + (size_t)b * topk;
    int32_t* slots = (int32_t*)malloc(sizeof(int32_t) * (size_t)(topk > 0 ? topk : 1));
    fp8_ctx ctx;
    int j, cnt = 0;
    for (j = 0; j < topk; ++j) {
      int32_t s = idx[j];
      if (s < 0) continue;
      if ((int64_t)s >= num_slots) {
        bad = 1;
        continue;
      }
      slots[cnt++] = s;
    }
    ctx.cache = cache;
    ctx.slots = slots;
    fused_row(q_raw + (size_t)flat * ORACLE_D, gain, eps, rope_base, (double)positions[b],
              fetch_fp8, &ctx, cnt, scale, codes + (size_t)r * ORACLE_D, out_scale + r, lse + r,
              0);
    free(slots);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------- sparse prefill */

/* bf16 latent rows [s_kv, 576] addressed by a list of row indices. */
typedef struct {
  const uint16_t* kv;
  const int32_t* slots;
} kv_rows_ctx;

static void fetch_kv_row(const void* vctx, int j, double* out) {
  const kv_rows_ctx* c = (const kv_rows_ctx*)vctx;
  const uint16_t* row = c->kv + (size_t)c->slots[j] * ORACLE_D;
  int d;
  for (d = 0; d < ORACLE_D; ++d) out[d] = bf16_bits_to_f64(row[d]);
}

/* Token-level sparse prefill (no batch dimension).
 *  q            [s_q, h_q, 576] bf16 bits
 *  kv           [s_kv, 576] bf16 bits (one latent KV head)
 *  indices      [s_q, topk] int32 rows of kv, -1 = invalid
 *  topk_length  [s_q] or NULL: only indices[t][0 .. topk_length[t]) count
 *  attn_sink    [h_q] or NULL: a per-head logit that joins the softmax
 *               normaliser without a value row
 *  out [rows, d_v], lse [rows] (rows of (t, h), or the sampled `rows`). */
int oracle_sparse_prefill(const uint16_t* q, const uint16_t* kv, int64_t s_kv,
                          const int32_t* indices, const int32_t* topk_length,
                          const double* attn_sink, int s_q, int h_q, int topk, int d_v,
                          double scale, const int64_t* rows, int64_t n_rows, double* out,
                          double* lse) {
  int64_t total = (int64_t)s_q * h_q;
  int64_t n = rows ? n_rows : total;
  int64_t r;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (r = 0; r < n; ++r) {
    int64_t flat = rows ? rows[r] : r;
    int t = (int)(flat / h_q), h = (int)(flat % h_q);
    const int32_t* idx = indices + (size_t)t * topk;
    int len = topk_length ? topk_length[t] : topk;
    const uint16_t* qr = q + (size_t)flat * ORACLE_D;
    double qv[ORACLE_D];
    int32_t* slots = (int32_t*)malloc(sizeof(int32_t) * (size_t)(topk > 0 ? topk : 1));
    kv_rows_ctx ctx;
    int j, d, cnt = 0;
    if (len > topk) len = topk;
    for (d = 0; d < ORACLE_D; ++d) qv[d] = bf16_bits_to_f64(qr[d]);
    for (j = 0; j < len; ++j) {
      int32_t s = idx[j];
      if (s < 0) continue;
      if ((int64_t)s >= s_kv) {
        bad = 1;
        continue;
      }
      slots[cnt++] = s;
    }
    ctx.kv = kv;
    ctx.slots = slots;
    attend_rows_ds(qv, ORACLE_D, fetch_kv_row, &ctx, cnt, d_v, scale,
                   attn_sink ? attn_sink[h] : -INFINITY, out + (size_t)r * d_v, lse + r);
    free(slots);
  }
  return bad ? -1 : 0;
}
