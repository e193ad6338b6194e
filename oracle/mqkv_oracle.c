/*
 * mqkv_oracle.c — plain CPU oracle for the chunk-adaptive mixed-bitwidth KV
 * cache path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load this library.  It is slow on
 * purpose: plain loops in the order the method is stated, fp64 for reference
 * values, IEEE fp32 exactly where the method fixes fp32 decisions.  It shares
 * no code, header, table or constant with the CUDA library; the byte formats
 * it writes are re-derived here from the prose of the public header.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math (never fast-math;
 * x86-64 evaluates float in SSE single precision, FLT_EVAL_METHOD == 0).
 *
 * Sources of each step:
 *  - Router, argmax, vote: MoQAE paper notes, 方法详解 › 整体框架 (chunks are
 *    routed; per-token choice; majority vote inside a chunk) and
 *    关键设计 › Quantization-Aware Experts (router maps a chunk C with D
 *    features to per-token expert scores through W1, W2, W3; experts are the
 *    FP16/INT4/INT2 quantisation settings).  The printed form f(CW1·CW2)W3 is
 *    garbled; it is read here as (SiLU(C W1) ⊙ (C W2)) W3 + b3.
 *  - Routing freezing: same notes, 路由冻结 (first chunk kept at FP16).
 *  - Routing sharing: same notes, 路由共享 (one decision reused by all layers);
 *    here that means one map per sequence, reused by the caller.
 *  - Regrouping by precision before quantisation: Cocktail abstract on the
 *    "Bin Zhang" scholarfeed author page (chunk-level KV cache computation).
 *  - Quantiser: the pages leave it open; asymmetric min-max per token over
 *    groups of 32 along head_dim, fp32, round half to even, fp16 scale/min.
 *  - Attention: same MoQAE notes, 整体框架 (ordinary attention after
 *    quantisation); single query, softmax scale 1/sqrt(d) by default.
 *
 * Pins: every function here is checked by the CPU tests against closed forms,
 * special cases, invariants and brute force (see tests/test_oracle_pins.py).
 * The router's decisions on real data are "parity unpinned" beyond those
 * special cases: no trained router exists to compare with.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define NEXP 3
#define GROUP 32

/* ------------------------------------------------------------------ fp16 */

static float half_bits_to_float(uint16_t h) {
  _Float16 v;
  memcpy(&v, &h, 2);
  return (float)v; /* exact widening */
}

static uint16_t float_to_half_bits(float f) {
  _Float16 v = (_Float16)f; /* IEEE round to nearest even */
  uint16_t h;
  memcpy(&h, &v, 2);
  return h;
}

int mqo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void mqo_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Element e of a [rows, cols] array stored as fp32 (dtype 0) or fp16 (1). */
static float load_elem(const void* base, int dtype, int64_t e) {
  if (dtype == 0) return ((const float*)base)[e];
  return half_bits_to_float(((const uint16_t*)base)[e]);
}

void mqo_f32_to_f16(const float* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = float_to_half_bits(in[i]);
}

void mqo_f16_to_f32(const uint16_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = half_bits_to_float(in[i]);
}

/* ---------------------------------------------------------------- router */

/*
 * Router scores for T tokens: z_t = (SiLU(C_t W1) ⊙ (C_t W2)) W3 + b3.
 * Every product and sum is taken in fp64 from the fp32 inputs; the result is
 * rounded to fp32 once (logits32) and also kept in fp64 (logits64).
 * C [T, D], W1/W2 [D, H], W3 [H, 3] row-major; b3 may be NULL (zero).
 */
void mqo_router_logits(int64_t T, int D, int H, const float* C, const float* W1,
                       const float* W2, const float* W3, const float* b3,
                       float* logits32, double* logits64) {
#pragma omp parallel
  {
    double* h1 = (double*)malloc(sizeof(double) * (size_t)H);
    double* h2 = (double*)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      const float* c = C + t * (int64_t)D;
      for (int j = 0; j < H; ++j) { h1[j] = 0.0; h2[j] = 0.0; }
      for (int k = 0; k < D; ++k) {
        const double ck = (double)c[k];
        const float* w1 = W1 + (int64_t)k * H;
        const float* w2 = W2 + (int64_t)k * H;
        for (int j = 0; j < H; ++j) {
          h1[j] += ck * (double)w1[j];
          h2[j] += ck * (double)w2[j];
        }
      }
      double z[NEXP];
      for (int e = 0; e < NEXP; ++e) z[e] = b3 ? (double)b3[e] : 0.0;
      for (int j = 0; j < H; ++j) {
        const double silu = h1[j] / (1.0 + exp(-h1[j]));
        const double g = silu * h2[j];
        for (int e = 0; e < NEXP; ++e) z[e] += g * (double)W3[(int64_t)j * NEXP + e];
      }
      for (int e = 0; e < NEXP; ++e) {
        if (logits64) logits64[t * NEXP + e] = z[e];
        if (logits32) logits32[t * NEXP + e] = (float)z[e];
      }
    }
    free(h1);
    free(h2);
  }
}

/* Index of the largest of three fp32 scores; an exact tie keeps the lower
 * index (= more bits). */
static int argmax3_f32(const float* z) {
  int best = 0;
  for (int e = 1; e < NEXP; ++e)
    if (z[e] > z[best]) best = e;
  return best;
}

void mqo_token_argmax(int64_t T, const float* logits32, uint8_t* token_expert) {
  for (int64_t t = 0; t < T; ++t) token_expert[t] = (uint8_t)argmax3_f32(logits32 + t * NEXP);
}

/* Difference between the largest and second-largest fp64 score of each token
 * (0 for an exact tie).  Used to exempt near-ties from map comparisons. */
void mqo_top2_gap(int64_t T, const double* logits64, double* gap) {
  for (int64_t t = 0; t < T; ++t) {
    const double* z = logits64 + t * NEXP;
    double a = z[0], b = -INFINITY;
    for (int e = 1; e < NEXP; ++e) {
      if (z[e] > a) { b = a; a = z[e]; }
      else if (z[e] > b) b = z[e];
    }
    gap[t] = a - b;
  }
}

int64_t mqo_num_chunks(int B, const int32_t* seq_lens, int L) {
  int64_t n = 0;
  for (int b = 0; b < B; ++b) n += (seq_lens[b] + L - 1) / L;
  return n;
}

/*
 * Majority vote per chunk over its tokens' choices; a count tie keeps the
 * lower index (more bits).  The tail chunk of a sequence votes over the tokens
 * it has.  With routing_freeze, chunk 0 of every sequence becomes FP16.
 * token_expert is indexed by token row (sequences back to back).
 */
void mqo_vote(int B, const int32_t* seq_lens, int L, const uint8_t* token_expert,
              int routing_freeze, uint8_t* chunk_expert) {
  int64_t row = 0, ci = 0;
  for (int b = 0; b < B; ++b) {
    const int Tb = seq_lens[b];
    const int nb = (Tb + L - 1) / L;
    for (int c = 0; c < nb; ++c) {
      int count[NEXP] = {0, 0, 0};
      const int t0 = c * L;
      const int t1 = (t0 + L < Tb) ? t0 + L : Tb;
      for (int t = t0; t < t1; ++t) count[token_expert[row + t]]++;
      int win = 0;
      for (int e = 1; e < NEXP; ++e)
        if (count[e] > count[win]) win = e;
      if (routing_freeze && c == 0) win = 0;
      chunk_expert[ci + c] = (uint8_t)win;
    }
    row += Tb;
    ci += nb;
  }
}

/* The whole routing step (scores, per-token argmax, vote, freezing). */
void mqo_route(int B, const int32_t* seq_lens, int L, int D, int H, const float* C,
               const float* W1, const float* W2, const float* W3, const float* b3,
               int routing_freeze, uint8_t* token_expert, uint8_t* chunk_expert,
               float* logits32, double* logits64) {
  int64_t T = 0;
  for (int b = 0; b < B; ++b) T += seq_lens[b];
  mqo_router_logits(T, D, H, C, W1, W2, W3, b3, logits32, logits64);
  mqo_token_argmax(T, logits32, token_expert);
  mqo_vote(B, seq_lens, L, token_expert, routing_freeze, chunk_expert);
}

/* -------------------------------------------------- similarity search */

/*
 * Chunk-level quantization search by similarity (Cocktail abstract on the
 * "Bin Zhang" scholarfeed author page: the bitwidth of each context chunk is
 * chosen from the similarity between the chunk and the query).  The page
 * gives neither the similarity nor the thresholds; the reading used here:
 *   sim(b, c) = cos(mean of C_t over the chunk's tokens, u_b)   (fp64)
 *   expert = FP16 if sim >= tau_hi, INT4 if sim >= tau_lo, else INT2;
 *   a zero vector gives sim = 0; with routing_freeze, chunk 0 is FP16.
 * C [T, D] fp32 (sequences back to back), u [B, D] fp32.
 */
void mqo_similarity_route(int B, const int32_t* seq_lens, int L, int D, const float* C,
                          const float* u, double tau_hi, double tau_lo, int routing_freeze,
                          uint8_t* chunk_expert, double* sim_out) {
  int64_t row = 0, ci = 0;
  double* mean = (double*)malloc(sizeof(double) * (size_t)D);
  for (int b = 0; b < B; ++b) {
    const int Tb = seq_lens[b];
    const int nb = (Tb + L - 1) / L;
    double unorm = 0.0;
    for (int k = 0; k < D; ++k) unorm += (double)u[(int64_t)b * D + k] * u[(int64_t)b * D + k];
    for (int c = 0; c < nb; ++c) {
      const int t0 = c * L, t1 = (t0 + L < Tb) ? t0 + L : Tb;
      for (int k = 0; k < D; ++k) mean[k] = 0.0;
      for (int t = t0; t < t1; ++t)
        for (int k = 0; k < D; ++k) mean[k] += (double)C[(row + t) * (int64_t)D + k];
      double dot = 0.0, mnorm = 0.0;
      for (int k = 0; k < D; ++k) {
        mean[k] /= (double)(t1 - t0);
        dot += mean[k] * (double)u[(int64_t)b * D + k];
        mnorm += mean[k] * mean[k];
      }
      const double sim = (mnorm > 0.0 && unorm > 0.0) ? dot / sqrt(mnorm * unorm) : 0.0;
      int e = sim >= tau_hi ? 0 : (sim >= tau_lo ? 1 : 2);
      if (routing_freeze && c == 0) e = 0;
      chunk_expert[ci + c] = (uint8_t)e;
      if (sim_out) sim_out[ci + c] = sim;
    }
    row += Tb;
    ci += nb;
  }
  free(mean);
}

/* --------------------------------------------------------------- layout */

/* Layout table as the public header describes it, rebuilt here from prose. */
#define LAYOUT_MAGIC 0x4C4B514Du
#define HEADER_BYTES 64
#define SEQ_BYTES 160

static uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

static const int kBits[NEXP] = {16, 4, 2};

/* Bytes of one row of codes (one token, one kv-head) at bitwidth bits. */
static uint64_t code_row_bytes(int d, int bits) { return (uint64_t)d * (uint64_t)bits / 8; }

/* Region size and scale offset of n tokens at expert e. */
static void region_geometry(int d, int e, int64_t n, uint64_t* region, uint64_t* scale_off) {
  if (e == 0) {
    *scale_off = 0;
    *region = align_up((uint64_t)n * code_row_bytes(d, 16), 128);
  } else {
    *scale_off = align_up((uint64_t)n * code_row_bytes(d, kBits[e]), 128);
    *region = *scale_off + align_up((uint64_t)n * (uint64_t)(d / GROUP) * 4u, 128);
  }
}

typedef struct {
  int64_t token_offset;
  int32_t num_tokens, num_chunks, chunk_offset;
  int32_t seg_chunks[NEXP], seg_chunk_begin[NEXP], seg_tokens[NEXP];
  uint64_t seg_base[NEXP], region_bytes[NEXP], scale_offset[NEXP];
} seq_info;

/* Per-sequence segment bookkeeping for a chunk map (stable by chunk index). */
static void describe_seq(int d, int Hkv, int L, int Tb, const uint8_t* map, int32_t* perm,
                         int32_t* inv, seq_info* si) {
  const int nb = (Tb + L - 1) / L;
  (void)Hkv;
  si->num_tokens = Tb;
  si->num_chunks = nb;
  int pos = 0;
  for (int e = 0; e < NEXP; ++e) {
    si->seg_chunk_begin[e] = pos;
    int nch = 0, ntok = 0;
    for (int c = 0; c < nb; ++c) {
      if (map[c] != e) continue;
      perm[pos] = c;
      inv[c] = pos;
      ++pos;
      ++nch;
      ntok += (c == nb - 1) ? Tb - c * L : L;
    }
    si->seg_chunks[e] = nch;
    si->seg_tokens[e] = ntok;
    region_geometry(d, e, ntok, &si->region_bytes[e], &si->scale_offset[e]);
  }
}

size_t mqo_layout_bytes(int B, const int32_t* seq_lens, int L) {
  const int64_t N = mqo_num_chunks(B, seq_lens, L);
  return HEADER_BYTES + (size_t)B * SEQ_BYTES + 2 * (size_t)align_up((uint64_t)N * 4, 16);
}

static void put32(uint8_t* p, int32_t v) { memcpy(p, &v, 4); }
static void putu32(uint8_t* p, uint32_t v) { memcpy(p, &v, 4); }
static void put64(uint8_t* p, int64_t v) { memcpy(p, &v, 8); }
static void putu64(uint8_t* p, uint64_t v) { memcpy(p, &v, 8); }

/*
 * Builds the layout table for a chunk map.  Schedule fields (work items) are
 * written as zero: they are implementation-defined and not part of the method.
 * Returns the packed size of one layer, or 0 if blob_bytes is too small.
 */
uint64_t mqo_build_layout(int B, int Hkv, int d, int L, const int32_t* seq_lens,
                          const uint8_t* chunk_expert, uint8_t* blob, size_t blob_bytes) {
  const int64_t N = mqo_num_chunks(B, seq_lens, L);
  if (blob_bytes < mqo_layout_bytes(B, seq_lens, L)) return 0;
  memset(blob, 0, mqo_layout_bytes(B, seq_lens, L));
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
  int32_t* inv = (int32_t*)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
  uint64_t base = 0;
  int64_t row = 0, coff = 0;
  uint8_t* seqs = blob + HEADER_BYTES;
  for (int b = 0; b < B; ++b) {
    seq_info si;
    memset(&si, 0, sizeof si);
    describe_seq(d, Hkv, L, seq_lens[b], chunk_expert + coff, perm + coff, inv + coff, &si);
    si.token_offset = row;
    si.chunk_offset = (int32_t)coff;
    uint8_t* r = seqs + (size_t)b * SEQ_BYTES;
    put64(r + 0, si.token_offset);
    put32(r + 8, si.num_tokens);
    put32(r + 12, si.num_chunks);
    put32(r + 16, si.chunk_offset);
    for (int e = 0; e < NEXP; ++e) {
      put32(r + 20 + 4 * e, si.seg_chunks[e]);
      put32(r + 32 + 4 * e, si.seg_chunk_begin[e]);
      put32(r + 44 + 4 * e, si.seg_tokens[e]);
      putu64(r + 56 + 8 * e, base);
      putu64(r + 80 + 8 * e, si.region_bytes[e]);
      putu64(r + 104 + 8 * e, si.scale_offset[e]);
      base += 2 * (uint64_t)Hkv * si.region_bytes[e];
    }
    row += seq_lens[b];
    coff += si.num_chunks;
  }
  putu32(blob + 0, LAYOUT_MAGIC);
  putu32(blob + 4, 1u);
  put32(blob + 8, B);
  put32(blob + 12, Hkv);
  put32(blob + 16, d);
  put32(blob + 20, L);
  put32(blob + 24, (int32_t)N);
  put32(blob + 28, 0); /* schedule */
  put64(blob + 32, row);
  putu64(blob + 40, base);
  uint8_t* pperm = blob + HEADER_BYTES + (size_t)B * SEQ_BYTES;
  uint8_t* pinv = pperm + align_up((uint64_t)N * 4, 16);
  if (N > 0) {
    memcpy(pperm, perm, (size_t)N * 4);
    memcpy(pinv, inv, (size_t)N * 4);
  }
  free(perm);
  free(inv);
  return base;
}

/* Packed size of one layer for a chunk map (no table written). */
uint64_t mqo_packed_bytes(int B, int Hkv, int d, int L, const int32_t* seq_lens,
                          const uint8_t* chunk_expert) {
  uint64_t total = 0;
  int64_t coff = 0;
  for (int b = 0; b < B; ++b) {
    const int Tb = seq_lens[b], nb = (Tb + L - 1) / L;
    for (int e = 0; e < NEXP; ++e) {
      int64_t ntok = 0;
      for (int c = 0; c < nb; ++c)
        if (chunk_expert[coff + c] == e) ntok += (c == nb - 1) ? Tb - c * L : L;
      uint64_t region, soff;
      region_geometry(d, e, ntok, &region, &soff);
      total += 2 * (uint64_t)Hkv * region;
    }
    coff += nb;
  }
  return total;
}

/* ------------------------------------------------------------- quantiser */

/*
 * One group of 32 values (fp32) at `bits` in {4, 2}:
 *   mn, mx = min, max;  s = (mx - mn) / (2^bits - 1)  (s = 1 if mx == mn)
 *   code_j = clamp(rint((x_j - mn) / s), 0, 2^bits - 1)
 * in IEEE fp32 with round-half-even rint; returns fp32 s and mn and their
 * fp16 (round to nearest even) bit patterns.
 */
void mqo_quantize_group(const float* x, int bits, uint8_t* codes, float* s_out, float* mn_out,
                        uint16_t* s_half, uint16_t* mn_half) {
  float mn = x[0], mx = x[0];
  for (int j = 1; j < GROUP; ++j) {
    if (x[j] < mn) mn = x[j];
    if (x[j] > mx) mx = x[j];
  }
  const float levels = (float)((1 << bits) - 1);
  float s = (mx - mn) / levels;
  if (mx == mn) s = 1.0f;
  for (int j = 0; j < GROUP; ++j) {
    const float t = x[j] - mn;
    float q = rintf(t / s);
    if (q < 0.0f) q = 0.0f;
    if (q > levels) q = levels;
    codes[j] = (uint8_t)q;
  }
  if (s_out) *s_out = s;
  if (mn_out) *mn_out = mn;
  if (s_half) *s_half = float_to_half_bits(s);
  if (mn_half) *mn_half = float_to_half_bits(mn);
}

/* Writes 32 codes of `bits` bits LSB-first into 4*bits bytes. */
void mqo_pack_codes(const uint8_t* codes, int bits, uint8_t* out) {
  const int per_word = 32 / bits;
  for (int w = 0; w < bits; ++w) {
    uint32_t word = 0;
    for (int i = 0; i < per_word; ++i) word |= (uint32_t)codes[w * per_word + i] << (bits * i);
    memcpy(out + 4 * w, &word, 4);
  }
}

void mqo_unpack_codes(const uint8_t* in, int bits, uint8_t* codes) {
  const int per_word = 32 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  for (int w = 0; w < bits; ++w) {
    uint32_t word;
    memcpy(&word, in + 4 * w, 4);
    for (int i = 0; i < per_word; ++i) codes[w * per_word + i] = (uint8_t)((word >> (bits * i)) & mask);
  }
}

/* Encodes one row (one token, one kv-head: d values) at expert e into a code
 * row and, for INT experts, a scale row of d/32 (scale, min) fp16 pairs. */
static void encode_row(const void* src, int dtype, int64_t elem0, int d, int e, uint8_t* code_row,
                       uint8_t* scale_row) {
  if (e == 0) {
    uint16_t* out = (uint16_t*)code_row;
    for (int j = 0; j < d; ++j) {
      if (dtype == 1)
        out[j] = ((const uint16_t*)src)[elem0 + j];
      else
        out[j] = float_to_half_bits(((const float*)src)[elem0 + j]);
    }
    return;
  }
  const int bits = kBits[e];
  for (int k = 0; k < d / GROUP; ++k) {
    float x[GROUP];
    uint8_t codes[GROUP];
    uint16_t sh, mh;
    for (int j = 0; j < GROUP; ++j) x[j] = load_elem(src, dtype, elem0 + k * GROUP + j);
    mqo_quantize_group(x, bits, codes, NULL, NULL, &sh, &mh);
    mqo_pack_codes(codes, bits, code_row + (size_t)k * 4 * bits);
    memcpy(scale_row + 4 * k, &sh, 2);
    memcpy(scale_row + 4 * k + 2, &mh, 2);
  }
}

/*
 * Packs one layer.  K, V are [T, Hkv, d] (dtype 0 = fp32, 1 = fp16); the
 * packed buffer follows the public format.  Returns 0 on success, 1 if
 * packed_bytes is too small.  Padding bytes are left as they were.
 */
int mqo_pack(int B, int Hkv, int d, int L, const int32_t* seq_lens, const uint8_t* chunk_expert,
             const void* K, const void* V, int dtype, uint8_t* packed, uint64_t packed_bytes) {
  if (packed_bytes < mqo_packed_bytes(B, Hkv, d, L, seq_lens, chunk_expert)) return 1;
  const int64_t N = mqo_num_chunks(B, seq_lens, L);
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
  int32_t* inv = (int32_t*)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
  seq_info* si = (seq_info*)calloc((size_t)B, sizeof(seq_info));
  uint64_t base = 0;
  int64_t row = 0, coff = 0;
  for (int b = 0; b < B; ++b) {
    describe_seq(d, Hkv, L, seq_lens[b], chunk_expert + coff, perm + coff, inv + coff, &si[b]);
    si[b].token_offset = row;
    si[b].chunk_offset = (int32_t)coff;
    for (int e = 0; e < NEXP; ++e) {
      si[b].seg_base[e] = base;
      base += 2 * (uint64_t)Hkv * si[b].region_bytes[e];
    }
    row += seq_lens[b];
    coff += si[b].num_chunks;
  }
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t ci = 0; ci < N; ++ci) {
    int b = 0;
    while (ci >= (int64_t)si[b].chunk_offset + si[b].num_chunks) ++b;
    const seq_info* s = &si[b];
    const int c = (int)(ci - s->chunk_offset);
    const int e = chunk_expert[ci];
    const int p = inv[ci];
    const int t0 = c * L;
    const int nt = (c == s->num_chunks - 1) ? s->num_tokens - t0 : L;
    const int64_t seg_row0 = (int64_t)(p - s->seg_chunk_begin[e]) * L;
    const uint64_t rb = code_row_bytes(d, kBits[e]);
    for (int kv = 0; kv < 2; ++kv) {
      const void* src = kv == 0 ? K : V;
      for (int g = 0; g < Hkv; ++g) {
        uint8_t* region = packed + s->seg_base[e] + ((uint64_t)kv * Hkv + g) * s->region_bytes[e];
        for (int t = 0; t < nt; ++t) {
          const int64_t tok = s->token_offset + t0 + t;
          const int64_t segrow = seg_row0 + t;
          encode_row(src, dtype, (tok * Hkv + g) * d, d, e, region + segrow * rb,
                     region + s->scale_offset[e] + segrow * (uint64_t)(d / GROUP) * 4u);
        }
      }
    }
  }
  free(perm);
  free(inv);
  free(si);
  return 0;
}

/* ------------------------------------------------------------- attention */

/* Dequantised row (fp64) of token row `segrow` of a region at expert e. */
static void decode_row(const uint8_t* region, uint64_t scale_off, int d, int e, int64_t segrow,
                       double* out) {
  if (e == 0) {
    const uint16_t* h = (const uint16_t*)(region + segrow * code_row_bytes(d, 16));
    for (int j = 0; j < d; ++j) out[j] = (double)half_bits_to_float(h[j]);
    return;
  }
  const int bits = kBits[e];
  const uint8_t* code_row = region + segrow * code_row_bytes(d, bits);
  const uint8_t* scale_row = region + scale_off + segrow * (uint64_t)(d / GROUP) * 4u;
  for (int k = 0; k < d / GROUP; ++k) {
    uint8_t codes[GROUP];
    uint16_t sh, mh;
    mqo_unpack_codes(code_row + (size_t)k * 4 * bits, bits, codes);
    memcpy(&sh, scale_row + 4 * k, 2);
    memcpy(&mh, scale_row + 4 * k + 2, 2);
    const double s = (double)half_bits_to_float(sh), m = (double)half_bits_to_float(mh);
    for (int j = 0; j < GROUP; ++j) out[k * GROUP + j] = (double)codes[j] * s + m;
  }
}

/*
 * Single-query attention over n tokens in fp64, as defined:
 *   score_t = scale * <q, k_t>,  o = sum_t exp(score_t - max) v_t / sum_t exp(score_t - max)
 * K, V are n rows of d doubles.  n == 0 gives zeros.
 */
static void attend_ml(int n, int d, const double* q, const double* Kd, const double* Vd,
                      double scale, double* o, double* ml) {
  for (int j = 0; j < d; ++j) o[j] = 0.0;
  if (ml) {
    ml[0] = -INFINITY;
    ml[1] = 0.0;
  }
  if (n == 0) return;
  double* sc = (double*)malloc(sizeof(double) * (size_t)n);
  double mx = -INFINITY;
  for (int t = 0; t < n; ++t) {
    double acc = 0.0;
    for (int j = 0; j < d; ++j) acc += q[j] * Kd[(int64_t)t * d + j];
    sc[t] = scale * acc;
    if (sc[t] > mx) mx = sc[t];
  }
  double den = 0.0;
  for (int t = 0; t < n; ++t) {
    const double p = exp(sc[t] - mx);
    den += p;
    for (int j = 0; j < d; ++j) o[j] += p * Vd[(int64_t)t * d + j];
  }
  for (int j = 0; j < d; ++j) o[j] /= den;
  if (ml) {
    ml[0] = mx;   /* largest scaled score */
    ml[1] = den;  /* sum of exp(score - mx) */
  }
  free(sc);
}

static void attend(int n, int d, const double* q, const double* Kd, const double* Vd, double scale,
                   double* o) {
  attend_ml(n, d, q, Kd, Vd, scale, o, 0);
}

/*
 * Decode attention over a packed layer (this oracle's own packing of the same
 * map): for every (b, h), tokens are visited in ORIGINAL order; kv-head
 * g = h / (Hq/Hkv).  q is [B, Hq, d] (dtype 0 fp32, 1 fp16); scale <= 0 means
 * 1/sqrt(d).  out is [B, Hq, d] fp64.
 */
static void decode_impl(int B, int Hq, int Hkv, int d, int L, const int32_t* seq_lens,
                        const uint8_t* chunk_expert, const uint8_t* packed, const void* q,
                        int q_dtype, double scale, double* out, double* ml) {
  if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
  const int64_t N = mqo_num_chunks(B, seq_lens, L);
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
  int32_t* inv = (int32_t*)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
  seq_info* si = (seq_info*)calloc((size_t)B, sizeof(seq_info));
  uint64_t base = 0;
  int64_t coff = 0;
  for (int b = 0; b < B; ++b) {
    describe_seq(d, Hkv, L, seq_lens[b], chunk_expert + coff, perm + coff, inv + coff, &si[b]);
    si[b].chunk_offset = (int32_t)coff;
    for (int e = 0; e < NEXP; ++e) {
      si[b].seg_base[e] = base;
      base += 2 * (uint64_t)Hkv * si[b].region_bytes[e];
    }
    coff += si[b].num_chunks;
  }
  const int qpg = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
    const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / qpg;
    const seq_info* s = &si[b];
    const int Tb = s->num_tokens;
    double* Kd = (double*)malloc(sizeof(double) * (size_t)(Tb > 0 ? Tb : 1) * d);
    double* Vd = (double*)malloc(sizeof(double) * (size_t)(Tb > 0 ? Tb : 1) * d);
    double qd[128];
    for (int j = 0; j < d; ++j) qd[j] = (double)load_elem(q, q_dtype, bh * d + j);
    for (int t = 0; t < Tb; ++t) {
      const int c = t / L;
      const int64_t ci = s->chunk_offset + c;
      const int e = chunk_expert[ci];
      const int64_t segrow = (int64_t)(inv[ci] - s->seg_chunk_begin[e]) * L + (t - c * L);
      const uint8_t* rk = packed + s->seg_base[e] + (uint64_t)g * s->region_bytes[e];
      const uint8_t* rv = packed + s->seg_base[e] + (uint64_t)(Hkv + g) * s->region_bytes[e];
      decode_row(rk, s->scale_offset[e], d, e, segrow, Kd + (int64_t)t * d);
      decode_row(rv, s->scale_offset[e], d, e, segrow, Vd + (int64_t)t * d);
    }
    attend_ml(Tb, d, qd, Kd, Vd, scale, out + bh * d, ml ? ml + 2 * bh : 0);
    free(Kd);
    free(Vd);
  }
  free(perm);
  free(inv);
  free(si);
}

void mqo_decode(int B, int Hq, int Hkv, int d, int L, const int32_t* seq_lens,
                const uint8_t* chunk_expert, const uint8_t* packed, const void* q, int q_dtype,
                double scale, double* out) {
  decode_impl(B, Hq, Hkv, d, L, seq_lens, chunk_expert, packed, q, q_dtype, scale, out, 0);
}

/*
 * The same attention, also returning for every (b, h) the largest scaled
 * score m and l = sum_t exp(score_t - m) (ml is [B, Hq, 2] fp64; an empty
 * sequence gives m = -inf, l = 0).  These are what a device holding only part
 * of a sequence's context contributes to the merge of a split softmax.
 */
void mqo_decode_partial(int B, int Hq, int Hkv, int d, int L, const int32_t* seq_lens,
                        const uint8_t* chunk_expert, const uint8_t* packed, const void* q,
                        int q_dtype, double scale, double* out, double* ml) {
  decode_impl(B, Hq, Hkv, d, L, seq_lens, chunk_expert, packed, q, q_dtype, scale, out, ml);
}

/*
 * Decode attention for selected (b, h) pairs straight from the raw K/V and the
 * map: each token is quantised and dequantised on the spot with the same
 * quantiser (no packed buffer).  pairs holds n_pairs (b, h) int32 pairs;
 * out is [n_pairs, d] fp64.  Used to check outputs sampled from large runs.
 */
void mqo_decode_pairs(int B, int Hq, int Hkv, int d, int L, const int32_t* seq_lens,
                      const uint8_t* chunk_expert, const void* K, const void* V, int kv_dtype,
                      const void* q, int q_dtype, double scale, const int32_t* pairs,
                      int n_pairs, double* out) {
  if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
  int64_t* row0 = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  int64_t* coff = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  row0[0] = 0;
  coff[0] = 0;
  for (int b = 0; b < B; ++b) {
    row0[b + 1] = row0[b] + seq_lens[b];
    coff[b + 1] = coff[b] + (seq_lens[b] + L - 1) / L;
  }
  const int qpg = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n_pairs; ++i) {
    const int b = pairs[2 * i], h = pairs[2 * i + 1], g = h / qpg;
    const int Tb = seq_lens[b];
    double* Kd = (double*)malloc(sizeof(double) * (size_t)(Tb > 0 ? Tb : 1) * d);
    double* Vd = (double*)malloc(sizeof(double) * (size_t)(Tb > 0 ? Tb : 1) * d);
    /* one encoded row: codes at [0, 256), scales at [256, 272) */
    uint8_t rowbuf[256 + 16];
    double qd[128];
    for (int j = 0; j < d; ++j) qd[j] = (double)load_elem(q, q_dtype, ((int64_t)b * Hq + h) * d + j);
    for (int t = 0; t < Tb; ++t) {
      const int e = chunk_expert[coff[b] + t / L];
      const int64_t elem0 = ((row0[b] + t) * Hkv + g) * d;
      encode_row(K, kv_dtype, elem0, d, e, rowbuf, rowbuf + 256);
      decode_row(rowbuf, 256, d, e, 0, Kd + (int64_t)t * d);
      encode_row(V, kv_dtype, elem0, d, e, rowbuf, rowbuf + 256);
      decode_row(rowbuf, 256, d, e, 0, Vd + (int64_t)t * d);
    }
    attend(Tb, d, qd, Kd, Vd, scale, out + (int64_t)i * d);
    free(Kd);
    free(Vd);
  }
  free(row0);
  free(coff);
}

/*
 * Dense single-query attention on the raw K/V (no quantisation), fp64.
 * Same argument conventions as mqo_decode; used for the all-FP16 check.
 */
void mqo_dense_attention(int B, int Hq, int Hkv, int d, const int32_t* seq_lens, const void* K,
                         const void* V, int kv_dtype, const void* q, int q_dtype, double scale,
                         double* out) {
  if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
  int64_t* row0 = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
  row0[0] = 0;
  for (int b = 0; b < B; ++b) row0[b + 1] = row0[b] + seq_lens[b];
  const int qpg = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
    const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / qpg;
    const int Tb = seq_lens[b];
    double* Kd = (double*)malloc(sizeof(double) * (size_t)(Tb > 0 ? Tb : 1) * d);
    double* Vd = (double*)malloc(sizeof(double) * (size_t)(Tb > 0 ? Tb : 1) * d);
    double qd[128];
    for (int j = 0; j < d; ++j) qd[j] = (double)load_elem(q, q_dtype, bh * d + j);
    for (int t = 0; t < Tb; ++t)
      for (int j = 0; j < d; ++j) {
        const int64_t e0 = ((row0[b] + t) * Hkv + g) * d + j;
        Kd[(int64_t)t * d + j] = (double)load_elem(K, kv_dtype, e0);
        Vd[(int64_t)t * d + j] = (double)load_elem(V, kv_dtype, e0);
      }
    attend(Tb, d, qd, Kd, Vd, scale, out + bh * d);
    free(Kd);
    free(Vd);
  }
  free(row0);
}
