// decode.cu — single-query decode attention straight from the mixed-bitwidth
// packed cache.
//
// MoQAE paper notes, 方法详解 › 整体框架: after quantisation the model runs
// ordinary attention over the cache; here one query per (sequence, query
// head) attends over all cached tokens of its sequence:
//   o = sum_t softmax_t(scale * q . khat_t) vhat_t,
//   khat, vhat = code * (half)s + (half)min   (or the stored fp16 value).
// Cocktail abstract (chunk-level KV cache computation): because chunks were
// regrouped by precision, every stretch of work below reads one precision
// only — no per-token branching between bitwidths.
//
// decode_partial_kernel — every warp is an independent persistent worker
// that takes work items from an atomic counter, one at a time (items differ
// in cost with their precision, so a static split leaves SMs idle).  A work
// item is
// (sequence b, segment s, kv-head g, token range of at most item_tokens[s]
// tokens).  The warp streams the item's four byte ranges (K codes, V codes, K
// scales, V scales) through its own 4-stage cp.async ring in shared memory,
// one tile of TPW tokens per stage, every lane copying 16-byte units so each
// instruction reads whole sectors.  Per tile:
//   lanes: LPT lanes cover one token (SL dims each), TPW tokens per tile; the
//          lane keeps its SL query values of all Hq/Hkv heads in registers
//   scores: q . code on the raw codes (one mask per code, see code_bits),
//          dequantisation folded in per
//          group: q . khat = s * (q . code) + min * sum(q); shuffle-reduced
//          over the token's LPT lanes
//   softmax: online, log2 domain, with a lazily moved reference maximum
//   values: acc += (p * s) * code per value pair and bias += p * min per head
//   end of item: the TPW token lanes are merged with shuffles and (m, l,
//          acc[d]) of every head goes to the workspace.
// decode_combine_kernel — one warp per (b, query head) merges the partials of
// all items of (b, g) with the usual max-rescaling.
#include "decode_ptx.cuh"

namespace mqkv {
namespace {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kRing = 4;  // stages of each warp's copy ring
constexpr float kRescale = 8.0f;

// Lane geometry of one precision: each lane owns SL consecutive dims of one
// token (SL * QPG query values and accumulators stay in registers), LPT lanes
// cover a token, TPW tokens are processed per warp iteration.
template <int D, int QPG, int E>
struct Geo {
  static constexpr int BITS = E == 0 ? 16 : (E == 1 ? 4 : 2);
  static constexpr int SL_INT = 32 / QPG;
  static constexpr int SL = E == 0 ? (SL_INT < 16 ? SL_INT : 16) : SL_INT;
  static constexpr int LPT = D / SL;
  static constexpr int TPW = 32 / LPT;
  static constexpr int PIECE = SL * BITS / 8;   // code bytes of one lane's slice
  static constexpr int CROW = D * BITS / 8;     // code bytes of one token row
  static constexpr int SROW = E == 0 ? 0 : D / kGroup * 4;
  static constexpr int CODES = TPW * CROW;      // code bytes of one iteration (K or V)
  static constexpr int SCALES = E == 0 ? 0 : (TPW * SROW + 15) / 16 * 16;
  static constexpr int STAGE = 2 * CODES + 2 * SCALES;
};

template <int D, int QPG>
constexpr int stage_bytes() {
  constexpr int a = Geo<D, QPG, 0>::STAGE, b = Geo<D, QPG, 1>::STAGE, c = Geo<D, QPG, 2>::STAGE;
  constexpr int m = a > b ? a : b;
  return (m > c ? m : c + 0) + 0;
}

template <int D, int QPG>
constexpr size_t decode_smem_bytes() {
  return (size_t)kDecWarps * kRing * stage_bytes<D, QPG>();
}

// Code extraction by masking in place.  A 32-bit pattern below 2^24, read as
// an fp32 number, is exactly pattern * 2^-149 (a subnormal, or exponent field
// 1 where the spacing is the same), so masking one code of a packed word
// leaves the float c * 2^(o - 149), o the code's bit offset; codes at offsets
// 24 and up are first moved down one byte (offset o - 8).  The f32x2 FMAs
// take subnormal operands without flushing (no .ftz), and the factor that
// multiplies a code carries the compensating power of two:
//   scores: query pre-scaled by 2^(kQExp - o), product q c 2^(kQExp - 149)
//   values: weight scaled by 2^kWExp; the accumulator of position o holds
//           sum p s c 2^(kWExp - 149 + o) and is rescaled at the end.
// A code has at most 4 significant bits and an fp16 query 11, so each score
// product is exact in fp32 (above the subnormal range, |q| >= 2^-41), and no
// offset is subtracted afterwards.  Bounds: |q| < 2^64 keeps the scaled
// query finite; weights stay below 2^8 (lazy rescaling) and s below 2^16, so
// the scaled weight stays below 2^124.
constexpr int kQExp = 64;
constexpr int kWExp = 100;

__device__ __forceinline__ constexpr float pow2f(int e) {
  float r = 1.0f;
  for (int i = 0; i < e; ++i) r *= 2.0f;
  for (int i = 0; i > e; --i) r *= 0.5f;
  return r;
}

// Bit offset of code v of a lane's slice after code_bits.
template <int BITS>
__device__ __forceinline__ constexpr int code_off(int v) {
  return (v * BITS) % 32 + BITS <= 24 ? (v * BITS) % 32 : (v * BITS) % 32 - 8;
}

// Code v of a lane's slice (words LSB-first), in place: c << code_off(v).
template <int BITS>
__device__ __forceinline__ uint32_t code_bits(const uint32_t* words, int v) {
  constexpr uint32_t m = (1u << BITS) - 1u;
  const uint32_t w = words[(v * BITS) / 32];
  const int o = (v * BITS) % 32;
  return o + BITS <= 24 ? (w & (m << o)) : ((w >> 8) & (m << (o - 8)));
}

// One lane's copy units of one iteration: 16-byte pieces of the iteration's
// token tile (K codes | V codes | K scales | V scales), located once per item.
template <int STAGE>
struct CopyPlan {
  static constexpr int U = (STAGE / 16 + 31) / 32;
  const unsigned char* src[U];  // source at iteration 0
  uint32_t step[U];             // source advance per iteration
  uint16_t dst[U];              // offset inside a stage
  int16_t row[U];               // first token row (inside the tile) the unit reads
  bool used[U];
};

template <typename Gm, int STAGE>
__device__ __forceinline__ void plan_copies(CopyPlan<STAGE>& cp, const unsigned char* regk,
                                            const unsigned char* regv, uint64_t soff, int64_t t0) {
  const int lane = threadIdx.x & 31;
  constexpr int CB = Gm::CODES, SB = Gm::SCALES;
  constexpr int UNITS = (2 * CB + 2 * SB) / 16;
#pragma unroll
  for (int i = 0; i < CopyPlan<STAGE>::U; ++i) {
    const int u = lane + 32 * i;
    cp.used[i] = u < UNITS;
    int off = u * 16;
    if (off < CB) {
      cp.src[i] = regk + t0 * Gm::CROW + off;
      cp.step[i] = Gm::TPW * Gm::CROW;
      cp.dst[i] = off;
      cp.row[i] = off / Gm::CROW;
    } else if ((off -= CB) < CB) {
      cp.src[i] = regv + t0 * Gm::CROW + off;
      cp.step[i] = Gm::TPW * Gm::CROW;
      cp.dst[i] = CB + off;
      cp.row[i] = off / Gm::CROW;
    } else if ((off -= CB) < SB) {
      cp.src[i] = regk + soff + t0 * Gm::SROW + off;
      cp.step[i] = Gm::TPW * Gm::SROW;
      cp.dst[i] = 2 * CB + off;
      cp.row[i] = off / (Gm::SROW > 0 ? Gm::SROW : 1);
    } else {
      off -= SB;
      cp.src[i] = regv + soff + t0 * Gm::SROW + off;
      cp.step[i] = Gm::TPW * Gm::SROW;
      cp.dst[i] = 2 * CB + SB + off;
      cp.row[i] = off / (Gm::SROW > 0 ? Gm::SROW : 1);
    }
  }
}

template <int D, int QPG, int QDT, int E>
__device__ __forceinline__ void run_item(const unsigned char* __restrict__ regk,
                                         const unsigned char* __restrict__ regv, uint64_t soff,
                                         int t0, int n, const void* __restrict__ q, int64_t qbase,
                                         float scale_log2, unsigned char* ring, int64_t w,
                                         float* __restrict__ ws_acc, float2* __restrict__ ws_ml) {
  using Gm = Geo<D, QPG, E>;
  constexpr int SL = Gm::SL, LPT = Gm::LPT, TPW = Gm::TPW;
  constexpr int STRIDE = stage_bytes<D, QPG>();
  constexpr int BITS = Gm::BITS;
  constexpr int NP = SL / 2;  // value pairs per lane
  const int lane = threadIdx.x & 31;
  const int tl = lane / LPT, sl = lane % LPT;
  const int iters = (n + TPW - 1) / TPW;

  CopyPlan<Gm::STAGE> cp;  // this precision's units (the ring stride fits the largest)
  plan_copies<Gm, Gm::STAGE>(cp, regk, regv, soff, t0);
  auto issue = [&](int it) {
    if (it < iters) {
      const int nv = min(TPW, n - it * TPW);
      unsigned char* st = ring + (it % kRing) * STRIDE;
#pragma unroll
      for (int i = 0; i < CopyPlan<Gm::STAGE>::U; ++i)
        if (cp.used[i] && cp.row[i] < nv)
          cp_async16(st + cp.dst[i], cp.src[i] + (uint64_t)it * cp.step[i]);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int it = 0; it < kRing - 1; ++it) issue(it);

  // ---- query slice of every head, in value pairs, pre-scaled per code position
  uint64_t qp[QPG][NP];
  float qs[QPG];
#pragma unroll
  for (int h = 0; h < QPG; ++h) {
    const int64_t base = qbase + (int64_t)h * D + sl * SL;
    qs[h] = 0.f;
#pragma unroll
    for (int j = 0; j < SL; j += 2) {
      float a, b;
      if constexpr (QDT == MQ_F16) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(static_cast<const __half*>(q) + base + j));
        a = f.x;
        b = f.y;
      } else {
        const float2 f = *reinterpret_cast<const float2*>(static_cast<const float*>(q) + base + j);
        a = f.x;
        b = f.y;
      }
      qs[h] += a + b;
      if constexpr (E != 0) {
        a *= pow2f(kQExp - code_off<BITS>(j));
        b *= pow2f(kQExp - code_off<BITS>(j + 1));
      }
      qp[h][j / 2] = pk2(a, b);
    }
  }

  uint64_t acc[QPG][NP];
  float bias[QPG], m[QPG], m8[QPG], l[QPG];  // m8 = m + kRescale
#pragma unroll
  for (int h = 0; h < QPG; ++h) {
    bias[h] = 0.f;
    m[h] = -INFINITY;
    m8[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j) acc[h][j] = 0ull;
  }
  const int grp = (sl * SL) / kGroup;

  for (int it = 0; it < iters; ++it) {
    issue(it + kRing - 1);
    cp_async_wait<kRing - 1>();
    __syncwarp();
    const unsigned char* st = ring + (it % kRing) * STRIDE;
    const bool valid = it * TPW + tl < n;
    const unsigned char* kp = st + tl * Gm::CROW + sl * Gm::PIECE;
    const unsigned char* vp = st + Gm::CODES + tl * Gm::CROW + sl * Gm::PIECE;
    float ks = 1.f, km = 0.f, vs = 1.f, vm = 0.f;
    if constexpr (E != 0) {
      const float2 a = half2_bits_to_float2(
          *reinterpret_cast<const uint32_t*>(st + 2 * Gm::CODES + tl * Gm::SROW + grp * 4));
      const float2 b = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(
          st + 2 * Gm::CODES + Gm::SCALES + tl * Gm::SROW + grp * 4));
      ks = a.x * pow2f(149 - kQExp); km = a.y; vs = b.x * pow2f(kWExp); vm = b.y;
    }
    // ---- scores: q . code (pairs) in kChains independent accumulator chains
    // (short dependency chains), then the group's scale and min
    // (with several query heads per kv-head the heads already give independent
    // chains)
    constexpr int kChains = QPG > 1 ? 1 : (NP >= 4 ? 4 : NP);
    uint64_t dot2[QPG][kChains];
#pragma unroll
    for (int h = 0; h < QPG; ++h)
#pragma unroll
      for (int c = 0; c < kChains; ++c) dot2[h][c] = 0ull;
    if constexpr (E == 0) {
      const uint32_t* wv = reinterpret_cast<const uint32_t*>(kp);
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const float2 f = half2_bits_to_float2(wv[i]);
        const uint64_t x = pk2(f.x, f.y);
#pragma unroll
        for (int h = 0; h < QPG; ++h) dot2[h][i % kChains] = fma2(x, qp[h][i], dot2[h][i % kChains]);
      }
    } else {
      constexpr int BYTES = SL * BITS / 8;
      uint32_t words[(BYTES + 3) / 4];
      if constexpr (BYTES >= 4) {
#pragma unroll
        for (int k = 0; k < BYTES / 4; ++k) words[k] = reinterpret_cast<const uint32_t*>(kp)[k];
      } else {
        words[0] = BYTES == 2 ? *reinterpret_cast<const unsigned short*>(kp) : *kp;
      }
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const uint64_t x = pk2u(code_bits<BITS>(words, 2 * i), code_bits<BITS>(words, 2 * i + 1));
#pragma unroll
        for (int h = 0; h < QPG; ++h) dot2[h][i % kChains] = fma2(x, qp[h][i], dot2[h][i % kChains]);
      }
    }
    float part[QPG];
#pragma unroll
    for (int h = 0; h < QPG; ++h) {
      uint64_t d2 = dot2[h][0];
      if constexpr (kChains == 4) {
        d2 = add2(add2(dot2[h][0], dot2[h][1]), add2(dot2[h][2], dot2[h][3]));
      } else {
#pragma unroll
        for (int c = 1; c < kChains; ++c) d2 = add2(d2, dot2[h][c]);
      }
      const float dot = lo2(d2) + hi2(d2);
      part[h] = E == 0 ? dot : fmaf(ks, dot, km * qs[h]);
    }
#pragma unroll
    for (int off = 1; off < LPT; off <<= 1)
#pragma unroll
      for (int h = 0; h < QPG; ++h) part[h] += __shfl_xor_sync(0xffffffffu, part[h], off);
    float p[QPG];
#pragma unroll
    for (int h = 0; h < QPG; ++h) {
      const float sc = valid ? part[h] * scale_log2 : -INFINITY;
      // lazy rescaling: the reference maximum moves only when a score exceeds
      // it by more than kRescale (log2 units), so weights stay below
      // 2^kRescale; (m, l, acc) remain consistent for any reference
      // (m8 is kept only with one query head per kv-head: with several, the
      // registers are better spent elsewhere)
      if (sc > (QPG == 1 ? m8[h] : m[h] + kRescale)) {
        const float a = ex2_ftz(m[h] - sc);
        const uint64_t a2 = pk2(a, a);
        l[h] *= a;
        bias[h] *= a;
#pragma unroll
        for (int j = 0; j < NP; ++j) acc[h][j] = fma2(acc[h][j], a2, 0ull);
        m[h] = sc;
        if constexpr (QPG == 1) m8[h] = sc + kRescale;
      }
      p[h] = valid ? ex2_ftz(sc - m[h]) : 0.f;
      l[h] += p[h];
    }
    // ---- values.  Lanes past the item's last token hold stale stage bytes:
    // their fp16 values and scales may be NaN, so FP16 tiles skip the
    // accumulation and quantised tiles zero the weight by a select (masked
    // codes are always finite, so they then add exactly 0).
    if (E != 0 || valid) {
      uint64_t w2[QPG];
#pragma unroll
      for (int h = 0; h < QPG; ++h) {
        const float wgt = E == 0 ? p[h] : (valid ? p[h] * vs : 0.f);
        w2[h] = pk2(wgt, wgt);
        if constexpr (E != 0) bias[h] = valid ? fmaf(p[h], vm, bias[h]) : bias[h];
      }
      if constexpr (E == 0) {
        const uint32_t* wv = reinterpret_cast<const uint32_t*>(vp);
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          const float2 f = half2_bits_to_float2(wv[i]);
          const uint64_t x = pk2(f.x, f.y);
#pragma unroll
          for (int h = 0; h < QPG; ++h) acc[h][i] = fma2(x, w2[h], acc[h][i]);
        }
      } else {
        constexpr int BYTES = SL * BITS / 8;
        uint32_t words[(BYTES + 3) / 4];
        if constexpr (BYTES >= 4) {
#pragma unroll
          for (int k = 0; k < BYTES / 4; ++k) words[k] = reinterpret_cast<const uint32_t*>(vp)[k];
        } else {
          words[0] = BYTES == 2 ? *reinterpret_cast<const unsigned short*>(vp) : *vp;
        }
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          const uint64_t x = pk2u(code_bits<BITS>(words, 2 * i), code_bits<BITS>(words, 2 * i + 1));
#pragma unroll
          for (int h = 0; h < QPG; ++h) acc[h][i] = fma2(x, w2[h], acc[h][i]);
        }
      }
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();

  // ---- undo the per-position code scaling, then merge the TPW token lanes
  float av[QPG][SL];
#pragma unroll
  for (int h = 0; h < QPG; ++h)
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      av[h][2 * j] = lo2(acc[h][j]) * (E == 0 ? 1.f : pow2f(149 - kWExp - code_off<BITS>(2 * j)));
      av[h][2 * j + 1] =
          hi2(acc[h][j]) * (E == 0 ? 1.f : pow2f(149 - kWExp - code_off<BITS>(2 * j + 1)));
    }
  if constexpr (QPG == 1) {
    // One query head: merge through the warp's ring, idle now (every copy has
    // landed and been read).  Each lane stores its slice (SL dims) with its
    // token lane's (m, l, bias); then lane i combines dims DPL i.. over the
    // TPW token lanes of their slice.
    constexpr int ROW = SL + 4;  // floats per lane: av[SL], m, l, bias, pad
    constexpr int DPL = D / 32;  // output dims per lane
    float* smf = reinterpret_cast<float*>(ring);
    float* row = smf + lane * ROW;
#pragma unroll
    for (int j = 0; j < SL; j += 4)
      *reinterpret_cast<float4*>(row + j) = make_float4(av[0][j], av[0][j + 1], av[0][j + 2], av[0][j + 3]);
    *reinterpret_cast<float4*>(row + SL) = make_float4(m[0], l[0], bias[0], 0.f);
    __syncwarp();
    const int d0 = lane * DPL;
    const int sld = d0 / SL, o = d0 % SL;
    float M = -INFINITY;
#pragma unroll
    for (int t = 0; t < TPW; ++t) M = fmaxf(M, smf[(t * LPT + sld) * ROW + SL]);
    float L = 0.f, Bs = 0.f, ad[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) ad[i] = 0.f;
#pragma unroll
    for (int t = 0; t < TPW; ++t) {
      const float* src = smf + (t * LPT + sld) * ROW;
      const float4 mlb = *reinterpret_cast<const float4*>(src + SL);
      const float a = mlb.x == -INFINITY ? 0.f : ex2_ftz(mlb.x - M);
      L = fmaf(a, mlb.y, L);
      Bs = fmaf(a, mlb.z, Bs);
      if constexpr (DPL == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src + o);
        ad[0] = fmaf(a, v.x, ad[0]);
        ad[1] = fmaf(a, v.y, ad[1]);
        ad[2] = fmaf(a, v.z, ad[2]);
        ad[3] = fmaf(a, v.w, ad[3]);
      } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) ad[i] = fmaf(a, src[o + i], ad[i]);
      }
    }
    float* dst = ws_acc + (size_t)w * D + d0;
#pragma unroll
    for (int i = 0; i < DPL; ++i) dst[i] = ad[i] + Bs;
    if (lane == 0) ws_ml[w] = make_float2(M, L);
  } else {
#pragma unroll
  for (int off = LPT; off < 32; off <<= 1) {
#pragma unroll
    for (int h = 0; h < QPG; ++h) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
      const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
      const float bo = __shfl_xor_sync(0xffffffffu, bias[h], off);
      const float M = fmaxf(m[h], mo);
      const float a = m[h] == -INFINITY ? 0.f : exp2f(m[h] - M);
      const float b = mo == -INFINITY ? 0.f : exp2f(mo - M);
      l[h] = l[h] * a + lo * b;
      bias[h] = bias[h] * a + bo * b;
#pragma unroll
      for (int j = 0; j < SL; ++j) {
        const float ao = __shfl_xor_sync(0xffffffffu, av[h][j], off);
        av[h][j] = av[h][j] * a + ao * b;
      }
      m[h] = M;
    }
  }
  if (tl == 0) {
#pragma unroll
    for (int h = 0; h < QPG; ++h) {
      float* dst = ws_acc + ((size_t)w * QPG + h) * D + sl * SL;
#pragma unroll
      for (int j = 0; j < SL; j += 4)
        *reinterpret_cast<float4*>(dst + j) =
            make_float4(av[h][j] + bias[h], av[h][j + 1] + bias[h], av[h][j + 2] + bias[h],
                        av[h][j + 3] + bias[h]);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < QPG; ++h) ws_ml[(size_t)w * QPG + h] = make_float2(m[h], l[h]);
  }
  }
  __syncwarp();  // (one query head: the ring is read before the next item's copies refill it)
}


// Each warp is an independent worker: it takes the next work item from a
// counter in the workspace whenever it finishes one, and streams each item
// through its own copy ring.  No block-wide barrier is used.
template <int D, int QPG, int QDT>
__global__ void __launch_bounds__(kDecThreads, 2)
decode_partial_kernel(const unsigned char* __restrict__ layout,
                      const unsigned char* __restrict__ packed, const void* __restrict__ q,
                      float scale_log2, float* __restrict__ ws_acc, float2* __restrict__ ws_ml,
                      unsigned int* __restrict__ counter, int64_t capacity_items,
                      unsigned int* status) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  if (h->magic != MQ_LAYOUT_MAGIC || h->head_dim != D) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_BAD_LAYOUT);
    return;
  }
  const int B = h->num_seqs, Hkv = h->num_kv_heads;
  const int64_t total = (int64_t)h->total_items * Hkv;
  if (total > capacity_items) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_WORKSPACE_TOO_SMALL);
    return;
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  unsigned char* ring = smem_raw + (size_t)warp * kRing * stage_bytes<D, QPG>();
  // dynamic assignment: a warp takes the next item when it is done with one,
  // so items of different cost even out across the SMs
  for (;;) {
    unsigned int wi = 0;
    if (lane == 0) wi = atomicAdd(counter, 1u);
    const int64_t w = (int64_t)__shfl_sync(0xffffffffu, wi, 0);
    if (w >= total) break;
    const int64_t bs = w / Hkv;
    const int g = (int)(w - bs * Hkv);
    const int b = find_item_seq(layout, B, bs);
    const mq_seq_layout* r = reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(b));
    const int s = bs < r->item_begin[1] ? 0 : (bs < r->item_begin[2] ? 1 : 2);
    const int j = (int)(bs - r->item_begin[s]);
    const int t0 = j * h->item_tokens[s];
    const int n = min(h->item_tokens[s], r->seg_tokens[s] - t0);
    if (n <= 0) {
      if ((threadIdx.x & 31) == 0) set_status(status, MQ_DEV_INDEX_RANGE);
      continue;
    }
    const unsigned char* regk = packed + r->seg_base[s] + (uint64_t)g * r->region_bytes[s];
    const unsigned char* regv = regk + (uint64_t)Hkv * r->region_bytes[s];
    const int64_t qbase = ((int64_t)b * Hkv + g) * QPG * D;
    if (s == 0)
      run_item<D, QPG, QDT, 0>(regk, regv, 0, t0, n, q, qbase, scale_log2, ring, w, ws_acc, ws_ml);
    else if (s == 1)
      run_item<D, QPG, QDT, 1>(regk, regv, r->scale_offset[1], t0, n, q, qbase, scale_log2, ring, w,
                               ws_acc, ws_ml);
    else
      run_item<D, QPG, QDT, 2>(regk, regv, r->scale_offset[2], t0, n, q, qbase, scale_log2, ring, w,
                               ws_acc, ws_ml);
  }
}

// One CTA per (sequence, query head): 8 warps split the items, each keeps a
// running (max, sum, accumulator) over its items, then the warps' states are
// merged in shared memory.
// PARTIAL: instead of the attention output, write the record of a context
// shard: [o (D values, normalised), m, l, 0, 0] with m the reference score of
// the merged softmax (natural-log units, within 8 ln 2 below the largest
// score) and l = sum exp(score - m) (mq_decode_attn_partial).
// Long sequences are split: gridDim.y = S CTAs per (b, h) each merge a fixed
// slice of the items into a split record [num (D values), M, L] in `split`;
// the CTA that finishes last (a counter per (b, h) in `done`, zero on entry
// and left at zero) merges the S records in slice order and writes the
// output, so the result does not depend on the CTAs' timing.
template <int D, int QPG, bool PARTIAL, int NW>
__global__ void __launch_bounds__(32 * NW)
decode_combine_kernel(const unsigned char* __restrict__ layout, int Hq,
                      const float* __restrict__ ws_acc, const float2* __restrict__ ws_ml,
                      float* __restrict__ out, float* __restrict__ split,
                      unsigned int* __restrict__ done) {
  constexpr int PER_LANE = D / 32;
  __shared__ float s_acc[NW][D];
  __shared__ float s_m[NW], s_l[NW];
  __shared__ int s_last;
  const int S = gridDim.y, k = blockIdx.y;
  pdl_wait();  // the partial records of the decode kernel
  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  const int Hkv = h->num_kv_heads;
  const int64_t bh = blockIdx.x;
  const int b = (int)(bh / Hq), hq = (int)(bh % Hq);
  const int g = hq / QPG, hh = hq % QPG;
  const int lane = threadIdx.x & 31, warp = threadIdx.x / 32;
  const mq_seq_layout* r = reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(b));
  const int n_items = r->item_begin[2] + r->item_count[2] - r->item_begin[0];
  const int i0 = r->item_begin[0] + (int)((int64_t)n_items * k / S);
  const int i1 = r->item_begin[0] + (int)((int64_t)n_items * (k + 1) / S);
  float M = -INFINITY, l = 0.f, acc[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) acc[i] = 0.f;
  // kU items per round, all loaded before any is merged (independent loads
  // in flight instead of one dependent load at a time)
  constexpr int kU = 8;
  for (int it0 = i0 + warp; it0 < i1; it0 += NW * kU) {
    float2 ml[kU];
    float v[kU][PER_LANE];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int it = it0 + u * NW;
      ml[u] = make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i) v[u][i] = 0.f;
      if (it < i1) {
        const int64_t wi = ((int64_t)it * Hkv + g) * QPG + hh;
        ml[u] = ws_ml[wi];
        const float* a = ws_acc + wi * D + lane * PER_LANE;
        if constexpr (PER_LANE == 4) {
          const float4 t = *reinterpret_cast<const float4*>(a);
          v[u][0] = t.x; v[u][1] = t.y; v[u][2] = t.z; v[u][3] = t.w;
        } else {
          const float2 t = *reinterpret_cast<const float2*>(a);
          v[u][0] = t.x; v[u][1] = t.y;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (ml[u].x == -INFINITY) continue;  // past the end, or an item with no tokens
      const float Mn = fmaxf(M, ml[u].x);
      const float fa = M == -INFINITY ? 0.f : exp2f(M - Mn);
      const float fb = exp2f(ml[u].x - Mn);
      l = l * fa + ml[u].y * fb;
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i) acc[i] = acc[i] * fa + v[u][i] * fb;
      M = Mn;
    }
  }
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) s_acc[warp][lane * PER_LANE + i] = acc[i];
  if (lane == 0) {
    s_m[warp] = M;
    s_l[warp] = l;
  }
  __syncthreads();
  float Mx = -INFINITY, num = 0.f, den = 0.f;
  if (threadIdx.x < D) {
#pragma unroll
    for (int w = 0; w < NW; ++w) Mx = fmaxf(Mx, s_m[w]);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = s_m[w] == -INFINITY ? 0.f : exp2f(s_m[w] - Mx);
      num += f * s_acc[w][threadIdx.x];
      den += f * s_l[w];
    }
  }
  if (S > 1) {
    // this slice's record, then the last slice's CTA merges all of them
    float* rec = split + ((size_t)bh * S + k) * (D + 2);
    if (threadIdx.x < D) rec[threadIdx.x] = num;
    if (threadIdx.x == 0) {
      rec[D] = Mx;
      rec[D + 1] = den;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(done + bh, 1u) == (unsigned int)(S - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) done[bh] = 0u;  // ready for the next call
    Mx = -INFINITY;
    num = den = 0.f;
    if (threadIdx.x < D) {
      const volatile float* base = split + (size_t)bh * S * (D + 2);
      for (int j = 0; j < S; ++j) Mx = fmaxf(Mx, base[j * (D + 2) + D]);
      for (int j = 0; j < S; ++j) {
        const float mj = base[j * (D + 2) + D];
        const float f = mj == -INFINITY ? 0.f : exp2f(mj - Mx);
        num += f * base[j * (D + 2) + threadIdx.x];
        den += f * base[j * (D + 2) + D + 1];
      }
    }
  }
  if (threadIdx.x < D) {
    if constexpr (PARTIAL) {
      float* rec = out + bh * (D + 4);
      rec[threadIdx.x] = den > 0.f ? num / den : 0.f;
      if (threadIdx.x == 0) {
        rec[D] = den > 0.f ? Mx * 0.6931471805599453f : -INFINITY;  // log2 -> natural units
        rec[D + 1] = den;
        rec[D + 2] = 0.f;
        rec[D + 3] = 0.f;
      }
    } else {
      out[bh * D + threadIdx.x] = den > 0.f ? num / den : 0.f;
    }
  }
}

// Merge of P context-shard records per (sequence, query head):
//   M = max_r m_r,  w_r = l_r exp(m_r - M),  o = sum_r w_r o_r / sum_r w_r
// (0 when every shard is empty).  One CTA per (b, h), one thread per value.
__global__ void __launch_bounds__(128)
combine_partials_kernel(int P, int64_t heads, int D, const float* __restrict__ parts,
                        float* __restrict__ out) {
  const int64_t bh = blockIdx.x;
  const int i = threadIdx.x;
  if (i >= D) return;  // no barrier below
  const size_t rec = (size_t)D + 4;
  float M = -INFINITY;
  for (int r = 0; r < P; ++r) {
    const float* p = parts + ((size_t)r * heads + bh) * rec;
    if (p[D + 1] > 0.f) M = fmaxf(M, p[D]);
  }
  float num = 0.f, den = 0.f;
  for (int r = 0; r < P; ++r) {
    const float* p = parts + ((size_t)r * heads + bh) * rec;
    const float l = p[D + 1];
    if (l > 0.f) {
      const float w = l * expf(p[D] - M);
      num = fmaf(w, p[i], num);
      den += w;
    }
  }
  out[bh * D + i] = den > 0.f ? num / den : 0.f;
}

// ============================================================================
// Tensor-core decode for several query heads per kv-head (fp16 queries).
//
// With Hq/Hkv = QPG > 1 the CUDA-core kernel above spreads one token over
// 32/(32/QPG) lanes and repeats the per-token softmax work on each of them.
// Here a warp takes 16 tokens at a time and lets mma.sync (m16n8k16, fp16
// operands, fp32 accumulation) form both products:
//   scores  S[16 tokens x 8 head slots] = Khat . Q^T, one accumulator per group
//           of 32 dims (the group's scale and min are applied afterwards:
//           q . khat = s (q . code) + min sum(q));
//   values  O^T[16 dims x 8 head slots] += Vhat^T . P', P' = p * s_v per group,
//           P' split into fp16 high and low parts (two MMAs) so that the
//           products keep fp32-level accuracy, O held in units of a power
//           of two raised with the largest scale seen so P' fits fp16; the
//           mins enter as sum_t p_t min_t per group.
// INT4 codes enter in place as fp16 c * 2^-24 (one shift and one mask per
// pair, see nib_sub); INT2 codes become exact fp16 integers (one
// byte-permute, one mask and one fma per pair).  The dims of a k-step are
// permuted identically in K and Q so that each lane reads whole bytes:
// k = 2t, 2t+1, 2t+8, 2t+9 of k-step (group g, half hh) are dims
// 32g + 8t + 2hh + {0, 4, 1, 5} for INT4 and 32g + 8t + 4hh + {0, 1, 2, 3}
// for INT2 (t = lane % 4).  V codes are expanded into a padded fp16 tile
// (INT4 dims in nib_dim order inside each 8) and fed to the MMA with
// ldmatrix.trans; FP16 segments feed K and V straight from the staged rows.
// ============================================================================
constexpr int kMmaWarps = 1;            // one worker warp per CTA: 12 resident per SM
constexpr int kMmaThreads = 32 * kMmaWarps;
constexpr int kMmaTile = 16;            // tokens per tile
constexpr int kMmaRing = 17408;         // shared bytes of one warp: 2 FP16 tiles at d=128, or
                                        // the quantised tiles' ring plus the V expansion tile
constexpr int kRowPad = 16;             // bytes added to every staged code row

template <int D, int E>
struct MG {
  static constexpr int BITS = E == 0 ? 16 : (E == 1 ? 4 : 2);
  static constexpr int CROW = D * BITS / 8;                 // code bytes of a token row
  static constexpr int KROW = CROW + kRowPad;               // staged row pitch
  static constexpr int SROW = E == 0 ? 0 : D / kGroup * 4;  // (scale, min) bytes of a row
  static constexpr int KOFF = 0;
  static constexpr int VOFF = kMmaTile * KROW;
  static constexpr int KSOFF = 2 * kMmaTile * KROW;
  static constexpr int VSOFF = KSOFF + kMmaTile * SROW;
  static constexpr int STAGE = (VSOFF + kMmaTile * SROW + 15) / 16 * 16;
  // quantised tiles leave the end of the warp's space to the V expansion tile
  static constexpr int RING = E == 0 ? kMmaRing : kMmaRing - kMmaTile * (128 + 8) * 2;
  static constexpr int STAGES = RING / STAGE < 8 ? RING / STAGE : 8;
  static constexpr int CU = CROW / 16;                      // 16-byte units per code row
};
static_assert(MG<128, 0>::STAGES >= 2 && MG<64, 0>::STAGES >= 2 && MG<128, 1>::STAGES >= 3 &&
                  MG<128, 2>::STAGES >= 3,
              "ring too small");

constexpr int kVbufRow = 128 + 8;       // fp16 elements of one expanded V row (padded)
constexpr int kVbufBytes = kMmaTile * kVbufRow * 2;

template <int D>
constexpr size_t mma_smem_bytes() {
  return (size_t)kMmaWarps * kMmaRing;
}

// byte j of w as [b, 0x64, b, 0x64]: two fp16 values 1024 + (low bits of b)
__device__ __forceinline__ uint32_t spread2(uint32_t w, int j) {
  return __byte_perm(w, 0x6464u, (uint32_t)j | 0x4000u | ((uint32_t)j << 8) | 0x0050u);
}
// INT4 in place: nibbles (i, i + 4) of w as an fp16 pair, each exactly
// c * 2^-24 (an fp16 pattern below 0x0800 is pattern * 2^-24: subnormal, or
// exponent field 1 with the same spacing).  No offset to remove; the 2^24
// goes into the group scale (scores) or the output unit (values).
__device__ __forceinline__ uint32_t nib_sub(uint32_t w, int i) {
  return (w >> (4 * i)) & 0x000F000Fu;
}
// Dim order of the INT4 in-place pairs inside a word's 8 dims: slot p of
// (nib_sub(w, 0), nib_sub(w, 1), nib_sub(w, 2), nib_sub(w, 3)) holds dim
// nib_dim(p) = (p / 2) + 4 (p % 2).
__device__ __forceinline__ constexpr int nib_dim(int p) { return (p >> 1) + 4 * (p & 1); }
// INT2: byte j of w -> two fp16 pairs (c0, c1), (c2, c3), exact
__device__ __forceinline__ void crumb_pairs(uint32_t w, int j, uint32_t& p01, uint32_t& p23) {
  const uint32_t x = spread2(w, j);
  p01 = h2_bits(__hfma2(bits_h2(x & 0xFF0CFF03u), __floats2half2_rn(1.0f, 0.25f),
                        __floats2half2_rn(-1024.0f, -256.0f)));
  p23 = h2_bits(__hfma2(bits_h2(x & 0xFFC0FF30u), __floats2half2_rn(0.0625f, 0.015625f),
                        __floats2half2_rn(-64.0f, -16.0f)));
}
// fp32 pair -> (high fp16 pair, low fp16 pair) with hi + lo ~ x to ~2^-22
__device__ __forceinline__ void split_h2(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x, y);
  const float2 hf = __half22float2(h);
  hi = h2_bits(h);
  lo = h2_bits(__floats2half2_rn(x - hf.x, y - hf.y));
}
// the same for a packed f32x2 pair (one packed subtract for the remainders)
__device__ __forceinline__ void split_h2p(uint64_t xy, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(lo2(xy), hi2(xy));
  const float2 hf = __half22float2(h);
  hi = h2_bits(h);
  const uint64_t r = sub2(xy, pk2(hf.x, hf.y));
  lo = h2_bits(__floats2half2_rn(lo2(r), hi2(r)));
}

template <int D, int QPG, int E>
__device__ __forceinline__ void mma_item(const unsigned char* __restrict__ regk,
                                         const unsigned char* __restrict__ regv, uint64_t soff,
                                         int t0, int n, const __half* __restrict__ q, int64_t qbase,
                                         float scale_log2, unsigned char* ring, __half* vbuf,
                                         int64_t w, float* __restrict__ ws_acc,
                                         float2* __restrict__ ws_ml) {
  using G = MG<D, E>;
  constexpr int NG = D / 32;  // groups of 32 dims
  constexpr int NK = D / 16;  // k-steps of the score MMA, m-tiles of O^T
  constexpr int VROW = D + 8; // fp16 elements of an expanded V row
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int iters = (n + kMmaTile - 1) / kMmaTile;

  // ---- copies of tile `it` into its stage (whole 16-byte units; code rows
  // padded): each lane keeps one column of the rows and steps over rows
  constexpr int RPI = 32 / G::CU;                  // rows per pass of the warp
  constexpr int PASSES = RPI >= kMmaTile ? 1 : kMmaTile / RPI;
  const int lrow = lane / G::CU, lcol = (lane % G::CU) * 16;
  auto issue = [&](int it) {
    if (it < iters) {
      unsigned char* st = ring + (it % G::STAGES) * G::STAGE;
      const int64_t row0 = t0 + (int64_t)it * kMmaTile;
      const int nv = min(kMmaTile, n - it * kMmaTile);
      const unsigned char* sk = regk + (row0 + lrow) * G::CROW + lcol;
      const unsigned char* sv = regv + (row0 + lrow) * G::CROW + lcol;
      unsigned char* dk = st + G::KOFF + lrow * G::KROW + lcol;
      unsigned char* dv = st + G::VOFF + lrow * G::KROW + lcol;
#pragma unroll
      for (int i = 0; i < PASSES; ++i) {
        if (lrow + i * RPI < nv) {
          cp_async16(dk + i * RPI * G::KROW, sk + i * RPI * G::CROW);
          cp_async16(dv + i * RPI * G::KROW, sv + i * RPI * G::CROW);
        }
      }
      if constexpr (E != 0) {
        // a tile's scales are SROW 16-byte units per array (K, then V)
        if (lane < 2 * G::SROW) {
          const int kv = lane >= G::SROW;
          const int off = (lane - kv * G::SROW) * 16;
          if (off / G::SROW < nv)
            cp_async16(st + (kv ? G::VSOFF : G::KSOFF) + off,
                       (kv ? regv : regk) + soff + row0 * G::SROW + off);
        }
      }
    }
    cp_async_commit();
  };
#pragma unroll 1
  for (int it = 0; it < G::STAGES - 1; ++it) issue(it);

  // ---- query operand (B of the score MMA): head slot gid, zero past QPG
  uint32_t qb[NK][2];
  // per group, the (head slot 2 tig, 2 tig + 1) pair of query sums; for INT4
  // in units of 2^24 (the codes enter as c * 2^-24, see score_scale)
  uint64_t qsum2[NG];
  {
    const bool hv = gid < QPG;
    const __half* qh = q + qbase + (int64_t)(hv ? gid : 0) * D;
    float part[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) part[g] = 0.f;
#pragma unroll
    for (int kk = 0; kk < NK; ++kk) {
      uint32_t b0, b1;
      if constexpr (E == 1) {
        // k = 2t, 2t+1 -> dims base + 2hh + {0, 4}; k = 2t+8, 2t+9 -> base + 2hh + {1, 5}
        const int base = 32 * (kk / 2) + 8 * tig + 2 * (kk % 2);
        const unsigned short* qs16 = reinterpret_cast<const unsigned short*>(qh);
        b0 = hv ? (uint32_t)qs16[base] | ((uint32_t)qs16[base + 4] << 16) : 0u;
        b1 = hv ? (uint32_t)qs16[base + 1] | ((uint32_t)qs16[base + 5] << 16) : 0u;
      } else {
        const int d0 = E == 0 ? 16 * kk + 2 * tig : 32 * (kk / 2) + 8 * tig + 4 * (kk % 2);
        const int d1 = E == 0 ? d0 + 8 : d0 + 2;
        b0 = hv ? *reinterpret_cast<const uint32_t*>(qh + d0) : 0u;
        b1 = hv ? *reinterpret_cast<const uint32_t*>(qh + d1) : 0u;
      }
      qb[kk][0] = b0;
      qb[kk][1] = b1;
      const float2 f0 = __half22float2(bits_h2(b0)), f1 = __half22float2(bits_h2(b1));
      part[kk / 2] += (f0.x + f0.y) + (f1.x + f1.y);
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      part[g] += __shfl_xor_sync(0xffffffffu, part[g], 1);
      part[g] += __shfl_xor_sync(0xffffffffu, part[g], 2);
      // sums of heads 2 tig and 2 tig + 1 live in lanes 8 tig and 8 tig + 4
      const float u = E == 1 ? 1.0f / 16777216.0f : 1.0f;
      qsum2[g] = pk2(__shfl_sync(0xffffffffu, part[g], 8 * tig) * u,
                     __shfl_sync(0xffffffffu, part[g], 8 * tig + 4) * u);
    }
  }

  const float score_scale = scale_log2 * (E == 1 ? 16777216.0f : 1.0f);
  float o[NK][4];
  float vb[NG][2];
  float mrun[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};
  // INT items hold O in units of 2^A (abits = bits of 2^A; 0 until the first
  // nonzero scale sets A to its binade); FP16 items in plain units
  uint32_t abits = 0u;
#pragma unroll
  for (int mt = 0; mt < NK; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
#pragma unroll
  for (int g = 0; g < NG; ++g) vb[g][0] = vb[g][1] = 0.f;
  const int r0 = gid, r1 = gid + 8;

#pragma unroll 1
  for (int it = 0; it < iters; ++it) {
    issue(it + G::STAGES - 1);
    cp_async_wait<G::STAGES - 1>();
    __syncwarp();
    unsigned char* st = ring + (it % G::STAGES) * G::STAGE;
    const int nv = min(kMmaTile, n - it * kMmaTile);
    const bool v0 = r0 < nv, v1 = r1 < nv;

    // ---- scores: C rows = tokens (r0, r1), columns = head slots (2 tig, 2 tig + 1)
    // scores of rows (r0, r1) x head slots (2 tig, 2 tig + 1), as f32x2 pairs;
    // INT4 scores in units of 2^-24
    uint64_t s01, s23;
    if constexpr (E == 0) {
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t kbase = smem_addr(st + G::KOFF);
      const int j = lane >> 3;
      const uint32_t arow = kbase + ((lane & 7) + (j & 1) * 8) * G::KROW + (j >> 1) * 16;
#pragma unroll
      for (int kk = 0; kk < NK; ++kk) {
        uint32_t a[4];
        ldsm_x4(a, arow + kk * 32);
        mma16816(s4, a[0], a[1], a[2], a[3], qb[kk][0], qb[kk][1]);
      }
      s01 = pk2(s4[0], s4[1]);
      s23 = pk2(s4[2], s4[3]);
    } else {
      // the rows' (scale, min) pairs of all groups, one vector load per row
      uint32_t ks0[NG], ks1[NG];
      if constexpr (NG == 4) {
        const uint4 a = *reinterpret_cast<const uint4*>(st + G::KSOFF + r0 * G::SROW);
        const uint4 b = *reinterpret_cast<const uint4*>(st + G::KSOFF + r1 * G::SROW);
        ks0[0] = a.x; ks0[1] = a.y; ks0[2] = a.z; ks0[3] = a.w;
        ks1[0] = b.x; ks1[1] = b.y; ks1[2] = b.z; ks1[3] = b.w;
      } else {
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          ks0[g] = *reinterpret_cast<const uint32_t*>(st + G::KSOFF + r0 * G::SROW + 4 * g);
          ks1[g] = *reinterpret_cast<const uint32_t*>(st + G::KSOFF + r1 * G::SROW + 4 * g);
        }
      }
      s01 = 0ull;
      s23 = 0ull;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (E == 1) {
          const uint32_t w0 = *reinterpret_cast<const uint32_t*>(st + G::KOFF + r0 * G::KROW + 4 * (4 * g + tig));
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(st + G::KOFF + r1 * G::KROW + 4 * (4 * g + tig));
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            mma16816(acc, nib_sub(w0, 2 * hh), nib_sub(w1, 2 * hh), nib_sub(w0, 2 * hh + 1),
                     nib_sub(w1, 2 * hh + 1), qb[2 * g + hh][0], qb[2 * g + hh][1]);
        } else {
          const uint32_t h0 = *reinterpret_cast<const unsigned short*>(st + G::KOFF + r0 * G::KROW + 8 * g + 2 * tig);
          const uint32_t h1 = *reinterpret_cast<const unsigned short*>(st + G::KOFF + r1 * G::KROW + 8 * g + 2 * tig);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t a0, a2, a1, a3;
            crumb_pairs(h0, hh, a0, a2);
            crumb_pairs(h1, hh, a1, a3);
            mma16816(acc, a0, a1, a2, a3, qb[2 * g + hh][0], qb[2 * g + hh][1]);
          }
        }
        const float2 sm0 = half2_bits_to_float2(ks0[g]), sm1 = half2_bits_to_float2(ks1[g]);
        s01 = fma2(pk2(acc[0], acc[1]), pk2(sm0.x, sm0.x), fma2(qsum2[g], pk2(sm0.y, sm0.y), s01));
        s23 = fma2(pk2(acc[2], acc[3]), pk2(sm1.x, sm1.x), fma2(qsum2[g], pk2(sm1.y, sm1.y), s23));
      }
    }

    // ---- online softmax per head slot (log2 domain, lazily moved reference;
    // rows past the item's end hold stale bytes and are masked, never used)
    float sc[4];
    sc[0] = v0 ? lo2(s01) * score_scale : -INFINITY;
    sc[1] = v0 ? hi2(s01) * score_scale : -INFINITY;
    sc[2] = v1 ? lo2(s23) * score_scale : -INFINITY;
    sc[3] = v1 ? hi2(s23) * score_scale : -INFINITY;
    float tm[2] = {fmaxf(sc[0], sc[2]), fmaxf(sc[1], sc[3])};
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      tm[0] = fmaxf(tm[0], __shfl_xor_sync(0xffffffffu, tm[0], off));
      tm[1] = fmaxf(tm[1], __shfl_xor_sync(0xffffffffu, tm[1], off));
    }
#pragma unroll
    for (int hj = 0; hj < 2; ++hj) {
      if (tm[hj] > mrun[hj] + kRescale) {
        const float a = exp2f(mrun[hj] - tm[hj]);
        lsum[hj] *= a;
#pragma unroll
        for (int g = 0; g < NG; ++g) vb[g][hj] *= a;
#pragma unroll
        for (int mt = 0; mt < NK; ++mt) {
          o[mt][hj] *= a;
          o[mt][2 + hj] *= a;
        }
        mrun[hj] = tm[hj];
      }
    }
    float p[4];
    p[0] = v0 ? exp2f(sc[0] - mrun[0]) : 0.f;
    p[1] = v0 ? exp2f(sc[1] - mrun[1]) : 0.f;
    p[2] = v1 ? exp2f(sc[2] - mrun[0]) : 0.f;
    p[3] = v1 ? exp2f(sc[3] - mrun[1]) : 0.f;
    lsum[0] += p[0] + p[2];
    lsum[1] += p[1] + p[3];

    // ---- values: O^T[dims x head slots] += Vhat^T . P'
    if constexpr (E != 0) {
      // expand this tile's V codes into vbuf (natural dim order), two lanes a row
      {
        const int row = lane >> 1, half = lane & 1;
        constexpr int HB = G::CROW / 2;  // code bytes of half a row
        const uint32_t* src = reinterpret_cast<const uint32_t*>(st + G::VOFF + row * G::KROW + half * HB);
        __half* dst = vbuf + row * VROW + half * (HB * 8 / G::BITS);
#pragma unroll
        for (int k = 0; k < HB / 4; ++k) {
          const uint32_t wv = src[k];
          if constexpr (E == 1) {  // dims in nib_dim order, values c * 2^-24
            *reinterpret_cast<uint4*>(dst + 8 * k) =
                make_uint4(nib_sub(wv, 0), nib_sub(wv, 1), nib_sub(wv, 2), nib_sub(wv, 3));
          } else {
            uint32_t c[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) crumb_pairs(wv, j, c[2 * j], c[2 * j + 1]);
            *reinterpret_cast<uint4*>(dst + 16 * k) = make_uint4(c[0], c[1], c[2], c[3]);
            *reinterpret_cast<uint4*>(dst + 16 * k + 8) = make_uint4(c[4], c[5], c[6], c[7]);
          }
        }
      }
      __syncwarp();
      const uint32_t vbase = smem_addr(vbuf);
      const int j = lane >> 3;
      const uint32_t arow = vbase + ((lane & 7) + (j >> 1) * 8) * (VROW * 2) + (j & 1) * 16;
      // O is kept in units of 2^A, A raised (like the softmax reference) when
      // a tile brings a scale of a higher binade, so that p * scale * 2^-A
      // stays within fp16 (p <= 2^8, scale <= 65504); both rescalings are
      // exact powers of two
      // scales of rows past the item's end are taken as 0 (their stage bytes
      // are stale and need not be numbers); p is 0 there as well, so those
      // rows add exactly 0 below
      float2 vsm[NG][2];
      float smax = 0.f;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(st + G::VSOFF + r0 * G::SROW + 4 * g);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(st + G::VSOFF + r1 * G::SROW + 4 * g);
        vsm[g][0] = half2_bits_to_float2(v0 ? b0 : 0u);
        vsm[g][1] = half2_bits_to_float2(v1 ? b1 : 0u);
        smax = fmaxf(smax, fmaxf(vsm[g][0].x, vsm[g][1].x));
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, off));
      const uint32_t eb = __float_as_uint(smax) & 0x7F800000u;
      if (eb > abits) {  // uniform over the warp
        if (abits != 0u) {
          const float f = __uint_as_float(0x3F800000u + abits - eb);  // 2^(A_old - A_new)
#pragma unroll
          for (int mt = 0; mt < NK; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[mt][i] *= f;
        }
        abits = eb;
      }
      const float down = __uint_as_float(0x7F000000u - abits);  // 2^-A
      // (head slot 2 tig, 2 tig + 1) pairs of p for rows r0 and r1, and p * 2^-A
      const uint64_t pp0 = pk2(p[0], p[1]), pp1 = pk2(p[2], p[3]);
      const uint64_t pd0 = mul2(pp0, pk2(down, down)), pd1 = mul2(pp1, pk2(down, down));
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const float2 sm0 = vsm[g][0], sm1 = vsm[g][1];
        const uint64_t xa = mul2(pd0, pk2(sm0.x, sm0.x));  // (x0, x1): row r0
        const uint64_t xb = mul2(pd1, pk2(sm1.x, sm1.x));  // (x2, x3): row r1
        const uint64_t vbg = fma2(pp1, pk2(sm1.y, sm1.y), fma2(pp0, pk2(sm0.y, sm0.y), pk2(vb[g][0], vb[g][1])));
        vb[g][0] = lo2(vbg);
        vb[g][1] = hi2(vbg);
        uint32_t hi0, lo0, hi1, lo1;
        split_h2p(xa, hi0, lo0);
        split_h2p(xb, hi1, lo1);
        const uint32_t bh0 = movm_t(hi0), bh1 = movm_t(hi1), bl0 = movm_t(lo0), bl1 = movm_t(lo1);
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
          const int mt = 2 * g + mm;
          uint32_t a[4];
          ldsm_x4_t(a, arow + mt * 32);
          mma16816(o[mt], a[0], a[1], a[2], a[3], bh0, bh1);
          mma16816(o[mt], a[0], a[1], a[2], a[3], bl0, bl1);
        }
      }
    } else {
      // FP16 rows straight from the stage; rows past the item's end are zeroed
      // first (stale bytes there need not be numbers, and 0 * NaN is NaN)
      if (nv < kMmaTile) {
        constexpr int RU = D * 2 / 16;  // 16-byte units of a row
        for (int u = lane; u < (kMmaTile - nv) * RU; u += 32) {
          const int row = nv + u / RU;
          *reinterpret_cast<uint4*>(st + G::VOFF + row * G::KROW + (u % RU) * 16) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      uint32_t hi0, lo0, hi1, lo1;
      split_h2(p[0], p[1], hi0, lo0);
      split_h2(p[2], p[3], hi1, lo1);
      const uint32_t bh0 = movm_t(hi0), bh1 = movm_t(hi1), bl0 = movm_t(lo0), bl1 = movm_t(lo1);
      const uint32_t vbase = smem_addr(st + G::VOFF);
      const int j = lane >> 3;
      const uint32_t arow = vbase + ((lane & 7) + (j >> 1) * 8) * G::KROW + (j & 1) * 16;
#pragma unroll
      for (int mt = 0; mt < NK; ++mt) {
        uint32_t a[4];
        ldsm_x4_t(a, arow + mt * 32);
        mma16816(o[mt], a[0], a[1], a[2], a[3], bh0, bh1);
        mma16816(o[mt], a[0], a[1], a[2], a[3], bl0, bl1);
      }
    }
    __syncwarp();  // the stage and vbuf are read before they are refilled
  }
  cp_async_wait<0>();

  // ---- partial results of the item: sum over the token lanes, then per head slot
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], off);
    lsum[1] += __shfl_xor_sync(0xffffffffu, lsum[1], off);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      vb[g][0] += __shfl_xor_sync(0xffffffffu, vb[g][0], off);
      vb[g][1] += __shfl_xor_sync(0xffffffffu, vb[g][1], off);
    }
  }
  // 2^A (and 2^24 for INT4 codes entered as c * 2^-24)
  const float up = (E == 0 || abits == 0u) ? 1.f
                   : __uint_as_float(abits) * (E == 1 ? 16777216.0f : 1.0f);
#pragma unroll
  for (int hj = 0; hj < 2; ++hj) {
    const int h = 2 * tig + hj;
    if (h < QPG) {
      float* dst = ws_acc + ((size_t)w * QPG + h) * D;
      // row p of O^T is vbuf column p: dim p for FP16 / INT2, INT4 in nib_dim order
      const int dg = E == 1 ? nib_dim(gid) : gid;
#pragma unroll
      for (int mt = 0; mt < NK; ++mt) {
        const int d0 = 16 * mt + dg, d1 = d0 + 8;
        dst[d0] = fmaf(o[mt][hj], up, vb[d0 / 32][hj]);
        dst[d1] = fmaf(o[mt][2 + hj], up, vb[d1 / 32][hj]);
      }
      if (gid == 0) ws_ml[(size_t)w * QPG + h] = make_float2(mrun[hj], lsum[hj]);
    }
  }
  __syncwarp();
}

template <int D, int QPG>
__global__ void __launch_bounds__(kMmaThreads, 12)
decode_mma_kernel(const unsigned char* __restrict__ layout, const unsigned char* __restrict__ packed,
                  const __half* __restrict__ q, float scale_log2, float* __restrict__ ws_acc,
                  float2* __restrict__ ws_ml, unsigned int* __restrict__ counter,
                  int64_t capacity_items, unsigned int* status) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  if (h->magic != MQ_LAYOUT_MAGIC || h->head_dim != D) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_BAD_LAYOUT);
    return;
  }
  const int B = h->num_seqs, Hkv = h->num_kv_heads;
  const int64_t total = (int64_t)h->total_items * Hkv;
  if (total > capacity_items) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_WORKSPACE_TOO_SMALL);
    return;
  }
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  unsigned char* ring = smem_raw + (size_t)warp * kMmaRing;
  __half* vbuf = reinterpret_cast<__half*>(ring + kMmaRing - kVbufBytes);  // quantised tiles only
  for (;;) {
    unsigned int wi = 0;
    if (lane == 0) wi = atomicAdd(counter, 1u);
    const int64_t w = (int64_t)__shfl_sync(0xffffffffu, wi, 0);
    if (w >= total) break;
    const int64_t bs = w / Hkv;
    const int g = (int)(w - bs * Hkv);
    const int b = find_item_seq(layout, B, bs);
    const mq_seq_layout* r = reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(b));
    const int s = bs < r->item_begin[1] ? 0 : (bs < r->item_begin[2] ? 1 : 2);
    const int j = (int)(bs - r->item_begin[s]);
    const int t0 = j * h->item_tokens[s];
    const int n = min(h->item_tokens[s], r->seg_tokens[s] - t0);
    if (n <= 0) {
      if (lane == 0) set_status(status, MQ_DEV_INDEX_RANGE);
      continue;
    }
    const unsigned char* regk = packed + r->seg_base[s] + (uint64_t)g * r->region_bytes[s];
    const unsigned char* regv = regk + (uint64_t)Hkv * r->region_bytes[s];
    const int64_t qbase = ((int64_t)b * Hkv + g) * QPG * D;
    if (s == 0)
      mma_item<D, QPG, 0>(regk, regv, 0, t0, n, q, qbase, scale_log2, ring, vbuf, w, ws_acc, ws_ml);
    else if (s == 1)
      mma_item<D, QPG, 1>(regk, regv, r->scale_offset[1], t0, n, q, qbase, scale_log2, ring, vbuf,
                          w, ws_acc, ws_ml);
    else
      mma_item<D, QPG, 2>(regk, regv, r->scale_offset[2], t0, n, q, qbase, scale_log2, ring, vbuf,
                          w, ws_acc, ws_ml);
  }
}

template <int D, int QPG, int QDT>
cudaError_t launch_decode_t(int64_t max_items, int Hq, const unsigned char* layout,
                            const unsigned char* packed, const void* q, float scale_log2,
                            float* out, float* ws_acc, float2* ws_ml, unsigned int* counter,
                            unsigned int* done, int* tab, float* split, int num_seqs,
                            unsigned int* status, cudaStream_t stream, bool partial) {
  // several query heads per kv-head with fp16 queries: the tensor-core kernel
  constexpr bool kMma = QDT == MQ_F16 && QPG >= 2;
  constexpr size_t smem = kMma ? mma_smem_bytes<D>() : decode_smem_bytes<D, QPG>();
  constexpr int threads = kMma ? kMmaThreads : kDecThreads;
  constexpr int warps = kMma ? kMmaWarps : kDecWarps;
  cudaError_t err;
  int dev = 0, sms = 0, per_sm = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
  const int64_t cap = max_items;  // work items x kv-heads the workspace holds
  auto run = [&](auto kern, auto qptr) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem)) != cudaSuccess)
      return e;
    int64_t grid = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
    const int64_t need = (cap + warps - 1) / warps;
    if (grid > need) grid = need;
    if (grid > 0) {
      // worker warps take items from a counter in the workspace; it and the
      // merge counters after it start at zero
      if ((e = cudaMemsetAsync(counter, 0, sizeof(unsigned int) * (1 + (size_t)num_seqs * Hq), stream)) !=
          cudaSuccess)
        return e;
      kern<<<(unsigned)grid, threads, smem, stream>>>(layout, packed, qptr, scale_log2, ws_acc, ws_ml,
                                                      counter, cap, status);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
  };
  if constexpr (D == 128 && QPG == 1 && QDT == MQ_F16)
    err = launch_decode_mha(cap, layout, packed, static_cast<const __half*>(q), scale_log2, ws_acc,
                            ws_ml, counter, tab, num_seqs, Hq, status, stream);
  else if constexpr (D == 128 && QPG == 4 && QDT == MQ_F16)
    err = launch_decode_gqa4(cap, layout, packed, static_cast<const __half*>(q), scale_log2, ws_acc,
                             ws_ml, counter, tab, num_seqs, Hq, status, stream);
  else if constexpr (kMma)
    err = run(decode_mma_kernel<D, QPG>, static_cast<const __half*>(q));
  else
    err = run(decode_partial_kernel<D, QPG, QDT>, q);
  if (err != cudaSuccess) return err;
  const int64_t heads = (int64_t)num_seqs * Hq;
  // long sequences are merged in up to kSplitMax slices of about 64 items;
  // with fewer heads than two thirds of the SMs, of about 16 (measured:
  // 40 heads of ~130 items merge 1% faster in 8 slices than in 2, 128 heads
  // of ~66 items 1.5% slower in 4 than in 1)
  const int64_t avg = max_items / Hq * QPG / (num_seqs > 0 ? num_seqs : 1);  // items per (b, h)
  const int64_t per = heads * 3 < (int64_t)sms * 2 ? 16 : 64;
  const int S = (int)(avg / per < 1 ? 1 : (avg / per > kSplitMax ? kSplitMax : avg / per));
  const dim3 grid((unsigned)heads, (unsigned)S);
  const float* acc_c = ws_acc;
  const float2* ml_c = ws_ml;
  cudaError_t e2;
  if (avg <= 32) {
    // few items per head: four warps, one round of loads each, and twice as
    // many heads resident at once
    e2 = partial ? launch_pdl(decode_combine_kernel<D, QPG, true, 4>, grid, dim3(128), 0, stream, layout,
                              Hq, acc_c, ml_c, out, split, done)
                 : launch_pdl(decode_combine_kernel<D, QPG, false, 4>, grid, dim3(128), 0, stream, layout,
                              Hq, acc_c, ml_c, out, split, done);
  } else {
    e2 = partial ? launch_pdl(decode_combine_kernel<D, QPG, true, 8>, grid, dim3(256), 0, stream, layout,
                              Hq, acc_c, ml_c, out, split, done)
                 : launch_pdl(decode_combine_kernel<D, QPG, false, 8>, grid, dim3(256), 0, stream, layout,
                              Hq, acc_c, ml_c, out, split, done);
  }
  if (e2 != cudaSuccess) return e2;
  return cudaGetLastError();
}

template <int D, int QDT>
cudaError_t dispatch_qpg(int qpg, int64_t max_items, int Hq, const unsigned char* layout,
                         const unsigned char* packed, const void* q, float scale_log2, float* out,
                         float* ws_acc, float2* ws_ml, unsigned int* counter, unsigned int* done,
                         int* tab, float* split, int B, unsigned int* status, cudaStream_t stream,
                         bool partial) {
  switch (qpg) {
    case 1: return launch_decode_t<D, 1, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, counter, done, tab, split, B, status, stream, partial);
    case 2: return launch_decode_t<D, 2, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, counter, done, tab, split, B, status, stream, partial);
    case 4: return launch_decode_t<D, 4, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, counter, done, tab, split, B, status, stream, partial);
    case 8: return launch_decode_t<D, 8, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, counter, done, tab, split, B, status, stream, partial);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t decode_workspace_bytes(const mq_shape& s, int64_t max_items) {
  const int64_t qpg = s.num_q_heads / s.num_kv_heads;
  const int64_t recs = max_items * s.num_kv_heads * qpg;
  // partial (acc) records, (m, l) records, control words (the work counter,
  // then one merge counter per (b, h)), the work-order prefix table of the
  // tensor-core kernels (3 x (B + 1) int32), the merge slices
  const uint64_t heads = (uint64_t)s.num_seqs * s.num_q_heads;
  return (size_t)align128((uint64_t)recs * s.head_dim * 4) + (size_t)align128((uint64_t)recs * 8) +
         (size_t)align128(4 + heads * 4) + (size_t)align128((uint64_t)3 * (s.num_seqs + 1) * 4) +
         (size_t)align128(heads * kSplitMax * (s.head_dim + 2) * 4);
}

cudaError_t launch_decode(const mq_shape& s, int64_t max_items, const void* layout,
                          const void* packed, const void* q, int q_dtype, float softmax_scale,
                          float* out, void* workspace, size_t workspace_bytes,
                          unsigned int* status, cudaStream_t stream, bool partial) {
  (void)workspace_bytes;
  const int64_t qpg = s.num_q_heads / s.num_kv_heads;
  const int64_t recs = max_items * s.num_kv_heads * qpg;
  float* ws_acc = static_cast<float*>(workspace);
  float2* ws_ml = reinterpret_cast<float2*>(static_cast<unsigned char*>(workspace) +
                                            align128((uint64_t)recs * s.head_dim * 4));
  unsigned int* counter = reinterpret_cast<unsigned int*>(
      static_cast<unsigned char*>(workspace) + align128((uint64_t)recs * s.head_dim * 4) +
      align128((uint64_t)recs * 8));
  const uint64_t heads = (uint64_t)s.num_seqs * s.num_q_heads;
  unsigned int* done = counter + 1;  // merge counters, zeroed with the work counter
  int* tab = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(counter) + align128(4 + heads * 4));
  float* split = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(tab) +
                                          align128((uint64_t)3 * (s.num_seqs + 1) * 4));
  const float scale_log2 = softmax_scale * 1.4426950408889634f;
  const unsigned char* lay = static_cast<const unsigned char*>(layout);
  const unsigned char* pk = static_cast<const unsigned char*>(packed);
  const int64_t cap = max_items * s.num_kv_heads;
  if (s.head_dim == 128) {
    if (q_dtype == MQ_F16)
      return dispatch_qpg<128, MQ_F16>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, counter, done, tab, split, s.num_seqs, status, stream, partial);
    return dispatch_qpg<128, MQ_F32>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, counter, done, tab, split, s.num_seqs, status, stream, partial);
  }
  if (q_dtype == MQ_F16)
    return dispatch_qpg<64, MQ_F16>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, counter, done, tab, split, s.num_seqs, status, stream, partial);
  return dispatch_qpg<64, MQ_F32>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, counter, done, tab, split, s.num_seqs, status, stream, partial);
}

cudaError_t launch_combine_partials(int P, int B, int Hq, int D, const float* parts, float* out,
                                    cudaStream_t stream) {
  const int64_t heads = (int64_t)B * Hq;
  if (heads == 0) return cudaSuccess;
  combine_partials_kernel<<<(unsigned)heads, 128, 0, stream>>>(P, heads, D, parts, out);
  return cudaGetLastError();
}

}  // namespace mqkv
