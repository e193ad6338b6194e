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
//   scores: q . code on the raw codes (expanded with one byte-permute and a
//          mask per value pair, see spread_byte), dequantisation folded in per
//          group: q . khat = s * (q . code) + min * sum(q); shuffle-reduced
//          over the token's LPT lanes
//   softmax: online, log2 domain, with a lazily moved reference maximum
//   values: acc += (p * s) * code per value pair and bias += p * min per head
//   end of item: the TPW token lanes are merged with shuffles and (m, l,
//          acc[d]) of every head goes to the workspace.
// decode_combine_kernel — one warp per (b, query head) merges the partials of
// all items of (b, g) with the usual max-rescaling.
#include "common.cuh"

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
  static constexpr int SL = E == 0 ? (SL_INT < 8 ? SL_INT : 8) : SL_INT;
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

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// exact small integer -> float: the integer is OR-ed into the mantissa of
// 2^23 and 2^23 subtracted again (both steps exact for c < 2^23)
__device__ __forceinline__ float code_to_float(uint32_t c) {
  return __uint_as_float(0x4B000000u | c) - 8388608.0f;
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t bits) {
  __half2 h;
  *reinterpret_cast<uint32_t*>(&h) = bits;
  return __half22float2(h);
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic, round to nearest)
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  return (uint64_t)__float_as_uint(a) | ((uint64_t)__float_as_uint(b) << 32);
}
__device__ __forceinline__ uint64_t pk2u(uint32_t a, uint32_t b) {
  return (uint64_t)a | ((uint64_t)b << 32);
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Code extraction without shifts.  __byte_perm puts byte m of a code word
// into bytes 2 and 1 of a word whose byte 3 is 0x43 (the exponent of 2^7):
//   [0x43 | B | B | 0].
// Masking keeps one code in the mantissa, giving exactly 128 + c * 2^k:
//   INT4: low nibble  & 0xFF0F0000 -> 128 + c        (k = 0)
//         high nibble & 0xFF00F000 -> 128 + c / 16   (k = -4, from byte 1)
//   INT2: & 0xFF030000 -> 128 + c, & 0xFF0C0000 -> 128 + 4c,
//         & 0xFF300000 -> 128 + 16c, & 0xFF00C000 -> 128 + c / 4.
// (Byte 2's top bit is the exponent's lowest bit, so the code in that
// position is read from the byte-1 copy instead.)  Each value has at most 12
// significant bits, so its product with an fp16 query (11 bits), pre-scaled
// by 2^-k, is exact in fp32.
__device__ __forceinline__ uint32_t spread_byte(uint32_t word, int m) {
  return __byte_perm(word, 0x43u, 0x4005u | ((uint32_t)m << 8) | ((uint32_t)m << 4));
}

// Per-position scale 2^-k of the code values above (query pre-scaling), and
// its inverse (applied to value accumulators at the end).
template <int BITS>
__device__ __forceinline__ constexpr float pos_scale(int i) {
  if constexpr (BITS == 4) return i % 2 == 0 ? 1.0f : 16.0f;
  else return (i % 4) == 0 ? 1.0f : ((i % 4) == 1 ? 0.25f : ((i % 4) == 2 ? 0.0625f : 4.0f));
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

  CopyPlan<STRIDE> cp;
  plan_copies<Gm, STRIDE>(cp, regk, regv, soff, t0);
  auto issue = [&](int it) {
    if (it < iters) {
      const int nv = min(TPW, n - it * TPW);
      unsigned char* st = ring + (it % kRing) * STRIDE;
#pragma unroll
      for (int i = 0; i < CopyPlan<STRIDE>::U; ++i)
        if (cp.used[i] && cp.row[i] < nv)
          cp_async16(st + cp.dst[i], cp.src[i] + (uint64_t)it * cp.step[i]);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int it = 0; it < kRing - 1; ++it) issue(it);

  // ---- query slice of every head, in value pairs, pre-scaled per code position
  uint64_t qp[QPG][NP];
  float qs[QPG], qb[QPG];
#pragma unroll
  for (int h = 0; h < QPG; ++h) {
    const int64_t base = qbase + (int64_t)h * D + sl * SL;
    qs[h] = 0.f;
    qb[h] = 0.f;
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
        a *= pos_scale<BITS>(j);
        b *= pos_scale<BITS>(j + 1);
        qb[h] += a + b;
      }
      qp[h][j / 2] = pk2(a, b);
    }
    qb[h] *= 128.0f;
  }

  uint64_t acc[QPG][NP];
  float bias[QPG], m[QPG], l[QPG];
#pragma unroll
  for (int h = 0; h < QPG; ++h) {
    bias[h] = 0.f;
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j) acc[h][j] = 0ull;
  }
  const uint64_t k128 = pk2(128.0f, 128.0f);
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
      ks = a.x; km = a.y; vs = b.x; vm = b.y;
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
      for (int mb = 0; mb < BYTES; ++mb) {
        const uint32_t t = spread_byte(words[mb / 4], mb % 4);
        if constexpr (BITS == 4) {
          const uint64_t x = pk2u(t & 0xFF0F0000u, t & 0xFF00F000u);
#pragma unroll
          for (int h = 0; h < QPG; ++h)
            dot2[h][mb % kChains] = fma2(x, qp[h][mb], dot2[h][mb % kChains]);
        } else {
          const uint64_t x0 = pk2u(t & 0xFF030000u, t & 0xFF0C0000u);
          const uint64_t x1 = pk2u(t & 0xFF300000u, t & 0xFF00C000u);
#pragma unroll
          for (int h = 0; h < QPG; ++h) {
            dot2[h][(2 * mb) % kChains] = fma2(x0, qp[h][2 * mb], dot2[h][(2 * mb) % kChains]);
            dot2[h][(2 * mb + 1) % kChains] =
                fma2(x1, qp[h][2 * mb + 1], dot2[h][(2 * mb + 1) % kChains]);
          }
        }
      }
    }
    float part[QPG];
#pragma unroll
    for (int h = 0; h < QPG; ++h) {
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < kChains; ++c) dot += lo2(dot2[h][c]) + hi2(dot2[h][c]);
      part[h] = E == 0 ? dot : fmaf(ks, dot - qb[h], km * qs[h]);
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
      if (sc > m[h] + kRescale) {
        const float a = exp2f(m[h] - sc);
        const uint64_t a2 = pk2(a, a);
        l[h] *= a;
        bias[h] *= a;
#pragma unroll
        for (int j = 0; j < NP; ++j) acc[h][j] = fma2(acc[h][j], a2, 0ull);
        m[h] = sc;
      }
      p[h] = valid ? exp2f(sc - m[h]) : 0.f;
      l[h] += p[h];
    }
    // ---- values (lanes past the item's last token hold stale stage bytes,
    // which may decode to NaN: they skip the accumulation instead)
    if (valid) {
      uint64_t w2[QPG];
#pragma unroll
      for (int h = 0; h < QPG; ++h) {
        const float wgt = E == 0 ? p[h] : p[h] * vs;
        w2[h] = pk2(wgt, wgt);
        if constexpr (E != 0) bias[h] = fmaf(p[h], vm, bias[h]);
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
        for (int mb = 0; mb < BYTES; ++mb) {
          const uint32_t t = spread_byte(words[mb / 4], mb % 4);
          if constexpr (BITS == 4) {
            const uint64_t x = sub2(pk2u(t & 0xFF0F0000u, t & 0xFF00F000u), k128);
#pragma unroll
            for (int h = 0; h < QPG; ++h) acc[h][mb] = fma2(x, w2[h], acc[h][mb]);
          } else {
            const uint64_t x0 = sub2(pk2u(t & 0xFF030000u, t & 0xFF0C0000u), k128);
            const uint64_t x1 = sub2(pk2u(t & 0xFF300000u, t & 0xFF00C000u), k128);
#pragma unroll
            for (int h = 0; h < QPG; ++h) {
              acc[h][2 * mb] = fma2(x0, w2[h], acc[h][2 * mb]);
              acc[h][2 * mb + 1] = fma2(x1, w2[h], acc[h][2 * mb + 1]);
            }
          }
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
      av[h][2 * j] = lo2(acc[h][j]) * (E == 0 ? 1.f : pos_scale<BITS>(2 * j));
      av[h][2 * j + 1] = hi2(acc[h][j]) * (E == 0 ? 1.f : pos_scale<BITS>(2 * j + 1));
    }
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
  __syncwarp();
}

__device__ __forceinline__ int find_item_seq(const unsigned char* layout, int B, int64_t bs) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    const mq_seq_layout* r =
        reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(mid));
    if (r->item_begin[0] <= bs) lo = mid; else hi = mid - 1;
  }
  return lo;
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
template <int D, int QPG, bool PARTIAL>
__global__ void __launch_bounds__(256)
decode_combine_kernel(const unsigned char* __restrict__ layout, int Hq,
                      const float* __restrict__ ws_acc, const float2* __restrict__ ws_ml,
                      float* __restrict__ out) {
  constexpr int PER_LANE = D / 32;
  constexpr int NW = 8;
  __shared__ float s_acc[NW][D];
  __shared__ float s_m[NW], s_l[NW];
  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  const int Hkv = h->num_kv_heads;
  const int64_t bh = blockIdx.x;
  const int b = (int)(bh / Hq), hq = (int)(bh % Hq);
  const int g = hq / QPG, hh = hq % QPG;
  const int lane = threadIdx.x & 31, warp = threadIdx.x / 32;
  const mq_seq_layout* r = reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(b));
  const int i0 = r->item_begin[0];
  const int i1 = r->item_begin[2] + r->item_count[2];
  float M = -INFINITY, l = 0.f, acc[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) acc[i] = 0.f;
  for (int it = i0 + warp; it < i1; it += NW) {
    const int64_t wi = ((int64_t)it * Hkv + g) * QPG + hh;
    const float2 ml = ws_ml[wi];
    const float* a = ws_acc + wi * D + lane * PER_LANE;
    float v[PER_LANE];
    if constexpr (PER_LANE == 4) {
      const float4 t = *reinterpret_cast<const float4*>(a);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
      const float2 t = *reinterpret_cast<const float2*>(a);
      v[0] = t.x; v[1] = t.y;
    }
    const float Mn = fmaxf(M, ml.x);
    const float fa = M == -INFINITY ? 0.f : exp2f(M - Mn);
    const float fb = ml.x == -INFINITY ? 0.f : exp2f(ml.x - Mn);
    l = l * fa + ml.y * fb;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) acc[i] = acc[i] * fa + v[i] * fb;
    M = Mn;
  }
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) s_acc[warp][lane * PER_LANE + i] = acc[i];
  if (lane == 0) {
    s_m[warp] = M;
    s_l[warp] = l;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float Mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) Mx = fmaxf(Mx, s_m[w]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = s_m[w] == -INFINITY ? 0.f : exp2f(s_m[w] - Mx);
      num += f * s_acc[w][threadIdx.x];
      den += f * s_l[w];
    }
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

template <int D, int QPG, int QDT>
cudaError_t launch_decode_t(int64_t max_items, int Hq, const unsigned char* layout,
                            const unsigned char* packed, const void* q, float scale_log2,
                            float* out, float* ws_acc, float2* ws_ml, unsigned int* counter,
                            int num_seqs, unsigned int* status, cudaStream_t stream,
                            bool partial) {
  constexpr size_t smem = decode_smem_bytes<D, QPG>();
  auto kern = decode_partial_kernel<D, QPG, QDT>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  int dev = 0, sms = 0, per_sm = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
  if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecThreads, smem)) != cudaSuccess)
    return err;
  const int64_t cap = max_items;  // work items x kv-heads the workspace holds
  int64_t grid = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
  const int64_t need = (cap + kDecWarps - 1) / kDecWarps;
  if (grid > need) grid = need;
  if (grid > 0) {
    // worker warps take items from a counter in the workspace, zeroed here
    if ((err = cudaMemsetAsync(counter, 0, sizeof(unsigned int), stream)) != cudaSuccess) return err;
    kern<<<(unsigned)grid, kDecThreads, smem, stream>>>(layout, packed, q, scale_log2, ws_acc, ws_ml,
                                                         counter, cap, status);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  const int64_t heads = (int64_t)num_seqs * Hq;
  if (partial)
    decode_combine_kernel<D, QPG, true><<<(unsigned)heads, 256, 0, stream>>>(layout, Hq, ws_acc,
                                                                             ws_ml, out);
  else
    decode_combine_kernel<D, QPG, false><<<(unsigned)heads, 256, 0, stream>>>(layout, Hq, ws_acc,
                                                                              ws_ml, out);
  return cudaGetLastError();
}

template <int D, int QDT>
cudaError_t dispatch_qpg(int qpg, int64_t max_items, int Hq, const unsigned char* layout,
                         const unsigned char* packed, const void* q, float scale_log2, float* out,
                         float* ws_acc, float2* ws_ml, unsigned int* counter, int B,
                         unsigned int* status, cudaStream_t stream, bool partial) {
  switch (qpg) {
    case 1: return launch_decode_t<D, 1, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, counter, B, status, stream, partial);
    case 2: return launch_decode_t<D, 2, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, counter, B, status, stream, partial);
    case 4: return launch_decode_t<D, 4, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, counter, B, status, stream, partial);
    case 8: return launch_decode_t<D, 8, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, counter, B, status, stream, partial);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t decode_workspace_bytes(const mq_shape& s, int64_t max_items) {
  const int64_t qpg = s.num_q_heads / s.num_kv_heads;
  const int64_t recs = max_items * s.num_kv_heads * qpg;
  // partial (acc) records, (m, l) records, the work counter
  return (size_t)align128((uint64_t)recs * s.head_dim * 4) + (size_t)align128((uint64_t)recs * 8) +
         128;
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
  const float scale_log2 = softmax_scale * 1.4426950408889634f;
  const unsigned char* lay = static_cast<const unsigned char*>(layout);
  const unsigned char* pk = static_cast<const unsigned char*>(packed);
  const int64_t cap = max_items * s.num_kv_heads;
  if (s.head_dim == 128) {
    if (q_dtype == MQ_F16)
      return dispatch_qpg<128, MQ_F16>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, counter, s.num_seqs, status, stream, partial);
    return dispatch_qpg<128, MQ_F32>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, counter, s.num_seqs, status, stream, partial);
  }
  if (q_dtype == MQ_F16)
    return dispatch_qpg<64, MQ_F16>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, counter, s.num_seqs, status, stream, partial);
  return dispatch_qpg<64, MQ_F32>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, counter, s.num_seqs, status, stream, partial);
}

cudaError_t launch_combine_partials(int P, int B, int Hq, int D, const float* parts, float* out,
                                    cudaStream_t stream) {
  const int64_t heads = (int64_t)B * Hq;
  if (heads == 0) return cudaSuccess;
  combine_partials_kernel<<<(unsigned)heads, 128, 0, stream>>>(P, heads, D, parts, out);
  return cudaGetLastError();
}

}  // namespace mqkv
