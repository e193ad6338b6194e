// decode_gqa.cu — decode attention on the tensor cores for four query heads
// per kv-head (fp16 queries, head_dim 128), straight from the mixed-bitwidth
// packed cache.
//
// MoQAE paper notes, 方法详解 › 整体框架: ordinary attention over the
// quantised cache, here with the query heads of one kv-head sharing every
// loaded token (the Llama-3 grouped-query shape):
//   o_h = sum_t softmax_t(scale * q_h . khat_t) vhat_t,  h = 0..3,
//   khat, vhat = code * (half)s + (half)min   per group of 32 dims.
// The per-item partial records (m, l, acc per query head) are merged by
// decode_combine_kernel.  Products run on mma.sync (m16n8k16, fp16 operands,
// fp32 accumulation) with the codes in place (see decode_mha.cu for the
// in-place operands); the work split, copy ring and claims are those of
// decode_tc.cuh.
//
// Scores: two accumulators of S[16 tokens x 8 columns].  In k-steps 0-3 the
//   A operand's lanes hold dims of groups 0 (tig even) and 1 (tig odd), in
//   k-steps 4-7 of groups 2 and 3, so column c carries query head c / 2
//   restricted to group c & 1 (first accumulator) or 2 + (c & 1) (second):
//   one MMA per k-step.  Lane (gid, tig) then holds, for its tokens gid and
//   gid + 8, the four groups' code dot products of head tig, applies each
//   group's scale and min and has the score of head tig without any exchange.
// Values: O^T[128 dims x 8 columns] += Vhat^T . B' per m-tile, B' holding
//   p_th * s_tg split into an fp16 high part and the fp16 remainder.  A
//   transposed ldmatrix of token rows puts one 16-bit word of two tokens
//   side by side, so a mask gives a dim's code pair.  Lane (gid, tig)
//   accumulates head tig for rows gid and gid + 8 of every m-tile.
//   INT4: a group is one 16-byte unit of a token row; m-tile 2 g + sh holds
//   group g's dims 4 i + 2 sh (rows i) and 4 i + 2 sh + 1 (rows i + 8), and
//   B'_g's column (h, hl) is head h's high (hl = 0) or low (hl = 1) part.
//   Partner lanes (the two columns of a head) each form both parts for two
//   of the four groups and exchange the halves the other needs.
//   INT2: a 16-byte unit holds two groups; m-tile 4 k + p holds dims
//   64 k + 8 i + p (rows i) and 64 k + 8 i + p + 4 (rows i + 8), both in
//   group 2 k + i / 4, and B'_k's column (h, gp) is head h, group 2 k + gp:
//   two MMAs per m-tile, high parts then low parts, into one accumulator,
//   of whose columns a lane keeps the one of its rows' group.
//   The codes' power-of-two position factors are removed from the finished
//   accumulator.
#include "decode_tc.cuh"

namespace mqkv {
namespace {

constexpr int kG = 4;  // query heads per kv-head

// Token of B' row pair slot j (0..3) on a lane with index tig in its quad.
// (the token pairs a transposed ldmatrix gives the V operand)
__device__ __forceinline__ int gq_tau(int tig, int j) { return 2 * tig + (j & 1) + 8 * (j >> 1); }

// Running state of the item in progress.
struct GqState {
  float o[8][4];   // O^T tiles: head tig, rows gid, gid + 8 of m-tile mt, columns hi / lo
  float m, m8, l;  // head tig: reference, reference + 8, sum over this lane's rows
  uint64_t bias2;  // head gid / 2, the lane's two groups: sum over its tokens of p * min
  float down, vlim;
};

__device__ __forceinline__ void gq_reset(GqState& S) {
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) S.o[mt][0] = S.o[mt][1] = S.o[mt][2] = S.o[mt][3] = 0.f;
  S.m = -INFINITY;
  S.m8 = -INFINITY;
  S.l = 0.f;
  S.bias2 = 0ull;
  S.down = 16384.0f;  // value unit 2^A, A = -14 until a larger scale arrives
  S.vlim = 1.0f / 8192.0f;
}

// Per-run query operands: the score B operand per k-step, and for head tig
// the group sums and the factor that turns a dot product into a log2-domain
// score.
struct GqQuery {
  uint32_t qb[8][2];
  float qs[4];  // scale_log2 x sum of q_tig over group g
  float sfac;
};

template <int E>
__device__ __forceinline__ void gq_query(GqQuery& Q, const __half* __restrict__ qh, float scale_log2,
                                         int lane) {
  const int gid = lane >> 2, tig = lane & 3;
  // lane L holds head L / 8, dims 16 (L % 8) .. 16 (L % 8) + 15
  const uint4 r0 = *reinterpret_cast<const uint4*>(qh + 16 * lane);
  const uint4 r1 = *reinterpret_cast<const uint4*>(qh + 16 * lane + 8);
  float qf[16];
  {
    const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 f = half2_bits_to_float2(w[i]);
      qf[2 * i] = f.x;
      qf[2 * i + 1] = f.y;
    }
  }
  float mx = 0.f, sm = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    mx = fmaxf(mx, fabsf(qf[i]));
    sm += qf[i];
  }
  sm += __shfl_xor_sync(0xffffffffu, sm, 1);  // lanes 8h + 2g, +1: group g of head h
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
#pragma unroll
  for (int g = 0; g < 4; ++g) Q.qs[g] = __shfl_sync(0xffffffffu, sm, 8 * tig + 2 * g) * scale_log2;
  if constexpr (E == 0) {
    // column c = head c / 2 (both columns of a head alike): b0 = q_h[16 ks + 2 tig, +1],
    // b1 = q_h[16 ks + 8 + 2 tig, +1], h = gid / 2
    const __half* qg = qh + (gid >> 1) * 128;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      Q.qb[ks][0] = *reinterpret_cast<const uint32_t*>(qg + 16 * ks + 2 * tig);
      Q.qb[ks][1] = *reinterpret_cast<const uint32_t*>(qg + 16 * ks + 8 + 2 * tig);
    }
    Q.sfac = scale_log2;
  } else {
    // one power of two per head brings max|q_h| to [2^14, 2^15)
    const int eb = (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127;
    const float qexp = mx > 0.f ? __uint_as_float((uint32_t)(127 + 14 - eb) << 23) : 1.f;
    const float qexp_b = __shfl_sync(0xffffffffu, qexp, 8 * (gid >> 1));  // head gid / 2 (B values)
    const float qexp_s = __shfl_sync(0xffffffffu, qexp, 8 * tig);         // head tig (scores)
    // B column gid is head gid / 2, group 2 (ks / 4) + (gid & 1); the lane's
    // k-indices are dims of group 2 (ks / 4) + (tig & 1), part th = tig / 2
    const bool on = (gid & 1) == (tig & 1);
    const int th = tig >> 1;
    const int hsrc = 8 * (gid >> 1);  // lanes of head gid / 2
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int gl = 2 * (ks / 4) + (tig & 1);
      int d0, d1, e;  // dims (inside group gl) of pairs b0 = (d0, d0 + e), b1 = (d1, d1 + e)
      float c0, c1;   // 1 / position scale
      if constexpr (E == 1) {
        d0 = 16 * th + 8 * ((ks % 4) / 2) + 2 * (ks % 2); d1 = d0 + 1; e = 4;
        c0 = 1.f; c1 = 1.f / 16.f;
      } else {
        const int p0 = 2 * (ks % 4);
        d0 = 16 * th + p0; d1 = d0 + 1; e = 8;
        c0 = 1.f / crumb_scale(p0); c1 = 1.f / crumb_scale(p0 + 1);
      }
      // dim 32 gl + d lives in lane hsrc + 2 gl + d / 16, element d % 16 (the
      // same element on every lane)
      const int base = hsrc + 2 * gl;
      const float a0 = __shfl_sync(0xffffffffu, qf[d0 & 15], base + d0 / 16);
      const float a1 = __shfl_sync(0xffffffffu, qf[(d0 + e) & 15], base + (d0 + e) / 16);
      const float b0 = __shfl_sync(0xffffffffu, qf[d1 & 15], base + d1 / 16);
      const float b1 = __shfl_sync(0xffffffffu, qf[(d1 + e) & 15], base + (d1 + e) / 16);
      const float f = on ? qexp_b : 0.f;
      Q.qb[ks][0] = h2_bits(__floats2half2_rn(a0 * f * c0, a1 * f * c0));
      Q.qb[ks][1] = h2_bits(__floats2half2_rn(b0 * f * c1, b1 * f * c1));
    }
    Q.sfac = scale_log2 / qexp_s * 16777216.0f;
  }
}

// Subtile u0 (tokens 16 u0 .. 16 u0 + 15) of a stage: scores of head tig,
// online softmax, B', values.
template <int E, int u0, bool FULL>
__device__ __forceinline__ void gq_sub(GqState& S, const GqQuery& Q, const unsigned char* st,
                                       int nv, int lane) {
  using G = TG<E>;
  constexpr int SUB = 1;
  const int gid = lane >> 2, tig = lane & 3;
  const bool hl = gid & 1;

  // ---- scores of head tig for rows gid, gid + 8 of each subtile
  float x[SUB][2];
#pragma unroll
  for (int u = 0; u < SUB; ++u) {
    float v0, v1;
    if constexpr (E == 0) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      const int j = lane >> 3;
      const uint32_t arow = smem_addr(st + G::KOFF) + ((lane & 7) + (j & 1) * 8) * G::KROW + (j >> 1) * 16;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, arow + ks * 32);
        mma16816(c, a[0], a[1], a[2], a[3], Q.qb[ks][0], Q.qb[ks][1]);
      }
      v0 = c[0] * Q.sfac;  // columns 2 tig and 2 tig + 1 are both head tig
      v1 = c[2] * Q.sfac;
    } else {
      float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};  // groups (0, 1), (2, 3)
      const unsigned char* kr = st + G::KOFF + (16 * (u0 + u) + gid) * G::CROW;
      const int th = tig >> 1, gt = tig & 1;
      if constexpr (E == 1) {
        // group 2 hv + gt, words 2 th, 2 th + 1 of it (16 dims)
        uint2 w[2][2];  // [hv][row gid, gid + 8]
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          const int off = 16 * int4_unit(gid, 2 * hv + gt) + 8 * th;  // rows gid, gid + 8 alike
          w[hv][0] = *reinterpret_cast<const uint2*>(kr + off);
          w[hv][1] = *reinterpret_cast<const uint2*>(kr + 8 * G::CROW + off);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint2 r0 = w[ks / 4][0], r1 = w[ks / 4][1];
          const uint32_t x0 = ((ks % 4) / 2) ? r0.y : r0.x, x1 = ((ks % 4) / 2) ? r1.y : r1.x;
          const uint32_t y0 = x0 >> 8, y1 = x1 >> 8;
          const int nb = 2 * (ks % 2);
          mma16816(ks < 4 ? c0 : c1, nib_at(x0, y0, nb), nib_at(x1, y1, nb), nib_at(x0, y0, nb + 1),
                   nib_at(x1, y1, nb + 1), Q.qb[ks][0], Q.qb[ks][1]);
        }
      } else {
        // group 2 hv + gt, word th of it (16 dims)
        uint32_t w[2][2];
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          const int off = 8 * (2 * hv + gt) + 4 * th;
          w[hv][0] = *reinterpret_cast<const uint32_t*>(kr + off);
          w[hv][1] = *reinterpret_cast<const uint32_t*>(kr + 8 * G::CROW + off);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t x0 = w[ks / 4][0], x1 = w[ks / 4][1];
          const uint32_t y0 = x0 >> 10, y1 = x1 >> 10;
          const int p0 = 2 * (ks % 4);
          mma16816(ks < 4 ? c0 : c1, crumb_at(x0, y0, p0), crumb_at(x1, y1, p0),
                   crumb_at(x0, y0, p0 + 1), crumb_at(x1, y1, p0 + 1), Q.qb[ks][0], Q.qb[ks][1]);
        }
      }
      // the rows' (scale, min) of all four groups
      const uint4 k0 = *reinterpret_cast<const uint4*>(st + G::KSOFF + (16 * (u0 + u) + gid) * 16);
      const uint4 k1 = *reinterpret_cast<const uint4*>(st + G::KSOFF + (16 * (u0 + u) + gid + 8) * 16);
      const float2 s00 = half2_bits_to_float2(k0.x), s01 = half2_bits_to_float2(k0.y);
      const float2 s02 = half2_bits_to_float2(k0.z), s03 = half2_bits_to_float2(k0.w);
      const float2 s10 = half2_bits_to_float2(k1.x), s11 = half2_bits_to_float2(k1.y);
      const float2 s12 = half2_bits_to_float2(k1.z), s13 = half2_bits_to_float2(k1.w);
      const float d0 = fmaf(s00.x, c0[0], fmaf(s01.x, c0[1], fmaf(s02.x, c1[0], s03.x * c1[1])));
      const float d1 = fmaf(s10.x, c0[2], fmaf(s11.x, c0[3], fmaf(s12.x, c1[2], s13.x * c1[3])));
      const float m0 = fmaf(s00.y, Q.qs[0], fmaf(s01.y, Q.qs[1], fmaf(s02.y, Q.qs[2], s03.y * Q.qs[3])));
      const float m1 = fmaf(s10.y, Q.qs[0], fmaf(s11.y, Q.qs[1], fmaf(s12.y, Q.qs[2], s13.y * Q.qs[3])));
      v0 = fmaf(d0, Q.sfac, m0);
      v1 = fmaf(d1, Q.sfac, m1);
    }
    // rows past the item's end hold stale bytes (maybe not numbers): select
    x[u][0] = (FULL || 16 * (u0 + u) + gid < nv) ? v0 : -INFINITY;
    x[u][1] = (FULL || 16 * (u0 + u) + gid + 8 < nv) ? v1 : -INFINITY;
  }

  // ---- online softmax of head tig, reference moved lazily
  float mx = fmaxf(x[0][0], x[0][1]);
  if constexpr (SUB == 2) mx = fmaxf(mx, fmaxf(x[1][0], x[1][1]));
  if (__any_sync(0xffffffffu, mx > S.m8)) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float mn = fmaxf(S.m, mx);
    const float a = ex2_ftz(S.m - mn);
    S.m = mn;
    S.m8 = mn + kTcRescale;
    S.l *= a;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) S.o[mt][i] *= a;
    const float ab = __shfl_sync(0xffffffffu, a, gid >> 1);  // head gid / 2's factor
    S.bias2 = mul2(S.bias2, pk2(ab, ab));
  }
  float p[SUB][2];
#pragma unroll
  for (int u = 0; u < SUB; ++u) {
    p[u][0] = ex2_ftz(x[u][0] - S.m);
    p[u][1] = ex2_ftz(x[u][1] - S.m);
    S.l += p[u][0] + p[u][1];
  }
  // this lane's B' rows are tokens tau_j = 2 tig + (j & 1) + 8 (j >> 1) of
  // head gid / 2
  float P[SUB][4];
#pragma unroll
  for (int u = 0; u < SUB; ++u)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tau = gq_tau(tig, j);
      P[u][j] = __shfl_sync(0xffffffffu, p[u][tau >> 3], 4 * (tau & 7) + (gid >> 1));
    }

  // ---- B' and values
  if constexpr (E == 0) {
    const uint32_t h01 = h2_bits(__floats2half2_rn(P[0][0], P[0][1]));
    const uint32_t h23 = h2_bits(__floats2half2_rn(P[0][2], P[0][3]));
    const float2 f01 = half2_bits_to_float2(h01), f23 = half2_bits_to_float2(h23);
    const uint32_t l01 = h2_bits(__floats2half2_rn(P[0][0] - f01.x, P[0][1] - f01.y));
    const uint32_t l23 = h2_bits(__floats2half2_rn(P[0][2] - f23.x, P[0][3] - f23.y));
    const uint32_t bb0 = hl ? l01 : h01, bb1 = hl ? l23 : h23;
    unsigned char* stw = const_cast<unsigned char*>(st);
    if (!FULL && nv < 16) {  // stale rows may not be numbers, and 0 * NaN is NaN
      constexpr int RU = 256 / 16;
      for (int i = lane; i < (16 - nv) * RU; i += 32)
        *reinterpret_cast<uint4*>(stw + G::VOFF + (nv + i / RU) * G::KROW + (i % RU) * 16) =
            make_uint4(0, 0, 0, 0);
      __syncwarp();
    }
    const int j = lane >> 3;
    const uint32_t arow = smem_addr(st + G::VOFF) + ((lane & 7) + (j >> 1) * 8) * G::KROW + (j & 1) * 16;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a[4];
      ldsm_x4_t(a, arow + mt * 32);
      mma16816(S.o[mt], a[0], a[1], a[2], a[3], bb0, bb1);
    }
  } else {
    // the lane's two groups of head gid / 2: INT4 ga, ga + 1 (ga = 2 (gid & 1)),
    // whose B' parts it forms for itself and for its partner lane (lane ^ 4,
    // the other column of the head); INT2 (gid & 1) and 2 + (gid & 1), the
    // groups of its own columns in the two B' matrices
    const int ga = 2 * (gid & 1);
    // per subtile: scales, value unit, B', value MMAs (fewer live registers)
#pragma unroll
    for (int u = 0; u < SUB; ++u) {
      float vs[4][2], vm[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = 16 * (u0 + u) + gq_tau(tig, j);
        const unsigned char* sr = st + G::VSOFF + row * 16;
        uint2 raw;
        if constexpr (E == 1) {
          raw = *reinterpret_cast<const uint2*>(sr + 4 * ga);
        } else {
          raw.x = *reinterpret_cast<const uint32_t*>(sr + 4 * (gid & 1));
          raw.y = *reinterpret_cast<const uint32_t*>(sr + 8 + 4 * (gid & 1));
        }
        if (!FULL && row >= nv) raw = make_uint2(0u, 0u);  // stale scales may not be numbers
        const float2 a = half2_bits_to_float2(raw.x), b = half2_bits_to_float2(raw.y);
        vs[j][0] = a.x; vm[j][0] = a.y;
        vs[j][1] = b.x; vm[j][1] = b.y;
      }
      float vmax = fmaxf(fmaxf(fmaxf(vs[0][0], vs[0][1]), fmaxf(vs[1][0], vs[1][1])),
                         fmaxf(fmaxf(vs[2][0], vs[2][1]), fmaxf(vs[3][0], vs[3][1])));
      if (__any_sync(0xffffffffu, vmax >= S.vlim)) {
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
        const uint32_t eb = __float_as_uint(vmax) & 0x7F800000u;  // 2^k, vmax in [2^k, 2^(k+1))
        const float dn = __uint_as_float(0x7F000000u - eb);        // 2^-k
        const float f = pow2_ratio(dn, S.down);                     // exact power of two
        S.down = dn;
        S.vlim = __uint_as_float(eb + 0x00800000u);                 // 2^(k+1)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) S.o[mt][i] *= f;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        S.bias2 = fma2(pk2(P[u][j], P[u][j]), pk2(vm[j][0], vm[j][1]), S.bias2);
      const uint64_t dn2 = pk2(S.down, S.down);
      const uint64_t p01 = mul2(pk2(P[u][0], P[u][1]), dn2), p23 = mul2(pk2(P[u][2], P[u][3]), dn2);
      // the lane's two groups k = 0, 1: p * s (* 2^-A) of rows (tau_0, tau_1)
      // and (tau_2, tau_3) split into fp16 high parts hi[k][pair] and
      // remainders lo[k][pair]
      uint32_t hi[2][2], lo[2][2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint64_t w01 = mul2(p01, pk2(vs[0][k], vs[1][k]));
        const uint64_t w23 = mul2(p23, pk2(vs[2][k], vs[3][k]));
        hi[k][0] = h2_bits(__floats2half2_rn(lo2(w01), hi2(w01)));
        hi[k][1] = h2_bits(__floats2half2_rn(lo2(w23), hi2(w23)));
        const float2 f01 = half2_bits_to_float2(hi[k][0]), f23 = half2_bits_to_float2(hi[k][1]);
        const uint64_t r01 = sub2(w01, pk2(f01.x, f01.y)), r23 = sub2(w23, pk2(f23.x, f23.y));
        lo[k][0] = h2_bits(__floats2half2_rn(lo2(r01), hi2(r01)));
        lo[k][1] = h2_bits(__floats2half2_rn(lo2(r23), hi2(r23)));
      }
      const int j8 = lane >> 3;
      const int vr = 16 * (u0 + u) + (lane & 7) + 8 * (j8 & 1);  // ldmatrix row of this lane
      if constexpr (E == 2) {
        // B'_k (k = 0, 1) column (h, gp) = head h, group 2 k + gp; this lane
        // holds column gid: its own parts.  A transposed ldmatrix of 8 token
        // rows x one 16-byte unit (dims 64 k .. 64 k + 63, groups 2 k, 2 k + 1)
        // gives lane (gid, tig) word gid (dims 64 k + 8 gid + 0..7, group
        // 2 k + gid / 4) of tokens 2 tig, 2 tig + 1; m-tile 4 k + p takes
        // crumbs p (rows gid) and p + 4 (rows gid + 8), so both of a lane's
        // rows lie in group 2 k + gid / 4 and one of its two columns is theirs.
        // The high and low parts go through two MMAs into one accumulator.
        uint32_t r[4];  // (unit 0, tokens 0-7), (0, 8-15), (1, 0-7), (1, 8-15)
        ldsm_x4_t(r, smem_addr(st + G::VOFF) + vr * 32 + 16 * int2_unit(vr, j8 >> 1));
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint32_t x0 = r[2 * k], x1 = r[2 * k + 1], y0 = x0 >> 10, y1 = x1 >> 10;
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) {
            const uint32_t a0 = crumb_at(x0, y0, pp), a1 = crumb_at(x0, y0, pp + 4);
            const uint32_t a2 = crumb_at(x1, y1, pp), a3 = crumb_at(x1, y1, pp + 4);
            mma16816(S.o[4 * k + pp], a0, a1, a2, a3, hi[k][0], hi[k][1]);
            mma16816(S.o[4 * k + pp], a0, a1, a2, a3, lo[k][0], lo[k][1]);
          }
        }
      } else {
        // B'_g column (h, hl) = head h, high (hl = 0) or low (hl = 1) part:
        // this lane's column takes its own kind of part; the partner lane
        // needs the other kind of the same groups
        uint32_t bb[4][2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {
            const uint32_t own = hl ? lo[k][pr] : hi[k][pr];
            const uint32_t rcv = __shfl_xor_sync(0xffffffffu, hl ? hi[k][pr] : lo[k][pr], 4);
            // groups 0, 1: own on even-gid lanes, received on odd ones; 2, 3 the reverse
            bb[k][pr] = hl ? rcv : own;
            bb[2 + k][pr] = hl ? own : rcv;
          }
        }
        // a group is one 16-byte unit of a token row: a transposed ldmatrix
        // gives lane (gid, tig) 16-bit word gid (dims 4 gid .. 4 gid + 3 of
        // the group) of tokens 2 tig (low half) and 2 tig + 1 (high half);
        // m-tile 2 g + sh takes nibbles 2 sh (rows gid) and 2 sh + 1 (rows
        // gid + 8) of group g, two masks per pair of tokens
        const uint32_t vrow = smem_addr(st + G::VOFF) + vr * 64;
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          uint32_t r[4];  // (group 2 hv, tokens 0-7), (2 hv, 8-15), (2 hv + 1, 0-7), (2 hv + 1, 8-15)
          ldsm_x4_t(r, vrow + 16 * int4_unit(vr, 2 * hv + (j8 >> 1)));
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const int g = 2 * hv + gg;
            const uint32_t x0 = r[2 * gg], x1 = r[2 * gg + 1], y0 = x0 >> 8, y1 = x1 >> 8;
            mma16816(S.o[2 * g], x0 & 0x000F000Fu, x0 & 0x00F000F0u, x1 & 0x000F000Fu, x1 & 0x00F000F0u,
                     bb[g][0], bb[g][1]);
            mma16816(S.o[2 * g + 1], y0 & 0x000F000Fu, y0 & 0x00F000F0u, y1 & 0x000F000Fu,
                     y1 & 0x00F000F0u, bb[g][0], bb[g][1]);
          }
        }
      }
    }
  }
}

// Partial records of a finished item, one per query head: unnormalised
// accumulator (with the mins' contribution) and (m, l).
template <int E>
__device__ __forceinline__ void gq_record(const GqState& S, int lane, int64_t w,
                                          float* __restrict__ ws_acc, float2* __restrict__ ws_ml) {
  const int gid = lane >> 2, tig = lane & 3;
  float l = S.l;
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  float bias[4] = {0.f, 0.f, 0.f, 0.f};
  float f = 1.f;
  if constexpr (E != 0) {
    // head gid / 2, the lane's two groups (INT4 2 (gid & 1) + {0, 1}, INT2
    // (gid & 1) + {0, 2})
    float b0 = lo2(S.bias2), b1 = hi2(S.bias2);
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      b0 += __shfl_xor_sync(0xffffffffu, b0, off);
      b1 += __shfl_xor_sync(0xffffffffu, b1, off);
    }
    // head tig's groups sit on lanes 8 tig (gid even) and 8 tig + 4 (gid odd)
    const float e0 = __shfl_sync(0xffffffffu, b0, 8 * tig), e1 = __shfl_sync(0xffffffffu, b1, 8 * tig);
    const float o0 = __shfl_sync(0xffffffffu, b0, 8 * tig + 4), o1 = __shfl_sync(0xffffffffu, b1, 8 * tig + 4);
    if constexpr (E == 1) {
      bias[0] = e0; bias[1] = e1; bias[2] = o0; bias[3] = o1;
    } else {
      bias[0] = e0; bias[1] = o0; bias[2] = e1; bias[3] = o1;
    }
    f = pow2_ratio(16777216.0f, S.down);  // 2^A and the codes' 2^-24
  }
  float* dst = ws_acc + ((size_t)w * kG + tig) * 128;
  if constexpr (E == 1) {
    // m-tile 2 g + sh: rows gid, gid + 8 are dims 32 g + 4 gid + 2 sh and
    // 32 g + 4 gid + 2 sh + 1 (nibbles at bit 4 carry a factor 16)
    const float f16 = f * 0.0625f;
#pragma unroll
    for (int g = 0; g < 4; ++g)
      *reinterpret_cast<float4*>(dst + 32 * g + 4 * gid) =
          make_float4(fmaf(S.o[2 * g][0] + S.o[2 * g][1], f, bias[g]),
                      fmaf(S.o[2 * g][2] + S.o[2 * g][3], f16, bias[g]),
                      fmaf(S.o[2 * g + 1][0] + S.o[2 * g + 1][1], f, bias[g]),
                      fmaf(S.o[2 * g + 1][2] + S.o[2 * g + 1][3], f16, bias[g]));
  } else if constexpr (E == 2) {
    // m-tile 4 k + p: rows gid, gid + 8 are dims 64 k + 8 gid + p and
    // 64 k + 8 gid + p + 4 (crumbs p, p + 4), group 2 k + gid / 4, whose
    // column is 2 tig + gid / 4
    const bool odd = gid & 4;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float bk = odd ? bias[2 * k + 1] : bias[2 * k];
      float r[8];
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        const float* c = S.o[4 * k + pp];
        r[pp] = fmaf(odd ? c[1] : c[0], f / crumb_scale(pp), bk);
        r[pp + 4] = fmaf(odd ? c[3] : c[2], f / crumb_scale(pp + 4), bk);
      }
      float4* d4 = reinterpret_cast<float4*>(dst + 64 * k + 8 * gid);
      d4[0] = make_float4(r[0], r[1], r[2], r[3]);
      d4[1] = make_float4(r[4], r[5], r[6], r[7]);
    }
  } else {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      dst[16 * mt + gid] = fmaf(S.o[mt][0] + S.o[mt][1], f, bias[mt / 2]);
      dst[16 * mt + gid + 8] = fmaf(S.o[mt][2] + S.o[mt][3], f, bias[mt / 2]);
    }
  }
  if (gid == 0) ws_ml[(size_t)w * kG + tig] = make_float2(S.m, l);
}

template <int E>
__device__ __forceinline__ void gq_run(const TcRun& R, int Hkv, const __half* __restrict__ q,
                                       float scale_log2, unsigned char* ring,
                                       float* __restrict__ ws_acc, float2* __restrict__ ws_ml) {
  using G = TG<E>;
  const int lane = threadIdx.x & 31;
  TcStream<E> cs;
  cs.init(ring, R.regk, R.regv, R.soff, R.T0, R.T1, lane);
#pragma unroll 1
  for (int s = 0; s < G::STAGES - 1; ++s) cs.issue_next(lane);

  GqQuery Q;
  gq_query<E>(Q, q + ((int64_t)R.b * Hkv + R.g) * kG * 128, scale_log2, lane);
  GqState S;
  gq_reset(S);
  int64_t w = R.w0;
  const int item_stages = R.IT / G::TOK;  // item boundaries fall on stage boundaries
  int left = item_stages;
  uint32_t soff = 0;

  // whole stages; a record at every item boundary
#pragma unroll 1
  for (int k = 0; k < cs.nfull; ++k) {
    cs.issue_next(lane);
    cp_async_wait<G::STAGES - 1>();
    __syncwarp();
    const unsigned char* st = ring + soff;
    gq_sub<E, 0, true>(S, Q, st, G::TOK, lane);
    if constexpr (G::SUB == 2) gq_sub<E, 1, true>(S, Q, st, G::TOK, lane);
    soff = soff + G::STAGE == G::STAGES * G::STAGE ? 0u : soff + G::STAGE;
    if (--left == 0) {
      gq_record<E>(S, lane, w, ws_acc, ws_ml);
      gq_reset(S);
      w += Hkv;
      left = item_stages;
    }
    __syncwarp();  // the stage is read before it is refilled
  }
  // the run's last item ends with a partial stage, or early at a stage boundary
  if (cs.tail > 0) {
    cs.issue_next(lane);
    cp_async_wait<G::STAGES - 1>();
    __syncwarp();
    const unsigned char* st = ring + soff;
    gq_sub<E, 0, false>(S, Q, st, cs.tail, lane);
    if constexpr (G::SUB == 2)
      if (cs.tail > 16) gq_sub<E, 1, false>(S, Q, st, cs.tail, lane);
    gq_record<E>(S, lane, w, ws_acc, ws_ml);
  } else if (left != item_stages) {
    gq_record<E>(S, lane, w, ws_acc, ws_ml);
  }
  cp_async_wait<0>();
  __syncwarp();
}

__global__ void __launch_bounds__(32, kTcCtasPerSm)
decode_gqa_kernel(const unsigned char* __restrict__ layout, const unsigned char* __restrict__ packed,
                  const __half* __restrict__ q, float scale_log2, float* __restrict__ ws_acc,
                  float2* __restrict__ ws_ml, unsigned int* __restrict__ counter,
                  const int* __restrict__ tab, int B, int64_t capacity_items, unsigned int* status) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  pdl_wait();     // the prep kernel's table and counters
  pdl_trigger();  // the combine may launch; it waits for this kernel
  if (!tc_layout_ok(layout, B, capacity_items, status)) return;
  const int Hkv = reinterpret_cast<const mq_layout_header*>(layout)->num_kv_heads;
  const int lane = threadIdx.x & 31;
  TcRun R;
  TcClaim C;
  while (tc_next_run(R, C, layout, packed, tab, counter, status, lane)) {
    if (R.s == 0)
      gq_run<0>(R, Hkv, q, scale_log2, smem_raw, ws_acc, ws_ml);
    else if (R.s == 1)
      gq_run<1>(R, Hkv, q, scale_log2, smem_raw, ws_acc, ws_ml);
    else
      gq_run<2>(R, Hkv, q, scale_log2, smem_raw, ws_acc, ws_ml);
  }
}

}  // namespace

cudaError_t launch_decode_gqa4(int64_t capacity_items, const unsigned char* layout,
                               const unsigned char* packed, const __half* q, float scale_log2,
                               float* ws_acc, float2* ws_ml, unsigned int* counter, int* tab,
                               int B, int Hq, unsigned int* status, cudaStream_t stream) {
  cudaError_t e;
  static std::atomic<int> workers_cache[kTcMaxDevices];
  const size_t smem = kTcRing;
  int64_t grid = 0;
  if ((e = tc_workers(reinterpret_cast<const void*>(decode_gqa_kernel), smem, workers_cache, &grid)) != cudaSuccess)
    return e;
  if (grid > capacity_items) grid = capacity_items;
  if (grid <= 0) return cudaSuccess;
  // the work order's prefix table, and the counter zeroed
  tc_prep_kernel<<<1, 256, 0, stream>>>(layout, B, B * Hq, tab, counter);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_pdl(decode_gqa_kernel, dim3((unsigned)grid), dim3(32), smem, stream, layout, packed, q,
                    scale_log2, ws_acc, ws_ml, counter, tab, B, capacity_items, status);
}

}  // namespace mqkv
