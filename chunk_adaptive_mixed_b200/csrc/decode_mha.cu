// decode_mha.cu — decode attention on the tensor cores for one query head per
// kv-head (fp16 queries, head_dim 128), straight from the mixed-bitwidth
// packed cache.
//
// MoQAE paper notes, 方法详解 › 整体框架: after quantisation the model runs
// ordinary attention over the cache,
//   o = sum_t softmax_t(scale * q . khat_t) vhat_t,
//   khat, vhat = code * (half)s + (half)min   per group of 32 dims,
// and the Cocktail abstract's chunk regrouping makes every work item read one
// precision only.  This kernel computes the per-item partial results
// (m, l, acc) that decode_combine_kernel merges, like decode_partial_kernel,
// but lets mma.sync (m16n8k16, fp16 operands, fp32 accumulation) form both
// products so that the CUDA cores only move codes into operand registers:
//
// Scores S[16 tokens x 8 columns] = Khat_codes . B.  Lane (gid, tig) of the
//   A operand holds tokens (gid, gid + 8) and only dims of group tig, so B's
//   column g carries the query restricted to group g (columns 4..7 are zero)
//   and D[t][g] is the code dot product of group g alone; the group's scale
//   and min are applied afterwards: q . khat_t = sum_g s_tg D[t][g] +
//   min_tg sum_{d in g} q_d.
// Values O^T[128 dims x 8 columns] += Vhat_codes^T . B'.  Column (g, hl) of
//   B' holds p_t * s_tg split into an fp16 high part (hl = 0) and the fp16
//   remainder (hl = 1), so the products keep fp32-level accuracy; the output
//   for dim d is the sum of its two columns of group g(d) (the other groups'
//   columns are computed and ignored).  The mins enter as sum_t p_t min_tg.
//
// Codes enter the MMAs in place: a 16-bit pattern below 2^11 read as fp16 is
// exactly pattern * 2^-24 (subnormal, or exponent field 1 with the same
// spacing), so masking a code inside its 16-bit half leaves c * 2^(o - 24)
// with o its bit offset there; codes at offsets that would reach 2^11 are
// first shifted down (INT4 by 8, INT2 by 10).  The power of two 2^o of each
// operand slot is divided out of the matching query element (scores; the
// query is first brought to [2^14, 2^15) by one power of two per item so the
// divided elements stay normal) or out of the finished accumulator (values).
// For the value product the A operand pairs two tokens of one dim: byte
// permutes interleave the 16-bit halves of two token rows, then masks pick
// each dim's code pair.
//
// One warp per CTA (12 per SM) is an independent persistent worker: it takes
// work items from an atomic counter and streams each item through its own
// cp.async ring of 16-token stages.  The stage layout keeps every lane's
// shared-memory reads conflict-free without padding for the quantised tiles
// (FP16 rows are padded for ldmatrix).
#include "decode_ptx.cuh"

namespace mqkv {
namespace {

constexpr int kTcTile = 16;        // tokens per stage
constexpr int kTcRing = 17408;     // shared bytes per worker warp
constexpr int kTcCtasPerSm = 12;   // one-warp CTAs resident per SM
constexpr float kTcRescale = 8.0f; // lazy softmax reference: weights stay below 2^8

template <int E>
struct TG {  // stage geometry at head_dim 128
  static constexpr int BITS = E == 0 ? 16 : (E == 1 ? 4 : 2);
  static constexpr int CROW = 128 * BITS / 8;            // code bytes of a token row
  static constexpr int KROW = E == 0 ? CROW + 16 : CROW; // staged pitch
  static constexpr int SROW = E == 0 ? 0 : 16;           // (scale, min) bytes of a row
  static constexpr int KOFF = 0;
  static constexpr int VOFF = kTcTile * KROW;
  static constexpr int KSOFF = 2 * kTcTile * KROW;
  static constexpr int VSOFF = KSOFF + kTcTile * SROW;
  static constexpr int STAGE = VSOFF + kTcTile * SROW;
  static constexpr int STAGES = kTcRing / STAGE < 8 ? kTcRing / STAGE : 8;
  static constexpr int CU = CROW / 16;                   // 16-byte units per code row
};
static_assert(TG<0>::STAGES >= 2 && TG<1>::STAGES >= 4 && TG<2>::STAGES >= 4, "ring too small");

// Copies of one stage (rows [row0, row0 + nv) of the item's regions) into st.
template <int E>
__device__ __forceinline__ void tc_issue(unsigned char* st, const unsigned char* regk,
                                         const unsigned char* regv, uint64_t soff, int64_t row0,
                                         int nv, int lane) {
  using G = TG<E>;
  if constexpr (E == 0) {
    // 16 units per row; lane covers rows r, r + 2, ... at column c
    const int r = lane >> 4, c = (lane & 15) * 16;
    const unsigned char* sk = regk + (row0 + r) * G::CROW + c;
    const unsigned char* sv = regv + (row0 + r) * G::CROW + c;
    unsigned char* dk = st + G::KOFF + r * G::KROW + c;
    unsigned char* dv = st + G::VOFF + r * G::KROW + c;
#pragma unroll
    for (int i = 0; i < kTcTile / 2; ++i)
      if (2 * i + r < nv) {
        cp_async16(dk + i * 2 * G::KROW, sk + i * 2 * G::CROW);
        cp_async16(dv + i * 2 * G::KROW, sv + i * 2 * G::CROW);
      }
  } else {
    // codes: one contiguous block of 16 rows per array; unit u = lane + 32 i
    constexpr int NI = kTcTile * G::CU / 32;
    const unsigned char* sk = regk + row0 * G::CROW + lane * 16;
    const unsigned char* sv = regv + row0 * G::CROW + lane * 16;
#pragma unroll
    for (int i = 0; i < NI; ++i)
      if ((lane + 32 * i) / G::CU < nv) {
        cp_async16(st + G::KOFF + (lane + 32 * i) * 16, sk + i * 512);
        cp_async16(st + G::VOFF + (lane + 32 * i) * 16, sv + i * 512);
      }
    // scales: one 16-byte row per token; lanes 0-15 K, 16-31 V
    const int sr = lane & 15;
    if (sr < nv)
      cp_async16(st + (lane < 16 ? G::KSOFF : G::VSOFF) + sr * 16,
                 (lane < 16 ? regk : regv) + soff + (row0 + sr) * 16);
  }
  cp_async_commit();
}

// In-place INT2 code pair at 2-bit position p (0..7) of both 16-bit halves:
// c * 4^(p or p - 5) * 2^-24 each (positions 5..7 come from x >> 10).
__device__ __forceinline__ uint32_t crumb_at(uint32_t x, uint32_t x10, int p) {
  return p <= 4 ? (x & (0x00030003u << (2 * p))) : (x10 & (0x00030003u << (2 * (p - 5))));
}
__host__ __device__ constexpr float crumb_scale(int p) {
  return p <= 4 ? (float)(1 << (2 * p)) : (float)(1 << (2 * (p - 5)));
}
// In-place INT4 code pair at nibble n (0..3) of both 16-bit halves:
// c * 16^(n & 1) * 2^-24 each (nibbles 2, 3 come from x >> 8).
__device__ __forceinline__ uint32_t nib_at(uint32_t x, uint32_t x8, int n) {
  return (n < 2 ? x : x8) & ((n & 1) ? 0x00F000F0u : 0x000F000Fu);
}

template <int E>
__device__ __forceinline__ void tc_item(const unsigned char* __restrict__ regk,
                                        const unsigned char* __restrict__ regv, uint64_t soff,
                                        int t0, int n, const __half* __restrict__ q,
                                        int64_t qbase, float scale_log2, unsigned char* ring,
                                        int64_t w, float* __restrict__ ws_acc,
                                        float2* __restrict__ ws_ml) {
  using G = TG<E>;
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  const int iters = (n + kTcTile - 1) / kTcTile;

#pragma unroll 1
  for (int s = 0; s < G::STAGES - 1; ++s) {
    if (s < iters)
      tc_issue<E>(ring + s * G::STAGE, regk, regv, soff, (int64_t)t0 + s * kTcTile,
                  min(kTcTile, n - s * kTcTile), lane);
    else
      cp_async_commit();
  }

  // ---- query: one power of two brings max|q| to [2^14, 2^15); per-group sums
  const __half* qh = q + qbase;
  float qsa, qsb, qexp;  // sums of groups 2(tig&1), 2(tig&1)+1 (x scale_log2); 2^E
  {
    const uint2 raw = *reinterpret_cast<const uint2*>(qh + 4 * lane);
    const float2 f0 = half2_bits_to_float2(raw.x), f1 = half2_bits_to_float2(raw.y);
    float mx = fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y)));
    float sm = (f0.x + f0.y) + (f1.x + f1.y);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) sm += __shfl_xor_sync(0xffffffffu, sm, off);
    const int ga = 2 * (tig & 1);
    qsa = __shfl_sync(0xffffffffu, sm, 8 * ga) * scale_log2;
    qsb = __shfl_sync(0xffffffffu, sm, 8 * ga + 8) * scale_log2;
    const int eb = (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127;  // floor(log2 max|q|)
    qexp = mx > 0.f ? __uint_as_float((uint32_t)(127 + 14 - eb) << 23) : 1.f;
  }
  // score B operand: qb[ks] for k-step ks
  uint32_t qb[8][2];
  if constexpr (E == 0) {
    const bool on = gid == 0;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const float2 x = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(qh + 16 * ks + 2 * tig));
      const float2 y = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(qh + 16 * ks + 8 + 2 * tig));
      const float f = on ? qexp : 0.f;
      qb[ks][0] = h2_bits(__floats2half2_rn(x.x * f, x.y * f));
      qb[ks][1] = h2_bits(__floats2half2_rn(y.x * f, y.y * f));
    }
  } else {
    const float f = gid == tig ? qexp : 0.f;
    const __half* qg = qh + 32 * tig;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      int d0, d1, e0, e1;  // dims of the (b0, b1) pairs; second element of each at +e
      float c0, c1;        // 1 / position scale of each pair
      if constexpr (E == 1) {
        d0 = 8 * (ks / 2) + 2 * (ks % 2); d1 = d0 + 1; e0 = e1 = 4;
        c0 = 1.f; c1 = 1.f / 16.f;
      } else {
        const int p0 = 2 * (ks % 4), p1 = p0 + 1;
        d0 = 16 * (ks / 4) + p0; d1 = 16 * (ks / 4) + p1; e0 = e1 = 8;
        c0 = 1.f / crumb_scale(p0); c1 = 1.f / crumb_scale(p1);
      }
      qb[ks][0] = h2_bits(__floats2half2_rn(__half2float(qg[d0]) * f * c0, __half2float(qg[d0 + e0]) * f * c0));
      qb[ks][1] = h2_bits(__floats2half2_rn(__half2float(qg[d1]) * f * c1, __half2float(qg[d1 + e1]) * f * c1));
    }
  }
  // score = sfac * (code or fp16 dot) [+ mins]: undoes 2^E and, for codes, the 2^-24
  const float sfac = scale_log2 / qexp * (E == 0 ? 1.f : 16777216.0f);

  // p redistribution: this lane's B' rows are tokens tau_j; source lanes of each
  int src[4], tau[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if constexpr (E == 0) {
      tau[j] = 2 * tig + (j & 1) + 8 * (j >> 1);
    } else {
      tau[j] = tig + 4 * j;
    }
    src[j] = 4 * (tau[j] & 7) + (tau[j] >> 3);
  }

  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float m = -INFINITY, m8 = -INFINITY, l = 0.f;
  uint64_t bias2 = 0ull;
  // value unit 2^A (INT tiles): B' = p * s * 2^-A stays below 2^9; A only rises
  float down = 16384.0f, vlim = 1.0f / 8192.0f;  // A = -14 until a larger scale arrives
  const int g = gid >> 1;
  const bool hl = gid & 1;

#pragma unroll 1
  for (int it = 0; it < iters; ++it) {
    {
      const int nx = it + G::STAGES - 1;
      if (nx < iters)
        tc_issue<E>(ring + (nx % G::STAGES) * G::STAGE, regk, regv, soff,
                    (int64_t)t0 + nx * kTcTile, min(kTcTile, n - nx * kTcTile), lane);
      else
        cp_async_commit();
    }
    cp_async_wait<G::STAGES - 1>();
    __syncwarp();
    unsigned char* st = ring + (it % G::STAGES) * G::STAGE;
    const int nv = min(kTcTile, n - it * kTcTile);

    // ---- scores (two accumulator chains)
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (E == 0) {
      const int j = lane >> 3;
      const uint32_t arow = smem_addr(st + G::KOFF) + ((lane & 7) + (j & 1) * 8) * G::KROW + (j >> 1) * 16;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, arow + ks * 32);
        mma16816(ks < 4 ? c0 : c1, a[0], a[1], a[2], a[3], qb[ks][0], qb[ks][1]);
      }
    } else if constexpr (E == 1) {
      const uint4 w0 = *reinterpret_cast<const uint4*>(st + G::KOFF + gid * 64 + 16 * tig);
      const uint4 w1 = *reinterpret_cast<const uint4*>(st + G::KOFF + (gid + 8) * 64 + 16 * tig);
      const uint32_t r0[4] = {w0.x, w0.y, w0.z, w0.w}, r1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t x0 = r0[ks / 2], x1 = r1[ks / 2];
        const uint32_t y0 = x0 >> 8, y1 = x1 >> 8;
        const int nb = 2 * (ks % 2);
        mma16816(ks < 4 ? c0 : c1, nib_at(x0, y0, nb), nib_at(x1, y1, nb), nib_at(x0, y0, nb + 1),
                 nib_at(x1, y1, nb + 1), qb[ks][0], qb[ks][1]);
      }
    } else {
      const uint2 w0 = *reinterpret_cast<const uint2*>(st + G::KOFF + gid * 32 + 8 * tig);
      const uint2 w1 = *reinterpret_cast<const uint2*>(st + G::KOFF + (gid + 8) * 32 + 8 * tig);
      const uint32_t r0[2] = {w0.x, w0.y}, r1[2] = {w1.x, w1.y};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t x0 = r0[ks / 4], x1 = r1[ks / 4];
        const uint32_t y0 = x0 >> 10, y1 = x1 >> 10;
        const int p0 = 2 * (ks % 4);
        mma16816(ks < 4 ? c0 : c1, crumb_at(x0, y0, p0), crumb_at(x1, y1, p0),
                 crumb_at(x0, y0, p0 + 1), crumb_at(x1, y1, p0 + 1), qb[ks][0], qb[ks][1]);
      }
    }
    // this lane's share of the scores of rows gid, gid + 8 (log2 units)
    float sc0, sc1;
    if constexpr (E == 0) {
      sc0 = ((c0[0] + c1[0]) + (c0[1] + c1[1])) * sfac;
      sc1 = ((c0[2] + c1[2]) + (c0[3] + c1[3])) * sfac;
    } else {
      const uint2 k0 = *reinterpret_cast<const uint2*>(st + G::KSOFF + gid * 16 + 8 * (tig & 1));
      const uint2 k1 = *reinterpret_cast<const uint2*>(st + G::KSOFF + (gid + 8) * 16 + 8 * (tig & 1));
      const float2 a0 = half2_bits_to_float2(k0.x), b0 = half2_bits_to_float2(k0.y);
      const float2 a1 = half2_bits_to_float2(k1.x), b1 = half2_bits_to_float2(k1.y);
      sc0 = fmaf(fmaf(a0.x, c0[0] + c1[0], b0.x * (c0[1] + c1[1])), sfac, fmaf(a0.y, qsa, b0.y * qsb));
      sc1 = fmaf(fmaf(a1.x, c0[2] + c1[2], b1.x * (c0[3] + c1[3])), sfac, fmaf(a1.y, qsa, b1.y * qsb));
    }
    sc0 += __shfl_xor_sync(0xffffffffu, sc0, 1);
    sc1 += __shfl_xor_sync(0xffffffffu, sc1, 1);
    // rows past the item's end hold stale bytes (maybe not numbers): masked by
    // a select; lanes tig >= 2 hold no score
    const float x0 = (tig < 2 && gid < nv) ? sc0 : -INFINITY;
    const float x1 = (tig < 2 && gid + 8 < nv) ? sc1 : -INFINITY;

    // ---- online softmax, reference moved lazily (uniform over the warp)
    if (__any_sync(0xffffffffu, fmaxf(x0, x1) > m8)) {
      float mx = fmaxf(x0, x1);
#pragma unroll
      for (int off = 2; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float a = ex2_ftz(m - mx);
      m = mx;
      m8 = mx + kTcRescale;
      l *= a;
      bias2 = mul2(bias2, pk2(a, a));
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[mt][i] *= a;
    }
    const float p0 = ex2_ftz(x0 - m), p1 = ex2_ftz(x1 - m);
    const float pv = (tig & 1) ? p1 : p0;
    float P[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) P[j] = __shfl_sync(0xffffffffu, pv, src[j]);
    l += (P[0] + P[1]) + (P[2] + P[3]);

    // ---- B' = p * s (* 2^-A), high or low fp16 part by column
    uint32_t bb0, bb1;
    if constexpr (E == 0) {
      const uint32_t h01 = h2_bits(__floats2half2_rn(P[0], P[1]));
      const uint32_t h23 = h2_bits(__floats2half2_rn(P[2], P[3]));
      const float2 f01 = half2_bits_to_float2(h01), f23 = half2_bits_to_float2(h23);
      const uint32_t l01 = h2_bits(__floats2half2_rn(P[0] - f01.x, P[1] - f01.y));
      const uint32_t l23 = h2_bits(__floats2half2_rn(P[2] - f23.x, P[3] - f23.y));
      bb0 = gid >= 2 ? 0u : (hl ? l01 : h01);
      bb1 = gid >= 2 ? 0u : (hl ? l23 : h23);
    } else {
      float vs[4], vm[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t raw = *reinterpret_cast<const uint32_t*>(st + G::VSOFF + tau[j] * 16 + 4 * g);
        const float2 f = half2_bits_to_float2(tau[j] < nv ? raw : 0u);
        vs[j] = f.x;
        vm[j] = f.y;
      }
      const float vmax = fmaxf(fmaxf(vs[0], vs[1]), fmaxf(vs[2], vs[3]));
      if (__any_sync(0xffffffffu, vmax >= vlim)) {
        float mx = vmax;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const uint32_t eb = __float_as_uint(mx) & 0x7F800000u;     // 2^k, mx in [2^k, 2^(k+1))
        const float dn = __uint_as_float(0x7F000000u - eb);         // 2^-k
        const float f = dn / down;                                  // exact power of two
        down = dn;
        vlim = __uint_as_float(eb + 0x00800000u);                    // 2^(k+1)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) o[mt][i] *= f;
      }
      bias2 = fma2(pk2(P[0], P[1]), pk2(vm[0], vm[1]), bias2);
      bias2 = fma2(pk2(P[2], P[3]), pk2(vm[2], vm[3]), bias2);
      const uint64_t w01 = mul2(pk2(P[0] * down, P[1] * down), pk2(vs[0], vs[1]));
      const uint64_t w23 = mul2(pk2(P[2] * down, P[3] * down), pk2(vs[2], vs[3]));
      const uint32_t h01 = h2_bits(__floats2half2_rn(lo2(w01), hi2(w01)));
      const uint32_t h23 = h2_bits(__floats2half2_rn(lo2(w23), hi2(w23)));
      const float2 f01 = half2_bits_to_float2(h01), f23 = half2_bits_to_float2(h23);
      const uint64_t r01 = sub2(w01, pk2(f01.x, f01.y)), r23 = sub2(w23, pk2(f23.x, f23.y));
      const uint32_t l01 = h2_bits(__floats2half2_rn(lo2(r01), hi2(r01)));
      const uint32_t l23 = h2_bits(__floats2half2_rn(lo2(r23), hi2(r23)));
      bb0 = hl ? l01 : h01;
      bb1 = hl ? l23 : h23;
    }

    // ---- values
    if constexpr (E == 0) {
      if (nv < kTcTile) {  // stale rows may not be numbers, and 0 * NaN is NaN
        constexpr int RU = 256 / 16;
        for (int u = lane; u < (kTcTile - nv) * RU; u += 32)
          *reinterpret_cast<uint4*>(st + G::VOFF + (nv + u / RU) * G::KROW + (u % RU) * 16) =
              make_uint4(0, 0, 0, 0);
        __syncwarp();
      }
      const int j = lane >> 3;
      const uint32_t arow = smem_addr(st + G::VOFF) + ((lane & 7) + (j >> 1) * 8) * G::KROW + (j & 1) * 16;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t a[4];
        ldsm_x4_t(a, arow + mt * 32);
        mma16816(o[mt], a[0], a[1], a[2], a[3], bb0, bb1);
      }
    } else if constexpr (E == 1) {
      uint2 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint2*>(st + G::VOFF + tau[j] * 64 + 8 * gid);
      // halves of token pairs (0, 1) and (2, 3): dims 0-3, 4-7 (word a), 8-11, 12-15 (word b)
      const uint32_t la01 = __byte_perm(v[0].x, v[1].x, 0x5410), ha01 = __byte_perm(v[0].x, v[1].x, 0x7632);
      const uint32_t lb01 = __byte_perm(v[0].y, v[1].y, 0x5410), hb01 = __byte_perm(v[0].y, v[1].y, 0x7632);
      const uint32_t la23 = __byte_perm(v[2].x, v[3].x, 0x5410), ha23 = __byte_perm(v[2].x, v[3].x, 0x7632);
      const uint32_t lb23 = __byte_perm(v[2].y, v[3].y, 0x5410), hb23 = __byte_perm(v[2].y, v[3].y, 0x7632);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const uint32_t xa01 = mt < 4 ? la01 : ha01, xb01 = mt < 4 ? lb01 : hb01;
        const uint32_t xa23 = mt < 4 ? la23 : ha23, xb23 = mt < 4 ? lb23 : hb23;
        const int nb = mt & 3;
        mma16816(o[mt], nib_at(xa01, xa01 >> 8, nb), nib_at(xb01, xb01 >> 8, nb),
                 nib_at(xa23, xa23 >> 8, nb), nib_at(xb23, xb23 >> 8, nb), bb0, bb1);
      }
    } else {
      uint32_t v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint32_t*>(st + G::VOFF + tau[j] * 32 + 4 * gid);
      const uint32_t l01 = __byte_perm(v[0], v[1], 0x5410), h01 = __byte_perm(v[0], v[1], 0x7632);
      const uint32_t l23 = __byte_perm(v[2], v[3], 0x5410), h23 = __byte_perm(v[2], v[3], 0x7632);
      const uint32_t l01s = l01 >> 10, h01s = h01 >> 10, l23s = l23 >> 10, h23s = h23 >> 10;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
        mma16816(o[mt], crumb_at(l01, l01s, mt), crumb_at(h01, h01s, mt), crumb_at(l23, l23s, mt),
                 crumb_at(h23, h23s, mt), bb0, bb1);
    }
    __syncwarp();  // the stage is read before it is refilled
  }
  cp_async_wait<0>();

  // ---- partial results of the item
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  float* dst = ws_acc + (size_t)w * 128;
  if constexpr (E == 0) {
    // O^T rows gid, gid + 8 of m-tile mt are dims 16 mt + gid (+8); columns 0, 1
    if (tig == 0) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        dst[16 * mt + gid] = o[mt][0] + o[mt][1];
        dst[16 * mt + gid + 8] = o[mt][2] + o[mt][3];
      }
    }
  } else {
    float bias = lo2(bias2) + hi2(bias2);
    bias += __shfl_xor_sync(0xffffffffu, bias, 1);
    bias += __shfl_xor_sync(0xffffffffu, bias, 2);
    // lanes whose columns (2 tig, 2 tig + 1) are their own dims' group hold
    // dims 16 gid + mt (row gid) and 16 gid + 8 + mt (row gid + 8)
    if (tig == g) {
      const float up = 16777216.0f / down;  // 2^A and the codes' 2^-24
      float r0[8], r1[8];
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const float f = up / (E == 1 ? ((mt & 1) ? 16.f : 1.f) : crumb_scale(mt));
        r0[mt] = fmaf(o[mt][0] + o[mt][1], f, bias);
        r1[mt] = fmaf(o[mt][2] + o[mt][3], f, bias);
      }
      float4* d4 = reinterpret_cast<float4*>(dst + 16 * gid);
      d4[0] = make_float4(r0[0], r0[1], r0[2], r0[3]);
      d4[1] = make_float4(r0[4], r0[5], r0[6], r0[7]);
      d4[2] = make_float4(r1[0], r1[1], r1[2], r1[3]);
      d4[3] = make_float4(r1[4], r1[5], r1[6], r1[7]);
    }
  }
  if (lane == 0) ws_ml[w] = make_float2(m, l);
  __syncwarp();
}

__global__ void __launch_bounds__(32, kTcCtasPerSm)
decode_mha_kernel(const unsigned char* __restrict__ layout, const unsigned char* __restrict__ packed,
                  const __half* __restrict__ q, float scale_log2, float* __restrict__ ws_acc,
                  float2* __restrict__ ws_ml, unsigned int* __restrict__ counter,
                  int64_t capacity_items, unsigned int* status) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  if (h->magic != MQ_LAYOUT_MAGIC || h->head_dim != 128) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_BAD_LAYOUT);
    return;
  }
  const int B = h->num_seqs, Hkv = h->num_kv_heads;
  const int64_t total = (int64_t)h->total_items * Hkv;
  if (total > capacity_items) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_WORKSPACE_TOO_SMALL);
    return;
  }
  const int lane = threadIdx.x & 31;
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
    const int64_t qbase = ((int64_t)b * Hkv + g) * 128;
    if (s == 0)
      tc_item<0>(regk, regv, 0, t0, n, q, qbase, scale_log2, smem_raw, w, ws_acc, ws_ml);
    else if (s == 1)
      tc_item<1>(regk, regv, r->scale_offset[1], t0, n, q, qbase, scale_log2, smem_raw, w, ws_acc,
                 ws_ml);
    else
      tc_item<2>(regk, regv, r->scale_offset[2], t0, n, q, qbase, scale_log2, smem_raw, w, ws_acc,
                 ws_ml);
  }
}

}  // namespace

cudaError_t launch_decode_mha(int64_t capacity_items, const unsigned char* layout,
                              const unsigned char* packed, const __half* q, float scale_log2,
                              float* ws_acc, float2* ws_ml, unsigned int* counter,
                              unsigned int* status, cudaStream_t stream) {
  cudaError_t e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const size_t smem = kTcRing;
  if ((e = cudaFuncSetAttribute(decode_mha_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)) != cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_mha_kernel, 32, smem)) !=
      cudaSuccess)
    return e;
  int64_t grid = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
  if (grid > capacity_items) grid = capacity_items;
  if (grid <= 0) return cudaSuccess;
  if ((e = cudaMemsetAsync(counter, 0, sizeof(unsigned int), stream)) != cudaSuccess) return e;
  decode_mha_kernel<<<(unsigned)grid, 32, smem, stream>>>(layout, packed, q, scale_log2, ws_acc, ws_ml,
                                                          counter, capacity_items, status);
  return cudaGetLastError();
}

}  // namespace mqkv
