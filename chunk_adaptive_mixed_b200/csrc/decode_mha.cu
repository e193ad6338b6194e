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
// query is first brought to [2^14, 2^15) by one power of two so the divided
// elements stay normal) or out of the finished accumulator (values).  For the
// value product the A operand pairs two tokens of one dim: a transposed
// ldmatrix over token rows puts the same 16-bit word of two tokens side by
// side, then masks pick each dim's code pair (so an m-tile's rows are dims in
// the order of their bit positions, undone when the record is written).
//
// Work: one warp per CTA (12 per SM) is a persistent worker.  Work items are
// numbered region by region — (sequence, segment, kv-head), then the items of
// that region in token order — and a worker claims a group of consecutive
// items from an atomic counter, the group shrinking as the work runs out
// (guided self-scheduling: long streams early, a short tail).  Consecutive
// items of one region form one run: the worker streams the run's token range
// through its cp.async ring (32-token stages for INT4 / INT2, 16-token stages
// for FP16) without draining the ring at item boundaries, and writes each
// item's partial record when the item's last stage is done.  Every item is
// computed from a fresh state, so its record does not depend on which worker
// took it or on the grouping.  Quantised stages are laid out so that every
// lane's shared-memory reads are conflict-free without padding; FP16 rows are
// padded for ldmatrix.
#include "decode_tc.cuh"

namespace mqkv {
namespace {

// Running state of the item in progress (one query head).
struct TcState {
  float o[8][4];
  float m, m8, l;
  uint64_t bias2;
  float down, vlim;  // value unit 2^A as 2^-A and 2^(A+1) (quantised items)
};

__device__ __forceinline__ void tc_reset(TcState& S) {
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) S.o[mt][0] = S.o[mt][1] = S.o[mt][2] = S.o[mt][3] = 0.f;
  S.m = -INFINITY;
  S.m8 = -INFINITY;
  S.l = 0.f;
  S.bias2 = 0ull;
  S.down = 16384.0f;          // A = -14 until a larger scale arrives
  S.vlim = 1.0f / 8192.0f;
}

// Per-run query operands and constants.
struct TcQuery {
  uint32_t qb[8][2];  // score B operand per k-step
  float qsa, qsb;     // (scale_log2 x) sums of q over groups 2(tig&1), 2(tig&1)+1
  float sfac;         // code or fp16 dot -> log2-domain score
};

template <int E>
__device__ __forceinline__ void tc_query(TcQuery& Q, const __half* __restrict__ qh, float scale_log2,
                                         int lane) {
  const int gid = lane >> 2, tig = lane & 3;
  // lane holds dims 4 lane .. 4 lane + 3
  const uint2 raw = *reinterpret_cast<const uint2*>(qh + 4 * lane);
  const float2 f0 = half2_bits_to_float2(raw.x), f1 = half2_bits_to_float2(raw.y);
  float mx = fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y)));
  float sm = (f0.x + f0.y) + (f1.x + f1.y);
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) sm += __shfl_xor_sync(0xffffffffu, sm, off);
  const int ga = 2 * (tig & 1);
  Q.qsa = __shfl_sync(0xffffffffu, sm, 8 * ga) * scale_log2;
  Q.qsb = __shfl_sync(0xffffffffu, sm, 8 * ga + 8) * scale_log2;
  if constexpr (E == 0) {
    // b0 = q[16 ks + 2 tig, +1], b1 = q[16 ks + 8 + 2 tig, +1] on lanes gid == 0
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int l0 = 4 * ks + (tig >> 1), l1 = 4 * ks + 2 + (tig >> 1);
      const uint32_t x0 = __shfl_sync(0xffffffffu, raw.x, l0), y0 = __shfl_sync(0xffffffffu, raw.y, l0);
      const uint32_t x1 = __shfl_sync(0xffffffffu, raw.x, l1), y1 = __shfl_sync(0xffffffffu, raw.y, l1);
      Q.qb[ks][0] = gid == 0 ? ((tig & 1) ? y0 : x0) : 0u;
      Q.qb[ks][1] = gid == 0 ? ((tig & 1) ? y1 : x1) : 0u;
    }
    Q.sfac = scale_log2;
  } else {
    // one power of two brings max|q| to [2^14, 2^15)
    const int eb = (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127;
    const float qexp = mx > 0.f ? __uint_as_float((uint32_t)(127 + 14 - eb) << 23) : 1.f;
    const float f = gid == tig ? qexp : 0.f;  // group tig's column is lane (tig, tig)'s
    const float qv[4] = {f0.x, f0.y, f1.x, f1.y};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      // dims (d, d + e) of pair b0 and (d1, d1 + e) of b1, inside group tig;
      // each dim's element index (d mod 4) is the same on every lane
      int d0, d1, e;
      float c0, c1;  // 1 / position scale
      if constexpr (E == 1) {
        d0 = 8 * (ks / 2) + 2 * (ks % 2); d1 = d0 + 1; e = 4;
        c0 = 1.f; c1 = 1.f / 16.f;
      } else {
        const int p0 = 2 * (ks % 4);
        d0 = 16 * (ks / 4) + p0; d1 = d0 + 1; e = 8;
        c0 = 1.f / crumb_scale(p0); c1 = 1.f / crumb_scale(p0 + 1);
      }
      const int src = 8 * tig;  // lane holding dims 32 tig .. 32 tig + 3
      const float a0 = __shfl_sync(0xffffffffu, qv[d0 & 3], src + d0 / 4);
      const float a1 = __shfl_sync(0xffffffffu, qv[d0 & 3], src + (d0 + e) / 4);
      const float b0 = __shfl_sync(0xffffffffu, qv[d1 & 3], src + d1 / 4);
      const float b1 = __shfl_sync(0xffffffffu, qv[d1 & 3], src + (d1 + e) / 4);
      Q.qb[ks][0] = h2_bits(__floats2half2_rn(a0 * f * c0, a1 * f * c0));
      Q.qb[ks][1] = h2_bits(__floats2half2_rn(b0 * f * c1, b1 * f * c1));
    }
    // undoes 2^E and the codes' 2^-24
    Q.sfac = scale_log2 / qexp * 16777216.0f;
  }
}

// One stage: scores of its subtiles, online softmax, B', values.
// FULL: a stage of TOK valid rows (no row checks); otherwise rows [0, nv).
template <int E, bool FULL>
__device__ __forceinline__ void tc_stage(TcState& S, const TcQuery& Q, const unsigned char* st,
                                         int nv, int lane) {
  using G = TG<E>;
  constexpr int SUB = G::SUB;
  const int gid = lane >> 2, tig = lane & 3;
  const int g = gid >> 1;
  const bool hl = gid & 1;

  // ---- scores of rows gid, gid + 8 of each subtile (one accumulator chain
  // per subtile; the two subtiles of a stage interleave)
  float sc[SUB][2];
#pragma unroll
  for (int u = 0; u < SUB; ++u) {
    float c0[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (E == 0) {
      const int j = lane >> 3;
      const uint32_t arow = smem_addr(st + G::KOFF) + ((lane & 7) + (j & 1) * 8) * G::KROW + (j >> 1) * 16;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, arow + ks * 32);
        mma16816(c0, a[0], a[1], a[2], a[3], Q.qb[ks][0], Q.qb[ks][1]);
      }
      sc[u][0] = (c0[0] + c0[1]) * Q.sfac;
      sc[u][1] = (c0[2] + c0[3]) * Q.sfac;
    } else {
      const unsigned char* kr = st + G::KOFF + (16 * u + gid) * G::CROW;
      if constexpr (E == 1) {
        const int un = 16 * int4_unit(gid, tig);  // rows gid, gid + 8 share the swizzle
        const uint4 w0 = *reinterpret_cast<const uint4*>(kr + un);
        const uint4 w1 = *reinterpret_cast<const uint4*>(kr + 8 * G::CROW + un);
        const uint32_t r0[4] = {w0.x, w0.y, w0.z, w0.w}, r1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t x0 = r0[ks / 2], x1 = r1[ks / 2];
          const uint32_t y0 = x0 >> 8, y1 = x1 >> 8;
          const int nb = 2 * (ks % 2);
          mma16816(c0, nib_at(x0, y0, nb), nib_at(x1, y1, nb), nib_at(x0, y0, nb + 1),
                   nib_at(x1, y1, nb + 1), Q.qb[ks][0], Q.qb[ks][1]);
        }
      } else {
        const uint2 w0 = *reinterpret_cast<const uint2*>(kr + 8 * tig);
        const uint2 w1 = *reinterpret_cast<const uint2*>(kr + 8 * G::CROW + 8 * tig);
        const uint32_t r0[2] = {w0.x, w0.y}, r1[2] = {w1.x, w1.y};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t x0 = r0[ks / 4], x1 = r1[ks / 4];
          const uint32_t y0 = x0 >> 10, y1 = x1 >> 10;
          const int p0 = 2 * (ks % 4);
          mma16816(c0, crumb_at(x0, y0, p0), crumb_at(x1, y1, p0),
                   crumb_at(x0, y0, p0 + 1), crumb_at(x1, y1, p0 + 1), Q.qb[ks][0], Q.qb[ks][1]);
        }
      }
      const unsigned char* ksr = st + G::KSOFF + (16 * u + gid) * 16 + 8 * (tig & 1);
      const uint2 k0 = *reinterpret_cast<const uint2*>(ksr);
      const uint2 k1 = *reinterpret_cast<const uint2*>(ksr + 8 * 16);
      const float2 a0 = half2_bits_to_float2(k0.x), b0 = half2_bits_to_float2(k0.y);
      const float2 a1 = half2_bits_to_float2(k1.x), b1 = half2_bits_to_float2(k1.y);
      sc[u][0] = fmaf(fmaf(a0.x, c0[0], b0.x * c0[1]), Q.sfac,
                      fmaf(a0.y, Q.qsa, b0.y * Q.qsb));
      sc[u][1] = fmaf(fmaf(a1.x, c0[2], b1.x * c0[3]), Q.sfac,
                      fmaf(a1.y, Q.qsa, b1.y * Q.qsb));
    }
  }
  // full scores (lanes tig 0, 1); rows past the item's end hold stale bytes
  // (maybe not numbers) and are masked by a select; lanes tig >= 2 hold none
  float x[SUB][2];
#pragma unroll
  for (int u = 0; u < SUB; ++u)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float v = sc[u][r] + __shfl_xor_sync(0xffffffffu, sc[u][r], 1);
      x[u][r] = (tig < 2 && (FULL || 16 * u + 8 * r + gid < nv)) ? v : -INFINITY;
    }

  // ---- online softmax, reference moved lazily (uniform over the warp)
  float mx = fmaxf(x[0][0], x[0][1]);
  if constexpr (SUB == 2) mx = fmaxf(mx, fmaxf(x[1][0], x[1][1]));
  if (__any_sync(0xffffffffu, mx > S.m8)) {
#pragma unroll
    for (int off = 2; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float a = ex2_ftz(S.m - mx);
    S.m = mx;
    S.m8 = mx + kTcRescale;
    S.l *= a;
    S.bias2 = mul2(S.bias2, pk2(a, a));
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) S.o[mt][i] *= a;
  }
  // this lane's B' rows are tokens tau_j = 2 tig + (j & 1) + 8 (j >> 1) of
  // each subtile, the token pairs of a transposed ldmatrix
  float P[SUB][4];
#pragma unroll
  for (int u = 0; u < SUB; ++u) {
    const float p0 = ex2_ftz(x[u][0] - S.m), p1 = ex2_ftz(x[u][1] - S.m);
    const float pv = (tig & 1) ? p1 : p0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tau = 2 * tig + (j & 1) + 8 * (j >> 1);
      P[u][j] = __shfl_sync(0xffffffffu, pv, 4 * (tau & 7) + (tau >> 3));
    }
    S.l += (P[u][0] + P[u][1]) + (P[u][2] + P[u][3]);
  }

  // ---- B' = p * s (* 2^-A), high or low fp16 part by column
  uint32_t bb[SUB][2];
  if constexpr (E == 0) {
    const uint32_t h01 = h2_bits(__floats2half2_rn(P[0][0], P[0][1]));
    const uint32_t h23 = h2_bits(__floats2half2_rn(P[0][2], P[0][3]));
    const float2 f01 = half2_bits_to_float2(h01), f23 = half2_bits_to_float2(h23);
    const uint32_t l01 = h2_bits(__floats2half2_rn(P[0][0] - f01.x, P[0][1] - f01.y));
    const uint32_t l23 = h2_bits(__floats2half2_rn(P[0][2] - f23.x, P[0][3] - f23.y));
    bb[0][0] = gid >= 2 ? 0u : (hl ? l01 : h01);
    bb[0][1] = gid >= 2 ? 0u : (hl ? l23 : h23);
  } else {
    float vs[SUB][4], vm[SUB][4];
#pragma unroll
    for (int u = 0; u < SUB; ++u)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = 16 * u + 2 * tig + (j & 1) + 8 * (j >> 1);
        uint32_t raw = *reinterpret_cast<const uint32_t*>(st + G::VSOFF + row * 16 + 4 * g);
        if (!FULL) raw = row < nv ? raw : 0u;  // stale scales may not be numbers
        const float2 f = half2_bits_to_float2(raw);
        vs[u][j] = f.x;
        vm[u][j] = f.y;
      }
    float vmax = fmaxf(fmaxf(vs[0][0], vs[0][1]), fmaxf(vs[0][2], vs[0][3]));
    if constexpr (SUB == 2) vmax = fmaxf(vmax, fmaxf(fmaxf(vs[1][0], vs[1][1]), fmaxf(vs[1][2], vs[1][3])));
    if (__any_sync(0xffffffffu, vmax >= S.vlim)) {
      float v = vmax;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
      const uint32_t eb = __float_as_uint(v) & 0x7F800000u;     // 2^k, v in [2^k, 2^(k+1))
      const float dn = __uint_as_float(0x7F000000u - eb);         // 2^-k
      const float f = pow2_ratio(dn, S.down);                      // exact power of two
      S.down = dn;
      S.vlim = __uint_as_float(eb + 0x00800000u);                  // 2^(k+1)
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) S.o[mt][i] *= f;
    }
#pragma unroll
    for (int u = 0; u < SUB; ++u) {
      S.bias2 = fma2(pk2(P[u][0], P[u][1]), pk2(vm[u][0], vm[u][1]), S.bias2);
      S.bias2 = fma2(pk2(P[u][2], P[u][3]), pk2(vm[u][2], vm[u][3]), S.bias2);
      const uint64_t dn2 = pk2(S.down, S.down);
      const uint64_t w01 = mul2(mul2(pk2(P[u][0], P[u][1]), dn2), pk2(vs[u][0], vs[u][1]));
      const uint64_t w23 = mul2(mul2(pk2(P[u][2], P[u][3]), dn2), pk2(vs[u][2], vs[u][3]));
      const uint32_t h01 = h2_bits(__floats2half2_rn(lo2(w01), hi2(w01)));
      const uint32_t h23 = h2_bits(__floats2half2_rn(lo2(w23), hi2(w23)));
      const float2 f01 = half2_bits_to_float2(h01), f23 = half2_bits_to_float2(h23);
      const uint64_t r01 = sub2(w01, pk2(f01.x, f01.y)), r23 = sub2(w23, pk2(f23.x, f23.y));
      const uint32_t l01 = h2_bits(__floats2half2_rn(lo2(r01), hi2(r01)));
      const uint32_t l23 = h2_bits(__floats2half2_rn(lo2(r23), hi2(r23)));
      bb[u][0] = hl ? l01 : h01;
      bb[u][1] = hl ? l23 : h23;
    }
  }

  // ---- values: O^T += Vhat^T . B'
  if constexpr (E == 0) {
    unsigned char* stw = const_cast<unsigned char*>(st);
    if (!FULL) {  // stale rows may not be numbers, and 0 * NaN is NaN
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
      mma16816(S.o[mt], a[0], a[1], a[2], a[3], bb[0][0], bb[0][1]);
    }
  } else {
    // a transposed ldmatrix of 8 token rows x one 16-byte unit gives lane
    // (gid, tig) 16-bit word gid of the unit for tokens 2 tig (low half) and
    // 2 tig + 1 (high half); masks then pick one dim's code pair
    const int j = lane >> 3;
#pragma unroll
    for (int u = 0; u < SUB; ++u) {
      const int row = 16 * u + (lane & 7) + 8 * (j & 1);
      if constexpr (E == 1) {
        // unit = group; m-tile 2 g + sh takes nibbles 2 sh (rows gid) and
        // 2 sh + 1 (rows gid + 8) of word gid: dims 32 g + 4 gid + 2 sh (+1)
        const uint32_t vrow = smem_addr(st + G::VOFF) + row * 64;
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          uint32_t r[4];  // (group 2 hv, tokens 0-7), (2 hv, 8-15), (2 hv + 1, 0-7), (2 hv + 1, 8-15)
          ldsm_x4_t(r, vrow + 16 * int4_unit(row, 2 * hv + (j >> 1)));
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const int mt = 2 * (2 * hv + gg);
            const uint32_t lo = r[2 * gg], hi = r[2 * gg + 1], lo8 = lo >> 8, hi8 = hi >> 8;
            mma16816(S.o[mt], lo & 0x000F000Fu, lo & 0x00F000F0u, hi & 0x000F000Fu, hi & 0x00F000F0u,
                     bb[u][0], bb[u][1]);
            mma16816(S.o[mt + 1], lo8 & 0x000F000Fu, lo8 & 0x00F000F0u, hi8 & 0x000F000Fu,
                     hi8 & 0x00F000F0u, bb[u][0], bb[u][1]);
          }
        }
      } else {
        // units 0, 1 hold dims 0-63, 64-127; m-tile p takes crumb p of word
        // gid: rows gid, gid + 8 are dims 8 gid + p and 64 + 8 gid + p
        uint32_t r[4];  // (unit 0, tokens 0-7), (0, 8-15), (1, 0-7), (1, 8-15)
        ldsm_x4_t(r, smem_addr(st + G::VOFF) + row * 32 + 16 * int2_unit(row, j >> 1));
        const uint32_t s0 = r[0] >> 10, s1 = r[1] >> 10, s2 = r[2] >> 10, s3 = r[3] >> 10;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
          mma16816(S.o[mt], crumb_at(r[0], s0, mt), crumb_at(r[2], s2, mt), crumb_at(r[1], s1, mt),
                   crumb_at(r[3], s3, mt), bb[u][0], bb[u][1]);
      }
    }
  }
}

// Partial record of a finished item: unnormalised accumulator (with the
// mins' contribution) and (m, l).
template <int E>
__device__ __forceinline__ void tc_record(const TcState& S, int lane, int64_t w,
                                          float* __restrict__ ws_acc, float2* __restrict__ ws_ml) {
  const int gid = lane >> 2, tig = lane & 3;
  float l = S.l;
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  float* dst = ws_acc + (size_t)w * 128;
  if constexpr (E == 0) {
    // O^T rows gid, gid + 8 of m-tile mt are dims 16 mt + gid (+8); columns 0, 1
    if (tig == 0) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        dst[16 * mt + gid] = S.o[mt][0] + S.o[mt][1];
        dst[16 * mt + gid + 8] = S.o[mt][2] + S.o[mt][3];
      }
    }
  } else {
    float bias = lo2(S.bias2) + hi2(S.bias2);  // group gid / 2, this lane's tokens
    bias += __shfl_xor_sync(0xffffffffu, bias, 1);
    bias += __shfl_xor_sync(0xffffffffu, bias, 2);
    // columns (2 tig, 2 tig + 1) are group tig's: a lane writes the dims of
    // group tig among its rows, with that group's sum of p * min
    bias = __shfl_sync(0xffffffffu, bias, 8 * tig);
    const float up = pow2_ratio(16777216.0f, S.down);  // 2^A and the codes' 2^-24
    if constexpr (E == 1) {
      // m-tiles 2 tig, 2 tig + 1: dims 32 tig + 4 gid + (0, 1, 2, 3), the odd
      // ones from nibbles at bit 4 (factor 16)
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int g = 0; g < 4; ++g)
        if (tig == g)
          v = make_float4(S.o[2 * g][0] + S.o[2 * g][1], S.o[2 * g][2] + S.o[2 * g][3],
                          S.o[2 * g + 1][0] + S.o[2 * g + 1][1], S.o[2 * g + 1][2] + S.o[2 * g + 1][3]);
      *reinterpret_cast<float4*>(dst + 32 * tig + 4 * gid) =
          make_float4(fmaf(v.x, up, bias), fmaf(v.y, up * 0.0625f, bias), fmaf(v.z, up, bias),
                      fmaf(v.w, up * 0.0625f, bias));
    } else {
      // rows gid hold dims 8 gid + mt (group gid / 4), rows gid + 8 dims
      // 64 + 8 gid + mt (group 2 + gid / 4)
      const bool upper = tig >= 2;
      if (tig == (gid >> 2) + (upper ? 2 : 0)) {
        float r[8];
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
          r[mt] = fmaf(upper ? S.o[mt][2] + S.o[mt][3] : S.o[mt][0] + S.o[mt][1], up / crumb_scale(mt),
                       bias);
        float4* d4 = reinterpret_cast<float4*>(dst + (upper ? 64 : 0) + 8 * gid);
        d4[0] = make_float4(r[0], r[1], r[2], r[3]);
        d4[1] = make_float4(r[4], r[5], r[6], r[7]);
      }
    }
  }
  if (lane == 0) ws_ml[w] = make_float2(S.m, l);
}

// One run: tokens [T0, T1) of one region (the region's items j0, j0 + 1, ...
// of IT tokens each; records w0, w0 + Hkv, ...), streamed through the ring.
template <int E>
__device__ __forceinline__ void tc_run(const TcRun& R, int Hkv, const __half* __restrict__ q,
                                       float scale_log2, unsigned char* ring,
                                       float* __restrict__ ws_acc, float2* __restrict__ ws_ml) {
  using G = TG<E>;
  const int lane = threadIdx.x & 31;
  TcStream<E> cs;
  cs.init(ring, R.regk, R.regv, R.soff, R.T0, R.T1, lane);
#pragma unroll 1
  for (int s = 0; s < G::STAGES - 1; ++s) cs.issue_next(lane);

  TcQuery Q;
  tc_query<E>(Q, q + ((int64_t)R.b * Hkv + R.g) * 128, scale_log2, lane);
  TcState S;
  tc_reset(S);
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
    tc_stage<E, true>(S, Q, ring + soff, G::TOK, lane);
    soff = soff + G::STAGE == G::STAGES * G::STAGE ? 0u : soff + G::STAGE;
    if (--left == 0) {
      tc_record<E>(S, lane, w, ws_acc, ws_ml);
      tc_reset(S);
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
    tc_stage<E, false>(S, Q, ring + soff, cs.tail, lane);
    tc_record<E>(S, lane, w, ws_acc, ws_ml);
  } else if (left != item_stages) {
    tc_record<E>(S, lane, w, ws_acc, ws_ml);
  }
  cp_async_wait<0>();
  __syncwarp();
}

__global__ void __launch_bounds__(32, kTcCtasPerSm)
decode_mha_kernel(const unsigned char* __restrict__ layout, const unsigned char* __restrict__ packed,
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
      tc_run<0>(R, Hkv, q, scale_log2, smem_raw, ws_acc, ws_ml);
    else if (R.s == 1)
      tc_run<1>(R, Hkv, q, scale_log2, smem_raw, ws_acc, ws_ml);
    else
      tc_run<2>(R, Hkv, q, scale_log2, smem_raw, ws_acc, ws_ml);
  }
}

}  // namespace

cudaError_t launch_decode_mha(int64_t capacity_items, const unsigned char* layout,
                              const unsigned char* packed, const __half* q, float scale_log2,
                              float* ws_acc, float2* ws_ml, unsigned int* counter, int* tab,
                              int B, int Hq, unsigned int* status, cudaStream_t stream) {
  cudaError_t e;
  static std::atomic<int> workers_cache[kTcMaxDevices];
  const size_t smem = kTcRing;
  int64_t grid = 0;
  if ((e = tc_workers(reinterpret_cast<const void*>(decode_mha_kernel), smem, workers_cache, &grid)) != cudaSuccess)
    return e;
  if (grid > capacity_items) grid = capacity_items;
  if (grid <= 0) return cudaSuccess;
  // the work order's prefix table, and the counter zeroed
  tc_prep_kernel<<<1, 256, 0, stream>>>(layout, B, B * Hq, tab, counter);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_pdl(decode_mha_kernel, dim3((unsigned)grid), dim3(32), smem, stream, layout, packed, q,
                    scale_log2, ws_acc, ws_ml, counter, tab, B, capacity_items, status);
}

}  // namespace mqkv
