// decode_tc.cuh — pieces shared by the tensor-core decode kernels
// (decode_mha.cu: one query head per kv-head; decode_gqa.cu: four): stage
// geometry of the per-warp copy ring, the in-place code operands, the stage
// copies, and the work claims.  Internal to libmqkv; not part of the ABI.
//
// Work: items are numbered segment by segment (all sequences' FP16 items,
// then INT4, then INT2, so that at any time nearly every worker runs the same
// precision's code), inside a segment region by region — (sequence,
// kv-head), then the region's items in token order — and a worker warp
// claims a group of consecutive items from an atomic counter, the group
// shrinking as the work runs out (guided self-scheduling).  The items of one
// region inside a group form a run: tokens [T0, T1) of that region, streamed
// through the worker's ring without draining it at item boundaries.  A small
// preparation kernel writes, per segment, the prefix sums of the sequences'
// item counts (the order's index) and zeroes the counter.
#pragma once

#include <atomic>

#include "decode_ptx.cuh"

namespace mqkv {
namespace {

constexpr int kTcRing = 17408;      // shared bytes per worker warp
constexpr int kTcCtasPerSm = 12;    // one-warp CTAs resident per SM
constexpr float kTcRescale = 8.0f;  // lazy softmax reference: weights stay below 2^8
constexpr int kTcMaxGroup = 8;      // items per claim at most

template <int E>
struct TG {  // stage geometry at head_dim 128
  static constexpr int BITS = E == 0 ? 16 : (E == 1 ? 4 : 2);
  static constexpr int SUB = E == 0 ? 1 : 2;             // 16-token subtiles per stage
  static constexpr int TOK = 16 * SUB;                   // tokens per stage
  static constexpr int CROW = 128 * BITS / 8;            // code bytes of a token row
  static constexpr int KROW = E == 0 ? CROW + 16 : CROW; // staged pitch
  static constexpr int SROW = E == 0 ? 0 : 16;           // (scale, min) bytes of a row
  static constexpr int KOFF = 0;
  static constexpr int VOFF = TOK * KROW;
  static constexpr int KSOFF = 2 * TOK * KROW;
  static constexpr int VSOFF = KSOFF + TOK * SROW;
  static constexpr int STAGE = VSOFF + TOK * SROW;
  static constexpr int STAGES = kTcRing / STAGE < 8 ? kTcRing / STAGE : 8;
  static constexpr int CU = CROW / 16;                   // 16-byte units per code row
};
static_assert(TG<0>::STAGES >= 2 && TG<1>::STAGES >= 3 && TG<2>::STAGES >= 3, "ring too small");

// a / b for powers of two a, b whose quotient is a normal float: the
// exponent fields subtract (exact, and no division).
__device__ __forceinline__ float pow2_ratio(float a, float b) {
  return __uint_as_float(__float_as_uint(a) - __float_as_uint(b) + 0x3F800000u);
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

// Staged INT4 code rows (64 bytes, four 16-byte units) keep unit c of row r
// at unit c ^ ((r >> 1) & 3), so that 16-byte reads of the same unit from
// rows r and r + 2 fall on different banks.  (Row parity and rows 8 apart keep
// the same pattern; unit r + 32 i shares row r's.)
__device__ __forceinline__ int int4_unit(int row, int c) { return c ^ ((row >> 1) & 3); }
// Staged INT2 value rows (32 bytes, two units) keep unit c of row r at unit
// c ^ ((r >> 2) & 1), so that the eight rows of a transposed ldmatrix phase
// fall on eight different 16-byte bank groups.  Key rows are not swizzled.
__device__ __forceinline__ int int2_unit(int row, int c) { return c ^ ((row >> 2) & 1); }

// Shared-memory byte offsets, inside a stage, of the lane's copy
// destinations: K codes, V codes (FP16: rows r, r + 2, ... at column c;
// quantised: unit lane + 32 i of each code block, INT4 rows keeping their
// four units XOR-swizzled (int4_unit), INT2 value rows their two
// (int2_unit)); the scale rows are row lane of each scale block.
template <int E>
__device__ __forceinline__ uint32_t tc_dst_k(int lane) {
  using G = TG<E>;
  if constexpr (E == 0) return G::KOFF + (lane >> 4) * G::KROW + (lane & 15) * 16;
  if constexpr (E == 1) return G::KOFF + (lane >> 2) * 64 + 16 * int4_unit(lane >> 2, lane & 3);
  return G::KOFF + lane * 16;
}
template <int E>
__device__ __forceinline__ uint32_t tc_dst_v(int lane) {
  using G = TG<E>;
  if constexpr (E == 0) return G::VOFF + (lane >> 4) * G::KROW + (lane & 15) * 16;
  if constexpr (E == 1) return G::VOFF + (lane >> 2) * 64 + 16 * int4_unit(lane >> 2, lane & 3);
  return G::VOFF + (lane >> 1) * 32 + 16 * int2_unit(lane >> 1, lane & 1);
}

// Copies of one stage into the slot at shared address sa: rows [0, nv) of
// the stage starting at the lane's source pointers (already advanced to the
// stage's first row).
template <int E, bool FULL>
__device__ __forceinline__ void tc_issue(uint32_t sa, uint32_t dk, uint32_t dv, const unsigned char* gk,
                                         const unsigned char* gv, const unsigned char* gks,
                                         const unsigned char* gvs, int nv, int lane) {
  using G = TG<E>;
  const uint64_t pol = l2_evict_first_policy();
  if constexpr (E == 0) {
    // 16 units per 256-byte row; the lane covers rows r, r + 2, ... at column c
    const int r = lane >> 4;
#pragma unroll
    for (int i = 0; i < G::TOK / 2; ++i)
      if (FULL || 2 * i + r < nv) {
        cp_async16h(sa + dk + i * 2 * G::KROW, gk + i * 2 * G::CROW, pol);
        cp_async16h(sa + dv + i * 2 * G::KROW, gv + i * 2 * G::CROW, pol);
      }
  } else {
#pragma unroll
    for (int i = 0; i < G::TOK * G::CU / 32; ++i)
      if (FULL || (lane + 32 * i) / G::CU < nv) {
        cp_async16h(sa + dk + i * 512, gk + i * 512, pol);
        cp_async16h(sa + dv + i * 512, gv + i * 512, pol);
      }
    if (FULL || lane < nv) {
      cp_async16h(sa + G::KSOFF + lane * 16, gks, pol);
      cp_async16h(sa + G::VSOFF + lane * 16, gvs, pol);
    }
  }
  cp_async_commit();
}

// The copy stream of one run: nfull whole stages, then a tail stage of
// tail rows if tail > 0; the lane's sources advance one stage per issue and
// the slots cycle through the ring.
template <int E>
struct TcStream {
  const unsigned char *gk, *gv, *gks, *gvs;
  uint32_t ring, dk, dv;  // ring's shared address; the lane's destination offsets
  uint32_t soff;          // offset of the slot of stage `issued`
  int nfull, tail, issued;

  __device__ __forceinline__ void init(unsigned char* ring_ptr, const unsigned char* regk,
                                       const unsigned char* regv, uint64_t soff_scales, int T0, int T1,
                                       int lane) {
    using G = TG<E>;
    const int ntok = T1 - T0;
    nfull = ntok / G::TOK;
    tail = ntok - nfull * G::TOK;
    issued = 0;
    ring = smem_addr(ring_ptr);
    soff = 0;
    dk = tc_dst_k<E>(lane);
    dv = tc_dst_v<E>(lane);
    if constexpr (E == 0) {
      const int64_t row = (int64_t)T0 + (lane >> 4);
      gk = regk + row * G::CROW + (lane & 15) * 16;
      gv = regv + row * G::CROW + (lane & 15) * 16;
      gks = gvs = nullptr;
    } else {
      gk = regk + (int64_t)T0 * G::CROW + lane * 16;
      gv = regv + (int64_t)T0 * G::CROW + lane * 16;
      gks = regk + soff_scales + ((int64_t)T0 + lane) * 16;
      gvs = regv + soff_scales + ((int64_t)T0 + lane) * 16;
    }
  }
  // Issues the run's next stage (or an empty group past its end).
  __device__ __forceinline__ void issue_next(int lane) {
    using G = TG<E>;
    if (issued < nfull)
      tc_issue<E, true>(ring + soff, dk, dv, gk, gv, gks, gvs, G::TOK, lane);
    else if (issued == nfull && tail > 0)
      tc_issue<E, false>(ring + soff, dk, dv, gk, gv, gks, gvs, tail, lane);
    else
      cp_async_commit();
    gk += G::TOK * G::CROW;
    gv += G::TOK * G::CROW;
    if constexpr (E != 0) {
      gks += G::TOK * 16;
      gvs += G::TOK * 16;
    }
    ++issued;
    soff = soff + G::STAGE == G::STAGES * G::STAGE ? 0u : soff + G::STAGE;
  }
};

// Worker warps (resident one-warp CTAs) of a decode kernel on the current
// device, its dynamic shared-memory limit raised first.  Both depend only on
// the kernel and the device, so each launcher keeps them in its own cache
// (one slot per device) and a call pays for the queries once.
constexpr int kTcMaxDevices = 64;
inline cudaError_t tc_workers(const void* kern, size_t smem, std::atomic<int>* cache, int64_t* workers) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < kTcMaxDevices) {
    const int c = cache[dev].load(std::memory_order_acquire);
    if (c > 0) {
      *workers = c;
      return cudaSuccess;
    }
  }
  int sms = 0, per_sm = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32, smem)) != cudaSuccess)
    return e;
  const int c = sms * (per_sm > 0 ? per_sm : 1);
  if (dev < kTcMaxDevices) cache[dev].store(c, std::memory_order_release);
  *workers = c;
  return cudaSuccess;
}

// A run: tokens [T0, T1) of one region, items of IT tokens, the first
// item's record w0 (the next ones w0 + Hkv, ...).
struct TcRun {
  const unsigned char* regk;
  const unsigned char* regv;
  uint64_t soff;
  int T0, T1, IT, s, b, g;
  int64_t w0;
};

struct TcClaim {
  int64_t v = 0, v1 = 0;
};

// Prefix table of the work order: tab[s * (B + 1) + b] = items of segment s
// (per kv-head) in sequences before b; tab[s * (B + 1) + B] = the segment's
// total.  One CTA; also zeroes the control words (the work counter and the
// nheads merge counters after it).  B is the caller's sequence count (the
// table was sized with it).
__global__ void __launch_bounds__(256)
tc_prep_kernel(const unsigned char* __restrict__ layout, int B, int nheads, int* __restrict__ tab,
               unsigned int* __restrict__ counter) {
  __shared__ int red[33];
  pdl_trigger();  // the decode kernel may launch now; it waits for this one
  for (int i = threadIdx.x; i <= nheads; i += blockDim.x) counter[i] = 0u;
  for (int s = 0; s < kNumExperts; ++s) {
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += blockDim.x) {
      const int b = b0 + threadIdx.x;
      const int c = b < B ? reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(b))
                                ->item_count[s]
                          : 0;
      int total = 0;
      const int ex = block_exclusive_scan<int>(c, red, &total);
      if (b < B) tab[s * (B + 1) + b] = carry + ex;
      carry += total;
    }
    if (threadIdx.x == 0) tab[s * (B + 1) + B] = carry;
  }
}

// The worker's next run, claiming a new group when the current one is used
// up.  Returns false when the work is exhausted.  Item j of kv-head g of
// sequence b in segment s has number
//   v = Hkv * (totals of segments before s + tab[s][b]) + g * count + j
// (count = the sequence's items in s) and record (item_begin[s] + j) * Hkv + g.
__device__ __forceinline__ bool tc_next_run(TcRun& R, TcClaim& C, const unsigned char* layout,
                                            const unsigned char* packed, const int* __restrict__ tab,
                                            unsigned int* counter, unsigned int* status, int lane) {
  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  const int B = h->num_seqs, Hkv = h->num_kv_heads;
  const int64_t total = (int64_t)h->total_items * Hkv;
  for (;;) {
    if (C.v >= C.v1) {
      // guided claim: up to kTcMaxGroup items, about the remaining work over
      // twice the workers
      unsigned int v0 = 0, cnt = 0;
      if (lane == 0) {
        const int64_t cur = (int64_t)*reinterpret_cast<volatile unsigned int*>(counter);
        const int64_t want = (total - cur) / (2 * (int64_t)gridDim.x);
        cnt = (unsigned int)(want < 1 ? 1 : (want > kTcMaxGroup ? kTcMaxGroup : want));
        v0 = atomicAdd(counter, cnt);
      }
      v0 = __shfl_sync(0xffffffffu, v0, 0);
      cnt = __shfl_sync(0xffffffffu, cnt, 0);
      if ((int64_t)v0 >= total) return false;
      C.v = v0;
      C.v1 = min((int64_t)v0 + cnt, total);
    }
    const int64_t v = C.v;
    const int64_t t0 = (int64_t)Hkv * tab[B], t1 = (int64_t)Hkv * tab[2 * B + 1];
    const int s = v < t0 ? 0 : (v < t0 + t1 ? 1 : 2);
    const int* ts = tab + s * (B + 1);
    const int64_t sbase = s == 0 ? 0 : (s == 1 ? t0 : t0 + t1);
    const int64_t ib = (v - sbase) / Hkv;  // item block inside the segment
    // the last sequence whose prefix is <= ib (sequences without items in s
    // share their successor's prefix and are skipped)
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ts[mid] <= ib) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int cntr = ts[b + 1] - ts[b];
    const int64_t base = sbase + (int64_t)Hkv * ts[b];
    const int64_t u = v - base;
    const int g = cntr > 0 ? (int)(u / cntr) : 0;
    const int j = cntr > 0 ? (int)(u - (int64_t)g * cntr) : 0;
    const int64_t vend = min(C.v1, base + (int64_t)(g + 1) * cntr);  // end of the region's items
    const mq_seq_layout* r = reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(b));
    const int IT = h->item_tokens[s];
    R.T0 = j * IT;
    R.T1 = (int)min((int64_t)r->seg_tokens[s], (int64_t)(j + (vend - v)) * IT);
    if (cntr <= 0 || g >= Hkv || u < 0 || R.T1 <= R.T0 || r->item_count[s] != cntr) {
      if (lane == 0) set_status(status, MQ_DEV_INDEX_RANGE);
      C.v = C.v1;  // drop the rest of this group
      continue;
    }
    R.IT = IT;
    R.s = s;
    R.b = b;
    R.g = g;
    R.regk = packed + r->seg_base[s] + (uint64_t)g * r->region_bytes[s];
    R.regv = R.regk + (uint64_t)Hkv * r->region_bytes[s];
    R.soff = s == 0 ? 0 : r->scale_offset[s];
    R.w0 = ((int64_t)r->item_begin[s] + j) * Hkv + g;
    C.v = vend;
    return true;
  }
}

// Header checks shared by the kernels; false (status set) when the layout is
// not usable.
__device__ __forceinline__ bool tc_layout_ok(const unsigned char* layout, int B,
                                             int64_t capacity_items, unsigned int* status) {
  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  if (h->magic != MQ_LAYOUT_MAGIC || h->head_dim != 128 || h->num_seqs != B) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_BAD_LAYOUT);
    return false;
  }
  if ((int64_t)h->total_items * h->num_kv_heads > capacity_items) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_WORKSPACE_TOO_SMALL);
    return false;
  }
  return true;
}

}  // namespace
}  // namespace mqkv
