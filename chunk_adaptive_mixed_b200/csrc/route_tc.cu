// route_tc.cu — router scores on the 5th-generation tensor cores.
//
// MoQAE paper notes, 关键设计 › Quantization-Aware Experts: every token of a
// chunk C is scored against the experts {FP16, INT4, INT2} by a small MLP,
// read here as z_t = (SiLU(C_t W1) ⊙ (C_t W2)) W3 + b3.  The two projections
// C·W1 and C·W2 are one dense contraction [T, D] x [D, 2H]: it runs on
// tcgen05.mma (kind::f16 with bf16 operands) by splitting both operands into
// a bf16 high part and the bf16 of the remainder (x ~ hi + lo) and
// accumulating hi·hi + hi·lo + lo·hi in fp32 (the dropped lo·lo term and the
// rounding of lo leave about 2^-16 relative per product; the scores stay
// within the tolerance the routing decisions allow, see include/mqkv.h).
//
// router_tc_kernel: one CTA owns 128 tokens and one block of HB hidden units
// of both branches (an N = 2*HB accumulator in tensor memory); the CTAs of
// one token tile are consecutive in the grid.
//   warps 0-7  load C (fp32) for the next k-tile, split it, store the two
//              halves into 128B-swizzled K-major shared tiles (eight warps
//              keep enough loads in flight), then run the epilogue: SiLU
//              gate, W3 projection of this hidden block.
//   warp 8     allocates tensor memory and issues the MMAs (one thread).
//   warp 9     brings the pre-split, pre-swizzled weight tiles with 1-D bulk
//              copies.
// Two shared-memory stages; per stage a full mbarrier (the producers), a
// weight mbarrier (the bulk copies' bytes) and an empty one; tcgen05.commit
// frees a stage when its MMAs complete.  Every wait is bounded: on timeout
// the kernel records MQ_DEV_WAIT_TIMEOUT, stops, lets the weight copies it
// started land, frees its tensor memory and returns.
#include <cuda_bf16.h>

#include "common.cuh"

namespace mqkv {
namespace {

constexpr int kTcBM = 128;     // tokens per CTA (MMA M)
constexpr int kTcKE = 64;      // bf16 k elements per k-tile (one 128-byte swizzle row)
constexpr int kTcStages = 2;
constexpr int kTcProdWarps = 8;                  // producer warps (C split, epilogue)
constexpr int kTcProd = 32 * kTcProdWarps;
constexpr int kTcMmaWarp = kTcProdWarps;         // one thread issues the MMAs
constexpr int kTcWeightWarp = kTcProdWarps + 1;  // one thread copies the weight tiles
constexpr int kTcThreads = 32 * (kTcProdWarps + 2);
static_assert(kTcThreads == 32 * (kTcWeightWarp + 1), "the weight warp is the block's last warp");
constexpr uint32_t kTcWaitLimit = 1u << 24;
constexpr uint32_t kTcTestWaitLimit = 1u << 12;  // under the test hook: a stop within milliseconds

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// bf16 high parts of (a, b) and the bf16 of their remainders, packed in pairs.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Byte offset of 16-byte chunk c (0..7) of row r inside a K-major tile with
// 128-byte rows and the 128-byte swizzle (chunk index XOR row-in-atom).
__host__ __device__ __forceinline__ uint32_t swz_off(int r, int c) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), leading offset unused (1), version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: fp32 accumulate, bf16 A and B, both K-major.
template <int M, int N>
constexpr uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int BN>
struct TcSmem {
  static constexpr int A_BYTES = kTcBM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE = 2 * A_BYTES + 2 * B_BYTES;
  static constexpr int TOTAL = kTcStages * STAGE + 1024 /*barriers*/ + 1024 /*alignment*/;
};

// ---------------------------------------------------------------- weights
// Wp[hb][kt][hi|lo][BN rows x 128 B] in the swizzled K-major tile layout;
// rows 0..HB-1 are W1's hidden units hb*HB.., rows HB..2HB-1 W2's.
template <int BN>
__global__ void prepack_weights_kernel(const float* __restrict__ W1, const float* __restrict__ W2,
                                       int D, int H, int nkt, unsigned char* __restrict__ Wp) {
  constexpr int HB = BN / 2;
  const int hb = blockIdx.y, kt = blockIdx.x;
  unsigned char* tile_hi = Wp + ((size_t)(hb * nkt + kt) * 2) * (BN * 128);
  unsigned char* tile_lo = tile_hi + BN * 128;
  for (int q = threadIdx.x; q < BN * 8; q += blockDim.x) {
    const int n = q / 8, c = q % 8;
    const float* W = n < HB ? W1 : W2;
    const int col = hb * HB + (n < HB ? n : n - HB);
    const uint32_t off = swz_off(n, c);
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = kt * kTcKE + 8 * c + i;
      x[i] = k < D ? W[(size_t)k * H + col] : 0.0f;
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_bf16x2(x[2 * i], x[2 * i + 1], hi[i], lo[i]);
    *reinterpret_cast<uint4*>(tile_hi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(tile_lo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

// ---------------------------------------------------------------- router
template <int BN>
__global__ void __launch_bounds__(kTcThreads, 1)
router_tc_kernel(const float* __restrict__ C, int64_t T, int D, int nkt,
                 const unsigned char* __restrict__ Wp, const float* __restrict__ W3,
                 float4* __restrict__ zpart, int nhb, unsigned int* status, uint32_t wait_limit,
                 int inject) {
  constexpr int HB = BN / 2;
  using S = TcSmem<BN>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* stages = base;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kTcStages * S::STAGE);
  uint64_t* empty = full + kTcStages;
  uint64_t* done = empty + kTcStages;
  uint64_t* wfull = done + 1;  // the weight tiles' bytes, per stage
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wfull + kTcStages);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  // the nhb hidden blocks of one token tile are adjacent CTAs, so they run
  // together and all but the first read the tile's C rows from L2
  const int64_t m0 = (int64_t)(blockIdx.x / nhb) * kTcBM;
  const int hb = (int)(blockIdx.x % nhb);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], kTcProd);
      mbar_init(&empty[s], 1);
      mbar_init(&wfull[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto a_hi = [&](int s) { return stages + s * S::STAGE; };
  auto a_lo = [&](int s) { return stages + s * S::STAGE + S::A_BYTES; };
  auto b_hi = [&](int s) { return stages + s * S::STAGE + 2 * S::A_BYTES; };
  auto b_lo = [&](int s) { return stages + s * S::STAGE + 2 * S::A_BYTES + S::B_BYTES; };
  auto fail = [&]() {
    set_status(status, MQ_DEV_WAIT_TIMEOUT);
    atomicExch(abort_flag, 1);
  };

  if (warp < kTcProdWarps) {
    // ---- producers: C tile (128 rows x kTcKE fp32) -> split -> swizzled stores
    const int t = threadIdx.x;  // 0..kTcProd-1
    constexpr int NV = kTcKE / 32;  // float4 loads per 16-byte chunk of a part
    constexpr int PER = 8 * kTcBM / kTcProd;  // 16-byte chunks per thread and k-tile
    // two register buffers: the loads of k-tile kt + 2 are issued as soon as
    // k-tile kt is stored, so two tiles of loads are in flight
    float4 buf0[PER * NV], buf1[PER * NV];
    auto load = [&](int kt, float4 (&buf)[PER * NV]) {
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int f = t + kTcProd * i;
        const int row = f >> 3, c = f & 7;
        const int64_t tok = m0 + row;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const int k = kt * kTcKE + (kTcKE / 8) * c + 4 * v;
          buf[NV * i + v] = (tok < T && k < D)
                                ? __ldg(reinterpret_cast<const float4*>(C + tok * D + k))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    };
    // split k-tile kt into its stage; false when the kernel gives up
    auto store = [&](int kt, const float4 (&buf)[PER * NV]) -> bool {
      const int s = kt % kTcStages;
      const uint32_t ph = (kt / kTcStages) & 1;
      if (*(volatile int*)abort_flag) return false;
      if (!mbar_wait(&empty[s], ph ^ 1, wait_limit)) { fail(); return false; }
      unsigned char* hi = a_hi(s);
      unsigned char* lo = a_lo(s);
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int f = t + kTcProd * i;
        const int row = f >> 3, c = f & 7;
        const uint32_t off = swz_off(row, c);
        const float4 x0 = buf[2 * i], x1 = buf[2 * i + 1];
        uint32_t h[4], l[4];
        split_bf16x2(x0.x, x0.y, h[0], l[0]);
        split_bf16x2(x0.z, x0.w, h[1], l[1]);
        split_bf16x2(x1.x, x1.y, h[2], l[2]);
        split_bf16x2(x1.z, x1.w, h[3], l[3]);
        *reinterpret_cast<uint4*>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
      }
      fence_proxy_async();  // generic-proxy stores -> visible to the tensor cores
      // (inject: the test hook withholds the first stage, so the MMA
      // thread's bounded wait runs out)
      if (!(inject && kt == 0)) mbar_arrive(&full[s]);
      return true;
    };
    load(0, buf0);
    if (nkt > 1) load(1, buf1);
    for (int kt = 0; kt < nkt; kt += 2) {
      if (!store(kt, buf0)) break;
      if (kt + 2 < nkt) load(kt + 2, buf0);
      if (kt + 1 >= nkt) break;
      if (!store(kt + 1, buf1)) break;
      if (kt + 3 < nkt) load(kt + 3, buf1);
    }
  } else if (warp == kTcMmaWarp) {
    // ---- MMA issue (one thread)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16<kTcBM, BN>();
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt % kTcStages;
        const uint32_t ph = (kt / kTcStages) & 1;
        if (*(volatile int*)abort_flag) break;
        if (!mbar_wait(&full[s], ph, wait_limit) || !mbar_wait(&wfull[s], ph, wait_limit)) {
          fail();
          break;
        }
        tc_fence_after();
        const uint32_t ah = smem_u32(a_hi(s)), al = smem_u32(a_lo(s));
        const uint32_t bh = smem_u32(b_hi(s)), bl = smem_u32(b_lo(s));
        const uint32_t pa[3] = {ah, ah, al}, pb[3] = {bh, bl, bh};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)  // K = 16 bf16 (32 bytes) per MMA
            umma_bf16(tmem, smem_desc(pa[pass] + 32 * ks), smem_desc(pb[pass] + 32 * ks), idesc,
                      (kt | pass | ks) != 0);
        umma_commit(&empty[s]);  // the stage is free once these MMAs are done
      }
      umma_commit(done);  // all issued MMAs complete -> epilogue may read
    }
    __syncwarp();
  } else {
    // ---- weight tiles (one thread)
    if (lane == 0) {
      int issued = 0;
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt % kTcStages;
        const uint32_t ph = (kt / kTcStages) & 1;
        if (*(volatile int*)abort_flag) break;
        if (!mbar_wait(&empty[s], ph ^ 1, wait_limit)) { fail(); break; }
        const unsigned char* src = Wp + ((size_t)(hb * nkt + kt) * 2) * S::B_BYTES;
        mbar_arrive_expect_tx(&wfull[s], 2 * S::B_BYTES);
        bulk_g2s(b_hi(s), src, S::B_BYTES, &wfull[s]);
        bulk_g2s(b_lo(s), src + S::B_BYTES, S::B_BYTES, &wfull[s]);
        issued = kt + 1;
      }
      // after a stop, the copies this thread started must land before the
      // CTA's shared memory goes away: each stage's latest one, waited on
      // (bounded) through its own barrier
      if (*(volatile int*)abort_flag)
        for (int kt = max(0, issued - kTcStages); kt < issued; ++kt)
          mbar_wait(&wfull[kt % kTcStages], (kt / kTcStages) & 1, wait_limit);
    }
    __syncwarp();
  }

  // ---- epilogue: producer warp w reads tensor-memory lanes 32 (w % 4).. (its
  // 32 tokens; a warp may only read its quarter of the lanes) and half w / 4
  // of the hidden block's columns; the halves' partial scores meet in shared
  // memory (the stages are free: every MMA has completed)
  if (warp < kTcProdWarps) {
    const int q4 = warp & 3, half = warp >> 2;
    const bool ok = mbar_wait(done, 0, wait_limit);
    if (!ok) fail();
    tc_fence_after();
    float z0 = 0.f, z1 = 0.f, z2 = 0.f;
    // tcgen05.ld is warp-collective: the whole warp takes the same branch
    const bool run = __all_sync(0xffffffffu, ok && !*(volatile int*)abort_flag);
    if (run) {
      const uint32_t lane_addr = tmem + ((uint32_t)(q4 * 32) << 16);
      for (int c0 = half * (HB / 2); c0 < (half + 1) * (HB / 2); c0 += 32) {
        float h1[32], h2[32];
        tmem_ld32(lane_addr + c0, h1);
        tmem_ld32(lane_addr + HB + c0, h2);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int hidden = hb * HB + c0 + j;
          const float g = h1[j] / (1.0f + expf(-h1[j])) * h2[j];
          z0 = fmaf(g, __ldg(W3 + hidden * 3 + 0), z0);
          z1 = fmaf(g, __ldg(W3 + hidden * 3 + 1), z1);
          z2 = fmaf(g, __ldg(W3 + hidden * 3 + 2), z2);
        }
      }
    }
    const int row = q4 * 32 + lane;
    float* zs = reinterpret_cast<float*>(stages);
    if (half == 1) {
      zs[3 * row + 0] = z0;
      zs[3 * row + 1] = z1;
      zs[3 * row + 2] = z2;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kTcProd) : "memory");  // producer warps only
    if (half == 0 && run) {
      const int64_t tok = m0 + row;
      z0 += zs[3 * row + 0];
      z1 += zs[3 * row + 1];
      z2 += zs[3 * row + 2];
      if (tok < T) zpart[tok * nhb + hb] = make_float4(z0, z1, z2, 0.f);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

// CTA (sequence b, block of 8 chunks), one warp per chunk: sum the hidden-block partial
// scores, add the bias, take each token's argmax (ties -> lower index = more
// bits), write them, and take the chunk's majority (ties -> more bits);
// chunk 0 is frozen to FP16 when asked (路由冻结).
__global__ void finish_vote_kernel(const int64_t* __restrict__ cu, int L,
                                   const float4* __restrict__ zpart, int nhb,
                                   const float* __restrict__ b3, int routing_freeze,
                                   uint8_t* __restrict__ token_expert, float* __restrict__ logits,
                                   uint8_t* __restrict__ chunk_expert) {
  __shared__ int64_t red[32];
  const int b = blockIdx.x;
  const int64_t row0 = cu[b];
  const int64_t Tb = cu[b + 1] - row0;
  const int64_t nb = (Tb + L - 1) / L;
  const int nw = blockDim.x / 32;
  if ((int64_t)blockIdx.y * nw >= nb) return;  // uniform for the whole block
  const int64_t coff = block_chunk_offset(b, cu, L, red);
  const int lane = threadIdx.x & 31, warp = threadIdx.x / 32 + blockIdx.y * nw;
  float bias0 = 0.f, bias1 = 0.f, bias2 = 0.f;
  if (b3) {
    bias0 = b3[0];
    bias1 = b3[1];
    bias2 = b3[2];
  }
  for (int64_t c = warp; c < nb; c += (int64_t)nw * gridDim.y) {
    const int64_t t0 = c * L;
    const int64_t t1 = min(t0 + (int64_t)L, Tb);
    int cnt[kNumExperts] = {0, 0, 0};
    for (int64_t t = t0; t < t1; t += 32) {
      const bool in = t + lane < t1;
      int e = -1;
      if (in) {
        const int64_t tok = row0 + t + lane;
        float z[3] = {0.f, 0.f, 0.f};
        for (int h = 0; h < nhb; ++h) {
          const float4 p = zpart[tok * nhb + h];
          z[0] += p.x;
          z[1] += p.y;
          z[2] += p.z;
        }
        z[0] += bias0;
        z[1] += bias1;
        z[2] += bias2;
        e = 0;
        if (z[1] > z[e]) e = 1;
        if (z[2] > z[e]) e = 2;
        token_expert[tok] = (uint8_t)e;
        if (logits) {
          logits[tok * 3 + 0] = z[0];
          logits[tok * 3 + 1] = z[1];
          logits[tok * 3 + 2] = z[2];
        }
      }
      cnt[0] += __popc(__ballot_sync(0xffffffffu, e == 0));
      cnt[1] += __popc(__ballot_sync(0xffffffffu, e == 1));
      cnt[2] += __popc(__ballot_sync(0xffffffffu, e == 2));
    }
    int win = 0;
    if (cnt[1] > cnt[win]) win = 1;
    if (cnt[2] > cnt[win]) win = 2;
    if (routing_freeze && c == 0) win = 0;
    if (lane == 0) chunk_expert[coff + c] = (uint8_t)win;
  }
}

template <int BN>
cudaError_t launch_tc(const float* C, int64_t T, int D, int H, const float* W1, const float* W2,
                      const float* W3, unsigned char* Wp, float4* zpart, unsigned int* status,
                      cudaStream_t stream) {
  // the test hook (mq_debug_arm_wait_timeout) applies to one launch
  const bool inject = debug_take(MQ_DEBUG_ROUTER);
  const int nkt = (D + kTcKE - 1) / kTcKE;
  const int nhb = H / (BN / 2);
  prepack_weights_kernel<BN><<<dim3(nkt, nhb), 256, 0, stream>>>(W1, W2, D, H, nkt, Wp);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (T == 0) return cudaSuccess;
  const size_t smem = TcSmem<BN>::TOTAL;
  if ((err = cudaFuncSetAttribute(router_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
    return err;
  const dim3 grid((unsigned)(((T + kTcBM - 1) / kTcBM) * nhb));
  router_tc_kernel<BN><<<grid, kTcThreads, smem, stream>>>(C, T, D, nkt, Wp, W3, zpart, nhb, status,
                                                            inject ? kTcTestWaitLimit : kTcWaitLimit,
                                                            inject ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

size_t route_workspace_bytes(int64_t T, int D, int H) {
  const int BN = H >= 128 ? 256 : 128;
  const int nhb = H / (BN / 2);
  const int nkt = (D + kTcKE - 1) / kTcKE;
  const size_t wp = (size_t)nhb * nkt * 2 * BN * 128;
  return (size_t)align128(wp) + (size_t)align128((uint64_t)T * nhb * 16) + 1024;
}

cudaError_t launch_router_tc(const float* C, int64_t T, int D, int H, const float* W1,
                             const float* W2, const float* W3, void* workspace,
                             unsigned int* status, cudaStream_t stream, const float4** zpart_out,
                             int* nhb_out) {
  const int BN = H >= 128 ? 256 : 128;
  const int nhb = H / (BN / 2);
  const int nkt = (D + kTcKE - 1) / kTcKE;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  unsigned char* Wp = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(ws) + 1023) & ~uintptr_t(1023));
  const size_t wp = (size_t)nhb * nkt * 2 * BN * 128;
  float4* zpart = reinterpret_cast<float4*>(Wp + align128(wp));
  *zpart_out = zpart;
  *nhb_out = nhb;
  if (BN == 256) return launch_tc<256>(C, T, D, H, W1, W2, W3, Wp, zpart, status, stream);
  return launch_tc<128>(C, T, D, H, W1, W2, W3, Wp, zpart, status, stream);
}

cudaError_t launch_finish_vote(int B, const int64_t* cu_seqlens, int L, int64_t max_chunks,
                               const float4* zpart, int nhb, const float* b3, int routing_freeze,
                               uint8_t* token_expert, float* logits, uint8_t* chunk_expert,
                               cudaStream_t stream) {
  const int64_t chunk_blocks = max_chunks > 0 ? (max_chunks + 7) / 8 : 1;  // 8 warps a block
  finish_vote_kernel<<<dim3(B, (unsigned)chunk_blocks), 256, 0, stream>>>(
      cu_seqlens, L, zpart, nhb, b3, routing_freeze, token_expert, logits, chunk_expert);
  return cudaGetLastError();
}

}  // namespace mqkv
