// route.cu — router scores, per-token argmax, per-chunk vote, routing freezing.
//
// MoQAE paper notes, 关键设计 › Quantization-Aware Experts: every token of a
// chunk C is scored against the quantisation experts {FP16, INT4, INT2} by a
// small MLP printed as f(CW1·CW2)W3; this library evaluates it as
//     z_t = (SiLU(C_t W1) ⊙ (C_t W2)) W3 + b3          (fp32 throughout)
// and takes the per-token argmax (ties -> lower index = more bits).
// 方法详解 › 整体框架: the chunk's bitwidth is the majority of its tokens'
// choices (ties -> more bits).  路由冻结 (Routing Freezing): chunk 0 of every
// sequence is forced to FP16.
//
// router_kernel: one CTA computes BM=64 tokens x all H hidden units of both
// branches (a 64 x 2H output tile) with fp32 FFMA, K-loop over D in steps of
// 16 with double-buffered shared memory; the gate, the H x 3 projection, the
// bias and the argmax run in the epilogue, so the [T, 2H] hidden activations
// never reach HBM.  C is read exactly once.
#include "common.cuh"

namespace mqkv {
namespace {

constexpr int kBM = 64;
constexpr int kBK = 16;
constexpr int kRouterThreads = 256;
constexpr int kTM = 8;  // tokens per thread (kBM / (kRouterThreads / 32))

// Column of hidden unit i (0 <= i < HC) owned by lane hc; groups of 4
// consecutive columns per lane, 128 columns apart, keep 128-bit shared loads
// conflict-free.
template <int HC>
__device__ __forceinline__ int hidden_col(int hc, int i) {
  constexpr int V = HC < 4 ? HC : 4;
  return (i / 4) * 128 + hc * V + (i % 4);
}

template <int H>
struct RouterSmem {
  float As[2][kBK][kBM];  // C tile, transposed ([k][token])
  float B1[2][kBK][H];
  float B2[2][kBK][H];
};

template <int H>
__global__ void __launch_bounds__(kRouterThreads, 1)
router_kernel(const float* __restrict__ C, int64_t T, int D, const float* __restrict__ W1,
              const float* __restrict__ W2, const float* __restrict__ W3,
              const float* __restrict__ b3, uint8_t* __restrict__ token_expert,
              float* __restrict__ logits) {
  constexpr int HC = H / 32;            // hidden units per thread per branch
  constexpr int V = HC < 4 ? HC : 4;    // floats per vector access of B rows
  constexpr int BQ = kBK * H / 4;       // float4s in one B tile
  constexpr int BLOADS = BQ / kRouterThreads;
  static_assert(BQ % kRouterThreads == 0, "B tile load split");

  extern __shared__ __align__(16) unsigned char smem_raw[];
  RouterSmem<H>& sm = *reinterpret_cast<RouterSmem<H>*>(smem_raw);

  const int tid = threadIdx.x;
  const int tm = tid / 32;  // token row block (warp)
  const int hc = tid % 32;  // hidden column lane
  const int64_t m0 = (int64_t)blockIdx.x * kBM;

  // global -> register staging
  const int a_row = tid / 4, a_kq = tid % 4;
  float4 ra;
  float4 rb1[BLOADS], rb2[BLOADS];

  auto load_tiles = [&](int k0) {
    const int64_t row = m0 + a_row;
    const int kc = k0 + 4 * a_kq;
    if (row < T && kc < D)
      ra = __ldg(reinterpret_cast<const float4*>(C + row * (int64_t)D + kc));
    else
      ra = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < BLOADS; ++r) {
      const int idx = tid + r * kRouterThreads;
      const int k = idx / (H / 4), jq = idx % (H / 4);
      if (k0 + k < D) {
        rb1[r] = __ldg(reinterpret_cast<const float4*>(W1 + (int64_t)(k0 + k) * H) + jq);
        rb2[r] = __ldg(reinterpret_cast<const float4*>(W2 + (int64_t)(k0 + k) * H) + jq);
      } else {
        rb1[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        rb2[r] = rb1[r];
      }
    }
  };
  auto store_tiles = [&](int buf) {
    sm.As[buf][4 * a_kq + 0][a_row] = ra.x;
    sm.As[buf][4 * a_kq + 1][a_row] = ra.y;
    sm.As[buf][4 * a_kq + 2][a_row] = ra.z;
    sm.As[buf][4 * a_kq + 3][a_row] = ra.w;
#pragma unroll
    for (int r = 0; r < BLOADS; ++r) {
      const int idx = tid + r * kRouterThreads;
      const int k = idx / (H / 4), jq = idx % (H / 4);
      reinterpret_cast<float4*>(&sm.B1[buf][k][0])[jq] = rb1[r];
      reinterpret_cast<float4*>(&sm.B2[buf][k][0])[jq] = rb2[r];
    }
  };

  float acc1[kTM][HC], acc2[kTM][HC];
#pragma unroll
  for (int r = 0; r < kTM; ++r)
#pragma unroll
    for (int i = 0; i < HC; ++i) { acc1[r][i] = 0.f; acc2[r][i] = 0.f; }

  const int nk = (D + kBK - 1) / kBK;
  load_tiles(0);
  store_tiles(0);
  __syncthreads();
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) load_tiles((kt + 1) * kBK);
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[kTM];
      const float4 a0 = *reinterpret_cast<const float4*>(&sm.As[buf][kk][tm * kTM]);
      const float4 a1 = *reinterpret_cast<const float4*>(&sm.As[buf][kk][tm * kTM + 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
      a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      float b1[HC], b2[HC];
#pragma unroll
      for (int v = 0; v < HC / V; ++v) {
        const int col = hidden_col<HC>(hc, v * 4);
        if constexpr (V == 4) {
          const float4 x1 = *reinterpret_cast<const float4*>(&sm.B1[buf][kk][col]);
          const float4 x2 = *reinterpret_cast<const float4*>(&sm.B2[buf][kk][col]);
          b1[v * 4 + 0] = x1.x; b1[v * 4 + 1] = x1.y; b1[v * 4 + 2] = x1.z; b1[v * 4 + 3] = x1.w;
          b2[v * 4 + 0] = x2.x; b2[v * 4 + 1] = x2.y; b2[v * 4 + 2] = x2.z; b2[v * 4 + 3] = x2.w;
        } else {
          const float2 x1 = *reinterpret_cast<const float2*>(&sm.B1[buf][kk][col]);
          const float2 x2 = *reinterpret_cast<const float2*>(&sm.B2[buf][kk][col]);
          b1[0] = x1.x; b1[1] = x1.y;
          b2[0] = x2.x; b2[1] = x2.y;
        }
      }
#pragma unroll
      for (int r = 0; r < kTM; ++r)
#pragma unroll
        for (int i = 0; i < HC; ++i) {
          acc1[r][i] = fmaf(a[r], b1[i], acc1[r][i]);
          acc2[r][i] = fmaf(a[r], b2[i], acc2[r][i]);
        }
    }
    if (kt + 1 < nk) {
      // buf ^ 1 was last read in iteration kt - 1, which every thread finished
      // before the barrier that closed it
      store_tiles(buf ^ 1);
      __syncthreads();
    }
  }

  // epilogue: gate, projection to 3 experts, bias, argmax
  float w3[HC][kNumExperts];
#pragma unroll
  for (int i = 0; i < HC; ++i) {
    const int j = hidden_col<HC>(hc, i);
#pragma unroll
    for (int e = 0; e < kNumExperts; ++e) w3[i][e] = __ldg(W3 + j * kNumExperts + e);
  }
  float bias[kNumExperts] = {0.f, 0.f, 0.f};
  if (b3) {
#pragma unroll
    for (int e = 0; e < kNumExperts; ++e) bias[e] = __ldg(b3 + e);
  }
#pragma unroll
  for (int r = 0; r < kTM; ++r) {
    float z[kNumExperts] = {0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < HC; ++i) {
      const float h1 = acc1[r][i];
      const float g = h1 / (1.0f + expf(-h1)) * acc2[r][i];
#pragma unroll
      for (int e = 0; e < kNumExperts; ++e) z[e] = fmaf(g, w3[i][e], z[e]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int e = 0; e < kNumExperts; ++e) z[e] += __shfl_xor_sync(0xffffffffu, z[e], off);
    const int64_t tok = m0 + tm * kTM + r;
    if (hc == 0 && tok < T) {
#pragma unroll
      for (int e = 0; e < kNumExperts; ++e) z[e] += bias[e];
      int best = 0;
      if (z[1] > z[best]) best = 1;
      if (z[2] > z[best]) best = 2;
      token_expert[tok] = (uint8_t)best;
      if (logits) {
        logits[tok * 3 + 0] = z[0];
        logits[tok * 3 + 1] = z[1];
        logits[tok * 3 + 2] = z[2];
      }
    }
  }
}

// One CTA per sequence; one warp per chunk: count the tokens' choices with
// ballots, take the majority (ties -> more bits), freeze chunk 0.
__global__ void vote_kernel(const int64_t* __restrict__ cu, int L,
                            const uint8_t* __restrict__ token_expert, int routing_freeze,
                            uint8_t* __restrict__ chunk_expert, unsigned int* status) {
  __shared__ int64_t red[32];
  const int b = blockIdx.x;
  const int64_t coff = block_chunk_offset(b, cu, L, red);
  const int64_t row0 = cu[b];
  const int64_t Tb = cu[b + 1] - row0;
  const int64_t nb = (Tb + L - 1) / L;
  const int lane = threadIdx.x & 31, warp = threadIdx.x / 32, nw = blockDim.x / 32;
  for (int64_t c = warp; c < nb; c += nw) {
    const int64_t t0 = c * L;
    const int64_t t1 = min(t0 + (int64_t)L, Tb);
    int cnt[kNumExperts] = {0, 0, 0};
    for (int64_t t = t0; t < t1; t += 32) {
      const bool in = t + lane < t1;
      const int e = in ? token_expert[row0 + t + lane] : -1;
      if (in && e > 2) set_status(status, MQ_DEV_INDEX_RANGE);
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

template <int H>
cudaError_t launch_router_h(const float* C, int64_t T, int D, const float* W1, const float* W2,
                            const float* W3, const float* b3, uint8_t* token_expert,
                            float* logits, cudaStream_t stream) {
  const size_t smem = sizeof(RouterSmem<H>);
  cudaError_t err = cudaFuncSetAttribute(router_kernel<H>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int64_t grid = (T + kBM - 1) / kBM;
  if (grid == 0) return cudaSuccess;
  router_kernel<H><<<(unsigned)grid, kRouterThreads, smem, stream>>>(C, T, D, W1, W2, W3, b3,
                                                                      token_expert, logits);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const float* C, int64_t T, int D, int H, const float* W1,
                          const float* W2, const float* W3, const float* b3,
                          uint8_t* token_expert, float* logits, cudaStream_t stream) {
  switch (H) {
    case 64: return launch_router_h<64>(C, T, D, W1, W2, W3, b3, token_expert, logits, stream);
    case 128: return launch_router_h<128>(C, T, D, W1, W2, W3, b3, token_expert, logits, stream);
    case 256: return launch_router_h<256>(C, T, D, W1, W2, W3, b3, token_expert, logits, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_vote(int B, const int64_t* cu_seqlens, int L, const uint8_t* token_expert,
                        int routing_freeze, uint8_t* chunk_expert, unsigned int* status,
                        cudaStream_t stream) {
  vote_kernel<<<B, 256, 0, stream>>>(cu_seqlens, L, token_expert, routing_freeze, chunk_expert,
                                     status);
  return cudaGetLastError();
}

}  // namespace mqkv
