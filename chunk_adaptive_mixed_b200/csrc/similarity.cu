// similarity.cu — chunk-level quantization search by chunk–query similarity.
//
// Cocktail abstract (scholarfeed "Bin Zhang" author page): the bitwidth of each
// context chunk is chosen from the similarity between that chunk and the query.
// The page defines neither the similarity nor the cut-offs; the reading built
// here (stated in include/mqkv.h) is the cosine between the chunk's mean router
// input row and one query vector per sequence, cut at two caller thresholds.
//
// One CTA per chunk streams the chunk's L x D block of C once (the only HBM
// traffic of any size), summing each column in fp64.  The cosine is
//   sum_k S_k u_k / sqrt(sum_k S_k^2 * sum_k u_k^2),  S = column sums,
// which equals the cosine of the mean (the 1/n factors cancel), so the
// threshold test is taken in fp64 like the CPU oracle's.
#include "common.cuh"

namespace mqkv {
namespace {

constexpr int kSimThreads = 256;
constexpr int kSimUnroll = 8;

__device__ inline void add4(double (&a)[4], const float4 v) {
  a[0] += (double)v.x;
  a[1] += (double)v.y;
  a[2] += (double)v.z;
  a[3] += (double)v.w;
}

__global__ void __launch_bounds__(kSimThreads)
similarity_route_kernel(const float* __restrict__ C, int D, const float* __restrict__ u,
                        const int64_t* __restrict__ cu, int L, double tau_hi, double tau_lo,
                        int routing_freeze, uint8_t* __restrict__ chunk_expert,
                        double* __restrict__ similarity) {
  __shared__ int64_t red_i[33];
  __shared__ double red[3][kSimThreads / 32];
  const int b = blockIdx.y;
  const int c = blockIdx.x;
  const int64_t row0 = cu[b];
  const int64_t Tb = cu[b + 1] - row0;
  const int64_t nb = (Tb + L - 1) / L;
  if (c >= nb) return;  // uniform over the block
  const int64_t off = block_chunk_offset(b, cu, L, red_i);

  const int64_t t0 = (int64_t)c * L;
  const int n = (int)((t0 + L < Tb ? t0 + L : Tb) - t0);
  const float4* base = reinterpret_cast<const float4*>(C + (row0 + t0) * (int64_t)D);
  const float4* ub = reinterpret_cast<const float4*>(u + (int64_t)b * D);
  const int D4 = D / 4;

  double dot = 0.0, ss = 0.0, uu = 0.0;
  for (int j = threadIdx.x; j < D4; j += kSimThreads) {
    double s[4] = {0.0, 0.0, 0.0, 0.0};
    const float4* p = base + j;
    int t = 0;
    for (; t + kSimUnroll <= n; t += kSimUnroll) {
      float4 v[kSimUnroll];
#pragma unroll
      for (int i = 0; i < kSimUnroll; ++i) v[i] = __ldcs(p + (int64_t)(t + i) * D4);
#pragma unroll
      for (int i = 0; i < kSimUnroll; ++i) add4(s, v[i]);
    }
    for (; t < n; ++t) add4(s, __ldcs(p + (int64_t)t * D4));
    const float4 w = __ldg(ub + j);
    dot += s[0] * (double)w.x + s[1] * (double)w.y + s[2] * (double)w.z + s[3] * (double)w.w;
    ss += s[0] * s[0] + s[1] * s[1] + s[2] * s[2] + s[3] * s[3];
    uu += (double)w.x * w.x + (double)w.y * w.y + (double)w.z * w.z + (double)w.w * w.w;
  }
  for (int o = 16; o > 0; o >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    uu += __shfl_xor_sync(0xffffffffu, uu, o);
  }
  const int warp = threadIdx.x / 32;
  if ((threadIdx.x & 31) == 0) {
    red[0][warp] = dot;
    red[1][warp] = ss;
    red[2][warp] = uu;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, m = 0.0, q = 0.0;
    for (int w = 0; w < kSimThreads / 32; ++w) {
      a += red[0][w];
      m += red[1][w];
      q += red[2][w];
    }
    const double sim = (m > 0.0 && q > 0.0) ? a / sqrt(m * q) : 0.0;
    int e = sim >= tau_hi ? 0 : (sim >= tau_lo ? 1 : 2);
    if (routing_freeze && c == 0) e = 0;
    chunk_expert[off + c] = (uint8_t)e;
    if (similarity) similarity[off + c] = sim;
  }
}

}  // namespace

cudaError_t launch_similarity_route(int B, const int64_t* cu_seqlens, int L, int64_t max_chunks,
                                    const float* C, int D, const float* u, double tau_hi,
                                    double tau_lo, int routing_freeze, uint8_t* chunk_expert,
                                    double* similarity, cudaStream_t stream) {
  if (max_chunks == 0) return cudaSuccess;
  const dim3 grid((unsigned)max_chunks, (unsigned)B);
  similarity_route_kernel<<<grid, kSimThreads, 0, stream>>>(C, D, u, cu_seqlens, L, tau_hi,
                                                            tau_lo, routing_freeze, chunk_expert,
                                                            similarity);
  return cudaGetLastError();
}

}  // namespace mqkv
