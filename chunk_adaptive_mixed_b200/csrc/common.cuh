// common.cuh — internal helpers shared by the libmqkv translation units.
//
// Nothing here is part of the public ABI (include/mqkv.h).  Kernels report
// device-side failures by OR-ing MQ_DEV_* bits into a status word whose
// address the launcher passes in; they never trap.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mqkv.h"
#include "mqkv_debug.h"

namespace mqkv {

constexpr int kNumExperts = 3;
constexpr int kGroup = 32;
// merge slices per (sequence, query head) in the decode combine, at most
constexpr int kSplitMax = 8;

__host__ __device__ constexpr int expert_bits(int e) { return e == 0 ? 16 : (e == 1 ? 4 : 2); }

__host__ __device__ inline uint64_t align128(uint64_t x) { return (x + 127) & ~uint64_t(127); }
__host__ __device__ inline uint64_t align16(uint64_t x) { return (x + 15) & ~uint64_t(15); }

// Byte offsets inside the layout blob (see include/mqkv.h).
__host__ __device__ inline size_t layout_seq_offset(int b) {
  return sizeof(mq_layout_header) + (size_t)b * sizeof(mq_seq_layout);
}
__host__ __device__ inline size_t layout_perm_offset(int B) { return layout_seq_offset(B); }
__host__ __device__ inline size_t layout_inv_offset(int B, int64_t N) {
  return layout_perm_offset(B) + (size_t)align16((uint64_t)N * 4);
}
__host__ __device__ inline size_t layout_total_bytes(int B, int64_t N) {
  return layout_inv_offset(B, N) + (size_t)align16((uint64_t)N * 4);
}

// Bytes of one row (token) of codes for one kv-head at expert e.
__host__ __device__ inline uint32_t code_row_bytes(int d, int e) {
  return (uint32_t)(d * expert_bits(e) / 8);
}
// Bytes of one row of (scale, min) pairs (INT experts only).
__host__ __device__ inline uint32_t scale_row_bytes(int d) { return (uint32_t)(d / kGroup * 4); }

__device__ inline void set_status(unsigned int* status, unsigned int bits) {
  if (status) atomicOr(status, bits);
}

// Sum over sequences b' < b of ceil(T_b' / L), computed by the whole block
// (blockDim.x a multiple of 32, red holds >= 32 entries).
__device__ inline int64_t block_chunk_offset(int b, const int64_t* cu, int L, int64_t* red) {
  int64_t part = 0;
  for (int i = threadIdx.x; i < b; i += blockDim.x) {
    const int64_t Tb = cu[i + 1] - cu[i];
    part += (Tb + L - 1) / L;
  }
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = part;
  __syncthreads();
  int64_t total = 0;
  for (int w = 0; w < (int)(blockDim.x / 32); ++w) total += red[w];
  __syncthreads();
  return total;
}

// Exclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024);
// *total receives the block's sum.  red holds >= 32 entries.
template <typename T>
__device__ inline T block_exclusive_scan(T v, T* red, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x / 32;
  T incl = v;
  for (int off = 1; off < 32; off <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) red[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x / 32;
    T w = lane < nw ? red[lane] : T(0);
    T wi = w;
    for (int off = 1; off < 32; off <<= 1) {
      const T y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    red[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) red[32] = wi;
  }
  __syncthreads();
  const T out = red[warp] + incl - v;
  *total = red[32];
  __syncthreads();
  return out;
}

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error; arguments are pre-validated.

// Decode work split: tokens per work item of each segment (implementation
// defined; depends only on the shape and the lengths).
struct ItemPolicy {
  int item_tokens[kNumExperts];
};
ItemPolicy item_policy(const mq_shape& s, const int32_t* h_seq_lens);
int64_t max_items_per_kv_head(const mq_shape& s, const int32_t* h_seq_lens, const ItemPolicy& p);

// Router on tcgen05 (3 x TF32): weights pre-split into the workspace, then
// per-hidden-block partial scores; finish_vote sums them, adds the bias, takes
// the argmax and the chunk vote.
size_t route_workspace_bytes(int64_t T, int D, int H);
// Test hook (include/mqkv_debug.h): true once after the kernel's bit was armed.
bool debug_take(uint32_t kernel_bit);

cudaError_t launch_router_tc(const float* C, int64_t T, int D, int H, const float* W1,
                             const float* W2, const float* W3, void* workspace,
                             unsigned int* status, cudaStream_t stream, const float4** zpart_out,
                             int* nhb_out);
cudaError_t launch_finish_vote(int B, const int64_t* cu_seqlens, int L, int64_t max_chunks,
                               const float4* zpart, int nhb, const float* b3, int routing_freeze,
                               uint8_t* token_expert, float* logits, uint8_t* chunk_expert,
                               cudaStream_t stream);
// Chunk-level search by chunk-query cosine (fp64), grid (max_chunks, B).
cudaError_t launch_similarity_route(int B, const int64_t* cu_seqlens, int L, int64_t max_chunks,
                                    const float* C, int D, const float* u, double tau_hi,
                                    double tau_lo, int routing_freeze, uint8_t* chunk_expert,
                                    double* similarity, cudaStream_t stream);
// grow < 0: fixed layout over total_slots = N chunks; grow >= 0: growable,
// total_slots = N + B * (grow + 1).
cudaError_t launch_layout(const mq_shape& s, const int64_t* cu_seqlens, const uint8_t* chunk_expert,
                          int64_t total_slots, const ItemPolicy& pol, int grow, void* layout,
                          unsigned int* status, cudaStream_t stream);
// Growth steps of a growable layout (sealed: device uint8[B] or NULL).
cudaError_t launch_grow_commit(const mq_shape& s, const uint8_t* sealed, int add, void* layout,
                               unsigned int* status, cudaStream_t stream);
cudaError_t launch_grow_seal(const mq_shape& s, const void* layout, const uint8_t* sealed,
                             void* packed, uint64_t packed_bytes, unsigned int* status,
                             cudaStream_t stream);
cudaError_t launch_grow_append(const mq_shape& s, const void* layout, const void* K_new,
                               const void* V_new, int kv_dtype, void* packed,
                               uint64_t packed_bytes, unsigned int* status, cudaStream_t stream);
cudaError_t launch_pack(const mq_shape& s, int64_t total_chunks, const void* layout, const void* K,
                        const void* V, int kv_dtype, void* packed, uint64_t packed_bytes,
                        unsigned int* status, cudaStream_t stream);
// partial: write context-shard records [B, Hq, d + 4] instead of the output.
cudaError_t launch_decode(const mq_shape& s, int64_t max_items, const void* layout,
                          const void* packed, const void* q, int q_dtype, float softmax_scale,
                          float* out, void* workspace, size_t workspace_bytes,
                          unsigned int* status, cudaStream_t stream, bool partial = false);
// Per-item partial results of decode on the tensor cores (one query head per
// kv-head, fp16 queries, head_dim 128): the same workspace records as the
// CUDA-core kernel; the counter is zeroed on the stream first.
cudaError_t launch_decode_mha(int64_t capacity_items, const unsigned char* layout,
                              const unsigned char* packed, const __half* q, float scale_log2,
                              float* ws_acc, float2* ws_ml, unsigned int* counter, int* tab, int B, int Hq,
                              unsigned int* status, cudaStream_t stream);
// The same for four query heads per kv-head (decode_gqa.cu).
cudaError_t launch_decode_gqa4(int64_t capacity_items, const unsigned char* layout,
                               const unsigned char* packed, const __half* q, float scale_log2,
                               float* ws_acc, float2* ws_ml, unsigned int* counter, int* tab, int B, int Hq,
                               unsigned int* status, cudaStream_t stream);
cudaError_t launch_combine_partials(int P, int B, int Hq, int D, const float* parts, float* out,
                                    cudaStream_t stream);

// Records a formatted reason for mq_last_error() and returns `status`.
mq_status report_error(mq_status status, const char* fmt, ...);

// Workspace layout of mq_decode_attn for a given item bound.
size_t decode_workspace_bytes(const mq_shape& s, int64_t max_items);

}  // namespace mqkv
