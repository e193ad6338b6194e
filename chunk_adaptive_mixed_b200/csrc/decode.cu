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
// decode_partial_kernel — persistent CTAs walk the work items of the layout's
// schedule.  A work item is (sequence b, segment s, kv-head g, token range of
// at most item_tokens[s] tokens); its four byte ranges (K codes, K scales,
// V codes, V scales) are staged into shared memory with 1-D TMA bulk copies
// completing on an mbarrier.  Then, for the Hq/Hkv query heads of g:
//   scores: one thread per (token, group of 32 dims); the group's dot product
//           uses the raw codes, dequantisation folded in per group:
//           q . khat = s * (q . code) + min * sum(q)
//   softmax: per head max / exp2 / sum over the item (log2 domain)
//   values:  one thread per (token lane, 8-dim slice); accumulates p*s*code
//           and p*min per group, reduced across token lanes in shared memory
//   partial: (m, l, acc[d]) per head to the workspace.
// decode_combine_kernel — one warp per (b, query head) merges the partials of
// all items of (b, g) with the usual max-rescaling.
#include "common.cuh"

namespace mqkv {
namespace {

constexpr int kDecThreads = 128;
constexpr int kStageBytes = 32768;
constexpr int kMaxScores = 2048;  // QPG * tokens of one item
constexpr int kMaxQpg = 8;
constexpr uint32_t kWaitLimit = 1u << 22;

struct DecodeSmem {
  alignas(128) unsigned char stage[kStageBytes + 64];
  alignas(16) float q[kMaxQpg][4][36];  // [head][group][dim], rows padded
  float qsum[kMaxQpg][4];
  float sc[kMaxScores];  // scores, then probabilities, [head][token]
  float m[kMaxQpg];
  float l[kMaxQpg];
  alignas(8) unsigned long long bar;
  int info[8];  // b, s, n, g, kc_off, ks_off, vc_off, vs_off (stage offsets)
  int abort_flag;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(unsigned long long* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(unsigned long long* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait; returns false when the limit was reached.
__device__ __forceinline__ bool mbar_wait_bounded(unsigned long long* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
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

template <int D>
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

template <int D, int QPG, int QDT>
__global__ void __launch_bounds__(kDecThreads)
decode_partial_kernel(const unsigned char* __restrict__ layout,
                      const unsigned char* __restrict__ packed, const void* __restrict__ q,
                      float scale_log2, float* __restrict__ ws_acc, float2* __restrict__ ws_ml,
                      int64_t capacity_items, unsigned int* status) {
  constexpr int G = D / kGroup;
  constexpr int S = D / 8;                 // 8-dim slices
  constexpr int TL = kDecThreads / S;      // token lanes in the value pass
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DecodeSmem& sm = *reinterpret_cast<DecodeSmem*>(smem_raw);

  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  if (h->magic != MQ_LAYOUT_MAGIC || h->head_dim != D) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_BAD_LAYOUT);
    return;
  }
  const int B = h->num_seqs, Hkv = h->num_kv_heads, L = h->chunk_len;
  (void)L;
  const int64_t total = (int64_t)h->total_items * Hkv;
  if (total > capacity_items) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, MQ_DEV_WORKSPACE_TOO_SMALL);
    return;
  }
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&sm.bar, 1);
    fence_barrier_init();
    sm.abort_flag = 0;
  }
  __syncthreads();
  uint32_t parity = 0;

  for (int64_t w = blockIdx.x; w < total; w += gridDim.x) {
    if (tid == 0) {
      const int64_t bs = w / Hkv;
      const int g = (int)(w - bs * Hkv);
      const int b = find_item_seq<D>(layout, B, bs);
      const mq_seq_layout* r =
          reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(b));
      const int s = bs < r->item_begin[1] ? 0 : (bs < r->item_begin[2] ? 1 : 2);
      const int j = (int)(bs - r->item_begin[s]);
      const int it = h->item_tokens[s];
      const int t0 = j * it;
      const int n = min(it, r->seg_tokens[s] - t0);
      const uint32_t crow = code_row_bytes(D, s);
      const unsigned char* regk = packed + r->seg_base[s] + (uint64_t)g * r->region_bytes[s];
      const unsigned char* regv = regk + (uint64_t)Hkv * r->region_bytes[s];
      const uint32_t cbytes = (uint32_t)align16((uint64_t)n * crow);
      const uint32_t sbytes = s == 0 ? 0u : (uint32_t)align16((uint64_t)n * scale_row_bytes(D));
      const int kc = 0, ks = (int)cbytes, vc = (int)(cbytes + sbytes), vs = (int)(2 * cbytes + sbytes);
      if (n <= 0 || n * QPG > kMaxScores || 2 * (cbytes + sbytes) > (uint32_t)kStageBytes) {
        set_status(status, MQ_DEV_INDEX_RANGE);
        sm.info[2] = 0;
      } else {
        sm.info[2] = n;
      }
      sm.info[0] = b; sm.info[1] = s; sm.info[3] = g;
      sm.info[4] = kc; sm.info[5] = ks; sm.info[6] = vc; sm.info[7] = vs;
      if (sm.info[2] > 0) {
        fence_proxy_async_smem();
        mbar_expect_tx(&sm.bar, 2 * (cbytes + sbytes));
        bulk_copy_g2s(sm.stage + kc, regk + (uint64_t)t0 * crow, cbytes, &sm.bar);
        bulk_copy_g2s(sm.stage + vc, regv + (uint64_t)t0 * crow, cbytes, &sm.bar);
        if (s != 0) {
          const uint32_t srow = scale_row_bytes(D);
          bulk_copy_g2s(sm.stage + ks, regk + r->scale_offset[s] + (uint64_t)t0 * srow, sbytes,
                        &sm.bar);
          bulk_copy_g2s(sm.stage + vs, regv + r->scale_offset[s] + (uint64_t)t0 * srow, sbytes,
                        &sm.bar);
        }
      }
    }
    __syncthreads();
    const int b = sm.info[0], s = sm.info[1], n = sm.info[2], g = sm.info[3];
    if (n == 0) {
      __syncthreads();
      continue;
    }

    // query heads of this kv-head, as fp32, while the copy is in flight
    const int64_t qbase = ((int64_t)b * Hkv * QPG + (int64_t)g * QPG) * D;
    for (int i = tid; i < QPG * D; i += kDecThreads) {
      const int hh = i / D, dd = i - hh * D;
      float v;
      if constexpr (QDT == MQ_F16)
        v = __half2float(static_cast<const __half*>(q)[qbase + i]);
      else
        v = static_cast<const float*>(q)[qbase + i];
      sm.q[hh][dd / kGroup][dd % kGroup] = v;
    }
    __syncthreads();
    if (tid < QPG * G) {
      const int hh = tid / G, k = tid % G;
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < kGroup; ++j) acc += sm.q[hh][k][j];
      sm.qsum[hh][k] = acc;
    }

    bool ok = mbar_wait_bounded(&sm.bar, parity);
    parity ^= 1u;
    if (!ok) {
      set_status(status, MQ_DEV_WAIT_TIMEOUT);
      atomicExch(&sm.abort_flag, 1);
      mbar_wait_bounded(&sm.bar, parity ^ 1u);  // give the copies one more chance to land
    }
    __syncthreads();
    if (sm.abort_flag) return;

    const unsigned char* st = sm.stage;
    // ---- scores
    {
      const int k = tid % G;
      // warp-uniform trip count: every lane of a warp runs every iteration,
      // because the group reduction below shuffles across the full warp
      for (int tb = (tid / 32) * (32 / G); tb < n; tb += kDecThreads / G) {
        const int t = tb + (tid & 31) / G;
        const bool valid = t < n;
        float part[QPG];
        if (!valid) {
#pragma unroll
          for (int hh = 0; hh < QPG; ++hh) part[hh] = 0.f;
        } else if (s == 0) {
          const uint4* src = reinterpret_cast<const uint4*>(st + sm.info[4] + t * (2 * D) + k * 64);
          float x[32];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 u = src[v];
            const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = half2_bits_to_float2(wds[i]);
              x[8 * v + 2 * i] = f.x;
              x[8 * v + 2 * i + 1] = f.y;
            }
          }
#pragma unroll
          for (int hh = 0; hh < QPG; ++hh) {
            float dot = 0.f;
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 qq = *reinterpret_cast<const float4*>(&sm.q[hh][k][4 * j4]);
              dot = fmaf(qq.x, x[4 * j4], dot);
              dot = fmaf(qq.y, x[4 * j4 + 1], dot);
              dot = fmaf(qq.z, x[4 * j4 + 2], dot);
              dot = fmaf(qq.w, x[4 * j4 + 3], dot);
            }
            part[hh] = dot;
          }
        } else {
          const uint32_t sp =
              *reinterpret_cast<const uint32_t*>(st + sm.info[5] + t * (D / kGroup * 4) + k * 4);
          const float2 sm2 = half2_bits_to_float2(sp);  // (scale, min)
          float x[32];
          if (s == 1) {
            const uint4 u = *reinterpret_cast<const uint4*>(st + sm.info[4] + t * (D / 2) + k * 16);
            const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd)
#pragma unroll
              for (int i = 0; i < 8; ++i) x[8 * wd + i] = code_to_float((wds[wd] >> (4 * i)) & 0xFu);
          } else {
            const uint2 u = *reinterpret_cast<const uint2*>(st + sm.info[4] + t * (D / 4) + k * 8);
            const uint32_t wds[2] = {u.x, u.y};
#pragma unroll
            for (int wd = 0; wd < 2; ++wd)
#pragma unroll
              for (int i = 0; i < 16; ++i) x[16 * wd + i] = code_to_float((wds[wd] >> (2 * i)) & 0x3u);
          }
#pragma unroll
          for (int hh = 0; hh < QPG; ++hh) {
            float dot = 0.f;
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 qq = *reinterpret_cast<const float4*>(&sm.q[hh][k][4 * j4]);
              dot = fmaf(qq.x, x[4 * j4], dot);
              dot = fmaf(qq.y, x[4 * j4 + 1], dot);
              dot = fmaf(qq.z, x[4 * j4 + 2], dot);
              dot = fmaf(qq.w, x[4 * j4 + 3], dot);
            }
            part[hh] = fmaf(sm2.x, dot, sm2.y * sm.qsum[hh][k]);
          }
        }
#pragma unroll
        for (int hh = 0; hh < QPG; ++hh) {
#pragma unroll
          for (int off = 1; off < G; off <<= 1) part[hh] += __shfl_xor_sync(0xffffffffu, part[hh], off);
          if (k == 0 && valid) sm.sc[hh * n + t] = part[hh] * scale_log2;
        }
      }
    }
    __syncthreads();
    // ---- softmax statistics per head (log2 domain)
    {
      const int warp = tid / 32, lane = tid & 31;
      for (int hh = warp; hh < QPG; hh += kDecThreads / 32) {
        float mx = -INFINITY;
        for (int t = lane; t < n; t += 32) mx = fmaxf(mx, sm.sc[hh * n + t]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float sum = 0.f;
        for (int t = lane; t < n; t += 32) {
          const float p = exp2f(sm.sc[hh * n + t] - mx);
          sm.sc[hh * n + t] = p;
          sum += p;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) {
          sm.m[hh] = mx;
          sm.l[hh] = sum;
        }
      }
    }
    __syncthreads();
    // ---- values
    float acc[QPG][8];
    {
      const int slice = tid % S, tl = tid / S;
      const int k = slice / 4;
      float bias[QPG];
#pragma unroll
      for (int hh = 0; hh < QPG; ++hh) {
        bias[hh] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[hh][i] = 0.f;
      }
      for (int t = tl; t < n; t += TL) {
        float x[8];
        if (s == 0) {
          const uint4 u = *reinterpret_cast<const uint4*>(st + sm.info[6] + t * (2 * D) + slice * 16);
          const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = half2_bits_to_float2(wds[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
          }
#pragma unroll
          for (int hh = 0; hh < QPG; ++hh) {
            const float p = sm.sc[hh * n + t];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[hh][i] = fmaf(p, x[i], acc[hh][i]);
          }
        } else {
          const uint32_t sp =
              *reinterpret_cast<const uint32_t*>(st + sm.info[7] + t * (D / kGroup * 4) + k * 4);
          const float2 sm2 = half2_bits_to_float2(sp);
          if (s == 1) {
            const uint32_t wd = *reinterpret_cast<const uint32_t*>(st + sm.info[6] + t * (D / 2) + slice * 4);
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = code_to_float((wd >> (4 * i)) & 0xFu);
          } else {
            const uint32_t wd = *reinterpret_cast<const unsigned short*>(st + sm.info[6] + t * (D / 4) + slice * 2);
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = code_to_float((wd >> (2 * i)) & 0x3u);
          }
#pragma unroll
          for (int hh = 0; hh < QPG; ++hh) {
            const float p = sm.sc[hh * n + t];
            const float ws = p * sm2.x;
            bias[hh] = fmaf(p, sm2.y, bias[hh]);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[hh][i] = fmaf(ws, x[i], acc[hh][i]);
          }
        }
      }
#pragma unroll
      for (int hh = 0; hh < QPG; ++hh)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[hh][i] += bias[hh];
    }
    __syncthreads();  // stage no longer needed: reuse it for the token-lane reduction
    {
      float* red = reinterpret_cast<float*>(sm.stage);  // [TL][QPG][D]
      const int slice = tid % S, tl = tid / S;
#pragma unroll
      for (int hh = 0; hh < QPG; ++hh) {
        float4* dst = reinterpret_cast<float4*>(red + ((size_t)tl * QPG + hh) * D + slice * 8);
        dst[0] = make_float4(acc[hh][0], acc[hh][1], acc[hh][2], acc[hh][3]);
        dst[1] = make_float4(acc[hh][4], acc[hh][5], acc[hh][6], acc[hh][7]);
      }
    }
    __syncthreads();
    {
      const float* red = reinterpret_cast<const float*>(sm.stage);
      float* dst = ws_acc + (size_t)w * QPG * D;
      for (int o = tid; o < QPG * D; o += kDecThreads) {
        float v = 0.f;
#pragma unroll
        for (int tl = 0; tl < TL; ++tl) v += red[(size_t)tl * QPG * D + o];
        dst[o] = v;
      }
      if (tid < QPG) ws_ml[(size_t)w * QPG + tid] = make_float2(sm.m[tid], sm.l[tid]);
    }
    __syncthreads();  // stage and scores are rewritten by the next item
  }
}

template <int D, int QPG>
__global__ void __launch_bounds__(128)
decode_combine_kernel(const unsigned char* __restrict__ layout, int Hq,
                      const float* __restrict__ ws_acc, const float2* __restrict__ ws_ml,
                      float* __restrict__ out) {
  constexpr int PER_LANE = D / 32;
  const mq_layout_header* h = reinterpret_cast<const mq_layout_header*>(layout);
  const int B = h->num_seqs, Hkv = h->num_kv_heads;
  const int64_t wg = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (wg >= (int64_t)B * Hq) return;
  const int b = (int)(wg / Hq), hq = (int)(wg % Hq);
  const int g = hq / QPG, hh = hq % QPG;
  const mq_seq_layout* r = reinterpret_cast<const mq_seq_layout*>(layout + layout_seq_offset(b));
  float* o = out + wg * D + lane * PER_LANE;
  const int i0 = r->item_begin[0];
  const int i1 = r->item_begin[2] + r->item_count[2];
  if (r->num_tokens == 0 || i1 <= i0) {
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) o[i] = 0.f;
    return;
  }
  float M = -INFINITY;
  for (int it = i0 + lane; it < i1; it += 32) M = fmaxf(M, ws_ml[((int64_t)it * Hkv + g) * QPG + hh].x);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float acc[PER_LANE];
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) acc[i] = 0.f;
  float l = 0.f;
  for (int it = i0; it < i1; ++it) {
    const int64_t wi = ((int64_t)it * Hkv + g) * QPG + hh;
    const float2 ml = ws_ml[wi];
    const float f = exp2f(ml.x - M);
    l = fmaf(f, ml.y, l);
    const float* a = ws_acc + wi * D + lane * PER_LANE;
    if constexpr (PER_LANE == 4) {
      const float4 v = *reinterpret_cast<const float4*>(a);
      acc[0] = fmaf(f, v.x, acc[0]); acc[1] = fmaf(f, v.y, acc[1]);
      acc[2] = fmaf(f, v.z, acc[2]); acc[3] = fmaf(f, v.w, acc[3]);
    } else {
      const float2 v = *reinterpret_cast<const float2*>(a);
      acc[0] = fmaf(f, v.x, acc[0]); acc[1] = fmaf(f, v.y, acc[1]);
    }
  }
  const float inv_l = 1.0f / l;
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) o[i] = acc[i] * inv_l;
}

template <int D, int QPG, int QDT>
cudaError_t launch_decode_t(int64_t max_items, int Hq, const unsigned char* layout,
                            const unsigned char* packed, const void* q, float scale_log2,
                            float* out, float* ws_acc, float2* ws_ml, int num_seqs,
                            unsigned int* status, cudaStream_t stream) {
  const size_t smem = sizeof(DecodeSmem);
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
  if (grid > cap) grid = cap;
  if (grid > 0) {
    kern<<<(unsigned)grid, kDecThreads, smem, stream>>>(layout, packed, q, scale_log2, ws_acc, ws_ml,
                                                         cap, status);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  const int64_t warps = (int64_t)num_seqs * Hq;
  decode_combine_kernel<D, QPG><<<(unsigned)((warps + 3) / 4), 128, 0, stream>>>(layout, Hq, ws_acc,
                                                                                ws_ml, out);
  return cudaGetLastError();
}

template <int D, int QDT>
cudaError_t dispatch_qpg(int qpg, int64_t max_items, int Hq, const unsigned char* layout,
                         const unsigned char* packed, const void* q, float scale_log2, float* out,
                         float* ws_acc, float2* ws_ml, int B, unsigned int* status,
                         cudaStream_t stream) {
  switch (qpg) {
    case 1: return launch_decode_t<D, 1, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, B, status, stream);
    case 2: return launch_decode_t<D, 2, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, B, status, stream);
    case 4: return launch_decode_t<D, 4, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, B, status, stream);
    case 8: return launch_decode_t<D, 8, QDT>(max_items, Hq, layout, packed, q, scale_log2, out, ws_acc, ws_ml, B, status, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t decode_workspace_bytes(const mq_shape& s, int64_t max_items) {
  const int64_t qpg = s.num_q_heads / s.num_kv_heads;
  const int64_t recs = max_items * s.num_kv_heads * qpg;
  return (size_t)align128((uint64_t)recs * s.head_dim * 4) + (size_t)align128((uint64_t)recs * 8);
}

cudaError_t launch_decode(const mq_shape& s, int64_t max_items, const void* layout,
                          const void* packed, const void* q, int q_dtype, float softmax_scale,
                          float* out, void* workspace, size_t workspace_bytes,
                          unsigned int* status, cudaStream_t stream) {
  (void)workspace_bytes;
  const int64_t qpg = s.num_q_heads / s.num_kv_heads;
  const int64_t recs = max_items * s.num_kv_heads * qpg;
  float* ws_acc = static_cast<float*>(workspace);
  float2* ws_ml = reinterpret_cast<float2*>(static_cast<unsigned char*>(workspace) +
                                            align128((uint64_t)recs * s.head_dim * 4));
  const float scale_log2 = softmax_scale * 1.4426950408889634f;
  const unsigned char* lay = static_cast<const unsigned char*>(layout);
  const unsigned char* pk = static_cast<const unsigned char*>(packed);
  const int64_t cap = max_items * s.num_kv_heads;
  if (s.head_dim == 128) {
    if (q_dtype == MQ_F16)
      return dispatch_qpg<128, MQ_F16>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, s.num_seqs, status, stream);
    return dispatch_qpg<128, MQ_F32>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, s.num_seqs, status, stream);
  }
  if (q_dtype == MQ_F16)
    return dispatch_qpg<64, MQ_F16>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, s.num_seqs, status, stream);
  return dispatch_qpg<64, MQ_F32>((int)qpg, cap, s.num_q_heads, lay, pk, q, scale_log2, out, ws_acc, ws_ml, s.num_seqs, status, stream);
}

}  // namespace mqkv
