// api.cu — the extern "C" entry points of libmqkv (include/mqkv.h).
//
// Every entry point validates its arguments on the host first (no CUDA call
// happens before validation passes), then launches asynchronously on the
// caller's stream.  The only library state is the device status word below
// (one 32-bit word per device, part of the module image, never allocated) and
// a thread-local error string.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "common.cuh"

namespace mqkv {

__device__ unsigned int g_device_status;

namespace {

thread_local char t_last_error[512] = "";

mq_status fail(mq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
  va_end(ap);
  return st;
}

mq_status cuda_fail(cudaError_t err, const char* what) {
  return fail(MQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

// Address of g_device_status on the current device (looked up once per device).
constexpr int kMaxDevices = 64;
std::mutex g_status_mutex;
unsigned int* g_status_ptr[kMaxDevices] = {};

cudaError_t status_word(unsigned int** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_status_mutex);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_device_status);
    if (err != cudaSuccess) return err;
    g_status_ptr[dev] = static_cast<unsigned int*>(p);
  }
  *out = g_status_ptr[dev];
  return cudaSuccess;
}

// Longest sequence (so that one (K|V, kv-head) region stays below 2^31 bytes).
constexpr int32_t kMaxSeqTokens = 1 << 23;

mq_status check_shape(const mq_shape* s) {
  if (!s) return fail(MQ_ERR_INVALID_ARG, "shape is NULL");
  if (s->num_seqs < 1) return fail(MQ_ERR_INVALID_ARG, "num_seqs must be >= 1 (got %d)", s->num_seqs);
  if (s->num_q_heads < 1 || s->num_kv_heads < 1)
    return fail(MQ_ERR_INVALID_ARG, "head counts must be >= 1 (Hq=%d, Hkv=%d)", s->num_q_heads,
                s->num_kv_heads);
  if (s->num_q_heads % s->num_kv_heads != 0)
    return fail(MQ_ERR_INVALID_ARG, "num_q_heads %% num_kv_heads != 0 (Hq=%d, Hkv=%d)",
                s->num_q_heads, s->num_kv_heads);
  const int qpg = s->num_q_heads / s->num_kv_heads;
  if (qpg != 1 && qpg != 2 && qpg != 4 && qpg != 8)
    return fail(MQ_ERR_UNSUPPORTED, "Hq/Hkv must be 1, 2, 4 or 8 (got %d)", qpg);
  if (s->head_dim != 64 && s->head_dim != 128)
    return fail(MQ_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", s->head_dim);
  if (s->chunk_len < 32 || s->chunk_len > 4096 || s->chunk_len % 32 != 0)
    return fail(MQ_ERR_INVALID_ARG, "chunk_len must be a multiple of 32 in [32, 4096] (got %d)",
                s->chunk_len);
  if (s->group_size != kGroup)
    return fail(MQ_ERR_UNSUPPORTED, "group_size must be 32 (got %d)", s->group_size);
  return MQ_OK;
}

// Validates the lengths; returns total tokens and chunks.
mq_status check_lens(const mq_shape* s, const int32_t* h_seq_lens, int64_t* T, int64_t* N) {
  if (!h_seq_lens) return fail(MQ_ERR_INVALID_ARG, "h_seq_lens is NULL");
  int64_t t = 0, n = 0;
  for (int b = 0; b < s->num_seqs; ++b) {
    if (h_seq_lens[b] < 0) return fail(MQ_ERR_INVALID_ARG, "h_seq_lens[%d] < 0", b);
    if (h_seq_lens[b] > kMaxSeqTokens)
      return fail(MQ_ERR_UNSUPPORTED, "h_seq_lens[%d] = %d exceeds %d tokens", b, h_seq_lens[b],
                  kMaxSeqTokens);
    t += h_seq_lens[b];
    n += (h_seq_lens[b] + s->chunk_len - 1) / s->chunk_len;
  }
  if (n >= (int64_t(1) << 31)) return fail(MQ_ERR_UNSUPPORTED, "more than 2^31 chunks");
  *T = t;
  *N = n;
  return MQ_OK;
}

#define MQ_TRY(x)                      \
  do {                                 \
    const mq_status st_ = (x);         \
    if (st_ != MQ_OK) return st_;      \
  } while (0)

#define MQ_NEED_PTR(p, name)                                                           \
  do {                                                                                 \
    if (!(p)) return fail(MQ_ERR_INVALID_ARG, "%s is NULL", name);                     \
    if (misaligned(p)) return fail(MQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

}  // namespace

mq_status report_error(mq_status status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
  va_end(ap);
  return status;
}

// ------------------------------------------------------------ item policy

ItemPolicy item_policy(const mq_shape& s, const int32_t* h_seq_lens) {
  // Work items are balanced by estimated decode time, not by bytes: a token
  // costs its packed bytes plus a fixed amount of arithmetic (code expansion,
  // dot products, softmax), about 374 byte-equivalents per query head group
  // for one query head (fitted to the single-precision decode rates: FP16
  // 5.2, INT4 2.7, INT2 1.85 TB/s), growing with the query heads that share a
  // kv-head.  An item carries about 2^18 byte-equivalents (2^19 with four or
  // more query heads per kv-head, whose per-item partial results are larger)
  // so the partial results, and the merge that reads them back, stay a few
  // percent of the bytes read (measured with one query head per kv-head:
  // 2^18 decodes 1.6% faster than 2^17 and as fast as 2^19; with four query
  // heads, 2^20 is no faster than 2^19).  Small
  // problems are split finer (by powers of two, down to 32 tokens) so that
  // every worker warp of a 148-SM part gets several items.  Depends only on
  // the shape and the lengths, so size queries and layout builds agree
  // without a GPU.
  const int d = s.head_dim;
  const int qpg = s.num_q_heads / s.num_kv_heads;
  const int bpt[kNumExperts] = {2 * 2 * d, 2 * (d / 2 + d / 8), 2 * (d / 4 + d / 8)};
  const int arith = (374 * d / 128) * (2 + 3 * qpg) / 5;  // 0.4 + 0.6 * qpg of one head's
  const int target = qpg >= 4 ? (1 << 19) : (1 << 18);
  ItemPolicy p;
  for (int e = 0; e < kNumExperts; ++e) {
    int m = (target / (bpt[e] + arith)) / 32 * 32;
    if (m < 32) m = 32;
    p.item_tokens[e] = m;
  }
  int64_t T = 0;
  for (int b = 0; b < s.num_seqs; ++b) T += h_seq_lens[b];
  const int64_t want = 148 * 2 * 8 * 4;  // worker warps of a 148-SM part x 4
  while (true) {
    const int64_t est = T * s.num_kv_heads / p.item_tokens[1];
    if (est >= want) break;
    bool shrunk = false;
    for (int e = 0; e < kNumExperts; ++e)
      if (p.item_tokens[e] >= 64) {
        p.item_tokens[e] = (p.item_tokens[e] / 2) / 32 * 32;
        shrunk = true;
      }
    if (!shrunk) break;
  }
  return p;
}

int64_t max_items_per_kv_head(const mq_shape& s, const int32_t* h_seq_lens, const ItemPolicy& p) {
  int it_min = p.item_tokens[0];
  for (int e = 1; e < kNumExperts; ++e) it_min = p.item_tokens[e] < it_min ? p.item_tokens[e] : it_min;
  int64_t n = 0;
  for (int b = 0; b < s.num_seqs; ++b) n += (h_seq_lens[b] + it_min - 1) / it_min + 3;
  return n;
}

// Growable layouts: lengths the layout is sized for (prefill + growth budget).
struct GrowDims {
  std::vector<int32_t> cap_lens;  // h_seq_lens[b] + grow_tokens
  int grow_chunks;                // chunks that can complete during growth
  int64_t slots;                  // chunk slots (perm / inv entries)
};

}  // namespace mqkv

using namespace mqkv;

namespace {

mq_status grow_dims(const mq_shape* shape, const int32_t* h_seq_lens, int32_t grow_tokens,
                    GrowDims* g, int64_t* T, int64_t* N) {
  MQ_TRY(check_shape(shape));
  MQ_TRY(check_lens(shape, h_seq_lens, T, N));
  if (grow_tokens < 0 || grow_tokens > kMaxSeqTokens)
    return fail(MQ_ERR_INVALID_ARG, "grow_tokens must be in [0, %d] (got %d)", kMaxSeqTokens,
                grow_tokens);
  g->cap_lens.resize(shape->num_seqs);
  for (int b = 0; b < shape->num_seqs; ++b) {
    const int64_t c = (int64_t)h_seq_lens[b] + grow_tokens;
    if (c > kMaxSeqTokens)
      return fail(MQ_ERR_UNSUPPORTED, "h_seq_lens[%d] + grow_tokens exceeds %d tokens", b,
                  kMaxSeqTokens);
    g->cap_lens[b] = (int32_t)c;
  }
  g->grow_chunks = (grow_tokens + shape->chunk_len - 1) / shape->chunk_len;
  g->slots = *N + (int64_t)shape->num_seqs * (g->grow_chunks + 1);
  if (g->slots >= (int64_t(1) << 31)) return fail(MQ_ERR_UNSUPPORTED, "more than 2^31 chunk slots");
  return MQ_OK;
}

}  // namespace

extern "C" {

const char* mq_status_string(mq_status status) {
  switch (status) {
    case MQ_OK: return "ok";
    case MQ_ERR_INVALID_ARG: return "invalid argument";
    case MQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case MQ_ERR_WORKSPACE: return "buffer too small";
    case MQ_ERR_CUDA: return "CUDA error";
    case MQ_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

const char* mq_last_error(void) { return t_last_error; }

size_t mq_layout_bytes(const mq_shape* shape, const int32_t* h_seq_lens) {
  int64_t T, N;
  if (check_shape(shape) != MQ_OK || check_lens(shape, h_seq_lens, &T, &N) != MQ_OK) return 0;
  return layout_total_bytes(shape->num_seqs, N);
}

size_t mq_packed_bytes_upper_bound(const mq_shape* shape, const int32_t* h_seq_lens) {
  int64_t T, N;
  if (check_shape(shape) != MQ_OK || check_lens(shape, h_seq_lens, &T, &N) != MQ_OK) return 0;
  uint64_t total = 0;
  for (int b = 0; b < shape->num_seqs; ++b)
    total += 2ull * shape->num_kv_heads *
             align128((uint64_t)h_seq_lens[b] * code_row_bytes(shape->head_dim, 0));
  return (size_t)total;
}

size_t mq_decode_workspace_bytes(const mq_shape* shape, const int32_t* h_seq_lens) {
  int64_t T, N;
  if (check_shape(shape) != MQ_OK || check_lens(shape, h_seq_lens, &T, &N) != MQ_OK) return 0;
  const ItemPolicy p = item_policy(*shape, h_seq_lens);
  return decode_workspace_bytes(*shape, max_items_per_kv_head(*shape, h_seq_lens, p));
}

mq_status mq_packed_bytes(const void* layout, size_t* h_bytes, void* stream) {
  MQ_NEED_PTR(layout, "layout");
  if (!h_bytes) return fail(MQ_ERR_INVALID_ARG, "h_bytes is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint64_t v = 0;
  cudaError_t err = cudaMemcpyAsync(&v, static_cast<const unsigned char*>(layout) +
                                            offsetof(mq_layout_header, packed_bytes),
                                    sizeof v, cudaMemcpyDeviceToHost, st);
  if (err != cudaSuccess) return cuda_fail(err, "mq_packed_bytes copy");
  if ((err = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(err, "mq_packed_bytes sync");
  *h_bytes = (size_t)v;
  return MQ_OK;
}

mq_status mq_device_status(uint32_t* h_flags, int32_t clear, void* stream) {
  if (!h_flags) return fail(MQ_ERR_INVALID_ARG, "h_flags is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* word = nullptr;
  cudaError_t err = status_word(&word);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  unsigned int v = 0;
  if ((err = cudaMemcpyAsync(&v, word, sizeof v, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return cuda_fail(err, "device status read");
  if (clear && (err = cudaMemsetAsync(word, 0, sizeof v, st)) != cudaSuccess)
    return cuda_fail(err, "device status clear");
  if ((err = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(err, "device status sync");
  *h_flags = v;
  if (v) return fail(MQ_ERR_DEVICE_CHECK, "device status 0x%x", v);
  return MQ_OK;
}

size_t mq_route_workspace_bytes(const mq_shape* shape, const int32_t* h_seq_lens, int32_t D,
                                int32_t H) {
  int64_t T, N;
  if (check_shape(shape) != MQ_OK || check_lens(shape, h_seq_lens, &T, &N) != MQ_OK) return 0;
  if (D < 1 || D % 4 != 0 || (H != 64 && H != 128 && H != 256)) {
    fail(MQ_ERR_INVALID_ARG, "D must be a positive multiple of 4 and H one of 64, 128, 256");
    return 0;
  }
  return route_workspace_bytes(T, D, H);
}

mq_status mq_route_chunks(const mq_shape* shape, const int32_t* h_seq_lens,
                          const int64_t* d_cu_seqlens, const float* C, int32_t D, int32_t H,
                          const float* W1, const float* W2, const float* W3, const float* b3,
                          int32_t routing_freeze, uint8_t* token_expert, uint8_t* chunk_expert,
                          float* logits, void* workspace, size_t workspace_bytes, void* stream) {
  MQ_TRY(check_shape(shape));
  int64_t T, N;
  MQ_TRY(check_lens(shape, h_seq_lens, &T, &N));
  if (D < 1 || D % 4 != 0) return fail(MQ_ERR_INVALID_ARG, "D must be a positive multiple of 4 (got %d)", D);
  if (H != 64 && H != 128 && H != 256)
    return fail(MQ_ERR_UNSUPPORTED, "H must be 64, 128 or 256 (got %d)", H);
  MQ_NEED_PTR(d_cu_seqlens, "d_cu_seqlens");
  MQ_NEED_PTR(C, "C");
  MQ_NEED_PTR(W1, "W1");
  MQ_NEED_PTR(W2, "W2");
  MQ_NEED_PTR(W3, "W3");
  if (b3 && misaligned(b3)) return fail(MQ_ERR_INVALID_ARG, "b3 is not 16-byte aligned");
  MQ_NEED_PTR(token_expert, "token_expert");
  MQ_NEED_PTR(chunk_expert, "chunk_expert");
  if (logits && misaligned(logits)) return fail(MQ_ERR_INVALID_ARG, "logits is not 16-byte aligned");
  const size_t need = route_workspace_bytes(T, D, H);
  if (workspace_bytes < need)
    return fail(MQ_ERR_WORKSPACE, "workspace_bytes %zu < %zu needed", workspace_bytes, need);
  MQ_NEED_PTR(workspace, "workspace");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  const float4* zpart = nullptr;
  int nhb = 0;
  err = launch_router_tc(C, T, D, H, W1, W2, W3, workspace, status, st, &zpart, &nhb);
  if (err != cudaSuccess) return cuda_fail(err, "router launch");
  int64_t max_chunks = 0;
  for (int b = 0; b < shape->num_seqs; ++b) {
    const int64_t nb = (h_seq_lens[b] + shape->chunk_len - 1) / shape->chunk_len;
    max_chunks = nb > max_chunks ? nb : max_chunks;
  }
  err = launch_finish_vote(shape->num_seqs, d_cu_seqlens, shape->chunk_len, max_chunks, zpart, nhb, b3,
                           routing_freeze, token_expert, logits, chunk_expert, st);
  if (err != cudaSuccess) return cuda_fail(err, "vote launch");
  return MQ_OK;
}

mq_status mq_similarity_route(const mq_shape* shape, const int32_t* h_seq_lens,
                              const int64_t* d_cu_seqlens, const float* C, int32_t D,
                              const float* u, double tau_hi, double tau_lo,
                              int32_t routing_freeze, uint8_t* chunk_expert, double* similarity,
                              void* stream) {
  MQ_TRY(check_shape(shape));
  int64_t T, N;
  MQ_TRY(check_lens(shape, h_seq_lens, &T, &N));
  if (D < 1 || D % 4 != 0) return fail(MQ_ERR_INVALID_ARG, "D must be a positive multiple of 4 (got %d)", D);
  if (shape->num_seqs > 65535)
    return fail(MQ_ERR_UNSUPPORTED, "num_seqs must be <= 65535 (got %d)", shape->num_seqs);
  if (tau_hi != tau_hi || tau_lo != tau_lo) return fail(MQ_ERR_INVALID_ARG, "a threshold is NaN");
  MQ_NEED_PTR(d_cu_seqlens, "d_cu_seqlens");
  if (T > 0) MQ_NEED_PTR(C, "C");
  MQ_NEED_PTR(u, "u");
  if (N > 0) MQ_NEED_PTR(chunk_expert, "chunk_expert");
  if (similarity && misaligned(similarity))
    return fail(MQ_ERR_INVALID_ARG, "similarity is not 16-byte aligned");
  int64_t max_chunks = 0;
  for (int b = 0; b < shape->num_seqs; ++b) {
    const int64_t nb = (h_seq_lens[b] + shape->chunk_len - 1) / shape->chunk_len;
    max_chunks = nb > max_chunks ? nb : max_chunks;
  }
  const cudaError_t err = launch_similarity_route(
      shape->num_seqs, d_cu_seqlens, shape->chunk_len, max_chunks, C, D, u, tau_hi, tau_lo,
      routing_freeze, chunk_expert, similarity, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "similarity launch");
  return MQ_OK;
}

mq_status mq_build_layout(const mq_shape* shape, const int32_t* h_seq_lens,
                          const int64_t* d_cu_seqlens, const uint8_t* chunk_expert, void* layout,
                          size_t layout_bytes, void* stream) {
  MQ_TRY(check_shape(shape));
  int64_t T, N;
  MQ_TRY(check_lens(shape, h_seq_lens, &T, &N));
  MQ_NEED_PTR(d_cu_seqlens, "d_cu_seqlens");
  if (N > 0) MQ_NEED_PTR(chunk_expert, "chunk_expert");
  MQ_NEED_PTR(layout, "layout");
  const size_t need = layout_total_bytes(shape->num_seqs, N);
  if (layout_bytes < need)
    return fail(MQ_ERR_WORKSPACE, "layout_bytes %zu < %zu needed", layout_bytes, need);
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  const ItemPolicy p = item_policy(*shape, h_seq_lens);
  err = launch_layout(*shape, d_cu_seqlens, chunk_expert, N, p, -1, layout, status,
                      static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "layout launch");
  return MQ_OK;
}

mq_status mq_pack_kv(const mq_shape* shape, const int32_t* h_seq_lens, const void* layout,
                     const void* K, const void* V, int32_t kv_dtype, void* packed,
                     size_t packed_bytes, void* stream) {
  MQ_TRY(check_shape(shape));
  int64_t T, N;
  MQ_TRY(check_lens(shape, h_seq_lens, &T, &N));
  if (kv_dtype != MQ_F16 && kv_dtype != MQ_F32)
    return fail(MQ_ERR_INVALID_ARG, "kv_dtype must be MQ_F16 or MQ_F32 (got %d)", kv_dtype);
  MQ_NEED_PTR(layout, "layout");
  if (T > 0) {
    MQ_NEED_PTR(K, "K");
    MQ_NEED_PTR(V, "V");
    MQ_NEED_PTR(packed, "packed");
  }
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  err = launch_pack(*shape, N, layout, K, V, kv_dtype, packed, packed_bytes, status,
                    static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "pack launch");
  return MQ_OK;
}

mq_status mq_decode_attn(const mq_shape* shape, const int32_t* h_seq_lens, const void* layout,
                         const void* packed, const void* q, int32_t q_dtype, float softmax_scale,
                         float* out, void* workspace, size_t workspace_bytes, void* stream) {
  MQ_TRY(check_shape(shape));
  int64_t T, N;
  MQ_TRY(check_lens(shape, h_seq_lens, &T, &N));
  if (q_dtype != MQ_F16 && q_dtype != MQ_F32)
    return fail(MQ_ERR_INVALID_ARG, "q_dtype must be MQ_F16 or MQ_F32 (got %d)", q_dtype);
  MQ_NEED_PTR(layout, "layout");
  MQ_NEED_PTR(q, "q");
  MQ_NEED_PTR(out, "out");
  if (T > 0) MQ_NEED_PTR(packed, "packed");
  const ItemPolicy p = item_policy(*shape, h_seq_lens);
  const int64_t items = max_items_per_kv_head(*shape, h_seq_lens, p);
  const size_t need = decode_workspace_bytes(*shape, items);
  if (workspace_bytes < need)
    return fail(MQ_ERR_WORKSPACE, "workspace_bytes %zu < %zu needed", workspace_bytes, need);
  MQ_NEED_PTR(workspace, "workspace");
  if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / sqrtf((float)shape->head_dim);
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  err = launch_decode(*shape, items, layout, packed, q, q_dtype, softmax_scale, out, workspace,
                      workspace_bytes, status, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "decode launch");
  return MQ_OK;
}

// ------------------------------------------------------------ context split

mq_status mq_decode_attn_partial(const mq_shape* shape, const int32_t* h_seq_lens,
                                 const void* layout, const void* packed, const void* q,
                                 int32_t q_dtype, float softmax_scale, float* partial,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  MQ_TRY(check_shape(shape));
  int64_t T, N;
  MQ_TRY(check_lens(shape, h_seq_lens, &T, &N));
  if (q_dtype != MQ_F16 && q_dtype != MQ_F32)
    return fail(MQ_ERR_INVALID_ARG, "q_dtype must be MQ_F16 or MQ_F32 (got %d)", q_dtype);
  MQ_NEED_PTR(layout, "layout");
  MQ_NEED_PTR(q, "q");
  MQ_NEED_PTR(partial, "partial");
  if (T > 0) MQ_NEED_PTR(packed, "packed");
  const ItemPolicy p = item_policy(*shape, h_seq_lens);
  const int64_t items = max_items_per_kv_head(*shape, h_seq_lens, p);
  const size_t need = decode_workspace_bytes(*shape, items);
  if (workspace_bytes < need)
    return fail(MQ_ERR_WORKSPACE, "workspace_bytes %zu < %zu needed", workspace_bytes, need);
  MQ_NEED_PTR(workspace, "workspace");
  if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / sqrtf((float)shape->head_dim);
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  err = launch_decode(*shape, items, layout, packed, q, q_dtype, softmax_scale, partial, workspace,
                      workspace_bytes, status, static_cast<cudaStream_t>(stream), true);
  if (err != cudaSuccess) return cuda_fail(err, "decode launch");
  return MQ_OK;
}

mq_status mq_combine_partials(int32_t num_parts, int32_t num_seqs, int32_t num_q_heads,
                              int32_t head_dim, const float* partials, float* out, void* stream) {
  if (num_parts < 1) return fail(MQ_ERR_INVALID_ARG, "num_parts must be >= 1 (got %d)", num_parts);
  if (num_seqs < 1 || num_q_heads < 1)
    return fail(MQ_ERR_INVALID_ARG, "num_seqs and num_q_heads must be >= 1");
  if (head_dim != 64 && head_dim != 128)
    return fail(MQ_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", head_dim);
  MQ_NEED_PTR(partials, "partials");
  MQ_NEED_PTR(out, "out");
  const cudaError_t err = launch_combine_partials(num_parts, num_seqs, num_q_heads, head_dim,
                                                  partials, out, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "combine launch");
  return MQ_OK;
}

// ---------------------------------------------------------------- growth

mq_status mq_grow_sizes(const mq_shape* shape, const int32_t* h_seq_lens, int32_t grow_tokens,
                        size_t* layout_bytes, size_t* packed_bytes_upper_bound,
                        size_t* decode_workspace_bytes) {
  GrowDims g;
  int64_t T, N;
  MQ_TRY(grow_dims(shape, h_seq_lens, grow_tokens, &g, &T, &N));
  const int L = shape->chunk_len, d = shape->head_dim, Hkv = shape->num_kv_heads;
  if (layout_bytes) *layout_bytes = layout_total_bytes(shape->num_seqs, g.slots);
  if (packed_bytes_upper_bound) {
    // every present chunk at FP16, plus the growth rows of all three segments
    uint64_t total = 0;
    for (int b = 0; b < shape->num_seqs; ++b) {
      const uint64_t nb = (h_seq_lens[b] + L - 1) / L;
      for (int e = 0; e < kNumExperts; ++e) {
        const uint64_t rows = ((e == 0 ? nb + 1 : 0) + g.grow_chunks) * (uint64_t)L;
        uint64_t rb = align128(rows * code_row_bytes(d, e));
        if (e != 0) rb += align128(rows * scale_row_bytes(d));
        total += 2ull * Hkv * rb;
      }
    }
    *packed_bytes_upper_bound = total;
  }
  if (decode_workspace_bytes) {
    const ItemPolicy p = item_policy(*shape, g.cap_lens.data());
    *decode_workspace_bytes =
        mqkv::decode_workspace_bytes(*shape, max_items_per_kv_head(*shape, g.cap_lens.data(), p));
  }
  return MQ_OK;
}

mq_status mq_grow_build_layout(const mq_shape* shape, const int32_t* h_seq_lens,
                               int32_t grow_tokens, const int64_t* d_cu_seqlens,
                               const uint8_t* chunk_expert, void* layout, size_t layout_bytes,
                               void* stream) {
  GrowDims g;
  int64_t T, N;
  MQ_TRY(grow_dims(shape, h_seq_lens, grow_tokens, &g, &T, &N));
  MQ_NEED_PTR(d_cu_seqlens, "d_cu_seqlens");
  if (N > 0) MQ_NEED_PTR(chunk_expert, "chunk_expert");
  MQ_NEED_PTR(layout, "layout");
  const size_t need = layout_total_bytes(shape->num_seqs, g.slots);
  if (layout_bytes < need)
    return fail(MQ_ERR_WORKSPACE, "layout_bytes %zu < %zu needed", layout_bytes, need);
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  const ItemPolicy p = item_policy(*shape, g.cap_lens.data());
  err = launch_layout(*shape, d_cu_seqlens, chunk_expert, g.slots, p, g.grow_chunks, layout,
                      status, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "layout launch");
  return MQ_OK;
}

mq_status mq_grow_pack_kv(const mq_shape* shape, const int32_t* h_seq_lens, int32_t grow_tokens,
                          const void* layout, const void* K, const void* V, int32_t kv_dtype,
                          void* packed, size_t packed_bytes, void* stream) {
  GrowDims g;
  int64_t T, N;
  MQ_TRY(grow_dims(shape, h_seq_lens, grow_tokens, &g, &T, &N));
  if (kv_dtype != MQ_F16 && kv_dtype != MQ_F32)
    return fail(MQ_ERR_INVALID_ARG, "kv_dtype must be MQ_F16 or MQ_F32 (got %d)", kv_dtype);
  MQ_NEED_PTR(layout, "layout");
  MQ_NEED_PTR(packed, "packed");
  if (T > 0) {
    MQ_NEED_PTR(K, "K");
    MQ_NEED_PTR(V, "V");
  }
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  err = launch_pack(*shape, g.slots, layout, K, V, kv_dtype, packed, packed_bytes, status,
                    static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "pack launch");
  return MQ_OK;
}

mq_status mq_grow_commit(const mq_shape* shape, void* layout, const uint8_t* sealed,
                         int32_t add_token, void* stream) {
  MQ_TRY(check_shape(shape));
  MQ_NEED_PTR(layout, "layout");
  if (sealed && misaligned(sealed)) return fail(MQ_ERR_INVALID_ARG, "sealed is not 16-byte aligned");
  if (add_token != 0 && add_token != 1)
    return fail(MQ_ERR_INVALID_ARG, "add_token must be 0 or 1 (got %d)", add_token);
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  err = launch_grow_commit(*shape, sealed, add_token, layout, status,
                           static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "grow commit launch");
  return MQ_OK;
}

mq_status mq_grow_append_kv(const mq_shape* shape, const void* layout, const void* K_new,
                            const void* V_new, int32_t kv_dtype, void* packed,
                            size_t packed_bytes, void* stream) {
  MQ_TRY(check_shape(shape));
  if (kv_dtype != MQ_F16 && kv_dtype != MQ_F32)
    return fail(MQ_ERR_INVALID_ARG, "kv_dtype must be MQ_F16 or MQ_F32 (got %d)", kv_dtype);
  MQ_NEED_PTR(layout, "layout");
  MQ_NEED_PTR(K_new, "K_new");
  MQ_NEED_PTR(V_new, "V_new");
  MQ_NEED_PTR(packed, "packed");
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  err = launch_grow_append(*shape, layout, K_new, V_new, kv_dtype, packed, packed_bytes, status,
                           static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "grow append launch");
  return MQ_OK;
}

mq_status mq_grow_seal(const mq_shape* shape, const void* layout, const uint8_t* sealed,
                       void* packed, size_t packed_bytes, void* stream) {
  MQ_TRY(check_shape(shape));
  MQ_NEED_PTR(layout, "layout");
  MQ_NEED_PTR(sealed, "sealed");
  MQ_NEED_PTR(packed, "packed");
  unsigned int* status = nullptr;
  cudaError_t err = status_word(&status);
  if (err != cudaSuccess) return cuda_fail(err, "device status word");
  err = launch_grow_seal(*shape, layout, sealed, packed, packed_bytes, status,
                         static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "grow seal launch");
  return MQ_OK;
}

}  // extern "C"
