// layout.cu — chunk regrouping by precision (Cocktail: chunk-level KV cache
// computation, from the Cocktail abstract on the "Bin Zhang" scholarfeed
// author page: reorder the KV chunks by precision before quantising, so that
// attention never mixes bitwidths inside one stretch of work).
//
// layout_seq_kernel (one CTA per sequence): stable partition of the
// sequence's chunks into FP16 -> INT4 -> INT2 segments with warp-ballot ranks,
// perm / inv tables, segment token counts, region geometry and the decode
// work-item counts of each segment.
// layout_finalize_kernel (one CTA): exclusive scans over sequences for the
// segment byte bases and the first work item of every (sequence, segment),
// then the table header.
#include "common.cuh"

namespace mqkv {
namespace {

constexpr int kLayoutThreads = 256;

__device__ inline mq_seq_layout* seq_rec(void* layout, int b) {
  return reinterpret_cast<mq_seq_layout*>(static_cast<unsigned char*>(layout) +
                                          layout_seq_offset(b));
}

__global__ void __launch_bounds__(kLayoutThreads)
layout_seq_kernel(const int64_t* __restrict__ cu, int L, int d, int Hkv,
                  const uint8_t* __restrict__ chunk_expert, int64_t total_chunks,
                  int it0, int it1, int it2, void* layout, unsigned int* status) {
  __shared__ int64_t red[33];
  __shared__ int wcount[kLayoutThreads / 32][kNumExperts];
  const int b = blockIdx.x;
  const int B = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid / 32;
  const int64_t coff = block_chunk_offset(b, cu, L, red);
  const int64_t row0 = cu[b];
  const int Tb = (int)(cu[b + 1] - row0);
  const int nb = (Tb + L - 1) / L;
  int32_t* perm = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(layout) +
                                             layout_perm_offset(B));
  int32_t* inv = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(layout) +
                                            layout_inv_offset(B, total_chunks));

  auto expert_of = [&](int c) -> int {
    int e = chunk_expert[coff + c];
    if (e > 2) {
      set_status(status, MQ_DEV_INDEX_RANGE);
      e = 2;
    }
    return e;
  };

  // pass 1: chunks per expert
  int cnt[kNumExperts] = {0, 0, 0};
  for (int c = tid; c < nb; c += blockDim.x) cnt[expert_of(c)]++;
  int seg_chunks[kNumExperts];
  for (int e = 0; e < kNumExperts; ++e) {
    int v = cnt[e];
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) wcount[warp][e] = v;
    __syncthreads();
    int tot = 0;
    for (int w = 0; w < kLayoutThreads / 32; ++w) tot += wcount[w][e];
    seg_chunks[e] = tot;
    __syncthreads();
  }
  const int begin[kNumExperts] = {0, seg_chunks[0], seg_chunks[0] + seg_chunks[1]};

  // pass 2: stable ranks inside each expert, 256 chunks at a time
  int running[kNumExperts] = {0, 0, 0};
  for (int base = 0; base < nb; base += kLayoutThreads) {
    const int c = base + tid;
    const int e = c < nb ? expert_of(c) : -1;
    const unsigned lt = (1u << lane) - 1u;
    int my_rank = 0;
    for (int x = 0; x < kNumExperts; ++x) {
      const unsigned m = __ballot_sync(0xffffffffu, e == x);
      if (e == x) my_rank = __popc(m & lt);
      if (lane == 0) wcount[warp][x] = __popc(m);
    }
    __syncthreads();
    int before = 0;
    int tile_tot[kNumExperts] = {0, 0, 0};
    for (int w = 0; w < kLayoutThreads / 32; ++w)
      for (int x = 0; x < kNumExperts; ++x) {
        if (w < warp && x == e) before += wcount[w][x];
        tile_tot[x] += wcount[w][x];
      }
    if (e >= 0) {
      const int pos = begin[e] + running[e] + before + my_rank;
      perm[coff + pos] = c;
      inv[coff + c] = pos;
    }
    for (int x = 0; x < kNumExperts; ++x) running[x] += tile_tot[x];
    __syncthreads();
  }

  if (tid == 0) {
    mq_seq_layout* r = seq_rec(layout, b);
    const int tail_e = nb > 0 ? expert_of(nb - 1) : -1;
    const int tail_short = nb > 0 ? nb * L - Tb : 0;
    const int it[kNumExperts] = {it0, it1, it2};
    r->token_offset = row0;
    r->num_tokens = Tb;
    r->num_chunks = nb;
    r->chunk_offset = (int32_t)coff;
    for (int e = 0; e < kNumExperts; ++e) {
      const int ntok = seg_chunks[e] * L - (e == tail_e ? tail_short : 0);
      r->seg_chunks[e] = seg_chunks[e];
      r->seg_chunk_begin[e] = begin[e];
      r->seg_tokens[e] = ntok;
      if (e == 0) {
        r->scale_offset[e] = 0;
        r->region_bytes[e] = align128((uint64_t)ntok * code_row_bytes(d, e));
      } else {
        const uint64_t so = align128((uint64_t)ntok * code_row_bytes(d, e));
        r->scale_offset[e] = so;
        r->region_bytes[e] = so + align128((uint64_t)ntok * scale_row_bytes(d));
      }
      r->item_count[e] = (ntok + it[e] - 1) / it[e];
      r->seg_base[e] = 0;    // finalize
      r->item_begin[e] = 0;  // finalize
    }
    r->reserved[0] = 0;
    r->reserved[1] = 0;
  }
}

__global__ void __launch_bounds__(1024)
layout_finalize_kernel(const int64_t* __restrict__ cu, int B, int L, int d, int Hkv,
                       int it0, int it1, int it2, void* layout) {
  __shared__ uint64_t red_u[33];
  __shared__ int64_t red_i[33];
  uint64_t byte_carry = 0;
  int64_t item_carry = 0, chunk_carry = 0;
  for (int base = 0; base < B; base += blockDim.x) {
    const int b = base + threadIdx.x;
    mq_seq_layout* r = b < B ? seq_rec(layout, b) : nullptr;
    uint64_t bytes = 0;
    int64_t items = 0, chunks = 0;
    if (r) {
      for (int e = 0; e < kNumExperts; ++e) {
        bytes += 2ull * (uint64_t)Hkv * r->region_bytes[e];
        items += r->item_count[e];
      }
      chunks = r->num_chunks;
    }
    uint64_t tb;
    int64_t ti, tc;
    const uint64_t bbase = block_exclusive_scan<uint64_t>(bytes, red_u, &tb) + byte_carry;
    const int64_t ibase = block_exclusive_scan<int64_t>(items, red_i, &ti) + item_carry;
    (void)block_exclusive_scan<int64_t>(chunks, red_i, &tc);
    if (r) {
      uint64_t off = bbase;
      int64_t it = ibase;
      for (int e = 0; e < kNumExperts; ++e) {
        r->seg_base[e] = off;
        off += 2ull * (uint64_t)Hkv * r->region_bytes[e];
        r->item_begin[e] = (int32_t)it;
        it += r->item_count[e];
      }
    }
    byte_carry += tb;
    item_carry += ti;
    chunk_carry += tc;
  }
  if (threadIdx.x == 0) {
    mq_layout_header* h = static_cast<mq_layout_header*>(layout);
    h->magic = MQ_LAYOUT_MAGIC;
    h->version = MQ_LAYOUT_VERSION;
    h->num_seqs = B;
    h->num_kv_heads = Hkv;
    h->head_dim = d;
    h->chunk_len = L;
    h->total_chunks = (int32_t)chunk_carry;
    h->total_items = (int32_t)item_carry;
    h->total_tokens = cu[B];
    h->packed_bytes = byte_carry;
    h->item_tokens[0] = it0;
    h->item_tokens[1] = it1;
    h->item_tokens[2] = it2;
    h->reserved[0] = 0;
  }
}

}  // namespace

cudaError_t launch_layout(const mq_shape& s, const int64_t* cu_seqlens, const uint8_t* chunk_expert,
                          int64_t total_chunks, const ItemPolicy& pol, void* layout,
                          unsigned int* status, cudaStream_t stream) {
  const int* it = pol.item_tokens;
  layout_seq_kernel<<<s.num_seqs, kLayoutThreads, 0, stream>>>(
      cu_seqlens, s.chunk_len, s.head_dim, s.num_kv_heads, chunk_expert, total_chunks, it[0],
      it[1], it[2], layout, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  layout_finalize_kernel<<<1, 1024, 0, stream>>>(cu_seqlens, s.num_seqs, s.chunk_len, s.head_dim,
                                                 s.num_kv_heads, it[0], it[1], it[2], layout);
  return cudaGetLastError();
}

}  // namespace mqkv
