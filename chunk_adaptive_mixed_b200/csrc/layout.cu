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

// grow < 0: a fixed layout (regions hold exactly the segment's tokens).
// grow >= 0: a growable layout — every segment region reserves room for
// `grow` more chunks (FP16 one more, for the open chunk), chunk slots are
// num_chunks + grow + 1 per sequence, and a partial last chunk is the open
// FP16 tail whatever the map says.
__global__ void __launch_bounds__(kLayoutThreads)
layout_seq_kernel(const int64_t* __restrict__ cu, int L, int d, int Hkv,
                  const uint8_t* __restrict__ chunk_expert, int64_t total_slots,
                  int it0, int it1, int it2, int grow, void* layout, unsigned int* status) {
  __shared__ int64_t red[33];
  __shared__ int wcount[kLayoutThreads / 32][kNumExperts];
  const int b = blockIdx.x;
  const int B = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid / 32;
  const int64_t in_off = block_chunk_offset(b, cu, L, red);  // index into chunk_expert
  const int64_t coff = in_off + (grow >= 0 ? (int64_t)b * (grow + 1) : 0);  // slot offset
  const int64_t row0 = cu[b];
  const int Tb = (int)(cu[b + 1] - row0);
  const int nb = (Tb + L - 1) / L;
  const bool open_tail = grow >= 0 && Tb % L != 0;
  int32_t* perm = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(layout) +
                                             layout_perm_offset(B));
  int32_t* inv = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(layout) +
                                            layout_inv_offset(B, total_slots));

  auto expert_of = [&](int c) -> int {
    if (open_tail && c == nb - 1) return 0;
    int e = chunk_expert[in_off + c];
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

  // unused slots of a growable layout name chunk nb, past the sequence's last
  // token, so a pack over every slot encodes nothing there
  if (grow >= 0)
    for (int p = nb + tid; p < nb + grow + 1; p += blockDim.x) perm[coff + p] = nb;

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
      // rows the regions hold: the tokens, or for a growable layout whole
      // chunk slots for the present chunks plus the growth budget
      const int64_t rows =
          grow < 0 ? ntok : (int64_t)(seg_chunks[e] + grow + (e == 0 ? 1 : 0)) * L;
      r->seg_chunks[e] = seg_chunks[e];
      r->seg_chunk_begin[e] = begin[e];
      r->seg_tokens[e] = ntok;
      if (e == 0) {
        r->scale_offset[e] = 0;
        r->region_bytes[e] = align128((uint64_t)rows * code_row_bytes(d, e));
      } else {
        const uint64_t so = align128((uint64_t)rows * code_row_bytes(d, e));
        r->scale_offset[e] = so;
        r->region_bytes[e] = so + align128((uint64_t)rows * scale_row_bytes(d));
      }
      r->item_count[e] = (ntok + it[e] - 1) / it[e];
      r->seg_base[e] = 0;    // finalize
      r->item_begin[e] = 0;  // finalize
    }
    r->chunk_capacity = grow < 0 ? 0 : nb + grow + 1;
    r->grow_state = open_tail ? MQ_GROW_OPEN : 0;
  }
}

__global__ void __launch_bounds__(1024)
layout_finalize_kernel(int B, int L, int d, int Hkv, int it0, int it1, int it2, int grow,
                       void* layout) {
  __shared__ uint64_t red_u[33];
  __shared__ int64_t red_i[33];
  if (it0 < 0) {  // after a growth step: keep the sizes the layout was built with
    const mq_layout_header* h0 = static_cast<const mq_layout_header*>(layout);
    it0 = h0->item_tokens[0];
    it1 = h0->item_tokens[1];
    it2 = h0->item_tokens[2];
    grow = h0->grow_chunks - 1;
    __syncthreads();  // all threads have read the header before it is rewritten
  }
  uint64_t byte_carry = 0;
  int64_t item_carry = 0, chunk_carry = 0, token_carry = 0;
  for (int base = 0; base < B; base += blockDim.x) {
    const int b = base + threadIdx.x;
    mq_seq_layout* r = b < B ? seq_rec(layout, b) : nullptr;
    uint64_t bytes = 0;
    int64_t items = 0, chunks = 0, tokens = 0;
    if (r) {
      for (int e = 0; e < kNumExperts; ++e) {
        bytes += 2ull * (uint64_t)Hkv * r->region_bytes[e];
        items += r->item_count[e];
      }
      chunks = grow < 0 ? r->num_chunks : r->chunk_capacity;
      tokens = r->num_tokens;
    }
    uint64_t tb;
    int64_t ti, tc, tt;
    const uint64_t bbase = block_exclusive_scan<uint64_t>(bytes, red_u, &tb) + byte_carry;
    const int64_t ibase = block_exclusive_scan<int64_t>(items, red_i, &ti) + item_carry;
    (void)block_exclusive_scan<int64_t>(chunks, red_i, &tc);
    (void)block_exclusive_scan<int64_t>(tokens, red_i, &tt);
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
    token_carry += tt;
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
    h->total_tokens = token_carry;
    h->packed_bytes = byte_carry;
    h->item_tokens[0] = it0;
    h->item_tokens[1] = it1;
    h->item_tokens[2] = it2;
    h->grow_chunks = grow < 0 ? 0 : grow + 1;
  }
}

// Shift perm entries [lo, hi) of one sequence by `dir` (+1 or -1) positions
// and update inv for the moved chunks.  Tiles are visited so that no entry is
// overwritten before it has been read (low to high for -1, high to low for +1).
__device__ void shift_positions(int32_t* perm, int32_t* inv, int64_t coff, int lo, int hi,
                                int dir) {
  const int n = hi - lo;
  const int ntiles = (n + kLayoutThreads - 1) / kLayoutThreads;
  for (int i = 0; i < ntiles; ++i) {
    const int tile = dir < 0 ? i : ntiles - 1 - i;
    const int p = lo + tile * kLayoutThreads + threadIdx.x;
    int32_t c = 0;
    if (p < hi) c = perm[coff + p];
    __syncthreads();
    if (p < hi) {
      perm[coff + p + dir] = c;
      inv[coff + c] = p + dir;
    }
    __syncthreads();
  }
}

// One decode step of a growable layout, one CTA per sequence:
//  1. seal: if the open chunk is full and sealed[b] names its expert, the
//     chunk leaves the end of the FP16 segment for the end of segment
//     sealed[b] (its codes were written there by mq_grow_seal beforehand);
//     expert 0 keeps it where it is;
//  2. reserve: with add != 0, one more token row at the end of the open chunk
//     (a new open FP16 chunk when there is none).
// A step that would exceed a reserved capacity is skipped for that sequence,
// flagged in grow_state and reported with MQ_DEV_CAPACITY.
__global__ void __launch_bounds__(kLayoutThreads)
grow_commit_kernel(int L, int d, const uint8_t* __restrict__ sealed, int add, void* layout,
                   unsigned int* status) {
  const int b = blockIdx.x;
  const int B = gridDim.x;
  const mq_layout_header* h = static_cast<const mq_layout_header*>(layout);
  mq_seq_layout* r = seq_rec(layout, b);
  int32_t* perm = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(layout) +
                                             layout_perm_offset(B));
  int32_t* inv = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(layout) +
                                            layout_inv_offset(B, h->total_chunks));
  if (h->magic != MQ_LAYOUT_MAGIC || h->grow_chunks <= 0) {
    if (threadIdx.x == 0) set_status(status, MQ_DEV_BAD_LAYOUT);
    return;
  }
  const int64_t coff = r->chunk_offset;
  int n = r->num_chunks, T = r->num_tokens;
  int state = r->grow_state & MQ_GROW_OPEN;
  int sc[kNumExperts], st[kNumExperts];
  for (int e = 0; e < kNumExperts; ++e) {
    sc[e] = r->seg_chunks[e];
    st[e] = r->seg_tokens[e];
  }
  auto rows_cap = [&](int e) -> int64_t {
    return e == 0 ? (int64_t)(r->region_bytes[0] / code_row_bytes(d, 0))
                  : (int64_t)(r->scale_offset[e] / code_row_bytes(d, e));
  };
  __syncthreads();  // every thread has read the record before thread 0 rewrites it

  // 1. seal the full open chunk
  if (sealed && (state & MQ_GROW_OPEN) && T > 0 && T % L == 0) {
    const int e = sealed[b];
    if (e == 255) {
      // no seal for this sequence in this step
    } else if (e > 2) {
      if (threadIdx.x == 0) set_status(status, MQ_DEV_INDEX_RANGE);
    } else if (e == 0) {
      state &= ~MQ_GROW_OPEN;
    } else if (st[e] + L > rows_cap(e)) {
      if (threadIdx.x == 0) set_status(status, MQ_DEV_CAPACITY);
      state |= MQ_GROW_FULL;
    } else {
      const int c_open = perm[coff + sc[0] - 1];
      const int end_e = sc[0] + sc[1] + (e == 2 ? sc[2] : 0);
      shift_positions(perm, inv, coff, sc[0], end_e, -1);
      if (threadIdx.x == 0) {
        perm[coff + end_e - 1] = c_open;
        inv[coff + c_open] = end_e - 1;
      }
      sc[0] -= 1;
      st[0] -= L;
      sc[e] += 1;
      st[e] += L;
      state &= ~MQ_GROW_OPEN;
    }
  }

  // 2. reserve one token row
  if (add) {
    if (state & MQ_GROW_OPEN) {
      if (T % L == 0 || st[0] + 1 > rows_cap(0)) {  // full and not sealed, or no room
        if (threadIdx.x == 0) set_status(status, MQ_DEV_CAPACITY);
        state |= MQ_GROW_FULL;
      } else {
        st[0] += 1;
        T += 1;
      }
    } else if (n + 1 > r->chunk_capacity || st[0] + 1 > rows_cap(0)) {
      if (threadIdx.x == 0) set_status(status, MQ_DEV_CAPACITY);
      state |= MQ_GROW_FULL;
    } else {
      // a new open chunk at the end of the FP16 segment
      shift_positions(perm, inv, coff, sc[0], sc[0] + sc[1] + sc[2], +1);
      if (threadIdx.x == 0) {
        perm[coff + sc[0]] = n;
        inv[coff + n] = sc[0];
      }
      sc[0] += 1;
      st[0] += 1;
      n += 1;
      T += 1;
      state |= MQ_GROW_OPEN;
    }
  }

  if (threadIdx.x == 0) {
    r->num_tokens = T;
    r->num_chunks = n;
    int begin = 0;
    for (int e = 0; e < kNumExperts; ++e) {
      r->seg_chunks[e] = sc[e];
      r->seg_chunk_begin[e] = begin;
      begin += sc[e];
      r->seg_tokens[e] = st[e];
      r->item_count[e] = (st[e] + h->item_tokens[e] - 1) / h->item_tokens[e];
    }
    r->grow_state = state;
  }
}

}  // namespace

cudaError_t launch_layout(const mq_shape& s, const int64_t* cu_seqlens, const uint8_t* chunk_expert,
                          int64_t total_slots, const ItemPolicy& pol, int grow, void* layout,
                          unsigned int* status, cudaStream_t stream) {
  const int* it = pol.item_tokens;
  layout_seq_kernel<<<s.num_seqs, kLayoutThreads, 0, stream>>>(
      cu_seqlens, s.chunk_len, s.head_dim, s.num_kv_heads, chunk_expert, total_slots, it[0],
      it[1], it[2], grow, layout, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  layout_finalize_kernel<<<1, 1024, 0, stream>>>(s.num_seqs, s.chunk_len, s.head_dim,
                                                 s.num_kv_heads, it[0], it[1], it[2], grow, layout);
  return cudaGetLastError();
}

cudaError_t launch_grow_commit(const mq_shape& s, const uint8_t* sealed, int add, void* layout,
                               unsigned int* status, cudaStream_t stream) {
  grow_commit_kernel<<<s.num_seqs, kLayoutThreads, 0, stream>>>(s.chunk_len, s.head_dim, sealed,
                                                                add, layout, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  layout_finalize_kernel<<<1, 1024, 0, stream>>>(s.num_seqs, s.chunk_len, s.head_dim,
                                                 s.num_kv_heads, -1, -1, -1, 0, layout);
  return cudaGetLastError();
}

}  // namespace mqkv
