// decode_noalloc.cu — mq_decode_attn_noalloc: decode attention for callers
// that cannot allocate device memory.
//
// mq_decode_attn needs a caller-provided workspace for its per-item partial
// results.  Some callers cannot get one: a serving runtime that reserves
// nearly all of HBM for its own KV pool at start-up and forbids any later
// cudaMalloc, or a plain C host program that has no device allocator of its
// own to hand.  For them this entry point uses a scratch array that is part
// of the library's module image instead: it is created when the module loads
// on a GPU and lives until the process exits, on every GPU that loads the
// library, whether or not this function is ever called.
//
// The work itself is mq_decode_attn's, unchanged: this file only supplies the
// workspace pointer.
#include <mutex>

#include "common.cuh"

namespace {

// The scratch array.  Its name is only meaningful in device code; on the host
// it is a stand-in symbol, so host code must ask the runtime for the device
// address (scratch_address below) and never pass the name itself to a kernel.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the first call on each device does the lookup).  The cached
// address belongs to the device's current primary context: after
// cudaDeviceReset the module is loaded afresh and the cache is stale, so a
// process that resets a device must not call mq_decode_attn_noalloc again on
// it.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" mq_status mq_decode_attn_noalloc(const mq_shape* shape, const int32_t* h_seq_lens,
                                            const void* layout, const void* packed,
                                            const void* q, int32_t q_dtype, float softmax_scale,
                                            float* out, void* stream) {
  // Size check first, on the host, so an oversized request fails before the
  // GPU is touched.  A zero size means the shape or the lengths are invalid:
  // mq_decode_attn's own validation then reports the precise reason.
  const size_t need = mq_decode_workspace_bytes(shape, h_seq_lens);
  if (need > (size_t)MQ_NOALLOC_SCRATCH_BYTES)
    return mqkv::report_error(
        MQ_ERR_WORKSPACE,
        "mq_decode_attn_noalloc: this batch needs %zu bytes of scratch, more than the %u bytes "
        "built into the library (MQ_NOALLOC_SCRATCH_BYTES); call mq_decode_attn with a "
        "workspace instead",
        need, (unsigned)MQ_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (need > 0) {
    const cudaError_t err = scratch_address(&scratch);
    if (err != cudaSuccess)
      return mqkv::report_error(MQ_ERR_CUDA,
                                "mq_decode_attn_noalloc: address of the scratch array: %s",
                                cudaGetErrorString(err));
  }
  // With no scratch (need == 0: invalid arguments) the capacity passed is 0,
  // so mq_decode_attn's argument checks report exactly what they report for a
  // caller with no workspace.
  return mq_decode_attn(shape, h_seq_lens, layout, packed, q, q_dtype, softmax_scale, out,
                        scratch, scratch ? (size_t)MQ_NOALLOC_SCRATCH_BYTES : 0, stream);
}
