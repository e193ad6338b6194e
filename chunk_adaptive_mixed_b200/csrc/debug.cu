// debug.cu — the test hook of include/mqkv_debug.h: a one-shot flag per
// kernel that its host launcher consumes (debug_take) and turns into a
// withheld stage and a short wait bound for that one launch.
#include <atomic>

#include "common.cuh"
#include "mqkv_debug.h"

namespace mqkv {
namespace {
std::atomic<uint32_t> g_armed{0};
}  // namespace

bool debug_take(uint32_t kernel_bit) {
  if ((g_armed.load(std::memory_order_relaxed) & kernel_bit) == 0) return false;
  return (g_armed.fetch_and(~kernel_bit, std::memory_order_acq_rel) & kernel_bit) != 0;
}

}  // namespace mqkv

extern "C" mq_status mq_debug_arm_wait_timeout(uint32_t kernels) {
  if (kernels & ~MQ_DEBUG_ROUTER) return MQ_ERR_INVALID_ARG;
  mqkv::g_armed.fetch_or(kernels, std::memory_order_acq_rel);
  return MQ_OK;
}
