/* mqkv_debug.h — test hooks of libmqkv.  Not part of the serving interface:
 * they exist so that tests can drive failure paths on a real GPU without a
 * fault, and do nothing unless called.
 *
 * Every wait a libmqkv kernel makes on a copy or a peer is bounded: when the
 * bound runs out the kernel sets MQ_DEV_WAIT_TIMEOUT in the device status
 * word (read with mq_device_status), lets the copies it started land,
 * releases what it holds (tensor memory) and returns, leaving the context
 * usable.  In normal operation nothing makes such a wait run out. */
#ifndef MQKV_DEBUG_H
#define MQKV_DEBUG_H

#include <stdint.h>

#include "mqkv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Kernels the hook can reach (bit mask). */
#define MQ_DEBUG_ROUTER 0x1u /* the tensor-core router of mq_route_chunks */

/* Arms, for the next launch in this process of each kernel named in
 * `kernels`, a stage whose arrival is withheld, with the kernel's wait bound
 * cut to a few thousand polls: that launch stops at its first wait, sets
 * MQ_DEV_WAIT_TIMEOUT and produces no valid output.  One launch consumes the
 * arming; later launches run normally.  Host only: no CUDA call is made.
 * Returns MQ_OK, or MQ_ERR_INVALID_ARG for bits outside MQ_DEBUG_*. */
mq_status mq_debug_arm_wait_timeout(uint32_t kernels);

#ifdef __cplusplus
}
#endif

#endif /* MQKV_DEBUG_H */
