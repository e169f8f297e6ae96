/*
 * quest_debug.h -- fault injection for tests of the library's own error paths.
 *
 * The pages define no failure handling; this header has no counterpart on them.
 * It lets a test make the library's error paths run without faulting a GPU:
 * the fault is a decision taken on the host, never a bad address, a trap or an
 * unbounded wait on the device.
 *
 * A fault is armed for the calling host thread and is consumed by the next call,
 * on that thread, of an entry point of include/quest.h that gets past its
 * argument checks to the point of launching (a call rejected with QUEST_EINVAL,
 * or one with no rows to process, leaves it armed).
 */
#ifndef QUEST_B200_DEBUG_H
#define QUEST_B200_DEBUG_H

#include "quest.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum quest_fault {
    QUEST_FAULT_NONE = 0,          /* disarm */
    /* The call launches nothing and returns QUEST_ECUDA as if the launch had
     * failed (quest_last_error_message() says the failure was injected); its
     * outputs are left untouched. */
    QUEST_FAULT_LAUNCH = 1,
    /* Consumed only by quest_w4a4_linear: the call runs the one-CTA-per-tile
     * kernel (whatever M is) with its operand copies withheld and every pipeline
     * wait bounded at 1 ms, so the waits run out with no copy or MMA in flight.
     * The call returns QUEST_OK (the launch succeeded), y is incomplete, and the
     * next quest_device_status() reports QUEST_ETIMEOUT, then clears it. */
    QUEST_FAULT_WAIT_TIMEOUT = 2
} quest_fault;

/* Arms `fault` for the calling host thread (replacing any armed fault).
 * Returns QUEST_OK, or QUEST_EINVAL for an unknown value. */
quest_status quest_debug_inject_fault(quest_fault fault);

#ifdef __cplusplus
}
#endif

#endif /* QUEST_B200_DEBUG_H */
