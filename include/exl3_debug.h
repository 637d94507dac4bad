/*
 * exl3_debug.h -- test hooks of the EXL3 B200 library (not needed by users).
 *
 * Every device-side wait in the library (mbarrier phases, stage hand-offs) is
 * bounded in wall time, 1 s by default; when the bound is reached the kernel
 * records EXL3_ERR_TIMEOUT in the workspace status word and returns early.
 * Tests shorten the bound to make a wait run out on purpose, without any
 * fault or hang, and check that the status is reported.
 */
#ifndef EXL3_B200_DEBUG_H
#define EXL3_B200_DEBUG_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Set the bound of device-side waits for launches made after this call, in
 * nanoseconds; 0 restores the default (1 s).  Process-wide. */
void exl3_debug_set_wait_limit_ns(uint64_t ns);

/* Current bound in nanoseconds. */
uint64_t exl3_debug_wait_limit_ns(void);

#ifdef __cplusplus
}
#endif

#endif /* EXL3_B200_DEBUG_H */
