/*
 * kivi_debug.h - entry point of the debug build of the library
 * (libkivi_debug.so, compiled with KIVI_DEBUG_BUILD, KIVI_DEBUG_BOUNDS and a
 * short wait budget).  The regular libkivi.so does not export it.
 *
 * The pages have no counterpart: this build exists to test the library's own
 * failure reporting without faulting a GPU.
 *   - Every mbarrier wait of the decode kernel gives up after about 1 ms
 *     (KIVI_DEBUG_WAIT_CYCLES) instead of about 2 s, sets bit 1 of the device
 *     status word and stops issuing work; the call completes and the host
 *     reads KIVI_ERR_DEVICE from kivi_check_device_status.
 *   - Every copy the decode kernel issues is first checked against the
 *     buffers implied by the configuration; an index outside them sets bit 8
 *     of the status word and the copy is skipped.
 */
#ifndef KIVI_DEBUG_H
#define KIVI_DEBUG_H

#include <stdint.h>

#include "kivi.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Adds `bytes` to every copy size the decode kernel expects on its mbarriers
 * (0 restores normal operation).  Every issued copy still lands whole; the
 * barrier simply waits for bytes that never come, so the bounded wait runs out.
 * Returns KIVI_ERR_CUDA if the device variable cannot be written. */
kivi_status kivi_debug_overstate_copies(uint32_t bytes);

#ifdef __cplusplus
}
#endif

#endif /* KIVI_DEBUG_H */
