/*
 * sla2_test.h -- test hooks of libsla2.so (not part of the forward-pass API).
 */
#ifndef SLA2_TEST_H
#define SLA2_TEST_H
#include "sla2.h"
#ifdef __cplusplus
extern "C" {
#endif

/* Launches one warp that waits on a device barrier nothing ever signals. The
 * wait is bounded by budget_ns (1 ns .. 10 s); when it runs out the kernel
 * writes SLA2_ERR_DEVICE_TIMEOUT (5) into *status (a device word, zeroed first
 * on `stream`) and returns, leaving the context usable. Exercises the same
 * bounded-wait path every pipeline wait of the forward pass uses.
 * Returns SLA2_ERR_INVALID_ARG for a NULL status or a budget outside the range. */
sla2_status sla2_selftest_timeout(unsigned int* status, unsigned long long budget_ns, void* stream);

/* Sets the budget (ns) of every bounded device wait in later launches of this
 * process; 0 restores the default (2 s). */
void sla2_set_wait_budget_ns(unsigned long long ns);

#ifdef __cplusplus
}
#endif
#endif
