/*
 * dsa_probe.h - measurement support for the benchmark's roofline (libdsaprobe.so); not part
 * of the layer.  The pages have no counterpart: this measures the hardware the attention
 * runs on.
 *
 * The sparse attention's dominant traffic is a gather of random 256-byte rows (one KV head
 * of one selected cache row, for K and for V).  dsa_probe_gather reads random 256-byte rows
 * of one buffer in the attention's access shape -- a warp takes 32 row indices with one
 * load, shares them by shuffle and moves two rows (512 contiguous bytes) per instruction in
 * 16-byte pieces -- and does nothing else, so its rate is the ceiling that gather can reach
 * on that buffer: from L2 when the buffer fits there, from HBM otherwise.
 */
#ifndef DSA_PROBE_H
#define DSA_PROBE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Gather rate, in bytes per second, of random 256-byte rows of `buf`.
 *   buf      device, n_rows rows of 256 bytes (n_rows a power of two), 16-byte aligned
 *   idx      device int32 scratch of n_idx entries (a power of two, >= 32): receives the row
 *            indices (a counter-based hash masked to n_rows, so every access is in bounds)
 *   variant  0: loads into registers (all 16 row pairs of a 32-row chunk in flight);
 *            1: cp.async into a shared-memory ring of two chunks per warp;
 *            2, 3: as 0, 1 with each piece addressed by a 32-bit index of 16-byte units
 *            added to buf (n_rows <= 2^28) instead of 64-bit arithmetic
 *   blocks   CTAs of 256 threads; chunks_per_warp chunks of 32 rows per warp
 *   reps     timed launches after one untimed launch
 *   sink     device scratch of >= blocks * 256 16-byte words (written only in a case that
 *            does not occur: it keeps the loads from being removed)
 * Returns 0 on an invalid argument or a CUDA error.  Synchronous, on the legacy default
 * stream; the caller owns every buffer.
 */
double dsa_probe_gather(const void* buf, uint32_t n_rows, int32_t* idx, uint32_t n_idx,
                        int variant, int blocks, int chunks_per_warp, int reps, void* sink);

#ifdef __cplusplus
}
#endif

#endif /* DSA_PROBE_H */
