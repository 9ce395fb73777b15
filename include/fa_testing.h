/*
 * fa_testing.h -- test hooks of libfa.so.  Not part of the attention call:
 * the pages have no counterpart; these exist so that a test can pin which of
 * the library's equivalent kernels runs a call, and check each against the
 * same reference.  Production callers never need them.
 */
#ifndef FA_B200_TESTING_H
#define FA_B200_TESTING_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * fa_testing_set_prefill_tiles -- which tcgen05 prefill / dense attention
 * kernel runs every following fa_fwd*, fa_fwd_varlen and prefill-path
 * fa_kvcache_fwd* call.
 *   tiles  0 = the planner's choice (the default), 1 = the one-tile kernel,
 *          2 = the two-tile kernel on pairs of query tiles, 3 = the two-tile
 *          kernel on one query tile with its key range split between the two
 *          softmax warpgroups (packed sequences run as 2); anything else is
 *          FA_ERR_INVALID_ARG.
 * Process-wide and not synchronised: set it while no other thread is
 * calling the library, and set it back to 0 when done.
 */
int fa_testing_set_prefill_tiles(int32_t tiles);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_TESTING_H */
