/*
 * muon_debug.h -- extra entry points of the bounds-checked build of the
 * library (libmuon_checked.so, built with -DMUON_BOUNDS_CHECK by
 * newton_schulz_norm_b200.build with checked=True).  The regular libmuon.so
 * does not export them.
 *
 * In the checked build every kernel validates the entries of the tables it
 * reads (tile lists, problem tables, work items) against the sizes it was
 * launched with before using them, and turns an invalid entry into
 * MUON_ERR_INVALID_ARG in the status word (reported by muon_status) instead
 * of an access out of bounds.  The entry point below lets a test plant such
 * an entry.  There is no counterpart of either on the pages; they are this
 * library's stand-in for a memory checker.
 */
#ifndef MUON_DEBUG_H_
#define MUON_DEBUG_H_

#include "muon.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * muon_debug_set_tile_row -- overwrite the first output row (i0) of tile
 * `index` of the chain launch of `ns_steps` iterations cached for this shape
 * set (built by an earlier muon_step with these shapes and ns_steps), so
 * that the next such muon_step meets an invalid tile.  Synchronises the
 * device.  Returns MUON_OK, or MUON_ERR_INVALID_ARG if no such plan, chain
 * or tile exists.  The plan stays corrupted until muon_release().
 */
MUON_API int muon_debug_set_tile_row(const int64_t* shapes, int n, int ns_steps, int index, int i0);

#ifdef __cplusplus
}
#endif

#endif /* MUON_DEBUG_H_ */
