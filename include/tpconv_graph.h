/* Graph preprocessing for the streaming convolution: a spatial node order.
 *
 * The receiver traversal of Sobek (section 4: each receiver streams over its incoming
 * edges and gathers the source rows x_j, and the source traversal gathers m_bar rows)
 * reads node rows in the order the graph lists them.  Numbering nodes along a Morton
 * (Z-order) curve of their positions puts the neighbours of a receiver close together
 * in memory, so those gathers hit the same cache lines and L2 sectors.  These calls
 * compute such an order and apply it to a graph and to node arrays; the convolution
 * entry points (tpconv.h) then run on the renumbered graph unchanged, and their
 * results are the renumbered results of the original graph.
 *
 * All calls are asynchronous on `stream`, allocate nothing and use only the caller's
 * workspace.  Pointers are device pointers; int32 indices.
 */
#ifndef TPCONV_GRAPH_H
#define TPCONV_GRAPH_H

#include <stddef.h>
#include <stdint.h>

#include "tpconv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Workspace bytes of tpconv_spatial_order for N nodes. */
tpconv_status tpconv_spatial_order_workspace_bytes(int64_t N, size_t* bytes);

/* perm[k] = the old id of the node placed at position k.  Nodes are sorted by the
 * 30-bit Morton code of their position, ties by node id, so the order is unique.  The
 * code interleaves (x lowest bit, then y, then z) the cell indices
 *   c_a = min(1023, floor((pos_a - lo_a) * (1024 / (hi_a - lo_a))))   (0 when hi_a == lo_a)
 * over the bounding box [lo, hi] of pos, evaluated in float32.
 * pos [N][3] float32, perm [N] int32 (written).  Errors: INVALID_ARG (N < 0 or
 * N >= 2^31, NULL pointers with N > 0), WORKSPACE_TOO_SMALL, CUDA. */
tpconv_status tpconv_spatial_order(int64_t N, const float* pos, int32_t* perm, void* ws, size_t ws_bytes,
                                   struct CUstream_st* stream);

/* Renumber a receiver-sorted CSR by a permutation perm (perm[k] = old id at k):
 * row k of the result lists the sources of old receiver perm[k] in their original
 * order, each relabelled old -> new.  row_ptr_out [N+1], src_out [E] and inv [N]
 * (inv[old] = new) are written.  perm must be a permutation of 0..N-1; entries out of
 * range are skipped (no memory outside the arrays is touched) and leave the result
 * unspecified.  Errors: INVALID_ARG, CUDA. */
tpconv_status tpconv_permute_graph(int64_t N, int64_t E, const int32_t* row_ptr, const int32_t* src,
                                   const int32_t* perm, int32_t* row_ptr_out, int32_t* src_out,
                                   int32_t* inv, struct CUstream_st* stream);

/* out[k][:] = in[perm[k]][:] for k < rows; rows of `width` float32 values (node
 * features, positions, gradients).  Out-of-range perm entries write zeros.
 * in and out must not overlap.  Errors: INVALID_ARG, CUDA. */
tpconv_status tpconv_gather_rows(int64_t rows, int64_t width, const float* in, const int32_t* perm,
                                 float* out, struct CUstream_st* stream);

#ifdef __cplusplus
}
#endif

#endif /* TPCONV_GRAPH_H */
