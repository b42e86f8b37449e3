// wq_sk_debug.cu -- host view of the stream-K cuts that the persistent
// kernels share (stream-K GEMV and GEMM, the role-split W4A16 GEMM, the
// integer tensor-core GEMMs), computed by the same helpers the kernels run
// (sk_start, sk_owner, SkTable in wq_device.cuh), so the tests can check the
// partition and the fix-ups' contributor ranges on the CPU.
//
// The weights are one stream of U units (128-row panel x 128-k block,
// panel-major, KB k-blocks per panel); CTA c of G takes units
// [start(c), start(c + 1)).  A panel whose units meet several ranges is
// finished by the last of those CTAs to take its ticket; each CTA keeps at
// most two partial slots (slot 0 for its first panel, 1 for its last).
#include <climits>

#include "wq.h"
#include "wq_device.cuh"

extern "C" int wq_stream_k_plan(long long U, int G, int KB, int *start, int *first, int *owner_table,
                                int *owner_div)
{
    if (!start || !first || !owner_table || !owner_div)
        return WQ_ERR_NULL;
    // the launchers cap the grid at the unit count, so no range is empty
    if (U < 1 || U > INT_MAX || G < 1 || G > U || KB < 1)
        return WQ_ERR_SHAPE;
    // the per-CTA table, filled as every CTA fills its shared-memory copy
    for (int c = 0; c <= G; ++c) {
        start[c] = wq::sk_start(U, G, c);
        first[c] = start[c] / KB;
    }
    const wq::SkTable sk{start, first};
    for (int u = 0; u < (int)U; ++u) {
        owner_table[u] = sk.owner(u, G);
        owner_div[u] = wq::sk_owner(U, G, u);
    }
    return WQ_OK;
}
