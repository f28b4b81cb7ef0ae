// rope_fast_pairx_staged.cu -- instantiations of the item-based rope kernel:
// PAIRX layout (NeoX rows, one vector per lane, the partner half by shuffle),
// angles staged per token in shared memory.
#include "rope_fast.cuh"

namespace qkr {

KernelFn pick_fast_pairx_staged(int lpr, int ns, int u, bool norm, int rmode)
{
    return pick_fast<PAIRX, false>(lpr, ns, u, norm, rmode);
}

}  // namespace qkr
