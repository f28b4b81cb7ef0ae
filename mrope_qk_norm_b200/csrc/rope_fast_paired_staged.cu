// rope_fast_paired_staged.cu -- instantiations of the item-based rope kernel:
// PAIRED layout, angles staged per token in shared memory.
#include "rope_fast.cuh"

namespace qkr {

KernelFn pick_fast_paired_staged(int lpr, int ns, int u, bool norm, int rmode)
{
    return pick_fast<PAIRED, false>(lpr, ns, u, norm, rmode);
}

}  // namespace qkr
