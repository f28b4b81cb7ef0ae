// rope_fast_paired_direct.cu -- instantiations of the item-based rope kernel:
// PAIRED layout, angles read per item straight from an fp32 table.
#include "rope_fast.cuh"

namespace qkr {

KernelFn pick_fast_paired_direct(int lpr, int ns, int u, bool norm, int rmode)
{
    return pick_fast<PAIRED, true>(lpr, ns, u, norm, rmode);
}

}  // namespace qkr
