// rope_fast_vector_staged.cu -- instantiations of the item-based rope kernel:
// VECTOR layout, angles staged per token in shared memory.
#include "rope_fast.cuh"

namespace qkr {

KernelFn pick_fast_vector_staged(int lpr, int ns, int u, bool norm, int rmode)
{
    return pick_fast<VECTOR, false>(lpr, ns, u, norm, rmode);
}

}  // namespace qkr
