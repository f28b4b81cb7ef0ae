// rope_stream_paired.cu -- instantiations of the streaming rope kernel
// (cp.async row ring, staged angles) for the PAIRED layout.
#include "rope_stream.cuh"

namespace qkr {

KernelFn pick_stream_paired(int lpr, int ns, int u, bool norm)
{
    return pick_stream<PAIRED>(lpr, ns, u, norm);
}

}  // namespace qkr
