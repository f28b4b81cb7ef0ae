// rope_stream_vector.cu -- instantiations of the streaming rope kernel
// (cp.async row ring, staged angles) for the VECTOR layout.
#include "rope_stream.cuh"

namespace qkr {

KernelFn pick_stream_vector(int lpr, int ns, int u, bool norm)
{
    return pick_stream<VECTOR>(lpr, ns, u, norm);
}

}  // namespace qkr
