// status.cu -- the library's device status word, and the launch-floor probe.
//
// Kernels that meet a condition the host could not check before the launch
// (rope_set_rows: a cache row index outside the cache, which the host cannot
// see without synchronising) set a bit here with atomicOr instead of writing
// out of bounds.  The word is per device and shared by every call of the
// process.  qkr_device_status reads it with one atomic exchange on the device
// (read and clear in one step, so a bit set by a kernel running concurrently
// on another stream is either returned by this read or left for the next
// one, never lost).

#include <mutex>

#include "qkr_internal.cuh"

namespace qkr {

__device__ unsigned int g_device_status;    // OR of the bits raised since the last clear
__device__ unsigned int g_status_snapshot;  // value taken by the last read

namespace {

__global__ void status_take_kernel(int reset)
{
    g_status_snapshot = reset ? atomicExch(&g_device_status, 0u) : atomicOr(&g_device_status, 0u);
}

std::mutex g_status_mu;  // one read at a time per process (they share the snapshot word)

// The launch floor: a kernel that does only what every library kernel does
// before its first memory access (the programmatic-launch wait and trigger).
__global__ void null_kernel()
{
    pdl_wait();
    pdl_trigger();
}

}  // namespace

cudaError_t launch_null(int64_t grid, int block, cudaStream_t stream, LaunchRecord *rec)
{
    cudaError_t e = launch(null_kernel, dim3((unsigned)grid), dim3(block), 0, stream, 1);
    if (e == cudaSuccess && rec) {
        *rec = LaunchRecord();
        rec->kernel = QKR_KERNEL_NULL;
        rec->block = block;
        rec->grid = grid;
        rec->launches = 1;
    }
    return e;
}

cudaError_t device_status_address(unsigned **addr)
{
    void *a = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&a, g_device_status);
    if (e == cudaSuccess)
        *addr = static_cast<unsigned *>(a);
    return e;
}

cudaError_t read_device_status(unsigned *status, bool reset)
{
    std::lock_guard<std::mutex> lock(g_status_mu);
    // legacy default stream: the exchange runs after the work of every
    // blocking stream; a copy from the symbol on the same stream follows it
    status_take_kernel<<<1, 1, 0, 0>>>(reset ? 1 : 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    return cudaMemcpyFromSymbol(status, g_status_snapshot, sizeof(unsigned));
}

}  // namespace qkr
