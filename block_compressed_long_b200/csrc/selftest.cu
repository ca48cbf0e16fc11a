// selftest.cu -- a check of the bounded device-side wait every kernel uses.
//
// The kernels' waits on mbarriers (bulk-copy and tensor-core completions,
// copies between the CTAs of a cluster) give up after a wall-clock limit and
// report LBCA_ERR_TIMEOUT through the status word instead of spinning forever.
// A real copy always completes, so this entry point builds the situation on
// purpose: one CTA waits on an mbarrier that nothing arrives at (or, as the
// control, at which its own thread arrives first), with the same helper and a
// short limit, and reports what the helper returned.
#include "common.cuh"
#include "lbca.h"

namespace lbca {
namespace {

__global__ void bounded_wait_kernel(int32_t arrive, uint64_t limit_ns, int32_t* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && arrive)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&bar)) : "memory");
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0, limit_ns);
    if (!__syncthreads_and(ok) && threadIdx.x == 0) set_status(status, LBCA_ERR_TIMEOUT);
}

}  // namespace
}  // namespace lbca

extern "C" lbca_status lbca_selftest_bounded_wait(int32_t arrive, uint64_t limit_ns, int32_t* d_status,
                                                  lbca_stream_t stream) {
    if (!d_status || (arrive != 0 && arrive != 1) || limit_ns == 0 || limit_ns > 2000000000ull) return LBCA_ERR_ARG;
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return LBCA_ERR_CUDA;
    if (major != 10 || minor != 0) return LBCA_ERR_UNSUPPORTED;
    lbca::bounded_wait_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(arrive, limit_ns, d_status);
    return cudaGetLastError() == cudaSuccess ? LBCA_OK : LBCA_ERR_CUDA;
}
