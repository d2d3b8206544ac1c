// selftest.cu -- exercises the failure path of the bounded device waits.
//
// Every wait of the tensor-core kernels on an mbarrier gives up after a time limit, records
// NQ_ERR_TIMEOUT in the device error word and lets the kernel finish; nq_sync_status reports
// and clears it.  This entry point makes exactly that happen on purpose, without a fault: one
// thread waits, with a short limit, on an mbarrier that nothing ever completes.
#include "tc_common.cuh"

namespace nq {

__global__ void __launch_bounds__(32) bounded_wait_kernel(unsigned int* err, uint64_t limit_ns) {
    __shared__ __align__(8) unsigned long long bar;
    const uint32_t b = tc::smem_u32(&bar);
    if (threadIdx.x == 0) {
        tc::mbar_init(b, 1);  // one arrival expected; none is ever made
        tc::mbar_fence_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) tc::mbar_wait_for(b, 0u, err, limit_ns);  // gives up after limit_ns
}

}  // namespace nq

extern "C" NQ_API nq_status nq_selftest_bounded_wait(int64_t limit_us, void* stream) {
    if (limit_us < 1000 || limit_us > 2000000) return NQ_ERR_SHAPE;
    unsigned int* err = nq_host::error_word();
    if (!err) return NQ_ERR_DEVICE;
    const uint64_t limit_ns = static_cast<uint64_t>(limit_us) * 1000u;
    nq::bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_ns);
    return cudaGetLastError() == cudaSuccess ? NQ_OK : NQ_ERR_LAUNCH;
}
