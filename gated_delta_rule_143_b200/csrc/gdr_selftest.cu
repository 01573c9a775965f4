// gdr_selftest.cu -- a self-test of the bounded waits the tensor-core kernels rely on.
//
// The warp-specialised kernels never wait without a limit: every mbarrier wait and every wait on a
// flag written by another CTA gives up after a wall-clock bound, records GDR_ERR_TIMEOUT in the
// status word and raises the CTA's abort flag, so that the other roles of the CTA stop waiting too.
// This kernel lays out the same chain of roles as the state pass -- a copy role waiting on a ring
// flag, an MMA-issue role waiting on the copy role's mbarrier, epilogue warps waiting on the issue
// role's mbarrier -- but the ring flag is one that nothing ever sets. The copy role's wait has a
// short bound, the others' a bound 100 times longer: the copy role's wait expires, the abort flag
// releases the others, and the kernel ends after about one short bound (not 100) with the status
// word set, leaving the context usable.
#include "gdr_sm100.cuh"

namespace gdr {
namespace {

__device__ int g_selftest_flag = 0;  // never written: the ring flag that does not come

__global__ void bounded_wait_selftest_kernel(const int* flag, uint64_t limit_ns, int* status,
                                             unsigned long long* elapsed_ns) {
    using namespace sm100;
    __shared__ uint64_t full, done;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        mbar_init(&done, 1);
        fence_mbar_init();
        abort_flag = 0;
    }
    __syncthreads();
    const uint64_t t0 = globaltimer_ns();
    if (warp == 0) {  // copy role: waits for the producer's flag, then would hand the block on
        if (lane == 0 && flag_wait_geq(flag, 1, status, &abort_flag, 1024, limit_ns)) mbar_arrive(&full);
        __syncwarp();
    } else if (warp == 1) {  // issue role: waits for the copy, then would start the products
        if (lane == 0 && mbar_wait_abort(&full, 0, status, &abort_flag, 100 * limit_ns)) mbar_arrive(&done);
        __syncwarp();
    } else {  // epilogue warps: wait for the products
        mbar_wait_abort(&done, 0, status, &abort_flag, 100 * limit_ns);
    }
    __syncthreads();
    if (threadIdx.x == 0) *elapsed_ns = globaltimer_ns() - t0;
}

__device__ unsigned long long g_selftest_elapsed = 0;

}  // namespace

cudaError_t launch_bounded_wait_selftest(int* status, uint64_t limit_ns, cudaStream_t stream) {
    void* flag = nullptr;
    void* el = nullptr;
    cudaError_t err = cudaGetSymbolAddress(&flag, g_selftest_flag);
    if (err == cudaSuccess) err = cudaGetSymbolAddress(&el, g_selftest_elapsed);
    if (err != cudaSuccess) return err;
    bounded_wait_selftest_kernel<<<1, 192, 0, stream>>>(static_cast<const int*>(flag), limit_ns, status,
                                                        static_cast<unsigned long long*>(el));
    return cudaGetLastError();
}

cudaError_t read_bounded_wait_selftest_elapsed(unsigned long long* elapsed_ns) {
    return cudaMemcpyFromSymbol(elapsed_ns, g_selftest_elapsed, sizeof(*elapsed_ns));
}

}  // namespace gdr
