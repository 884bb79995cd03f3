// Test helper: the bounded mbarrier wait and the device error word that every
// liblq kernel relies on (lq_common.cuh), run on their own.  A wait on a
// barrier that one arrival completes must succeed; a wait on a barrier that
// nothing ever arrives on must give up after its budget, and the error report
// must land in the error word, first report winning.  No copy is in flight and
// every loop is bounded, so nothing here can hang or fault.
#include <cstdint>

#include "lq_common.cuh"

namespace {

__global__ void wait_probe_kernel(int32_t *err, long long *out, long long budget) {
    __shared__ __align__(8) uint64_t bars[2];
    if (threadIdx.x == 0) {
        lq::mbar_init(&bars[0], 1);
        lq::mbar_init(&bars[1], 1);
        lq::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    // bars[1]: the single expected arrival completes phase 0
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(lq::smem_u32(&bars[1])) : "memory");
    const bool done = lq::mbar_wait(&bars[1], 0u, budget);
    // bars[0]: no arrival ever comes, so the wait has to run out
    const long long t0 = clock64();
    const bool never = lq::mbar_wait(&bars[0], 0u, budget);
    const long long waited = clock64() - t0;
    if (!never) lq::report_error(err, LQ_DEVERR_TIMEOUT, 11, 22);
    lq::report_error(err, LQ_DEVERR_RANGE, 33, 44);      // a later report must not overwrite
    out[0] = done ? 1 : 0;
    out[1] = never ? 1 : 0;
    out[2] = waited;
}

}  // namespace

// Runs the probe with the given budget (SM clocks).  host_out receives
// {completed wait ok, empty wait ok, cycles waited, err[0], err[1], err[2]}.
// Returns the CUDA error code of the launch and copies (0 on success).
extern "C" int lq_test_wait_probe(long long budget, long long *host_out) {
    int32_t *err = nullptr;
    long long *out = nullptr;
    cudaError_t e = cudaMalloc(&err, 64 * sizeof(int32_t));
    if (e == cudaSuccess) e = cudaMalloc(&out, 3 * sizeof(long long));
    if (e == cudaSuccess) e = cudaMemset(err, 0, 64 * sizeof(int32_t));
    if (e == cudaSuccess) {
        wait_probe_kernel<<<1, 32>>>(err, out, budget);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    int32_t herr[3] = {0, 0, 0};
    long long hout[3] = {0, 0, 0};
    if (e == cudaSuccess) e = cudaMemcpy(hout, out, sizeof(hout), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(herr, err, sizeof(herr), cudaMemcpyDeviceToHost);
    for (int i = 0; i < 3; ++i) {
        host_out[i] = hout[i];
        host_out[3 + i] = herr[i];
    }
    if (out) cudaFree(out);
    if (err) cudaFree(err);
    return (int)e;
}
