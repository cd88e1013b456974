// A check of the library's failure handling that needs no fault: one CTA whose barrier wait can
// never complete (nothing ever arrives on it), to show that a bounded wait gives up, records its
// tag in a device error word, raises the CTA's abort flag so that the CTA's other waits return at
// once, and that the kernel then returns and leaves the context usable.
#include "sm100_ptx.cuh"

namespace {

constexpr int kErrSelfTest = 0x401;

__device__ int g_selftest_error = 0;
__device__ int g_selftest_out[4];

__global__ void __launch_bounds__(64) bounded_wait_kernel() {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        lad::ptx::mbar_init(lad::ptx::smem_u32(&bars[0]), 1);
        lad::ptx::mbar_init(lad::ptx::smem_u32(&bars[1]), 1);
        abort_flag = 0;
        lad::ptx::mbar_fence_init();
    }
    __syncthreads();
    volatile int *ab = &abort_flag;
    if (warp == 0) {
        // phase 0 of bars[0] never completes: this wait runs out after the limit
        const bool ok = lad::ptx::wait_bar(lad::ptx::smem_u32(&bars[0]), 0, ab, &g_selftest_error, kErrSelfTest);
        if (lane == 0) g_selftest_out[0] = ok ? 1 : 0;
    } else {
        // a second wait that cannot complete either, started half a limit later: it must return
        // when warp 0 raises the flag, half a limit before it would reach its own (another tag)
        const uint64_t ts = lad::dev::globaltimer_ns();
        while (lad::dev::globaltimer_ns() - ts < lad::dev::kWaitLimitNs / 2) {
        }
        const uint64_t t0 = lad::dev::globaltimer_ns();
        const bool ok = lad::ptx::wait_bar(lad::ptx::smem_u32(&bars[1]), 0, ab, &g_selftest_error, kErrSelfTest + 1);
        const uint64_t t1 = lad::dev::globaltimer_ns();
        if (lane == 0) {
            g_selftest_out[1] = ok ? 1 : 0;
            g_selftest_out[2] = static_cast<int>((t1 - t0) / 1000000ull);  // ms waited
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) g_selftest_out[3] = abort_flag;
}

}  // namespace

extern "C" int lad_check_bounded_wait(int *tag, int *results, void *stream) {
    using lad::set_error;
    if (!tag || !results) return set_error(LAD_EINVAL, "lad_check_bounded_wait: null output");
    cudaStream_t s = lad::as_stream(stream);
    int zero[4] = {0, 0, 0, 0};
    cudaError_t e = cudaMemcpyToSymbolAsync(g_selftest_out, zero, sizeof zero, 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_selftest_error, zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_check_bounded_wait: %s", cudaGetErrorString(e));
    bounded_wait_kernel<<<1, 64, 0, s>>>();
    int rc = lad::check_launch("lad_check_bounded_wait");
    if (rc != LAD_OK) return rc;
    e = cudaMemcpyFromSymbolAsync(results, g_selftest_out, 4 * sizeof(int), 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyFromSymbolAsync(tag, g_selftest_error, sizeof(int), 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_error(LAD_ECUDA, "lad_check_bounded_wait: %s", cudaGetErrorString(e));
    return LAD_OK;
}
