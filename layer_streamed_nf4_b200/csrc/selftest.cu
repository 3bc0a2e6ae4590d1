// Self-test of the bounded wait every tensor-core kernel relies on: a kernel
// waits on an mbarrier that nothing ever arrives on, with a short limit, and
// must give up and report it instead of hanging; the context stays usable.
#include "common.cuh"
#include "launch.cuh"

namespace lsn {
namespace {

__device__ int g_wait_probe_result;

__global__ void wait_probe_kernel(long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);                       // one arrival expected, none will come
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) g_wait_probe_result = mbar_wait(&bar, 0, nullptr, limit_cycles) ? 0 : 1;
}

}  // namespace
}  // namespace lsn

using namespace lsn;

extern "C" lsn_status lsn_selftest_wait_timeout(int limit_us, lsn_stream_t stream) {
    LSN_CHECK_ARG(limit_us > 0 && limit_us <= 1000000, "lsn_selftest_wait_timeout: limit_us must be in [1, 1e6]");
    int dev = 0, khz = 0;
    LSN_CUDA_TRY(cudaGetDevice(&dev));
    LSN_CUDA_TRY(cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev));
    if (khz <= 0) khz = 2000000;
    const long long cycles = (long long)limit_us * (khz / 1000);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int minus_one = -1;
    LSN_CUDA_TRY(cudaMemcpyToSymbolAsync(g_wait_probe_result, &minus_one, sizeof(int), 0, cudaMemcpyHostToDevice, st));
    wait_probe_kernel<<<1, 32, 0, st>>>(cycles);
    LSN_CUDA_TRY(cudaGetLastError());
    int result = -1;
    LSN_CUDA_TRY(cudaMemcpyFromSymbolAsync(&result, g_wait_probe_result, sizeof(int), 0, cudaMemcpyDeviceToHost, st));
    LSN_CUDA_TRY(cudaStreamSynchronize(st));
    if (result == 1) return fail(LSN_ERR_TIMEOUT, "the bounded wait gave up as it should");
    return fail(LSN_ERR_STATE, "the bounded wait did not report a timeout (result " + std::to_string(result) + ")");
}
