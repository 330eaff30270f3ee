// selftest.cu -- a drill for the failure-detection path of the bounded waits.
//
// One warp waits, through the same bounded mbarrier wait every tensor-core
// kernel uses, on an mbarrier that nothing ever arrives on.  The wait gives
// up after the caller's limit, latches DART_ERR_TIMEOUT with this kernel's id
// and the wait site in the device status word, and the kernel returns: no
// copy, tensor-core operation or TMEM allocation is in flight, so the context
// stays usable and the next call runs clean once dart_sync_status has read
// and cleared the word.
#include "sm100.cuh"

namespace dart {

constexpr int kDrillKernelId = 9;
constexpr int kDrillSite = 1;

namespace {

__global__ void __launch_bounds__(32) wait_drill_kernel(int* status, unsigned long long limit_ns) {
    __shared__ __align__(8) unsigned long long bar;
    __shared__ volatile int abort_flag;
    const uint32_t b = sm100::smem_u32(&bar);
    if (threadIdx.x == 0) {
        abort_flag = 0;
        sm100::mbar_init(b, 1);   // one arrival expected; none will come
        sm100::fence_mbar_init();
    }
    __syncwarp();
    const sm100::WaitCtx wc{&abort_flag, status, kDrillKernelId};
    sm100::mbar_wait_warp(b, 0, wc, kDrillSite, limit_ns);
}

}  // namespace

cudaError_t launch_wait_drill(int* status, unsigned long long limit_ns, cudaStream_t st) {
    wait_drill_kernel<<<1, 32, 0, st>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace dart
