// selftest.cu -- exercises the bounded-wait mechanism every kernel of the library relies on,
// without any fault: the threads of one small CTA wait on an mbarrier phase that nothing
// will ever complete.  Each wait gives up after the usual limit (about a second of SM
// clocks) or as soon as another thread of the CTA has given up (the abort flag), records
// CSA_ERR_DEVICE_TIMEOUT and returns.  Each thread records whether its wait returned
// "gave up" and how many clocks it spent.
#include <cuda_runtime.h>
#include <stdint.h>

#include "csa_internal.h"
#include "ptx.cuh"

namespace csa {

struct SelftestOut {
    int gave_up[128];        // 1 when the wait returned false
    long long cycles[128];   // clocks spent in the wait
};

__global__ void __launch_bounds__(128, 1) k_selftest_wait(int* status, SelftestOut* out) {
    __shared__ uint64_t never[2];
    __shared__ int abort_flag;
    const int tid = threadIdx.x;
    if (tid == 0) {
        mbar_init(&never[0], 1);
        mbar_init(&never[1], 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    volatile int* abort_v = &abort_flag;
    const long long t0 = clock64();
    const bool ok = mbar_wait(&never[tid < 32 ? 0 : 1], 0, abort_v, status);
    out->cycles[tid] = clock64() - t0;
    out->gave_up[tid] = ok ? 0 : 1;
}

int run_selftest_wait(int* status, void* out, cudaStream_t st) {
    k_selftest_wait<<<1, 128, 0, st>>>(status, static_cast<SelftestOut*>(out));
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_LAUNCH;
}

size_t selftest_out_bytes() { return sizeof(SelftestOut); }

}  // namespace csa
