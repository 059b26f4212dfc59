// Test-only kernels for the bounded pipeline waits of libgqa (sm100_ptx.cuh: mbar_wait).
// One CTA waits on an mbarrier; in the timeout case nothing ever arrives on it, so the wait must give
// up after its time limit, set the timeout bit in the error word and raise the CTA's abort flag,
// and the kernel must return normally.  Built and run by tests/test_failure_detection.py.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../grouped_query_attention_gqa_b200/csrc/sm100_ptx.cuh"

using namespace gqa::ptx;

__global__ void wait_kernel(int* err, int* out, int arrive_first) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        abort_flag = 0;
    }
    __syncthreads();
    if (arrive_first && threadIdx.x == 0) mbar_arrive(&bar);
    const bool ok = mbar_wait(&bar, 0, err, &abort_flag);
    if (threadIdx.x == 0) {
        out[0] = ok ? 1 : 0;
        out[1] = abort_flag;
    }
}

// Returns 0 on success and fills ok / abort / error word / elapsed milliseconds.
extern "C" int run_wait(int arrive_first, int* ok, int* abort_flag, int* err_word, float* ms) {
    int *d_err = nullptr, *d_out = nullptr;
    if (cudaMalloc(&d_err, sizeof(int)) != cudaSuccess) return -1;
    if (cudaMalloc(&d_out, 2 * sizeof(int)) != cudaSuccess) return -1;
    cudaMemset(d_err, 0, sizeof(int));
    cudaMemset(d_out, 0xff, 2 * sizeof(int));
    cudaEvent_t a, b;
    cudaEventCreate(&a);
    cudaEventCreate(&b);
    cudaEventRecord(a);
    wait_kernel<<<1, 32>>>(d_err, d_out, arrive_first);
    cudaEventRecord(b);
    if (cudaEventSynchronize(b) != cudaSuccess) return -2;
    cudaEventElapsedTime(ms, a, b);
    int h_out[2];
    cudaMemcpy(h_out, d_out, sizeof(h_out), cudaMemcpyDeviceToHost);
    cudaMemcpy(err_word, d_err, sizeof(int), cudaMemcpyDeviceToHost);
    *ok = h_out[0];
    *abort_flag = h_out[1];
    cudaFree(d_err);
    cudaFree(d_out);
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
