// Failure-detection check of the bounded waits (fca_selftest_wait_timeout).
//
// Every spin-wait in this library goes through dev::mbar_wait, which gives up
// after dev::kWaitLimitNs of wall-clock time, records kErrWaitTimeout in a
// device error word and returns false, so that a kernel whose data never
// arrives ends with a status the host can read instead of hanging the GPU.
// This file makes such a wait run out on purpose, without any fault: one
// thread waits for phase 0 of a fresh mbarrier that nothing arrives on.
#include "fca_device.cuh"
#include "fca_internal.h"

namespace fca {

namespace {

__global__ void k_wait_selftest(int32_t* word) {
    __shared__ uint64_t bar;
    dev::mbar_init(&bar, 1);
    dev::fence_mbarrier_init();
    volatile int abort = 0;
    (void)dev::mbar_wait(&bar, 0, &abort, word);
}

}  // namespace

}  // namespace fca

extern "C" fca_status fca_selftest_wait_timeout(void* stream, int32_t* out_word) {
    if (!out_word) return FCA_ERR_INVALID_ARG;
    *out_word = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* word = nullptr;
    cudaError_t e = fca::note_cuda(cudaMallocAsync(reinterpret_cast<void**>(&word), sizeof(int32_t), s));
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return e == cudaErrorMemoryAllocation ? FCA_ERR_OOM : FCA_ERR_CUDA;
    }
    int32_t v = 0;
    e = fca::note_cuda(cudaMemsetAsync(word, 0, sizeof(int32_t), s));
    if (e == cudaSuccess) {
        fca::k_wait_selftest<<<1, 1, 0, s>>>(word);
        e = fca::note_cuda(cudaGetLastError());
    }
    if (e == cudaSuccess) e = fca::note_cuda(cudaMemcpyAsync(&v, word, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
    const cudaError_t ef = fca::note_cuda(cudaFreeAsync(word, s));
    const cudaError_t es = fca::note_cuda(cudaStreamSynchronize(s));
    if (e != cudaSuccess || ef != cudaSuccess || es != cudaSuccess) {
        (void)cudaGetLastError();
        return FCA_ERR_CUDA;
    }
    *out_word = v;
    return FCA_OK;
}
