// Self-test of the bounded waits the decode kernels rely on (see
// mla_selftest_wait_timeout in include/mla_sparse_decode.h).  Its own
// translation unit: it shares only the inline-PTX layer (ptx.cuh), whose
// wait() is the one every kernel uses.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mla_sparse_decode.h"
// The inline-PTX layer (its out-of-line helpers are static: this translation
// unit and the decode's each hold their own copy of the same wait()).
#include "ptx.cuh"

namespace {

// One thread waits on an mbarrier that nothing arrives on.  After
// kWaitLimitNs the wait must give up, set the CTA's abort flag and write
// MLA_ERR_DEVICE_TIMEOUT to *d_status; a second wait must then return at
// once.  *d_result: bit 0 = the first wait reported completion, bit 1 = the
// second did, bit 2 = the abort flag was set (a healthy result is exactly 4).
__global__ void __launch_bounds__(32, 1) wait_selftest_kernel(int* d_status, int* d_result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mla::mbar_init(mla::smem_u32(&bar), 1);
    mla::fence_mbarrier_init_cluster();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const mla::AbortState ab{&abort_flag, d_status};
    const bool first = mla::wait(mla::smem_u32(&bar), 0, ab);
    const bool second = mla::wait(mla::smem_u32(&bar), 0, ab);
    *d_result = (first ? 1 : 0) | (second ? 2 : 0) | (*ab.flag ? 4 : 0);
  }
}

}  // namespace

extern "C" int mla_selftest_wait_timeout(int* d_status, int* d_result, cudaStream_t stream) {
  if (!d_status || !d_result || (reinterpret_cast<uintptr_t>(d_status) & 3u) ||
      (reinterpret_cast<uintptr_t>(d_result) & 3u))
    return MLA_ERR_INVALID_ARG;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (major != 10 || minor != 0) return MLA_ERR_UNSUPPORTED;
  wait_selftest_kernel<<<1, 32, 0, stream>>>(d_status, d_result);
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
