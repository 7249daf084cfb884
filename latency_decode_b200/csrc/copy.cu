// copy.cu -- a PDL-chained copy kernel for a decode step's inputs and outputs.
//
// [XZY] "程序化依赖启动（PDL）" and [NV] "Programmatic Dependent Launch": the
// gaps between consecutive kernels of a step are closed by letting the next
// kernel start its independent preamble (for the GEMMs: streaming their static
// weights) while the previous one still runs.  A cudaMemcpy node between two
// kernels is not a kernel and breaks that chain; this kernel moves the bytes
// instead, so a step that begins by fetching its activations from the host
// (or ends by returning its results) stays one PDL chain.  Under unified
// addressing, pinned host memory from cudaHostAlloc is directly addressable by
// kernels, so either side of the copy may be host memory.
#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

constexpr int kCopyThreads = 256;
constexpr int kCopyBatch = 4;  // 16-byte loads in flight per thread per round

__global__ void __launch_bounds__(kCopyThreads) copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          long long n16, int wait_first) {
  // src may be written, and dst still read, by the preceding kernel, unless
  // the caller has vouched that neither is
  if (wait_first) pdl_wait();
  pdl_trigger();
  const long long stride = static_cast<long long>(gridDim.x) * kCopyThreads;
  for (long long i0 = blockIdx.x * static_cast<long long>(kCopyThreads) + threadIdx.x; i0 < n16;
       i0 += stride * kCopyBatch) {
    uint4 v[kCopyBatch];
#pragma unroll
    for (int j = 0; j < kCopyBatch; ++j) {
      const long long i = i0 + j * stride;
      if (i < n16) v[j] = __ldcg(src + i);
    }
#pragma unroll
    for (int j = 0; j < kCopyBatch; ++j) {
      const long long i = i0 + j * stride;
      if (i < n16) dst[i] = v[j];
    }
  }
}

cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t s, bool pdl, bool wait_first) {
  const long long n16 = static_cast<long long>(bytes / 16);
  if (n16 == 0) return cudaSuccess;
  long long blocks = (n16 + kCopyThreads * kCopyBatch - 1) / (kCopyThreads * kCopyBatch);
  if (blocks > 2ll * sm_count()) blocks = 2ll * sm_count();
  Launch L(dim3(static_cast<unsigned>(blocks)), dim3(kCopyThreads), 0, s, 0, pdl);
  return cudaLaunchKernelEx(&L.cfg, copy_kernel, reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst),
                            n16, wait_first ? 1 : 0);
}

}  // namespace dl
