// pack.cu -- A0: offline weight swizzle ([XZY] "GEMM 权重重排"; [NV] "CUDA
// kernel optimisation and fusion").  Rearranges a canonical row-major e4m3
// [N][K] weight into 16 KB blocks, each the exact shared-memory image of a
// 128-row x 128-K-byte tcgen05 operand in the K-major 128-byte-swizzle layout,
// ordered so that the K range one GEMM CTA streams is one contiguous run of
// bytes.  The GEMM then fetches weights with plain bulk copies (no tensor map).
// Layout definition: include/dl.h, dl_pack_fp8_weight.
#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

// One thread per 16-byte chunk of the packed output.
__global__ void pack_kernel(const uint8_t* __restrict__ w, uint8_t* __restrict__ out, int N, int K,
                            int kind) {
  const long long chunks = static_cast<long long>(N) * K / 16;
  const int KB = K / 128;
  const int F = N / 2;
  for (long long c = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; c < chunks;
       c += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long blk = c >> 10;          // 1024 chunks of 16 B per 16 KB block
    const int in_blk = static_cast<int>(c & 1023);
    const int r = in_blk >> 3;              // 8 chunks per 128-byte row image
    const int pos = in_blk & 7;             // physical chunk position within the row
    const int src_chunk = pos ^ (r & 7);    // 128-byte swizzle
    long long row;
    int kb;
    if (kind == DL_PACK_SWIGLU) {
      const long long pair = blk >> 1;
      const int which = static_cast<int>(blk & 1);  // 0 gate, 1 up
      const long long t = pair / KB;
      kb = static_cast<int>(pair % KB);
      row = (which ? F : 0) + t * 128 + r;
    } else {
      const long long t = blk / KB;
      kb = static_cast<int>(blk % KB);
      row = t * 128 + r;
    }
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(w + row * K + kb * 128 + src_chunk * 16));
    reinterpret_cast<uint4*>(out)[c] = v;
  }
}

cudaError_t launch_pack(const uint8_t* w_nk, uint8_t* w_packed, int N, int K, int kind,
                        cudaStream_t s) {
  const long long chunks = static_cast<long long>(N) * K / 16;
  long long blocks = (chunks + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  Launch L(dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, 0, false);
  return cudaLaunchKernelEx(&L.cfg, pack_kernel, w_nk, w_packed, N, K, kind);
}

}  // namespace dl
