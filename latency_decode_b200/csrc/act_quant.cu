// act_quant.cu -- A1: dynamic per-tensor e4m3 quantisation of the GEMM input.
//
// [XZY] "CUDA 内核优化与融合", item "运算融合", and [NV] "CUDA kernel
// optimisation and fusion": a Quantize step is fused ahead of the FP8 GEMM so
// the GEMM consumes e4m3 activations.  Scale rule (per-tensor, dynamic):
//   amax = max|x|, inv = 448/amax, s_x = amax/448 (both single IEEE roundings),
//   x_q  = e4m3_rn_satfinite(x * inv) (one IEEE rounding for the product).
//
// One thread-block cluster of C <= 8 CTAs covers the whole [M][K] input: each
// CTA reduces |x| over its slice, the cluster merges the C partial maxima
// through distributed shared memory (no global round trip), and each CTA then
// quantises its own slice from registers (the input is read from memory once).
#include <cuda_fp8.h>

#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

constexpr int kAqThreads = 512;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float absmax8(uint4 u) {
  float m = fabsf(bf16_lo(u.x));
  m = fmaxf(m, fabsf(bf16_hi(u.x)));
  m = fmaxf(m, fabsf(bf16_lo(u.y)));
  m = fmaxf(m, fabsf(bf16_hi(u.y)));
  m = fmaxf(m, fabsf(bf16_lo(u.z)));
  m = fmaxf(m, fabsf(bf16_hi(u.z)));
  m = fmaxf(m, fabsf(bf16_lo(u.w)));
  m = fmaxf(m, fabsf(bf16_hi(u.w)));
  return m;
}

__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, float inv) {
  const __nv_fp8x2_storage_t a = __nv_cvt_float2_to_fp8x2(
      make_float2(__fmul_rn(bf16_lo(w0), inv), __fmul_rn(bf16_hi(w0), inv)), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(
      make_float2(__fmul_rn(bf16_lo(w1), inv), __fmul_rn(bf16_hi(w1), inv)), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16);
}

// Launched as one cluster of gridDim.x CTAs.
__global__ void __launch_bounds__(kAqThreads) act_quant_kernel(const uint16_t* __restrict__ x, int n,
                                                               uint8_t* __restrict__ xq,
                                                               float* __restrict__ s_x) {
  __shared__ float warp_max[kAqThreads / 32];
  __shared__ float cta_amax;

  // x may be produced by the preceding kernel: wait before reading it (through
  // L2, ld.global.cg), then let the dependent GEMM start streaming its weights.
  pdl_wait();
  pdl_trigger();

  const int C = gridDim.x;
  const int r = static_cast<int>(cluster_rank());
  const int nv = n >> 3;  // 16-byte vectors of 8 bf16
  const int v0 = static_cast<int>(static_cast<long long>(nv) * r / C);
  const int v1 = static_cast<int>(static_cast<long long>(nv) * (r + 1) / C);
  const uint4* xv = reinterpret_cast<const uint4*>(x);

  // One pass over memory: this CTA's slice (<= kKeep vectors per thread, which
  // covers M*K <= 8*512*12*8 = 393216 with 8 CTAs) is loaded once, all loads in
  // flight together, and kept in registers for the quantisation after the
  // cluster amax; larger inputs read the remainder twice.
  constexpr int kKeep = 12;
  uint4 u[kKeep];
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < kKeep; ++j) {
    const int i = v0 + threadIdx.x + j * kAqThreads;
    u[j] = i < v1 ? __ldcg(xv + i) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int j = 0; j < kKeep; ++j) m = fmaxf(m, absmax8(u[j]));
  for (int i = v0 + threadIdx.x + kKeep * kAqThreads; i < v1; i += kAqThreads)  // larger inputs
    m = fmaxf(m, absmax8(__ldcg(xv + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float w = threadIdx.x < kAqThreads / 32 ? warp_max[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, o));
    if (threadIdx.x == 0) cta_amax = w;
  }
  cluster_sync();  // every CTA's partial maximum is now visible cluster-wide

  float amax = 0.0f;
  const uint32_t local = smem_u32(&cta_amax);
  for (int p = 0; p < C; ++p) amax = fmaxf(amax, dsmem_ld_f32(dsmem_addr(local, p)));

  uint2* q2 = reinterpret_cast<uint2*>(xq);
  const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
#pragma unroll
  for (int j = 0; j < kKeep; ++j) {
    const int i = v0 + threadIdx.x + j * kAqThreads;
    if (i < v1)
      q2[i] = amax > 0.0f ? make_uint2(quant4(u[j].x, u[j].y, inv), quant4(u[j].z, u[j].w, inv)) : make_uint2(0u, 0u);
  }
  for (int i = v0 + threadIdx.x + kKeep * kAqThreads; i < v1; i += kAqThreads) {
    const uint4 w = __ldcg(xv + i);
    q2[i] = amax > 0.0f ? make_uint2(quant4(w.x, w.y, inv), quant4(w.z, w.w, inv)) : make_uint2(0u, 0u);
  }
  if (r == 0 && threadIdx.x == 0) *s_x = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;

  cluster_sync();  // peers have finished reading cta_amax before this CTA exits
}

cudaError_t launch_act_quant(const uint16_t* x, int M, int K, uint8_t* xq, float* s_x,
                             cudaStream_t s, bool pdl) {
  const long long n = static_cast<long long>(M) * K;
  int C = static_cast<int>((n + 32767) / 32768);  // ~32K elements (64 KB of bf16) per CTA
  if (C < 1) C = 1;
  if (C > 8) C = 8;
  Launch L(dim3(C), dim3(kAqThreads), 0, s, static_cast<unsigned>(C), pdl);
  return cudaLaunchKernelEx(&L.cfg, act_quant_kernel, x, static_cast<int>(n), xq, s_x);
}

}  // namespace dl
