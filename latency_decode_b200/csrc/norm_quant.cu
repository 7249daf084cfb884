// norm_quant.cu -- residual add + RMSNorm + Quantize: the producer of an FP8
// GEMM input, as one kernel.
//
// [XZY] "CUDA 内核优化与融合", item "运算融合", and [NV] "CUDA kernel
// optimisation and fusion" fuse (AllReduce +) RMSNorm + Quantize into one
// kernel ahead of the FP8 GEMM.  On one GPU the AllReduce is absent; the
// residual add of the pre-norm block takes its place:
//   h = bf16_rne(x + r)                         (the residual stream, bf16)
//   y = (h * rsqrt(mean(h^2) + eps)) * gamma     (fp32, per token row)
//   amax = max|y| over the whole [M][K] tensor, inv = 448/amax, s_x = amax/448
//   x_q = e4m3_rn_satfinite(y * inv)
// x_q and s_x land in a GEMM workspace, whose GEMM then runs with
// DL_FLAG_XQ_READY and skips its own quantisation.
//
// One thread-block cluster of C <= 8 CTAs covers the tensor.  Each CTA owns R
// consecutive token rows and 16/R warps per row; a row's h stays in registers
// from the load to the quantisation, so x and r are read from memory once.
// Row sums of squares are reduced in a fixed order (deterministic), the
// tensor amax across the cluster through distributed shared memory.
#include <cuda_fp8.h>

#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

constexpr int kNqThreads = 512;
constexpr int kNqWarps = kNqThreads / 32;
constexpr int kNqKeep = 10;  // 16-byte vectors of h per thread held in registers

struct NormQuantArgs {
  const uint16_t* x;
  const uint16_t* r;      // may be null
  uint16_t* h_out;        // may be null
  const uint16_t* gamma;  // [K]
  uint8_t* xq;            // [M][K]
  float* s_x;
  int M, K;
  int R;                  // rows per CTA (power of two, <= 16)
  float eps;
};

// h of vector v again, beyond the register set: from h_out when this thread
// stored it there (whatever h_out aliases), else recomputed from x and r.
__device__ __forceinline__ uint4 reload_h(const uint4* xv, const uint4* rv, const uint4* hv, int v) {
  if (hv != nullptr) return __ldcg(hv + v);
  const uint4 u = __ldcg(xv + v);
  return rv != nullptr ? add8_bf16(u, __ldcg(rv + v)) : u;
}

// Launched as one cluster of gridDim.x CTAs.
__global__ void __launch_bounds__(kNqThreads) add_rmsnorm_quant_kernel(const __grid_constant__ NormQuantArgs a) {
  __shared__ float red[kNqWarps];
  __shared__ float cta_amax;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = gridDim.x;
  const int crank = static_cast<int>(cluster_rank());
  const int WR = kNqWarps / a.R;          // warps per row
  const int TPR = WR * 32;                // threads per row
  const int rr = warp / WR;
  const int tr = (warp - rr * WR) * 32 + lane;
  const int row = crank * a.R + rr;
  const bool live = row < a.M;
  const int VR = a.K >> 3;                // 16-byte vectors per row
  const long long rbase = static_cast<long long>(row) * VR;
  const uint4* xv = reinterpret_cast<const uint4*>(a.x) + rbase;
  const uint4* rv = a.r != nullptr ? reinterpret_cast<const uint4*>(a.r) + rbase : nullptr;
  uint4* hv = a.h_out != nullptr ? reinterpret_cast<uint4*>(a.h_out) + rbase : nullptr;
  const uint4* gv = reinterpret_cast<const uint4*>(a.gamma);

  // gamma is a static input: its vectors are loaded before the wait for the
  // preceding kernel, so they are in registers when the norm needs them
  uint4 gk[kNqKeep];
#pragma unroll
  for (int j = 0; j < kNqKeep; ++j) {
    const int v = tr + j * TPR;
    gk[j] = (live && v < VR) ? __ldg(gv + v) : make_uint4(0u, 0u, 0u, 0u);
  }

  // x and r may be produced by the preceding kernel: wait before reading them,
  // then let the dependent GEMM start streaming its weights.
  pdl_wait();
  pdl_trigger();

  // ---- h = x (+ r), kept in registers; row sum of squares -------------------
  uint4 h[kNqKeep];
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < kNqKeep; ++j) {
    const int v = tr + j * TPR;
    h[j] = make_uint4(0u, 0u, 0u, 0u);
    if (live && v < VR) {
      h[j] = __ldcg(xv + v);
      if (rv != nullptr) h[j] = add8_bf16(h[j], __ldcg(rv + v));
    }
  }
#pragma unroll
  for (int j = 0; j < kNqKeep; ++j) {
    const int v = tr + j * TPR;
    if (live && v < VR) {
      if (hv != nullptr) hv[v] = h[j];
      ss += sumsq8(h[j]);
    }
  }
  for (int v = tr + kNqKeep * TPR; live && v < VR; v += TPR) {  // rows longer than the register set
    uint4 u = __ldcg(xv + v);
    if (rv != nullptr) u = add8_bf16(u, __ldcg(rv + v));
    if (hv != nullptr) hv[v] = u;
    ss += sumsq8(u);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  float tot = 0.0f;
  for (int w = 0; w < WR; ++w) tot += red[rr * WR + w];  // fixed order: deterministic
  const float rs = __frsqrt_rn(__fadd_rn(__fdiv_rn(tot, static_cast<float>(a.K)), a.eps));
  __syncthreads();  // red[] is reused below

  // ---- amax of y over the tensor ----------------------------------------------
  float m = 0.0f;
  float y[8];
#pragma unroll
  for (int j = 0; j < kNqKeep; ++j) {
    const int v = tr + j * TPR;
    if (live && v < VR) m = fmaxf(m, norm8(h[j], gk[j], rs, y));
  }
  for (int v = tr + kNqKeep * TPR; live && v < VR; v += TPR) {
    const uint4 u = reload_h(xv, rv, hv, v);
    m = fmaxf(m, norm8(u, __ldg(gv + v), rs, y));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float w = threadIdx.x < kNqWarps ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, o));
    if (threadIdx.x == 0) cta_amax = w;
  }
  cluster_sync();  // every CTA's maximum is visible cluster-wide
  float amax = 0.0f;
  const uint32_t local = smem_u32(&cta_amax);
  for (int p = 0; p < C; ++p) amax = fmaxf(amax, dsmem_ld_f32(dsmem_addr(local, p)));

  // ---- quantise from registers ------------------------------------------------
  const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
  uint2* q2 = reinterpret_cast<uint2*>(a.xq) + rbase;
#pragma unroll
  for (int j = 0; j < kNqKeep; ++j) {
    const int v = tr + j * TPR;
    if (live && v < VR) {
      norm8(h[j], gk[j], rs, y);
      q2[v] = amax > 0.0f ? quant8(y, inv) : make_uint2(0u, 0u);
    }
  }
  for (int v = tr + kNqKeep * TPR; live && v < VR; v += TPR) {
    const uint4 u = reload_h(xv, rv, hv, v);
    norm8(u, __ldg(gv + v), rs, y);
    q2[v] = amax > 0.0f ? quant8(y, inv) : make_uint2(0u, 0u);
  }
  if (crank == 0 && threadIdx.x == 0) *a.s_x = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;

  cluster_sync();  // peers have finished reading cta_amax before this CTA exits
}

cudaError_t launch_add_rmsnorm_quant(const uint16_t* x, const uint16_t* r, uint16_t* h_out, const uint16_t* gamma,
                                     int M, int K, float eps, uint8_t* xq, float* s_x, cudaStream_t s, bool pdl) {
  // rows per CTA: the smallest power of two that fits M rows in <= 16 CTAs
  // (a cluster above 8 CTAs is non-portable; more CTAs shorten each one's
  // share of the loads at large M)
  int R = 1;
  while (R < 16 && (M + R - 1) / R > 16) R <<= 1;
  const int C = (M + R - 1) / R;
  if (C > 16) return cudaErrorInvalidValue;
  if (C > 8) {
    cudaError_t e = ensure_kernel_attrs(reinterpret_cast<const void*>(add_rmsnorm_quant_kernel), 0, true);
    if (e != cudaSuccess) return e;
  }
  NormQuantArgs a;
  a.x = x;
  a.r = r;
  a.h_out = h_out;
  a.gamma = gamma;
  a.xq = xq;
  a.s_x = s_x;
  a.M = M;
  a.K = K;
  a.R = R;
  a.eps = eps;
  Launch L(dim3(C), dim3(kNqThreads), 0, s, static_cast<unsigned>(C), pdl);
  return cudaLaunchKernelEx(&L.cfg, add_rmsnorm_quant_kernel, a);
}

}  // namespace dl
