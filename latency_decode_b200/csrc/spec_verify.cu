// spec_verify.cu -- greedy speculative verification on the device.
//
// [XZY] "推测解码" / "端到端的工作流": the target model checks the draft tokens
// of one step in parallel, keeps the drafts that match the token it would
// itself generate, and at the first mismatch emits its own token instead.
// [XZY] "通过 CUDA Graph 和重叠调度器减少主机端开销": the verification stays on
// the device so that the target forward, the verification and the draft
// forward fit in one CUDA graph with no host synchronisation.
//
// One thread-block cluster per sequence.  CTA r of the cluster scans the r-th
// slice of the vocabulary for all T positions of its sequence; every
// (logit, index) pair becomes one 64-bit key (order-preserving float bits above,
// with -0 taken as +0, inverted index below), so an unsigned max picks the
// largest logit and, on a tie, the lowest index -- whatever order the threads
// arrive in.  The cluster
// merges the per-CTA maxima through distributed shared memory, and CTA 0
// decides the accepted prefix and writes the results.
#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

constexpr int kSvThreads = 512;
constexpr int kSvMaxT = 32;
constexpr int kSvBatch = 8;  // 16-byte loads in flight per thread per round

struct VerifyArgs {
  const uint16_t* logits;  // [B][T][V] bf16
  const int32_t* draft;    // [B][T-1]
  int32_t* target_ids;     // [B][T]
  int32_t* n_accepted;     // [B]
  int32_t* emitted;        // [B][T]
  int32_t* seq_lens;       // [B], may be null
  int B, T, V;
};

// Order-preserving map of a float onto uint32 (finite inputs).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// (logit, index) as one key: order-preserving value bits above, the inverted
// index below, so that the larger key is the larger logit and, among equal
// logits, the lower index.  -0 and +0 are the same logit value: -0 is keyed as
// +0, so that a tie between them, like any other tie, goes to the lower index.
__device__ __forceinline__ unsigned long long sv_key(float v, int index) {
  if (v == 0.0f) v = 0.0f;
  return (static_cast<unsigned long long>(ordered_bits(v)) << 32) |
         static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(index));
}

__device__ __forceinline__ float bf16_at(uint4 u, int e) {  // element e (0..7) of 8 packed bf16
  const uint32_t w = e < 2 ? u.x : e < 4 ? u.y : e < 6 ? u.z : u.w;
  return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

// Launched as grid (C, B) with clusters of (C, 1, 1).  kMinBlocks = 2 caps the
// registers at 64 so that two CTAs share an SM (a 16-CTA cluster then spans 8
// SMs of a GPC and grids beyond one CTA per SM run in one wave); grids that
// fit one CTA per SM use the unconstrained build, which is faster there.
template <int kMinBlocks>
__global__ void __launch_bounds__(kSvThreads, kMinBlocks) spec_verify_kernel(const __grid_constant__ VerifyArgs a) {
  __shared__ unsigned long long best[kSvMaxT];
  __shared__ unsigned long long wbest[kSvThreads / 32];

  // the logits are the output of the preceding kernel (the LM head)
  pdl_wait();
  pdl_trigger();

  const int C = gridDim.x;
  const int r = static_cast<int>(cluster_rank());
  const int b = blockIdx.y;
  const int T = a.T;
  const int nv = a.V >> 3;  // 16-byte vectors per row
  const int c0 = static_cast<int>(static_cast<long long>(nv) * r / C);
  const int c1 = static_cast<int>(static_cast<long long>(nv) * (r + 1) / C);
  const int per = c1 - c0;  // vectors of this CTA's slice, per row
  const uint4* base = reinterpret_cast<const uint4*>(a.logits) + static_cast<long long>(b) * T * nv;
  // Each of the T rows gets its own group of G = 512 / T' threads (T' = T
  // rounded up to a power of two; groups past T idle), which scans the row's
  // slice with 16-byte loads, kSvBatch in flight per thread.  A thread meets
  // its vectors in increasing index order, so only a strictly larger value
  // replaces its best one (the first of equal values stays); the row's best
  // over the group is then the largest (value, lowest index) key, reduced by
  // shuffles and, for groups wider than a warp, one shared slot per warp.
  int Tp = 1;
  while (Tp < T) Tp <<= 1;
  const int G = kSvThreads / Tp;
  const int t = threadIdx.x / G;
  const int gi = threadIdx.x - t * G;
  float best_v = 0.0f;
  int best_i = -1;
  if (t < T) {
    const uint4* row = base + static_cast<long long>(t) * nv + c0;
    for (int v0 = gi; v0 < per; v0 += G * kSvBatch) {
      uint4 u[kSvBatch];
#pragma unroll
      for (int j = 0; j < kSvBatch; ++j)
        if (v0 + j * G < per) u[j] = __ldcg(row + v0 + j * G);
#pragma unroll
      for (int j = 0; j < kSvBatch; ++j) {
        if (v0 + j * G < per) {
          // the vector's largest value (packed bf16 maxima), then, only when it
          // beats the best so far, its first position
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
          const __nv_bfloat162 m2 = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
          const float vmax = fmaxf(__low2float(m2), __high2float(m2));
          if (best_i < 0 || vmax > best_v) {
            int e = 7;
#pragma unroll
            for (int k = 6; k >= 0; --k)
              if (bf16_at(u[j], k) == vmax) e = k;
            best_v = vmax;
            best_i = (c0 + v0 + j * G) * 8 + e;
          }
        }
      }
    }
  }
  unsigned long long key = best_i >= 0 ? sv_key(best_v, best_i) : 0ull;
  const int width = G < 32 ? G : 32;  // G is a power of two >= 16
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    if (o < width) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
      key = other > key ? other : key;
    }
  }
  const int warp = threadIdx.x >> 5;
  if (G <= 32) {
    if (t < T && gi == 0) best[t] = key;
  } else {
    if ((threadIdx.x & 31) == 0) wbest[warp] = key;
  }
  __syncthreads();
  if (G > 32 && threadIdx.x < T) {  // the G / 32 warps of row threadIdx.x
    unsigned long long k = 0ull;
    for (int w = threadIdx.x * (G / 32); w < (threadIdx.x + 1) * (G / 32); ++w) k = wbest[w] > k ? wbest[w] : k;
    best[threadIdx.x] = k;
  }
  cluster_sync();  // every CTA's row maxima are final and visible cluster-wide

  if (r == 0 && threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int tid = 0;
    if (lane < T) {
      unsigned long long k = 0ull;
      const uint32_t local = smem_u32(&best[lane]);
      for (int p = 0; p < C; ++p) {
        const uint32_t addr = dsmem_addr(local, static_cast<uint32_t>(p));
        const unsigned long long lo = dsmem_ld_u32(addr);
        const unsigned long long hi = dsmem_ld_u32(addr + 4u);
        const unsigned long long kp = (hi << 32) | lo;
        k = kp > k ? kp : k;
      }
      tid = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(k & 0xFFFFFFFFull));
      a.target_ids[static_cast<long long>(b) * T + lane] = tid;
    }
    // accepted prefix: draft i is kept while it equals the target's token at i
    const bool match = lane < T - 1 && __ldcg(a.draft + static_cast<long long>(b) * (T - 1) + lane) == tid;
    const unsigned miss = __ballot_sync(0xffffffffu, !match);
    const int n = min(__ffs(miss) - 1, T - 1);  // lanes >= T-1 never match
    if (lane < T) a.emitted[static_cast<long long>(b) * T + lane] = lane <= n ? tid : -1;
    if (lane == 0) {
      a.n_accepted[b] = n;
      if (a.seq_lens != nullptr) a.seq_lens[b] -= (T - 1 - n);  // drop the rejected drafts' cache entries
    }
  }
  cluster_sync();  // CTA 0 has read every peer's maxima before they exit
}

cudaError_t launch_spec_verify(const uint16_t* logits, int B, int T, int V, const int32_t* draft,
                               int32_t* target_ids, int32_t* n_accepted, int32_t* emitted, int32_t* seq_lens,
                               cudaStream_t s, bool pdl) {
  // enough CTAs to keep the memory system busy: about two per SM over all sequences
  int C = (2 * sm_count() + B - 1) / B;
  if (C > 16) C = 16;
  if (C < 1) C = 1;
  const int nv = V / 8;
  if (C > nv) C = nv;
  const bool two = static_cast<long long>(C) * B > sm_count();
  const void* fn = two ? reinterpret_cast<const void*>(spec_verify_kernel<2>)
                       : reinterpret_cast<const void*>(spec_verify_kernel<1>);
  if (C > 8) {
    cudaError_t e = ensure_kernel_attrs(fn, 0, true);
    if (e != cudaSuccess) return e;
  }
  VerifyArgs a;
  a.logits = logits;
  a.draft = draft;
  a.target_ids = target_ids;
  a.n_accepted = n_accepted;
  a.emitted = emitted;
  a.seq_lens = seq_lens;
  a.B = B;
  a.T = T;
  a.V = V;
  Launch L(dim3(C, B), dim3(kSvThreads), 0, s, static_cast<unsigned>(C), pdl);
  return two ? cudaLaunchKernelEx(&L.cfg, spec_verify_kernel<2>, a) : cudaLaunchKernelEx(&L.cfg, spec_verify_kernel<1>, a);
}

}  // namespace dl
