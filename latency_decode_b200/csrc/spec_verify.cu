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

// -0 and +0 are the same logit value: -0 is keyed as +0, so that a tie between
// them, like any other tie, goes to the lower index.
__device__ __forceinline__ unsigned long long sv_key(uint32_t bf16_bits, int index) {
  if (bf16_bits == 0x8000u) bf16_bits = 0u;
  return (static_cast<unsigned long long>(ordered_bits(__uint_as_float(bf16_bits << 16))) << 32) |
         static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(index));
}

// Best key among the 8 bf16 logits of one 16-byte vector starting at index v8.
__device__ __forceinline__ unsigned long long best8(uint4 u, int v8) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  unsigned long long k = 0ull;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const unsigned long long lo = sv_key(w[i] & 0xFFFFu, v8 + 2 * i);
    const unsigned long long hi = sv_key(w[i] >> 16, v8 + 2 * i + 1);
    k = lo > k ? lo : k;
    k = hi > k ? hi : k;
  }
  return k;
}

// Launched as grid (C, B) with clusters of (C, 1, 1).
__global__ void __launch_bounds__(kSvThreads) spec_verify_kernel(const __grid_constant__ VerifyArgs a) {
  __shared__ unsigned long long best[kSvMaxT];

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
  if (threadIdx.x < T) best[threadIdx.x] = 0ull;
  __syncthreads();

  const uint4* base = reinterpret_cast<const uint4*>(a.logits) + static_cast<long long>(b) * T * nv;
  const int items = per * T;  // (row, vector) pairs, row-major
  int cur_row = -1;
  unsigned long long cur = 0ull;
  for (int i0 = threadIdx.x; i0 < items; i0 += kSvThreads * kSvBatch) {
    uint4 u[kSvBatch];
#pragma unroll
    for (int j = 0; j < kSvBatch; ++j) {
      const int i = i0 + j * kSvThreads;
      if (i < items) {
        const int t = i / per;
        u[j] = __ldcg(base + static_cast<long long>(t) * nv + c0 + (i - t * per));
      }
    }
#pragma unroll
    for (int j = 0; j < kSvBatch; ++j) {
      const int i = i0 + j * kSvThreads;
      if (i < items) {
        const int t = i / per;
        if (t != cur_row) {
          if (cur_row >= 0) atomicMax(&best[cur_row], cur);
          cur_row = t;
          cur = 0ull;
        }
        const unsigned long long k = best8(u[j], (c0 + (i - t * per)) * 8);
        cur = k > cur ? k : cur;
      }
    }
  }
  if (cur_row >= 0) atomicMax(&best[cur_row], cur);
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
  if (C > 8) {
    cudaError_t e = ensure_kernel_attrs(reinterpret_cast<const void*>(spec_verify_kernel), 0, true);
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
  return cudaLaunchKernelEx(&L.cfg, spec_verify_kernel, a);
}

}  // namespace dl
