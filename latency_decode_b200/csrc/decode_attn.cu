// decode_attn.cu -- A3/A4: split-KV grouped-query decode attention with a
// cluster distributed-shared-memory log-sum-exp merge.
//
// Sources: [XZY] "CUDA 内核优化与融合", item "Attention内核并行优化" (the work is
// split along the sequence dimension of K and V over several thread blocks;
// the blocks of one thread-block cluster reduce their partial results through
// distributed shared memory, avoiding global memory); [NV] "CUDA kernel
// optimisation and fusion" (same two points).
//
// Design (B200-native; the pages give no code):
//  * the keys of one (sequence b, kv head) are split into P*S contiguous
//    chunks of ceil(L/(P*S)) keys (rounded up to 16), one per CTA; the S CTAs
//    of a thread-block cluster hold S neighbouring chunks.  The G = Hq/Hkv query
//    heads and the T query tokens share every K/V byte loaded, so K and V are
//    read exactly once.
//  * a producer warp moves 64-key tiles of K and V with TMA tensor copies in the
//    128-byte swizzle (bank-conflict-free ldmatrix), into a ring of stages; it
//    does not wait for the preceding kernel (the KV cache is static), so under
//    PDL the ring fills while the QKV GEMM still runs.
//  * four consumer warps each take 16 keys of a tile and run swapped-AB
//    tensor-core MMAs (mma.sync m16n8k16, bf16 -> fp32): S^T = K Q^T with the
//    keys as the M dimension and the R = G*T query rows as N (padded to 8, not
//    16), then O^T += V^T P^T.  P^T is formed in registers with movmatrix; the
//    Q^T fragments are read from shared memory, which keeps two CTAs per SM.
//  * online softmax in the log2 domain; the row max is a 3-step warp shuffle.
//  * merges: the four warp states merge in shared memory; the S CTA states of
//    a cluster merge through distributed shared memory (M* = max m_i,
//    L* = sum l_i 2^(m_i-M*), o = sum o_i 2^(m_i-M*) / L*), each CTA owning
//    1/S of the outputs.  With P = 1 that is the final result.  With P > 1
//    (used when B*Hkv*S CTAs would leave the GPU half idle) each cluster
//    stores its merged state in the workspace and bumps a per-(b, kv head)
//    counter; the cluster that arrives last merges the P states the same way
//    and resets the counter.  Nothing ever waits for another cluster.
#include <cudaTypedefs.h>

#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

// W consumer warps take 16 keys each of a stage of 16*W keys; one more warp
// is the TMA producer.  W = 8 (one CTA per SM, enough warps to hide the MMA and
// softmax latency) for clusters of up to 8 CTAs; W = 4 (two CTAs per SM where
// they fit) for 16-CTA clusters, which pack onto the GPCs only that way.
constexpr int kAttnMaxSplits = 16;    // clusters per (b, kv head)
constexpr int kLazyRescale = 8;       // log2 headroom before the running max is raised

struct AttnArgs {
  const uint16_t* q;
  long long q_stride;
  int B, T, Hq, Hkv, G, R, Lcap;
  const int32_t* seq_lens;
  float scale_log2;  // softmax scale * log2(e)
  uint16_t* out;
  uint32_t* status;
  uint32_t* counters;  // [B*Hkv][S], P > 1 only
  float* part_ml;      // [B*Hkv][P][S][R][2] per-owner (m, l)
  float* part_o;       // [B*Hkv][P][R*D/4] float4
  int P;
  int stages;
  int recv_off;        // byte offset of the DSMEM receive buffer
  int debug;
};

__device__ __forceinline__ uint32_t ld_b32(const uint16_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

template <int D, int NT, int W>
__global__ void __launch_bounds__(32 * (W + 1), W == 4 ? 2 : 1)
    decode_attn_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       const __grid_constant__ AttnArgs a) {
  constexpr int kAttnConsumers = W;
  constexpr int kAttnThreads = 32 * (W + 1);
  constexpr int kAttnKT = 16 * W;             // keys per pipeline stage
  constexpr int HALVES = D / 64;              // a swizzled row holds 64 bf16 (128 bytes)
  constexpr int HALF_BYTES = kAttnKT * 128;   // kAttnKT keys x 128 bytes
  constexpr int STAGE_BYTES = 2 * HALVES * HALF_BYTES;
  constexpr int KS = D / 16;                  // MMA k-steps over d, and m-tiles of d
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint2* qs = reinterpret_cast<uint2*>(ring + a.stages * STAGE_BYTES);        // [KS][NT][32]
  uint8_t* recv_base = smem + a.recv_off;                                      // DSMEM receive buffer
  uint64_t* bars = reinterpret_cast<uint64_t*>(qs + KS * NT * 32);
  int* abort_word = reinterpret_cast<int*>(bars + 2 * a.stages);
  int* last_word = abort_word + 1;
  volatile int* abort_flag = abort_word;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8u * a.stages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = gridDim.x;
  const int rank = static_cast<int>(cluster_rank());
  const int hk = blockIdx.y;
  const int b = blockIdx.z / a.P;
  const int split = blockIdx.z - b * a.P;
  const long long budget = a.debug ? kWaitBudgetDebug : kWaitBudget;

  // ---- this CTA's key chunk ----
  int L = __ldg(a.seq_lens + b);
  if (L < a.T || L > a.Lcap) {
    if (threadIdx.x == 0 && rank == 0 && hk == 0 && split == 0) set_status(a.status, kStatusBadSeqLen);
    L = 0;  // no visible keys: the output of this sequence is zero
  }
  const int nchunks = a.P * S;
  const int chunk = (((L + nchunks - 1) / nchunks) + 15) & ~15;
  const int lo = min((split * S + rank) * chunk, L);
  const int hi = min(lo + chunk, L);
  const int n_tiles = (hi - lo + kAttnKT - 1) / kAttnKT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, kAttnConsumers);
    }
    *abort_word = 0;
    *last_word = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int g = lane >> 2;   // MMA group id (row of the A/C fragments)
  const int q4 = lane & 3;   // thread in group

  // per-warp online-softmax state for rows nt*8 + 2*q4 + j
  float o[KS][NT][4];
  float m_run[NT][2], l_run[NT][2];
#pragma unroll
  for (int mt = 0; mt < KS; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) o[mt][nt][c] = 0.0f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      m_run[nt][j] = -INFINITY;
      l_run[nt][j] = 0.0f;
    }

  if (warp == kAttnConsumers) {
    // ---- producer ----
    if (lane == 0) {
      prefetch_tensormap(&tk);
      prefetch_tensormap(&tv);
      const int z = b * a.Hkv + hk;
      const int n_issue = (a.debug && n_tiles > 0) ? n_tiles - 1 : n_tiles;  // test hook
      int issued = 0;
      for (int i = 0; i < n_issue; ++i) {
        const int s = i % a.stages;
        if (i >= a.stages &&
            !mbar_wait(empty0 + 8u * s, static_cast<uint32_t>((i / a.stages) - 1) & 1u, budget, abort_flag)) {
          set_status(a.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        const uint32_t st = smem_u32(ring + s * STAGE_BYTES);
        const uint32_t fb = full0 + 8u * s;
        mbar_arrive_expect_tx(fb, STAGE_BYTES);
        const int key0 = lo + i * kAttnKT;
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          tma_load_3d(st + h * HALF_BYTES, &tk, h * 64, key0, z, fb);
          tma_load_3d(st + (HALVES + h) * HALF_BYTES, &tv, h * 64, key0, z, fb);
        }
        issued = i + 1;
      }
      if (*abort_flag) {
        const int first = issued > a.stages ? issued - a.stages : 0;
        for (int i = first; i < issued; ++i)
          mbar_wait(full0 + 8u * (i % a.stages), static_cast<uint32_t>(i / a.stages) & 1u, budget, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ---- consumers ----
    pdl_wait();  // q is written by the preceding QKV GEMM
    if (threadIdx.x == 0) pdl_trigger();

    // Q^T fragments (B operand of S^T = K Q^T), column n = query row g of tile nt,
    // staged once in shared memory by the four consumer warps.
    for (int f = threadIdx.x; f < KS * NT * 32; f += 32 * kAttnConsumers) {
      const int ln = f & 31;
      const int nt = (f >> 5) % NT;
      const int ks = (f >> 5) / NT;
      const int rho = nt * 8 + (ln >> 2);
      uint2 v = make_uint2(0u, 0u);
      if (rho < a.R) {
        const int t = rho / a.G;
        const int hq = hk * a.G + rho % a.G;
        const uint16_t* qrow =
            a.q + (static_cast<long long>(b) * a.T + t) * a.q_stride + static_cast<long long>(hq) * D;
        v.x = ld_b32(qrow + ks * 16 + 2 * (ln & 3));
        v.y = ld_b32(qrow + ks * 16 + 8 + 2 * (ln & 3));
      }
      qs[f] = v;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kAttnConsumers) : "memory");

    int lim[NT][2];  // last visible key of the rows this thread accumulates
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int r2 = nt * 8 + 2 * q4 + j;
        lim[nt][j] = r2 < a.R ? L - a.T + r2 / a.G : -1;
      }

    for (int i = 0; i < n_tiles; ++i) {
      const int s = i % a.stages;
      bool ok = !*abort_flag;
      if (ok && !mbar_wait(full0 + 8u * s, static_cast<uint32_t>(i / a.stages) & 1u, budget, abort_flag)) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);  // the warp-wide MMA path below needs a uniform decision
      const int key_base = lo + i * kAttnKT + warp * 16;
      if (ok && key_base < hi) {
        const uint32_t kbase = smem_u32(ring + s * STAGE_BYTES);
        const uint32_t vbase = kbase + HALVES * HALF_BYTES;
        // ---- S^T[16 keys x 8*NT rows] = K . Q^T ----
        float sc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) sc[nt][c] = 0.0f;
        {
          const int j = lane >> 3;
          const int key_l = warp * 16 + (j & 1) * 8 + (lane & 7);
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const int half = ks >> 2;
            const int ch = (ks & 3) * 2 + (j >> 1);
            const uint32_t addr = kbase + half * HALF_BYTES + key_l * 128 + ((ch ^ (key_l & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(addr, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint2 qf = qs[(ks * NT + nt) * 32 + lane];
              mma_bf16_16816(sc[nt], a0, a1, a2, a3, qf.x, qf.y);
            }
          }
        }
        // ---- online softmax (log2 domain) ----
        const int kA = key_base + g;
        const int kB = kA + 8;
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float p[4];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float x0 = (kA < hi && kA <= lim[nt][j]) ? sc[nt][j] * a.scale_log2 : -INFINITY;
            const float x1 = (kB < hi && kB <= lim[nt][j]) ? sc[nt][2 + j] * a.scale_log2 : -INFINITY;
            float mx = fmaxf(x0, x1);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            // Lazy rescale: the reference max m_run moves only when this tile's
            // max exceeds it by more than 2^kLazyRescale, so the O rescale below
            // is rarely needed; p stays <= 2^kLazyRescale, far from overflow.
            if (mx > m_run[nt][j] + static_cast<float>(kLazyRescale)) {
              const float m_new = mx;
              const float alpha = ex2(m_run[nt][j] - m_new);  // 0 when m_run is -inf
              l_run[nt][j] *= alpha;
#pragma unroll
              for (int mt = 0; mt < KS; ++mt) {
                o[mt][nt][j] *= alpha;
                o[mt][nt][2 + j] *= alpha;
              }
              m_run[nt][j] = m_new;
            }
            const float m_use = (m_run[nt][j] == -INFINITY) ? 0.0f : m_run[nt][j];
            p[j] = ex2(x0 - m_use);
            p[2 + j] = ex2(x1 - m_use);
            l_run[nt][j] += p[j] + p[2 + j];
          }
          // P^T as the B operand [k = key][n = row]: transpose each 8x8 block
          pb[nt][0] = movmatrix_t(pack_bf16x2(p[0], p[1]));
          pb[nt][1] = movmatrix_t(pack_bf16x2(p[2], p[3]));
        }
        // ---- O^T[d x rows] += V^T . P^T ----
        {
          const int j = lane >> 3;
          const int key_l = warp * 16 + (j >> 1) * 8 + (lane & 7);
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            const int half = mt >> 2;
            const int ch = (mt & 3) * 2 + (j & 1);
            const uint32_t addr = vbase + half * HALF_BYTES + key_l * 128 + ((ch ^ (key_l & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(addr, a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8u * s);
    }
    // full row sums: add the partial sums of the 8 lanes that share a row
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float l = l_run[nt][j];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        l_run[nt][j] = l;
      }
  }

  __syncthreads();  // the ring is drained: reuse it for the per-warp states
  pdl_wait();
  const int R = a.R;
  float* wo = reinterpret_cast<float*>(ring);             // [W][R][D] per-warp o
  float* wm = wo + kAttnConsumers * R * D;                // [W][R]
  float* wl = wm + kAttnConsumers * R;                    // [W][R]
  if (warp < kAttnConsumers) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int rho = nt * 8 + 2 * q4 + j;
        if (rho < R) {
          if (g == 0) {
            wm[warp * R + rho] = m_run[nt][j];
            wl[warp * R + rho] = l_run[nt][j];
          }
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            wo[(warp * R + rho) * D + mt * 16 + g] = o[mt][nt][j];
            wo[(warp * R + rho) * D + mt * 16 + g + 8] = o[mt][nt][2 + j];
          }
        }
      }
  }
  __syncthreads();

  // ---- merge the four warp states and push the CTA state to the slice owners ----
  // Outputs are I = R*D/4 float4 items; CTA c of the cluster owns items
  // [c*Q, (c+1)*Q).  Every CTA stores its state of item i straight into the
  // receive buffer of the owner of i (remote shared-memory stores, no round
  // trip), and the (m, l) of each row into every peer; one cluster barrier
  // later each owner merges the S states of its items locally.
  const int I = R * (D / 4);
  const int Q = (I + S - 1) / S;
  float4* rv_o = reinterpret_cast<float4*>(recv_base);     // [S][Q]
  float* rv_m = reinterpret_cast<float*>(rv_o + S * Q);   // [S][R]
  float* rv_l = rv_m + S * R;                             // [S][R]
  const uint32_t rv_o_l = smem_u32(rv_o), rv_m_l = smem_u32(rv_m), rv_l_l = smem_u32(rv_l);
  for (int it = threadIdx.x; it < I; it += kAttnThreads) {
    const int rho = it / (D / 4);
    const int c4 = it - rho * (D / 4);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnConsumers; ++w)
      if (wl[w * R + rho] > 0.0f) M = fmaxf(M, wm[w * R + rho]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < kAttnConsumers; ++w) {
      const float lw = wl[w * R + rho];
      if (lw > 0.0f) {
        const float f = ex2(wm[w * R + rho] - M);
        const float4 v = *reinterpret_cast<const float4*>(wo + (w * R + rho) * D + c4 * 4);
        acc.x += v.x * f;
        acc.y += v.y * f;
        acc.z += v.z * f;
        acc.w += v.w * f;
        lsum += lw * f;
      }
    }
    const int owner = it / Q;
    dsmem_st_f32x4(dsmem_addr(rv_o_l + 16u * (rank * Q + (it - owner * Q)), owner), acc);
    if (c4 == 0) {
      for (int p = 0; p < S; ++p) {
        dsmem_st_f32(dsmem_addr(rv_m_l + 4u * (rank * R + rho), p), M);
        dsmem_st_f32(dsmem_addr(rv_l_l + 4u * (rank * R + rho), p), lsum);
      }
    }
  }
  cluster_sync();  // every state of my items has landed in my receive buffer

  // ---- merge the S CTA states of my items ----
  const long long head = static_cast<long long>(b) * a.Hkv + hk;
  const long long slot = head * a.P + split;
  const int my0 = rank * Q;
  const int cnt = max(0, min(I, my0 + Q) - my0);
  for (int k = threadIdx.x; k < cnt; k += kAttnThreads) {
    const int it = my0 + k;
    const int rho = it / (D / 4);
    const int c4 = it - rho * (D / 4);
    float M = -INFINITY;
    for (int p = 0; p < S; ++p)
      if (rv_l[p * R + rho] > 0.0f) M = fmaxf(M, rv_m[p * R + rho]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.0f;
    for (int p = 0; p < S; ++p) {
      const float lp = rv_l[p * R + rho];
      if (lp > 0.0f) {
        const float f = ex2(rv_m[p * R + rho] - M);
        const float4 v = rv_o[p * Q + k];
        acc.x += v.x * f;
        acc.y += v.y * f;
        acc.z += v.z * f;
        acc.w += v.w * f;
        lsum += lp * f;
      }
    }
    if (a.P == 1) {
      const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
      const int t = rho / a.G;
      const int hq = hk * a.G + rho % a.G;
      uint16_t* dst = a.out + ((static_cast<long long>(b) * a.T + t) * a.Hq + hq) * D + c4 * 4;
      uint2 packed;
      packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
      packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(dst) = packed;
    } else {
      // this cluster's merged state of my items, unnormalised, for the cross-cluster merge
      *reinterpret_cast<float4*>(a.part_o + (slot * I + it) * 4) = acc;
      if (c4 == 0 || k == 0) {
        float* ml = a.part_ml + ((slot * S + rank) * R + rho) * 2;
        ml[0] = M;
        ml[1] = lsum;
      }
    }
  }
  if (a.P > 1) {
    // The P CTAs that own the same items in the P clusters of this head meet
    // through the workspace: the last one to arrive merges and stores them.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const unsigned prev = atomicAdd(a.counters + head * S + rank, 1u);
      const int last = prev == static_cast<unsigned>(a.P - 1);
      if (last) {
        __threadfence();
        a.counters[head * S + rank] = 0u;  // all P have arrived: reset for the next call
      }
      *last_word = last;
    }
    __syncthreads();
    if (*last_word) {
      __threadfence();
      for (int k = threadIdx.x; k < cnt; k += kAttnThreads) {
        const int it = my0 + k;
        const int rho = it / (D / 4);
        const int c4 = it - rho * (D / 4);
        float M = -INFINITY;
        for (int p = 0; p < a.P; ++p) {
          const float* ml = a.part_ml + (((head * a.P + p) * S + rank) * R + rho) * 2;
          if (__ldcg(ml + 1) > 0.0f) M = fmaxf(M, __ldcg(ml));
        }
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float lsum = 0.0f;
        for (int p = 0; p < a.P; ++p) {
          const float* ml = a.part_ml + (((head * a.P + p) * S + rank) * R + rho) * 2;
          const float lq = __ldcg(ml + 1);
          if (lq > 0.0f) {
            const float f = ex2(__ldcg(ml) - M);
            const float4 v = __ldcg(reinterpret_cast<const float4*>(a.part_o + ((head * a.P + p) * I + it) * 4));
            acc.x += v.x * f;
            acc.y += v.y * f;
            acc.z += v.z * f;
            acc.w += v.w * f;
            lsum += lq * f;
          }
        }
        const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
        const int t = rho / a.G;
        const int hq = hk * a.G + rho % a.G;
        uint16_t* dst = a.out + ((static_cast<long long>(b) * a.T + t) * a.Hq + hq) * D + c4 * 4;
        uint2 packed;
        packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2*>(dst) = packed;
      }
    }
  }
  // No trailing cluster barrier: after the one above, no CTA touches another CTA's shared memory.
}

// ---- host side ----------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

static bool encode_kv_map(CUtensorMap* m, const uint16_t* base, int d, int Lcap, int BH, int kt) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Lcap), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(Lcap) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kt), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Workspace of dl_decode_attn with P clusters per (b, kv head) of S CTAs: the
// 256-byte header, the per-(head, owner) counters, the per-owner (m, l) of each
// cluster, and the merged item states of each cluster.
size_t attn_ws_bytes(int B, int Hkv, int R, int d, int P, int S) {
  if (P <= 1) return kWsHeader;
  const size_t heads = static_cast<size_t>(B) * Hkv;
  const size_t counters = (heads * S * 4 + 255) / 256 * 256;
  const size_t ml = (heads * P * S * R * 2 * 4 + 255) / 256 * 256;
  return kWsHeader + counters + ml + heads * P * R * d * 4;
}

// Shared-memory plan of one attention CTA: two CTAs per SM when a 3-stage
// ring (6 for d=64) fits, else one CTA per SM with the deepest ring (<= 6
// stages) that fits.  The per-warp merge buffers reuse the drained ring.
struct AttnPlan {
  int stages, smem, recv_off;
};

template <int D, int NT, int W>
static AttnPlan attn_plan(int R, int S) {
  constexpr int STAGE_BYTES = 2 * (D / 64) * (16 * W) * 128;
  const int merge_bytes = (W * R * D + 2 * W * R) * 4;
  const int I = R * (D / 4);
  const int Q = (I + S - 1) / S;
  const int recv_bytes = S * Q * 16 + 2 * S * R * 4;
  const int qs_bytes = (D / 16) * NT * 32 * 8;
  auto smem_for = [&](int st) { return 1024 + st * STAGE_BYTES + qs_bytes + 2 * st * 8 + 16 + recv_bytes + 16; };
  int stages = W == 4 ? (D == 128 ? 3 : 6) : (D == 128 ? 3 : 6);
  if (W == 8 || 2 * (smem_for(stages) + 1024) > 233472) {
    stages = 6;
    while (stages > 2 && smem_for(stages) > 232448) --stages;
  }
  while (stages * STAGE_BYTES < merge_bytes) ++stages;
  AttnPlan pl;
  pl.stages = stages;
  pl.smem = smem_for(stages);
  pl.recv_off = ((stages * STAGE_BYTES + qs_bytes + 2 * stages * 8 + 16) + 15) & ~15;
  return pl;
}

template <int D, int NT, int W>
static cudaError_t attn_configure(const AttnPlan& pl, int S) {
  auto kern = decode_attn_kernel<D, NT, W>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
  if (e == cudaSuccess && S > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

// Clusters of S CTAs of this kernel that can be resident on the GPU at once.
template <int D, int NT, int W>
static int attn_max_clusters_t(int R, int S) {
  const AttnPlan pl = attn_plan<D, NT, W>(R, S);
  const int per_sm = 233472 / (pl.smem + 1024) >= 2 ? 2 : 1;
  int fallback = (sm_count() * per_sm) / S;
  if (attn_configure<D, NT, W>(pl, S) != cudaSuccess) {
    (void)cudaGetLastError();
    return fallback;
  }
  Launch L(dim3(S, 1, 1), dim3(32 * (W + 1)), static_cast<size_t>(pl.smem), nullptr, static_cast<unsigned>(S), false);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_attn_kernel<D, NT, W>, &L.cfg) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    return fallback;
  }
  return n;
}

static int attn_warps(int S) { return S >= 16 ? 4 : 8; }

template <int W>
static int attn_max_clusters_w(int d, int R, int S) {
  const int NT = (R + 7) / 8;
  if (d == 128) {
    switch (NT) {
      case 1: return attn_max_clusters_t<128, 1, W>(R, S);
      case 2: return attn_max_clusters_t<128, 2, W>(R, S);
      case 3: return attn_max_clusters_t<128, 3, W>(R, S);
      default: return attn_max_clusters_t<128, 4, W>(R, S);
    }
  }
  switch (NT) {
    case 1: return attn_max_clusters_t<64, 1, W>(R, S);
    case 2: return attn_max_clusters_t<64, 2, W>(R, S);
    case 3: return attn_max_clusters_t<64, 3, W>(R, S);
    default: return attn_max_clusters_t<64, 4, W>(R, S);
  }
}

static int attn_max_clusters(int d, int R, int S) {
  return attn_warps(S) == 8 ? attn_max_clusters_w<8>(d, R, S) : attn_max_clusters_w<4>(d, R, S);
}

// Clusters per (b, kv head).  Splitting a head over P clusters costs a merge
// through the workspace (~2-3 us), so it is used only when each CTA would
// otherwise stream long chunks (>= 2048 keys), with >= 1024 keys per CTA
// left, and never beyond the clusters that can be resident at once.
int attn_auto_splits(int B, int Hkv, int cluster, int Lcap, int d, int R) {
  const long long keys_per_cta = Lcap / cluster;
  if (keys_per_cta < 2048) return 1;
  const long long heads = static_cast<long long>(B) * Hkv;
  const long long resident = attn_max_clusters(d, R, cluster);
  long long P = resident / heads;
  if (P > keys_per_cta / 1024) P = keys_per_cta / 1024;
  if (P > kAttnMaxSplits) P = kAttnMaxSplits;
  return P < 1 ? 1 : static_cast<int>(P);
}

template <int D, int NT, int W>
static cudaError_t launch_attn_t(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                                 const AttnLaunch& p, cudaStream_t s) {
  const AttnPlan pl = attn_plan<D, NT, W>(a.R, p.cluster);
  AttnArgs args = a;
  args.stages = pl.stages;
  args.recv_off = pl.recv_off;
  cudaError_t e = attn_configure<D, NT, W>(pl, p.cluster);
  if (e != cudaSuccess) return e;
  Launch L(dim3(p.cluster, p.Hkv, p.B * a.P), dim3(32 * (W + 1)), static_cast<size_t>(pl.smem), s,
           static_cast<unsigned>(p.cluster), p.pdl);
  return cudaLaunchKernelEx(&L.cfg, decode_attn_kernel<D, NT, W>, tk, tv, args);
}

template <int W>
static cudaError_t launch_attn_w(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                                 const AttnLaunch& p, cudaStream_t s, int NT) {
  if (p.d == 128) {
    switch (NT) {
      case 1: return launch_attn_t<128, 1, W>(tk, tv, a, p, s);
      case 2: return launch_attn_t<128, 2, W>(tk, tv, a, p, s);
      case 3: return launch_attn_t<128, 3, W>(tk, tv, a, p, s);
      case 4: return launch_attn_t<128, 4, W>(tk, tv, a, p, s);
    }
  } else if (p.d == 64) {
    switch (NT) {
      case 1: return launch_attn_t<64, 1, W>(tk, tv, a, p, s);
      case 2: return launch_attn_t<64, 2, W>(tk, tv, a, p, s);
      case 3: return launch_attn_t<64, 3, W>(tk, tv, a, p, s);
      case 4: return launch_attn_t<64, 4, W>(tk, tv, a, p, s);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn(const AttnLaunch& p, cudaStream_t s) {
  const int W = attn_warps(p.cluster);
  const int kt = 16 * W;  // keys per stage of the chosen variant
  CUtensorMap tk, tv;
  if (!encode_kv_map(&tk, p.k, p.d, p.Lcap, p.B * p.Hkv, kt) ||
      !encode_kv_map(&tv, p.v, p.d, p.Lcap, p.B * p.Hkv, kt))
    return cudaErrorInvalidValue;
  AttnArgs a;
  a.q = p.q;
  a.q_stride = p.q_stride;
  a.B = p.B;
  a.T = p.T;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.G = p.Hq / p.Hkv;
  a.R = a.G * p.T;
  a.Lcap = p.Lcap;
  a.seq_lens = p.seq_lens;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.out = p.out;
  a.status = p.status;
  a.stages = 3;
  a.debug = p.debug ? 1 : 0;
  // clusters per (b, kv head): forced, else automatic; then as many as the workspace holds
  int P = p.splits > 0 ? p.splits : attn_auto_splits(p.B, p.Hkv, p.cluster, p.Lcap, p.d, a.R);
  while (P > 1 && attn_ws_bytes(p.B, p.Hkv, a.R, p.d, P, p.cluster) > p.ws_bytes) --P;
  if (static_cast<long long>(p.B) * P > 65535) P = 1;
  a.P = P;
  a.counters = nullptr;
  a.part_ml = a.part_o = nullptr;
  if (P > 1) {
    const size_t heads = static_cast<size_t>(p.B) * p.Hkv;
    uint8_t* base = reinterpret_cast<uint8_t*>(p.status) + kWsHeader;
    a.counters = reinterpret_cast<uint32_t*>(base);
    base += (heads * p.cluster * 4 + 255) / 256 * 256;
    a.part_ml = reinterpret_cast<float*>(base);
    base += (heads * P * p.cluster * a.R * 2 * 4 + 255) / 256 * 256;
    a.part_o = reinterpret_cast<float*>(base);
  }
  const int NT = (a.R + 7) / 8;
  if (W == 8) return launch_attn_w<8>(tk, tv, a, p, s, NT);
  return launch_attn_w<4>(tk, tv, a, p, s, NT);
}

}  // namespace dl
