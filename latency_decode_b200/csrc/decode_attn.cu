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
//  * one cluster of S CTAs per (sequence b, kv head); CTA r streams the r-th
//    contiguous chunk of ceil(L/S) keys (rounded up to 16).  The G = Hq/Hkv
//    query heads of the group and the T query tokens share every K/V byte
//    loaded, so K and V are read exactly once.
//  * a producer warp moves 64-key tiles of K and V with TMA tensor copies in the
//    128-byte swizzle (bank-conflict-free ldmatrix), into a ring of stages; it
//    does not wait for the preceding kernel (the KV cache is static), so under
//    PDL the ring fills while the QKV GEMM still runs.
//  * four consumer warps each take 16 keys of a tile and run swapped-AB
//    tensor-core MMAs (mma.sync m16n8k16, bf16 -> fp32): S^T = K Q^T with the
//    keys as the M dimension and the R = G*T query rows as N (padded to 8, not
//    16), then O^T += V^T P^T.  P^T is formed in registers with movmatrix.
//  * online softmax in the log2 domain; the row max is a 3-step warp shuffle.
//  * the four warp states merge in shared memory, then the S CTA states merge
//    through distributed shared memory: M* = max m_i, L* = sum l_i 2^(m_i-M*),
//    o = sum o_i 2^(m_i-M*) / L*; each CTA finalises 1/S of the outputs.
#include <cudaTypedefs.h>

#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

constexpr int kAttnKT = 64;           // keys per pipeline stage
constexpr int kAttnConsumers = 4;     // consumer warps, 16 keys each per stage
constexpr int kAttnThreads = 32 * (kAttnConsumers + 1);

struct AttnArgs {
  const uint16_t* q;
  long long q_stride;
  int B, T, Hq, Hkv, G, R, Lcap;
  const int32_t* seq_lens;
  float scale_log2;  // softmax scale * log2(e)
  uint16_t* out;
  uint32_t* status;
  int stages;
  int debug;
};

__device__ __forceinline__ uint32_t ld_b32(const uint16_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

template <int D, int NT>
__global__ void __launch_bounds__(kAttnThreads, 1)
    decode_attn_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       const __grid_constant__ AttnArgs a) {
  constexpr int HALVES = D / 64;              // a swizzled row holds 64 bf16 (128 bytes)
  constexpr int HALF_BYTES = kAttnKT * 128;   // 64 keys x 128 bytes
  constexpr int STAGE_BYTES = 2 * HALVES * HALF_BYTES;
  constexpr int KS = D / 16;                  // MMA k-steps over d, and m-tiles of d
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + a.stages * STAGE_BYTES);
  int* abort_word = reinterpret_cast<int*>(bars + 2 * a.stages);
  volatile int* abort_flag = abort_word;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8u * a.stages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = gridDim.x;
  const int rank = static_cast<int>(cluster_rank());
  const int hk = blockIdx.y;
  const int b = blockIdx.z;
  const long long budget = a.debug ? kWaitBudgetDebug : kWaitBudget;

  // ---- this CTA's key chunk ----
  int L = __ldg(a.seq_lens + b);
  if (L < a.T || L > a.Lcap) {
    if (threadIdx.x == 0 && rank == 0 && hk == 0) set_status(a.status, kStatusBadSeqLen);
    L = 0;  // no visible keys: the output of this sequence is zero
  }
  const int chunk = (((L + S - 1) / S) + 15) & ~15;
  const int lo = min(rank * chunk, L);
  const int hi = min(lo + chunk, L);
  const int n_tiles = (hi - lo + kAttnKT - 1) / kAttnKT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, kAttnConsumers);
    }
    *abort_word = 0;
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

    // Q^T fragments (B operand of S^T = K Q^T): column n = query row g of tile nt
    uint32_t qf[KS][NT][2];
    int lim[NT][2];  // last visible key of the rows this thread accumulates
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int rho = nt * 8 + g;
      const bool valid = rho < a.R;
      const int t = valid ? rho / a.G : 0;
      const int hq = hk * a.G + (valid ? rho % a.G : 0);
      const uint16_t* qrow = a.q + (static_cast<long long>(b) * a.T + t) * a.q_stride + static_cast<long long>(hq) * D;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qf[ks][nt][0] = valid ? ld_b32(qrow + ks * 16 + 2 * q4) : 0u;
        qf[ks][nt][1] = valid ? ld_b32(qrow + ks * 16 + 8 + 2 * q4) : 0u;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int r2 = nt * 8 + 2 * q4 + j;
        lim[nt][j] = r2 < a.R ? L - a.T + r2 / a.G : -1;
      }
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
            for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(sc[nt], a0, a1, a2, a3, qf[ks][nt][0], qf[ks][nt][1]);
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
            const float m_new = fmaxf(m_run[nt][j], mx);
            const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
            const float alpha = ex2(m_run[nt][j] - m_use);
            p[j] = ex2(x0 - m_use);
            p[2 + j] = ex2(x1 - m_use);
            l_run[nt][j] = l_run[nt][j] * alpha + p[j] + p[2 + j];
            m_run[nt][j] = m_new;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
              o[mt][nt][j] *= alpha;
              o[mt][nt][2 + j] *= alpha;
            }
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

  __syncthreads();  // the ring is drained: reuse it for the merge buffers
  pdl_wait();
  const int R = a.R;
  float* wo = reinterpret_cast<float*>(ring);             // [4][R][D] per-warp o
  float* wm = wo + kAttnConsumers * R * D;                // [4][R]
  float* wl = wm + kAttnConsumers * R;                    // [4][R]
  float* cm = wl + kAttnConsumers * R;                    // [R]   CTA state, read by peers
  float* cl = cm + R;                                     // [R]
  float* co = cl + R + ((4 - ((2 * R) & 3)) & 3);         // [R][D], 16-byte aligned
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
  // ---- merge the four warp states into this CTA's state ----
  for (int idx = threadIdx.x; idx < R * D; idx += kAttnThreads) {
    const int rho = idx / D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnConsumers; ++w)
      if (wl[w * R + rho] > 0.0f) M = fmaxf(M, wm[w * R + rho]);
    float acc = 0.0f, lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < kAttnConsumers; ++w) {
      const float lw = wl[w * R + rho];
      if (lw > 0.0f) {
        const float f = ex2(wm[w * R + rho] - M);
        acc += wo[(w * R + rho) * D + (idx - rho * D)] * f;
        lsum += lw * f;
      }
    }
    co[idx] = acc;
    if (idx - rho * D == 0) {
      cm[rho] = M;
      cl[rho] = lsum;
    }
  }
  cluster_sync();  // every CTA state of the cluster is visible through DSMEM

  // ---- merge the S CTA states; CTA `rank` finalises a 1/S slice of the outputs ----
  const int items = R * (D / 4);
  const int i0 = static_cast<int>(static_cast<long long>(items) * rank / S);
  const int i1 = static_cast<int>(static_cast<long long>(items) * (rank + 1) / S);
  const uint32_t cm_l = smem_u32(cm), cl_l = smem_u32(cl), co_l = smem_u32(co);
  for (int it = i0 + threadIdx.x; it < i1; it += kAttnThreads) {
    const int rho = it / (D / 4);
    const int c4 = it - rho * (D / 4);
    float M = -INFINITY;
    for (int p = 0; p < S; ++p) {
      const float lp = dsmem_ld_f32(dsmem_addr(cl_l + 4u * rho, p));
      if (lp > 0.0f) M = fmaxf(M, dsmem_ld_f32(dsmem_addr(cm_l + 4u * rho, p)));
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.0f;
    for (int p = 0; p < S; ++p) {
      const float lp = dsmem_ld_f32(dsmem_addr(cl_l + 4u * rho, p));
      if (lp > 0.0f) {
        const float f = ex2(dsmem_ld_f32(dsmem_addr(cm_l + 4u * rho, p)) - M);
        const float4 v = dsmem_ld_f32x4(dsmem_addr(co_l + 4u * (rho * D + c4 * 4), p));
        acc.x += v.x * f;
        acc.y += v.y * f;
        acc.z += v.z * f;
        acc.w += v.w * f;
        lsum += lp * f;
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
  cluster_sync();  // keep this CTA's state alive until every peer has read it
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

static bool encode_kv_map(CUtensorMap* m, const uint16_t* base, int d, int Lcap, int BH) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Lcap), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(Lcap) * d * 2};
  cuuint32_t box[3] = {64, kAttnKT, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int NT>
static cudaError_t launch_attn_t(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                                 const AttnLaunch& p, cudaStream_t s) {
  constexpr int STAGE_BYTES = 2 * (D / 64) * kAttnKT * 128;
  const int R = a.R;
  const int merge_bytes = (kAttnConsumers * R * D + 2 * kAttnConsumers * R + 2 * R + 4 + R * D) * 4;
  int stages = a.stages;
  while (stages * STAGE_BYTES < merge_bytes) ++stages;
  AttnArgs args = a;
  args.stages = stages;
  const int smem = 1024 + stages * STAGE_BYTES + 2 * stages * 8 + 16;
  auto kern = decode_attn_kernel<D, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (p.cluster > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  Launch L(dim3(p.cluster, p.Hkv, p.B), dim3(kAttnThreads), static_cast<size_t>(smem), s,
           static_cast<unsigned>(p.cluster), p.pdl);
  return cudaLaunchKernelEx(&L.cfg, kern, tk, tv, args);
}

cudaError_t launch_attn(const AttnLaunch& p, cudaStream_t s) {
  CUtensorMap tk, tv;
  if (!encode_kv_map(&tk, p.k, p.d, p.Lcap, p.B * p.Hkv) || !encode_kv_map(&tv, p.v, p.d, p.Lcap, p.B * p.Hkv))
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
  a.stages = 4;
  a.debug = p.debug ? 1 : 0;
  const int NT = (a.R + 7) / 8;
  if (p.d == 128) {
    switch (NT) {
      case 1: return launch_attn_t<128, 1>(tk, tv, a, p, s);
      case 2: return launch_attn_t<128, 2>(tk, tv, a, p, s);
      case 3: return launch_attn_t<128, 3>(tk, tv, a, p, s);
      case 4: return launch_attn_t<128, 4>(tk, tv, a, p, s);
    }
  } else if (p.d == 64) {
    switch (NT) {
      case 1: return launch_attn_t<64, 1>(tk, tv, a, p, s);
      case 2: return launch_attn_t<64, 2>(tk, tv, a, p, s);
      case 3: return launch_attn_t<64, 3>(tk, tv, a, p, s);
      case 4: return launch_attn_t<64, 4>(tk, tv, a, p, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace dl
