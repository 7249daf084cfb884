// gemm_e4m3.cu -- A2/A5/A6: FP8 (e4m3, per-tensor scale) weight-streaming
// GEMM at tiny M on the 5th-generation tensor cores, with the FC13+SwiGLU and
// FC_QKV+attention-scaling epilogues and the grouped per-expert (MoE) variant.
//
// Sources: [XZY] "CUDA 内核优化与融合" (items "空间分区与高效内存加载" -- warp
// specialisation so weight loads use the HBM bandwidth, "GEMM 权重重排" -- the
// offline weight swizzle, "运算融合" -- SwiGLU fused into the GEMM); [NV]
// "CUDA kernel optimisation and fusion" (low-latency GEMM kernels, FC13 +
// SwiGLU and FC_QKV + attn_scaling fusions, FP8 MoE).
//
// Design (B200-native; the pages give no code):
//  * swap-AB: the weight tile (128 output rows x 128 K-bytes) is the M=128
//    operand A of tcgen05.mma.kind::f8f6f4, the few tokens are the N operand
//    (N = tokens rounded up to 8), the fp32 accumulator lives in Tensor Memory
//    with one output row per TMEM lane.
//  * weights are pre-swizzled offline (pack.cu), so one 16 KB cp.async.bulk per
//    pipeline stage lands a ready tcgen05 operand in shared memory.
//  * warp roles: warp 0 streams weights through a ring of 16 KB stages (it does
//    not wait for the preceding kernel: weights are static, so under PDL the
//    ring fills while the predecessor still runs), warp 1 issues the MMAs,
//    warps 2-3 stage the activations into the swizzled B operand; all four
//    warps then read the accumulators back with tcgen05.ld.
//  * split-K over a cluster of S CTAs: each CTA reduces 1/S of K, the S partial
//    accumulators are summed through distributed shared memory (each CTA owns
//    128/S output rows), and the nonlinear epilogue runs on the full sums.
//  * SwiGLU: the gate rows and the up rows of the same output columns are two
//    MMAs into two TMEM column ranges of the same lanes, so one thread holds
//    both g and u of its output and applies silu(g)*u directly.
//  * MoE: grid z is an expert slot; every CTA derives the slot's expert and its
//    tokens from expert_ids on the device (no host sync), and CTAs of unused
//    slots exit at once, so only touched experts are read from HBM.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

constexpr int kGemmThreads = 128;
constexpr int kSubBytes = 16384;  // one packed block: 128 rows x 128 K-bytes
constexpr int kMaxTok = 64;
constexpr int kMaxExperts = 1024;
constexpr int kBStages = 4;       // B ring depth when the activations stream in with the weights

struct GemmArgs {
  CUtensorMap xq_map;         // tma_b: x_q [M][K] as 128-byte x npad boxes, 128-byte swizzle
  const uint8_t* w;           // packed weights (expert 0 block for MoE)
  long long w_expert_bytes;   // bytes per expert block (0 for dense)
  const float* w_scale;       // [1] or [E]
  const uint8_t* xq;          // e4m3 activations [M][K] (read; or written when x != null)
  float* s_x;                 // activation scale (read; or written when x != null)
  const uint16_t* x;          // bf16 activations [M][K]: quantise inside this kernel (dense, small M*K)
  uint32_t* status;
  uint16_t* out;              // bf16 [tokens][ldo]
  const int32_t* expert_ids;  // MoE routing (null for dense)
  int M, K, KB, ldo, E;
  int q_cols;
  float q_scale;
  int stages;
  int bsm_bytes;
  int tmem_cols;
  int recv_bytes;             // > 0: split-K partials are pushed into a dedicated receive buffer
  int coop;                   // fused quantiser: the cluster shares the amax (each CTA reads its K slice)
  int tma_b;                  // streamed B (dense): one tensor load per k-block, issued by the producer
  int debug;
};

struct GemmMisc {
  uint32_t tmem_base;
  int abort;
  float sx;                   // activation scale used by the epilogue
  float wmax[2];              // per-warp |x| maxima of the fused quantiser
  float peer_amax[8];         // cooperative quantiser: the slice maxima of the cluster's CTAs
  int n_tok;
  int expert;
  int tokens[kMaxTok];
  uint32_t touched[kMaxExperts / 32];
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float absmax8(uint4 u) {
  float m = fmaxf(fabsf(bf16_lo(u.x)), fabsf(bf16_hi(u.x)));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(u.y)), fabsf(bf16_hi(u.y))));
  m = fmaxf(m, fmaxf(fabsf(bf16_lo(u.z)), fabsf(bf16_hi(u.z))));
  return fmaxf(m, fmaxf(fabsf(bf16_lo(u.w)), fabsf(bf16_hi(u.w))));
}

// e4m3 codes of 4 bf16 values (two 32-bit words) scaled by inv: one IEEE
// rounding for the product, then round-to-nearest-even with saturation.
__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, float inv) {
  const __nv_fp8x2_storage_t a = __nv_cvt_float2_to_fp8x2(
      make_float2(__fmul_rn(bf16_lo(w0), inv), __fmul_rn(bf16_hi(w0), inv)), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(
      make_float2(__fmul_rn(bf16_lo(w1), inv), __fmul_rn(bf16_hi(w1), inv)), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16);
}

template <bool kSwiglu>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_e4m3_kernel(const __grid_constant__ GemmArgs a) {
  constexpr int SUBS = kSwiglu ? 2 : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint8_t* bsm = ring + a.stages * kSubBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bsm + a.bsm_bytes);
  GemmMisc* misc = reinterpret_cast<GemmMisc*>(bars + 2 * a.stages + 3 + 2 * kBStages);
  float* recv = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(misc) + ((sizeof(GemmMisc) + 15) & ~15));
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8u * a.stages;
  const uint32_t xready = empty0 + 8u * a.stages;
  const uint32_t done = xready + 8u;
  const uint32_t bfull0 = done + 8u;                 // B ring (streamed activations)
  const uint32_t bempty0 = bfull0 + 8u * kBStages;
  const uint32_t amaxbar = bempty0 + 8u * kBStages;  // cooperative quantiser: the cluster's slice maxima
  // Fused quantiser: the whole B slice is written once (xready).  Otherwise the
  // e4m3 activations stream through a kBStages ring beside the weight ring.
  const bool stream_b = a.x == nullptr;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = gridDim.x;  // split-K factor == cluster size
  const int rank = static_cast<int>(cluster_rank());
  const int tile = blockIdx.y;
  const long long budget = a.debug ? kWaitBudgetDebug : kWaitBudget;
  volatile int* abort_flag = &misc->abort;

  // ---- which expert and which tokens this CTA serves --------------------------
  if (a.expert_ids != nullptr) {
    if (warp == 0) {
      const int nw = (a.E + 31) >> 5;
      for (int i = lane; i < nw; i += 32) misc->touched[i] = 0u;
      __syncwarp();
      int id0 = lane < a.M ? __ldg(a.expert_ids + lane) : -1;
      int id1 = lane + 32 < a.M ? __ldg(a.expert_ids + lane + 32) : -1;
      if ((lane < a.M && (id0 < 0 || id0 >= a.E)) || (lane + 32 < a.M && (id1 < 0 || id1 >= a.E))) {
        if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) set_status(a.status, kStatusBadExpert);
      }
      if (id0 >= a.E) id0 = -1;
      if (id1 >= a.E) id1 = -1;
      if (id0 >= 0) atomicOr(&misc->touched[id0 >> 5], 1u << (id0 & 31));
      if (id1 >= 0) atomicOr(&misc->touched[id1 >> 5], 1u << (id1 & 31));
      __syncwarp();
      // the slot-th touched expert, experts in increasing id order
      const uint32_t word = lane < nw ? misc->touched[lane] : 0u;
      const int cnt = __popc(word);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = incl - cnt;
      const int slot = blockIdx.z;
      int mine = -1;
      if (slot >= excl && slot < incl) {
        uint32_t v = word;
        for (int j = 0; j < slot - excl; ++j) v &= v - 1u;
        mine = lane * 32 + __ffs(v) - 1;
      }
      mine = __reduce_max_sync(0xffffffffu, mine);
      // this expert's tokens, in token order
      const unsigned lt = (1u << lane) - 1u;
      const unsigned b0 = __ballot_sync(0xffffffffu, mine >= 0 && id0 == mine);
      const unsigned b1 = __ballot_sync(0xffffffffu, mine >= 0 && id1 == mine);
      if (mine >= 0 && id0 == mine) misc->tokens[__popc(b0 & lt)] = lane;
      if (mine >= 0 && id1 == mine) misc->tokens[__popc(b0) + __popc(b1 & lt)] = lane + 32;
      if (lane == 0) {
        misc->n_tok = mine >= 0 ? __popc(b0) + __popc(b1) : 0;
        misc->expert = mine >= 0 ? mine : 0;
      }
    }
  } else if (threadIdx.x == 0) {
    misc->n_tok = a.M;
    misc->expert = 0;
  }
  __syncthreads();
  const int n_tok = misc->n_tok;
  const int expert = misc->expert;
  if (n_tok == 0) {  // unused expert slot: every CTA of the cluster leaves here
    // One early leaver still waits for the predecessor, so that this grid never
    // completes before it even when no slot is used (completion stays ordered
    // along the PDL chain).
    if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == gridDim.z - 1) pdl_wait();
    return;
  }
  const int npad = (n_tok + 7) & ~7;
  const bool routed = a.expert_ids != nullptr;

  const int kb0 = static_cast<int>(static_cast<long long>(a.KB) * rank / S);
  const int kb1 = static_cast<int>(static_cast<long long>(a.KB) * (rank + 1) / S);
  const int nkb = kb1 - kb0;
  const int nsub = nkb * SUBS;
  const uint8_t* wsrc = a.w + expert * a.w_expert_bytes +
                        (static_cast<long long>(tile) * a.KB + kb0) * SUBS * kSubBytes;

  // The fused quantiser reads all of x right after the PDL wait: warm L2 with
  // its lines now, while the CTA sets up (a hint only; x is read after the wait).
  if (a.x != nullptr && warp >= 2) {
    const char* xb = reinterpret_cast<const char*>(a.x);
    const long long xbytes = static_cast<long long>(a.M) * a.K * 2;
    for (long long off = static_cast<long long>(threadIdx.x - 64) * 128; off < xbytes; off += 64 * 128)
      prefetch_l2_line(xb + off);
  }

  // ---- barriers and Tensor Memory ---------------------------------------------------
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 1);
    }
    mbar_init(xready, 64);
    mbar_init(done, 1);
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(bfull0 + 8u * s, a.tma_b ? 1 : 64);
      mbar_init(bempty0 + 8u * s, 1);
    }
    mbar_init(amaxbar, 1);
    misc->abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(&misc->tmem_base), static_cast<uint32_t>(a.tmem_cols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;
  // First phase of a split cluster barrier: every thread arrives here, and
  // waits before it first stores into a peer's shared memory (so every peer's
  // barriers are initialised; thread 0 published them with
  // fence.mbarrier_init before the block barrier above, hence a relaxed
  // arrive): the cooperative quantiser's stagers before they send their slice
  // maxima, every other thread at the epilogue.
  if (S > 1) cluster_arrive_relaxed();

  if (warp == 0) {
    // ---- weight producer ----
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      const int n_issue = a.debug ? nsub - 1 : nsub;  // test hook: withhold the last stage
      int issued = 0;
      // Streamed B by tensor loads (dense): the activations of k-block kb land
      // in B slot kb % kBStages with one copy of npad rows x 128 bytes (the
      // tensor map swizzles them into the operand layout and zero-fills the
      // padding rows).  They exist only once the preceding kernel has written
      // them, so the first `stages` weight blocks are issued before the PDL
      // wait and their k-blocks' activations right after it; from then on each
      // k-block's activations go out just ahead of its first weight block.
      const bool tma_b = a.tma_b != 0;
      const int prefill = a.stages < n_issue ? a.stages : n_issue;
      int kb_b = 0;  // next k-block whose activations are to be issued
      auto issue_b = [&](int kb) -> bool {
        const int bs = kb % kBStages;
        if (kb >= kBStages &&
            !mbar_wait(bempty0 + 8u * bs, static_cast<uint32_t>((kb / kBStages) - 1) & 1u, budget, abort_flag))
          return false;
        mbar_arrive_expect_tx(bfull0 + 8u * bs, static_cast<uint32_t>(npad * 128));
        tma_load_3d(smem_u32(bsm + bs * npad * 128), &a.xq_map, (kb0 + kb) * 128, 0, 0, bfull0 + 8u * bs);
        return true;
      };
      auto issue_b_upto = [&](int kb_end) -> bool {  // k-blocks kb_b .. kb_end - 1
        for (; kb_b < kb_end; ++kb_b)
          if (!issue_b(kb_b)) return false;
        return true;
      };
      if (tma_b) prefetch_tensormap(&a.xq_map);
      // stage s and round parity kept incrementally (no division by the
      // runtime ring depth on this single-thread issue path)
      int s = 0;
      uint32_t round_par = 0;  // (i / stages) & 1
      for (int i = 0; i < n_issue; ++i) {
        if (tma_b && i >= prefill) {
          if (i == prefill) pdl_wait();  // x_q is written by the preceding kernel
          if (!issue_b_upto(i / SUBS + 1)) {
            set_status(a.status, kStatusTimeout);
            *abort_flag = 1;
            break;
          }
        }
        if (i >= a.stages && !mbar_wait(empty0 + 8u * s, round_par ^ 1u, budget, abort_flag)) {
          set_status(a.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(full0 + 8u * s, kSubBytes);
        bulk_load(smem_u32(ring + s * kSubBytes), wsrc + static_cast<long long>(i) * kSubBytes, kSubBytes,
                  full0 + 8u * s, pol);
        issued = i + 1;
        if (++s == a.stages) {
          s = 0;
          round_par ^= 1u;
        }
      }
      if (tma_b && !*abort_flag) {  // the activations of every k-block not issued yet
        if (prefill >= n_issue) pdl_wait();
        if (!issue_b_upto(nkb)) {
          set_status(a.status, kStatusTimeout);
          *abort_flag = 1;
        }
      }
      if (*abort_flag) {  // let the copies still in flight land before the CTA can exit
        const int first = issued > a.stages ? issued - a.stages : 0;
        for (int i = first; i < issued; ++i)
          mbar_wait(full0 + 8u * (i % a.stages), static_cast<uint32_t>(i / a.stages) & 1u, budget, nullptr);
        for (int kb = kb_b > kBStages ? kb_b - kBStages : 0; kb < kb_b; ++kb)
          mbar_wait(bfull0 + 8u * (kb % kBStages), static_cast<uint32_t>(kb / kBStages) & 1u, budget, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      int n_mma = 0;
      if (!stream_b && !mbar_wait(xready, 0, budget, abort_flag)) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      } else {
        const uint32_t idesc = e4m3_idesc(128, npad);
        int s = 0;
        uint32_t round_par = 0;  // (i / stages) & 1, kept incrementally like the producer's
        for (int i = 0; i < nsub; ++i) {
          const int kbl = i / SUBS;
          const int which = i % SUBS;
          const int bslot = kbl % kBStages;
          if (stream_b && which == 0 &&
              !mbar_wait(bfull0 + 8u * bslot, static_cast<uint32_t>(kbl / kBStages) & 1u, budget, abort_flag)) {
            set_status(a.status, kStatusTimeout);
            *abort_flag = 1;
            break;
          }
          if (!mbar_wait(full0 + 8u * s, round_par, budget, abort_flag)) {
            set_status(a.status, kStatusTimeout);
            *abort_flag = 1;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sw128_kmajor_desc(smem_u32(ring + s * kSubBytes));
          const uint64_t bdesc =
              sw128_kmajor_desc(smem_u32(bsm + (stream_b ? bslot : kbl) * npad * 128));
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 4 x K=32 bytes per 128-byte swizzle row
            tc_mma_e4m3(tmem + static_cast<uint32_t>(which * npad), adesc + 2u * k, bdesc + 2u * k, idesc,
                        (kbl > 0 || k > 0) ? 1u : 0u);
          }
          ++n_mma;
          tc_commit(empty0 + 8u * s);  // stage free once these MMAs have read it
          if (stream_b && which == SUBS - 1) tc_commit(bempty0 + 8u * bslot);  // B slot free too
          if (++s == a.stages) {
            s = 0;
            round_par ^= 1u;
          }
        }
      }
      if (n_mma > 0) tc_commit(done);
      else mbar_arrive(done);
    }
    __syncwarp();
  } else {
    // ---- activation stager: e4m3 rows -> swizzled K-major B operand ----
    const int t = threadIdx.x - 64;
    const int per_row = nkb * 8;  // 16-byte chunks per token row of this K slice
    const int chunks = npad * per_row;
    // row and chunk-in-row of this thread's first chunk; the loops below step
    // them by 64 chunks without a division
    const int row_t = t / per_row;
    const int rem_t = t - row_t * per_row;
    if (a.x != nullptr) {
      // The B operand's token-padding rows (n_tok .. npad-1) stay zero: write the
      // whole slice as zeros now, before the wait, so that after it only the
      // real rows are quantised.
      for (int c = t; c < chunks; c += 64) *reinterpret_cast<uint4*>(bsm + c * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    pdl_wait();  // x (or x_q and s_x) is written by the preceding kernel
    pdl_trigger();
    if (a.x != nullptr) {
      // Fused quantiser (A1): amax over the whole [M][K] input, then this CTA's
      // K slice straight into the B operand.  Same arithmetic as act_quant.cu.
      // x (like x_q and s_x below) may be written by the preceding kernel while
      // this one already runs, so it is read through L2 (ld.global.cg), never
      // through the read-only path.
      const uint4* xv = reinterpret_cast<const uint4*>(a.x);
      const int nv = (a.M * a.K) >> 3;
      // This thread's first kKeep chunks of the CTA's K slice are loaded into
      // registers in the same batch as the amax loads, so quantising them
      // needs no second trip to memory.  With the cooperative quantiser these
      // chunks are the whole slice, and the only loads.
      constexpr int kKeep = 5;
      uint4 keep[2 * kKeep];
      {
        int row = row_t, rem = rem_t;
#pragma unroll
        for (int j = 0; j < kKeep; ++j) {
          keep[2 * j] = make_uint4(0u, 0u, 0u, 0u);
          keep[2 * j + 1] = keep[2 * j];
          const int c = t + 64 * j;
          if (c < chunks && row < n_tok) {
            const uint4* src =
                xv + ((static_cast<long long>(row) * a.K + (kb0 + (rem >> 3)) * 128 + (rem & 7) * 16) >> 3);
            keep[2 * j] = __ldcg(src);
            keep[2 * j + 1] = __ldcg(src + 1);
          }
          rem += 64;
          while (rem >= per_row) {
            rem -= per_row;
            ++row;
          }
        }
      }
      // amax over all of x: 16 independent 16-byte loads in flight per thread per
      // round, so x (10 KB at batch 1) arrives in one memory round trip.  The
      // cooperative quantiser takes the amax of its slice (the kept chunks)
      // and exchanges it with the cluster instead.
      constexpr int kBatch = 16;
      float m = 0.0f;
      if (a.coop) {
#pragma unroll
        for (int j = 0; j < 2 * kKeep; ++j) m = fmaxf(m, absmax8(keep[j]));
      }
      for (int base = a.coop ? nv : t; base < nv; base += 64 * kBatch) {
        uint4 u[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const int i = base + 64 * j;
          u[j] = i < nv ? __ldcg(xv + i) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) m = fmaxf(m, absmax8(u[j]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) misc->wmax[warp - 2] = m;
      asm volatile("bar.sync 1, 64;" ::: "memory");  // the two stager warps only
      float amax = fmaxf(misc->wmax[0], misc->wmax[1]);
      if (a.coop) {
        // The S slices of the cluster cover all of x: each CTA sends its slice
        // maximum to every CTA of the cluster (itself included), counted on the
        // receiver's amaxbar, and takes the maximum of the S values it receives.
        cluster_wait();  // every CTA of the cluster has initialised its barriers
        if (t == 0) {
          mbar_arrive_expect_tx(amaxbar, static_cast<uint32_t>(4 * S));
          const uint32_t slot = smem_u32(&misc->peer_amax[rank]);
          for (int p = 0; p < S; ++p)
            dsmem_st_async_f32(dsmem_addr(slot, static_cast<uint32_t>(p)), amax,
                               dsmem_addr(amaxbar, static_cast<uint32_t>(p)));
        }
        if (!mbar_wait_cluster(amaxbar, 0, budget)) {
          set_status(a.status, kStatusTimeout);
          *abort_flag = 1;
        }
        amax = 0.0f;
        for (int p = 0; p < S; ++p) amax = fmaxf(amax, misc->peer_amax[p]);
      }
      const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
      if (t == 0) misc->sx = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
      const bool publish = blockIdx.y == 0 && blockIdx.z == 0;  // one CTA column writes x_q / s_x
      if (publish && rank == 0 && t == 0) *a.s_x = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
      // This thread's chunks, in order; rows only grow with c, so the work ends
      // at the first padding row.  The first kKeep chunks come from registers,
      // in one unrolled block (independent chains), the rest are loaded here.
      auto put = [&](int row, int rem, uint4 v) {
        const int kbl = rem >> 3;
        const int ch = rem & 7;
        if (publish)
          *reinterpret_cast<uint4*>(const_cast<uint8_t*>(a.xq) + static_cast<long long>(row) * a.K +
                                    (kb0 + kbl) * 128 + ch * 16) = v;
        *reinterpret_cast<uint4*>(bsm + kbl * npad * 128 + (row >> 3) * 1024 + (row & 7) * 128 +
                                  ((ch ^ (row & 7)) << 4)) = v;
      };
      auto quant16 = [&](uint4 u0, uint4 u1) {
        return amax > 0.0f ? make_uint4(quant4(u0.x, u0.y, inv), quant4(u0.z, u0.w, inv),
                                        quant4(u1.x, u1.y, inv), quant4(u1.z, u1.w, inv))
                           : make_uint4(0u, 0u, 0u, 0u);
      };
      int row = row_t, rem = rem_t;
#pragma unroll
      for (int j = 0; j < kKeep; ++j) {
        if (t + 64 * j < chunks && row < n_tok) put(row, rem, quant16(keep[2 * j], keep[2 * j + 1]));
        rem += 64;
        while (rem >= per_row) {
          rem -= per_row;
          ++row;
        }
      }
      for (int c = t + 64 * kKeep; c < chunks && row < n_tok; c += 64) {
        const uint4* src = xv + ((static_cast<long long>(row) * a.K + (kb0 + (rem >> 3)) * 128 + (rem & 7) * 16) >> 3);
        put(row, rem, quant16(__ldcg(src), __ldcg(src + 1)));
        rem += 64;
        while (rem >= per_row) {
          rem -= per_row;
          ++row;
        }
      }
      fence_async_smem();
      mbar_arrive(xready);
    } else {
    if (t == 0) misc->sx = __ldcg(a.s_x);
    if (!a.tma_b) {
    // Stream the e4m3 activations of each k-block into the B ring with 16-byte
    // async copies, one commit group per k-block, kBStages-1 k-blocks in
    // flight: a block is published (bfull) as soon as its own group has landed,
    // so the L2 latency of one block overlaps the copies of the next ones.
    auto issue_kb = [&](int kb) -> bool {
      const int bslot = kb % kBStages;
      if (kb >= kBStages &&
          !mbar_wait(bempty0 + 8u * bslot, static_cast<uint32_t>((kb / kBStages) - 1) & 1u, budget, abort_flag)) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        return false;
      }
      uint8_t* blk = bsm + bslot * npad * 128;
      for (int c = t; c < npad * 8; c += 64) {
        const int row = c >> 3;
        const int ch = c & 7;
        uint8_t* dst = blk + (row >> 3) * 1024 + (row & 7) * 128 + ((ch ^ (row & 7)) << 4);
        if (row < n_tok) {
          const int tok = routed ? misc->tokens[row] : row;
          cp_async_16(smem_u32(dst), a.xq + static_cast<long long>(tok) * a.K + (kb0 + kb) * 128 + ch * 16);
        } else {
          *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      return true;
    };
    int committed = 0;  // commit groups so far, one per k-block issued (empty ones at the tail)
    bool alive = true;
    for (int kb = 0; kb < nkb && kb < kBStages - 1; ++kb) {
      alive = alive && issue_kb(kb);
      cp_async_commit();
      ++committed;
    }
    for (int kbl = 0; kbl < nkb && alive; ++kbl) {
      // publish k-block kbl as soon as its own group has landed ...
      cp_async_wait_pending(committed - (kbl + 1));
      fence_async_smem();
      mbar_arrive(bfull0 + 8u * (kbl % kBStages));
      // ... then refill the slot k-block kbl-1 used, once its MMAs are done
      // (waiting for them before the publish would chain the MMAs to this warp)
      const int kb_next = kbl + kBStages - 1;
      if (kb_next < nkb) alive = issue_kb(kb_next);
      cp_async_commit();
      ++committed;
    }
    cp_async_wait_pending(0);  // nothing in flight when the stager moves on
    }
    }
  }

  // ---- epilogue: TMEM -> shared partials -> cluster reduction -> bf16 ----------
  if (S > 1 && !(a.coop && warp >= 2)) cluster_wait();  // first phase (the cooperative stagers waited already)
  if (!mbar_wait(done, 0, budget, nullptr)) set_status(a.status, kStatusTimeout);
  tc_fence_after();
  pdl_wait();
  fence_async_smem();
  const float scale_w = __ldg(a.w_scale + expert);
  if (a.recv_bytes > 0) {
    // Push: each thread owns one accumulator row (its TMEM lane) and stores it
    // straight into the receive buffer of the CTA that owns that output row;
    // one cluster barrier later every owner holds all S partials locally.
    // (Non-blocking st.async stores counted on the owner's mbarrier instead of
    // the barrier were measured slower at M = 1.)
    const int Qr = (128 + S - 1) / S;
    const int row = warp * 32 + lane;
    const int owner = row / Qr;
    const int k = row - owner * Qr;
    const uint32_t dst = dsmem_addr(smem_u32(recv), static_cast<uint32_t>(owner));
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    for (int c0 = 0; c0 < SUBS * npad; c0 += 8) {
      uint32_t r[8];
      tmem_ld_x8(lane_base + static_cast<uint32_t>(c0), r);
      tmem_wait_ld();
      // npad is a multiple of 8, so the 8 columns share one sub-accumulator
      const int which = (SUBS == 2 && c0 >= npad) ? 1 : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int m = c0 - which * npad + j;
        if (m < n_tok)
          dsmem_st_f32(dst + static_cast<uint32_t>((((rank * SUBS + which) * npad + m) * Qr + k) * 4),
                       __uint_as_float(r[j]));
      }
    }
    tc_fence_before();
    cluster_sync();  // every partial of my rows has landed in my receive buffer
    const float scale = misc->sx * scale_w;
    const int rows = min(Qr, 128 - rank * Qr);
    const int items = rows > 0 ? rows * n_tok : 0;
    for (int it = threadIdx.x; it < items; it += kGemmThreads) {
      const int m = it / rows;
      const int kk = it - m * rows;
      const int orow = rank * Qr + kk;
      const int tok = routed ? misc->tokens[m] : m;
      // the S partials: every load issued up front (indices past S clamped to
      // rank 0's slot, in bounds, and not added), then summed in rank order
      float gp[8], up[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const int pp = p < S ? p : 0;
        gp[p] = recv[((pp * SUBS + 0) * npad + m) * Qr + kk];
        up[p] = kSwiglu ? recv[((pp * SUBS + 1) * npad + m) * Qr + kk] : 0.0f;
      }
      float g = gp[0];
      float u = up[0];
#pragma unroll
      for (int p = 1; p < 8; ++p) {
        if (p < S) {
          g += gp[p];
          u += up[p];
        }
      }
      if (kSwiglu) {
        const float yg = g * scale;
        const float yu = u * scale;
        const float o = yg / (1.0f + expf(-yg)) * yu;
        const __nv_bfloat16 bv = __float2bfloat16_rn(o);
        a.out[static_cast<long long>(tok) * a.ldo + tile * 128 + orow] = *reinterpret_cast<const uint16_t*>(&bv);
      } else {
        const int col = tile * 128 + orow;
        float y = g * scale;
        if (col < a.q_cols) y *= a.q_scale;
        const __nv_bfloat16 bv = __float2bfloat16_rn(y);
        a.out[static_cast<long long>(tok) * a.ldo + col] = *reinterpret_cast<const uint16_t*>(&bv);
      }
    }
    if (warp == 2) {
      tc_fence_after();
      tmem_dealloc(tmem, static_cast<uint32_t>(a.tmem_cols));
    }
    return;
  }
  // Pull (large M): partials parked in the drained ring, summed through DSMEM loads.
  float* part = reinterpret_cast<float*>(ring);  // [SUBS*npad][128]
  {
    const int row = warp * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int ncols = SUBS * npad;
    for (int c0 = 0; c0 < ncols; c0 += 64) {  // up to eight 8-column loads in flight per wait
      uint32_t r[8][8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (c0 + 8 * q < ncols) tmem_ld_x8(lane_base + static_cast<uint32_t>(c0 + 8 * q), r[q]);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int cq = c0 + 8 * q;  // 8 columns of one sub-accumulator (npad is a multiple of 8)
        const int mq = cq - ((SUBS == 2 && cq >= npad) ? npad : 0);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (cq < ncols && mq + j < n_tok) part[(cq + j) * 128 + row] = __uint_as_float(r[q][j]);
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // all S partial accumulators are complete and visible

  const float scale = misc->sx * scale_w;
  // This CTA owns output rows [4*g0, 4*(g0+ng)): groups of 4 consecutive rows,
  // so every peer read is one 16-byte load (a group's partials of one token
  // are contiguous in the parked [column][128 rows] layout).
  const int g0 = 32 * rank / S;
  const int ng = 32 * (rank + 1) / S - g0;
  const int items = ng * n_tok;  // (token, row group)
  const uint32_t part_base = smem_u32(part);
  // kPullBatch items per thread per round: all their peer loads are issued
  // before the first sum, so a round costs one DSMEM round trip, not one per item.
  constexpr int kPullBatch = 2;
  for (int it0 = threadIdx.x; it0 < items; it0 += kGemmThreads * kPullBatch) {
    float4 gv[kPullBatch][8], uv[kPullBatch][8];
#pragma unroll
    for (int q = 0; q < kPullBatch; ++q) {
      const int it = it0 + q * kGemmThreads;
      const int m = it / ng;
      const int row = 4 * (g0 + (it - m * ng));
      const uint32_t off_g = part_base + static_cast<uint32_t>((m * 128 + row) * 4);
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        gv[q][p] = make_float4(0.f, 0.f, 0.f, 0.f);
        uv[q][p] = gv[q][p];
        if (it < items && p < S) {
          gv[q][p] = dsmem_ld_f32x4(dsmem_addr(off_g, p));
          if (kSwiglu) uv[q][p] = dsmem_ld_f32x4(dsmem_addr(off_g + static_cast<uint32_t>(npad * 128 * 4), p));
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kPullBatch; ++q) {
      const int it = it0 + q * kGemmThreads;
      if (it >= items) continue;
      const int m = it / ng;
      const int row = 4 * (g0 + (it - m * ng));
      const int tok = routed ? misc->tokens[m] : m;
      float g[4] = {0.f, 0.f, 0.f, 0.f};
      float u[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int p = 0; p < 8; ++p) {  // peers summed in rank order
        g[0] += gv[q][p].x;
        g[1] += gv[q][p].y;
        g[2] += gv[q][p].z;
        g[3] += gv[q][p].w;
        u[0] += uv[q][p].x;
        u[1] += uv[q][p].y;
        u[2] += uv[q][p].z;
        u[3] += uv[q][p].w;
      }
      float o[4];
      const int col = tile * 128 + row;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (kSwiglu) {
          const float yg = g[i] * scale;
          const float yu = u[i] * scale;
          o[i] = yg / (1.0f + expf(-yg)) * yu;
        } else {
          o[i] = g[i] * scale;
          if (col + i < a.q_cols) o[i] *= a.q_scale;
        }
      }
      uint2 packed;
      packed.x = pack_bf16x2(o[0], o[1]);
      packed.y = pack_bf16x2(o[2], o[3]);
      *reinterpret_cast<uint2*>(a.out + static_cast<long long>(tok) * a.ldo + col) = packed;
    }
  }
  tc_fence_before();
  cluster_sync();  // peers are done reading this CTA's partials
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(a.tmem_cols));
  }
}

static int pow2_at_least(int v, int lo) {
  int p = lo;
  while (p < v) p <<= 1;
  return p;
}

cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t s) {
  const int KB = g.K / 128;
  const int SUBS = g.swiglu ? 2 : 1;
  const int n_tiles = g.swiglu ? (g.N / 2) / 128 : g.N / 128;
  const int npad_max = (g.M + 7) & ~7;
  const int b_per_kb = npad_max * 128;
  const int sms = sm_count();

  // split-K: about 1.6 CTAs per SM (measured best at batch 1-4), at least
  // enough that each CTA's slice of the activations fits the B buffer, at most
  // 8 (portable cluster) and KB.
  const bool stream_b = g.x == nullptr;
  int S;
  if (g.split > 0) {
    S = g.split;
  } else {
    S = (16 * sms / (n_tiles * g.slots) + 5) / 10;
    const int s_fit = (KB * b_per_kb + 45055) / 45056;  // keep a preloaded B <= 44 KB when possible
    if (!stream_b && s_fit <= 8 && S < s_fit) S = s_fit;
  }
  const int s_min = stream_b ? 1 : (KB * b_per_kb + 65535) / 65536;  // hard cap: preloaded B <= 64 KB
  if (S < s_min) S = s_min;
  if (S < 1) S = 1;
  if (S > 8) S = 8;
  if (S > KB) S = KB;
  if (S < s_min) return cudaErrorInvalidValue;
  const int nkb_max = (KB + S - 1) / S;
  const int bsm_bytes = stream_b ? kBStages * b_per_kb : nkb_max * b_per_kb;
  const int part_bytes = SUBS * npad_max * 128 * 4;
  // split-K partials are pushed into a dedicated receive buffer when it is small
  const int Qr = (128 + S - 1) / S;
  int recv_bytes = S * Qr * SUBS * npad_max * 4;
  if (recv_bytes > 20 * 1024 || S == 1) recv_bytes = 0;
  const int misc_bytes = static_cast<int>((sizeof(GemmMisc) + 15) & ~static_cast<size_t>(15)) + recv_bytes;
  auto smem_for = [&](int st) {
    return 1024 + st * kSubBytes + bsm_bytes + (2 * st + 3 + 2 * kBStages) * 8 + misc_bytes;
  };
  // the deepest ring (<= 6 stages) that keeps two CTAs per SM, else 6 stages at one CTA per SM
  int stages = 6;
  while (stages > 3 && 2 * (smem_for(stages) + 1024) > 233472) --stages;
  if (2 * (smem_for(stages) + 1024) > 233472) stages = 6;
  while (stages * kSubBytes < part_bytes) ++stages;
  int smem = smem_for(stages);
  if (smem > 232448) return cudaErrorInvalidValue;
  const int tmem_cols = pow2_at_least(SUBS * npad_max, 32);
  // TMEM safety: the CTAs that can share an SM must fit in its 512 columns.
  while ((233472 / (smem + 1024)) * tmem_cols > 512) smem += 1024;

  GemmArgs a{};
  a.w = g.w;
  a.w_expert_bytes = g.w_expert_bytes;
  a.w_scale = g.w_scale;
  a.xq = g.xq;
  a.s_x = g.s_x;
  a.x = g.x;
  a.status = g.status;
  a.out = g.out;
  a.expert_ids = g.expert_ids;
  a.M = g.M;
  a.K = g.K;
  a.KB = KB;
  a.ldo = g.ldo;
  a.E = g.E;
  a.q_cols = g.q_cols;
  a.q_scale = g.q_scale;
  a.stages = stages;
  a.bsm_bytes = bsm_bytes;
  a.tmem_cols = tmem_cols;
  a.recv_bytes = recv_bytes;
  // The fused quantiser shares the amax across the cluster once all of x no
  // longer arrives in one batch of loads per thread (16 vectors of 8 values
  // for each of the 64 stager threads) and each CTA's slice fits its kept
  // registers (5 chunks of 16 values per thread: M = 4 at K = 5120).
  a.coop = (g.x != nullptr && S > 1 && static_cast<long long>(g.M) * g.K > 64 * 16 * 8 &&
            static_cast<long long>(g.M) * nkb_max * 8 <= 64 * 5)
               ? 1
               : 0;
  a.debug = g.debug ? 1 : 0;
  // Dense streamed activations come in by tensor loads (routed tokens are
  // gathered row by row by the stager warps instead)
  a.tma_b = (stream_b && g.expert_ids == nullptr &&
             encode_u8_rows_sw128(&a.xq_map, g.xq, g.K, g.M, npad_max))
                ? 1
                : 0;

  Launch L(dim3(S, n_tiles, g.slots), dim3(kGemmThreads), static_cast<size_t>(smem), s,
           static_cast<unsigned>(S), g.pdl);
  cudaError_t e;
  if (g.swiglu) {
    e = ensure_kernel_attrs(reinterpret_cast<const void*>(gemm_e4m3_kernel<true>), smem, false);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&L.cfg, gemm_e4m3_kernel<true>, a);
  }
  e = ensure_kernel_attrs(reinterpret_cast<const void*>(gemm_e4m3_kernel<false>), smem, false);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&L.cfg, gemm_e4m3_kernel<false>, a);
}

}  // namespace dl
