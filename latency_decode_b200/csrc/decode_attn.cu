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
//  * a producer warp moves tiles of 16*W keys of K and V with TMA tensor copies
//    in the 128-byte swizzle (bank-conflict-free ldmatrix) into a ring of
//    stages; it does not wait for the preceding kernel (the KV cache is
//    static), so under PDL the ring fills while the QKV GEMM still runs.
//  * W consumer warps each take 16 keys of a tile and run swapped-AB
//    tensor-core MMAs (mma.sync m16n8k16, fp32 accumulation): S^T = K Q^T with
//    the keys as the M dimension and the R = G*T query rows as N (padded to 8,
//    not 16), then O^T += V^T P^T.  P^T is formed in registers with movmatrix;
//    the Q^T fragments are read from shared memory.
//  * online softmax in the log2 domain with a lazily raised running max; the
//    row max is a 3-step warp shuffle.
//  * merges: the W warp states merge in shared memory; each CTA then pushes
//    its state of every output item (a float4 of o and the row's (m, l)) into
//    the receive buffer of the CTA of the cluster that owns the item, through
//    distributed shared memory, with non-blocking stores that count their
//    bytes on the owner's mbarrier; once its bytes are in, each owner merges
//    the S states (M* = max m_i, L* = sum l_i 2^(m_i-M*), o = sum o_i
//    2^(m_i-M*) / L*).  With P = 1 that is the final result.  With P > 1 (used
//    when B*Hkv*S CTAs would leave the GPU half idle) each cluster stores its
//    merged state in the workspace and bumps a per-(b, kv head, owner)
//    counter; the cluster that arrives last merges the P states the same way
//    and resets the counter.  Nothing ever waits for another cluster.
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

// W consumer warps take 16 keys each of a stage of 16*W keys; one more warp
// is the TMA producer.  W = 8 (one CTA per SM, enough warps to hide the MMA and
// softmax latency) for clusters of up to 8 CTAs; W = 4 (two CTAs per SM where
// they fit) for 16-CTA clusters, which pack onto the GPCs only that way.
constexpr int kAttnMaxSplits = 16;    // clusters per (b, kv head)
constexpr int kAttnMaxCluster = 16;   // CTAs per cluster
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
  const float* kv_scale;  // FP8 cache only: device [2] = {s_k, s_v}
  int lpt;             // 1: grid z visits the sequences longest first
  int P;
  int stages;
  uint32_t stages_magic;  // ceil(2^32 / stages): i / stages == umulhi(i, magic) for i < 2^32 / stages
  int recv_off;        // byte offset of the DSMEM receive buffer
  int kv_evict_first;  // 1: K/V tiles are brought into L2 with the evict-first policy
  int debug;
};

// The four e4m3 codes of a 32-bit word (low byte first) -> two f16x2 words
// (codes 0-1, then 2-3; low half first).  Exact, since every e4m3 value is an
// f16 value.  The word's halves are the 16-bit operands of the two
// conversions directly: masking or shifting them out first cost two more
// instructions per pair on the attention's critical path.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi) : "r"(w));
}

__device__ __forceinline__ uint32_t ld_b32(const uint16_t* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

// F8: the KV cache holds e4m3 codes (one byte per element) with per-tensor
// scales s_k, s_v; K is [key][d] and V is stored transposed, [d][key].  The
// ring carries half the bytes, and the MMA operands are converted to f16 in
// registers straight from the TMA-landed tiles (cvt e4m3x2 -> f16x2), with no
// staging pass: inside each warp's 16 keys the MMA key index r stands for the
// physical key pi(r) = 4*((r%8)/2) + 2*(r/8) + r%2, and inside each k-step the
// d index of thread t for element e stands for physical d = 32t + 4ks + e.
// Both are fixed permutations of a dot product's terms (Q's fragments use the
// same d map; the causal mask uses pi), chosen so that every fragment a thread
// needs is 4 (V^T) or 16 (K) contiguous bytes.  Q and P are rounded to f16.
template <int D, int NT, int W, bool F8>
__global__ void __launch_bounds__(32 * (W + 1), W == 4 ? 2 : 1)
    decode_attn_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       const __grid_constant__ AttnArgs a) {
  static_assert(!F8 || D == 128, "the FP8 cache path is built for d = 128");
  constexpr int kAttnConsumers = W;
  constexpr int kAttnThreads = 32 * (W + 1);
  constexpr int kAttnKT = 16 * W;             // keys per pipeline stage
  constexpr int HALVES = D / 64;              // a swizzled row holds 64 16-bit values (128 bytes)
  constexpr int HALF_BYTES = kAttnKT * 128;   // kAttnKT keys x 128 bytes
  constexpr int KV_BYTES = F8 ? kAttnKT * D : HALVES * HALF_BYTES;  // one of K, V in a stage
  constexpr int STAGE_BYTES = 2 * KV_BYTES;
  constexpr int KS = D / 16;                  // MMA k-steps over d, and m-tiles of d
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint2* qs = reinterpret_cast<uint2*>(ring + a.stages * STAGE_BYTES);        // [KS][NT][32]
  uint8_t* recv_base = smem + a.recv_off;                                      // DSMEM receive buffer
  uint64_t* bars = reinterpret_cast<uint64_t*>(qs + KS * NT * 32);
  // bars: [stages] full, [stages] empty, then the receive barrier of the merge
  int* abort_word = reinterpret_cast<int*>(bars + 2 * a.stages + 1);
  int* last_word = abort_word + 1;
  volatile int* abort_flag = abort_word;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8u * a.stages;
  const uint32_t recv_bar = empty0 + 8u * a.stages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = gridDim.x;
  const int rank = static_cast<int>(cluster_rank());
  const int hk = blockIdx.y;
  const int zb = blockIdx.z / a.P;  // dispatch slot of the sequence
  const int split = blockIdx.z - zb * a.P;
  const long long budget = a.debug ? kWaitBudgetDebug : kWaitBudget;

  // Longest-first order: CTAs are dispatched in grid order, so when the grid
  // runs in several waves, mapping slot zb to the zb-th longest sequence (ties
  // by index) makes the hardware's in-order dispatch a longest-processing-time
  // schedule.  seq_lens is a static input, read before the PDL wait.
  __shared__ int lpt_seq;
  int b = zb;
  if (a.lpt) {
    for (int j = threadIdx.x; j < a.B; j += blockDim.x) {
      int Lj = __ldg(a.seq_lens + j);
      Lj = (Lj < a.T || Lj > a.Lcap) ? 0 : Lj;
      int rank_j = 0;
      for (int i = 0; i < a.B; ++i) {
        int Li = __ldg(a.seq_lens + i);
        Li = (Li < a.T || Li > a.Lcap) ? 0 : Li;
        rank_j += (Li > Lj || (Li == Lj && i < j)) ? 1 : 0;
      }
      if (rank_j == zb) lpt_seq = j;
    }
    __syncthreads();
    b = lpt_seq;
  }

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
    if (F8) mbar_init(recv_bar, 1);
    *abort_word = 0;
    *last_word = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // F8: every CTA's receive barrier is initialised before any peer stores into
  // it (the matching wait comes just before the merge's pushes).
  if constexpr (F8) cluster_arrive();

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
      const bool kv_ef = a.kv_evict_first != 0;
      const uint64_t kvpol = l2_policy_evict_first();
      const int z = b * a.Hkv + hk;
      const int n_issue = (a.debug && n_tiles > 0) ? n_tiles - 1 : n_tiles;  // test hook
      int issued = 0;
      int s = 0;               // stage of tile i, and
      uint32_t round_par = 0;  // (i / stages) & 1, both kept without a division
      for (int i = 0; i < n_issue; ++i) {
        if (i >= a.stages && !mbar_wait(empty0 + 8u * s, round_par ^ 1u, budget, abort_flag)) {
          set_status(a.status, kStatusTimeout);
          *abort_flag = 1;
          break;
        }
        const uint32_t st = smem_u32(ring + s * STAGE_BYTES);
        const uint32_t fb = full0 + 8u * s;
        mbar_arrive_expect_tx(fb, STAGE_BYTES);
        const int key0 = lo + i * kAttnKT;
        if (F8) {  // K: KT rows of 128 bytes; V^T: 128 rows (d) of KT bytes
          if (kv_ef) {
            tma_load_3d_policy(st, &tk, 0, key0, z, fb, kvpol);
            tma_load_3d_policy(st + KV_BYTES, &tv, key0, 0, z, fb, kvpol);
          } else {
            tma_load_3d(st, &tk, 0, key0, z, fb);
            tma_load_3d(st + KV_BYTES, &tv, key0, 0, z, fb);
          }
        } else {
#pragma unroll
          for (int h = 0; h < HALVES; ++h) {
            if (kv_ef) {
              tma_load_3d_policy(st + h * HALF_BYTES, &tk, h * 64, key0, z, fb, kvpol);
              tma_load_3d_policy(st + (HALVES + h) * HALF_BYTES, &tv, h * 64, key0, z, fb, kvpol);
            } else {
              tma_load_3d(st + h * HALF_BYTES, &tk, h * 64, key0, z, fb);
              tma_load_3d(st + (HALVES + h) * HALF_BYTES, &tv, h * 64, key0, z, fb);
            }
          }
        }
        issued = i + 1;
        if (++s == a.stages) {
          s = 0;
          round_par ^= 1u;
        }
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
    // staged once in shared memory by the consumer warps.  Each thread's QI
    // entries are loaded in one unrolled pass before any is stored, so the
    // staging costs one memory round trip, not one per entry.
    constexpr int QN = KS * NT * 32;                       // entries
    constexpr int QI = (QN + 32 * kAttnConsumers - 1) / (32 * kAttnConsumers);
    uint2 qv[QI];
#pragma unroll
    for (int i = 0; i < QI; ++i) {
      const int f = threadIdx.x + i * 32 * kAttnConsumers;
      const int ln = f & 31;
      const int nt = (f >> 5) % NT;
      const int ks = (f >> 5) / NT;
      const int rho = nt * 8 + (ln >> 2);
      qv[i] = make_uint2(0u, 0u);
      if (f < QN && rho < a.R) {
        const int t = rho / a.G;
        const int hq = hk * a.G + rho % a.G;
        const uint16_t* qrow =
            a.q + (static_cast<long long>(b) * a.T + t) * a.q_stride + static_cast<long long>(hq) * D;
        if (F8) {  // k-step ks, thread t: physical d = 32t + 4ks + e; bf16 -> f16
          const int d0 = 32 * (ln & 3) + 4 * ks;
          const uint32_t w0 = ld_b32(qrow + d0), w1 = ld_b32(qrow + d0 + 2);
          qv[i].x = pack_f16x2(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xFFFF0000u));
          qv[i].y = pack_f16x2(__uint_as_float(w1 << 16), __uint_as_float(w1 & 0xFFFF0000u));
        } else {
          qv[i].x = ld_b32(qrow + ks * 16 + 2 * (ln & 3));
          qv[i].y = ld_b32(qrow + ks * 16 + 8 + 2 * (ln & 3));
        }
      }
    }
#pragma unroll
    for (int i = 0; i < QI; ++i) {
      const int f = threadIdx.x + i * 32 * kAttnConsumers;
      if (f < QN) qs[f] = qv[i];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kAttnConsumers) : "memory");

    // F8: the cache holds k / s_k, so the logits take s_k into their scale
    const float scale_log2 = F8 ? a.scale_log2 * __ldg(a.kv_scale) : a.scale_log2;
    // F8: physical key offsets (within the warp's 16) of MMA rows g and g+8
    const int pA = F8 ? 4 * (g >> 1) + (g & 1) : g;
    const int pB = F8 ? pA + 2 : g + 8;

    int lim[NT][2];  // last visible key of the rows this thread accumulates
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int r2 = nt * 8 + 2 * q4 + j;
        lim[nt][j] = r2 < a.R ? L - a.T + r2 / a.G : -1;
      }

    for (int i = 0; i < n_tiles; ++i) {
      // stage and round of tile i: a multiply-high by the ring depth's
      // reciprocal instead of a division
      const uint32_t round = __umulhi(static_cast<uint32_t>(i), a.stages_magic);
      const int s = i - static_cast<int>(round) * a.stages;
      bool ok = !*abort_flag;
      if (ok && !mbar_wait(full0 + 8u * s, round & 1u, budget, abort_flag)) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);  // the warp-wide MMA path below needs a uniform decision
      const int key_base = lo + i * kAttnKT + warp * 16;
      if (ok && key_base < hi) {
        const uint32_t kbase = smem_u32(ring + s * STAGE_BYTES);
        const uint32_t vbase = kbase + KV_BYTES;
        // ---- S^T[16 keys x 8*NT rows] = K . Q^T ----
        float sc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) sc[nt][c] = 0.0f;
        if (F8) {
          // rows pi(g), pi(g+8) of K: bytes 32t .. 32t+31 (chunks 2t, 2t+1) hold
          // e = 0..3 of k-steps 0..7 for this thread
          const int rA = warp * 16 + pA, rB = warp * 16 + pB;
          const uint8_t* kt = ring + s * STAGE_BYTES;
          uint4 kA[2], kB[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            kA[h] = *reinterpret_cast<const uint4*>(kt + rA * 128 + (((2 * q4 + h) ^ (rA & 7)) << 4));
            kB[h] = *reinterpret_cast<const uint4*>(kt + rB * 128 + (((2 * q4 + h) ^ (rB & 7)) << 4));
          }
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const uint32_t wA = (&kA[ks >> 2].x)[ks & 3];
            const uint32_t wB = (&kB[ks >> 2].x)[ks & 3];
            uint32_t a0, a1, a2, a3;
            e4m3x4_to_f16x2x2(wA, a0, a2);
            e4m3x4_to_f16x2x2(wB, a1, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint2 qf = qs[(ks * NT + nt) * 32 + lane];
              mma_f16_16816(sc[nt], a0, a1, a2, a3, qf.x, qf.y);
            }
          }
        } else {
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
        const int kA = key_base + pA;  // physical keys of MMA rows g and g+8
        const int kB = key_base + pB;
        // A tile that every row sees in full (any but a chunk's last and the
        // causal diagonal) needs no mask: padding rows then see it too, but
        // their states are never stored.
        const bool full = key_base + 16 <= hi && key_base + 15 <= L - a.T;
        float x[NT][4];
        bool raise = false;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            x[nt][j] = (full || (kA < hi && kA <= lim[nt][j])) ? sc[nt][j] * scale_log2 : -INFINITY;
            x[nt][2 + j] = (full || (kB < hi && kB <= lim[nt][j])) ? sc[nt][2 + j] * scale_log2 : -INFINITY;
            const float thr = m_run[nt][j] + static_cast<float>(kLazyRescale);
            raise = raise || x[nt][j] > thr || x[nt][2 + j] > thr;
          }
        // Lazy rescale: the reference max m_run of a row moves only when this
        // tile's row max exceeds it by more than 2^kLazyRescale, so the O
        // rescale below is rarely needed and p stays <= 2^kLazyRescale, far
        // from overflow.  Whether any score of the warp exceeds its row's
        // threshold is one vote; only then are the row maxima taken (three
        // shuffle rounds per row) and the rows that need it rescaled.
        if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float mx = fmaxf(x[nt][j], x[nt][2 + j]);
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
              mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
              if (mx > m_run[nt][j] + static_cast<float>(kLazyRescale)) {
                const float alpha = ex2(m_run[nt][j] - mx);  // 0 when m_run is -inf
                l_run[nt][j] *= alpha;
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                  o[mt][nt][j] *= alpha;
                  o[mt][nt][2 + j] *= alpha;
                }
                m_run[nt][j] = mx;
              }
            }
        }
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float p[4];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float m_use = (m_run[nt][j] == -INFINITY) ? 0.0f : m_run[nt][j];
            p[j] = ex2(x[nt][j] - m_use);
            p[2 + j] = ex2(x[nt][2 + j] - m_use);
            l_run[nt][j] += p[j] + p[2 + j];
          }
          // P^T as the B operand [k = key][n = row]: transpose each 8x8 block
          pb[nt][0] = movmatrix_t(F8 ? pack_f16x2(p[0], p[1]) : pack_bf16x2(p[0], p[1]));
          pb[nt][1] = movmatrix_t(F8 ? pack_f16x2(p[2], p[3]) : pack_bf16x2(p[2], p[3]));
        }
        // ---- O^T[d x rows] += V^T . P^T ----
        if (F8) {
          // V^T rows 16mt+g and 16mt+g+8 (d), bytes warp*16 + 4t .. +3 = MMA keys
          // 2t, 2t+1 (e = 0, 1) and 2t+8, 2t+9 (e = 2, 3)
          // Two m-tiles per ldmatrix: lane l addresses row l % 8 of matrix l / 8,
          // matrices 0-3 being V^T rows 16mt + {0, 8} and 16(mt+1) + {0, 8}.  A
          // matrix row is this warp's 16-byte chunk (keys warp*16 .. +15) of a
          // V^T row as TMA swizzled it: chunk index XOR the row's low 3 bits
          // (128-byte rows) or bits 1-2 (64-byte rows).  Thread t of group g so
          // receives bytes 4t .. 4t+3 of that chunk in row g of each matrix.
          const int mi = lane >> 3, rr = lane & 7;
          const int vch = kAttnKT == 128 ? ((warp ^ rr) & 7) : ((warp ^ (rr >> 1)) & 3);
          const uint32_t vaddr = smem_u32(ring + s * STAGE_BYTES + KV_BYTES) +
                                 static_cast<uint32_t>((16 * (mi >> 1) + 8 * (mi & 1) + rr) * kAttnKT + (vch << 4));
#pragma unroll
          for (int mt = 0; mt < KS; mt += 2) {
            uint32_t w[4];
            ldsm_x4(vaddr + static_cast<uint32_t>(mt * 16 * kAttnKT), w[0], w[1], w[2], w[3]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t a0, a1, a2, a3;
              e4m3x4_to_f16x2x2(w[2 * h], a0, a2);
              e4m3x4_to_f16x2x2(w[2 * h + 1], a1, a3);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_f16_16816(o[mt + h][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
            }
          }
        } else {
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
  // Rows of the per-warp o are padded to D + 4 floats: the 4 lanes of a fragment
  // that write the same column of 4 different rows then hit 4 different banks.
  constexpr int DP = D + 4;
  float* wo = reinterpret_cast<float*>(ring);             // [W][R][DP] per-warp o
  float* wm = wo + kAttnConsumers * R * DP;               // [W][R]
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
            wo[(warp * R + rho) * DP + mt * 16 + g] = o[mt][nt][j];
            wo[(warp * R + rho) * DP + mt * 16 + g + 8] = o[mt][nt][2 + j];
          }
        }
      }
  }
  __syncthreads();

  // ---- merge the W warp states and push the CTA state to the slice owners ----
  // Outputs are I = R*D/4 float4 items; CTA c of the cluster owns items
  // [c*Q, (c+1)*Q).  Every CTA stores its state of item i -- the float4 of o
  // and the (m, l) of its row -- straight into the receive buffer of the owner
  // of i (two remote shared-memory stores per item, no round trip).  bf16
  // cache: plain remote stores, then one cluster barrier.  FP8 cache:
  // non-blocking remote stores (st.async) that count their bytes on the
  // owner's receive barrier, where the owner waits (measured faster for this
  // variant only).  Each owner then merges the S states of its items locally.
  const int I = R * (D / 4);
  const int Q = (I + S - 1) / S;
  const int my0 = rank * Q;
  const int cnt = max(0, min(I, my0 + Q) - my0);
  float4* rv_o = reinterpret_cast<float4*>(recv_base);      // [S][Q]
  float2* rv_ml = reinterpret_cast<float2*>(rv_o + S * Q);  // [S][Q] (m, l)
  const uint32_t rv_o_l = smem_u32(rv_o), rv_ml_l = smem_u32(rv_ml);
  if constexpr (F8) {
    cluster_wait();  // every receive barrier of the cluster is initialised
    // (test hook: 16 bytes more are expected than the peers send, so the
    // owner's bounded receive wait below runs out)
    if (threadIdx.x == 0)
      mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>(S * cnt * (16 + 8) + (a.debug ? 16 : 0)));
  }
  for (int it = threadIdx.x; it < I; it += kAttnThreads) {
    const int rho = it / (D / 4);
    const int c4 = it - rho * (D / 4);
    // Every load is issued up front and unconditionally (all are in bounds), so
    // the W states cost one shared-memory round trip rather than one per warp;
    // a warp without visible keys (l = 0) gets weight 0.
    float mw[kAttnConsumers], lw[kAttnConsumers];
    float4 ow[kAttnConsumers];
#pragma unroll
    for (int w = 0; w < kAttnConsumers; ++w) {
      mw[w] = wm[w * R + rho];
      lw[w] = wl[w * R + rho];
      ow[w] = *reinterpret_cast<const float4*>(wo + (w * R + rho) * DP + c4 * 4);
    }
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnConsumers; ++w) M = lw[w] > 0.0f ? fmaxf(M, mw[w]) : M;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < kAttnConsumers; ++w) {
      const float f = lw[w] > 0.0f ? ex2(mw[w] - M) : 0.0f;
      acc.x += ow[w].x * f;
      acc.y += ow[w].y * f;
      acc.z += ow[w].z * f;
      acc.w += ow[w].w * f;
      lsum += lw[w] * f;
    }
    const int owner = it / Q;
    const uint32_t slot_i = static_cast<uint32_t>(rank * Q + (it - owner * Q));
    if constexpr (F8) {
      const uint32_t owner_bar = dsmem_addr(recv_bar, owner);
      dsmem_st_async_f32x4(dsmem_addr(rv_o_l + 16u * slot_i, owner), acc, owner_bar);
      dsmem_st_async_f32x2(dsmem_addr(rv_ml_l + 8u * slot_i, owner), M, lsum, owner_bar);
    } else {
      dsmem_st_f32x4(dsmem_addr(rv_o_l + 16u * slot_i, owner), acc);
      dsmem_st_f32x2(dsmem_addr(rv_ml_l + 8u * slot_i, owner), M, lsum);
    }
  }
  // every state of my items has landed in my receive buffer
  bool recv_ok = true;
  if constexpr (F8) {
    cluster_arrive();  // this CTA's pushes are issued (waited for before the CTA exits)
    recv_ok = mbar_wait_cluster(recv_bar, 0, budget);
    if (!recv_ok) set_status(a.status, kStatusTimeout);
  } else {
    cluster_sync();
  }

  // ---- merge the S CTA states of my items ----
  const float out_scale = F8 ? __ldg(a.kv_scale + 1) : 1.0f;  // F8: the cache holds v / s_v
  const long long head = static_cast<long long>(b) * a.Hkv + hk;
  const long long slot = head * a.P + split;
  for (int k = threadIdx.x; k < cnt; k += kAttnThreads) {
    const int it = my0 + k;
    const int rho = it / (D / 4);
    const int c4 = it - rho * (D / 4);
    // All (m, l) first, then the o states in groups of 4, each group's loads
    // issued together; indices past S are clamped to S - 1 (in bounds) and get
    // weight 0, so no load sits behind a branch.
    float mp[kAttnMaxCluster], lp[kAttnMaxCluster];
#pragma unroll
    for (int p = 0; p < kAttnMaxCluster; ++p) {
      const float2 ml = rv_ml[(p < S ? p : S - 1) * Q + k];
      mp[p] = ml.x;
      lp[p] = p < S ? ml.y : 0.0f;
    }
    float M = -INFINITY;
#pragma unroll
    for (int p = 0; p < kAttnMaxCluster; ++p) M = lp[p] > 0.0f ? fmaxf(M, mp[p]) : M;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float lsum = 0.0f;
#pragma unroll
    for (int p0 = 0; p0 < kAttnMaxCluster; p0 += 4) {
      if (p0 >= S) break;
      float4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = rv_o[(p0 + q < S ? p0 + q : S - 1) * Q + k];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float f = lp[p0 + q] > 0.0f ? ex2(mp[p0 + q] - M) : 0.0f;
        acc.x += v[q].x * f;
        acc.y += v[q].y * f;
        acc.z += v[q].z * f;
        acc.w += v[q].w * f;
        lsum += lp[p0 + q] * f;
      }
    }
    if (a.P == 1) {
      const float inv = lsum > 0.0f ? out_scale / lsum : 0.0f;
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
        // as in the owner merge: every load of a group issued together, indices
        // past P clamped and weighted 0
        float mq[kAttnMaxSplits], lq[kAttnMaxSplits];
#pragma unroll
        for (int p = 0; p < kAttnMaxSplits; ++p) {
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(
              a.part_ml + (((head * a.P + (p < a.P ? p : a.P - 1)) * S + rank) * R + rho) * 2));
          mq[p] = ml.x;
          lq[p] = p < a.P ? ml.y : 0.0f;
        }
        float M = -INFINITY;
#pragma unroll
        for (int p = 0; p < kAttnMaxSplits; ++p) M = lq[p] > 0.0f ? fmaxf(M, mq[p]) : M;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float lsum = 0.0f;
#pragma unroll
        for (int p0 = 0; p0 < kAttnMaxSplits; p0 += 4) {
          if (p0 >= a.P) break;
          float4 v[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            v[q] = __ldcg(reinterpret_cast<const float4*>(
                a.part_o + ((head * a.P + (p0 + q < a.P ? p0 + q : a.P - 1)) * I + it) * 4));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float f = lq[p0 + q] > 0.0f ? ex2(mq[p0 + q] - M) : 0.0f;
            acc.x += v[q].x * f;
            acc.y += v[q].y * f;
            acc.z += v[q].z * f;
            acc.w += v[q].w * f;
            lsum += lq[p0 + q] * f;
          }
        }
        const float inv = lsum > 0.0f ? out_scale / lsum : 0.0f;
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
  // bf16 cache: no trailing cluster barrier; once a CTA has passed the cluster
  // barrier above, every peer's stores into its shared memory have landed.
  // FP8 cache: a CTA leaves only once every CTA of the cluster has issued its
  // pushes, so that no peer can still store into the shared memory of a CTA
  // whose bounded receive wait ran out; the bytes issued before that barrier
  // are then given one more bounded wait to land.
  if constexpr (F8) {
    cluster_wait();
    if (!recv_ok) (void)mbar_wait_cluster(recv_bar, 0, budget);
  }
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

// A cache as a 3-D tensor map.  [BH][Lcap][d] with 128-byte rows per box: bf16
// in boxes of 64 elements (two per key for d = 128), or e4m3 in one box of
// d = 128 bytes.  transposed (the e4m3 V^T cache, [BH][d][Lcap]): boxes of d
// rows of kt bytes (128: 128-byte swizzle; 64: 64-byte swizzle).
static bool encode_kv_map(CUtensorMap* m, const void* base, int d, int Lcap, int BH, int kt, bool fp8,
                          bool transposed) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t esz = fp8 ? 1 : 2;
  cuuint32_t estr[3] = {1, 1, 1};
  if (transposed) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(Lcap), static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(Lcap), static_cast<cuuint64_t>(Lcap) * d};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(kt), static_cast<cuuint32_t>(d), 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, kt == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(Lcap), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esz, static_cast<cuuint64_t>(Lcap) * d * esz};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(kt), 1};
  return enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_u8_rows_sw128(CUtensorMap* m, const void* base, int row_bytes, int rows, int box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr || row_bytes < 128 || row_bytes % 16 != 0 || rows < 1 || box_rows < 1 || box_rows > 256)
    return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows), 1};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes),
                           static_cast<cuuint64_t>(row_bytes) * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
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

template <int D, int NT, int W, bool F8>
static AttnPlan attn_plan(int R, int S) {
  constexpr int STAGE_BYTES = F8 ? 2 * (16 * W) * D : 2 * (D / 64) * (16 * W) * 128;
  const int merge_bytes = (W * R * (D + 4) + 2 * W * R) * 4;  // per-warp o rows padded to D + 4
  const int I = R * (D / 4);
  const int Q = (I + S - 1) / S;
  const int recv_bytes = S * Q * (16 + 8);
  const int qs_bytes = (D / 16) * NT * 32 * 8;
  auto smem_for = [&](int st) {
    return 1024 + st * STAGE_BYTES + qs_bytes + (2 * st + 1) * 8 + 16 + recv_bytes + 16;
  };
  int stages = D == 128 ? 3 : 6;
  // W = 4 is chosen to put two CTAs on each SM: give up ring depth (down to
  // two stages) before that
  while (W == 4 && stages > 2 && 2 * (smem_for(stages) + 1024) > 233472) --stages;
  if (W == 8 || 2 * (smem_for(stages) + 1024) > 233472) {
    stages = 6;
    while (stages > 2 && smem_for(stages) > 232448) --stages;
  }
  while (stages * STAGE_BYTES < merge_bytes) ++stages;  // the merge reuses the drained ring
  AttnPlan pl;
  pl.stages = stages;
  pl.smem = smem_for(stages);
  pl.recv_off = ((stages * STAGE_BYTES + qs_bytes + (2 * stages + 1) * 8 + 16) + 15) & ~15;
  return pl;
}

template <int D, int NT, int W, bool F8>
static cudaError_t attn_configure(const AttnPlan& pl, int S) {
  return ensure_kernel_attrs(reinterpret_cast<const void*>(decode_attn_kernel<D, NT, W, F8>), pl.smem, S > 8);
}

// Clusters of S CTAs of this kernel that can be resident on the GPU at once.
template <int D, int NT, int W, bool F8>
static int attn_max_clusters_t(int R, int S) {
  const AttnPlan pl = attn_plan<D, NT, W, F8>(R, S);
  const int per_sm = 233472 / (pl.smem + 1024) >= 2 ? 2 : 1;
  int fallback = (sm_count() * per_sm) / S;
  if (attn_configure<D, NT, W, F8>(pl, S) != cudaSuccess) {
    (void)cudaGetLastError();
    return fallback;
  }
  Launch L(dim3(S, 1, 1), dim3(32 * (W + 1)), static_cast<size_t>(pl.smem), nullptr, static_cast<unsigned>(S), false);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_attn_kernel<D, NT, W, F8>, &L.cfg) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    return fallback;
  }
  return n;
}

// Consumer warps per CTA.  W = 8 (one CTA per SM) when the grid fits in one
// wave; W = 4 (two CTAs per SM, each overlapping the other's start-up and
// merge) for 16-CTA clusters and for grids of more CTAs than SMs, where a CTA's
// fixed costs would otherwise repeat once per wave (batch16x4: 118 -> 97 us).
static int attn_warps(int S, long long ctas) { return (S >= 16 || ctas > sm_count()) ? 4 : 8; }

template <int W, bool F8>
static int attn_max_clusters_w(int d, int R, int S) {
  const int NT = (R + 7) / 8;
  if (F8 || d == 128) {
    switch (NT) {
      case 1: return attn_max_clusters_t<128, 1, W, F8>(R, S);
      case 2: return attn_max_clusters_t<128, 2, W, F8>(R, S);
      case 3: return attn_max_clusters_t<128, 3, W, F8>(R, S);
      default: return attn_max_clusters_t<128, 4, W, F8>(R, S);
    }
  }
  switch (NT) {
    case 1: return attn_max_clusters_t<64, 1, W, false>(R, S);
    case 2: return attn_max_clusters_t<64, 2, W, false>(R, S);
    case 3: return attn_max_clusters_t<64, 3, W, false>(R, S);
    default: return attn_max_clusters_t<64, 4, W, false>(R, S);
  }
}

struct AttnShapeKey {
  int d, R, S, W;
  bool fp8;
};

static int attn_max_clusters_query(const void* ctx) {
  const AttnShapeKey& k = *static_cast<const AttnShapeKey*>(ctx);
  if (k.fp8)
    return k.W == 8 ? attn_max_clusters_w<8, true>(k.d, k.R, k.S) : attn_max_clusters_w<4, true>(k.d, k.R, k.S);
  return k.W == 8 ? attn_max_clusters_w<8, false>(k.d, k.R, k.S) : attn_max_clusters_w<4, false>(k.d, k.R, k.S);
}

// The occupancy query costs a runtime round trip: asked once per device and shape.
static int attn_max_clusters(int d, int R, int S, bool fp8, int W) {
  const AttnShapeKey k{d, R, S, W, fp8};
  const unsigned long long key = (1ull << 60) | (static_cast<unsigned long long>(W) << 52) |
                                 (static_cast<unsigned long long>(fp8) << 48) |
                                 (static_cast<unsigned long long>(d) << 32) |
                                 (static_cast<unsigned long long>(R) << 16) | static_cast<unsigned long long>(S);
  return memo_int(key, attn_max_clusters_query, &k);
}

// Clusters per (b, kv head).  Splitting a head over P clusters costs a merge
// through the workspace (~2-3 us), so it is used only when each CTA would
// otherwise stream long chunks (>= 2048 keys), with >= 1024 keys per CTA
// left, and never beyond the clusters that can be resident at once.
int attn_auto_splits(int B, int Hkv, int cluster, int Lcap, int d, int R, bool fp8) {
  const long long keys_per_cta = Lcap / cluster;
  if (keys_per_cta < 2048) return 1;
  const long long heads = static_cast<long long>(B) * Hkv;
  const long long resident = attn_max_clusters(d, R, cluster, fp8, attn_warps(cluster, heads * cluster));
  long long P = resident / heads;
  if (P > keys_per_cta / 1024) P = keys_per_cta / 1024;
  if (P > kAttnMaxSplits) P = kAttnMaxSplits;
  return P < 1 ? 1 : static_cast<int>(P);
}

template <int D, int NT, int W, bool F8>
static cudaError_t launch_attn_t(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                                 const AttnLaunch& p, cudaStream_t s) {
  const AttnPlan pl = attn_plan<D, NT, W, F8>(a.R, p.cluster);
  AttnArgs args = a;
  args.stages = pl.stages;
  args.stages_magic = static_cast<uint32_t>((0x100000000ull + pl.stages - 1) / pl.stages);
  args.recv_off = pl.recv_off;
  cudaError_t e = attn_configure<D, NT, W, F8>(pl, p.cluster);
  if (e != cudaSuccess) return e;
  Launch L(dim3(p.cluster, p.Hkv, p.B * a.P), dim3(32 * (W + 1)), static_cast<size_t>(pl.smem), s,
           static_cast<unsigned>(p.cluster), p.pdl);
  return cudaLaunchKernelEx(&L.cfg, decode_attn_kernel<D, NT, W, F8>, tk, tv, args);
}

template <int W>
static cudaError_t launch_attn_w(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a,
                                 const AttnLaunch& p, cudaStream_t s, int NT) {
  if (p.fp8) {
    if (p.d != 128) return cudaErrorInvalidValue;
    switch (NT) {
      case 1: return launch_attn_t<128, 1, W, true>(tk, tv, a, p, s);
      case 2: return launch_attn_t<128, 2, W, true>(tk, tv, a, p, s);
      case 3: return launch_attn_t<128, 3, W, true>(tk, tv, a, p, s);
      case 4: return launch_attn_t<128, 4, W, true>(tk, tv, a, p, s);
    }
  } else if (p.d == 128) {
    switch (NT) {
      case 1: return launch_attn_t<128, 1, W, false>(tk, tv, a, p, s);
      case 2: return launch_attn_t<128, 2, W, false>(tk, tv, a, p, s);
      case 3: return launch_attn_t<128, 3, W, false>(tk, tv, a, p, s);
      case 4: return launch_attn_t<128, 4, W, false>(tk, tv, a, p, s);
    }
  } else if (p.d == 64) {
    switch (NT) {
      case 1: return launch_attn_t<64, 1, W, false>(tk, tv, a, p, s);
      case 2: return launch_attn_t<64, 2, W, false>(tk, tv, a, p, s);
      case 3: return launch_attn_t<64, 3, W, false>(tk, tv, a, p, s);
      case 4: return launch_attn_t<64, 4, W, false>(tk, tv, a, p, s);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn(const AttnLaunch& p, cudaStream_t s) {
  const int W = attn_warps(p.cluster, static_cast<long long>(p.B) * p.Hkv * p.cluster);
  const int kt = 16 * W;  // keys per stage of the chosen variant
  CUtensorMap tk, tv;
  if (!encode_kv_map(&tk, p.k, p.d, p.Lcap, p.B * p.Hkv, kt, p.fp8, false) ||
      !encode_kv_map(&tv, p.v, p.d, p.Lcap, p.B * p.Hkv, kt, p.fp8, p.fp8))
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
  int P = p.splits > 0 ? p.splits : attn_auto_splits(p.B, p.Hkv, p.cluster, p.Lcap, p.d, a.R, p.fp8);
  while (P > 1 && attn_ws_bytes(p.B, p.Hkv, a.R, p.d, P, p.cluster) > p.ws_bytes) --P;
  if (static_cast<long long>(p.B) * P > 65535) P = 1;
  a.P = P;
  a.counters = nullptr;
  a.part_ml = a.part_o = nullptr;
  a.kv_scale = p.kv_scale;
  a.lpt = (p.B > 1 && p.B <= 128) ? 1 : 0;  // the in-kernel ranking is O(B^2 / threads)
  // A cache larger than half of L2 streams through it once per call: its lines
  // are marked evict-first, so that they leave L2 before anything the
  // neighbouring kernels re-read (measured: verify4 chain 63.8 -> 60.0 us,
  // batch16x4 134.5 -> 125.0 us; a 16.8 MB cache at batch 1 lost 0.2 us with it).
  const double kv_bytes = 2.0 * p.B * p.Hkv * static_cast<double>(p.Lcap) * p.d * (p.fp8 ? 1 : 2);
  a.kv_evict_first = kv_bytes > 64.0 * 1024 * 1024 ? 1 : 0;
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
