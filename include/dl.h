/*
 * dl.h -- C ABI of libdl.so, the B200 (sm_100a) low-latency FP8 decode kernels.
 *
 * The library implements the decode hot path described by the NVIDIA technical
 * blog "Blackwell breaks the 1,000 TPS/user barrier with Meta's Llama 4
 * Maverick" (cited below as [NV], Korean edition) and its Chinese rewrite by
 * Xinzhiyuan (cited as [XZY]):
 *   - an FP8 (e4m3, per-tensor scale) weight-streaming GEMM at tiny M with two
 *     fused epilogues, FC13+SwiGLU and FC_QKV+attention scaling, plus a grouped
 *     per-expert (MoE) variant;
 *   - grouped-query decode attention split along the KV sequence, whose per-block
 *     partial softmax states are merged across a thread-block cluster through
 *     distributed shared memory;
 *   - consecutive kernels chained with Programmatic Dependent Launch.
 *
 * Conventions that hold for every entry point
 * -------------------------------------------
 * - Every data pointer is a DEVICE pointer unless stated otherwise; the caller
 *   allocates and owns every buffer.  The library never allocates, frees or
 *   synchronises in these calls (dl_read_status is the one call that
 *   synchronises the stream).
 * - bf16 tensors are passed as their raw 16-bit patterns (uint16_t); e4m3
 *   tensors as raw bytes (uint8_t, OCP FP8 E4M3 "e4m3fn" encoding).
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).
 * - Errors the host can see (null pointers, shapes, alignment, workspace size)
 *   are returned BEFORE anything is launched.  A failed launch returns
 *   DL_ERR_CUDA.  Errors only the device can see (a bounded wait that ran out,
 *   a sequence length or expert id out of range) are OR-ed into the status
 *   word of the workspace and reported by dl_read_status; the outputs of that
 *   call are then undefined.
 * - Outputs are written in full on success.
 * - With DL_FLAG_PDL each kernel is launched with programmatic stream
 *   serialisation.  Every kernel of this library waits for its predecessor
 *   before it triggers its own dependents, and reads only "static" inputs
 *   (packed weights, weight scales, KV cache, sequence lengths, expert ids)
 *   before that wait.  Hence: with DL_FLAG_PDL, those static inputs must not be
 *   outputs of the kernel that immediately precedes the call in the stream
 *   when that kernel is itself one of this library's kernels.
 * - Workspace: `ws` is device memory of at least dl_workspace_bytes(...) bytes,
 *   256-byte aligned, zero-filled by the caller once before first use.  Layout:
 *     [0, 4)        uint32 status word (bits: 1 timeout, 2 bad sequence length,
 *                   4 bad expert id); cleared by dl_read_status
 *     [8, 12)       float  s_x, the activation scale of the last GEMM call
 *     [256, 256+M*K) uint8 x_q, the e4m3 activations [M][K] of the last GEMM call
 *   Two calls that may run concurrently (or overlap under PDL) must not share
 *   a workspace, except dl_add_rmsnorm_quant and the GEMM that follows it with
 *   DL_FLAG_XQ_READY, which hand x_q over through it.
 */
#ifndef LATENCY_DECODE_DL_H
#define LATENCY_DECODE_DL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dl_status {
  DL_OK = 0,
  DL_ERR_INVALID_ARG = 1,   /* null pointer, shape or range error (host-side) */
  DL_ERR_UNSUPPORTED = 2,   /* a shape this build does not implement */
  DL_ERR_ALIGNMENT = 3,     /* a pointer or stride is not aligned as required */
  DL_ERR_WORKSPACE = 4,     /* ws is null, misaligned or smaller than required */
  DL_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
  DL_ERR_TIMEOUT = 6,       /* a bounded device wait ran out (from dl_read_status) */
  DL_ERR_DEVICE_ARG = 7     /* the device found a bad seq_len / expert id (from dl_read_status) */
} dl_status;

/* flags (bitwise OR) */
#define DL_FLAG_PDL 1u            /* launch with Programmatic Dependent Launch */
#define DL_FLAG_DEBUG_TIMEOUT 2u  /* test hook: shortens every bounded wait to ~2 ms and
                                     withholds the last pipeline load, so the consumer's
                                     wait runs out and DL_ERR_TIMEOUT is reported; in the
                                     FP8-cache attention merge each owner CTA also expects
                                     16 bytes more than its peers send, so its receive
                                     wait runs out as well */
#define DL_FLAG_XQ_READY 4u        /* GEMM entry points: the workspace already holds x_q and
                                     s_x, written into this same workspace by
                                     dl_add_rmsnorm_quant; the GEMM skips its activation
                                     quantisation and `x` may be NULL */
#define DL_FLAG_COPY_NO_WAIT 16u   /* dl_copy only: the copy neither reads what the kernel
                                     before it in the stream writes nor writes what that
                                     kernel reads, so under DL_FLAG_PDL it starts without
                                     waiting for it (the caller vouches for this) */
#define DL_FLAG_SPLIT_SHIFT 8     /* bits [8,13): if non-zero, force the GEMM split-K
                                     cluster size (1..8), or the number of clusters per
                                     (b, kv head) of dl_decode_attn (1..16), instead of
                                     the built-in choice */

/* weight pack kinds */
#define DL_PACK_PLAIN 0   /* FC_QKV and other plain projections */
#define DL_PACK_SWIGLU 1  /* FC13: gate rows [0,F) and up rows [F,2F) paired per tile */

/* ---------------------------------------------------------------------------
 * Offline weight swizzle.  [XZY] "CUDA 内核优化与融合", item "GEMM 权重重排";
 * [NV] "CUDA kernel optimisation and fusion": the GEMM weights are rearranged
 * offline into a swizzled layout so that the result read back from Tensor
 * Memory after the tensor-core MMA lands in a convenient order.
 *
 * Input  w_nk: canonical e4m3 weight, row-major [N][K] (nn.Linear layout).
 * Output w_packed: N*K bytes.  Let KB = K/128.  The packed tensor is a
 * sequence of 16384-byte blocks; each block is the shared-memory image of 128
 * weight rows x 128 K-bytes in the tcgen05 K-major 128-byte-swizzle layout:
 * byte c of row r sits at (r/8)*1024 + (r%8)*128 + ((c/16) ^ (r%8))*16 + c%16.
 *   DL_PACK_PLAIN  (N % 128 == 0): block (t*KB + kb) holds rows 128t..128t+127,
 *                  K-bytes 128kb..128kb+127.
 *   DL_PACK_SWIGLU (N % 256 == 0, F = N/2): block 2*(t*KB + kb) holds gate rows
 *                  128t..128t+127 and block 2*(t*KB + kb)+1 the up rows
 *                  F+128t..F+128t+127, for the same K-bytes.  The gate and up
 *                  accumulators of one output column then land in the same
 *                  Tensor Memory lane, so SwiGLU needs no data exchange.
 * Requirements: K % 128 == 0, pointers 16-byte aligned, w_nk and w_packed must
 * not overlap.  The pack is an exact byte permutation.
 * ------------------------------------------------------------------------- */
dl_status dl_pack_fp8_weight(const uint8_t* w_nk, uint8_t* w_packed, int N, int K, int kind,
                             void* stream);

/* Bytes of workspace a GEMM call with M rows of K activations needs
 * (256 + M*K rounded up to 256).  dl_workspace_bytes(0, 0) = 256 (the status
 * word only) is the least dl_decode_attn accepts; see
 * dl_decode_attn_workspace_bytes for the size it can use. */
size_t dl_workspace_bytes(int M, int K);

/* ---------------------------------------------------------------------------
 * FC13 + SwiGLU.  [XZY] "运算融合" and [NV] fusion list: SwiGLU is fused into
 * the GEMM before it; the activation Quantize is fused ahead of the GEMM.
 *   x       bf16 [M][K], row-major, 16-byte aligned
 *   w_packed e4m3, DL_PACK_SWIGLU layout of the [N2][K] weight, 16-byte aligned
 *   w_scale device float[1], the per-tensor weight scale s_w
 *   out     bf16 [M][N2/2], row-major, 16-byte aligned
 * Computes s_x and x_q = e4m3(x / s_x) (one dynamic per-tensor scale,
 * s_x = max|x| / 448), y = s_x * s_w * x_q . W^T accumulated in fp32 on the
 * tensor cores, and out[m][j] = silu(y[m][j]) * y[m][F+j] rounded to bf16.
 * Supported: 1 <= M <= 64, K % 128 == 0, N2 % 256 == 0.
 * ------------------------------------------------------------------------- */
dl_status dl_fc13_swiglu(const uint16_t* x, int M, int K, const uint8_t* w_packed,
                         const float* w_scale, int N2, uint16_t* out, void* ws,
                         size_t ws_bytes, void* stream, unsigned flags);

/* ---------------------------------------------------------------------------
 * FC13 + SwiGLU without a caller workspace.  The source pages have no
 * counterpart of this entry point; it exists for callers that cannot allocate
 * device memory: a plugin that its host runtime hands only input and output
 * buffers, an engine that reserves its whole memory pool at start-up and
 * forbids later allocations, or a latency-critical loop where cudaMalloc or
 * cudaFree would synchronise the device.
 *
 * Same computation, arguments and requirements as dl_fc13_swiglu, except:
 *   - the activation scratch (e4m3 x_q and s_x) lives in one fixed device
 *     array inside libdl.so of 256 + 64*8192 bytes, held by every GPU that
 *     loads the library until the process exits.  M > 64 or M*K > 64*8192
 *     returns DL_ERR_WORKSPACE before anything is launched.
 *   - `status` is an optional device uint32 that the caller zeroes; device-
 *     side errors (bit 1 timeout) are OR-ed into it.  NULL turns device-side
 *     error reporting off for the call (a wait that runs out still ends the
 *     kernel; the output is then undefined and nothing says so).
 *   - nothing is allocated or freed: no cudaMalloc, cudaFree or allocating
 *     library routine is called.
 *   - the first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress, once per device, with that device current);
 *     make that first call before any stream capture.
 *   - every call shares the array and leaves its contents behind; calls that
 *     overlap on the GPU (concurrent streams or unordered host threads) race
 *     on it.  Calls queued in order on one stream, with or without
 *     DL_FLAG_PDL, are safe.
 * ------------------------------------------------------------------------- */
dl_status dl_fc13_swiglu_static_ws(const uint16_t* x, int M, int K, const uint8_t* w_packed,
                                   const float* w_scale, int N2, uint16_t* out, uint32_t* status,
                                   void* stream, unsigned flags);

/* ---------------------------------------------------------------------------
 * FC_QKV + attention scaling.  [XZY] "运算融合"; [NV] fusion list.
 *   w_packed e4m3, DL_PACK_PLAIN layout of the [(Hq+2*Hkv)*d][K] weight
 *   qkv     bf16 [M][(Hq+2*Hkv)*d], row-major: Q heads, then K heads, then V heads
 * y as above; the Q columns [0, Hq*d) are multiplied by q_scale (normally
 * 1/sqrt(d)), the K and V columns are not.  Supported: 1 <= M <= 64,
 * K % 128 == 0, (Hq+2*Hkv)*d % 128 == 0.
 * ------------------------------------------------------------------------- */
dl_status dl_fc_qkv_scale(const uint16_t* x, int M, int K, const uint8_t* w_packed,
                          const float* w_scale, int Hq, int Hkv, int d, float q_scale,
                          uint16_t* qkv, void* ws, size_t ws_bytes, void* stream,
                          unsigned flags);

/* ---------------------------------------------------------------------------
 * Grouped MoE expert FC13 + SwiGLU, top-1.  [XZY] FP8 for GEMM, MoE and
 * attention; [NV] "CUDA kernel optimisation and fusion" (MoE kernels).
 *   x          bf16 [T][K]
 *   expert_ids device int32[T], each in [0, E)
 *   w_packed   E consecutive DL_PACK_SWIGLU blocks of N2*K bytes (expert e at
 *              byte offset e*N2*K)
 *   w_scales   device float[E]
 *   out        bf16 [T][N2/2], rows in token order
 * One activation scale over all T tokens.  Token t uses expert expert_ids[t].
 * Only the experts that some token selects are read from memory.  Routing is
 * computed on the device from expert_ids (no host synchronisation).
 * Supported: 1 <= T <= 64, 1 <= E <= 1024, K % 128 == 0, N2 % 256 == 0.
 * ------------------------------------------------------------------------- */
dl_status dl_moe_fc13_swiglu_grouped(const uint16_t* x, int T, int K, const int32_t* expert_ids,
                                     int E, const uint8_t* w_packed, const float* w_scales,
                                     int N2, uint16_t* out, void* ws, size_t ws_bytes,
                                     void* stream, unsigned flags);

/* ---------------------------------------------------------------------------
 * Plain-epilogue FP8 projection: the attention output projection and the FC2
 * down projection of the layer.  [NV] "CUDA kernel optimisation and fusion"
 * (the layer's GEMMs are low-latency FP8 weight-streaming GEMMs); [XZY]
 * "CUDA 内核优化与融合" (FP8 GEMMs, Quantize fused ahead of them).
 *   x        bf16 [M][K] (may be NULL with DL_FLAG_XQ_READY)
 *   w_packed e4m3, DL_PACK_PLAIN layout of the [N][K] weight
 *   out      bf16 [M][N], row-major
 * out = bf16(s_x * s_w * x_q . W^T), accumulated in fp32 on the tensor cores,
 * with x_q, s_x as for dl_fc13_swiglu (or taken from the workspace with
 * DL_FLAG_XQ_READY).  Supported: 1 <= M <= 64, M*K <= 64*8192, K % 128 == 0,
 * N % 128 == 0.
 * ------------------------------------------------------------------------- */
dl_status dl_gemm_e4m3(const uint16_t* x, int M, int K, const uint8_t* w_packed,
                       const float* w_scale, int N, uint16_t* out, void* ws, size_t ws_bytes,
                       void* stream, unsigned flags);

/* ---------------------------------------------------------------------------
 * Grouped MoE expert projection with a plain epilogue (the expert FC2 down
 * projection), top-1.  Same routing, arguments and rules as
 * dl_moe_fc13_swiglu_grouped, with E consecutive DL_PACK_PLAIN blocks of N*K
 * bytes and out bf16 [T][N] in token order.  Supported: 1 <= T <= 64,
 * T*K <= 64*8192, 1 <= E <= 1024, K % 128 == 0, N % 128 == 0.
 * ------------------------------------------------------------------------- */
dl_status dl_moe_gemm_grouped(const uint16_t* x, int T, int K, const int32_t* expert_ids, int E,
                              const uint8_t* w_packed, const float* w_scales, int N,
                              uint16_t* out, void* ws, size_t ws_bytes, void* stream,
                              unsigned flags);

/* ---------------------------------------------------------------------------
 * Residual add + RMSNorm + Quantize, one kernel producing the FP8 input of the
 * next GEMM.  [XZY] "CUDA 内核优化与融合", item "运算融合", and [NV] "CUDA
 * kernel optimisation and fusion" fuse (AllReduce +) RMSNorm + Quantize; on
 * one GPU the AllReduce is absent and the residual add takes its place.
 *   x         bf16 [M][K], the sub-layer output (or the hidden state)
 *   residual  bf16 [M][K] or NULL
 *   h_out     bf16 [M][K] or NULL; receives h = bf16_rne(x + residual)
 *             (h = x when residual is NULL).  It may be x or residual itself
 *             (in-place update) but must not partially overlap either.
 *   gamma     bf16 [K], the RMSNorm gain
 *   eps       > 0
 *   ws        the workspace of the GEMM that consumes the result (at least
 *             dl_workspace_bytes(M, K)); x_q [M][K] and s_x are written there.
 * Per token row: y = (h * rsqrt(mean(h^2) + eps)) * gamma in fp32; then one
 * per-tensor scale s_x = max|y| / 448 and x_q = e4m3(y * (448 / max|y|)), as
 * in the GEMMs' own quantisation.  Run the consuming GEMM next on the same
 * stream with DL_FLAG_XQ_READY and the same ws: these two calls share the
 * workspace by design (under DL_FLAG_PDL the GEMM reads x_q only after it
 * waited for this kernel).
 * Supported: 1 <= M <= 64, M*K <= 64*8192, K % 128 == 0; pointers 16-byte
 * aligned.
 * ------------------------------------------------------------------------- */
dl_status dl_add_rmsnorm_quant(const uint16_t* x, const uint16_t* residual, uint16_t* h_out,
                               const uint16_t* gamma, int M, int K, float eps, void* ws,
                               size_t ws_bytes, void* stream, unsigned flags);

/* ---------------------------------------------------------------------------
 * Residual add + RMSNorm + Quantize, then the GEMM that consumes it, in one call.
 * [XZY] "运算融合" / [NV] fusion list: the (AllReduce +) RMSNorm + Quantize
 * producer of a GEMM input.  Exactly dl_add_rmsnorm_quant(x, residual, h_out,
 * gamma, M, K, eps, ws) followed by dl_fc_qkv_scale / dl_fc13_swiglu with
 * DL_FLAG_XQ_READY and the same ws: two kernels chained under DL_FLAG_PDL, so
 * the GEMM streams its weights while the producer runs.  (Computing the
 * producer inside every GEMM CTA instead was measured slower: each CTA re-reads
 * x, residual and gamma.)  h_out may be x or residual itself but must not
 * partially overlap either.  The remaining arguments are those of
 * dl_fc_qkv_scale / dl_fc13_swiglu; x is required.
 * ------------------------------------------------------------------------- */
dl_status dl_rmsnorm_fc_qkv_scale(const uint16_t* x, const uint16_t* residual, uint16_t* h_out,
                                  const uint16_t* gamma, float eps, int M, int K,
                                  const uint8_t* w_packed, const float* w_scale, int Hq, int Hkv,
                                  int d, float q_scale, uint16_t* qkv, void* ws, size_t ws_bytes,
                                  void* stream, unsigned flags);
dl_status dl_rmsnorm_fc13_swiglu(const uint16_t* x, const uint16_t* residual, uint16_t* h_out,
                                 const uint16_t* gamma, float eps, int M, int K,
                                 const uint8_t* w_packed, const float* w_scale, int N2, uint16_t* out,
                                 void* ws, size_t ws_bytes, void* stream, unsigned flags);

/* ---------------------------------------------------------------------------
 * Split-KV grouped-query decode attention with a cluster DSMEM merge.
 * [XZY] "CUDA 内核优化与融合", item "Attention内核并行优化"; [NV] "CUDA kernel
 * optimisation and fusion": the work is split along the sequence dimension of
 * K and V over several thread blocks, and the blocks of one thread-block
 * cluster reduce their partial results through distributed shared memory
 * instead of global memory.
 *   q         bf16, q[b][t][h][i] at q[(b*T + t)*q_token_stride + h*d + i]
 *             (q may point into the qkv output of dl_fc_qkv_scale, with
 *             q_token_stride = (Hq+2*Hkv)*d and softmax_scale = 1, since those
 *             Q columns are already scaled)
 *   k_cache, v_cache  bf16 [B][Hkv][Lcap][d], contiguous, 16-byte aligned
 *   seq_lens  device int32[B]; sequence b has L = seq_lens[b] keys, the last T
 *             of which are the new tokens: query t sees keys 0 .. L-T+t
 *             (bottom-right causal).  T <= L <= Lcap is required (checked on
 *             the device: DL_ERR_DEVICE_ARG from dl_read_status, output zero).
 *   out       bf16 [B][T][Hq][d], contiguous
 * o = softmax(softmax_scale * q K^T) V per (b, t, head); q head h reads kv
 * head h / (Hq/Hkv).  Each (b, kv head) is handled by one cluster of
 * cluster_size CTAs (1, 2, 4, 8 or 16); CTA r streams the r-th contiguous
 * chunk of ceil(L/cluster_size) keys (rounded up to 16).
 * When the workspace allows (dl_decode_attn_workspace_bytes), each (b, kv
 * head) may be split over several clusters of cluster_size CTAs; their
 * DSMEM-merged states are merged once more through the workspace.  The
 * DL_FLAG_SPLIT_SHIFT bits, when non-zero, force that number of clusters
 * (1..16).  ws must be zero-filled before its first use; every call leaves
 * its counters at zero again.
 * Supported: d in {64, 128}, Hq % Hkv == 0, (Hq/Hkv)*T <= 32, q_token_stride
 * a multiple of 8 and >= Hq*d.
 * ------------------------------------------------------------------------- */
dl_status dl_decode_attn(const uint16_t* q, long long q_token_stride, int B, int T, int Hq,
                         int Hkv, int d, const uint16_t* k_cache, const uint16_t* v_cache,
                         int Lcap, const int32_t* seq_lens, float softmax_scale,
                         int cluster_size, uint16_t* out, void* ws, size_t ws_bytes,
                         void* stream, unsigned flags);

/* ---------------------------------------------------------------------------
 * Split-KV decode attention over an FP8 (e4m3) KV cache.  [TC] and [XZY]
 * (section "CUDA 内核优化与融合" and the FP8 rationale): FP8 is used for
 * attention as well as for the GEMMs and MoE; it halves the KV bytes streamed.
 * Same computation, split, merge and rules as dl_decode_attn, except:
 *   k_cache   e4m3 bytes [B][Hkv][Lcap][d] (OCP E4M3 "e4m3fn"), holding k / s_k
 *   vt_cache  e4m3 bytes [B][Hkv][d][Lcap]: V stored transposed, holding v / s_v
 *             (key j, dim i of a head at i*Lcap + j)
 *   kv_scale  device float[2] = {s_k, s_v}, the per-tensor cache scales (a
 *             static input: read before the PDL wait)
 *   Lcap      a multiple of 16 (DL_ERR_ALIGNMENT otherwise)
 * o = softmax(softmax_scale * q (s_k K)^T) (s_v V).  The MMA operands are
 * converted to f16 in registers (exact for e4m3) and the products run in f16
 * with fp32 accumulation (q and the probabilities are rounded to f16).
 * Supported: d = 128, (Hq/Hkv)*T <= 32.  The workspace rules are those of
 * dl_decode_attn, sized by dl_decode_attn_fp8kv_workspace_bytes.
 * ------------------------------------------------------------------------- */
dl_status dl_decode_attn_fp8kv(const uint16_t* q, long long q_token_stride, int B, int T, int Hq,
                               int Hkv, int d, const uint8_t* k_cache, const uint8_t* vt_cache,
                               const float* kv_scale, int Lcap, const int32_t* seq_lens,
                               float softmax_scale, int cluster_size, uint16_t* out, void* ws,
                               size_t ws_bytes, void* stream, unsigned flags);

/* Workspace bytes for dl_decode_attn_fp8kv at these shapes (0 for invalid shapes). */
size_t dl_decode_attn_fp8kv_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int Lcap,
                                            int cluster_size);

/* ---------------------------------------------------------------------------
 * Greedy speculative verification, on the device.  [XZY] "推测解码" /
 * "端到端的工作流" (the target verifies the draft tokens of a step in parallel,
 * keeps those that match the token it would generate itself, and emits its own
 * token at the first mismatch) and "通过 CUDA Graph 和重叠调度器减少主机端开销"
 * (the verification stays on the device, inside the step's CUDA graph).
 *   logits     bf16 [B][T][V]: the target's outputs at the step's T input
 *              positions (the last accepted token, then the T-1 drafts); finite
 *   draft_ids  int32 [B][T-1]: the drafts fed at positions 1..T-1 (may be NULL
 *              when T == 1)
 *   target_ids int32 [B][T] out: argmax over V of each position (the lowest
 *              index wins a tie)
 *   n_accepted int32 [B] out: n = the number of leading drafts with
 *              draft_ids[b][i] == target_ids[b][i]
 *   emitted    int32 [B][T] out: target_ids[b][0..n], then -1: the n accepted
 *              drafts and the target's own next token (n + 1 tokens)
 *   seq_lens   int32 [B] or NULL: if given, decreased in place by T-1-n, so it
 *              again counts only the cache entries of accepted tokens (the
 *              caller's cache held all T inputs of this step)
 * No workspace; no device-side errors.  Under DL_FLAG_PDL the logits and draft
 * ids are read after the wait.  seq_lens is written here, so the next call that
 * reads it (dl_decode_attn) must not immediately follow this one under PDL.
 * Supported: 1 <= T <= 32, 1 <= B <= 65535, V % 8 == 0; logits 16-byte aligned.
 * ------------------------------------------------------------------------- */
dl_status dl_spec_verify_greedy(const uint16_t* logits, int B, int T, int V,
                                const int32_t* draft_ids, int32_t* target_ids,
                                int32_t* n_accepted, int32_t* emitted, int32_t* seq_lens,
                                void* stream, unsigned flags);

/* Workspace bytes for dl_decode_attn at these shapes.  When B*Hkv*cluster_size
 * CTAs would leave the GPU half idle, dl_decode_attn splits each (b, kv head)
 * over several clusters whose merged states meet in the workspace (the last
 * cluster to finish merges them and resets its counter); this returns the size
 * that allows the built-in choice.  A smaller workspace (down to 256 bytes)
 * is accepted and simply allows fewer clusters per head.  Returns 0 for
 * invalid shapes. */
size_t dl_decode_attn_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int Lcap,
                                      int cluster_size);

/* ---------------------------------------------------------------------------
 * A copy as a kernel, so that a step which fetches its activations from the
 * host (or returns its results there) stays one PDL chain.  [XZY]
 * "程序化依赖启动（PDL）" and [NV] "Programmatic Dependent Launch": the next
 * kernel's independent preamble (a GEMM's weight stream) overlaps the one
 * before it; a copy node of a CUDA graph is not a kernel and would break that.
 *   src, dst  device memory, or pinned host memory from cudaHostAlloc (which
 *             kernels address directly under unified addressing); 16-byte
 *             aligned, not overlapping
 *   bytes     a multiple of 16 (0 launches nothing)
 * With DL_FLAG_PDL the kernel waits for its predecessor before it reads src or
 * writes dst, unless DL_FLAG_COPY_NO_WAIT says that neither is touched by that
 * predecessor: then it runs beside it (an upload beside the previous step's
 * download uses both directions of the host link at once).  Host memory
 * written this way is visible to the host once the stream has been
 * synchronised.
 * ------------------------------------------------------------------------- */
dl_status dl_copy(const void* src, void* dst, size_t bytes, void* stream, unsigned flags);

/* Synchronises `stream`, reads the status word of `ws`, clears it, and returns
 * DL_OK, DL_ERR_TIMEOUT or DL_ERR_DEVICE_ARG (timeout takes precedence). */
dl_status dl_read_status(void* ws, void* stream);

/* A static, human-readable name of a status code. */
const char* dl_status_string(dl_status s);

#ifdef __cplusplus
}
#endif
#endif /* LATENCY_DECODE_DL_H */
