/*
 * oracle.h -- plain, slow CPU reference for the low-latency FP8 decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, calls or
 * includes this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark load the compiled oracle.  It shares no code, header, table
 * or constant generator with the CUDA path.
 *
 * Every routine takes the same canonical bytes the GPU receives (bf16 as raw
 * uint16, e4m3 as raw uint8, weights unpacked in nn.Linear [N][K] row-major
 * order) and accumulates in IEEE double.  Where the method itself fixes a
 * single-precision step (the activation scale 448/amax and the product x*inv
 * that feeds the e4m3 rounding), the oracle performs that step in float, so
 * that the integer e4m3 codes it produces are decided in the same precision as
 * on the device.
 *
 * Page references (titles and sections of the source pages):
 *   [NV]  "Blackwell breaks the 1,000 TPS/user barrier with Meta's Llama 4
 *         Maverick", NVIDIA technical blog (Korean edition).
 *   [XZY] Xinzhiyuan report on the same blog (Chinese), guosisoft.com.
 *   [TC]  tech-critter.com rewrite of the same blog (English).
 *
 * Parity status of every function is pinned by tests/test_oracle.py against
 * closed forms, invariants, library routines and brute force; see the header
 * comment of each function.
 */
#ifndef LATENCY_DECODE_ORACLE_H
#define LATENCY_DECODE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- number formats (format definitions, not the method) ---------------- */

/* bf16 bit pattern -> double (exact). */
double oracle_bf16_to_f64(uint16_t bits);
/* double -> bf16 bit pattern, round to nearest even, overflow to +-inf. */
uint16_t oracle_f64_to_bf16(double v);
/* OCP FP8 E4M3 ("e4m3fn": bias 7, no infinities, S.1111.111 = NaN) -> double. */
double oracle_e4m3_to_f64(uint8_t code);
/* float -> e4m3 code, round to nearest even, saturate finite values to +-448.
 * NaN input gives 0x7F.  The sign of zero is kept. */
uint8_t oracle_f32_to_e4m3(float v);

/* ---- A1: activation quantisation ---------------------------------------
 * [XZY] "CUDA 内核优化与融合" / "运算融合" and [NV] "CUDA kernel optimisation and
 * fusion": a Quantize step is fused ahead of the FP8 GEMM, so the GEMM sees
 * e4m3 activations.  Reading (design notes, open point 2): one dynamic
 * per-tensor scale over the whole [M][K] input:
 *   amax = max |x|;  inv = 448f / amax (float);  s_x = amax / 448f (float);
 *   xq   = e4m3_rne_sat((float)x * inv).
 * amax == 0 gives s_x = 1 and all-zero codes. */
void oracle_act_quant(const uint16_t* x, int M, int K, uint8_t* xq, float* s_x);

/* ---- A2/A5: FP8 GEMM ----------------------------------------------------
 * y[m][n] = s_x * s_w * sum_k dec(xq[m][k]) * dec(w[n][k]), all in double.
 * w is [N][K] row-major e4m3 (the nn.Linear layout). */
void oracle_gemm_q(const uint8_t* xq, float s_x, const uint8_t* w, float s_w,
                   int M, int N, int K, double* y);

/* ---- A5: FC13 + SwiGLU ([XZY] "运算融合"; [NV] kernel fusion list) ---------
 * w is [N2][K] with rows [0,F) the gate projection (FC1) and rows [F,2F) the
 * up projection (FC3), F = N2/2.  out[m][j] = silu(g) * u with
 * g = y[m][j], u = y[m][F+j], silu(g) = g / (1 + exp(-g)).  out is [M][F]. */
void oracle_fc13_swiglu_q(const uint8_t* xq, float s_x, const uint8_t* w, float s_w,
                          int M, int K, int N2, double* out);
void oracle_fc13_swiglu(const uint16_t* x, int M, int K, const uint8_t* w, float s_w,
                        int N2, double* out);

/* ---- A2: FC_QKV + attention scaling ([XZY] "运算融合"; [NV] fusion list) ----
 * Columns are [Q (Hq*d) | K (Hkv*d) | V (Hkv*d)]; the Q columns are multiplied
 * by q_scale, K and V columns are left as they are.  out is [M][(Hq+2Hkv)*d]. */
void oracle_fc_qkv_scale_q(const uint8_t* xq, float s_x, const uint8_t* w, float s_w,
                           int M, int K, int Hq, int Hkv, int d, float q_scale,
                           double* out);
void oracle_fc_qkv_scale(const uint16_t* x, int M, int K, const uint8_t* w, float s_w,
                         int Hq, int Hkv, int d, float q_scale, double* out);

/* ---- A6: MoE expert FC13 + SwiGLU, top-1 ([XZY] FP8 for GEMM/MoE/Attention) -
 * One activation scale over all T tokens; token t uses expert ids[t] with its
 * weight block w + ids[t]*N2*K and scale s_w[ids[t]].  Output rows stay in
 * token order.  out is [T][N2/2]. */
void oracle_moe_fc13_swiglu(const uint16_t* x, int T, int K, const int32_t* ids, int E,
                            const uint8_t* w, const float* s_w, int N2, double* out);

/* ---- Plain-epilogue projections (attention output projection, FC2 down
 * projection): [NV] "CUDA kernel optimisation and fusion" lists the layer's
 * GEMMs as FP8 weight-streaming GEMMs; without a fused epilogue the output is
 * y itself.  oracle_linear: out[m][n] = y[m][n] of act_quant(x) and w [N][K].
 * oracle_moe_linear: one activation scale over all T tokens, token t uses
 * expert ids[t] (block w + ids[t]*N*K, scale s_w[ids[t]]); out is [T][N] in
 * token order, a NaN row for an id outside [0, E). */
void oracle_linear(const uint16_t* x, int M, int K, const uint8_t* w, float s_w, int N,
                   double* out);
void oracle_moe_linear(const uint16_t* x, int T, int K, const int32_t* ids, int E,
                       const uint8_t* w, const float* s_w, int N, double* out);

/* ---- Residual add + RMSNorm, the producer of the next GEMM's input ---------
 * [XZY] "CUDA 内核优化与融合" / "运算融合" and [NV] "CUDA kernel optimisation and
 * fusion" fuse (AllReduce +) RMSNorm + Quantize into one kernel ahead of the
 * FP8 GEMM; on one GPU the AllReduce is absent and the residual add remains.
 * Readings (the pages give no formula): the residual stream is bf16, so
 *   h = bf16_rne(x + r)   (h = x when r is NULL), written to h_out;
 *   y[m][k] = h[m][k] / sqrt(mean_k h[m][k]^2 + eps) * gamma[k]   (double).
 * The Quantize step then takes y in the kernel's precision: oracle_quant_f32
 * of (float)y. */
void oracle_add_rmsnorm(const uint16_t* x, const uint16_t* r, const uint16_t* gamma, int M,
                        int K, float eps, uint16_t* h_out, double* y);
/* Per-tensor dynamic quantisation of float values, the rule of oracle_act_quant
 * applied to fp32 inputs: amax = max|y|, inv = 448f/amax, s_x = amax/448f,
 * xq = e4m3_rne_sat(y * inv) (one float rounding for the product). */
void oracle_quant_f32(const float* y, long long n, uint8_t* xq, float* s_x);

/* ---- Greedy speculative verification on the device ([XZY] "推测解码",
 * "端到端的工作流" and "通过 CUDA Graph 和重叠调度器减少主机端开销"; [NV]
 * speculative-decoding section) ----------------------------------------------
 * The target step reads T inputs per sequence: the last accepted token, then
 * the T-1 draft tokens draft[b][0..T-2].  logits [B][T][V] (bf16) are the
 * target's outputs at those positions.  Readings: the token the target itself
 * would generate is the greedy argmax (lowest index on a tie); draft[b][i] is
 * accepted while it equals target_ids[b][i] for every earlier i; at the first
 * mismatch the target's own token is emitted instead, and with no mismatch the
 * token after the last draft is emitted as well.
 *   target_ids [B][T]; n_accepted[b] = accepted drafts (0..T-1);
 *   emitted [B][T] = target_ids[b][0..n] followed by -1 (n + 1 tokens). */
void oracle_spec_verify_greedy(const uint16_t* logits, int B, int T, int V, const int32_t* draft,
                               int32_t* target_ids, int32_t* n_accepted, int32_t* emitted);

/* ---- A3: grouped-query decode attention, computed unsplit ----------------
 * [XZY] "Attention内核并行优化"; [NV] "CUDA kernel optimisation and fusion".
 * q[b][t][h][i] sits at q[(b*T + t)*q_stride + h*d + i]; K and V caches are
 * [B][Hkv][Lcap][d].  q head h reads kv head h / (Hq/Hkv).  With L = seq_lens[b],
 * query t (0-based among the T new tokens) sees keys 0 .. L-T+t (bottom-right
 * causal alignment).  s_j = scale * <q, k_j>; o = sum_j softmax(s)_j v_j.
 * out is [B][T][Hq][d]. */
void oracle_decode_attn(const uint16_t* q, long long q_stride, int B, int T, int Hq,
                        int Hkv, int d, const uint16_t* k, const uint16_t* v, int Lcap,
                        const int32_t* seq_lens, float scale, double* out);

/* ---- A3 with an FP8 KV cache ([TC] and [XZY]: FP8 is used for attention as
 * well as for the GEMMs and MoE).  Reading: the cache holds e4m3 codes with one
 * per-tensor scale each for K and V, k = s_k * e4m3(code), v = s_v * e4m3(code);
 * q stays bf16.  k is [B][Hkv][Lcap][d] bytes as in oracle_decode_attn; the V
 * cache is stored transposed, v_t [B][Hkv][d][Lcap] (key j, dim i at
 * i*Lcap + j).  Otherwise exactly oracle_decode_attn (GQA map, bottom-right
 * causal rule). */
void oracle_decode_attn_fp8kv(const uint16_t* q, long long q_stride, int B, int T, int Hq, int Hkv,
                              int d, const uint8_t* k, const uint8_t* v_t, int Lcap,
                              const int32_t* seq_lens, float scale, float s_k, float s_v,
                              double* out);

/* Partial softmax state of one (b, q head, query t) over the visible keys that
 * fall in [key_lo, key_hi): m = max logit (-inf if none), l = sum exp(s - m),
 * o = sum exp(s - m) v (unnormalised, length d).  Used only to check the
 * log-sum-exp merge identity of A4. */
void oracle_attn_partial(const uint16_t* q, long long q_stride, int T, int Hq, int Hkv,
                         int d, const uint16_t* k, const uint16_t* v, int Lcap,
                         int b, int t, int h, int L, float scale, int key_lo, int key_hi,
                         double* m, double* l, double* o);

/* ---- A4: log-sum-exp merge of S partial states ([XZY] cluster / distributed
 * shared memory reduction of the per-block results).
 *   M* = max_i m_i;  L* = sum_i l_i e^(m_i - M*);  o = sum_i o_i e^(m_i - M*) / L*.
 * Partials with l_i == 0 carry no weight.  o_parts is [S][d]. */
void oracle_lse_combine(int S, const double* m, const double* l, const double* o_parts,
                        int d, double* out);

#ifdef __cplusplus
}
#endif
#endif
