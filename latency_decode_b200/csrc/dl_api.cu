// dl_api.cu -- the C ABI of libdl.so (include/dl.h): argument validation, the
// launch sequence of each entry point, and the status word.
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "dl_device.cuh"
#include "dl_internal.h"

namespace dl {

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev < 64) cached[dev] = n;
  return n;
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return dev;
}

namespace {
std::mutex g_attr_mu;
std::map<std::pair<int, const void*>, std::pair<int, bool>> g_attrs;  // (device, kernel) -> (smem, nonportable)
std::mutex g_memo_mu;
std::map<std::pair<int, unsigned long long>, int> g_memo;
}  // namespace

cudaError_t ensure_kernel_attrs(const void* func, int smem_bytes, bool nonportable_cluster) {
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(g_attr_mu);
  auto& slot = g_attrs[{dev, func}];
  if (smem_bytes > slot.first) {
    cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    slot.first = smem_bytes;
  }
  if (nonportable_cluster && !slot.second) {
    cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    slot.second = true;
  }
  return cudaSuccess;
}

int memo_int(unsigned long long key, int (*fn)(const void*), const void* ctx) {
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lock(g_memo_mu);
    auto it = g_memo.find({dev, key});
    if (it != g_memo.end()) return it->second;
  }
  const int v = fn(ctx);  // computed outside the lock (it may call ensure_kernel_attrs)
  std::lock_guard<std::mutex> lock(g_memo_mu);
  g_memo[{dev, key}] = v;
  return v;
}

}  // namespace dl

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

dl_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return DL_OK;
  (void)cudaGetLastError();  // clear a sticky launch-configuration error
  return DL_ERR_CUDA;
}

dl_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < need) return DL_ERR_WORKSPACE;
  return DL_OK;
}

// x may be null when DL_FLAG_XQ_READY says the workspace already holds x_q.
dl_status check_gemm_common(const uint16_t* x, int M, int K, const uint8_t* w, const float* w_scale,
                            const void* out, unsigned flags) {
  const bool xq_ready = (flags & DL_FLAG_XQ_READY) != 0;
  if ((x == nullptr && !xq_ready) || w == nullptr || w_scale == nullptr || out == nullptr) return DL_ERR_INVALID_ARG;
  if (M < 1 || K < 128) return DL_ERR_INVALID_ARG;
  if (K % 128 != 0) return DL_ERR_UNSUPPORTED;
  if (M > 64) return DL_ERR_UNSUPPORTED;
  if (static_cast<long long>(M) * K > 64ll * 8192) return DL_ERR_UNSUPPORTED;
  if (!aligned(x, 16) || !aligned(w, 16) || !aligned(out, 16) || !aligned(w_scale, 4)) return DL_ERR_ALIGNMENT;
  return DL_OK;
}

unsigned forced_split(unsigned flags) { return (flags >> DL_FLAG_SPLIT_SHIFT) & 31u; }

}  // namespace

extern "C" {

size_t dl_workspace_bytes(int M, int K) {
  if (M < 0 || K < 0) return 0;
  const size_t q = static_cast<size_t>(M) * static_cast<size_t>(K);
  return dl::kWsHeader + ((q + 255) / 256) * 256;
}

static size_t attn_ws_for(int B, int T, int Hq, int Hkv, int d, int Lcap, int cluster_size, bool fp8) {
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || d < 1 || Lcap < 1 || cluster_size < 1 || Hq % Hkv != 0) return 0;
  if (d != 128 && (fp8 || d != 64)) return 0;
  const int P = dl::attn_auto_splits(B, Hkv, cluster_size, Lcap, d, (Hq / Hkv) * T, fp8);
  return dl::attn_ws_bytes(B, Hkv, (Hq / Hkv) * T, d, P, cluster_size);
}

size_t dl_decode_attn_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int Lcap, int cluster_size) {
  return attn_ws_for(B, T, Hq, Hkv, d, Lcap, cluster_size, false);
}

size_t dl_decode_attn_fp8kv_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int Lcap, int cluster_size) {
  return attn_ws_for(B, T, Hq, Hkv, d, Lcap, cluster_size, true);
}

dl_status dl_pack_fp8_weight(const uint8_t* w_nk, uint8_t* w_packed, int N, int K, int kind,
                             void* stream) {
  if (w_nk == nullptr || w_packed == nullptr || N < 1 || K < 1) return DL_ERR_INVALID_ARG;
  if (kind != DL_PACK_PLAIN && kind != DL_PACK_SWIGLU) return DL_ERR_INVALID_ARG;
  if (K % 128 != 0) return DL_ERR_UNSUPPORTED;
  if (N % (kind == DL_PACK_SWIGLU ? 256 : 128) != 0) return DL_ERR_UNSUPPORTED;
  if (!aligned(w_nk, 16) || !aligned(w_packed, 16)) return DL_ERR_ALIGNMENT;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(w_nk), b0 = reinterpret_cast<uintptr_t>(w_packed);
  const uintptr_t bytes = static_cast<uintptr_t>(N) * static_cast<uintptr_t>(K);
  if (a0 < b0 + bytes && b0 < a0 + bytes) return DL_ERR_INVALID_ARG;  // overlap
  return cuda_status(dl::launch_pack(w_nk, w_packed, N, K, kind, static_cast<cudaStream_t>(stream)));
}

struct NormSpec {  // residual add + RMSNorm ahead of the GEMM (gamma == null: none)
  const uint16_t* residual = nullptr;
  uint16_t* h_out = nullptr;
  const uint16_t* gamma = nullptr;
  float eps = 0.0f;
};

static dl_status run_dense_gemm(const uint16_t* x, int M, int K, const uint8_t* w_packed, const float* w_scale,
                                int N, bool swiglu, int q_cols, float q_scale, uint16_t* out, void* ws,
                                void* stream, unsigned flags, const NormSpec& norm = NormSpec()) {
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool pdl = (flags & DL_FLAG_PDL) != 0;
  if (norm.gamma != nullptr) {
    // The producer of the input as its own kernel, PDL-chained ahead of the GEMM
    // (computing it inside every GEMM CTA measured slower: each re-reads x, r and gamma).
    cudaError_t e = dl::launch_add_rmsnorm_quant(x, norm.residual, norm.h_out, norm.gamma, M, K, norm.eps,
                                                 dl::ws_xq(ws), dl::ws_sx(ws), s, pdl);
    if (e != cudaSuccess) return cuda_status(e);
    flags |= DL_FLAG_XQ_READY;
  }
  // Small inputs are quantised inside the GEMM (one launch); larger ones by the
  // cluster quantise kernel first.  Both write x_q and s_x to the workspace.
  // With DL_FLAG_XQ_READY a producer kernel (dl_add_rmsnorm_quant) has
  // already written them there.
  const bool xq_ready = (flags & DL_FLAG_XQ_READY) != 0;
  const bool fused = !xq_ready && static_cast<long long>(M) * K <= dl::kFusedQuantMaxElems;
  if (!fused && !xq_ready) {
    cudaError_t e = dl::launch_act_quant(x, M, K, dl::ws_xq(ws), dl::ws_sx(ws), s, pdl);
    if (e != cudaSuccess) return cuda_status(e);
  }
  dl::GemmLaunch g{};
  g.x = fused ? x : nullptr;
  g.w = w_packed;
  g.w_expert_bytes = 0;
  g.w_scale = w_scale;
  g.xq = dl::ws_xq(ws);
  g.s_x = dl::ws_sx(ws);
  g.status = dl::ws_status(ws);
  g.out = out;
  g.expert_ids = nullptr;
  g.M = M;
  g.K = K;
  g.N = N;
  g.ldo = swiglu ? N / 2 : N;
  g.E = 1;
  g.q_cols = q_cols;
  g.q_scale = q_scale;
  g.swiglu = swiglu;
  g.slots = 1;
  g.split = static_cast<int>(forced_split(flags));
  g.debug = (flags & DL_FLAG_DEBUG_TIMEOUT) != 0;
  g.pdl = pdl;
  return cuda_status(dl::launch_gemm(g, s));
}

dl_status dl_fc13_swiglu(const uint16_t* x, int M, int K, const uint8_t* w_packed, const float* w_scale, int N2,
                         uint16_t* out, void* ws, size_t ws_bytes, void* stream, unsigned flags) {
  dl_status st = check_gemm_common(x, M, K, w_packed, w_scale, out, flags);
  if (st != DL_OK) return st;
  if (N2 < 256) return DL_ERR_INVALID_ARG;
  if (N2 % 256 != 0) return DL_ERR_UNSUPPORTED;
  if (forced_split(flags) > 8) return DL_ERR_INVALID_ARG;
  st = check_ws(ws, ws_bytes, dl_workspace_bytes(M, K));
  if (st != DL_OK) return st;
  return run_dense_gemm(x, M, K, w_packed, w_scale, N2, true, 0, 1.0f, out, ws, stream, flags);
}

dl_status dl_fc_qkv_scale(const uint16_t* x, int M, int K, const uint8_t* w_packed, const float* w_scale, int Hq,
                          int Hkv, int d, float q_scale, uint16_t* qkv, void* ws, size_t ws_bytes, void* stream,
                          unsigned flags) {
  dl_status st = check_gemm_common(x, M, K, w_packed, w_scale, qkv, flags);
  if (st != DL_OK) return st;
  if (Hq < 1 || Hkv < 0 || d < 1) return DL_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(Hq + 2 * Hkv) * d;
  if (N % 128 != 0 || N > (1ll << 24)) return DL_ERR_UNSUPPORTED;
  if (forced_split(flags) > 8) return DL_ERR_INVALID_ARG;
  st = check_ws(ws, ws_bytes, dl_workspace_bytes(M, K));
  if (st != DL_OK) return st;
  return run_dense_gemm(x, M, K, w_packed, w_scale, static_cast<int>(N), false, Hq * d, q_scale, qkv, ws, stream,
                        flags);
}

static dl_status run_moe_gemm(const uint16_t* x, int T, int K, const int32_t* expert_ids, int E,
                              const uint8_t* w_packed, const float* w_scales, int N, bool swiglu, uint16_t* out,
                              void* ws, size_t ws_bytes, void* stream, unsigned flags) {
  dl_status st = check_gemm_common(x, T, K, w_packed, w_scales, out, flags);
  if (st != DL_OK) return st;
  const int granule = swiglu ? 256 : 128;
  if (expert_ids == nullptr || E < 1 || N < granule) return DL_ERR_INVALID_ARG;
  if (E > 1024 || N % granule != 0) return DL_ERR_UNSUPPORTED;
  if (!aligned(expert_ids, 4)) return DL_ERR_ALIGNMENT;
  if (forced_split(flags) > 8) return DL_ERR_INVALID_ARG;
  st = check_ws(ws, ws_bytes, dl_workspace_bytes(T, K));
  if (st != DL_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool pdl = (flags & DL_FLAG_PDL) != 0;
  if ((flags & DL_FLAG_XQ_READY) == 0) {
    cudaError_t e = dl::launch_act_quant(x, T, K, dl::ws_xq(ws), dl::ws_sx(ws), s, pdl);
    if (e != cudaSuccess) return cuda_status(e);
  }
  dl::GemmLaunch g{};
  g.w = w_packed;
  g.w_expert_bytes = static_cast<long long>(N) * K;
  g.w_scale = w_scales;
  g.xq = dl::ws_xq(ws);
  g.s_x = dl::ws_sx(ws);
  g.status = dl::ws_status(ws);
  g.out = out;
  g.expert_ids = expert_ids;
  g.M = T;
  g.K = K;
  g.N = N;
  g.ldo = swiglu ? N / 2 : N;
  g.E = E;
  g.q_cols = 0;
  g.q_scale = 1.0f;
  g.swiglu = swiglu;
  g.slots = T < E ? T : E;
  g.split = static_cast<int>(forced_split(flags));
  g.debug = (flags & DL_FLAG_DEBUG_TIMEOUT) != 0;
  g.pdl = pdl;
  return cuda_status(dl::launch_gemm(g, s));
}

dl_status dl_moe_fc13_swiglu_grouped(const uint16_t* x, int T, int K, const int32_t* expert_ids, int E,
                                     const uint8_t* w_packed, const float* w_scales, int N2, uint16_t* out,
                                     void* ws, size_t ws_bytes, void* stream, unsigned flags) {
  return run_moe_gemm(x, T, K, expert_ids, E, w_packed, w_scales, N2, true, out, ws, ws_bytes, stream, flags);
}

dl_status dl_moe_gemm_grouped(const uint16_t* x, int T, int K, const int32_t* expert_ids, int E,
                              const uint8_t* w_packed, const float* w_scales, int N, uint16_t* out, void* ws,
                              size_t ws_bytes, void* stream, unsigned flags) {
  return run_moe_gemm(x, T, K, expert_ids, E, w_packed, w_scales, N, false, out, ws, ws_bytes, stream, flags);
}

dl_status dl_gemm_e4m3(const uint16_t* x, int M, int K, const uint8_t* w_packed, const float* w_scale, int N,
                       uint16_t* out, void* ws, size_t ws_bytes, void* stream, unsigned flags) {
  dl_status st = check_gemm_common(x, M, K, w_packed, w_scale, out, flags);
  if (st != DL_OK) return st;
  if (N < 128) return DL_ERR_INVALID_ARG;
  if (N % 128 != 0) return DL_ERR_UNSUPPORTED;
  if (forced_split(flags) > 8) return DL_ERR_INVALID_ARG;
  st = check_ws(ws, ws_bytes, dl_workspace_bytes(M, K));
  if (st != DL_OK) return st;
  return run_dense_gemm(x, M, K, w_packed, w_scale, N, false, 0, 1.0f, out, ws, stream, flags);
}

static dl_status check_norm_spec(const uint16_t* x, const uint16_t* residual, const uint16_t* h_out,
                                 const uint16_t* gamma, int M, int K, float eps) {
  if (x == nullptr || gamma == nullptr) return DL_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || !(eps < 3.0e38f)) return DL_ERR_INVALID_ARG;
  if (M > 64 || static_cast<long long>(M) * K > 64ll * 8192) return DL_ERR_UNSUPPORTED;
  if (!aligned(residual, 16) || !aligned(h_out, 16) || !aligned(gamma, 16)) return DL_ERR_ALIGNMENT;
  // h_out may be x or residual itself (in-place update), but no partial overlap
  const uintptr_t bytes = static_cast<uintptr_t>(M) * static_cast<uintptr_t>(K) * 2u;
  if (h_out != nullptr) {
    const uintptr_t hb = reinterpret_cast<uintptr_t>(h_out);
    for (const void* p : {static_cast<const void*>(x), static_cast<const void*>(residual)}) {
      const uintptr_t pb = reinterpret_cast<uintptr_t>(p);
      if (p != nullptr && pb != hb && pb < hb + bytes && hb < pb + bytes) return DL_ERR_INVALID_ARG;
    }
  }
  return DL_OK;
}

dl_status dl_rmsnorm_fc_qkv_scale(const uint16_t* x, const uint16_t* residual, uint16_t* h_out,
                                  const uint16_t* gamma, float eps, int M, int K, const uint8_t* w_packed,
                                  const float* w_scale, int Hq, int Hkv, int d, float q_scale, uint16_t* qkv,
                                  void* ws, size_t ws_bytes, void* stream, unsigned flags) {
  flags &= ~DL_FLAG_XQ_READY;
  dl_status st = check_gemm_common(x, M, K, w_packed, w_scale, qkv, flags);
  if (st != DL_OK) return st;
  st = check_norm_spec(x, residual, h_out, gamma, M, K, eps);
  if (st != DL_OK) return st;
  if (Hq < 1 || Hkv < 0 || d < 1) return DL_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(Hq + 2 * Hkv) * d;
  if (N % 128 != 0 || N > (1ll << 24)) return DL_ERR_UNSUPPORTED;
  if (forced_split(flags) > 8) return DL_ERR_INVALID_ARG;
  st = check_ws(ws, ws_bytes, dl_workspace_bytes(M, K));
  if (st != DL_OK) return st;
  NormSpec ns;
  ns.residual = residual;
  ns.h_out = h_out;
  ns.gamma = gamma;
  ns.eps = eps;
  return run_dense_gemm(x, M, K, w_packed, w_scale, static_cast<int>(N), false, Hq * d, q_scale, qkv, ws, stream,
                        flags, ns);
}

dl_status dl_rmsnorm_fc13_swiglu(const uint16_t* x, const uint16_t* residual, uint16_t* h_out,
                                 const uint16_t* gamma, float eps, int M, int K, const uint8_t* w_packed,
                                 const float* w_scale, int N2, uint16_t* out, void* ws, size_t ws_bytes,
                                 void* stream, unsigned flags) {
  flags &= ~DL_FLAG_XQ_READY;
  dl_status st = check_gemm_common(x, M, K, w_packed, w_scale, out, flags);
  if (st != DL_OK) return st;
  st = check_norm_spec(x, residual, h_out, gamma, M, K, eps);
  if (st != DL_OK) return st;
  if (N2 < 256) return DL_ERR_INVALID_ARG;
  if (N2 % 256 != 0) return DL_ERR_UNSUPPORTED;
  if (forced_split(flags) > 8) return DL_ERR_INVALID_ARG;
  st = check_ws(ws, ws_bytes, dl_workspace_bytes(M, K));
  if (st != DL_OK) return st;
  NormSpec ns;
  ns.residual = residual;
  ns.h_out = h_out;
  ns.gamma = gamma;
  ns.eps = eps;
  return run_dense_gemm(x, M, K, w_packed, w_scale, N2, true, 0, 1.0f, out, ws, stream, flags, ns);
}

dl_status dl_add_rmsnorm_quant(const uint16_t* x, const uint16_t* residual, uint16_t* h_out, const uint16_t* gamma,
                               int M, int K, float eps, void* ws, size_t ws_bytes, void* stream, unsigned flags) {
  if (x == nullptr || gamma == nullptr) return DL_ERR_INVALID_ARG;
  if (M < 1 || K < 128 || !(eps > 0.0f) || !(eps < 3.0e38f)) return DL_ERR_INVALID_ARG;
  if (K % 128 != 0 || M > 64 || static_cast<long long>(M) * K > 64ll * 8192) return DL_ERR_UNSUPPORTED;
  if (!aligned(x, 16) || !aligned(residual, 16) || !aligned(h_out, 16) || !aligned(gamma, 16))
    return DL_ERR_ALIGNMENT;
  // h_out may be x or residual itself (in-place update), but no partial overlap
  const uintptr_t bytes = static_cast<uintptr_t>(M) * static_cast<uintptr_t>(K) * 2u;
  if (h_out != nullptr) {
    const uintptr_t hb = reinterpret_cast<uintptr_t>(h_out);
    for (const void* p : {static_cast<const void*>(x), static_cast<const void*>(residual)}) {
      const uintptr_t pb = reinterpret_cast<uintptr_t>(p);
      if (p != nullptr && pb != hb && pb < hb + bytes && hb < pb + bytes) return DL_ERR_INVALID_ARG;
    }
  }
  dl_status st = check_ws(ws, ws_bytes, dl_workspace_bytes(M, K));
  if (st != DL_OK) return st;
  return cuda_status(dl::launch_add_rmsnorm_quant(x, residual, h_out, gamma, M, K, eps, dl::ws_xq(ws),
                                                  dl::ws_sx(ws), static_cast<cudaStream_t>(stream),
                                                  (flags & DL_FLAG_PDL) != 0));
}

dl_status dl_spec_verify_greedy(const uint16_t* logits, int B, int T, int V, const int32_t* draft_ids,
                                int32_t* target_ids, int32_t* n_accepted, int32_t* emitted, int32_t* seq_lens,
                                void* stream, unsigned flags) {
  if (logits == nullptr || target_ids == nullptr || n_accepted == nullptr || emitted == nullptr)
    return DL_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || V < 8) return DL_ERR_INVALID_ARG;
  if (T > 1 && draft_ids == nullptr) return DL_ERR_INVALID_ARG;
  if (T > 32 || B > 65535 || V % 8 != 0) return DL_ERR_UNSUPPORTED;
  if (!aligned(logits, 16) || !aligned(draft_ids, 4) || !aligned(target_ids, 4) || !aligned(n_accepted, 4) ||
      !aligned(emitted, 4) || !aligned(seq_lens, 4))
    return DL_ERR_ALIGNMENT;
  return cuda_status(dl::launch_spec_verify(logits, B, T, V, draft_ids, target_ids, n_accepted, emitted, seq_lens,
                                            static_cast<cudaStream_t>(stream), (flags & DL_FLAG_PDL) != 0));
}

static dl_status run_attn(const uint16_t* q, long long q_token_stride, int B, int T, int Hq, int Hkv, int d,
                          const void* k_cache, const void* v_cache, bool fp8, const float* kv_scale, int Lcap,
                          const int32_t* seq_lens, float softmax_scale, int cluster_size, uint16_t* out, void* ws,
                          size_t ws_bytes, void* stream, unsigned flags) {
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || seq_lens == nullptr || out == nullptr)
    return DL_ERR_INVALID_ARG;
  if (fp8 && kv_scale == nullptr) return DL_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Lcap < 1 || d < 1) return DL_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return DL_ERR_INVALID_ARG;
  if (d != 128 && (fp8 || d != 64)) return DL_ERR_UNSUPPORTED;
  if ((Hq / Hkv) * T > 32) return DL_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return DL_ERR_UNSUPPORTED;
  if (cluster_size != 1 && cluster_size != 2 && cluster_size != 4 && cluster_size != 8 && cluster_size != 16)
    return DL_ERR_INVALID_ARG;
  if (q_token_stride < static_cast<long long>(Hq) * d || q_token_stride % 8 != 0) return DL_ERR_ALIGNMENT;
  if (forced_split(flags) > 16) return DL_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(seq_lens, 4) || !aligned(kv_scale, 4))
    return DL_ERR_ALIGNMENT;
  if (fp8 && Lcap % 16 != 0) return DL_ERR_ALIGNMENT;  // the V^T rows (Lcap bytes) are a TMA stride
  dl_status st = check_ws(ws, ws_bytes, dl_workspace_bytes(0, 0));
  if (st != DL_OK) return st;
  dl::AttnLaunch a{};
  a.q = q;
  a.q_stride = q_token_stride;
  a.B = B;
  a.T = T;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.Lcap = Lcap;
  a.k = k_cache;
  a.v = v_cache;
  a.fp8 = fp8;
  a.kv_scale = kv_scale;
  a.seq_lens = seq_lens;
  a.scale = softmax_scale;
  a.cluster = cluster_size;
  a.splits = static_cast<int>(forced_split(flags));
  a.ws_bytes = ws_bytes;
  a.out = out;
  a.status = dl::ws_status(ws);
  a.debug = (flags & DL_FLAG_DEBUG_TIMEOUT) != 0;
  a.pdl = (flags & DL_FLAG_PDL) != 0;
  return cuda_status(dl::launch_attn(a, static_cast<cudaStream_t>(stream)));
}

dl_status dl_decode_attn(const uint16_t* q, long long q_token_stride, int B, int T, int Hq, int Hkv, int d,
                         const uint16_t* k_cache, const uint16_t* v_cache, int Lcap, const int32_t* seq_lens,
                         float softmax_scale, int cluster_size, uint16_t* out, void* ws, size_t ws_bytes,
                         void* stream, unsigned flags) {
  return run_attn(q, q_token_stride, B, T, Hq, Hkv, d, k_cache, v_cache, false, nullptr, Lcap, seq_lens,
                  softmax_scale, cluster_size, out, ws, ws_bytes, stream, flags);
}

dl_status dl_decode_attn_fp8kv(const uint16_t* q, long long q_token_stride, int B, int T, int Hq, int Hkv, int d,
                               const uint8_t* k_cache, const uint8_t* vt_cache, const float* kv_scale, int Lcap,
                               const int32_t* seq_lens, float softmax_scale, int cluster_size, uint16_t* out,
                               void* ws, size_t ws_bytes, void* stream, unsigned flags) {
  return run_attn(q, q_token_stride, B, T, Hq, Hkv, d, k_cache, vt_cache, true, kv_scale, Lcap, seq_lens,
                  softmax_scale, cluster_size, out, ws, ws_bytes, stream, flags);
}

dl_status dl_copy(const void* src, void* dst, size_t bytes, void* stream, unsigned flags) {
  if (src == nullptr || dst == nullptr) return DL_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(dst, 16) || bytes % 16 != 0) return DL_ERR_ALIGNMENT;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(src), b0 = reinterpret_cast<uintptr_t>(dst);
  if (bytes > 0 && a0 < b0 + bytes && b0 < a0 + bytes) return DL_ERR_INVALID_ARG;  // overlap
  return cuda_status(dl::launch_copy(src, dst, bytes, static_cast<cudaStream_t>(stream), (flags & DL_FLAG_PDL) != 0,
                                     (flags & DL_FLAG_COPY_NO_WAIT) == 0));
}

dl_status dl_read_status(void* ws, void* stream) {
  if (ws == nullptr || !aligned(ws, 256)) return DL_ERR_WORKSPACE;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && word != 0) {
    e = cudaMemsetAsync(ws, 0, sizeof(word), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return cuda_status(e);
  if (word & dl::kStatusTimeout) return DL_ERR_TIMEOUT;
  if (word & (dl::kStatusBadSeqLen | dl::kStatusBadExpert)) return DL_ERR_DEVICE_ARG;
  return DL_OK;
}

const char* dl_status_string(dl_status s) {
  switch (s) {
    case DL_OK: return "DL_OK";
    case DL_ERR_INVALID_ARG: return "DL_ERR_INVALID_ARG";
    case DL_ERR_UNSUPPORTED: return "DL_ERR_UNSUPPORTED";
    case DL_ERR_ALIGNMENT: return "DL_ERR_ALIGNMENT";
    case DL_ERR_WORKSPACE: return "DL_ERR_WORKSPACE";
    case DL_ERR_CUDA: return "DL_ERR_CUDA";
    case DL_ERR_TIMEOUT: return "DL_ERR_TIMEOUT";
    case DL_ERR_DEVICE_ARG: return "DL_ERR_DEVICE_ARG";
  }
  return "DL_ERR_UNKNOWN";
}

}  // extern "C"
