// dl_api.cu -- the C ABI of libdl.so (include/dl.h): argument validation, the
// launch sequence of each entry point, and the status word.
#include <cstdio>
#include <cstring>

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

dl_status check_gemm_common(const uint16_t* x, int M, int K, const uint8_t* w, const float* w_scale,
                            const void* out) {
  if (x == nullptr || w == nullptr || w_scale == nullptr || out == nullptr) return DL_ERR_INVALID_ARG;
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

size_t dl_decode_attn_workspace_bytes(int B, int T, int Hq, int Hkv, int d, int Lcap, int cluster_size) {
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || d < 1 || Lcap < 1 || cluster_size < 1 || Hq % Hkv != 0) return 0;
  if (d != 64 && d != 128) return 0;
  const int P = dl::attn_auto_splits(B, Hkv, cluster_size, Lcap, d, (Hq / Hkv) * T);
  return dl::attn_ws_bytes(B, Hkv, (Hq / Hkv) * T, d, P, cluster_size);
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

static dl_status run_dense_gemm(const uint16_t* x, int M, int K, const uint8_t* w_packed, const float* w_scale,
                                int N, bool swiglu, int q_cols, float q_scale, uint16_t* out, void* ws,
                                void* stream, unsigned flags) {
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool pdl = (flags & DL_FLAG_PDL) != 0;
  // Small inputs are quantised inside the GEMM (one launch); larger ones by the
  // cluster quantise kernel first.  Both write x_q and s_x to the workspace.
  const bool fused = static_cast<long long>(M) * K <= dl::kFusedQuantMaxElems;
  if (!fused) {
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
  dl_status st = check_gemm_common(x, M, K, w_packed, w_scale, out);
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
  dl_status st = check_gemm_common(x, M, K, w_packed, w_scale, qkv);
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

dl_status dl_moe_fc13_swiglu_grouped(const uint16_t* x, int T, int K, const int32_t* expert_ids, int E,
                                     const uint8_t* w_packed, const float* w_scales, int N2, uint16_t* out,
                                     void* ws, size_t ws_bytes, void* stream, unsigned flags) {
  dl_status st = check_gemm_common(x, T, K, w_packed, w_scales, out);
  if (st != DL_OK) return st;
  if (expert_ids == nullptr || E < 1 || N2 < 256) return DL_ERR_INVALID_ARG;
  if (E > 1024 || N2 % 256 != 0) return DL_ERR_UNSUPPORTED;
  if (!aligned(expert_ids, 4)) return DL_ERR_ALIGNMENT;
  if (forced_split(flags) > 8) return DL_ERR_INVALID_ARG;
  st = check_ws(ws, ws_bytes, dl_workspace_bytes(T, K));
  if (st != DL_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool pdl = (flags & DL_FLAG_PDL) != 0;
  cudaError_t e = dl::launch_act_quant(x, T, K, dl::ws_xq(ws), dl::ws_sx(ws), s, pdl);
  if (e != cudaSuccess) return cuda_status(e);
  dl::GemmLaunch g{};
  g.w = w_packed;
  g.w_expert_bytes = static_cast<long long>(N2) * K;
  g.w_scale = w_scales;
  g.xq = dl::ws_xq(ws);
  g.s_x = dl::ws_sx(ws);
  g.status = dl::ws_status(ws);
  g.out = out;
  g.expert_ids = expert_ids;
  g.M = T;
  g.K = K;
  g.N = N2;
  g.ldo = N2 / 2;
  g.E = E;
  g.q_cols = 0;
  g.q_scale = 1.0f;
  g.swiglu = true;
  g.slots = T < E ? T : E;
  g.split = static_cast<int>(forced_split(flags));
  g.debug = (flags & DL_FLAG_DEBUG_TIMEOUT) != 0;
  g.pdl = pdl;
  return cuda_status(dl::launch_gemm(g, s));
}

dl_status dl_decode_attn(const uint16_t* q, long long q_token_stride, int B, int T, int Hq, int Hkv, int d,
                         const uint16_t* k_cache, const uint16_t* v_cache, int Lcap, const int32_t* seq_lens,
                         float softmax_scale, int cluster_size, uint16_t* out, void* ws, size_t ws_bytes,
                         void* stream, unsigned flags) {
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || seq_lens == nullptr || out == nullptr)
    return DL_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || Hq < 1 || Hkv < 1 || Lcap < 1 || d < 1) return DL_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return DL_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return DL_ERR_UNSUPPORTED;
  if ((Hq / Hkv) * T > 32) return DL_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535) return DL_ERR_UNSUPPORTED;
  if (cluster_size != 1 && cluster_size != 2 && cluster_size != 4 && cluster_size != 8 && cluster_size != 16)
    return DL_ERR_INVALID_ARG;
  if (q_token_stride < static_cast<long long>(Hq) * d || q_token_stride % 8 != 0) return DL_ERR_ALIGNMENT;
  if (forced_split(flags) > 16) return DL_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(seq_lens, 4))
    return DL_ERR_ALIGNMENT;
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
