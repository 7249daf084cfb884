// static_ws.cu -- dl_fc13_swiglu_static_ws: FC13 + SwiGLU for callers that
// cannot allocate device memory.
//
// dl_fc13_swiglu needs a caller-allocated workspace for the e4m3 activations
// and their scale.  Some callers have no way to obtain one: a plugin handed only
// its input and output buffers by a host runtime that owns all device memory,
// an engine that sizes its memory pool once at start-up and forbids any later
// allocation, or a latency-critical loop where cudaMalloc/cudaFree would
// synchronise the device and stall the pipeline.  This variant keeps that
// scratch in a fixed array inside the library instead, so the caller passes
// only inputs and outputs.
//
// The scratch is one file-scope device array of 256 + 64*8192 bytes (512 KiB
// plus a 256-byte header), the same layout as the workspace of
// dl_fc13_swiglu.  Every GPU that loads the library holds it until the
// process exits.  Every call on a device shares it and leaves its contents
// behind; the kernels overwrite all of it that they read, so nothing needs
// clearing between calls.  Two calls that run at the same time on the GPU
// (different streams, or different host threads without ordering) race on
// the array.  Calls queued one after another on one stream are ordered,
// with or without PDL.
#include <mutex>

#include "dl_device.cuh"
#include "dl_internal.h"

namespace {

constexpr int kStaticMaxM = 64;
constexpr long long kStaticMaxElems = 64ll * 8192;  // M*K limit of the array
constexpr size_t kStaticScratchBytes = dl::kWsHeader + static_cast<size_t>(kStaticMaxElems);

static __device__ __align__(256) uint8_t g_fc13_scratch[kStaticScratchBytes];

// Device address of g_fc13_scratch, looked up once per device.  In host code
// the array's name stands in for the symbol only; it is not a device address.
constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fc13_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" dl_status dl_fc13_swiglu_static_ws(const uint16_t* x, int M, int K, const uint8_t* w_packed,
                                              const float* w_scale, int N2, uint16_t* out, uint32_t* status,
                                              void* stream, unsigned flags) {
  if (x == nullptr || w_packed == nullptr || w_scale == nullptr || out == nullptr) return DL_ERR_INVALID_ARG;
  if (M < 1 || K < 128 || N2 < 256) return DL_ERR_INVALID_ARG;
  if (K % 128 != 0 || N2 % 256 != 0) return DL_ERR_UNSUPPORTED;
  // the fixed scratch holds at most 64 rows and 64*8192 activation bytes
  if (M > kStaticMaxM || static_cast<long long>(M) * K > kStaticMaxElems) return DL_ERR_WORKSPACE;
  if (!is_aligned(x, 16) || !is_aligned(w_packed, 16) || !is_aligned(out, 16) || !is_aligned(w_scale, 4) ||
      (status != nullptr && !is_aligned(status, 4)))
    return DL_ERR_ALIGNMENT;
  if (((flags >> DL_FLAG_SPLIT_SHIFT) & 31u) > 8u) return DL_ERR_INVALID_ARG;

  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) {
    (void)cudaGetLastError();
    return DL_ERR_CUDA;
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool pdl = (flags & DL_FLAG_PDL) != 0;
  // As in dl_fc13_swiglu: small inputs are quantised inside the GEMM, larger
  // ones by the quantise kernel first; both write x_q and s_x to the array.
  const bool fused = static_cast<long long>(M) * K <= dl::kFusedQuantMaxElems;
  cudaError_t e = fused ? cudaSuccess : dl::launch_act_quant(x, M, K, dl::ws_xq(scratch), dl::ws_sx(scratch), s, pdl);
  if (e == cudaSuccess) {
    dl::GemmLaunch g{};
    g.x = fused ? x : nullptr;
    g.w = w_packed;
    g.w_expert_bytes = 0;
    g.w_scale = w_scale;
    g.xq = dl::ws_xq(scratch);
    g.s_x = dl::ws_sx(scratch);
    g.status = status;
    g.out = out;
    g.expert_ids = nullptr;
    g.M = M;
    g.K = K;
    g.N = N2;
    g.ldo = N2 / 2;
    g.E = 1;
    g.q_cols = 0;
    g.q_scale = 1.0f;
    g.swiglu = true;
    g.slots = 1;
    g.split = static_cast<int>((flags >> DL_FLAG_SPLIT_SHIFT) & 31u);
    g.debug = (flags & DL_FLAG_DEBUG_TIMEOUT) != 0;
    g.pdl = pdl;
    e = dl::launch_gemm(g, s);
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return DL_ERR_CUDA;
  }
  return DL_OK;
}
