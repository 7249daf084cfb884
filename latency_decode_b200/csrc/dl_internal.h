// dl_internal.h -- host-side declarations shared by the .cu files of libdl.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dl.h"

namespace dl {

// Fills the launch attributes for an optional cluster shape and PDL.
struct Launch {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[2];
  Launch(dim3 grid, dim3 block, size_t smem, cudaStream_t s, unsigned cluster_x, bool pdl) {
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    int n = 0;
    if (cluster_x > 0) {
      attr[n].id = cudaLaunchAttributeClusterDimension;
      attr[n].val.clusterDim.x = cluster_x;
      attr[n].val.clusterDim.y = 1;
      attr[n].val.clusterDim.z = 1;
      ++n;
    }
    if (pdl) {
      attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[n].val.programmaticStreamSerializationAllowed = 1;
      ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
  }
};

int sm_count();  // SMs of the current device (cached per device)
int current_device();

// Raises the dynamic shared-memory limit of a kernel (and allows non-portable
// cluster sizes) on the current device only when a launch needs more than was
// set before: launches after the first cost no runtime call.
cudaError_t ensure_kernel_attrs(const void* func, int smem_bytes, bool nonportable_cluster);

// Memoised per (device, key): returns the cached value, or computes it with
// fn(), stores it and returns it.  Thread-safe.
int memo_int(unsigned long long key, int (*fn)(const void*), const void* ctx);

// Workspace layout (see dl.h).
constexpr size_t kWsHeader = 256;
inline uint32_t* ws_status(void* ws) { return static_cast<uint32_t*>(ws); }
inline float* ws_sx(void* ws) { return reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 8); }
inline uint8_t* ws_xq(void* ws) { return static_cast<uint8_t*>(ws) + kWsHeader; }

// ---- kernels' host launchers (return a CUDA error code) ----
cudaError_t launch_act_quant(const uint16_t* x, int M, int K, uint8_t* xq, float* s_x,
                             cudaStream_t s, bool pdl);
cudaError_t launch_add_rmsnorm_quant(const uint16_t* x, const uint16_t* r, uint16_t* h_out, const uint16_t* gamma,
                                     int M, int K, float eps, uint8_t* xq, float* s_x, cudaStream_t s, bool pdl);
cudaError_t launch_spec_verify(const uint16_t* logits, int B, int T, int V, const int32_t* draft,
                               int32_t* target_ids, int32_t* n_accepted, int32_t* emitted, int32_t* seq_lens,
                               cudaStream_t s, bool pdl);
cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t s, bool pdl, bool wait_first);
cudaError_t launch_pack(const uint8_t* w_nk, uint8_t* w_packed, int N, int K, int kind,
                        cudaStream_t s);

// A 2-D TMA map over rows of row_bytes bytes (row pitch row_bytes): boxes of
// 128 bytes x box_rows rows with the 128-byte swizzle (the tcgen05 SW128
// K-major operand layout); rows past `rows` read as zeros.  false when the
// driver's encoder is unavailable or refuses the shape.
bool encode_u8_rows_sw128(CUtensorMap* m, const void* base, int row_bytes, int rows, int box_rows);

struct GemmLaunch {
  const uint8_t* w;
  long long w_expert_bytes;
  const float* w_scale;
  uint8_t* xq;
  float* s_x;
  const uint16_t* x;          // non-null: quantise x inside the GEMM (dense, small M*K)
  uint32_t* status;
  uint16_t* out;
  const int32_t* expert_ids;  // null for dense
  int M, K, N, ldo, E;        // N = output rows streamed per expert (N2 for SwiGLU)
  int q_cols;
  float q_scale;
  bool swiglu;
  int slots;                  // grid z (1 for dense)
  int split;                  // forced split-K cluster size (0 = choose)
  bool debug;
  bool pdl;
};
cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t s);
// Largest M*K for which a dense GEMM quantises its activations itself.
constexpr long long kFusedQuantMaxElems = 32768;

struct AttnLaunch {
  const uint16_t* q;
  long long q_stride;
  int B, T, Hq, Hkv, d, Lcap;
  const void* k;              // bf16 [B][Hkv][Lcap][d], or e4m3 bytes when fp8
  const void* v;
  bool fp8;                   // e4m3 cache with kv_scale = device {s_k, s_v}
  const float* kv_scale;
  const int32_t* seq_lens;
  float scale;
  int cluster;
  int splits;        // clusters per (b, kv head); 0 = automatic
  size_t ws_bytes;   // workspace available (limits the number of clusters per head)
  uint16_t* out;
  uint32_t* status;  // start of the workspace
  bool debug;
  bool pdl;
};
cudaError_t launch_attn(const AttnLaunch& a, cudaStream_t s);
size_t attn_ws_bytes(int B, int Hkv, int R, int d, int P, int S);
int attn_auto_splits(int B, int Hkv, int cluster, int Lcap, int d, int R, bool fp8);

}  // namespace dl
