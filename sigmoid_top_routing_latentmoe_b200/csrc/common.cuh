// Shared device helpers of the LatentMoE CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/latent_moe.h"

namespace lmoe {

// Status word values written on the device (same codes as lmoe_status).
constexpr int kStatusDevice = LMOE_EDEVICE;
constexpr int kStatusTimeout = LMOE_ETIMEOUT;

// Routed GEMMs are scheduled in row tiles of at most this many sorted pairs
// of one expert: kTileM for single-CTA tiles (and the CUDA-core kernels), and
// kRoutedPairTileM for the tensor-core GEMMs on CTA pairs.  Workspaces size
// the tile list for kTileM, which bounds both.
constexpr int kTileM = 128;
constexpr int kRoutedPairTileM = 256;

// Words of the synchronisation area that follows the workspace header: the
// final GEMM with the fused combine counts the RMSNorm(u) rows ready per
// 256-row tile there (up to kSyncWords - 1 tiles) and keeps a finished-CTA
// counter in the last word; every such launch leaves it zeroed again.
constexpr int kSyncWords = 1024;

// Header at the start of every workspace.
struct WsHeader {
  int32_t status;        // 0, or the first failure code recorded on the device
  int32_t n_mtiles;      // number of routed row tiles (written by dispatch)
  int32_t n_mtiles2;     // routed GEMM2's own list, when its tile height differs
  int32_t pad[61];
};

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ void record_status(int32_t* status, int code) {
  atomicCAS(status, 0, code);
}

// Exact fp32 SiTU-GLU hidden unit: beta1 tanh(a/beta1) sigmoid(a) * beta2 tanh(c/beta2).
__device__ __forceinline__ float situ_exact(float a, float c, float beta1, float beta2) {
  float gate = beta1 * tanhf(a / beta1) * (1.0f / (1.0f + expf(-a)));
  float up = beta2 * tanhf(c / beta2);
  return gate * up;
}

// Programmatic dependent launch: every kernel of the library lets the next
// kernel in its stream launch as soon as all of its CTAs have started
// (pdl_trigger), and waits for the previous kernel to complete -- memory
// included -- before it touches anything (pdl_wait).  Both are no-ops when
// the kernel was launched without the attribute.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace lmoe
