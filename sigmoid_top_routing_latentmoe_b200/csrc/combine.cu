// Weighted combine + RMSNorm (kda/layers/latent_moe.py: the index_add of
// p-weighted expert outputs back to their tokens, then self.norm; sec-07
// compute flow steps 3 and 5):
//   u_t = sum_{i < k} p[t, i] * expert_out[inv_pair[t, i]]     (slot order, fp32)
//   u_normed_t = u_t * (1 / sqrt(mean(u_t^2) + eps)) * w
// Each token is reduced by one warp in a fixed order: no float atomics, so
// the result is deterministic.  Rows are read with 16-byte vectors.
#include "combine_row.cuh"
#include "common.cuh"
#include "kernels.h"
#include "launch.h"

namespace lmoe {
namespace {

template <typename T, int VPL>  // VPL: 16-byte vectors per lane
__global__ void __launch_bounds__(256) combine_kernel(const T* __restrict__ eo,
                                                      const int32_t* __restrict__ inv_pair,
                                                      const float* __restrict__ probs,
                                                      const float* __restrict__ rms_w, int64_t n,
                                                      int k, int L, float eps, T* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n) return;
  combine_row<T, VPL>(eo, inv_pair, probs, rms_w, t, k, L, eps, out);
}

// Wide rows (l > 1024): one 128-thread block per token, VPT 16-byte vectors
// per thread; the k expert rows are read UNROLL slots at a time so that many
// loads are in flight.  Same arithmetic order per element as combine_kernel:
// u = sum over slots in order, then RMSNorm.
template <typename T, int VPT>
__global__ void __launch_bounds__(128) combine_block_kernel(const T* __restrict__ eo,
                                                            const int32_t* __restrict__ inv_pair,
                                                            const float* __restrict__ probs,
                                                            const float* __restrict__ rms_w,
                                                            int k, int L, float eps,
                                                            T* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  constexpr int E = 16 / sizeof(T);
  constexpr int UNROLL = 4;
  __shared__ float red[4];
  const int64_t t = blockIdx.x;
  const int nvec = L / E;
  float u[VPT][E];
#pragma unroll
  for (int v = 0; v < VPT; ++v)
#pragma unroll
    for (int e = 0; e < E; ++e) u[v][e] = 0.0f;
  for (int i0 = 0; i0 < k; i0 += UNROLL) {
    uint4 raw[UNROLL][VPT];
    float pw[UNROLL];
#pragma unroll
    for (int j = 0; j < UNROLL; ++j) {
      const int i = i0 + j;
      pw[j] = 0.0f;
      const int64_t r = i < k ? inv_pair[t * k + i] : -1;
      if (r >= 0) {  // r < 0: a pair the dispatch dropped (out-of-range id)
        pw[j] = probs[t * k + i];
        const uint4* row = reinterpret_cast<const uint4*>(eo + r * L);
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          const int vi = v * 128 + threadIdx.x;
          raw[j][v] = vi < nvec ? row[vi] : make_uint4(0, 0, 0, 0);
        }
      } else {
#pragma unroll
        for (int v = 0; v < VPT; ++v) raw[j][v] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int j = 0; j < UNROLL; ++j) {
      if (i0 + j < k && pw[j] != 0.0f) {
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          const T* el = reinterpret_cast<const T*>(&raw[j][v]);
#pragma unroll
          for (int e = 0; e < E; ++e) u[v][e] = fmaf(pw[j], to_f(el[e]), u[v][e]);
        }
      }
    }
  }
  float ss = 0.0f;
#pragma unroll
  for (int v = 0; v < VPT; ++v)
#pragma unroll
    for (int e = 0; e < E; ++e) ss = fmaf(u[v][e], u[v][e], ss);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  ss = red[0] + red[1] + red[2] + red[3];
  const float inv = rsqrtf(ss / (float)L + eps);
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    const int vi = v * 128 + threadIdx.x;
    if (vi < nvec) {
      uint4 raw;
      T* el = reinterpret_cast<T*>(&raw);
#pragma unroll
      for (int e = 0; e < E; ++e) el[e] = from_f<T>(u[v][e] * inv * rms_w[vi * E + e]);
      reinterpret_cast<uint4*>(out + t * L)[vi] = raw;
    }
  }
}

}  // namespace

template <typename T>
cudaError_t launch_combine(const T* eo, const int32_t* inv_pair, const float* probs,
                           const float* rms_w, int64_t n, int k, int L, float eps, T* out,
                           cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  constexpr int E = 16 / sizeof(T);
  const int nvec = L / E;
  const int vpl = (nvec + 31) / 32;
  if (vpl > 4) {  // wide rows: a block per token
    const int vpt = (nvec + 127) / 128;
#define LMOE_COMBINE_BLOCK_CASE(V)                                                     \
    if (vpt <= V) {                                                                    \
      count_launch();                                                                  \
      return launch_pdl(combine_block_kernel<T, V>, dim3((unsigned)n), dim3(128), 0, st, 1, eo, \
                        inv_pair, probs, rms_w, k, L, eps, out);                       \
    }
    LMOE_COMBINE_BLOCK_CASE(2)
    LMOE_COMBINE_BLOCK_CASE(4)
#undef LMOE_COMBINE_BLOCK_CASE
    return cudaErrorInvalidValue;
  }
  const int warps = 8;
  unsigned blocks = (unsigned)((n + warps - 1) / warps);
#define LMOE_COMBINE_CASE(V)                                                              \
  if (vpl <= V) {                                                                         \
    count_launch();                                                                       \
    return launch_pdl(combine_kernel<T, V>, dim3(blocks), dim3(warps * 32), 0, st, 1, eo,    \
                      inv_pair, probs, rms_w, n, k, L, eps, out);                         \
  }
  LMOE_COMBINE_CASE(1)
  LMOE_COMBINE_CASE(2)
  LMOE_COMBINE_CASE(4)
#undef LMOE_COMBINE_CASE
  return cudaErrorInvalidValue;
}
template cudaError_t launch_combine<float>(const float*, const int32_t*, const float*,
                                           const float*, int64_t, int, int, float, float*,
                                           cudaStream_t);
template cudaError_t launch_combine<__nv_bfloat16>(const __nv_bfloat16*, const int32_t*,
                                                   const float*, const float*, int64_t, int, int,
                                                   float, __nv_bfloat16*, cudaStream_t);

}  // namespace lmoe
