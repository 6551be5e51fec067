// Router balancing losses (kda/layers/latent_moe.py LatentMoE._balancing_losses;
// the pages' test_moe_aux_loss_penalizes_collapse), before their coefficients:
//   frac_e      = (pairs routed to e) / max(N k, 1)
//   prob_mean_e = mean_t sigmoid(l_te)
//   aux         = R sum_e frac_e prob_mean_e        (Switch/GShard form on sigmoid scores)
//   z           = mean_t (logsumexp_e l_te)^2      (z-loss on the raw logits)
// Two launches, both deterministic: every block of kLossRows tokens writes its
// per-expert sums of sigmoid(l), its integer expert histogram and its sum of
// squared row logsumexps; one CTA then adds the blocks in order.
#include "common.cuh"
#include "kernels.h"
#include "launch.h"

namespace lmoe {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float sigmoid_l(float l) { return 1.0f / (1.0f + expf(-l)); }

__global__ void __launch_bounds__(kThreads) loss_partial_kernel(
    const float* __restrict__ logits, int64_t ld, const int32_t* __restrict__ ids, int64_t n,
    int k, int R, float* __restrict__ part_s, int32_t* __restrict__ part_c,
    float* __restrict__ part_z, int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int32_t hist[];  // [R]
  __shared__ float wz[kThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kLossRows;
  const int rows = (int)(n - t0 < kLossRows ? n - t0 : kLossRows);
  for (int e = threadIdx.x; e < R; e += kThreads) hist[e] = 0;
  __syncthreads();
  // integer histogram of this block's pairs (order-free)
  for (int i = threadIdx.x; i < rows * k; i += kThreads) {
    const int e = ids[t0 * k + i];
    if ((unsigned)e < (unsigned)R) atomicAdd(&hist[e], 1);
    else record_status(status, kStatusDevice);
  }
  // per-expert sums of sigmoid over the block's rows, rows in order
  for (int e = threadIdx.x; e < R; e += kThreads) {
    float acc = 0.0f;
    for (int r = 0; r < rows; ++r) acc += sigmoid_l(logits[(t0 + r) * ld + e]);
    part_s[(int64_t)blockIdx.x * R + e] = acc;
  }
  // squared logsumexp of each row: a warp per row, rows of a warp in order
  float zacc = 0.0f;
  for (int r = warp; r < rows; r += kThreads / 32) {
    const float* lr = logits + (t0 + r) * ld;
    float m = -INFINITY;
    for (int e = lane; e < R; e += 32) m = fmaxf(m, lr[e]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float se = 0.0f;
    for (int e = lane; e < R; e += 32) se += expf(lr[e] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
    const float lse = m + logf(se);
    zacc += lse * lse;
  }
  if (lane == 0) wz[warp] = zacc;
  __syncthreads();
  for (int e = threadIdx.x; e < R; e += kThreads) part_c[(int64_t)blockIdx.x * R + e] = hist[e];
  if (threadIdx.x == 0) {
    float zs = 0.0f;
    for (int w = 0; w < kThreads / 32; ++w) zs += wz[w];
    part_z[blockIdx.x] = zs;
  }
}

__global__ void __launch_bounds__(kThreads) loss_final_kernel(
    const float* __restrict__ part_s, const int32_t* __restrict__ part_c,
    const float* __restrict__ part_z, int blocks, int64_t n, int k, int R,
    float* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[kThreads];
  const float inv_n = n > 0 ? 1.0f / (float)n : 0.0f;
  const int64_t pairs = n * k;
  const float inv_pairs = 1.0f / (float)(pairs > 0 ? pairs : 1);
  float aux = 0.0f;
  for (int e = threadIdx.x; e < R; e += kThreads) {
    float s = 0.0f;
    int64_t c = 0;
    for (int b = 0; b < blocks; ++b) {
      s += part_s[(int64_t)b * R + e];
      c += part_c[(int64_t)b * R + e];
    }
    const float pm = s * inv_n, fr = (float)c * inv_pairs;
    out[2 + e] = fr;
    out[2 + R + e] = pm;
    aux += fr * pm;
  }
  red[threadIdx.x] = aux;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.0f, z = 0.0f;
    for (int i = 0; i < kThreads; ++i) a += red[i];
    for (int b = 0; b < blocks; ++b) z += part_z[b];
    out[0] = (float)R * a;
    out[1] = z * inv_n;
  }
}

}  // namespace

cudaError_t launch_router_losses(const float* logits, int64_t ld, const int32_t* ids, int64_t n,
                                 int k, int R, float* part_s, int32_t* part_c, float* part_z,
                                 int32_t* status, float* out, cudaStream_t st) {
  const int blocks = loss_blocks(n);
  if (blocks > 0) {
    const size_t smem = (size_t)R * sizeof(int32_t);
    cudaError_t e = cudaFuncSetAttribute(loss_partial_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    e = launch_pdl(loss_partial_kernel, dim3(blocks), dim3(kThreads), smem, st, 1, logits, ld, ids,
                   n, k, R, part_s, part_c, part_z, status);
    if (e != cudaSuccess) return e;
  }
  count_launch();
  return launch_pdl(loss_final_kernel, dim3(1), dim3(kThreads), 0, st, 1, (const float*)part_s,
                    (const int32_t*)part_c, (const float*)part_z, blocks, n, k, R, out);
}

}  // namespace lmoe
