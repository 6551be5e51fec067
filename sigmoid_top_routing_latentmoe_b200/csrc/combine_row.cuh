// One token of the weighted combine + RMSNorm, by one warp (kda/layers/
// latent_moe.py: the index_add of p-weighted expert outputs, then self.norm;
// sec-07 compute flow steps 3 and 5):
//   u_t = sum_{i < k} p[t, i] * expert_out[inv_pair[t, i]]     (slot order, fp32)
//   out_t = u_t * (1 / sqrt(mean(u_t^2) + eps)) * w
// Shared by the combine kernel and the final GEMM's fused combine, so both give
// the same bits.  VPL: 16-byte vectors of the row per lane; the row's
// L / (16 / sizeof(T)) vectors must fit in 32 VPL.  Slots whose inv_pair entry
// is negative (pairs the dispatch dropped) add nothing.
#pragma once

#include "common.cuh"

namespace lmoe {

template <typename T, int VPL>
__device__ __forceinline__ void combine_row(const T* __restrict__ eo,
                                            const int32_t* __restrict__ inv_pair,
                                            const float* __restrict__ probs,
                                            const float* __restrict__ rms_w, int64_t t, int k,
                                            int L, float eps, T* __restrict__ out) {
  constexpr int E = 16 / sizeof(T);  // elements per vector
  const int lane = threadIdx.x & 31;
  const int nvec = L / E;
  float u[VPL][E];
#pragma unroll
  for (int v = 0; v < VPL; ++v)
#pragma unroll
    for (int e = 0; e < E; ++e) u[v][e] = 0.0f;
#pragma unroll 4
  for (int i = 0; i < k; ++i) {  // unrolled: up to four slots' rows in flight
    const int64_t r = inv_pair[t * k + i];
    if (r < 0) continue;  // a pair the dispatch dropped (out-of-range id)
    const float p = probs[t * k + i];
    const uint4* row = reinterpret_cast<const uint4*>(eo + r * L);
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      int vi = v * 32 + lane;
      if (vi < nvec) {
        uint4 raw = row[vi];
        const T* el = reinterpret_cast<const T*>(&raw);
#pragma unroll
        for (int e = 0; e < E; ++e) u[v][e] = fmaf(p, to_f(el[e]), u[v][e]);
      }
    }
  }
  float ss = 0.0f;
#pragma unroll
  for (int v = 0; v < VPL; ++v)
#pragma unroll
    for (int e = 0; e < E; ++e) ss = fmaf(u[v][e], u[v][e], ss);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = rsqrtf(ss / (float)L + eps);
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    int vi = v * 32 + lane;
    if (vi < nvec) {
      uint4 raw;
      T* el = reinterpret_cast<T*>(&raw);
#pragma unroll
      for (int e = 0; e < E; ++e) el[e] = from_f<T>(u[v][e] * inv * rms_w[vi * E + e]);
      reinterpret_cast<uint4*>(out + t * L)[vi] = raw;
    }
  }
}

}  // namespace lmoe
