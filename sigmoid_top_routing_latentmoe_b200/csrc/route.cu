// Router kernels: K3 sigmoid routing (sec-07 compute flow step 2, K3 eq.13;
// kda/layers/latent_moe.py LatentMoE._route):
//   l = W_r x,  s = sigmoid(l),  T = TopK(s + b, k),  p_i = s_i / max(sum_T s, 1e-9).
// The bias enters the selection only.  router == 1 is the rule latent_moe.py
// had before it: T = TopK(l, k), p = softmax over the k selected logits.
// Slots are written in descending key order; equal keys go to the lower
// expert index.
#include "common.cuh"
#include "kernels.h"
#include "launch.h"

namespace lmoe {
namespace {

__device__ __forceinline__ float sigmoid_f(float l) { return 1.0f / (1.0f + expf(-l)); }

// Warp-wide selection of the largest key (ties: lower expert index).
__device__ __forceinline__ void warp_argmax(float& key, int& idx) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float ok = __shfl_xor_sync(0xffffffffu, key, off);
    int oi = __shfl_xor_sync(0xffffffffu, idx, off);
    if (ok > key || (ok == key && oi < idx)) {
      key = ok;
      idx = oi;
    }
  }
}

// Top-k over R <= 32 * VPL experts held VPL per lane (expert e = j*32 + lane),
// then p = s / max(sum s, 1e-9); with softmax != 0, s holds the logits and
// p = exp(s - s_first) / sum over the slots (slot 0 holds the largest).
// Called by all 32 lanes of a warp.
template <int VPL, bool SOFTMAX>
__device__ __forceinline__ void select_topk(const float (&s)[VPL], const float (&key_in)[VPL], int R,
                                            int k, int32_t* ids_row, float* probs_row) {
  const int lane = threadIdx.x & 31;
  float key[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) key[j] = (j * 32 + lane < R) ? key_in[j] : -INFINITY;
  float den = 0.0f;
  float sel_s = 0.0f;  // score of the slot this lane will write (lane == slot)
  int sel_id = 0;
  float first = 0.0f;  // softmax: the largest selected logit
  for (int slot = 0; slot < k; ++slot) {
    float bk = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      int e = j * 32 + lane;
      if (e < R && (key[j] > bk || (key[j] == bk && e < bi))) {
        bk = key[j];
        bi = e;
      }
    }
    warp_argmax(bk, bi);
    // owner lane retires the winner and broadcasts its raw score
    float sc = 0.0f;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      if (j * 32 + lane == bi) {
        key[j] = -INFINITY;
        sc = s[j];
      }
    }
    sc = __shfl_sync(0xffffffffu, sc, bi & 31);
    if (SOFTMAX) {
      if (slot == 0) first = sc;
      sc = expf(sc - first);
    }
    den += sc;
    if ((slot & 31) == lane) {
      sel_s = sc;
      sel_id = bi;
    }
    if ((slot & 31) == 31 || slot == k - 1) {
      // flush a group of up to 32 slots
      int base = slot & ~31;
      if (lane <= (slot & 31)) ids_row[base + lane] = sel_id;
      // probs need the full sum: stash scores in probs_row for now
      if (lane <= (slot & 31)) probs_row[base + lane] = sel_s;
    }
  }
  if (!SOFTMAX) den = fmaxf(den, 1e-9f);
  __syncwarp();
  for (int slot = lane; slot < k; slot += 32) probs_row[slot] = probs_row[slot] / den;
}

// One warp per token, RMAX >= R accumulators per lane.  Each lane reads x and
// the matching slice of every W_r row in 16-byte vectors (W_r stays in L1/L2),
// so lane j owns columns [8j, 8j+8) of every 256-column block.  A butterfly
// transpose-reduction then leaves lane e holding expert e's logit.
template <typename T, int RMAX>
__global__ void __launch_bounds__(256) route_gemv_kernel(const T* __restrict__ x,
                                                         const T* __restrict__ w_r,
                                                         const float* __restrict__ bias, int64_t n,
                                                         int d, int R, int k, int router,
                                                         int32_t* __restrict__ ids,
                                                         float* __restrict__ probs,
                                                         float* __restrict__ logits_out,
                                                         int64_t ld) {
  pdl_trigger();
  pdl_wait();
  constexpr int E = 16 / sizeof(T);  // elements per 16-byte vector
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
  const int nvec = d / E;
  float acc[RMAX];
#pragma unroll
  for (int e = 0; e < RMAX; ++e) acc[e] = 0.0f;
  for (int v = lane; v < nvec; v += 32) {
    const uint4 xv = xr[v];
    const T* xe = reinterpret_cast<const T*>(&xv);
    float xf[E];
#pragma unroll
    for (int i = 0; i < E; ++i) xf[i] = to_f(xe[i]);
#pragma unroll
    for (int e = 0; e < RMAX; ++e) {
      if (e < R) {
        const uint4 wv = reinterpret_cast<const uint4*>(w_r + (int64_t)e * d)[v];
        const T* we = reinterpret_cast<const T*>(&wv);
#pragma unroll
        for (int i = 0; i < E; ++i) acc[e] = fmaf(to_f(we[i]), xf[i], acc[e]);
      }
    }
  }
  // sum over lanes; lane e keeps expert e
#pragma unroll
  for (int e = 0; e < RMAX; ++e) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  float logit = 0.0f;
#pragma unroll
  for (int e = 0; e < RMAX; ++e)
    if (e == lane) logit = acc[e];
  if (logits_out != nullptr && lane < R) logits_out[t * ld + lane] = logit;
  float s[1], key[1];
  if (router) {
    s[0] = key[0] = logit;
  } else {
    s[0] = sigmoid_f(logit);
    key[0] = s[0] + ((bias != nullptr && lane < R) ? bias[lane] : 0.0f);
  }
  if (router) select_topk<1, true>(s, key, R, k, ids + t * k, probs + t * k);
  else select_topk<1, false>(s, key, R, k, ids + t * k, probs + t * k);
}

template <int VPL, bool SOFTMAX>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits,
                                                         int64_t ld, const float* __restrict__ bias,
                                                         int64_t n, int R, int k,
                                                         int32_t* __restrict__ ids,
                                                         float* __restrict__ probs) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n) return;
  const float* lr = logits + t * ld;
  float s[VPL], key[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    int e = j * 32 + lane;
    float l = (e < R) ? lr[e] : 0.0f;
    if (SOFTMAX) {
      s[j] = key[j] = l;
    } else {
      s[j] = sigmoid_f(l);
      key[j] = s[j] + ((bias != nullptr && e < R) ? bias[e] : 0.0f);
    }
  }
  select_topk<VPL, SOFTMAX>(s, key, R, k, ids + t * k, probs + t * k);
}

// Order-preserving map of a float to uint32 (larger float -> larger code).
__device__ __forceinline__ uint32_t orderable(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Bitonic sort of 64 keys held two per lane (element i = lane + 32 r),
// descending: afterwards element i is the i-th largest.
__device__ __forceinline__ void warp_sort64_desc(uint64_t (&v)[2]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {  // partner is the lane's other element
        const bool desc = (lane & size) == 0;  // size == 64 here: always descending
        const uint64_t hi = v[0] > v[1] ? v[0] : v[1], lo = v[0] > v[1] ? v[1] : v[0];
        v[0] = desc ? hi : lo;
        v[1] = desc ? lo : hi;
      } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int i = lane + 32 * r;
          const uint64_t pv = __shfl_xor_sync(0xffffffffu, v[r], stride);
          const bool desc = (i & size) == 0;
          const bool keep_max = ((lane & stride) == 0) == desc;  // lower index of the pair
          v[r] = keep_max ? (v[r] > pv ? v[r] : pv) : (v[r] < pv ? v[r] : pv);
        }
      }
    }
  }
}

// Bitonic sort of 32 floats across the warp, descending (lane i gets the
// i-th largest).
__device__ __forceinline__ float warp_sort32_desc(float v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const float pv = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool desc = (lane & size) == 0 || size == 32;
      const bool keep_max = ((lane & stride) == 0) == desc;
      v = keep_max ? fmaxf(v, pv) : fminf(v, pv);
    }
  }
  return v;
}

// Expert held as value j of a lane in the wide top-k: the row is read as
// float4 groups, group g of 128 experts giving lane l experts 128 g + 4 l ...
// 128 g + 4 l + 3.
__device__ __forceinline__ int wide_expert(int j, int lane) {
  return (j >> 2) * 128 + lane * 4 + (j & 3);
}

// k rounds of a warp argmax over keys held VPL per lane (expert
// wide_expert(j, lane); ties to the lower expert), the selected experts'
// scores read back from the logits row lr: the same slots and weights as
// select_topk, without a second array of scores in registers.
template <int VPL, bool SOFTMAX>
__device__ __noinline__ void select_topk_keys(float (&key)[VPL], const float* __restrict__ lr, int R,
                                              int k, int32_t* ids_row, float* probs_row) {
  const int lane = threadIdx.x & 31;
  float den = 0.0f, first = 0.0f;
  for (int slot = 0; slot < k; ++slot) {
    float bk = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = wide_expert(j, lane);
      if (e < R && (key[j] > bk || (key[j] == bk && e < bi))) {
        bk = key[j];
        bi = e;
      }
    }
    warp_argmax(bk, bi);
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      if (wide_expert(j, lane) == bi) key[j] = -INFINITY;
    float sc = SOFTMAX ? lr[bi] : sigmoid_f(lr[bi]);
    if (SOFTMAX) {
      if (slot == 0) first = sc;
      sc = expf(sc - first);
    }
    den += sc;
    if (lane == 0) {
      ids_row[slot] = bi;
      probs_row[slot] = sc;  // divided by the sum below
    }
  }
  if (!SOFTMAX) den = fmaxf(den, 1e-9f);
  __syncwarp();
  for (int slot = lane; slot < k; slot += 32) probs_row[slot] = probs_row[slot] / den;
}

// Top-k for many experts (R > 96, k <= 32), one warp per token, same result
// as select_topk (keys descending, ties to the lower expert index; p from the
// exact scores in slot order):
//   1. the k-th largest of the 32 lane maxima is a lower bound Lk on the k-th
//      largest key (k distinct keys reach it), so every key of the top k is
//      >= Lk;
//   2. the keys >= Lk (typically a few dozen of R) are compacted by ballot
//      into a per-warp list of (orderable key << 32 | ~expert) codes;
//   3. up to 64 candidates are sorted by a warp bitonic sort; the first k are
//      the slots.  More than 64 candidates (clustered keys) take the k-round
//      selection over all R keys instead.
// The selection keys use the fast exponential and division (|error| ~1e-7,
// far below the routing margins); the selected scores are recomputed exactly.
template <int VPL, bool SOFTMAX>
__global__ void __launch_bounds__(256, VPL <= 32 ? (SOFTMAX ? 3 : 4) : 1) route_topk_wide_kernel(const float* __restrict__ logits,
                                                              int64_t ld,
                                                              const float* __restrict__ bias,
                                                              int64_t n, int R, int k,
                                                              int32_t* __restrict__ ids,
                                                              float* __restrict__ probs) {
  pdl_trigger();
  __shared__ uint64_t cand[8][64];
  extern __shared__ float sbias[];  // [R]: the bias, read once per block
  if (!SOFTMAX) {
    for (int e = threadIdx.x; e < R; e += blockDim.x) sbias[e] = bias != nullptr ? bias[e] : 0.0f;
    __syncthreads();
  }
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= n) return;
  const float* lr = logits + t * ld;  // ld: a multiple of 16 floats, >= R
  float key[VPL];
  float lmax = -INFINITY;
#pragma unroll
  for (int g = 0; g < VPL / 4; ++g) {
    const int e0 = g * 128 + lane * 4;
    float4 l4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (VPL <= 64) {  // one 16-byte load per group (e0 + 3 < ld)
      if (e0 < R) l4 = *reinterpret_cast<const float4*>(lr + e0);
    } else {  // the widest rows: scalar loads keep fewer values live
      if (e0 < R) l4.x = lr[e0];
      if (e0 + 1 < R) l4.y = lr[e0 + 1];
      if (e0 + 2 < R) l4.z = lr[e0 + 2];
      if (e0 + 3 < R) l4.w = lr[e0 + 3];
    }
    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float kv = -INFINITY;
      if (e0 + c < R)
        kv = SOFTMAX ? lv[c] : __fdividef(1.0f, 1.0f + __expf(-lv[c])) + sbias[e0 + c];
      key[4 * g + c] = kv;
      lmax = fmaxf(lmax, kv);
    }
  }
  const float lk = __shfl_sync(0xffffffffu, warp_sort32_desc(lmax), k - 1);
  int mine = 0;
#pragma unroll
  for (int j = 0; j < VPL; ++j) mine += key[j] >= lk ? 1 : 0;
  int incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total > 64) {  // clustered keys: the k-round selection over everything
    // exact keys (the fast ones above may differ in the last bits)
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = wide_expert(j, lane);
      if (e < R) {
        const float l = lr[e];
        key[j] = SOFTMAX ? l : sigmoid_f(l) + sbias[e];
      }
    }
    select_topk_keys<VPL, SOFTMAX>(key, lr, R, k, ids + t * k, probs + t * k);
    return;
  }
  int at = incl - mine;
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    if (key[j] >= lk) {
      const uint32_t e = (uint32_t)wide_expert(j, lane);
      cand[warp][at++] = ((uint64_t)orderable(key[j]) << 32) | (uint64_t)(0xffffffffu - e);
    }
  }
  __syncwarp();
  uint64_t v[2];
  v[0] = lane < total ? cand[warp][lane] : 0ull;
  v[1] = lane + 32 < total ? cand[warp][lane + 32] : 0ull;
  warp_sort64_desc(v);
  // lane i < k holds slot i
  const int e = (int)(0xffffffffu - (uint32_t)(v[0] & 0xffffffffu));
  float sc = 0.0f;
  if (lane < k) sc = SOFTMAX ? lr[e] : sigmoid_f(lr[e]);
  float den = 0.0f, first = __shfl_sync(0xffffffffu, sc, 0);
  if (SOFTMAX && lane < k) sc = expf(sc - first);
  for (int slot = 0; slot < k; ++slot) den += __shfl_sync(0xffffffffu, sc, slot);
  if (!SOFTMAX) den = fmaxf(den, 1e-9f);
  if (lane < k) {
    ids[t * k + lane] = e;
    probs[t * k + lane] = sc / den;
  }
}

}  // namespace

template <typename T>
cudaError_t launch_route_gemv(const T* x, const T* w_r, const float* bias, int64_t n, int d, int R,
                              int k, int router, int32_t* ids, float* probs, float* logits_out,
                              int64_t ld, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int warps = 8;
  int64_t blocks = (n + warps - 1) / warps;
  cudaError_t e;
  if (R <= 16)
    e = launch_pdl(route_gemv_kernel<T, 16>, dim3((unsigned)blocks), dim3(warps * 32), 0, st, 1, x,
                   w_r, bias, n, d, R, k, router, ids, probs, logits_out, ld);
  else
    e = launch_pdl(route_gemv_kernel<T, 32>, dim3((unsigned)blocks), dim3(warps * 32), 0, st, 1, x,
                   w_r, bias, n, d, R, k, router, ids, probs, logits_out, ld);
  count_launch();
  return e;
}
template cudaError_t launch_route_gemv<float>(const float*, const float*, const float*, int64_t,
                                              int, int, int, int, int32_t*, float*, float*,
                                              int64_t, cudaStream_t);
template cudaError_t launch_route_gemv<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                      const float*, int64_t, int, int, int, int,
                                                      int32_t*, float*, float*, int64_t,
                                                      cudaStream_t);

cudaError_t launch_route_topk(const float* logits, int64_t ld, const float* bias, int64_t n, int R,
                              int k, int router, int32_t* ids, float* probs, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int warps = 8;
  unsigned blocks = (unsigned)((n + warps - 1) / warps);
  int vpl = (R + 31) / 32;
  if (vpl >= 4 && k <= 32) {
#define LMOE_TOPK_WIDE(V)                                                                    \
    if (vpl <= V) {                                                                          \
      count_launch();                                                                        \
      return router ? launch_pdl(route_topk_wide_kernel<V, true>, dim3(blocks),              \
                                 dim3(warps * 32), 0, st, 1, logits, ld, bias, n, R, k, ids, \
                                 probs)                                                      \
                    : launch_pdl(route_topk_wide_kernel<V, false>, dim3(blocks),             \
                                 dim3(warps * 32), (size_t)R * sizeof(float), st, 1, logits, \
                                 ld, bias, n, R, k, ids, probs);                             \
    }
    LMOE_TOPK_WIDE(4)
    LMOE_TOPK_WIDE(8)
    LMOE_TOPK_WIDE(16)
    LMOE_TOPK_WIDE(32)
    LMOE_TOPK_WIDE(64)
    LMOE_TOPK_WIDE(128)
#undef LMOE_TOPK_WIDE
  }
#define LMOE_TOPK_CASE(V)                                                                  \
  if (vpl <= V) {                                                                          \
    count_launch();                                                                        \
    return router ? launch_pdl(route_topk_kernel<V, true>, dim3(blocks), dim3(warps * 32), 0, st, \
                               1, logits, ld, bias, n, R, k, ids, probs)                  \
                  : launch_pdl(route_topk_kernel<V, false>, dim3(blocks), dim3(warps * 32), 0,    \
                               st, 1, logits, ld, bias, n, R, k, ids, probs);             \
  }
  LMOE_TOPK_CASE(1)
  LMOE_TOPK_CASE(2)
  LMOE_TOPK_CASE(4)
  LMOE_TOPK_CASE(8)
  LMOE_TOPK_CASE(16)
  LMOE_TOPK_CASE(32)
  LMOE_TOPK_CASE(64)
  LMOE_TOPK_CASE(128)
#undef LMOE_TOPK_CASE
  return cudaErrorInvalidValue;
}

}  // namespace lmoe
