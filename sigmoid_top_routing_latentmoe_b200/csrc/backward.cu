// Backward of the LatentMoE layer (gradients of <dy, y>; the pages train the
// layer and test its gradients: test_moe_unselected_experts_have_zero_grad and
// the sparse == dense checks of tests/integration/test_k3_arch.py).
//
// It recomputes the forward's internals in fp32 (routing with the same kernels,
// dispatch, z, the routed pre-activations a = W_g z and c = W_u z, the expert
// outputs, u, RMSNorm, the shared pre-activations) and then applies the chain
// rule step by step:
//   y = s_sh + W_up uhat     dW_up = dy^T uhat,          duhat = dy W_up
//   uhat = u r w             dw = sum_t duhat u r,       du = r w duhat - u r^3/l <w duhat u>
//   u = sum_i p_i E_i(z)     dp_i = <du, E_i(z)>,         dE_i = p_i du
//   E(v) = W_o h, h = g(a) up(c)
//                            dW_o = dE^T h, dh = dE W_o,  da = dh up g', dc = dh g up'
//                            dW_g = da^T v, dW_u = dc^T v, dv = da W_g + dc W_u
//   routing (ids fixed)      K3: dl_i = (dp_i - <p, dp>) / S * s_i (1 - s_i)
//                            softmax over the top-k logits: dl_i = p_i (dp_i - <p, dp>)
//   z = W_down x             dW_down = dz^T x, dx = dz W_down + dl W_r + (shared terms)
// Every contraction runs through one CUDA-core fp32 GEMM kernel with generic
// strides (any operand layout; bf16 or fp32 operands, a template parameter
// each), in three forms: plain;
// grouped over the routed row tiles (one expert's weights per tile); grouped
// along K per expert (weight gradients: a sum over that expert's rows).  No
// atomics: every result is a fixed-order sum, so the gradients are
// deterministic.  Weight gradients of experts that no token selects are 0.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "launch.h"
#include "umma_gemm.h"

namespace lmoe {
namespace {

constexpr int GB = 128;  // output tile (rows and columns)
constexpr int GK = 8;    // K per smem stage
constexpr int GT = 256;  // threads: 16 x 16, each 8 x 8 outputs
constexpr int GE = GB * GK / GT;  // elements of each operand a thread loads per stage
constexpr int kRmsRows = 32;  // tokens per partial sum of the RMSNorm weight gradient
int rms_blocks(int64_t n) { return (int)((n + kRmsRows - 1) / kRmsRows); }

struct GemmDesc {
  const void* A;
  int a_bf16;
  int64_t sam, sak;         // A(m, k) = A[m * sam + k * sak]
  const void* B;
  int b_bf16;
  int64_t sbk, sbn;         // B(k, n) = B[k * sbk + n * sbn]
  float* C;
  int64_t ldc;
  int M, N, K;
  int accumulate;           // C += result instead of C = result
  int form;                 // 0 plain; 1 grouped over routed tiles; 2 grouped along K per expert
  const int4* tiles;        // form 1: (expert, first row, rows), rows <= 128
  const int32_t* n_tiles;
  const int32_t* offsets;   // form 2: expert e sums rows [offsets[e], offsets[e+1])
  int64_t b_estride;        // form 1: B advances by this per expert
  int64_t c_estride;        // form 2: C advances by this per expert
  int k_chunk;              // form 0 split along K: blockIdx.z takes [z k_chunk, (z+1) k_chunk)
};

// Operand loads keep the raw bits (a bf16 zero-extended to 32 bits) so that no
// instruction waits on a load until the stage is written to smem, one stage
// later: the loads stay in flight behind the current stage's FMAs.
template <int BF>
__device__ __forceinline__ uint32_t ld_raw(const void* p, int64_t i) {
  if (BF) return (uint32_t)__ldg(static_cast<const unsigned short*>(p) + i);
  return __float_as_uint(__ldg(static_cast<const float*>(p) + i));
}
template <int BF>
__device__ __forceinline__ float from_raw(uint32_t r) {
  return BF ? __uint_as_float(r << 16) : __uint_as_float(r);
}

// A 128 x 128 tile of C per CTA (two CTAs per SM).  Each stage stages A
// [128 x GK] and B [GK x 128] in smem as As[k][m], Bs[k][n] (the global reads
// run along whichever index is contiguous), double-buffered so that one barrier
// per stage suffices; thread (tx, ty) owns rows {4ty..4ty+3, 64+4ty..64+4ty+3}
// and the same pattern of columns, read as float4 (conflict-free).
// ABF / BBF: A / B hold bf16 (else fp32).
template <int ABF, int BBF>
__global__ void __launch_bounds__(GT, 2) bwd_gemm_kernel(const GemmDesc g) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) float As[2][GK][GB + 4];
  __shared__ __align__(16) float Bs[2][GK][GB + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  int m_lo, m_hi, k_lo, k_hi;
  const void* Bp = g.B;
  float* Cp = g.C;
  const int n0 = blockIdx.y * GB;
  if (g.form == 1) {
    const int t = blockIdx.x;
    if (t >= *g.n_tiles) return;
    const int4 tl = g.tiles[t];
    m_lo = tl.y;
    m_hi = tl.y + tl.z;
    Bp = BBF ? (const void*)(static_cast<const __nv_bfloat16*>(g.B) + tl.x * g.b_estride)
             : (const void*)(static_cast<const float*>(g.B) + tl.x * g.b_estride);
    k_lo = 0;
    k_hi = g.K;
  } else {
    m_lo = blockIdx.x * GB;
    m_hi = min(g.M, m_lo + GB);
    k_lo = 0;
    k_hi = g.K;
    if (g.form == 2) {
      const int e = blockIdx.z;
      k_lo = g.offsets[e];
      k_hi = g.offsets[e + 1];
      Cp = g.C + e * g.c_estride;
    } else if (g.k_chunk > 0) {  // one slice of K; C is this slice's partial block
      k_lo = blockIdx.z * g.k_chunk;
      k_hi = min(g.K, k_lo + g.k_chunk);
      Cp = g.C + (int64_t)blockIdx.z * g.M * g.ldc;
    }
  }
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  const bool a_kc = g.sak == 1, b_nc = g.sbn == 1;
  uint32_t ra[GE], rb[GE];
  // a K-contiguous operand is read as GK consecutive elements per row, else as
  // 128 consecutive rows per k
  auto fetch = [&](int k0) {
#pragma unroll
    for (int q = 0; q < GE; ++q) {
      const int mi = a_kc ? tid / GK + (GT / GK) * q : tid & 127;
      const int ki = a_kc ? tid % GK : (tid >> 7) + 2 * q;
      const int m = m_lo + mi, k = k0 + ki;
      ra[q] = (m < m_hi && k < k_hi) ? ld_raw<ABF>(g.A, (int64_t)m * g.sam + (int64_t)k * g.sak)
                                     : 0u;
    }
#pragma unroll
    for (int q = 0; q < GE; ++q) {
      const int ki = b_nc ? (tid >> 7) + 2 * q : tid % GK;
      const int ni = b_nc ? tid & 127 : tid / GK + (GT / GK) * q;
      const int k = k0 + ki, n = n0 + ni;
      rb[q] = (k < k_hi && n < g.N) ? ld_raw<BBF>(Bp, (int64_t)k * g.sbk + (int64_t)n * g.sbn)
                                    : 0u;
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int q = 0; q < GE; ++q) {
      if (a_kc) As[buf][tid % GK][tid / GK + (GT / GK) * q] = from_raw<ABF>(ra[q]);
      else As[buf][(tid >> 7) + 2 * q][tid & 127] = from_raw<ABF>(ra[q]);
      if (b_nc) Bs[buf][(tid >> 7) + 2 * q][tid & 127] = from_raw<BBF>(rb[q]);
      else Bs[buf][tid % GK][tid / GK + (GT / GK) * q] = from_raw<BBF>(rb[q]);
    }
  };
  if (k_lo < k_hi) {
    fetch(k_lo);
    stash(0);
  }
  __syncthreads();
  int buf = 0;
  for (int k0 = k_lo; k0 < k_hi; k0 += GK) {
    const bool more = k0 + GK < k_hi;
    if (more) fetch(k0 + GK);  // in flight while this stage is multiplied out
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    // the other buffer was last read before the previous barrier
    if (more) stash(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m_lo + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (m >= m_hi) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (n >= g.N) continue;
      float* c = Cp + (int64_t)m * g.ldc + n;
      *c = g.accumulate ? *c + acc[i][j] : acc[i][j];
    }
  }
}

// C (+)= the sum of the K slices' partial blocks, slices in order.
__global__ void split_sum_kernel(const float* __restrict__ part, int splits, int M, int N,
                                 float* __restrict__ C, int64_t ldc, int accumulate) {
  pdl_trigger();
  pdl_wait();
  const int64_t total = (int64_t)M * N;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = i / N, n = i - m * N;
    float v = accumulate ? C[m * ldc + n] : 0.0f;
    for (int s = 0; s < splits; ++s) v += part[(int64_t)s * total + i];
    C[m * ldc + n] = v;
  }
}

// Scratch for the K slices of plain GEMMs with few output tiles (floats).
constexpr int64_t kSplitScratch = (int64_t)16 << 20;

using GemmKernel = void (*)(GemmDesc);
GemmKernel gemm_kernel(const GemmDesc& g) {
  if (g.a_bf16) return g.b_bf16 ? bwd_gemm_kernel<1, 1> : bwd_gemm_kernel<1, 0>;
  return g.b_bf16 ? bwd_gemm_kernel<0, 1> : bwd_gemm_kernel<0, 0>;
}

// SMs of the device current at the first call (B200: 148); thread-safe init.
int sm_count() {
  static const int n = [] {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
  }();
  return n;
}

// Number of K slices of a plain GEMM with `tiles` output tiles: the one with the
// least estimated time, taken as the K steps of the busiest SM (its CTAs times
// the slice length; a CTA alone on its SM runs at about 0.7 of the rate of two
// sharing one, which hide each other's latencies) with 3 % more per extra slice
// (its partial block is written and summed once more).
int choose_splits(int64_t tiles, int64_t MN, int K) {
  const int64_t sms = sm_count();
  if (tiles >= 2 * sms) return 1;
  const int max_s = std::min(16, K / 128);  // slices of at least 128
  auto load = [&](int64_t ctas) {
    const int64_t per_sm = (ctas + sms - 1) / sms;
    return per_sm == 1 ? 1.43 : (double)per_sm;
  };
  int best = 1;
  double best_cost = load(tiles) * K;
  for (int s = 2; s <= max_s; ++s) {
    if ((int64_t)s * MN > kSplitScratch) break;
    const double cost = load(tiles * s) * ((double)K / s) * (1.0 + 0.03 * (s - 1));
    if (cost < best_cost * (1.0 - 1e-9)) {
      best = s;
      best_cost = cost;
    }
  }
  return best;
}

cudaError_t gemm(const GemmDesc& g0, int max_tiles, int R, cudaStream_t st,
                 float* split_scratch = nullptr) {
  GemmDesc g = g0;
  const GemmKernel kern = gemm_kernel(g);
  // A plain GEMM with too few output tiles to fill the GPU runs as K slices
  // (a fixed number, summed in order by a second kernel).
  if (g.form == 0 && split_scratch != nullptr) {
    const int64_t tiles = (int64_t)((g.M + GB - 1) / GB) * ((g.N + GB - 1) / GB);
    int splits = choose_splits(tiles, (int64_t)g.M * g.N, g.K);
    if (splits > 1) {
      const int chunk = ((g.K + splits - 1) / splits + GK - 1) / GK * GK;
      splits = (g.K + chunk - 1) / chunk;
      GemmDesc p = g;
      p.C = split_scratch;
      p.ldc = g.N;
      p.accumulate = 0;
      p.k_chunk = chunk;
      count_launch();
      cudaError_t e = launch_pdl(kern,
                                 dim3((unsigned)((g.M + GB - 1) / GB), (unsigned)((g.N + GB - 1) / GB),
                                      (unsigned)splits),
                                 dim3(GT), 0, st, 1, p);
      if (e != cudaSuccess) return e;
      const int64_t total = (int64_t)g.M * g.N;
      count_launch();
      return launch_pdl(split_sum_kernel,
                        dim3((unsigned)std::min<int64_t>((total + 255) / 256, 148 * 16)), dim3(256),
                        0, st, 1, (const float*)split_scratch, splits, g.M, g.N, g.C, g.ldc,
                        g.accumulate);
    }
  }
  dim3 grid;
  if (g.form == 1) grid = dim3((unsigned)max_tiles, (unsigned)((g.N + GB - 1) / GB), 1);
  else grid = dim3((unsigned)((g.M + GB - 1) / GB), (unsigned)((g.N + GB - 1) / GB),
                   g.form == 2 ? (unsigned)R : 1u);
  if (grid.x == 0 || grid.y == 0) return cudaSuccess;
  count_launch();
  return launch_pdl(kern, grid, dim3(GT), 0, st, 1, g);
}

__device__ __forceinline__ float sigmoid_b(float v) { return 1.0f / (1.0f + expf(-v)); }

// h = g(a) up(c) (forward), elementwise over n values.
__global__ void situ_fwd_kernel(const float* __restrict__ a, const float* __restrict__ c,
                                int64_t n, float b1, float b2, float* __restrict__ h) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    h[i] = b1 * tanhf(a[i] / b1) * sigmoid_b(a[i]) * b2 * tanhf(c[i] / b2);
}

// da = dh up(c) g'(a), dc = dh g(a) up'(c), written over a and c.
__global__ void situ_bwd_kernel(float* __restrict__ a, float* __restrict__ c,
                                const float* __restrict__ dh, int64_t n, float b1, float b2) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float tg = tanhf(a[i] / b1), sg = sigmoid_b(a[i]), tu = tanhf(c[i] / b2);
    const float gv = b1 * tg * sg, up = b2 * tu;
    const float dg = (1.0f - tg * tg) * sg + gv * (1.0f - sg);
    const float du = 1.0f - tu * tu;
    a[i] = dh[i] * up * dg;
    c[i] = dh[i] * gv * du;
  }
}

// Per token (a warp): u = sum_slot p o[inv], r = (mean u^2 + eps)^-1/2, uhat = u r w.
__global__ void combine_f32_kernel(const float* __restrict__ o, const int32_t* __restrict__ inv,
                                   const float* __restrict__ probs, const float* __restrict__ w,
                                   int64_t n, int k, int L, float eps, float* __restrict__ u,
                                   float* __restrict__ uhat, float* __restrict__ rr) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n) return;
  float ss = 0.0f;
  for (int j = lane; j < L; j += 32) {
    float v = 0.0f;
    for (int i = 0; i < k; ++i) v = fmaf(probs[t * k + i], o[(int64_t)inv[t * k + i] * L + j], v);
    u[t * L + j] = v;
    ss = fmaf(v, v, ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float r = rsqrtf(ss / (float)L + eps);
  for (int j = lane; j < L; j += 32) uhat[t * L + j] = u[t * L + j] * r * w[j];
  if (lane == 0) rr[t] = r;
}

// Per token (a warp): du = r w duhat - u r^3 / l <w duhat u>; then for each slot
// dp = <du, o[inv]> and dE[inv] = p du.
__global__ void rms_dp_kernel(const float* __restrict__ u, const float* __restrict__ duhat,
                              const float* __restrict__ rr, const float* __restrict__ w,
                              const float* __restrict__ o, const int32_t* __restrict__ inv,
                              const float* __restrict__ probs, int64_t n, int k, int L,
                              float* __restrict__ du, float* __restrict__ dp,
                              float* __restrict__ dE) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n) return;
  const float r = rr[t];
  float s = 0.0f;
  for (int j = lane; j < L; j += 32) s = fmaf(w[j] * duhat[t * L + j], u[t * L + j], s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float c3 = r * r * r / (float)L * s;
  for (int j = lane; j < L; j += 32) du[t * L + j] = r * w[j] * duhat[t * L + j] - u[t * L + j] * c3;
  __syncwarp();
  for (int i = 0; i < k; ++i) {
    const int64_t row = inv[t * k + i];
    const float p = probs[t * k + i];
    float d = 0.0f;
    for (int j = lane; j < L; j += 32) {
      const float g = du[t * L + j];
      d = fmaf(g, o[row * L + j], d);
      dE[row * L + j] = p * g;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    if (lane == 0) dp[t * k + i] = d;
  }
}

// RMSNorm weight gradient: part[b][j] = sum over block b's kRmsRows tokens of
// duhat u r (tokens in order), then drms[j] = sum_b part[b][j] (blocks in order).
__global__ void rms_dw_part_kernel(const float* __restrict__ u, const float* __restrict__ duhat,
                                   const float* __restrict__ rr, int64_t n, int L,
                                   float* __restrict__ part) {
  pdl_trigger();
  pdl_wait();
  const int64_t t0 = (int64_t)blockIdx.x * kRmsRows;
  const int64_t t1 = min(n, t0 + kRmsRows);
  for (int j = threadIdx.x; j < L; j += blockDim.x) {
    float acc = 0.0f;
    for (int64_t t = t0; t < t1; ++t) acc = fmaf(duhat[t * L + j] * u[t * L + j], rr[t], acc);
    part[(int64_t)blockIdx.x * L + j] = acc;
  }
}
__global__ void rms_dw_final_kernel(const float* __restrict__ part, int blocks, int L,
                                    float* __restrict__ drms) {
  pdl_trigger();
  pdl_wait();
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < L; j += gridDim.x * blockDim.x) {
    float acc = 0.0f;
    for (int b = 0; b < blocks; ++b) acc += part[(int64_t)b * L + j];
    drms[j] = acc;
  }
}

// Per token (a warp): the logit gradient row dl [R] (0 off the selected
// experts) from dp, p and the logits.
__global__ void router_bwd_kernel(const float* __restrict__ logits, int64_t ld,
                                  const int32_t* __restrict__ ids, const float* __restrict__ probs,
                                  const float* __restrict__ dp, int64_t n, int k, int R,
                                  int router, float* __restrict__ dl) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= n) return;
  for (int e = lane; e < R; e += 32) dl[t * R + e] = 0.0f;
  __syncwarp();
  if (lane == 0) {
    float pdp = 0.0f, ssum = 0.0f;
    for (int i = 0; i < k; ++i) {
      pdp = fmaf(probs[t * k + i], dp[t * k + i], pdp);
      ssum += sigmoid_b(logits[t * ld + ids[t * k + i]]);
    }
    for (int i = 0; i < k; ++i) {
      const int e = ids[t * k + i];
      float g;
      if (router == 1) {
        g = probs[t * k + i] * (dp[t * k + i] - pdp);
      } else {
        const float s = sigmoid_b(logits[t * ld + e]);
        const float ds = ssum >= 1e-9f ? (dp[t * k + i] - pdp) / ssum : dp[t * k + i] / 1e-9f;
        g = ds * s * (1.0f - s);
      }
      dl[t * R + e] = g;
    }
  }
}

// dz[t] = sum over slots of dzp[inv[t, slot]] (slots in order).
__global__ void gather_sum_kernel(const float* __restrict__ dzp, const int32_t* __restrict__ inv,
                                  int64_t n, int k, int L, float* __restrict__ dz) {
  pdl_trigger();
  pdl_wait();
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n * L) return;
  const int64_t t = i / L;
  const int j = (int)(i - t * L);
  float v = 0.0f;
  for (int s = 0; s < k; ++s) v += dzp[(int64_t)inv[t * k + s] * L + j];
  dz[i] = v;
}

unsigned grid_for(int64_t n, int threads) {
  return (unsigned)std::min<int64_t>((n + threads - 1) / threads, 148 * 32);
}

GemmDesc desc(const void* A, int a_bf16, int64_t sam, int64_t sak, const void* B, int b_bf16,
              int64_t sbk, int64_t sbn, float* C, int64_t ldc, int M, int N, int K,
              int accumulate = 0) {
  GemmDesc g;
  memset(&g, 0, sizeof(g));
  g.A = A; g.a_bf16 = a_bf16; g.sam = sam; g.sak = sak;
  g.B = B; g.b_bf16 = b_bf16; g.sbk = sbk; g.sbn = sbn;
  g.C = C; g.ldc = ldc; g.M = M; g.N = N; g.K = K; g.accumulate = accumulate;
  return g;
}

}  // namespace

// Sizes of the backward's scratch, in the order it is carved from the workspace.
BwdLayout bwd_layout(const BwdDims& d) {
  BwdLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t at = off; off += (bytes + 255) & ~(size_t)255; return at; };
  const int64_t N = d.N, P = d.N * d.k;
  L.ld_logits = (d.R + 15) / 16 * 16;
  L.max_tiles = (int)(P / kTileM + d.R + 1);
  L.header = take(256);
  L.logits = take((size_t)N * L.ld_logits * 4);
  L.ids = take((size_t)P * 4);
  L.probs = take((size_t)P * 4);
  L.counts = take((size_t)d.R * 4);
  L.offsets = take((size_t)(d.R + 1) * 4);
  L.perm = take((size_t)P * 4);
  L.inv = take((size_t)P * 4);
  L.block_counts = take((size_t)dispatch_blocks(P) * d.R * 4);
  L.tiles = take((size_t)L.max_tiles * 16);
  L.z = take((size_t)N * d.L * 4);
  L.zp = take((size_t)P * d.L * 4);
  L.a = take((size_t)P * d.F * 4);
  L.c = take((size_t)P * d.F * 4);
  L.h = take((size_t)P * d.F * 4);
  L.dh = take((size_t)P * d.F * 4);
  L.o = take((size_t)P * d.L * 4);
  L.dE = take((size_t)P * d.L * 4);
  L.u = take((size_t)N * d.L * 4);
  L.uhat = take((size_t)N * d.L * 4);
  L.duhat = take((size_t)N * d.L * 4);
  L.du = take((size_t)N * d.L * 4);
  L.rr = take((size_t)N * 4);
  L.dp = take((size_t)P * 4);
  L.dl = take((size_t)N * d.R * 4);
  L.rms_part = take((size_t)rms_blocks(N) * d.L * 4);
  L.ash = take((size_t)N * d.S * d.G * 4);
  L.csh = take((size_t)N * d.S * d.G * 4);
  L.hsh = take((size_t)N * d.S * d.G * 4);
  L.dhsh = take((size_t)N * d.S * d.G * 4);
  L.split = take((size_t)kSplitScratch * 4);
  L.total = off;
  return L;
}

cudaError_t run_backward(const BwdDims& d, const BwdArgs& a, void* ws, cudaStream_t st) {
  const BwdLayout L = bwd_layout(d);
  char* base = static_cast<char*>(ws);
  auto F32 = [&](size_t off) { return reinterpret_cast<float*>(base + off); };
  auto I32 = [&](size_t off) { return reinterpret_cast<int32_t*>(base + off); };
  const int64_t N = d.N, P = d.N * d.k;
  const int bf = d.bf16;
  const int Lt = d.L, D = d.d, R = d.R, F = d.F, S = d.S, G = d.G, k = d.k;
  int32_t* status = I32(L.header);
  int32_t* n_mtiles = I32(L.header) + 1;
  float* logits = F32(L.logits);
  int32_t* ids = I32(L.ids);
  float* probs = F32(L.probs);
  int32_t* offsets = I32(L.offsets);
  int32_t* perm = I32(L.perm);
  int32_t* inv = I32(L.inv);
  int4* tiles = reinterpret_cast<int4*>(base + L.tiles);
  float *z = F32(L.z), *zp = F32(L.zp), *pa = F32(L.a), *pc = F32(L.c), *h = F32(L.h), *dh = F32(L.dh);
  float *o = F32(L.o), *dE = F32(L.dE), *u = F32(L.u), *uhat = F32(L.uhat);
  float *duhat = F32(L.duhat), *du = F32(L.du), *rr = F32(L.rr), *dp = F32(L.dp);
  float *dl = F32(L.dl), *rms_part = F32(L.rms_part);
  float *ash = F32(L.ash), *csh = F32(L.csh), *hsh = F32(L.hsh), *dhsh = F32(L.dhsh);
  float* split = F32(L.split);
  const int64_t FL = (int64_t)F * Lt;
  cudaError_t e;
#define LMOE_STEP(call) do { if ((e = (call)) != cudaSuccess) return e; } while (0)
  // ---- forward, recomputed in fp32
  // bf16 operands: the contractions with x (z, the router logits and the shared
  // experts' gate / up pre-activations) are one tensor-core pass over x, exact
  // products with fp32 sums, that also routes as the forward does (the same
  // epilogue for R <= 32, else the same top-k kernel); fp32 operands: CUDA-core GEMMs
  const int SG = S * G;
  if (bf) {
    XpassArgs xa{};
    xa.x = static_cast<const __nv_bfloat16*>(a.x);
    xa.N = N;
    xa.d = D;
    xa.w_down = static_cast<const __nv_bfloat16*>(a.w_down);
    xa.L = Lt;
    xa.w_router = static_cast<const __nv_bfloat16*>(a.w_router);
    xa.R = R;
    xa.ws_g = static_cast<const __nv_bfloat16*>(a.ws_g);
    xa.ws_u = static_cast<const __nv_bfloat16*>(a.ws_u);
    xa.S = S;
    xa.G = G;
    xa.z32 = z;
    xa.logits = logits;
    xa.logits_ld = L.ld_logits;
    xa.a_sh = ash;
    xa.c_sh = csh;
    xa.beta1 = d.beta1;
    xa.beta2 = d.beta2;
    xa.router = d.router;
    xa.bias = a.bias;
    xa.ids = R <= 32 ? ids : nullptr;
    xa.probs = probs;
    xa.top_k = k;
    LMOE_STEP(umma_xpass(xa, status, st));
    if (R > 32)
      LMOE_STEP(launch_route_topk(logits, L.ld_logits, a.bias, N, R, k, d.router, ids, probs, st));
  } else {
    // router logits, then the same top-k kernel as the forward
    LMOE_STEP(gemm(desc(a.x, bf, D, 1, a.w_router, bf, 1, D, logits, L.ld_logits, (int)N, R, D),
                   0, R, st, split));
    LMOE_STEP(launch_route_topk(logits, L.ld_logits, a.bias, N, R, k, d.router, ids, probs, st));
  }
  DispatchScratch ds;
  ds.block_counts = I32(L.block_counts);
  ds.status = status;
  ds.n_mtiles = n_mtiles;
  ds.tiles = tiles;
  LMOE_STEP(launch_dispatch(ids, N, k, R, I32(L.counts), offsets, perm, inv, ds, st));
  // z = x W_down^T
  if (!bf)
    LMOE_STEP(gemm(desc(a.x, bf, D, 1, a.w_down, bf, 1, D, z, Lt, (int)N, Lt, D), 0, R, st, split));
  // zp = z[perm], the sorted rows; a, c = zp W_g,e^T, zp W_u,e^T on the routed tiles
  LMOE_STEP(launch_gather_rows<float>(z, perm, P, Lt, zp, st));
  {
    GemmDesc g = desc(zp, 0, Lt, 1, a.w_g, bf, 1, Lt, pa, F, 0, F, Lt);
    g.form = 1; g.tiles = tiles; g.n_tiles = n_mtiles; g.b_estride = FL;
    LMOE_STEP(gemm(g, L.max_tiles, R, st));
    g.B = a.w_u; g.C = pc;
    LMOE_STEP(gemm(g, L.max_tiles, R, st));
  }
  count_launch();
  LMOE_STEP(launch_pdl(situ_fwd_kernel, dim3(grid_for(P * F, 256)), dim3(256), 0, st, 1,
                       (const float*)pa, (const float*)pc, P * F, d.beta1, d.beta2, h));
  // o = h W_o,e^T
  {
    GemmDesc g = desc(h, 0, F, 1, a.w_o, bf, 1, F, o, Lt, 0, Lt, F);
    g.form = 1; g.tiles = tiles; g.n_tiles = n_mtiles; g.b_estride = FL;
    LMOE_STEP(gemm(g, L.max_tiles, R, st));
  }
  const unsigned warps_grid = (unsigned)((N + 7) / 8);
  count_launch();
  LMOE_STEP(launch_pdl(combine_f32_kernel, dim3(warps_grid), dim3(256), 0, st, 1,
                       (const float*)o, (const int32_t*)inv, (const float*)probs, a.rms_weight, N,
                       k, Lt, d.rms_eps, u, uhat, rr));
  // ---- step 5: y = s_sh + W_up uhat
  LMOE_STEP(gemm(desc(a.dy, bf, D, 1, a.w_up, bf, Lt, 1, duhat, Lt, (int)N, Lt, D), 0, R, st, split));
  LMOE_STEP(gemm(desc(a.dy, bf, 1, D, uhat, 0, Lt, 1, a.g.dw_up, Lt, D, Lt, (int)N), 0, R, st, split));
  // ---- RMSNorm, and the routing weights' and experts' output gradients
  count_launch();
  LMOE_STEP(launch_pdl(rms_dp_kernel, dim3(warps_grid), dim3(256), 0, st, 1, (const float*)u,
                       (const float*)duhat, (const float*)rr, a.rms_weight, (const float*)o,
                       (const int32_t*)inv, (const float*)probs, N, k, Lt, du, dp, dE));
  const int rb = rms_blocks(N);
  count_launch();
  LMOE_STEP(launch_pdl(rms_dw_part_kernel, dim3(rb), dim3(256), 0, st, 1, (const float*)u,
                       (const float*)duhat, (const float*)rr, N, Lt, rms_part));
  count_launch();
  LMOE_STEP(launch_pdl(rms_dw_final_kernel, dim3((Lt + 255) / 256), dim3(256), 0, st, 1,
                       (const float*)rms_part, rb, Lt, a.g.drms));
  // ---- routed experts
  {  // dh = dE W_o,e
    GemmDesc g = desc(dE, 0, Lt, 1, a.w_o, bf, F, 1, dh, F, 0, F, Lt);
    g.form = 1; g.tiles = tiles; g.n_tiles = n_mtiles; g.b_estride = FL;
    LMOE_STEP(gemm(g, L.max_tiles, R, st));
  }
  {  // dW_o,e = dE^T h over expert e's rows
    GemmDesc g = desc(dE, 0, 1, Lt, h, 0, F, 1, a.g.dw_o, F, Lt, F, 0);
    g.form = 2; g.offsets = offsets; g.c_estride = FL;
    LMOE_STEP(gemm(g, 0, R, st, split));
  }
  count_launch();
  LMOE_STEP(launch_pdl(situ_bwd_kernel, dim3(grid_for(P * F, 256)), dim3(256), 0, st, 1, pa, pc,
                       (const float*)dh, P * F, d.beta1, d.beta2));
  {  // dW_g,e = da^T zp, dW_u,e = dc^T zp
    GemmDesc g = desc(pa, 0, 1, F, zp, 0, Lt, 1, a.g.dw_g, Lt, F, Lt, 0);
    g.form = 2; g.offsets = offsets; g.c_estride = FL;
    LMOE_STEP(gemm(g, 0, R, st, split));
    g.A = pc; g.C = a.g.dw_u;
    LMOE_STEP(gemm(g, 0, R, st, split));
  }
  {  // dzp = da W_g,e + dc W_u,e (written over o)
    GemmDesc g = desc(pa, 0, F, 1, a.w_g, bf, Lt, 1, o, Lt, 0, Lt, F);
    g.form = 1; g.tiles = tiles; g.n_tiles = n_mtiles; g.b_estride = FL;
    LMOE_STEP(gemm(g, L.max_tiles, R, st));
    g.A = pc; g.B = a.w_u; g.accumulate = 1;
    LMOE_STEP(gemm(g, L.max_tiles, R, st));
  }
  count_launch();  // dz (written over du)
  LMOE_STEP(launch_pdl(gather_sum_kernel, dim3((unsigned)((N * Lt + 255) / 256)), dim3(256), 0,
                       st, 1, (const float*)o, (const int32_t*)inv, N, k, Lt, du));
  // ---- routing, through p
  count_launch();
  LMOE_STEP(launch_pdl(router_bwd_kernel, dim3(warps_grid), dim3(256), 0, st, 1,
                       (const float*)logits, (int64_t)L.ld_logits, (const int32_t*)ids,
                       (const float*)probs, (const float*)dp, N, k, R, d.router, dl));
  LMOE_STEP(gemm(desc(dl, 0, 1, R, a.x, bf, D, 1, a.g.dw_router, D, R, D, (int)N), 0, R, st, split));
  // ---- step 1
  LMOE_STEP(gemm(desc(du, 0, 1, Lt, a.x, bf, D, 1, a.g.dw_down, D, Lt, D, (int)N), 0, R, st, split));
  LMOE_STEP(gemm(desc(du, 0, Lt, 1, a.w_down, bf, D, 1, a.g.dx, D, (int)N, D, Lt), 0, R, st, split));
  LMOE_STEP(gemm(desc(dl, 0, R, 1, a.w_router, bf, D, 1, a.g.dx, D, (int)N, D, R, 1), 0, R, st, split));
  // ---- step 4: shared experts, dE = dy
  if (S > 0) {
    if (!bf) {
      LMOE_STEP(gemm(desc(a.x, bf, D, 1, a.ws_g, bf, 1, D, ash, SG, (int)N, SG, D), 0, R, st, split));
      LMOE_STEP(gemm(desc(a.x, bf, D, 1, a.ws_u, bf, 1, D, csh, SG, (int)N, SG, D), 0, R, st, split));
    }
    count_launch();
    LMOE_STEP(launch_pdl(situ_fwd_kernel, dim3(grid_for(N * SG, 256)), dim3(256), 0, st, 1,
                         (const float*)ash, (const float*)csh, N * SG, d.beta1, d.beta2, hsh));
    for (int j = 0; j < S; ++j) {
      const void* wo = bf ? (const void*)(static_cast<const __nv_bfloat16*>(a.ws_o) +
                                          (int64_t)j * D * G)
                          : (const void*)(static_cast<const float*>(a.ws_o) + (int64_t)j * D * G);
      // dh_sh,j = dy W_o,sh,j ;  dW_o,sh,j = dy^T h_sh,j
      LMOE_STEP(gemm(desc(a.dy, bf, D, 1, wo, bf, G, 1, dhsh + (int64_t)j * G, SG, (int)N, G, D),
                     0, R, st, split));
      LMOE_STEP(gemm(desc(a.dy, bf, 1, D, hsh + (int64_t)j * G, 0, SG, 1,
                          a.g.dws_o + (int64_t)j * D * G, G, D, G, (int)N),
                     0, R, st, split));
    }
    count_launch();
    LMOE_STEP(launch_pdl(situ_bwd_kernel, dim3(grid_for(N * SG, 256)), dim3(256), 0, st, 1, ash,
                         csh, (const float*)dhsh, N * SG, d.beta1, d.beta2));
    LMOE_STEP(gemm(desc(ash, 0, 1, SG, a.x, bf, D, 1, a.g.dws_g, D, SG, D, (int)N), 0, R, st, split));
    LMOE_STEP(gemm(desc(csh, 0, 1, SG, a.x, bf, D, 1, a.g.dws_u, D, SG, D, (int)N), 0, R, st, split));
    LMOE_STEP(gemm(desc(ash, 0, SG, 1, a.ws_g, bf, D, 1, a.g.dx, D, (int)N, D, SG, 1), 0, R, st, split));
    LMOE_STEP(gemm(desc(csh, 0, SG, 1, a.ws_u, bf, D, 1, a.g.dx, D, (int)N, D, SG, 1), 0, R, st, split));
  }
#undef LMOE_STEP
  return cudaGetLastError();
}

}  // namespace lmoe
