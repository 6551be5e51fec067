// CUDA-core (FFMA) GEMM with the LatentMoE epilogues.  This is the fp32
// path of the library: tcgen05 has no fp32 operand kind, and the fp32 mode
// must hold the oracle to 1e-5 relative.  The bf16 path uses the tcgen05
// engine (umma_gemm.cu) instead.
//
//   C[m, n] = sum_s sum_k A_s[m, k] * B_s[n, k]          (store mode)
//   C[m, n] = SiTU(A[m,:].B[n,:], A[m,:].B_up[n,:])     (SiTU mode, sec-07 SiTU formula)
// Row tiles come either from a dense range [0, M) or from the routed tile list
// (expert, first row, rows); in the latter case B advances by one expert's
// weight block per expert id.
#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T, bool SITU>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtGemm g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float Us[SITU ? BK : 1][SITU ? BN + 4 : 1];

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  int row_begin, row_end;
  int64_t b_off = 0;
  if (g.tiles != nullptr) {
    const int tile = blockIdx.x >> 1;
    if (tile >= *g.n_tiles) return;
    const int4 tl = g.tiles[tile];
    row_begin = tl.y + (blockIdx.x & 1) * BM;
    row_end = tl.y + tl.z;
    if (row_begin >= row_end) return;
    row_end = min(row_end, row_begin + BM);
    b_off = (int64_t)tl.x * g.b_expert_stride;
  } else {
    row_begin = blockIdx.x * BM;
    row_end = min(g.M, row_begin + BM);
  }
  const int col0 = blockIdx.y * BN;

  float acc[4][4], accu[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = accu[i][j] = 0.0f;

  for (int s = 0; s < g.nseg; ++s) {
    const T* A = static_cast<const T*>(g.A[s]);
    const T* B = static_cast<const T*>(g.B[s]) + b_off;
    const T* U = SITU ? static_cast<const T*>(g.B_up) + b_off : nullptr;
    const int64_t lda = g.lda[s], ldb = g.ldb[s];
    const int K = g.K[s];
    for (int k0 = 0; k0 < K; k0 += BK) {
      // 64 x 16 tiles: 1024 elements, 4 per thread
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int idx = threadIdx.x + q * 256;
        int r = idx >> 4, kk = idx & 15;
        int gr = row_begin + r, gk = k0 + kk;
        As[kk][r] = (gr < row_end && gk < K) ? to_f(A[(int64_t)gr * lda + gk]) : 0.0f;
        int gn = col0 + r;
        Bs[kk][r] = (gn < g.N && gk < K) ? to_f(B[(int64_t)gn * ldb + gk]) : 0.0f;
        if (SITU) Us[kk][r] = (gn < g.N && gk < K) ? to_f(U[(int64_t)gn * ldb + gk]) : 0.0f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        float a[4], b[4], u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          b[j] = Bs[kk][tx * 4 + j];
          if (SITU) u[j] = Us[kk][tx * 4 + j];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            if (SITU) accu[i][j] = fmaf(a[i], u[j], accu[i][j]);
          }
      }
      __syncthreads();
    }
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gr = row_begin + ty * 4 + i;
    if (gr >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = col0 + tx * 4 + j;
      if (gn >= g.N) continue;
      float v = SITU ? situ_exact(acc[i][j], accu[i][j], g.beta1, g.beta2) : acc[i][j];
      if (g.out_f32)
        static_cast<float*>(g.C)[(int64_t)gr * g.ldc + gn] = v;
      else
        static_cast<T*>(g.C)[(int64_t)gr * g.ldc + gn] = from_f<T>(v);
    }
  }
}

}  // namespace

template <typename T>
cudaError_t launch_simt_gemm(const SimtGemm& g, cudaStream_t st) {
  unsigned gx = g.tiles != nullptr ? (unsigned)(2 * g.max_tiles) : (unsigned)((g.M + BM - 1) / BM);
  unsigned gy = (unsigned)((g.N + BN - 1) / BN);
  if (gx == 0 || gy == 0) return cudaSuccess;
  if (g.mode == kSitu)
    simt_gemm_kernel<T, true><<<dim3(gx, gy), 256, 0, st>>>(g);
  else
    simt_gemm_kernel<T, false><<<dim3(gx, gy), 256, 0, st>>>(g);
  count_launch();
  return cudaGetLastError();
}
template cudaError_t launch_simt_gemm<float>(const SimtGemm&, cudaStream_t);
template cudaError_t launch_simt_gemm<__nv_bfloat16>(const SimtGemm&, cudaStream_t);

}  // namespace lmoe
