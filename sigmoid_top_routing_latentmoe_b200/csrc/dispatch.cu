// Pair permutation (kda/layers/latent_moe.py LatentMoE._routed_u; sec-07
// sparse dispatch, step 1): the N*k (token, expert) pairs, flattened
// token-major, are stably sorted by expert id -- the pages' argsort(stable) +
// bincount + cumsum -- as a deterministic three-pass counting sort:
//   1. per-block histograms of a fixed chunk of pairs,
//   2. one block scans them (per expert over blocks, then over experts) into
//      counts, offsets and each block's starting slot per expert, and writes
//      the routed row-tile list (expert, first row, rows) used by the GEMMs,
//   3. each block ranks its pairs in pair order inside each expert and
//      scatters perm_token / inv_pair.
// No step depends on atomic ordering, so the output is bit-exact.
#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

constexpr int kChunk = 4096;       // pairs per block
constexpr int kThreads = 256;      // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kPerWarp = kChunk / kWarps;  // 512 pairs, walked 32 at a time

__global__ void __launch_bounds__(kThreads) hist_kernel(const int32_t* __restrict__ ids,
                                                        int64_t n_pairs, int R,
                                                        int32_t* __restrict__ block_counts,
                                                        int32_t* __restrict__ status) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < R; e += kThreads) hist[e] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk;
  for (int j = threadIdx.x; j < kChunk; j += kThreads) {
    int64_t p = base + j;
    if (p < n_pairs) {
      int e = ids[p];
      if ((unsigned)e < (unsigned)R)
        atomicAdd(&hist[e], 1);
      else
        record_status(status, kStatusDevice);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < R; e += kThreads)
    block_counts[(int64_t)blockIdx.x * R + e] = hist[e];
}

// Single block.  block_counts[b, e] becomes the first sorted slot of block b's
// pairs of expert e.
__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ block_counts,
                                                    int n_blocks, int R, int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ n_mtiles,
                                                    int4* __restrict__ tiles) {
  extern __shared__ int32_t sm[];  // [R] counts, then [R] tile starts
  int32_t* cnt = sm;
  int32_t* tstart = sm + R;
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry[2];
  // per-expert exclusive scan over blocks
  for (int e = threadIdx.x; e < R; e += blockDim.x) {
    int32_t run = 0;
    for (int b = 0; b < n_blocks; ++b) {
      int32_t c = block_counts[(int64_t)b * R + e];
      block_counts[(int64_t)b * R + e] = run;
      run += c;
    }
    cnt[e] = run;
  }
  if (threadIdx.x == 0) { carry[0] = 0; carry[1] = 0; }
  __syncthreads();
  // exclusive scan over experts of counts (-> offsets) and of tile counts
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int base = 0; base < R; base += blockDim.x) {
    int e = base + threadIdx.x;
    int32_t c = (e < R) ? cnt[e] : 0;
    int32_t nt = (c + kTileM - 1) / kTileM;
    // scan pair counts
    for (int pass = 0; pass < 2; ++pass) {
      int32_t v = pass == 0 ? c : nt;
      int32_t inc = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int32_t o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
      }
      if (lane == 31) warp_sums[warp] = inc;
      __syncthreads();
      if (warp == 0) {
        int32_t ws = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          int32_t o = __shfl_up_sync(0xffffffffu, ws, off);
          if (lane >= off) ws += o;
        }
        if (lane < nw) warp_sums[lane] = ws;  // inclusive over warps
      }
      __syncthreads();
      int32_t excl = inc - v + (warp > 0 ? warp_sums[warp - 1] : 0) + carry[pass];
      if (e < R) {
        if (pass == 0) {
          offsets[e] = excl;
          counts[e] = c;
        } else {
          tstart[e] = excl;
        }
      }
      __syncthreads();
      if (threadIdx.x == blockDim.x - 1) carry[pass] = excl + v;
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) {
    offsets[R] = carry[0];
    *n_mtiles = carry[1];
  }
  __syncthreads();
  // tile list: expert e owns tiles [tstart[e], tstart[e] + ceil(cnt/128))
  for (int e = warp; e < R; e += nw) {
    int32_t c = cnt[e];
    int32_t nt = (c + kTileM - 1) / kTileM;
    int32_t off = offsets[e];
    for (int j = lane; j < nt; j += 32) {
      int32_t rows = min(kTileM, c - j * kTileM);
      tiles[tstart[e] + j] = make_int4(e, off + j * kTileM, rows, 0);
    }
  }
}

__global__ void __launch_bounds__(kThreads) scatter_kernel(const int32_t* __restrict__ ids,
                                                           int64_t n_pairs, int k, int R,
                                                           const int32_t* __restrict__ block_first,
                                                           const int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ perm_token,
                                                           int32_t* __restrict__ inv_pair) {
  extern __shared__ int32_t wcnt[];  // [kWarps][R]: per-warp counts, then running slots
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kWarps * R; i += kThreads) wcnt[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kChunk + (int64_t)warp * kPerWarp;
  // pass 1: per-warp histogram of its contiguous sub-range
  for (int j = lane; j < kPerWarp; j += 32) {
    int64_t p = base + j;
    if (p < n_pairs) {
      int e = ids[p];
      if ((unsigned)e < (unsigned)R) atomicAdd(&wcnt[warp * R + e], 1);
    }
  }
  __syncthreads();
  // pass 2: first slot of each warp's pairs of expert e
  for (int e = threadIdx.x; e < R; e += kThreads) {
    int32_t run = offsets[e] + block_first[(int64_t)blockIdx.x * R + e];
    for (int w = 0; w < kWarps; ++w) {
      int32_t c = wcnt[w * R + e];
      wcnt[w * R + e] = run;
      run += c;
    }
  }
  __syncthreads();
  // pass 3: walk the sub-range in pair order, 32 pairs at a time
  for (int j0 = 0; j0 < kPerWarp; j0 += 32) {
    int64_t p = base + j0 + lane;
    bool valid = p < n_pairs;
    int e = valid ? ids[p] : -1;
    valid = valid && (unsigned)e < (unsigned)R;
    unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1 - lane);
    unsigned lower = same & ((1u << lane) - 1u);
    int32_t slot = 0;
    if (valid) slot = wcnt[warp * R + e] + __popc(lower);
    __syncwarp();
    if (valid && lower == 0) wcnt[warp * R + e] += __popc(same);
    __syncwarp();
    if (valid) {
      perm_token[slot] = (int32_t)(p / k);
      inv_pair[p] = slot;
    }
  }
}

template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ z, const int32_t* __restrict__ perm_token,
                                   int64_t n_rows, int width, T* __restrict__ zp) {
  // one warp per row, 16-byte vectors
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= n_rows) return;
  const int64_t src = perm_token[r];
  const int vec = 16 / sizeof(T);
  const uint4* s = reinterpret_cast<const uint4*>(z + src * width);
  uint4* d = reinterpret_cast<uint4*>(zp + r * width);
  for (int i = lane; i < width / vec; i += 32) d[i] = s[i];
}

// Tile list from offsets alone (for moe_expert_ffn called on its own).  One
// warp: each lane scans a contiguous run of experts.
__global__ void build_tiles_kernel(const int32_t* __restrict__ offsets, int R,
                                   int32_t* __restrict__ n_mtiles, int4* __restrict__ tiles) {
  const int lane = threadIdx.x;
  const int per = (R + 31) / 32;
  const int e0 = min(R, lane * per), e1 = min(R, e0 + per);
  int32_t mine = 0;
  for (int e = e0; e < e1; ++e) mine += (offsets[e + 1] - offsets[e] + kTileM - 1) / kTileM;
  int32_t inc = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int32_t o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  int32_t t = inc - mine;
  for (int e = e0; e < e1; ++e) {
    const int32_t off = offsets[e], c = offsets[e + 1] - off;
    for (int j = 0; j * kTileM < c; ++j) tiles[t++] = make_int4(e, off + j * kTileM, min(kTileM, c - j * kTileM), 0);
  }
  if (lane == 31) *n_mtiles = inc;
}

}  // namespace

cudaError_t launch_build_tiles(const int32_t* offsets, int R, int32_t* n_mtiles, int4* tiles,
                               cudaStream_t st) {
  build_tiles_kernel<<<1, 32, 0, st>>>(offsets, R, n_mtiles, tiles);
  count_launch();
  return cudaGetLastError();
}

int dispatch_blocks(int64_t n_pairs) { return (int)((n_pairs + kChunk - 1) / kChunk); }

cudaError_t launch_dispatch(const int32_t* ids, int64_t n, int k, int R, int32_t* counts,
                            int32_t* offsets, int32_t* perm_token, int32_t* inv_pair,
                            const DispatchScratch& s, cudaStream_t st) {
  const int64_t n_pairs = n * k;
  const int nb = dispatch_blocks(n_pairs);
  if (nb > 0) {
    hist_kernel<<<nb, kThreads, R * sizeof(int32_t), st>>>(ids, n_pairs, R, s.block_counts,
                                                           s.status);
    count_launch();
  }
  scan_kernel<<<1, 1024, 2 * R * sizeof(int32_t), st>>>(s.block_counts, nb, R, counts, offsets,
                                                        s.n_mtiles, s.tiles);
  count_launch();
  if (nb > 0) {
    size_t smem = (size_t)kWarps * R * sizeof(int32_t);
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
    }
    scatter_kernel<<<nb, kThreads, smem, st>>>(ids, n_pairs, k, R, s.block_counts, offsets,
                                               perm_token, inv_pair);
    count_launch();
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gather_rows(const T* z, const int32_t* perm_token, int64_t n_rows, int width,
                               T* zp, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  const int warps = 8;
  gather_rows_kernel<T><<<(unsigned)((n_rows + warps - 1) / warps), warps * 32, 0, st>>>(
      z, perm_token, n_rows, width, zp);
  count_launch();
  return cudaGetLastError();
}
template cudaError_t launch_gather_rows<float>(const float*, const int32_t*, int64_t, int, float*,
                                               cudaStream_t);
template cudaError_t launch_gather_rows<__nv_bfloat16>(const __nv_bfloat16*, const int32_t*,
                                                       int64_t, int, __nv_bfloat16*, cudaStream_t);

}  // namespace lmoe
