// Pair permutation (kda/layers/latent_moe.py LatentMoE._routed_u; sec-07
// sparse dispatch, step 1): the N*k (token, expert) pairs, flattened
// token-major, are stably sorted by expert id -- the pages' argsort(stable) +
// bincount + cumsum -- as a deterministic counting sort over chunks of pairs:
//   1. hist:    one CTA per chunk counts its pairs per expert (skipped when
//               the x-pass's routing epilogue already wrote the expert
//               counts of every 32 tokens: R <= 32),
//   2. colscan: (large count matrices only) one CTA per 32 experts turns
//               each expert's column of chunk counts into exclusive prefixes
//               and the expert's total,
//   3. scatter: one CTA per chunk derives each expert's first sorted slot for
//               its chunk (offsets = exclusive scan of the totals), ranks its
//               pairs in pair order inside each expert and writes perm_token /
//               inv_pair; CTA 0 also writes counts, offsets and the routed
//               row-tile list (expert, first row, rows) the GEMMs walk.
// No result depends on the order of atomic operations: bit-exact.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "launch.h"

namespace lmoe {
namespace {

constexpr int kThreads = 256;  // 8 warps per chunk
constexpr int kWarps = kThreads / 32;
constexpr int kMaxChunks = 128;

// Pairs per chunk: at least 256 (one 32-pair step per warp), and large enough
// that there are at most kMaxChunks chunks.
int64_t chunk_pairs(int64_t n_pairs) {
  const int64_t per = (n_pairs + kMaxChunks - 1) / kMaxChunks;
  const int64_t step = 32 * kWarps;
  return std::max<int64_t>(step, (per + step - 1) / step * step);
}

// Block-wide exclusive scan of one value per thread; *total gets the sum.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_sums,
                                                        int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
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
    if (lane < nw) warp_sums[lane] = ws;
    if (lane == nw - 1) *total = ws;
  }
  __syncthreads();
  const int32_t excl = inc - v + (warp > 0 ? warp_sums[warp - 1] : 0);
  __syncthreads();
  return excl;
}

// Chunk-count matrices up to this many ints are scanned inside the scatter
// kernel (every CTA walks the columns it needs); larger ones get a column-scan
// kernel first.
constexpr int kSmallScan = 8192;

// One CTA per chunk counts the chunk's pairs per expert.
__global__ void __launch_bounds__(kThreads) hist_kernel(const int32_t* __restrict__ ids,
                                                        int64_t n_pairs, int64_t chunk, int R,
                                                        int32_t* __restrict__ chunk_counts,
                                                        int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < R; e += kThreads) hist[e] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t per_warp = chunk / kWarps;
  const int64_t p0 = (int64_t)blockIdx.x * chunk + warp * per_warp;
  const int64_t p1 = min(n_pairs, p0 + per_warp);
  for (int64_t q = p0; q < p1; q += 32) {
    const int64_t p = q + lane;
    int e = p < p1 ? ids[p] : -1;
    if (p < p1 && (unsigned)e >= (unsigned)R) {
      record_status(status, kStatusDevice);
      e = -1;
    }
    // one shared-memory add per distinct expert among the warp's 32 pairs
    const unsigned same = __match_any_sync(0xffffffffu, e < 0 ? -1 - lane : e);
    if (e >= 0 && (same & ((1u << lane) - 1u)) == 0) atomicAdd(&hist[e], __popc(same));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < R; e += kThreads)
    chunk_counts[(int64_t)blockIdx.x * R + e] = hist[e];
}

// Large count matrices: one CTA per 32 experts turns each column of chunk
// counts into its exclusive prefix over the chunks (in place) and writes the
// expert's total.  The block is staged in smem (rows padded to 33 ints); a
// warp scans one expert with each lane owning consecutive chunks.
__global__ void __launch_bounds__(kThreads) colscan_kernel(int32_t* __restrict__ chunk_counts,
                                                           int C, int R,
                                                           int32_t* __restrict__ counts) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t col[kMaxChunks][33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e0 = blockIdx.x * 32;
  const bool in = e0 + lane < R;
  for (int c = warp; c < C; c += kWarps)
    col[c][lane] = in ? chunk_counts[(int64_t)c * R + e0 + lane] : 0;
  __syncthreads();
  const int per = (C + 31) / 32;  // chunks per lane (<= 4)
  for (int j = warp; j < 32; j += kWarps) {
    const int c0 = lane * per;
    int32_t s = 0;
    for (int i = 0; i < per; ++i)
      if (c0 + i < C) s += col[c0 + i][j];
    int32_t inc = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t o = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += o;
    }
    int32_t run = inc - s;
    for (int i = 0; i < per; ++i)
      if (c0 + i < C) {
        const int32_t v = col[c0 + i][j];
        col[c0 + i][j] = run;
        run += v;
      }
    const int32_t total = __shfl_sync(0xffffffffu, inc, 31);
    if (lane == 0 && e0 + j < R) counts[e0 + j] = total;
  }
  __syncthreads();
  for (int c = warp; c < C; c += kWarps)
    if (in) chunk_counts[(int64_t)c * R + e0 + lane] = col[c][lane];
}

// No pairs at all: every count and offset is zero, no tiles.
__global__ void empty_scan_kernel(int R, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                  int32_t* __restrict__ n_mtiles) {
  pdl_trigger();
  pdl_wait();
  for (int e = threadIdx.x; e <= R; e += blockDim.x) {
    if (e < R) counts[e] = 0;
    offsets[e] = 0;
  }
  if (threadIdx.x == 0) *n_mtiles = 0;
}

// Ranks each chunk's pairs inside their expert in pair order and scatters.
// Prologue: every CTA derives, for each expert, its chunk's first sorted slot
// -- offsets[e] (an exclusive scan of the per-expert totals) plus the pairs of
// expert e in earlier chunks -- from the count rows: summed here when
// `prefixed` is 0, or read as the column scan left them.  The count rows are
// the histogram's (one per chunk, sub_rows = 1) or the x-pass's (one per 32
// tokens, sub_rows of them per chunk); crows rows in all.  CTA 0 also writes
// counts (unless prefixed), offsets and the routed row-tile list.
// With z != nullptr each chunk has `subs` CTAs: all of them rank the chunk's
// pairs (cheap), sub-CTA 0 writes perm_token / inv_pair, and sub-CTA s copies
// the z rows of the pairs whose index is s modulo subs to their sorted slots in
// zp (row_vecs 16-byte vectors per row), a warp's rows copied together so that
// many loads are in flight.
__global__ void __launch_bounds__(kThreads) scatter_kernel(
    const int32_t* __restrict__ ids, int64_t n_pairs, int64_t chunk, int k, int R, int crows,
    int sub_rows, const int32_t* __restrict__ chunk_counts, int prefixed,
    int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ n_mtiles, int4* __restrict__ tiles,
    int32_t* __restrict__ perm_token, int32_t* __restrict__ inv_pair, int subs,
    const uint4* __restrict__ z, uint4* __restrict__ zp, int row_vecs, int tile_m) {
  pdl_trigger();
  pdl_wait();
  // [kWarps][R] per-warp counts, then first slots; [R] this chunk's first slot
  extern __shared__ int32_t wcnt[];
  int32_t* base = wcnt + kWarps * R;
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t totals[2];
  __shared__ int32_t carry[2];
  __shared__ int32_t row_slot[kWarps][32], row_tok[kWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cb = blockIdx.x / subs, sub = blockIdx.x - cb * subs;
  for (int i = threadIdx.x; i < kWarps * R; i += kThreads) wcnt[i] = 0;
  if (threadIdx.x == 0) carry[0] = carry[1] = 0;
  const int lim = cb * sub_rows;  // count rows before this chunk
  // R <= 32: warp w sums rows w, w + 8, ... (lane = expert), then the warps'
  // partial sums are added per expert
  __shared__ int32_t part[2][kWarps][32];
  const bool by_warps = !prefixed && R <= 32;
  if (by_warps) {
    int32_t f = 0, t = 0;
    if (lane < R) {
      for (int c0 = warp; c0 < crows; c0 += kWarps * 16) {  // 16 loads in flight
        int32_t v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int c = c0 + u * kWarps;
          v[u] = c < crows ? chunk_counts[(int64_t)c * R + lane] : 0;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          f += c0 + u * kWarps < lim ? v[u] : 0;
          t += v[u];
        }
      }
    }
    part[0][warp][lane] = f;
    part[1][warp][lane] = t;
  }
  __syncthreads();
  for (int e0 = 0; e0 < R; e0 += kThreads) {
    const int e = e0 + threadIdx.x;
    int32_t first = 0, tot = 0;
    if (e < R) {
      if (prefixed) {
        first = chunk_counts[(int64_t)cb * R + e];
        tot = counts[e];
      } else if (by_warps) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          first += part[0][w][e];
          tot += part[1][w][e];
        }
      } else {
        for (int c0 = 0; c0 < crows; c0 += 32) {  // up to 32 loads in flight
          int32_t v[32];
#pragma unroll
          for (int u = 0; u < 32; ++u)
            v[u] = c0 + u < crows ? chunk_counts[(int64_t)(c0 + u) * R + e] : 0;
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            first += c0 + u < lim ? v[u] : 0;
            tot += v[u];
          }
        }
      }
    }
    const int32_t nt = (tot + tile_m - 1) / tile_m;
    const int32_t ex_c = block_exclusive_scan(tot, warp_sums, &totals[0]) + carry[0];
    const int32_t ex_t = block_exclusive_scan(nt, warp_sums, &totals[1]) + carry[1];
    if (e < R) {
      base[e] = ex_c + first;
      if (cb == 0 && sub == 0) {
        if (!prefixed) counts[e] = tot;
        offsets[e] = ex_c;
        for (int t = 0; t * tile_m < tot; ++t)
          tiles[ex_t + t] = make_int4(e, ex_c + t * tile_m, min(tile_m, tot - t * tile_m), 0);
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      carry[0] += totals[0];
      carry[1] += totals[1];
    }
    __syncthreads();
  }
  if (cb == 0 && sub == 0 && threadIdx.x == 0) {
    offsets[R] = carry[0];
    *n_mtiles = carry[1];
  }
  const int64_t per_warp = chunk / kWarps;
  const int64_t p0 = (int64_t)cb * chunk + warp * per_warp;
  const int64_t p1 = min(n_pairs, p0 + per_warp);
  int32_t* my = wcnt + warp * R;
  // pass 1: this warp's counts per expert (only this warp writes its row)
  for (int64_t q = p0; q < p1; q += 32) {
    const int64_t p = q + lane;
    const int e = p < p1 ? ids[p] : -1;
    const bool valid = (unsigned)e < (unsigned)R;
    const unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1 - lane);
    if (valid && (same & ((1u << lane) - 1u)) == 0) my[e] += __popc(same);
  }
  __syncthreads();
  // pass 2: first sorted slot of each warp's pairs of expert e
  for (int e = threadIdx.x; e < R; e += kThreads) {
    int32_t run = base[e];
    for (int w = 0; w < kWarps; ++w) {
      const int32_t c = wcnt[w * R + e];
      wcnt[w * R + e] = run;
      run += c;
    }
  }
  __syncthreads();
  // pass 3: walk the warp's pairs in order, 32 at a time
  for (int64_t q = p0; q < p1; q += 32) {
    const int64_t p = q + lane;
    const int e = p < p1 ? ids[p] : -1;
    const bool valid = (unsigned)e < (unsigned)R;
    const unsigned same = __match_any_sync(0xffffffffu, valid ? e : -1 - lane);
    const unsigned lower = same & ((1u << lane) - 1u);
    int32_t slot = -1;
    if (valid) slot = my[e] + __popc(lower);
    __syncwarp();
    if (valid && lower == 0) my[e] += __popc(same);
    __syncwarp();
    const int32_t tok = (int32_t)((uint32_t)p / (uint32_t)k);  // pairs < 2^31
    if (valid && sub == 0) {
      perm_token[slot] = tok;
      inv_pair[p] = slot;
    } else if (!valid && p < p1 && sub == 0) {
      inv_pair[p] = -1;  // an out-of-range id: the pair takes no slot
    }
    if (z != nullptr) {
      // this sub-CTA's rows of the step: pairs p with p mod subs == sub
      const bool mine = valid && (int)(p % subs) == sub;
      const unsigned sel = __ballot_sync(0xffffffffu, mine);
      const int at = __popc(sel & ((1u << lane) - 1u));
      if (mine) {
        row_slot[warp][at] = slot;
        row_tok[warp][at] = tok;
      }
      __syncwarp();
      const int n_vec = __popc(sel) * row_vecs;
      for (int i0 = 0; i0 < n_vec; i0 += 32 * 8) {  // 8 loads in flight per lane
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * 32 + lane;
          if (i < n_vec) {
            const int r = i / row_vecs, c = i - r * row_vecs;
            v[u] = z[(int64_t)row_tok[warp][r] * row_vecs + c];
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * 32 + lane;
          if (i < n_vec) {
            const int r = i / row_vecs, c = i - r * row_vecs;
            zp[(int64_t)row_slot[warp][r] * row_vecs + c] = v[u];
          }
        }
      }
      __syncwarp();
    }
  }
}

template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ z, const int32_t* __restrict__ perm_token,
                                   int64_t n_rows, int width, T* __restrict__ zp) {
  pdl_trigger();
  pdl_wait();
  // one warp per row, 16-byte vectors: up to 8 loads per lane in flight
  // before their stores; the sorted copy is written once and read once by
  // routed GEMM1, so its stores stream past L2 (st.global.cs)
  constexpr int U = 8;
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= n_rows) return;
  const int64_t src = perm_token[r];
  const int nv = width / (int)(16 / sizeof(T));
  const uint4* s = reinterpret_cast<const uint4*>(z + src * width);
  uint4* d = reinterpret_cast<uint4*>(zp + r * width);
  for (int i0 = lane; i0 < nv; i0 += 32 * U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (i0 + 32 * u < nv) v[u] = __ldg(s + i0 + 32 * u);
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (i0 + 32 * u < nv) __stcs(d + i0 + 32 * u, v[u]);
  }
}

// Consistency check of a permutation: ids in range, counts summing to N k,
// offsets the exclusive sum of counts, inv_pair a bijection onto the sorted
// slots (a bitmap, every slot set exactly once), perm_token[inv_pair[t, i]] = t,
// slots of expert e inside [offsets[e], offsets[e+1]) and tokens ascending
// inside an expert.  A violation sets kStatusDevice in the status word.
__global__ void check_counts_kernel(const int32_t* __restrict__ counts,
                                    const int32_t* __restrict__ offsets, int R, int64_t n_pairs,
                                    int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  if (threadIdx.x != 0) return;
  int64_t run = 0;
  bool bad = offsets[0] != 0;
  for (int e = 0; e < R; ++e) {
    if (counts[e] < 0 || offsets[e + 1] - offsets[e] != counts[e]) bad = true;
    run += counts[e];
  }
  if (run != n_pairs || offsets[R] != n_pairs) bad = true;
  if (bad) record_status(status, kStatusDevice);
}
__global__ void check_pairs_kernel(const int32_t* __restrict__ ids,
                                   const int32_t* __restrict__ offsets,
                                   const int32_t* __restrict__ perm_token,
                                   const int32_t* __restrict__ inv_pair, int64_t n_pairs, int k,
                                   int R, uint32_t* __restrict__ bitmap,
                                   int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < n_pairs;
       p += (int64_t)gridDim.x * blockDim.x) {
    const int e = ids[p];
    const int64_t slot = inv_pair[p];
    const int32_t t = (int32_t)(p / k);
    bool bad = (unsigned)e >= (unsigned)R || slot < 0 || slot >= n_pairs;
    if (!bad) {
      bad = perm_token[slot] != t || slot < offsets[e] || slot >= offsets[e + 1];
      // tokens ascend inside an expert: the next slot of the same expert holds a later token
      if (!bad && slot + 1 < offsets[e + 1] && slot + 1 < n_pairs && perm_token[slot + 1] <= t)
        bad = true;
      const uint32_t bit = 1u << (slot & 31);
      if (!bad && (atomicOr(&bitmap[slot >> 5], bit) & bit)) bad = true;  // slot taken twice
    }
    if (bad) record_status(status, kStatusDevice);
  }
}
__global__ void check_bitmap_kernel(const uint32_t* __restrict__ bitmap, int64_t n_pairs,
                                    int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < (n_pairs + 31) / 32;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t left = n_pairs - w * 32;
    const uint32_t want = left >= 32 ? 0xffffffffu : ((1u << left) - 1u);
    if (bitmap[w] != want) record_status(status, kStatusDevice);  // a slot nobody maps to
  }
}

// Tile list from offsets alone (for moe_expert_ffn called on its own).  One
// warp: each lane scans a contiguous run of experts.
__global__ void build_tiles_kernel(const int32_t* __restrict__ offsets, int R, int tile_m,
                                   int32_t* __restrict__ n_mtiles, int4* __restrict__ tiles) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x;
  const int per = (R + 31) / 32;
  const int e0 = min(R, lane * per), e1 = min(R, e0 + per);
  int32_t mine = 0;
  for (int e = e0; e < e1; ++e) mine += (offsets[e + 1] - offsets[e] + tile_m - 1) / tile_m;
  int32_t inc = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int32_t o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  int32_t t = inc - mine;
  for (int e = e0; e < e1; ++e) {
    const int32_t off = offsets[e], c = offsets[e + 1] - off;
    for (int j = 0; j * tile_m < c; ++j)
      tiles[t++] = make_int4(e, off + j * tile_m, min(tile_m, c - j * tile_m), 0);
  }
  if (lane == 31) *n_mtiles = inc;
}

template <typename K>
cudaError_t set_smem(K* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

int dispatch_blocks(int64_t n_pairs) {
  const int64_t chunk = chunk_pairs(n_pairs);
  return (int)((n_pairs + chunk - 1) / chunk);
}

bool dispatch_takes_row_counts(int64_t n, int k, int R) {
  const int64_t n_pairs = n * k;
  if (n_pairs == 0 || R > 32) return false;
  const int64_t rows = (n + kCountRowTokens - 1) / kCountRowTokens;
  return chunk_pairs(n_pairs) % ((int64_t)kCountRowTokens * k) == 0 && rows * R <= kSmallScan;
}

int64_t dispatch_count_rows(int64_t n, int k) {
  return std::max<int64_t>(dispatch_blocks(n * k), (n + kCountRowTokens - 1) / kCountRowTokens);
}

cudaError_t launch_dispatch(const int32_t* ids, int64_t n, int k, int R, int32_t* counts,
                            int32_t* offsets, int32_t* perm_token, int32_t* inv_pair,
                            const DispatchScratch& s, cudaStream_t st, const void* z, void* zp,
                            int row_bytes, int tile_m, bool row_counts) {
  const int64_t n_pairs = n * k;
  const int64_t chunk = chunk_pairs(n_pairs);
  const int nb = dispatch_blocks(n_pairs);
  if (nb == 0) {
    count_launch();
    return launch_pdl(empty_scan_kernel, dim3(1), dim3(32), 0, st, 1, R, counts, offsets,
                      s.n_mtiles);
  }
  if (row_counts && !dispatch_takes_row_counts(n, k, R)) return cudaErrorInvalidValue;
  cudaError_t e = cudaSuccess;
  int crows = nb, sub_rows = 1;
  if (row_counts) {
    crows = (int)((n + kCountRowTokens - 1) / kCountRowTokens);
    sub_rows = (int)(chunk / ((int64_t)kCountRowTokens * k));
  } else {
    e = set_smem(hist_kernel, R * sizeof(int32_t));
    if (e != cudaSuccess) return e;
    count_launch();
    e = launch_pdl(hist_kernel, dim3(nb), dim3(kThreads), R * sizeof(int32_t), st, 1, ids,
                   n_pairs, chunk, R, s.block_counts, s.status);
    if (e != cudaSuccess) return e;
  }
  const int prefixed = !row_counts && (int64_t)nb * R > kSmallScan ? 1 : 0;
  if (prefixed) {
    count_launch();
    e = launch_pdl(colscan_kernel, dim3((R + 31) / 32), dim3(kThreads), 0, st, 1, s.block_counts,
                   nb, R, counts);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = (size_t)(kWarps + 1) * R * sizeof(int32_t);
  e = set_smem(scatter_kernel, smem);
  if (e != cudaSuccess) return e;
  // with the row copy: enough CTAs per chunk to cover the SMs twice (at most 16)
  const int subs = z != nullptr ? std::max(1, std::min(16, (2 * 148 + nb - 1) / nb)) : 1;
  count_launch();
  e = launch_pdl(scatter_kernel, dim3((unsigned)(nb * subs)), dim3(kThreads), smem, st, 1, ids,
                 n_pairs, chunk, k, R, crows, sub_rows, (const int32_t*)s.block_counts, prefixed,
                 counts,
                 offsets, s.n_mtiles, s.tiles, perm_token, inv_pair, subs,
                 static_cast<const uint4*>(z), static_cast<uint4*>(zp), row_bytes / 16, tile_m);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}


cudaError_t launch_check_dispatch(const int32_t* ids, int64_t n, int k, int R,
                                  const int32_t* counts, const int32_t* offsets,
                                  const int32_t* perm_token, const int32_t* inv_pair,
                                  uint32_t* bitmap, int32_t* status, cudaStream_t st) {
  const int64_t n_pairs = n * k;
  cudaError_t e = cudaMemsetAsync(bitmap, 0, (size_t)((n_pairs + 31) / 32) * 4, st);
  if (e != cudaSuccess) return e;
  count_launch();
  e = launch_pdl(check_counts_kernel, dim3(1), dim3(32), 0, st, 1, counts, offsets, R, n_pairs,
                 status);
  if (e != cudaSuccess || n_pairs == 0) return e;
  const unsigned blocks = (unsigned)std::min<int64_t>((n_pairs + 255) / 256, 148 * 8);
  count_launch();
  e = launch_pdl(check_pairs_kernel, dim3(blocks), dim3(256), 0, st, 1, ids, offsets, perm_token,
                 inv_pair, n_pairs, k, R, bitmap, status);
  if (e != cudaSuccess) return e;
  count_launch();
  return launch_pdl(check_bitmap_kernel, dim3(blocks), dim3(256), 0, st, 1, (const uint32_t*)bitmap,
                    n_pairs, status);
}

cudaError_t launch_build_tiles(const int32_t* offsets, int R, int32_t* n_mtiles, int4* tiles,
                               cudaStream_t st, int tile_m) {
  count_launch();
  return launch_pdl(build_tiles_kernel, dim3(1), dim3(32), 0, st, 1, offsets, R, tile_m, n_mtiles,
                    tiles);
}

template <typename T>
cudaError_t launch_gather_rows(const T* z, const int32_t* perm_token, int64_t n_rows, int width,
                               T* zp, cudaStream_t st) {
  if (n_rows == 0) return cudaSuccess;
  const int warps = 8;
  count_launch();
  return launch_pdl(gather_rows_kernel<T>, dim3((unsigned)((n_rows + warps - 1) / warps)),
                    dim3(warps * 32), 0, st, 1, z, perm_token, n_rows, width, zp);
}
template cudaError_t launch_gather_rows<float>(const float*, const int32_t*, int64_t, int, float*,
                                               cudaStream_t);
template cudaError_t launch_gather_rows<__nv_bfloat16>(const __nv_bfloat16*, const int32_t*,
                                                       int64_t, int, __nv_bfloat16*, cudaStream_t);

}  // namespace lmoe
