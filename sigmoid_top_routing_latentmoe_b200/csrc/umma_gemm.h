// Host interface of the tcgen05 (5th-generation tensor core) GEMM engine.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lmoe {

// x-pass: one pass over x [N, d] computes
//   z      [N, L]  bf16 = x W_down^T
//   logits [N, R]  fp32 = x W_r^T          (row stride logits_ld)
//   hsh    [N, S*G] bf16 = SiTU(x W_g,sh^T, x W_u,sh^T) per shared expert
struct XpassArgs {
  const __nv_bfloat16* x;
  int64_t N;
  int d;
  const __nv_bfloat16* w_down;  // [L, d]
  int L;
  const __nv_bfloat16* w_router;  // [R, d]
  int R;
  const __nv_bfloat16* ws_g;  // [S, G, d]
  const __nv_bfloat16* ws_u;
  int S, G;
  __nv_bfloat16* z;
  float* logits;
  int64_t logits_ld;
  __nv_bfloat16* hsh;
  // z32 != nullptr: fp32 pre-activations instead (for the backward's recompute):
  // z32 [N, L] = x W_down^T, a_sh / c_sh [N, S*G] = x W_g,sh^T / x W_u,sh^T, and
  // no SiTU; z and hsh are not written.
  float* z32;
  float* a_sh;
  float* c_sh;
  float beta1, beta2;
  // When R <= 32 and ids != nullptr the epilogue also routes each row (K3 top-k
  // + L1 normalisation with bias b, or router == 1: top-k of the logits +
  // softmax) and writes ids/probs; the logits are written either way.
  int router;
  const float* bias;
  int32_t* ids;
  float* probs;
  int top_k;
  // With routing in the epilogue and row_counts != nullptr: row j of
  // row_counts [ceil(N / 32), R] gets, for each expert, the number of pairs of
  // tokens [32 j, 32 j + 32) routed to it (the dispatch's count rows).
  int32_t* row_counts;
  int max_units;  // at most this many CTA pairs (0: one per pair of SMs)
  // 1: 256 x 512 tiles (two N = 256 MMAs per K step, one TMEM accumulator);
  // 0: 256 x 256 tiles (double-buffered accumulator).  Ignored for z32.
  int wide;
  // Stream-K as in FinalArgs (few row tiles, e.g. a decode step): a tile
  // split between CTA pairs gets the others' fp32 partials added into its
  // accumulator before the epilogue.  Not with z32.
  float* sk_part;
  size_t sk_bytes;
  int32_t* sync;  // kSyncWords zeroed words (left zeroed)
  int stream_k;   // -1 by the wave fill, 0 never, 1 whenever sk_part fits
};

// final: y [N, d] = sum_j hsh[:, jG:(j+1)G] W_o,sh_j^T + uhat W_up^T
struct FinalArgs {
  const __nv_bfloat16* hsh;  // [N, S*G]
  int64_t N;
  int S, G;
  const __nv_bfloat16* ws_o;  // [S, d, G]
  int d;
  const __nv_bfloat16* uhat;  // [N, L]
  int L;
  const __nv_bfloat16* w_up;  // [d, L]
  __nv_bfloat16* y;
  int max_units;  // at most this many CTA pairs (0: one per pair of SMs)
  int wide;       // 1: 256 x 512 tiles (two N = 256 MMAs per K step, one accumulator)
  // Fused combine (eo != nullptr, L <= 1024): the kernel's epilogue warps first
  // write uhat = RMSNorm(sum_i probs[t, i] eo[inv[t, i]]) * rms_w for an even
  // share of the rows (the combine kernel's arithmetic), counting finished rows
  // per 256-row tile in sync[]; each CTA's producer waits for its tile's count
  // before loading the uhat K blocks, which come after the shared experts' ones.
  const __nv_bfloat16* eo;  // [N k, L] expert outputs, sorted-pair order
  const int32_t* inv;       // [N, k]
  const float* probs;       // [N, k]
  const float* rms_w;       // [L]
  int top_k;
  float rms_eps;
  int32_t* sync;            // kSyncWords zeroed words (left zeroed)
  // Stream-K: when whole tiles would leave a late wave part-empty, each CTA
  // pair takes an equal share of the tiles x K-blocks iterations; a tile split
  // between pairs is summed in fp32 through sk_part (sk_bytes long, scratch)
  // by the pair holding its first K blocks.  Flags live in sync[].
  // stream_k: -1 chooses by the wave fill, 0 never, 1 whenever sk_part fits.
  float* sk_part;
  size_t sk_bytes;
  int stream_k;
};

// routed GEMM1: h [P, F] = SiTU(zp W_g,e^T, zp W_u,e^T) per row tile of expert e
// routed GEMM2: eo [P, L] = h W_o,e^T
struct RoutedArgs {
  const __nv_bfloat16* a;  // zp [P, L] (gemm1) or h [P, F] (gemm2)
  int64_t P;
  int L, F, R;
  const __nv_bfloat16* w0;  // gemm1: w_g [R, F, L]; gemm2: w_o [R, L, F]
  const __nv_bfloat16* w1;  // gemm1: w_u [R, F, L]
  __nv_bfloat16* out;       // gemm1: h; gemm2: eo
  const int4* tiles;        // routed row tiles (expert, first row, rows)
  const int32_t* n_mtiles;
  int max_tiles;
  float beta1, beta2;
  int max_units;  // at most this many CTAs or CTA pairs (0: one per SM / pair of SMs)
  // 1: CTA pairs (tcgen05 cta_group::2) over row tiles of <= 256 sorted pairs;
  // 0: single CTAs over row tiles of <= 128.  The tile list must have been
  // built with the matching height (kRoutedPairTileM or kTileM).
  int pairs;
  // GEMM1 with pairs: 1 = tiles of 256 hidden units (256 x 512 accumulator).
  int wide;
};

cudaError_t umma_xpass(const XpassArgs& a, int32_t* status, cudaStream_t st);
cudaError_t umma_final(const FinalArgs& a, int32_t* status, cudaStream_t st);
cudaError_t umma_routed1(const RoutedArgs& a, int32_t* status, cudaStream_t st);
cudaError_t umma_routed2(const RoutedArgs& a, int32_t* status, cudaStream_t st);

}  // namespace lmoe
