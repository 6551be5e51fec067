// Internal launch interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lmoe {

// ---------------------------------------------------------------- routing
// Warp-per-token router for small R (<= 32): fp32 GEMV over W_r, sigmoid,
// biased top-k in registers, L1 normalisation.  T = float or bf16.
template <typename T>
// router: 0 K3 sigmoid rule, 1 softmax over the top-k logits.  logits_out
// (row stride ld) receives the fp32 logits when not null.
cudaError_t launch_route_gemv(const T* x, const T* w_r, const float* bias, int64_t n, int d, int R,
                              int k, int router, int32_t* ids, float* probs, float* logits_out,
                              int64_t ld, cudaStream_t st);
// Top-k + normalisation from precomputed fp32 logits [n, ld] (R valid columns).
cudaError_t launch_route_topk(const float* logits, int64_t ld, const float* bias, int64_t n, int R,
                              int k, int router, int32_t* ids, float* probs, cudaStream_t st);

// ------------------------------------------------------ router balancing losses
// Blocks of this many tokens each leave fixed-order partial sums.
constexpr int kLossRows = 256;
inline int loss_blocks(int64_t n) { return (int)((n + kLossRows - 1) / kLossRows); }
// out [2 + 2R] = aux, z, frac[R], prob_mean[R]; part_s / part_c [blocks][R],
// part_z [blocks] are scratch.
cudaError_t launch_router_losses(const float* logits, int64_t ld, const int32_t* ids, int64_t n,
                                 int k, int R, float* part_s, int32_t* part_c, float* part_z,
                                 int32_t* status, float* out, cudaStream_t st);

// ----------------------------------------------------------- permutation
// Tokens per row of the expert counts the x-pass's routing epilogue writes
// (one warp's rows): row j holds, for each expert, the pairs of tokens
// [32 j, 32 j + 32) routed to it.
constexpr int kCountRowTokens = 32;

struct DispatchScratch {
  int32_t* block_counts;  // [dispatch_count_rows, R]: chunk counts or the x-pass's row counts
  int32_t* status;        // workspace status word
  int32_t* n_mtiles;      // out: number of routed row tiles
  int4* tiles;            // out: [max_tiles] (expert, row0, rows, 0)
};
int dispatch_blocks(int64_t n_pairs);
// Rows of block_counts the dispatch needs (either kind of count row).
int64_t dispatch_count_rows(int64_t n, int k);
// Whether the dispatch can start from per-32-token expert counts (R <= 32,
// each chunk of the counting sort a whole number of count rows, and the rows
// few enough to be summed inside the scatter).
bool dispatch_takes_row_counts(int64_t n, int k, int R);
// With z != nullptr the scatter also copies each pair's z row (row_bytes, a
// multiple of 16) to its sorted slot in zp.  The routed tile list holds tiles
// of at most tile_m rows of one expert (kTileM or kRoutedPairTileM).  With
// row_counts, block_counts already holds the x-pass's count rows for these
// ids and the histogram kernel is not launched (cudaErrorInvalidValue when
// dispatch_takes_row_counts is false).
cudaError_t launch_dispatch(const int32_t* ids, int64_t n, int k, int R, int32_t* counts,
                            int32_t* offsets, int32_t* perm_token, int32_t* inv_pair,
                            const DispatchScratch& s, cudaStream_t st, const void* z = nullptr,
                            void* zp = nullptr, int row_bytes = 0, int tile_m = 128,
                            bool row_counts = false);
cudaError_t launch_build_tiles(const int32_t* offsets, int R, int32_t* n_mtiles, int4* tiles,
                               cudaStream_t st, int tile_m = 128);
// Consistency check of a permutation (bitmap: (N k + 31) / 32 words of scratch).
cudaError_t launch_check_dispatch(const int32_t* ids, int64_t n, int k, int R,
                                  const int32_t* counts, const int32_t* offsets,
                                  const int32_t* perm_token, const int32_t* inv_pair,
                                  uint32_t* bitmap, int32_t* status, cudaStream_t st);
// zp[r, :] = z[perm_token[r], :]
template <typename T>
cudaError_t launch_gather_rows(const T* z, const int32_t* perm_token, int64_t n_rows, int width,
                               T* zp, cudaStream_t st);

// ------------------------------------------------------------ SIMT GEMM
// C[m, n] = sum_s A_s[m, :K_s] . B_s[n, :K_s]  (all operands K-contiguous).
// mode kStore: C = acc (T or fp32 out);  kSitu: two accumulators against B and
// B_up, C = SiTU(acc_g, acc_u).  Ragged: rows come from the tile list and B
// pointers advance by b_expert_stride elements per expert.
constexpr int kMaxSeg = 8;
enum SimtMode { kStore = 0, kSitu = 1 };
struct SimtGemm {
  const void* A[kMaxSeg];
  int64_t lda[kMaxSeg];
  const void* B[kMaxSeg];
  int64_t ldb[kMaxSeg];
  int K[kMaxSeg];
  int nseg;
  const void* B_up;        // SiTU mode: up-projection rows (same ldb as B[0])
  int64_t b_expert_stride; // ragged mode: elements between experts' weights
  void* C;
  int64_t ldc;
  int M, N;                // dense mode rows; output columns
  int out_f32;             // 1: C is fp32 regardless of T
  const int4* tiles;       // ragged mode tile list or nullptr
  const int32_t* n_tiles;
  int max_tiles;
  float beta1, beta2;
  int mode;
};
template <typename T>
cudaError_t launch_simt_gemm(const SimtGemm& g, cudaStream_t st);

// -------------------------------------------------------------- combine
template <typename T>
cudaError_t launch_combine(const T* expert_out, const int32_t* inv_pair, const float* probs,
                           const float* rms_w, int64_t n, int k, int L, float eps, T* out,
                           cudaStream_t st);

// ------------------------------------------------------------ self-test
cudaError_t launch_capped_wait(int32_t* flag, int32_t* status, int cap_ms, cudaStream_t st);

// Launch counter (api.cu)
void count_launch(int n = 1);
// Sets the per-thread message returned by lmoe_last_error (api.cu).
void set_last_error(const char* msg);

// ------------------------------------------------------------------ backward
struct BwdDims {
  int64_t N;
  int d, L, R, k, S, F, G;
  float beta1, beta2, rms_eps;
  int router;
  int bf16;  // x, dy and the weights are bf16 (else fp32); gradients are fp32
};
struct BwdGrads {
  float *dx, *dw_down, *dw_router, *dw_up, *drms, *dw_g, *dw_u, *dw_o, *dws_g, *dws_u, *dws_o;
};
struct BwdArgs {
  const void *x, *dy, *w_down, *w_router, *w_up, *w_g, *w_u, *w_o, *ws_g, *ws_u, *ws_o;
  const float *rms_weight, *bias;
  BwdGrads g;
};
struct BwdLayout {
  size_t header, logits, ids, probs, counts, offsets, perm, inv, block_counts, tiles, z, zp, a, c, h,
      dh, o, dE, u, uhat, duhat, du, rr, dp, dl, rms_part, ash, csh, hsh, dhsh, split, total;
  int ld_logits, max_tiles;
};
BwdLayout bwd_layout(const BwdDims& d);
// The workspace header (its first 256 bytes) must be zero on entry.
cudaError_t run_backward(const BwdDims& d, const BwdArgs& a, void* ws, cudaStream_t st);

}  // namespace lmoe
