// tcgen05 GEMM engine for the bf16 LatentMoE forward (sm_100a).
//
// One persistent, warp-specialised kernel template serves the four GEMMs of
// the layer.  Every tile is 128 rows x (128 or 256) columns, K in blocks of 64
// bf16 (one 128-byte swizzle atom):
//   warp 0   TMA producer: cp.async.bulk.tensor loads of the A tile and of
//            one or two 128-row B sub-tiles into a 4-stage smem ring,
//   warp 1   MMA issuer: tcgen05.mma.kind::f16 (bf16 x bf16 -> fp32) into a
//            double-buffered TMEM accumulator (2 x 256 columns), and the
//            TMEM allocator,
//   warps 2-9 epilogue: tcgen05.ld of the accumulator, the fused epilogue of
//            the GEMM (bf16/fp32 store, or the SiTU-GLU hidden unit of a
//            gate/up column pair), then bf16 blocks of 32 rows x 64 columns
//            transposed through a per-warp smem buffer so that every global
//            store instruction writes whole 128-byte row segments.
// The four GEMMs (sec-07 compute flow; kda/layers/latent_moe.py):
//   XPASS   x [N, d] against [W_down | W_r | (W_g,sh, W_u,sh) pairs]: z, the
//           router logits (step 2) and the shared experts' SiTU hidden units
//           (step 4) in one pass over x.
//   ROUTED1 sorted pairs z[perm] against (W_g,e, W_u,e) pairs: SiTU hidden
//           units of the routed experts (step 3), row tiles from the device
//           tile list (no padding to a capacity).
//   ROUTED2 routed hidden units against W_o,e.
//   FINAL   [h_sh | RMSNorm(u)] against [W_o,sh | W_up]: the shared experts'
//           output projection and the latent restore summed in one
//           accumulator (step 5, y = s_sh + W_up RMSNorm(u)).
// Every mbarrier wait is capped: after ~2 s the kernel records LMOE_ETIMEOUT,
// stops issuing work, drains what it issued, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "combine_row.cuh"
#include "common.cuh"
#include "kernels.h"
#include "umma_gemm.h"
#include "launch.h"

namespace lmoe {
namespace {

constexpr int BM = 128;          // rows per CTA (TMEM lanes)
constexpr int BK = 64;           // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int SUB = 128;         // rows of a full B sub-tile
constexpr int A_BYTES = BM * BK * 2;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 2 * ACC_COLS;
#ifndef LMOE_EPI_WARPS
#define LMOE_EPI_WARPS 8
#endif
// Epilogue warps: 8 = two per TMEM lane quarter, splitting the column blocks;
// 4 = one per quarter, each taking every column block.
constexpr int EPI_WARPS = LMOE_EPI_WARPS;
static_assert(EPI_WARPS == 4 || EPI_WARPS == 8, "4 or 8 epilogue warps");
constexpr int HS = EPI_WARPS / 4;  // column-block stride of one epilogue warp
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr uint64_t WAIT_CAP_NS = 2000000000ull;

// XPASS_F32: the x-pass with fp32 z and shared gate / up pre-activations (no SiTU)
// XPASS_WIDE, FINAL_WIDE, ROUTED1_WIDE: those GEMMs on 256 x 512 pair tiles (see Cfg)
// XPASS_SK, XPASS_WIDE_SK: the x-pass under stream-K (their own instantiations,
//   so that the stream-K code costs the plain x-pass no registers)
enum Mode {
  XPASS = 0, FINAL = 1, ROUTED1 = 2, ROUTED2 = 3, XPASS_F32 = 4,
  XPASS_WIDE = 5, FINAL_WIDE = 6, ROUTED1_WIDE = 7, XPASS_SK = 8, XPASS_WIDE_SK = 9
};
template <int MODE>
constexpr bool is_wide() {
  return MODE == XPASS_WIDE || MODE == FINAL_WIDE || MODE == ROUTED1_WIDE || MODE == XPASS_WIDE_SK;
}
// the GEMM a mode computes (a wide mode computes its base mode's GEMM)
template <int MODE>
constexpr int base_of() {
  return MODE == XPASS_WIDE || MODE == XPASS_SK || MODE == XPASS_WIDE_SK ? XPASS
         : MODE == FINAL_WIDE                                           ? FINAL
         : MODE == ROUTED1_WIDE                                         ? ROUTED1
                                                                        : MODE;
}
template <int MODE>
constexpr bool is_xpass() {
  return MODE == XPASS || MODE == XPASS_F32 || MODE == XPASS_WIDE || MODE == XPASS_SK ||
         MODE == XPASS_WIDE_SK;
}
template <int MODE>
constexpr bool is_xpass_sk() { return MODE == XPASS_SK || MODE == XPASS_WIDE_SK; }

// CG = 1: one CTA computes a 128-row tile and loads every B sub-tile.
// CG = 2: a CTA pair (cluster of 2) computes a 256-row tile with
//         tcgen05.mma.cta_group::2; each CTA loads its own 128 rows of A and
//         one of the two B sub-tiles (half of N), so each SM streams half of
//         B per FLOP.
// W = 2 (XPASS_WIDE, pairs only): each K step issues two N = 256 MMAs into
//         the 512 TMEM columns, a 256 x 512 tile; each CTA loads 128 rows of A
//         and two 128-row B sub-tiles per stage, so every byte an SM streams
//         feeds 1.33x the FLOPs of a 256 x 256 tile.  The accumulator takes
//         all of TMEM (one buffer): the next tile's MMAs wait for the
//         epilogue, while the TMA ring keeps filling.
template <int MODE, int CG>
struct Cfg {
  static constexpr int W = is_wide<MODE>() ? 2 : 1;
  static constexpr int B_BYTES = (CG == 1 ? 2 : W) * SUB * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB or 32 KB
  static constexpr int STAGES = CG == 1 ? 4 : (W == 2 ? 4 : 6);
  static constexpr int EPI_STAGE = 32 * 128;             // per epilogue warp: 32 rows x 128 B
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_WARPS * EPI_STAGE + 1024;
  static constexpr int MT = BM * CG;                     // tile rows
  static constexpr int NACC = W == 2 ? 1 : 2;            // accumulator buffers in TMEM
  static constexpr int ACC_STRIDE = TMEM_COLS / NACC;    // columns per buffer
};
static_assert(Cfg<XPASS_WIDE, 2>::SMEM_BYTES <= 232448, "wide tiles exceed shared memory");

enum Epi { EPI_Z = 1, EPI_SITU = 3, EPI_STORE = 4 };
// B sub-tile sources of the x-pass: 0 W_down, 1 W_r, 2 W_g,sh, 3 W_u,sh,
// 5 zero padding (a box outside W_r: loads zeros, stores nothing).
constexpr int kPadMap = 5;

struct Params {
  CUtensorMap tmA0, tmA1;              // A operands (FINAL: h_sh, uhat)
  CUtensorMap tmB0, tmB1, tmB2, tmB3;  // B operands (see decode_tile)
  int map_mask;                        // encoded maps: bit 0 A0, 1 A1, 2 B0, 3 B1, 4 B2, 5 B3
  int M;                               // dense rows
  int n_tiles;                         // tiles along the output columns
  int kb0, kb1;                        // K blocks (FINAL: per shared expert, then uhat)
  int S, G, L, R, F, d;
  int nz_sub, nr_sub, n_zr_tiles, g_blocks;
  int bn;                              // FINAL / ROUTED2 tile width: 128, 192 or 256
  int fuse_topk;                       // XPASS: top-k in the epilogue (R <= 32)
  int router;                          // 0: K3 sigmoid rule; 1: softmax over the top-k logits
  int top_k;
  const float* bias;
  int32_t* ids;
  float* probs;
  int32_t* row_counts;                 // XPASS with fuse_topk: per 32 rows, pairs per expert
  void* out0;
  void* out1;
  void* out2;
  void* out3;                          // XPASS_F32: up pre-activations (row stride ld2)
  int64_t ld0, ld1, ld2;
  const int4* tiles;
  const int32_t* n_mtiles;
  int32_t* status;
  float beta1, beta2, inv_beta1, inv_beta2, beta12;
  // FINAL with the fused combine (see FinalArgs)
  const __nv_bfloat16* c_eo;
  const int32_t* c_inv;
  const float* c_probs;
  const float* c_rms;
  __nv_bfloat16* c_uhat;
  int32_t* c_sync;
  int c_k, c_vpl, fuse_combine;
  float c_eps;
  // FINAL with stream-K scheduling: each unit (CTA pair) takes an equal share
  // of the tiles' K-block iterations; see work_begin / work_next and the epilogue
  int stream_k;
  float* sk_part;     // [units][2 ranks][4 lane quarters][bn / 64][16][32] float4 partials
  int32_t* sk_flags;  // [units] warps that stored the unit's partial
};

template <int NS>  // at most NS B sub-tiles
struct TileT {
  int m0, rows, n_sub;
  int ncols;                       // MMA N: sum of the sub-tiles' rows
  int bmap[NS], brow[NS], bz[NS];  // B source map, first row, expert (3-D maps)
  int srows[NS];                   // rows of each sub-tile load
  int scol[NS];                    // accumulator / output column of each sub-tile
  int epi, ocol;
};
template <int MODE, int CG>
using Tile = TileT<2 * Cfg<MODE, CG>::W>;

// ------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Capped wait: false if the cap ran out (status recorded) or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  uint32_t it = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++it & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > WAIT_CAP_NS) {
        *abort_flag = 1;
        record_status(status, kStatusTimeout);
        return false;
      }
    }
  }
  return true;
}
// Capped wait until the counter at c reaches target (acquire), then a proxy
// fence so that TMA loads issued afterwards see the global writes it counted.
__device__ __forceinline__ bool wait_count(const int32_t* c, int target, volatile int* abort_flag,
                                           int32_t* status) {
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
    if (v >= target) break;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      const uint64_t now = global_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > WAIT_CAP_NS) {
        *abort_flag = 1;
        record_status(status, kStatusTimeout);
        return false;
      }
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 lanes x 32 columns of fp32: thread i of the warp gets row (lane base + i).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Two 32-column TMEM loads in flight before one wait.
__device__ __forceinline__ void tc_ld32x2(uint32_t ta, float (&va)[32], uint32_t tb,
                                          float (&vb)[32]) {
  uint32_t r[32], q[32];
#define LMOE_TC_LD32(ADDR, R)                                                                   \
  asm volatile(                                                                                 \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                                 \
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"                                 \
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"               \
      : "=r"(R[0]), "=r"(R[1]), "=r"(R[2]), "=r"(R[3]), "=r"(R[4]), "=r"(R[5]), "=r"(R[6]),     \
        "=r"(R[7]), "=r"(R[8]), "=r"(R[9]), "=r"(R[10]), "=r"(R[11]), "=r"(R[12]),             \
        "=r"(R[13]), "=r"(R[14]), "=r"(R[15]), "=r"(R[16]), "=r"(R[17]), "=r"(R[18]),          \
        "=r"(R[19]), "=r"(R[20]), "=r"(R[21]), "=r"(R[22]), "=r"(R[23]), "=r"(R[24]),          \
        "=r"(R[25]), "=r"(R[26]), "=r"(R[27]), "=r"(R[28]), "=r"(R[29]), "=r"(R[30]),          \
        "=r"(R[31])                                                                             \
      : "r"(ADDR))
  LMOE_TC_LD32(ta, r);
  LMOE_TC_LD32(tb, q);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(q[i]);
  }
}
// Two 32-column TMEM stores, then a wait for both (32 lanes x 32 columns each).
__device__ __forceinline__ void tc_st32x2(uint32_t ta, const float (&va)[32], uint32_t tb,
                                          const float (&vb)[32]) {
#define LMOE_TC_ST32(ADDR, V)                                                                   \
  asm volatile(                                                                                 \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "                                           \
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"                                \
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"                       \
      ::"r"(ADDR), "f"(V[0]), "f"(V[1]), "f"(V[2]), "f"(V[3]), "f"(V[4]), "f"(V[5]), "f"(V[6]), \
      "f"(V[7]), "f"(V[8]), "f"(V[9]), "f"(V[10]), "f"(V[11]), "f"(V[12]), "f"(V[13]),          \
      "f"(V[14]), "f"(V[15]), "f"(V[16]), "f"(V[17]), "f"(V[18]), "f"(V[19]), "f"(V[20]),       \
      "f"(V[21]), "f"(V[22]), "f"(V[23]), "f"(V[24]), "f"(V[25]), "f"(V[26]), "f"(V[27]),       \
      "f"(V[28]), "f"(V[29]), "f"(V[30]), "f"(V[31])                                            \
      : "memory")
  LMOE_TC_ST32(ta, va);
  LMOE_TC_ST32(tb, vb);
#undef LMOE_TC_ST32
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Two 16-column TMEM loads in flight before one wait.
__device__ __forceinline__ void tc_ld16x2(uint32_t ta, float (&va)[16], uint32_t tb,
                                          float (&vb)[16]) {
  uint32_t r[16], q[16];
#define LMOE_TC_LD16(ADDR, R)                                                                   \
  asm volatile(                                                                                 \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "                                                 \
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"                         \
      : "=r"(R[0]), "=r"(R[1]), "=r"(R[2]), "=r"(R[3]), "=r"(R[4]), "=r"(R[5]), "=r"(R[6]),     \
        "=r"(R[7]), "=r"(R[8]), "=r"(R[9]), "=r"(R[10]), "=r"(R[11]), "=r"(R[12]),             \
        "=r"(R[13]), "=r"(R[14]), "=r"(R[15])                                                   \
      : "r"(ADDR))
  LMOE_TC_LD16(ta, r);
  LMOE_TC_LD16(tb, q);
#undef LMOE_TC_LD16
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(q[i]);
  }
}
// Four 32-column TMEM loads in flight before one wait.
__device__ __forceinline__ void tc_ld32x4(uint32_t ta, float (&va)[32], uint32_t tb,
                                          float (&vb)[32], uint32_t tc, float (&vc)[32],
                                          uint32_t td, float (&vd)[32]) {
  uint32_t r[32], q[32], x[32], y[32];
  LMOE_TC_LD32(ta, r);
  LMOE_TC_LD32(tb, q);
  LMOE_TC_LD32(tc, x);
  LMOE_TC_LD32(td, y);
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(q[i]);
    vc[i] = __uint_as_float(x[i]);
    vd[i] = __uint_as_float(y[i]);
  }
}
#undef LMOE_TC_LD32

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row
// core groups 1024 bytes apart (SBO), descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}
__device__ __forceinline__ uint32_t tanh_h2(uint32_t v) {
  uint32_t r;
  asm("tanh.approx.f16x2 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}
__device__ __forceinline__ uint32_t ex2_h2(uint32_t v) {
  uint32_t r;
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}
__device__ __forceinline__ __half2 mufu_h2(uint32_t (*f)(uint32_t), __half2 x) {
  uint32_t u = f(*reinterpret_cast<const uint32_t*>(&x));
  return *reinterpret_cast<__half2*>(&u);
}
// Two SiTU-GLU hidden units at once, packed to bf16x2:
//   h = beta1 tanh(a/beta1) sigmoid(a) * beta2 tanh(c/beta2),
// on f16x2 pairs: a and c are rounded to f16 once and scaled there; the
// sigmoid is formed without cancellation for negative a,
//   sigmoid(a) = 2^(min(a, 0) log2 e) * (1/2 + tanh(|a|/2)/2),
// (e^a sigmoid(-a) = sigmoid(a)), so its error stays relative over the whole
// range; the three tanh and the exponential are one MUFU op per pair each,
// and the bounded factors (|tanh| <= 1, sigmoid <= 1) are multiplied in f16x2
// after the scale beta1*beta2 (|h| <= beta1*beta2).  An |a| or |c| beyond the
// f16 range rounds to infinity, where every factor reaches its limit.
struct SituConsts {
  __half2 inv_b1, inv_b2, b12, half, log2e, zero;
};
__device__ __forceinline__ SituConsts situ_consts(const Params& p) {
  return {__float2half2_rn(p.inv_beta1), __float2half2_rn(p.inv_beta2),
          __float2half2_rn(p.beta12), __float2half2_rn(0.5f),
          __float2half2_rn(1.4426950408889634f), __float2half2_rn(0.0f)};
}
__device__ __forceinline__ uint32_t situ2_bf16(float a0, float a1, float c0, float c1,
                                               const SituConsts& k) {
  const __half2 a = __floats2half2_rn(a0, a1);
  const __half2 c = __floats2half2_rn(c0, c1);
  const __half2 t1 = mufu_h2(tanh_h2, __hmul2(a, k.inv_b1));
  const __half2 t2 = mufu_h2(tanh_h2, __hmul2(__habs2(a), k.half));
  const __half2 em = mufu_h2(ex2_h2, __hmul2(__hmin2(a, k.zero), k.log2e));
  const __half2 t3 = mufu_h2(tanh_h2, __hmul2(c, k.inv_b2));
  const __half2 sg = __hmul2(__hfma2(t2, k.half, k.half), em);
  const __half2 h = __hmul2(__hmul2(__hmul2(t1, k.b12), sg), t3);
  const float2 f = __half22float2(h);
  __nv_bfloat162 o = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t*>(&o);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA loads of one CTA of a pair; the transaction bytes land on the barrier
// at `bar` (a cluster address: the leader CTA's barrier).
__device__ __forceinline__ void tma2_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                             int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma2_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                             int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tc2_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive (when the issuing thread's MMAs complete) on the barrier at this
// offset in both CTAs of the pair.
__device__ __forceinline__ void tc2_commit_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
// Instruction descriptor: D fp32, A and B bf16, both K-major, M = 128 * CG, N = n.
template <int CG>
__device__ __forceinline__ uint32_t instr_desc_cg(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)((BM * CG) >> 4) << 24);
}

// ---------------------------------------------------------- tile decoding
template <int MODE, int CG>
__device__ __forceinline__ int total_tiles(const Params& p) {
  if (is_xpass<MODE>() || base_of<MODE>() == FINAL) return ((p.M + Cfg<MODE, CG>::MT - 1) / Cfg<MODE, CG>::MT) * p.n_tiles;
  return (*p.n_mtiles) * p.n_tiles;
}

template <int MODE, int CG>
__device__ __forceinline__ Tile<MODE, CG> decode_tile(const Params& p, int t) {
  Tile<MODE, CG> tl;
#pragma unroll
  for (int s = 0; s < 2 * Cfg<MODE, CG>::W; ++s) {
    tl.bz[s] = 0;
    tl.srows[s] = SUB;
    tl.scol[s] = s * SUB;
  }
  if (is_xpass<MODE>() || base_of<MODE>() == FINAL) {
    constexpr int MT = Cfg<MODE, CG>::MT;
    const int m_tiles = (p.M + MT - 1) / MT;
    // From 32 row tiles on, tiles go in groups of kGroupM row tiles, rows
    // fastest inside a group: the tiles in flight at once (one per CTA pair)
    // cover a few row tiles times many column tiles, so both operands' tiles
    // are reused from L2 instead of the rows being streamed from DRAM once per
    // column tile (mid shape: x-pass 495 -> 473 us, final GEMM DRAM reads
    // 1.2 GB before).  Fewer row tiles keep rows fastest over all of them (the
    // 0.5b shape, whose operands stay in L2 either way, was 0.4 us slower grouped).
    constexpr int kGroupM = 8;
    const int gsize = m_tiles >= 32 ? kGroupM : m_tiles;
    const int per_group = gsize * p.n_tiles;
    const int g = t / per_group, r = t - g * per_group;
    const int gm = min(gsize, m_tiles - g * gsize);  // row tiles in this group
    const int mt = g * gsize + r % gm, n = r / gm;
    tl.m0 = mt * MT;
    tl.rows = min(MT, p.M - tl.m0);
    if (base_of<MODE>() == FINAL) {
      const int n0 = n * p.bn;
      if (Cfg<MODE, CG>::W == 2) {  // four 128-row sub-tiles: CTA r loads r and r + 2
        tl.n_sub = 4;
#pragma unroll
        for (int sb = 0; sb < 2 * Cfg<MODE, CG>::W; ++sb) {
          tl.brow[sb] = n0 + sb * SUB;
          tl.bmap[sb] = 0;
        }
        tl.ncols = 4 * SUB;
      } else if (CG == 2) {  // each CTA loads half of the tile's columns
        tl.n_sub = 2;
        tl.srows[0] = tl.srows[1] = p.bn / 2;
        tl.scol[1] = p.bn / 2;
        tl.brow[0] = n0;
        tl.brow[1] = n0 + p.bn / 2;
        tl.ncols = p.bn;
      } else {
        tl.n_sub = (p.bn > SUB && n0 + SUB < p.d) ? 2 : 1;
        tl.srows[1] = p.bn - SUB;
        tl.brow[0] = n0;
        tl.brow[1] = n0 + SUB;
        tl.ncols = tl.n_sub == 2 ? p.bn : SUB;
      }
      tl.bmap[0] = tl.bmap[1] = 0;
      tl.epi = EPI_STORE;
      tl.ocol = n0;
    } else if (n < p.n_zr_tiles) {
      // 2 W sub-tiles of z / router rows (sub-tile s: accumulator columns [128 s, 128 s + 128))
      constexpr int NS = 2 * Cfg<MODE, CG>::W;
      tl.n_sub = 0;
      for (int s = 0; s < NS; ++s) {
        const int idx = NS * n + s;
        if (idx < p.nz_sub) {
          tl.bmap[s] = 0;
          tl.brow[s] = idx * SUB;
          tl.n_sub = s + 1;
        } else if (idx < p.nz_sub + p.nr_sub) {
          tl.bmap[s] = 1;
          tl.brow[s] = (idx - p.nz_sub) * SUB;
          tl.n_sub = s + 1;
        } else {  // a pair tile always loads two sub-tiles: pad with zeros
          tl.bmap[s] = kPadMap;
          tl.brow[s] = p.nr_sub * SUB;
        }
      }
      if (CG == 2) tl.n_sub = NS;
      tl.epi = EPI_Z;  // per sub-tile: z, routing or padding, resolved in the epilogue
      tl.ocol = 0;
      tl.ncols = tl.n_sub * SUB;
    } else {
      // W blocks of 128 hidden units of shared expert j: sub-tile 2b holds the gate
      // rows of block b, sub-tile 2b + 1 the matching up rows
      constexpr int W = Cfg<MODE, CG>::W;
      const int q = n - p.n_zr_tiles;
      const int j = q / p.g_blocks, fb = q % p.g_blocks;
      tl.n_sub = 2 * W;
#pragma unroll
      for (int sb = 0; sb < 2 * W; ++sb) {
        tl.bmap[sb] = (sb & 1) ? 3 : 2;
        tl.brow[sb] = fb * W * SUB + (sb >> 1) * SUB;
        tl.bz[sb] = j;
      }
      tl.epi = EPI_SITU;
      tl.ocol = j * p.G + fb * W * SUB;
      tl.ncols = 2 * W * SUB;
    }
  } else {
    const int mt = t / p.n_tiles, n = t % p.n_tiles;
    const int4 e = p.tiles[mt];
    tl.m0 = e.y;
    tl.rows = e.z;
#pragma unroll
    for (int sb = 0; sb < 2 * Cfg<MODE, CG>::W; ++sb) tl.bz[sb] = e.x;
    if (Cfg<MODE, CG>::W == 2) {  // ROUTED1_WIDE: 256 hidden units of expert e
      // sub-tile 2b: gate rows of block b of W_g,e; 2b + 1: the up rows of W_u,e
      // (CTA 0 loads the gate sub-tiles, CTA 1 the up ones)
      tl.n_sub = 4;
#pragma unroll
      for (int sb = 0; sb < 2 * Cfg<MODE, CG>::W; ++sb) {
        tl.bmap[sb] = sb & 1;
        tl.brow[sb] = n * 2 * SUB + (sb >> 1) * SUB;
      }
      tl.epi = EPI_SITU;
      tl.ocol = n * 2 * SUB;
      tl.ncols = 4 * SUB;
    } else if (base_of<MODE>() == ROUTED1) {
      // gate rows of W_g,e and the matching up rows of W_u,e (CG = 2: CTA 0
      // loads the gate half, CTA 1 the up half)
      tl.n_sub = 2;
      tl.bmap[0] = 0;
      tl.bmap[1] = 1;
      tl.brow[0] = tl.brow[1] = n * SUB;
      tl.epi = EPI_SITU;
      tl.ocol = n * SUB;
      tl.ncols = 2 * SUB;
    } else if (CG == 2) {  // ROUTED2 on a pair: each CTA loads half of the bn W_o rows
      const int n0 = n * p.bn;
      tl.n_sub = 2;
      tl.bmap[0] = tl.bmap[1] = 0;
      tl.srows[0] = tl.srows[1] = p.bn / 2;
      tl.scol[1] = p.bn / 2;
      tl.brow[0] = n0;
      tl.brow[1] = n0 + p.bn / 2;
      tl.ncols = p.bn;
      tl.epi = EPI_STORE;
      tl.ocol = n0;
    } else {
      const int n0 = n * p.bn;
      tl.n_sub = (p.bn > SUB && n0 + SUB < p.L) ? 2 : 1;
      tl.bmap[0] = 0;
      tl.bmap[1] = 1;  // map 1: the (bn - 128)-row box
      tl.brow[0] = n0;
      tl.brow[1] = n0 + SUB;
      tl.srows[1] = p.bn - SUB;
      tl.ncols = tl.n_sub == 2 ? p.bn : SUB;
      tl.epi = EPI_STORE;
      tl.ocol = n0;
    }
  }
  return tl;
}

template <int MODE>
__device__ __forceinline__ int k_blocks(const Params& p) {
  return base_of<MODE>() == FINAL ? p.S * p.kb0 + p.kb1 : p.kb0;
}

// The work of one unit (a CTA or CTA pair): K blocks [kb0, kb1) of tile t.
// Plain scheduling gives a unit whole tiles unit, unit + n_units, ...; stream-K
// (FINAL, p.stream_k) gives it the iterations [u Q / U, (u + 1) Q / U) of the
// Q = tiles x K-blocks iterations, in order, so a tile can be split between
// consecutive units.  All three roles walk the same sequence.
struct Work {
  int t, kb0, kb1;
};
struct WorkIter {
  int64_t cur, end;
  int nkb, step;
  bool sk;
};
template <int MODE, int CG>
__device__ __forceinline__ WorkIter work_begin(const Params& p, int unit, int n_units) {
  WorkIter it;
  it.nkb = k_blocks<MODE>(p);
  it.sk = (base_of<MODE>() == FINAL || is_xpass_sk<MODE>()) && p.stream_k;
  const int64_t total = total_tiles<MODE, CG>(p);
  if (it.sk) {
    const int64_t q = total * it.nkb;
    it.cur = q * unit / n_units;
    it.end = q * (unit + 1) / n_units;
    it.step = 0;
  } else {
    it.cur = unit;
    it.end = total;
    it.step = n_units;
  }
  return it;
}
__device__ __forceinline__ bool work_next(WorkIter& it, Work& w) {
  if (it.cur >= it.end) return false;
  if (!it.sk) {
    w.t = (int)it.cur;
    w.kb0 = 0;
    w.kb1 = it.nkb;
    it.cur += it.step;
    return true;
  }
  w.t = (int)(it.cur / it.nkb);
  w.kb0 = (int)(it.cur - (int64_t)w.t * it.nkb);
  w.kb1 = (int)min((int64_t)it.nkb, w.kb0 + (it.end - it.cur));
  it.cur += w.kb1 - w.kb0;
  return true;
}
// Stream-K: the unit whose share holds iteration i.
__device__ __forceinline__ int sk_unit_of(int64_t i, int64_t q, int n_units) {
  int u = (int)((i * n_units) / q);
  while (u + 1 < n_units && q * (u + 1) / n_units <= i) ++u;
  while (u > 0 && q * u / n_units > i) --u;
  return u;
}

__device__ __forceinline__ const CUtensorMap* bmap_ptr(const Params& p, int i) {
  return i == 0 ? &p.tmB0 : i == 1 ? &p.tmB1 : i == 2 ? &p.tmB2 : &p.tmB3;
}

// Loads one B sub-tile (CG = 1 loads into the CTA's own barrier; CG = 2 into
// the leader's).
template <int CG>
__device__ __forceinline__ void load_b(uint32_t dst, const CUtensorMap* map, bool three_d,
                                       uint32_t bar, int kk, int row, int z) {
  if (CG == 1) {
    if (three_d)
      tma_load_3d(dst, map, bar, kk, row, z);
    else
      tma_load_2d(dst, map, bar, kk, row);
  } else {
    if (three_d)
      tma2_load_3d(dst, map, bar, kk, row, z);
    else
      tma2_load_2d(dst, map, bar, kk, row);
  }
}

// ------------------------------------------------------------- producer
template <int MODE, int CG>
__device__ __forceinline__ void produce(const Params& p, uint8_t* ring, uint64_t* full,
                                        uint64_t* empty, volatile int* abort_flag, uint32_t rank,
                                        int unit, int n_units) {
  using C = Cfg<MODE, CG>;
  // This one thread refills every stage, so its per-stage path is kept short:
  // everything that depends only on the tile is resolved before the K loop
  // (no tile-array indexing inside it), and which stages hold loads in flight
  // is tracked in two bit masks.
  int stage = 0;
  uint32_t phase = 0;
  uint32_t issued = 0, issued_phase = 0;  // bit s: stage s was filled; its phase
  const uint32_t ring0 = smem_u32(ring);
  const uint32_t full0 = smem_u32(full), empty0 = smem_u32(empty);
  const uint32_t full0_leader = CG == 1 ? full0 : map_to_rank(full0, 0);
  bool ok = true;
  WorkIter wi = work_begin<MODE, CG>(p, unit, n_units);
  Work wk;
  while (ok && work_next(wi, wk)) {
    const Tile<MODE, CG> tl = decode_tile<MODE, CG>(p, wk.t);
    const int arow = tl.m0 + (CG == 2 ? BM * (int)rank : 0);
    // A routed pair tile of <= 128 rows has none in CTA 1: it loads no A there
    // (its accumulator rows are never stored) and the leader expects fewer bytes.
    constexpr bool kRoutedPair = CG == 2 && (base_of<MODE>() == ROUTED1 || MODE == ROUTED2);
    int a_ctas = CG;
    if constexpr (kRoutedPair) a_ctas = tl.rows <= BM ? 1 : 2;
    const bool load_a = CG == 1 || !kRoutedPair || (int)rank < a_ctas;
    const uint32_t tx_bytes = (uint32_t)(a_ctas * A_BYTES + tl.ncols * BK * 2);
    // the B sub-tiles this CTA loads: CG = 1 sub-tiles 0 (and 1); CG = 2 the
    // sub-tile of its rank (and, for wide tiles, rank + 2 at B offset 1)
    const int sa = CG == 1 ? 0 : (int)rank;
    const bool two = (CG == 1 && tl.n_sub > 1) || C::W == 2;
    const int sb = CG == 1 ? 1 : (int)rank + 2;
    int ma = tl.bmap[sa], mb = two ? tl.bmap[sb] : 0;
    const int row_a = tl.brow[sa], z_a = tl.bz[sa];
    const int row_b = two ? tl.brow[sb] : 0, z_b = two ? tl.bz[sb] : 0;
    if (is_xpass<MODE>() && ma == kPadMap) ma = 1;
    if (is_xpass<MODE>() && mb == kPadMap) mb = 1;
    const bool td_a = !(is_xpass<MODE>() && ma < 2), td_b = !(is_xpass<MODE>() && mb < 2);
    const CUtensorMap* map_a = bmap_ptr(p, ma);
    const CUtensorMap* map_b = bmap_ptr(p, mb);
    const uint32_t off_b = SUB * BK * 2;  // the second sub-tile's B offset
    for (int kb = wk.kb0; kb < wk.kb1; ++kb) {
      if (base_of<MODE>() == FINAL && p.fuse_combine && kb == max(p.S * p.kb0, wk.kb0)) {
        // the uhat rows of this tile are written by the kernel's own epilogue
        // warps (checked before this unit's first uhat K block of the tile)
        if (!wait_count(p.c_sync + tl.m0 / Cfg<MODE, CG>::MT, tl.rows, abort_flag, p.status)) {
          ok = false;
          break;
        }
      }
      if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, p.status)) {
        ok = false;
        break;
      }
      const uint32_t a_dst = ring0 + stage * C::STAGE_BYTES;
      const uint32_t b_dst = a_dst + A_BYTES;
      const uint32_t own_bar = full0 + 8 * stage;
      const uint32_t bar = full0_leader + 8 * stage;
      if (CG == 1 || rank == 0) mbar_expect_tx(own_bar, tx_bytes);
      if (base_of<MODE>() == FINAL) {
        const int kb_sh = p.S * p.kb0;
        if (kb < kb_sh) {
          const int j = kb / p.kb0, kk = (kb % p.kb0) * BK;
          if (CG == 1) tma_load_2d(a_dst, &p.tmA0, bar, j * p.G + kk, arow);
          else tma2_load_2d(a_dst, &p.tmA0, bar, j * p.G + kk, arow);
          load_b<CG>(b_dst, sa == 0 ? &p.tmB0 : &p.tmB2, true, bar, kk, row_a, j);
          if (two) load_b<CG>(b_dst + off_b, &p.tmB2, true, bar, kk, row_b, j);
        } else {
          const int kk = (kb - kb_sh) * BK;
          if (CG == 1) tma_load_2d(a_dst, &p.tmA1, bar, kk, arow);
          else tma2_load_2d(a_dst, &p.tmA1, bar, kk, arow);
          load_b<CG>(b_dst, sa == 0 ? &p.tmB1 : &p.tmB3, false, bar, kk, row_a, 0);
          if (two) load_b<CG>(b_dst + off_b, &p.tmB3, false, bar, kk, row_b, 0);
        }
      } else {
        const int kk = kb * BK;
        if (CG == 1) tma_load_2d(a_dst, &p.tmA0, bar, kk, arow);
        else if (load_a) tma2_load_2d(a_dst, &p.tmA0, bar, kk, arow);
        load_b<CG>(b_dst, map_a, td_a, bar, kk, row_a, z_a);
        if (two) load_b<CG>(b_dst + off_b, map_b, td_b, bar, kk, row_b, z_b);
      }
      issued |= 1u << stage;
      issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  // drain: every load issued into this CTA's barriers has landed before exit
  // (a pair's loads all land on the leader's barriers)
  if (CG == 1 || rank == 0) {
#pragma unroll
    for (int s = 0; s < C::STAGES; ++s)
      if (issued & (1u << s)) {
        volatile int no_abort = 0;
        mbar_wait(full0 + 8 * s, (issued_phase >> s) & 1u, &no_abort, p.status);
      }
  }
}

// ------------------------------------------------------------ MMA issuer
template <int MODE, int CG>
__device__ __forceinline__ void mma_issue(const Params& p, uint8_t* ring, uint64_t* full,
                                          uint64_t* empty, uint64_t* tfull, uint64_t* tempty,
                                          uint64_t* drain, uint32_t tmem, volatile int* abort_flag,
                                          int unit, int n_units) {
  using C = Cfg<MODE, CG>;
  int stage = 0;
  uint32_t phase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  bool ok = true;
  WorkIter wi = work_begin<MODE, CG>(p, unit, n_units);
  Work wk;
  while (ok && work_next(wi, wk)) {
    const Tile<MODE, CG> tl = decode_tile<MODE, CG>(p, wk.t);
    const uint32_t idesc = instr_desc_cg<CG>(tl.ncols / C::W);
    if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, p.status)) break;
    tc_fence_after();
    const uint32_t d_tmem = tmem + acc * C::ACC_STRIDE;
    for (int kb = wk.kb0; kb < wk.kb1; ++kb) {
      if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a_addr = smem_u32(ring + stage * C::STAGE_BYTES);
      const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
      for (int k = 0; k < BK / 16; ++k) {
        const uint32_t accum = (kb > wk.kb0 || k > 0) ? 1u : 0u;
#pragma unroll
        for (int w = 0; w < C::W; ++w) {  // W = 2: columns [256 w, 256 w + 256) from B block w
          const uint32_t bw = b_addr + w * SUB * BK * 2 + k * 32;
          if (CG == 1)
            tc_mma(d_tmem + w * 256, smem_desc(a_addr + k * 32), smem_desc(bw), idesc, accum);
          else
            tc2_mma(d_tmem + w * 256, smem_desc(a_addr + k * 32), smem_desc(bw), idesc, accum);
        }
      }
      if (CG == 1)
        tc_commit(smem_u32(&empty[stage]));
      else
        tc2_commit_both(smem_u32(&empty[stage]));
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    if (CG == 1)
      tc_commit(smem_u32(&tfull[acc]));
    else
      tc2_commit_both(smem_u32(&tfull[acc]));
    if (++acc == C::NACC) {
      acc = 0;
      acc_phase ^= 1u;
    }
  }
  // drain: all MMAs this thread issued are complete before TMEM is freed
  if (CG == 1)
    tc_commit(smem_u32(drain));
  else
    tc2_commit_both(smem_u32(drain));
  volatile int no_abort = 0;
  mbar_wait(smem_u32(drain), 0, &no_abort, p.status);
}

// ------------------------------------------------------------- epilogue
// A 32-row x 128-byte block of this warp (lane i holds row i as 32 words: 64
// bf16 or 32 fp32 columns) goes through the warp's 4 KB smem buffer: rows of
// 128 bytes whose 16-byte chunks are XOR-swizzled by (row mod 8), so that the
// row-wise writes and the column-wise reads are both free of bank conflicts.
// Read back, each store instruction covers 4 rows x 128 contiguous bytes
// instead of 32 rows x 16 bytes.  rows / bytes: how many of the block's rows
// and leading bytes of each row (a multiple of 16) exist; ld in bytes.
// 16-byte chunk q (0..7) of this lane's row in the warp's staging block.
__device__ __forceinline__ void stage_chunk(uint32_t stage, int q, uint32_t w0, uint32_t w1,
                                            uint32_t w2, uint32_t w3) {
  const int lane = threadIdx.x & 31;
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                   stage + lane * 128 + ((q ^ (lane & 7)) << 4)),
               "r"(w0), "r"(w1), "r"(w2), "r"(w3)
               : "memory");
}
// Stores the staged block (rows of 128 bytes; see warp_store_block).
__device__ __forceinline__ void warp_flush_block(uint32_t stage, char* base, int64_t ld, int rows,
                                                 int bytes);

__device__ __forceinline__ void warp_store_block(uint32_t stage, const uint32_t (&w)[32],
                                                 char* base, int64_t ld, int rows, int bytes) {
#pragma unroll
  for (int q = 0; q < 8; ++q) stage_chunk(stage, q, w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  warp_flush_block(stage, base, ld, rows, bytes);
}

__device__ __forceinline__ void warp_flush_block(uint32_t stage, char* base, int64_t ld, int rows,
                                                 int bytes) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  const int q = lane & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = i * 4 + (lane >> 3);
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(stage + row * 128 + ((q ^ (row & 7)) << 4))
                 : "memory");
    if (row < rows && q * 16 < bytes)
      *reinterpret_cast<uint4*>(base + (int64_t)row * ld + q * 16) = v;
  }
  __syncwarp();
}

// SiTU of the 64 hidden units at gate columns [c0, c0 + 64) and up columns
// [c0 + 128, c0 + 192) of this warp's 32 TMEM lanes, packed to bf16 and
// written to the warp's staging block (row = lane, 128 bytes); store it with
// warp_flush_block.  Each quarter of 16 units is read from TMEM at once and its
// eight-unit chunks go to shared memory as soon as they are formed, so that
// few values are live besides 32 accumulator columns (the epilogue runs at the
// 168-register cap of 320-thread CTAs).
__device__ __forceinline__ void situ_stage64(uint32_t tbase, uint32_t c0, uint32_t stage,
                                             const SituConsts& sk) {
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    float g[16], u[16];
    tc_ld16x2(tbase + c0 + 16 * h, g, tbase + SUB + c0 + 16 * h, u);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = 8 * q + 2 * j;
        w[j] = situ2_bf16(g[i], g[i + 1], u[i], u[i + 1], sk);
      }
      stage_chunk(stage, 2 * h + q, w[0], w[1], w[2], w[3]);
    }
  }
}

__device__ __forceinline__ void warp_store_bf16(uint32_t stage, const uint32_t (&w)[32],
                                                __nv_bfloat16* base, int64_t ld, int rows,
                                                int cols) {
  warp_store_block(stage, w, reinterpret_cast<char*>(base), ld * 2, rows, cols * 2);
}

// 32 fp32 accumulator columns of the warp's rows (lane = row), cols <= 32 of them.
__device__ __forceinline__ void warp_store_f32(uint32_t stage, const float (&v)[32], float* base,
                                               int64_t ld, int rows, int cols) {
  uint32_t w[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(v[j]);
  warp_store_block(stage, w, reinterpret_cast<char*>(base), ld * 4, rows, cols * 4);
}

// 64 fp32 accumulator columns -> 32 packed bf16x2 words.
__device__ __forceinline__ void pack_block(const float (&a)[32], const float (&b)[32],
                                           uint32_t (&w)[32]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    w[j] = pack_bf16(a[2 * j], a[2 * j + 1]);
    w[16 + j] = pack_bf16(b[2 * j], b[2 * j + 1]);
  }
}

// Routing of one row from its fp32 logits (R <= 32, one TMEM chunk): the K3
// rule s = sigmoid(l), T = TopK(s + b, k) in descending key order (ties to the
// lower expert), p = s_T / max(sum s_T, 1e-9); or (router == 1) T = TopK(l, k),
// p = softmax over the selected logits.  Same operations, in the same order,
// as the standalone top-k kernel.
__device__ __forceinline__ void route_row32(const Params& p, const float (&lg)[32], int64_t row) {
  float sc[32], key[32];
  const bool soft = p.router == 1;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    sc[e] = soft ? lg[e] : 1.0f / (1.0f + expf(-lg[e]));
    key[e] = (e < p.R) ? (soft ? lg[e] : sc[e] + (p.bias != nullptr ? p.bias[e] : 0.0f))
                       : -INFINITY;
  }
  float den = 0.0f, first = 0.0f;
  int32_t* ids = p.ids + row * p.top_k;
  float* probs = p.probs + row * p.top_k;
#pragma unroll 1
  for (int slot = 0; slot < p.top_k; ++slot) {
    int best = 0;
    float bk = key[0];
#pragma unroll
    for (int e = 1; e < 32; ++e)
      if (key[e] > bk) {
        bk = key[e];
        best = e;
      }
    float sel = 0.0f;
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (e == best) {
        sel = sc[e];
        key[e] = -INFINITY;
      }
    if (soft) {
      if (slot == 0) first = sel;
      sel = expf(sel - first);
    }
    ids[slot] = best;
    probs[slot] = sel;
    den += sel;
  }
  if (!soft) den = fmaxf(den, 1e-9f);
#pragma unroll 1
  for (int slot = 0; slot < p.top_k; ++slot) probs[slot] = probs[slot] / den;
}

// Pairs per expert among one warp's 32 rows of a routed x-pass tile (the
// dispatch's count row grow0 / 32): lane e counts the ids equal to e, matching
// the five bits of each id by ballots.  The warp's own ids were just written
// by its lanes, each lane reading its own row.  Kept out of line so that the
// epilogue's registers stay as they are.
__device__ __noinline__ void count_row_experts(const int32_t* ids, int top_k, int R,
                                               int32_t* row_counts, int64_t grow0, int rows) {
  const int lane = threadIdx.x & 31;
  const unsigned have = __ballot_sync(0xffffffffu, lane < rows);
  int32_t cnt = 0;
#pragma unroll 1
  for (int j = 0; j < top_k; ++j) {
    const int e = lane < rows ? ids[(grow0 + lane) * top_k + j] : 0;
    unsigned m = have;
#pragma unroll
    for (int bit = 0; bit < 5; ++bit) {
      const unsigned set = __ballot_sync(0xffffffffu, (e >> bit) & 1);
      m &= ((lane >> bit) & 1) ? set : ~set;
    }
    cnt += __popc(m);
  }
  if (lane < R) row_counts[(grow0 >> 5) * R + lane] = cnt;
}

// x-pass stream-K share of one tile (see the epilogue).  Role 1: store the
// raw accumulator (NB 64-column blocks of this warp's lane quarter, if any
// of its rows exist) and count
// the warp in sk_flags; returns false (no epilogue).  Role 2: wait for the
// shares of units unit + 1 .. sk_last, add them into TMEM in unit order, and
// meet the other epilogue warps at the fix-up barrier (capped), so that the
// epilogue reads fixed columns only; returns whether all of that completed.
template <int NB, int CG>
__device__ __noinline__ bool xpass_sk_fixup(const Params& p, uint32_t tbase, int sk_role, int unit,
                                            int sk_last, uint32_t rank, int ew, int h0,
                                            bool has_rows, uint64_t* fixbar, uint32_t& fix_phase,
                                            volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  auto part = [&](int u, int cb) {
    return reinterpret_cast<float4*>(p.sk_part) +
           ((((size_t)u * 2 + rank) * 4 + ew) * NB + cb) * 16 * 32 + lane;
  };
  bool waited = true;
  if (sk_role == 2 && lane == 0)
    for (int u2 = unit + 1; u2 <= sk_last && waited; ++u2)
      waited = wait_count(p.sk_flags + u2, CG * EPI_WARPS, abort_flag, p.status);
  waited = __shfl_sync(0xffffffffu, (int)waited, 0) != 0;
  __syncwarp();
  // a warp whose 32 rows lie past the tile's last row neither stores nor
  // reads partials (they would never be stored)
#pragma unroll 1
  for (int cb = h0; has_rows && waited && cb < NB; cb += HS) {
    float a[32], b[32];
    tc_ld32x2(tbase + cb * 64, a, tbase + cb * 64 + 32, b);
    if (sk_role == 1) {
      float4* dst = part(unit, cb);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        dst[j * 32] = make_float4(a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]);
        dst[(8 + j) * 32] = make_float4(b[4 * j], b[4 * j + 1], b[4 * j + 2], b[4 * j + 3]);
      }
      continue;
    }
    for (int u2 = unit + 1; u2 <= sk_last; ++u2) {
      const float4* src = part(u2, cb);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 pa = __ldcg(src + j * 32), pb = __ldcg(src + (8 + j) * 32);
        a[4 * j] += pa.x; a[4 * j + 1] += pa.y; a[4 * j + 2] += pa.z; a[4 * j + 3] += pa.w;
        b[4 * j] += pb.x; b[4 * j + 1] += pb.y; b[4 * j + 2] += pb.z; b[4 * j + 3] += pb.w;
      }
    }
    tc_st32x2(tbase + cb * 64, a, tbase + cb * 64 + 32, b);
  }
  if (sk_role == 1) {
    __threadfence();
    __syncwarp();
    if (lane == 0) atomicAdd(p.sk_flags + unit, 1);
    return false;
  }
  // the other epilogue warps' columns are fixed too: an mbarrier with a
  // capped wait (a warp that gave up earlier cannot hang the others)
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(fixbar));
  const bool fixed = mbar_wait(smem_u32(fixbar), fix_phase, abort_flag, p.status);
  fix_phase ^= 1u;
  tc_fence_after();
  return waited && fixed;
}

template <int MODE, int CG>
__device__ __forceinline__ void epilogue(const Params& p, uint64_t* tfull, uint64_t* tempty,
                                         uint64_t* fixbar, uint32_t tmem, uint32_t stage,
                                         volatile int* abort_flag, uint32_t rank, int unit,
                                         int n_units) {
  const int ew = (threadIdx.x >> 5) & 3;  // TMEM lane quarter this warp may access
  // first column block of this warp (then every HS-th)
  const int h0 = EPI_WARPS == 8 ? ((threadIdx.x >> 5) - 2) >> 2 : 0;
  const int lane = threadIdx.x & 31;
  const int wrow = ew * 32 + (CG == 2 ? BM * (int)rank : 0);  // first tile row of this warp
  const SituConsts sk = situ_consts(p);
  if (base_of<MODE>() == FINAL && p.fuse_combine) {
    // The fused combine: uhat rows of an even share per CTA, one warp per row,
    // each row counted in its 256-row tile's word once written.  Runs while the
    // first tile's K loop goes through the shared experts' blocks.
    const int ewarp = (threadIdx.x >> 5) - 2;
    const int64_t per = (p.M + gridDim.x - 1) / gridDim.x;
    const int64_t r0 = (int64_t)blockIdx.x * per, r1 = min((int64_t)p.M, r0 + per);
    for (int64_t t = r0 + ewarp; t < r1; t += EPI_WARPS) {
      if (p.c_vpl == 1)
        combine_row<__nv_bfloat16, 1>(p.c_eo, p.c_inv, p.c_probs, p.c_rms, t, p.c_k, p.L, p.c_eps,
                                      p.c_uhat);
      else if (p.c_vpl == 2)
        combine_row<__nv_bfloat16, 2>(p.c_eo, p.c_inv, p.c_probs, p.c_rms, t, p.c_k, p.L, p.c_eps,
                                      p.c_uhat);
      else
        combine_row<__nv_bfloat16, 4>(p.c_eo, p.c_inv, p.c_probs, p.c_rms, t, p.c_k, p.L, p.c_eps,
                                      p.c_uhat);
      __threadfence();  // every lane's stores of the row, then one count
      __syncwarp();
      if (lane == 0) atomicAdd(p.c_sync + t / Cfg<MODE, CG>::MT, 1);
    }
  }
  int acc = 0;
  uint32_t acc_phase = 0;
  uint32_t fix_phase = 0;  // x-pass stream-K: phase of the fix-up barrier
  const int nkb = k_blocks<MODE>(p);
  const int64_t q_sk = (int64_t)total_tiles<MODE, CG>(p) * nkb;  // stream-K iterations
  WorkIter wi = work_begin<MODE, CG>(p, unit, n_units);
  Work wk;
  while (work_next(wi, wk)) {
    const Tile<MODE, CG> tl = decode_tile<MODE, CG>(p, wk.t);
    // Stream-K (FINAL): a unit that holds K blocks after the first of a tile
    // stores its fp32 partial (role 1) and counts its warps in sk_flags; the
    // unit that holds the tile's first K blocks (role 2) works on them last,
    // waits for the partials of the units after it that hold the rest, and
    // adds them in unit order before the epilogue: a fixed summation order.
    int sk_role = 0, sk_last = unit;
    if ((base_of<MODE>() == FINAL || is_xpass_sk<MODE>()) && p.stream_k) {
      if (wk.kb0 > 0) {
        sk_role = 1;
      } else if (wk.kb1 < nkb) {
        sk_role = 2;
        sk_last = sk_unit_of((int64_t)wk.t * nkb + nkb - 1, q_sk, n_units);
      }
    }
    if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.status)) break;
    tc_fence_after();
    const uint32_t tbase = tmem + ((uint32_t)(ew * 32) << 16) + acc * Cfg<MODE, CG>::ACC_STRIDE;
    const int rows = min(32, tl.rows - wrow);  // rows of this warp inside the tile
    const int64_t grow0 = (int64_t)tl.m0 + wrow;
    bool sk_skip = false;  // x-pass role 1: partial stored, no epilogue
    if constexpr (is_xpass_sk<MODE>()) {
      if (sk_role != 0) {
        // x-pass stream-K: role 1 stores the raw accumulator and skips the
        // epilogue; role 2 adds the other shares into TMEM first
        sk_skip = !xpass_sk_fixup<Cfg<MODE, CG>::W * 4, CG>(p, tbase, sk_role, unit, sk_last,
                                                           rank, ew, h0, rows > 0, fixbar,
                                                           fix_phase, abort_flag);
      }
    }
    if (rows <= 0 || sk_skip) {
      // nothing of this warp's rows exists in the tile (or a stream-K share)
    } else if (tl.epi == EPI_SITU) {
      // columns [0,128) hold gate pre-activations, [128,256) the matching up ones;
      // this warp writes the blocks of 64 hidden units h0, h0 + HS, ...
      int width;
      __nv_bfloat16* out;
      int64_t ld;
      if (is_xpass<MODE>()) {
        width = p.G - (tl.ocol - (tl.ocol / p.G) * p.G);  // hidden units left in this expert
        out = static_cast<__nv_bfloat16*>(p.out2);
        ld = p.ld2;
      } else {
        width = p.F - tl.ocol;
        out = static_cast<__nv_bfloat16*>(p.out0);
        ld = p.ld0;
      }
      if (Cfg<MODE, CG>::W == 2) {
        // blocks of 64 hidden units b (of 4): gate columns 256 (b / 2) + 64 (b % 2),
        // up columns 128 further
#pragma unroll 1
        for (int b = h0; b < 4; b += HS) {
          const int bcols = min(64, width - 64 * b);
          if (bcols <= 0) break;
          const uint32_t c0 = (uint32_t)((b >> 1) * 256 + (b & 1) * 64);
          situ_stage64(tbase, c0, stage, sk);
          warp_flush_block(stage, reinterpret_cast<char*>(out + grow0 * ld + tl.ocol + 64 * b),
                           ld * 2, rows, bcols * 2);
        }
      } else if (MODE == XPASS_F32) {
#pragma unroll 1
        for (int b = h0; b < 2; b += HS) {  // the pre-activations themselves, fp32
          const int cols = min(64, width - b * 64);
          if (cols <= 0) break;
          float g0[32], u0[32], g1[32], u1[32];
          const uint32_t c0 = b * 64;
          tc_ld32x4(tbase + c0, g0, tbase + SUB + c0, u0, tbase + c0 + 32, g1,
                    tbase + SUB + c0 + 32, u1);
          const int64_t at = grow0 * p.ld2 + tl.ocol + b * 64;
          float* ga = static_cast<float*>(p.out2) + at;
          float* ua = static_cast<float*>(p.out3) + at;
          warp_store_f32(stage, g0, ga, p.ld2, rows, min(32, cols));
          warp_store_f32(stage, u0, ua, p.ld2, rows, min(32, cols));
          if (cols > 32) {
            warp_store_f32(stage, g1, ga + 32, p.ld2, rows, cols - 32);
            warp_store_f32(stage, u1, ua + 32, p.ld2, rows, cols - 32);
          }
        }
      } else {
#pragma unroll 1
        for (int b = h0; b < 2; b += HS) {
          const int cols = min(64, width - b * 64);
          if (cols <= 0) break;
          situ_stage64(tbase, (uint32_t)(b * 64), stage, sk);
          warp_flush_block(stage, reinterpret_cast<char*>(out + grow0 * ld + tl.ocol + b * 64),
                           ld * 2, rows, cols * 2);
        }
      }
    } else if (is_xpass<MODE>()) {
#pragma unroll 1
      for (int s = 0; s < tl.n_sub; ++s) {
        if (tl.bmap[s] == kPadMap) continue;
        if (tl.bmap[s] == 1) {  // router logits
          if (p.fuse_topk) {
            // all R <= 32 router logits of a row sit in one 32-column chunk
            if (h0 == 0) {
              float lg[32];
              tc_ld32(tbase + tl.scol[s], lg);
              if (lane < rows) {
                float* dst = static_cast<float*>(p.out1) + (grow0 + lane) * p.ld1;
#pragma unroll
                for (int g4 = 0; g4 < 8; ++g4)
                  if (g4 * 4 < p.R)
                    reinterpret_cast<float4*>(dst)[g4] =
                        make_float4(lg[g4 * 4], lg[g4 * 4 + 1], lg[g4 * 4 + 2], lg[g4 * 4 + 3]);
                route_row32(p, lg, grow0 + lane);
              }
              if (p.row_counts != nullptr && rows > 0)
                count_row_experts(p.ids, p.top_k, p.R, p.row_counts, grow0, rows);
            }
            continue;
          }
#pragma unroll 1
          for (int c = h0; c < tl.srows[s] / 32; c += HS) {
            float v[32];
            tc_ld32(tbase + tl.scol[s] + c * 32, v);
            if (lane >= rows) continue;
            const int col = tl.brow[s] + c * 32;
            float* dst = static_cast<float*>(p.out1) + (grow0 + lane) * p.ld1 + col;
#pragma unroll
            for (int g4 = 0; g4 < 8; ++g4)
              if (col + g4 * 4 < p.R)
                reinterpret_cast<float4*>(dst)[g4] =
                    make_float4(v[g4 * 4], v[g4 * 4 + 1], v[g4 * 4 + 2], v[g4 * 4 + 3]);
          }
          continue;
        }
        // z columns [brow + 64 hb, +64) for the blocks hb of this warp
#pragma unroll 1
        for (int hb = h0; hb < 2; hb += HS) {
          const int col = tl.brow[s] + hb * 64;
          const int cols = min(64, p.L - col);
          if (cols <= 0) break;
          float a[32], b[32];
          tc_ld32x2(tbase + tl.scol[s] + hb * 64, a, tbase + tl.scol[s] + hb * 64 + 32, b);
          if (MODE == XPASS_F32) {
            float* zf = static_cast<float*>(p.out0) + grow0 * p.ld0 + col;
            warp_store_f32(stage, a, zf, p.ld0, rows, min(32, cols));
            if (cols > 32) warp_store_f32(stage, b, zf + 32, p.ld0, rows, cols - 32);
            continue;
          }
          uint32_t w[32];
          pack_block(a, b, w);
          warp_store_bf16(stage, w, static_cast<__nv_bfloat16*>(p.out0) + grow0 * p.ld0 + col,
                          p.ld0, rows, cols);
        }
      }
    } else {
      // FINAL / ROUTED2: accumulator columns [0, ncols) are output columns
      // [ocol, ocol + ncols); this warp writes the 64-column blocks h0, h0 + HS, ...
      const int width = (base_of<MODE>() == FINAL ? p.d : p.L) - tl.ocol;
      const int ncols = min(tl.ncols, width);
      bool waited = true;
      if (sk_role == 2 && lane == 0)  // the partials of units unit + 1 .. sk_last
        for (int u2 = unit + 1; u2 <= sk_last && waited; ++u2)
          waited = wait_count(p.sk_flags + u2, CG * EPI_WARPS, abort_flag, p.status);
      waited = __shfl_sync(0xffffffffu, (int)waited, 0) != 0;
      __syncwarp();  // lane 0's acquire orders the other lanes' partial reads
      const int nblk = p.bn / 64;
#pragma unroll 1
      for (int cb = h0; waited && cb * 64 < ncols; cb += HS) {
        const int cols = min(64, ncols - cb * 64);
        const int64_t col = tl.ocol + cb * 64;
        float a[32], b[32];
        tc_ld32x2(tbase + cb * 64, a, tbase + cb * 64 + 32, b);
        if (sk_role != 0) {
          // partial blocks: [unit][rank][lane quarter][64-column block][16 float4][32 lanes]
          auto part = [&](int u) {
            return reinterpret_cast<float4*>(p.sk_part) +
                   ((((size_t)u * 2 + rank) * 4 + ew) * nblk + cb) * 16 * 32 + lane;
          };
          if (sk_role == 1) {
            float4* dst = part(unit);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              dst[j * 32] = make_float4(a[4 * j], a[4 * j + 1], a[4 * j + 2], a[4 * j + 3]);
              dst[(8 + j) * 32] = make_float4(b[4 * j], b[4 * j + 1], b[4 * j + 2], b[4 * j + 3]);
            }
            continue;
          }
          for (int u2 = unit + 1; u2 <= sk_last; ++u2) {
            const float4* src = part(u2);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 pa = __ldcg(src + j * 32), pb = __ldcg(src + (8 + j) * 32);
              a[4 * j] += pa.x; a[4 * j + 1] += pa.y; a[4 * j + 2] += pa.z; a[4 * j + 3] += pa.w;
              b[4 * j] += pb.x; b[4 * j + 1] += pb.y; b[4 * j + 2] += pb.z; b[4 * j + 3] += pb.w;
            }
          }
        }
        uint32_t w[32];
        pack_block(a, b, w);
        warp_store_bf16(stage, w, static_cast<__nv_bfloat16*>(p.out0) + grow0 * p.ld0 + col,
                        p.ld0, rows, cols);
      }
    }
    if (base_of<MODE>() == FINAL && sk_role == 1) {  // every warp counts, rows or not
      __threadfence();
      __syncwarp();
      if (lane == 0) atomicAdd(p.sk_flags + unit, 1);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (CG == 1)
        mbar_arrive(smem_u32(&tempty[acc]));
      else  // the leader's MMA thread waits for both CTAs' epilogues
        mbar_arrive_cluster(map_to_rank(smem_u32(&tempty[acc]), 0));
    }
    if (++acc == Cfg<MODE, CG>::NACC) {
      acc = 0;
      acc_phase ^= 1u;
    }
  }
}

template <int MODE, int CG>
__global__ void __launch_bounds__(THREADS, 1) umma_gemm_kernel(const __grid_constant__ Params p) {
  using C = Cfg<MODE, CG>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[C::STAGES], empty[C::STAGES], tfull[2], tempty[2], drain,
      fixbar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const uint32_t rank = CG == 2 ? cluster_rank() : 0;
  const int unit = CG == 2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = CG == 2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), EPI_WARPS * CG);
    }
    mbar_init(smem_u32(&drain), 1);
    mbar_init(smem_u32(&fixbar), EPI_WARPS);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x == 32) {  // fetch the encoded tensor maps while the previous kernel finishes
    const CUtensorMap* maps[6] = {&p.tmA0, &p.tmA1, &p.tmB0, &p.tmB1, &p.tmB2, &p.tmB3};
#pragma unroll
    for (int i = 0; i < 6; ++i)
      if (p.map_mask & (1 << i))
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(maps[i]))
                     : "memory");
  }
  if (warp == 1) {
    if (CG == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&tmem_slot)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&tmem_slot)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // everything above overlaps the previous kernel; inputs are read only below
  pdl_trigger();
  pdl_wait();

  if (warp == 0) {
    if ((threadIdx.x & 31) == 0)
      produce<MODE, CG>(p, ring, full, empty, &abort_flag, rank, unit, n_units);
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0 && rank == 0)
      mma_issue<MODE, CG>(p, ring, full, empty, tfull, tempty, &drain, tmem, &abort_flag, unit,
                          n_units);
  } else {
    const uint32_t stage =
        smem_u32(ring) + C::STAGES * C::STAGE_BYTES + (warp - 2) * C::EPI_STAGE;
    epilogue<MODE, CG>(p, tfull, tempty, &fixbar, tmem, stage, &abort_flag, rank, unit, n_units);
  }

  tc_fence_before();
  __syncthreads();
  if (CG == 2) cluster_sync();  // neither CTA frees TMEM or exits while its pair still works
  tc_fence_after();
  if ((base_of<MODE>() == FINAL || is_xpass_sk<MODE>()) && (p.fuse_combine || p.stream_k) &&
      threadIdx.x == 0) {
    // the last CTA to finish (every CTA is past its waits) zeroes the counts
    // and flags for the next launch
    __threadfence();
    if (atomicAdd(p.c_sync + (kSyncWords - 1), 1) == (int)gridDim.x - 1) {
      if (p.fuse_combine) {
        const int n_mt = (p.M + C::MT - 1) / C::MT;
        for (int i = 0; i < n_mt; ++i) atomicExch(p.c_sync + i, 0);
      }
      if (p.stream_k)
        for (int i = 0; i < n_units; ++i) atomicExch(p.sk_flags + i, 0);
      atomicExch(p.c_sync + (kSyncWords - 1), 0);
    }
  }
  if (warp == 1) {
    if (CG == 1)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(TMEM_COLS)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(TMEM_COLS)
                   : "memory");
  }
}

// ------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// bf16 tensor [dim2][dim1][dim0] (dim0 contiguous) with a box of 64 x rows
// (x 1), 128-byte swizzle, zero fill outside the tensor; rank 2 or 3.
// Encoded maps are cached per host thread: a map is a function of the base
// address, the extents, the box and the rank only, so a cached entry with the
// same key is the map the encoder would return (a forward encodes about a
// dozen maps, every call, otherwise).
struct MapKey {
  const void* base;
  uint64_t d0, d1, d2;
  uint32_t box, rank;
  bool operator==(const MapKey& o) const {
    return base == o.base && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && box == o.box &&
           rank == o.rank;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool valid;
};
constexpr int kMapCache = 64;

static bool encode_map(CUtensorMap* m, const void* base, uint64_t dim0, uint64_t dim1,
                       uint64_t dim2, uint32_t box_rows, uint32_t rank) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || dim0 == 0 || dim1 == 0 || dim2 == 0) return false;
  static thread_local MapEntry cache[kMapCache];
  const MapKey key{base, dim0, dim1, dim2, box_rows, rank};
  uint64_t h = reinterpret_cast<uintptr_t>(base) ^ (dim0 * 0x9E3779B97F4A7C15ull) ^
               (dim1 * 0xC2B2AE3D27D4EB4Full) ^ (dim2 << 17) ^ ((uint64_t)box_rows << 7) ^ rank;
  h ^= h >> 29;
  MapEntry& e = cache[h % kMapCache];
  if (e.valid && e.key == key) {
    *m = e.map;
    return true;
  }
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {dim0 * 2, dim0 * dim1 * 2};
  cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  e.key = key;
  e.map = *m;
  e.valid = true;
  return true;
}
static bool make_map(CUtensorMap* m, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                     uint32_t box_rows) {
  return encode_map(m, base, dim0, dim1, dim2, box_rows, dim2 > 1 ? 3 : 2);
}
// Always 3D maps for expert-stacked weights (so the kernel can pass 3 coordinates).
static bool make_map3(CUtensorMap* m, const void* base, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                      uint32_t box_rows) {
  return encode_map(m, base, dim0, dim1, dim2, box_rows, 3);
}

// Per-device launch state: the SM count, and whether each kernel instance has
// had its dynamic shared-memory limit raised on that device (the attribute is
// per device).  Guarded by one mutex; read once per device.
constexpr int kMaxDevices = 64;
static std::mutex g_dev_mu;
static int g_sms[kMaxDevices] = {0};

static int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  return dev;
}

static int num_sms() {
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_sms[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sms[dev] = n > 0 ? n : 148;
  }
  return g_sms[dev];
}

// grid: CTAs (CG = 1) or CTA pairs (CG = 2).
template <int MODE, int CG>
static cudaError_t launch(const Params& p, int grid, cudaStream_t st) {
  static bool attr[kMaxDevices] = {false};
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!attr[dev]) {
      cudaError_t e = cudaFuncSetAttribute(umma_gemm_kernel<MODE, CG>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           Cfg<MODE, CG>::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      attr[dev] = true;
    }
  }
  if (grid <= 0) return cudaSuccess;
  count_launch();
  return launch_pdl(umma_gemm_kernel<MODE, CG>, dim3(CG * grid), dim3(THREADS),
                    (size_t)Cfg<MODE, CG>::SMEM_BYTES, st, CG, p);
}

// Tile width for the plain-store GEMMs: the one of 256, 192, 128 columns that
// minimises (waves of tiles over the SMs) x (columns per tile), ties to the
// wider tile.
static int pick_bn(int m_tiles, int width, int units) {
  int best = 256;
  int64_t best_cost = -1;
  for (int bn : {256, 192, 128}) {
    const int64_t tiles = (int64_t)m_tiles * ((width + bn - 1) / bn);
    const int64_t waves = (tiles + units - 1) / units;
    const int64_t cost = waves * bn;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

static Params base_params(int32_t* status) {
  Params p;
  memset(&p, 0, sizeof(p));
  p.status = status;
  return p;
}

}  // namespace

cudaError_t umma_xpass(const XpassArgs& a, int32_t* status, cudaStream_t st) {
  if (a.N == 0) return cudaSuccess;
  Params p = base_params(status);
  bool ok = make_map(&p.tmA0, a.x, a.d, a.N, 1, BM) &&
            (a.L == 0 || make_map(&p.tmB0, a.w_down, a.d, a.L, 1, SUB)) &&
            (a.R == 0 || make_map(&p.tmB1, a.w_router, a.d, a.R, 1, SUB));
  if (a.S > 0)
    ok = ok && make_map3(&p.tmB2, a.ws_g, a.d, a.G, a.S, SUB) &&
         make_map3(&p.tmB3, a.ws_u, a.d, a.G, a.S, SUB);
  if (!ok) return cudaErrorInvalidValue;
  p.map_mask = 1 | (a.L > 0 ? 4 : 0) | (a.R > 0 ? 8 : 0) | (a.S > 0 ? 16 | 32 : 0);
  p.M = (int)a.N;
  p.kb0 = (a.d + BK - 1) / BK;
  p.L = a.L;
  p.R = a.R;
  p.S = a.S;
  p.G = a.G;
  p.d = a.d;
  const bool f32 = a.z32 != nullptr;
  const bool wide = a.wide && !f32;
  const int ns = wide ? 4 : 2;  // B sub-tiles of 128 rows per tile
  p.nz_sub = (a.L + SUB - 1) / SUB;
  p.nr_sub = (a.R + SUB - 1) / SUB;
  p.n_zr_tiles = (p.nz_sub + p.nr_sub + ns - 1) / ns;
  p.g_blocks = a.S > 0 ? (a.G + SUB * (ns / 2) - 1) / (SUB * (ns / 2)) : 0;
  p.n_tiles = p.n_zr_tiles + a.S * p.g_blocks;
  p.out0 = f32 ? (void*)a.z32 : (void*)a.z;
  p.ld0 = a.L;
  p.out1 = a.logits;
  p.ld1 = a.logits_ld;
  p.out2 = f32 ? (void*)a.a_sh : (void*)a.hsh;
  p.out3 = a.c_sh;
  p.ld2 = (int64_t)a.S * a.G;
  p.beta1 = a.beta1;
  p.beta2 = a.beta2;
  p.inv_beta1 = 1.0f / a.beta1;
  p.inv_beta2 = 1.0f / a.beta2;
  p.beta12 = a.beta1 * a.beta2;
  p.fuse_topk = (a.ids != nullptr && a.R <= 32) ? 1 : 0;
  p.router = a.router;
  p.top_k = a.top_k;
  p.bias = a.bias;
  p.ids = a.ids;
  p.probs = a.probs;
  p.row_counts = p.fuse_topk ? a.row_counts : nullptr;
  const int total = (int)((a.N + 2 * BM - 1) / (2 * BM)) * p.n_tiles;
  const int units = a.max_units > 0 ? std::min(a.max_units, num_sms() / 2) : num_sms() / 2;
  if (f32) return launch<XPASS_F32, 2>(p, std::min(total, units), st);
  int grid = std::min(total, units);
  // Stream-K by the final GEMM's rule (a decode step at the K3 width: 17 row x
  // column tiles of 112 K blocks for 74 pairs)
  const int64_t iters = (int64_t)total * p.kb0;
  const int waves = (total + units - 1) / units;
  const size_t part_bytes = (size_t)units * 2 * BM * (wide ? 4 : 2) * SUB * 4;
  const bool sk_fits = a.sk_part != nullptr && a.sync != nullptr && part_bytes <= a.sk_bytes &&
                       units <= kSyncWords - 1;
  const bool sk_pays = (double)total < 0.9 * waves * units && iters >= 8LL * units;
  if (sk_fits && (a.stream_k == 1 || (a.stream_k < 0 && sk_pays))) {
    p.stream_k = 1;
    p.sk_part = a.sk_part;
    p.sk_flags = a.sync + (kSyncWords - 1 - units);
    p.c_sync = a.sync;
    grid = (int)std::min<int64_t>(units, iters);
  }
  if (p.stream_k)
    return wide ? launch<XPASS_WIDE_SK, 2>(p, grid, st) : launch<XPASS_SK, 2>(p, grid, st);
  return wide ? launch<XPASS_WIDE, 2>(p, grid, st) : launch<XPASS, 2>(p, grid, st);
}

cudaError_t umma_final(const FinalArgs& a, int32_t* status, cudaStream_t st) {
  if (a.N == 0) return cudaSuccess;
  Params p = base_params(status);
  const int m_tiles = (int)((a.N + 2 * BM - 1) / (2 * BM));
  const int units = a.max_units > 0 ? std::min(a.max_units, num_sms() / 2) : num_sms() / 2;
  // wide: 256 x 512 tiles, each CTA loading two 128-row B sub-tiles
  p.bn = a.wide ? 4 * SUB : pick_bn(m_tiles, a.d, units);
  const uint32_t hb = a.wide ? SUB : p.bn / 2;  // rows of each B box a CTA loads
  bool ok = make_map(&p.tmA1, a.uhat, a.L, a.N, 1, BM) && make_map(&p.tmB1, a.w_up, a.L, a.d, 1, hb) &&
            make_map(&p.tmB3, a.w_up, a.L, a.d, 1, hb);
  if (a.S > 0)
    ok = ok && make_map(&p.tmA0, a.hsh, (uint64_t)a.S * a.G, a.N, 1, BM) &&
         make_map3(&p.tmB0, a.ws_o, a.G, a.d, a.S, hb) &&
         make_map3(&p.tmB2, a.ws_o, a.G, a.d, a.S, hb);
  if (!ok) return cudaErrorInvalidValue;
  p.map_mask = 2 | 8 | 32 | (a.S > 0 ? 1 | 4 | 16 : 0);
  p.M = (int)a.N;
  p.S = a.S;
  p.G = a.G;
  p.kb0 = a.S > 0 ? (a.G + BK - 1) / BK : 0;
  p.kb1 = (a.L + BK - 1) / BK;
  p.L = a.L;
  p.d = a.d;
  p.n_tiles = (a.d + p.bn - 1) / p.bn;
  p.out0 = a.y;
  p.ld0 = a.d;
  if (a.eo != nullptr) {
    const int nvec = a.L / 8;
    p.fuse_combine = 1;
    p.c_eo = a.eo;
    p.c_inv = a.inv;
    p.c_probs = a.probs;
    p.c_rms = a.rms_w;
    p.c_uhat = const_cast<__nv_bfloat16*>(a.uhat);
    p.c_sync = a.sync;
    p.c_k = a.top_k;
    p.c_eps = a.rms_eps;
    p.c_vpl = nvec <= 32 ? 1 : nvec <= 64 ? 2 : 4;
    if (nvec > 128 || m_tiles > kSyncWords - 1) return cudaErrorInvalidValue;
  }
  const int total = m_tiles * p.n_tiles;
  int grid = std::min(total, units);
  // Stream-K where whole tiles fill the last wave below 90% (and every pair
  // still gets >= 8 K blocks): the pairs' flags sit after the combine's counts.
  // With the fused combine only while the tiles fill at most half the pairs:
  // a pair's first share is the tail of a tile, whose uhat K blocks then wait
  // for the combine rows at once instead of after the shared experts' blocks
  // (0.5b shape, 64 tiles: final 35 -> 51 us; 12 and 24 tiles at 512 and
  // 1024 tokens: forward 75 -> 71 and 80 -> 75 us).
  const int64_t iters = (int64_t)total * (p.S * p.kb0 + p.kb1);
  const int waves = (total + units - 1) / units;
  const bool sk_fits = a.sk_part != nullptr && a.sync != nullptr &&
                       (size_t)units * 2 * BM * p.bn * 4 <= a.sk_bytes &&
                       (p.fuse_combine ? m_tiles : 0) + units <= kSyncWords - 1;
  const bool sk_pays = (!p.fuse_combine || 2 * total <= units) &&
                       (double)total < 0.9 * waves * units && iters >= 8LL * units;
  if (sk_fits && (a.stream_k == 1 || (a.stream_k < 0 && sk_pays))) {
    p.stream_k = 1;
    p.sk_part = a.sk_part;
    p.sk_flags = a.sync + (kSyncWords - 1 - units);
    p.c_sync = a.sync;  // its last word counts finished CTAs for the flags' reset
    grid = (int)std::min<int64_t>(units, iters);  // every pair holds >= 1 iteration
  }
  return a.wide ? launch<FINAL_WIDE, 2>(p, grid, st) : launch<FINAL, 2>(p, grid, st);
}

cudaError_t umma_routed1(const RoutedArgs& a, int32_t* status, cudaStream_t st) {
  if (a.P == 0) return cudaSuccess;
  Params p = base_params(status);
  bool ok = make_map(&p.tmA0, a.a, a.L, a.P, 1, BM) && make_map3(&p.tmB0, a.w0, a.L, a.F, a.R, SUB) &&
            make_map3(&p.tmB1, a.w1, a.L, a.F, a.R, SUB);
  if (!ok) return cudaErrorInvalidValue;
  p.map_mask = 1 | 4 | 8;
  p.kb0 = (a.L + BK - 1) / BK;
  p.L = a.L;
  p.F = a.F;
  p.R = a.R;
  const bool wide = a.wide && a.pairs;  // 256 hidden units per tile (pairs only)
  p.n_tiles = wide ? (a.F + 2 * SUB - 1) / (2 * SUB) : (a.F + SUB - 1) / SUB;
  p.out0 = a.out;
  p.ld0 = a.F;
  p.tiles = a.tiles;
  p.n_mtiles = a.n_mtiles;
  p.beta1 = a.beta1;
  p.beta2 = a.beta2;
  p.inv_beta1 = 1.0f / a.beta1;
  p.inv_beta2 = 1.0f / a.beta2;
  p.beta12 = a.beta1 * a.beta2;
  const int64_t bound = (int64_t)a.max_tiles * p.n_tiles;
  const int cg = a.pairs ? 2 : 1;
  const int cap = num_sms() / cg;
  const int units = a.max_units > 0 ? std::min(a.max_units, cap) : cap;
  const int grid = (int)std::min<int64_t>(bound, units);
  if (wide) return launch<ROUTED1_WIDE, 2>(p, grid, st);
  return a.pairs ? launch<ROUTED1, 2>(p, grid, st) : launch<ROUTED1, 1>(p, grid, st);
}

cudaError_t umma_routed2(const RoutedArgs& a, int32_t* status, cudaStream_t st) {
  if (a.P == 0) return cudaSuccess;
  Params p = base_params(status);
  const int cg = a.pairs ? 2 : 1;
  const int cap0 = num_sms() / cg;
  const int cap = a.max_units > 0 ? std::min(a.max_units, cap0) : cap0;
  const int tile_m = BM * cg;
  p.bn = pick_bn((int)((a.P + tile_m - 1) / tile_m) + a.R / 2, a.L, cap);
  bool ok = make_map(&p.tmA0, a.a, a.F, a.P, 1, BM);
  if (a.pairs) {  // each CTA of a pair loads bn / 2 rows of W_o,e
    ok = ok && make_map3(&p.tmB0, a.w0, a.F, a.L, a.R, p.bn / 2);
    p.map_mask = 1 | 4;
  } else {
    ok = ok && make_map3(&p.tmB0, a.w0, a.F, a.L, a.R, SUB) &&
         (p.bn == SUB || make_map3(&p.tmB1, a.w0, a.F, a.L, a.R, p.bn - SUB));
    p.map_mask = 1 | 4 | (p.bn == SUB ? 0 : 8);
  }
  if (!ok) return cudaErrorInvalidValue;
  p.kb0 = (a.F + BK - 1) / BK;
  p.L = a.L;
  p.F = a.F;
  p.R = a.R;
  p.n_tiles = (a.L + p.bn - 1) / p.bn;
  p.out0 = a.out;
  p.ld0 = a.L;
  p.tiles = a.tiles;
  p.n_mtiles = a.n_mtiles;
  const int64_t bound = (int64_t)a.max_tiles * p.n_tiles;
  const int grid = (int)std::min<int64_t>(bound, cap);
  return a.pairs ? launch<ROUTED2, 2>(p, grid, st) : launch<ROUTED2, 1>(p, grid, st);
}

}  // namespace lmoe
