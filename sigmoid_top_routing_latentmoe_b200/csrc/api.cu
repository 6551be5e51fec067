// C ABI of the LatentMoE forward library: argument checks, workspace layout
// and the launch sequence of each entry point.  See include/latent_moe.h.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "umma_gemm.h"

namespace lmoe {

static thread_local std::string g_last_error;
static thread_local uint64_t g_launches = 0;

void count_launch(int n) { g_launches += (uint64_t)n; }
void set_last_error(const char* msg) { g_last_error = msg; }

// --------------------------------------------------------------- profiling
// Optional CUDA-event brackets around the launches of named kernels.  Off
// unless lmoe_profile_enable names tags.  Each event is recorded on a side
// branch forked from the launching stream at that point (a library-owned
// stream per thread and device), so no event sits between two kernels of the
// launching stream: it would cut their programmatic (PDL) overlap, about
// 3 us per bracket in a graph replay.  The branch is joined back into the
// launching stream when the public call returns (ProfJoin).
struct ProfRec {
  std::string tag;
  cudaEvent_t a, b;
};
static thread_local std::string g_prof_tags;  // "" off, "*" all, else ",tag1,tag2,"
static thread_local std::vector<ProfRec> g_prof;

static bool prof_wanted(const char* tag) {
  if (g_prof_tags.empty()) return false;
  if (g_prof_tags == "*") return true;
  return g_prof_tags.find("," + std::string(tag) + ",") != std::string::npos;
}

static thread_local cudaStream_t g_prof_side[64];
static thread_local cudaStream_t g_prof_forked = nullptr;  // side stream forked in this call

static bool prof_record(cudaEvent_t ev, cudaStream_t st, unsigned flags) {
  int dev = 0;
  cudaStream_t side = nullptr;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
    if (g_prof_side[dev] == nullptr &&
        cudaStreamCreateWithFlags(&g_prof_side[dev], cudaStreamNonBlocking) != cudaSuccess)
      g_prof_side[dev] = nullptr;
    side = g_prof_side[dev];
  }
  if (side == nullptr) return cudaEventRecordWithFlags(ev, st, flags) == cudaSuccess;
  cudaEvent_t fork;
  if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess) return false;
  const bool ok = cudaEventRecord(fork, st) == cudaSuccess &&
                  cudaStreamWaitEvent(side, fork, 0) == cudaSuccess &&
                  cudaEventRecordWithFlags(ev, side, flags) == cudaSuccess;
  cudaEventDestroy(fork);
  g_prof_forked = side;
  return ok;
}

// Joins the profiling side branch back into the call's stream (a stream
// capture must end with every forked stream joined).
struct ProfJoin {
  cudaStream_t st;
  explicit ProfJoin(cudaStream_t s) : st(s) {}
  ~ProfJoin() {
    if (g_prof_forked == nullptr) return;
    cudaEvent_t j;
    if (cudaEventCreateWithFlags(&j, cudaEventDisableTiming) == cudaSuccess) {
      cudaEventRecord(j, g_prof_forked);
      cudaStreamWaitEvent(st, j, 0);
      cudaEventDestroy(j);
    }
    g_prof_forked = nullptr;
  }
};

struct ProfScope {
  bool on = false;
  cudaStream_t st;
  ProfRec r{};
  unsigned flags = cudaEventRecordDefault;
  ProfScope(const char* tag, cudaStream_t s) : st(s) {
    if (!prof_wanted(tag)) return;
    r.tag = tag;
    if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) return;
    // inside a stream capture the events become event-record nodes of the graph
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
      flags = cudaEventRecordExternal;
    on = prof_record(r.a, st, flags);
  }
  ~ProfScope() {
    if (!on) return;
    prof_record(r.b, st, flags);
    g_prof.push_back(r);
  }
};

static lmoe_status fail(lmoe_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

static lmoe_status cuda_fail(cudaError_t e, const char* where) {
  return fail(LMOE_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define LMOE_CUDA(call, where)                      \
  do {                                              \
    cudaError_t _e = (call);                        \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

// ------------------------------------------------------------- device check
static lmoe_status check_device() {
  static std::mutex mu;
  static int arch_ok[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  LMOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LMOE_EUNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  if (arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    LMOE_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev), "attr");
    LMOE_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev), "attr");
    arch_ok[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  if (arch_ok[dev] != 1) return fail(LMOE_EUNSUPPORTED, "device %d is not sm_100 (B200)", dev);
  return LMOE_OK;
}

// ------------------------------------------------------------- validation
static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static lmoe_status check_dims(const lmoe_dims* d) {
  if (d == nullptr) return fail(LMOE_EINVAL, "dims is NULL");
  if (d->dtype != LMOE_F32 && d->dtype != LMOE_BF16) return fail(LMOE_EINVAL, "dtype %d", d->dtype);
  if (d->n_tokens < 0) return fail(LMOE_EINVAL, "n_tokens < 0");
  if (d->d <= 0 || d->latent <= 0 || d->ff_routed <= 0)
    return fail(LMOE_EINVAL, "d, latent and ff_routed must be positive");
  if (d->n_routed < 1 || d->n_routed > 4096) return fail(LMOE_EUNSUPPORTED, "n_routed out of [1, 4096]");
  if (d->top_k < 1 || d->top_k > d->n_routed) return fail(LMOE_EINVAL, "top_k out of [1, n_routed]");
  if (d->n_shared < 0 || d->n_shared > kMaxSeg - 1) return fail(LMOE_EUNSUPPORTED, "n_shared out of [0, 7]");
  if (d->n_shared > 0 && d->ff_shared <= 0) return fail(LMOE_EINVAL, "ff_shared must be positive");
  if (d->d % 8 || d->latent % 8 || d->ff_routed % 8 || (d->n_shared > 0 && d->ff_shared % 8))
    return fail(LMOE_EINVAL, "d, latent, ff_routed and ff_shared must be multiples of 8");
  if (d->latent > 4096) return fail(LMOE_EUNSUPPORTED, "latent > 4096");
  if (d->d > 65536) return fail(LMOE_EUNSUPPORTED, "d > 65536");
  if (d->n_tokens * (int64_t)d->top_k >= ((int64_t)1 << 31) - kTileM * 8)
    return fail(LMOE_EUNSUPPORTED, "n_tokens * top_k too large");
  if (!(d->beta1 > 0.0f) || !(d->beta2 > 0.0f) || !(d->rms_eps >= 0.0f))
    return fail(LMOE_EINVAL, "beta1, beta2 must be > 0 and rms_eps >= 0");
  if (d->router != LMOE_ROUTER_K3 && d->router != LMOE_ROUTER_SOFTMAX_TOPK)
    return fail(LMOE_EINVAL, "router %d", d->router);
  return LMOE_OK;
}

#define LMOE_PTR(p, name)                                                          \
  do {                                                                             \
    if ((p) == nullptr) return fail(LMOE_EINVAL, "%s is NULL", name);              \
    if (!aligned16(p)) return fail(LMOE_EINVAL, "%s is not 16-byte aligned", name); \
  } while (0)

// ------------------------------------------------------------ workspace
static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }
constexpr int kSkMaxPairs = 80;  // CTA pairs the stream-K scratch is sized for

struct Layout {
  size_t header, sync, z, logits, ids, probs, counts, offsets, perm, inv, block_counts, tiles, tiles2,
      zp, h, skx, eo, hsh, uhat, loss, x, y, total;
  int64_t logits_ld;
  int max_tiles;
};

static Layout layout(const lmoe_dims* d, bool host_copies) {
  Layout L{};
  const int64_t N = d->n_tokens, P = N * d->top_k;
  const size_t es = d->dtype == LMOE_BF16 ? 2 : 4;
  const int R = d->n_routed;
  L.logits_ld = (R + 15) / 16 * 16;
  L.max_tiles = (int)(P / kTileM + R + 1);
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t at = off; off += align256(bytes); return at; };
  L.header = take(sizeof(WsHeader));
  L.sync = take((size_t)kSyncWords * 4);  // right after the header: cleared with it
  L.z = take((size_t)N * d->latent * es);
  L.logits = take((size_t)N * L.logits_ld * 4);
  L.ids = take((size_t)P * 4);
  L.probs = take((size_t)P * 4);
  L.counts = take((size_t)R * 4);
  L.offsets = take((size_t)(R + 1) * 4);
  L.perm = take((size_t)P * 4);
  L.inv = take((size_t)P * 4);
  L.block_counts = take((size_t)dispatch_count_rows(N, d->top_k) * R * 4);
  L.tiles = take((size_t)L.max_tiles * sizeof(int4));
  L.tiles2 = take((size_t)L.max_tiles * sizeof(int4));
  L.zp = take((size_t)P * d->latent * es);
  L.h = take((size_t)P * d->ff_routed * es);
  // The stream-K partials of the x-pass (before the dispatch writes zp) and of
  // the final GEMM (after the routed GEMMs) reuse [zp, eo); this tops it up
  // to one 256-row tile of fp32 per CTA pair (up to kSkMaxPairs).
  if (d->dtype == LMOE_BF16) {
    const size_t bn_max = d->d >= 4096 ? 512 : 256;
    const size_t need = (size_t)kSkMaxPairs * 2 * 128 * bn_max * 4, have = off - L.zp;
    L.skx = take(need > have ? need - have : 0);
  } else {
    L.skx = take(0);
  }
  L.eo = take((size_t)P * d->latent * es);
  L.hsh = take((size_t)N * d->n_shared * (size_t)d->ff_shared * es);
  L.uhat = take((size_t)N * d->latent * es);
  // scratch of moe_router_losses: per block of tokens, R sigmoid sums, R counts, one z sum
  L.loss = take((size_t)loss_blocks(N) * (2 * (size_t)R + 1) * 4);
  if (host_copies) {
    L.x = take((size_t)N * d->d * es);
    L.y = take((size_t)N * d->d * es);
  }
  L.total = off;
  return L;
}

template <typename P>
static P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

static lmoe_status check_ws(const lmoe_dims* d, void* ws, size_t ws_bytes, bool host) {
  LMOE_PTR(ws, "ws");
  if (((uintptr_t)ws & 255u) != 0) return fail(LMOE_EINVAL, "ws must be 256-byte aligned");
  size_t need = layout(d, host).total;
  if (ws_bytes < need)
    return fail(LMOE_EWORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
  return LMOE_OK;
}

#define LMOE_TRY(expr)                  \
  do {                                  \
    lmoe_status _s = (expr);            \
    if (_s != LMOE_OK) return _s;       \
  } while (0)

// ------------------------------------------------------------- launchers
template <typename T>
static lmoe_status run_route(const lmoe_dims* d, const void* x, const void* w_r, const float* bias,
                             int32_t* ids, float* probs, void* ws, cudaStream_t st) {
  const Layout L = layout(d, false);
  const int64_t N = d->n_tokens;
  if (N == 0) return LMOE_OK;
  float* logits = at<float>(ws, L.logits);
  if (d->n_routed <= 32) {
    ProfScope ps("route", st);
    LMOE_CUDA(launch_route_gemv<T>((const T*)x, (const T*)w_r, bias, N, d->d, d->n_routed,
                                   d->top_k, d->router, ids, probs, logits, L.logits_ld, st),
              "route_gemv");
    return LMOE_OK;
  }
  ProfScope ps("route", st);
  if (std::is_same<T, __nv_bfloat16>::value) {
    XpassArgs a{};
    a.x = (const __nv_bfloat16*)x; a.N = N; a.d = d->d; a.L = 0; a.w_router = (const __nv_bfloat16*)w_r;
    a.R = d->n_routed; a.S = 0; a.logits = logits; a.logits_ld = L.logits_ld;
    a.beta1 = d->beta1; a.beta2 = d->beta2;
    LMOE_CUDA(umma_xpass(a, &at<WsHeader>(ws, L.header)->status, st), "router logits (tcgen05)");
  } else {
    SimtGemm g{};
    g.A[0] = x; g.lda[0] = d->d; g.B[0] = w_r; g.ldb[0] = d->d; g.K[0] = d->d; g.nseg = 1;
    g.C = logits; g.ldc = L.logits_ld; g.M = (int)N; g.N = d->n_routed; g.out_f32 = 1;
    g.mode = kStore;
    LMOE_CUDA(launch_simt_gemm<T>(g, st), "router logits");
  }
  LMOE_CUDA(launch_route_topk(logits, L.logits_ld, bias, N, d->n_routed, d->top_k, d->router, ids,
                              probs, st),
            "route_topk");
  return LMOE_OK;
}

// The bf16 routed GEMMs run on CTA pairs over <= 256-row tiles, or on single
// CTAs over <= 128.  Pairs when experts average 64 to 256 sorted pairs: one
// pair tile then covers an expert's rows, so its weights stream once per
// output tile, half through each SM (K3 width, 146 rows per expert: W_o GEMM
// 1093 -> 889 us).  With more rows per expert GEMM1 stays on pairs only for a
// long K (l >= 1024; mid shape, 2048 rows per expert: GEMM1 528 -> 469 us on
// pairs, while GEMM2 went 280 -> 418 us, so GEMM2 stays single; 0.5b shape,
// l = 384: both slower on pairs, 14.7 -> 19.8 and 8.1 -> 10.8 us).  For
// decode-like loads of a few rows a 256-row MMA would mostly multiply empty rows.
static bool routed_pairs(const lmoe_dims* d, int gemm) {
  const int64_t pairs = d->n_tokens * (int64_t)d->top_k, R = d->n_routed;
  if (d->dtype != LMOE_BF16 || pairs < 64 * R) return false;
  return pairs <= 256 * R || (gemm == 1 && d->latent >= 1024);
}
// height of the tile list the dispatch writes (GEMM1's)
static int routed_tile_m(const lmoe_dims* d, int gemm = 1) {
  return routed_pairs(d, gemm) ? kRoutedPairTileM : kTileM;
}

// z != nullptr: the scatter also writes the sorted rows of z to the workspace
// (the A operand of the routed GEMMs).
// row_counts: the x-pass wrote the expert counts of every 32 tokens to the
// dispatch's count scratch (counts_in_xpass), so no histogram is launched.
static lmoe_status run_dispatch(const lmoe_dims* d, const int32_t* ids, int32_t* counts,
                                int32_t* offsets, int32_t* perm, int32_t* inv, void* ws,
                                cudaStream_t st, const void* z = nullptr,
                                bool row_counts = false) {
  const Layout L = layout(d, false);
  DispatchScratch s;
  s.block_counts = at<int32_t>(ws, L.block_counts);
  s.status = &at<WsHeader>(ws, L.header)->status;
  s.n_mtiles = &at<WsHeader>(ws, L.header)->n_mtiles;
  s.tiles = at<int4>(ws, L.tiles);
  ProfScope ps("dispatch", st);
  const int es = d->dtype == LMOE_BF16 ? 2 : 4;
  LMOE_CUDA(launch_dispatch(ids, d->n_tokens, d->top_k, d->n_routed, counts, offsets, perm, inv,
                            s, st, z, z != nullptr ? at<char>(ws, L.zp) : nullptr,
                            d->latent * es, routed_tile_m(d), row_counts),
            "dispatch");
  return LMOE_OK;
}

// Routed experts on sorted pairs; the tile list must already be in the workspace.
// perm holds the token of each sorted pair: its rows of z are first copied in
// sorted order, the A operand of GEMM1, unless the dispatch already did
// (rows_sorted).
template <typename T>
static lmoe_status run_expert_ffn(const lmoe_dims* d, const void* z, const int32_t* perm,
                                  const int32_t* offsets, const void* w_g, const void* w_u,
                                  const void* w_o, void* eo, void* ws, cudaStream_t st,
                                  bool rows_sorted = false) {
  const Layout L = layout(d, false);
  const int64_t P = d->n_tokens * d->top_k;
  if (P == 0) return LMOE_OK;
  const int Lt = d->latent, F = d->ff_routed;
  T* zp = at<T>(ws, L.zp);
  T* h = at<T>(ws, L.h);
  const int4* tiles = at<int4>(ws, L.tiles);
  const int32_t* n_tiles = &at<WsHeader>(ws, L.header)->n_mtiles;
  const bool tc = std::is_same<T, __nv_bfloat16>::value;
  // GEMM2's tile list: GEMM1's, or its own at the other height
  const int4* tiles2 = tiles;
  const int32_t* n_tiles2 = n_tiles;
  if (routed_tile_m(d, 2) != routed_tile_m(d, 1)) {
    tiles2 = at<int4>(ws, L.tiles2);
    n_tiles2 = &at<WsHeader>(ws, L.header)->n_mtiles2;
    LMOE_CUDA(launch_build_tiles(offsets, d->n_routed, const_cast<int32_t*>(n_tiles2),
                                 const_cast<int4*>(tiles2), st, routed_tile_m(d, 2)),
              "build_tiles");
  }
  if (!rows_sorted) {
    ProfScope ps("gather", st);
    LMOE_CUDA(launch_gather_rows<T>((const T*)z, perm, P, Lt, zp, st), "gather");
  }
  SimtGemm g1{};
  g1.A[0] = zp; g1.lda[0] = Lt; g1.B[0] = w_g; g1.ldb[0] = Lt; g1.K[0] = Lt; g1.nseg = 1;
  g1.B_up = w_u; g1.b_expert_stride = (int64_t)F * Lt;
  g1.C = h; g1.ldc = F; g1.N = F; g1.tiles = tiles; g1.n_tiles = n_tiles;
  g1.max_tiles = L.max_tiles; g1.beta1 = d->beta1; g1.beta2 = d->beta2; g1.mode = kSitu;
  int32_t* status = &at<WsHeader>(ws, L.header)->status;
  RoutedArgs ra{};
  ra.P = P; ra.L = Lt; ra.F = F; ra.R = d->n_routed; ra.tiles = tiles; ra.n_mtiles = n_tiles;
  ra.max_tiles = L.max_tiles; ra.beta1 = d->beta1; ra.beta2 = d->beta2;
  ra.pairs = routed_pairs(d, 1) ? 1 : 0;
  // pairs with a long K (l >= 2048): GEMM1 on 256 x 512 tiles, 256 hidden units each
  ra.wide = ra.pairs && Lt >= 2048 ? 1 : 0;
  {
    ProfScope ps("expert_gemm1", st);
    if (tc) {
      ra.a = (const __nv_bfloat16*)zp; ra.w0 = (const __nv_bfloat16*)w_g;
      ra.w1 = (const __nv_bfloat16*)w_u; ra.out = (__nv_bfloat16*)h;
      LMOE_CUDA(umma_routed1(ra, status, st), "routed gemm1 (tcgen05)");
    } else {
      LMOE_CUDA(launch_simt_gemm<T>(g1, st), "routed gemm1");
    }
  }
  SimtGemm g2{};
  g2.A[0] = h; g2.lda[0] = F; g2.B[0] = w_o; g2.ldb[0] = F; g2.K[0] = F; g2.nseg = 1;
  g2.b_expert_stride = (int64_t)Lt * F;
  g2.C = eo; g2.ldc = Lt; g2.N = Lt; g2.tiles = tiles2; g2.n_tiles = n_tiles2;
  g2.max_tiles = L.max_tiles; g2.mode = kStore;
  {
    ProfScope ps("expert_gemm2", st);
    if (tc) {
      ra.a = (const __nv_bfloat16*)h; ra.w0 = (const __nv_bfloat16*)w_o; ra.w1 = nullptr;
      ra.out = (__nv_bfloat16*)eo;
      ra.pairs = routed_pairs(d, 2) ? 1 : 0;
      ra.tiles = tiles2; ra.n_mtiles = n_tiles2;
      LMOE_CUDA(umma_routed2(ra, status, st), "routed gemm2 (tcgen05)");
    } else {
      LMOE_CUDA(launch_simt_gemm<T>(g2, st), "routed gemm2");
    }
  }
  return LMOE_OK;
}

// Stream-K for the x-pass and the final GEMM: chosen by the wave fill unless
// LMOE_STREAM_K is 0 (never) or 1 (whenever its scratch fits).
static int stream_k_mode() {
  if (const char* v = getenv("LMOE_STREAM_K")) {
    if (v[0] == '0') return 0;
    if (v[0] == '1') return 1;
  }
  return -1;
}

// The forward's x-pass runs on 256 x 256 tiles with a double-buffered
// accumulator.  The engine's 256 x 512 x-pass tiles (1.33x the FLOPs per
// streamed byte, one accumulator, the SiTU epilogue exposed once per tile) won
// at d >= 2048 only while the tiles went rows-fastest over all row tiles;
// with the grouped tile order the 256 x 256 tiles measured faster at every
// shape (mid: x-pass 470 -> 420 us; K3 width 708 -> 688 us; decode step
// 76 -> 59 us), so the wide x-pass is not chosen (XpassArgs.wide still works).
static int xpass_wide(const lmoe_dims*) { return 0; }

// The scatter also writes the sorted copy of z when it is at most 16 MiB and
// there are at least 4096 pairs (enough chunks to spread the copy over many
// CTAs); otherwise the gather kernel does (decode step, 1024 pairs: dispatch +
// copy 26 -> 17 us).
static bool rows_in_scatter(const lmoe_dims* d) {
  const size_t es = d->dtype == LMOE_BF16 ? 2 : 4;
  const int64_t P = d->n_tokens * (int64_t)d->top_k;
  return (uint64_t)P * d->latent * es <= (16u << 20) && P >= 4096;
}

// With routing in the x-pass's epilogue (R <= 32) the epilogue also counts
// each 32 tokens' pairs per expert, and the dispatch starts from those counts
// instead of launching its histogram kernel (0.5b shape: one launch fewer).
// LMOE_XPASS_COUNTS=0 keeps the histogram kernel.
static bool counts_in_xpass(const lmoe_dims* d) {
  if (const char* v = getenv("LMOE_XPASS_COUNTS"))
    if (v[0] == '0') return false;
  return d->dtype == LMOE_BF16 && d->n_routed <= 32 &&
         dispatch_takes_row_counts(d->n_tokens, d->top_k, d->n_routed);
}

// The combine inside the final GEMM (bf16, l <= 1024, <= 64 MB of expert outputs).
static bool combine_fused(const lmoe_dims* d) {
  return d->dtype == LMOE_BF16 && d->latent <= 1024 &&
         (d->n_tokens + 255) / 256 <= kSyncWords - 1 &&
         (double)d->n_tokens * d->top_k * d->latent * 2.0 <= 64.0 * (1 << 20);
}

// bf16 forward on the tensor cores, one stream: the x-pass (z, routing and the
// shared experts' hidden units), dispatch, the routed experts, combine +
// RMSNorm, and one GEMM for y = shared + W_up RMSNorm(u).
static lmoe_status run_forward_tc(const lmoe_dims* d, const lmoe_weights* w, const void* x,
                                  void* y, int32_t* ids_out, float* probs_out, int32_t* counts_out,
                                  void* ws, cudaStream_t st) {
  typedef __nv_bfloat16 T;
  const Layout L = layout(d, false);
  const int64_t N = d->n_tokens;
  const int Lt = d->latent, S = d->n_shared, G = d->ff_shared, D = d->d, R = d->n_routed;
  const int k = d->top_k;
  int32_t* ids = ids_out ? ids_out : at<int32_t>(ws, L.ids);
  float* probs = probs_out ? probs_out : at<float>(ws, L.probs);
  int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  T* z = at<T>(ws, L.z);
  T* hsh = at<T>(ws, L.hsh);
  T* eo = at<T>(ws, L.eo);
  T* uhat = at<T>(ws, L.uhat);
  float* logits = at<float>(ws, L.logits);
  int32_t* status = &at<WsHeader>(ws, L.header)->status;
  if (N == 0) {
    LMOE_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * R, st), "memset");
    return LMOE_OK;
  }
  const bool row_counts = counts_in_xpass(d);
  // steps 1, 2 and 4 in one pass over x (routing in the epilogue when R <= 32)
  {
    XpassArgs a{};
    a.x = (const T*)x; a.N = N; a.d = D;
    a.w_down = (const T*)w->w_down; a.L = Lt;
    a.w_router = (const T*)w->w_router; a.R = R;
    a.ws_g = (const T*)w->ws_g; a.ws_u = (const T*)w->ws_u; a.S = S; a.G = G;
    a.z = z; a.logits = logits; a.logits_ld = L.logits_ld;
    a.hsh = hsh; a.beta1 = d->beta1; a.beta2 = d->beta2;
    a.bias = w->expert_bias; a.ids = ids; a.probs = probs; a.top_k = k; a.router = d->router;
    if (row_counts) a.row_counts = at<int32_t>(ws, L.block_counts);
    a.wide = xpass_wide(d);
    // stream-K scratch: the sorted-z / routed-hidden region, unused until the dispatch
    a.sync = at<int32_t>(ws, L.sync);
    a.sk_part = at<float>(ws, L.zp);
    a.sk_bytes = L.eo - L.zp;
    a.stream_k = stream_k_mode();
    ProfScope ps("xpass", st);
    LMOE_CUDA(umma_xpass(a, status, st), "x-pass (tcgen05)");
  }
  if (R > 32) {
    ProfScope ps("route", st);
    LMOE_CUDA(launch_route_topk(logits, L.logits_ld, w->expert_bias, N, R, k, d->router, ids,
                                probs, st),
              "route_topk");
  }
  // step 3: dispatch, routed experts, combine + RMSNorm
  // Mid-sized sorted copies of z are made by the scatter itself, saving a
  // launch; others by the gather kernel (rows_in_scatter).
  const bool fuse_rows = rows_in_scatter(d);
  LMOE_TRY(run_dispatch(d, ids, counts, offsets, perm, inv, ws, st, fuse_rows ? z : nullptr,
                        row_counts));
  LMOE_TRY(run_expert_ffn<T>(d, z, perm, offsets, w->w_g, w->w_u, w->w_o, eo, ws, st, fuse_rows));
  // For l <= 1024 and up to 64 MB of expert outputs the combine runs inside
  // the final GEMM (its epilogue warps write RMSNorm(u) while the K loop goes
  // through the shared experts' blocks; 0.5b shape: combine + final 34 -> 31 us).
  // Larger volumes get the combine kernel first: their reads compete with the
  // final GEMM's own (mid shape, 268 MB: +23 us per step fused).
  const bool fuse_combine = combine_fused(d);
  if (!fuse_combine) {
    ProfScope ps("combine", st);
    LMOE_CUDA(launch_combine<T>(eo, inv, probs, w->rms_weight, N, k, Lt, d->rms_eps, uhat, st),
              "combine");
  }
  // step 5: y = shared + W_up uhat in one accumulator
  {
    FinalArgs a{};
    a.hsh = hsh; a.N = N; a.S = S; a.G = G; a.ws_o = (const T*)w->ws_o; a.d = D;
    a.uhat = uhat; a.L = Lt; a.w_up = (const T*)w->w_up; a.y = (T*)y;
    // wide output rows (d >= 4096) with a long K: 256 x 512 tiles
    a.wide = D >= 4096 && S * G + Lt >= 4096 ? 1 : 0;
    if (fuse_combine) {
      a.eo = eo; a.inv = inv; a.probs = probs; a.rms_w = w->rms_weight; a.top_k = k;
      a.rms_eps = d->rms_eps;
    }
    a.sync = at<int32_t>(ws, L.sync);
    // stream-K partials go to the sorted z copy and the routed hidden units,
    // both dead once the routed GEMMs are done
    a.sk_part = at<float>(ws, L.zp);
    a.sk_bytes = L.eo - L.zp;
    a.stream_k = stream_k_mode();
    ProfScope ps("final", st);
    LMOE_CUDA(umma_final(a, status, st), "final (tcgen05)");
  }
  return LMOE_OK;
}

// fp32 forward on the CUDA cores (the debug/reference-precision mode).
template <typename T>
static lmoe_status run_forward(const lmoe_dims* d, const lmoe_weights* w, const void* x, void* y,
                               int32_t* ids_out, float* probs_out, int32_t* counts_out, void* ws,
                               cudaStream_t st) {
  const Layout L = layout(d, false);
  const int64_t N = d->n_tokens;
  const int Lt = d->latent, S = d->n_shared, G = d->ff_shared, D = d->d;
  int32_t* ids = ids_out ? ids_out : at<int32_t>(ws, L.ids);
  float* probs = probs_out ? probs_out : at<float>(ws, L.probs);
  int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  T* z = at<T>(ws, L.z);
  T* hsh = at<T>(ws, L.hsh);
  T* eo = at<T>(ws, L.eo);
  T* uhat = at<T>(ws, L.uhat);
  if (N == 0) {
    LMOE_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * d->n_routed, st), "memset");
    return LMOE_OK;
  }
  // step 1: z = W_down x
  {
    SimtGemm g{};
    g.A[0] = x; g.lda[0] = D; g.B[0] = w->w_down; g.ldb[0] = D; g.K[0] = D; g.nseg = 1;
    g.C = z; g.ldc = Lt; g.M = (int)N; g.N = Lt; g.mode = kStore;
    ProfScope ps("xpass", st);
    LMOE_CUDA(launch_simt_gemm<T>(g, st), "down");
  }
  // step 4 (independent of routing): h_sh = SiTU hidden of the shared experts
  if (S > 0) {
    SimtGemm g{};
    g.A[0] = x; g.lda[0] = D; g.B[0] = w->ws_g; g.ldb[0] = D; g.K[0] = D; g.nseg = 1;
    g.B_up = w->ws_u; g.C = hsh; g.ldc = (int64_t)S * G; g.M = (int)N; g.N = S * G;
    g.beta1 = d->beta1; g.beta2 = d->beta2; g.mode = kSitu;
    ProfScope ps("xpass", st);
    LMOE_CUDA(launch_simt_gemm<T>(g, st), "shared gemm1");
  }
  // step 2: routing
  LMOE_TRY(run_route<T>(d, x, w->w_router, w->expert_bias, ids, probs, ws, st));
  // step 3: dispatch, routed experts, combine + RMSNorm
  // Mid-sized sorted copies of z are made by the scatter itself, saving a
  // launch; others by the gather kernel (rows_in_scatter).
  const bool fuse_rows = rows_in_scatter(d);
  LMOE_TRY(run_dispatch(d, ids, counts, offsets, perm, inv, ws, st, fuse_rows ? z : nullptr));
  LMOE_TRY(run_expert_ffn<T>(d, z, perm, offsets, w->w_g, w->w_u, w->w_o, eo, ws, st, fuse_rows));
  {
    ProfScope ps("combine", st);
    LMOE_CUDA(launch_combine<T>(eo, inv, probs, w->rms_weight, N, d->top_k, Lt, d->rms_eps, uhat,
                                st),
              "combine");
  }
  // step 5: y = sum_j W_o,sh_j h_sh_j + W_up uhat
  {
    SimtGemm g{};
    int s = 0;
    for (int j = 0; j < S; ++j, ++s) {
      g.A[s] = hsh + (int64_t)j * G; g.lda[s] = (int64_t)S * G;
      g.B[s] = static_cast<const T*>(w->ws_o) + (int64_t)j * D * G; g.ldb[s] = G; g.K[s] = G;
    }
    g.A[s] = uhat; g.lda[s] = Lt; g.B[s] = w->w_up; g.ldb[s] = Lt; g.K[s] = Lt; ++s;
    g.nseg = s; g.C = y; g.ldc = D; g.M = (int)N; g.N = D; g.mode = kStore;
    ProfScope ps("final", st);
    LMOE_CUDA(launch_simt_gemm<T>(g, st), "final");
  }
  return LMOE_OK;
}

static lmoe_status check_weights(const lmoe_dims* d, const lmoe_weights* w) {
  if (w == nullptr) return fail(LMOE_EINVAL, "weights is NULL");
  LMOE_PTR(w->w_down, "w_down");
  LMOE_PTR(w->w_router, "w_router");
  LMOE_PTR(w->w_up, "w_up");
  LMOE_PTR(w->rms_weight, "rms_weight");
  if (w->expert_bias != nullptr && !aligned16(w->expert_bias))
    return fail(LMOE_EINVAL, "expert_bias is not 16-byte aligned");
  LMOE_PTR(w->w_g, "w_g");
  LMOE_PTR(w->w_u, "w_u");
  LMOE_PTR(w->w_o, "w_o");
  if (d->n_shared > 0) {
    LMOE_PTR(w->ws_g, "ws_g");
    LMOE_PTR(w->ws_u, "ws_u");
    LMOE_PTR(w->ws_o, "ws_o");
  }
  return LMOE_OK;
}

// ------------------------------------------------------ host entry point
// latent_moe_forward_host pipelines chunks of tokens: the x chunks go to the
// device on one copy stream, each chunk's forward runs on the caller's stream
// as soon as its x has landed, and its y returns on a second copy stream while
// the next chunk computes.  The two copy streams and the events are created
// once per device and kept for the life of the process.
constexpr int kMaxHostChunks = 8;
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in_done[kMaxHostChunks] = {}, fwd_done[kMaxHostChunks] = {};
};

static lmoe_status host_pipe(HostPipe** out) {
  static std::mutex mu;
  static HostPipe pipes[64];
  static bool ready[64] = {false};
  int dev = 0;
  LMOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LMOE_EUNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(mu);
  HostPipe& p = pipes[dev];
  if (!ready[dev]) {
    const unsigned ef = cudaEventDisableTiming;
    LMOE_CUDA(cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking), "copy stream");
    LMOE_CUDA(cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking), "copy stream");
    LMOE_CUDA(cudaEventCreateWithFlags(&p.start, ef), "event");
    LMOE_CUDA(cudaEventCreateWithFlags(&p.done, ef), "event");
    for (int c = 0; c < kMaxHostChunks; ++c) {
      LMOE_CUDA(cudaEventCreateWithFlags(&p.in_done[c], ef), "event");
      LMOE_CUDA(cudaEventCreateWithFlags(&p.fwd_done[c], ef), "event");
    }
    ready[dev] = true;
  }
  *out = &p;
  return LMOE_OK;
}

// Number of token chunks for the host entry point, from a cost model of the
// pipeline copy_in(first) + sum over chunks of the slowest stage +
// copy_out(last): per chunk of n tokens the copies take n d es / 50 GB/s each
// way, and the forward its dense GEMMs' FLOPs at 0.8 PFLOP/s plus the routed
// experts' max(FLOPs at 0.8 PFLOP/s, weights of the experts the chunk selects
// at 6 TB/s) plus 60 us of launch latency and tile tails (a 1024-token chunk of
// the 0.5b layer takes ~90 us against 122 us for 4096 tokens: small chunks
// leave most SMs idle).  A chunked plan must beat one chunk by 15 %, and of
// the counts within 3 % of the best estimate the smallest is taken (measured:
// 0.5b shape 2 chunks 12.0 M tokens/s against 10.8 M for one and 9.7 M for
// four; mid shape 4 chunks 6.5 M, 7 chunks 6.2 M, one 4.0 M).
static int host_chunks(const lmoe_dims* d) {
  // LMOE_HOST_CHUNKS=c (1..8) overrides the model
  if (const char* v = getenv("LMOE_HOST_CHUNKS")) {
    const int c = atoi(v);
    if (c >= 1 && c <= kMaxHostChunks) return c;
  }
  const double N = (double)d->n_tokens, es = d->dtype == LMOE_BF16 ? 2.0 : 4.0;
  const double D = d->d, L = d->latent, R = d->n_routed, k = d->top_k, F = d->ff_routed;
  const double SG = (double)d->n_shared * (d->n_shared > 0 ? d->ff_shared : 0);
  const double dense_tok = 2 * D * L + 2 * D * R + 6 * SG * D + 2 * L * D;
  const double routed_tok = 6 * k * L * F;
  const double w_expert = 3 * F * L * es;
  const double copy_bw = 50e9, flop_rate = d->dtype == LMOE_BF16 ? 0.8e15 : 2.0e13,
               hbm = 6.0e12, fixed = 60e-6;
  double est[kMaxHostChunks + 1] = {0.0};
  int n_c = 0;
  double best = 0.0;
  for (int c = 1; c <= kMaxHostChunks; ++c) {
    const double n = std::ceil(N / c);
    if (c > 1 && n < 256) break;
    const double used = R * (1.0 - std::pow(1.0 - k / R, n));  // experts a chunk selects
    const double t_copy = n * D * es / copy_bw;
    const double t_fwd = n * dense_tok / flop_rate +
                         std::max(n * routed_tok / flop_rate, used * w_expert / hbm) + fixed;
    est[c] = 2 * t_copy + c * std::max(t_copy, t_fwd);
    n_c = c;
    if (c == 1 || (est[c] < best && est[c] < 0.85 * est[1])) best = est[c];
  }
  for (int c = 1; c <= n_c; ++c)
    if (est[c] <= 1.03 * best && (c == 1 || est[c] < 0.85 * est[1])) return c;
  return 1;
}

}  // namespace lmoe

using namespace lmoe;

extern "C" {

size_t lmoe_workspace_size(const lmoe_dims* dims) {
  if (check_dims(dims) != LMOE_OK) return 0;
  return layout(dims, false).total;
}

size_t lmoe_workspace_size_host(const lmoe_dims* dims) {
  if (check_dims(dims) != LMOE_OK) return 0;
  return layout(dims, true).total;
}

lmoe_status moe_route(const lmoe_dims* dims, const void* x, const void* w_router,
                      const float* expert_bias, int32_t* ids, float* probs, void* ws,
                      size_t ws_bytes, lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  if (dims->n_tokens > 0) {
    LMOE_PTR(x, "x");
    LMOE_PTR(ids, "ids");
    LMOE_PTR(probs, "probs");
  }
  LMOE_PTR(w_router, "w_router");
  if (expert_bias != nullptr && !aligned16(expert_bias))
    return fail(LMOE_EINVAL, "expert_bias is not 16-byte aligned");
  LMOE_TRY(check_ws(dims, ws, ws_bytes, false));
  LMOE_TRY(check_device());
  ProfJoin pj((cudaStream_t)stream);  // joins the profiling branch on return
  cudaStream_t st = (cudaStream_t)stream;
  if (dims->dtype == LMOE_BF16)
    return run_route<__nv_bfloat16>(dims, x, w_router, expert_bias, ids, probs, ws, st);
  return run_route<float>(dims, x, w_router, expert_bias, ids, probs, ws, st);
}

lmoe_status moe_dispatch(const lmoe_dims* dims, const int32_t* ids, int32_t* counts,
                         int32_t* offsets, int32_t* perm_token, int32_t* inv_pair, void* ws,
                         size_t ws_bytes, lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  if (dims->n_tokens > 0) {
    LMOE_PTR(ids, "ids");
    LMOE_PTR(perm_token, "perm_token");
    LMOE_PTR(inv_pair, "inv_pair");
  }
  LMOE_PTR(counts, "counts");
  LMOE_PTR(offsets, "offsets");
  LMOE_TRY(check_ws(dims, ws, ws_bytes, false));
  LMOE_TRY(check_device());
  ProfJoin pj((cudaStream_t)stream);  // joins the profiling branch on return
  return run_dispatch(dims, ids, counts, offsets, perm_token, inv_pair, ws, (cudaStream_t)stream);
}

lmoe_status moe_expert_ffn(const lmoe_dims* dims, const void* z, const int32_t* perm_token,
                           const int32_t* offsets, const void* w_g, const void* w_u,
                           const void* w_o, void* expert_out, void* ws, size_t ws_bytes,
                           lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  if (dims->n_tokens > 0) {
    LMOE_PTR(z, "z");
    LMOE_PTR(perm_token, "perm_token");
    LMOE_PTR(expert_out, "expert_out");
  }
  LMOE_PTR(offsets, "offsets");
  LMOE_PTR(w_g, "w_g");
  LMOE_PTR(w_u, "w_u");
  LMOE_PTR(w_o, "w_o");
  LMOE_TRY(check_ws(dims, ws, ws_bytes, false));
  LMOE_TRY(check_device());
  ProfJoin pj((cudaStream_t)stream);  // joins the profiling branch on return
  cudaStream_t st = (cudaStream_t)stream;
  const Layout L = layout(dims, false);
  LMOE_CUDA(launch_build_tiles(offsets, dims->n_routed, &at<WsHeader>(ws, L.header)->n_mtiles,
                               at<int4>(ws, L.tiles), st, routed_tile_m(dims)),
            "build_tiles");
  if (dims->dtype == LMOE_BF16)
    return run_expert_ffn<__nv_bfloat16>(dims, z, perm_token, offsets, w_g, w_u, w_o, expert_out,
                                         ws, st);
  return run_expert_ffn<float>(dims, z, perm_token, offsets, w_g, w_u, w_o, expert_out, ws, st);
}

lmoe_status lmoe_check_dispatch(const lmoe_dims* dims, const int32_t* ids, const int32_t* counts,
                                const int32_t* offsets, const int32_t* perm_token,
                                const int32_t* inv_pair, void* ws, size_t ws_bytes,
                                lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  LMOE_PTR(counts, "counts");
  LMOE_PTR(offsets, "offsets");
  if (dims->n_tokens > 0) {
    LMOE_PTR(ids, "ids");
    LMOE_PTR(perm_token, "perm_token");
    LMOE_PTR(inv_pair, "inv_pair");
  }
  LMOE_TRY(check_ws(dims, ws, ws_bytes, false));
  LMOE_TRY(check_device());
  const Layout L = layout(dims, false);
  // the bitmap lives in the sorted-row area of the workspace (N*k*l elements >= N*k/32 words)
  uint32_t* bitmap = at<uint32_t>(ws, L.eo);
  LMOE_CUDA(launch_check_dispatch(ids, dims->n_tokens, dims->top_k, dims->n_routed, counts, offsets,
                                  perm_token, inv_pair, bitmap, &at<WsHeader>(ws, L.header)->status,
                                  (cudaStream_t)stream),
            "check dispatch");
  return LMOE_OK;
}

static BwdDims bwd_dims(const lmoe_dims* d) {
  BwdDims b;
  b.N = d->n_tokens; b.d = d->d; b.L = d->latent; b.R = d->n_routed; b.k = d->top_k;
  b.S = d->n_shared; b.F = d->ff_routed; b.G = d->n_shared > 0 ? d->ff_shared : 0;
  b.beta1 = d->beta1; b.beta2 = d->beta2; b.rms_eps = d->rms_eps; b.router = d->router;
  b.bf16 = d->dtype == LMOE_BF16 ? 1 : 0;
  return b;
}

size_t lmoe_backward_workspace_size(const lmoe_dims* dims) {
  if (check_dims(dims) != LMOE_OK) return 0;
  return bwd_layout(bwd_dims(dims)).total;
}

lmoe_status latent_moe_backward(const lmoe_dims* dims, const lmoe_weights* w, const void* x,
                                const void* dy, const lmoe_grads* g, void* ws, size_t ws_bytes,
                                lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  if (w == nullptr || g == nullptr) return fail(LMOE_EINVAL, "weights or grads is NULL");
  LMOE_PTR(w->w_down, "w_down");
  LMOE_PTR(w->w_router, "w_router");
  LMOE_PTR(w->w_up, "w_up");
  LMOE_PTR(w->rms_weight, "rms_weight");
  LMOE_PTR(w->w_g, "w_g");
  LMOE_PTR(w->w_u, "w_u");
  LMOE_PTR(w->w_o, "w_o");
  LMOE_PTR(g->dw_down, "dw_down");
  LMOE_PTR(g->dw_router, "dw_router");
  LMOE_PTR(g->dw_up, "dw_up");
  LMOE_PTR(g->drms_weight, "drms_weight");
  LMOE_PTR(g->dw_g, "dw_g");
  LMOE_PTR(g->dw_u, "dw_u");
  LMOE_PTR(g->dw_o, "dw_o");
  if (dims->n_shared > 0) {
    LMOE_PTR(w->ws_g, "ws_g");
    LMOE_PTR(w->ws_u, "ws_u");
    LMOE_PTR(w->ws_o, "ws_o");
    LMOE_PTR(g->dws_g, "dws_g");
    LMOE_PTR(g->dws_u, "dws_u");
    LMOE_PTR(g->dws_o, "dws_o");
  }
  if (dims->n_tokens > 0) {
    LMOE_PTR(x, "x");
    LMOE_PTR(dy, "dy");
    LMOE_PTR(g->dx, "dx");
  }
  LMOE_PTR(ws, "ws");
  if (((uintptr_t)ws & 255u) != 0) return fail(LMOE_EINVAL, "ws must be 256-byte aligned");
  const BwdDims bd = bwd_dims(dims);
  const size_t need = bwd_layout(bd).total;
  if (ws_bytes < need)
    return fail(LMOE_EWORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
  LMOE_TRY(check_device());
  ProfJoin pj((cudaStream_t)stream);  // joins the profiling branch on return
  cudaStream_t st = (cudaStream_t)stream;
  LMOE_CUDA(cudaMemsetAsync(ws, 0, 256, st), "clear the header");
  if (dims->n_tokens == 0) {  // no tokens: every gradient is 0
    const size_t L = dims->latent, d = dims->d, R = dims->n_routed, F = dims->ff_routed;
    LMOE_CUDA(cudaMemsetAsync(g->dw_down, 0, L * d * 4, st), "memset");
    LMOE_CUDA(cudaMemsetAsync(g->dw_router, 0, R * d * 4, st), "memset");
    LMOE_CUDA(cudaMemsetAsync(g->dw_up, 0, d * L * 4, st), "memset");
    LMOE_CUDA(cudaMemsetAsync(g->drms_weight, 0, L * 4, st), "memset");
    LMOE_CUDA(cudaMemsetAsync(g->dw_g, 0, R * F * L * 4, st), "memset");
    LMOE_CUDA(cudaMemsetAsync(g->dw_u, 0, R * F * L * 4, st), "memset");
    LMOE_CUDA(cudaMemsetAsync(g->dw_o, 0, R * L * F * 4, st), "memset");
    if (dims->n_shared > 0) {
      const size_t SG = (size_t)dims->n_shared * dims->ff_shared;
      LMOE_CUDA(cudaMemsetAsync(g->dws_g, 0, SG * d * 4, st), "memset");
      LMOE_CUDA(cudaMemsetAsync(g->dws_u, 0, SG * d * 4, st), "memset");
      LMOE_CUDA(cudaMemsetAsync(g->dws_o, 0, SG * d * 4, st), "memset");
    }
    return LMOE_OK;
  }
  BwdArgs a;
  a.x = x; a.dy = dy; a.w_down = w->w_down; a.w_router = w->w_router; a.w_up = w->w_up;
  a.w_g = w->w_g; a.w_u = w->w_u; a.w_o = w->w_o; a.ws_g = w->ws_g; a.ws_u = w->ws_u;
  a.ws_o = w->ws_o; a.rms_weight = w->rms_weight; a.bias = w->expert_bias;
  a.g.dx = g->dx; a.g.dw_down = g->dw_down; a.g.dw_router = g->dw_router; a.g.dw_up = g->dw_up;
  a.g.drms = g->drms_weight; a.g.dw_g = g->dw_g; a.g.dw_u = g->dw_u; a.g.dw_o = g->dw_o;
  a.g.dws_g = g->dws_g; a.g.dws_u = g->dws_u; a.g.dws_o = g->dws_o;
  ProfScope ps("backward", st);
  LMOE_CUDA(run_backward(bd, a, ws, st), "backward");
  return LMOE_OK;
}

lmoe_status moe_router_losses(const lmoe_dims* dims, const float* logits, int64_t ld,
                              const int32_t* ids, float* out, void* ws, size_t ws_bytes,
                              lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  LMOE_PTR(out, "out");
  if (dims->n_tokens > 0) LMOE_PTR(ids, "ids");
  LMOE_TRY(check_ws(dims, ws, ws_bytes, false));
  const Layout L = layout(dims, false);
  if (logits == nullptr) {
    logits = at<float>(ws, L.logits);
    ld = L.logits_ld;
  } else if (ld < dims->n_routed || (uintptr_t)logits % 4 != 0) {
    return fail(LMOE_EINVAL, "logits: ld < n_routed or misaligned");
  }
  LMOE_TRY(check_device());
  ProfJoin pj((cudaStream_t)stream);  // joins the profiling branch on return
  const int64_t nb = loss_blocks(dims->n_tokens);
  float* part_s = at<float>(ws, L.loss);
  int32_t* part_c = reinterpret_cast<int32_t*>(part_s + nb * dims->n_routed);
  float* part_z = reinterpret_cast<float*>(part_c + nb * dims->n_routed);
  ProfScope ps("router_losses", (cudaStream_t)stream);
  LMOE_CUDA(launch_router_losses(logits, ld, ids, dims->n_tokens, dims->top_k, dims->n_routed,
                                 part_s, part_c, part_z, &at<WsHeader>(ws, L.header)->status, out,
                                 (cudaStream_t)stream),
            "router losses");
  return LMOE_OK;
}

lmoe_status moe_combine(const lmoe_dims* dims, const void* expert_out, const int32_t* inv_pair,
                        const float* probs, const float* rms_weight, void* u_normed,
                        lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  if (dims->n_tokens > 0) {
    LMOE_PTR(expert_out, "expert_out");
    LMOE_PTR(inv_pair, "inv_pair");
    LMOE_PTR(probs, "probs");
    LMOE_PTR(u_normed, "u_normed");
  }
  LMOE_PTR(rms_weight, "rms_weight");
  LMOE_TRY(check_device());
  cudaStream_t st = (cudaStream_t)stream;
  if (dims->dtype == LMOE_BF16) {
    LMOE_CUDA(launch_combine<__nv_bfloat16>((const __nv_bfloat16*)expert_out, inv_pair, probs,
                                            rms_weight, dims->n_tokens, dims->top_k, dims->latent,
                                            dims->rms_eps, (__nv_bfloat16*)u_normed, st),
              "combine");
  } else {
    LMOE_CUDA(launch_combine<float>((const float*)expert_out, inv_pair, probs, rms_weight,
                                    dims->n_tokens, dims->top_k, dims->latent, dims->rms_eps,
                                    (float*)u_normed, st),
              "combine");
  }
  return LMOE_OK;
}

lmoe_status latent_moe_forward(const lmoe_dims* dims, const lmoe_weights* weights, const void* x,
                               void* y, int32_t* ids_out, float* probs_out, int32_t* counts_out,
                               void* ws, size_t ws_bytes, lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  LMOE_TRY(check_weights(dims, weights));
  if (dims->n_tokens > 0) {
    LMOE_PTR(x, "x");
    LMOE_PTR(y, "y");
  }
  if (ids_out && !aligned16(ids_out)) return fail(LMOE_EINVAL, "ids_out is not 16-byte aligned");
  if (probs_out && !aligned16(probs_out)) return fail(LMOE_EINVAL, "probs_out is not 16-byte aligned");
  if (counts_out && !aligned16(counts_out)) return fail(LMOE_EINVAL, "counts_out is not 16-byte aligned");
  LMOE_TRY(check_ws(dims, ws, ws_bytes, false));
  LMOE_TRY(check_device());
  ProfJoin pj((cudaStream_t)stream);  // joins the profiling branch on return
  cudaStream_t st = (cudaStream_t)stream;
  if (dims->dtype == LMOE_BF16)
    return run_forward_tc(dims, weights, x, y, ids_out, probs_out, counts_out, ws, st);
  return run_forward<float>(dims, weights, x, y, ids_out, probs_out, counts_out, ws, st);
}

lmoe_status latent_moe_forward_host(const lmoe_dims* dims, const lmoe_weights* weights,
                                    const void* x_host, void* y_host, void* ws, size_t ws_bytes,
                                    lmoe_stream stream) {
  LMOE_TRY(check_dims(dims));
  LMOE_TRY(check_weights(dims, weights));
  if (dims->n_tokens > 0 && (x_host == nullptr || y_host == nullptr))
    return fail(LMOE_EINVAL, "x_host / y_host is NULL");
  LMOE_TRY(check_ws(dims, ws, ws_bytes, true));
  LMOE_TRY(check_device());
  ProfJoin pj((cudaStream_t)stream);  // joins the profiling branch on return
  cudaStream_t st = (cudaStream_t)stream;
  const Layout L = layout(dims, true);
  const int64_t N = dims->n_tokens;
  const size_t row = (size_t)dims->d * (dims->dtype == LMOE_BF16 ? 2 : 4);
  char* xd = at<char>(ws, L.x);
  char* yd = at<char>(ws, L.y);
  if (N == 0) {
    LMOE_TRY(dims->dtype == LMOE_BF16
                 ? run_forward_tc(dims, weights, xd, yd, nullptr, nullptr, nullptr, ws, st)
                 : run_forward<float>(dims, weights, xd, yd, nullptr, nullptr, nullptr, ws, st));
    LMOE_CUDA(cudaStreamSynchronize(st), "sync");
    return LMOE_OK;
  }
  HostPipe* hp = nullptr;
  LMOE_TRY(host_pipe(&hp));
  const int C = host_chunks(dims);
  const int64_t per = (N + C - 1) / C;
  // copies wait for whatever the caller queued on its stream before this call
  LMOE_CUDA(cudaEventRecord(hp->start, st), "event");
  LMOE_CUDA(cudaStreamWaitEvent(hp->in, hp->start, 0), "wait");
  LMOE_CUDA(cudaStreamWaitEvent(hp->out, hp->start, 0), "wait");
  for (int c = 0; c < C; ++c) {  // every chunk's x in flight first (the copy engine streams them)
    const int64_t t0 = c * per, n = std::min<int64_t>(per, N - t0);
    if (n <= 0) break;
    LMOE_CUDA(cudaMemcpyAsync(xd + t0 * row, static_cast<const char*>(x_host) + t0 * row, n * row,
                              cudaMemcpyHostToDevice, hp->in),
              "H2D x");
    LMOE_CUDA(cudaEventRecord(hp->in_done[c], hp->in), "event");
  }
  for (int c = 0; c < C; ++c) {  // chunk c's forward on the caller's stream, its y copied back
    const int64_t t0 = c * per, n = std::min<int64_t>(per, N - t0);
    if (n <= 0) break;
    lmoe_dims dc = *dims;
    dc.n_tokens = n;
    LMOE_CUDA(cudaStreamWaitEvent(st, hp->in_done[c], 0), "wait");
    lmoe_status s = dims->dtype == LMOE_BF16
                        ? run_forward_tc(&dc, weights, xd + t0 * row, yd + t0 * row, nullptr,
                                         nullptr, nullptr, ws, st)
                        : run_forward<float>(&dc, weights, xd + t0 * row, yd + t0 * row, nullptr,
                                             nullptr, nullptr, ws, st);
    if (s != LMOE_OK) return s;
    LMOE_CUDA(cudaEventRecord(hp->fwd_done[c], st), "event");
    LMOE_CUDA(cudaStreamWaitEvent(hp->out, hp->fwd_done[c], 0), "wait");
    LMOE_CUDA(cudaMemcpyAsync(static_cast<char*>(y_host) + t0 * row, yd + t0 * row, n * row,
                              cudaMemcpyDeviceToHost, hp->out),
              "D2H y");
  }
  LMOE_CUDA(cudaEventRecord(hp->done, hp->out), "event");
  LMOE_CUDA(cudaStreamWaitEvent(st, hp->done, 0), "wait");
  LMOE_CUDA(cudaStreamSynchronize(st), "sync");
  return LMOE_OK;
}

lmoe_status lmoe_forward_plan(const lmoe_dims* dims, int32_t* flags) {
  LMOE_TRY(check_dims(dims));
  if (flags == nullptr) return fail(LMOE_EINVAL, "flags is NULL");
  const lmoe_dims* d = dims;
  const bool bf16 = d->dtype == LMOE_BF16;
  const bool fuse_rows = rows_in_scatter(d);
  int32_t f = 0;
  if (bf16 && combine_fused(d)) f |= LMOE_PLAN_COMBINE_FUSED;
  if (bf16 && xpass_wide(d)) f |= LMOE_PLAN_XPASS_WIDE;
  if (routed_pairs(d, 1)) f |= LMOE_PLAN_GEMM1_PAIRS;
  if (routed_pairs(d, 2)) f |= LMOE_PLAN_GEMM2_PAIRS;
  if (routed_pairs(d, 1) && d->latent >= 2048) f |= LMOE_PLAN_GEMM1_WIDE;
  if (fuse_rows) f |= LMOE_PLAN_ROWS_IN_SCATTER;
  if (counts_in_xpass(d)) f |= LMOE_PLAN_COUNTS_IN_XPASS;
  *flags = f;
  return LMOE_OK;
}

lmoe_status lmoe_workspace_layout(const lmoe_dims* dims, size_t* offsets, int32_t n) {
  LMOE_TRY(check_dims(dims));
  if (offsets == nullptr || n < 8) return fail(LMOE_EINVAL, "offsets needs 8 entries");
  const Layout L = layout(dims, false);
  const size_t v[11] = {L.z,  L.logits, L.hsh, L.uhat,    L.eo,  L.h,
                        L.zp, (size_t)L.logits_ld, L.offsets, L.perm, L.inv};
  for (int i = 0; i < (n >= 11 ? 11 : 8); ++i) offsets[i] = v[i];
  return LMOE_OK;
}

lmoe_status lmoe_workspace_init(void* ws, size_t ws_bytes, lmoe_stream stream) {
  LMOE_PTR(ws, "ws");
  if (ws_bytes < sizeof(WsHeader)) return fail(LMOE_EWORKSPACE, "workspace smaller than its header");
  // the header and the synchronisation area after it
  const size_t n = std::min(ws_bytes, align256(sizeof(WsHeader)) + (size_t)kSyncWords * 4);
  LMOE_CUDA(cudaMemsetAsync(ws, 0, n, (cudaStream_t)stream), "memset header");
  return LMOE_OK;
}

lmoe_status lmoe_get_device_status(void* ws, lmoe_stream stream) {
  LMOE_PTR(ws, "ws");
  cudaStream_t st = (cudaStream_t)stream;
  int32_t v = 0;
  LMOE_CUDA(cudaMemcpyAsync(&v, &static_cast<WsHeader*>(ws)->status, sizeof(v),
                            cudaMemcpyDeviceToHost, st),
            "read status");
  LMOE_CUDA(cudaStreamSynchronize(st), "sync");
  if (v != 0) {
    LMOE_CUDA(cudaMemsetAsync(&static_cast<WsHeader*>(ws)->status, 0, sizeof(int32_t), st),
              "clear status");
    LMOE_CUDA(cudaStreamSynchronize(st), "sync");
    return v == LMOE_ETIMEOUT ? LMOE_ETIMEOUT : LMOE_EDEVICE;
  }
  return LMOE_OK;
}

lmoe_status lmoe_selftest_capped_wait(void* ws, size_t ws_bytes, int32_t cap_ms,
                                      lmoe_stream stream) {
  LMOE_PTR(ws, "ws");
  if (ws_bytes < sizeof(WsHeader)) return fail(LMOE_EWORKSPACE, "workspace smaller than its header");
  if (cap_ms < 1 || cap_ms > 10000) return fail(LMOE_EINVAL, "cap_ms out of [1, 10000]");
  LMOE_TRY(check_device());
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader* h = static_cast<WsHeader*>(ws);
  // the flag nothing sets: a zeroed word of the header padding
  LMOE_CUDA(cudaMemsetAsync(&h->pad[0], 0, sizeof(int32_t), st), "memset flag");
  LMOE_CUDA(launch_capped_wait(&h->pad[0], &h->status, cap_ms, st), "capped wait");
  return LMOE_OK;
}

const char* lmoe_status_string(lmoe_status s) {
  switch (s) {
    case LMOE_OK: return "LMOE_OK";
    case LMOE_EINVAL: return "LMOE_EINVAL";
    case LMOE_EUNSUPPORTED: return "LMOE_EUNSUPPORTED";
    case LMOE_EWORKSPACE: return "LMOE_EWORKSPACE";
    case LMOE_ECUDA: return "LMOE_ECUDA";
    case LMOE_EDEVICE: return "LMOE_EDEVICE";
    case LMOE_ETIMEOUT: return "LMOE_ETIMEOUT";
  }
  return "LMOE_UNKNOWN";
}

const char* lmoe_last_error(void) { return g_last_error.c_str(); }

lmoe_status lmoe_profile_enable(const char* tags) {
  if (tags == nullptr || tags[0] == 0) {
    g_prof_tags.clear();
  } else if (std::string(tags) == "*") {
    g_prof_tags = "*";
  } else {
    g_prof_tags = "," + std::string(tags) + ",";
  }
  return LMOE_OK;
}

lmoe_status lmoe_profile_read_tag(const char* tag, double* total_ms, int64_t* launches) {
  double tot = 0.0;
  int64_t n = 0;
  std::vector<ProfRec> keep;
  for (auto& r : g_prof) {
    if (tag != nullptr && r.tag != tag) {
      keep.push_back(r);
      continue;
    }
    float ms = 0.0f;
    LMOE_CUDA(cudaEventSynchronize(r.b), "event sync");
    LMOE_CUDA(cudaEventElapsedTime(&ms, r.a, r.b), "elapsed");
    tot += ms;
    ++n;
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  g_prof.swap(keep);
  if (total_ms) *total_ms = tot;
  if (launches) *launches = n;
  return LMOE_OK;
}

lmoe_status lmoe_profile_peek_tag(const char* tag, double* total_ms, int64_t* launches) {
  double tot = 0.0;
  int64_t n = 0;
  for (auto& r : g_prof) {
    if (tag != nullptr && r.tag != tag) continue;
    float ms = 0.0f;
    LMOE_CUDA(cudaEventSynchronize(r.b), "event sync");
    LMOE_CUDA(cudaEventElapsedTime(&ms, r.a, r.b), "elapsed");
    tot += ms;
    ++n;
  }
  if (total_ms) *total_ms = tot;
  if (launches) *launches = n;
  return LMOE_OK;
}

lmoe_status lmoe_profile_read(double* total_ms, int64_t* launches) {
  return lmoe_profile_read_tag(nullptr, total_ms, launches);
}

uint64_t lmoe_launch_count(int32_t reset) {
  uint64_t v = g_launches;
  if (reset) g_launches = 0;
  return v;
}

}  // extern "C"
