// moe_dispatch_noalloc: the pair permutation for callers that cannot hand
// the library a workspace.
//
// Some callers cannot allocate device memory at the point where they need the
// permutation: code running inside a region where allocation is forbidden or
// would break its guarantees (a plugin host that offers no scratch buffer, a
// memory-capped pool that is already full, a latency-critical thread that must
// not enter the driver's allocator), or bindings that only see the tensors
// they were given.  This variant needs only its inputs and outputs.  The
// scratch of the counting sort (per-block histograms, the routed row-tile
// list and a status word) lives in one fixed array in device memory that the
// library defines at file scope; every GPU that loads the library holds it
// until the process exits.
//
// Behaviour that differs from moe_dispatch:
//   - The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current).  Make that first call
//     before any stream capture.
//   - All calls share the one array and it keeps the last call's contents.
//     Two calls whose work overlaps on the GPU (different streams, or
//     different host threads) race on it: serialise them.
//   - Out-of-range ids are dropped, as in moe_dispatch (their inv_pair
//     entries are -1), but they are not reported: the status word is
//     private to this variant.
//   - Sizes whose scratch does not fit the array are rejected with
//     LMOE_EUNSUPPORTED before anything is launched.
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace lmoe {
namespace {

// Capacity of the fixed scratch array, in int32 words (1 MiB).
constexpr int64_t kNoAllocWords = 1 << 18;
constexpr int64_t kHeaderWords = 64;  // [0] status, [1] routed tile count

static __device__ __align__(256) int32_t g_dispatch_scratch[kNoAllocWords];

constexpr int kMaxDevices = 64;
static std::mutex g_mu;
static int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};

// Messages go to the library's per-thread error string (lmoe_last_error).
lmoe_status noalloc_fail(lmoe_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  set_last_error(buf);
  return st;
}

// Words of scratch one call needs: header, per-block histograms, tile list.
int64_t scratch_words(int64_t n_pairs, int R) {
  const int64_t hist = (int64_t)dispatch_blocks(n_pairs) * R;
  const int64_t max_tiles = n_pairs / kTileM + R + 1;
  const int64_t hist_padded = (hist + 3) / 4 * 4;  // keep the tile list 16-byte aligned
  return kHeaderWords + hist_padded + 4 * max_tiles;
}

// Device address of the array on the current device (looked up once per device).
lmoe_status scratch_on_current_device(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(LMOE_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(LMOE_EUNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (!(major == 10 && minor == 0))
      return noalloc_fail(LMOE_EUNSUPPORTED, "device %d is not sm_100 (B200)", dev);
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (e != cudaSuccess || p == nullptr)
      return noalloc_fail(LMOE_ECUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return LMOE_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace
}  // namespace lmoe

using namespace lmoe;

extern "C" {

LMOE_API lmoe_status moe_dispatch_noalloc(const lmoe_dims* dims, const int32_t* ids,
                                          int32_t* counts, int32_t* offsets, int32_t* perm_token,
                                          int32_t* inv_pair, lmoe_stream stream) {
  if (dims == nullptr) return noalloc_fail(LMOE_EINVAL, "dims is NULL");
  const int64_t N = dims->n_tokens;
  const int R = dims->n_routed, k = dims->top_k;
  if (N < 0) return noalloc_fail(LMOE_EINVAL, "n_tokens < 0");
  if (R < 1 || R > 4096) return noalloc_fail(LMOE_EUNSUPPORTED, "n_routed out of [1, 4096]");
  if (k < 1 || k > R) return noalloc_fail(LMOE_EINVAL, "top_k out of [1, n_routed]");
  if (N * (int64_t)k >= ((int64_t)1 << 31) - kTileM * 8)
    return noalloc_fail(LMOE_EUNSUPPORTED, "n_tokens * top_k too large");
  const int64_t need = scratch_words(N * k, R);
  if (need > kNoAllocWords)
    return noalloc_fail(LMOE_EUNSUPPORTED,
                        "n_tokens*top_k = %lld with n_routed = %d needs %lld bytes of scratch; "
                        "the fixed array holds %lld bytes (use moe_dispatch with a workspace)",
                        (long long)(N * k), R, (long long)(need * 4),
                        (long long)(kNoAllocWords * 4));
  const void* must[] = {counts, offsets};
  for (const void* p : must)
    if (p == nullptr || !aligned16(p)) return noalloc_fail(LMOE_EINVAL, "counts/offsets NULL or misaligned");
  if (N > 0 && (ids == nullptr || perm_token == nullptr || inv_pair == nullptr || !aligned16(ids) ||
                !aligned16(perm_token) || !aligned16(inv_pair)))
    return noalloc_fail(LMOE_EINVAL, "ids/perm_token/inv_pair NULL or misaligned");

  int32_t* scratch = nullptr;
  lmoe_status s = scratch_on_current_device(&scratch);
  if (s != LMOE_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  // The status word is the scratch that must start at zero; the histograms
  // and the tile list are fully rewritten by every call.
  cudaError_t e = cudaMemsetAsync(scratch, 0, kHeaderWords * sizeof(int32_t), st);
  if (e != cudaSuccess) return noalloc_fail(LMOE_ECUDA, "clear status: %s", cudaGetErrorString(e));
  const int64_t hist = (int64_t)dispatch_blocks(N * k) * R;
  DispatchScratch ds;
  ds.status = scratch;
  ds.n_mtiles = scratch + 1;
  ds.block_counts = scratch + kHeaderWords;
  ds.tiles = reinterpret_cast<int4*>(scratch + kHeaderWords + (hist + 3) / 4 * 4);
  e = launch_dispatch(ids, N, k, R, counts, offsets, perm_token, inv_pair, ds, st);
  if (e != cudaSuccess) return noalloc_fail(LMOE_ECUDA, "dispatch: %s", cudaGetErrorString(e));
  return LMOE_OK;
}

}  // extern "C"
