// Sort-by-expert without any device allocation: the same two kernels as
// moe_sort (per-tile expert histogram, then the multi-CTA stable scatter),
// with their scratch (the histograms, the grouped GEMM's m-tile table, its
// length and the status word) in a fixed-size array in the library's own
// device memory instead of a handle's workspace.
//
// It serves callers that cannot allocate device memory when they sort:
// a serving runtime that has reserved its HBM budget up front (weights, KV
// cache, activation pools) and refuses further allocations during a step;
// a scheduler thread that must not stall the device, since cudaFree
// synchronises the whole device and cudaMalloc may; and code that receives
// routing from elsewhere and holds no moe_handle (whose workspace moe_create
// allocates).  Nothing here calls cudaMalloc, cudaFree or a library routine
// that allocates.
//
// The scratch is one array per device, so calls that overlap in time on the
// same device (other streams, other host threads) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace {

constexpr int kMaxT = MOE_SORT_STATIC_MAX_TOKENS;
constexpr int kTokenTiles = (kMaxT + moe::kBM - 1) / moe::kBM;
// Scratch layout (byte offsets, each 256-byte aligned):
//   hist     [kTokenTiles, MOE_MAX_EXPERTS] int32
//   tiles    [kMaxT * MOE_MAX_TOP_K / 128 + MOE_MAX_EXPERTS + 1] int2
//   n_mtiles [1] int32
//   status   [1] int32
constexpr size_t align256(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t kHistOff = 0;
constexpr size_t kHistBytes = size_t(kTokenTiles) * MOE_MAX_EXPERTS * 4;
constexpr size_t kTilesOff = align256(kHistOff + kHistBytes);
constexpr size_t kTilesBytes =
    (size_t(kMaxT) * MOE_MAX_TOP_K / moe::kBM + MOE_MAX_EXPERTS + 1) * sizeof(int2);
constexpr size_t kNTilesOff = align256(kTilesOff + kTilesBytes);
constexpr size_t kStatusOff = kNTilesOff + 256;
constexpr size_t kScratchBytes = kStatusOff + 256;  // about 75 KB

static __device__ __align__(256) unsigned char g_sort_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char* g_scratch[kMaxDevices];  // device address of g_sort_scratch, per device

// Device address of the scratch array on the current device.  The first call
// on a device resolves the symbol (this also loads the module there if it is
// not yet loaded); later calls only read the cached pointer.
moe_status scratch_on_current_device(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        major != 10)
      return MOE_ERR_DEVICE;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sort_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_scratch[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_sort_static(const int32_t* idx, int32_t num_tokens, int32_t top_k,
                                      int32_t num_experts, int32_t* perm, int32_t* inv,
                                      int32_t* off, int32_t* status, void* stream) {
  if (!idx || !perm || !inv || !off) return MOE_ERR_NULL_POINTER;
  if (top_k < 1 || top_k > MOE_MAX_TOP_K || num_experts < 1 || num_experts > MOE_MAX_EXPERTS ||
      top_k > num_experts)
    return MOE_ERR_INVALID_CONFIG;
  if (num_tokens < 1 || num_tokens > MOE_SORT_STATIC_MAX_TOKENS)
    return MOE_ERR_TOKENS_OUT_OF_RANGE;
  unsigned char* s = nullptr;
  const moe_status st = scratch_on_current_device(&s);
  if (st != MOE_OK) return st;
  int* hist = reinterpret_cast<int*>(s + kHistOff);
  int2* tiles = reinterpret_cast<int2*>(s + kTilesOff);
  int* n_mtiles = reinterpret_cast<int*>(s + kNTilesOff);
  int* dstatus = status ? status : reinterpret_cast<int*>(s + kStatusOff);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // The status word is OR-ed into, so it starts at zero; the histogram and
  // the tile table are overwritten in full by the kernels.
  if (cudaMemsetAsync(dstatus, 0, sizeof(int32_t), cs) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::launch_tile_hist(idx, num_tokens, top_k, num_experts, hist, dstatus, cs) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::launch_sort(idx, hist, num_tokens, top_k, num_experts, perm, inv, off, tiles, n_mtiles,
                       dstatus, cs) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
