// lmoe_route_noalloc: the routing and segment build of lmoe_route with its
// scratch in a file-scope device array instead of caller-provided memory.
//
// Some callers cannot hand this library device memory: a serving engine that
// reserves all of HBM for its own pool at start-up and has no allocation hook
// to lend, or a host path where cudaMalloc (which may synchronize the device)
// is not allowed.  For them the scratch lives in a static __device__ array of
// fixed size that every GPU loading the library holds until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "kernels.h"
#include "lmoe.h"

namespace {

constexpr int64_t kMaxTokens = LMOE_NOALLOC_MAX_TOKENS;
constexpr int64_t kMaxRouted = LMOE_NOALLOC_MAX_ROUTED;
constexpr int64_t kMaxExperts = 1024;
constexpr int64_t kBlockRows = 256;   // token-block width of the segment list

constexpr size_t a256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// scratch carve-up: per-chunk histograms, per-row weights, token-block list,
// block count, error word
constexpr size_t kChunkBytes = a256(((kMaxTokens + 31) / 32) * kMaxExperts * 4);
constexpr size_t kWrowBytes = a256(kMaxRouted * 4);
constexpr size_t kBlocksBytes = a256((kMaxRouted / kBlockRows + kMaxExperts + 1) * 16);
constexpr size_t kScratchBytes = kChunkBytes + kWrowBytes + kBlocksBytes + 256 + 256;

}  // namespace

// Host code must not use this name as a device address: it is a host-side
// stand-in.  The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

static std::mutex g_scratch_mu;
static void* g_scratch_addr[256];   // per device ordinal, set on first use

// Device address of g_route_scratch on the current device (looked up once per
// device, with that device current).
static int scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LMOE_ERR_CUDA;
  }
  if (dev < 0 || dev >= 256) return LMOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return LMOE_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LMOE_OK;
}

// the error word's byte offset inside the array
constexpr size_t kErrOffset = kChunkBytes + kWrowBytes + kBlocksBytes + 256;

extern "C" int lmoe_route_noalloc(const float* logits, const float* bias, int64_t T, int32_t N,
                                  int32_t K, int32_t* topk_idx, float* topk_w, int32_t* counts,
                                  int32_t* offsets, int32_t* perm, int32_t* inv, void* stream) {
  if (T < 0 || N <= 0 || K <= 0 || K > N) return LMOE_ERR_INVALID_ARG;
  if (N % 32 || N > kMaxExperts || K > 32) return LMOE_ERR_UNSUPPORTED;
  if (T > kMaxTokens || T * K > kMaxRouted) return LMOE_ERR_UNSUPPORTED;
  if (!counts || !offsets || (T > 0 && (!logits || !topk_idx || !topk_w || !perm || !inv)))
    return LMOE_ERR_INVALID_ARG;
  void* base = nullptr;
  int rc = scratch_on_current_device(&base);
  if (rc != LMOE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* s = static_cast<char*>(base);
  int32_t* chunk = reinterpret_cast<int32_t*>(s);
  float* wrow = reinterpret_cast<float*>(s + kChunkBytes);
  int4* blocks = reinterpret_cast<int4*>(s + kChunkBytes + kWrowBytes);
  int32_t* nblocks = reinterpret_cast<int32_t*>(s + kChunkBytes + kWrowBytes + kBlocksBytes);
  int* err = reinterpret_cast<int*>(s + kErrOffset);
  // the array keeps the previous call's contents: the error word starts at 0
  if (cudaMemsetAsync(err, 0, 4, st) != cudaSuccess) return LMOE_ERR_CUDA;
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, N * 4, st) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, (N + 1) * 4, st) != cudaSuccess)
      return LMOE_ERR_CUDA;
    return LMOE_OK;
  }
  // every chunk histogram used below is written in full by the hist kernel
  if (lmoe::launch_route(logits, bias, T, N, K, topk_idx, topk_w, st) != cudaSuccess ||
      lmoe::launch_hist(topk_idx, T, N, K, chunk, err, st) != cudaSuccess ||
      lmoe::launch_scan(chunk, T, N, counts, st) != cudaSuccess ||
      lmoe::launch_scatter(topk_idx, topk_w, chunk, counts, T, N, K, kBlockRows, offsets, perm,
                           inv, wrow, blocks, nblocks, nullptr, err, st) != cudaSuccess)
    return LMOE_ERR_CUDA;
  return LMOE_OK;
}

extern "C" int lmoe_route_noalloc_status(void* stream) {
  void* base = nullptr;
  int rc = scratch_on_current_device(&base);
  if (rc != LMOE_OK) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return LMOE_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpy(&flag, static_cast<char*>(base) + kErrOffset, 4, cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return LMOE_ERR_CUDA;
  return flag ? LMOE_ERR_DEVICE : LMOE_OK;
}
