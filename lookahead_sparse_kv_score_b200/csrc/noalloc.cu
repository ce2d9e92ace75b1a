// lsa_topk_noalloc: the top-k inside the fetched set with its scratch in a file-scope
// device array instead of a caller-supplied workspace.
//
// For callers that cannot allocate device memory when they call the library: a host
// framework that owns every device allocation and hands plugins no allocator, or a
// latency-critical loop whose memory is fixed once at start-up.  They pass inputs and
// outputs as usual; the candidate keys live in g_topk_scratch below, which every GPU
// that loads the library holds until the process exits.
#include <mutex>

#include "lsa_common.cuh"

namespace lsa {
namespace {

// One 32-bit ordered key per candidate slot: B * cap slots per call at most.
constexpr size_t kTopkScratchSlots = size_t(1) << 23;   // 8,388,608 slots = 32 MiB

__device__ __align__(256) uint32_t g_topk_scratch[kTopkScratchSlots];

// The array's name is a host-side stand-in in host code, not a device address: the
// address is resolved per device with cudaGetSymbolAddress, with that device current.
// It is looked up again on every call made outside stream capture (so a device reset,
// which reloads the module at a new address, is picked up by the next such call); a
// call made while its stream is capturing reuses the address of the last call on that
// device, since the lookup may load the module, which capture does not allow.
constexpr int kMaxDevices = 128;
uint32_t* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

int scratch_address(cudaStream_t stream, uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LSA_ERR_CUDA, "topk_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  }
  if (dev < 0 || dev >= kMaxDevices) return fail(LSA_ERR_UNSUPPORTED, "topk_noalloc: device %d", dev);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cap);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(LSA_ERR_CUDA, "topk_noalloc: cudaStreamIsCapturing: %s", cudaGetErrorString(e));
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap != cudaStreamCaptureStatusNone) {
    if (g_scratch_addr[dev] == nullptr)
      return fail(LSA_ERR_UNSUPPORTED,
                  "topk_noalloc: first call on device %d made during stream capture; call it once outside capture first",
                  dev);
  } else {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return fail(LSA_ERR_CUDA, "topk_noalloc: cudaGetSymbolAddress on device %d: %s", dev,
                  cudaGetErrorString(e));
    }
    g_scratch_addr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_scratch_addr[dev];
  return LSA_OK;
}

}  // namespace
}  // namespace lsa

extern "C" int lsa_topk_noalloc(int B, int L, int N, int k, const int32_t* idx, int cap, const int32_t* count,
                                const float* logit, int32_t* topk, int32_t* topk_count, void* stream) {
  const lsa::CallRange range("lsa_topk_noalloc");
  using namespace lsa;
  clear_error();
  if (B < 0 || L <= 0 || N < 0 || k < 0 || cap < 0)
    return fail(LSA_ERR_INVALID_ARG, "topk_noalloc: bad size (L must be >= 1)");
  if (B == 0) return LSA_OK;
  if (!count || (cap > 0 && !idx) || (k > 0 && !topk) || (N > 0 && !logit))
    return fail(LSA_ERR_INVALID_ARG, "topk_noalloc: null pointer");
  if (static_cast<size_t>(B) * static_cast<size_t>(cap) > kTopkScratchSlots)
    return fail(LSA_ERR_NOMEM, "topk_noalloc: B*cap = %zu exceeds the built-in scratch of %zu slots (32 MiB)",
                static_cast<size_t>(B) * static_cast<size_t>(cap), kTopkScratchSlots);
  uint32_t* scratch = nullptr;
  const int rc = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (rc != LSA_OK) return rc;
  // No clearing needed: each call writes every scratch slot it reads before reading it.
  return launch_topk(B, L, N, k, idx, cap, count, logit, topk, topk_count, scratch,
                     static_cast<cudaStream_t>(stream));
}
