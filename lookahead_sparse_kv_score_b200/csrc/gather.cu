// Cold pool -> hot pool gather of the fetched compressed-KV rows.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.1 "dynamic fetch":
// marked entries are brought from the CPU cold pool into GPU memory; the review page
// (paper.oopus.info, part 二) adds that the copy is asynchronous and overlapped with
// compute.  The cold pool is page-locked host memory mapped into the device address
// space; this kernel reads it directly over the host link (no staging buffer, no
// per-row copy calls) and writes the hot pool in HBM.  Each thread keeps eight
// 16-byte loads in flight so that enough requests cover the link latency.
#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 256;
constexpr int kInFlight = 8;

__global__ void __launch_bounds__(kThreads)
gather_kernel(int N, int vpr, const uint4* __restrict__ cold, const int32_t* __restrict__ idx,
              const int32_t* __restrict__ count, int cap, uint4* __restrict__ hot,
              int32_t* status) {
  const int b = blockIdx.y;
  const int n = max(0, min(count[b], cap));
  const size_t total = static_cast<size_t>(n) * vpr;
  const size_t stride = static_cast<size_t>(gridDim.x) * kThreads;
  const int32_t* ib = idx + static_cast<size_t>(b) * cap;
  const uint4* cb = cold + static_cast<size_t>(b) * N * vpr;
  uint4* hb = hot + static_cast<size_t>(b) * cap * vpr;
  for (size_t i0 = blockIdx.x * static_cast<size_t>(kThreads) + threadIdx.x; i0 < total;
       i0 += stride * kInFlight) {
    uint4 v[kInFlight];
    size_t dst[kInFlight];
    bool ok[kInFlight];
#pragma unroll
    for (int t = 0; t < kInFlight; ++t) {
      const size_t i = i0 + t * stride;
      ok[t] = false;
      if (i < total) {
        const int j = static_cast<int>(i / vpr);
        const int c = static_cast<int>(i - static_cast<size_t>(j) * vpr);
        const int e = ib[j];
        if (e >= 0 && e < N) {
          v[t] = cb[static_cast<size_t>(e) * vpr + c];
          dst[t] = i;
          ok[t] = true;
        } else {
          raise_status(status, LSA_ERR_RANGE);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kInFlight; ++t)
      if (ok[t]) hb[dst[t]] = v[t];
  }
}

}  // namespace

int launch_gather(int B, int N, size_t row_bytes, const void* cold_dev, const int32_t* idx,
                  const int32_t* count, int cap, void* hot, int32_t* status, cudaStream_t s) {
  if (B == 0 || cap == 0) return LSA_OK;
  const int vpr = static_cast<int>(row_bytes / 16);
  const size_t work = static_cast<size_t>(cap) * vpr;
  const unsigned gx = (unsigned)std::max<size_t>(
      1, std::min<size_t>((work + kThreads * kInFlight - 1) / (kThreads * kInFlight),
                          std::max(1, 148 * 4 / B)));
  gather_kernel<<<dim3(gx, B), kThreads, 0, s>>>(N, vpr, static_cast<const uint4*>(cold_dev), idx, count,
                                                 cap, static_cast<uint4*>(hot), status);
  return check_launch("gather_cold");
}

}  // namespace lsa
