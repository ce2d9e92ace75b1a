// Cold pool -> hot pool gather of the fetched compressed-KV rows.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.1 "dynamic fetch":
// marked entries are brought from the CPU cold pool into GPU memory; the review page
// (paper.oopus.info, part 二) adds that the copy is asynchronous and overlapped with
// compute.  The cold pool is page-locked host memory mapped into the device address
// space; this kernel reads it directly over the host link (no staging buffer, no
// per-row copy calls) and writes the hot pool in HBM.  Each thread keeps eight
// 16-byte loads in flight so that enough requests cover the link latency.
//
// The link bounds this kernel (about 51 GB/s on B200 with 1152-byte rows, 93% of a
// contiguous pinned copy), but reaching it beside other kernels takes many loads in
// flight.  Each block therefore moves one chunk of kChunk 16-byte pieces and exits: the
// grid covers every row the launch could have, blocks past the actual rows exit at
// once, and a kernel on a higher-priority stream (the selection running beside the
// gather) gets each SM as soon as a chunk retires.  The rows of all sequences form one
// flat range, so sequences with very different fetch counts spread over all blocks.
#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 256;
constexpr int kInFlight = 8;
constexpr int kChunk = kThreads * kInFlight * 4;   // 16-byte pieces per block (128 KB)
constexpr int kSeqPerLaunch = 4096;   // sequences whose row prefix one launch holds in shared memory

__global__ void __launch_bounds__(kThreads)
gather_kernel(int B, int N, int vpr, const uint4* __restrict__ cold, const int32_t* __restrict__ idx,
              const int32_t* __restrict__ count, int cap, uint4* __restrict__ hot, int32_t* status) {
  extern __shared__ long long pre[];   // [B + 1]: pre[b] = rows of sequences before b
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    long long run = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      long long v = b < B ? max(0, min(count[b], cap)) : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      if (b < B) pre[b + 1] = run + v;
      run += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) pre[0] = 0;
  }
  __syncthreads();
  const size_t total = static_cast<size_t>(pre[B]) * vpr;
  for (size_t c0 = static_cast<size_t>(blockIdx.x) * kChunk; c0 < total;
       c0 += static_cast<size_t>(gridDim.x) * kChunk) {
    const size_t end = c0 + kChunk < total ? c0 + kChunk : total;
    for (size_t i0 = c0 + threadIdx.x; i0 < end; i0 += static_cast<size_t>(kThreads) * kInFlight) {
      uint4 v[kInFlight];
      size_t dst[kInFlight];
      bool ok[kInFlight];
#pragma unroll
      for (int t = 0; t < kInFlight; ++t) {
        const size_t i = i0 + static_cast<size_t>(t) * kThreads;
        ok[t] = false;
        if (i < end) {
          const long long g = static_cast<long long>(i / vpr);     // flat row
          const int c = static_cast<int>(i - static_cast<size_t>(g) * vpr);
          int lo = 0, hi = B;                                        // pre[lo] <= g < pre[hi]
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= g) lo = mid; else hi = mid;
          }
          const int j = static_cast<int>(g - pre[lo]);
          const int e = idx[static_cast<size_t>(lo) * cap + j];
          if (e >= 0 && e < N) {
            v[t] = cold[(static_cast<size_t>(lo) * N + e) * vpr + c];
            dst[t] = (static_cast<size_t>(lo) * cap + j) * vpr + c;
            ok[t] = true;
          } else {
            raise_status(status, LSA_ERR_RANGE);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kInFlight; ++t)
        if (ok[t]) hot[dst[t]] = v[t];
    }
  }
}

}  // namespace

int launch_gather(int B, int N, size_t row_bytes, const void* cold_dev, const int32_t* idx,
                  const int32_t* count, int cap, void* hot, int32_t* status, cudaStream_t s) {
  if (B == 0 || cap == 0) return LSA_OK;
  const int vpr = static_cast<int>(row_bytes / 16);
  const size_t seq_cold = static_cast<size_t>(N) * vpr, seq_hot = static_cast<size_t>(cap) * vpr;
  int launches = 0;
  for (int b0 = 0; b0 < B; b0 += kSeqPerLaunch) {
    const int nb = std::min(kSeqPerLaunch, B - b0);
    const size_t work = static_cast<size_t>(nb) * cap * vpr;   // upper bound on this launch's 16-byte moves
    const unsigned grid = (unsigned)std::max<size_t>(1, std::min<size_t>((work + kChunk - 1) / kChunk, 1u << 30));
    gather_kernel<<<grid, kThreads, (nb + 1) * sizeof(long long), s>>>(nb, N, vpr, static_cast<const uint4*>(cold_dev) + b0 * seq_cold,
                                            idx + static_cast<size_t>(b0) * cap, count + b0, cap,
                                            static_cast<uint4*>(hot) + b0 * seq_hot, status);
    ++launches;
  }
  return check_launch("gather_cold", launches);
}

}  // namespace lsa
