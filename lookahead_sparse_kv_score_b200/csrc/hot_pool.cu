// Hot-pool residency across triggers: only rows of the fetch set that are not yet in
// GPU memory cross the host link.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.1, and the review page
// (paper.oopus.info), part 二: every tau decode steps the indexer predicts which
// compressed KV blocks will be needed and only those are kept in GPU memory, fetched
// from the CPU cold pool.  What happens to a row fetched by an earlier trigger is not
// stated; here it stays in its slot until the slot is needed: a trigger keeps the
// resident rows of its fetch set U (their stamp becomes the trigger index t), and each
// missing row of U takes a free or the least recently needed slot, slots ordered by
// (stamp, slot index), the i-th missing entry (ascending) pairing with the i-th taken
// slot (ascending).  An update whose |U| exceeds the pool moves nothing.
//
// One update, per batch of sequences:
//   1. need = U & ~resident                         (hot_need_kernel)
//   2. need list = ascending set bits of need       (the fetch-list compaction)
//   3. slot keys: kept slot -> stamp t, key 0;      (hot_slot_keys_kernel)
//      other slot -> key ~stamp (older is larger, a free slot has stamp 0)
//   4. the |need| largest keys, ties to the lower slot, in ascending slot order
//                                                   (the cluster radix select, direct keys)
//   5. move row need[i] into slot taken[i] and update the maps and the resident bits
//                                                   (hot_assign_kernel)
#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 256;
constexpr int kInFlight = 8;
constexpr int kChunk = kThreads * kInFlight * 4;   // 16-byte pieces per block (128 KB)
constexpr int kSeqPerLaunch = 4096;   // sequences whose move prefix one assign launch holds in shared memory

__global__ void hot_need_kernel(int B, int N, const uint32_t* __restrict__ U, const uint32_t* __restrict__ R,
                                uint32_t* __restrict__ need) {
  const int Nw = (N + 31) / 32;
  const size_t total = static_cast<size_t>(B) * Nw;
  const uint32_t tail = (N & 31) ? ((1u << (N & 31)) - 1u) : 0xffffffffu;   // bits of the last word below N
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int w = static_cast<int>(i % Nw);
    need[i] = U[i] & ~R[i] & (w == Nw - 1 ? tail : 0xffffffffu);
  }
}

__global__ void hot_slot_keys_kernel(int N, int slots, const uint32_t* __restrict__ U, uint32_t t,
                                     const int32_t* __restrict__ entry_of, uint32_t* __restrict__ stamp,
                                     uint32_t* __restrict__ key, int32_t* __restrict__ kept_count) {
  const int b = blockIdx.y;
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  const int Nw = (N + 31) / 32;
  int kept = 0;
  if (s < slots) {
    const size_t i = static_cast<size_t>(b) * slots + s;
    const int e = entry_of[i];
    const bool in = e >= 0 && e < N && ((U[static_cast<size_t>(b) * Nw + (e >> 5)] >> (e & 31)) & 1u);
    if (in) {
      stamp[i] = t;
      key[i] = 0u;
      kept = 1;
    } else {
      key[i] = ~stamp[i];
    }
  }
  kept = __syncthreads_count(kept);
  if (threadIdx.x == 0 && kept) atomicAdd(&kept_count[b], kept);
}

// Moves of all sequences form one flat range of (row, 16-byte piece); each block moves
// one chunk and exits (as in the fetch-list gather).  The first piece of a row also
// updates the maps: the evicted entry (if any) leaves, the new one enters.
__global__ void __launch_bounds__(kThreads)
hot_assign_kernel(int B, int N, int slots, int vpr, uint32_t t, const uint4* __restrict__ cold,
                  const int32_t* __restrict__ need, const int32_t* __restrict__ taken,
                  const int32_t* __restrict__ moved, uint4* __restrict__ hot, int32_t* __restrict__ slot_of,
                  int32_t* __restrict__ entry_of, uint32_t* __restrict__ stamp, uint32_t* __restrict__ R,
                  int32_t* status) {
  extern __shared__ long long pre[];   // [B + 1]: rows moved by the sequences before b
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    long long run = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      long long v = b < B ? max(0, min(moved[b], slots)) : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
      }
      if (b < B) pre[b + 1] = run + v;
      run += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) pre[0] = 0;
  }
  __syncthreads();
  const int Nw = (N + 31) / 32;
  const size_t total = static_cast<size_t>(pre[B]) * vpr;
  for (size_t c0 = static_cast<size_t>(blockIdx.x) * kChunk; c0 < total;
       c0 += static_cast<size_t>(gridDim.x) * kChunk) {
    const size_t end = c0 + kChunk < total ? c0 + kChunk : total;
    for (size_t i0 = c0 + threadIdx.x; i0 < end; i0 += static_cast<size_t>(kThreads) * kInFlight) {
      uint4 v[kInFlight];
      size_t dst[kInFlight];
      bool ok[kInFlight];
#pragma unroll
      for (int u = 0; u < kInFlight; ++u) {
        const size_t i = i0 + static_cast<size_t>(u) * kThreads;
        ok[u] = false;
        if (i < end) {
          const long long g = static_cast<long long>(i / vpr);
          const int c = static_cast<int>(i - static_cast<size_t>(g) * vpr);
          int lo = 0, hi = B;                                        // pre[lo] <= g < pre[hi]
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= g) lo = mid; else hi = mid;
          }
          const int j = static_cast<int>(g - pre[lo]);
          const int e = need[static_cast<size_t>(lo) * slots + j];
          const int s = taken[static_cast<size_t>(lo) * slots + j];
          if (e >= 0 && e < N && s >= 0 && s < slots) {
            if (c == 0) {
              const size_t si = static_cast<size_t>(lo) * slots + s;
              const int old = entry_of[si];
              uint32_t* Rb = R + static_cast<size_t>(lo) * Nw;
              if (old >= 0 && old < N) {
                slot_of[static_cast<size_t>(lo) * N + old] = -1;
                atomicAnd(Rb + (old >> 5), ~(1u << (old & 31)));
              }
              entry_of[si] = e;
              stamp[si] = t;
              slot_of[static_cast<size_t>(lo) * N + e] = s;
              atomicOr(Rb + (e >> 5), 1u << (e & 31));
            }
            v[u] = cold[(static_cast<size_t>(lo) * N + e) * vpr + c];
            dst[u] = (static_cast<size_t>(lo) * slots + s) * vpr + c;
            ok[u] = true;
          } else {
            raise_status(status, LSA_ERR_RANGE);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kInFlight; ++u)
        if (ok[u]) hot[dst[u]] = v[u];
    }
  }
}

}  // namespace

HotLayout hot_layout(int B, int N, int slots) {
  HotLayout o{};
  const size_t Bs = static_cast<size_t>(B), Nw = (static_cast<size_t>(N) + 31) / 32;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off = align_up(off + bytes, 256); return at; };
  o.slot_of = take(Bs * N * 4);
  o.entry_of = take(Bs * slots * 4);
  o.stamp = take(Bs * slots * 4);
  o.resident = take(Bs * Nw * 4);
  o.state_bytes = off;
  off = 0;
  o.need_bits = take(Bs * Nw * 4);
  o.keys = take(Bs * slots * 4);
  o.need = take(Bs * slots * 4);
  o.need_count = take(Bs * 4);
  o.kept_count = take(Bs * 4);
  o.taken = take(Bs * slots * 4);
  o.moved = take(Bs * 4);
  o.select_ws = take(Bs * slots * 4);
  o.ws_bytes = off;
  return o;
}

int launch_hot_update(int B, int N, int slots, size_t row_bytes, uint32_t t, const uint32_t* U,
                      const void* cold_dev, void* hot, void* state, int32_t* moved_out, int32_t* status,
                      void* ws, cudaStream_t s) {
  const HotLayout lay = hot_layout(B, N, slots);
  uint8_t* st = static_cast<uint8_t*>(state);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* slot_of = reinterpret_cast<int32_t*>(st + lay.slot_of);
  int32_t* entry_of = reinterpret_cast<int32_t*>(st + lay.entry_of);
  uint32_t* stamp = reinterpret_cast<uint32_t*>(st + lay.stamp);
  uint32_t* R = reinterpret_cast<uint32_t*>(st + lay.resident);
  uint32_t* need_bits = reinterpret_cast<uint32_t*>(w + lay.need_bits);
  uint32_t* keys = reinterpret_cast<uint32_t*>(w + lay.keys);
  int32_t* need = reinterpret_cast<int32_t*>(w + lay.need);
  int32_t* need_count = reinterpret_cast<int32_t*>(w + lay.need_count);
  int32_t* kept_count = reinterpret_cast<int32_t*>(w + lay.kept_count);
  int32_t* taken = reinterpret_cast<int32_t*>(w + lay.taken);
  int32_t* moved = moved_out ? moved_out : reinterpret_cast<int32_t*>(w + lay.moved);
  uint32_t* select_ws = reinterpret_cast<uint32_t*>(w + lay.select_ws);
  const int Nw = (N + 31) / 32;
  int rc;
  if (cudaMemsetAsync(kept_count, 0, static_cast<size_t>(B) * 4, s) != cudaSuccess)
    return check_launch("hot_pool_update/memset", 0);
  const size_t words = static_cast<size_t>(B) * Nw;
  const unsigned g1 = static_cast<unsigned>(std::max<size_t>(1, std::min<size_t>((words + 255) / 256, 148 * 8)));
  hot_need_kernel<<<g1, 256, 0, s>>>(B, N, U, R, need_bits);
  if ((rc = check_launch("hot_pool_update/need")) != LSA_OK) return rc;
  // missing rows beyond the pool raise LSA_ERR_CAPACITY here or in the slot select
  if ((rc = launch_compact(B, N, need_bits, slots, need, need_count, status, s)) != LSA_OK) return rc;
  int launches = 0;
  for (int b0 = 0; b0 < B; b0 += 65535) {   // the sequence index is gridDim.y
    const int nb = std::min(65535, B - b0);
    const size_t so = static_cast<size_t>(b0) * slots;
    hot_slot_keys_kernel<<<dim3((slots + 255) / 256, nb), 256, 0, s>>>(
        N, slots, U + static_cast<size_t>(b0) * Nw, t, entry_of + so, stamp + so, keys + so, kept_count + b0);
    ++launches;
  }
  if ((rc = check_launch("hot_pool_update/slot_keys", launches)) != LSA_OK) return rc;
  if ((rc = launch_select_keys(B, slots, keys, need_count, kept_count, status, taken, moved, select_ws, s)) != LSA_OK)
    return rc;
  const int vpr = static_cast<int>(row_bytes / 16);
  launches = 0;
  for (int b0 = 0; b0 < B; b0 += kSeqPerLaunch) {
    const int nb = std::min(kSeqPerLaunch, B - b0);
    const size_t so = static_cast<size_t>(b0) * slots, no = static_cast<size_t>(b0) * N;
    const size_t work = static_cast<size_t>(nb) * slots * vpr;   // upper bound on this launch's 16-byte moves
    const unsigned grid =
        static_cast<unsigned>(std::max<size_t>(1, std::min<size_t>((work + kChunk - 1) / kChunk, 1u << 30)));
    hot_assign_kernel<<<grid, kThreads, (nb + 1) * sizeof(long long), s>>>(
        nb, N, slots, vpr, t, static_cast<const uint4*>(cold_dev) + no * vpr, need + so, taken + so, moved + b0,
        static_cast<uint4*>(hot) + so * vpr, slot_of + no, entry_of + so, stamp + so,
        R + static_cast<size_t>(b0) * Nw, status);
    ++launches;
  }
  return check_launch("hot_pool_update/assign", launches);
}

}  // namespace lsa
