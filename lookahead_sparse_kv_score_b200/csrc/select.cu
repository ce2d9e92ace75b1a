// Selection after scoring: OR-union of indexer layers, fetch-list compaction and the
// fine top-k inside the fetched subset.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science): §2.4 (three indexer
// layers whose predictions are combined by union, OR mode), §2.1 "dynamic fetch"
// (every entry with I >= 0.5 is fetched) and "hierarchical selection" (a top-k runs
// inside the fetched subset once it is in GPU memory).
#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

// ------------------------------------------------------------------ union
__global__ void union_kernel(size_t nwords, const uint32_t* __restrict__ m, uint32_t* __restrict__ U,
                             uint32_t* __restrict__ nw) {
  const size_t n4 = nwords / 4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t t0 = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  const uint4* m4 = reinterpret_cast<const uint4*>(m);
  uint4* U4 = reinterpret_cast<uint4*>(U);
  uint4* n4p = reinterpret_cast<uint4*>(nw);
  for (size_t i = t0; i < n4; i += stride) {
    const uint4 a = m4[i];
    uint4 u = U4[i];
    if (nw) n4p[i] = make_uint4(a.x & ~u.x, a.y & ~u.y, a.z & ~u.z, a.w & ~u.w);
    u.x |= a.x; u.y |= a.y; u.z |= a.z; u.w |= a.w;
    U4[i] = u;
  }
  for (size_t i = n4 * 4 + t0; i < nwords; i += stride) {
    const uint32_t a = m[i], u = U[i];
    if (nw) nw[i] = a & ~u;
    U[i] = u | a;
  }
}

// ------------------------------------------------------------------ block scan
// Exclusive scan of one int per thread over a 1024-thread block; returns the
// exclusive prefix and writes the block total to *total (shared).
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tmp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nwarps = blockDim.x >> 5;
    int x = lane < nwarps ? warp_tmp[lane] : 0;
    int xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += t;
    }
    if (lane < nwarps) warp_tmp[lane] = xi - x;
    if (lane == 31) *total = xi;
  }
  __syncthreads();
  const int r = warp_tmp[warp] + incl - v;
  __syncthreads();   // warp_tmp / total may be reused by the caller's next scan
  return r;
}

// ------------------------------------------------------------------ compact
__global__ void __launch_bounds__(1024)
compact_kernel(const uint32_t* __restrict__ bits, int Nw, int cap, int32_t* __restrict__ idx,
               int32_t* __restrict__ count, int32_t* status) {
  __shared__ int warp_tmp[32];
  __shared__ int total;
  const int b = blockIdx.x;
  const uint32_t* row = bits + static_cast<size_t>(b) * Nw;
  int32_t* out = idx + static_cast<size_t>(b) * cap;
  int base = 0;
  for (int w0 = 0; w0 < Nw; w0 += blockDim.x) {
    const int wi = w0 + threadIdx.x;
    uint32_t word = wi < Nw ? row[wi] : 0u;
    const int c = __popc(word);
    int pos = base + block_exclusive_scan(c, warp_tmp, &total);
    while (word) {
      const int bit = __ffs(word) - 1;
      word &= word - 1;
      if (pos < cap) out[pos] = wi * 32 + bit;
      ++pos;
    }
    base += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    count[b] = base;
    if (base > cap) raise_status(status, LSA_ERR_CAPACITY);
  }
}

// ------------------------------------------------------------------ top-k
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);   // larger float -> larger key
}

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;

// One block per sequence: keys, 4 radix passes of 8 bits for the k-th largest key,
// then a stable pass that keeps every key above it and the lowest-index ties.
__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(int B, int L, int N, int k, const int32_t* __restrict__ idx, int cap,
            const int32_t* __restrict__ count, const float* __restrict__ logit,
            int32_t* __restrict__ topk, int32_t* __restrict__ topk_count,
            uint32_t* __restrict__ keys_ws) {
  __shared__ int sub[kTopkWarps][256];
  __shared__ int hist[256];
  __shared__ int warp_tmp[32];
  __shared__ int total;
  __shared__ uint32_t s_prefix;
  __shared__ int s_kk;
  const int b = blockIdx.x, tid = threadIdx.x, warp = tid >> 5;
  int n = count[b];
  n = max(0, min(n, cap));
  const int32_t* ib = idx + static_cast<size_t>(b) * cap;
  int32_t* ob = topk + static_cast<size_t>(b) * k;
  if (n <= k) {
    for (int j = tid; j < k; j += kTopkThreads) ob[j] = j < n ? ib[j] : -1;
    if (tid == 0 && topk_count) topk_count[b] = n;
    return;
  }
  uint32_t* kb = keys_ws + static_cast<size_t>(b) * cap;
  uint32_t prefix = 0, himask = 0;
  int kk = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < kTopkWarps * 256; i += kTopkThreads) (&sub[0][0])[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += kTopkThreads) {
      uint32_t u;
      if (pass == 0) {
        const int e = ib[j];
        float key = -INFINITY;
        if (e >= 0 && e < N)
          for (int l = 0; l < L; ++l) key = fmaxf(key, logit[(static_cast<size_t>(l) * B + b) * N + e]);
        u = order_key(key);
        kb[j] = u;
      } else {
        u = kb[j];
      }
      if ((u & himask) == prefix) atomicAdd(&sub[warp][(u >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 256) {
      int h = 0;
      for (int w = 0; w < kTopkWarps; ++w) h += sub[w][tid];
      hist[tid] = h;
    }
    __syncthreads();
    if (tid == 0) {
      int cum = 0, sel = 0;
      for (int d = 255; d >= 0; --d) {
        if (cum + hist[d] >= kk) { sel = d; break; }
        cum += hist[d];
      }
      s_kk = kk - cum;
      s_prefix = prefix | (static_cast<uint32_t>(sel) << shift);
    }
    __syncthreads();
    kk = s_kk;
    prefix = s_prefix;
    himask |= 255u << shift;
    __syncthreads();
  }
  // prefix = k-th largest key T; kk = how many keys equal to T to keep (lowest j first)
  const uint32_t T = prefix;
  int gt_base = 0, eq_base = 0;
  for (int j0 = 0; j0 < n; j0 += kTopkThreads) {
    const int j = j0 + tid;
    const uint32_t u = j < n ? kb[j] : 0u;
    const int gt = (j < n && u > T) ? 1 : 0;
    const int eq = (j < n && u == T) ? 1 : 0;
    const int packed = gt | (eq << 16);
    const int ex = block_exclusive_scan(packed, warp_tmp, &total);
    const int gt_before = gt_base + (ex & 0xFFFF);
    const int eq_before = eq_base + (ex >> 16);
    if (gt || (eq && eq_before < kk)) ob[gt_before + min(eq_before, kk)] = ib[j];
    gt_base += total & 0xFFFF;
    eq_base += total >> 16;
    __syncthreads();
  }
  if (tid == 0 && topk_count) topk_count[b] = k;
}

}  // namespace

int launch_union(int B, int Nw, const uint32_t* m, uint32_t* U, uint32_t* nw, cudaStream_t s) {
  const size_t n = static_cast<size_t>(B) * Nw;
  if (n == 0) return LSA_OK;
  const unsigned grid = (unsigned)std::min<size_t>((n / 4 + 255) / 256 + 1, 148 * 8);
  union_kernel<<<grid, 256, 0, s>>>(n, m, U, nw);
  return check_launch("select_union");
}

int launch_compact(int B, int N, const uint32_t* bits, int cap, int32_t* idx, int32_t* count,
                   int32_t* status, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  compact_kernel<<<B, 1024, 0, s>>>(bits, (N + 31) / 32, cap, idx, count, status);
  return check_launch("compact");
}

int launch_topk(int B, int L, int N, int k, const int32_t* idx, int cap, const int32_t* count,
                const float* logit, int32_t* topk, int32_t* topk_count, uint32_t* keys_ws,
                cudaStream_t s) {
  if (B == 0) return LSA_OK;
  topk_kernel<<<B, kTopkThreads, 0, s>>>(B, L, N, k, idx, cap, count, logit, topk, topk_count, keys_ws);
  return check_launch("topk");
}

}  // namespace lsa
