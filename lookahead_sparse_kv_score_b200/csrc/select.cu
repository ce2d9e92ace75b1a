// Selection after scoring: OR-union of indexer layers, fetch-list compaction and the
// fine top-k inside the fetched subset.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science): §2.4 (three indexer
// layers whose predictions are combined by union, OR mode), §2.1 "dynamic fetch"
// (every entry with I >= 0.5 is fetched) and "hierarchical selection" (a top-k runs
// inside the fetched subset once it is in GPU memory).
#include <algorithm>
#include <type_traits>

#include <cooperative_groups.h>

#include "lsa_common.cuh"

namespace lsa {
namespace {

namespace cg = cooperative_groups;

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
// Block (chunk, b) owns words [chunk*kCompactWords, ...) of sequence b.  Its output
// base is the popcount of all earlier words of the sequence (re-read from L2, at most
// a few tens of KB); its indices are staged in shared memory and written coalesced.
constexpr int kCompactWords = 256;
constexpr int kCompactThreads = 256;

__global__ void __launch_bounds__(kCompactThreads)
compact_kernel(const uint32_t* __restrict__ bits, int Nw, int cap, int32_t* __restrict__ idx,
               int32_t* __restrict__ count, int32_t* status) {
  __shared__ int warp_tmp[32];
  __shared__ int total;
  __shared__ int sred[kCompactThreads / 32];
  __shared__ int32_t sidx[kCompactWords * 32];
  const int b = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
  const uint32_t* row = bits + static_cast<size_t>(b) * Nw;
  const int w0 = chunk * kCompactWords;
  // base: set bits in words [0, w0)
  int pc = 0;
  const int nvec = w0 / 4;             // w0 is a multiple of 4; row is 16-byte aligned when Nw % 4 == 0
  if ((Nw & 3) == 0) {
    const uint4* r4 = reinterpret_cast<const uint4*>(row);
    for (int i = tid; i < nvec; i += kCompactThreads) {
      const uint4 v = __ldg(r4 + i);
      pc += __popc(v.x) + __popc(v.y) + __popc(v.z) + __popc(v.w);
    }
  } else {
    for (int i = tid; i < w0; i += kCompactThreads) pc += __popc(__ldg(row + i));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) pc += __shfl_xor_sync(0xffffffffu, pc, o);
  if ((tid & 31) == 0) sred[tid >> 5] = pc;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < kCompactThreads / 32; ++w) base += sred[w];
  // own words
  const int wi = w0 + tid;
  uint32_t word = wi < Nw ? __ldg(row + wi) : 0u;
  int pos = block_exclusive_scan(__popc(word), warp_tmp, &total);
  while (word) {
    const int bit = __ffs(word) - 1;
    word &= word - 1;
    sidx[pos++] = wi * 32 + bit;
  }
  __syncthreads();
  const int n = total;
  int32_t* out = idx + static_cast<size_t>(b) * cap;
  for (int i = tid; i < n; i += kCompactThreads)
    if (base + i < cap) out[base + i] = sidx[i];
  if (chunk == static_cast<int>(gridDim.x) - 1 && tid == 0) {
    count[b] = base + n;
    if (base + n > cap) raise_status(status, LSA_ERR_CAPACITY);
  }
}

// ------------------------------------------------------------------ union + fetch lists
// The whole selection of one trigger in two launches over the L layer masks (three with
// the union's top-k keys): per word, new_l = mask_l & ~(mask_0 | .. | mask_{l-1}) and
// U = mask_0 | .. | mask_{L-1}, and the L + 1 fetch lists (new_0 .. new_{L-1}, U) with
// their counts.  Block (chunk, b) owns words [chunk*kCompactWords, ...) of sequence b.
// The first launch writes each chunk's popcounts of the L + 1 sets; the second takes its
// output bases from the earlier chunks' counts; each warp stages its run of every list in
// shared memory and copies it out with full stores; the third (select_keys_kernel) forms
// the keys of the union's list.
constexpr int kSelMaxLayers = 8;

// Per (chunk, sequence): the popcounts of the chunk's words in the L new sets and the
// union, written to counts[b][chunk][kSelMaxLayers + 1] (slot kSelMaxLayers = union).
// kML >= L bounds the layers the kernel is compiled for (3 or kSelMaxLayers).
template <int kML>
__global__ void __launch_bounds__(kCompactThreads)
select_count_kernel(const uint32_t* __restrict__ mask, int L, size_t lstride, int Nw, int32_t* __restrict__ counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ int sred[kML + 1][kCompactThreads / 32];
  const int b = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t* mb = mask + static_cast<size_t>(b) * Nw;
  const int wi = chunk * kCompactWords + tid;
  int pc[kML + 1];
  uint32_t mw[kML];
#pragma unroll
  for (int l = 0; l < kML; ++l) {            // every layer's word loaded before any is used
    mw[l] = 0u;
    if (l < L && wi < Nw) mw[l] = __ldg(mb + l * lstride + wi);
  }
  uint32_t acc = 0;
#pragma unroll
  for (int l = 0; l < kML; ++l) {
    pc[l] = __popc(mw[l] & ~acc);
    acc |= mw[l];
  }
  pc[kML] = __popc(acc);
#pragma unroll
  for (int j = 0; j <= kML; ++j) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pc[j] += __shfl_xor_sync(0xffffffffu, pc[j], o);
    if (lane == 0) sred[j][warp] = pc[j];
  }
  __syncthreads();
  if (tid <= kML) {
    int t = 0;
    for (int w = 0; w < kCompactThreads / 32; ++w) t += sred[tid][w];
    const int slot = tid == kML ? kSelMaxLayers : tid;
    counts[(static_cast<size_t>(b) * gridDim.x + chunk) * (kSelMaxLayers + 1) + slot] = t;
  }
}

template <int kML>
__global__ void __launch_bounds__(kCompactThreads, 4)
select_fetch_kernel(const uint32_t* __restrict__ mask, int L, size_t lstride, int Nw, int cap,
                    const int32_t* __restrict__ counts, uint32_t* __restrict__ U, uint32_t* __restrict__ nw,
                    int32_t* __restrict__ idx_new, int32_t* __restrict__ cnt_new, size_t cstride,
                    int32_t* __restrict__ idx_U, int32_t* __restrict__ cnt_U, int32_t* status,
                    int32_t* __restrict__ ubase) {
  pdl_wait();
  pdl_trigger();
  __shared__ int base_s[kML + 1];
  __shared__ int wsum[kML + 1][kCompactThreads / 32];
  __shared__ int32_t wstage[kCompactThreads / 32][32 * 32];   // one warp's words hold at most 1024 indices
  const int b = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t* mb = mask + static_cast<size_t>(b) * Nw;
  const int w0 = chunk * kCompactWords;
  // own word: every layer's word loaded first, so that these loads and the bases' below
  // are in flight together
  const int wi = w0 + tid;
  uint32_t word[kML + 1];
  uint32_t mw[kML];
#pragma unroll
  for (int l = 0; l < kML; ++l) {
    mw[l] = 0u;
    if (l < L && wi < Nw) mw[l] = __ldg(mb + l * lstride + wi);
  }
  // bases: the lists' set bits in the earlier chunks of this sequence (list q, q = kML
  // the union, summed by warp q mod 8, its lanes over the chunks, so no load waits on
  // another)
  for (int q = warp; q <= kML; q += kCompactThreads / 32) {
    const int slot = q == kML ? kSelMaxLayers : q;
    int t = 0;
    const int32_t* cb = counts + static_cast<size_t>(b) * gridDim.x * (kSelMaxLayers + 1) + slot;
    for (int c = lane; c < chunk; c += 32) t += __ldg(cb + c * (kSelMaxLayers + 1));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) base_s[q] = t;
  }
  {
    uint32_t acc = 0;
#pragma unroll
    for (int l = 0; l < kML; ++l) {
      word[l] = mw[l] & ~acc;
      acc |= mw[l];
      if (nw && l < L && wi < Nw) nw[l * lstride + static_cast<size_t>(b) * Nw + wi] = word[l];
    }
    word[kML] = acc;
    if (U && wi < Nw) U[static_cast<size_t>(b) * Nw + wi] = acc;
  }
  const bool last = chunk == static_cast<int>(gridDim.x) - 1;
  // every list's offsets for the block in one pass: warp prefix sums of the popcounts,
  // one barrier, then the warps' bases (a warp's threads cover one contiguous run of
  // each list)
  int incl[kML + 1];
#pragma unroll
  for (int q = 0; q <= kML; ++q) {
    const int v = (q < L || q == kML) ? __popc(word[q]) : 0;
    incl[q] = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl[q], o);
      if (lane >= o) incl[q] += t;
    }
    if (lane == 31) wsum[q][warp] = incl[q];
  }
  __syncthreads();
#pragma unroll 1
  for (int j = 0; j <= L; ++j) {
    const int jj = j == L ? kML : j;
    const int base = base_s[jj];
    int before = 0, total = 0;
    for (int w = 0; w < kCompactThreads / 32; ++w) {
      const int ws = wsum[jj][w];
      before += w < warp ? ws : 0;
      total += ws;
    }
    uint32_t bits = 0;
    int inc = 0;
#pragma unroll
    for (int q = 0; q <= kML; ++q)
      if (q == jj) { bits = word[q]; inc = incl[q]; }
    // the warp's run of this list: staged in its own shared buffer in list order, then
    // copied out with full 128-byte stores
    int32_t* stage = wstage[warp];
    int wp = inc - __popc(bits);                     // this lane's offset inside the warp's run
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      stage[wp++] = wi * 32 + bit;
    }
    __syncwarp();
    const int wtot = __shfl_sync(0xffffffffu, inc, 31);
    const int wbase = base + before;
    int32_t* out = (j == L ? idx_U + static_cast<size_t>(b) * cap : idx_new + j * cstride * cap + static_cast<size_t>(b) * cap);
    for (int i = lane; i < wtot; i += 32)
      if (wbase + i < cap) out[wbase + i] = stage[i];
    if (j == L && ubase && lane == 0) ubase[static_cast<size_t>(b) * (gridDim.x * (kCompactThreads / 32)) +
                                          chunk * (kCompactThreads / 32) + warp] = wbase;
    __syncwarp();
    if (last && tid == 0) {
      int32_t* cnt = j == L ? cnt_U + b : cnt_new + j * cstride + b;
      *cnt = base + total;
      if (base + total > cap) raise_status(status, LSA_ERR_CAPACITY);
    }
  }
}

// The union's top-k keys: key_U[b][j] = order_key(max over layers of logit[l][b][e]) for
// the j-th union entry e.  One warp per 32 union words (1024 entries), independent of
// the others: its run of the union list starts at ubase[b][warp] (from the fetch
// kernel), each word's offset is a warp prefix sum of the popcounts, and the logits are
// read densely (lane t: the four entries 128 k + 4 t, k = 0..7; groups without a
// candidate are skipped), every load of the warp issued before the first is used; the
// keys are staged in shared memory in list order and written out with full stores.
template <int kML>
__global__ void __launch_bounds__(256)
select_keys_kernel(const uint32_t* __restrict__ U, int Nw, int L, int N, int cap, const int32_t* __restrict__ ubase,
                   int wpb, const float* __restrict__ logit, int Bfull, int b_off, uint32_t* __restrict__ key_U) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t kstage[8][32 * 32];          // a warp's keys in list order, then copied out
  const int b = blockIdx.y, lane = threadIdx.x & 31;
  const int wg = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);   // warp of words [32 wg, 32 wg + 32)
  if (wg * 32 >= Nw) return;
  uint32_t* stage = kstage[threadIdx.x >> 5];
  const int wi = wg * 32 + lane;
  const uint32_t uw = wi < Nw ? __ldg(U + static_cast<size_t>(b) * Nw + wi) : 0u;
  const int base = __ldg(ubase + static_cast<size_t>(b) * wpb + wg);
  int inc = __popc(uw);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  const int ex = inc - __popc(uw);
  const float* lb = logit + static_cast<size_t>(b_off + b) * N;
  const size_t lstep = static_cast<size_t>(Bfull) * N;
  uint32_t* kout = key_U + static_cast<size_t>(b) * cap;
  const bool vec = (N % 4 == 0) && (reinterpret_cast<uintptr_t>(logit) % 16 == 0);
  const int sh = (lane & 7) * 4;                    // bit of entry 128 k + 4 lane in its word
  constexpr int kGroups = 8;
  constexpr int kHalf = kML <= 3 ? 4 : 1;          // groups whose loads are in flight together
#pragma unroll
  for (int k0 = 0; k0 < kGroups; k0 += kHalf) {
    uint32_t wd[kHalf], nib[kHalf];
    int off[kHalf];
    float m[kHalf][4];
#pragma unroll
    for (int u = 0; u < kHalf; ++u) {
      const int src = 4 * (k0 + u) + (lane >> 3);   // the word holding those entries
      wd[u] = __shfl_sync(0xffffffffu, uw, src);
      off[u] = __shfl_sync(0xffffffffu, ex, src);
      nib[u] = (wd[u] >> sh) & 0xFu;
#pragma unroll
      for (int i = 0; i < 4; ++i) m[u][i] = -INFINITY;
    }
    if (vec) {
      // every load first (predicated, no branch between a load and its use), then the maxima
      float4 v[kHalf][kML];
#pragma unroll
      for (int l = 0; l < kML; ++l)
#pragma unroll
        for (int u = 0; u < kHalf; ++u) {
          const int e0 = wg * 1024 + 128 * (k0 + u) + 4 * lane;
          v[u][l] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
          if (l < L && nib[u] != 0u && e0 < N)
            v[u][l] = __ldg(reinterpret_cast<const float4*>(lb + l * lstep + e0));
        }
#pragma unroll
      for (int l = 0; l < kML; ++l)
#pragma unroll
        for (int u = 0; u < kHalf; ++u) {
          m[u][0] = fmaxf(m[u][0], v[u][l].x); m[u][1] = fmaxf(m[u][1], v[u][l].y);
          m[u][2] = fmaxf(m[u][2], v[u][l].z); m[u][3] = fmaxf(m[u][3], v[u][l].w);
        }
    } else {
      for (int l = 0; l < L; ++l)
#pragma unroll
        for (int u = 0; u < kHalf; ++u) {
          const int e0 = wg * 1024 + 128 * (k0 + u) + 4 * lane;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (((nib[u] >> i) & 1u) && e0 + i < N) m[u][i] = fmaxf(m[u][i], __ldg(lb + l * lstep + e0 + i));
        }
    }
#pragma unroll
    for (int u = 0; u < kHalf; ++u) {
      int pos = off[u] + __popc(wd[u] & ((1u << sh) - 1u));   // offset in the warp's run
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if ((nib[u] >> i) & 1u) stage[pos++] = order_key(m[u][i]);
    }
  }
  __syncwarp();
  const int wtot = __shfl_sync(0xffffffffu, inc, 31);
  for (int i = lane; i < wtot; i += 32)
    if (base + i < cap) kout[base + i] = stage[i];
}

// ------------------------------------------------------------------ top-k

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSmemKeys = 32768;   // keys of one CTA's candidate slice held in shared memory
constexpr int kSubHists = 8;           // digit histograms, one per four warps (fewer same-bin collisions)
constexpr int kDigitBins = 2048;       // radix digits of 11, 11 and 10 bits
constexpr int kKeyBatch = 8;           // keys a thread loads before using any
constexpr int kKeptCap = 512;          // positions of kept keys a warp records (in the digit histograms' space)
constexpr int kBinsPerThread = kDigitBins / kTopkThreads;
static_assert(kBinsPerThread == 2, "two digit bins per thread");
static_assert(kTopkWarps * kKeptCap <= kSubHists * kDigitBins, "kept positions fit in the digit histograms");

struct TopkShared {
  int sub[kSubHists][kDigitBins];   // digit histograms, one per four warps
  int hist[2][kDigitBins];   // this CTA's digit histogram by pass parity, read by the whole cluster
  int warp_tmp[32];
  int wgt[kTopkWarps], weq[kTopkWarps];   // per-warp counts of keys above T and equal to T
  int cnt[2];                // this CTA's counts above T and equal to T, read by the cluster
  int gbase, ebase;
  uint32_t prefix;
  int kk;
  int total;
};
constexpr int kTopkStateBytes = (static_cast<int>(sizeof(TopkShared)) + 15) / 16 * 16;

// Candidates and keys come in one of three ways.  Fetched-set mode: candidate j is entry
// idx[b][j] (j < count[b]) with key order_key(max over layers of logit[l][b][entry]),
// and k is the same for every sequence.  Keyed mode (idx and dkeys given): the same
// candidates with the keys given per candidate, dkeys[b][j].  Direct mode (dkeys without
// idx): candidate j is j itself for j < cap, its key is dkeys[b][j], and sequence b keeps
// kdev[b] of them, or none (raising LSA_ERR_CAPACITY) when kdev[b] exceeds cap - kept[b];
// the output row stride is then cap.
//
// One thread-block cluster per sequence; CTA `rank` owns the contiguous candidate slice
// [rank m, (rank + 1) m), m = ceil(n / cluster size).  Its keys go to shared memory when
// the slice fits in kTopkSmemKeys; otherwise given keys are read in place and computed
// keys go to the key workspace.  Three radix passes (digits of 11, 11 and 10 bits, most
// significant first) find the k-th largest key T and the number kk of keys equal to T to
// keep; each pass adds the CTAs' digit histograms through distributed shared memory and
// picks the digit with one block-wide scan.  The kept entries, all keys above T and the
// kk lowest-index ties, are written in ascending candidate (= entry) order: each warp
// owns a contiguous part of its CTA's slice, records where its keys at or above T are
// while counting them, and takes its output offset from the counts of the CTAs and warps
// before it.
__global__ void __launch_bounds__(kTopkThreads, 1)
topk_cluster_kernel(int B, int L, int N, int k, const int32_t* __restrict__ idx, int cap,
                    const int32_t* __restrict__ count, const float* __restrict__ logit,
                    const uint32_t* __restrict__ dkeys, const int32_t* __restrict__ kdev,
                    const int32_t* __restrict__ kept, int32_t* status,
                    uint32_t* __restrict__ keys_ws, int32_t* __restrict__ topk, int32_t* __restrict__ topk_count) {
  pdl_wait();
  pdl_trigger();
  // dynamic shared memory: the shared state, then the key slice
  extern __shared__ __align__(16) uint8_t topk_smem[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(topk_smem);
  uint32_t* skeys = reinterpret_cast<uint32_t*>(topk_smem + kTopkStateBytes);
  cg::cluster_group cl = cg::this_cluster();
  const int cs = static_cast<int>(cl.num_blocks());
  const int rank = static_cast<int>(cl.block_rank());
  const int b = blockIdx.x / cs;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool direct = dkeys != nullptr && idx == nullptr;   // keys given per slot, outputs are slots
  const bool keyed = dkeys != nullptr && idx != nullptr;     // keys given per candidate of idx
  int n, kb;                         // candidates and keys to keep for this sequence
  if (direct) {
    n = cap;
    kb = max(0, kdev[b]);
    if (kb > cap - kept[b]) {
      if (rank == 0 && tid == 0) raise_status(status, LSA_ERR_CAPACITY);
      kb = 0;
    }
  } else {
    n = max(0, min(count[b], cap));
    kb = k;
  }
  const int32_t* ib = direct ? nullptr : idx + static_cast<size_t>(b) * cap;
  int32_t* ob = topk + static_cast<size_t>(b) * (direct ? cap : k);
  if (n <= kb || kb == 0) {          // the same for every CTA of the cluster: no barrier follows
    if (rank == 0) {
      const int m = min(n, kb);
      for (int j = tid; j < (direct ? m : k); j += kTopkThreads) ob[j] = j < m ? (direct ? j : ib[j]) : -1;
      if (tid == 0 && topk_count) topk_count[b] = m;
    }
    return;
  }
  const int m = (n + cs - 1) / cs;
  const int j0 = min(n, rank * m), mloc = min(n, j0 + m) - j0;
  // the slice's keys: in shared memory when they fit; otherwise read in place (given keys)
  // or computed into the key workspace
  const bool in_smem = m <= kTopkSmemKeys;
  uint32_t* key = in_smem ? skeys
                          : ((direct || keyed) ? const_cast<uint32_t*>(dkeys) + static_cast<size_t>(b) * cap + j0
                                               : keys_ws + static_cast<size_t>(b) * cap + j0);
  if (direct || keyed) {
    if (in_smem) {
      const uint32_t* src = dkeys + static_cast<size_t>(b) * cap + j0;
      for (int jb = 0; jb < mloc; jb += kKeyBatch * kTopkThreads) {
        uint32_t v[kKeyBatch];
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
          const int j = jb + u * kTopkThreads + tid;
          v[u] = j < mloc ? __ldg(src + j) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
          const int j = jb + u * kTopkThreads + tid;
          if (j < mloc) key[j] = v[u];
        }
      }
    }
  } else {
    // eight candidates per thread in flight: their entries first, then every layer's logits
    constexpr int kBatch = 8;
    for (int jb = 0; jb < mloc; jb += kBatch * kTopkThreads) {
      int e[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = jb + u * kTopkThreads + tid;
        e[u] = j < mloc ? __ldg(ib + j0 + j) : -1;
      }
      float z[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) z[u] = -INFINITY;
      for (int l = 0; l < L; ++l) {
        const float* lb = logit + (static_cast<size_t>(l) * B + b) * N;
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (e[u] >= 0 && e[u] < N) z[u] = fmaxf(z[u], __ldg(lb + e[u]));
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = jb + u * kTopkThreads + tid;
        if (j < mloc) key[j] = order_key(z[u]);
      }
    }
  }
  __syncthreads();
  uint32_t prefix = 0, himask = 0;
  int kk = kb;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const uint32_t dmask = pass == 2 ? 1023u : 2047u;
    for (int i = tid; i < kSubHists * kDigitBins; i += kTopkThreads) (&sh.sub[0][0])[i] = 0;
    __syncthreads();
    int* mysub = sh.sub[warp % kSubHists];
    for (int jb = 0; jb < mloc; jb += kKeyBatch * kTopkThreads) {
      uint32_t v[kKeyBatch];   // loaded before use: slices in global memory stay latency-hidden
#pragma unroll
      for (int u = 0; u < kKeyBatch; ++u) {
        const int j = jb + u * kTopkThreads + tid;
        v[u] = j < mloc ? key[j] : 0u;
      }
#pragma unroll
      for (int u = 0; u < kKeyBatch; ++u) {
        const int j = jb + u * kTopkThreads + tid;
        if (j < mloc && (v[u] & himask) == prefix) atomicAdd(&mysub[(v[u] >> shift) & dmask], 1);
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kBinsPerThread; ++q) {
      const int d = tid * kBinsPerThread + q;
      int h = 0;
#pragma unroll
      for (int c = 0; c < kSubHists; ++c) h += sh.sub[c][d];
      sh.hist[pass & 1][d] = h;
    }
    // After this barrier every CTA's histogram of the pass is complete.  A CTA rewrites
    // hist[pass & 1] two passes later, after the next barrier, which no CTA passes
    // before it has finished reading this pass's histograms.
    cl.sync();
    // thread t holds the totals of digits D - 1 - 2t and D - 2 - 2t (descending order),
    // so an exclusive scan in thread order counts the keys in higher digits
    int tot[kBinsPerThread], mine = 0;
#pragma unroll
    for (int q = 0; q < kBinsPerThread; ++q) {
      const int d = kDigitBins - 1 - (tid * kBinsPerThread + q);
      int v[8];                 // every rank's count loaded before any is added
#pragma unroll
      for (int r = 0; r < 8; ++r) v[r] = r < cs ? cl.map_shared_rank(&sh.hist[pass & 1][0], r)[d] : 0;
      int t = 0;
#pragma unroll
      for (int r = 0; r < 8; ++r) t += v[r];
      tot[q] = t;
      mine += t;
    }
    int above = block_exclusive_scan(mine, sh.warp_tmp, &sh.total);
#pragma unroll
    for (int q = 0; q < kBinsPerThread; ++q) {
      const int d = kDigitBins - 1 - (tid * kBinsPerThread + q);
      if (above < kk && above + tot[q] >= kk) {   // the digit holding the kk-th largest key
        sh.kk = kk - above;
        sh.prefix = prefix | (static_cast<uint32_t>(d) << shift);
      }
      above += tot[q];
    }
    __syncthreads();
    kk = sh.kk;
    prefix = sh.prefix;
    himask |= dmask << shift;
  }
  const uint32_t T = prefix;
  // this warp's contiguous part of the slice
  const int per = (mloc + kTopkWarps - 1) / kTopkWarps;
  const int w0 = min(mloc, warp * per), w1 = min(mloc, w0 + per);
  // The warp counts its keys above and equal to T and records where they are (ascending,
  // in the digit histograms' space, free after the last pass), so that the output needs
  // no second pass over the part unless more than kKeptCap of them fell in it.
  const uint32_t lt = (1u << lane) - 1u;
  int* wpos = &sh.sub[0][0] + warp * kKeptCap;
  int nk = 0;
  {
    int gt = 0, eq = 0;
    for (int jb = w0; jb < w1; jb += 32 * kKeyBatch) {
      uint32_t v[kKeyBatch];
#pragma unroll
      for (int u = 0; u < kKeyBatch; ++u) {
        const int j = jb + u * 32 + lane;
        v[u] = j < w1 ? key[j] : 0u;
      }
#pragma unroll
      for (int u = 0; u < kKeyBatch; ++u) {
        const int j = jb + u * 32 + lane;
        const bool g = j < w1 && v[u] > T, q = j < w1 && v[u] == T;
        const uint32_t gm = __ballot_sync(0xffffffffu, g), qm = __ballot_sync(0xffffffffu, q);
        const uint32_t km = gm | qm;
        const int at = nk + __popc(km & lt);
        if ((g || q) && at < kKeptCap) wpos[at] = j;
        nk += __popc(km);
        gt += __popc(gm);
        eq += __popc(qm);
      }
    }
    if (lane == 0) { sh.wgt[warp] = gt; sh.weq[warp] = eq; }
    __syncthreads();
    if (warp == 0) {
      int g = sh.wgt[lane], q = sh.weq[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        q += __shfl_xor_sync(0xffffffffu, q, o);
      }
      if (lane == 0) { sh.cnt[0] = g; sh.cnt[1] = q; }
    }
    cl.sync();
    if (warp == 0) {            // lane r reads rank r's counts; the lower ranks' are summed
      int g = 0, q = 0;
      if (lane < rank) {
        const int* rc = cl.map_shared_rank(&sh.cnt[0], lane);
        g = rc[0];
        q = rc[1];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        g += __shfl_xor_sync(0xffffffffu, g, o);
        q += __shfl_xor_sync(0xffffffffu, q, o);
      }
      if (lane == 0) { sh.gbase = g; sh.ebase = q; }
    }
    cl.sync();   // no CTA leaves while another may still read its shared memory
  }
  int gt_before = sh.gbase, eq_before = sh.ebase;
  for (int w = 0; w < warp; ++w) { gt_before += sh.wgt[w]; eq_before += sh.weq[w]; }
  if (nk <= kKeptCap) {
    for (int i0 = 0; i0 < nk; i0 += 32) {
      const int i = i0 + lane;
      const int j = i < nk ? wpos[i] : 0;
      const uint32_t u = i < nk ? key[j] : 0u;
      const bool g = i < nk && u > T, q = i < nk && u == T;
      const uint32_t gm = __ballot_sync(0xffffffffu, g), qm = __ballot_sync(0xffffffffu, q);
      const int gb = gt_before + __popc(gm & lt), qb = eq_before + __popc(qm & lt);
      const int c = j0 + j;
      if (g) ob[gb + min(qb, kk)] = direct ? c : __ldg(ib + c);
      else if (q && qb < kk) ob[gb + qb] = direct ? c : __ldg(ib + c);
      gt_before += __popc(gm);
      eq_before += __popc(qm);
    }
    if (rank == 0 && tid == 0 && topk_count) topk_count[b] = kb;
    return;
  }
  constexpr int kOutBatch = 4;
  for (int jb0 = w0; jb0 < w1; jb0 += 32 * kOutBatch) {
    uint32_t v[kOutBatch];
#pragma unroll
    for (int u = 0; u < kOutBatch; ++u) {
      const int j = jb0 + u * 32 + lane;
      v[u] = j < w1 ? key[j] : 0u;
    }
#pragma unroll
    for (int u = 0; u < kOutBatch; ++u) {
      const int j = jb0 + u * 32 + lane;
      const bool g = j < w1 && v[u] > T, q = j < w1 && v[u] == T;
      const uint32_t gm = __ballot_sync(0xffffffffu, g), qm = __ballot_sync(0xffffffffu, q);
      const int gb = gt_before + __popc(gm & lt), qb = eq_before + __popc(qm & lt);
      const int c = j0 + j;
      if (g) ob[gb + min(qb, kk)] = direct ? c : __ldg(ib + c);
      else if (q && qb < kk) ob[gb + qb] = direct ? c : __ldg(ib + c);
      gt_before += __popc(gm);
      eq_before += __popc(qm);
    }
  }
  if (rank == 0 && tid == 0 && topk_count) topk_count[b] = kb;
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
  const int Nw = (N + 31) / 32;
  constexpr int kSeqPerLaunch = 65535;   // the sequence index is gridDim.y
  int launches = 0;
  for (int b0 = 0; b0 < B; b0 += kSeqPerLaunch) {
    const int nb = std::min(kSeqPerLaunch, B - b0);
    const dim3 grid(std::max(1, (Nw + kCompactWords - 1) / kCompactWords), nb);
    compact_kernel<<<grid, kCompactThreads, 0, s>>>(bits + static_cast<size_t>(b0) * Nw, Nw, cap,
                                                    idx + static_cast<size_t>(b0) * cap, count + b0, status);
    ++launches;
  }
  return check_launch("compact", launches);
}

// Workspace: per-chunk counts [B][chunks][kSelMaxLayers + 1], the union list's base of
// every warp of words [B][chunks * 8], and room for the union words [B][Nw] when the
// caller does not ask for them (the key kernel reads them).
struct SelWs {
  size_t counts, ubase, U, total;
};
static SelWs sel_ws(int B, int N) {
  const int Nw = (N + 31) / 32;
  const size_t chunks = std::max(1, (Nw + kCompactWords - 1) / kCompactWords);
  SelWs w{};
  w.counts = 0;
  w.ubase = align_up(static_cast<size_t>(B) * chunks * (kSelMaxLayers + 1) * 4, 256);
  w.U = align_up(w.ubase + static_cast<size_t>(B) * chunks * (kCompactThreads / 32) * 4, 256);
  w.total = align_up(w.U + static_cast<size_t>(B) * Nw * 4, 256);
  return w;
}

size_t select_fetch_workspace_bytes(int B, int N) { return sel_ws(B, N).total; }

int launch_select_fetch(int B, int L, int N, const uint32_t* mask, uint32_t* U, uint32_t* nw, int cap,
                        int32_t* idx_new, int32_t* cnt_new, int32_t* idx_U, int32_t* cnt_U, int32_t* status,
                        int32_t* ws, const float* logit, uint32_t* key_U, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  const int Nw = (N + 31) / 32;
  const size_t lstride = static_cast<size_t>(B) * Nw;
  const int chunks = std::max(1, (Nw + kCompactWords - 1) / kCompactWords);
  const int wpb = chunks * (kCompactThreads / 32);             // warps of words per sequence
  const SelWs lay = sel_ws(B, N);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  int32_t* counts = reinterpret_cast<int32_t*>(wsb + lay.counts);
  int32_t* ubase = key_U ? reinterpret_cast<int32_t*>(wsb + lay.ubase) : nullptr;
  // the key kernel reads the union words: the caller's, else a workspace copy
  uint32_t* Uw = U ? U : (key_U ? reinterpret_cast<uint32_t*>(wsb + lay.U) : nullptr);
  constexpr int kSeqPerLaunch = 65535;   // the sequence index is gridDim.y
  int launches = 0;
  for (int b0 = 0; b0 < B; b0 += kSeqPerLaunch) {
    const int nb = std::min(kSeqPerLaunch, B - b0);
    const dim3 grid(chunks, nb);
    const size_t o = static_cast<size_t>(b0) * Nw;
    int32_t* cnt = counts + static_cast<size_t>(b0) * chunks * (kSelMaxLayers + 1);
    auto go = [&](auto ml) {
      constexpr int kML = decltype(ml)::value;
      launch_dependent(select_count_kernel<kML>, grid, dim3(kCompactThreads), 0, s, mask + o, L, lstride, Nw, cnt);
      launch_dependent(select_fetch_kernel<kML>, grid, dim3(kCompactThreads), 0, s, mask + o, L, lstride, Nw, cap,
                       static_cast<const int32_t*>(cnt), Uw ? Uw + o : nullptr, nw ? nw + o : nullptr,
                       idx_new + static_cast<size_t>(b0) * cap, cnt_new + b0, static_cast<size_t>(B),
                       idx_U + static_cast<size_t>(b0) * cap, cnt_U + b0, status,
                       ubase ? ubase + static_cast<size_t>(b0) * wpb : nullptr);
      launches += 2;
      if (key_U) {
        const dim3 kgrid((wpb + 7) / 8, nb);
        launch_dependent(select_keys_kernel<kML>, kgrid, dim3(256), 0, s, static_cast<const uint32_t*>(Uw + o), Nw,
                         L, N, cap, static_cast<const int32_t*>(ubase + static_cast<size_t>(b0) * wpb), wpb, logit,
                         B, b0, key_U + static_cast<size_t>(b0) * cap);
        ++launches;
      }
    };
    if (L <= 3)
      go(std::integral_constant<int, 3>{});
    else
      go(std::integral_constant<int, kSelMaxLayers>{});
  }
  return check_launch("select_fetch", launches);
}

namespace {

int launch_topk_cluster(int B, int L, int N, int k, const int32_t* idx, int cap, const int32_t* count,
                        const float* logit, const uint32_t* dkeys, const int32_t* kdev, const int32_t* kept,
                        int32_t* status, int32_t* topk, int32_t* topk_count, uint32_t* keys_ws, cudaStream_t s) {
  const int smem = kTopkStateBytes + kTopkSmemKeys * 4;
  // per device, once: the kernel's attributes, the SM count and the largest cluster size
  // the occupancy calculator accepts (kept so that a launch makes no query calls)
  constexpr int kMaxDevices = 64;
  static int dev_sms[kMaxDevices] = {}, dev_max_cs[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  if (dev_sms[dev] == 0) {
    cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    int best = 1;
    for (int c = 8; c > 1; c >>= 1) {
      cudaLaunchConfig_t q = {};
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = c;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      q.gridDim = dim3(c);
      q.blockDim = dim3(kTopkThreads);
      q.dynamicSmemBytes = smem;
      q.attrs = qa;
      q.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, topk_cluster_kernel, &q) == cudaSuccess && clusters > 0) {
        best = c;
        break;
      }
      cudaGetLastError();
    }
    dev_max_cs[dev] = best;
    dev_sms[dev] = n;
  }
  const int sms = dev_sms[dev];
  // CTAs per sequence: as many as keep B x cs within one wave, at most 8 (portable); when
  // the keys are computed from the logits, at least enough that a full list (cap
  // candidates) keeps every CTA's slice in shared memory (the busiest sequence sets the
  // kernel's time, and computing a slice into global memory costs more than a second
  // wave of clusters).
  int cs = 8;
  while (cs > 1 && B * cs > sms) cs >>= 1;
  // keys computed here must fit in shared memory; given keys can be read in place
  if (dkeys == nullptr)
    while (cs < 8 && (cap + cs - 1) / cs > kTopkSmemKeys) cs <<= 1;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // a dependent launch (pdl_wait in the kernel)
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kTopkThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cs = std::min(cs, dev_max_cs[dev]);
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(B * cs);
  cudaLaunchKernelEx(&cfg, topk_cluster_kernel, B, L, N, k, idx, cap, count, logit, dkeys, kdev, kept, status,
                     keys_ws, topk, topk_count);
  return check_launch("topk");
}

}  // namespace

int launch_topk(int B, int L, int N, int k, const int32_t* idx, int cap, const int32_t* count,
                const float* logit, int32_t* topk, int32_t* topk_count, uint32_t* keys_ws,
                cudaStream_t s) {
  if (B == 0) return LSA_OK;
  return launch_topk_cluster(B, L, N, k, idx, cap, count, logit, nullptr, nullptr, nullptr, nullptr, topk,
                             topk_count, keys_ws, s);
}

int launch_topk_keyed(int B, int k, const int32_t* idx, int cap, const int32_t* count, const uint32_t* keys,
                      int32_t* topk, int32_t* topk_count, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  return launch_topk_cluster(B, 1, 0, k, idx, cap, count, nullptr, keys, nullptr, nullptr, nullptr, topk, topk_count,
                             nullptr, s);
}

int launch_select_keys(int B, int n, const uint32_t* keys, const int32_t* kdev, const int32_t* kept,
                       int32_t* status, int32_t* out, int32_t* out_count, uint32_t* keys_ws, cudaStream_t s) {
  if (B == 0) return LSA_OK;
  return launch_topk_cluster(B, 0, n, 0, nullptr, n, nullptr, nullptr, keys, kdev, kept, status, out, out_count,
                             keys_ws, s);
}

}  // namespace lsa
