// Cross-layer majority-vote labels and their BCE + focal loss.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.2: the indexer logits
// of each layer are turned into probabilities with a softmax, each layer keeps its
// high-confidence entries by nucleus (top-p, p = 0.6) selection, and an entry is a
// golden label when at least theta = 3 of the L layers select it.  §2.3: the indexer
// is trained with binary cross-entropy plus a focal loss.
//
// Nucleus of one row (layer l, position p) over N entries, without sorting:
//   pi_s = e_s / Z with e_s = exp(x_s - max x) (fp32 exp, fp64 sums).  In descending
//   order of x (equal x: lower index first) an entry is selected iff the mass before
//   it is < top_p * Z.  Since pi is increasing in x, the boundary is a threshold key T
//   on the order-preserving integer image of x: everything above T is selected, and of
//   the c entries tied at T the first c_sel in index order, where
//   c_sel = ceil((top_p * Z - mass above T) / e_T).  T is found by a radix select on
//   the keys (four 8-bit digits, most significant first) whose histograms accumulate
//   both counts and mass: each pass keeps the digit whose cumulative mass from the top
//   first reaches the target.
#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int kRowThreads = 512;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kBins = 256;

__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, T* tmp, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  T r = tmp[0];
  for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) r = op(r, tmp[w]);
  __syncthreads();
  return r;
}

// One row per iteration of the block.  selbits [L*P][Nw]; rowparam [L*P] = (T, cutoff index).
__global__ void __launch_bounds__(kRowThreads, 2)
vote_rows_kernel(const float* __restrict__ logits, int rows, int N, float top_p,
                 uint32_t* __restrict__ selbits, int2* __restrict__ rowparam) {
  extern __shared__ __align__(16) uint8_t vsm[];
  double* hmass = reinterpret_cast<double*>(vsm);                          // [warps][256]
  int* hcnt = reinterpret_cast<int*>(hmass + kRowWarps * kBins);           // [warps][256]
  __shared__ float ftmp[kRowWarps];
  __shared__ double dtmp[kRowWarps];
  __shared__ double s_bin_mass[kBins];
  __shared__ int s_bin_cnt[kBins];
  __shared__ int s_sel, s_cnt;
  __shared__ double s_above, s_target;
  __shared__ int s_cut;
  __shared__ int s_tie_base;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Nw = (N + 31) / 32;
  for (int row = blockIdx.x; row < rows; row += gridDim.x) {
    const float* x = logits + static_cast<size_t>(row) * N;
    // ---- max
    float m = -INFINITY;
    for (int s = tid; s < N; s += kRowThreads) m = fmaxf(m, x[s]);
    m = block_reduce(m, ftmp, [](float a, float b) { return fmaxf(a, b); });
    // ---- radix select on the keys with mass histograms
    uint32_t prefix = 0, hmask = 0;
    double above = 0.0, target = 0.0;
    int cnt_final = 0;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = lane; i < kBins; i += 32) {
        hmass[warp * kBins + i] = 0.0;
        hcnt[warp * kBins + i] = 0;
      }
      __syncwarp();
      for (int s = tid; s < N; s += kRowThreads) {
        const float xv = x[s];
        const uint32_t u = order_key(xv);
        if ((u & hmask) == prefix) {
          const int bin = (u >> shift) & (kBins - 1);
          atomicAdd(&hcnt[warp * kBins + bin], 1);
          atomicAdd(&hmass[warp * kBins + bin], static_cast<double>(__expf(xv - m)));
        }
      }
      __syncthreads();
      if (tid < kBins) {
        double ms = 0.0;
        int c = 0;
        for (int w = 0; w < kRowWarps; ++w) {
          ms += hmass[w * kBins + tid];
          c += hcnt[w * kBins + tid];
        }
        s_bin_mass[tid] = ms;
        s_bin_cnt[tid] = c;
      }
      __syncthreads();
      if (warp == 0) {
        // Lane j owns bins 255-8j .. 248-8j (descending).  The selected bin is the first,
        // in descending order, at which base + cumulative mass reaches the target; if
        // rounding keeps the total below the target (top_p close to 1), the lowest
        // non-empty bin is taken (every entry above it is selected).
        double loc = 0.0;
        int nonempty = 0;
        for (int i = 0; i < 8; ++i) {
          const int b = kBins - 1 - (8 * lane + i);
          loc += s_bin_mass[b];
          nonempty |= s_bin_cnt[b] > 0;
        }
        double total = loc;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
        double incl = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const double excl = incl - loc;
        const double tgt = pass == 0 ? static_cast<double>(top_p) * total : s_target;
        const double base = pass == 0 ? 0.0 : s_above;
        const unsigned reach = __ballot_sync(0xffffffffu, nonempty && base + incl >= tgt);
        const unsigned ne = __ballot_sync(0xffffffffu, nonempty);
        const int owner = reach ? __ffs(reach) - 1 : 31 - __clz(ne ? ne : 1u);
        if (lane == owner) {
          double cum = base + excl;
          int sel = -1;
          for (int i = 0; i < 8; ++i) {
            const int b = kBins - 1 - (8 * lane + i);
            if (s_bin_cnt[b] == 0) continue;
            if (reach && cum + s_bin_mass[b] >= tgt) { sel = b; break; }
            sel = b;                       // no reach: ends at the lowest non-empty bin
            if (!reach) { cum += s_bin_mass[b]; continue; }
            cum += s_bin_mass[b];
          }
          if (!reach) cum -= s_bin_mass[sel];   // mass strictly above the selected bin
          s_sel = sel;
          s_above = cum;
          s_cnt = s_bin_cnt[sel];
          if (pass == 0) s_target = tgt;
        }
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(s_sel) << shift;
      hmask |= 255u << shift;
      above = s_above;
      target = s_target;
      cnt_final = s_cnt;
      __syncthreads();
    }
    const uint32_t T = prefix;
    // number of entries tied at T to select, in index order
    const double eT = static_cast<double>(__expf(key_value(T) - m));
    long long want = eT > 0.0 ? static_cast<long long>(ceil((target - above) / eT)) : cnt_final;
    want = want < 1 ? 1 : (want > cnt_final ? cnt_final : want);
    // cutoff index: the want-th tie in index order (all ties when want == cnt_final)
    int cut = N;
    if (want < cnt_final) {
      if (tid == 0) { s_cut = N; s_tie_base = 0; }
      __syncthreads();
      for (int s0 = 0; s0 < N; s0 += kRowThreads) {
        const int s = s0 + tid;
        const bool tie = s < N && order_key(x[s]) == T;
        const unsigned b = __ballot_sync(0xffffffffu, tie);
        if (lane == 0) hcnt[warp] = __popc(b);
        __syncthreads();
        int before = s_tie_base;
        for (int w = 0; w < warp; ++w) before += hcnt[w];
        before += __popc(b & ((1u << lane) - 1));
        if (tie && before + 1 == want) s_cut = s;
        __syncthreads();
        if (tid == 0) {
          int tot = 0;
          for (int w = 0; w < kRowWarps; ++w) tot += hcnt[w];
          s_tie_base += tot;
        }
        __syncthreads();
        if (s_cut < N) break;
      }
      cut = s_cut;
      __syncthreads();
    }
    if (tid == 0) rowparam[row] = make_int2(static_cast<int>(T), cut);
    // ---- selection bits of the row
    uint32_t* out = selbits + static_cast<size_t>(row) * Nw;
    for (int s = tid; s < Nw * 32; s += kRowThreads) {
      bool sel = false;
      if (s < N) {
        const uint32_t u = order_key(x[s]);
        sel = u > T || (u == T && s <= cut);
      }
      const unsigned bits = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) out[s >> 5] = bits;
    }
    __syncthreads();
  }
}

// Per (position, word): count over layers, golden bits (count >= theta), counts.
__global__ void vote_count_kernel(const uint32_t* __restrict__ selbits, int L, int P, int N, int theta,
                                  uint32_t* __restrict__ golden, uint8_t* __restrict__ counts) {
  const int Nw = (N + 31) / 32;
  const int p = blockIdx.y;
  const int w = blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= Nw) return;
  uint8_t cnt[32];
#pragma unroll
  for (int b = 0; b < 32; ++b) cnt[b] = 0;
  for (int l = 0; l < L; ++l) {
    const uint32_t bits = selbits[(static_cast<size_t>(l) * P + p) * Nw + w];
#pragma unroll
    for (int b = 0; b < 32; ++b) cnt[b] += (bits >> b) & 1u;
  }
  uint32_t g = 0;
#pragma unroll
  for (int b = 0; b < 32; ++b) g |= static_cast<uint32_t>(cnt[b] >= theta) << b;
  if (w * 32 + 32 > N) g &= (N - w * 32 >= 32) ? 0xffffffffu : ((1u << (N - w * 32)) - 1u);
  golden[static_cast<size_t>(p) * Nw + w] = g;
  if (counts) {
    uint8_t* c = counts + static_cast<size_t>(p) * N + static_cast<size_t>(w) * 32;
    for (int b = 0; b < 32 && w * 32 + b < N; ++b) c[b] = cnt[b];
  }
}

// Sums of the BCE and focal terms over all P*N entries (fp64), then means.
__global__ void vote_loss_kernel(const float* __restrict__ scores, const uint32_t* __restrict__ golden, int P,
                                 int N, float gamma, double* __restrict__ acc) {
  __shared__ double tmp[2][32];
  const int Nw = (N + 31) / 32;
  const size_t total = static_cast<size_t>(P) * N;
  const double eps = 1.0 / 1048576.0;   // 2^-20: probabilities clamped to [eps, 1 - eps]
  double bce = 0.0, fl = 0.0;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t p = i / N, s = i - p * N;
    const bool y = (golden[p * Nw + (s >> 5)] >> (s & 31)) & 1u;
    double pr = static_cast<double>(scores[i]);
    pr = pr < eps ? eps : (pr > 1.0 - eps ? 1.0 - eps : pr);
    if (y) {
      const double lp = log(pr);
      bce -= lp;
      fl -= pow(1.0 - pr, static_cast<double>(gamma)) * lp;
    } else {
      const double lq = log1p(-pr);
      bce -= lq;
      fl -= pow(pr, static_cast<double>(gamma)) * lq;
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    bce += __shfl_xor_sync(0xffffffffu, bce, o);
    fl += __shfl_xor_sync(0xffffffffu, fl, o);
  }
  if (lane == 0) { tmp[0][warp] = bce; tmp[1][warp] = fl; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) { a += tmp[0][w]; b += tmp[1][w]; }
    atomicAdd(&acc[0], a);
    atomicAdd(&acc[1], b);
  }
}

__global__ void vote_loss_finalize(const double* __restrict__ acc, double n, double* __restrict__ loss) {
  loss[0] = acc[0] / n;
  loss[1] = acc[1] / n;
}

}  // namespace

int launch_vote(const VoteArgs& a, cudaStream_t st) {
  const int rows = a.L * a.P;
  const int Nw = (a.N + 31) / 32;
  int rc = LSA_OK;
  if (rows > 0) {
    const size_t smem = static_cast<size_t>(kRowWarps) * kBins * (sizeof(double) + sizeof(int));
    cudaFuncSetAttribute(vote_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(rows, 2 * sms);
    vote_rows_kernel<<<grid, kRowThreads, smem, st>>>(a.logits, rows, a.N, a.top_p, a.selbits,
                                                      reinterpret_cast<int2*>(a.rowparam));
    if ((rc = check_launch("vote_labels/rows")) != LSA_OK) return rc;
  }
  vote_count_kernel<<<dim3((Nw + 255) / 256, a.P), 256, 0, st>>>(a.selbits, a.L, a.P, a.N, a.theta, a.golden,
                                                                 a.counts);
  if ((rc = check_launch("vote_labels/count")) != LSA_OK) return rc;
  if (a.scores) {
    cudaMemsetAsync(a.lossacc, 0, 2 * sizeof(double), st);
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    vote_loss_kernel<<<2 * sms, 256, 0, st>>>(a.scores, a.golden, a.P, a.N, a.gamma, a.lossacc);
    vote_loss_finalize<<<1, 1, 0, st>>>(a.lossacc, static_cast<double>(a.P) * a.N, a.loss);
    if ((rc = check_launch("vote_labels/loss", 2)) != LSA_OK) return rc;
  }
  return LSA_OK;
}

}  // namespace lsa
