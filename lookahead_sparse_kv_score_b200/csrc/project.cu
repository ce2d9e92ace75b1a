// Low-rank indexer query: c = h W_down, q = c W_up, w = h W_w.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.1 "memory indexer":
// the hidden state h_t is mapped to a low-rank indexer query; §2.3: only these
// low-rank query projections are trained.  For bf16 models c and q are rounded to
// bf16 (nearest even) from an fp32 sum; w stays fp32.
//
// These are skinny products (B <= a few dozen rows against weight matrices of
// millions of elements), bound by the weight bytes.  Each block owns 64 output
// columns and a 256-long slice of the reduction dimension for up to 32 rows at a
// time; the slices are summed in a fixed order by a second kernel, so results do not
// depend on scheduling.
#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int kCols = 64;      // output columns per block
constexpr int kGroups = 4;     // reduction-dimension groups per block (256 threads)
constexpr int kSplit = 256;    // reduction slice per block
constexpr int kRows = 32;      // rows (sequences) per pass
constexpr int kXStride = 36;   // padded row of the staged X slice (floats)

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// part[s][li][b][m] = sum_{k in slice s} X[li][b][k] * W[l0+li][k][m]
template <typename XT, typename WT>
__global__ void __launch_bounds__(256)
skinny_partial(const XT* __restrict__ X, const WT* __restrict__ W, int B, int K, int M, int l0,
               float* __restrict__ part) {
  __shared__ __align__(16) float xs[kSplit * kXStride];
  const int tid = threadIdx.x;
  const int c = tid % kCols, g = tid / kCols;
  const int m = blockIdx.x * kCols + c;
  const int s = blockIdx.y, li = blockIdx.z, nL = gridDim.z;
  const int k0 = s * kSplit, kn = min(kSplit, K - k0);
  const XT* Xl = X + static_cast<size_t>(li) * B * K;
  const WT* Wl = W + static_cast<size_t>(l0 + li) * K * M;
  for (int b0 = 0; b0 < B; b0 += kRows) {
    const int nb = min(kRows, B - b0);
    __syncthreads();
    for (int i = tid; i < kSplit * kRows; i += 256) {
      const int kk = i % kSplit, bb = i / kSplit;
      float v = 0.f;
      if (kk < kn && bb < nb) v = to_f(Xl[static_cast<size_t>(b0 + bb) * K + k0 + kk]);
      xs[kk * kXStride + bb] = v;
    }
    __syncthreads();
    float acc[kRows];
#pragma unroll
    for (int bb = 0; bb < kRows; ++bb) acc[bb] = 0.f;
    if (m < M) {
      for (int kk = g; kk < kn; kk += kGroups) {
        const float wv = to_f(Wl[static_cast<size_t>(k0 + kk) * M + m]);
        const float4* xr = reinterpret_cast<const float4*>(xs + kk * kXStride);
#pragma unroll
        for (int j = 0; j < kRows / 4; ++j) {
          const float4 x4 = xr[j];
          acc[4 * j + 0] = fmaf(x4.x, wv, acc[4 * j + 0]);
          acc[4 * j + 1] = fmaf(x4.y, wv, acc[4 * j + 1]);
          acc[4 * j + 2] = fmaf(x4.z, wv, acc[4 * j + 2]);
          acc[4 * j + 3] = fmaf(x4.w, wv, acc[4 * j + 3]);
        }
      }
    }
    __syncthreads();
    float* red = xs;   // [kGroups][kRows][kCols]
#pragma unroll
    for (int bb = 0; bb < kRows; ++bb) red[(g * kRows + bb) * kCols + c] = acc[bb];
    __syncthreads();
    for (int i = tid; i < kRows * kCols; i += 256) {
      const int bb = i / kCols, cc = i % kCols;
      const int mm = blockIdx.x * kCols + cc;
      if (bb < nb && mm < M) {
        float v = 0.f;
        for (int gg = 0; gg < kGroups; ++gg) v += red[(gg * kRows + bb) * kCols + cc];
        part[((static_cast<size_t>(s) * nL + li) * B + b0 + bb) * M + mm] = v;
      }
    }
  }
}

// out[i] = sum_s part[s][i] (fixed order), optionally rounded to bf16; written as
// float to outf (if any) and as the storage type to out1 / out2 (if any).
template <typename OT>
__global__ void reduce_splits(const float* __restrict__ part, int S, size_t n, int round_bf16,
                              float* __restrict__ outf, OT* __restrict__ out1, OT* __restrict__ out2) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < S; ++s) v += part[s * n + i];
    if (round_bf16) v = __bfloat162float(__float2bfloat16_rn(v));
    if (outf) outf[i] = v;
    OT o;
    if constexpr (sizeof(OT) == 2) o = __float2bfloat16_rn(v); else o = v;
    if (out1) out1[i] = o;
    if (out2) out2[i] = o;
  }
}

template <typename WT>
int project_typed(const ProjectArgs& a, cudaStream_t st) {
  const WT* h = static_cast<const WT*>(a.h) + static_cast<size_t>(a.l0) * a.B * a.D;
  const int SA = project_splits(a.D), SB = project_splits(a.r);
  const int rb = a.wdt == LSA_BF16;
  const size_t HD = static_cast<size_t>(a.H) * a.dI;
  if (a.do_w) {   // w = h W_w
    skinny_partial<WT, WT><<<dim3((a.H + kCols - 1) / kCols, SA, a.nL), 256, 0, st>>>(
        h, static_cast<const WT*>(a.W_w), a.B, a.D, a.H, a.l0, a.partW);
    const size_t nw = static_cast<size_t>(a.nL) * a.B * a.H;
    const size_t woff = static_cast<size_t>(a.l0) * a.B * a.H;
    reduce_splits<float><<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(
        a.partW, SA, nw, 0, a.w_ws + woff, a.w_out ? a.w_out + woff : nullptr, nullptr);
  }
  if (!a.do_q) return check_launch("project", a.do_w ? 2 : 0);
  // c = h W_down (rounded to bf16 for bf16 models)
  skinny_partial<WT, WT><<<dim3((a.r + kCols - 1) / kCols, SA, a.nL), 256, 0, st>>>(
      h, static_cast<const WT*>(a.W_down), a.B, a.D, a.r, a.l0, a.partA);
  const size_t nc = static_cast<size_t>(a.nL) * a.B * a.r;
  reduce_splits<float><<<(unsigned)((nc + 255) / 256), 256, 0, st>>>(a.partA, SA, nc, rb, a.cbuf, nullptr, nullptr);
  // q = c W_up in the storage type
  skinny_partial<float, WT><<<dim3((unsigned)((HD + kCols - 1) / kCols), SB, a.nL), 256, 0, st>>>(
      a.cbuf, static_cast<const WT*>(a.W_up), a.B, a.r, static_cast<int>(HD), a.l0, a.partB);
  const size_t nq = static_cast<size_t>(a.nL) * a.B * HD;
  const size_t qoff = static_cast<size_t>(a.l0) * a.B * HD;
  unsigned gq = (unsigned)std::min<size_t>((nq + 255) / 256, 148 * 16);
  reduce_splits<WT><<<gq, 256, 0, st>>>(a.partB, SB, nq, rb, nullptr,
                                        static_cast<WT*>(a.q_ws) + qoff,
                                        a.q_out ? static_cast<WT*>(a.q_out) + qoff : nullptr);
  return check_launch("project", (a.do_w ? 2 : 0) + 4);
}

}  // namespace

int project_splits(int K) { return (K + kSplit - 1) / kSplit; }

int launch_project(const ProjectArgs& a, cudaStream_t s) {
  if (a.wdt == LSA_BF16) return project_typed<__nv_bfloat16>(a, s);
  return project_typed<float>(a, s);
}

}  // namespace lsa
