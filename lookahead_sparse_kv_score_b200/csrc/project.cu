// Low-rank indexer query: c = h W_down, q = c W_up, w = h W_w.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.1 "memory indexer":
// the hidden state h_t is mapped to a low-rank indexer query; §2.3: only these
// low-rank query projections are trained.  For bf16 models c and q are rounded to
// bf16 (nearest even) from an fp32 sum; w stays fp32.
//
// These are skinny products (B rows, a few dozen at most, against weight matrices of
// millions of elements) bound by the weight bytes.  A block owns 32 rows x 256 output
// columns of a slice of the reduction dimension: the weight rows stream through a
// cp.async ring in shared memory, each thread holds a 4-row x 8-column tile in
// registers (packed two-wide fp32 FMAs) and reads the four X values of its rows from a
// staged, transposed X slice.  Slices are summed in a fixed order by a second kernel,
// so the results do not depend on scheduling.
#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int kTileCols = 256;     // output columns per block (32 threads x 8)
constexpr int kTileRows = 32;      // rows per pass (8 row groups x 4)
constexpr int kThreads = 256;
constexpr int kXStride = 36;       // padded row of the transposed X slice (floats)
constexpr int kSliceA = 256;       // reduction slice of h W_down / h W_w
constexpr int kSliceB = 128;       // reduction slice of c W_up

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// acc += x * w for a pair of columns (two fp32 FMAs, round to nearest).
__device__ __forceinline__ void fma2(float2& acc, float x, float2 w) {
  unsigned long long a = *reinterpret_cast<unsigned long long*>(&acc);
  const float2 xx = make_float2(x, x);
  const unsigned long long xb = *reinterpret_cast<const unsigned long long*>(&xx);
  const unsigned long long wb = *reinterpret_cast<const unsigned long long*>(&w);
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a) : "l"(xb), "l"(wb));
  acc = *reinterpret_cast<float2*>(&a);
}

// 16-byte global -> shared copy, zero-filled when `valid` is false (nothing is read).
__device__ __forceinline__ void cp16(void* dst, const void* src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory"); }

__device__ __forceinline__ void unpack8(const __nv_bfloat16* p, float2 (&w)[4]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    w[i] = make_float2(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xFFFF0000u));
}
__device__ __forceinline__ void unpack8(const float* p, float2 (&w)[4]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  w[0] = make_float2(a.x, a.y); w[1] = make_float2(a.z, a.w);
  w[2] = make_float2(b.x, b.y); w[3] = make_float2(b.z, b.w);
}

constexpr int kStageRows = 8;      // weight rows per pipeline stage
constexpr int kStages = 4;         // cp.async ring depth

template <typename WT>
constexpr size_t proj_smem(int slice) {
  return static_cast<size_t>(slice) * kXStride * sizeof(float) +
         static_cast<size_t>(kStages) * kStageRows * kTileCols * sizeof(WT);
}

// part[s][li][b][m] = sum_{k in slice s} X[li][b][k] * W[l0+li][k][m] for the columns of
// W1 (m < M1) and, when blockIdx.x >= nb1, of W2 (written to part2 with M2 columns).
// The weight rows of the slice stream through a kStages-deep cp.async ring of
// kStageRows x 256 columns; X of the block's rows is staged once, transposed.
template <typename XT, typename WT, int kSlice>
__global__ void __launch_bounds__(kThreads)
proj_partial(const XT* __restrict__ X, int B, int K, int l0,
             const WT* __restrict__ W1, int M1, float* __restrict__ part1,
             const WT* __restrict__ W2, int M2, float* __restrict__ part2) {
  extern __shared__ __align__(16) uint8_t psm[];
  float* xs = reinterpret_cast<float*>(psm);                                          // [kSlice][kXStride]
  WT* ring = reinterpret_cast<WT*>(psm + static_cast<size_t>(kSlice) * kXStride * sizeof(float));
  constexpr int kStageElems = kStageRows * kTileCols;                                  // per stage
  constexpr int kVec = 16 / sizeof(WT);                                                // elements per copy
  constexpr int kCopies = kStageElems / kVec / kThreads;                               // copies per thread
  const int nb1 = (M1 + kTileCols - 1) / kTileCols;
  const bool second = static_cast<int>(blockIdx.x) >= nb1;
  const WT* W = second ? W2 : W1;
  const int M = second ? M2 : M1;
  float* part = second ? part2 : part1;
  const int col0 = (second ? blockIdx.x - nb1 : blockIdx.x) * kTileCols;
  const int tid = threadIdx.x, cg = tid & 31, rg = tid >> 5;
  const int m = col0 + cg * 8;
  const int s = blockIdx.y, li = blockIdx.z, nL = gridDim.z;
  const int k0 = s * kSlice, kn = min(kSlice, K - k0);
  const int nstages = (kn + kStageRows - 1) / kStageRows;
  const XT* Xl = X + static_cast<size_t>(li) * B * K;
  const WT* Wl = W + (static_cast<size_t>(l0 + li) * K + k0) * M;
  auto issue = [&](int st) {
    if (st < nstages) {
      WT* dst = ring + (st % kStages) * kStageElems;
#pragma unroll
      for (int c = 0; c < kCopies; ++c) {
        const int e = (c * kThreads + tid) * kVec;                 // element within the stage
        const int kr = e / kTileCols, col = e % kTileCols;
        const int k = st * kStageRows + kr;
        const bool ok = k < kn && col0 + col < M;
        cp16(dst + e, ok ? static_cast<const void*>(Wl + static_cast<size_t>(k) * M + col0 + col) : Wl, ok);
      }
    }
    cp_commit();
  };
  for (int b0 = 0; b0 < B; b0 += kTileRows) {
    const int nb = min(kTileRows, B - b0);
    __syncthreads();
    for (int st = 0; st < kStages - 1; ++st) issue(st);
    for (int i = tid; i < kSlice * kTileRows; i += kThreads) {
      const int kk = i % kSlice, bb = i / kSlice;
      float v = 0.f;
      if (kk < kn && bb < nb) v = to_f(Xl[static_cast<size_t>(b0 + bb) * K + k0 + kk]);
      xs[kk * kXStride + bb] = v;
    }
    const bool active = rg * 4 < nb && m < M;    // warp-uniform in rows; M is a multiple of 8
    float2 acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = make_float2(0.f, 0.f);
    for (int st = 0; st < nstages; ++st) {
      cp_wait<kStages - 2>();
      __syncthreads();
      issue(st + kStages - 1);
      if (active) {
        const WT* wst = ring + (st % kStages) * kStageElems + cg * 8;
#pragma unroll
        for (int kr = 0; kr < kStageRows; ++kr) {
          const int k = st * kStageRows + kr;
          float2 w[4];
          unpack8(wst + kr * kTileCols, w);
          const float4 x = *reinterpret_cast<const float4*>(xs + k * kXStride + rg * 4);
          const float xr[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) fma2(acc[r][c], xr[r], w[c]);
        }
      }
    }
    cp_wait<0>();
    if (active) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int b = b0 + rg * 4 + r;
        if (b - b0 >= nb) break;
        float4* out = reinterpret_cast<float4*>(part + ((static_cast<size_t>(s) * nL + li) * B + b) * M + m);
        out[0] = make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
        out[1] = make_float4(acc[r][2].x, acc[r][2].y, acc[r][3].x, acc[r][3].y);
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

unsigned grid_for(size_t n) { return static_cast<unsigned>(std::min<size_t>((n + 255) / 256, 148 * 16)); }

// The two stage-A reductions of the tensor-core path in one launch: elements [0, nw) are
// the head weights w (fp32 outputs), elements [nw, nw + nc) the elements of c (rounded to
// bf16); each sums its S slices in order.
__global__ void reduce_cw_kernel(const float* __restrict__ partW, size_t nw, float* __restrict__ w1,
                                 float* __restrict__ w2, const float* __restrict__ partA, size_t nc,
                                 __nv_bfloat16* __restrict__ c, int S) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < nw + nc;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    if (i < nw) {
      float v = 0.f;
      for (int s = 0; s < S; ++s) v += partW[s * nw + i];
      w1[i] = v;
      if (w2) w2[i] = v;
    } else {
      const size_t k = i - nw;
      float v = 0.f;
      for (int s = 0; s < S; ++s) v += partA[s * nc + k];
      c[k] = __float2bfloat16_rn(v);
    }
  }
}

template <typename WT>
int project_typed(const ProjectArgs& a, cudaStream_t st) {
  const WT* h = static_cast<const WT*>(a.h) + static_cast<size_t>(a.l0) * a.B * a.D;
  const int SA = project_splits(a.D), SB = project_splits_b(a.r);
  const int rb = a.wdt == LSA_BF16;
  const size_t HD = static_cast<size_t>(a.H) * a.dI;
  int launches = 0;
  // c = h W_down and w = h W_w in one launch (W_w's column blocks after W_down's)
  const int nbd = a.do_q ? (a.r + kTileCols - 1) / kTileCols : 0;
  const int nbw = a.do_w ? (a.H + kTileCols - 1) / kTileCols : 0;
  constexpr size_t smA = proj_smem<WT>(kSliceA), smB = proj_smem<WT>(kSliceB);
  cudaFuncSetAttribute(proj_partial<WT, WT, kSliceA>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smA);
  cudaFuncSetAttribute(proj_partial<float, WT, kSliceB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smB);
  proj_partial<WT, WT, kSliceA><<<dim3(nbd + nbw, SA, a.nL), kThreads, smA, st>>>(
      h, a.B, a.D, a.l0, static_cast<const WT*>(a.W_down), a.do_q ? a.r : 0, a.partA,
      static_cast<const WT*>(a.W_w), a.H, a.partW);
  ++launches;
  if (a.do_w) {
    const size_t nw = static_cast<size_t>(a.nL) * a.B * a.H;
    const size_t woff = static_cast<size_t>(a.l0) * a.B * a.H;
    reduce_splits<float><<<grid_for(nw), 256, 0, st>>>(a.partW, SA, nw, 0, a.w_ws + woff,
                                                        a.w_out ? a.w_out + woff : nullptr, nullptr);
    ++launches;
  }
  if (a.do_q) {
    const size_t nc = static_cast<size_t>(a.nL) * a.B * a.r;
    reduce_splits<float><<<grid_for(nc), 256, 0, st>>>(a.partA, SA, nc, rb, a.cbuf, nullptr, nullptr);
    // q = c W_up in the storage type
    proj_partial<float, WT, kSliceB><<<dim3(static_cast<unsigned>((HD + kTileCols - 1) / kTileCols), SB, a.nL),
                                       kThreads, smB, st>>>(a.cbuf, a.B, a.r, a.l0, static_cast<const WT*>(a.W_up),
                                                          static_cast<int>(HD), a.partB, nullptr, 0, nullptr);
    const size_t nq = static_cast<size_t>(a.nL) * a.B * HD;
    const size_t qoff = static_cast<size_t>(a.l0) * a.B * HD;
    reduce_splits<WT><<<grid_for(nq), 256, 0, st>>>(a.partB, SB, nq, rb, nullptr, static_cast<WT*>(a.q_ws) + qoff,
                                                    a.q_out ? static_cast<WT*>(a.q_out) + qoff : nullptr);
    launches += 3;
  }
  return check_launch("project", launches);
}

}  // namespace

int project_splits(int K) { return (K + kSliceA - 1) / kSliceA; }
int project_splits_b(int K) { return (K + kSliceB - 1) / kSliceB; }

// Fixed-order sums of S slices for the tensor-core path: w (fp32) and c (rounded to bf16,
// stored as bf16 for q = c W_up).
int launch_project_reductions(const ProjectArgs& a, int S, const ProjectTcBufs& t, cudaStream_t st) {
  if (a.do_w && a.do_q) {
    const size_t nw = static_cast<size_t>(a.nL) * a.B * a.H;
    const size_t woff = static_cast<size_t>(a.l0) * a.B * a.H;
    const size_t nc = static_cast<size_t>(a.nL) * a.B * a.r;
    launch_dependent(reduce_cw_kernel, dim3(grid_for(nw + nc)), dim3(256), 0, st, a.partW, nw, a.w_ws + woff,
                     a.w_out ? a.w_out + woff : nullptr, a.partA, nc, t.c_bf16, S);
    return check_launch("project/reduce");
  }
  int launches = 0;
  if (a.do_w) {
    const size_t nw = static_cast<size_t>(a.nL) * a.B * a.H;
    const size_t woff = static_cast<size_t>(a.l0) * a.B * a.H;
    reduce_splits<float><<<grid_for(nw), 256, 0, st>>>(a.partW, S, nw, 0, a.w_ws + woff,
                                                        a.w_out ? a.w_out + woff : nullptr, nullptr);
    ++launches;
  }
  if (a.do_q) {
    const size_t nc = static_cast<size_t>(a.nL) * a.B * a.r;
    reduce_splits<__nv_bfloat16><<<grid_for(nc), 256, 0, st>>>(a.partA, S, nc, 1, nullptr, t.c_bf16, nullptr);
    ++launches;
  }
  return check_launch("project/reduce", launches);
}

int launch_project_q_reduction(const ProjectArgs& a, int S, cudaStream_t st) {
  const size_t HD = static_cast<size_t>(a.H) * a.dI;
  const size_t nq = static_cast<size_t>(a.nL) * a.B * HD;
  const size_t qoff = static_cast<size_t>(a.l0) * a.B * HD;
  reduce_splits<__nv_bfloat16><<<grid_for(nq), 256, 0, st>>>(
      a.partB, S, nq, 1, nullptr, static_cast<__nv_bfloat16*>(a.q_ws) + qoff,
      a.q_out ? static_cast<__nv_bfloat16*>(a.q_out) + qoff : nullptr);
  return check_launch("project/reduce q");
}

int launch_project(const ProjectArgs& a, cudaStream_t s) {
  if ((a.r % 8) != 0 || (a.H % 8) != 0 || ((static_cast<size_t>(a.H) * a.dI) % 8) != 0)
    return fail(LSA_ERR_UNSUPPORTED, "project: r, H and H*dI must be multiples of 8");
  if (a.wdt == LSA_BF16) {
    if (project_tc_supported(a))
      return launch_project_tc(a, ProjectTcBufs{reinterpret_cast<__nv_bfloat16*>(a.cbuf)}, s);
    return project_typed<__nv_bfloat16>(a, s);
  }
  return project_typed<float>(a, s);
}

}  // namespace lsa
