// CUDA-core path of the head-fused gated score (fp32 models, and any shape the
// tensor-core path does not take).
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.1 "scoring" and
// "dynamic fetch":  z_s = kscale_s * sum_h w_h * ReLU(q_h . khat_s) + b,  I = sigmoid(z),
// fetched iff I >= 0.5, i.e. z >= 0.
//
// One thread per entry; the (sequence, layer) query and head weights sit in shared
// memory as fp32.  Heads are processed 16 at a time so the key row is re-read from L1
// only H/16 times.
#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 128;
constexpr int kHeadChunk = 16;

template <typename QT>
__device__ __forceinline__ float q_elem(const QT* q, size_t i) { return load_elem(q, i); }

template <typename KT, typename QT>
__global__ void __launch_bounds__(kThreads)
score_simt_kernel(const QT* __restrict__ q, const float* __restrict__ w, const float* __restrict__ bias,
                  const KT* __restrict__ K, const float* __restrict__ kscale,
                  int B, int N, int H, int dI, int l0,
                  uint32_t* __restrict__ mask, float* __restrict__ logit, float* __restrict__ score) {
  extern __shared__ float sm[];
  float* qs = sm;                 // [H][dI]
  float* ws = sm + H * dI;        // [H]
  const int b = blockIdx.y, l = l0 + blockIdx.z;
  const size_t unit = static_cast<size_t>(l) * B + b;
  for (int i = threadIdx.x; i < H * dI; i += kThreads) qs[i] = q_elem(q, unit * H * dI + i);
  for (int i = threadIdx.x; i < H; i += kThreads) ws[i] = w[unit * H + i];
  __syncthreads();

  const int s = blockIdx.x * kThreads + threadIdx.x;
  const bool valid = s < N;
  float z = 0.f;
  if (valid) {
    const KT* kr = K + (unit * N + s) * dI;
    for (int h0 = 0; h0 < H; h0 += kHeadChunk) {
      const int hn = min(kHeadChunk, H - h0);
      float acc[kHeadChunk];
#pragma unroll
      for (int j = 0; j < kHeadChunk; ++j) acc[j] = 0.f;
      for (int d = 0; d < dI; ++d) {
        const float kd = load_elem(kr, d);
#pragma unroll
        for (int j = 0; j < kHeadChunk; ++j)
          if (j < hn) acc[j] = fmaf(qs[(h0 + j) * dI + d], kd, acc[j]);
      }
#pragma unroll
      for (int j = 0; j < kHeadChunk; ++j)
        if (j < hn) z = fmaf(ws[h0 + j], fmaxf(acc[j], 0.f), z);
    }
    if (kscale != nullptr) z *= kscale[unit * N + s];
    z += bias[l];
    if (logit) logit[unit * N + s] = z;
    if (score) score[unit * N + s] = sigmoid_f(z);
  }
  const unsigned bits = __ballot_sync(0xffffffffu, valid && z >= 0.f);
  const int Nw = (N + 31) / 32;
  const int word = s / 32;
  if ((threadIdx.x & 31) == 0 && word < Nw) mask[unit * Nw + word] = bits;
}

template <typename KT>
int launch_k(const ScoreArgs& a, cudaStream_t st) {
  const dim3 grid((a.N + kThreads - 1) / kThreads, a.B, a.nL);
  const size_t smem = (static_cast<size_t>(a.H) * a.dI + a.H) * sizeof(float);
  if (smem > 48 * 1024) {
    if (a.wdt == LSA_BF16)
      cudaFuncSetAttribute(score_simt_kernel<KT, __nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    else
      cudaFuncSetAttribute(score_simt_kernel<KT, float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  }
  if (a.wdt == LSA_BF16)
    score_simt_kernel<KT, __nv_bfloat16><<<grid, kThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(a.q), a.w, a.bias, static_cast<const KT*>(a.K), a.kscale,
        a.B, a.N, a.H, a.dI, a.l0, a.mask, a.logit, a.score);
  else
    score_simt_kernel<KT, float><<<grid, kThreads, smem, st>>>(
        static_cast<const float*>(a.q), a.w, a.bias, static_cast<const KT*>(a.K), a.kscale,
        a.B, a.N, a.H, a.dI, a.l0, a.mask, a.logit, a.score);
  return check_launch("score_simt");
}

// Gathered candidates (the native indexer's fine score): thread j of sequence b scores
// entry e = idx[b][j] for j < min(count[b], cap) and writes score[b][e].
template <typename KT, typename QT>
__global__ void __launch_bounds__(kThreads)
fine_simt_kernel(const QT* __restrict__ q, const float* __restrict__ w, const KT* __restrict__ K,
                 const float* __restrict__ kscale, const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                 int cap, int N, int H, int dI, float* __restrict__ score) {
  extern __shared__ float sm[];
  float* qs = sm;                 // [H][dI]
  float* ws = sm + H * dI;        // [H]
  const int b = blockIdx.y;
  const int n = min(count[b], cap);
  if (static_cast<int>(blockIdx.x) * kThreads >= n) return;
  for (int i = threadIdx.x; i < H * dI; i += kThreads) qs[i] = load_elem(q, static_cast<size_t>(b) * H * dI + i);
  for (int i = threadIdx.x; i < H; i += kThreads) ws[i] = w[static_cast<size_t>(b) * H + i];
  __syncthreads();
  const int j = blockIdx.x * kThreads + threadIdx.x;
  if (j >= n) return;
  const int e = idx[static_cast<size_t>(b) * cap + j];
  if (e < 0 || e >= N) return;
  const KT* kr = K + (static_cast<size_t>(b) * N + e) * dI;
  float z = 0.f;
  for (int h0 = 0; h0 < H; h0 += kHeadChunk) {
    const int hn = min(kHeadChunk, H - h0);
    float acc[kHeadChunk];
#pragma unroll
    for (int t = 0; t < kHeadChunk; ++t) acc[t] = 0.f;
    for (int d = 0; d < dI; ++d) {
      const float kd = load_elem(kr, d);
#pragma unroll
      for (int t = 0; t < kHeadChunk; ++t)
        if (t < hn) acc[t] = fmaf(qs[(h0 + t) * dI + d], kd, acc[t]);
    }
#pragma unroll
    for (int t = 0; t < kHeadChunk; ++t)
      if (t < hn) z = fmaf(ws[h0 + t], fmaxf(acc[t], 0.f), z);
  }
  if (kscale != nullptr) z *= kscale[static_cast<size_t>(b) * N + e];
  score[static_cast<size_t>(b) * N + e] = z;
}

template <typename KT, typename QT>
int launch_fine_k(const FineArgs& a, cudaStream_t st) {
  const dim3 grid((a.cap + kThreads - 1) / kThreads, a.B);
  const size_t smem = (static_cast<size_t>(a.H) * a.dI + a.H) * sizeof(float);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(fine_simt_kernel<KT, QT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  fine_simt_kernel<KT, QT><<<grid, kThreads, smem, st>>>(static_cast<const QT*>(a.q), a.w,
                                                         static_cast<const KT*>(a.K), a.kscale, a.idx, a.count, a.cap,
                                                         a.N, a.H, a.dI, a.score);
  return check_launch("fine_score_simt");
}

template <typename KT>
int launch_fine_q(const FineArgs& a, cudaStream_t st) {
  return a.qdt == LSA_BF16 ? launch_fine_k<KT, __nv_bfloat16>(a, st) : launch_fine_k<KT, float>(a, st);
}

}  // namespace

int launch_fine_score_simt(const FineArgs& a, cudaStream_t s) {
  if (a.N == 0 || a.B == 0 || a.cap == 0) return LSA_OK;
  switch (a.kdt) {
    case LSA_F32: return launch_fine_q<float>(a, s);
    case LSA_BF16: return launch_fine_q<__nv_bfloat16>(a, s);
    case LSA_E4M3: return launch_fine_q<uint8_t>(a, s);
  }
  return fail(LSA_ERR_UNSUPPORTED, "fine_score: key dtype %d", a.kdt);
}

int launch_fine_score(const FineArgs& a, cudaStream_t s) {
  if (a.N == 0 || a.B == 0 || a.cap == 0) return LSA_OK;
  if (tc_supported(a.H, a.dI, a.qdt, a.kdt)) return launch_fine_score_tc(a, s);
  return launch_fine_score_simt(a, s);
}

int launch_score_simt(const ScoreArgs& a, cudaStream_t s) {
  if (a.N == 0 || a.B == 0 || a.nL == 0) return LSA_OK;
  switch (a.kdt) {
    case LSA_F32: return launch_k<float>(a, s);
    case LSA_BF16: return launch_k<__nv_bfloat16>(a, s);
    case LSA_E4M3: return launch_k<uint8_t>(a, s);
  }
  return fail(LSA_ERR_UNSUPPORTED, "score_simt: key dtype %d", a.kdt);
}

}  // namespace lsa
