// Low-rank indexer query on the tensor cores (bf16 weights): c = h W_down, w = h W_w,
// q = c W_up.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.1 "memory indexer" and
// §2.3 (the low-rank query projections are what the indexer trains).  These are skinny
// products: a few dozen rows X [B][K] against weights W [K][M] of millions of elements,
// so the weight bytes bound them; a CUDA-core version is bound by its own fp32 FMA rate
// first.  Here each CTA computes Y^T = W^T X^T for 128 output features of one layer and
// one reduction slice with tcgen05.mma (kind::f16, bf16 operands, fp32 accumulator in
// TMEM): A = W^T, read straight from the row-major weights as an MN-major operand (TMA
// boxes of 64 features x 64 reduction rows, 128-byte swizzle), B = X^T, K-major (boxes of
// 64 reduction elements x all rows, rows past B zero-filled).  Warp 0 loads through a
// 4-stage ring, warp 1 issues the MMAs, all four warps drain the accumulator: fp32
// partial sums per slice, or for a single slice the bf16-rounded result itself.
#include <cuda.h>

#include <algorithm>

#include "lsa_common.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int kPM = 128;           // output features per CTA (MMA M)
constexpr int kPK = 64;            // reduction elements per stage (128 bytes of bf16)
constexpr int kPStages = 4;
constexpr int kPThreads = 128;
constexpr int kPSlice = 512;       // reduction elements per CTA
constexpr int kABoxBytes = kPK * 64 * 2;          // one 64-feature half of the A tile (8 KB)
constexpr int kABytes = 2 * kABoxBytes;           // A tile of a stage (16 KB)

struct PjParams {
  int B, K, l0, nL;
  int M1, M2, nb1;        // features of the first / second weight; CTAs of the first
  int npad, slices;       // MMA N (rows padded to 16) and reduction slices
  int round_bf16;         // no partial buffer: round the result to bf16
  float* part1;           // [slices][nL][B][M1] fp32 partial sums, or null
  float* part2;           // [slices][nL][B][M2] fp32, or null
  __nv_bfloat16* out1a;   // with part1 null (single slice): [nL][B][M1] bf16 outputs
  __nv_bfloat16* out1b;
  int32_t* status;
};

// MN-major operand, 128-byte swizzle: 64-feature atoms of 8 reduction rows (1024 bytes,
// stride byte offset between the 8-row groups), the second 64-feature half kABoxBytes
// further (leading byte offset).
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(kABoxBytes >> 4) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// K-major operand, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// fp32 accumulate, bf16 A (MN-major) and B (K-major), M = 128, N = n.
__host__ __device__ constexpr uint32_t pj_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kPM >> 4) << 24);
}

// Bounded wait that ends only on completion or on the time limit.
__device__ __forceinline__ bool wait_timed(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// grid: (nb1 + nb2 feature blocks, slices, nL layers).  Maps: W1/W2 3-D (M, K, L) with
// 64 x 64 boxes; X 3-D (K, B, nL) with 64 x npad boxes.
__global__ void __launch_bounds__(kPThreads, 1)
proj_tc_kernel(const __grid_constant__ CUtensorMap mapW1, const __grid_constant__ CUtensorMap mapW2,
               const __grid_constant__ CUtensorMap mapX, const PjParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  const int xbytes = p.npad * 128;
  const int stage_bytes = kABytes + xbytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kPStages * stage_bytes);
  uint64_t* empty = full + kPStages;
  uint64_t* accum = empty + kPStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool second = static_cast<int>(blockIdx.x) >= p.nb1;
  const CUtensorMap* mapW = second ? &mapW2 : &mapW1;
  const int M = second ? p.M2 : p.M1;
  const int m0 = (second ? blockIdx.x - p.nb1 : blockIdx.x) * kPM;
  const int s = blockIdx.y, li = blockIdx.z;
  const int k0 = s * kPSlice, kn = min(kPSlice, p.K - k0);
  const int nst = (kn + kPK - 1) / kPK;
  uint32_t ncols = 32;
  while (static_cast<int>(ncols) < p.npad) ncols <<= 1;
  if (tid == 0) {
    for (int i = 0; i < kPStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(accum, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0 && lane == 0) {
    // producer: stage st holds reduction rows k0 + st*64 .. +63
    const uint64_t pol = evict_first_policy();
    int issued = 0;
    for (int st = 0; st < nst; ++st) {
      const int slot = st % kPStages;
      if (st >= kPStages && !mbar_wait(&empty[slot], ((st / kPStages) - 1) & 1, abort_flag)) break;
      uint8_t* base = sm + slot * stage_bytes;
      mbar_expect_tx(&full[slot], static_cast<uint32_t>(stage_bytes));
      const int kc = k0 + st * kPK;
      tma_load_3d(base, mapW, m0, kc, p.l0 + li, &full[slot], pol);
      tma_load_3d(base + kABoxBytes, mapW, m0 + 64, kc, p.l0 + li, &full[slot], pol);
      tma_load_3d(base + kABytes, &mapX, kc, 0, li, &full[slot], pol);
      issued = st + 1;
    }
    // before leaving, every copy issued must have landed (bounded)
    for (int st = (issued > kPStages ? issued - kPStages : 0); st < issued; ++st)
      mbar_wait(&full[st % kPStages], (st / kPStages) & 1, abort_flag);
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    const uint32_t idesc = pj_idesc(p.npad);
    for (int st = 0; st < nst; ++st) {
      const int slot = st % kPStages;
      if (!mbar_wait(&full[slot], (st / kPStages) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(sm + slot * stage_bytes), x0 = a0 + kABytes;
#pragma unroll
      for (int ks = 0; ks < kPK / 16; ++ks)
        mma<false>(tmem, desc_mn(a0 + ks * 2048), desc_k(x0 + ks * 32), idesc, (st > 0 || ks > 0) ? 1u : 0u);
      mma_commit(&empty[slot]);
    }
    // also after an abort: the commit arrives once the MMAs already issued are done
    mma_commit(accum);
  }
  __syncwarp();
  // epilogue: thread t holds accumulator lane t = feature m0 + t.  The wait ends on the
  // commit (or the time limit), not on the abort flag, so no MMA is in flight below.
  const bool got = wait_timed(accum, 0) && !*abort_flag;
  tc_fence_after();
  if (got) {
    const int m = m0 + tid;
    for (int c0 = 0; c0 < p.B; c0 += 32) {
      float v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0), v);
      if (m < M) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int b = c0 + j;
          if (b >= p.B) break;
          const size_t row = static_cast<size_t>(li) * p.B + b;
          float* part = second ? p.part2 : p.part1;
          if (part) {
            part[(static_cast<size_t>(s) * p.nL * p.B + row) * M + m] = v[j];
          } else {
            const float r = p.round_bf16 ? __bfloat162float(__float2bfloat16_rn(v[j])) : v[j];
            const __nv_bfloat16 o = __float2bfloat16_rn(r);
            if (p.out1a) p.out1a[row * M + m] = o;
            if (p.out1b) p.out1b[row * M + m] = o;
          }
        }
      }
    }
  } else if (tid == 0) {
    raise_status(p.status, LSA_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

int encode(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0, uint32_t b1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(LSA_ERR_CUDA, "project_tc: cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LSA_OK : fail(LSA_ERR_CUDA, "project_tc: tensor map encode failed (%d)", (int)r);
}

int pj_smem(int npad) { return kPStages * (kABytes + npad * 128) + 64 + 1024; }

// One launch of proj_tc_kernel over X [nL][B][K] and the weights of layers l0 .. l0+nL-1.
int launch_pj(const void* X, int B, int K, int L, int l0, int nL, const void* W1, int M1, const void* W2, int M2,
              float* part1, float* part2, __nv_bfloat16* out1a, __nv_bfloat16* out1b, int round_bf16,
              int32_t* status, cudaStream_t st) {
  CUtensorMap m1, m2, mx;
  const int npad = std::max(16, (B + 15) / 16 * 16);
  int rc;
  if ((rc = encode(&m1, W1, M1, K, L, 64, kPK)) != LSA_OK) return rc;
  if ((rc = encode(&m2, W2 ? W2 : W1, W2 ? M2 : M1, K, L, 64, kPK)) != LSA_OK) return rc;
  if ((rc = encode(&mx, X, K, B, nL, kPK, npad)) != LSA_OK) return rc;
  PjParams p{};
  p.B = B; p.K = K; p.l0 = l0; p.nL = nL;
  p.M1 = M1; p.M2 = W2 ? M2 : 0; p.nb1 = (M1 + kPM - 1) / kPM;
  p.npad = npad; p.slices = (K + kPSlice - 1) / kPSlice;
  p.round_bf16 = round_bf16;
  p.part1 = part1; p.part2 = part2; p.out1a = out1a; p.out1b = out1b; p.status = status;
  const int nb2 = W2 ? (M2 + kPM - 1) / kPM : 0;
  const int smem = pj_smem(npad);
  cudaFuncSetAttribute(proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  launch_dependent(proj_tc_kernel, dim3(p.nb1 + nb2, p.slices, nL), dim3(kPThreads), smem, st, m1, m2, mx, p);
  return check_launch("project_tc");
}

}  // namespace

bool project_tc_supported(const ProjectArgs& a) {
  return a.wdt == LSA_BF16 && a.B >= 1 && a.B <= 256 && a.D % 8 == 0 && a.r % 8 == 0 && a.H % 8 == 0 &&
         (static_cast<size_t>(a.H) * a.dI) % 8 == 0 && pj_smem(std::max(16, (a.B + 15) / 16 * 16)) <= 227 * 1024;
}

int project_tc_slices(int K) { return (K + kPSlice - 1) / kPSlice; }

// Stage A: partial sums of c = h W_down and w = h W_w over D-slices, then their fixed-order
// sums (c rounded to bf16, stored as bf16 for stage B; w fp32).  Stage B: q = c W_up in
// one slice (K = r <= 512) written rounded, or in slices with a final reduction.
int launch_project_tc(const ProjectArgs& a, const ProjectTcBufs& t, cudaStream_t st) {
  const __nv_bfloat16* h = static_cast<const __nv_bfloat16*>(a.h) + static_cast<size_t>(a.l0) * a.B * a.D;
  const size_t HD = static_cast<size_t>(a.H) * a.dI;
  const int SA = project_tc_slices(a.D);
  int rc = launch_pj(h, a.B, a.D, a.L, a.l0, a.nL, a.do_q ? a.W_down : a.W_w, a.do_q ? a.r : a.H,
                     (a.do_q && a.do_w) ? a.W_w : nullptr, a.H, a.do_q ? a.partA : a.partW,
                     (a.do_q && a.do_w) ? a.partW : nullptr, nullptr, nullptr, 0, a.status, st);
  if (rc != LSA_OK) return rc;
  if ((rc = launch_project_reductions(a, SA, t, st)) != LSA_OK) return rc;
  if (!a.do_q) return LSA_OK;
  const int SB = project_tc_slices(a.r);
  __nv_bfloat16* q1 = static_cast<__nv_bfloat16*>(a.q_ws) + static_cast<size_t>(a.l0) * a.B * HD;
  __nv_bfloat16* q2 = a.q_out ? static_cast<__nv_bfloat16*>(a.q_out) + static_cast<size_t>(a.l0) * a.B * HD : nullptr;
  if (SB == 1)
    return launch_pj(t.c_bf16, a.B, a.r, a.L, a.l0, a.nL, a.W_up, static_cast<int>(HD), nullptr, 0, nullptr, nullptr,
                     q1, q2, 1, a.status, st);
  rc = launch_pj(t.c_bf16, a.B, a.r, a.L, a.l0, a.nL, a.W_up, static_cast<int>(HD), nullptr, 0, a.partB, nullptr,
                 nullptr, nullptr, 0, a.status, st);
  if (rc != LSA_OK) return rc;
  return launch_project_q_reduction(a, SB, st);
}

}  // namespace lsa
