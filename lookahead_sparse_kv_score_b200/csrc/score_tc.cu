// Tensor-core path of the head-fused gated score on sm_100a: TMA -> shared memory ->
// tcgen05.mma -> tensor memory -> fused epilogue.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.1 "scoring" and
// "dynamic fetch": z_s = kscale_s * sum_h w_h * ReLU(q_h . khat_s) + b; an entry is
// fetched iff sigmoid(z_s) >= 0.5, i.e. z_s >= 0.
//
// Shape of the contraction.  The entries are the MMA's M dimension: one tile is 128
// compressed keys (rows of K_IComp), the B operand is the (sequence, layer) query with
// the H heads as N, and the head dimension dI is the reduction.  The accumulator
// D[128 entries][H heads] lands in tensor memory with one entry per TMEM lane, so each
// epilogue thread owns one entry: it loads its H dot products, applies ReLU, the head
// weights, the per-entry scale and the bias, and the warp's 32 threshold bits become
// one mask word through a ballot.  Scores never go back to HBM unless asked for.
//
// fp8 keys.  tcgen05 kind::f8f6f4 needs both operands in 8-bit formats, while the
// query is bf16.  Each head row q_h is scaled by a power of two s_h (exact) so that
// max |q_h / s_h| <= 448, then split as hi = e4m3(q/s), lo = e4m3(q/s - hi).  A bf16
// value has 8 significant bits and the residual after a 4-bit e4m3 rounding has at
// most 4, so hi + lo reproduces q/s exactly unless lo falls below the e4m3 subnormal
// range (|q| < 2^-10 s_h).  The MMA runs the key tile against hi and then against lo
// into the same accumulator, and s_h > 0 folds into the head weight:
// w_h ReLU(s_h x) = (w_h s_h) ReLU(x).
//
// Pipeline (one persistent CTA per SM, 6 warps):
//   warp 0       TMA producer: key tiles into an S-stage ring, query images into two
//                slots (one per (sequence, layer) change).
//   warp 1       TMEM allocation and the single-thread MMA issuer; two accumulators
//                so the epilogue of tile i overlaps the MMA of tile i+1.
//   warps 2..5   epilogue, one per TMEM lane quadrant (warp id mod 4).
// Every mbarrier wait is bounded by a time limit; on expiry the kernel records
// LSA_ERR_TIMEOUT in the status word, drains what it issued and frees its TMEM.
#include <cuda.h>

#include <algorithm>

#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int kTileM = 128;
constexpr int kThreads = 192;
constexpr int kSmemLimit = 227 * 1024;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: true when the phase completed; false (and the abort flag raised) when
// the time limit passed or another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u) {
      if (*abort_flag) return false;
      if (global_timer() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

template <bool kFp8>
__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                    uint32_t accumulate) {
  const uint32_t z = 0;
  if constexpr (kFp8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z));
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z));
  }
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, 8-row core
// groups 1024 bytes apart (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);         // start address
  d |= static_cast<uint64_t>(1u) << 16;                         // leading byte offset (unused for SW128 K-major)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                 // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;                         // version
  d |= static_cast<uint64_t>(2u) << 61;                         // SWIZZLE_128B
  return d;
}

// Instruction descriptor: fp32 accumulate, K-major A and B, M = 128, N = n.
__host__ __device__ constexpr uint32_t instr_desc(bool fp8, int n) {
  return (1u << 4)                                   // D format F32
         | ((fp8 ? 0u : 1u) << 7)                    // A format: E4M3 (f8f6f4) or BF16 (f16)
         | ((fp8 ? 0u : 1u) << 10)                   // B format
         | (static_cast<uint32_t>(n >> 3) << 17)     // N >> 3
         | (static_cast<uint32_t>(kTileM >> 4) << 24);   // M >> 4
}

// ------------------------------------------------------------------ layout constants
struct TcLayout {
  int chunks;       // 128-byte K chunks of one key row
  int a_bytes;      // one key tile (128 rows)
  int img_bytes;    // one query image (hi+lo for fp8)
  int ksteps;       // MMA instructions per tile
  int stages;       // key-tile ring depth
  int tmem_cols;    // allocated TMEM columns (2 accumulators)
  size_t smem;      // dynamic shared memory
};

__host__ __device__ inline TcLayout tc_layout(int H, int dI, bool fp8) {
  TcLayout t{};
  const int row_bytes = fp8 ? dI : 2 * dI;
  t.chunks = row_bytes / 128;
  t.a_bytes = kTileM * row_bytes;
  t.img_bytes = (fp8 ? 2 : 1) * H * row_bytes;
  t.ksteps = (fp8 ? 2 : 1) * row_bytes / 32;
  int cols = 32;
  while (cols < 2 * H) cols *= 2;
  t.tmem_cols = cols;
  const int fixed = 2 * t.img_bytes + 2 * H * 4 + 1024 /*barriers*/ + 1024 /*alignment*/;
  int s = (kSmemLimit - fixed) / t.a_bytes;
  t.stages = s > 8 ? 8 : s;
  t.smem = static_cast<size_t>(t.stages) * t.a_bytes + fixed;
  return t;
}

struct TcParams {
  int B, N, H, dI, l0, nUnits, tiles_per_unit;
  const uint8_t* qimg;     // [L][B][img_bytes]
  const float* wfold;      // [L][B][H]
  const float* bias;       // [L]
  const float* kscale;     // [L][B][N] or null
  uint32_t* mask;          // [L][B][Nw]
  float* logit;            // [L][B][N] or null
  float* score;            // [L][B][N] or null
  int32_t* status;         // device status word or null
};

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const TcLayout lay = tc_layout(p.H, p.dI, kFp8);
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_ring = smem;                                                   // [stages][a_bytes]
  uint8_t* q_slot = a_ring + static_cast<size_t>(lay.stages) * lay.a_bytes;  // [2][img_bytes]
  float* wf_slot = reinterpret_cast<float*>(q_slot + 2 * lay.img_bytes);     // [2][H]
  uint64_t* bars = reinterpret_cast<uint64_t*>(wf_slot + 2 * p.H);
  uint64_t* full = bars;                    // [8]
  uint64_t* empty = bars + 8;               // [8]
  uint64_t* qfull = bars + 16;              // [2]
  uint64_t* qempty = bars + 18;             // [2]
  uint64_t* tfull = bars + 20;              // [2]
  uint64_t* tempty = bars + 22;             // [2]
  uint64_t* drain = bars + 24;              // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 26);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 27);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < lay.stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 1 + 4);     // MMA commit + four epilogue warps
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], 4);         // four epilogue warps
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, lay.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long T = static_cast<long long>(p.nUnits) * p.tiles_per_unit;
  const long long t_begin = T * blockIdx.x / gridDim.x, t_end = T * (blockIdx.x + 1) / gridDim.x;
  const int Nw = (p.N + 31) / 32;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- producer
    const uint64_t policy = evict_first_policy();
    long long cur = -1;
    int k = -1;
    long long issued = 0;
    for (long long t = t_begin; t < t_end; ++t, ++issued) {
      const long long unit = t / p.tiles_per_unit;
      const int n0 = static_cast<int>(t - unit * p.tiles_per_unit) * kTileM;
      const int uabs = p.l0 * p.B + static_cast<int>(unit);
      if (unit != cur) {
        cur = unit;
        ++k;
        const int slot = k & 1;
        if (!mbar_wait(&qempty[slot], ((k >> 1) & 1) ^ 1, abort_flag)) break;
        mbar_expect_tx(&qfull[slot], lay.img_bytes + p.H * 4);
        bulk_load(q_slot + slot * lay.img_bytes, p.qimg + static_cast<size_t>(uabs) * lay.img_bytes,
                  lay.img_bytes, &qfull[slot]);
        bulk_load(wf_slot + slot * p.H, p.wfold + static_cast<size_t>(uabs) * p.H, p.H * 4, &qfull[slot]);
      }
      const int s = static_cast<int>(issued % lay.stages);
      if (!mbar_wait(&empty[s], ((issued / lay.stages) & 1) ^ 1, abort_flag)) break;
      mbar_expect_tx(&full[s], lay.a_bytes);
      uint8_t* dst = a_ring + static_cast<size_t>(s) * lay.a_bytes;
      for (int c = 0; c < lay.chunks; ++c)
        tma_load_3d(dst + c * (kTileM * 128), &kmap, c * (kFp8 ? 128 : 64), n0, uabs, &full[s], policy);
    }
    // drain: every key tile this thread issued has landed before the CTA exits
    for (long long j = std::max(0ll, issued - lay.stages); j < issued; ++j) {
      const int s = static_cast<int>(j % lay.stages);
      volatile int no_abort = 0;
      if (!mbar_wait(&full[s], (j / lay.stages) & 1, &no_abort)) break;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = instr_desc(kFp8, p.H);
    long long cur = -1;
    int k = -1, slot = 0;
    long long i = 0;
    bool ok = true;
    for (long long t = t_begin; t < t_end && ok; ++t, ++i) {
      const long long unit = t / p.tiles_per_unit;
      if (unit != cur) {
        if (cur != -1) mma_commit(&qempty[slot]);
        cur = unit;
        ++k;
        slot = k & 1;
        if (!(ok = mbar_wait(&qfull[slot], (k >> 1) & 1, abort_flag))) break;
      }
      const int acc = static_cast<int>(i & 1);
      if (!(ok = mbar_wait(&tempty[acc], ((i >> 1) & 1) ^ 1, abort_flag))) break;
      tc_fence_after();
      const int s = static_cast<int>(i % lay.stages);
      if (!(ok = mbar_wait(&full[s], (i / lay.stages) & 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t a_base = smem_u32(a_ring + static_cast<size_t>(s) * lay.a_bytes);
      const uint32_t b_base = smem_u32(q_slot + slot * lay.img_bytes);
      const uint32_t d_tmem = tmem_base + acc * p.H;
      const int steps_per_pass = lay.chunks * 4;     // 32-byte K steps over one key row
      for (int ks = 0; ks < lay.ksteps; ++ks) {
        const int ka = ks % steps_per_pass;           // fp8: second pass re-reads the same key tile
        const uint32_t a_addr = a_base + (ka >> 2) * (kTileM * 128) + (ka & 3) * 32;
        const uint32_t b_addr = b_base + (ks >> 2) * (p.H * 128) + (ks & 3) * 32;
        mma<kFp8>(d_tmem, smem_desc(a_addr), smem_desc(b_addr), idesc, ks > 0 ? 1u : 0u);
      }
      mma_commit(&empty[s]);
      mma_commit(&tfull[acc]);
    }
    if (cur != -1 && ok) mma_commit(&qempty[slot]);
    // drain: all MMAs issued by this thread have completed
    mma_commit(drain);
    volatile int no_abort = 0;
    mbar_wait(drain, 0, &no_abort);
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    long long cur = -1;
    int k = -1, slot = 0;
    float bias_l = 0.f;
    long long i = 0;
    for (long long t = t_begin; t < t_end; ++t, ++i) {
      const long long unit = t / p.tiles_per_unit;
      const int n0 = static_cast<int>(t - unit * p.tiles_per_unit) * kTileM;
      const size_t uabs = static_cast<size_t>(p.l0) * p.B + static_cast<size_t>(unit);
      if (unit != cur) {
        if (cur != -1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&qempty[slot]);
        }
        cur = unit;
        ++k;
        slot = k & 1;
        bias_l = p.bias[p.l0 + static_cast<int>(unit / p.B)];
        if (!__all_sync(0xffffffffu, mbar_wait(&qfull[slot], (k >> 1) & 1, abort_flag))) break;
      }
      const int n = n0 + row;
      const bool valid = n < p.N;
      float ks = 1.f;
      if (kFp8 && valid) ks = p.kscale[uabs * p.N + n];
      const int acc = static_cast<int>(i & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], (i >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      float z = 0.f;
      const float* wf = wf_slot + slot * p.H;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * p.H;
      for (int c0 = 0; c0 < p.H; c0 += 32) {
        float v[32];
        tmem_ld32(taddr + c0, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) z = fmaf(wf[c0 + j], fmaxf(v[j], 0.f), z);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      z = fmaf(z, ks, bias_l);
      if (valid) {
        if (p.logit) p.logit[uabs * p.N + n] = z;
        if (p.score) p.score[uabs * p.N + n] = sigmoid_f(z);
      }
      const unsigned bits = __ballot_sync(0xffffffffu, valid && z >= 0.f);
      const int word = (n0 + quad * 32) >> 5;
      if (lane == 0 && word < Nw) p.mask[uabs * Nw + word] = bits;
    }
    if (cur != -1) {      // warp-uniform: every lane left the loop at the same tile
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[slot]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) raise_status(p.status, LSA_ERR_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, lay.tmem_cols);
  }
}

// ------------------------------------------------------------------ query images
// One block per (layer, sequence).  bf16: the query rows in the 128-byte-swizzled
// K-major layout the MMA reads (16-byte unit j of row h stored at unit j ^ (h % 8)).
// fp8: per-head power-of-two scale, hi and lo e4m3 rows in the same layout, and the
// folded head weights w_h * s_h.
template <bool kFp8>
__global__ void build_qimg_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                                  int B, int H, int dI, int l0, uint8_t* __restrict__ img,
                                  float* __restrict__ wfold) {
  const size_t uabs = static_cast<size_t>(l0) * B + blockIdx.x;
  const __nv_bfloat16* qu = q + uabs * H * dI;
  const int row_bytes = kFp8 ? dI : 2 * dI;
  const int img_bytes = (kFp8 ? 2 : 1) * H * row_bytes;
  uint8_t* out = img + uabs * img_bytes;
  if constexpr (!kFp8) {
    for (int e = threadIdx.x; e < H * dI; e += blockDim.x) {
      const int h = e / dI, d = e % dI;
      const int c = d / 64, j = (d % 64) / 8, x = d % 8;
      const size_t off = static_cast<size_t>(c) * H * 128 + h * 128 + ((j ^ (h & 7)) * 16) + x * 2;
      *reinterpret_cast<__nv_bfloat16*>(out + off) = qu[e];
    }
    for (int h = threadIdx.x; h < H; h += blockDim.x) wfold[uabs * H + h] = w[uabs * H + h];
  } else {
    // one warp per head
    const int lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const size_t lo_base = static_cast<size_t>(H) * dI;
    for (int h = threadIdx.x >> 5; h < H; h += nwarps) {
      float amax = 0.f;
      for (int d = lane; d < dI; d += 32) amax = fmaxf(amax, fabsf(__bfloat162float(qu[h * dI + d])));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      // smallest power of two s with amax <= 448 s
      int e = 0;
      if (amax > 0.f) {
        e = static_cast<int>(ceilf(log2f(amax / 448.f)));
        while (amax > ldexpf(448.f, e)) ++e;
        while (e > -126 && amax <= ldexpf(448.f, e - 1)) --e;
      }
      const float inv = ldexpf(1.f, -e);
      for (int d = lane; d < dI; d += 32) {
        const float x = __bfloat162float(qu[h * dI + d]) * inv;   // exact (power of two)
        const __nv_fp8_e4m3 hi(x);
        const __nv_fp8_e4m3 lo(x - static_cast<float>(hi));
        const int c = d / 128, j = (d % 128) / 16, xx = d % 16;
        const size_t off = static_cast<size_t>(c) * H * 128 + h * 128 + ((j ^ (h & 7)) * 16) + xx;
        out[off] = hi.__x;
        out[lo_base + off] = lo.__x;
      }
      if (lane == 0) wfold[uabs * H + h] = w[uabs * H + h] * ldexpf(1.f, e);
    }
  }
}

// ------------------------------------------------------------------ tensor map
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

bool tc_supported(int H, int dI, int wdt, int kdt) {
  if (wdt != LSA_BF16) return false;
  if (H < 32 || H > 256 || H % 32 != 0) return false;
  const bool fp8 = kdt == LSA_E4M3;
  if (kdt == LSA_BF16) {
    if (dI % 64 != 0 || dI < 64 || dI > 256) return false;
  } else if (fp8) {
    if (dI % 128 != 0 || dI > 256) return false;
  } else {
    return false;
  }
  return tc_layout(H, dI, fp8).stages >= 2;
}

size_t tc_image_bytes(int H, int dI, int kdt) {
  return static_cast<size_t>(tc_layout(H, dI, kdt == LSA_E4M3).img_bytes);
}

int launch_score_tc(const TcArgs& a, cudaStream_t st) {
  const ScoreArgs& s = a.sc;
  if (s.N == 0 || s.B == 0 || s.nL == 0) return LSA_OK;
  const bool fp8 = s.kdt == LSA_E4M3;
  const TcLayout lay = tc_layout(s.H, s.dI, fp8);
  // query images and folded head weights for the processed layers
  if (fp8)
    build_qimg_kernel<true><<<s.B * s.nL, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(s.q), s.w, s.B, s.H,
                                                        s.dI, s.l0, a.qimg, a.wfold);
  else
    build_qimg_kernel<false><<<s.B * s.nL, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(s.q), s.w, s.B,
                                                         s.H, s.dI, s.l0, a.qimg, a.wfold);
  int rc = check_launch("score_tc/query image");
  if (rc != LSA_OK) return rc;

  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(LSA_ERR_CUDA, "score_tc: cuTensorMapEncodeTiled unavailable");
  CUtensorMap map;
  const int esz = fp8 ? 1 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(s.dI), static_cast<cuuint64_t>(s.N),
                              static_cast<cuuint64_t>(s.L) * s.B};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(s.dI) * esz, static_cast<cuuint64_t>(s.N) * s.dI * esz};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(kTileM), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult cr = enc(&map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                          const_cast<void*>(s.K), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return fail(LSA_ERR_CUDA, "score_tc: tensor map encode failed (%d)", (int)cr);

  TcParams p{};
  p.B = s.B; p.N = s.N; p.H = s.H; p.dI = s.dI; p.l0 = s.l0; p.nUnits = s.nL * s.B;
  p.tiles_per_unit = (s.N + kTileM - 1) / kTileM;
  p.qimg = a.qimg; p.wfold = a.wfold; p.bias = s.bias; p.kscale = s.kscale;
  p.mask = s.mask; p.logit = s.logit; p.score = s.score; p.status = a.status;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = static_cast<long long>(p.nUnits) * p.tiles_per_unit;
  const int grid = static_cast<int>(std::min<long long>(sms, tiles));
  if (fp8) {
    cudaFuncSetAttribute(score_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.smem);
    score_tc_kernel<true><<<grid, kThreads, lay.smem, st>>>(map, p);
  } else {
    cudaFuncSetAttribute(score_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.smem);
    score_tc_kernel<false><<<grid, kThreads, lay.smem, st>>>(map, p);
  }
  return check_launch("score_tc");
}

}  // namespace lsa
