// One indexer training step on the tensor cores: loss and gradients of the query side
// against frozen compressed keys.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.3: K_IComp is frozen,
// only the low-rank query projections are trained, the objective is BCE combined with a
// focal loss; §2.2: the labels are the cross-layer majority-vote bits.  For P query
// positions of one indexer layer:
//   a_phs = q_ph . k_s,  z_ps = sum_h w_ph ReLU(a_phs) + b,  J = mean BCE + mean FL,
//   g_ps = dJ/dz_ps,  U_ph = sum_s g_ps 1[a_phs > 0] k_s,
//   dq_ph = w_ph U_ph,  dw_ph = q_ph . U_ph,  db = sum g,
//   dW_up = c^T dq,  dc = dq W_up^T,  dW_down = h^T dc,  dW_w = h^T dw.
//
// train_tc_kernel fuses the forward scores, the loss terms, g and U.  A CTA owns a group
// of 128 / H positions (128 (position, head) rows) and a chunk of key tiles of 128
// entries.  Per tile: tcgen05.mma A = the key tile (K-major), B = the group's query
// image -> F [entries x (p, h)] in TMEM; the epilogue warps (one thread per entry) read
// F, form z, the loss terms and g, and write G' = g 1[a > 0] as bf16 hi and lo parts
// (hi + lo carries g to ~2^-17) into shared memory as an MN-major operand; then
// tcgen05.mma A = G' (MN-major, (p, h) x entries), B = the same key tile read MN-major
// -> U [(p, h) x dI] accumulated in TMEM over the chunk.  Partial U per chunk, the loss
// sums and db go to global memory; small CUDA-core kernels finish dq, dw and the
// projection gradients.
#include <cuda.h>

#include <algorithm>

#include "lsa_common.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int kTE = 128;          // entries per key tile
constexpr int kTR = 128;          // (position, head) rows per group
// warp 0 producer, warp 1 MMA, warps 4 .. 19 epilogue: four per TMEM lane quarter, each
// owning 32 of the 128 (position, head) columns
constexpr int kEpiWarps = 16;
template <int kH>
constexpr int train_threads() { return 128 + 32 * kEpiWarps; }
constexpr int kTStages = 3;       // key tiles in flight: the next tile's load must not wait on the MMAs
constexpr int kTChunks = 4;       // entry chunks per group
constexpr int kGBufs = 1;         // gated-gradient tiles (hi + lo) in shared memory

struct TrainParams {
  int P, N, H, dI, chunks, ntiles;
  const uint8_t* qimg;            // [groups][kTR x dI bf16], K-major, 128-byte swizzle
  const float* w;                 // [P][H]
  float bias, gamma;
  const uint32_t* labels;         // [P][Nw]
  float* Upart;                   // [chunks][P*H][dI]
  double* acc;                    // [3]: sum BCE, sum FL, sum g
  int32_t* status;
};

__device__ __forceinline__ uint64_t desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// fp32 accumulate, bf16 operands, M = 128; transposes select MN-major operands.
__host__ __device__ constexpr uint32_t t_idesc(int n, bool ta, bool tb) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((ta ? 1u : 0u) << 15) | ((tb ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ bool wait_timed(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
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

// dJ/dz of BCE + focal (gamma) for one pair, before the 1/n of the means (zero where
// the probability clamp [2^-20, 1 - 2^-20] is active); also the pair's BCE and FL terms.
// Everything is taken from z: the clamp is |z| > ln(2^20 - 1), p = sigmoid(z) and
// 1 - p = sigmoid(-z) are each computed directly, ln p = -log1p(e^-z) and
// ln(1 - p) = -log1p(e^z), so nothing near saturation rests on 1 - p in fp32.
__device__ __forceinline__ float pair_grad(float z, bool y, float gamma, double& bce, double& fl) {
  const float eps = 1.f / 1048576.f;
  const float zc = 13.862942f;                 // ln(2^20 - 1): sigmoid(zc) = 1 - 2^-20
  const bool clamped = z > zc || z < -zc;
  float pc, qc, lp, lq;
  if (z > zc) {
    pc = 1.f - eps; qc = eps; lp = log1pf(-eps); lq = logf(eps);
  } else if (z < -zc) {
    pc = eps; qc = 1.f - eps; lp = logf(eps); lq = log1pf(-eps);
  } else {
    const float en = expf(-z), ep = expf(z);
    pc = 1.f / (1.f + en);
    qc = 1.f / (1.f + ep);
    lp = -log1pf(en);
    lq = -log1pf(ep);
  }
  const float fw = gamma == 2.f ? (y ? qc * qc : pc * pc) : (y ? powf(qc, gamma) : powf(pc, gamma));
  float d;
  if (y) {
    bce -= lp;
    fl -= static_cast<double>(fw * lp);
    d = -qc + gamma * pc * fw * lp - fw * qc;                 // (p - 1) + g p (1-p)^g ln p - (1-p)^(g+1)
  } else {
    bce -= lq;
    fl -= static_cast<double>(fw * lq);
    d = pc + fw * pc - gamma * fw * qc * lq;                  // p + p^(g+1) - g p^g (1-p) ln(1-p)
  }
  return clamped ? 0.f : d;
}

template <int kH, int kDI>
__global__ void __launch_bounds__(train_threads<kH>(), 1)
train_tc_kernel(const __grid_constant__ CUtensorMap mapK, const TrainParams p) {
  constexpr int kPg = kTR / kH;                        // positions per group
  constexpr int kBoxes = kDI / 64;                     // 64-element key columns per tile row
  constexpr int kBoxBytes = kTE * 128;                 // one box: 128 entries x 128 bytes
  constexpr int kKeyBytes = kBoxes * kBoxBytes;
  constexpr int kQBytes = kTR * kDI * 2;
  constexpr int kGBytes = kTR * kTE * 2;               // one of G'hi / G'lo
  constexpr int kGHalf = kGBytes / 2;                  // 64 (p, h) columns x 128 entry rows
  extern __shared__ __align__(1024) uint8_t smraw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  uint8_t* keys = sm;
  uint8_t* qs = keys + kTStages * kKeyBytes;
  uint8_t* gbuf = qs + kQBytes;                                        // [kGBufs][hi, lo] G' tiles
  float* ws = reinterpret_cast<float*>(gbuf + kGBufs * 2 * kGBytes);   // [kTR] head weights of the group
  float* zsm = ws + kTR;                                               // [2][4 quarters][4][32] partial z
  uint64_t* full = reinterpret_cast<uint64_t*>(zsm + 2 * 4 * 4 * 32);
  uint64_t* empty = full + kTStages;
  uint64_t* f_full = empty + kTStages;          // [2]: forward accumulator b ready
  uint64_t* f_free = f_full + 2;                // [2]: forward accumulator b read
  uint64_t* g_full = f_free + 2;                // [2]: G' buffer b written
  uint64_t* g_free = g_full + 2;                // [2]: G' buffer b consumed
  uint64_t* u_done = g_free + 2;
  uint64_t* q_bar = u_done + 1;
  uint64_t* z_bar = q_bar + 1;                  // [2 parities][4 quarters]: partial z written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(z_bar + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int group = blockIdx.x, chunk = blockIdx.y;
  const int t0 = (p.ntiles * chunk) / p.chunks, t1 = (p.ntiles * (chunk + 1)) / p.chunks;
  const int nt = t1 - t0;
  if (tid == 0) {
    for (int i = 0; i < kTStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 2); }   // 2 issuers
    for (int b = 0; b < 2; ++b) { mbar_init(&f_full[b], 1); mbar_init(&f_free[b], 32 * kEpiWarps); }
    for (int b = 0; b < 2; ++b) { mbar_init(&g_full[b], 32 * kEpiWarps); mbar_init(&g_free[b], 2); }
    mbar_init(u_done, 2);
    mbar_init(q_bar, 1);
    for (int b = 0; b < 8; ++b) mbar_init(&z_bar[b], 128);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid < kTR) ws[tid] = p.w[static_cast<size_t>(group * kPg) * kH + tid];
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // F buffers at columns 0 and 128; U from the hi parts at 256, from the lo parts at 384
  const uint32_t tF = tmem, tU = tmem + 256, tUlo = tmem + 384;

  if (warp == 0 && lane == 0) {
    // producer: the group's query image once, then the chunk's key tiles
    mbar_expect_tx(q_bar, kQBytes);
    bulk_load(qs, p.qimg + static_cast<size_t>(group) * kQBytes, kQBytes, q_bar);
    const uint64_t pol = evict_first_policy();
    int issued = 0;
    for (int i = 0; i < nt; ++i) {
      const int slot = i % kTStages;
      if (i >= kTStages && !mbar_wait(&empty[slot], ((i / kTStages) - 1) & 1, abort_flag)) break;
      uint8_t* dst = keys + slot * kKeyBytes;
      mbar_expect_tx(&full[slot], kKeyBytes);
#pragma unroll
      for (int bx = 0; bx < kBoxes; ++bx)
        tma_load_3d(dst + bx * kBoxBytes, &mapK, bx * 64, (t0 + i) * kTE, 0, &full[slot], pol);
      issued = i + 1;
    }
    for (int i = (issued > kTStages ? issued - kTStages : 0); i < issued; ++i)
      wait_timed(&full[i % kTStages], (i / kTStages) & 1);
    wait_timed(q_bar, 0);
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    // Two MMA issuers (one thread issues a tcgen05.mma every ~90 cycles): warp 1 issues
    // the forward products, tile i+1's ahead of tile i's backward ones, and the backward
    // product of the hi parts of G' into U; warp 2 the backward product of the lo parts
    // into a second accumulator.  A key tile or a G' tile is free once both have
    // committed.
    const bool first = warp == 1;
    const uint32_t id_f = t_idesc(kTR, false, false), id_b = t_idesc(kDI, true, true);
    bool ok = mbar_wait(q_bar, 0, abort_flag);
    const uint32_t q0 = smem_u32(qs), g0 = smem_u32(gbuf);
    auto forward = [&](int i) -> bool {
      const int slot = i % kTStages, fb = i & 1;
      if (!mbar_wait(&full[slot], (i / kTStages) & 1, abort_flag)) return false;
      if (i >= 2 && !mbar_wait(&f_free[fb], ((i >> 1) - 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t k0 = smem_u32(keys + slot * kKeyBytes);
#pragma unroll
      for (int ks = 0; ks < kDI / 16; ++ks) {
        const uint32_t off = (ks >> 2) * kBoxBytes + (ks & 3) * 32;
        mma<false>(tF + fb * 128, desc(k0 + off, 16, 1024),
                   desc(q0 + (ks >> 2) * (kTR * 128) + (ks & 3) * 32, 16, 1024), id_f, ks > 0 ? 1u : 0u);
      }
      mma_commit(&f_full[fb]);
      return true;
    };
    if (first && ok && nt > 0) ok = forward(0);
    for (int i = 0; ok && i < nt; ++i) {
      if (first && i + 1 < nt && !forward(i + 1)) { ok = false; break; }
      const int slot = i % kTStages;
      if (!first && !mbar_wait(&full[slot], (i / kTStages) & 1, abort_flag)) { ok = false; break; }
      const int gb = i % kGBufs;
      if (!mbar_wait(&g_full[gb], (i / kGBufs) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t k0 = smem_u32(keys + slot * kKeyBytes);
      const uint32_t a0 = g0 + gb * 2 * kGBytes + (first ? 0 : kGBytes);
#pragma unroll
      for (int ks = 0; ks < kTE / 16; ++ks)
        mma<false>(first ? tU : tUlo, desc(a0 + ks * 2048, kGHalf, 1024), desc(k0 + ks * 2048, kBoxBytes, 1024),
                   id_b, (i > 0 || ks > 0) ? 1u : 0u);
      mma_commit(&g_free[gb]);
      mma_commit(&empty[slot]);
    }
    mma_commit(u_done);          // also after an abort: arrives once issued MMAs are done
  } else if (warp >= 4) {
    // epilogue warp (quarter, wq): lanes = entries quarter*32 .. +31 of the tile, columns
    // wq*32 .. +31 = heads of position j = wq*32 / kH.  The kH/32 warps of a position add
    // their partial z through shared memory, synchronised by a bounded mbarrier wait.
    constexpr int kParts = kH / 32;                     // warps per position
    const int we = warp - 4, quarter = we & 3, wq = we >> 2;
    const int j = wq / kParts, part = wq % kParts;
    const int e = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int Nw = (p.N + 31) / 32;
    const int pp = group * kPg + j;
    const float inv_n = 1.f / (static_cast<float>(p.P) * static_cast<float>(p.N));
    const uint32_t* lrow = p.labels + static_cast<size_t>(pp) * Nw;
    double bce = 0.0, fl = 0.0, gsum = 0.0;
    for (int i = 0; i < nt; ++i) {
      const int s = (t0 + i) * kTE + e;
      const uint32_t lab = s < p.N ? __ldg(lrow + (s >> 5)) : 0u;   // issued before the wait
      const int fb = i & 1;
      if (!mbar_wait(&f_full[fb], (i >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      float a[32];
      ld32(tF + fb * 128 + lane_off + wq * 32, a);
      tc_fence_before();
      mbar_arrive(&f_free[fb]);
      float zp[4] = {0.f, 0.f, 0.f, 0.f};                 // four independent chains
      const float4* w4 = reinterpret_cast<const float4*>(ws + wq * 32);
#pragma unroll
      for (int hh = 0; hh < 32; hh += 4) {
        const float4 wv = w4[hh >> 2];
        zp[0] = fmaf(wv.x, fmaxf(a[hh], 0.f), zp[0]);
        zp[1] = fmaf(wv.y, fmaxf(a[hh + 1], 0.f), zp[1]);
        zp[2] = fmaf(wv.z, fmaxf(a[hh + 2], 0.f), zp[2]);
        zp[3] = fmaf(wv.w, fmaxf(a[hh + 3], 0.f), zp[3]);
      }
      float z = (zp[0] + zp[1]) + (zp[2] + zp[3]);
      if constexpr (kParts > 1) {
        // this tile parity's buffer is rewritten two tiles later, after the next exchange
        float* zb = zsm + ((fb * 4 + quarter) * 4) * 32;
        zb[wq * 32 + lane] = z;
        mbar_arrive(&z_bar[fb * 4 + quarter]);
        if (!mbar_wait(&z_bar[fb * 4 + quarter], (i >> 1) & 1, abort_flag)) break;
        z = 0.f;
#pragma unroll
        for (int k = 0; k < kParts; ++k) z += zb[(j * kParts + k) * 32 + lane];
      }
      z += p.bias;
      float g = 0.f;
      if (s < p.N) {
        const bool y = (lab >> (s & 31)) & 1u;
        double b2 = 0.0, f2 = 0.0;
        g = pair_grad(z, y, p.gamma, b2, f2) * inv_n;
        if (part == 0) {                                  // one warp per position counts the pair
          bce += b2;
          fl += f2;
          gsum += g;
        }
      }
      // G' = g 1[a > 0]: the bf16 bit patterns of g's hi and lo parts, masked per column
      const __nv_bfloat16 bh = __float2bfloat16_rn(g);
      const uint32_t hb = __bfloat16_as_ushort(bh);
      const uint32_t lb = __bfloat16_as_ushort(__float2bfloat16_rn(g - __bfloat162float(bh)));
      const int gb = i % kGBufs;
      if (i >= kGBufs && !mbar_wait(&g_free[gb], ((i / kGBufs) - 1) & 1, abort_flag)) break;
      uint8_t* ghi = gbuf + gb * 2 * kGBytes;
      uint8_t* glo = ghi + kGBytes;
      // G' row e, columns wq*32 .. +31, MN-major 128-byte swizzle
      const uint32_t rowoff = (e >> 3) * 1024 + (e & 7) * 128;
#pragma unroll
      for (int cidx = 0; cidx < 4; ++cidx) {
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t m = (a[cidx * 8 + 2 * u] > 0.f ? 0x0000FFFFu : 0u) | (a[cidx * 8 + 2 * u + 1] > 0.f ? 0xFFFF0000u : 0u);
          wh[u] = (hb | (hb << 16)) & m;
          wl[u] = (lb | (lb << 16)) & m;
        }
        const int col = wq * 32 + cidx * 8;               // first (p, h) column of this 16-byte unit
        const int half = col >> 6, chunk16 = (col & 63) >> 3;
        const uint32_t off = half * kGHalf + rowoff + ((chunk16 ^ (e & 7)) << 4);
        *reinterpret_cast<uint4*>(ghi + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        *reinterpret_cast<uint4*>(glo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&g_full[gb]);
    }
    // all MMAs of the chunk done (or abandoned)
    const bool got = wait_timed(u_done, 0) && !*abort_flag;
    tc_fence_after();
    if (got) {
      // U rows: (p, h) = TMEM lane e of this quarter; the four warps of a quarter split dI
      float* dst = p.Upart + (static_cast<size_t>(chunk) * p.P * p.H + static_cast<size_t>(group) * kTR + e) * kDI;
      for (int c0 = wq * 32; c0 < kDI; c0 += 128) {
        float v[32], vl[32];
        ld32(tU + lane_off + c0, v);
        ld32(tUlo + lane_off + c0, vl);
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] += vl[u];
        if (nt == 0) {                       // an empty chunk: no MMA wrote U
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = 0.f;
        }
#pragma unroll
        for (int u = 0; u < 32; u += 4) *reinterpret_cast<float4*>(dst + c0 + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        bce += __shfl_xor_sync(0xffffffffu, bce, o);
        fl += __shfl_xor_sync(0xffffffffu, fl, o);
        gsum += __shfl_xor_sync(0xffffffffu, gsum, o);
      }
      if (lane == 0 && part == 0) {
        atomicAdd(&p.acc[0], bce);
        atomicAdd(&p.acc[1], fl);
        atomicAdd(&p.acc[2], gsum);
      }
    } else if (e == 0 && wq == 0) {
      raise_status(p.status, LSA_ERR_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// K-major, 128-byte-swizzled image of the query rows of each group: row m = (position
// group*Pg + m / H, head m % H), dI bf16; chunks of 64 columns, each [128 rows x 128 B].
__global__ void train_qimg_kernel(const __nv_bfloat16* __restrict__ q, int P, int H, int dI, int Pg,
                                  uint8_t* __restrict__ img) {
  const int group = blockIdx.y;
  const int units = kTR * (dI / 8);                    // 16-byte units per group
  for (int u = blockIdx.x * blockDim.x + threadIdx.x; u < units; u += gridDim.x * blockDim.x) {
    const int m = u / (dI / 8), c8 = u % (dI / 8);     // row, 8-element unit along dI
    const int pp = group * Pg + m / H, hh = m % H;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (pp < P) v = *reinterpret_cast<const uint4*>(q + (static_cast<size_t>(pp) * H + hh) * dI + c8 * 8);
    const int chunk = c8 / 8, unit = c8 % 8;
    const size_t off = static_cast<size_t>(group) * kTR * dI * 2 + chunk * (kTR * 128) + (m >> 3) * 1024 +
                       (m & 7) * 128 + ((unit ^ (m & 7)) << 4);
    *reinterpret_cast<uint4*>(img + off) = v;
  }
}

// U = sum over chunks; dq = w U ([P][H*dI]); dw = q . U ([P][H]).  One block per (p, h).
// One warp per (position, head) row: U = the chunks' partial sums in chunk order, dq = w U,
// dw = q . U; block 0's first thread also writes the loss means and the bias gradient
// (the fused kernel's sums are complete when this launch runs).
__global__ void __launch_bounds__(256)
train_finish_kernel(const float* __restrict__ Upart, int chunks, int rows, int dI,
                    const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                    float* __restrict__ dq, float* __restrict__ dw, const double* __restrict__ acc, double n,
                    double* __restrict__ loss, double* __restrict__ dbias) {
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (loss) { loss[0] = acc[0] / n; loss[1] = acc[1] / n; }
    if (dbias) dbias[0] = acc[2];
  }
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float wr = w[row];
  float part = 0.f;
  for (int d = lane; d < dI; d += 32) {
    float u = 0.f;
    for (int c = 0; c < chunks; ++c) u += Upart[(static_cast<size_t>(c) * rows + row) * dI + d];
    dq[static_cast<size_t>(row) * dI + d] = wr * u;
    part = fmaf(__bfloat162float(q[static_cast<size_t>(row) * dI + d]), u, part);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if (lane == 0) dw[row] = part;
}

// out[m][n] = sum_p X[p][m] Y[p][n]  (X bf16 [P][M], Y fp32 [P][Nn]; M % 8 == 0, Nn % 4 == 0,
// all three pointers 16-byte aligned).  128 x 128 tiles; a thread owns 8 x 8 outputs, rows
// ty*4 + {0..3} and 64 + ty*4 + {0..3} and columns likewise from tx, so that every
// shared-memory read is a 16-byte vector; the positions p are staged 16 at a time.  One
// launch can serve a second product with the same X: column tiles from nbx1 on belong to
// (Y2, Nn2, out2).
constexpr int kOT = 128;   // tile edge
constexpr int kOK = 16;    // positions per stage

__global__ void __launch_bounds__(256)
outer_acc_kernel(const __nv_bfloat16* __restrict__ X, int M, const float* __restrict__ Y, int Nn, int P,
                 float* __restrict__ out, int nbx1 = 0x7fffffff, const float* __restrict__ Y2 = nullptr,
                 int Nn2 = 0, float* __restrict__ out2 = nullptr) {
  __shared__ __align__(16) float xs[kOK][kOT];
  __shared__ __align__(16) float ys[kOK][kOT];
  int bx = blockIdx.x;
  if (bx >= nbx1) {
    bx -= nbx1;
    Y = Y2;
    Nn = Nn2;
    out = out2;
  }
  const int m0 = blockIdx.y * kOT, n0 = bx * kOT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  // The next stage's values are loaded into registers while the current one is used
  // (thread t: X positions t / 16, values (t % 16) * 8 .. + 7; Y two float4).
  const int xk = threadIdx.x >> 4, xc = (threadIdx.x & 15) * 8;
  auto load_x = [&](int p0) {
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    const int pp = p0 + xk, m = m0 + xc;
    if (pp < P && m < M) raw = *reinterpret_cast<const uint4*>(X + static_cast<size_t>(pp) * M + m);   // M % 8 == 0
    return raw;
  };
  auto load_y = [&](int p0, int u) {
    const int t = threadIdx.x + u * 256;
    const int kk = t / (kOT / 4), c = (t % (kOT / 4)) * 4;
    const int pp = p0 + kk, n = n0 + c;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (pp < P && n < Nn) v = *reinterpret_cast<const float4*>(Y + static_cast<size_t>(pp) * Nn + n);
    return v;
  };
  static_assert(kOK * kOT / 4 == 2 * 256, "two float4 of Y per thread and stage");
  uint4 xr = load_x(0);
  float4 yr0 = load_y(0, 0), yr1 = load_y(0, 1);
  for (int p0 = 0; p0 < P; p0 += kOK) {
    {   // X: bf16 -> fp32 is exact
      const uint32_t wv[4] = {xr.x, xr.y, xr.z, xr.w};
      float v[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(wv[e] << 16);
        v[2 * e + 1] = __uint_as_float(wv[e] & 0xffff0000u);
      }
      *reinterpret_cast<float4*>(&xs[xk][xc]) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(&xs[xk][xc + 4]) = make_float4(v[4], v[5], v[6], v[7]);
      const int t0 = threadIdx.x, t1 = threadIdx.x + 256;
      *reinterpret_cast<float4*>(&ys[t0 / (kOT / 4)][(t0 % (kOT / 4)) * 4]) = yr0;
      *reinterpret_cast<float4*>(&ys[t1 / (kOT / 4)][(t1 % (kOT / 4)) * 4]) = yr1;
    }
    __syncthreads();
    if (p0 + kOK < P) {
      xr = load_x(p0 + kOK);
      yr0 = load_y(p0 + kOK, 0);
      yr1 = load_y(p0 + kOK, 1);
    }
#pragma unroll
    for (int k = 0; k < kOK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&ys[k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&ys[k][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i >> 2) * 64 + ty * 4 + (i & 3);
    if (m >= M) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = n0 + h * 64 + tx * 4;   // Nn % 4 == 0: n < Nn covers all four
      if (n < Nn)
        *reinterpret_cast<float4*>(out + static_cast<size_t>(m) * Nn + n) =
            make_float4(acc[i][4 * h], acc[i][4 * h + 1], acc[i][4 * h + 2], acc[i][4 * h + 3]);
    }
  }
}

// dc[p][i] = sum_j dq[p][j] W_up[i][j]  (W_up bf16 [r][J]).  Tiles of 64 positions x 256
// rows i, 8 x 8 outputs per thread (two float4 of each operand per reduction step), the
// reduction split into kDcSplits slices written as partial sums and added in a fixed order
// by dc_reduce_kernel; within a slice j ascends, so the tile shape changes no result bit.
// The next 32-wide chunk of both operands is loaded into registers while the current one
// is used.
constexpr int kDcSplits = 64;
constexpr int kDcP = 64, kDcI = 256, kDcJ = 32;

__global__ void __launch_bounds__(256)
dc_kernel(const float* __restrict__ dq, int P, int J, const __nv_bfloat16* __restrict__ Wu, int r,
          float* __restrict__ part) {
  __shared__ __align__(16) float as[kDcJ][kDcP];   // [j][p]
  __shared__ __align__(16) float bs[kDcJ][kDcI];   // [j][i]
  const int i0 = blockIdx.x * kDcI, p0 = blockIdx.y * kDcP, sl = blockIdx.z;
  const int js = (J * sl) / kDcSplits, je = (J * (sl + 1)) / kDcSplits;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // i groups of 4 (x2), p groups of 4 (x2)
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  // thread t loads dq float4 f = t + 256 u (row f % 64, j f / 64 * 4) and W_up 8-wide
  // pieces f = t + 256 u (row f % 256, j f / 256 * 8); positions past P, rows past r and
  // columns past the slice read zero (J % 8 == 0, so a piece is all in or all out)
  auto load_a = [&](int j0, int u) {
    const int f = threadIdx.x + 256 * u, row = f % kDcP, j = j0 + (f / kDcP) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p0 + row < P && j < je) v = *reinterpret_cast<const float4*>(dq + static_cast<size_t>(p0 + row) * J + j);
    return v;
  };
  auto load_b = [&](int j0, int u) {
    const int f = threadIdx.x + 256 * u, row = f % kDcI, j = j0 + (f / kDcI) * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (i0 + row < r && j < je) v = *reinterpret_cast<const uint4*>(Wu + static_cast<size_t>(i0 + row) * J + j);
    return v;
  };
  float4 ar[2];
  uint4 br[4];
#pragma unroll
  for (int u = 0; u < 2; ++u) ar[u] = load_a(js, u);
#pragma unroll
  for (int u = 0; u < 4; ++u) br[u] = load_b(js, u);
  for (int j0 = js; j0 < je; j0 += kDcJ) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int f = threadIdx.x + 256 * u, row = f % kDcP, jj = (f / kDcP) * 4;
      as[jj][row] = ar[u].x; as[jj + 1][row] = ar[u].y; as[jj + 2][row] = ar[u].z; as[jj + 3][row] = ar[u].w;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int f = threadIdx.x + 256 * u, row = f % kDcI, jj = (f / kDcI) * 8;
      const uint32_t wv[4] = {br[u].x, br[u].y, br[u].z, br[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        bs[jj + 2 * e][row] = __uint_as_float(wv[e] << 16);              // bf16 -> fp32 is exact
        bs[jj + 2 * e + 1][row] = __uint_as_float(wv[e] & 0xffff0000u);
      }
    }
    __syncthreads();
    if (j0 + kDcJ < je) {
#pragma unroll
      for (int u = 0; u < 2; ++u) ar[u] = load_a(j0 + kDcJ, u);
#pragma unroll
      for (int u = 0; u < 4; ++u) br[u] = load_b(j0 + kDcJ, u);
    }
    const int kn = min(kDcJ, je - j0);
    for (int k = 0; k < kn; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&as[k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&as[k][32 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&bs[k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&bs[k][128 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int pp = p0 + (a >> 2) * 32 + ty * 4 + (a & 3);
    if (pp >= P) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int i = i0 + (b >> 2) * 128 + tx * 4 + (b & 3);
      if (i < r) part[(static_cast<size_t>(sl) * P + pp) * r + i] = acc[a][b];
    }
  }
}

__global__ void dc_reduce_kernel(const float* __restrict__ part, size_t n, float* __restrict__ dc) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float v = 0.f;
#pragma unroll 16
    for (int s = 0; s < kDcSplits; ++s) v += part[s * n + i];   // loads issued ahead, sums in slice order
    dc[i] = v;
  }
}

int train_smem(int dI) {
  return kTStages * (dI / 64) * kTE * 128 + kTR * dI * 2 + kGBufs * 2 * kTR * kTE * 2 + kTR * 4 + 2 * 4 * 4 * 32 * 4 +
         1024 + 1024;
}

}  // namespace

bool train_supported(int P, int H, int dI, int wdt, int kdt) {
  return wdt == LSA_BF16 && kdt == LSA_BF16 && (H == 32 || H == 64 || H == 128) && (dI == 64 || dI == 128) &&
         P >= 1 && P % (kTR / H) == 0 && P <= 4096;
}

TrainLayout train_layout(int P, int N, int D, int r, int H, int dI) {
  TrainLayout o{};
  const size_t Pz = static_cast<size_t>(P), HD = static_cast<size_t>(H) * dI;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off = align_up(off + bytes, 1024); return at; };
  const int groups = P / std::max(1, kTR / std::max(1, H));
  o.qimg = take(static_cast<size_t>(groups) * kTR * dI * 2);
  o.upart = take(static_cast<size_t>(kTChunks) * Pz * HD * 4);
  o.dq = take(Pz * HD * 4);
  o.dw = take(Pz * H * 4);
  o.dc = take(Pz * r * 4);
  o.dcpart = take(static_cast<size_t>(kDcSplits) * Pz * r * 4);
  o.acc = take(4 * 8);
  o.total = off;
  (void)N; (void)D;
  return o;
}

int launch_train(const TrainArgs& a, cudaStream_t st) {
  const TrainLayout lay = train_layout(a.P, a.N, a.D, a.r, a.H, a.dI);
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  const int Pg = kTR / a.H, groups = a.P / Pg;
  const size_t HD = static_cast<size_t>(a.H) * a.dI;
  uint8_t* qimg = ws + lay.qimg;
  float* Upart = reinterpret_cast<float*>(ws + lay.upart);
  float* dq = reinterpret_cast<float*>(ws + lay.dq);
  float* dw = reinterpret_cast<float*>(ws + lay.dw);
  float* dc = reinterpret_cast<float*>(ws + lay.dc);
  double* acc = reinterpret_cast<double*>(ws + lay.acc);
  int rc;
  if (cudaMemsetAsync(acc, 0, 4 * 8, st) != cudaSuccess) return check_launch("train/memset", 0);
  train_qimg_kernel<<<dim3((kTR * a.dI / 8 + 255) / 256, groups), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), a.P, a.H, a.dI, Pg, qimg);
  if ((rc = check_launch("train/query image")) != LSA_OK) return rc;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(LSA_ERR_CUDA, "train: cuTensorMapEncodeTiled unavailable");
  CUtensorMap mapK;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(a.dI), static_cast<cuuint64_t>(a.N), 1};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.dI) * 2, static_cast<cuuint64_t>(a.N) * a.dI * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kTE), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult cr = enc(&mapK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.K), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return fail(LSA_ERR_CUDA, "train: tensor map encode failed (%d)", (int)cr);
  TrainParams p{};
  p.P = a.P; p.N = a.N; p.H = a.H; p.dI = a.dI; p.chunks = kTChunks;
  p.ntiles = (a.N + kTE - 1) / kTE;
  p.qimg = qimg; p.w = a.w; p.bias = a.bias; p.gamma = a.gamma; p.labels = a.labels;
  p.Upart = Upart; p.acc = acc; p.status = a.status;
  const int smem = train_smem(a.dI);
  const dim3 grid(groups, kTChunks);
  auto go = [&](auto kern, int threads) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    kern<<<grid, threads, smem, st>>>(mapK, p);
  };
  switch (a.H * 1000 + a.dI) {
    case 32064: go(train_tc_kernel<32, 64>, train_threads<32>()); break;
    case 32128: go(train_tc_kernel<32, 128>, train_threads<32>()); break;
    case 64064: go(train_tc_kernel<64, 64>, train_threads<64>()); break;
    case 64128: go(train_tc_kernel<64, 128>, train_threads<64>()); break;
    case 128064: go(train_tc_kernel<128, 64>, train_threads<128>()); break;
    case 128128: go(train_tc_kernel<128, 128>, train_threads<128>()); break;
    default: return fail(LSA_ERR_UNSUPPORTED, "train: H=%d dI=%d", a.H, a.dI);
  }
  if ((rc = check_launch("train/fused")) != LSA_OK) return rc;
  const int frows = a.P * a.H;
  train_finish_kernel<<<(frows + 7) / 8, 256, 0, st>>>(Upart, kTChunks, frows, a.dI,
                                                       static_cast<const __nv_bfloat16*>(a.q), a.w, dq, dw, acc,
                                                       static_cast<double>(a.P) * a.N, a.loss, a.dbias);
  if ((rc = check_launch("train/finish")) != LSA_OK) return rc;
  // projection gradients
  const __nv_bfloat16* c = static_cast<const __nv_bfloat16*>(a.c);
  const __nv_bfloat16* h = static_cast<const __nv_bfloat16*>(a.h);
  outer_acc_kernel<<<dim3(static_cast<unsigned>((HD + kOT - 1) / kOT), (a.r + kOT - 1) / kOT), 256, 0, st>>>(
      c, a.r, dq, static_cast<int>(HD), a.P, a.dW_up);
  float* dcpart = reinterpret_cast<float*>(ws + lay.dcpart);
  dc_kernel<<<dim3((a.r + kDcI - 1) / kDcI, (a.P + kDcP - 1) / kDcP, kDcSplits), 256, 0, st>>>(
      dq, a.P, static_cast<int>(HD), static_cast<const __nv_bfloat16*>(a.W_up), a.r, dcpart);
  const size_t ndc = static_cast<size_t>(a.P) * a.r;
  dc_reduce_kernel<<<static_cast<unsigned>(std::min<size_t>((ndc + 255) / 256, 1184)), 256, 0, st>>>(dcpart, ndc, dc);
  const int nb_r = (a.r + kOT - 1) / kOT, nb_h = (a.H + kOT - 1) / kOT;   // dW_down and dW_w in one launch
  outer_acc_kernel<<<dim3(nb_r + nb_h, (a.D + kOT - 1) / kOT), 256, 0, st>>>(h, a.D, dc, a.r, a.P, a.dW_down, nb_r,
                                                                           dw, a.H, a.dW_w);
  return check_launch("train/projection gradients", 4);
}

}  // namespace lsa
