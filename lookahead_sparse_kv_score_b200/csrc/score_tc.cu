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
// range (|q| < 2^-10 s_h).  The B operand stacks the hi rows and the lo rows (N = 2H),
// so one MMA gives both dot products and the epilogue adds them; s_h > 0 folds into
// the head weight: w_h ReLU(s_h x) = (w_h s_h) ReLU(x).
//
// Pipeline (one persistent CTA per SM, 12 warps).  Issuing a tcgen05.mma or a commit
// costs a single thread on the order of a hundred cycles, comparable to the MMA's own
// work at these small N, so the CTA runs two independent pipelines over the even and
// the odd tiles of its range:
//   warps 0, 1   TMA producers (one per pipeline) into that pipeline's half of the
//                key-tile ring; warp 0 also loads the query image into one of two
//                slots at each (sequence, layer) change.
//   warps 2, 3   single-thread MMA issuers; warp 2 also owns the TMEM allocation.
//                Each pipeline has two accumulators (one when N > 128).
//   warps 4..11  two epilogue groups of four warps (one per TMEM lane quadrant).
// Per-tile bookkeeping is incremental (no integer division on the critical path) and
// the MMA descriptors are formed by adding constant offsets to a base descriptor.
// Every mbarrier wait is bounded by a time limit; on expiry the kernel records
// LSA_ERR_TIMEOUT in the status word, drains what it issued and frees its TMEM.
#include <cuda.h>

#include <algorithm>

#include "lsa_common.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int kTileM = 128;
constexpr int kSmemLimit = 227 * 1024;

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
// Accumulator columns per tile: H for bf16; 2H for fp8 (hi heads then lo heads).
template <bool kFp8, int kH>
struct TcShape {
  static constexpr int kN = kFp8 ? 2 * kH : kH;               // MMA N
  static constexpr int kNumAcc = kN <= 128 ? 4 : 2;           // TMEM accumulators
  static constexpr int kThreads = 128 + 128 * kNumAcc;        // 4 role warps + one epilogue group per accumulator
  static constexpr int kTmemCols = kNumAcc * kN;              // 128, 256 or 512
};

struct TcLayout {
  int chunks;       // 128-byte K chunks of one key row
  int a_bytes;      // one key tile (128 rows)
  int img_bytes;    // one query image (hi and lo rows for fp8)
  int ksteps;       // MMA instructions per tile
  int stages;       // key-tile ring depth (even; half per pipeline)
  size_t smem;      // dynamic shared memory
};

__host__ __device__ inline TcLayout tc_layout(int H, int dI, bool fp8) {
  TcLayout t{};
  const int row_bytes = fp8 ? dI : 2 * dI;
  t.chunks = row_bytes / 128;
  t.a_bytes = kTileM * row_bytes;
  t.img_bytes = (fp8 ? 2 : 1) * H * row_bytes;
  t.ksteps = row_bytes / 32;
  const int fixed = 2 * t.img_bytes + 1024 /*barriers*/ + 1024 /*alignment*/;
  int s = (kSmemLimit - fixed) / t.a_bytes;
  s = s > 8 ? 8 : s;
  t.stages = s & ~1;
  t.smem = static_cast<size_t>(t.stages) * t.a_bytes + fixed;
  return t;
}

struct TcParams {
  int B, N, H, dI, l0, nUnits, tiles_per_unit;
  // Gathered mode (the fine indexer): unit b scores the candidates idx[b][0..n_b),
  // n_b = min(count[b], cap), in tiles of 128; tile_start [nUnits + 1] is the prefix of
  // the units' tile counts.  Key rows are gathered by entry; logit is written at the
  // entry (logit[b][idx[b][j]]); no mask, score or bias.
  const int32_t* idx;      // [B][cap] or null
  const int32_t* count;    // [B]
  const int32_t* tile_start;
  int cap;
  const uint8_t* qimg;     // [L][B][img_bytes]
  const float* wfold;      // [L][B][H]
  const float* bias;       // [L]
  const float* kscale;     // [L][B][N] or null
  uint32_t* mask;          // [L][B][Nw]
  float* logit;            // [L][B][N] or null
  float* score;            // [L][B][N] or null
  int32_t* status;         // device status word or null
};

// Two 32-column TMEM loads of this thread's lane, one wait.
__device__ __forceinline__ void tmem_ld32x2(uint32_t t0, uint32_t t1, float (&v0)[32], float (&v1)[32]) {
  uint32_t r[64];
#define LSA_LD32(base, off)                                                                              \
  asm volatile(                                                                                          \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "                                                          \
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "                          \
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"        \
      : "=r"(r[base + 0]), "=r"(r[base + 1]), "=r"(r[base + 2]), "=r"(r[base + 3]), "=r"(r[base + 4]),  \
        "=r"(r[base + 5]), "=r"(r[base + 6]), "=r"(r[base + 7]), "=r"(r[base + 8]), "=r"(r[base + 9]),  \
        "=r"(r[base + 10]), "=r"(r[base + 11]), "=r"(r[base + 12]), "=r"(r[base + 13]),                 \
        "=r"(r[base + 14]), "=r"(r[base + 15]), "=r"(r[base + 16]), "=r"(r[base + 17]),                 \
        "=r"(r[base + 18]), "=r"(r[base + 19]), "=r"(r[base + 20]), "=r"(r[base + 21]),                 \
        "=r"(r[base + 22]), "=r"(r[base + 23]), "=r"(r[base + 24]), "=r"(r[base + 25]),                 \
        "=r"(r[base + 26]), "=r"(r[base + 27]), "=r"(r[base + 28]), "=r"(r[base + 29]),                 \
        "=r"(r[base + 30]), "=r"(r[base + 31])                                                           \
      : "r"(off))
  LSA_LD32(0, t0);
  LSA_LD32(32, t1);
#undef LSA_LD32
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) { v0[j] = __uint_as_float(r[j]); v1[j] = __uint_as_float(r[32 + j]); }
}

// Two pipelines per CTA, split by local tile parity p: producer warp p and MMA warp 2+p.
// Local tile i uses accumulator i % kNumAcc, drained by epilogue group i % kNumAcc
// (warps 4+4g .. 7+4g).  The pipelines share the query slots (loaded by producer 0 and
// released by both MMA issuers) and nothing else.
template <bool kFp8, int kH, int kKSteps, bool kGather>
__global__ void __launch_bounds__(TcShape<kFp8, kH>::kThreads, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const TcParams p) {
  pdl_wait();
  pdl_trigger();
  using S = TcShape<kFp8, kH>;
  constexpr int kN = S::kN, kNumAcc = S::kNumAcc;
  extern __shared__ uint8_t smem_raw[];
  const TcLayout lay = tc_layout(kH, p.dI, kFp8);
  const int S2 = lay.stages / 2;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_ring = smem;                                                   // [stages][a_bytes]
  uint8_t* q_slot = a_ring + static_cast<size_t>(lay.stages) * lay.a_bytes;  // [2][img_bytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(q_slot + 2 * lay.img_bytes);
  uint64_t* full = bars;                    // [8]
  uint64_t* empty = bars + 8;               // [8]
  uint64_t* qfull = bars + 16;              // [2]
  uint64_t* qempty = bars + 18;             // [2]
  uint64_t* tfull = bars + 20;              // [4]
  uint64_t* tempty = bars + 24;             // [4]
  uint64_t* drain = bars + 28;              // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 30);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 31);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < lay.stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 2);         // both MMA issuers
      mbar_init(&drain[s], 1);
    }
    for (int a = 0; a < kNumAcc; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 4); }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) tmem_alloc(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Tiles of a unit, the unit holding a flat tile index, and the walk to a later tile.
  auto tiles_of = [&](int u) -> int {
    if constexpr (kGather) return __ldg(p.tile_start + u + 1) - __ldg(p.tile_start + u);
    else return p.tiles_per_unit;
  };
  auto unit_of = [&](long long t) -> int {   // the last unit whose first tile is <= t
    if constexpr (kGather) {
      int lo = 0, hi = p.nUnits - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.tile_start + mid) <= t) lo = mid; else hi = mid - 1;
      }
      return lo;
    } else {
      return static_cast<int>(t / p.tiles_per_unit);
    }
  };
  auto first_tile = [&](int u) -> long long {
    if constexpr (kGather) return __ldg(p.tile_start + u);
    else return static_cast<long long>(u) * p.tiles_per_unit;
  };
  auto advance = [&](int& unit, int& tile, int by) {
    tile += by;
    if constexpr (kGather) {
      while (unit < p.nUnits && tile >= tiles_of(unit)) { tile -= tiles_of(unit); ++unit; }
    } else {
      while (tile >= p.tiles_per_unit) { tile -= p.tiles_per_unit; ++unit; }
    }
  };
  const long long T = kGather ? static_cast<long long>(__ldg(p.tile_start + p.nUnits))
                              : static_cast<long long>(p.nUnits) * p.tiles_per_unit;
  const long long t_begin = T * blockIdx.x / gridDim.x, t_end = T * (blockIdx.x + 1) / gridDim.x;
  const int n_local = static_cast<int>(t_end - t_begin);
  const int unit0 = n_local > 0 ? unit_of(t_begin) : 0;
  const int tile0 = n_local > 0 ? static_cast<int>(t_begin - first_tile(unit0)) : 0;
  const int Nw = (p.N + 31) / 32;
  const int uabs0 = p.l0 * p.B;

  // Local tile i of this CTA belongs to unit (i + t_begin) / tiles_per_unit; query slot
  // k = unit - unit0 of every unit in the range is loaded once by producer 0 and
  // released by both MMA issuers, in unit order.
  const int k_last = n_local > 0 ? unit_of(t_end - 1) - unit0 : -1;
  if (warp < 2 && (kGather || lane == 0)) {
    // ---------------------------------------------------------------- producers
    // Producer pp loads the key tiles of parity pp (local tiles pp, pp+2, ...) into
    // stages [pp*S2, pp*S2+S2); producer 0 also loads the query image of every unit.
    // Tiled mode: lane 0 alone, one TMA box per 128-byte K chunk.  Gathered mode: the
    // whole warp, lane l fetching candidates 4l .. 4l+3 of the tile with one four-row
    // gather per K chunk; lane 0 keeps the barriers.
    const int pp = warp;
    const uint64_t policy = evict_first_policy();
    int unit = unit0, tile = tile0;
    advance(unit, tile, pp);
    int kq = -1;                              // last query slot loaded (producer 0)
    auto load_q_through = [&](int k_to) -> bool {
      while (kq < k_to) {
        ++kq;
        const int slot = kq & 1;
        if (!mbar_wait(&qempty[slot], ((kq >> 1) & 1) ^ 1, abort_flag)) return false;
        mbar_expect_tx(&qfull[slot], lay.img_bytes);
        bulk_load(q_slot + slot * lay.img_bytes, p.qimg + static_cast<size_t>(uabs0 + unit0 + kq) * lay.img_bytes,
                  lay.img_bytes, &qfull[slot]);
      }
      return true;
    };
    int j = 0, s = 0;
    uint32_t ph = 0;
    bool ok = true;
    // Gathered mode: the rows (tensor-map row coordinates) of this lane's four candidates
    // of a tile; loaded one tile ahead so their latency overlaps the barrier waits.
    // Rows past the list repeat the tile's first candidate (always present).
    int rows[4] = {0, 0, 0, 0};
    auto rows_of = [&](int u, int t) {
      const int32_t* ib = p.idx + static_cast<size_t>(u) * p.cap;
      const int nb = min(__ldg(p.count + u), p.cap);
      const int first = __ldg(ib + t * kTileM);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int jj = t * kTileM + 4 * lane + e;
        int ent = __ldg(ib + min(jj, p.cap - 1));
        ent = jj < nb ? ent : first;
        ent = min(max(ent, 0), p.N - 1);
        rows[e] = (uabs0 + u) * p.N + ent;
      }
    };
    if constexpr (kGather) {
      if (pp < n_local) rows_of(unit, tile);
    }
    for (int i = pp; i < n_local; i += 2) {
      const int st = pp * S2 + s;
      if (lane == 0) {
        if (pp == 0) ok = load_q_through(unit - unit0);
        if (ok) ok = mbar_wait(&empty[st], ph ^ 1, abort_flag);
        if (ok) mbar_expect_tx(&full[st], lay.a_bytes);
      }
      if constexpr (kGather) ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      uint8_t* dst = a_ring + static_cast<size_t>(st) * lay.a_bytes;
      if constexpr (kGather) {
#pragma unroll
        for (int c = 0; c < kKSteps / 4; ++c)
          tma_gather4_2d(dst + c * (kTileM * 128) + lane * 4 * 128, &kmap, c * (kFp8 ? 128 : 64), rows[0], rows[1],
                         rows[2], rows[3], &full[st], policy);
      } else {
#pragma unroll
        for (int c = 0; c < kKSteps / 4; ++c)     // 128-byte K chunks of a key row
          tma_load_3d(dst + c * (kTileM * 128), &kmap, c * (kFp8 ? 128 : 64), tile * kTileM, uabs0 + unit,
                      &full[st], policy);
      }
      ++j;
      if (++s == S2) { s = 0; ph ^= 1; }
      advance(unit, tile, 2);
      if constexpr (kGather) {
        if (i + 2 < n_local) rows_of(unit, tile);
      }
    }
    if (lane == 0) {
      if (pp == 0 && ok) load_q_through(k_last);
      // drain: every key tile this warp issued has landed before the CTA exits
      for (int jj = j > S2 ? j - S2 : 0; jj < j; ++jj) {
        volatile int no_abort = 0;
        if (!mbar_wait(&full[pp * S2 + jj % S2], (jj / S2) & 1, &no_abort)) break;
      }
    }
  } else if ((warp == 2 || warp == 3) && lane == 0) {
    // ---------------------------------------------------------------- MMA issuers
    const int pp = warp - 2;
    const uint32_t idesc = instr_desc(kFp8, kN);
    const uint64_t dhi = smem_desc(0);
    const uint32_t a_ring_u = smem_u32(a_ring), q_slot_u = smem_u32(q_slot);
    int unit = unit0, tile = tile0;
    advance(unit, tile, pp);
    int kq = -1;                              // query slot in use
    // release the current slot and acquire every later one through k_to, in order
    auto acquire_q_through = [&](int k_to) -> bool {
      while (kq < k_to) {
        if (kq >= 0) mma_commit(&qempty[kq & 1]);
        ++kq;
        if (!mbar_wait(&qfull[kq & 1], (kq >> 1) & 1, abort_flag)) return false;
      }
      return true;
    };
    int s = 0;
    uint32_t ph = 0, aph = 0;     // aph: phase bit of each accumulator
    bool ok = true;
    for (int i = pp; i < n_local; i += 2) {
      if (!(ok = acquire_q_through(unit - unit0))) break;
      const int a = i % kNumAcc;
      const int st = pp * S2 + s;
      if (!(ok = mbar_wait(&tempty[a], ((aph >> a) & 1) ^ 1, abort_flag))) break;
      if (!(ok = mbar_wait(&full[st], ph, abort_flag))) break;
      tc_fence_after();
      const uint64_t adesc = dhi | (((a_ring_u + st * lay.a_bytes) >> 4) & 0x3FFFu);
      const uint64_t bdesc = dhi | (((q_slot_u + (kq & 1) * lay.img_bytes) >> 4) & 0x3FFFu);
      const uint32_t d_tmem = tmem_base + a * kN;
#pragma unroll
      for (int ks = 0; ks < kKSteps; ++ks) {
        constexpr uint32_t kA = (kTileM * 128) >> 4, kB = (kN * 128) >> 4;
        mma<kFp8>(d_tmem, adesc + (ks >> 2) * kA + (ks & 3) * 2, bdesc + (ks >> 2) * kB + (ks & 3) * 2, idesc,
                  ks > 0 ? 1u : 0u);
      }
      mma_commit(&empty[st]);
      mma_commit(&tfull[a]);
      aph ^= 1u << a;
      if (++s == S2) { s = 0; ph ^= 1; }
      advance(unit, tile, 2);
    }
    if (ok && acquire_q_through(k_last) && kq >= 0) mma_commit(&qempty[kq & 1]);
    // drain: all MMAs issued by this thread have completed
    mma_commit(&drain[pp]);
    volatile int no_abort = 0;
    mbar_wait(&drain[pp], 0, &no_abort);
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue
    const int g = (warp - 4) >> 2;            // accumulator: local tiles i = g, g + kNumAcc, ...
    const int quad = warp & 3;                // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    int unit = unit0, tile = tile0;
    advance(unit, tile, g);
    int cur = -1;
    float bias_l = 0.f;
    const float4* wf4 = nullptr;
    uint32_t aph = 0;
    // Gathered mode: the entry this thread's row scores in a tile (the candidate's entry
    // index, -1 past the unit's list); tiled mode: the row of the tile itself.
    auto entry_of = [&](int u, int t) -> int {
      const int jj = t * kTileM + row;
      return jj < min(__ldg(p.count + u), p.cap) ? __ldg(p.idx + static_cast<size_t>(u) * p.cap + jj) : -1;
    };
    int e_next = 0;
    if constexpr (kGather) e_next = g < n_local ? entry_of(unit, tile) : -1;
    // per-entry scale of the next tile, loaded one tile ahead
    float ks_next = 1.f;
    if (kFp8 && g < n_local) {
      const int n = kGather ? e_next : tile * kTileM + row;
      if (n >= 0 && n < p.N) ks_next = __ldg(p.kscale + static_cast<size_t>(uabs0 + unit) * p.N + n);
    }
    for (int i = g; i < n_local; i += kNumAcc) {
      const size_t uabs = static_cast<size_t>(uabs0 + unit);
      if (unit != cur) {
        cur = unit;
        bias_l = p.bias ? __ldg(p.bias + p.l0 + unit / p.B) : 0.f;
        wf4 = reinterpret_cast<const float4*>(p.wfold + uabs * kH);
      }
      const int n0 = tile * kTileM;
      const int n = kGather ? e_next : n0 + row;
      const bool valid = n >= 0 && n < p.N;
      const float ks = ks_next;
      // advance to this group's next tile and prefetch its scale (and entry)
      advance(unit, tile, kNumAcc);
      if (i + kNumAcc < n_local) {
        if constexpr (kGather) e_next = entry_of(unit, tile);
        if (kFp8) {
          const int nn = kGather ? e_next : tile * kTileM + row;
          ks_next = nn >= 0 && nn < p.N ? __ldg(p.kscale + static_cast<size_t>(uabs0 + unit) * p.N + nn) : 1.f;
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[g], aph, abort_flag))) break;
      aph ^= 1;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + g * kN;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      constexpr int kStep = kFp8 ? 32 : (kH >= 64 ? 64 : 32);
#pragma unroll
      for (int c0 = 0; c0 < kH; c0 += kStep) {
        float v0[32], v1[32];
        if constexpr (kFp8) {
          tmem_ld32x2(taddr + c0, taddr + kH + c0, v0, v1);         // hi heads, lo heads
        } else if constexpr (kStep == 64) {
          tmem_ld32x2(taddr + c0, taddr + c0 + 32, v0, v1);         // two head chunks
        } else {
          tmem_ld32x2(taddr + c0, taddr + c0, v0, v1);
        }
        if (c0 + kStep >= kH) {              // last load of this tile: release the accumulator
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[g]);
        }
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const float4 w = __ldg(wf4 + c0 / 4 + q4);
          const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int jj = 4 * q4 + e;
            const float x = kFp8 ? v0[jj] + v1[jj] : v0[jj];
            acc[e] = fmaf(wv[e], fmaxf(x, 0.f), acc[e]);
          }
        }
        if constexpr (!kFp8 && kStep == 64) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 w = __ldg(wf4 + (c0 + 32) / 4 + q4);
            const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] = fmaf(wv[e], fmaxf(v1[4 * q4 + e], 0.f), acc[e]);
          }
        }
      }
      const float z = fmaf((acc[0] + acc[1]) + (acc[2] + acc[3]), ks, bias_l);
      if (valid) {
        if (p.logit) p.logit[uabs * p.N + n] = z;
        if (p.score) p.score[uabs * p.N + n] = sigmoid_f(z);
      }
      if (p.mask) {
        const unsigned bits = __ballot_sync(0xffffffffu, valid && z >= 0.f);
        const int word = (n0 + quad * 32) >> 5;
        if (lane == 0 && word < Nw) p.mask[uabs * Nw + word] = bits;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) raise_status(p.status, LSA_ERR_TIMEOUT);
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

// ------------------------------------------------------------------ query images
// bf16: the query rows in the 128-byte-swizzled K-major layout the MMA reads (16-byte
// unit j of row h stored at unit j ^ (h % 8)); one 16-byte unit per thread.
__global__ void build_qimg_bf16_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                                       int B, int H, int dI, int l0, uint8_t* __restrict__ img,
                                       float* __restrict__ wfold) {
  pdl_wait();
  pdl_trigger();
  const size_t uabs = static_cast<size_t>(l0) * B + blockIdx.y;
  const int units = H * dI / 8;
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u < units) {
    const int h = u / (dI / 8), d0 = (u % (dI / 8)) * 8;
    const int c = d0 / 64, j = (d0 % 64) / 8;
    const uint4 v = *reinterpret_cast<const uint4*>(q + uabs * H * dI + static_cast<size_t>(h) * dI + d0);
    *reinterpret_cast<uint4*>(img + uabs * H * dI * 2 + static_cast<size_t>(c) * H * 128 + h * 128 +
                              ((j ^ (h & 7)) * 16)) = v;
  }
  if (blockIdx.x == 0)
    for (int hh = threadIdx.x; hh < H; hh += blockDim.x) wfold[uabs * H + hh] = w[uabs * H + hh];
}

// fp8: one warp per head: power-of-two scale s_h with max|q_h / s_h| <= 448, hi and lo
// e4m3 values, and the folded head weight w_h * s_h.  In each 128-byte K chunk the
// image holds 2H rows: row h = hi of head h, row H + h = lo of head h, swizzled like
// the bf16 image.  Each lane handles four consecutive elements of the head row.
__global__ void build_qimg_fp8_kernel(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                                      int B, int H, int dI, int l0, uint8_t* __restrict__ img,
                                      float* __restrict__ wfold) {
  pdl_wait();
  pdl_trigger();
  const size_t uabs = static_cast<size_t>(l0) * B + blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (h >= H) return;
  const __nv_bfloat16* qr = q + (uabs * H + h) * dI;
  uint8_t* out = img + uabs * 2 * H * dI;
  float amax = 0.f;
  for (int d = lane * 4; d < dI; d += 128)
    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(__bfloat162float(qr[d + e])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int ex = 0;   // smallest power of two s = 2^ex with amax <= 448 s
  if (amax > 0.f) {
    ex = static_cast<int>(ceilf(log2f(amax / 448.f)));
    while (amax > ldexpf(448.f, ex)) ++ex;
    while (ex > -126 && amax <= ldexpf(448.f, ex - 1)) --ex;
  }
  const float inv = ldexpf(1.f, -ex);
  const int rows = 2 * H;
  for (int d = lane * 4; d < dI; d += 128) {
    uint32_t hi4 = 0, lo4 = 0;
    for (int e = 0; e < 4; ++e) {
      const float x = __bfloat162float(qr[d + e]) * inv;   // exact (power of two)
      const __nv_fp8_e4m3 hi(x);
      const __nv_fp8_e4m3 lo(x - static_cast<float>(hi));
      hi4 |= static_cast<uint32_t>(hi.__x) << (8 * e);
      lo4 |= static_cast<uint32_t>(lo.__x) << (8 * e);
    }
    const int c = d / 128, j = (d % 128) / 16, x = d % 16;
    const size_t chunk = static_cast<size_t>(c) * rows * 128;
    const int rh = h, rl = H + h;
    *reinterpret_cast<uint32_t*>(out + chunk + rh * 128 + ((j ^ (rh & 7)) * 16) + x) = hi4;
    *reinterpret_cast<uint32_t*>(out + chunk + rl * 128 + ((j ^ (rl & 7)) * 16) + x) = lo4;
  }
  if (lane == 0) wfold[uabs * H + h] = w[uabs * H + h] * ldexpf(1.f, ex);
}

// ------------------------------------------------------------------ tensor map
template <bool kFp8, int kH, int kKSteps>
int launch_kernel(const CUtensorMap& map, const TcParams& p, const TcLayout& lay, int grid, cudaStream_t st) {
  if (p.idx != nullptr) {
    auto kern = score_tc_kernel<kFp8, kH, kKSteps, true>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.smem);
    launch_dependent(kern, dim3(grid), dim3(TcShape<kFp8, kH>::kThreads), lay.smem, st, map, p);
    return check_launch("fine_score_tc");
  }
  auto kern = score_tc_kernel<kFp8, kH, kKSteps, false>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.smem);
  launch_dependent(kern, dim3(grid), dim3(TcShape<kFp8, kH>::kThreads), lay.smem, st, map, p);
  return check_launch("score_tc");
}

template <bool kFp8, int kH>
int launch_k(const CUtensorMap& map, const TcParams& p, const TcLayout& lay, int grid, cudaStream_t st) {
  switch (lay.ksteps) {
    case 4: return launch_kernel<kFp8, kH, 4>(map, p, lay, grid, st);
    case 8: return launch_kernel<kFp8, kH, 8>(map, p, lay, grid, st);
    case 12:
      if constexpr (!kFp8) return launch_kernel<false, kH, 12>(map, p, lay, grid, st);
      break;
    case 16:
      if constexpr (!kFp8) return launch_kernel<false, kH, 16>(map, p, lay, grid, st);
      break;
  }
  return fail(LSA_ERR_UNSUPPORTED, "score_tc: %d MMA steps per tile", lay.ksteps);
}

template <bool kFp8>
int launch_h(const CUtensorMap& map, const TcParams& p, const TcLayout& lay, int grid, cudaStream_t st) {
  switch (p.H) {
    case 32: return launch_k<kFp8, 32>(map, p, lay, grid, st);
    case 64: return launch_k<kFp8, 64>(map, p, lay, grid, st);
    case 128: return launch_k<kFp8, 128>(map, p, lay, grid, st);
    case 256:
      if constexpr (!kFp8) return launch_k<false, 256>(map, p, lay, grid, st);
      break;
  }
  return fail(LSA_ERR_UNSUPPORTED, "score_tc: H=%d", p.H);
}

// tile_start[b] = sum over b' < b of ceil(min(count[b'], cap) / 128), b = 0..B (one block).
__global__ void tile_prefix_kernel(const int32_t* __restrict__ count, int B, int cap, int32_t* __restrict__ tile_start) {
  pdl_wait();
  pdl_trigger();
  __shared__ int wsum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < B; b0 += blockDim.x) {
    const int b = b0 + tid;
    const int n = b < B ? min(max(count[b], 0), cap) : 0;
    const int t = (n + kTileM - 1) / kTileM;
    int incl = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = carry;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (b < B) tile_start[b] = before + incl - t;
    __syncthreads();
    if (tid == blockDim.x - 1) carry = before + incl;
    __syncthreads();
  }
  if (tid == 0) tile_start[B] = carry;
}

}  // namespace

int launch_fine_score_tc(const FineArgs& a, cudaStream_t st) {
  const bool fp8 = a.kdt == LSA_E4M3;
  const TcLayout lay = tc_layout(a.H, a.dI, fp8);
  const dim3 ig(fp8 ? (a.H + 7) / 8 : (a.H * a.dI / 8 + 255) / 256, a.B);
  if (fp8)
    launch_dependent(build_qimg_fp8_kernel, ig, dim3(256), 0, st, static_cast<const __nv_bfloat16*>(a.q), a.w, a.B,
                     a.H, a.dI, 0, a.qimg, a.wfold);
  else
    launch_dependent(build_qimg_bf16_kernel, ig, dim3(256), 0, st, static_cast<const __nv_bfloat16*>(a.q), a.w, a.B,
                     a.H, a.dI, 0, a.qimg, a.wfold);
  launch_dependent(tile_prefix_kernel, dim3(1), dim3(1024), 0, st, a.count, a.B, a.cap, a.tile_start);
  int rc = check_launch("fine_score/query image and tile prefix", 2);
  if (rc != LSA_OK) return rc;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(LSA_ERR_CUDA, "fine_score: cuTensorMapEncodeTiled unavailable");
  CUtensorMap map;
  const int esz = fp8 ? 1 : 2;
  // rows of all sequences' keys, one row per box: the four-row gathers pick them by entry
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.dI), static_cast<cuuint64_t>(a.B) * a.N};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.dI) * esz};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), 1};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult cr = enc(&map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                          const_cast<void*>(a.K), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return fail(LSA_ERR_CUDA, "fine_score: tensor map encode failed (%d)", (int)cr);
  TcParams p{};
  p.B = a.B; p.N = a.N; p.H = a.H; p.dI = a.dI; p.l0 = 0; p.nUnits = a.B; p.tiles_per_unit = 0;
  p.qimg = a.qimg; p.wfold = a.wfold; p.bias = nullptr; p.kscale = a.kscale;
  p.mask = nullptr; p.logit = a.score; p.score = nullptr; p.status = a.status;
  p.idx = a.idx; p.count = a.count; p.tile_start = a.tile_start; p.cap = a.cap;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // the tile count is on the device: one CTA per SM, each takes an equal share of it
  return fp8 ? launch_h<true>(map, p, lay, sms, st) : launch_h<false>(map, p, lay, sms, st);
}

bool tc_supported(int H, int dI, int wdt, int kdt) {
  if (wdt != LSA_BF16) return false;
  if (H != 32 && H != 64 && H != 128 && H != 256) return false;
  const bool fp8 = kdt == LSA_E4M3;
  if (fp8 && H > 128) return false;   // hi and lo heads share one MMA: N = 2H <= 256
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
  const dim3 ig(fp8 ? (s.H + 7) / 8 : (s.H * s.dI / 8 + 255) / 256, s.B * s.nL);
  if (fp8)
    launch_dependent(build_qimg_fp8_kernel, ig, dim3(256), 0, st, static_cast<const __nv_bfloat16*>(s.q), s.w, s.B,
                     s.H, s.dI, s.l0, a.qimg, a.wfold);
  else
    launch_dependent(build_qimg_bf16_kernel, ig, dim3(256), 0, st, static_cast<const __nv_bfloat16*>(s.q), s.w, s.B,
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
  return fp8 ? launch_h<true>(map, p, lay, grid, st) : launch_h<false>(map, p, lay, grid, st);
}

}  // namespace lsa
