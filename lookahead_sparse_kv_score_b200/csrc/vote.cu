// Cross-layer majority-vote labels and their BCE + focal loss.
//
// Technical summary of FlashMemory-DeepSeek-V4 (gist.science), §2.2: the indexer logits
// of each layer are turned into probabilities with a softmax, each layer keeps its
// high-confidence entries by nucleus (top-p, p = 0.6) selection, and an entry is a
// golden label when at least theta = 3 of the L layers select it.  §2.3: the indexer
// is trained with binary cross-entropy plus a focal loss.
//
// Nucleus of one row (layer l, position p) over N entries, without sorting the row:
//   pi_s = e_s / Z with e_s = exp(x_s - c) for a constant c near max x (fp32 exp, fp64
//   sums).  In descending order of x (equal x: lower index first) an entry is selected
//   iff the mass before it is < top_p * Z.  Since pi is increasing in x, the boundary
//   is a threshold key T on the order-preserving integer image of x plus a cutoff index
//   among the entries tied at T.  The kernel finds the crossing inside a short run of
//   candidate entries located by a count-only histogram (window_nucleus below) and
//   falls back to a mass-weighted radix select over the whole row (radix_nucleus) for
//   rows the window does not resolve.
#include <algorithm>
#include <cmath>
#include <type_traits>

#include "lsa_common.cuh"

namespace lsa {
namespace {

#ifndef LSA_VOTE_THREADS
#define LSA_VOTE_THREADS 512
#endif
constexpr int kRowThreads = LSA_VOTE_THREADS;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kBins = 256;            // radix digit bins of the whole-row select
constexpr int kFineBins = 4096;       // linear bins of the candidate window
constexpr int kListCap = 8192;        // candidates resolved exactly in shared memory
constexpr float kHeadroom = 4.0f;     // window extent above the sampled maximum
constexpr int kSubBins = 1024;      // second-level bins over the run
constexpr int kHistInts = kFineBins + 32;   // bins plus a trash bin for entries outside the window
constexpr int kFineSmem = kHistInts * 4 + kListCap * 8;
constexpr int kRadixSmem = kRowWarps * kBins * 12;
constexpr int kRowSmem = kFineSmem > kRadixSmem ? kFineSmem : kRadixSmem;
static_assert(kFineBins % kRowThreads == 0, "bins per thread");
static_assert(kSubBins % kRowThreads == 0, "sub-bins per thread");
static_assert(kSubBins * 12 <= kHistInts * 4, "sub-bins reuse the histogram");

__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Selection words of a row (workspace) are kept in blocked order, which one ballot per
// element of a warp's float4 loads produces directly: for the 128 entries
// 128j .. 128j+127, word 4j + e holds in bit i the entry 128j + 4i + e.  A row has
// 4 ceil(N / 128) words; vote_count_kernel returns the labels to entry order.
__device__ __forceinline__ size_t sel_word(uint32_t idx) { return 4 * static_cast<size_t>(idx >> 7) + (idx & 3); }
__device__ __forceinline__ uint32_t sel_bit(uint32_t idx) { return 1u << ((idx >> 2) & 31); }

// 2^x by the hardware approximation (relative error ~2^-22; flushes denormals).
// e^(x - m) = 2^(x log2 e - m log2 e): one fma and one approximation per entry.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;
// The mass term e^(x - m0) of the window path, given nm = -m0 log2 e; every mass of a
// row's window path (Z, the mass above the run, the run's entries) uses this one form.
__device__ __forceinline__ float win_term(float x, float nm) { return ex2_approx(fmaf(x, kLog2e, nm)); }

// Paired fp32 arithmetic (one instruction for two lanes of values, each rounded as the
// scalar instruction rounds it).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  unsigned long long ra, rb, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}

// max(a, b, c) in one instruction; like fmaxf, a NaN operand is ignored.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// One count into the shared-memory histogram at a 32-bit shared address.
__device__ __forceinline__ void red_shared_inc(uint32_t addr) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr) : "memory");
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, T* tmp, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  T r = tmp[0];
#pragma unroll 8
  for (int w = 1; w < kRowWarps; ++w) r = op(r, tmp[w]);
  __syncthreads();
  return r;
}

// Exclusive prefix over threads (in thread order) of two fp64 values at once.
__device__ __forceinline__ void block_scan2(double a, double b, double2* tmp, double& ea, double& eb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double ta = __shfl_up_sync(0xffffffffu, ia, o), tb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) { ia += ta; ib += tb; }
  }
  double xa = __shfl_up_sync(0xffffffffu, ia, 1), xb = __shfl_up_sync(0xffffffffu, ib, 1);
  if (lane == 0) { xa = 0.0; xb = 0.0; }
  if (lane == 31) tmp[warp] = make_double2(ia, ib);
  __syncthreads();
  double wa = 0.0, wb = 0.0;
  for (int w = 0; w < warp; ++w) { wa += tmp[w].x; wb += tmp[w].y; }
  __syncthreads();
  ea = wa + xa;
  eb = wb + xb;
}

// Exclusive prefix over threads (in thread order) of two fp32 values at once.
__device__ __forceinline__ void block_scan2f(float a, float b, float2* tmp, float& ea, float& eb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float ta = __shfl_up_sync(0xffffffffu, ia, o), tb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) { ia += ta; ib += tb; }
  }
  float xa = __shfl_up_sync(0xffffffffu, ia, 1), xb = __shfl_up_sync(0xffffffffu, ib, 1);
  if (lane == 0) { xa = 0.f; xb = 0.f; }
  if (lane == 31) tmp[warp] = make_float2(ia, ib);
  __syncthreads();
  float wa = 0.f, wb = 0.f;
  for (int w = 0; w < warp; ++w) { wa += tmp[w].x; wb += tmp[w].y; }
  __syncthreads();
  ea = wa + xa;
  eb = wb + xb;
}

// Four consecutive logits starting at s (s % 4 == 0); entries at or beyond N read NaN
// and are skipped by the callers' s + j < N checks.
__device__ __forceinline__ float4 load4(const float* x, int s, int N, bool vec) {
  if (vec && s + 3 < N) return __ldg(reinterpret_cast<const float4*>(x + s));
  float4 v = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                         __int_as_float(0x7fc00000));
  if (s < N) v.x = x[s];
  if (s + 1 < N) v.y = x[s + 1];
  if (s + 2 < N) v.z = x[s + 2];
  if (s + 3 < N) v.w = x[s + 3];
  return v;
}

// 16-byte read-only loads with an L2 eviction priority: a row's first pass keeps it in
// L2 for the second (evict_last), the second pass is its last use (evict_first).
__device__ __forceinline__ uint64_t l2_policy_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ float4 ldg4_hint(const float4* p, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

// Ascending bitonic sort of n entries (n a power of two, >= 64).  Stages whose partner
// distance is below 64 stay inside 64-entry blocks, one warp per block, with warp
// barriers only.
__device__ void bitonic_sort(unsigned long long* a, int n) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto local = [&](int kmin, int kmax) {
    for (int blk = warp; blk < n / 64; blk += kRowWarps) {
      unsigned long long* b = a + blk * 64;
      const int base = blk * 64;
      for (int k = kmin; k <= kmax; k <<= 1) {
        for (int j = (k >> 1) < 32 ? (k >> 1) : 32; j > 0; j >>= 1) {
          const int i = ((lane & ~(j - 1)) << 1) | (lane & (j - 1));
          const unsigned long long u = b[i], v = b[i | j];
          if ((u > v) == (((base + i) & k) == 0)) { b[i] = v; b[i | j] = u; }
          __syncwarp();
        }
      }
    }
  };
  local(2, 64);
  __syncthreads();
  for (int k = 128; k <= n; k <<= 1) {
    for (int j = k >> 1; j >= 64; j >>= 1) {
      for (int q = tid; q < n / 2; q += kRowThreads) {
        const int i = ((q & ~(j - 1)) << 1) | (q & (j - 1));
        const unsigned long long u = a[i], v = a[i | j];
        if ((u > v) == ((i & k) == 0)) { a[i] = v; a[i | j] = u; }
      }
      __syncthreads();
    }
    local(k, k);
    __syncthreads();
  }
}

struct RowShared {
  float ftmp[32];
  double dtmp[32];
  int itmp[32];
  double2 d2tmp[32];
  float2 f2tmp[32];
  double bin_mass[kBins];
  int bin_cnt[kBins];
  double above, target;
  int sel, cnt, cut, tie_base, ilo, ihi, count, jstar, sstar;
  int nsel;
  double before;               // mass before the crossing sub-bin
  unsigned long long last;     // the last selected entry of the run
  unsigned long long sub[32];  // the crossing sub-bin's entries
};

// Nucleus threshold of one row by a radix select over all N keys (four 8-bit digits,
// most significant first) whose histograms carry counts and mass.  Used when the
// candidate window does not apply: top_p = 1, non-finite logits, or more than
// kListCap entries in the window's crossing bins (heavily tied rows).  Returns
// (T, cut): an entry is selected iff key > T, or key == T and index <= cut.
__device__ int2 radix_nucleus(const float* x, int N, float m, float top_p, uint8_t* dsm, RowShared& sh) {
  double* hmass = reinterpret_cast<double*>(dsm);                          // [warps][256]
  int* hcnt = reinterpret_cast<int*>(hmass + kRowWarps * kBins);           // [warps][256]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
      sh.bin_mass[tid] = ms;
      sh.bin_cnt[tid] = c;
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
        loc += sh.bin_mass[b];
        nonempty |= sh.bin_cnt[b] > 0;
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
      const double tgt = pass == 0 ? static_cast<double>(top_p) * total : sh.target;
      const double base = pass == 0 ? 0.0 : sh.above;
      const unsigned reach = __ballot_sync(0xffffffffu, nonempty && base + incl >= tgt);
      const unsigned ne = __ballot_sync(0xffffffffu, nonempty);
      const int owner = reach ? __ffs(reach) - 1 : 31 - __clz(ne ? ne : 1u);
      if (lane == owner) {
        double cum = base + excl;
        int sel = -1;
        for (int i = 0; i < 8; ++i) {
          const int b = kBins - 1 - (8 * lane + i);
          if (sh.bin_cnt[b] == 0) continue;
          if (reach && cum + sh.bin_mass[b] >= tgt) { sel = b; break; }
          sel = b;                       // no reach: ends at the lowest non-empty bin
          cum += sh.bin_mass[b];
        }
        if (!reach) cum -= sh.bin_mass[sel];   // mass strictly above the selected bin
        sh.sel = sel;
        sh.above = cum;
        sh.cnt = sh.bin_cnt[sel];
        if (pass == 0) sh.target = tgt;
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sh.sel) << shift;
    hmask |= 255u << shift;
    above = sh.above;
    target = sh.target;
    cnt_final = sh.cnt;
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
    if (tid == 0) { sh.cut = N; sh.tie_base = 0; }
    __syncthreads();
    for (int s0 = 0; s0 < N; s0 += kRowThreads) {
      const int s = s0 + tid;
      const bool tie = s < N && order_key(x[s]) == T;
      const unsigned b = __ballot_sync(0xffffffffu, tie);
      if (lane == 0) hcnt[warp] = __popc(b);
      __syncthreads();
      int before = sh.tie_base;
      for (int w = 0; w < warp; ++w) before += hcnt[w];
      before += __popc(b & ((1u << lane) - 1));
      if (tie && before + 1 == want) sh.cut = s;
      __syncthreads();
      if (tid == 0) {
        int tot = 0;
        for (int w = 0; w < kRowWarps; ++w) tot += hcnt[w];
        sh.tie_base += tot;
      }
      __syncthreads();
      if (sh.cut < N) break;
    }
    cut = sh.cut;
    __syncthreads();
  }
  return make_int2(static_cast<int>(T), cut);
}

// Crossing inside a gathered run of C entries (list: ~key << 32 | index) by a full
// sort: the run sorted by (key descending, index ascending), its mass scanned in that
// order; the first entry whose mass before reaches the target is the first one not
// selected.  The selected entries are or-ed into the row's words.
__device__ bool sorted_run_crossing(unsigned long long* list, int C, double above, double target, float m0,
                                    RowShared& sh, uint32_t* out, int2& res) {
  const int tid = threadIdx.x;
  int P2 = 64;
  while (P2 < C) P2 <<= 1;
  for (int i = C + tid; i < P2; i += kRowThreads) list[i] = ~0ull;
  __syncthreads();
  bitonic_sort(list, P2);
  const float nm = -m0 * kLog2e;
  const int chunk = (C + kRowThreads - 1) / kRowThreads;
  const int j0 = tid * chunk < C ? tid * chunk : C, j1 = j0 + chunk < C ? j0 + chunk : C;
  double loc = 0.0;
  for (int j = j0; j < j1; ++j) loc += static_cast<double>(win_term(key_value(~static_cast<uint32_t>(list[j] >> 32)), nm));
  double ex, ex2;
  block_scan2(loc, 0.0, sh.d2tmp, ex, ex2);
  if (tid == 0) sh.jstar = C + 1;     // C + 1: the crossing lies below the run
  __syncthreads();
  {
    double run = ex;
    for (int j = j0; j < j1; ++j) {
      if (above + run >= target) { atomicMin(&sh.jstar, j); break; }
      run += static_cast<double>(win_term(key_value(~static_cast<uint32_t>(list[j] >> 32)), nm));
    }
    // every entry of the run selected, the first one below it not
    if (j1 == C && j0 < j1 && above + run >= target) atomicMin(&sh.jstar, C);
  }
  __syncthreads();
  const int js = sh.jstar;
  if (js == 0 || js > C) return false;
  for (int j = tid; j < js; j += kRowThreads) {
    const uint32_t idx = static_cast<uint32_t>(list[j] & 0xffffffffu);
    atomicOr(&out[sel_word(idx)], sel_bit(idx));
  }
  const unsigned long long last = list[js - 1];
  res = make_int2(static_cast<int>(~static_cast<uint32_t>(last >> 32)), static_cast<int>(last & 0xffffffffu));
  __syncthreads();
  return true;
}

// Nucleus of one row from a candidate window.  Every entry outside the window
// [m - R, m], R = ln(N / (1 - top_p)) + 1, lies below the threshold: their total mass
// is below N e^-R < (1 - top_p) <= (1 - top_p) Z (Z >= 1 counts the maximum itself),
// so the entries inside already hold more than top_p Z.  The window is cut into
// kFineBins linear bins and only counts are histogrammed; with each bin's exponentials
// bounded by its edges, the crossing bin lies in a short run [ilo, ihi] of bins.  A
// second pass sums the exact mass above the run, writes the row's selection words
// (entries above the run set, the run's entries clear) and gathers the run's entries,
// which are sorted by (key descending, index ascending) and scanned for the crossing;
// the selected part of the run is then or-ed into the words.  Returns false when the
// run does not resolve the row (the words are then rewritten by the caller).
__device__ bool window_nucleus(const float* x, int N, bool vec, float top_p, float R, uint8_t* dsm,
                              RowShared& sh, uint32_t* out, int2& res) {
  int* hist = reinterpret_cast<int*>(dsm);
  unsigned long long* list = reinterpret_cast<unsigned long long*>(dsm + kHistInts * 4);
  const int tid = threadIdx.x, lane = tid & 31;
  constexpr int kPer = kFineBins / kRowThreads;
  const int G = (N + 3) >> 2;
  const int Gf = vec ? (N >> 2) : 0;   // float4 groups read without checks
  // anchor: the maximum of the first 4 * kRowThreads logits, plus headroom
  float m0;
  {
    const float4 v = load4(x, 4 * tid, N, vec);
    float mv = -INFINITY;
    if (4 * tid < N) mv = v.x;
    if (4 * tid + 1 < N) mv = fmaxf(mv, v.y);
    if (4 * tid + 2 < N) mv = fmaxf(mv, v.z);
    if (4 * tid + 3 < N) mv = fmaxf(mv, v.w);
    m0 = block_reduce(mv, sh.ftmp, [](float a, float b) { return fmaxf(a, b); });
  }
  if (!isfinite(m0)) return false;
  const float inv_w = static_cast<float>(kFineBins) / (R + kHeadroom);
  float m = -INFINITY;
  double Z = 0.0;
  float a = 0.f;
  for (int attempt = 0; attempt < 2; ++attempt) {
    a = attempt == 0 ? m0 + kHeadroom : m;
    for (int i = tid; i < kHistInts; i += kRowThreads) hist[i] = 0;
    __syncthreads();
    float mloc = -INFINITY;
    double zloc = 0.0;
    // Entries above a (only when the row gets re-anchored) and NaN spoil Z, which is
    // then discarded; entries outside the window land in the trash bin.
    // a inv_w rounded up: every x <= a then gets t >= 0, bin 0 included.  The bin of x:
    // u = sat((a inv_w - x inv_w) / kFineBins) by one saturating fma, then
    // 2^23 + floor(u kFineBins) by a round-down fma; that float's bit pattern times 4
    // plus a constant is the bin's shared-memory address (u = 1: the trash bin).
    const float ainv = __fmul_ru(a, inv_w);
    const float c1 = -inv_w / kFineBins, c0 = ainv / kFineBins;
    const uint32_t hbase = static_cast<uint32_t>(__cvta_generic_to_shared(hist)) - 0x4B000000u * 4u;
    const float nm = -m0 * kLog2e;
    auto body = [&](auto full, const float4& v, int s) -> float {
      constexpr bool kFull = decltype(full)::value;
      const float xs[4] = {v.x, v.y, v.z, v.w};
      float ez = 0.f;              // at most four terms <= e^4
      if constexpr (kFull) {
        // two three-input maxima, the exponents' arguments and the sum in pairs
        mloc = fmax3(mloc, xs[0], xs[1]);
        mloc = fmax3(mloc, xs[2], xs[3]);
        const float2 l2 = make_float2(kLog2e, kLog2e), n2 = make_float2(nm, nm);
        const float2 a01 = ffma2(make_float2(xs[0], xs[1]), l2, n2), a23 = ffma2(make_float2(xs[2], xs[3]), l2, n2);
        const float2 e = fadd2(make_float2(ex2_approx(a01.x), ex2_approx(a01.y)),
                               make_float2(ex2_approx(a23.x), ex2_approx(a23.y)));
        ez = e.x + e.y;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (kFull || s + j < N) {
          if constexpr (!kFull) {
            mloc = fmaxf(mloc, xs[j]);
            ez += ex2_approx(fmaf(xs[j], kLog2e, nm));
          }
          const float u = __saturatef(fmaf(xs[j], c1, c0));
          red_shared_inc(__float_as_uint(__fmaf_rd(u, static_cast<float>(kFineBins), 8388608.f)) * 4u + hbase);
        }
      }
      return ez;
    };
    int g0 = tid;
    const uint64_t keep = l2_policy_last();
    for (; g0 + 3 * kRowThreads < Gf; g0 += 4 * kRowThreads) {
      float4 v4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v4[u] = ldg4_hint(reinterpret_cast<const float4*>(x) + g0 + u * kRowThreads, keep);
      float ez = 0.f;              // sixteen terms in fp32, then the fp64 sum
#pragma unroll
      for (int u = 0; u < 4; ++u) ez += body(std::true_type{}, v4[u], 4 * (g0 + u * kRowThreads));
      zloc += static_cast<double>(ez);
    }
    for (; g0 < G; g0 += 4 * kRowThreads) {
      float4 v4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v4[u] = load4(x, 4 * (g0 + u * kRowThreads), N, vec);
      float ez = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) ez += body(std::false_type{}, v4[u], 4 * (g0 + u * kRowThreads));
      zloc += static_cast<double>(ez);
    }
    m = block_reduce(mloc, sh.ftmp, [](float p, float q) { return fmaxf(p, q); });
    Z = block_reduce(zloc, sh.dtmp, [](double p, double q) { return p + q; });
    if (!isfinite(m)) return false;
    if (m <= a) break;
    if (attempt == 1) return false;
    m0 = m - kHeadroom;           // a maximum above the headroom: re-anchor at it
  }
  if (!(Z > 0.0) || !isfinite(Z)) return false;
  const double target = static_cast<double>(top_p) * Z;
  // Bounds of each bin's mass from its edges: half a bin of slack for rounding in
  // fine_bin, 2^-10 relative for the fp32 exponentials and these fp32 sums (whose own
  // rounding stays below 3e-6 relative).  Only the run's extent depends on them: the
  // crossing found inside it is checked exactly below.
  const float w = 1.f / inv_w;
  const float A = static_cast<float>(static_cast<double>(a) - static_cast<double>(m0));
  const float targetf = static_cast<float>(target);
  const int b0 = tid * kPer;
  int cnt[kPer];
  float lo[kPer], hi[kPer], slo = 0.f, shi = 0.f;
  {
    const float r = expf(-w);
    float ehi = expf(A - (b0 - 0.5f) * w) * (1.f + 1.f / 1024.f);
    float elo = expf(A - (b0 + 1.5f) * w) * (1.f - 1.f / 1024.f);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      cnt[i] = hist[b0 + i];
      hi[i] = cnt[i] * ehi;
      lo[i] = cnt[i] * elo;
      shi += hi[i];
      slo += lo[i];
      ehi *= r;
      elo *= r;
    }
  }
  float chi, clo;
  block_scan2f(shi, slo, sh.f2tmp, chi, clo);
  if (tid == 0) { sh.ilo = kFineBins; sh.ihi = kFineBins - 1; }
  __syncthreads();
  {
    int ilo = kFineBins, ihi = kFineBins;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      chi += hi[i];
      clo += lo[i];
      if (ilo == kFineBins && cnt[i] > 0 && chi >= targetf) ilo = b0 + i;
      if (ihi == kFineBins && cnt[i] > 0 && clo >= targetf) ihi = b0 + i;
    }
    if (ilo < kFineBins) atomicMin(&sh.ilo, ilo);
    if (ihi < kFineBins) atomicMin(&sh.ihi, ihi);
  }
  __syncthreads();
  const int ilo = sh.ilo, ihi = sh.ihi;
  if (ilo >= kFineBins || ihi < ilo) return false;
  int c = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) c += (b0 + i >= ilo && b0 + i <= ihi) ? cnt[i] : 0;
  const int Cbins = block_reduce(c, sh.itmp, [](int p, int q) { return p + q; });
  if (Cbins > kListCap || Cbins == 0) return false;
  // Exact mass above the run, the row's words, the run's entries.  The pass splits the
  // row at two thresholds in x placed at the run's bin edges; any split monotone in x
  // serves, since the crossing found among the gathered entries is checked exactly
  // against the mass above them.
  const float xu = a - static_cast<float>(ilo) * w;        // above the run: x > xu
  const float xl = a - static_cast<float>(ihi + 1) * w;    // in the run: xl < x <= xu
  if (tid == 0) sh.count = 0;
  __syncthreads();
  double aloc = 0.0;
  {
    // A warp's lanes hold 32 consecutive float4 groups, i.e. one 128-entry block: one
    // ballot per element gives that block's four selection words (blocked order).
    const int Gr = (G + 31) & ~31;      // whole warps per iteration
    const float nm = -m0 * kLog2e;
    auto body = [&](auto full, const float4& v, int s) -> float {
      constexpr bool kFull = decltype(full)::value;
      const float xs[4] = {v.x, v.y, v.z, v.w};   // NaN past N: neither above nor in the run
      float ea = 0.f;
      uint32_t wd[4];
      uint32_t runm = 0;
      const float2 l2 = make_float2(kLog2e, kLog2e), n2 = make_float2(nm, nm);
      const float2 a01 = ffma2(make_float2(xs[0], xs[1]), l2, n2), a23 = ffma2(make_float2(xs[2], xs[3]), l2, n2);
      const float arg[4] = {a01.x, a01.y, a23.x, a23.y};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool up = (kFull || s + j < N) && xs[j] > xu;
        wd[j] = __ballot_sync(0xffffffffu, up);
        const float e = ex2_approx(arg[j]);
        if (up) ea += e;
        runm |= (!up && xs[j] > xl) ? (1u << j) : 0u;
      }
      if (runm) {   // the run's entries (a fraction of a percent): each takes its own list slot
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (runm & (1u << j)) {
            const int at = atomicAdd(&sh.count, 1);
            if (at < kListCap)
              list[at] = (static_cast<unsigned long long>(~order_key(xs[j])) << 32) | static_cast<uint32_t>(s + j);
          }
      }
      if (lane == 0 && s < N) *reinterpret_cast<uint4*>(out + 4 * (s >> 7)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      return ea;
    };
    int g0 = tid;
    const uint64_t last = l2_policy_first();
    // whole warps whose four groups are all full
    for (; (g0 - lane) + 31 + 3 * kRowThreads < Gf; g0 += 4 * kRowThreads) {
      float4 v4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v4[u] = ldg4_hint(reinterpret_cast<const float4*>(x) + g0 + u * kRowThreads, last);
      float ea = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) ea += body(std::true_type{}, v4[u], 4 * (g0 + u * kRowThreads));
      aloc += static_cast<double>(ea);
    }
    for (; g0 < Gr; g0 += 4 * kRowThreads) {
      float4 v4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v4[u] = load4(x, 4 * (g0 + u * kRowThreads), N, vec);
      float ea = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) ea += body(std::false_type{}, v4[u], 4 * (g0 + u * kRowThreads));
      aloc += static_cast<double>(ea);
    }
  }
  const double above = block_reduce(aloc, sh.dtmp, [](double p, double q) { return p + q; });
  const int C = sh.count;
  if (!(above < target) || C == 0 || C > kListCap) return false;
  // Second level: the run's entries in kSubBins sub-bins by x (monotone, so every entry
  // of a sub-bin precedes every entry of a later one), with counts and fp64 mass.  The
  // crossing sub-bin is the first whose cumulative mass reaches the target; its few
  // entries are ranked by (key descending, index ascending) in one warp.
  int* scnt = hist;
  double* smass = reinterpret_cast<double*>(dsm + kSubBins * 4);
  const float nm = -m0 * kLog2e;
  const float inv_ws = static_cast<float>(kSubBins) / fmaxf(xu - xl, 1e-30f);
  auto sub_bin = [&](unsigned long long ent) {
    const float xv = key_value(~static_cast<uint32_t>(ent >> 32));
    const int sb = __float_as_int(__fadd_rd((xu - xv) * inv_ws, 8388608.f)) - 0x4B000000;
    return sb < 0 ? 0 : (sb >= kSubBins ? kSubBins - 1 : sb);
  };
  for (int i = tid; i < kSubBins; i += kRowThreads) { scnt[i] = 0; smass[i] = 0.0; }
  if (tid == 0) { sh.sstar = kSubBins; sh.nsel = 0; }
  __syncthreads();
  for (int j = tid; j < C; j += kRowThreads) {
    const unsigned long long ent = list[j];
    const int sb = sub_bin(ent);
    atomicAdd(&scnt[sb], 1);
    atomicAdd(&smass[sb], static_cast<double>(win_term(key_value(~static_cast<uint32_t>(ent >> 32)), nm)));
  }
  __syncthreads();
  constexpr int kSubPer = kSubBins / kRowThreads;
  const int s0 = tid * kSubPer;
  double ms[kSubPer], sloc = 0.0;
#pragma unroll
  for (int i = 0; i < kSubPer; ++i) { ms[i] = smass[s0 + i]; sloc += ms[i]; }
  double sex, sex2;
  block_scan2(sloc, 0.0, sh.d2tmp, sex, sex2);
  {
    double cum = above + sex;
#pragma unroll
    for (int i = 0; i < kSubPer; ++i) {
      if (cum + ms[i] >= target) { atomicMin(&sh.sstar, s0 + i); break; }
      cum += ms[i];
    }
  }
  __syncthreads();
  const int S = sh.sstar;
  if (S >= kSubBins) return false;    // the crossing lies below the run
  if (tid == S / kSubPer) {           // only the owner of S holds the sum before it
    double cum = above + sex;
    for (int i = 0; i < S - s0; ++i) cum += ms[i];
    sh.before = cum;
  }
  const int nS = scnt[S];
  if (nS > 32) return sorted_run_crossing(list, C, above, target, m0, sh, out, res);   // dense: sort the run
  for (int j = tid; j < C; j += kRowThreads) {
    const unsigned long long ent = list[j];
    if (sub_bin(ent) == S) {
      const int at = atomicAdd(&sh.nsel, 1);
      if (at < 32) sh.sub[at] = ent;
    }
  }
  __syncthreads();
  if (tid < 32) {
    const unsigned long long mine = lane < nS ? sh.sub[lane] : ~0ull;
    const double em =
        lane < nS ? static_cast<double>(win_term(key_value(~static_cast<uint32_t>(mine >> 32)), nm)) : 0.0;
    double mb = 0.0;                  // mass of the sub-bin's entries before this one
    for (int o = 0; o < nS; ++o) {
      const unsigned long long other = __shfl_sync(0xffffffffu, mine, o);
      const double eo = __shfl_sync(0xffffffffu, em, o);
      if (other < mine) mb += eo;
    }
    const bool sel = lane < nS && sh.before + mb < target;
    unsigned long long lastv = sel ? mine : 0ull;   // the largest selected, in sorted order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long t = __shfl_xor_sync(0xffffffffu, lastv, o);
      lastv = t > lastv ? t : lastv;
    }
    if (lane == 0) sh.last = lastv;
  }
  __syncthreads();
  const unsigned long long last = sh.last;
  if (last == 0ull) return false;
  // the selected part of the run: earlier sub-bins, and the crossing sub-bin's entries
  // up to the last selected one
  for (int j = tid; j < C; j += kRowThreads) {
    const unsigned long long ent = list[j];
    const int sb = sub_bin(ent);
    if (sb < S || (sb == S && ent <= last)) {
      const uint32_t idx = static_cast<uint32_t>(ent & 0xffffffffu);
      atomicOr(&out[sel_word(idx)], sel_bit(idx));
    }
  }
  res = make_int2(static_cast<int>(~static_cast<uint32_t>(last >> 32)), static_cast<int>(last & 0xffffffffu));
  __syncthreads();
  return true;
}

// One row per iteration of the block.  selbits [L*P][4 ceil(N/128)] in blocked order;
// rowparam [L*P] = (T, cutoff index).
__global__ void __launch_bounds__(kRowThreads, kRowThreads >= 1024 ? 1 : 2)
vote_rows_kernel(const float* __restrict__ logits, int rows, int N, float top_p, float R,
                 uint32_t* __restrict__ selbits, int2* __restrict__ rowparam) {
  extern __shared__ __align__(16) uint8_t vsm[];
  __shared__ RowShared sh;
  const int tid = threadIdx.x, lane = tid & 31;
  const size_t Nwb = 4 * static_cast<size_t>((N + 127) / 128);   // blocked words per row
  for (int row = blockIdx.x; row < rows; row += gridDim.x) {
    const float* x = logits + static_cast<size_t>(row) * N;
    const bool vec = (N % 4 == 0) && (reinterpret_cast<uintptr_t>(x) % 16 == 0);
    uint32_t* out = selbits + static_cast<size_t>(row) * Nwb;
    int2 tc;
    const bool ok = top_p < 1.f && window_nucleus(x, N, vec, top_p, R, vsm, sh, out, tc);
    if (tid == 0 && ok) rowparam[row] = tc;
    if (ok) continue;   // window_nucleus ends on a block barrier
    float mv = -INFINITY;
    for (int s = tid; s < N; s += kRowThreads) mv = fmaxf(mv, x[s]);
    const float m = block_reduce(mv, sh.ftmp, [](float p, float q) { return fmaxf(p, q); });
    tc = radix_nucleus(x, N, m, top_p, vsm, sh);
    if (tid == 0) rowparam[row] = tc;
    const uint32_t T = static_cast<uint32_t>(tc.x);
    const int cut = tc.y;
    // selection words in blocked order: one ballot per element of a warp's float4 groups
    const int G = (N + 3) >> 2;
    const int Gr = (G + 31) & ~31;
    for (int g0 = tid; g0 < Gr; g0 += 4 * kRowThreads) {
      float4 v4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v4[u] = load4(x, 4 * (g0 + u * kRowThreads), N, vec);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = 4 * (g0 + u * kRowThreads);
        const float xs[4] = {v4[u].x, v4[u].y, v4[u].z, v4[u].w};
        uint32_t wd[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t k = order_key(xs[j]);
          wd[j] = __ballot_sync(0xffffffffu, s + j < N && (k > T || (k == T && s + j <= cut)));
        }
        if (lane == 0 && s < N) *reinterpret_cast<uint4*>(out + 4 * (s >> 7)) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      }
    }
    __syncthreads();
  }
}

// Bits 0..7 of x moved to bits 0, 4, 8, .., 28.
__device__ __forceinline__ uint32_t spread_byte(uint32_t x) {
  x &= 0xFFu;
  x = (x | (x << 12)) & 0x000F000Fu;
  x = (x | (x << 6)) & 0x03030303u;
  x = (x | (x << 3)) & 0x11111111u;
  return x;
}

// Per (position, 128-entry block): the layer counts of its entries as bit-sliced
// counters (plane k holds bit k of every count) over the block's four blocked-order
// selection words, golden bits (count >= theta) turned back into entry order, and the
// optional byte counts.
template <int kPlanes>
__global__ void vote_count_kernel(const uint32_t* __restrict__ selbits, int L, int P, int N, int theta,
                                  uint32_t* __restrict__ golden, uint8_t* __restrict__ counts) {
  const int Nb = (N + 127) / 128;
  const int Nw = (N + 31) / 32;
  const int p = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= Nb) return;
  uint32_t pl[4][kPlanes];
#pragma unroll
  for (int e = 0; e < 4; ++e)
#pragma unroll
    for (int k = 0; k < kPlanes; ++k) pl[e][k] = 0u;
  const uint4* src = reinterpret_cast<const uint4*>(selbits) + static_cast<size_t>(p) * Nb + j;
  const size_t stride = static_cast<size_t>(P) * Nb;
  auto add = [&](uint32_t carry, uint32_t* plane) {
#pragma unroll
    for (int k = 0; k < kPlanes; ++k) {
      const uint32_t t = plane[k] & carry;
      plane[k] ^= carry;
      carry = t;
    }
  };
  int l = 0;
  constexpr int kLoads = 8;    // layers' words in flight together
  for (; l + kLoads <= L; l += kLoads) {
    uint4 bw[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i) bw[i] = __ldg(src + (l + i) * stride);
#pragma unroll
    for (int i = 0; i < kLoads; ++i) {
      add(bw[i].x, pl[0]); add(bw[i].y, pl[1]); add(bw[i].z, pl[2]); add(bw[i].w, pl[3]);
    }
  }
  for (; l < L; ++l) {
    const uint4 b = __ldg(src + l * stride);
    add(b.x, pl[0]); add(b.y, pl[1]); add(b.z, pl[2]); add(b.w, pl[3]);
  }
  // count >= theta  <=>  no borrow out of count - theta (0 < theta < 2^kPlanes)
  uint32_t g[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    if (theta <= 0) {
      g[e] = 0xffffffffu;
    } else if (theta >= (1 << kPlanes)) {
      g[e] = 0u;
    } else {
      uint32_t borrow = 0u;
#pragma unroll
      for (int k = 0; k < kPlanes; ++k)
        borrow = ((theta >> k) & 1) ? (~pl[e][k] | borrow) : (~pl[e][k] & borrow);
      g[e] = ~borrow;
    }
  }
  // entry order: bit 4k + e of word 4j + m is entry 128j + 32m + 4k + e = 128j + 4(8m + k) + e,
  // i.e. bit 8m + k of blocked word e
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int w = 4 * j + m;
    if (w >= Nw) break;
    uint32_t gw = spread_byte(g[0] >> (8 * m)) | (spread_byte(g[1] >> (8 * m)) << 1) |
                  (spread_byte(g[2] >> (8 * m)) << 2) | (spread_byte(g[3] >> (8 * m)) << 3);
    const int valid = N - w * 32;
    if (valid < 32) gw &= (1u << valid) - 1u;
    golden[static_cast<size_t>(p) * Nw + w] = gw;
  }
  if (counts) {
    // byte 128j + 4i + e = count of blocked word e, bit i
    uint8_t* c = counts + static_cast<size_t>(p) * N + static_cast<size_t>(j) * 128;
    const int valid = N - j * 128;
    const bool vec = valid >= 128 && (reinterpret_cast<uintptr_t>(c) & 15) == 0;
#pragma unroll
    for (int i4 = 0; i4 < 32; i4 += 4) {
      uint32_t v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i4 + q;
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t cnt = 0;
#pragma unroll
          for (int k = 0; k < kPlanes; ++k) cnt |= ((pl[e][k] >> i) & 1u) << k;
          word |= cnt << (8 * e);
        }
        v[q] = word;
      }
      if (vec) {
        reinterpret_cast<uint4*>(c)[i4 / 4] = make_uint4(v[0], v[1], v[2], v[3]);
      } else {
        for (int q = 0; q < 4; ++q)
          for (int e = 0; e < 4; ++e) {
            const int at = 4 * (i4 + q) + e;
            if (at < valid) c[at] = static_cast<uint8_t>(v[q] >> (8 * e));
          }
      }
    }
  }
}

// Sums of the BCE and focal terms over all P*N entries, then means.  One logarithm per
// entry, of the probability of its label: ln p for a golden entry, ln(1 - p) otherwise
// (1 - p is exact in fp32 down to p = 2^-24 relative spacing, far below the clamp),
// by the hardware's fast log2 (absolute error ~1e-7 in ln, far below the means'
// tolerance); the focal factor is the squared probability of the other label.  Terms
// are summed in fp32 over groups of eight entries, the groups in fp64.
__device__ __forceinline__ float focal_pow(float q, float gamma) {
  return gamma == 2.f ? q * q : (gamma == 1.f ? q : (gamma == 0.f ? 1.f : powf(q, gamma)));
}

// acc [2] doubles, then a block counter: the last block to finish writes the means.
__global__ void vote_loss_kernel(const float* __restrict__ scores, const uint32_t* __restrict__ golden, int P,
                                 int N, float gamma, double* __restrict__ acc, double* __restrict__ loss) {
  __shared__ double tmp[2][32];
  const int Nw = (N + 31) / 32;
  const int p = blockIdx.y;
  const float eps = 1.f / 1048576.f;   // 2^-20: probabilities clamped to [eps, 1 - eps]
  const float* sc = scores + static_cast<size_t>(p) * N;
  const uint32_t* gw = golden + static_cast<size_t>(p) * Nw;
  double bce = 0.0, fl = 0.0;
  float gb = 0.f, gf = 0.f;    // the current group's fp32 sums
  auto term = [&](float pr, bool y) {
    pr = fminf(fmaxf(pr, eps), 1.f - eps);
    const float py = y ? pr : 1.f - pr;          // probability of the entry's label
    const float lp = __logf(py);
    gb -= lp;
    gf -= focal_pow(1.f - py, gamma) * lp;
  };
  const int stride = gridDim.x * blockDim.x;
  if ((N & 7) == 0 && (reinterpret_cast<uintptr_t>(sc) & 15) == 0) {
    const int G = N >> 3;       // groups of eight entries: two float4 and one byte of labels
    constexpr int kGroups = 2;  // groups whose loads are in flight together
    for (int g0 = blockIdx.x * blockDim.x + threadIdx.x; g0 < G; g0 += kGroups * stride) {
      float4 a[kGroups], c[kGroups];
      uint32_t bits[kGroups];
#pragma unroll
      for (int u = 0; u < kGroups; ++u) {
        const int g = g0 + u * stride;
        if (g < G) {
          a[u] = __ldg(reinterpret_cast<const float4*>(sc) + 2 * g);
          c[u] = __ldg(reinterpret_cast<const float4*>(sc) + 2 * g + 1);
          bits[u] = __ldg(gw + (g >> 2)) >> (8 * (g & 3));
        }
      }
#pragma unroll
      for (int u = 0; u < kGroups; ++u) {
        if (g0 + u * stride >= G) break;
        gb = 0.f;
        gf = 0.f;
        term(a[u].x, bits[u] & 1u);
        term(a[u].y, (bits[u] >> 1) & 1u);
        term(a[u].z, (bits[u] >> 2) & 1u);
        term(a[u].w, (bits[u] >> 3) & 1u);
        term(c[u].x, (bits[u] >> 4) & 1u);
        term(c[u].y, (bits[u] >> 5) & 1u);
        term(c[u].z, (bits[u] >> 6) & 1u);
        term(c[u].w, (bits[u] >> 7) & 1u);
        bce += static_cast<double>(gb);
        fl += static_cast<double>(gf);
      }
    }
  } else {
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < N; s += stride) {
      gb = 0.f;
      gf = 0.f;
      term(__ldg(sc + s), (__ldg(gw + (s >> 5)) >> (s & 31)) & 1u);
      bce += static_cast<double>(gb);
      fl += static_cast<double>(gf);
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
    __threadfence();
    unsigned int* done = reinterpret_cast<unsigned int*>(acc + 2);
    if (atomicAdd(done, 1u) == gridDim.x * gridDim.y - 1) {   // every other block's sums are in
      __threadfence();
      const double n = static_cast<double>(P) * N;
      loss[0] = *reinterpret_cast<volatile double*>(&acc[0]) / n;
      loss[1] = *reinterpret_cast<volatile double*>(&acc[1]) / n;
    }
  }
}

}  // namespace

int launch_vote(const VoteArgs& a, cudaStream_t st) {
  const int rows = a.L * a.P;
  int rc = LSA_OK;
  if (rows > 0 && a.N > 0) {
    const int smem = kRowSmem;
    cudaFuncSetAttribute(vote_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int per_sm = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, vote_rows_kernel, kRowThreads, smem);
    per_sm = per_sm < 1 ? 1 : per_sm;
    const int grid = std::min(rows, per_sm * sms);
    // window half-width ln(N / (1 - top_p)) + 1 (unused when top_p = 1)
    const float R = a.top_p < 1.f ? static_cast<float>(std::log(static_cast<double>(a.N) / (1.0 - a.top_p)) + 1.0)
                                  : 0.f;
    vote_rows_kernel<<<grid, kRowThreads, smem, st>>>(a.logits, rows, a.N, a.top_p, R, a.selbits,
                                                      reinterpret_cast<int2*>(a.rowparam));
    if ((rc = check_launch("vote_labels/rows")) != LSA_OK) return rc;
  }
  constexpr int kCountThreads = 128;
  const dim3 cgrid(((a.N + 127) / 128 + kCountThreads - 1) / kCountThreads, a.P);
  if (a.L <= 31)
    vote_count_kernel<5><<<cgrid, kCountThreads, 0, st>>>(a.selbits, a.L, a.P, a.N, a.theta, a.golden, a.counts);
  else
    vote_count_kernel<8><<<cgrid, kCountThreads, 0, st>>>(a.selbits, a.L, a.P, a.N, a.theta, a.golden, a.counts);
  if ((rc = check_launch("vote_labels/count")) != LSA_OK) return rc;
  if (a.scores) {
    cudaMemsetAsync(a.lossacc, 0, 3 * sizeof(double), st);   // the two sums and the block counter
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int per_row = std::max(1, std::min((a.N + 1023) / 1024, (4 * sms + a.P - 1) / a.P));
    vote_loss_kernel<<<dim3(per_row, a.P), 256, 0, st>>>(a.scores, a.golden, a.P, a.N, a.gamma, a.lossacc, a.loss);
    if ((rc = check_launch("vote_labels/loss")) != LSA_OK) return rc;
  }
  return LSA_OK;
}

}  // namespace lsa
