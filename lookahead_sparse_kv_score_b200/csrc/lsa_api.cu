// The C ABI of liblsa: argument checks, workspace layout and dispatch to the kernels.
// Every entry point is declared and documented in include/lsa.h.
#include <stdarg.h>
#include <stdio.h>

#include <algorithm>
#include <atomic>

#include <cstdlib>
#include <cstring>

#include "lsa_common.cuh"

namespace lsa {

static thread_local char g_err[512] = "";
static std::atomic<unsigned long long> g_launches{0};

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_err[0] = 0; }

// Host-side fault injection for the error-path tests: with LSA_FAULT=launch in the
// environment every launch check reports a failed launch (read once per process).
static bool injected_launch_fault() {
  static const bool on = [] {
    const char* v = std::getenv("LSA_FAULT");
    return v != nullptr && std::strcmp(v, "launch") == 0;
  }();
  return on;
}

int check_launch(const char* what, int kernels) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(LSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  if (injected_launch_fault()) return fail(LSA_ERR_CUDA, "%s: injected launch failure (LSA_FAULT=launch)", what);
  g_launches.fetch_add(static_cast<unsigned long long>(kernels), std::memory_order_relaxed);
  return LSA_OK;
}

static size_t esize(int dt) { return dt == LSA_F32 ? 4 : dt == LSA_BF16 ? 2 : 1; }
static bool valid_dtype(int dt) { return dt == LSA_F32 || dt == LSA_BF16 || dt == LSA_E4M3; }

// Workspace of lsa_index_score: regions in this order, each 1024-byte aligned.
struct ScoreWs {
  size_t partA, partW, partB, cbuf, q, w, qimg, wfold, total;
};

static ScoreWs score_ws(int B, int L, int D, int r, int H, int dI, int wdt, int kdt) {
  ScoreWs o{};
  const size_t BL = static_cast<size_t>(B) * L;
  const size_t SA = project_splits(D), SB = project_splits_b(r);
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off = align_up(off + bytes, 1024); return at; };
  o.partA = take(SA * BL * r * 4);
  o.partW = take(SA * BL * H * 4);
  o.partB = take(SB * BL * H * dI * 4);
  o.cbuf = take(BL * r * 4);
  o.q = take(BL * H * dI * esize(wdt));
  o.w = take(BL * H * 4);
  const bool tc = tc_supported(H, dI, wdt, kdt);
  o.qimg = take(tc ? BL * tc_image_bytes(H, dI, kdt) : 0);
  o.wfold = take(tc ? BL * H * 4 : 0);
  o.total = off;
  return o;
}

}  // namespace lsa

using namespace lsa;

extern "C" {

const char* lsa_status_string(int status) {
  switch (status) {
    case LSA_OK: return "ok";
    case LSA_ERR_INVALID_ARG: return "invalid argument";
    case LSA_ERR_UNSUPPORTED: return "unsupported dtype or shape";
    case LSA_ERR_CAPACITY: return "list longer than its capacity";
    case LSA_ERR_NOMEM: return "workspace too small";
    case LSA_ERR_CUDA: return "CUDA error";
    case LSA_ERR_TIMEOUT: return "bounded wait timed out";
    case LSA_ERR_RANGE: return "entry index out of range";
  }
  return "unknown status";
}

const char* lsa_last_error(void) { return g_err; }

int lsa_abi_version(void) { return 1; }

unsigned long long lsa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

size_t lsa_index_project_workspace_bytes(int B, int L, int D, int r, int H, int dI, int wdt) {
  if (B < 0 || L < 0 || D < 0 || r < 0 || H < 0 || dI < 0) return 0;
  const ScoreWs ws = score_ws(B, L, D, r, H, dI, wdt, LSA_F32);
  return ws.q;   // the projection scratch regions come first
}

int lsa_index_project(int B, int L, int D, int r, int H, int dI, int wdt, const void* h,
                      const void* W_down, const void* W_up, const void* W_w, int layer,
                      void* q_out, float* w_out, void* workspace, size_t workspace_bytes, void* stream) {
  const CallRange range("lsa_index_project");
  g_err[0] = 0;
  if (B < 0 || L < 0 || D <= 0 || r <= 0 || H <= 0 || dI <= 0)
    return fail(LSA_ERR_INVALID_ARG, "index_project: bad size");
  if (wdt != LSA_F32 && wdt != LSA_BF16) return fail(LSA_ERR_UNSUPPORTED, "index_project: wdt %d", wdt);
  if (layer < -1 || layer >= L) return fail(LSA_ERR_INVALID_ARG, "index_project: layer %d of %d", layer, L);
  if (B == 0 || L == 0) return LSA_OK;
  if (layer < 0 && L > 65535)
    return fail(LSA_ERR_UNSUPPORTED, "index_project: %d layers in one call (at most 65535)", L);
  if (!h || !W_down || !W_up || !W_w || !q_out || !w_out)
    return fail(LSA_ERR_INVALID_ARG, "index_project: null pointer");
  const void* ptrs[] = {h, W_down, W_up, W_w, q_out, w_out};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return fail(LSA_ERR_INVALID_ARG, "index_project: pointer %p not 16-byte aligned", p);
  const ScoreWs ws = score_ws(B, L, D, r, H, dI, wdt, LSA_F32);
  if (!workspace || workspace_bytes < ws.q || !aligned(workspace, 256))
    return fail(LSA_ERR_NOMEM, "index_project: workspace %zu bytes (need %zu)", workspace_bytes, ws.q);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  ProjectArgs pa{};
  pa.B = B; pa.L = L; pa.D = D; pa.r = r; pa.H = H; pa.dI = dI; pa.wdt = wdt;
  pa.l0 = layer < 0 ? 0 : layer; pa.nL = layer < 0 ? L : 1;
  pa.h = h; pa.W_down = W_down; pa.W_up = W_up; pa.W_w = W_w;
  pa.partA = reinterpret_cast<float*>(base + ws.partA);
  pa.partW = reinterpret_cast<float*>(base + ws.partW);
  pa.partB = reinterpret_cast<float*>(base + ws.partB);
  pa.cbuf = reinterpret_cast<float*>(base + ws.cbuf);
  pa.q_ws = q_out;          // written directly into the caller's buffers
  pa.w_ws = w_out;
  pa.q_out = nullptr;
  pa.w_out = nullptr;
  pa.do_q = pa.do_w = true;
  return launch_project(pa, static_cast<cudaStream_t>(stream));
}

size_t lsa_index_score_workspace_bytes(int B, int L, int N, int D, int r, int H, int dI, int wdt,
                                       int kdt) {
  (void)N;
  if (B < 0 || L < 0 || D < 0 || r < 0 || H < 0 || dI < 0) return 0;
  return score_ws(B, L, D, r, H, dI, wdt, kdt).total;
}

int lsa_index_score(int B, int L, int N, int D, int r, int H, int dI,
                    int wdt, const void* h, const void* W_down, const void* W_up,
                    const void* W_w, const float* bias,
                    int kdt, const void* K, const float* kscale,
                    int layer,
                    const void* q_in, const float* w_in,
                    void* q_out, float* w_out,
                    uint32_t* mask, float* logit, float* score, int32_t* status,
                    void* workspace, size_t workspace_bytes,
                    void* stream) {
  const CallRange range("lsa_index_score");
  g_err[0] = 0;
  if (B < 0 || L < 0 || N < 0 || D < 0 || r < 0 || H <= 0 || dI <= 0)
    return fail(LSA_ERR_INVALID_ARG, "index_score: negative size or H/dI < 1");
  if (wdt != LSA_F32 && wdt != LSA_BF16) return fail(LSA_ERR_UNSUPPORTED, "index_score: wdt %d", wdt);
  if (!valid_dtype(kdt)) return fail(LSA_ERR_UNSUPPORTED, "index_score: kdt %d", kdt);
  if (layer < -1 || layer >= L) return fail(LSA_ERR_INVALID_ARG, "index_score: layer %d of %d", layer, L);
  if (B == 0 || L == 0) return LSA_OK;
  if (static_cast<long long>(B) * (layer < 0 ? L : 1) > 65535)
    return fail(LSA_ERR_UNSUPPORTED,
                "index_score: B x scored layers = %lld (at most 65535 sequence-layer pairs per call)",
                static_cast<long long>(B) * (layer < 0 ? L : 1));
  if (w_in && !q_in) return fail(LSA_ERR_INVALID_ARG, "index_score: w_in needs q_in");
  const bool need_q = q_in == nullptr, need_w = w_in == nullptr;
  if (need_q && (D <= 0 || r <= 0 || !h || !W_down || !W_up))
    return fail(LSA_ERR_INVALID_ARG, "index_score: projection needs h, W_down, W_up, D, r");
  if (need_w && (D <= 0 || !h || !W_w))
    return fail(LSA_ERR_INVALID_ARG, "index_score: head weights need h, W_w, D");
  if (!bias) return fail(LSA_ERR_INVALID_ARG, "index_score: bias is null");
  if (N > 0 && (!K || !mask)) return fail(LSA_ERR_INVALID_ARG, "index_score: K or mask is null");
  if ((kdt == LSA_E4M3) != (kscale != nullptr))
    return fail(LSA_ERR_INVALID_ARG, "index_score: kscale must be given exactly for e4m3 keys");
  const void* ptrs[] = {h, W_down, W_up, W_w, bias, K, kscale, q_in, w_in, q_out, w_out, mask, logit, score};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return fail(LSA_ERR_INVALID_ARG, "index_score: pointer %p not 16-byte aligned", p);
  const bool tc = tc_supported(H, dI, wdt, kdt);
  if (!tc && static_cast<size_t>(H) * dI > 16384)
    return fail(LSA_ERR_UNSUPPORTED, "index_score: H*dI=%d too large for the CUDA-core path", H * dI);
  if (tc && !aligned(K, 128)) return fail(LSA_ERR_INVALID_ARG, "index_score: K must be 128-byte aligned");
  const ScoreWs ws = score_ws(B, L, D, r, H, dI, wdt, kdt);
  if (!workspace || workspace_bytes < ws.total || !aligned(workspace, 256))
    return fail(LSA_ERR_NOMEM, "index_score: workspace %zu bytes (need %zu, 256-byte aligned)",
                workspace_bytes, ws.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const int l0 = layer < 0 ? 0 : layer, nL = layer < 0 ? L : 1;

  int rc = LSA_OK;
  if (need_q || need_w) {
    ProjectArgs pa{};
    pa.B = B; pa.L = L; pa.D = D; pa.r = r; pa.H = H; pa.dI = dI; pa.wdt = wdt; pa.l0 = l0; pa.nL = nL;
    pa.h = h; pa.W_down = W_down; pa.W_up = W_up; pa.W_w = W_w;
    pa.partA = reinterpret_cast<float*>(base + ws.partA);
    pa.partW = reinterpret_cast<float*>(base + ws.partW);
    pa.partB = reinterpret_cast<float*>(base + ws.partB);
    pa.cbuf = reinterpret_cast<float*>(base + ws.cbuf);
    pa.q_ws = base + ws.q;
    pa.w_ws = reinterpret_cast<float*>(base + ws.w);
    pa.q_out = q_out;
    pa.w_out = w_out;
    pa.do_q = need_q;
    pa.do_w = need_w;
    pa.status = status;
    rc = launch_project(pa, st);
    if (rc != LSA_OK) return rc;
  }
  if (N == 0) return LSA_OK;
  ScoreArgs sa{};
  sa.B = B; sa.L = L; sa.N = N; sa.H = H; sa.dI = dI; sa.wdt = wdt; sa.kdt = kdt; sa.l0 = l0; sa.nL = nL;
  sa.q = need_q ? static_cast<const void*>(base + ws.q) : q_in;
  sa.w = need_w ? reinterpret_cast<const float*>(base + ws.w) : w_in;
  sa.bias = bias; sa.K = K; sa.kscale = kscale;
  sa.mask = mask; sa.logit = logit; sa.score = score;
  if (tc) {
    TcArgs ta{};
    ta.sc = sa;
    ta.qimg = base + ws.qimg;
    ta.wfold = reinterpret_cast<float*>(base + ws.wfold);
    ta.status = status;
    return launch_score_tc(ta, st);
  }
  return launch_score_simt(sa, st);
}

int lsa_select_union(int B, int Nw, const uint32_t* mask_l, uint32_t* U, uint32_t* new_l,
                     void* stream) {
  const CallRange range("lsa_select_union");
  g_err[0] = 0;
  if (B < 0 || Nw < 0) return fail(LSA_ERR_INVALID_ARG, "select_union: negative size");
  if (static_cast<size_t>(B) * Nw == 0) return LSA_OK;
  if (!mask_l || !U) return fail(LSA_ERR_INVALID_ARG, "select_union: null pointer");
  if (!aligned(mask_l, 16) || !aligned(U, 16) || (new_l && !aligned(new_l, 16)))
    return fail(LSA_ERR_INVALID_ARG, "select_union: pointers must be 16-byte aligned");
  return launch_union(B, Nw, mask_l, U, new_l, static_cast<cudaStream_t>(stream));
}

int lsa_compact(int B, int N, const uint32_t* bits, int cap, int32_t* idx, int32_t* count,
                int32_t* status, void* stream) {
  const CallRange range("lsa_compact");
  g_err[0] = 0;
  if (B < 0 || N < 0 || cap < 0) return fail(LSA_ERR_INVALID_ARG, "compact: negative size");
  if (B == 0) return LSA_OK;
  if (!count || (N > 0 && !bits) || (cap > 0 && !idx))
    return fail(LSA_ERR_INVALID_ARG, "compact: null pointer");
  if ((bits && !aligned(bits, 16)) || (idx && !aligned(idx, 16)) || !aligned(count, 4))
    return fail(LSA_ERR_INVALID_ARG, "compact: misaligned pointer");
  return launch_compact(B, N, bits, cap, idx, count, status, static_cast<cudaStream_t>(stream));
}

size_t lsa_select_fetch_workspace_bytes(int B, int N) {
  if (B < 0 || N < 0) return 0;
  return select_fetch_workspace_bytes(B, N) + 256;
}

int lsa_select_fetch(int B, int L, int N, const uint32_t* mask, uint32_t* U, uint32_t* new_l, int cap,
                     int32_t* idx_new, int32_t* cnt_new, int32_t* idx_U, int32_t* cnt_U, const float* logit,
                     uint32_t* key_U, int32_t* status, void* workspace, size_t workspace_bytes, void* stream) {
  const CallRange range("lsa_select_fetch");
  g_err[0] = 0;
  if (B < 0 || L < 0 || N < 0 || cap < 0) return fail(LSA_ERR_INVALID_ARG, "select_fetch: negative size");
  if (L < 1 || L > 8) return fail(LSA_ERR_UNSUPPORTED, "select_fetch: L = %d layers (1 to 8)", L);
  if (B == 0) return LSA_OK;
  if (!cnt_new || !cnt_U || (N > 0 && !mask) || (cap > 0 && (!idx_new || !idx_U)))
    return fail(LSA_ERR_INVALID_ARG, "select_fetch: null pointer");
  if ((mask && !aligned(mask, 16)) || (U && !aligned(U, 16)) || (new_l && !aligned(new_l, 16)) ||
      (idx_new && !aligned(idx_new, 16)) || (idx_U && !aligned(idx_U, 16)) || !aligned(cnt_new, 4) ||
      !aligned(cnt_U, 4) || (key_U && !aligned(key_U, 16)) || (logit && !aligned(logit, 4)))
    return fail(LSA_ERR_INVALID_ARG, "select_fetch: misaligned pointer");
  if (key_U && cap > 0 && !logit) return fail(LSA_ERR_INVALID_ARG, "select_fetch: key_U needs the logits");
  const size_t need = lsa_select_fetch_workspace_bytes(B, N);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
    return fail(LSA_ERR_NOMEM, "select_fetch: workspace %zu bytes (need %zu)", workspace_bytes, need);
  return launch_select_fetch(B, L, N, mask, U, new_l, cap, idx_new, cnt_new, idx_U, cnt_U, status,
                             static_cast<int32_t*>(workspace), logit, key_U, static_cast<cudaStream_t>(stream));
}

int lsa_topk_keyed(int B, int k, const int32_t* idx, int cap, const int32_t* count, const uint32_t* key,
                   int32_t* topk, int32_t* topk_count, void* stream) {
  const CallRange range("lsa_topk_keyed");
  g_err[0] = 0;
  if (B < 0 || k < 0 || cap < 0) return fail(LSA_ERR_INVALID_ARG, "topk_keyed: negative size");
  if (B == 0) return LSA_OK;
  if (!count || (cap > 0 && (!idx || !key)) || (k > 0 && !topk))
    return fail(LSA_ERR_INVALID_ARG, "topk_keyed: null pointer");
  if ((idx && !aligned(idx, 4)) || (key && !aligned(key, 4)) || !aligned(count, 4))
    return fail(LSA_ERR_INVALID_ARG, "topk_keyed: misaligned pointer");
  return launch_topk_keyed(B, k, idx, cap, count, key, topk, topk_count, static_cast<cudaStream_t>(stream));
}

// Workspace of lsa_fine_score: query images, folded head weights, tile prefix.
struct FineWs {
  size_t qimg, wfold, tiles, total;
};
static FineWs fine_ws(int B, int H, int dI, int kdt) {
  FineWs o{};
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off = align_up(off + bytes, 1024); return at; };
  o.qimg = take(static_cast<size_t>(B) * tc_image_bytes(H, dI, kdt));
  o.wfold = take(static_cast<size_t>(B) * H * 4);
  o.tiles = take((static_cast<size_t>(B) + 1) * 4);
  o.total = off;
  return o;
}

size_t lsa_fine_score_workspace_bytes(int B, int H, int dI, int kdt) {
  if (B < 0 || H < 0 || dI < 0) return 0;
  return fine_ws(B, H, dI, kdt).total + 256;
}

int lsa_fine_score(int B, int N, int H, int dI, int qdt, const void* q, const float* w, int kdt, const void* K,
                   const float* kscale, const int32_t* idx, int cap, const int32_t* count, float* score,
                   int32_t* status, void* workspace, size_t workspace_bytes, void* stream) {
  const CallRange range("lsa_fine_score");
  g_err[0] = 0;
  if (B < 0 || N < 0 || H <= 0 || dI <= 0 || cap < 0) return fail(LSA_ERR_INVALID_ARG, "fine_score: bad size");
  if (B == 0 || N == 0 || cap == 0) return LSA_OK;
  if (qdt != LSA_F32 && qdt != LSA_BF16) return fail(LSA_ERR_UNSUPPORTED, "fine_score: query dtype %d", qdt);
  if (kdt != LSA_F32 && kdt != LSA_BF16 && kdt != LSA_E4M3)
    return fail(LSA_ERR_UNSUPPORTED, "fine_score: key dtype %d", kdt);
  if (!q || !w || !K || !idx || !count || !score || (kdt == LSA_E4M3 && !kscale))
    return fail(LSA_ERR_INVALID_ARG, "fine_score: null pointer (e4m3 keys need kscale)");
  if (static_cast<long long>(B) * N > 0x7fffffffLL)
    return fail(LSA_ERR_UNSUPPORTED, "fine_score: B*N = %lld rows (at most 2^31 - 1)", static_cast<long long>(B) * N);
  const bool tc = tc_supported(H, dI, qdt, kdt);
  if (!tc && (static_cast<size_t>(H) * dI + H) * 4 > 227 * 1024)
    return fail(LSA_ERR_UNSUPPORTED, "fine_score: H*dI = %d too large for the CUDA-core path", H * dI);
  if (!aligned(K, 128) || !aligned(q, 16) || !aligned(w, 16) || !aligned(idx, 16) || !aligned(count, 4) ||
      !aligned(score, 4) || (kscale && !aligned(kscale, 4)))
    return fail(LSA_ERR_INVALID_ARG, "fine_score: misaligned pointer (K 128 bytes, q, w, idx 16)");
  const FineWs ws = fine_ws(B, H, dI, kdt);
  if (tc && (!workspace || workspace_bytes < ws.total || !aligned(workspace, 256)))
    return fail(LSA_ERR_NOMEM, "fine_score: workspace %zu bytes (need %zu)", workspace_bytes, ws.total);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  FineArgs fa{};
  fa.B = B; fa.N = N; fa.H = H; fa.dI = dI; fa.qdt = qdt; fa.kdt = kdt; fa.cap = cap;
  fa.q = q; fa.w = w; fa.K = K; fa.kscale = kscale; fa.idx = idx; fa.count = count; fa.score = score;
  fa.qimg = tc ? base + ws.qimg : nullptr;
  fa.wfold = tc ? reinterpret_cast<float*>(base + ws.wfold) : nullptr;
  fa.tile_start = tc ? reinterpret_cast<int32_t*>(base + ws.tiles) : nullptr;
  fa.status = status;
  return launch_fine_score(fa, static_cast<cudaStream_t>(stream));
}

size_t lsa_topk_workspace_bytes(int B, int cap) {
  if (B < 0 || cap < 0) return 0;
  return align_up(static_cast<size_t>(B) * cap * 4, 256) + 256;
}

int lsa_topk(int B, int L, int N, int k, const int32_t* idx, int cap, const int32_t* count,
             const float* logit, int32_t* topk, int32_t* topk_count,
             void* workspace, size_t workspace_bytes, void* stream) {
  const CallRange range("lsa_topk");
  g_err[0] = 0;
  if (B < 0 || L <= 0 || N < 0 || k < 0 || cap < 0)
    return fail(LSA_ERR_INVALID_ARG, "topk: bad size (L must be >= 1)");
  if (B == 0) return LSA_OK;
  if (!count || (cap > 0 && !idx) || (k > 0 && !topk) || (N > 0 && !logit))
    return fail(LSA_ERR_INVALID_ARG, "topk: null pointer");
  if (workspace_bytes < lsa_topk_workspace_bytes(B, cap) || (cap > 0 && !workspace) ||
      (workspace && !aligned(workspace, 256)))
    return fail(LSA_ERR_NOMEM, "topk: workspace %zu bytes (need %zu)", workspace_bytes,
                lsa_topk_workspace_bytes(B, cap));
  return launch_topk(B, L, N, k, idx, cap, count, logit, topk, topk_count,
                     static_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream));
}

int lsa_gather_cold(int B, int N, size_t row_bytes, const void* cold_host,
                    const int32_t* idx, const int32_t* count, int cap, void* hot,
                    int32_t* status, void* stream) {
  const CallRange range("lsa_gather_cold");
  g_err[0] = 0;
  if (B < 0 || N < 0 || cap < 0) return fail(LSA_ERR_INVALID_ARG, "gather_cold: negative size");
  if (row_bytes == 0 || row_bytes % 16 != 0)
    return fail(LSA_ERR_INVALID_ARG, "gather_cold: row_bytes %zu is not a positive multiple of 16", row_bytes);
  if (B == 0 || cap == 0) return LSA_OK;
  if (!cold_host || !idx || !count || !hot) return fail(LSA_ERR_INVALID_ARG, "gather_cold: null pointer");
  if (!aligned(cold_host, 16) || !aligned(hot, 16) || !aligned(idx, 16))
    return fail(LSA_ERR_INVALID_ARG, "gather_cold: pointers must be 16-byte aligned");
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, cold_host) != cudaSuccess || attr.type != cudaMemoryTypeHost ||
      attr.devicePointer == nullptr) {
    cudaGetLastError();
    return fail(LSA_ERR_INVALID_ARG, "gather_cold: cold pool is not page-locked, mapped host memory");
  }
  return launch_gather(B, N, row_bytes, attr.devicePointer, idx, count, cap, hot, status,
                       static_cast<cudaStream_t>(stream));
}

static int hot_sizes_ok(int B, int N, int slots) { return B >= 0 && N >= 0 && slots >= 0; }

size_t lsa_hot_pool_state_bytes(int B, int N, int slots) {
  return hot_sizes_ok(B, N, slots) ? hot_layout(B, N, slots).state_bytes : 0;
}

size_t lsa_hot_pool_workspace_bytes(int B, int N, int slots) {
  return hot_sizes_ok(B, N, slots) ? hot_layout(B, N, slots).ws_bytes : 0;
}

int lsa_hot_pool_layout(int B, int N, int slots, size_t offsets[4]) {
  g_err[0] = 0;
  if (!hot_sizes_ok(B, N, slots)) return fail(LSA_ERR_INVALID_ARG, "hot_pool_layout: negative size");
  if (!offsets) return fail(LSA_ERR_INVALID_ARG, "hot_pool_layout: null pointer");
  const HotLayout l = hot_layout(B, N, slots);
  offsets[0] = l.slot_of;
  offsets[1] = l.entry_of;
  offsets[2] = l.stamp;
  offsets[3] = l.resident;
  return LSA_OK;
}

int lsa_hot_pool_reset(int B, int N, int slots, void* state, void* stream) {
  const CallRange range("lsa_hot_pool_reset");
  g_err[0] = 0;
  if (!hot_sizes_ok(B, N, slots)) return fail(LSA_ERR_INVALID_ARG, "hot_pool_reset: negative size");
  if (!state) return fail(LSA_ERR_INVALID_ARG, "hot_pool_reset: null pointer");
  if (!aligned(state, 256)) return fail(LSA_ERR_INVALID_ARG, "hot_pool_reset: state must be 256-byte aligned");
  const HotLayout l = hot_layout(B, N, slots);
  uint8_t* st = static_cast<uint8_t*>(state);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t Nw = (static_cast<size_t>(N) + 31) / 32;
  if (cudaMemsetAsync(st + l.slot_of, 0xff, static_cast<size_t>(B) * N * 4, s) != cudaSuccess ||
      cudaMemsetAsync(st + l.entry_of, 0xff, static_cast<size_t>(B) * slots * 4, s) != cudaSuccess ||
      cudaMemsetAsync(st + l.stamp, 0, static_cast<size_t>(B) * slots * 4, s) != cudaSuccess ||
      cudaMemsetAsync(st + l.resident, 0, static_cast<size_t>(B) * Nw * 4, s) != cudaSuccess) {
    const cudaError_t e = cudaGetLastError();
    return fail(LSA_ERR_CUDA, "hot_pool_reset: %s", cudaGetErrorString(e));
  }
  return LSA_OK;
}

int lsa_hot_pool_update(int B, int N, int slots, size_t row_bytes, uint32_t trigger,
                        const uint32_t* U, const void* cold_host, void* hot, void* state,
                        int32_t* moved, int32_t* status,
                        void* workspace, size_t workspace_bytes, void* stream) {
  const CallRange range("lsa_hot_pool_update");
  g_err[0] = 0;
  if (!hot_sizes_ok(B, N, slots)) return fail(LSA_ERR_INVALID_ARG, "hot_pool_update: negative size");
  if (row_bytes == 0 || row_bytes % 16 != 0)
    return fail(LSA_ERR_INVALID_ARG, "hot_pool_update: row_bytes %zu is not a positive multiple of 16", row_bytes);
  if (trigger == 0 || trigger == 0xffffffffu)
    return fail(LSA_ERR_INVALID_ARG, "hot_pool_update: trigger must be in [1, 2^32 - 2]");
  if (slots < 1) return fail(LSA_ERR_INVALID_ARG, "hot_pool_update: slots must be >= 1");
  if (B == 0 || N == 0) return LSA_OK;
  if (!U || !cold_host || !state || !hot)
    return fail(LSA_ERR_INVALID_ARG, "hot_pool_update: null pointer");
  if (!aligned(state, 256) || !aligned(U, 16) || !aligned(cold_host, 16) || (hot && !aligned(hot, 16)))
    return fail(LSA_ERR_INVALID_ARG, "hot_pool_update: misaligned pointer (state 256 B, others 16 B)");
  const HotLayout l = hot_layout(B, N, slots);
  if (!workspace || workspace_bytes < l.ws_bytes || !aligned(workspace, 256))
    return fail(LSA_ERR_NOMEM, "hot_pool_update: workspace %zu bytes (need %zu, 256-byte aligned)", workspace_bytes,
                l.ws_bytes);
  cudaPointerAttributes attr{};
  if (cudaPointerGetAttributes(&attr, cold_host) != cudaSuccess || attr.type != cudaMemoryTypeHost ||
      attr.devicePointer == nullptr) {
    cudaGetLastError();
    return fail(LSA_ERR_INVALID_ARG, "hot_pool_update: cold pool is not page-locked, mapped host memory");
  }
  return launch_hot_update(B, N, slots, row_bytes, trigger, U, attr.devicePointer, hot, state, moved, status,
                           workspace, static_cast<cudaStream_t>(stream));
}

// Workspace of lsa_index_train_step: the projection's regions (as lsa_index_score with
// B = P, L = 1), then the training regions.
static size_t train_ws_bytes(int P, int N, int D, int r, int H, int dI, int wdt, size_t* proj_bytes) {
  const ScoreWs pw = score_ws(P, 1, D, r, H, dI, wdt, LSA_BF16);
  const size_t pb = align_up(pw.qimg, 1024);      // regions up to (not including) the query images
  if (proj_bytes) *proj_bytes = pb;
  return pb + train_layout(P, N, D, r, H, dI).total;
}

size_t lsa_index_train_step_workspace_bytes(int P, int N, int D, int r, int H, int dI) {
  if (P <= 0 || N < 0 || D <= 0 || r <= 0 || H <= 0 || dI <= 0) return 0;
  return train_ws_bytes(P, N, D, r, H, dI, LSA_BF16, nullptr);
}

int lsa_index_train_step(int P, int N, int D, int r, int H, int dI, int wdt,
                         const void* h, const void* W_down, const void* W_up, const void* W_w, float bias,
                         int kdt, const void* K, const float* kscale, const uint32_t* labels, float gamma,
                         const void* c_in, const void* q_in, const float* w_in,
                         double* loss, float* dW_down, float* dW_up, float* dW_w, double* dbias,
                         int32_t* status, void* workspace, size_t workspace_bytes, void* stream) {
  const CallRange range("lsa_index_train_step");
  g_err[0] = 0;
  if (P <= 0 || N < 0 || D <= 0 || r <= 0 || H <= 0 || dI <= 0)
    return fail(LSA_ERR_INVALID_ARG, "index_train_step: bad size");
  if (!train_supported(P, H, dI, wdt, kdt) || kscale != nullptr || D % 8 != 0 || r % 8 != 0)
    return fail(LSA_ERR_UNSUPPORTED,
                "index_train_step: needs bf16 weights and keys, H in {32, 64, 128}, dI in {64, 128}, P a multiple "
                "of 128/H and at most 4096, D and r multiples of 8");
  const bool given = c_in || q_in || w_in;
  if (given && !(c_in && q_in && w_in))
    return fail(LSA_ERR_INVALID_ARG, "index_train_step: give all of c_in, q_in, w_in or none");
  if (!given && P > 256) return fail(LSA_ERR_UNSUPPORTED, "index_train_step: projecting P > 256 positions");
  if (!h || !W_up || !K || !labels || !dW_down || !dW_up || !dW_w || (!given && (!W_down || !W_w)))
    return fail(LSA_ERR_INVALID_ARG, "index_train_step: null pointer");
  const void* ptrs[] = {h, W_down, W_up, W_w, K, labels, c_in, q_in, w_in, dW_down, dW_up, dW_w};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return fail(LSA_ERR_INVALID_ARG, "index_train_step: pointer %p not 16-byte aligned", p);
  size_t pb = 0;
  const size_t need = train_ws_bytes(P, N, D, r, H, dI, wdt, &pb);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
    return fail(LSA_ERR_NOMEM, "index_train_step: workspace %zu bytes (need %zu)", workspace_bytes, need);
  if (N == 0) return LSA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const ScoreWs pw = score_ws(P, 1, D, r, H, dI, wdt, LSA_BF16);
  TrainArgs ta{};
  ta.P = P; ta.N = N; ta.D = D; ta.r = r; ta.H = H; ta.dI = dI;
  ta.h = h; ta.W_up = W_up; ta.K = K; ta.bias = bias; ta.gamma = gamma; ta.labels = labels;
  ta.loss = loss; ta.dbias = dbias; ta.dW_down = dW_down; ta.dW_up = dW_up; ta.dW_w = dW_w;
  ta.status = status; ta.ws = base + pb;
  if (given) {
    ta.c = c_in; ta.q = q_in; ta.w = w_in;
  } else {
    ProjectArgs pa{};
    pa.B = P; pa.L = 1; pa.D = D; pa.r = r; pa.H = H; pa.dI = dI; pa.wdt = wdt; pa.l0 = 0; pa.nL = 1;
    pa.h = h; pa.W_down = W_down; pa.W_up = W_up; pa.W_w = W_w;
    pa.partA = reinterpret_cast<float*>(base + pw.partA);
    pa.partW = reinterpret_cast<float*>(base + pw.partW);
    pa.partB = reinterpret_cast<float*>(base + pw.partB);
    pa.cbuf = reinterpret_cast<float*>(base + pw.cbuf);
    pa.q_ws = base + pw.q;
    pa.w_ws = reinterpret_cast<float*>(base + pw.w);
    pa.do_q = pa.do_w = true;
    pa.status = status;
    if (!project_tc_supported(pa)) return fail(LSA_ERR_UNSUPPORTED, "index_train_step: projection shape");
    const int rc = launch_project(pa, st);      // leaves c (bf16) in cbuf, q and w in the workspace
    if (rc != LSA_OK) return rc;
    ta.c = base + pw.cbuf; ta.q = base + pw.q; ta.w = reinterpret_cast<const float*>(base + pw.w);
  }
  return launch_train(ta, st);
}

int lsa_check_bounded_wait(uint32_t limit_us, int32_t* status, void* stream) {
  const CallRange range("lsa_check_bounded_wait");
  g_err[0] = 0;
  if (!status) return fail(LSA_ERR_INVALID_ARG, "check_bounded_wait: null status");
  if (limit_us == 0 || limit_us > 2000000u)
    return fail(LSA_ERR_INVALID_ARG, "check_bounded_wait: limit %u us outside [1, 2000000]", limit_us);
  return launch_wait_check(static_cast<unsigned long long>(limit_us) * 1000ull, status,
                           static_cast<cudaStream_t>(stream));
}

// Per-row selection words in the vote kernels' blocked order: 4 per 128 entries.
static size_t vote_row_words(int N) { return 4 * ((static_cast<size_t>(N) + 127) / 128); }

size_t lsa_vote_labels_workspace_bytes(int L, int P, int N) {
  if (L < 0 || P < 0 || N < 0) return 0;
  const size_t Nw = vote_row_words(N);
  return align_up(static_cast<size_t>(L) * P * Nw * 4, 256) +
         align_up(static_cast<size_t>(L) * P * 4 * 4, 256) + 256;
}

int lsa_vote_labels(int L, int P, int N, const float* logits, float top_p, int theta,
                    uint32_t* golden, uint8_t* counts,
                    const float* scores, float gamma, double* loss,
                    void* workspace, size_t workspace_bytes, void* stream) {
  const CallRange range("lsa_vote_labels");
  g_err[0] = 0;
  if (L < 0 || P < 0 || N < 0) return fail(LSA_ERR_INVALID_ARG, "vote_labels: negative size");
  if (L > 255) return fail(LSA_ERR_UNSUPPORTED, "vote_labels: L = %d layers (at most 255: counts are bytes)", L);
  if (P > 65535) return fail(LSA_ERR_UNSUPPORTED, "vote_labels: P = %d positions (at most 65535)", P);
  if (!(top_p > 0.f && top_p <= 1.f)) return fail(LSA_ERR_INVALID_ARG, "vote_labels: top_p must be in (0, 1]");
  if (static_cast<size_t>(P) * N == 0) return LSA_OK;
  if ((L > 0 && !logits) || !golden) return fail(LSA_ERR_INVALID_ARG, "vote_labels: null pointer");
  if (scores && !loss) return fail(LSA_ERR_INVALID_ARG, "vote_labels: scores given without loss output");
  const size_t need = lsa_vote_labels_workspace_bytes(L, P, N);
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
    return fail(LSA_ERR_NOMEM, "vote_labels: workspace %zu bytes (need %zu)", workspace_bytes, need);
  const size_t Nw = vote_row_words(N);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  VoteArgs va{};
  va.L = L; va.P = P; va.N = N; va.logits = logits; va.top_p = top_p; va.theta = theta;
  va.golden = golden; va.counts = counts; va.scores = scores; va.gamma = gamma; va.loss = loss;
  va.selbits = reinterpret_cast<uint32_t*>(base);
  va.rowparam = reinterpret_cast<float*>(base + align_up(static_cast<size_t>(L) * P * Nw * 4, 256));
  va.lossacc = reinterpret_cast<double*>(base + need - 256);
  return launch_vote(va, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
