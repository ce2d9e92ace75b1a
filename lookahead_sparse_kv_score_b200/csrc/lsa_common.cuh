// Shared device helpers and internal launch declarations of liblsa.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stddef.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "lsa.h"

namespace lsa {

// One NVTX range per library call, named after the call, so that a profiler's timeline
// (or an ncu --nvtx filter) shows which call launched which kernels.  With no tool
// attached a range costs a few nanoseconds.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// ------------------------------------------------------------------ host-side errors
int fail(int code, const char* fmt, ...);   // records the message, returns code
void clear_error();                         // empties the calling thread's last message
int check_launch(const char* what, int kernels = 1);   // LSA_OK or LSA_ERR_CUDA after launching
                                                        // `kernels` kernels (counted when OK)

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ------------------------------------------------------------------ dependent launches
// The kernels of the scoring and selection chain are launched as programmatic dependents of
// the kernel before them on the stream: a kernel's blocks may be scheduled while its
// predecessor's last blocks still run, and each such kernel waits at its first
// instruction (pdl_wait) until the predecessor has completed and its writes are visible;
// it then lets its own dependents be scheduled (pdl_trigger).  For a kernel launched
// without the attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... Params, typename... Args>
inline cudaError_t launch_dependent(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Params>(args)...);
}

// ------------------------------------------------------------------ device helpers
__device__ __forceinline__ void raise_status(int32_t* status, int code) {
  if (status != nullptr) atomicMax(status, code);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ float e4m3_to_float(uint8_t code) {
  __nv_fp8_e4m3 v;
  v.__x = code;
  return static_cast<float>(v);   // exact: every e4m3 value is a float
}

// Element loaders for the three storage types.
__device__ __forceinline__ float load_elem(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ float load_elem(const uint8_t* p, size_t i) { return e4m3_to_float(p[i]); }

__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + __expf(-z)); }

// Order-preserving integer image of a float: x < y  <=>  order_key(x) < order_key(y)
// (the two zeros map to one key; non-negative x map to keys >= 2^31, so 0 is below
// every non-negative logit's key).
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------------ internal launches
// Projection: fills q_ws ([L][B][H][dI], wdt) and w_ws ([L][B][H] fp32) for layers
// l0 .. l0+nL-1.  Scratch regions come from the caller's workspace.
struct ProjectArgs {
  int B, L, D, r, H, dI, wdt, l0, nL;
  const void *h, *W_down, *W_up, *W_w;
  float *partA, *partW, *partB, *cbuf;
  void* q_ws;
  float* w_ws;
  void* q_out;
  float* w_out;
  bool do_q, do_w;      // project the query / the head weights
  int32_t* status;      // device status word or null (a tensor-core pipeline wait that gave up)
};
int launch_project(const ProjectArgs& a, cudaStream_t s);
// Tensor-core projection (bf16 weights, B <= 256) and the reductions it shares with the
// CUDA-core version.
struct ProjectTcBufs {
  __nv_bfloat16* c_bf16;   // [nL][B][r]: c rounded to bf16, the input of q = c W_up
};
bool project_tc_supported(const ProjectArgs& a);
int launch_project_tc(const ProjectArgs& a, const ProjectTcBufs& t, cudaStream_t s);
int launch_project_reductions(const ProjectArgs& a, int S, const ProjectTcBufs& t, cudaStream_t s);
int launch_project_q_reduction(const ProjectArgs& a, int S, cudaStream_t s);
int project_splits(int K);     // reduction slices of h W_down / h W_w (length K = D)
int project_splits_b(int K);   // reduction slices of c W_up (length K = r)

// CUDA-core scoring of layers l0 .. l0+nL-1.
struct ScoreArgs {
  int B, L, N, H, dI, wdt, kdt, l0, nL;
  const void* q;        // [L][B][H][dI] wdt
  const float* w;       // [L][B][H]
  const float* bias;    // [L]
  const void* K;        // [L][B][N][dI] kdt
  const float* kscale;  // [L][B][N] or null
  uint32_t* mask;
  float* logit;
  float* score;
};
int launch_score_simt(const ScoreArgs& a, cudaStream_t s);

// Tensor-core scoring (tcgen05 + TMA).  qimg/wfold are workspace regions.
struct TcArgs {
  ScoreArgs sc;
  uint8_t* qimg;        // [L][B][img_bytes], 1024-byte aligned
  float* wfold;         // [L][B][H]
  int32_t* status;      // caller's device status word (bounded-wait timeouts), may be null
};
size_t tc_image_bytes(int H, int dI, int kdt);
bool tc_supported(int H, int dI, int wdt, int kdt);
int launch_score_tc(const TcArgs& a, cudaStream_t s);

// Native-indexer fine score of gathered candidates (tensor cores when tc_supported,
// else CUDA cores): score[b][idx[b][j]] for j < min(count[b], cap).
struct FineArgs {
  int B, N, H, dI, qdt, kdt, cap;
  const void* q;            // [B][H][dI] qdt (f32 or bf16)
  const float* w;           // [B][H]
  const void* K;            // [B][N][dI] kdt
  const float* kscale;      // [B][N] or null
  const int32_t* idx;       // [B][cap]
  const int32_t* count;     // [B]
  float* score;             // [B][N]
  uint8_t* qimg;            // workspace [B][img_bytes] (tensor-core path)
  float* wfold;             // workspace [B][H]
  int32_t* tile_start;      // workspace [B + 1]
  int32_t* status;
};
int launch_fine_score(const FineArgs& a, cudaStream_t s);
int launch_fine_score_tc(const FineArgs& a, cudaStream_t s);
int launch_fine_score_simt(const FineArgs& a, cudaStream_t s);

// Selection.
int launch_union(int B, int Nw, const uint32_t* m, uint32_t* U, uint32_t* nw, cudaStream_t s);
int launch_compact(int B, int N, const uint32_t* bits, int cap, int32_t* idx, int32_t* count,
                   int32_t* status, cudaStream_t s);
size_t select_fetch_workspace_bytes(int B, int N);
int launch_select_fetch(int B, int L, int N, const uint32_t* mask, uint32_t* U, uint32_t* nw, int cap,
                        int32_t* idx_new, int32_t* cnt_new, int32_t* idx_U, int32_t* cnt_U, int32_t* status,
                        int32_t* ws, const float* logit, uint32_t* key_U, cudaStream_t s);
// The top-k with given per-candidate order keys (keys[b][j] for candidate idx[b][j]).
int launch_topk_keyed(int B, int k, const int32_t* idx, int cap, const int32_t* count, const uint32_t* keys,
                      int32_t* topk, int32_t* topk_count, cudaStream_t s);
int launch_topk(int B, int L, int N, int k, const int32_t* idx, int cap, const int32_t* count,
                const float* logit, int32_t* topk, int32_t* topk_count, uint32_t* keys_ws,
                cudaStream_t s);
// One indexer training step (bf16 weights and keys): loss sums, db and the gradients of
// W_down, W_up, W_w from P positions' c [P][r], q [P][H][dI] (bf16) and w [P][H].
struct TrainArgs {
  int P, N, D, r, H, dI;
  const void *h, *c, *q, *W_up, *K;
  const float* w;
  float bias, gamma;
  const uint32_t* labels;
  double *loss, *dbias;
  float *dW_down, *dW_up, *dW_w;
  int32_t* status;
  void* ws;
};
struct TrainLayout {
  size_t qimg, upart, dq, dw, dc, dcpart, acc, total;
};
bool train_supported(int P, int H, int dI, int wdt, int kdt);
TrainLayout train_layout(int P, int N, int D, int r, int H, int dI);
int launch_train(const TrainArgs& a, cudaStream_t s);

// One kernel whose bounded wait on an mbarrier nothing arrives at gives up after
// limit_ns and raises *status to LSA_ERR_TIMEOUT.
int launch_wait_check(unsigned long long limit_ns, int32_t* status, cudaStream_t s);

// Direct-key selection: per sequence b, the kdev[b] largest of keys[b][0..n) (ties to the
// lower index) in ascending index order, or none with LSA_ERR_CAPACITY when kdev[b]
// exceeds n - kept[b].  out [B][n], out_count [B].
int launch_select_keys(int B, int n, const uint32_t* keys, const int32_t* kdev, const int32_t* kept,
                       int32_t* status, int32_t* out, int32_t* out_count, uint32_t* keys_ws, cudaStream_t s);

// Hot-pool residency: byte offsets of the state arrays and of the update's workspace.
struct HotLayout {
  size_t slot_of, entry_of, stamp, resident, state_bytes;
  size_t need_bits, keys, need, need_count, kept_count, taken, moved, select_ws, ws_bytes;
};
HotLayout hot_layout(int B, int N, int slots);
int launch_hot_update(int B, int N, int slots, size_t row_bytes, uint32_t t, const uint32_t* U,
                      const void* cold_dev, void* hot, void* state, int32_t* moved, int32_t* status,
                      void* ws, cudaStream_t s);

int launch_gather(int B, int N, size_t row_bytes, const void* cold_dev, const int32_t* idx,
                  const int32_t* count, int cap, void* hot, int32_t* status, cudaStream_t s);

struct VoteArgs {
  int L, P, N;
  const float* logits;
  float top_p;
  int theta;
  uint32_t* golden;
  uint8_t* counts;
  const float* scores;
  float gamma;
  double* loss;
  uint32_t* selbits;    // workspace [L][P][Nw]
  float* rowparam;      // workspace [L][P][4]
  double* lossacc;      // workspace: [2] loss sums, then the loss blocks' counter
};
int launch_vote(const VoteArgs& a, cudaStream_t s);

}  // namespace lsa
