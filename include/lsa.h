/*
 * lsa.h -- C ABI of the Lookahead Sparse Attention (LSA) indexer hot path on B200.
 *
 * The operations follow the pages describing FlashMemory-DeepSeek-V4:
 *   [SUMMARY] "技术摘要：通过前瞻性稀疏注意力机制实现的 FlashMemory-DeepSeek-V4"
 *             (gist.science technical summary), §2.1 架构设计 (periodic trigger,
 *             memory indexer, scoring, dynamic fetch, hierarchical selection),
 *             §2.2 数据策展与标注 (cross-layer majority vote), §2.3 (BCE + focal loss),
 *             §2.4 最优配置 (three indexer layers, OR mode).
 *   [REVIEW]  "论文综述：FlashMemory-DeepSeek-V4 用前瞻稀疏注意力压缩超长上下文KV缓存"
 *             (paper.oopus.info review), part 二 核心方法与创新.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer is a DEVICE pointer unless the comment says "host".  The caller
 *    owns every buffer, including workspaces; the library allocates no memory.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronises, prints, traps or aborts.
 *  - Argument errors are detected on the host before anything is launched and
 *    returned as LSA_ERR_INVALID_ARG / LSA_ERR_UNSUPPORTED / LSA_ERR_NOMEM (workspace
 *    too small).  A failed launch returns LSA_ERR_CUDA.  lsa_last_error() gives a
 *    one-line description of the last error on the calling thread.
 *  - Conditions only the device can see (a fetch list longer than its capacity, an
 *    entry index out of range) are reported through an optional device status word
 *    (int32): the kernel raises it to the lsa_status code with atomicMax, so the
 *    caller zeroes it first and reads it after synchronising.
 *  - Per-(layer, sequence) tensors are stored LAYER-MAJOR: [L][B][...], so the slice
 *    of one indexer layer is one contiguous [B][...] block.
 *  - Bit sets are uint32 words; bit i of word j is entry 32*j + i; Nw = ceil(N/32);
 *    bits at or past N are zero.
 *  - Pointers must be 16-byte aligned; K_IComp must be 128-byte aligned.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LSA_OK = 0,
  LSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer          */
  LSA_ERR_UNSUPPORTED = 2,   /* dtype / shape combination not built                 */
  LSA_ERR_CAPACITY = 3,      /* (device status) a list did not fit its capacity     */
  LSA_ERR_NOMEM = 4,         /* workspace smaller than the *_workspace_bytes answer  */
  LSA_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed                 */
  LSA_ERR_TIMEOUT = 6,       /* (device status) a bounded wait gave up               */
  LSA_ERR_RANGE = 7          /* (device status) an entry index was out of [0, N)     */
} lsa_status;

typedef enum { LSA_F32 = 0, LSA_BF16 = 1, LSA_E4M3 = 2 } lsa_dtype;

/* Static string for a status code.  Never NULL. */
const char* lsa_status_string(int status);

/* Description of the last error returned on this thread ("" if none). */
const char* lsa_last_error(void);

/* ABI version of this header: 1. */
int lsa_abi_version(void);

/* Number of kernels this library has launched in this process (all threads).  A
 * diagnostic for callers that account for device work; it never resets. */
unsigned long long lsa_kernel_launches(void);

/* ------------------------------------------------------------------------------------
 * lsa_index_score -- low-rank indexer query + head-fused gated score + threshold.
 *
 * [SUMMARY] §2.1: every tau decode steps the memory indexer maps the hidden state
 * h_t of the current token to a low-rank indexer query and scores every earlier
 * compressed entry s with a head-fused, sigmoid-gated matching score I_{t,s}; entries
 * with I >= 0.5 are fetched ([REVIEW] 二).  Per (layer l, sequence b):
 *     c = h W_down[l]                    (rank r; rounded to bf16 when wdt = BF16)
 *     q = c W_up[l]  -> [H][dI]          (rounded to bf16 when wdt = BF16)
 *     w = h W_w[l]   -> [H]              (fp32, not rounded)
 *     z_s = kscale_s * sum_h w_h * ReLU(q_h . khat_s) + bias[l]
 *     I_s = sigmoid(z_s);  mask bit s = (z_s >= 0)  (<=> I_s >= 0.5)
 *
 * Sizes: B sequences, L indexer layers, N entries per sequence, D hidden, r rank,
 *        H heads, dI head dim.
 * Inputs (layer-major):
 *   h       [L][B][D]        wdt (LSA_F32 or LSA_BF16)
 *   W_down  [L][D][r]        wdt
 *   W_up    [L][r][H*dI]     wdt
 *   W_w     [L][D][H]        wdt
 *   bias    [L]              fp32
 *   K       [L][B][N][dI]    kdt (LSA_F32, LSA_BF16, or LSA_E4M3 codes)
 *   kscale  [L][B][N]        fp32, > 0; required iff kdt = LSA_E4M3, else NULL
 *   q_in    [L][B][H][dI]    wdt, optional: use this query instead of projecting
 *   w_in    [L][B][H]        fp32, optional: use these head weights (needs q_in)
 * Outputs (any may be NULL except mask):
 *   q_out   [L][B][H][dI]    wdt: the projected query (ignored when q_in is given)
 *   w_out   [L][B][H]        fp32
 *   mask    [L][B][Nw]       uint32 bit set of marked entries
 *   logit   [L][B][N]        fp32 z_s
 *   score   [L][B][N]        fp32 I_s
 * status: device int32 or NULL; raised to LSA_ERR_TIMEOUT if a bounded pipeline wait
 *   inside the tensor-core kernel gave up (the outputs are then incomplete).
 * layer: -1 processes all L layers in one pass; 0 <= layer < L processes that layer
 *   only and touches only that layer's slices of every output.
 * workspace: at least lsa_index_score_workspace_bytes(...) bytes, 256-byte aligned;
 *   contents are scratch and may be reused by the caller after the call completes.
 * Supported: kdt LSA_F32 with wdt LSA_F32 (CUDA-core path); kdt LSA_BF16 or
 *   LSA_E4M3 with wdt LSA_BF16 (tensor-core path: dI in {64,128,192,256} for bf16 and
 *   {128,256} for e4m3, H a multiple of 32 from 32 to 256).  Other combinations with
 *   H*dI <= 16384 run on the CUDA-core path; anything else is LSA_ERR_UNSUPPORTED.
 *   B x (layers scored in the call) <= 65535, else LSA_ERR_UNSUPPORTED (split the batch).
 * ---------------------------------------------------------------------------------- */
size_t lsa_index_score_workspace_bytes(int B, int L, int N, int D, int r, int H, int dI,
                                       int wdt, int kdt);

int lsa_index_score(int B, int L, int N, int D, int r, int H, int dI,
                    int wdt, const void* h, const void* W_down, const void* W_up,
                    const void* W_w, const float* bias,
                    int kdt, const void* K, const float* kscale,
                    int layer,
                    const void* q_in, const float* w_in,
                    void* q_out, float* w_out,
                    uint32_t* mask, float* logit, float* score, int32_t* status,
                    void* workspace, size_t workspace_bytes,
                    void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_index_project -- the low-rank indexer query alone (the first half of
 * lsa_index_score, [SUMMARY] §2.1 memory indexer / §2.3 low-rank query projections):
 *     q_out[l][b] = (h[l][b] W_down[l]) W_up[l]   (bf16 rounding at c and q for BF16)
 *     w_out[l][b] = h[l][b] W_w[l]                 (fp32)
 * Same layouts and dtypes as lsa_index_score; q_out [L][B][H][dI] in wdt and
 * w_out [L][B][H] fp32 are required.  Feed them to lsa_index_score as q_in / w_in to
 * score several times against one query, or to time the scoring on its own.
 * workspace: lsa_index_project_workspace_bytes(...) bytes, 256-byte aligned.
 * At most 65535 layers per call (layer = -1), else LSA_ERR_UNSUPPORTED.
 * ---------------------------------------------------------------------------------- */
size_t lsa_index_project_workspace_bytes(int B, int L, int D, int r, int H, int dI, int wdt);

int lsa_index_project(int B, int L, int D, int r, int H, int dI, int wdt, const void* h,
                      const void* W_down, const void* W_up, const void* W_w, int layer,
                      void* q_out, float* w_out, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_select_union -- multi-layer routing in OR mode ([SUMMARY] §2.4; [REVIEW] 二:
 * an entry any indexer layer asks for is fetched).  For one layer's mask, per word:
 *     new_l = mask_l & ~U;   U = U | mask_l
 * so calling it for the layers in order leaves U = OR of all layers and new_l = the
 * entries first asked for by layer l (what an incremental fetch must still move).
 *   mask_l [B][Nw] in, U [B][Nw] in/out (zero it before the first layer),
 *   new_l  [B][Nw] out or NULL.  Nw >= 0.
 * ---------------------------------------------------------------------------------- */
int lsa_select_union(int B, int Nw, const uint32_t* mask_l, uint32_t* U, uint32_t* new_l,
                     void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_compact -- fetch list of a bit set ([SUMMARY] §2.1 dynamic fetch: every entry
 * with I >= 0.5 is fetched).  For each sequence b:
 *     count[b] = popcount(bits[b]);  idx[b][0..] = ascending indices of the set bits.
 *   bits [B][Nw], idx [B][cap] int32, count [B] int32 (the true count, which may
 *   exceed cap; then only the first cap indices are written and *status is raised to
 *   LSA_ERR_CAPACITY).  status: device int32 or NULL.  N >= 0, cap >= 0.  One launch
 *   per block of 65535 sequences.
 * ---------------------------------------------------------------------------------- */
int lsa_compact(int B, int N, const uint32_t* bits, int cap, int32_t* idx, int32_t* count,
                int32_t* status, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_select_fetch -- the union, the per-layer new sets and all fetch lists of one
 * trigger in one launch ([SUMMARY] §2.4 OR mode over the indexer layers; §2.1 dynamic
 * fetch: every marked entry is fetched, incrementally as layers finish).  Equal to
 * zeroing U, calling lsa_select_union for layers 0..L-1 in order and lsa_compact on
 * each new set and on the union:
 *     new_l = mask_l & ~(mask_0 | .. | mask_{l-1}),   U = mask_0 | .. | mask_{L-1},
 *     idx_new[l][b][..] = ascending entries of new_l[b], cnt_new[l][b] = |new_l[b]|,
 *     idx_U[b][..] = ascending entries of U[b],           cnt_U[b] = |U[b]|.
 *   mask [L][B][Nw] (Nw = ceil(N/32); bits past N must be zero, as lsa_index_score
 *   leaves them); U [B][Nw] and new_l [L][B][Nw] outputs or NULL; idx_new [L][B][cap],
 *   cnt_new [L][B], idx_U [B][cap], cnt_U [B] int32 outputs.  A count above cap is
 *   reported as is, only cap indices are written and *status (device int32 or NULL) is
 *   raised to LSA_ERR_CAPACITY.  logit [L][B][N] fp32 and key_U [B][cap] uint32, both
 *   or neither: key_U[b][j] = order key of max over layers of logit[l][b][idx_U[b][j]]
 *   (the float's sign-magnitude bits mapped so that larger floats give larger keys),
 *   the keys lsa_topk ranks by, for lsa_topk_keyed.
 *   1 <= L <= 8, else LSA_ERR_UNSUPPORTED.  Device
 *   pointers 16-byte aligned (counts 4-byte).  Two launches (per-chunk counts, then the
 *   lists), and a third for key_U (the keys, from dense reads of the logits), per block
 *   of 65535 sequences.
 * workspace: lsa_select_fetch_workspace_bytes(B, N) bytes, 256-byte aligned.
 * ---------------------------------------------------------------------------------- */
size_t lsa_select_fetch_workspace_bytes(int B, int N);

int lsa_select_fetch(int B, int L, int N, const uint32_t* mask, uint32_t* U, uint32_t* new_l, int cap,
                     int32_t* idx_new, int32_t* cnt_new, int32_t* idx_U, int32_t* cnt_U, const float* logit,
                     uint32_t* key_U, int32_t* status, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_topk_keyed -- lsa_topk with the candidates' keys given: candidate j of sequence b
 * is entry idx[b][j] with key key[b][j] (an unsigned integer; larger ranks first, equal
 * keys by ascending j, i.e. ascending entry for an ascending list), j < min(count[b],
 * cap).  Results as lsa_topk: the first min(k, n) in ascending entry order in
 * topk[b][0..], -1 after them, topk_count[b] = min(k, n).  With key_U from
 * lsa_select_fetch it returns exactly what lsa_topk returns on the same lists and
 * logits ([SUMMARY] §2.1 hierarchical selection), without gathering the logits again.
 *   idx, key [B][cap], count [B], topk [B][k], topk_count [B] or NULL.  No workspace.
 * ---------------------------------------------------------------------------------- */
int lsa_topk_keyed(int B, int k, const int32_t* idx, int cap, const int32_t* count, const uint32_t* key,
                   int32_t* topk, int32_t* topk_count, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_topk -- fine top-k inside the fetched subset ([SUMMARY] §2.1 hierarchical
 * selection: once the critical subset is in GPU memory, a top-k runs inside it).
 * Candidate j of sequence b is entry e = idx[b][j], j < min(count[b], cap); its key is
 *     max over layers l of logit[l][b][e]
 * (for a fetched entry this equals the largest logit among the layers that marked it).
 * Keys are ordered descending, equal keys by ascending entry index; the first
 * min(k, n) are returned in ASCENDING ENTRY ORDER in topk[b][0..]; remaining slots are
 * set to -1; topk_count[b] = min(k, n).
 *   idx [B][cap] ascending (as written by lsa_compact), count [B],
 *   logit [L][B][N] fp32, topk [B][k] int32, topk_count [B] int32 (may be NULL).
 * workspace: lsa_topk_workspace_bytes(B, cap) bytes.
 * ---------------------------------------------------------------------------------- */
size_t lsa_topk_workspace_bytes(int B, int cap);

int lsa_topk(int B, int L, int N, int k, const int32_t* idx, int cap, const int32_t* count,
             const float* logit, int32_t* topk, int32_t* topk_count,
             void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_fine_score -- the backbone's native indexer scores the fetched subset for the
 * current token ([SUMMARY] §2.1 hierarchical selection: once the critical subset is in
 * GPU memory, the native Lightning Indexer makes a fine top-k choice inside it).  The
 * pages do not print the native indexer's formula; the reading taken is the lookahead
 * score's head-fused ReLU form with its own per-token query and keys, no bias or gate:
 *     score[b][e] = kscale[b][e] * sum_h w[b][h] * ReLU(q[b][h] . khat[b][e])
 * for every candidate e = idx[b][j], j < min(count[b], cap); other entries of score are
 * not written.  Ranking the candidates with lsa_topk(B, 1, N, k, idx, cap, count, score,
 * ...) then gives the fine top-k.
 *   q [B][H][dI] (qdt: LSA_F32 or LSA_BF16), w [B][H] fp32, K [B][N][dI] (kdt: LSA_F32,
 *   LSA_BF16 or LSA_E4M3 codes with kscale [B][N] fp32; NULL otherwise), idx [B][cap]
 *   entries in [0, N) (others are skipped), count [B], score [B][N] fp32.
 *   bf16 queries with H in {32, 64, 128, 256} and the key shapes of lsa_index_score run
 *   on the tensor cores (key rows gathered by entry, four rows per TMA gather), other
 *   shapes on the CUDA cores.  B * N < 2^31.  K 128-byte aligned; q, w, idx 16-byte.
 * workspace: lsa_fine_score_workspace_bytes(B, H, dI, kdt) bytes, 256-byte aligned.
 * ---------------------------------------------------------------------------------- */
size_t lsa_fine_score_workspace_bytes(int B, int H, int dI, int kdt);

int lsa_fine_score(int B, int N, int H, int dI, int qdt, const void* q, const float* w, int kdt, const void* K,
                   const float* kscale, const int32_t* idx, int cap, const int32_t* count, float* score,
                   int32_t* status, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_topk_noalloc -- lsa_topk without a workspace argument.  The pages have no
 * counterpart of this call: it exists for callers that cannot allocate device memory
 * when they call the library, such as a plugin inside a host framework that owns every
 * device allocation and exposes no allocator, or a latency-critical loop whose memory
 * is fixed once at start-up.  Arguments, results and errors are those of lsa_topk.
 *   Scratch: a file-scope device array of 2^23 uint32 slots (32 MiB) that every GPU
 *   which loads this part of the library's device code keeps until the process exits.  B * cap must not exceed
 *   8,388,608; larger calls return LSA_ERR_NOMEM and launch nothing.
 *   Set-up: a call resolves the array's device address (cudaGetSymbolAddress, with the
 *   call's device current) and remembers it per device.  A call made while its stream
 *   is capturing reuses the remembered address instead, so make the first call on each
 *   device before any stream capture (a first call during capture returns
 *   LSA_ERR_UNSUPPORTED).  A device reset moves the array: the next call outside capture
 *   picks up the new address, but a capture begun before that call still holds the old one.
 *   Sharing: all calls on a device use the same array, which keeps the last call's
 *   contents (nothing needs clearing: a call writes each slot before reading it).
 *   Calls that overlap on the GPU (for example on two streams) race on the array;
 *   serialise them.
 *   Allocation: no cudaMalloc, cudaFree or allocating library routine is called.
 * ---------------------------------------------------------------------------------- */
int lsa_topk_noalloc(int B, int L, int N, int k, const int32_t* idx, int cap, const int32_t* count,
                     const float* logit, int32_t* topk, int32_t* topk_count, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_gather_cold -- cold pool -> hot pool copy of the fetched rows ([SUMMARY] §2.1:
 * marked compressed KV entries move from the CPU cold pool into GPU memory; [REVIEW]
 * 二: asynchronously, overlapped with compute).  For j < min(count[b], cap):
 *     hot[b][j][0..row_bytes) = cold[b][idx[b][j]][0..row_bytes)
 *   cold   HOST pointer [B][N][row_bytes], page-locked and mapped into the device
 *          address space (cudaHostAlloc / pinned torch memory); read by the kernel
 *          over the host link, no staging copy.
 *   idx [B][cap], count [B], hot [B][cap][row_bytes] device.
 *   row_bytes: a positive multiple of 16.  Indices outside [0, N) are skipped and
 *   raise *status (if not NULL) to LSA_ERR_RANGE.
 * Launch it on a side stream to overlap the host-link transfer with scoring.
 * ---------------------------------------------------------------------------------- */
int lsa_gather_cold(int B, int N, size_t row_bytes, const void* cold_host,
                    const int32_t* idx, const int32_t* count, int cap, void* hot,
                    int32_t* status, void* stream);

/* ------------------------------------------------------------------------------------
 * Hot-pool residency across triggers ([SUMMARY] §2.1 and [REVIEW] 二: every tau decode
 * steps the indexer predicts which compressed KV blocks will be needed, and only those
 * are kept in GPU memory, fetched from the CPU cold pool).  The pages do not say what
 * becomes of a row fetched by an earlier trigger; here it stays in its slot until a
 * later trigger needs the slot, so only rows not yet resident cross the host link.
 *
 * State (device, caller-allocated, lsa_hot_pool_state_bytes; 256-byte aligned), four
 * arrays at the offsets lsa_hot_pool_layout returns:
 *   slot_of  [B][N] int32      slot holding entry e, or -1
 *   entry_of [B][slots] int32  entry held by slot s, or -1 (free)
 *   stamp    [B][slots] uint32 last trigger whose fetch set held the slot's entry (0: never)
 *   resident [B][ceil(N/32)] uint32 bits, bit e set iff slot_of[e] >= 0
 * lsa_hot_pool_reset empties the pool (no kernel: four memsets on the stream).
 *
 * lsa_hot_pool_update, for trigger index `trigger` (>= 1, increasing across calls) and
 * fetch set U [B][ceil(N/32)] (bits past N ignored), per sequence b:
 *   1. resident entries of U keep their slots; their stamp becomes `trigger`;
 *   2. if |U| > slots nothing moves and *status is raised to LSA_ERR_CAPACITY;
 *   3. else the missing entries of U (ascending) take the free or least recently
 *      needed slots: slots not kept, ordered by (stamp, slot index), the first as many
 *      as needed, paired in ascending slot order; each evicts the entry it held;
 *   4. hot[b][slot][0..row_bytes) = cold[b][entry][0..row_bytes) for each move.
 *   moved [B] (device, or NULL): rows moved per sequence.
 *   cold  HOST pointer [B][N][row_bytes], page-locked and mapped (as lsa_gather_cold);
 *   hot   device [B][slots][row_bytes]; slots >= 1; row_bytes a positive multiple of 16.
 *   workspace: lsa_hot_pool_workspace_bytes(B, N, slots) bytes, 256-byte aligned.
 * Six launches for B <= 4096 (the move step runs per block of 4096 sequences, the slot
 * keys per block of 65535); asynchronous on `stream`; calls on one state must not overlap.
 * ---------------------------------------------------------------------------------- */
size_t lsa_hot_pool_state_bytes(int B, int N, int slots);
size_t lsa_hot_pool_workspace_bytes(int B, int N, int slots);
/* offsets[0..3] = byte offsets of slot_of, entry_of, stamp, resident in the state */
int lsa_hot_pool_layout(int B, int N, int slots, size_t offsets[4]);
int lsa_hot_pool_reset(int B, int N, int slots, void* state, void* stream);
int lsa_hot_pool_update(int B, int N, int slots, size_t row_bytes, uint32_t trigger,
                        const uint32_t* U, const void* cold_host, void* hot, void* state,
                        int32_t* moved, int32_t* status,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_index_train_step -- loss and gradients of one indexer training step ([SUMMARY]
 * §2.3: K_IComp frozen, only the query-side projections trained, BCE combined with a
 * focal loss; §2.2: vote labels).  For P query positions of one indexer layer against N
 * frozen keys:
 *   c = h W_down, q = c W_up (both rounded to bf16), w = h W_w;
 *   z_ps = sum_h w_ph ReLU(q_ph . k_s) + bias;  prob = sigmoid(z) clamped to [2^-20, 1 - 2^-20];
 *   J = mean BCE(prob, y) + mean focal(prob, y; gamma) over all P*N pairs;
 *   outputs: loss[0] = mean BCE, loss[1] = mean focal (device doubles, or NULL);
 *   dW_down [D][r], dW_up [r][H*dI], dW_w [D][H] fp32 = dJ/dW; *dbias = dJ/dbias (device
 *   double, or NULL).  The bf16 roundings pass gradients straight through; where the
 *   probability clamp is active the derivative is zero.
 *   h [P][D], W_down [D][r], W_up [r][H*dI], W_w [D][H]: bf16 (wdt = LSA_BF16).
 *   K [N][dI] bf16 (kdt = LSA_BF16, kscale NULL); labels [P][ceil(N/32)] bits.
 *   c_in [P][r] bf16, q_in [P][H][dI] bf16, w_in [P][H] fp32: all three (the forward
 *   projection, e.g. from lsa_index_project) or none (then projected here; P <= 256).
 *   Supported: H in {32, 64, 128}, dI in {64, 128}, P a multiple of 128/H and at most
 *   4096; else LSA_ERR_UNSUPPORTED.  workspace: lsa_index_train_step_workspace_bytes bytes.
 *   The product of the keys with the positions' queries (forward) and with the gated
 *   gradients (backward) runs on the tensor cores; a stalled pipeline ends as
 *   LSA_ERR_TIMEOUT in *status.
 * ---------------------------------------------------------------------------------- */
size_t lsa_index_train_step_workspace_bytes(int P, int N, int D, int r, int H, int dI);
int lsa_index_train_step(int P, int N, int D, int r, int H, int dI, int wdt,
                         const void* h, const void* W_down, const void* W_up, const void* W_w, float bias,
                         int kdt, const void* K, const float* kscale, const uint32_t* labels, float gamma,
                         const void* c_in, const void* q_in, const float* w_in,
                         double* loss, float* dW_down, float* dW_up, float* dW_w, double* dbias,
                         int32_t* status, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_check_bounded_wait -- self-check of the pipeline waits (no counterpart on the pages).
 * Every wait inside the tensor-core kernels is bounded: when a pipeline stage does not
 * arrive within its limit (2 s) the kernel drains what it issued, frees its tensor
 * memory, raises the status word to LSA_ERR_TIMEOUT and returns.  This call launches one
 * kernel whose wait, the same bounded wait shortened to limit_us (1 .. 2,000,000), is on
 * a barrier that nothing arrives at: *status (device) becomes LSA_ERR_TIMEOUT after about
 * limit_us and the context stays usable.
 * Environment: LSA_FAULT=launch makes every call report a failed launch (LSA_ERR_CUDA),
 * for testing callers' error paths; it is read once per process.
 * ---------------------------------------------------------------------------------- */
int lsa_check_bounded_wait(uint32_t limit_us, int32_t* status, void* stream);

/* ------------------------------------------------------------------------------------
 * lsa_vote_labels -- cross-layer majority-vote golden labels and their loss
 * ([SUMMARY] §2.2: softmax over the indexer logits, per-layer nucleus top-p, an entry
 * is golden when at least theta of the L layers select it; §2.3 / [REVIEW] 二: BCE
 * plus focal loss).  For each (layer l, position p):
 *     pi = softmax_N(logits[l][p]);  S_{l,p} = nucleus: entries in descending pi
 *     (equal pi: lower index first) whose preceding mass is < top_p.
 *     count[p][s] = #{l : s in S_{l,p}};  golden[p] bit s = count >= theta.
 *   logits [L][P][N] fp32, golden [P][Nw] uint32, counts [P][N] uint8 or NULL.
 *   L <= 255 and P <= 65535, else LSA_ERR_UNSUPPORTED.
 *   scores [P][N] fp32 probabilities in (0,1) or NULL; when given, loss[0] = mean BCE
 *   and loss[1] = mean focal loss with exponent gamma over all P*N (device doubles).
 * workspace: lsa_vote_labels_workspace_bytes(L, P, N) bytes.
 * ---------------------------------------------------------------------------------- */
size_t lsa_vote_labels_workspace_bytes(int L, int P, int N);

int lsa_vote_labels(int L, int P, int N, const float* logits, float top_p, int theta,
                    uint32_t* golden, uint8_t* counts,
                    const float* scores, float gamma, double* loss,
                    void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
