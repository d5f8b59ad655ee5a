/*
 * rsm.h -- C ABI of librsm, a B200 (sm_100a) implementation of the routing-state-model (RSM)
 * sequence mixer of Raven ("Raven: High-Recall Sequence Modeling with Sparse Memory Routing").
 *
 * The mixer, per batch b, head h and token t (Raven README, github.com/xiaol/SelectingMemory,
 * "How Raven Works"):
 *   S_t      = the K of M slots with the largest router logits (ties: lower slot index first)
 *   s_i      = sigmoid(logit_i)                         for i in S_t, 0 otherwise
 *   a_i      = exp(s_i * f)                             f = per-head or per-slot log-decay, f <= 0
 *   H[i,:]   = a_i * H[i,:] + (1 - a_i) * k_i * v       for i in S_t; other rows keep their bits
 *   o_t      = sum_i q_i * H[i,:]                       (read after the write)
 * with a state H of M slot rows by Dv columns per (b,h). "Model Structure" of the same README
 * names the two decay families (Mamba2: one log-decay per head and token; GLA: one per slot) and
 * the two kernels (chunked for training/prefill, fused recurrent for generation).
 *
 * Conventions for every entry point:
 *   - The caller owns all memory. Pointers are DEVICE pointers unless stated otherwise, 16-byte
 *     aligned, row-major and contiguous in the layouts given below. The library never allocates.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Work is
 *     enqueued asynchronously; argument errors are returned synchronously before any launch,
 *     and a failed launch returns RSM_ERR_CUDA. rsm_last_error() describes the last failure of
 *     the calling host thread.
 *   - Logits and f must be finite and f <= 0 (a very negative finite f stands for "forget").
 *     These are preconditions; they are checked only when RSM_FLAG_VALIDATE is set.
 *   - Slots not selected at a step (decode) or in the whole call (prefill) are left bit-identical
 *     in the state.
 *   - Supported sizes: 32 <= M <= 256 with M a power of two, 1 <= K <= M, 1 <= Dv <= 256 with
 *     Dv % 4 == 0. Other sizes return RSM_ERR_UNSUPPORTED.
 */
#ifndef RSM_H_
#define RSM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RSM_API __attribute__((visibility("default")))
#else
#define RSM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rsm_status {
  RSM_OK = 0,
  RSM_ERR_INVALID_ARG = 1,  /* null pointer where one is required, bad size, misalignment */
  RSM_ERR_UNSUPPORTED = 2,  /* valid arguments outside the sizes this build implements */
  RSM_ERR_CUDA = 3,         /* a CUDA call or launch failed; see rsm_last_error() */
  RSM_ERR_NONFINITE = 4,    /* RSM_FLAG_VALIDATE found a non-finite logit or a non-finite/positive f */
  RSM_ERR_WORKSPACE = 5,    /* workspace missing or smaller than rsm_forward_workspace_size() */
  RSM_ERR_TIMEOUT = 6       /* a bounded device wait gave up (reported by rsm_get_device_status) */
} rsm_status;

typedef enum rsm_dtype { RSM_F32 = 0, RSM_BF16 = 1 } rsm_dtype;

typedef enum rsm_decay {
  RSM_DECAY_HEAD = 0,  /* f has one value per (b,t,h): Mamba2-style scalar log-decay            */
  RSM_DECAY_SLOT = 1   /* f has one value per (b,t,h,slot): GLA-style per-slot log-decay         */
} rsm_decay;

typedef enum rsm_path {
  RSM_PATH_AUTO = 0,    /* tensor-core path when the shape allows it, else the CUDA-core path    */
  RSM_PATH_SIMT = 1,    /* CUDA-core fp32 chunked path (any supported size, any input dtype)     */
  RSM_PATH_TENSOR = 2   /* tcgen05/TMEM tensor-core path; RSM_ERR_UNSUPPORTED when not available */
} rsm_path;

/* Router score of a selected slot (the selected set is the same for every variant: both scores
 * are monotone in the logit). Raven README "Model Structure" (top-k sigmoid/softmax router) and
 * "Usage" (router_score 'sigmoid' or 'softmax'); paperlayer.ai summary section 6.2.1 (sigmoid vs
 * softmax scores) and section 4.1 (the selected weights are normalised to sum to one). */
typedef enum rsm_router {
  RSM_ROUTER_SIGMOID = 0,       /* s_i = sigmoid(l_i) (default; the README pseudocode)                 */
  RSM_ROUTER_SOFTMAX = 1,       /* s_i = e^{l_i} / sum over all M slots of e^{l_j}                    */
  RSM_ROUTER_SIGMOID_NORM = 2,  /* sigmoid scores divided by their sum over the K selected slots      */
  RSM_ROUTER_SOFTMAX_NORM = 3   /* softmax scores divided by their sum over the K selected slots      */
} rsm_router;

enum {
  /* Device-side check of the preconditions: a non-finite logit or a non-finite or positive f is
   * reported as RSM_ERR_NONFINITE by rsm_get_device_status (results are then undefined). */
  RSM_FLAG_VALIDATE = 1,
  /* Testing aid for the bounded-wait error paths (no counterpart on the pages; never set in normal
   * use): in rsm_decode_step the routing warps hand over no routing slot and the warps waiting for
   * one give up after a short bound, so every CTA takes its timeout exit, the call writes neither o
   * nor the state, and rsm_get_device_status reports RSM_ERR_TIMEOUT. In rsm_backward the first token's
   * copy is withheld and the sweeps' waits get a bound of one poll, so the first wait expires with
   * the next tokens' copies in flight: the kernel stops, drains those copies (with the normal
   * bound) and reports RSM_ERR_TIMEOUT; the gradients are then undefined. Other calls ignore it. */
  RSM_FLAG_TEST_STALL_ROUTING = 256
};

/* ---------------------------------------------------------------------------------------------
 * rsm_route -- TopK routing of router logits.
 *   Raven README "How Raven Works" (route_scores = TopK(sigmoid(r_proj(x)))); paperlayer.ai summary
 *   section 4.1 (keep the top-K scores, set the rest to zero). Ranking is on the fp32 logits
 *   (sigmoid is monotone and saturates in fp32); exact ties go to the lower slot index, and
 *   -0.0 ties +0.0.
 *   logits    [rows, M] fp32 (device)
 *   idx_out   [rows, K] int32 (device): selected slots in rank order (logit desc, index asc)
 *   score_out [rows, K] fp32 (device, may be NULL): sigmoid(logit) of each selected slot
 *   rows may be 0 (nothing is launched).
 * ------------------------------------------------------------------------------------------- */
RSM_API rsm_status rsm_route(const float* logits, int64_t rows, int M, int K, int32_t* idx_out,
                     float* score_out, void* stream);

/* rsm_route with a router variant (score_out holds that variant's scores) and RSM_FLAG_* flags
 * (RSM_FLAG_VALIDATE reports non-finite logits through rsm_get_device_status). */
RSM_API rsm_status rsm_route_ex(const float* logits, int64_t rows, int M, int K, rsm_router router,
                                int flags, int32_t* idx_out, float* score_out, void* stream);

/* ---------------------------------------------------------------------------------------------
 * rsm_forward -- chunked prefill over T tokens.
 *   The recurrence above, evaluated chunk by chunk (paperlayer.ai summary, section A.5: the
 *   sequence is split into n chunks of length C, T = n*C, for stability and parallelism; a
 *   ragged last chunk is allowed here). The result does not depend on the chunk length beyond
 *   rounding.
 *   q, k    [B,T,H,M] in qkv_dtype (fp32 or bf16)
 *   v       [B,T,H,Dv] in qkv_dtype
 *   logits  [B,T,H,M] fp32
 *   f       [B,T,H] fp32 (RSM_DECAY_HEAD) or [B,T,H,M] fp32 (RSM_DECAY_SLOT)
 *   H0      [B,H,M,Dv] fp32 initial state, or NULL for zeros. May alias HT.
 *   o       [B,T,H,Dv] fp32 output (required)
 *   HT      [B,H,M,Dv] fp32 final state, or NULL to skip
 *   idx_out, score_out  [B,T,H,K] (int32, fp32), or NULL to skip: the routing of every token
 *   workspace / workspace_bytes: device scratch of at least rsm_forward_workspace_size(args)
 *     bytes (256-byte aligned); may be NULL when that size is 0. Its contents are not preserved.
 *   path: which implementation to run (RSM_PATH_AUTO normally).
 * ------------------------------------------------------------------------------------------- */
typedef struct rsm_forward_args {
  int B, T, H, M, K, Dv;
  rsm_dtype qkv_dtype;
  rsm_decay decay;
  const void* q;
  const void* k;
  const void* v;
  const float* logits;
  const float* f;
  const float* H0;
  float* o;
  float* HT;
  int32_t* idx_out;
  float* score_out;
  void* workspace;
  size_t workspace_bytes;
  rsm_path path;
  int flags; /* RSM_FLAG_* */
  rsm_router router;     /* score of the selected slots (RSM_ROUTER_SIGMOID = 0 by default)        */
  int32_t* slot_counts;  /* [B,H,M] int32 or NULL: the number of tokens of the call that selected
                            each slot is ADDED to it (the per-slot counts behind the paper's
                            "effective sequence length" analysis, paperlayer.ai summary 7.1) */
} rsm_forward_args;

/* Bytes of device workspace rsm_forward needs for these arguments (0 when none). Depends only on
 * the sizes, dtype, decay and path fields. Returns (size_t)-1 for arguments rsm_forward rejects. */
RSM_API size_t rsm_forward_workspace_size(const rsm_forward_args* args);
RSM_API rsm_status rsm_forward(const rsm_forward_args* args, void* stream);

/* The implementation rsm_forward would run for these arguments: RSM_PATH_SIMT or RSM_PATH_TENSOR
 * (RSM_PATH_AUTO resolved), or -1 for arguments rsm_forward rejects. Host-only. */
RSM_API int rsm_forward_selected_path(const rsm_forward_args* args);

/* Number of kernel launches one rsm_forward call makes for these arguments (for accounting and
 * profiling: tensor path = routing records + [segment summary + segment scan +] chunk scan; SIMT
 * path = 1; 0 when B*H == 0 or T == 0), or -1 for arguments rsm_forward rejects. Host-only. */
RSM_API int rsm_forward_kernel_launches(const rsm_forward_args* args);

/* Profiling aid (no counterpart on the pages): while set, every rsm_forward call made on the
 * calling host thread records `events[0]` on its stream before its first kernel and `events[i]`
 * after its i-th kernel (i = 1 .. rsm_forward_kernel_launches(args)), so that the caller can time
 * each kernel with cudaEventElapsedTime. `events` are cudaEvent_t handles passed as void*, owned
 * by the caller; `n_events` must be at least the launches of the calls that follow plus one (a
 * call that needs more returns RSM_ERR_INVALID_ARG before any launch). NULL / 0 stops recording.
 * The events are only recorded, never waited on or destroyed, by the library. Host-only. */
RSM_API rsm_status rsm_forward_set_profile_events(void* const* events, int n_events);

/* ---------------------------------------------------------------------------------------------
 * rsm_forward_noalloc -- rsm_forward for callers that cannot allocate device memory.
 *   The pages have no counterpart to this call; it exists for callers with no way to allocate:
 *   work recorded into a CUDA graph capture (an allocation would break the capture), programs
 *   whose allocator owns every byte of the device, or runtimes with a fixed memory plan. Where
 *   rsm_forward needs a caller-supplied workspace (the tensor-core path: routing records of every
 *   token, 144 bytes per token and head for K <= 16 and 288 for K <= 32, plus the segment states
 *   when a long sequence is split), this call uses a scratch array built into the library instead;
 *   the caller passes only the inputs and outputs (args->workspace and args->workspace_bytes are
 *   ignored). Results are bit-identical to those of rsm_forward.
 *   Limit: the scratch holds rsm_forward_noalloc_max_scratch() bytes (16 MiB), about 116,000
 *   token-heads (B*T*H) at K <= 16 before segment states; sizes whose workspace would exceed it
 *   return RSM_ERR_WORKSPACE with the sizes in rsm_last_error(), before anything is launched.
 *   The array occupies device memory on every GPU that loads the library, until exit. The first
 *   call on each device (and the first after a device reset) looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before any stream
 *   capture. All calls share the array and it keeps the last call's contents (nothing in it needs
 *   to start at zero): calls whose GPU work overlaps in time, on any streams or host threads of
 *   one device, race and must not be issued. No CUDA allocation routine is called.
 * ------------------------------------------------------------------------------------------- */
RSM_API rsm_status rsm_forward_noalloc(const rsm_forward_args* args, void* stream);
RSM_API size_t rsm_forward_noalloc_max_scratch(void);

/* ---------------------------------------------------------------------------------------------
 * rsm_decode_step -- one generation token per (b,h): fused routing, sparse decay/write of the K
 *   selected rows of the carried state in place, and the read o = q.H over all M rows.
 *   Raven README "Model Structure" (fused recurrent computation for inference).
 *   q, k    [B,H,M] in qkv_dtype;  v [B,H,Dv] in qkv_dtype
 *   logits  [B,H,M] fp32;          f [B,H] or [B,H,M] fp32
 *   state   [B,H,M,Dv] fp32, read and updated in place (only the K selected rows are written)
 *   o       [B,H,Dv] fp32 output
 *   idx_out, score_out [B,H,K] or NULL
 * ------------------------------------------------------------------------------------------- */
typedef struct rsm_decode_args {
  int B, H, M, K, Dv;
  rsm_dtype qkv_dtype;
  rsm_decay decay;
  const void* q;
  const void* k;
  const void* v;
  const float* logits;
  const float* f;
  float* state;
  float* o;
  int32_t* idx_out;
  float* score_out;
  int flags; /* RSM_FLAG_* */
  rsm_router router;     /* score of the selected slots (RSM_ROUTER_SIGMOID = 0 by default)        */
  int32_t* slot_counts;  /* [B,H,M] int32 or NULL: 1 is added for every slot selected at the step */
} rsm_decode_args;

RSM_API rsm_status rsm_decode_step(const rsm_decode_args* args, void* stream);

/* ---------------------------------------------------------------------------------------------
 * rsm_backward -- gradients of the prefill (training). Reverse-mode differentiation of the
 *   recurrence above with the sigmoid router: given dO = dL/do and dHT = dL/dH_T, it returns
 *   dL/dq, dL/dk, dL/dv, dL/dlogits, dL/df and dL/dH0. The TopK cut is piecewise constant in the
 *   logits, so unselected slots get no key or logit gradient. Raven README "Model Structure"
 *   (chunked computation for training) and the fork's reverse-scan backward.
 *   Inputs as rsm_forward (q, k, v in qkv_dtype; logits, f, H0 fp32; H0 may be NULL = zeros)
 *   dO    [B,T,H,Dv] fp32, or NULL for zero
 *   dHT   [B,H,M,Dv] fp32, or NULL for zero
 *   dq, dk, dlogits [B,T,H,M] fp32; dv [B,T,H,Dv] fp32; df [B,T,H] or [B,T,H,M] fp32;
 *   dH0 [B,H,M,Dv] fp32 (each output may be NULL to skip it)
 *   workspace: at least rsm_backward_workspace_size(args) bytes (256-byte aligned): the routing
 *     of every token, its K entries (slot, decay, write weight, score, rate, key; 32 bytes each)
 *     and a tape of the K state rows each token overwrites (T*K*Dv*4 bytes per (b,h) stream).
 *   Supported: the sizes of rsm_forward with M*Dv <= 24576 (the state and its gradient stay in
 *   shared memory), router RSM_ROUTER_SIGMOID. The arithmetic is fp32 on CUDA cores.
 * ------------------------------------------------------------------------------------------- */
typedef struct rsm_backward_args {
  int B, T, H, M, K, Dv;
  rsm_dtype qkv_dtype;
  rsm_decay decay;
  const void* q;
  const void* k;
  const void* v;
  const float* logits;
  const float* f;
  const float* H0;
  const float* dO;
  const float* dHT;
  float* dq;
  float* dk;
  float* dv;
  float* dlogits;
  float* df;
  float* dH0;
  void* workspace;
  size_t workspace_bytes;
  rsm_router router;
  int flags; /* RSM_FLAG_* */
} rsm_backward_args;

/* Bytes of workspace rsm_backward needs, or (size_t)-1 for arguments it rejects. Host-only. */
RSM_API size_t rsm_backward_workspace_size(const rsm_backward_args* args);
RSM_API rsm_status rsm_backward(const rsm_backward_args* args, void* stream);

/* Human-readable name of a status code (static storage). */
RSM_API const char* rsm_status_string(rsm_status status);

/* Detail of the last failure on the calling host thread ("" if none). */
RSM_API const char* rsm_last_error(void);

/* Synchronizes `stream`, then reads and clears the library's device status word for the current
 * device: RSM_OK, RSM_ERR_NONFINITE (validation found bad inputs) or RSM_ERR_TIMEOUT (a bounded
 * device wait expired). Errors of the synchronization itself return RSM_ERR_CUDA. */
RSM_API rsm_status rsm_get_device_status(void* stream);

/* Library version as major*10000 + minor*100 + patch. */
RSM_API int rsm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RSM_H_ */
