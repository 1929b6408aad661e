/*
 * moe_b200.h -- C ABI of the single-GPU Mixture-of-Experts layer forward for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (sources: "ops-transformer MoE operators" blog, 原理 Steps 1-4 and
 * 实现; "MoE Router: who decides which expert a token goes to"; "MegaBlocks 01 -
 * why MoE is hard", sections 1-5; "Integrating MoE into your model with
 * Colossal-AI", step 2):
 *
 *   route    logits = x Wg (+ b), p = softmax(logits), top-k (ties -> lower
 *            expert index), w = p_sel / sum(p_sel), aux = E * sum_i f_i P_i
 *   permute  histogram of the T*k slots per expert, inclusive scan (bins),
 *            stable counting sort on the low max(ceil(log2 E),1) key bits,
 *            capacity C = int(cf * k * T / E) with drop by arrival order
 *   gather   x_perm[row] = x[slot / k] for every kept slot, expert-contiguous
 *   ffn      per expert e over its rows: SwiGLU  h = silu(x W_gate[e]) * (x W_up[e])
 *                                      GELU    h = gelu(x W1[e])          (exact erf)
 *            then y = h W_down[e] (or h W2[e])
 *   combine  out[t] = sum_{j<k, slot kept} w[t,j] * y[row(t,j)]   (zero if all dropped)
 *
 * Conventions for every entry point below:
 *  - All tensor pointers are DEVICE pointers unless the name says host, and
 *    are owned by the caller. The library never allocates or frees device
 *    memory and never synchronises the stream, except moe_get_device_error.
 *  - Layouts are row-major. A slot is s = t * k + j (token t, choice j).
 *    Weights: Wg [d, E]; W1 / W_gate / W_up [E, d, F]; W2 / W_down [E, F, d]
 *    (the [E, hs, ffn] layout of the MegaBlocks page, section 4.3).
 *  - Gathered rows: the kept slots of expert 0 in ascending slot order, then
 *    expert 1, ...; expert e owns rows [seg_offsets[e], seg_offsets[e+1]).
 *  - dtype MOE_BF16: x, weights, x_perm, h, y_perm and out are bf16; router
 *    logits/probabilities/weights, the bias and the aux loss are fp32 and all
 *    accumulation is fp32. dtype MOE_F32: every tensor is fp32.
 *  - Limits: 1 <= E <= 256, 1 <= k <= min(E, 8), T >= 0, T * k < 2^31.
 *    bf16: d % 128 == 0 and F % 128 == 0. f32: d % 4 == 0 and F % 4 == 0.
 *    Every device pointer 16-byte aligned.
 *  - Host-checkable problems return a status synchronously and launch
 *    nothing. Data-dependent problems found on the device (an expert id out of
 *    range, a row index out of range, a bounded wait that timed out) set bits
 *    in a device error word kept in the first bytes of the workspace; kernels
 *    never trap and never write out of bounds; outputs of that call are then
 *    unspecified. Read the word with moe_get_device_error.
 *  - Workspace: every entry point takes (ws, ws_bytes). Its first 256 bytes
 *    are a control block (error word and counters) that must be zeroed once
 *    with moe_workspace_init before first use; the same workspace may then be
 *    reused by any number of calls on one stream. Calls that share a
 *    workspace must not run concurrently.
 *  - stream: a cudaStream_t (NULL = legacy default stream).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same object as cudaStream_t */
typedef struct CUevent_st* moe_event_t;   /* same object as cudaEvent_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_NULL = 1,        /* a required pointer is NULL */
  MOE_ERR_INVALID = 2,     /* a size or parameter is out of range */
  MOE_ERR_UNSUPPORTED = 3, /* valid but outside this build's limits (divisibility) */
  MOE_ERR_WORKSPACE = 4,   /* ws_bytes smaller than the matching *_workspace_size */
  MOE_ERR_ALIGN = 5,       /* a pointer is not 16-byte aligned */
  MOE_ERR_CUDA = 6,        /* a CUDA call or kernel launch failed */
  MOE_ERR_DEVICE = 7       /* the device error word is non-zero */
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;
typedef enum { MOE_ACT_GELU = 0, MOE_ACT_SWIGLU = 1 } moe_act_t;

/* Bits of the device error word. */
#define MOE_DEVERR_EXPERT_RANGE 0x1u /* a top-k expert id outside [0, E), or a router
                                        row with fewer than k selectable logits
                                        (NaN is never selected); expert 0 is
                                        written in that pick's place */
#define MOE_DEVERR_ROW_RANGE 0x2u    /* a slot/row index outside its buffer */
#define MOE_DEVERR_TIMEOUT 0x4u      /* a bounded on-chip wait gave up */

/* One MoE layer: shapes, activation, capacity and the weight pointers. */
typedef struct {
  int d;                    /* hidden size */
  int E;                    /* number of experts */
  int k;                    /* experts per token */
  int F;                    /* expert FFN size */
  moe_dtype_t dtype;
  moe_act_t act;
  double capacity_factor;   /* <= 0: dropless; else C = int(cf * (k * T / E)) */
  const void* w_router;     /* Wg [d, E] */
  const float* router_bias; /* fixed logit bias [E] (fp32) or NULL */
  const void* w1;           /* W_gate (SwiGLU) or W1 (GELU), [E, d, F] */
  const void* w3;           /* W_up [E, d, F] (SwiGLU), NULL for GELU */
  const void* w2;           /* W_down / W2 [E, F, d] */
  int flags;                /* MOE_LAYER_* bits, 0 for the default path */
  /* Training-side router inputs (NULL for inference):
   *   x_router     the router's input [T, d] (dtype) in place of x, e.g. x
   *                jittered by moe_router_jitter; the experts still read x
   *   logit_noise  [T, E] fp32 added to the gate logits after the bias,
   *                e.g. from moe_router_noise
   *   router_temperature  the softmax's tau (see moe_route_train); 0 means 1 */
  const void* x_router;
  const float* logit_noise;
  float router_temperature;
} moe_layer_t;

/* moe_layer_t.flags. MOE_LAYER_GATHER_IN_GEMM (bf16 only): moe_forward skips
 * the gather kernel and x_perm; the up projection loads its A rows straight
 * from x with TMA tile::gather4 (row r = token row_slot[r] / k). Same results
 * bit for bit; slower on every workload measured on B200 (each A tile is
 * re-gathered for every output column block), so it is off by default. */
#define MOE_LAYER_GATHER_IN_GEMM 1
/* MOE_LAYER_BINNED: the padded-binned [E, C, hs] layout of the pages'
 * standard MoE path ("MegaBlocks", sections 4.3-4.6; see moe_permute_binned):
 * expert e's rows are [e*C, e*C + kept_counts[e]) of a bucket of E*C rows
 * (gathered padding rows are zero). capacity_factor > 0 fixes C =
 * int(cf * k * T / E); capacity_factor <= 0 means dynamic capacity, C = the
 * largest per-expert count of the call (nothing dropped), computed on the
 * device, and the workspace is sized for the worst case C = T*k. The layer's
 * output is the same as the default layout's; only the intermediates'
 * layout differs. The expert FFN (bf16) skips the padding rows: h and y_perm
 * rows past kept_counts[e] in each bin are not written. */
#define MOE_LAYER_BINNED 2
/* MOE_LAYER_Z_LOSS: moe_forward also computes the router z-loss (see
 * moe_route_train) into the workspace (moe_views_t.z_loss). */
#define MOE_LAYER_Z_LOSS 4
/* MOE_LAYER_COMBINE_IN_GEMM (bf16, k = 1 only; MOE_ERR_UNSUPPORTED
 * otherwise): the combine runs in the down projection's epilogue ("MegaBlocks"
 * section 4.3 multiplies each expert output by its gate weight as it is
 * scattered back to the token). Each row's output, rounded to bf16 as y_perm
 * would hold it, is multiplied by its slot's weight in fp32 and written
 * straight to its token's row of out; the gather kernel zeroes the rows of
 * tokens whose slot was dropped. No combine kernel and no y_perm; out is the
 * same as the default path's bit for bit. */
#define MOE_LAYER_COMBINE_IN_GEMM 8

/* Device pointers into a moe_forward workspace where that call leaves its
 * intermediate results (see moe_forward_views). */
typedef struct {
  int32_t* topk_idx;     /* [T, k] */
  float* topk_w;         /* [T, k] */
  float* aux_loss;       /* [1] */
  float* z_loss;         /* [1], written with MOE_LAYER_Z_LOSS */
  int32_t* counts;       /* [E] */
  int32_t* bins;         /* [E] */
  int32_t* kept_counts;  /* [E] */
  int32_t* seg_offsets;  /* [E + 1] */
  int32_t* sorted_slot;  /* [T * k] */
  int32_t* slot_to_row;  /* [T * k] */
  int32_t* row_slot;     /* [rows_max] */
  uint8_t* drop_mask;    /* [T * k] */
  void* x_perm;          /* [rows_max, d]; NULL with MOE_LAYER_GATHER_IN_GEMM */
  void* h;               /* [rows_max, F] */
  void* y_perm;          /* [rows_max, d]; NULL with MOE_LAYER_COMBINE_IN_GEMM */
  int64_t rows_max;
  int64_t capacity;      /* C, or -1 when dropless */
} moe_views_t;

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(moe_status_t status);

/* Zero the control block (first 256 bytes) of a workspace, asynchronously
 * on `stream`. Needed once per workspace before its first use, and again
 * after a call reported MOE_DEVERR_TIMEOUT: a wait that gave up leaves the
 * grid-barrier words of the control block in an unknown state, and the next
 * call on that workspace could pass its barrier early. Zeroing also clears
 * the error word and restores the default wait limit. */
MOE_API moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Set how long a kernel using this workspace waits at a barrier between its
 * CTAs (the permute's grid barrier, where every CTA waits for all others to
 * publish their counts) before it gives up: it then sets MOE_DEVERR_TIMEOUT,
 * skips the work that needed the barrier and returns, leaving the GPU
 * context usable. limit_us in microseconds; 0 restores the default of 2 s.
 * Written asynchronously on `stream` (one small kernel). The waits inside a
 * CTA (on TMA and tensor-core completion) keep their fixed 2 s bound. */
MOE_API moe_status_t moe_workspace_set_wait_limit(void* ws, size_t ws_bytes, uint32_t limit_us,
                                                  moe_stream_t stream);

/* Number of CUDA kernels this library has launched in this process so far
 * (all devices, all streams, every entry point), counted on the host at each
 * launch. Read it before and after a region to count that region's launches.
 * Never fails; needs no device. */
MOE_API uint64_t moe_kernel_launches(void);

/* Read (synchronises `stream`) and optionally clear the device error word of
 * a workspace into *host_bits. Returns MOE_ERR_DEVICE if it was non-zero. */
MOE_API moe_status_t moe_get_device_error(void* ws, moe_stream_t stream, uint32_t* host_bits,
                                  int clear);

/* Capacity C = int(cf * (k * T / E)) evaluated in double, as the MegaBlocks
 * page's expert_capacity (section 4.2, world size 1); -1 (dropless) when
 * cf <= 0. */
MOE_API int64_t moe_capacity(double capacity_factor, int T, int k, int E);

/* Upper bound on gathered rows: T*k when capacity < 0 (dropless), else
 * min(T*k, E*C). */
MOE_API int64_t moe_rows_max(int T, int k, int E, int64_t capacity);

/* ------------------------------------------------------------------ route
 * Router gate Linear(d, E) without learned bias (+ optional fixed fp32 logit
 * bias), softmax over E, top-k by selection with ties to the lower expert
 * index (selection compares the fp32 logits), renormalisation of the k
 * weights to sum 1, and the load-balance loss aux = E * sum_i f_i * P_i with
 * f_i = (slots routed to i, before any capacity drop) / (T*k) and
 * P_i = mean_t p[t,i]. ("ops-transformer MoE operators", 实现: softmax,
 * top-K selection, NormalizeWeights; "MoE Router": gate without bias,
 * softmax, topk, renormalise.)
 *   x          [T, d] (dtype)          w_router [d, E] (dtype)
 *   bias       [E] fp32 or NULL
 *   topk_idx   out [T, k] int32        topk_w out [T, k] fp32
 *   aux_loss   out [1] fp32 (device)
 *   logits, probs  optional out [T, E] fp32 (NULL to skip)
 *   ws         >= moe_route_workspace_size(T, d, E) bytes */
MOE_API size_t moe_route_workspace_size(int T, int d, int E);
MOE_API moe_status_t moe_route(const void* x, const void* w_router, const float* bias, moe_dtype_t dtype,
                       int T, int d, int E, int k, int32_t* topk_idx, float* topk_w,
                       float* aux_loss, float* logits, float* probs, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* moe_route with the training-side variants:
 *   logit_noise  [T, E] fp32 added to each logit after the bias, or NULL
 *                ("Integrating MoE into your model with Colossal-AI", step 2:
 *                NormalNoiseGenerator adds Gaussian noise to the gate logits;
 *                see moe_router_noise)
 *   z_loss       out [1] fp32 or NULL: mean over tokens of the squared
 *                log-sum-exp of the logits the softmax sees (bias and noise
 *                included). The pages name the loss only (router_z_loss);
 *                this is its usual definition. Deterministic (fixed-order
 *                reductions).
 *   temperature  tau > 0 (MOE_ERR_INVALID otherwise): the softmax sees
 *                logits / tau ("ops-transformer MoE operators", 坑3: soft
 *                top-K, a softmax with a temperature so that experts not
 *                picked keep some probability; no formula is given, this is
 *                the plain reading). The pick is unchanged; probabilities,
 *                weights, the aux loss's P_i and the z-loss use l / tau.
 *                tau = 1 gives moe_route's results bit for bit.
 * Probabilities, top-k, weights and the aux loss are those of the noisy
 * logits. For jitter, pass the jittered x (moe_router_jitter) as x. */
MOE_API moe_status_t moe_route_train(const void* x, const void* w_router, const float* bias,
                             const float* logit_noise, float temperature, moe_dtype_t dtype, int T,
                             int d, int E, int k, int32_t* topk_idx, float* topk_w,
                             float* aux_loss, float* z_loss, float* logits, float* probs, void* ws,
                             size_t ws_bytes, moe_stream_t stream);

/* Router backward: the gradients of
 *     L = sum_{t,j} d_topk_w[t,j] * topk_w[t,j] + d_aux * aux + d_z * z_loss
 * through the tempered softmax and the gate, with the pick and the aux
 * loss's counts held fixed ("ops-transformer MoE operators", 实现: the gating
 * operator has a forward and a backward; 坑3: gradients reach the experts
 * through the softmax; the pages print no formula, this is the chain rule of
 * moe_route_train's forward):
 *     dL/dp_{i_j} = (d_topk_w[t,j] - sum_m d_topk_w[t,m] topk_w[t,m]) / sum_j p_{i_j}
 *     dL/dp[t,e] += d_aux * E * f_e / T     (f_e = picks of e / (T*k))
 *     d_logits    = p * (dL/dp - sum_e p_e dL/dp_e) / tau
 *                   + d_z * (2/T) * lse(l_t / tau) * p / tau
 *     dx = d_logits Wg^T,  d_wg = x^T d_logits
 * The fixed bias and the logit noise take no gradient (d_logits is also
 * theirs, if a caller wants them).
 *   x, w_router   the forward's inputs, [T, d] and [d, E] (dtype)
 *   probs         [T, E] fp32, the forward's probabilities (at tau)
 *   logits        [T, E] fp32, the forward's logits before tau; read only
 *                 when d_z != 0 (NULL otherwise)
 *   topk_idx, topk_w  the forward's picks and renormalised weights [T, k]
 *   d_topk_w      [T, k] fp32 upstream gradient of topk_w, or NULL (zero)
 *   d_aux, d_z    upstream gradients of the two losses (host scalars)
 *   temperature   tau > 0, as in the forward
 *   d_logits      out [T, E] fp32, or NULL
 *   dx            out [T, d] (dtype, rounded once), or NULL
 *   d_wg          out [d, E] fp32, or NULL
 *   ws            >= moe_route_backward_workspace_size(T, d, E) bytes
 * d follows the general limits above (a multiple of 128 for bf16, of 4 for
 * fp32; MOE_ERR_UNSUPPORTED otherwise). d_logits is
 * computed in fp32. dx and d_wg: for bf16 with E <= 64 (16-byte aligned x,
 * w_router and d_logits) on the tensor cores, d_logits entering as two bf16
 * terms hi = bf16(v), lo = bf16(v - hi) (|v - hi - lo| <= 2^-17 |v| for
 * |v| >= 2^-117, <= 2^-134 below, where v - hi leaves bf16's normal range)
 * and the products summed in fp32; otherwise fp32 on CUDA cores. d_wg adds its
 * partial sums in a fixed order (deterministic). */
MOE_API size_t moe_route_backward_workspace_size(int T, int d, int E);
MOE_API moe_status_t moe_route_backward(const void* x, const void* w_router, moe_dtype_t dtype,
                                int T, int d, int E, int k, const float* probs,
                                const float* logits, const int32_t* topk_idx,
                                const float* topk_w, const float* d_topk_w, float d_aux,
                                float d_z, float temperature, float* d_logits, void* dx,
                                float* d_wg, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Router jitter ("MegaBlocks", section 5: the router input is multiplied by
 * uniform noise in [1 - eps, 1 + eps] during training): x_out = x * m with
 * m uniform in [1 - eps, 1 + eps) per element, from the counter-based
 * generator Philox4x32-10 (Salmon et al., SC 2011) keyed by seed. Element n =
 * t*d + i uses word n % 4 of the generator's call n / 4 on counter
 * (lo32, hi32, 0, 0): u = (word >> 8) * 2^-24, m = (1 - eps) + (2 eps) u in
 * fp32, x * m in fp32 (rounded to bf16 for bf16). 0 <= eps < 1. x and x_out
 * [T, d] (dtype), device; they may not overlap. */
MOE_API moe_status_t moe_router_jitter(const void* x, moe_dtype_t dtype, int T, int d, float eps,
                               uint64_t seed, void* x_out, moe_stream_t stream);

/* Gaussian logit noise noise_out [T, E] fp32 (device) = std_dev * N(0, 1), by
 * Box-Muller from Philox4x32-10: value n = t*E + e uses words 2(n % 2) and
 * 2(n % 2) + 1 of call n / 2 on counter (lo32, hi32, 1, 0). The Colossal-AI
 * page scales the noise by the number of experts: std_dev = 1/E in that
 * reading. */
MOE_API moe_status_t moe_router_noise(int T, int E, float std_dev, uint64_t seed, float* noise_out,
                              moe_stream_t stream);

/* ---------------------------------------------------------------- permute
 * Sorting metadata of the T*k slots by expert id ("MegaBlocks", section 4.1:
 * sort, histogram, inclusive cumsum; only max(ceil(log2 E),1) key bits are
 * sorted), then capacity drop by arrival order (sections 3, 4.2, 4.5).
 *   topk_idx     [T, k] int32, values in [0, E)
 *   capacity     C >= 0 (0 drops every slot), or any negative value for dropless
 *   counts       out [E]    slots per expert (before the drop)
 *   bins         out [E]    inclusive prefix sum of counts
 *   sorted_slot  out [T*k]  slots in stable order of expert id
 *   slot_to_row  out [T*k]  gathered row of each slot, -1 if dropped
 *   row_slot     out [moe_rows_max(...)]  slot of each gathered row (rows
 *                past seg_offsets[E] are left untouched)
 *   drop_mask    out [T*k]  1 if the slot is dropped (u8)
 *   kept_counts  out [E]    min(counts, C)
 *   seg_offsets  out [E+1]  exclusive prefix sum of kept_counts
 *   ws           >= moe_permute_workspace_size(T, k, E) bytes */
MOE_API size_t moe_permute_workspace_size(int T, int k, int E);
MOE_API moe_status_t moe_permute(const int32_t* topk_idx, int T, int k, int E, int64_t capacity,
                         int32_t* counts, int32_t* bins, int32_t* sorted_slot,
                         int32_t* slot_to_row, int32_t* row_slot, uint8_t* drop_mask,
                         int32_t* kept_counts, int32_t* seg_offsets, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* moe_permute into the padded-binned [E, C] layout ("MegaBlocks", sections
 * 4.3 binned_gather into [E, C, hs], 4.5 short bins zero-padded and ranks >= C
 * dropped, 4.6 capacity 0 = the largest per-expert count):
 *   capacity     C >= 0, or negative for dynamic capacity: C = max(counts),
 *                computed on the device (no slot dropped)
 *   slot_to_row  out [T*k]  e*C + (rank of the slot within expert e), -1 if dropped
 *   row_slot     out [moe_rows_max_binned(...)]  slot of each bucket row; -1
 *                for padding rows; rows past seg_offsets[E] = E*C untouched
 *   kept_counts  out [E]    min(counts, C)
 *   seg_offsets  out [E+1]  e*C (so seg_offsets[1] is C)
 * counts, bins, sorted_slot and drop_mask as moe_permute. */
MOE_API moe_status_t moe_permute_binned(const int32_t* topk_idx, int T, int k, int E,
                                int64_t capacity, int32_t* counts, int32_t* bins,
                                int32_t* sorted_slot, int32_t* slot_to_row, int32_t* row_slot,
                                uint8_t* drop_mask, int32_t* kept_counts, int32_t* seg_offsets,
                                void* ws, size_t ws_bytes, moe_stream_t stream);

/* Rows of the binned bucket: E*C for capacity C >= 0, E*T*k (the worst case
 * of dynamic capacity) for capacity < 0. */
MOE_API int64_t moe_rows_max_binned(int T, int k, int E, int64_t capacity);

/* --------------------------------------------------- permute, no allocation
 * The same permute for callers that cannot allocate device memory: code that
 * runs where the CUDA allocator is not reachable or not allowed (a library
 * handed only pre-allocated tensors, a runtime whose memory pool is fixed
 * before the first call, a plugin in a process that forbids cudaMalloc after
 * start-up). It takes no workspace and calls no allocating routine. The paper
 * has no counterpart to this entry point; it exists for such callers only.
 *   Outputs and their meaning are those of moe_permute.
 *   device_error  out [1] u32 (device) or NULL: the call's device error bits.
 *   Limit: T*k <= MOE_PERMUTE_NOALLOC_MAX_SLOTS; larger sizes return
 *   MOE_ERR_WORKSPACE and launch nothing.
 * Its scratch is one file-scope static device array (256 bytes of control
 * block + 4 bytes per slot up to the limit, ~256 KB), which every GPU that
 * loads this library holds until the process exits. Each call looks up that
 * array's device address (cudaGetSymbolAddress, with the caller's device
 * current), so the address stays right after a cudaDeviceReset. The first
 * call on a device may load the library's device code (the CUDA runtime
 * loads modules lazily) and loading allocates device memory, the array
 * included: a caller that must not allocate makes one call at start-up, and
 * makes that first call before any stream capture. Every call shares the
 * array and clears its control block first: calls that overlap on the GPU
 * (other streams, other host threads) race and give wrong results. */
#define MOE_PERMUTE_NOALLOC_MAX_SLOTS 65536
MOE_API moe_status_t moe_permute_noalloc(const int32_t* topk_idx, int T, int k, int E,
                                         int64_t capacity, int32_t* counts, int32_t* bins,
                                         int32_t* sorted_slot, int32_t* slot_to_row,
                                         int32_t* row_slot, uint8_t* drop_mask,
                                         int32_t* kept_counts, int32_t* seg_offsets,
                                         uint32_t* device_error, moe_stream_t stream);

/* ------------------------------------------------ expert-parallel dispatch
 * Plans for running the experts on several ranks ("MoE Router: who decides
 * which expert a token goes to": per-device send counts with
 * device = expert / experts_per_device, an all-to-all-v with per-pair counts
 * and displacements, the experts computed where they live; "ops-transformer
 * MoE operators", 坑2: tokens go to the cards holding their experts and come
 * back after the compute; "Integrating MoE into your model with Colossal-AI",
 * step 2: all-to-all to the expert's GPU, expert MLP, all-to-all back).
 * Experts are owned in contiguous blocks: rank g holds experts
 * [g*E/world, (g+1)*E/world). Each rank routes, permutes (its own capacity)
 * and gathers its own tokens as on one GPU; because the gathered rows are
 * sorted by expert, the rows for rank g are one contiguous range of x_perm.
 * The exchanges are the caller's (e.g. NCCL all-to-all-v); these calls only
 * plan them. A layer computed this way gives each rank exactly the output of
 * moe_forward on its own tokens.
 *
 * Send plan: send_rows[g] = rows of x_perm for rank g (the kept counts of
 * g's experts summed), send_offsets[g] = its first row (seg_offsets of g's
 * first expert); send_offsets[world] = seg_offsets[E]. The per-expert counts
 * the receiver needs are kept_counts itself: its slice
 * [g*E/world, (g+1)*E/world) goes to rank g.
 *   kept_counts [E], seg_offsets [E+1] (moe_permute's outputs, device)
 *   send_rows [world], send_offsets [world+1] (device, out)
 *   ws >= 256 bytes (control block; a negative count sets MOE_DEVERR_ROW_RANGE)
 * E in [1, 256] and a multiple of world, else MOE_ERR_INVALID. */
MOE_API moe_status_t moe_ep_send_plan(const int32_t* kept_counts, const int32_t* seg_offsets, int E,
                                      int world, int32_t* send_rows, int32_t* send_offsets,
                                      void* ws, size_t ws_bytes, moe_stream_t stream);

/* Receive plan. recv_counts [world][experts_per_rank] (device): from each
 * source rank, its kept counts for this rank's experts, as received. Rows
 * arrive source-major (source 0's rows in expert order, then source 1's ...).
 *   recv_rows [world], recv_offsets [world+1]: rows from each source and
 *     where they start in the received buffer
 *   local_seg [experts_per_rank+1]: expert-major segment offsets (for local
 *     expert e: source 0's rows, then source 1's ...), for moe_expert_ffn
 *   local_to_recv [rows]: received row of each expert-major row (gather the
 *     received rows into expert-major order with moe_gather, k = 1)
 *   recv_to_local [rows]: the inverse (gather the expert outputs back into
 *     received order before the return exchange)
 *   rows_cap: capacity of the two maps; a total above it sets
 *     MOE_DEVERR_ROW_RANGE in ws and writes no map
 * world * experts_per_rank <= 256. */
MOE_API moe_status_t moe_ep_recv_plan(const int32_t* recv_counts, int world, int experts_per_rank,
                                      int64_t rows_cap, int32_t* recv_rows, int32_t* recv_offsets,
                                      int32_t* local_seg, int32_t* local_to_recv,
                                      int32_t* recv_to_local, void* ws, size_t ws_bytes,
                                      moe_stream_t stream);

/* ----------------------------------------------------------------- gather
 * x_perm[r] = x[row_slot[r] / k] for r < seg_offsets[E] ("MegaBlocks",
 * section 4.3, binned_gather in compact form), moved row by row with bulk
 * (TMA) copies. rows_max bounds seg_offsets[E].
 *   ws  >= 256 bytes (control block) */
MOE_API moe_status_t moe_gather(const void* x, moe_dtype_t dtype, int T, int d, int k,
                        const int32_t* row_slot, const int32_t* seg_offsets, int E,
                        int64_t rows_max, void* x_perm, void* ws, size_t ws_bytes,
                        moe_stream_t stream);

/* ------------------------------------------------------------- expert FFN
 * Grouped expert MLP over the expert-contiguous rows ("MegaBlocks", section
 * 4.3: bmm -> activation -> bmm, weights [E, hs, ffn]). bf16 runs on the
 * tcgen05 tensor cores (fp32 accumulation in tensor memory, SwiGLU/GELU in
 * the up-projection epilogue, h rounded to bf16); f32 runs on CUDA cores.
 * Experts with no rows read no weights.
 *   x_perm  [rows_max, d]   h out [rows_max, F]   y_perm out [rows_max, d]
 *   w1 W_gate/W1 [E, d, F], w3 W_up [E, d, F] (SwiGLU) or NULL, w2 [E, F, d]
 *   seg_offsets [E+1] from moe_permute
 *   ws  >= 256 bytes (control block) */
MOE_API moe_status_t moe_expert_ffn(const void* x_perm, const void* w1, const void* w3, const void* w2,
                            moe_dtype_t dtype, moe_act_t act, int64_t rows_max, int d, int F,
                            int E, const int32_t* seg_offsets, void* h, void* y_perm, void* ws,
                            size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- combine
 * out[t] = sum_{j=0..k-1, slot_to_row[t*k+j] >= 0} topk_w[t,j] * y_perm[row]
 * in fp32, j ascending; zero row when every slot of t is dropped
 * ("ops-transformer", 原理 Step 4; "MegaBlocks", sections 4.3 and 5).
 * Each output row is written by one thread group that gathers its k rows:
 * no atomics, deterministic.
 *   ws  >= 256 bytes (control block) */
MOE_API moe_status_t moe_combine(const void* y_perm, const float* topk_w, const int32_t* slot_to_row,
                         moe_dtype_t dtype, int T, int d, int k, int64_t rows_max, void* out,
                         void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- forward
 * The whole layer on one stream with no host synchronisation: route ->
 * permute -> gather -> expert FFN (up, down) -> combine. With
 * MOE_LAYER_GATHER_IN_GEMM the gather is part of the up projection and the
 * "gather" events bracket only the zeroing of dropped tokens' rows (with
 * MOE_LAYER_COMBINE_IN_GEMM) or no work; with MOE_LAYER_COMBINE_IN_GEMM the
 * combine is part of the down projection and the "combine" events bracket
 * no work.
 *   x [T, d], out [T, d] (dtype); aux_loss out [1] fp32 device or NULL.
 *   events: NULL, or 7 cudaEvent_t recorded on `stream` before route and
 *   after route, permute, gather, up-projection, down-projection, combine.
 *   ws >= moe_forward_workspace_size(layer, T) bytes; it holds every
 *   intermediate (see moe_forward_views). */
MOE_API size_t moe_forward_workspace_size(const moe_layer_t* layer, int T);
MOE_API moe_status_t moe_forward(const moe_layer_t* layer, const void* x, int T, void* out,
                         float* aux_loss, void* ws, size_t ws_bytes, moe_stream_t stream,
                         const moe_event_t* events);

/* Where moe_forward(layer, ., T, ...) leaves its intermediates in `ws`. */
MOE_API moe_status_t moe_forward_views(const moe_layer_t* layer, int T, void* ws, size_t ws_bytes,
                               moe_views_t* views);

/* moe_forward with HOST input and output: copies x_host (T*d elements,
 * pinned host memory recommended) into the workspace, runs the forward,
 * copies the output into out_host and the aux loss into *aux_host. All
 * copies are asynchronous on `stream`; the host buffers must stay valid
 * until the stream reaches this point. ws >= moe_forward_host_workspace_size. */
MOE_API size_t moe_forward_host_workspace_size(const moe_layer_t* layer, int T);
MOE_API moe_status_t moe_forward_host(const moe_layer_t* layer, const void* x_host, int T, void* out_host,
                              float* aux_host, void* ws, size_t ws_bytes, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
