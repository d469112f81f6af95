/*
 * fgs_moe.h -- C ABI of the B200 (sm_100a) DeepSeekMoE layer forward.
 *
 * The layer (DeepSeekMoE, arXiv 2401.06066, Abstract; blog summary sections
 * "Fine-Grained Expert Segmentation (Section 3.1)" and "Shared Expert
 * Isolation (Section 3.2)"): mN fine-grained routed experts of which mK are
 * active per token, plus K_s shared experts that every token uses.  For a
 * token u_t (a row of x):
 *
 *   z_{t,i} = u_t . e_i (+ c_i)                       affinity logits
 *   s_{t,i} = softmax_i(z_t)  or  sigmoid(z_{t,i})    affinities
 *   Sel_t   = the mK experts with the largest s (softmax) or s + b (sigmoid),
 *             ordered by that key descending, ties to the lower expert index
 *   g_{t,k} = s of the k-th selected expert (softmax), or that s divided by
 *             the sum of the selected s (sigmoid)
 *   FFN(u)  = W_down (SiLU(W_gate u) * (W_up u))
 *   h_t     = u_t + sum_j FFN^shared_j(u_t) + sum_k g_{t,k} FFN_{Sel_t,k}(u_t)
 *
 * The sigmoid variant with a per-expert selection bias b is the
 * auxiliary-loss-free routing of the DeepSeek-V3 technical report (section 2,
 * "Auxiliary-Loss-Free Load Balancing"); no token is ever dropped (same
 * section).  The pages state the layer in prose; the formulas above are the
 * standard reading of it.
 *
 * Conventions for every call:
 *   - bf16 means IEEE bfloat16 stored as 2-byte little-endian values; all
 *     matrices are row-major.
 *   - Device pointers are borrowed for the duration of the enqueued work; the
 *     caller owns them and must keep them alive until the stream reaches the
 *     end of the call.  Every device pointer must be 16-byte aligned.
 *   - Calls are asynchronous on the given stream unless stated otherwise.
 *   - Host-detectable errors return before anything is enqueued.  Errors the
 *     kernels detect (a bounded wait that ran out) are recorded on the device
 *     and returned by moe_status_query().
 *   - One handle serves one stream at a time; calls on one handle that overlap
 *     on the GPU race on its workspace.
 */
#ifndef FGS_MOE_H
#define FGS_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, K outside [1, min(max_k, mN)], bad enum, aliasing */
  MOE_ERR_SHAPE = 2,       /* T < 0, T > max_tokens, or a size outside the supported range */
  MOE_ERR_ALIGNMENT = 3,   /* d, I or I_s not a multiple of 16, or a pointer not 16-byte aligned */
  MOE_ERR_UNSUPPORTED = 4, /* mN > 256, max_k > 8, or a device that is not sm_100 */
  MOE_ERR_NOMEM = 5,       /* workspace allocation failed */
  MOE_ERR_CUDA = 6,        /* a CUDA runtime or driver call failed */
  MOE_ERR_TIMEOUT = 7      /* a device-side wait ran out; the kernel stopped early */
} moe_status;

typedef enum moe_gate_kind {
  MOE_GATE_SOFTMAX = 0,        /* s = softmax over all mN experts; gates not renormalised */
  MOE_GATE_SIGMOID_BIASED = 1  /* s = sigmoid; select on s + b; gates renormalised over Sel */
} moe_gate_kind;

/* moe_config.flags: leave terms out of h_t so each can be checked alone. */
#define MOE_FLAG_NO_RESIDUAL 0x1u /* drop u_t */
#define MOE_FLAG_NO_SHARED 0x2u   /* drop the shared experts */
#define MOE_FLAG_NO_ROUTED 0x4u   /* drop the routed experts (routing still runs) */
/* The handle also holds the workspace of moe_forward_fp8 (FP8 copies of the
 * permuted activations and of H, with their scales).  Requires d_model, d_ff
 * and d_ff_shared to be multiples of 128 (else MOE_ERR_ALIGNMENT) and at most
 * 8192 (else MOE_ERR_SHAPE). */
#define MOE_FLAG_FP8 0x8u
/* Test only: the first grouped-GEMM CTA waits on a barrier that nothing
 * arrives on, with a 20 ms limit; the call then reports MOE_ERR_TIMEOUT. */
#define MOE_FLAG_DEBUG_WAIT_TIMEOUT 0x100u

/* Sizes fixed for the life of a handle.  Limits: 16 <= d_model, d_ff,
 * d_ff_shared (each a multiple of 16); 1 <= n_routed <= 256;
 * 1 <= max_k <= min(8, n_routed); 0 <= n_shared; 1 <= max_tokens <= 2^20. */
typedef struct moe_config {
  int32_t d_model;     /* d: hidden size */
  int32_t n_routed;    /* mN: routed experts */
  int32_t d_ff;        /* I: intermediate size of one routed expert */
  int32_t n_shared;    /* K_s: shared experts (0 allowed) */
  int32_t d_ff_shared; /* I_s: intermediate size of one shared expert */
  int32_t max_tokens;  /* largest T passed to moe_forward */
  int32_t max_k;       /* largest mK passed to moe_forward */
  int32_t gate;        /* moe_gate_kind */
  uint32_t flags;      /* MOE_FLAG_* */
  /* Node-limited routing (DeepSeek-V3 technical report summary, section 2:
   * each token is sent to at most M nodes, chosen among those holding its
   * highest-affinity experts).  route_nodes = the number of nodes the mN
   * experts sit on, in equal contiguous ranges (expert i on node
   * i / (mN / route_nodes)); route_max_nodes = M.  A node ranks by the largest
   * selection key among its experts (ties to the lower node); the token's K
   * experts are the top K of the chosen nodes' experts.  Gates as without the
   * limit (softmax over all mN experts, or the selected sigmoids renormalised).
   * Both 0: no limit.  Otherwise 1 <= route_nodes <= 16 dividing mN,
   * 1 <= route_max_nodes <= route_nodes, max_k <= route_max_nodes * mN /
   * route_nodes (else MOE_ERR_INVALID_ARG). */
  int32_t route_nodes;
  int32_t route_max_nodes;
  /* Expert parallelism (see moe_ep_route below).  ep_ranks = G ranks that
   * split the mN routed experts in equal contiguous ranges (expert i on rank
   * i / (mN / G)); this handle is rank ep_rank and holds mN / G of them.
   * 0 or 1: a single-GPU handle (moe_forward).  Otherwise 2 <= G <= 32
   * dividing mN and 0 <= ep_rank < G (else MOE_ERR_INVALID_ARG); with
   * MOE_FLAG_FP8 the dispatch sends FP8 rows (moe_ep_experts_fp8). */
  int32_t ep_ranks;
  int32_t ep_rank;
} moe_config;

/* Router.  weight: bf16 [mN, d], row i is e_i.
 * logit_bias: float32 [mN] or NULL; softmax only: c_i added to z before
 *   the softmax (moves both selection and gate values).
 * select_bias: float32 [mN] or NULL; sigmoid only: b_i added to s for the
 *   selection alone (the gate values use s). */
typedef struct moe_router {
  const void* weight;
  const float* logit_bias;
  const float* select_bias;
} moe_router;

/* Routed experts, stacked: w_gate, w_up bf16 [mN, I, d]; w_down bf16 [mN, d, I]
 * (each expert's matrices in the [out, in] layout of a linear layer). */
typedef struct moe_experts {
  const void* w_gate;
  const void* w_up;
  const void* w_down;
} moe_experts;

/* Shared experts, stacked: w_gate, w_up bf16 [K_s, I_s, d]; w_down bf16 [K_s, d, I_s]. */
typedef struct moe_shared {
  const void* w_gate;
  const void* w_up;
  const void* w_down;
} moe_shared;

/* Expert weights in fine-grained FP8, as moe_quantize_fp8_blocks writes them:
 * E4M3 codes in the layout of the bf16 matrices (w_gate, w_up uint8 [n, I, d];
 * w_down uint8 [n, d, I]) and one UE8M0 scale byte per 128 x 128 block
 * (s_gate, s_up uint8 [n, I/128, d/128]; s_down uint8 [n, d/128, I/128]).
 * n = mN and I = d_ff for the routed experts; n = K_s and I = d_ff_shared for
 * the shared ones. */
typedef struct moe_experts_fp8 {
  const uint8_t* w_gate;
  const uint8_t* w_up;
  const uint8_t* w_down;
  const uint8_t* s_gate;
  const uint8_t* s_up;
  const uint8_t* s_down;
} moe_experts_fp8;

typedef struct moe_ctx* moe_handle;

/* Device bytes the handle allocates for cfg (host only; no CUDA call). */
moe_status moe_workspace_bytes(const moe_config* cfg, uint64_t* bytes);

/* Validate cfg and allocate the workspace on `device`.  The caller's current
 * device is restored before returning.
 * Returns MOE_ERR_UNSUPPORTED if the device is not sm_100. */
moe_status moe_create(const moe_config* cfg, int device, moe_handle* out);

/* Enqueue one layer forward on `stream` (a cudaStream_t; NULL = the legacy
 * default stream).  x: bf16 [T, d] device; out: bf16 [T, d] device, must not
 * overlap x or any weight.  shared must be NULL iff cfg.n_shared == 0.
 * T == 0 enqueues nothing and returns MOE_OK.  Asynchronous. */
moe_status moe_forward(moe_handle h, const void* x, int64_t T, const moe_router* router,
                       const moe_experts* experts, const moe_shared* shared, int32_t K,
                       void* out, void* stream);

/* The same forward for callers whose activations live in host memory:
 * x_host: bf16 [T, d] host; out_host: bf16 [T, d] host (pinned memory makes
 * the copies asynchronous to other host work and lets them overlap the
 * compute).  Copies x to the device, runs moe_forward on `stream`, copies the
 * result back and returns when out_host holds it.  Batches of 4096 tokens or
 * more run as up to 5 chunks of whole tokens (the first and last T/16) whose
 * copies in and out overlap the other chunks' compute (on two copy streams
 * the handle owns); the
 * output is bit-identical to one moe_forward over the whole batch, and
 * moe_get_routing afterwards returns the last chunk's routing.  The weights
 * stay device pointers. */
moe_status moe_forward_host(moe_handle h, const void* x_host, int64_t T, const moe_router* router,
                            const moe_experts* experts, const moe_shared* shared, int32_t K,
                            void* out_host, void* stream);

/* The layer forward with FP8 expert GEMMs (DeepSeek-V3 technical report,
 * section 3.3 "FP8 Training" and Appendix B.2 "Discussion About Block-Wise
 * Quantization"): routing as moe_forward (bf16 affinities, fp32 softmax or
 * sigmoid and top-K); each token row x_t is quantized once to E4M3 with one
 * power-of-two scale per 1 x 128 group (e = the smallest integer with
 * max|x| <= 448 * 2^e, codes rounded to nearest even); the gate/up GEMM runs
 * on those codes and the 128 x 128 block-quantized W_gate and W_up with
 * block-scaled tensor-core MMAs and fp32 accumulation; H = SiLU(gate) * up is
 * quantized 1 x 128 the same way in the GEMM's epilogue; the down GEMM runs on
 * H's codes and W_down's, scales by g and forms h_t = u_t + shared + sum_k
 * g FFN in k order (fp32, rounded once to bf16).  The residual u_t is the
 * unquantized input.  x, out: bf16 [T, d] device; experts and shared (NULL iff
 * K_s == 0): device FP8 weights as above.  The handle must have been created
 * with MOE_FLAG_FP8 (else MOE_ERR_UNSUPPORTED); the other arguments and errors
 * as moe_forward.  Asynchronous; moe_get_routing, moe_update_bias and
 * moe_status_query see it as they see moe_forward. */
moe_status moe_forward_fp8(moe_handle h, const void* x, int64_t T, const moe_router* router,
                           const moe_experts_fp8* experts, const moe_experts_fp8* shared, int32_t K,
                           void* out, void* stream);

/* Stream-ordered copies of the last forward's routing into device buffers
 * (any may be NULL): idx int32 [T, K] and gate float32 [T, K] (Sel_t and
 * g_t in selection order); counts int32 [mN] tokens per expert; offsets
 * int32 [mN + 1] exclusive prefix sum of counts; src int32 [T*K] token ids
 * grouped by expert, ascending within an expert. */
moe_status moe_get_routing(moe_handle h, int32_t* idx, float* gate, int32_t* counts,
                           int32_t* offsets, int32_t* src, void* stream);

/* Auxiliary-loss-free load balancing: one update of the per-expert selection
 * biases from the last forward's per-expert loads (DeepSeek-V3 technical
 * report summary, section 2 "Auxiliary-Loss-Free Load Balancing": after each
 * step a bias moves according to whether its expert was overloaded or
 * underloaded).  With load_i the (token, slot) pairs routed to expert i by the
 * last moe_forward on this handle and mean = sum(load) / mN (after a
 * moe_forward_host that ran in chunks, the loads are its last chunk's, as for
 * moe_get_routing; to balance on a whole batch, forward it from device
 * buffers with moe_forward):
 *   bias[i] += gamma * sign(mean - load_i)
 * (an overloaded expert's bias drops, an underloaded one's rises, an expert at
 * exactly the mean keeps its bias; the comparison is exact, on integers).
 * bias: float32 [mN] device, 4-byte aligned, updated in place -- normally the
 * moe_router select_bias of a MOE_GATE_SIGMOID_BIASED layer; gamma: the
 * update speed, finite.  Stream-ordered on `stream` after the forward whose
 * loads it reads; asynchronous.  MOE_ERR_INVALID_ARG for a NULL handle or
 * bias, a misaligned bias, a non-finite gamma, or no forward yet. */
moe_status moe_update_bias(moe_handle h, float* bias, float gamma, void* stream);

/* Synchronize the stream of the last forward and report (then clear) any
 * error the kernels recorded: MOE_ERR_TIMEOUT if a device-side wait ran out. */
moe_status moe_status_query(moe_handle h);

/* Free the workspace and the handle (synchronizes first).  NULL is a no-op. */
moe_status moe_destroy(moe_handle h);

/* Per-kernel timing.  moe_set_timing(h, kernel_mask): bit k of kernel_mask
 * (k a moe_kernel_id) makes moe_forward record a CUDA event pair around each
 * launch of kernel k, on its stream; 0 turns timing off; MOE_TIMING_ALL times
 * every kernel.  Event records add a few microseconds per launch, so time only
 * the kernels you need in a timed loop.  moe_kernel_times synchronizes those
 * events, writes each kernel's summed duration in milliseconds
 * (total_ms[MOE_KERNEL_COUNT]) and launch count (launches[MOE_KERNEL_COUNT];
 * either array may be NULL) and clears them. */
typedef enum moe_kernel_id {
  MOE_KERNEL_ROUTER = 0,   /* affinities, top-K, histogram, scan */
  MOE_KERNEL_PERMUTE = 1,  /* expert-contiguous rows of x */
  MOE_KERNEL_GATE_UP = 2,  /* SwiGLU(x W_gate^T, x W_up^T): shared experts on x, routed ones grouped */
  MOE_KERNEL_DOWN = 3,     /* shared experts: Hs W_down^T; routed experts: g * (H W_down^T) */
  MOE_KERNEL_COMBINE = 4,  /* h = x + shared + sum_k g * routed, k ascending */
  MOE_KERNEL_COUNT = 5
} moe_kernel_id;
#define MOE_TIMING_ALL ((1u << MOE_KERNEL_COUNT) - 1u)
moe_status moe_set_timing(moe_handle h, uint32_t kernel_mask);
moe_status moe_kernel_times(moe_handle h, float* total_ms, int32_t* launches);

/* Routing without any device allocation (the pages have no counterpart: this
 * serves callers, not the method).  For callers that cannot call cudaMalloc --
 * a serving runtime that plans all device memory before it starts, a framework
 * whose allocator must own every allocation, or a latency-critical loop that
 * cannot take cudaMalloc's implicit device synchronisation -- this runs the
 * router kernel of moe_forward (affinities, top-K, per-expert histogram and
 * offsets) with its scratch in a fixed 528 KB device array that the library
 * holds on every GPU that loads it, until the process exits.
 *
 * Runs on the calling thread's current device, on `stream`.  x: bf16 [T, d]
 * device; router as for moe_forward; gate: moe_gate_kind; outputs (device,
 * caller-allocated): idx int32 [T, K], gate_out float32 [T, K], counts int32
 * [mN], offsets int32 [mN + 1].  These are the values moe_get_routing returns
 * after moe_forward on the same inputs: idx, counts and offsets bit for bit
 * (batches of more than 256 tokens run the very same kernel; for smaller ones
 * moe_forward computes the logits on the CUDA cores in another summation
 * order, so a token whose K-th and (K+1)-th keys are closer than float32
 * rounding may pick differently), gates within 1e-5.
 * err: required device word (4-byte aligned) into which the kernel ORs its
 * error bits if a device-side wait runs out (the outputs are then not valid);
 * the caller clears it and reads it after the stream has finished.
 * Limits: T <= 65536 (else MOE_ERR_SHAPE: the static scratch is full),
 * mN <= 256, K <= 8, d a multiple of 16, 16-byte aligned pointers (x, router
 * and its biases, idx, gate_out, counts, offsets).  A null input or output
 * pointer, err included, -> MOE_ERR_INVALID_ARG; err not 4-byte aligned ->
 * MOE_ERR_ALIGNMENT.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * The first call on a device looks up the scratch array's device address and
 * sets the kernels' shared-memory limits; make that first call before any
 * stream capture.  Every call shares the one array and finds the previous
 * call's contents there (the call clears what must start at zero itself), so
 * calls that overlap on the GPU -- on different streams or different threads
 * of one device -- race and must be serialised by the caller. */
moe_status moe_route_noalloc(const void* x, int64_t T, int32_t d_model, const moe_router* router,
                             int32_t n_routed, int32_t gate, int32_t K, int32_t* idx, float* gate_out,
                             int32_t* counts, int32_t* offsets, uint32_t* err, void* stream);

/* Fine-grained FP8 quantization of GEMM operands (the first step of an FP8
 * expert path).  DeepSeek-V3 technical report, section 3.3 "FP8 Training":
 * GEMM inputs in FP8 with one scale per small group of values (fine-grained
 * scaling), activation scales powers of two; Appendix B.2 "Discussion About
 * Block-Wise Quantization": activations grouped 1 x 128 along the channels in
 * the forward pass, weights in 128 x 128 blocks.
 *
 * Per group, e is the smallest integer with max|x| <= 448 * 2^e, clamped to
 * [-127, 127] (an all-zero group takes -127); each element becomes the E4M3
 * code ("fn" variant: largest finite 448, no infinities) of x * 2^-e, rounded
 * to nearest with ties to the even code, keeping the sign (a negative value
 * that rounds to zero is 0x80).  The scale is stored as the byte e + 127
 * (UE8M0: the value it stands for is 2^(byte - 127)).  Inputs must be finite.
 *
 * Both run on the calling thread's current device, on `stream`, asynchronously;
 * all pointers are caller-owned device memory.  Errors, returned before any
 * launch: a null pointer -> MOE_ERR_INVALID_ARG; a negative size, cols <= 0, or
 * a grid dimension past CUDA's limits -> MOE_ERR_SHAPE; cols not a multiple of
 * 16, or x / w / q not 16-byte aligned -> MOE_ERR_ALIGNMENT; a failed launch ->
 * MOE_ERR_CUDA.  An empty input launches nothing and returns MOE_OK.
 *
 * moe_quantize_fp8_rows: x bf16 [rows, cols] row-major (activations, one token
 *   per row) -> q uint8 [rows, cols], scale uint8 [rows, ceil(cols / 128)];
 *   group g of a row is columns [128 g, 128 g + 128) (the last may be shorter).
 * moe_quantize_fp8_blocks: w bf16 [batch, rows, cols] (batch weight matrices,
 *   [out, in] each) -> q uint8 [batch, rows, cols], scale uint8
 *   [batch, ceil(rows / 128), ceil(cols / 128)]; batch <= 65535. */
moe_status moe_quantize_fp8_rows(const void* x, int64_t rows, int32_t cols, uint8_t* q, uint8_t* scale,
                                 void* stream);
moe_status moe_quantize_fp8_blocks(const void* w, int32_t batch, int32_t rows, int32_t cols, uint8_t* q,
                                   uint8_t* scale, void* stream);

/* The backward pass: gradients for the input, the router and the expert
 * weights (DeepSeek-V3 technical
 * report summary, section 3.2.1 "DualPipe and Computation-Communication
 * Overlap": a training step runs the MoE layer's backward for input and its
 * backward for weights as separate pieces; the pages print no formula, so
 * these are the chain rule through the forward above, with the top-K choice
 * held fixed: the gradient reaches the router through the chosen experts'
 * gate values only, and the sigmoid variant's selection bias gets none).
 *
 * For the last moe_forward on this handle -- called with the same x, T,
 * router, experts, shared and K, with no other forward (moe_forward_fp8,
 * moe_forward_host) on the handle since: its routing and expert-ordered rows
 * are read from the workspace -- and the gradient dh = dL/dh of its output:
 *   dx        bf16 [T, d] out: dL/du, the residual's dh + the shared experts'
 *             and the routed experts' input gradients + the router's (dz E)
 *   d_router  float32 [mN, d] out or NULL: dL/dE = dz^T u
 *   d_logit_bias float32 [mN] out or NULL: dL/dc = sum_t dz_t (only with a
 *             logit bias: else MOE_ERR_INVALID_ARG)
 *   dgate     float32 [T, K] out or NULL: dL/dg_{t,k} = dh_t . FFN_{Sel_t,k}(u_t)
 *   wgrad     NULL, or the expert weights' gradients (every pointer set; the
 *             shared ones when K_s > 0), float32 in the weights' layouts:
 *             dW_down,e = sum over e's rows of (g dh) m^T, dW_gate,e = sum of
 *             da u^T, dW_up,e = sum of db u^T (m = SiLU(a) b, da, db as below);
 *             the shared experts' the same with g = 1 over every token
 * where dz is dL/dz of the affinity logits (softmax: dz = s (ds - s . ds),
 * ds_i the dgate of the slot that chose expert i, 0 for the others; sigmoid:
 * ds_k = (dgate_k - g . dgate) / sum of the chosen s, dz = ds s (1 - s) on the
 * chosen experts, 0 elsewhere); for a routed row, da = g dm b SiLU'(a) and
 * db = g dm SiLU(a) with dm = W_down^T dh.  The debug flags leave the same
 * terms out as in the forward (a left-out part's weight gradients are zero).
 *
 * Asynchronous on `stream`, which must be the forward's stream or ordered after
 * it.  The first call allocates the backward's buffers
 * (a K-major copy of the expert weights, rewritten by every call, and
 * row-major activations of the forward's row count).  Errors: the last forward was not a
 * moe_forward with this T and K, or another argument error of moe_forward
 * -> MOE_ERR_INVALID_ARG / SHAPE / ALIGNMENT; dx overlapping x or dh ->
 * MOE_ERR_INVALID_ARG; an expert-parallel handle -> MOE_ERR_UNSUPPORTED; no
 * memory for the buffers -> MOE_ERR_NOMEM.  Overwrites the forward's
 * intermediate rows (H, Y, Hs, Ys) in the workspace. */
typedef struct moe_weight_grads {
  float* w_gate;  /* [mN, I, d] */
  float* w_up;    /* [mN, I, d] */
  float* w_down;  /* [mN, d, I] */
  float* ws_gate; /* [K_s, I_s, d] */
  float* ws_up;   /* [K_s, I_s, d] */
  float* ws_down; /* [K_s, d, I_s] */
} moe_weight_grads;

moe_status moe_backward(moe_handle h, const void* x, int64_t T, const moe_router* router, const moe_experts* experts,
                        const moe_shared* shared, int32_t K, const void* dh, void* dx, float* d_router,
                        float* d_logit_bias, float* dgate, const moe_weight_grads* wgrad, void* stream);

/* Expert parallelism (DeepSeek-V3 technical report summary, section 3.1
 * "Compute Clusters": the routed experts of a layer spread over many GPUs;
 * section 3.2.1 "DualPipe and Computation-Communication Overlap": an
 * all-to-all dispatch sends each token to the GPUs of its experts and an
 * all-to-all combine brings the results back; section 2: node-limited routing
 * bounds how many of them a token reaches -- moe_config.route_nodes /
 * route_max_nodes, with route_nodes = G to limit the ranks).
 *
 * G handles, one per rank (usually one per GPU of one NVLink domain), each
 * created with ep_ranks = G and its own ep_rank, all with the same other
 * fields.  Each rank passes its own tokens; the layer's result for a token is
 * the single-GPU layer's.  A forward is four calls, each asynchronous on
 * `stream`, separated on every rank by a barrier across the ranks that is
 * ordered on the same stream (for example a one-element all-reduce):
 *
 *   moe_ep_route     router and top-K of this rank's T tokens (T may be 0);
 *                    the per-expert counts that the other ranks read
 *   -- barrier --
 *   moe_ep_dispatch  from every rank's counts: where each row goes; stores
 *                    each (token, slot) row of x and its gate into the row
 *                    buffer of the rank that holds the slot's expert
 *   -- barrier --
 *   moe_ep_experts   the grouped GEMMs of this rank's experts on the rows it
 *                    received (all ranks' rows of expert e in ascending rank,
 *                    then ascending token), and of the shared experts on its
 *                    own T tokens
 *   -- barrier --
 *   moe_ep_combine   out = x + shared + the K g-scaled rows, read from the
 *                    ranks that computed them, summed in ascending k
 *
 * Before the next moe_ep_route every rank must have passed the third barrier
 * (the calls above on one stream, in this order, ensure it).  x stays
 * borrowed from moe_ep_route to moe_ep_combine.  The row buffers hold
 * G * max_tokens * max_k rows (plus padding), so every rank may send all of
 * its rows to one rank.  Batches of any size run the grouped GEMMs (the decode
 * FFN of moe_forward is not used).
 *
 * The ranks address each other's workspaces directly: moe_ep_set_peers takes
 * every rank's workspace pointer as this device addresses it (handles on one
 * GPU, or GPUs of one process with peer access enabled); moe_ep_ipc_handle /
 * moe_ep_open_peers exchange and open CUDA IPC handles between processes.
 * The calls below return MOE_ERR_INVALID_ARG on a single-GPU handle, before
 * the peers are set, or out of order (dispatch before route, ...); other
 * errors as for moe_forward.  moe_forward and moe_forward_fp8 return
 * MOE_ERR_UNSUPPORTED on an expert-parallel handle. */

/* This handle's workspace (device pointer), for moe_ep_set_peers of the other
 * handles when all are in one process. */
moe_status moe_ep_workspace(moe_handle h, void** workspace);
/* workspaces[r], r < G: rank r's workspace as this handle's device addresses
 * it; workspaces[ep_rank] must be this handle's own.  The pointers stay
 * borrowed for the life of the handle. */
moe_status moe_ep_set_peers(moe_handle h, void* const* workspaces);
/* The CUDA IPC handle (64 bytes, written to `handle`) of this handle's
 * workspace, for the other processes' moe_ep_open_peers. */
moe_status moe_ep_ipc_handle(moe_handle h, void* handle);
/* handles: G x 64 bytes, rank r's IPC handle at byte 64 r (this rank's own
 * entry is ignored).  Opens the others' workspaces (closed by moe_destroy)
 * and sets them as the peers. */
moe_status moe_ep_open_peers(moe_handle h, const void* handles);

/* router as for moe_forward; x bf16 [T, d], 0 <= T <= max_tokens. */
moe_status moe_ep_route(moe_handle h, const void* x, int64_t T, const moe_router* router, int32_t K, void* stream);
moe_status moe_ep_dispatch(moe_handle h, void* stream);
/* experts: this rank's mN / G routed experts, stacked as for moe_forward
 * (w_gate, w_up bf16 [mN / G, I, d]; w_down bf16 [mN / G, d, I]); local
 * expert l is global expert ep_rank * mN / G + l.  shared as for moe_forward
 * (every rank holds all K_s shared experts). */
moe_status moe_ep_experts(moe_handle h, const moe_experts* experts, const moe_shared* shared, void* stream);
/* The FP8 layer's step 3 (handles created with MOE_FLAG_FP8, whose dispatch
 * quantized each row once, 1 x 128 groups as moe_forward_fp8 does, and sent
 * its E4M3 codes and scale bytes instead of the bf16 row: the FP8 dispatch of
 * the DeepSeek-V3 report, section 3.3): this rank's mN / G experts and the
 * shared experts in the moe_experts_fp8 format of moe_forward_fp8.
 * moe_ep_experts returns MOE_ERR_UNSUPPORTED on such a handle, and this call
 * on a bf16 one. */
moe_status moe_ep_experts_fp8(moe_handle h, const moe_experts_fp8* experts, const moe_experts_fp8* shared,
                              void* stream);
/* out: bf16 [T, d] of the T tokens of the last moe_ep_route. */
moe_status moe_ep_combine(moe_handle h, void* out, void* stream);

/* The dispatch plan on the host, from every rank's counts (counts_all int32
 * [G, mN], row r = rank r's rows per global expert): base int32 [mN] = the
 * first row, in the buffer of expert e's rank, of rank `rank`'s rows of e; and
 * rank `rank`'s own tables over its mN / G experts, each int32 [mN / G + 1]:
 * counts_local (rows received per expert; the last entry 0), row_start
 * (padded to multiples of 256 rows), mtile_start (prefix sum of
 * ceil(rows / 256)), mtile128_start (prefix sum of ceil(rows / 128)); the
 * last entry of each prefix is the total.  moe_ep_dispatch computes the same
 * on the device.  Plain host arithmetic: needs no GPU.  Errors: a null
 * pointer, G outside [2, 32], mN outside [1, 256] or not a multiple of G,
 * rank outside [0, G), a negative count -> MOE_ERR_INVALID_ARG. */
moe_status moe_ep_plan(const int32_t* counts_all, int32_t G, int32_t n_routed, int32_t rank, int32_t* base,
                       int32_t* counts_local, int32_t* row_start, int32_t* mtile_start, int32_t* mtile128_start);

/* A static string naming the status. */
const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* FGS_MOE_H */
