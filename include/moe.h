/*
 * moe.h -- C ABI of the B200 (sm_100a) top-k mixture-of-experts FFN layer.
 *
 * The layer is the MoE FFN of DiffusionGemma 26B-A4B applied to a whole
 * denoising canvas at once:
 *   - 128 experts, 8 active per token (Quant-Tuner pull request "Add
 *     DiffusionGemma (Gemma-4 MoE block-diffusion) support", Summary; Hugging
 *     Face card "kingjones777/DiffusionGemma-26B-A4B-it-ROCmFP4-GGUF", header);
 *   - the router reads the raw residual through its own (1+gamma) RMSNorm,
 *     and a fused 3-D gate_up projection feeds the experts (Quant-Tuner pull
 *     request, "Answers to the motivating questions");
 *   - per expert gate/up 2816->704, down 704->2816, act GELUTanh; optional
 *     symmetric int4 weights in groups of 128 (auto-round pull request "Add
 *     quantization support for DiffusionGemma", transformers backend test
 *     log), or 8-bit floating-point weights (the ROCmFP4-GGUF card's FP8
 *     builds; E4M3 with one fp32 scale per weight row here), or 4-bit
 *     floating-point weights (the card's FP4 builds; MX E2M1 with an E4M3
 *     scale per 16 weights and an fp32 scale per row here);
 *   - the canvas of 256 tokens is denoised in parallel, so each step is a set
 *     of large batched expert matmuls (the ROCmFP4-GGUF card, section "The
 *     4-bit is NOT the fastest here").
 *
 * For each token t (x_t bf16 [d]):
 *   u   = x_t / sqrt(mean(x_t^2) + eps) * (1 + gamma)
 *   xe  = x_t, or bf16(x_t / sqrt(mean(x_t^2) + eps) * (1 + expert_gamma))
 *   z_e = router_w[e] . u (+ router_bias[e])            fp32
 *   S   = the k largest z_e, ties to the lower index; j order = (z desc, e asc)
 *   w_j = softmax(z)[S_j] / sum_j' softmax(z)[S_j']
 *   h   = gelu_tanh(Wgu[S_j][0:f] xe) * (Wgu[S_j][f:2f] xe)     (bf16 h)
 *   y_j = Wd[S_j] h          (bf16 y by default; fp32 with MOE_OPT_Y_BF16 = 0)
 *   out_t = residual_t + sum_j w_j y_j  (j order, fp32, one rounding to bf16)
 *
 * Conventions for every entry point:
 *   - All tensor arguments are DEVICE pointers on the plan's device, owned by
 *     the caller, contiguous row-major, 16-byte aligned (moe_forward_host is
 *     the one exception: its x and out are HOST pointers).
 *   - bf16 / fp16 data are passed as raw 16-bit words (void*).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous on that stream except where stated.
 *     A plan is used by one stream at a time.
 *   - On any invalid argument nothing is launched and an error is returned.
 *     Launch failures return MOE_ERR_CUDA.
 *   - Token counts: 0 <= T <= MOE_MAX_T and T * k <= MOE_MAX_ASSIGNMENTS;
 *     a larger T returns MOE_ERR_UNSUPPORTED before anything is launched.  Faults the kernels detect
 *     themselves (a bounded wait that ran out, an index out of range) are
 *     recorded in a device status word read by moe_plan_sync_status.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_plan_s* moe_plan_t;

/* Largest token count of one call, and largest T * k (token-expert
 * assignments) of one call. */
#define MOE_MAX_T 65536
#define MOE_MAX_ASSIGNMENTS (1 << 19)

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or aliasing      */
  MOE_ERR_UNSUPPORTED = 2,  /* shape or dtype outside what the kernels cover */
  MOE_ERR_ALLOC = 3,        /* workspace allocation failed                   */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed          */
  MOE_ERR_TIMEOUT = 5,      /* a device-side bounded wait ran out            */
  MOE_ERR_DEVICE_CHECK = 6  /* a kernel saw an out-of-range routing index    */
} moe_status_t;

typedef enum {
  MOE_W_BF16 = 0,      /* w_gate_up bf16 [E,2f,d]; w_down bf16 [E,d,f]           */
  MOE_W_INT4_G128 = 1, /* w_gate_up u8 [E,2f,d/2]; w_down u8 [E,d,f/2]; element i
                          of a row in byte i/2, low nibble for even i, 4-bit two's
                          complement; value = code * scale[row][i/128] (fp16)  */
  MOE_W_FP8_E4M3 = 2,  /* w_gate_up u8 [E,2f,d]; w_down u8 [E,d,f]; element i of a
                          row is byte i, an OFP8 E4M3 value (OCP 8-bit Floating
                          Point Specification; the NaN codes 0x7F / 0xFF must not
                          occur); value = e4m3 * scale[row] with one fp32 scale
                          per weight row.  The FP4 / FP8 weight builds are on the
                          Hugging Face card "kingjones777/DiffusionGemma-26B-A4B-
                          it-ROCmFP4-GGUF"; the pages do not fix the encoding.
                          Activations (the experts' input rows and h) are carried
                          as fp16 on this path: |x| (after the optional expert
                          norm) and |h| must stay below 65504.                 */
  MOE_W_FP4_E2M1 = 3   /* w_gate_up u8 [E,2f,d/2]; w_down u8 [E,d,f/2]; element i
                          of a row in byte i/2, low nibble for even i, an MX E2M1
                          value (OCP Microscaling Formats specification: 0, 0.5,
                          1, 1.5, 2, 3, 4, 6 and their negatives); value =
                          e2m1 * block[i/16][row] * s[row].  The scales of each
                          expert form one record {fp32 s[R]; u8 block[R*C/16]},
                          R the tensor's rows, C its columns, block[j][r] the
                          OFP8 E4M3 scale (no NaN) of elements 16j..16j+15 of
                          row r; records back to back, R*(4 + C/16) bytes each.
                          Activations are fp16 as for MOE_W_FP8_E4M3.          */
} moe_wdtype_t;

/* Options for moe_plan_set_option. */
enum {
  MOE_OPT_EPS = 0,        /* RMSNorm epsilon (default 1e-6)                        */
  MOE_OPT_TIMEOUT_MS = 1, /* bound of every device-side wait, ms (default 1000)    */
  MOE_OPT_PROFILE = 2,    /* 1: moe_forward records CUDA events around each kernel */
  MOE_OPT_TEST_STALL = 3, /* test hook: 1 makes the expert kernel wait on a flag
                             nothing sets, so the bounded wait runs out and the
                             call reports MOE_ERR_TIMEOUT (no trap, no hang)     */
  MOE_OPT_PDL = 4,        /* 1 (default): launch each kernel with programmatic
                             dependent launch so it overlaps the previous one's
                             tail; 0: plain stream-ordered launches              */
  MOE_OPT_ROUTER = 6,     /* router path: 0 (default) automatic -- tensor cores
                             when E <= 128, FFMA otherwise; 1 FFMA; 2 tensor
                             cores (E <= 128)                                    */
  MOE_OPT_L2_PREFETCH_MB = 5, /* MiB of the gate_up weight (from its start) the
                             router pulls into L2 while routing runs, so the
                             expert kernel's first wave finds it there
                             (default 0 = off)                                   */
  MOE_OPT_Y_BF16 = 7,     /* 1 (default): the per-slot expert outputs y are kept
                             in bf16 (one more rounding before the fp32
                             combine, half the bytes); 0: fp32                   */
  MOE_OPT_DEBUG = 8,      /* 1: the workspace is laid out with a 256-byte guard
                             block after every region, filled with a fixed
                             pattern when the workspace is (re)allocated;
                             moe_plan_sync_status then also checks every guard
                             and returns MOE_ERR_DEVICE_CHECK if a kernel wrote
                             past its region.  Takes effect at the next
                             workspace (re)allocation (set it before the first
                             call or moe_plan_reserve).  Default 0.             */
  MOE_OPT_CHUNK_TOKENS = 9 /* bf16 weights: tokens per work chunk of an expert,
                             128 or 256; 0 (default) picks 128 for a call of
                             at most 256 tokens and 256 above.  An expert
                             with more tokens than a chunk is split into
                             chunks, each streaming the expert's weights;
                             chunks of at most 128 tokens are multiplied by
                             two UMMA issuers that split K, so the fp32
                             summation order, and the result's last bits,
                             depend on the chunking: give two plans whose
                             results must agree byte for byte (expert-parallel
                             owners and moe_forward) the same explicit value.
                             The int4, fp8 and fp4 kernels always use 128.   */
};

/* Kernels of one moe_forward, for moe_plan_profile. */
enum {
  MOE_K_ROUTER = 0,   /* norm + logits + softmax + top-k                         */
  MOE_K_PLAN = 1,     /* histogram + scan + stable permutation, then the gather
                         of x rows in slot order                                */
  MOE_K_EXPERT = 2,   /* grouped gate_up(+GELU*up) and down GEMMs               */
  MOE_K_COMBINE = 3,  /* weighted k-order sum (+ residual)                       */
  MOE_K_COUNT = 4
};

/* Create a plan for E experts, top-k, hidden d, per-expert intermediate f.
 * Limits: 1 <= E <= 256; 1 <= k <= min(E, 32); d % 128 == 0, 128 <= d <= 4096;
 * f % 64 == 0, 64 <= f <= 4096 (every DiffusionGemma shape and the test
 * shapes fit; d % 128 keeps an int4 scale group inside one row of x).  Binds the plan to the current CUDA device.
 * Returns MOE_ERR_UNSUPPORTED outside the limits, MOE_ERR_INVALID_ARG on a
 * NULL `out`.  Allocates nothing on the device until the first call. */
moe_status_t moe_plan_create(int E, int k, int d, int f, moe_wdtype_t wdtype, moe_plan_t* out);

/* Set an option (see MOE_OPT_*).  Synchronous, host only. */
moe_status_t moe_plan_set_option(moe_plan_t plan, int key, double value);

/* Grow the plan-owned workspace to hold max_T tokens (allocated on the
 * legacy default stream, then synchronised).  moe_forward grows it on demand,
 * stream-ordered: the old workspace is released with cudaFreeAsync and the
 * new one taken with cudaMallocAsync on the call's stream, so the call does
 * not synchronise the host.  Call this first when the calls are to be
 * captured in a CUDA graph: a call that would grow the workspace while its
 * stream is capturing returns MOE_ERR_UNSUPPORTED and launches nothing. */
moe_status_t moe_plan_reserve(moe_plan_t plan, int max_T);

/* The whole layer for T tokens (T = 0 is a no-op).
 *   x              bf16 [T,d]
 *   router_w       fp32 [E,d]
 *   router_gamma   fp32 [d]    (applied as 1 + gamma)
 *   router_bias    fp32 [E] or NULL
 *   expert_gamma   fp32 [d] or NULL: the experts then read the expert-side
 *                  RMSNorm x / sqrt(mean(x^2) + eps) * (1 + expert_gamma)
 *                  (rounded to bf16), the model's pre-FFN norm whose only
 *                  consumer is the fused gate_up (Quant-Tuner pull request,
 *                  "Answers to the motivating questions"); NULL: raw x.
 *                  The router and the residual always see the raw x.
 *   w_gate_up      see moe_wdtype_t (rows [0,f) gate, [f,2f) up)
 *   w_down         see moe_wdtype_t
 *   scales_gate_up int4: fp16 [E,2f,ceil(d/128)]; fp8: fp32 [E,2f]; NULL for bf16
 *   scales_down    int4: fp16 [E,d,ceil(f/128)];  fp8: fp32 [E,d];  NULL for bf16
 *                  fp4: E scale records each (see MOE_W_FP4_E2M1), R = 2f, C = d for
 *                  gate_up and R = d, C = f for down
 *   residual       bf16 [T,d] or NULL; may alias `out`
 *   out            bf16 [T,d]; must not overlap x
 * Asynchronous on `stream`; the plan's workspace holds the routing tables
 * until the next call. */
moe_status_t moe_forward(moe_plan_t plan, int T, const void* x, const float* router_w,
                         const float* router_gamma, const float* router_bias,
                         const float* expert_gamma, const void* w_gate_up, const void* w_down, const void* scales_gate_up,
                         const void* scales_down, const void* residual, void* out, void* stream);

/* moe_forward with x, residual and out in HOST memory (pinned or pageable):
 * copies x (and residual) to the plan's device buffers, runs the layer, copies
 * out back and synchronises `stream` before returning.  Weights and router
 * tensors are device pointers as in moe_forward. */
moe_status_t moe_forward_host(moe_plan_t plan, int T, const void* x_host, const float* router_w,
                              const float* router_gamma, const float* router_bias,
                              const float* expert_gamma, const void* w_gate_up, const void* w_down,
                              const void* scales_gate_up, const void* scales_down,
                              const void* residual_host, void* out_host, void* stream);

/* Size of the fixed device array used by moe_forward_noalloc (40 MiB). */
#define MOE_NOALLOC_SCRATCH_BYTES (40u * 1024u * 1024u)

/* moe_forward for callers that cannot allocate device memory: a host that
 * owns and pre-assigns every byte of the GPU (an inference server or plugin
 * host with its own allocator), or a latency-critical loop that must never
 * enter the CUDA allocator.  The pages describe no such entry point; it is
 * this library's addition.
 *
 * Same arguments, layouts, results and errors as moe_forward, plus
 * status_out: a DEVICE int32 (or NULL) that receives this call's device
 * status word (MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE_CHECK) in stream
 * order.  The same status also stays in the array: moe_plan_sync_status on
 * the plan reports it (with the plan's own status word, first error first)
 * as long as no later moe_forward_noalloc call on the device has replaced
 * it, so a caller that passes NULL still learns of a device-side error.  The caller still passes every input and output.  All intermediates
 * (routing tables, gathered rows, h, y, counters) live in one file-scope
 * __device__ array of MOE_NOALLOC_SCRATCH_BYTES; the call never calls
 * cudaMalloc, cudaFree or any allocating routine.
 *   - Limit: the intermediates of T tokens must fit the array (about
 *     T*k*(6d + 2f) + T*(16k + 4) bytes plus small tables; one
 *     256-token canvas of the 2816/704/128/top-8 layer needs 37.5 MB).  A larger call
 *     returns MOE_ERR_UNSUPPORTED and launches nothing.
 *   - Set-up: a call looks up the array's device address on its device
 *     (cudaGetSymbolAddress, the device current) whenever its stream is not
 *     capturing, so the address stays right after a device reset reloads the
 *     library's module; while a capture is in progress the address of the
 *     last lookup on that device is used.  Make the first call on each device
 *     before any stream capture.
 *   - The array is part of the library's device image: every GPU that loads
 *     it holds the 40 MiB until the process exits.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents (each call clears the words that must start at zero).
 *     Calls that overlap on the GPU (other streams, other threads, other
 *     plans) race on it and must be serialised by the caller.
 *   - bf16 plans only (int4, fp8 and fp4 plans return MOE_ERR_UNSUPPORTED);
 *     MOE_OPT_PROFILE and MOE_OPT_DEBUG are ignored. */
moe_status_t moe_forward_noalloc(moe_plan_t plan, int T, const void* x, const float* router_w,
                                 const float* router_gamma, const float* router_bias,
                                 const float* expert_gamma, const void* w_gate_up, const void* w_down,
                                 const void* scales_gate_up, const void* scales_down,
                                 const void* residual, void* out, int32_t* status_out,
                                 void* stream);

/* Routing only: idx int32 [T,k] (j order), w fp32 [T,k], gap fp32 [T] or NULL
 * (gap = z_(k) - z_(k+1), +inf when k == E). */
moe_status_t moe_route(moe_plan_t plan, int T, const void* x, const float* router_w,
                       const float* router_gamma, const float* router_bias, int32_t* idx_out,
                       float* w_out, float* gap_out, void* stream);

/* ---- expert parallelism over the GPUs of one node -----------------------
 *
 * The pages run the whole model on one device (Hugging Face card
 * "Infatoshi/diffusiongemma-26B-A4B-iq2xxs-4070": every layer offloaded to one
 * card; auto-round pull request, transformers backend test log: one GPU).
 * These three calls are the library's own extension that spreads each
 * layer's experts
 * over N ranks of one node, rank r owning experts [r*E/N, (r+1)*E/N).
 * The pages' model has 128 experts with 8 active per token (Quant-Tuner pull
 * request, Summary; the ROCmFP4-GGUF card's header).  A layer call is:
 *   1. moe_route (every rank, its own tokens) -> idx, w;
 *   2. moe_ep_dispatch: the token-expert assignments sorted by owner, each
 *      owner's rows contiguous in (token, j) order, x rows packed to match;
 *   3. the caller exchanges counts, rows and expert ids with an all-to-all
 *      (e.g. NCCL through torch.distributed; no library kernel reads another
 *      GPU's memory);
 *   4. moe_expert_rows on every owner (a plan of its E/N experts, k = 1):
 *      y rows in the order received;
 *   5. the caller returns the y rows with the reverse all-to-all;
 *   6. moe_combine_rows: out_t = residual_t + sum_j w_tj y_(t,j) in j order.
 * With bf16 y rows (MOE_OPT_Y_BF16 on, the default) every rank's out equals
 * moe_forward's bytes for bf16 and int4 weights (and for fp8 / fp4 weights
 * without expert_gamma: those paths carry fp16 rows, and a row normalised
 * on the sender travels as bf16), provided the owner plan and moe_forward's
 * plan have the same explicit MOE_OPT_CHUNK_TOKENS (its default depends on
 * the call's size, which differs between them): an expert's tokens then
 * form the same chunks on the owner as in moe_forward, and the expert
 * kernels' arithmetic for a chunk depends on that chunk alone. */

/* Step 2, on the routing plan (E experts, top-k) of the sending rank.
 *   x             bf16 [T, d]  the rank's tokens
 *   idx           int32 [T, k] the experts moe_route chose
 *   n_ranks       owners; E % n_ranks == 0, 1 <= n_ranks <= min(E, 256)
 *   expert_gamma  fp32 [d] or NULL: rows are sent as the expert-side RMSNorm
 *                 of x (as in moe_forward), else as x
 *   send_rows     bf16 [T*k, d] out: rows for owner 0, then owner 1, ...
 *   send_expert   int32 [T*k] out: each send row's expert index on its owner
 *   pos           int32 [T*k] out: send row of assignment t*k + j
 *   send_counts   int32 [n_ranks] out (device): rows for each owner
 * Asynchronous on `stream`; an expert id outside [0, E) is reported as
 * MOE_ERR_DEVICE_CHECK by moe_plan_sync_status. */
moe_status_t moe_ep_dispatch(moe_plan_t plan, int T, const void* x, const int32_t* idx,
                             int n_ranks, const float* expert_gamma, void* send_rows,
                             int32_t* send_expert, int32_t* pos, int32_t* send_counts,
                             void* stream);

/* Step 4, on a plan created with the owner's expert count and k = 1: y_rows[r]
 * = expert row_expert[r] applied to x_rows[r] (gate_up, GELU-tanh * up,
 * down), rounded to bf16.  Weights and scales are the owner's slice of the
 * layer's tensors, laid out as for moe_forward.
 *   x_rows        bf16 [R, d]   rows as received (already normalised)
 *   row_expert    int32 [R]     expert of each row on this owner, [0, E)
 *   expert_gamma  fp32 [d] or NULL (normally NULL: the sender normalised)
 *   y_rows        bf16 [R, d]   out, same row order
 * R = 0 is a no-op.  A plan with k != 1 returns MOE_ERR_INVALID_ARG. */
moe_status_t moe_expert_rows(moe_plan_t plan, int R, const void* x_rows, const int32_t* row_expert,
                             const float* expert_gamma, const void* w_gate_up, const void* w_down,
                             const void* scales_gate_up, const void* scales_down, void* y_rows,
                             void* stream);

/* Step 6, on the sending rank's routing plan: out_t = residual_t + sum_j
 * w[t,j] * y_rows[pos[t*k+j]], j in order, fp32, one rounding to bf16.
 *   y_rows    bf16 [T*k, d] the returned rows, in send order
 *   pos, w    from moe_ep_dispatch / moe_route
 *   residual  bf16 [T, d] or NULL; may alias out
 * A pos outside [0, T*k) is clamped and reported as MOE_ERR_DEVICE_CHECK. */
moe_status_t moe_combine_rows(moe_plan_t plan, int T, const void* y_rows, const int32_t* pos,
                              const float* w, const void* residual, void* out, void* stream);

/* Device-to-device copies of the last moe_forward's routing tables (NULL to
 * skip one): offsets int32 [E+1] (expert segment starts in slot order),
 * perm int32 [T*k] (token of each slot), slot_of int32 [T*k] (slot of
 * assignment t*k+j).  Asynchronous on `stream`. */
moe_status_t moe_plan_routing(moe_plan_t plan, int32_t* offsets, int32_t* perm, int32_t* slot_of,
                              void* stream);

/* Synchronise `stream`, return the device status word (MOE_OK, MOE_ERR_TIMEOUT
 * or MOE_ERR_DEVICE_CHECK) and clear it.  The plan's own word comes first;
 * if it is clear, the word of the plan's last moe_forward_noalloc call (see
 * there) is reported and cleared.  With MOE_OPT_DEBUG on, a damaged
 * workspace guard block is reported as MOE_ERR_DEVICE_CHECK. */
moe_status_t moe_plan_sync_status(moe_plan_t plan, void* stream);

/* With MOE_OPT_PROFILE on: total device time (ms) and number of launches of
 * kernel `kernel` (MOE_K_*) recorded since the last read; synchronises the
 * recorded events and clears the record. */
moe_status_t moe_plan_profile(moe_plan_t plan, int kernel, double* total_ms, int* launches);

/* Release the plan and its workspace (synchronous). NULL is ignored. */
void moe_plan_destroy(moe_plan_t plan);

/* Static description of a status code. */
const char* moe_status_str(moe_status_t status);

/* ---- lm_head over the canvas and the entropy-bound acceptance step -------
 *
 * The step after the layer stack (fucina docs "DiffusionGemma 26B-A4B --
 * block text-diffusion": 256-token canvases denoised with the entropy-bound
 * sampler, temperature 0.8 -> 0.4, bound 0.1; auto-round pull request:
 * EntropyBoundSamplerConfig entropy_bound 0.1).  For each token t (h_t bf16
 * [d], the lm_head / tied embedding W bf16 [V, d]):
 *   z_v = h_t . W[v]  (fp32 accumulation), optionally softcap*tanh(z_v/softcap)
 *   u_v = z_v / temperature;  logZ_t = log sum_v exp(u_v)
 *   H_t = logZ_t - sum_v softmax(u)_v u_v            (entropy, nats)
 *   token_t = argmax_v z_v (lowest v on ties)
 * then, over the positions still masked: sorted by (H_t, t), accept the
 * longest prefix whose entropies, all but the last, sum (in fp64) to at most
 * entropy_bound; the lowest-entropy masked position is always accepted.
 * The pages name the rule but do not state it; this is the entropy-bounded
 * unmasking rule it is named after (the library's reading).
 * The [T, V] logits are never written: the GEMM's epilogue folds them into
 * per-(token, 256-row tile) softmax statistics on chip. */
typedef struct moe_lmhead_s* moe_lmhead_t;

/* Handle for a vocabulary of V rows of width d (1 <= V <= 2^24, d a multiple
 * of 64 in [64, 8192]); no device memory until the first call. */
moe_status_t moe_lmhead_create(int V, int d, moe_lmhead_t* out);

/* Arguments (device pointers; h and w 16-byte aligned, outputs 4-byte
 * aligned except accept_out):
 *   T              tokens, 1..4096 (0: nothing launched)
 *   h              bf16 [T, d]   final hidden states (after the final norm)
 *   w              bf16 [V, d]   lm_head weight
 *   temperature    > 0
 *   softcap        >= 0 (0: no soft cap)
 *   masked         uint8 [T], nonzero = still masked, or NULL (all masked)
 *   entropy_bound  >= 0
 *   token_out      int32 [T]     argmax token of every position
 *   entropy_out    fp32 [T]      H_t
 *   logz_out       fp32 [T]      logZ_t (NULL to skip)
 *   accept_out     uint8 [T]     1 = masked and accepted this step
 * Asynchronous on `stream`; bounded-wait expiry is reported by
 * moe_lmhead_sync_status.  The handle's workspace grows stream-ordered on
 * `stream` when T exceeds every earlier call's (a growth while the stream is
 * capturing returns MOE_ERR_UNSUPPORTED: make a call of the largest T first). */
moe_status_t moe_lmhead_forward(moe_lmhead_t lh, int T, const void* h, const void* w,
                                float temperature, float softcap, const uint8_t* masked,
                                float entropy_bound, int32_t* token_out, float* entropy_out,
                                float* logz_out, uint8_t* accept_out, void* stream);

/* Synchronise `stream`, return the handle's device status word and clear it. */
moe_status_t moe_lmhead_sync_status(moe_lmhead_t lh, void* stream);

/* on != 0: moe_lmhead_forward records CUDA events around its GEMM launch
 * (and launches without programmatic dependent launch, so the events bound
 * the GEMM alone); moe_lmhead_profile returns the total GEMM time (ms) and
 * the number of launches recorded since the last read, and clears them. */
moe_status_t moe_lmhead_set_profile(moe_lmhead_t lh, int on);
moe_status_t moe_lmhead_profile(moe_lmhead_t lh, double* gemm_ms, int* launches);

/* Release the handle and its workspace (synchronous). NULL is ignored. */
void moe_lmhead_destroy(moe_lmhead_t lh);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
