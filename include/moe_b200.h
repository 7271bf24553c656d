/*
 * moe_b200.h - C ABI of the B200 (sm_100a) Nemotron-H MoE FFN layer.
 *
 * The layer (NemotronMoeLayer, nemotron_moe.rs, module documentation): the
 * tokens are RMS-normalised and scored by the gate; a sigmoid top-k picks the
 * routed experts of each token.  Each chosen expert applies its up projection,
 * relu^2 and its down projection (between an fc1 into and an fc2 out of the
 * latent width for LatentMoE), and the expert outputs are combined with the
 * routing weights.  The always-on shared expert (up, relu^2, down) runs on the
 * normed tokens too, and both results are added to `hidden`.  The routing
 * never leaves the device: a forward pass copies nothing back to the host
 * (same module documentation; MoeLayer, `forward`).
 *
 * Notation: T tokens, H hidden_size, E num_experts, k top_k, I moe_inter,
 * S shared_inter, L latent_size (0 = direct), D = (L ? L : H) the width the
 * routed experts work on, R = T*k routed rows.
 *
 * Layouts: every matrix is row-major with the input dimension contiguous,
 * i.e. weights are [out, in] (nn.Linear layout).  Routed expert weights are
 * STACKED: up [E, I, D], down [E, D, I] (expert e's matrix starts at element
 * e*I*D).  BF16 values are IEEE binary32's upper 16 bits; FP8 values are OCP
 * E4M3 ("fn") bytes with one float32 scale per output row.
 *
 * Ownership: every pointer passed to moe_create is BORROWED; it must stay
 * valid and unchanged until moe_destroy.  The handle owns a device workspace
 * sized for max_tokens, allocated in moe_create and freed in moe_destroy.
 * moe_forward allocates nothing, never synchronises the host and never reads
 * device memory back; it only enqueues kernels on the caller's stream.
 *
 * Streams: `stream` arguments are cudaStream_t values passed as void*
 * (NULL = the legacy default stream).  One handle must not run two calls
 * concurrently on different streams (they share the workspace).
 *
 * Errors: every entry point validates its arguments on the host before any
 * launch and returns a moe_status; nothing is enqueued when it fails.  Launch
 * failures come back as MOE_ERR_CUDA.  A handle belongs to the device that
 * was current at moe_create: every call that takes a handle (except
 * moe_destroy, which switches to that device itself) returns MOE_ERR_DEVICE
 * when another device is current.  Device-side bounded waits that time out
 * set a device status word, read by moe_get_device_status.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_CONFIG = 1,      /* sizes, top_k bounds, dtype, divisibility */
  MOE_ERR_NULL_POINTER = 2,        /* a required pointer is NULL */
  MOE_ERR_MISALIGNED = 3,          /* a pointer is not 16-byte aligned */
  MOE_ERR_TOKENS_OUT_OF_RANGE = 4, /* num_tokens outside [1, max_tokens] */
  MOE_ERR_OUT_OF_MEMORY = 5,       /* workspace allocation failed in moe_create */
  MOE_ERR_CUDA = 6,                /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE = 7,              /* no sm_100 device is current, or not the handle's */
  MOE_ERR_INVALID_HANDLE = 8       /* NULL or destroyed handle */
} moe_status;

typedef enum {
  MOE_WEIGHTS_BF16 = 0,            /* stored as BF16 */
  MOE_WEIGHTS_FP8_E4M3_ROWSCALE = 1/* stored as E4M3 + float32 scale per output row */
} moe_weight_dtype;

/* Routing-kernel bounds (NemotronMoeLayer `new` refuses a top_k outside
 * 1..=num_experts or above the routing kernels' bounds; the pages do not
 * print the bound values, these are this library's). */
#define MOE_MAX_TOP_K 16
#define MOE_MAX_EXPERTS 256

/* Layer sizes (NemotronMoeLayer fields and the ModelConfig fields its
 * `prefill` reads: hidden_size, shared_expert_intermediate_size,
 * num_experts, rms_norm_eps, routed_scaling_factor, moe_latent_size,
 * moe_intermediate_size, num_experts_per_tok).
 * Requirements checked by moe_create (else MOE_ERR_INVALID_CONFIG):
 *   1 <= top_k <= num_experts, top_k <= MOE_MAX_TOP_K,
 *   num_experts <= MOE_MAX_EXPERTS, max_tokens >= 1,
 *   hidden_size, moe_inter, shared_inter, latent_size all multiples of 64
 *   (latent_size may be 0), rms_eps >= 0, routed_scaling_factor finite,
 *   expert_wdtype, shared_wdtype and latent_wdtype moe_weight_dtype values,
 *   and not FP8 routed experts together with latent_size > 0.
 * FP8 weights (nemotron_moe.rs `new` keeps FP8 copies of the routed
 * experts, the shared expert and fc1 / fc2) run as W8A8 on the tensor
 * cores: their input rows are quantised to E4M3 with one scale per row. */
typedef struct {
  int32_t hidden_size;           /* H */
  int32_t num_experts;           /* E */
  int32_t top_k;                 /* k */
  int32_t moe_inter;             /* I */
  int32_t shared_inter;          /* S */
  int32_t latent_size;           /* L, 0 = direct layer */
  int32_t max_tokens;            /* largest num_tokens a forward call may pass */
  float rms_eps;                 /* RMSNorm epsilon */
  float routed_scaling_factor;   /* multiplies the renormalised routing weights */
  int32_t expert_wdtype;         /* moe_weight_dtype of the routed experts' up / down */
  int32_t shared_wdtype;         /* moe_weight_dtype of the shared expert's up / down */
  int32_t latent_wdtype;         /* moe_weight_dtype of fc1 / fc2 (latent layers) */
} moe_config;

/* Device pointers to the layer's weights (all borrowed, 16-byte aligned). */
typedef struct {
  const void* norm_w;        /* [H] bf16, RMSNorm weight (multiplies x * rsqrt(mean x^2 + eps)) */
  const void* gate_w;        /* [E, H] bf16, router */
  const float* gate_bias;    /* [E] f32 added to the sigmoid scores for selection only; NULL = none */
  const void* up_w;          /* [E, I, D] bf16 or e4m3 */
  const void* down_w;        /* [E, D, I] bf16 or e4m3 */
  const float* up_scale;     /* [E, I] f32, FP8 only (else NULL) */
  const float* down_scale;   /* [E, D] f32, FP8 only (else NULL) */
  const void* shared_up_w;   /* [S, H] bf16 or e4m3 */
  const void* shared_down_w; /* [H, S] bf16 or e4m3 */
  const void* fc1_w;         /* [L, H] bf16 or e4m3, latent only (else NULL) */
  const void* fc2_w;         /* [H, L] bf16 or e4m3, latent only (else NULL) */
  const float* shared_up_scale;   /* [S] f32, FP8 shared expert only (else NULL) */
  const float* shared_down_scale; /* [H] f32, FP8 shared expert only (else NULL) */
  const float* fc1_scale;         /* [L] f32, FP8 fc1 / fc2 only (else NULL) */
  const float* fc2_scale;         /* [H] f32, FP8 fc1 / fc2 only (else NULL) */
} moe_weights;

/* A layer instance.  Its workspace serves one forward at a time: calls on one
 * handle are made from one host thread at a time, and passes enqueued on
 * different streams must not overlap on the device. */
typedef struct moe_handle moe_handle;

/* Which implementation moe_forward_path runs. */
typedef enum {
  MOE_PATH_AUTO = 0,     /* the decode path for num_tokens <= MOE_DECODE_MAX_TOKENS (with FP8 routed
                            experts: num_tokens == 1) where the layer supports it, else prefill */
  MOE_PATH_DECODE = 1,   /* weight-streaming tensor-core decode in one launch, weights x tokens
                            (num_tokens <= MOE_DECODE_MAX_TOKENS; direct layers with a BF16 shared
                            expert; FP8 routed experts are dequantised in shared memory) */
  MOE_PATH_PREFILL = 2   /* sort by expert + tcgen05 grouped GEMMs (any num_tokens) */
} moe_path;

#define MOE_DECODE_MAX_TOKENS 8

/* Validate the configuration and weights, build the TMA descriptors and
 * allocate the workspace on the current device.  Mirrors NemotronMoeLayer
 * `new` (nemotron_moe.rs): refuses top_k outside 1..=num_experts or above
 * the routing bounds.  The workspace keeps a copy of the gate with the norm
 * weight folded in (for the prefill router, which multiplies the raw rows
 * by it), made here and synchronously: norm_w and gate_w must not change
 * while the handle lives (the other weights are read at every forward).
 * On success *out receives a handle; on failure *out is set to NULL and
 * nothing stays allocated. */
MOE_API moe_status moe_create(const moe_config* config, const moe_weights* weights, moe_handle** out);

/* One forward pass over num_tokens tokens, enqueued on `stream`
 * (NemotronMoeLayer `prefill` / `decode`, which update hidden in place).
 *   hidden   [T, H] bf16, device, read then overwritten with the layer output
 *            residual_in + routed + shared (rounded once to bf16);
 *   residual [T, H] bf16, device, written with the pre-layer hidden (its
 *            input value is not read).
 * hidden and residual must not overlap.  Errors: MOE_ERR_INVALID_HANDLE,
 * MOE_ERR_NULL_POINTER, MOE_ERR_MISALIGNED, MOE_ERR_TOKENS_OUT_OF_RANGE,
 * MOE_ERR_CUDA. */
MOE_API moe_status moe_forward(moe_handle* h, void* hidden, void* residual, int32_t num_tokens,
                       void* stream);

/* moe_forward with an explicit choice of path (both compute the same layer). */
MOE_API moe_status moe_forward_path(moe_handle* h, void* hidden, void* residual, int32_t num_tokens,
                            int32_t path, void* stream);

/* Host-buffer variant for callers that hold the activations in host memory:
 * copies hidden_host [T, H] bf16 to the device, runs moe_forward, and copies
 * the output back into hidden_host and the pre-layer hidden into
 * residual_host (may be NULL to skip it).  Copies are cudaMemcpyAsync on
 * `stream`; the call returns after enqueueing them, so the caller
 * synchronises the stream before reading the host buffers.  Page-locked host
 * memory gives asynchronous copies.  Staging buffers come from the workspace
 * (no allocation).  With at most MOE_DECODE_MAX_TOKENS tokens on the
 * single-launch decode path, page-locked buffers that the device can address
 * are written by the kernel itself (the output rows and the residual go over
 * the bus as the kernel finishes them): one copy and one launch per call
 * instead of up to three copies. */
MOE_API moe_status moe_forward_host(moe_handle* h, void* hidden_host, void* residual_host,
                            int32_t num_tokens, void* stream);

/* Free the workspace and the handle.  Weights are not touched.  Waits for
 * the device to finish work that may still use the workspace. */
MOE_API moe_status moe_destroy(moe_handle* h);

/* Static string for a status code. */
MOE_API const char* moe_status_string(moe_status s);

/* --- parity / debug entry points (not needed for inference) ------------ */

/* Routing only (RMSNorm, FP32 gate, sigmoid top-k) for T tokens:
 *   idx [T, k] int32 expert ids, slots ordered by selection key descending
 *   (ties: lower expert index first); w [T, k] float32 routing weights
 *   (renormalised, times routed_scaling_factor).  Device pointers. */
MOE_API moe_status moe_route(moe_handle* h, const void* hidden, int32_t num_tokens, int32_t* idx,
                     float* w, void* stream);

/* Sort-by-expert of given routing idx [T, k] (device): perm [R] (sorted
 * position -> flat row t*k + j), inv [R] (flat row -> sorted position), off
 * [E+1] (exclusive prefix of per-expert counts).  Rows of one expert keep
 * token order.  Device pointers; idx values must lie in [0, E): a row with
 * an id outside it is left out of perm and off, gets inv = -1, and sets bit 2
 * of the device status word (moe_get_device_status). */
MOE_API moe_status moe_sort(moe_handle* h, const int32_t* idx, int32_t num_tokens, int32_t* perm,
                    int32_t* inv, int32_t* off, void* stream);

/* Largest num_tokens moe_sort_static accepts. */
#define MOE_SORT_STATIC_MAX_TOKENS 8192

/* The same sort-by-expert as moe_sort (same outputs, bit for bit), without a
 * handle and without allocating device memory.  The pages have no
 * counterpart: the layer they describe always sorts inside its forward
 * pass, from its own scratch.
 *
 * For callers that cannot allocate at the call: a runtime whose device
 * memory budget is fixed up front, a thread that must not stall the device
 * (cudaFree synchronises it), or code holding routing from elsewhere and no
 * moe_handle.  The scratch (about 75 KB: per-tile expert histograms, the
 * m-tile table, the status word) is a fixed array in the library's device
 * memory, one per device.
 *
 *   idx [num_tokens, top_k] int32 expert ids in [0, num_experts) (device).
 *   perm [R], inv [R], off [num_experts + 1] int32 (device, caller-owned,
 *   R = num_tokens * top_k): as moe_sort.
 *   status: optional device int32; set to 0, then bit 2 is OR-ed in if an
 *   id lies outside [0, num_experts) (that row is skipped).  NULL uses a
 *   word in the scratch that the caller cannot read: a bad id then goes
 *   unreported.  Either way the row gets inv = -1, and the entries of perm
 *   it would have filled (perm[off[E]..R)) are left unwritten.  Pass a
 *   status word unless the ids are known to be in range.
 *   stream: cudaStream_t (NULL = legacy default stream).
 *
 * Errors (nothing is launched): MOE_ERR_NULL_POINTER for a NULL idx, perm,
 * inv or off; MOE_ERR_INVALID_CONFIG for top_k outside [1, MOE_MAX_TOP_K],
 * num_experts outside [1, MOE_MAX_EXPERTS] or top_k > num_experts;
 * MOE_ERR_TOKENS_OUT_OF_RANGE for num_tokens outside
 * [1, MOE_SORT_STATIC_MAX_TOKENS]; MOE_ERR_DEVICE if the current device is
 * not sm_100; MOE_ERR_CUDA if resolving the scratch or a launch fails.
 *
 * The first call on a device does set-up (it looks up the scratch array's
 * device address, which may load the module on that device); make it before
 * any stream capture.  The address is kept for the device's primary context
 * (the runtime's context): call it with that context current, and not after
 * cudaDeviceReset, which discards the context the address belongs to.  The scratch is shared by all calls on a device, so
 * calls that overlap in time there (other streams or host threads) race;
 * the caller serialises them. */
MOE_API moe_status moe_sort_static(const int32_t* idx, int32_t num_tokens, int32_t top_k,
                                   int32_t num_experts, int32_t* perm, int32_t* inv, int32_t* off,
                                   int32_t* status, void* stream);

/* Copy the routing used by the last moe_forward* call on this handle (either
 * path) into idx [T, k] int32 and w [T, k] float32 (device pointers, same
 * meaning as moe_route's outputs); num_tokens must equal that call's. */
MOE_API moe_status moe_copy_routing(moe_handle* h, int32_t* idx, float* w, int32_t num_tokens,
                                    void* stream);

/* Copy the sort by expert used by the last moe_forward* call on this handle
 * (prefill path) into perm [R], inv [R] and off [E+1] int32 (device
 * pointers, R = num_tokens * top_k; same meaning as moe_sort's outputs, for
 * the routing moe_copy_routing returns).  num_tokens must equal that call's.
 * MOE_ERR_INVALID_CONFIG when that call took the decode path, which groups
 * tokens by expert without a sort. */
MOE_API moe_status moe_copy_sort(moe_handle* h, int32_t* perm, int32_t* inv, int32_t* off,
                                 int32_t num_tokens, void* stream);

/* Copy the device status word into *status (0 = no device-side timeout) and
 * clear it; after a non-zero status also reset the handle's device-side
 * tile and schedule counters, which a pass that gave up may have left
 * mid-count.  Synchronises the stream (debug use only). */
MOE_API moe_status moe_get_device_status(moe_handle* h, int32_t* status, void* stream);

/* Profiling: every following moe_forward* call records caller-owned CUDA
 * events (cudaEvent_t values passed as void*) on its stream: events[0] before
 * its first kernel launch and events[i] after its i-th launch, for i < count.
 * The array is borrowed and must stay valid while enabled; count = 0
 * disables.  Recording adds no device work besides the event records. */
MOE_API moe_status moe_set_stage_events(moe_handle* h, void* const* events, int32_t count);

/* Number of kernel launches the last moe_forward* call enqueued. */
MOE_API int32_t moe_last_launch_count(const moe_handle* h);

/* Path the last moe_forward* call took: MOE_PATH_DECODE or MOE_PATH_PREFILL
 * (-1 for an invalid handle or before the first forward). */
MOE_API int32_t moe_last_path(const moe_handle* h);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
