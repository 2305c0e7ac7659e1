/*
 * gdit.h -- C ABI of the B200 (sm_100a) flow-matching DiT action head.
 *
 * The library computes GR00T's action-head inference loop ("get_action"): a
 * K-step Euler integration x <- x + dt * v(x, t) of an action chunk
 * [B, H, A], where v is the 32-layer AlternateVLDiT conditioned on the VLM
 * backbone features (cross-attention on even layers, self-attention on odd
 * layers) and on per-embodiment state/action encoders and action decoder.
 *
 * Sources (page title, then section):
 *   Isaac-GR00T "Model architecture" page (nvidia-isaac-gr00t.mintlify.app/
 *     architecture.md): "Action head architecture", "Diffusion transformer
 *     (DiT)" (Architecture details, Transformer block structure, AlternateVLDiT
 *     variant), "Flow matching diffusion" (Inference (denoising)),
 *     "Embodiment-specific projectors" (CategorySpecificLinear, Multi-embodiment
 *     action encoder).
 *   Isaac-GR00T "GR00T model class" page (api/model/gr00t-model.md):
 *     get_action returns action_pred of shape (B, action_horizon, action_dim);
 *     "Flow matching diffusion" config (num_inference_timesteps = 4,
 *     num_timestep_buckets = 1000).
 *   PhyAI "Single-GPU inference for GR00T-N1.7" (phyai.mintlify.app/models/
 *     gr00t/ws1.md): Overview (the embodiment id routes the encoders and the
 *     decoder; it is not a token), "Prepare a request and construct the engine"
 *     (optional fixed noise for deterministic regression; CUDA-graph profiles,
 *     an unlisted profile is an error; max_batch_size fixed at build), "Close
 *     the engine" (close releases the graph registries), "Current limitations"
 *     (one GPU; normalized, padded actions are returned).
 *
 * Conventions shared by every entry point
 *   - Every function returns an int status: GDIT_OK (0) or a negative GDIT_E*
 *     code.  Nothing throws across the ABI.  gdit_strerror() names a code and
 *     gdit_last_error() gives the detail message of the last failed call on a
 *     handle (or of the last failed gdit_create when the handle is NULL).
 *   - "device" pointers are CUDA device (or managed) memory of the handle's
 *     device, owned by the caller, and must stay valid until the work enqueued
 *     on the call's stream has finished.  "host" pointers are read before the
 *     call returns unless stated otherwise.
 *   - Row-major, densely packed tensors; shapes are given as [dim0, dim1, ...].
 *   - Calls on one handle must not run concurrently from several host threads.
 *     The handle's workspace (activations, K/V cache, status word) is shared by
 *     its calls: calls on different streams must be ordered by the caller (an
 *     event or a synchronize), or use one handle per stream.  Handles are
 *     independent of one another.
 */
#ifndef GDIT_H
#define GDIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */
#define GDIT_OK 0
#define GDIT_EINVAL (-1)    /* bad argument: null pointer, size out of range, missing/ill-shaped weight */
#define GDIT_ENOMEM (-2)    /* device or host allocation failed */
#define GDIT_ECUDA (-3)     /* a CUDA runtime/driver call failed (message says which) */
#define GDIT_EPROFILE (-4)  /* strict-profile handle: (batch, seq, steps) was not prepared */
#define GDIT_ETIMEOUT (-5)  /* a device-side bounded wait expired; the kernel returned early */
#define GDIT_EDEVICE (-6)   /* device-detected bad input (e.g. embodiment_id out of range) */
#define GDIT_ENODEV (-7)    /* no usable sm_100 device */

/* dtype codes for gdit_tensor.dtype and gdit_get_action's bb_dtype */
#define GDIT_F32 0
#define GDIT_BF16 1         /* raw bfloat16 bit patterns (uint16) */

/* flags for gdit_config.flags */
#define GDIT_FLAG_STRICT_PROFILES 1u  /* unprepared (batch, seq, steps) -> GDIT_EPROFILE, never a capture */
#define GDIT_FLAG_NO_GRAPH 2u         /* run eagerly (no CUDA graph); same kernels, for debugging */
#define GDIT_FLAG_NO_SMALL 4u         /* never use the persistent loop of batches 1-4 (one CTA group per
                                         sample); they then run the same per-layer kernels as larger
                                         batches */
#define GDIT_FLAG_NO_TMA_STORE 8u     /* DiT GEMMs store their outputs thread by thread instead of by TMA */
#define GDIT_FLAG_NO_PAIR 16u         /* the DiT GEMMs and the cross K/V projection never run on CTA pairs
                                         (cta_group::2, 256-row tiles) */
#define GDIT_FLAG_NO_SKINNY 32u       /* the DiT GEMMs of few rows (batches of up to 9 samples on the
                                         per-layer path) run on the tensor-core GEMM instead of the
                                         skinny-M kernel */

/* ------------------------------------------------------------------ config
 * Model geometry and capacity.  Every size is explicit.  Defaults of the
 * pages' model (hidden etc. of the full-size workloads): num_layers 32,
 * hidden 1024, num_heads 16, head_dim 64 (hidden = num_heads * head_dim),
 * mlp_hidden 4096, backbone_dim 2048, action_dim 32, state_dim 64,
 * action_horizon 16, num_embodiments 32, time_freq_dim 256,
 * num_timestep_buckets 1000, ln_eps 1e-5.
 * Constraints (else GDIT_EINVAL): num_layers even and >= 2; head_dim 32 or 64;
 * hidden in {128, 256, 512, 1024, 2048}; mlp_hidden, backbone_dim multiples of
 * 64; action_dim and state_dim multiples of 32 and <= 256; action_horizon in
 * [1, 63]; num_embodiments in [1, 64]; time_freq_dim even and >= 2;
 * num_timestep_buckets >= 1; ln_eps > 0; max_batch in [1, 4096];
 * max_backbone_seq in [1, 65536]; attend_text_every_n_blocks >= 0. */
typedef struct {
  int num_layers, hidden, num_heads, head_dim, mlp_hidden, backbone_dim;
  int action_dim, state_dim, action_horizon, num_embodiments;
  int max_batch, max_backbone_seq, time_freq_dim, num_timestep_buckets;
  float ln_eps;
  unsigned flags;           /* GDIT_FLAG_* */
  int device;               /* CUDA device ordinal */
  /* AlternateVLDiT image/text split (Isaac-GR00T architecture page,
   * "AlternateVLDiT variant"): 0 = every cross layer attends to all valid
   * tokens; n >= 1 = cross block idx attends to the valid text tokens when
   * idx % (2n) == 0, else to the valid image tokens (image_mask of
   * gdit_get_action_vl; without it no token is an image token). */
  int attend_text_every_n_blocks;
} gdit_config;

/* One named host weight tensor.  Names and shapes (D hidden, F mlp_hidden,
 * C num_embodiments, Dvl backbone_dim, A action_dim, Sd state_dim,
 * Tf time_freq_dim; even l: Din = Dvl, odd l: Din = D):
 *   t_enc.l1.w [D,Tf] t_enc.l1.b [D] t_enc.l2.w [D,D] t_enc.l2.b [D]
 *   blk{l}.ada.w [2D,D] .ada.b [2D]  blk{l}.q.w [D,D] .q.b [D]
 *   blk{l}.k.w [D,Din] .k.b [D]      blk{l}.v.w [D,Din] .v.b [D]
 *   blk{l}.o.w [D,D] .o.b [D]        blk{l}.ln3.g [D] .ln3.b [D]
 *   blk{l}.ff1.w [F,D] .ff1.b [F]    blk{l}.ff2.w [D,F] .ff2.b [D]
 *   out.ada.w [2D,D] out.ada.b [2D]  out.proj.w [D,D] out.proj.b [D]
 *   state_enc.l1.W [C,Sd,D] .b [C,D] state_enc.l2.W [C,D,D] .b [C,D]
 *   act_enc.W1.W [C,A,D] .b [C,D]    act_enc.W2.W [C,2D,D] .b [C,D]
 *   act_enc.W3.W [C,D,D] .b [C,D]    act_dec.l1.W [C,D,D] .b [C,D]
 *   act_dec.l2.W [C,D,A] .b [C,A]
 * Optional, given together: vlln.g [Dvl] vlln.b [Dvl], the vision-language
 * LayerNorm of each backbone token's features before the cross K/V (needs
 * Dvl a multiple of 256, at most 4096).
 * Plain linears are PyTorch [out, in] (y = x W^T + b).  Category-specific
 * weights keep CategorySpecificLinear's [C, in, out] (y = x W[c] + b[c]).
 * dtype GDIT_F32 (float) or GDIT_BF16 (uint16 bit patterns); matrices are
 * stored on the device in bf16 (rounded to nearest even from f32), biases,
 * LayerNorm parameters and the per-step tables in f32. */
typedef struct {
  const char* name;
  int dtype;
  int ndim;
  const int64_t* shape;
  const void* host_ptr;
} gdit_tensor;

typedef struct gdit_handle gdit_handle;

/* Validates config and the weight table (every name above present exactly
 * once with its shape; unknown names are an error), uploads the weights and
 * allocates the workspace for max_batch x max_backbone_seq.  The host weight
 * buffers are read before the call returns and are not retained.
 * On success *out owns all device memory of the model.  On failure *out is
 * NULL and gdit_last_error(NULL) holds the reason (e.g. the missing weight);
 * everything allocated before the failure has been freed.
 * Host-side fault injection (for testing callers' error paths): the
 * environment variable GDIT_FAULT, read here, is a comma-separated list of
 * kind:N items.  alloc:N makes the handle's N-th device allocation fail
 * (GDIT_ENOMEM), upload:N its N-th weight or table upload (GDIT_ECUDA), and
 * graph:N its N-th CUDA-graph instantiation, at the first call of a profile
 * or in gdit_prepare (GDIT_ECUDA); N counts from 1.  Only the host-side call
 * is made to fail: nothing runs on the device for it.  A malformed value
 * makes gdit_create return GDIT_EINVAL. */
int gdit_create(const gdit_config* cfg, const gdit_tensor* weights, int n_weights, gdit_handle** out);

/* Frees graphs, weights and workspace.  Waits for the handle's outstanding work.
 * NULL is accepted.  (PhyAI "Close the engine".) */
void gdit_destroy(gdit_handle* h);

/* Inference: out_actions = x_K where x_0 = init_noise and
 * x_{k+1} = x_k + (1/K) v(x_k, t_k), t_k = k/K, t_discretized = floor(t_k * buckets)
 * (Isaac-GR00T architecture page, "Inference (denoising)").
 *   backbone_features  device [batch, seq, backbone_dim], f32 or bf16 (bb_dtype)
 *   vl_mask            device uint8 [batch, seq]; 1 = token valid (attention_mask == 1);
 *                      any pattern; a sample with no valid token gets a zero
 *                      cross-attention output
 *   state              device f32 [batch, 1, state_dim]
 *   embodiment_id      device int32 [batch], each in [0, num_embodiments); an id out of
 *                      range is not read out of bounds: that sample's output is NaN
 *                      and gdit_sync_status() reports GDIT_EDEVICE
 *   init_noise         device f32 [batch, action_horizon, action_dim]
 *   num_steps          K in [1, 64]
 *   out_actions        device f32 [batch, action_horizon, action_dim]; may alias init_noise
 *   batch in [1, max_batch], seq in [1, max_backbone_seq]
 *   cuda_stream        cudaStream_t (NULL = legacy default stream)
 * Buffer sizes are the caller's contract: the library reads and writes every
 * buffer by (batch, seq) and the handle's dimensions and cannot see a device
 * buffer's size, so a smaller buffer is read or written past its end.  (The
 * Python binding checks the tensors' shapes before the call.)
 * Asynchronous on cuda_stream.  The first call of a new (batch, seq, K) profile
 * captures a CUDA graph of the whole loop (unless GDIT_FLAG_NO_GRAPH); with
 * GDIT_FLAG_STRICT_PROFILES that profile must have been gdit_prepare()d.
 * The per-K timestep tables (TimestepEncoder, AdaLN modulation, the timestep
 * half of the action encoder's W2) depend only on the weights and K and are
 * computed by the library's kernels on the first call with that K, then kept. */
int gdit_get_action(gdit_handle* h, const void* backbone_features, int bb_dtype,
                    const uint8_t* vl_mask, const float* state, const int32_t* embodiment_id,
                    const float* init_noise, int num_steps, float* out_actions,
                    int batch, int seq, void* cuda_stream);

/* gdit_get_action with the image/text split's image_mask: device uint8
 * [batch, seq], 1 = image token (input_ids == image_token_index), used when
 * the handle's attend_text_every_n_blocks > 0; NULL = no image token.  The
 * cross layers' K/V are computed once over all valid tokens; each cross
 * layer's attention keeps the keys of its kind (a sample with no key of that
 * kind gets a zero cross-attention output). */
int gdit_get_action_vl(gdit_handle* h, const void* backbone_features, int bb_dtype,
                       const uint8_t* vl_mask, const uint8_t* image_mask, const float* state,
                       const int32_t* embodiment_id, const float* init_noise, int num_steps,
                       float* out_actions, int batch, int seq, void* cuda_stream);

/* Same computation with HOST buffers (same shapes and meanings as above).
 * Copies the inputs to handle-owned device buffers, runs, copies out_actions
 * back and synchronizes cuda_stream before returning.  Host buffers may be
 * pageable; pinned buffers make the copies asynchronous to the CPU. */
int gdit_get_action_host(gdit_handle* h, const void* backbone_features, int bb_dtype,
                         const uint8_t* vl_mask, const float* state, const int32_t* embodiment_id,
                         const float* init_noise, int num_steps, float* out_actions,
                         int batch, int seq, void* cuda_stream);

/* Captures the graph of profile (batch, seq, num_steps) ahead of time and
 * computes that K's tables.  Required per profile on strict-profile handles. */
int gdit_prepare(gdit_handle* h, int batch, int seq, int num_steps, int bb_dtype, void* cuda_stream);

/* Synchronizes the stream of the last call and returns its device status:
 * GDIT_OK, GDIT_EDEVICE (bad embodiment id) or GDIT_ETIMEOUT.  Clears it. */
int gdit_sync_status(gdit_handle* h);

const char* gdit_strerror(int code);
const char* gdit_last_error(const gdit_handle* h);

/* Library version string (not a model property). */
const char* gdit_version(void);

/* ------------------------------------------------------------ diagnostics
 * Read-only views of the state left by the last gdit_get_action on the
 * handle's stream (call gdit_sync_status first).  For tests and profiling. */

/* Routing of the last call: perm[i] = original index of the i-th sample in
 * embodiment order (stable counting sort by id, ties by sample index);
 * seg[c] .. seg[c+1] = sorted positions of category c; vofs[i] = first packed
 * valid backbone token of sorted sample i, vofs[batch] = total.  Host outputs:
 * perm int32 [batch], seg int32 [num_embodiments+1], vofs int32 [batch+1]. */
int gdit_debug_routing(gdit_handle* h, int32_t* perm, int32_t* seg, int32_t* vofs);

/* Cross-attention keys/values of cross layer `layer` (even, 0 <= layer <
 * num_layers) for the packed valid tokens of the last call, as f32 host
 * arrays k_out/v_out [total_valid, hidden] in packed (embodiment-sorted)
 * order.  *total_valid receives the row count; pass NULL buffers to query it. */
int gdit_debug_kv(gdit_handle* h, int layer, float* k_out, float* v_out, int* total_valid);

/* Failure detection check: launches one thread on `device` that waits, through
 * the bounded mbarrier wait every kernel of the library uses, on an mbarrier
 * that nothing ever arrives at, with a limit of limit_ns nanoseconds (1 us to
 * 1 s) instead of the kernels' 2 s.  No GPU fault or hang: the wait gives up,
 * records the timeout in a status word, and the thread exits.  Returns
 * GDIT_ETIMEOUT when the expiry was detected and reported (the expected
 * outcome), GDIT_EINVAL for a bad limit or device, GDIT_ENODEV without a GPU.
 * Allocates and frees one status word on the device; synchronous. */
int gdit_debug_wait_expiry(int device, unsigned long long limit_ns);

/* The plan of the skinny-M GEMM (the DiT linears of a few samples; a host
 * computation, no GPU needed): for out[M, N] = X[M, K] W[N, K]^T on num_sms
 * SMs, the row block (*mt m16 tiles), the units of 8 output features per
 * item (*nu), the ring depth (*stages), the CTAs (*ctas: one item each) and a
 * CTA's dynamic shared memory (*smem_bytes).  Returns GDIT_OK with a plan, or
 * GDIT_EINVAL for a shape the kernel does not take or when no plan fits one
 * item per SM (such a GEMM runs on the tensor-core kernel).  For tests. */
int gdit_debug_skinny_plan(long long M, int N, int K, int num_sms, int* mt, int* nu, int* stages, int* ctas,
                           int* smem_bytes);

/* Whether a call of `batch` samples and num_steps Euler steps on a model of
 * geometry *cfg runs the whole loop as the persistent kernel, on num_sms SMs
 * (a host computation, no GPU needed): *group_ctas = CTAs per sample group
 * (num_sms / batch), 0 when the call runs the per-layer kernels; *grouped = 1
 * when the grouped instantiation runs (several samples, or a CTA with more
 * than 4 units of 8 features in some linear).  GDIT_EINVAL for an invalid
 * configuration or arguments.  For tests. */
int gdit_debug_small_plan(const gdit_config* cfg, int batch, int num_steps, int num_sms, int* group_ctas,
                          int* grouped);

/* Range-checked build.  libgdit_checked.so is the same library compiled with
 * GDIT_CHECKED=1 (same entry points, same results):
 *   - every device allocation of a handle sits between two 4 KiB guard bands
 *     filled with 0xA5 when allocated;
 *   - the kernels check the indices they derive from the caller's inputs
 *     before following them: the packed-token rows each sample writes (inside
 *     the packed buffer), the key spans of the cross attention (inside a
 *     head's block of the K/V cache) and the sample permutation (inside the
 *     batch).  An index out of range is not followed: the access is skipped
 *     and gdit_sync_status returns GDIT_EDEVICE.
 * gdit_is_checked returns 1 in that build and 0 in libgdit.so.
 * gdit_check_canaries synchronizes the device and writes to *corrupted_bytes
 * the number of guard bytes of h's allocations that no longer hold 0xA5 (0
 * unless something wrote past the end or before the start of a buffer);
 * GDIT_EINVAL in a regular build.
 * gdit_debug_poke_guard (test hook) overwrites the first guard byte after
 * allocation `which` (0-based, in allocation order) from the host, as a
 * one-element overrun would; GDIT_EINVAL in a regular build or for a bad
 * index. */
int gdit_is_checked(void);
int gdit_check_canaries(gdit_handle* h, long long* corrupted_bytes);
int gdit_debug_poke_guard(gdit_handle* h, int which);

/* Per-kernel-class timing of one eager (graph-free) run of gdit_get_action
 * with the given device inputs, each launch bracketed by CUDA events on
 * cuda_stream.  Fills up to max_stats entries; returns the count (>= 0) or an
 * error.  flops / bytes are the algorithmic work of all launches of the class. */
typedef struct {
  char name[32];
  int launches;
  double total_ms;
  double flops;
  double bytes;
} gdit_kernel_stat;

int gdit_profile_get_action(gdit_handle* h, const void* backbone_features, int bb_dtype,
                            const uint8_t* vl_mask, const float* state, const int32_t* embodiment_id,
                            const float* init_noise, int num_steps, float* out_actions,
                            int batch, int seq, void* cuda_stream,
                            gdit_kernel_stat* stats, int max_stats);

/* Unit hook for the tcgen05 GEMM: C[M,N] (f32) = A[M,K] B[N,K]^T + bias[N]
 * with A, B bf16 device matrices (row-major, K contiguous), bias f32 device
 * (may be NULL), C f32 device.  bn in {32, 64, 128, 256}, splits >= 1 (split-K).
 * Requires N % 32 == 0 and K % 8 == 0.  Synchronizes cuda_stream. */
int gdit_test_gemm(const void* A, const void* B, const float* bias, float* C,
                   int M, int N, int K, int bn, int splits, void* cuda_stream);

/* Split-K GEMM that allocates nothing (no counterpart in the source pages: it
 * serves callers, not the method).  Same operation, layouts and limits as
 * gdit_test_gemm: C[M,N] (f32) = A[M,K] B[N,K]^T + bias[N], A and B bf16 device
 * matrices (row-major, K contiguous), bias f32 device or NULL, C f32 device;
 * all owned by the caller.
 * For callers that cannot call cudaMalloc at call time, for example a robot's
 * control loop, where cudaMalloc/cudaFree may synchronise the device and take
 * unbounded time, or a deployment whose memory budget is fixed up front.  The
 * split-K partials, per-tile counters and status word live in one fixed
 * device array inside the library (4 MiB of partials, 4096 output tiles),
 * which every GPU that loads the library keeps until the process exits.
 * Limits (else GDIT_EINVAL): ceil(M/128) * ceil(N/bn) <= 4096 and, when
 * splits > 1, splits * M * N <= 1048576.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture begins on that device.  Every call shares the
 * array and leaves its contents behind: calls that overlap on the GPU
 * (several streams, several host threads) race and give wrong results.  Each
 * call clears the status word and the tile counters on cuda_stream, launches
 * the GEMM, reads the status word back and synchronizes cuda_stream before it
 * returns.  Returns GDIT_OK, GDIT_EINVAL or GDIT_ETIMEOUT. */
int gdit_gemm_static_scratch(const void* A, const void* B, const float* bias, float* C,
                             int M, int N, int K, int bn, int splits, void* cuda_stream);

#ifdef __cplusplus
}
#endif
#endif /* GDIT_H */
