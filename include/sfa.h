/*
 * sfa.h — C ABI of the Signal Field Attention (SFA) operator for one NVIDIA
 * B200 (sm_100a).
 *
 * The operator (definitions by source page):
 *   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
 *        §2.1: near-field softmax attention over the last k tokens (eq.
 *        O_near), far-field EWMA of keys (eq. S_t), fusion O = O_near + α·S
 *        (eq. O).  §2.2: O(k·d) state.
 *   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
 *        §2.1: ring-buffer mean (16 slots), EMA field (γ = 0.98), semantic
 *        pool (64 slots, T = 0.07).  §2.2: enhancement = ring_mean +
 *        0.5·field + 0.5·semantic, clipped to ±ε, scaled by
 *        α_layer = α_base·(0.3 + 0.7·layer/(L−1))·decay^layer, added to the
 *        attention output.
 *   [P2] "Signal Field Attention (SFA)" (README page): SFA_Config defaults
 *        and the engine calls init(n_layers, hidden) /
 *        compute_enhancement(layer, attn_output), which this ABI follows
 *        with caller-owned buffers.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device and
 *     must be 16-byte aligned.  The caller owns all of them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; nothing synchronises except
 *     sfa_check_device_status.
 *   - Return value: SFA_OK (0) or a negative sfa_status.  No call throws, no
 *     kernel traps.  Errors detected on the device (a state whose header does
 *     not match the handle, a bounded wait that ran out) are latched in the
 *     handle and reported by sfa_check_device_status.
 *   - Layer-major, token-major layouts (d = head_dim, H = n_q_heads·d):
 *       prefill q   [L][batch][n][n_q_heads][d]    in_dtype
 *               k,v [L][batch][n][n_kv_heads][d]   in_dtype
 *               out [L][batch][n][H]               fp32 (bf16 in the bf16 output
 *                                                  modes, sfa_set_output_mode)
 *       decode  q   [L][batch][n_q_heads][d], k,v [L][batch][n_kv_heads][d],
 *               out [L][batch][H].
 *   - One state buffer serves `batch` sequences for all layers.  A state is
 *     used by one stream at a time; stream order serialises calls.  The
 *     compute calls never modify the handle, so it may be shared across
 *     streams and host threads (only sfa_set_decode_input_prefetch, the
 *     sfa_debug_* hooks and sfa_destroy modify it: call those while no other
 *     host thread uses the handle).
 */
#ifndef SFA_H
#define SFA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SFA_API __attribute__((visibility("default")))
#else
#define SFA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define SFA_ABI_VERSION 3

typedef enum sfa_status {
  SFA_OK = 0,
  SFA_ERR_INVALID_ARG = -1,     /* null pointer, negative size, bad value  */
  SFA_ERR_UNSUPPORTED = -2,     /* valid but not built: see sfa_init       */
  SFA_ERR_ALIGNMENT = -3,       /* a pointer is not 16-byte aligned         */
  SFA_ERR_STATE_MISMATCH = -4,  /* state header is not this handle's/batch */
  SFA_ERR_CUDA = -5,            /* a CUDA runtime call or launch failed     */
  SFA_ERR_DEVICE_TIMEOUT = -6,  /* a bounded device-side wait ran out       */
  SFA_ERR_WORKSPACE = -7        /* workspace smaller than required          */
} sfa_status;

typedef enum sfa_dtype { SFA_F32 = 0, SFA_BF16 = 1 } sfa_dtype;

/* What the compute calls write into `out` ([P3 §2.2]: output = attention
 * output + enhancement, with enhancement = alpha_layer * clip(ring_mean +
 * 0.5*field + 0.5*semantic, -eps, eps) and the attention output x = O_near +
 * alpha_far*S [P1 §2.1 eq. O]).  Set per handle by sfa_set_output_mode. */
typedef enum sfa_out_mode {
  SFA_OUT_F32 = 0,      /* out fp32 = x + enhancement (default)                       */
  SFA_OUT_BF16 = 1,     /* out bf16 = x + enhancement, rounded to nearest              */
  SFA_OUT_ADD_F32 = 2,  /* out fp32 += enhancement: out holds the caller's attention
                           output on entry ([P2] compute_enhancement(layer, attn_output)) */
  SFA_OUT_ADD_BF16 = 3  /* out bf16 += enhancement, rounded to nearest                 */
} sfa_out_mode;

/* Operator configuration.  Field names follow the pages' SFA_Config. */
typedef struct sfa_config {
  int n_layers;        /* L >= 1                                            */
  int n_q_heads;       /* query heads; hidden = n_q_heads*head_dim <= 8192  */
  int n_kv_heads;      /* KV heads, divides n_q_heads (GQA)                  */
  int head_dim;        /* 64 or 128                                          */
  int window_k;        /* near window k, 1..256            [P1 §2.1, §2.2]   */
  float gamma_far;     /* far-field EWMA decay, [0, 1]     [P1 eq. S_t]      */
  float alpha_far;     /* far-field mixing coefficient     [P1 eq. O]        */
  int ring_size;       /* must be 16                       [P3 §2.1 ch. 1]   */
  float ema_gamma;     /* EMA field decay (0.98)           [P3 §2.1 ch. 2]   */
  int n_slots;         /* must be 64                       [P3 §2.1 ch. 3]   */
  float temperature;   /* pool temperature (0.07), > 0, 1/T finite [P3 §2.1] */
  float clip_eps;      /* enhancement clip ε (0.5), >= 0   [P3 §2.2]         */
  float alpha_base;    /* base strength (0.1)              [P3 §2.2]         */
  float cross_decay;   /* per-layer decay (0.8)            [P3 §2.2]         */
  int in_dtype;        /* sfa_dtype of q, k, v; state and out are fp32       */
  const float* slots;  /* DEVICE [L][n_slots][hidden] fp32 semantic slots;
                          copied by sfa_init, may be freed afterwards        */
} sfa_config;

typedef struct sfa_handle sfa_handle;

/* Byte layout of a state buffer (host-side arithmetic only).
 * The buffer is a 256-byte header followed by L*batch stream blocks of
 * stream_stride bytes, stream (layer l, sequence b) at index l*batch + b.
 * Offsets below are relative to the start of a stream block. */
typedef struct sfa_state_layout {
  size_t header_bytes;   /* 256                                            */
  size_t stream_stride;  /* bytes per (layer, sequence) stream, 256-aligned */
  size_t total_bytes;    /* header + L*batch*stream_stride                 */
  size_t off_pos;        /* int64 position (tokens folded in)              */
  size_t off_win_k;      /* [window_k][n_kv][d] in_dtype, slot = pos mod k */
  size_t off_win_v;      /* same                                           */
  size_t off_far;        /* S [n_kv][d] fp32                               */
  size_t off_field;      /* EMA field [hidden] fp32                        */
  size_t off_ring_sum;   /* sum of the ring slots [hidden] fp32            */
  size_t off_ring;       /* ring [16][hidden] fp32, slot = pos mod 16      */
} sfa_state_layout;

/* Fills `cfg` with the pages' defaults ([P2 SFA_Config] usage example:
 * alpha_base 0.1, cross_decay 0.8, ema_gamma 0.98, ring_size 16, 64 slots,
 * clip 0.5; [P3 §2.1] temperature 0.07; [P1 §2.2] k = 16) plus
 * gamma_far 0.9, alpha_far 0.1, bf16 inputs.  Shape fields are zeroed and
 * slots is NULL.  No CUDA call. */
SFA_API void sfa_config_default(sfa_config* cfg);

/* Validates a configuration without touching the GPU: SFA_OK,
 * SFA_ERR_INVALID_ARG (null, non-positive sizes, non-finite or out-of-range
 * scalars, n_q % n_kv != 0) or SFA_ERR_UNSUPPORTED (head_dim not 64/128,
 * window_k > 256, ring_size != 16, n_slots != 64, hidden > 8192, or no
 * divisor cs <= 16 of n_q_heads with (n_q_heads / cs) * head_dim <= 512:
 * the decode kernel splits the hidden vector over a cluster of cs CTAs).
 * The slots pointer is checked for NULL and alignment only. */
SFA_API int sfa_config_validate(const sfa_config* cfg);

/* State layout for `batch` sequences of `cfg` (host arithmetic, no CUDA). */
SFA_API int sfa_state_layout_for(const sfa_config* cfg, int batch, sfa_state_layout* out);

/* [P2] engine init(n_layers, hidden): the operator's constants for one model.
 * Creates a handle on the current device: validates cfg, copies the slots,
 * precomputes slot norms and the alpha_layer table, allocates the device
 * error word.  *out receives the handle, or NULL on error.  Returns the
 * status of sfa_config_validate for a bad configuration, SFA_ERR_UNSUPPORTED
 * when a kernel's shared-memory plan does not fit the current device, and
 * SFA_ERR_CUDA when a CUDA call fails (no device, out of memory). */
SFA_API int sfa_init(const sfa_config* cfg, sfa_handle** out);

/* [P2] engine lifetime: the counterpart of sfa_init.
 * Frees the handle's device memory (synchronises the device first). */
SFA_API int sfa_destroy(sfa_handle* h);

/* [P1 §2.2] O(k·d) state: its size depends on the window, the heads and
 * the hidden size, never on the context length.
 * Bytes of a state buffer for `batch` sequences; 0 on invalid input. */
SFA_API size_t sfa_state_bytes(const sfa_handle* h, int batch);

/* Bytes of prefill workspace for a call of n tokens x `batch`; 0 on invalid
 * input or a call beyond sfa_prefill's limits (below).  The workspace holds
 * each stream's position at the start of the call, the far-field state at its
 * end, and per 64-token tile and stream the pool weights (16 KB) and the
 * far-field state at the tile's start (n_kv x d fp32); its content need not
 * be initialised. */
SFA_API size_t sfa_prefill_workspace_bytes(const sfa_handle* h, int batch, long long n);

/* [P1 §2.2] state of the window, the far field and [P3 §2.1] the ring,
 * field and position, all back to their empty values.
 * Zeroes `state` (state_bytes(h, batch) bytes) and writes its header for
 * this handle and batch: every stream back to position 0. */
SFA_API int sfa_state_reset(const sfa_handle* h, void* state, int batch, void* stream);

/* [P1 §2.1] near field (eq. O_near), far field (eq. S_t) and their sum
 * (eq. O); [P3 §2.1] ring, field and semantic pool; [P3 §2.2] fusion, clip
 * and alpha_layer, for n consecutive tokens of every sequence.
 * Folds n >= 0 tokens per sequence into the state and writes their outputs.
 * Equivalent to n calls of sfa_decode_step (same results within rounding).
 * Continues from each stream's current position.  n == 0 enqueues nothing.
 * SFA_ERR_UNSUPPORTED when layers x batch exceeds 65535, n exceeds
 * 64 x (2^31 - 1), or layers x batch x n exceeds 2^31 - 1 with bf16 inputs
 * and k <= 16 (the tensor copies use 32-bit row coordinates; split the
 * call).
 * workspace: sfa_prefill_workspace_bytes(h, batch, n) bytes (may be NULL
 * when n == 0); workspace_bytes is its size, checked.
 * Before any launch: SFA_ERR_INVALID_ARG (bad handle, n < 0, batch <= 0, a
 * NULL tensor), SFA_ERR_ALIGNMENT, SFA_ERR_WORKSPACE, SFA_ERR_UNSUPPORTED.
 * A state whose header does not match the handle or batch is left untouched
 * and latched as SFA_ERR_STATE_MISMATCH for sfa_check_device_status. */
SFA_API int sfa_prefill(const sfa_handle* h, const void* q, const void* k, const void* v,
                long long n, int batch, void* state, void* out, void* workspace,
                size_t workspace_bytes, void* stream);

/* [P1 §2.1] and [P3 §2.1–2.2] for one token of every sequence: the
 * per-step form of [P2]'s compute_enhancement(layer, attn_output), over all
 * layers at once.
 * Folds one token per sequence into the state and writes its output.
 * One launch covers all layers and sequences (for 64 or more sequences a
 * near-field kernel, then a pool kernel); no workspace.
 * The first kernel may start while the previous kernel on the stream is
 * still running (programmatic dependent launch): it fetches the handle's
 * constants at once, and the state, q, k and v only once that kernel has
 * finished, so inputs produced by the kernel just before are safe.  See
 * sfa_set_decode_input_prefetch for fetching q, k and v earlier.
 * Before any launch: SFA_ERR_INVALID_ARG (bad handle, batch <= 0, a NULL
 * tensor), SFA_ERR_ALIGNMENT, SFA_ERR_UNSUPPORTED (batch > 65535).  A state
 * whose header does not match is left untouched and latched as
 * SFA_ERR_STATE_MISMATCH, as for sfa_prefill. */
SFA_API int sfa_decode_step(const sfa_handle* h, const void* q, const void* k, const void* v,
                    int batch, void* state, void* out, void* stream);

/* Serving variants.  The pages call the enhancement once per layer from
 * inside the model's attention ([P2] usage example and llama.cpp
 * integration: one call per layer with that layer's attention output); a
 * serving loop also drops finished sequences from a decode step.  These
 * calls serve a range of layers and, for decode, a list of sequences; the
 * arithmetic is exactly that of the full calls.
 *
 * Bytes of prefill workspace for a sfa_prefill_layers call of layer_count
 * layers; 0 on invalid input (layer_count outside 1 .. n_layers) or a call
 * beyond sfa_prefill's limits. */
SFA_API size_t sfa_prefill_layers_workspace_bytes(const sfa_handle* h, int layer_count, int batch,
                                                  long long n);

/* sfa_prefill for layers layer_begin .. layer_begin + layer_count - 1 of the
 * state only.  q, k, v and out hold those layers alone, [layer_count][batch]
 * [n][...] in the layouts of sfa_prefill; workspace:
 * sfa_prefill_layers_workspace_bytes(h, layer_count, batch, n).  Other layers'
 * streams are untouched.  SFA_ERR_INVALID_ARG for a range outside 0 .. L-1. */
SFA_API int sfa_prefill_layers(const sfa_handle* h, int layer_begin, int layer_count,
                               const void* q, const void* k, const void* v, long long n, int batch,
                               void* state, void* out, void* workspace, size_t workspace_bytes,
                               void* stream);

/* sfa_decode_step for layers layer_begin .. layer_begin + layer_count - 1 and
 * n_seq sequences of the batch.  seq_ids: NULL (then n_seq must equal batch
 * and row i is sequence i) or a DEVICE array of n_seq DISTINCT sequence
 * indices in [0, batch) (row i is sequence seq_ids[i]; duplicates race on
 * that sequence's state).  q [layer_count][n_seq][n_q][d], k and v
 * [layer_count][n_seq][n_kv][d], out [layer_count][n_seq][hidden] fp32.
 * Sequences not listed keep their state and position.  An index out of range
 * is skipped on the device and latched as SFA_ERR_INVALID_ARG for
 * sfa_check_device_status; host-visible errors, and the input prefetch
 * option, as for sfa_decode_step. */
SFA_API int sfa_decode_step_ex(const sfa_handle* h, int layer_begin, int layer_count,
                               const int* seq_ids, int n_seq, const void* q, const void* k,
                               const void* v, int batch, void* state, void* out, void* stream);

/* Decode input prefetch (default off).  enable = 1 declares that, for every
 * later decode call on this handle, q, k and v are complete when the call is
 * enqueued and nothing that may still be running on the stream writes them:
 * for example inputs written before a synchronisation, copied in by
 * cudaMemcpyAsync, or written by a kernel on another stream that the call's
 * stream waits for through an event.  The per-sequence decode kernel then
 * fetches them before the previous kernel on the stream has finished, which
 * takes one memory round trip off each call.  With enable = 1, inputs
 * written by a kernel still running on the stream (a projection launched
 * just before the call, or an earlier SFA call's out) may be read before
 * they are written.  enable = 0 restores the default.  SFA_ERR_INVALID_ARG
 * for another value.  Results are identical either way. */
SFA_API int sfa_set_decode_input_prefetch(sfa_handle* h, int enable);

/* Output mode of later compute calls on this handle (sfa_out_mode; default
 * SFA_OUT_F32).  In the bf16 modes `out` points at bf16 elements; in the
 * add modes the calls read out (the caller's attention output, in the
 * mode's dtype) and add the enhancement to it in place.  Outside
 * SFA_OUT_F32 the prefill keeps x in its workspace instead of in out, so
 * sfa_prefill_workspace_bytes grows by layers x batch x n x hidden x 4
 * bytes, and decode calls of many sequences run the per-sequence kernel.
 * SFA_ERR_INVALID_ARG for another value. */
SFA_API int sfa_set_output_mode(sfa_handle* h, int mode);

/* Synchronises `stream`, then returns and clears the first error latched on
 * the device since the last check (SFA_OK if none), or SFA_ERR_CUDA if the
 * stream reports a CUDA error. */
SFA_API int sfa_check_device_status(const sfa_handle* h, void* stream);

/* Static description of a status code. */
SFA_API const char* sfa_status_string(int status);

/* ABI version of the loaded library (SFA_ABI_VERSION it was built with). */
SFA_API int sfa_abi_version(void);

/* Ragged prefill.  A serving engine's batch holds prompts of different
 * lengths, and [P2]'s engine is called per layer with whatever tokens each
 * sequence has; this call folds lens[b] tokens into sequence b (0 <= lens[b]
 * <= n_max), every sequence from its own position, with the arithmetic of
 * sfa_prefill.  q, k, v and out keep the layouts of sfa_prefill with n =
 * n_max: sequence b's tokens are its rows 0 .. lens[b]-1; the rows past
 * lens[b] take no part in any result, and out keeps what it held there.
 * lens: DEVICE array of `batch` int32, read by the kernels, so an earlier
 * kernel on the stream may write it.  workspace:
 * sfa_prefill_workspace_bytes(h, batch, n_max) bytes.  A count outside
 * 0 .. n_max leaves that sequence's state and output untouched and is
 * latched as SFA_ERR_INVALID_ARG for sfa_check_device_status; lens == NULL
 * is SFA_ERR_INVALID_ARG.  Otherwise the returns of sfa_prefill; n_max == 0
 * enqueues nothing. */
SFA_API int sfa_prefill_ragged(const sfa_handle* h, const void* q, const void* k, const void* v,
                               long long n_max, const int* lens, int batch, void* state, void* out,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the fixed device scratch behind sfa_prefill_static_ws. */
#define SFA_STATIC_WORKSPACE_BYTES (16u << 20)

/* sfa_prefill without a caller-provided workspace, for callers that cannot
 * allocate: an operator hook inside another engine that receives only its
 * input/output tensors and no allocator, or a serving loop that forbids
 * cudaMalloc in steady state because it can synchronise the device.  (The
 * pages have no counterpart: this is a deployment variant of sfa_prefill.)
 * The cross-tile scratch is one file-scope device array of
 * SFA_STATIC_WORKSPACE_BYTES that every GPU loading the library holds until
 * the process exits; nothing is allocated or freed.  The first call on a
 * device looks up the array's device address (with that device current)
 * and caches it; the runtime reserves the array on the device at that
 * point (device arrays of the library are loaded lazily), so the first call
 * may allocate and synchronise once: make it before any stream capture and
 * outside any region that must not allocate.  Every
 * call on a device shares the array, which keeps the last call's contents
 * (nothing in it has to start at zero), and calls that overlap on the GPU
 * (other streams, other host threads) race on it.  Returns SFA_ERR_WORKSPACE when
 * sfa_prefill_workspace_bytes(h, batch, n) exceeds the array (split the
 * prefill into smaller chunks), otherwise exactly what sfa_prefill returns;
 * results equal sfa_prefill's. */
SFA_API int sfa_prefill_static_ws(const sfa_handle* h, const void* q, const void* k, const void* v,
                                  long long n, int batch, void* state, void* out, void* stream);

/* Test hook for the device-side bounded waits of sfa_prefill (not needed in
 * normal use).  withhold_tile: tile index (tile * streams + stream, streams =
 * layers x batch of the call) whose pool-weight CTA waits on a barrier that
 * nothing completes (-1 disables); spin_limit: polls before that wait gives
 * up and latches SFA_ERR_DEVICE_TIMEOUT (0 restores the default).  The
 * kernel still finishes and the context stays usable.  Affects later calls
 * on this handle only. */
SFA_API int sfa_debug_set_wait_limit(sfa_handle* h, unsigned int spin_limit, long long withhold_tile);

/* Test hook that pins the kernel variants, so that every variant can be
 * checked on one workload (not needed in normal use; results agree within
 * the operator's tolerance whichever runs).  decode_tile: -1 chooses the
 * decode kernel by the number of sequences per call (the default), 0 always
 * the per-sequence kernel, 1 always the batch-tiled kernel.
 * prefill_near: where the tensor cores apply to the prefill near field
 * (bf16 inputs, k <= 16), 3 chooses by call size (the default: 2 for calls
 * of at least four 64-token tiles per SM, else 1), 2 runs it fused with the
 * pool scores in one kernel, 1 on the tensor cores followed by a separate
 * pool kernel, 0 on the CUDA cores.  SFA_ERR_INVALID_ARG for other values,
 * SFA_ERR_UNSUPPORTED if the requested kernel does not fit this
 * configuration (nothing changes then).  Affects later calls on this handle
 * only. */
SFA_API int sfa_debug_set_paths(sfa_handle* h, int decode_tile, int prefill_near);

#ifdef __cplusplus
}
#endif
#endif /* SFA_H */
