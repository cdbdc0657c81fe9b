/*
 * fi.h -- exact online causal long convolution for stacks of long-convolution
 * (LCSM, Hyena-style) mixer layers, with the relaxed block schedule of
 * "Flash Inference: Near Linear Time Inference for Long Convolution Sequence
 * Models and Beyond" (Oncescu, Purandare, Idreos, Kakade; arXiv 2410.12982),
 * built for NVIDIA B200 (sm_100a).
 *
 * What is computed (summary page, "Definizione del Compito" and "Architettura
 * del Modello"): for layers l = 1..M, channels d, sequences b and positions t,
 *
 *     y^l_t[b][d] = sum_{s <= t} h^l[d][t-s] * a^{l-1}_s[b][d]      (the mixer)
 *     a^l_t       = R(tanh(y^l_t))                                 (the block)
 *     a^0_t       = x_t                                            (the tokens)
 *
 * with R the identity (FI_F32) or round-to-nearest-even to bfloat16 (FI_BF16).
 * Each position is computed once every earlier position is known ("online"):
 * at step i the library adds the contribution of inputs [i-U, i) to outputs
 * [i, i+U), U = largest power of two dividing i (Algorithm 1 / 2 on the page),
 * for all layers at once (Algorithm 3), then finishes position i with the
 * h[0] term ("red cell") and the block, layer after layer.
 *
 * Conventions shared by every call:
 *   - All pointers named in a call are DEVICE pointers unless the name ends in
 *     "_host". Token-shaped buffers are row-major [B][D] (or [n][B][D]).
 *   - fp32 buffers are 4-byte aligned, bf16 buffers 2-byte aligned.
 *   - Every call is asynchronous on the context's CUDA stream (the stream given
 *     to fi_init or fi_set_stream); buffers passed in must stay valid until the
 *     stream reaches that point. Only fi_init, fi_destroy, fi_sync, the *_host
 *     call and fi_profile_read synchronise.
 *   - Errors are returned as fi_status; no exception crosses this boundary.
 *     fi_last_error() gives a message for the last failing call on this thread.
 *     After FI_E_CUDA the context should be destroyed.
 *   - A context is not thread-safe; use one per host thread.
 */
#ifndef FI_H
#define FI_H

#include <stdint.h>

#if defined(__GNUC__)
#define FI_API __attribute__((visibility("default")))
#else
#define FI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FI_OK = 0,
  FI_E_INVALID = 1,     /* bad argument: null pointer, size out of range, L not a power of two */
  FI_E_OOM = 2,         /* a device or pinned-host allocation failed */
  FI_E_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  FI_E_STATE = 4,       /* not allowed in the current state (e.g. stepping past max_len) */
  FI_E_TIMEOUT = 5,     /* a bounded device-side wait gave up (reported by fi_sync and the calls that synchronise) */
  FI_E_UNSUPPORTED = 6  /* valid request outside what the library implements */
} fi_status;

typedef enum { FI_F32 = 0, FI_BF16 = 1 } fi_dtype;

typedef struct {
  int32_t layers;    /* M >= 1 */
  int32_t channels;  /* D >= 1 */
  int32_t max_len;   /* L, a power of two, 2 <= L <= 2^17 */
  int32_t batch;     /* B >= 1 (independent sequences sharing the filters) */
  int32_t dtype;     /* fi_dtype of filters and tokens; accumulation is always fp32 */
  int32_t chunk;     /* 0 = automatic; else block sides below this run on chip (power of two, 2..64) */
  int32_t fft_from;  /* 0 = automatic; else the smallest block side computed by FFT (power of two >= 64) */
  int32_t tc_max;    /* 0 = automatic (bf16 with batch >= 32: sides 64..256, 64..512 from batch 64;
                        otherwise none), -1 = never;
                        else block sides 64..tc_max (power of two >= 64) run on the tensor cores as
                        Toeplitz products (bf16 contexts: exact bf16 products; fp32 contexts: three
                        bf16 products of split operands), ahead of FFT */
  int32_t reserved[4]; /* must be 0 */
} fi_config;

typedef struct fi_ctx fi_ctx;

/* Create a context.
 * h: filters, device, [M][D][L] of cfg->dtype (h^l[d][t] at ((l*D)+d)*L+t).
 *    The library copies them (widened to fp32) and precomputes, for every block
 *    side U >= fft_from, the spectrum of h[0..2U) (page: "Precomputazione FFT"),
 *    so the caller may free h once fi_init returns.
 * stream: a cudaStream_t (NULL = legacy default stream).
 * Allocates the state (fp32, (M+1)*B*D*L values), filters and spectra on the
 * current device. On error *out is NULL and nothing is leaked.
 * Errors: FI_E_INVALID (null, sizes, reserved != 0), FI_E_UNSUPPORTED (sizes this
 * build cannot schedule), FI_E_OOM, FI_E_CUDA. */
FI_API fi_status fi_init(fi_ctx** out, const fi_config* cfg, const void* h, void* stream);

/* One position (Algorithm 2, one iteration): with t = current position,
 * add the step-t block (U = lowbit(t)) into every layer's accumulators, then run
 * the red cell and block through the M layers.
 * x_t: device [B][D] of cfg->dtype, the token at position t.
 * y_t: device [B][D] fp32, receives y^M_t (last layer's mixer output, before tanh).
 * Errors: FI_E_INVALID (null), FI_E_STATE (position == max_len). */
FI_API fi_status fi_step(fi_ctx* ctx, const void* x_t, float* y_t);

/* Closed-loop generation of n positions from the current position p on device:
 * x_p = x0, and for t >= p: x_{t+1} = R(tanh(y^M_t) + eps_scale * eps[t-p]).
 * The page states the autoregressive loop (Algorithm 2: red cells and blocks
 * per layer, then the sampler) but has no call that runs many positions at
 * once: this one runs that loop on the device so that no host round trip sits
 * between positions. The sampler rule is the workloads' (tanh of the last
 * layer's output plus scaled noise; the page's synthetic sampler "adds noise",
 * "Configurazione Sperimentale").
 * x0:    device [B][D] of cfg->dtype; or NULL when p > 0, to continue with the
 *        token the sampler produced at the end of the previous call.
 * eps:   device [n][B][D] fp32 sampler noise.
 * y_out: device [n][B][D] fp32, receives y^M_t for t = p..p+n-1.
 * rec:   NULL, or device [M][n][B][D] fp32 that receives y^l_t for every layer
 *        (test and inspection hook; costs one extra write per layer and position).
 * Leaves the context at position p+n with the same state fi_step would leave.
 * Errors: FI_E_INVALID (null, x0 NULL at p = 0, n < 0), FI_E_STATE (p + n > max_len). */
FI_API fi_status fi_generate(fi_ctx* ctx, int32_t n, const void* x0, const float* eps,
                      float eps_scale, float* y_out, float* rec);

/* Prompt prefill (page, "Limitazioni" 4, Fase di Prompt: with a long prompt the
 * prefill dominates, and every prompt position is known at once). Starts a
 * sequence from position 0 with the p prompt tokens x[p][B][D] (device, of
 * cfg->dtype) and computes, layer by layer, the offline causal convolution of
 * the whole prompt by one FFT per (layer, sequence, channel) with the filter's
 * spectrum zero-padded to twice the transform, then the block. It leaves the
 * context at position p with the state p calls of fi_step would leave (the
 * blocks of steps below p whose targets reach past the prompt are added for
 * their targets >= p), so fi_generate (with the token at p as x0) or fi_step
 * continue from there.
 * y_out: NULL or device [p][B][D] fp32, receives y^M_t for t < p.
 * rec:   NULL or device [M][p][B][D] fp32, receives y^l_t for every layer.
 * Allocates scratch for the padded spectra (M*D*(2^ceil(log2 p)+1) complex) on
 * first use and keeps it.
 * Errors: FI_E_INVALID (NULL, p out of [1, max_len]), FI_E_STATE (position != 0),
 * FI_E_UNSUPPORTED (p > 16384), FI_E_OOM. */
FI_API fi_status fi_prefill(fi_ctx* ctx, int32_t p, const void* x, float* y_out, float* rec);

/* fi_generate with HOST buffers: copies x0_host and eps_host to the device,
 * generates, copies y^M back to y_out_host, and returns when the copy is done.
 * The work runs in segments of whole chunks (about 16 per call, none shorter
 * than 256 positions): the noise of later segments uploads and the outputs of
 * earlier ones download on two streams of the context's own while a segment
 * generates, so with pinned host buffers the copies overlap the generation.
 * The results equal those of one fi_generate call. Host buffers may be
 * pageable (no overlap) or pinned. Staging device buffers are allocated on
 * first use and kept by the context. */
FI_API fi_status fi_generate_host(fi_ctx* ctx, int32_t n, const void* x0_host, const float* eps_host,
                           float eps_scale, float* y_out_host);

/* The same closed-loop generation by the Lazy method of the page ("Tre Strategie
 * di Calcolo": every y^l_t summed in full when needed, O(L^2) in total), with
 * all layers' sums for a position in one launch (the page's parallel Lazy).
 * Arguments and state effects as fi_generate (rec not offered). This is the
 * quadratic baseline the relaxed schedule is measured against. */
FI_API fi_status fi_generate_lazy(fi_ctx* ctx, int32_t n, const void* x0, const float* eps,
                           float eps_scale, float* y_out);

/* Wait until every call issued on the context's stream has finished. Returns
 * FI_E_TIMEOUT if a bounded device-side wait inside a kernel gave up since the
 * last check (the results of those calls are then invalid; the flag is cleared).
 * The kernels' internal waits are all bounded, so no call can hang the GPU. */
FI_API fi_status fi_sync(fi_ctx* ctx);

/* Rewind to position 0. O(1): no memory is cleared, because every accumulator
 * is first written (not added to) by the block that first reaches it.
 * Not on the page (which runs one generation per model call); the filters and
 * their precomputed spectra ("Precomputazione FFT") are kept. */
FI_API fi_status fi_reset(fi_ctx* ctx);

/* Channel-mixing block (summary page, "Architettura del Modello": block^l maps
 * R^D to R^D and includes an MLP; "Configurazione Sperimentale": in the
 * synthetic setting the blocks are MLP + GELU and the sampler adds noise).
 * Replaces the elementwise tanh after every layer by
 *   a^l_t = R(W2^l GELU(W1^l y^l_t + b1^l) + b2^l)   per sequence, across channels,
 * GELU(u) = u Phi(u) (exact, erf form), R = bf16 rounding in bf16 contexts; the
 * sampler becomes x_{t+1} = R(a^M_t + eps_scale eps_t). fi_step and fi_generate
 * then run position by position (every layer's block needs all channels of the
 * layer below), blocks of the schedule as before; fi_generate replays the
 * layers of a position as one CUDA graph, captured on the first call of more
 * than one position after this one. Synchronises the context's stream.
 * hidden: Dh >= 1, or 0 to return to the tanh block (weights may be NULL).
 * w1 [M][Dh][D], b1 [M][Dh], w2 [M][D][Dh], b2 [M][D]: fp32, device pointers,
 * copied (the caller may free them after the call's stream work completes).
 * Errors: FI_E_INVALID (NULL weight, hidden < 0), FI_E_STATE (position != 0:
 * call fi_reset first), FI_E_UNSUPPORTED (min(B, 8) x D or min(B, 8) x Dh
 * floats beyond one CTA's shared memory), FI_E_OOM, FI_E_CUDA. fi_prefill and fi_generate_lazy return
 * FI_E_UNSUPPORTED while the block is set. */
FI_API fi_status fi_set_mlp_block(fi_ctx* ctx, int32_t hidden, const float* w1, const float* b1, const float* w2,
                                  const float* b2);

/* Current position (number of positions already produced). */
FI_API fi_status fi_position(const fi_ctx* ctx, int32_t* pos);

/* Copy the recorded activations a^layer_t for t < position into dst,
 * device [position][B][D] fp32; layer in [0, M-1] (layer 0 = the tokens).
 * These are the a^l_i the page keeps for every position ("Ottimizzazione della
 * Memoria": the slot of a^l_i also holds b^l_i until it is consumed); reading
 * them is a test hook, not on the page. */
FI_API fi_status fi_read_activations(fi_ctx* ctx, int32_t layer, float* dst);

/* Change the stream later calls run on. */
FI_API fi_status fi_set_stream(fi_ctx* ctx, void* stream);

/* The plan the context chose (after automatic selection): block sides below
 * *chunk run on chip, sides 64..*tc_max on the tensor cores (0: none), sides
 * from *fft_from up by FFT (0: none), any other side directly from HBM.
 * Each pointer may be NULL. */
FI_API fi_status fi_get_plan(const fi_ctx* ctx, int32_t* chunk, int32_t* fft_from, int32_t* tc_max);

/* Kernel timing. With profiling on, every kernel launch of fi_generate is
 * bracketed by CUDA events on the context's stream; fi_profile_read
 * synchronises and returns, per kernel class, the count of kernels launched
 * and the summed device time in milliseconds since the last read (a replayed
 * graph is one bracket and counts its kernels). Classes: 0 = on-chip chunk
 * (small blocks + red cells), 1 = direct blocks from HBM, 2 = FFT blocks,
 * 3 = per-position red cells (fi_step / lazy), 4 = lazy sums, 5 = tensor-core
 * blocks. */
#define FI_NUM_KERNEL_CLASSES 6
FI_API fi_status fi_profile(fi_ctx* ctx, int32_t enable);
FI_API fi_status fi_profile_read(fi_ctx* ctx, int32_t counts[FI_NUM_KERNEL_CLASSES],
                          double ms[FI_NUM_KERNEL_CLASSES]);
/* fi_profile_read, plus the block launches (direct, FFT, tensor-core) split by
 * block side: side_counts[q] and side_ms[q] for side 2^q (either may be NULL). */
FI_API fi_status fi_profile_read_sides(fi_ctx* ctx, int32_t counts[FI_NUM_KERNEL_CLASSES],
                                       double ms[FI_NUM_KERNEL_CLASSES], int32_t side_counts[32],
                                       double side_ms[32]);

/* Release everything the context owns (synchronises its stream first). NULL is allowed. */
FI_API fi_status fi_destroy(fi_ctx* ctx);

FI_API const char* fi_status_str(fi_status s);
FI_API const char* fi_last_error(void);

/* One closed-loop generation from position 0 that allocates no device memory.
 * For callers that cannot call cudaMalloc: code on a thread with a hard latency
 * budget (an allocation can block in the driver), code inside a host framework
 * whose device memory belongs to its own allocator, or code running where
 * allocation is not permitted. The paper has no counterpart to this call.
 * Computes what fi_init(cfg, h) followed by fi_generate(n, x0, eps, eps_scale,
 * y_out, NULL) would, with every block of side >= the on-chip chunk summed
 * directly (no filter spectra). Arguments as for those two calls; cfg->fft_from
 * is ignored; returns once the generation has finished on `stream`.
 * Working memory is one file-scope device array of 8 Mi floats (32 MiB) that
 * every GPU loading the library keeps until the process exits; the call needs
 * M*D*L + (M+1)*B*D*L + 64 floats of it (rounded up to 64 per part) and
 * returns FI_E_INVALID, with the sizes in fi_last_error(), when that is more.
 * All calls share the array and it keeps the last call's contents (each call
 * rewrites what it reads); calls whose work overlaps on the GPU race on it.
 * The first call on a device, with that device current, looks up the array's
 * device address and keeps it for the life of the process: make that first call
 * before any stream capture, and do not call this entry point again after a
 * cudaDeviceReset of that device (the kept address would no longer be valid).
 * Errors: FI_E_INVALID (NULL, sizes, L > 2^15), FI_E_CUDA, FI_E_TIMEOUT. */
FI_API fi_status fi_generate_noalloc(const fi_config* cfg, const void* h, int32_t n, const void* x0,
                                     const float* eps, float eps_scale, float* y_out, void* stream);

/* Test hook: the number of barrier checks after which a device-side wait in
 * later fi_generate calls gives up (negative restores the default, about a
 * second of waiting). 0 makes every wait that is not already satisfied give up
 * at once, which exercises the FI_E_TIMEOUT path of fi_sync without any wait. */
FI_API fi_status fi_debug_set_wait_limit(fi_ctx* ctx, int32_t limit);

/* Test hook (host only, no device work): the table of on-chip block pieces the
 * chunk kernel runs for a chunk of `chunk` positions (a power of two, 2..64):
 * retimed != 0 gives the table of a launch that covers a whole chunk (the chain
 * adds the terms of the first *chain_lags lags itself; the page's tiling of the
 * other pairs is shifted that many positions later, and its blocks are cut into
 * pieces spread over steps; retimed == 2: the coarser cut used for stacks of at
 * most 8 layers), 0 the page's tiling (the block of step r, side lowbit(r), at
 * step r; *chain_lags = 0). Writes up to `cap` entries of 5 int32
 * (step, first source, sources, first target, targets; positions relative to
 * the chunk start) to out, the entry count to *count, the lags to *chain_lags
 * (may be NULL).
 * Errors: FI_E_INVALID (NULL, chunk). */
FI_API fi_status fi_debug_chunk_schedule(int32_t chunk, int32_t retimed, int32_t* out, int32_t cap,
                                         int32_t* count, int32_t* chain_lags);

/* Test hook: run the library's device FFT (the one its FFT blocks use) on
 * `count` complex sequences of length 2^log2n (6 <= log2n <= 14), interleaved
 * (re, im) fp32, device buffers in[count][2^log2n][2] -> out (may alias in).
 * Forward is exp(-2 pi i k n / N), inverse exp(+...), both unnormalised.
 * Synchronous. */
FI_API fi_status fi_debug_fft(int32_t log2n, int32_t count, const float* in, float* out,
                       int32_t inverse, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FI_H */
