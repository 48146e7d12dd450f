/*
 * gdpa.h - C ABI of the B200 (sm_100a) GDPA library, libgdpa.so.
 *
 * GDPA (Generalized Dot-Product Attention) is Kunlun's Personalized FFN
 * recast as a multi-head attention operator.  The Kunlun technical summary
 * (gist.science/es/paper/2602.10016, section 2.2 "Optimizaciones de Modulos
 * de Bajo Nivel", GDPA bullet) states that the sequence tokens act as the
 * queries, that weights derived from the non-sequential context act as the
 * keys and values, and that the transformation is fused into one
 * FlashAttention-like kernel instead of separate memory-bound matmuls.  The
 * RecSysChannel review ("Kunlun: Establishing Scaling Laws for Massive-Scale
 * Recommendation Systems [2/2]", items 1 and 2) adds that K and V are
 * obtained from the context features and the event sequence is turned into
 * Q.  Neither page prints the formula; this library computes, for every
 * sample b and head j (token rows t in [offsets[b], offsets[b+1])):
 *
 *     S = scale * Q_bj K_bj^T,    P = phi(S),    O_bj = P V_bj
 *
 * with phi = identity, SiLU (x * logistic(x)), a row softmax, ReLU or GELU
 * (the PFFN variants' other activations), and its gradient.  Heads and
 * samples are independent; there is no normalisation for the elementwise phi,
 * no bias and no head mixing.
 *
 * Layouts (row-major, contiguous, every base pointer 16-byte aligned):
 *   q, o, dout, dq : [T, h, dh]      jagged tokens, T = offsets[B]
 *   k, v, dk, dv   : [B, h, m, dh]   one context key/value set per sample, head
 *   offsets        : int32 [B + 1]   device memory, offsets[0] = 0,
 *                                     non-decreasing, offsets[B] = T
 *   lse            : fp32 [h, T]     natural-log row log-sum-exp (softmax)
 * Element type of q, k, v, o, dout, dq, dk, dv: fp32 or bf16 (problem dtype).
 *
 * Ownership: the caller allocates every buffer, including the workspace whose
 * size the *_workspace_size calls report.  The library allocates no device
 * memory and keeps only small per-device host caches (launch attributes).
 *
 * Asynchrony: gdpa_fwd and gdpa_bwd only enqueue work on `stream` (a
 * cudaStream_t passed as void*) and never synchronise.  All pointers passed to
 * them are device pointers unless stated otherwise.
 *
 * Errors: argument errors are detected on the host and returned before any
 * launch (GDPA_ERR_INVALID_ARG / GDPA_ERR_UNSUPPORTED).  A failed launch
 * returns GDPA_ERR_CUDA.  Inconsistent device offsets (decreasing, a length
 * above max_n, offsets[B] != T) and bounded-wait time-outs inside a kernel are
 * detected on the device: the kernels then skip the bad work, and the code is
 * left in the workspace's status word, which gdpa_workspace_status() reads.
 */
#ifndef GDPA_H_
#define GDPA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDPA_API __attribute__((visibility("default")))
#else
#define GDPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* phi applied to the scaled logits x = s * q.k: identity, SiLU x*logistic(x),
 * row softmax, and the PFFN variants' other activations ReLU max(x, 0) and
 * GELU in its exact form x * Phi(x) (Phi the standard normal CDF). */
typedef enum {
  GDPA_PHI_IDENTITY = 0,
  GDPA_PHI_SILU = 1,
  GDPA_PHI_SOFTMAX = 2,
  GDPA_PHI_RELU = 3,
  GDPA_PHI_GELU = 4
} gdpa_phi_t;

typedef enum {
  GDPA_DTYPE_F32 = 0,   /* fp32 in / fp32 accumulate / fp32 out (SIMT kernels) */
  GDPA_DTYPE_BF16 = 1   /* bf16 in / fp32 accumulate / bf16 out (tcgen05 kernels) */
} gdpa_dtype_t;

typedef enum {
  GDPA_OK = 0,
  GDPA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad offsets */
  GDPA_ERR_UNSUPPORTED = 2,   /* valid but unsupported (e.g. dh not in {32,64,128}) */
  GDPA_ERR_CUDA = 3,          /* a CUDA runtime/driver call or a launch failed */
  GDPA_ERR_TIMEOUT = 4,       /* a bounded wait inside a kernel gave up */
  GDPA_ERR_WORKSPACE = 5      /* workspace null, misaligned or too small */
} gdpa_status_t;

/* Problem description (host memory, read during the call only). */
typedef struct {
  int32_t B;             /* samples, >= 1 */
  int32_t h;             /* heads, >= 1 */
  int32_t dh;            /* head dim: 32, 64 or 128 */
  int32_t m;             /* context keys/values per sample and head, >= 1 */
  int32_t max_n;         /* upper bound on every n_b = offsets[b+1]-offsets[b], >= 0 */
  int32_t dtype;         /* gdpa_dtype_t */
  int64_t total_tokens;  /* T = offsets[B], 0 <= T < 2^31 */
  int32_t phi;           /* gdpa_phi_t */
  float scale;           /* s in S = s Q K^T */
} gdpa_problem_t;

/* Workspace bytes gdpa_fwd needs for `p` (written to *bytes). Host only. */
GDPA_API gdpa_status_t gdpa_fwd_workspace_size(const gdpa_problem_t* p, size_t* bytes);

/* Workspace bytes gdpa_bwd needs for `p` (written to *bytes). Host only. */
GDPA_API gdpa_status_t gdpa_bwd_workspace_size(const gdpa_problem_t* p, size_t* bytes);

/*
 * Forward: o = phi(scale * q k^T) v per (sample, head).
 *   q [T,h,dh], k/v [B,h,m,dh], offsets int32 [B+1]: inputs (device).
 *   o [T,h,dh]: output (device), every valid row written.
 *   lse fp32 [h,T]: output for phi = softmax (needed by gdpa_bwd); may be NULL
 *     for softmax when no backward follows; ignored for the other phi.
 *   workspace: device, >= gdpa_fwd_workspace_size bytes, 256-byte aligned.
 *   stream: cudaStream_t (void*), may be NULL for the legacy default stream.
 */
GDPA_API gdpa_status_t gdpa_fwd(const gdpa_problem_t* p, const void* q, const int32_t* offsets,
                       const void* k, const void* v, void* o, float* lse,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward for an upstream gradient dout of o.
 *   q, k, v, offsets: as in gdpa_fwd.  o and lse: gdpa_fwd's outputs (read for
 *   phi = softmax only; may be NULL otherwise).  dout [T,h,dh]: input.
 *   dq [T,h,dh], dk/dv [B,h,m,dh]: outputs, every element written (dk, dv of a
 *   sample with no tokens are zero).
 *   workspace: device, >= gdpa_bwd_workspace_size bytes, 256-byte aligned.
 */
GDPA_API gdpa_status_t gdpa_bwd(const gdpa_problem_t* p, const void* q, const int32_t* offsets,
                       const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * The PFFN variant with biases (reading of the Kunlun summary, section 2.2,
 * GDPA bullet: GDPA is the Personalized FFN y = W2 phi(W1 x + b1) + b2 with
 * per-sample weights, recast as attention; the pages print neither the
 * formula nor the biases):
 *
 *     O_bj = phi(scale * Q_bj K_bj^T + 1 b1_bj^T) V_bj + 1 b2_bj^T
 *
 *   b1 fp32 [B, h, m]: per-sample, per-head key bias, added to every row of
 *     the scaled logits before phi (softmax: inside the exponent).
 *   b2 fp32 [B, h, dh]: per-sample, per-head output bias, added to every row
 *     of O (and not to LSE).
 *   Either may be NULL (a zero bias); with both NULL this is gdpa_fwd.  Device
 *   pointers, 4-byte aligned.  Every other argument, the workspace size and
 *   the error behaviour are those of gdpa_fwd.
 */
GDPA_API gdpa_status_t gdpa_fwd_bias(const gdpa_problem_t* p, const void* q,
                                     const int32_t* offsets, const void* k, const void* v,
                                     const float* b1, const float* b2, void* o, float* lse,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of gdpa_fwd_bias for an upstream gradient dout of o.
 *   b1, b2: the forward's biases (either may be NULL).  o: the biased
 *   forward output (read for phi = softmax, whose row sums D = rowsum(dout *
 *   (o - b2)) need it).
 *   dq, dk, dv: as gdpa_bwd.  db1 fp32 [B, h, m] = the sum over each sample's
 *   tokens of dS (the gradient of the biased logits); db2 fp32 [B, h, dh] = the
 *   sum over each sample's tokens of dout.  Either may be NULL (not computed);
 *   a sample with no tokens gets zeros.  Same workspace as gdpa_bwd.
 */
GDPA_API gdpa_status_t gdpa_bwd_bias(const gdpa_problem_t* p, const void* q,
                                     const int32_t* offsets, const void* k, const void* v,
                                     const float* b1, const float* b2, const void* o,
                                     const float* lse, const void* dout, void* dq, void* dk,
                                     void* dv, float* db1, float* db2, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * Weight Generation: each sample's GDPA keys (or values) from its context
 * vector.  The Kunlun summary (gist.science/es/paper/2602.10016, section 2.1)
 * lists Weight Generation in the Interaction Block, and the RecSysChannel
 * review ("Kunlun ... [2/2]", item 1) says that K and V are obtained from the
 * context features; neither page gives the map.  This library computes its
 * plainest reading, a learned linear map per output tensor:
 *
 *     y[b, f] = sum_c w[f, c] * ctx[b, c],   b < B, f < F,
 *
 * rounded to bf16, with y[b] viewed as [h, m, dh] (F = h * m * dh): K or V of
 * gdpa_fwd for sample b.
 *   w   fp32 [F, C] (device, 16-byte aligned), C = 32 or 64 (the backward: 64),
 *       F a multiple of 8.
 *   ctx fp32 [B, C] (device, 16-byte aligned).
 *   y   bf16 [B, F] (device, 16-byte aligned): output, every element written.
 *   status_ws: NULL, or a device buffer of >= 256 bytes, 256-byte aligned,
 *     whose status word is cleared and receives GDPA_ERR_TIMEOUT if a bounded
 *     wait inside the kernel expires (read with gdpa_workspace_status).
 * The products run on the tensor cores in tf32 (10 mantissa bits) with fp32
 * accumulation.  Returns GDPA_ERR_UNSUPPORTED for another C or F % 8 != 0,
 * GDPA_ERR_INVALID_ARG for a null or misaligned pointer; asynchronous on
 * `stream`; allocates nothing.
 */
GDPA_API gdpa_status_t gdpa_weight_gen(int32_t B, int64_t F, int32_t C, const float* w,
                                       const float* ctx, void* y, void* status_ws,
                                       void* stream);

/* Workspace bytes gdpa_weight_gen_bwd needs (written to *bytes).  Host only. */
GDPA_API gdpa_status_t gdpa_weight_gen_bwd_workspace_size(int32_t B, int64_t F, int32_t C,
                                                          size_t* bytes);

/*
 * Backward of gdpa_weight_gen for an upstream gradient dy of y:
 *     dw[f, c] = sum_b dy[b, f] * ctx[b, c],   dctx[b, c] = sum_f dy[b, f] * w[f, c].
 *   w, ctx: the forward's inputs (fp32, device, 16-byte aligned).
 *   dy bf16 [B, F]: input (e.g. the dk or dv of gdpa_bwd viewed as [B, h*m*dh]).
 *   dw fp32 [F, C], dctx fp32 [B, C]: outputs (device, 16-byte aligned), every
 *     element written.
 *   workspace: device, >= gdpa_weight_gen_bwd_workspace_size bytes, 256-byte
 *     aligned (bf16 copies of w and ctx, and the status word that a bounded-wait
 *     expiry sets to GDPA_ERR_TIMEOUT; read with gdpa_workspace_status).
 * Supported: C = 64, F a multiple of 8, B <= 896 (GDPA_ERR_UNSUPPORTED
 * otherwise).  The products run on the tensor cores with bf16 operands and
 * fp32 accumulation; dctx is reduced across CTAs in fp32 in a non-deterministic
 * order.  Asynchronous on `stream`; allocates nothing.
 */
GDPA_API gdpa_status_t gdpa_weight_gen_bwd(int32_t B, int64_t F, int32_t C, const float* w,
                                           const float* ctx, const void* dy, float* dw,
                                           float* dctx, void* workspace, size_t workspace_bytes,
                                           void* stream);

/*
 * Seed-query attention pooling, the first level of Hierarchical Seed Pooling
 * (HSP).  The Kunlun summary (section 2.2, HSP bullet) says HSP replaces the
 * random learnable queries of pooling by multi-head attention with learned
 * seed-level representations for long sequences (then compressed by
 * SumKronLinear, which is not part of this call); the RecSysChannel review
 * (item 3) places it after GDPA.  Read as attention with learned seeds: for
 * every sample b and head j,
 *
 *     O[b, j] = softmax_rows(scale * seeds[j] K_bj^T) V_bj,
 *     LSE[b, j, i] = ln sum_t exp(scale * seeds[j, i] . k_t)   (natural log),
 *
 * with K_bj, V_bj the rows t in [offsets[b], offsets[b+1]) of head j.  A
 * sample without tokens gets O = 0 and LSE = -inf.
 *   seeds bf16 [h, S, dh], k and v bf16 [T, h, dh], offsets int32 [B+1]
 *   (device, as in gdpa_fwd), o bf16 [B, h, S, dh] (output, every element
 *   written), lse fp32 [B, h, S] (output; may be NULL).  Base pointers 16-byte
 *   aligned (lse and offsets 4-byte).
 *   Supported: dh = 32 or 64, 1 <= S <= 128, B <= 4096 (GDPA_ERR_UNSUPPORTED
 *   otherwise); max_n, total_tokens and the error behaviour as in gdpa_fwd.
 *   workspace: device, >= gdpa_pool_workspace_size bytes, 256-byte aligned;
 *   device-detected errors go to its status word (gdpa_workspace_status).
 */
GDPA_API gdpa_status_t gdpa_pool_workspace_size(int32_t B, int32_t h, int32_t dh, int32_t S,
                                                size_t* bytes);
GDPA_API gdpa_status_t gdpa_pool_fwd(int32_t B, int32_t h, int32_t dh, int32_t S,
                                     int64_t total_tokens, int32_t max_n, float scale,
                                     const void* seeds, const int32_t* offsets, const void* k,
                                     const void* v, void* o, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * Gradient of gdpa_pool_fwd for an upstream dO (same passage; the softmax
 * attention gradient with the seeds as queries):
 *
 *     dV_t = sum_i P[i, t] dO_i,   dS = P * (dP - D),   dP = dO V^T,   D_i = dO_i . O_i,
 *     dK_t = scale * sum_i dS[i, t] seeds_i,   dseeds_i = scale * sum_b sum_t dS[i, t] k_t,
 *
 * per sample b and head j; the seeds' gradient sums over every sample.
 *   seeds, k, v, o (from gdpa_pool_fwd), lse (its fp32 [B, h, S] output,
 *   natural log, required), dout bf16 [B, h, S, dh]; outputs dseeds fp32
 *   [h, S, dh] (overwritten), dk, dv bf16 [T, h, dh] (every row written).
 *   Same shapes, limits, alignment and error behaviour as gdpa_pool_fwd.
 *   workspace: device, >= gdpa_pool_bwd_workspace_size bytes, 256-byte
 *   aligned; device-detected errors go to its status word.
 */
GDPA_API gdpa_status_t gdpa_pool_bwd_workspace_size(int32_t B, int32_t h, int32_t dh, int32_t S,
                                                    int64_t total_tokens, size_t* bytes);
GDPA_API gdpa_status_t gdpa_pool_bwd(int32_t B, int32_t h, int32_t dh, int32_t S,
                                     int64_t total_tokens, int32_t max_n, float scale,
                                     const void* seeds, const int32_t* offsets, const void* k,
                                     const void* v, const void* o, const float* lse,
                                     const void* dout, float* dseeds, void* dk, void* dv,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sliding-window self-attention on the jagged token sequence.  The Kunlun
 * summary (section 2.2, sliding-window bullet) restricts self-attention on the
 * sequence to local windows, from O(T^2) to O(T w), without giving the
 * window's alignment; this library takes the causal window of width `window`:
 * token t of a sample attends to the tokens t' of the same sample with
 * t - window < t' <= t.  Per head j:
 *
 *     O_t = sum_t' softmax_t'(scale * q_t . k_t') v_t',   LSE[j, t] = ln sum_t' exp(...)
 *
 *   q, k, v, o bf16 [T, h, dh] (device; o every row written), offsets int32
 *   [B+1] (device), lse fp32 [h, T] (output; may be NULL).  Base pointers
 *   16-byte aligned (lse, offsets 4-byte).  dh = 32 or 64; window >= 1.
 *   workspace: device, >= gdpa_window_workspace_size bytes, 256-byte aligned.
 *   max_n, total_tokens and the error behaviour as in gdpa_fwd.
 */
GDPA_API gdpa_status_t gdpa_window_workspace_size(int32_t B, int32_t h, int32_t dh,
                                                  int64_t total_tokens, size_t* bytes);
GDPA_API gdpa_status_t gdpa_window_fwd(int32_t B, int32_t h, int32_t dh, int64_t total_tokens,
                                       int32_t max_n, int32_t window, float scale,
                                       const void* q, const int32_t* offsets, const void* k,
                                       const void* v, void* o, float* lse, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * Gradient of gdpa_window_fwd for an upstream dO: dQ, dK, dV of the causal
 * window's softmax attention (same passage), with D_t = dO_t . O_t.
 *   q, k, v, o (from gdpa_window_fwd), lse (its fp32 [h, T] output, natural
 *   log, required), dout bf16 [T, h, dh]; outputs dq, dk, dv bf16 [T, h, dh]
 *   (every row written).  Same limits, alignment and error behaviour as
 *   gdpa_window_fwd, and B <= 4096 (GDPA_ERR_UNSUPPORTED otherwise).
 *   workspace: device, >= gdpa_window_bwd_workspace_size bytes, 256-byte
 *   aligned; device-detected errors go to its status word.
 */
GDPA_API gdpa_status_t gdpa_window_bwd_workspace_size(int32_t B, int32_t h, int32_t dh,
                                                      int64_t total_tokens, size_t* bytes);
GDPA_API gdpa_status_t gdpa_window_bwd(int32_t B, int32_t h, int32_t dh, int64_t total_tokens,
                                       int32_t max_n, int32_t window, float scale,
                                       const void* q, const int32_t* offsets, const void* k,
                                       const void* v, const void* o, const float* lse,
                                       const void* dout, void* dq, void* dk, void* dv,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Device-detected status of the last gdpa_fwd/gdpa_bwd that used `workspace`
 * (GDPA_OK, GDPA_ERR_INVALID_ARG for inconsistent offsets, GDPA_ERR_TIMEOUT).
 * Synchronises `stream`; writes the code to *status (host).
 */
GDPA_API gdpa_status_t gdpa_workspace_status(const void* workspace, void* stream, int32_t* status);

/* Static, human-readable name of a status code. */
GDPA_API const char* gdpa_status_string(gdpa_status_t s);

/* Number of kernels the last gdpa_fwd / gdpa_bwd call on this thread launched. */
GDPA_API int32_t gdpa_last_launch_count(void);

/*
 * Per-kernel timing (host-thread local; for benchmarks, not for production).
 * While enabled, each kernel launch of gdpa_fwd / gdpa_bwd on this host thread
 * is bracketed by two CUDA events recorded on the call's stream.  Enabling
 * (or disabling) discards any unread records.  Returns GDPA_ERR_CUDA if an
 * event could not be created.
 */
GDPA_API gdpa_status_t gdpa_timing_enable(int32_t enable);

typedef struct {
  char name[48];       /* kernel name, NUL-terminated */
  int32_t launches;    /* launches recorded since gdpa_timing_enable(1) */
  float total_ms;      /* sum of their event-measured durations */
} gdpa_kernel_time_t;

/*
 * Waits for the recorded events, then writes up to `cap` per-kernel sums to
 * `out` (host) and returns how many distinct kernels were recorded (which may
 * exceed cap), or -1 on a CUDA error.  The records are cleared.
 */
GDPA_API int32_t gdpa_timing_read(gdpa_kernel_time_t* out, int32_t cap);

/*
 * Self-test of the device-side failure path.  Launches one small kernel on
 * `stream` whose thread waits, with the same bounded mbarrier wait the GDPA
 * kernels use, on a barrier that nothing ever completes.  After timeout_us
 * microseconds (1 .. 5,000,000) the wait gives up, GDPA_ERR_TIMEOUT is written
 * to the status word of `workspace` (>= 256 bytes, 256-byte aligned, device)
 * and the kernel returns; the context stays usable.  Read the result with
 * gdpa_workspace_status().  The Kunlun pages have no counterpart of this call.
 */
GDPA_API gdpa_status_t gdpa_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                                  uint32_t timeout_us, void* stream);

/*
 * Self-test of the FMA-pipe exp2 that the softmax kernels use for part of
 * their exponentials (Cody-Waite range reduction and a degree-3 minimax
 * polynomial; relative error <= 7.5e-5 for -126 <= x < 127).  For n device
 * floats x, writes that exp2 to y_fma and the hardware ex2.approx result to
 * y_mufu (all device pointers, n >= 0), on `stream`.  Returns
 * GDPA_ERR_INVALID_ARG for n < 0 or a null pointer with n > 0.  The Kunlun
 * pages have no counterpart of this call.
 */
GDPA_API gdpa_status_t gdpa_selftest_exp2(const float* x, float* y_fma, float* y_mufu,
                                          int64_t n, void* stream);

/*
 * gdpa_fwd_no_alloc: gdpa_fwd for callers that cannot allocate device memory
 * at call time (for example a host framework that has reserved all device
 * memory for its own pool and gives plug-in operators no allocator, or a
 * serving loop that cannot afford cudaMalloc's implicit synchronisation).
 * The Kunlun pages have no counterpart of this call; it only moves gdpa_fwd's
 * scratch out of the caller's hands.
 *   Arguments as in gdpa_fwd, without the workspace: the caller passes inputs
 *   and outputs only.  The scratch (status header + tile list) is a static
 *   2 MiB device array inside the library, held by every device that loads
 *   the library until the process exits.  Problems whose forward workspace
 *   (gdpa_fwd_workspace_size) exceeds 2 MiB are rejected with
 *   GDPA_ERR_WORKSPACE before any launch; that allows h * (T / r + B) <= 131,056
 *   tiles, with r = 128 query rows per tile for bf16 and 64 for fp32.
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.  Allocates nothing: no cudaMalloc, cudaFree or allocating library
 *   routine.  All calls share the one array, so calls that overlap on the GPU
 *   (different streams, or different host threads, without ordering between
 *   them) race on it and must be serialised by the caller.  The device status
 *   of the last call is read with gdpa_fwd_no_alloc_status, not with
 *   gdpa_workspace_status.
 */
GDPA_API gdpa_status_t gdpa_fwd_no_alloc(const gdpa_problem_t* p, const void* q,
                                         const int32_t* offsets, const void* k, const void* v,
                                         void* o, float* lse, void* stream);

/*
 * Device-detected status (GDPA_OK, GDPA_ERR_INVALID_ARG for inconsistent
 * device offsets, GDPA_ERR_TIMEOUT) of the last gdpa_fwd_no_alloc call on the
 * current device, read from the header of its static scratch.  Copies four
 * bytes on `stream`, synchronises it, and writes the code to *status (host).
 * Allocates nothing.  The Kunlun pages have no counterpart of this call.
 */
GDPA_API gdpa_status_t gdpa_fwd_no_alloc_status(void* stream, int32_t* status);

#ifdef __cplusplus
}
#endif

#endif /* GDPA_H_ */
