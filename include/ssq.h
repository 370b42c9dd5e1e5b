/*
 * ssq.h -- libssq: the Mamba-2 recurrent-state update with the per-request
 * state stored in low-bit form, on NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources are page title + section):
 *
 *   "ssm-state-quantization" README, Setup:
 *     - each head decays its state by lambda = exp(dt*A) per step;
 *     - the quantizer keeps one scale per row of the state (per head and
 *       head_dim, over the d_state entries) and refits it every step;
 *     - symmetric grid [-amax, amax] with step amax/(2^(b-1)-1), or
 *       asymmetric grid [min, max] with an integer zero point and step
 *       (max-min)/(2^b-1);
 *     - the output is read from the quantized state;
 *     - heads are grouped into decay bands (lambda <= 0.9, 0.9 < lambda <=
 *       0.99, lambda > 0.99) and a band can be rounded on its own.
 *   "ssm-state-quantization" README, Findings 1: nearest rounding (RTN).
 *   "Mamba state quantization for inference":
 *     - "Recurrent state is fixed per request, not free": each live request
 *       owns one state, and a token reads, updates and stores all of it;
 *     - "Mixed precision spends bits on persistent channels": decoding the
 *       low-bit part, the fp32 update, the new scales and the packed store
 *       belong in one kernel, and each precision tier is one contiguous
 *       region so nothing is gathered per token;
 *     - "Mamba state quantization needs phase-aware benchmarks": a prefill
 *       keeps its state in fp32 and hands its last state to the packed
 *       cache.
 *   "SSDi8: Accurate and Efficient 8-bit Quantization for State Space
 *   Duality", 4 Methodology, State quantization: per-(H,P) state scales,
 *   nothing along N.
 *
 * One step for one (layer, request, head h, row p), entries n < d_state:
 *     s_n   = decode(stored row)                 (q - z)*Delta, q*Delta, fp
 *     lam   = (float) exp((double)(dt_h * A_h))
 *     s'_n  = fma(lam, s_n, (dt_h * x_p) * B_{g(h),n})        all fp32
 *     refit Delta (and z) from s', round s'_n*inv to nearest (ties to even)
 *     y_p   = sum_n C_{g(h),n} * decode(new row)_n + D_h * x_p
 * with g(h) = h / (nheads/ngroups).  Quantized codes are bit-identical to a
 * plain scalar evaluation of these formulas in that order; y is fp32 with
 * fp32 accumulation.  A head whose mask entry is 0 keeps an fp32 row.
 *
 * ---------------------------------------------------------------------------
 * Conventions for every entry point
 *   - Device pointers are CUDA device (or managed) memory owned by the caller;
 *     the library never allocates, frees or synchronises except where an
 *     entry point says so.  Every launch is asynchronous on `stream`.
 *   - Argument errors are detected on the host before anything is launched
 *     and nothing is written; the call returns SSQ_ERR_INVALID_ARG,
 *     SSQ_ERR_UNSUPPORTED or SSQ_ERR_ALIGNMENT.  A failed launch returns
 *     SSQ_ERR_CUDA.  ssq_last_error_detail() gives a one-line reason.
 *   - Values that live on the device (slot indices, state contents) are
 *     checked by the kernels: a bad value sets a bit in the pool's error word
 *     (SSQ_DEVERR_*), the affected request is skipped, and no kernel traps.
 *     Read the word with ssq_pool_error().
 *   - Results are deterministic: no atomics on any output.
 *   - Two calls that write the same slot and layer must not overlap on the
 *     GPU; one call must not name a slot twice in slot_idx.
 * ---------------------------------------------------------------------------
 */
#ifndef SSQ_H
#define SSQ_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols of libssq (the library is built with hidden default
 * visibility). */
#if defined(__GNUC__)
#define SSQ_API __attribute__((visibility("default")))
#else
#define SSQ_API
#endif

#define SSQ_MAX_HEADS 512
#define SSQ_POOL_HEADER_BYTES 256
#define SSQ_POOL_ALIGN 256

typedef enum {
    SSQ_OK = 0,
    SSQ_ERR_INVALID_ARG = 1, /* null pointer, bad size or index          */
    SSQ_ERR_UNSUPPORTED = 2, /* shape or format this build does not cover */
    SSQ_ERR_ALIGNMENT = 3,   /* pointer not aligned as documented        */
    SSQ_ERR_CUDA = 4         /* a CUDA call or launch failed              */
} ssq_status;

/* State storage formats.  b = 8 or 4 bits per code; "sym" uses the
 * symmetric grid, "asym" the asymmetric grid with an integer zero point. */
typedef enum {
    SSQ_F32 = 0,     /* fp32 state, no rounding                        */
    SSQ_BF16 = 1,    /* bf16 state, fp32 -> bf16 round to nearest even  */
    SSQ_I8_SYM = 2,  /* int8 two's complement codes in [-127, 127]     */
    SSQ_I8_ASYM = 3, /* uint8 codes in [0, 255]                        */
    SSQ_I4_SYM = 4,  /* 4-bit two's complement codes in [-7, 7]         */
    SSQ_I4_ASYM = 5  /* 4-bit codes in [0, 15]                          */
} ssq_format;

/* Bits of the pool's device error word (SSQ_DEVERR_*). */
#define SSQ_DEVERR_SLOT 0x1u      /* slot index outside [0, n_slots)      */
#define SSQ_DEVERR_NONFINITE 0x2u /* a row's updated values were not finite */
#define SSQ_DEVERR_TIMEOUT 0x4u   /* a pipeline wait gave up (about 1 s)    */
#define SSQ_DEVERR_CHANNEL 0x8u   /* a DAMP channel map entry outside [0, d_state) */

/* Shape of one state pool.  Every request slot holds the state of n_layers
 * layers; each layer holds nheads x headdim rows of d_state entries.
 *   nheads      1 .. SSQ_MAX_HEADS
 *   headdim     1 .. 2048
 *   d_state     16, 32, 64, 128 or 256
 *   ngroups     >= 1 and divides nheads; B and C are shared by the
 *               nheads/ngroups consecutive heads of a group
 *   head_mask   HOST array of nheads bytes, or NULL.  For the integer
 *               formats, heads with mask 0 keep an fp32 row and are never
 *               rounded ("ssm-state-quantization", Setup: rounding one decay
 *               band only).  Ignored for SSQ_F32 and SSQ_BF16.  Read during
 *               each call; the library keeps no pointer to it. */
typedef struct {
    int n_layers;
    int n_slots;
    int nheads;
    int headdim;
    int d_state;
    int ngroups;
    ssq_format fmt;
    const uint8_t* head_mask;
} ssq_config;

/* Byte layout of a pool (all offsets in bytes).
 *
 *   pool = [header: SSQ_POOL_HEADER_BYTES][slot 0][slot 1] ... [slot n-1]
 *   slot s starts at header_bytes + s*slot_bytes.  Inside a slot, layer l's
 *   block of each region starts at region_off + l*region_layer_bytes:
 *     codes  at codes_off: [n_quant_heads][headdim][row_code_bytes]
 *     meta   at meta_off:  [n_quant_heads][headdim][row_meta_bytes]
 *     fp     at fp_off:    [n_fp_heads][headdim][d_state] elements of
 *                          fp_elem_bytes (fp32, or bf16 for SSQ_BF16)
 *   and the *_layer_bytes strides are those sizes rounded up to
 *   SSQ_POOL_ALIGN.
 *   Heads are stored in region order: the quantized heads first in increasing
 *   head index, then the fp heads (head_perm of ssq_pool_layout).  So a
 *   masked band is one contiguous region and no kernel gathers per token
 *   ("Mamba state quantization for inference", mixed-precision layout).
 *   Codes of a row: 8-bit formats store entry n in byte n; 4-bit formats store
 *   entries 2k and 2k+1 in the low and high nibble of byte k.  Sym codes are
 *   two's complement (int8 / 4-bit).  Meta of a row: asym {float Delta,
 *   float z} (8 bytes), sym {float Delta} (4 bytes).
 *   Header: uint32 error word (SSQ_DEVERR_* bits) at byte 0; the rest is
 *   reserved.  Every region and slot starts on a SSQ_POOL_ALIGN boundary.
 *   An all-zero pool is a valid all-zero state in every format. */
typedef struct {
    size_t pool_bytes;
    size_t header_bytes;
    size_t slot_bytes;
    size_t codes_off, meta_off, fp_off;
    size_t codes_layer_bytes, meta_layer_bytes, fp_layer_bytes;
    size_t row_code_bytes, row_meta_bytes, fp_elem_bytes;
    int n_quant_heads, n_fp_heads;
} ssq_layout;

/* Compute the pool layout for cfg ("Mamba state quantization for
 * inference", "Recurrent state is fixed per request, not free": one state
 * per live request, sized by the format; "Mixed precision spends bits on
 * persistent channels": each precision tier one contiguous region).
 * head_perm (HOST, nheads int32, may be NULL) receives the natural head
 * index stored at each region position.  Host only; no CUDA call. */
SSQ_API ssq_status ssq_pool_layout(const ssq_config* cfg, ssq_layout* out,
                           int32_t* head_perm);

/* Set a whole pool to the all-zero state and clear its error word
 * (cudaMemsetAsync of layout.pool_bytes bytes).  pool: device, aligned to
 * SSQ_POOL_ALIGN. */
SSQ_API ssq_status ssq_pool_init(const ssq_config* cfg, void* pool,
                         cudaStream_t stream);

/* Read the pool's error word into *flags (HOST) and clear it.  This call
 * synchronises `stream`. */
SSQ_API ssq_status ssq_pool_error(const ssq_config* cfg, void* pool,
                          uint32_t* flags, cudaStream_t stream);

/* Write fp32 states into pool slots through the row quantizer: the prefill
 * hand-off of "Mamba state quantization for inference" ("Mamba state
 * quantization needs phase-aware benchmarks": the fp32 state at the end of a
 * prefill chunk enters the packed cache), and pool initialisation.
 *   S         device fp32 [nl][batch][nheads][headdim][d_state], natural head
 *             order, 16-byte aligned
 *   slot_idx  device int32 [batch]: pool slot of request b; NULL = slot b
 *   layers    layer0 .. layer0+nl-1 of each slot are written */
SSQ_API ssq_status ssq_quantize_rows(const ssq_config* cfg, void* pool,
                             const int32_t* slot_idx, int batch, int layer0,
                             int nl, const float* S, cudaStream_t stream);

/* Read pool slots back as fp32 (checkpointing, tests): the inverse layout of
 * ssq_quantize_rows, each row decoded as (q - z)*Delta (asymmetric grid),
 * q*Delta (symmetric grid) or the fp value ("ssm-state-quantization"
 * README, Setup: the two grids and the per-row scale).
 *   S_out  device fp32 [nl][batch][nheads][headdim][d_state], natural head
 *          order, 16-byte aligned; slot_idx, layer0, nl as ssq_quantize_rows.
 * Rows of a request whose slot index is out of range are not written. */
SSQ_API ssq_status ssq_dequantize_rows(const ssq_config* cfg, const void* pool,
                               const int32_t* slot_idx, int batch,
                               int layer0, int nl, float* S_out,
                               cudaStream_t stream);

/* Diagnostics of one decode step, read-only ("ssm-state-quantization"
 * README, Findings 4 and 5: an entry reverses when rounding turns its change
 * against the direction of the step's input; the page relates damage to the
 * part of the reversal error that reaches the output, measured against the
 * output itself).  For
 * every row the step ssq_decode_step would take is evaluated (same update
 * s' = fma(lambda, s, w), w = fl(fl(dt*x)*B_n), same refit and nearest
 * rounding) and, with e_n = fl(deq_n - s'_n) the rounding error, four fp32
 * numbers are written:
 *   [0] reversals: entries with w_n != 0 whose increment fl(e_n + w_n) has
 *       the other sign than w_n
 *   [1] sum over the reversed entries of C_n e_n
 *   [2] sum over all entries of C_n e_n
 *   [3] the readout signal, sum over all entries of C_n s'_n
 * Rows stored as fp32 / bf16 are not rounded: [0..2] = 0.  The pool is not
 * changed; y and D are not involved (the D*x term does not see the state).
 *   x, B, C, dt, A, slot_idx  as ssq_decode_step
 *   diag  device fp32 [nl][batch][nheads][headdim][4], natural head order,
 *         16-byte aligned; rows of a request whose slot index is out of
 *         range are not written (the pool's error word records it). */
SSQ_API ssq_status ssq_decode_diag(const ssq_config* cfg, const void* pool,
                           const int32_t* slot_idx, int batch, int layer0,
                           int nl, const float* x, const float* B,
                           const float* C, const float* dt, const float* A,
                           float* diag, cudaStream_t stream);

/* One decode token for a batch of live requests over nl layers, in one
 * launch: the fused read -> recurrence -> refit -> requantize -> write-back
 * -> readout of "Mamba state quantization for inference" (mixed-precision
 * section) with the quantizer of "ssm-state-quantization", Setup.  The nl
 * layer updates are independent (a model calls nl = 1 per layer because
 * layer l+1's input depends on layer l's output).
 *   slot_idx  device int32 [batch] or NULL (slot b)
 *   x         device fp32 [nl][batch][nheads][headdim]      (16-B aligned)
 *   B, C      device fp32 [nl][batch][ngroups][d_state]     (16-B aligned)
 *   dt        device fp32 [nl][batch][nheads], already positive (softplus
 *             and bias applied by the caller)
 *   A, D      device fp32 [nl][nheads]
 *   y         device fp32 [nl][batch][nheads][headdim]      (16-B aligned)
 * The state of layers layer0 .. layer0+nl-1 of each named slot is updated
 * in place.  y of a request whose slot index is out of range is not
 * written. */
SSQ_API ssq_status ssq_decode_step(const ssq_config* cfg, void* pool,
                           const int32_t* slot_idx, int batch, int layer0,
                           int nl, const float* x, const float* B,
                           const float* C, const float* dt, const float* A,
                           const float* D, float* y, cudaStream_t stream);

/* ssq_decode_step with stochastic rounding of the quantized rows
 * ("ssm-state-quantization" README, Findings 9: stochastic rounding of the
 * state keeps 8 bits within 0.4 ppl of the control).  Entry n of row r =
 * h*headdim + p rounds to floor(s'*inv + u) (+ z), clamped to the code
 * range, on the grid refit as for nearest rounding; u = d/65536 with d 16
 * bits of Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC 2011) under key
 * (seed low word, seed high word) and counter (r*(d_state/8) + n/8, layer,
 * slot, step): word (n%8)/2 of the output, low half for even n.  Pass a new
 * step (e.g. the token position) at every call for fresh draws.  fp32 /
 * bf16 rows are unaffected.  Other arguments as ssq_decode_step. */
SSQ_API ssq_status ssq_decode_step_sr(const ssq_config* cfg, void* pool,
                              const int32_t* slot_idx, int batch, int layer0,
                              int nl, const float* x, const float* B,
                              const float* C, const float* dt, const float* A,
                              const float* D, float* y, uint64_t seed,
                              uint32_t step, cudaStream_t stream);

/* T tokens of one layer with the state rounded at every token and held on
 * chip between tokens ("ssm-state-quantization", Setup: a sequential
 * per-token scan in place of the chunked scan, so the state can be rounded
 * at every step).  Equal, bit for bit in the stored codes and meta, to T
 * calls of ssq_decode_step with nl = 1.
 *   x   device fp32 [batch][T][nheads][headdim]     (16-B aligned)
 *   B,C device fp32 [batch][T][ngroups][d_state]    (16-B aligned)
 *   dt  device fp32 [batch][T][nheads]
 *   A,D device fp32 [nheads]
 *   y   device fp32 [batch][T][nheads][headdim]     (16-B aligned)
 * Only the final state is written to the pool. */
SSQ_API ssq_status ssq_scan(const ssq_config* cfg, void* pool,
                    const int32_t* slot_idx, int batch, int layer, int T,
                    const float* x, const float* B, const float* C,
                    const float* dt, const float* A, const float* D,
                    float* y, cudaStream_t stream);

/* ssq_scan with stochastic rounding at every token, token t drawing with
 * step counter step0 + t (draws as ssq_decode_step_sr); equal to T calls of
 * ssq_decode_step_sr with nl = 1 and steps step0 .. step0+T-1. */
SSQ_API ssq_status ssq_scan_sr(const ssq_config* cfg, void* pool,
                       const int32_t* slot_idx, int batch, int layer, int T,
                       const float* x, const float* B, const float* C,
                       const float* dt, const float* A, const float* D,
                       float* y, uint64_t seed, uint32_t step0,
                       cudaStream_t stream);

/* Prefill hand-off ("Mamba state quantization for inference", "Mamba state
 * quantization needs phase-aware benchmarks": the prefill runs in fp32 and
 * only its last state is packed).  T tokens of one layer from the stored state with the
 * recurrence in fp32 and no rounding between tokens; y_t is read from the
 * fp32 state; after the last token the state is refit and quantized once
 * (quantized heads; fp heads are stored as fp32, or rounded to bf16 for
 * SSQ_BF16) and written to the pool.  Arguments, layouts, ownership and
 * errors as ssq_scan.  A fresh request starts from a zero slot
 * (ssq_pool_init, or ssq_quantize_rows of zeros); a chunked prefill passes
 * each chunk in turn (the state is requantized between chunks). */
SSQ_API ssq_status ssq_prefill(const ssq_config* cfg, void* pool,
                       const int32_t* slot_idx, int batch, int layer, int T,
                       const float* x, const float* B, const float* C,
                       const float* dt, const float* A, const float* D,
                       float* y, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * DAMP mixed-tier state ("Mamba state quantization for inference", "Mixed
 * precision spends bits on persistent channels").  Per head the state
 * S[p][n] (p < headdim the value dimension, n < d_state the key channel) is
 * held as d_state key channels, each the Hadamard-rotated value vector
 *     t[k] = sum_p H[k][p] S[p][n],   H[k][p] = (-1)^popcount(k & p)
 * (the +-1 Sylvester-Hadamard matrix of order headdim; H/sqrt(headdim) is
 * orthonormal), formed in double by the fast Walsh-Hadamard transform
 * (butterfly stages of span 1, 2, ..., headdim/2) and rounded once to fp32.  A per-(layer, head) channel map chan[m] (a permutation of
 * 0..d_state-1, chosen by calibration outside the library) puts the
 * n_protected protected channels first: positions m < n_protected keep t in
 * FP16 (round to nearest even), the others in INT8 on the asymmetric grid of
 * the row quantizer above, one {fp32 Delta, fp32 z} per position over its
 * headdim values.  Bits per value: 16 for the FP16 tier, 8 + 64/headdim for
 * the INT8 tier (9 at headdim 64); 16 of 128 channels protected at headdim
 * 64 gives 9.875.
 *
 * The decode step runs the recurrence on the rotated state with the rotated
 * input xr = H x (rounded as above):
 *     t'_m[k] = fma(lambda, t_m[k], fl(fl(dt*xr[k]) * B[chan[m]]))
 * FP16 positions store fp16(t'), INT8 positions refit and round t' exactly
 * as ssq_decode_step rounds a row (codes, steps, zero points and FP16 values
 * are bit-identical to a scalar evaluation); y is read from the stored state
 * and rotated back:
 *     y[p] = D x[p] + (1/headdim) sum_k H[p][k] sum_m C[chan[m]] t'_m[k]
 * accumulated in fp32.
 *
 * Shapes: headdim 16, 32, 64 or 128; d_state 16 .. 256, a multiple of 16;
 * 0 <= n_protected <= d_state; ngroups divides nheads.
 * ------------------------------------------------------------------------ */
typedef struct {
    int n_layers;
    int n_slots;
    int nheads;
    int headdim;
    int d_state;
    int ngroups;
    int n_protected;
} ssq_damp_config;

/* Byte layout of a DAMP pool.
 *   pool = [header: SSQ_POOL_HEADER_BYTES][slot 0] ... [slot n_slots-1]
 *   slot = [layer 0] ... [layer n_layers-1], layer = [head 0] ... [head H-1]
 *   head block (head_bytes, a multiple of 16), offsets within it:
 *     hi_off    [n_protected][headdim] fp16, position-major
 *     codes_off [d_state - n_protected][headdim] uint8 codes
 *     meta_off  [d_state - n_protected] x {float Delta, float z}
 *   each region starts on a 16-byte boundary; slot_bytes is rounded up to
 *   SSQ_POOL_ALIGN.  Header: the uint32 error word at byte 0.  An all-zero
 *   pool is the all-zero state.  bits_per_value counts codes, FP16 values
 *   and meta per state value (padding excluded). */
typedef struct {
    size_t pool_bytes;
    size_t header_bytes;
    size_t slot_bytes;
    size_t layer_bytes;
    size_t head_bytes;
    size_t hi_off, codes_off, meta_off;
    double bits_per_value;
} ssq_damp_layout;

/* Host only; no CUDA call.  SSQ_ERR_UNSUPPORTED for shapes outside the
 * list above. */
SSQ_API ssq_status ssq_damp_pool_layout(const ssq_damp_config* cfg, ssq_damp_layout* out);

/* Write fp32 states into DAMP pool slots (the prefill hand-off for this
 * layout): every key channel rotated, then stored in its tier.
 *   chan      device int32 [n_layers][nheads][d_state]: the channel map of
 *             every layer (a permutation per head; an entry outside
 *             [0, d_state) sets SSQ_DEVERR_CHANNEL and that head is skipped)
 *   S         device fp32 [nl][batch][nheads][headdim][d_state], 16-B aligned
 *   slot_idx  device int32 [batch] or NULL; layers layer0 .. layer0+nl-1
 * pool: device, aligned to SSQ_POOL_ALIGN. */
SSQ_API ssq_status ssq_damp_quantize(const ssq_damp_config* cfg, void* pool,
                             const int32_t* chan, const int32_t* slot_idx,
                             int batch, int layer0, int nl, const float* S,
                             cudaStream_t stream);

/* Read DAMP pool slots back as fp32: S[p][chan[m]] = (1/headdim) sum_k
 * H[p][k] t_m[k], formed in double by the same butterfly transform and
 * rounded once.
 *   S_out  device fp32 [nl][batch][nheads][headdim][d_state] */
SSQ_API ssq_status ssq_damp_dequantize(const ssq_damp_config* cfg, const void* pool,
                               const int32_t* chan, const int32_t* slot_idx,
                               int batch, int layer0, int nl, float* S_out,
                               cudaStream_t stream);

/* One decode token on DAMP pool slots over nl layers.  x, B, C, dt, A, D, y
 * and slot_idx as ssq_decode_step; chan as ssq_damp_quantize.  The pool's
 * error word (read with ssq_pool_error or ssq_damp_pool_error) records bad
 * slots (the request is skipped), bad channel maps (the head is skipped) and
 * non-finite INT8 groups. */
SSQ_API ssq_status ssq_damp_decode_step(const ssq_damp_config* cfg, void* pool,
                                const int32_t* chan, const int32_t* slot_idx,
                                int batch, int layer0, int nl, const float* x,
                                const float* B, const float* C,
                                const float* dt, const float* A,
                                const float* D, float* y, cudaStream_t stream);

/* Read the DAMP pool's error word into *flags (HOST) and clear it; this
 * call synchronises `stream`. */
SSQ_API ssq_status ssq_damp_pool_error(const ssq_damp_config* cfg, void* pool,
                               uint32_t* flags, cudaStream_t stream);

/* Static string for a status code. */
SSQ_API const char* ssq_status_string(ssq_status s);

/* One-line reason for the last non-OK status returned on this host thread
 * (static thread-local storage; valid until the next call). */
SSQ_API const char* ssq_last_error_detail(void);

/* Test support for the failure path of the decode step; not for production
 * use.  Applies to the ssq_decode_step / ssq_decode_step_sr launches issued
 * later on the calling host thread:
 *   wait_limit_cycles  the kernel's bound on each pipeline wait, in SM clock
 *                      cycles (0: the default, about one second)
 *   withhold_first_tile  nonzero: the producer of the first thread block
 *                      issues no copy for its first tile, so the waits on it
 *                      run out; the call sets SSQ_DEVERR_TIMEOUT in the
 *                      pool's error word and returns, no copy in flight and
 *                      the context usable (that block's tiles are skipped).
 * ssq_test_hooks(0, 0) restores normal behaviour.  SSQ_ERR_INVALID_ARG for a
 * negative limit.  Host only; no CUDA call. */
SSQ_API ssq_status ssq_test_hooks(int withhold_first_tile, long long wait_limit_cycles);

#ifdef __cplusplus
}
#endif
#endif /* SSQ_H */
