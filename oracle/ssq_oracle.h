/*
 * ssq_oracle.h -- plain, slow CPU oracle for the quantized Mamba-2
 * recurrent-state update.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link
 * or call this code: only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA library; the two meet only through the seeded input
 * generators and through the documented pool byte layout, which the tests
 * pack and unpack on their own.
 *
 * Sources (page title, section):
 *   [SQ]   "ssm-state-quantization" README, Setup: decay lambda = exp(dt*A)
 *          per head and step; one scale per (head, head_dim) row over the
 *          d_state entries, refit every step; symmetric grid [-amax, amax]
 *          with step amax/(2^(b-1)-1); asymmetric grid [min, max] with an
 *          integer zero point and step (max-min)/(2^b-1); the output is read
 *          from the quantized state.  Findings 1: nearest rounding (RTN).
 *   [FAN]  "Mamba state quantization for inference", "Quantization error
 *          returns on the next token": S_t = A_t S_(t-1) + W_t and the stored
 *          state S_q,t = A_t S_q,(t-1) + W_t + R_t.  "Mixed precision spends
 *          bits on persistent channels": the update runs in FP32 and the new
 *          quantization parameters are derived from the updated state.
 *   [SSDi8] "SSDi8: Accurate and Efficient 8-bit Quantization for State
 *          Space Duality", 3.1 Quantization (nearest level, scale from the
 *          maximum absolute value and the bit width) and 4 Methodology, State
 *          quantization (per-(H,P) scales, nothing along N).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - input term dt*B (x) x, the Mamba-2 form; dt arrives already positive;
 *   - group map g(h) = h / (H/G);
 *   - round half to even (rint under FE_TONEAREST) on the exact product
 *     s'*inv (one rounding; the product is formed in double, where the
 *     product of two floats is exact), and the zero point likewise;
 *   - inv = 1/Delta once per row, then a multiply per entry;
 *   - zero point z = rint(-lo*inv) kept unclamped in an fp32 slot;
 *   - constant row: Delta := |lo|; Delta below FLT_MIN flushes the row to
 *     zero (Delta = 0, inv = 0, z = 0, all codes 0);
 *   - metadata is fp32 Delta (and fp32 z for the asymmetric grid);
 *   - bf16 storage rounds fp32 to nearest even;
 *   - heads whose mask entry is 0 keep an fp32 row and skip the quantizer.
 *
 * Parity status of each function is stated at its definition.
 */
#ifndef SSQ_ORACLE_H
#define SSQ_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Storage formats, numbered as in the library's public header so the tests
 * can pass one integer to both sides. */
enum { OREF_F32 = 0, OREF_BF16 = 1, OREF_I8_SYM = 2, OREF_I8_ASYM = 3,
       OREF_I4_SYM = 4, OREF_I4_ASYM = 5 };

typedef struct {
    int fmt;
    int nheads, headdim, d_state, ngroups;
    const uint8_t* head_mask; /* nheads entries, 1 = quantized; NULL = all */
} oref_cfg;

/* Logical state of one (layer, request): rows are (head, p) in natural head
 * order, rows = nheads*headdim.
 *   q[rows*N]    integer codes (quantized rows; unsigned for asym, signed
 *                for sym);
 *   delta[rows]  step Delta; zero[rows] zero point z (0 for sym);
 *   val[rows*N]  stored value of fp rows (f32 / bf16 formats, masked heads).
 * For a row only one of (q, delta, zero) or val is meaningful. */
typedef struct {
    int32_t* q;
    float* delta;
    float* zero;
    float* val;
} oref_state;

int   oref_bits(int fmt);
int   oref_is_quant(int fmt);
int   oref_is_sym(int fmt);
int   oref_row_is_quant(const oref_cfg* c, int h);

float oref_lambda(float dt, float A);
float oref_bf16_round(float v);

void  oref_quantize_row(int fmt, int N, const float* v, int32_t* q,
                        float* delta, float* zero);
void  oref_quantize_row_dbg(int fmt, int N, const float* v, int32_t* q,
                            float* delta, float* zero, float* pre);
void  oref_dequantize_row(int fmt, int N, const int32_t* q, float delta,
                          float zero, float* out);

void  oref_state_from_f32(const oref_cfg* c, const float* S, oref_state* st);
void  oref_state_to_f32(const oref_cfg* c, const oref_state* st, float* S);

void  oref_step(const oref_cfg* c, oref_state* st, const float* x,
                const float* B, const float* C, const float* dt,
                const float* A, const float* D, float* y, float* pre);

void  oref_scan(const oref_cfg* c, oref_state* st, int T, const float* x,
                const float* B, const float* C, const float* dt,
                const float* A, const float* D, float* y);

void  oref_step_diag(const oref_cfg* c, const oref_state* st, const float* x,
                     const float* B, const float* C, const float* dt,
                     const float* A, const float* D, float* diag);

/* Stochastic rounding.  The random draw of entry n of row r (= h*P + p) at
 * a step is 16 bits of Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
 * random numbers: as easy as 1, 2, 3", SC 2011) with key (seed low, seed
 * high) and counter (r*(N/8) + n/8, layer, slot, step): word (n%8)/2 of the
 * output, low half for even n, high half for odd n. */
typedef struct {
    uint64_t seed;
    uint32_t step;   /* token counter: decode position, or the first token of a scan */
    uint32_t layer;
    uint32_t slot;
} oref_sr;

void  oref_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
uint32_t oref_sr_u16(const oref_sr* r, int row, int n, int N);
void  oref_quantize_row_sr(int fmt, int N, const float* v, const uint32_t* u16,
                           int32_t* q, float* delta, float* zero);
void  oref_step_sr(const oref_cfg* c, oref_state* st, const oref_sr* r,
                   const float* x, const float* B, const float* C,
                   const float* dt, const float* A, const float* D, float* y);
void  oref_scan_sr(const oref_cfg* c, oref_state* st, const oref_sr* r, int T,
                   const float* x, const float* B, const float* C,
                   const float* dt, const float* A, const float* D, float* y);

void  oref_prefill(const oref_cfg* c, oref_state* st, int T, const float* x,
                   const float* B, const float* C, const float* dt,
                   const float* A, const float* D, float* y);

void  oref_scan_f64(const oref_cfg* c, double* S, int T, const float* x,
                    const float* B, const float* C, const float* dt,
                    const float* A, const float* D, double* y);

void  oref_decode_batch(const oref_cfg* c, int nl, int batch,
                        oref_state* states, const float* x, const float* B,
                        const float* C, const float* dt, const float* A,
                        const float* D, float* y);

/* DAMP mixed-tier state ("Mamba state quantization for inference", "Mixed
 * precision spends bits on persistent channels").  Per head, position m of
 * chan[h][.] names a key channel; positions 0..n_protected-1 hold the
 * channel's Hadamard-rotated value vector in FP16 (hi, widened to fp32
 * here), the others in INT8 on the asymmetric grid (codes q, step delta,
 * zero point zero per position).  headdim a power of two. */
typedef struct {
    int nheads, headdim, d_state, ngroups;
    int n_protected;
    const int32_t* chan;     /* [nheads][d_state], a permutation per head */
} oref_damp_cfg;

typedef struct {
    float* hi;       /* [nheads][K][P] */
    int32_t* q;      /* [nheads][N-K][P] */
    float* delta;    /* [nheads][N-K] */
    float* zero;     /* [nheads][N-K] */
} oref_damp_state;

void  oref_hadamard(int P, const float* v, int stride, float* out);
float oref_fp16_round(float v);
void  oref_damp_from_f32(const oref_damp_cfg* c, const float* S, oref_damp_state* st);
void  oref_damp_to_f32(const oref_damp_cfg* c, const oref_damp_state* st, float* S);
void  oref_damp_step(const oref_damp_cfg* c, oref_damp_state* st, const float* x,
                     const float* B, const float* C, const float* dt, const float* A,
                     const float* D, float* y);

#ifdef __cplusplus
}
#endif
#endif
