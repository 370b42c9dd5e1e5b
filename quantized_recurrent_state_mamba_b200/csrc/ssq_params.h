// ssq_params.h -- launch parameters shared by the host API and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ssq.h"

namespace ssq {

// Everything a kernel needs to address one pool and one call's tensors.
// Passed by value as a __grid_constant__ kernel parameter (< 4 KB).
struct PoolView {
    uint8_t* pool;             // base of the pool (header at offset 0)
    long long header_bytes, slot_bytes;
    long long codes_off, meta_off, fp_off;
    long long codes_layer_bytes, meta_layer_bytes, fp_layer_bytes;
    int n_slots, n_layers;
    int H, P, N, G, hpg;       // heads, head_dim, d_state, groups, heads/group
    int Hq, Hf;                // heads in the quantized / fp region
    // n / P and h / hpg as (n * m) >> 32 with m = floor(2^32 / d) + 1: exact
    // for n < 2^32 / d (row and head indices are far below that)
    unsigned long long mP, mHpg;
    uint16_t perm[SSQ_MAX_HEADS];  // region position -> natural head index
};

struct CallView {
    const int32_t* slot_idx;   // [batch] or null (identity)
    int batch, layer0, nl;
    int rows_per_tile;         // rows of the quantized region handled per tile
    int rows_per_tile_f;       // rows of the fp region handled per tile
    int qtiles, ftiles;        // tiles per (layer, request) in each region
    long long total_tiles;
    int T;                     // tokens (scan only)
    int tiles_per_head;        // scan: CTAs per head
    int scan_chunk;            // scan: tokens staged per shared-memory buffer
    unsigned long long sr_seed;  // stochastic rounding: Philox key
    unsigned sr_step;            // stochastic rounding: step counter (first token)
    // Test support (ssq_test_hooks): the decode kernel's wait limit in clock
    // cycles (0: the default, about a second) and whether CTA 0's producer
    // withholds the copy of its first tile.
    long long wait_limit;
    int test_withhold;
    const float* x;
    const float* B;
    const float* C;
    const float* dt;
    const float* A;
    const float* D;
    float* y;
    const float* S_in;         // quantize_rows input
    float* S_out;              // dequantize_rows output
    float* diag;               // step diagnostics output, float4 per row
};

// The DAMP mixed-tier pool: every (slot, layer, head) owns one block of
// head_bytes: FP16 tier at hi_off ([K][P] halves), INT8 codes at codes_off
// ([N-K][P] bytes), meta at meta_off ([N-K] x {float Delta, float z}).
struct DampView {
    uint8_t* pool;
    long long header_bytes, slot_bytes, layer_bytes, head_bytes;
    int hi_off, codes_off, meta_off;
    int n_slots, n_layers;
    int H, P, N, G, hpg, K;
    const int32_t* chan;       // [n_layers][H][N] position -> key channel
};

struct DampCall {
    const int32_t* slot_idx;
    int batch, layer0, nl;
    const float* x;
    const float* B;
    const float* C;
    const float* dt;
    const float* A;
    const float* D;
    float* y;
    const float* S_in;
    float* S_out;
};

// which: 0 decode step, 1 quantize (hand-off from fp32), 2 dequantize
cudaError_t launch_damp(const DampView& dv, const DampCall& dc, int which, cudaStream_t stream);

// Host-side launchers (one per kernel family); each returns the CUDA error of
// its launch.  The decode and rows kernels run a grid-stride loop over tiles
// on a grid sized to the device's resident capacity.
// sr: stochastic rounding of the quantized rows (cv.sr_seed, cv.sr_step)
cudaError_t launch_decode(const PoolView& pv, const CallView& cv, int fmt, bool sr,
                          cudaStream_t stream);
cudaError_t launch_quantize(const PoolView& pv, const CallView& cv, int fmt,
                            cudaStream_t stream);
cudaError_t launch_dequantize(const PoolView& pv, const CallView& cv, int fmt,
                              cudaStream_t stream);
// Step diagnostics (read-only): per row {reversals, reversal error, total
// rounding error, readout signal} as float4 in [nl][batch][H][P] order, to
// cv.diag.  The decode kernel in its diagnostics mode; tiles as
// decode_tile_rows.
cudaError_t launch_decode_diag(const PoolView& pv, const CallView& cv, int fmt,
                               cudaStream_t stream);
// The decode kernel of one state format in a mode (0 nearest rounding, 1
// stochastic rounding, 2 diagnostics), specialised in ssq_decode_<format>.cu.
template <int FMT>
cudaError_t launch_decode_fmt(const PoolView& pv, const CallView& cv, int mode,
                              cudaStream_t stream);
// How the scan splits its rows: entries per lane, warps per CTA, rows per
// CTA, CTAs per head, tokens per staged chunk, dynamic shared memory.
struct ScanPlan {
    int E, warps, rows, tiles_per_head, chunk;
    size_t smem_bytes;
};
ScanPlan scan_plan(int d_state, int headdim, long long batch_heads, int sms);
// prefill: keep the state fp32 over all T tokens and quantize it once at
// the end (the prefill hand-off) instead of rounding at every token.
// sr: stochastic rounding at every token (not with prefill)
cudaError_t launch_scan(const PoolView& pv, const CallView& cv, int fmt, const ScanPlan& sp,
                        bool prefill, bool sr, cudaStream_t stream);

// Rows per decode tile in the quantized and the fp region.
void decode_tile_rows(int fmt, int d_state, int* rows_q, int* rows_f);
// Whether the decode kernel's per-unit shared memory (B and C of every group,
// per-head arrays) fits one CTA.
bool decode_fits(int fmt, int d_state, int nheads, int ngroups);

// Grid for a grid-stride kernel: resident blocks on the current device,
// capped by the number of tiles.
int grid_for(const void* kernel, int threads, long long tiles);

__host__ __device__ inline int fdiv(int n, unsigned long long m)
{
    return (int)(((unsigned long long)(unsigned)n * m) >> 32);
}
inline unsigned long long fdiv_magic(int d)
{
    return (1ull << 32) / (unsigned long long)d + 1ull;
}

// Rows handled per tile for a given d_state (256 threads, LPR lanes per row).
inline int rows_per_tile(int d_state)
{
    const int E = d_state >= 32 ? 32 : d_state;
    const int lpr = d_state / E;
    return 256 / lpr;
}

}  // namespace ssq
