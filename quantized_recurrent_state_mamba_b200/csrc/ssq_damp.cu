// ssq_damp.cu -- the DAMP mixed-tier state: decode step, hand-off from fp32,
// read-back.
//
// "Mamba state quantization for inference", "Mixed precision spends bits on
// persistent channels": each key channel's vector over head_dim is rotated
// by a Hadamard matrix; a chosen set of channels stays in FP16 and the rest
// is stored as 8-bit codes with a step and an offset; each tier is one
// contiguous block, so a kernel reads both with no gather; every token
// decodes the 8-bit tier, updates in fp32, fits new steps and stores the
// packed state again, all in one kernel.
//
// Per head the state is N key channels ("positions" m = 0..N-1 after the
// caller's channel permutation chan[layer][h][m]; positions < K form the
// FP16 tier) of P rotated values t[m][k] = sum_p H[k][p] S[p][chan[m]], H the
// +-1 Sylvester-Hadamard matrix.  The recurrence is linear, so it runs on the
// rotated state with the rotated input xr = H x:
//   t'[m][k] = fma(lambda, t[m][k], fl(fl(dt * xr[k]) * B[chan[m]]))
// and the readout rotates back once per head:
//   y[p] = D x[p] + (1/P) sum_k H[p][k] sum_m C[chan[m]] stored'[m][k].
// Rotations that decide stored values (xr, the hand-off, the read-back) are
// the fast Walsh-Hadamard transform in double, butterfly stages h = 1, 2,
// ..., P/2, rounded once, so every stored code, step, zero point and FP16
// value is bit-identical to a scalar evaluation in that order; the readout
// accumulates and rotates back in fp32.
//
// Thread mapping: a position's P values sit on LPR consecutive lanes, E per
// lane (lane j of the group holds rotated indices jE .. jE+E-1); a warp
// covers 32/LPR positions per pass.  The hand-off and read-back kernels use
// E = 16 with one CTA per head; the decode step uses E = 32 (16 at P = 16)
// with one warp per head (below).
#include <cuda_fp16.h>

#include <type_traits>

#include "ssq_common.cuh"
#include "ssq_params.h"
#include "ssq_pipe.cuh"

namespace ssq {

namespace {

constexpr int kDampE = 16;   // rotated entries per lane (hand-off, read-back)

// Reduce-scatter of a lane's E partial sums over the positions of its warp:
// at each round a lane keeps half of its values and sends the other half to
// the partner lane (xor OFF), so after log2(32/LPR) rounds the warp's sums
// over all its positions are spread over the lanes.  base gets the offset
// (within the lane's E) of the values the lane ends with.
template <int CUR, int OFF, int REM, int E>
__device__ __forceinline__ void reduce_scatter(float (&v)[E], int lane, int& base)
{
    if constexpr (REM > 0) {
        if constexpr (CUR > 1) {
            constexpr int H = CUR / 2;
            const bool up = (lane & OFF) != 0;
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const float send = up ? v[i] : v[i + H];
                const float keep = up ? v[i + H] : v[i];
                v[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, OFF));
            }
            if (up) base += H;
            reduce_scatter<H, OFF * 2, REM - 1, E>(v, lane, base);
        } else {
            v[0] = __fadd_rn(v[0], __shfl_xor_sync(0xffffffffu, v[0], OFF));
            reduce_scatter<1, OFF * 2, REM - 1, E>(v, lane, base);
        }
    }
}

template <int N>
__host__ __device__ constexpr int ilog2() { return N <= 1 ? 0 : 1 + ilog2<N / 2>(); }

// Fast Walsh-Hadamard transform in double of a vector of E*LPR values held
// E per lane by LPR consecutive lanes (lane j of the group holds indices
// j*E .. j*E+E-1): stages h = 1, 2, ..., E*LPR/2 in turn; at each stage the
// pair (i, i+h), bit h of i clear, becomes (a_i + a_(i+h), a_i - a_(i+h)).
// Stages h < E pair values inside a lane, the others pair lanes j and j^(h/E).
template <int E, int LPR>
__device__ __forceinline__ void fwht_lanes(double (&a)[E], int lane)
{
#pragma unroll
    for (int h = 1; h < E; h *= 2) {
#pragma unroll
        for (int e = 0; e < E; ++e)
            if ((e & h) == 0) {
                const double x = a[e], y = a[e + h];
                a[e] = __dadd_rn(x, y);
                a[e + h] = __dsub_rn(x, y);
            }
    }
#pragma unroll
    for (int o = 1; o < LPR; o *= 2) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const double other = __shfl_xor_sync(0xffffffffu, a[e], o);
            a[e] = up ? __dsub_rn(other, a[e]) : __dadd_rn(a[e], other);
        }
    }
}

struct DampUnit {
    int l, b, h, slot, layer, g;
    long long lb;
    uint8_t* head;          // this unit's head block
    const int32_t* chan;    // [N] position -> key channel
};

__device__ __forceinline__ DampUnit damp_unit(const DampView& dv, const DampCall& dc, long long u)
{
    DampUnit t;
    t.lb = u / dv.H;
    t.h = (int)(u - t.lb * dv.H);
    t.l = (int)(t.lb / dc.batch);
    t.b = (int)(t.lb - (long long)t.l * dc.batch);
    t.slot = dc.slot_idx ? __ldg(dc.slot_idx + t.b) : t.b;
    t.layer = dc.layer0 + t.l;
    t.g = t.h / dv.hpg;
    t.head = dv.pool + dv.header_bytes + (long long)t.slot * dv.slot_bytes
             + (long long)t.layer * dv.layer_bytes + (long long)t.h * dv.head_bytes;
    t.chan = dv.chan + ((long long)t.layer * dv.H + t.h) * dv.N;
    return t;
}

// The lane's position for pass `pass` and its key channel (the unit's
// channel map was checked by damp_chan_ok).
struct DampPos {
    int m, n;
    bool active, hi;
};

template <int LPR>
__device__ __forceinline__ DampPos damp_pos(const DampView& dv, const DampUnit& u, int pass,
                                            int tid)
{
    DampPos ps;
    const int m = pass * (kThreads / LPR) + tid / LPR;
    ps.active = m < dv.N;
    ps.m = ps.active ? m : 0;
    ps.n = __ldg(u.chan + ps.m);
    ps.hi = ps.m < dv.K;
    return ps;
}

// Every channel index of the unit's map lies in [0, N) (N <= kThreads); a
// barrier for the whole CTA.
__device__ __forceinline__ bool damp_chan_ok(const DampView& dv, const DampUnit& u, int tid)
{
    int bad = 0;
    if (tid < dv.N) {
        const int n = __ldg(u.chan + tid);
        bad = (n < 0 || n >= dv.N);
    }
    return __syncthreads_or(bad) == 0;
}

// Reads the lane's 16 stored values of position ps.m (FP16 tier widened,
// INT8 tier decoded).  Every lane of the warp calls this.
__device__ __forceinline__ void damp_load(const DampView& dv, const DampUnit& u, const DampPos& ps,
                                          int j, float (&t)[kDampE])
{
    constexpr int E = kDampE;
    const int P = dv.P;
    Chunk<E> codes;
    float delta = 0.0f, z = 0.0f;
    if (ps.hi) {
        Chunk<2 * E> hv;
        load_chunk<2 * E>(hv, u.head + dv.hi_off + ((long long)ps.m * P + j * E) * 2);
#pragma unroll
        for (int i = 0; i < E / 2; ++i) {
            t[2 * i] = __half2float(__ushort_as_half((unsigned short)(hv.w[i] & 0xffffu)));
            t[2 * i + 1] = __half2float(__ushort_as_half((unsigned short)(hv.w[i] >> 16)));
        }
#pragma unroll
        for (int i = 0; i < E / 4; ++i) codes.w[i] = 0u;
    } else {
        const int i = ps.m - dv.K;
        load_chunk<E>(codes, u.head + dv.codes_off + (long long)i * P + j * E);
        const float2 mz = *reinterpret_cast<const float2*>(u.head + dv.meta_off + (long long)i * 8);
        delta = mz.x;
        z = mz.y;
    }
    float s[E];
    decode_row<SSQ_I8_ASYM, E>(codes, delta, z, s);   // warp-uniform inside
    if (!ps.hi) {
#pragma unroll
        for (int e = 0; e < E; ++e) t[e] = s[e];
    }
}

// Writes the updated values of position ps.m (tiers as above) and leaves in
// t what the stored state now decodes to.  Every lane of the warp calls this.
template <int LPR>
__device__ __forceinline__ void damp_store(const DampView& dv, const DampUnit& u, const DampPos& ps,
                                           int j, float (&t)[kDampE], bool write, uint32_t* err)
{
    constexpr int E = kDampE;
    const int P = dv.P;
    // INT8 tier: refit over the position's P values (LPR lanes), round
    const RowParams rp = refit_row<SSQ_I8_ASYM, E, LPR>(t);
    float r[E];
    uint32_t k[E];
    round_row<SSQ_I8_ASYM, E>(rp, t, r, k);
    if (ps.hi) {
        Chunk<2 * E> hv;
#pragma unroll
        for (int i = 0; i < E / 2; ++i) {
            const __half a = __float2half_rn(t[2 * i]);
            const __half b = __float2half_rn(t[2 * i + 1]);
            hv.w[i] = (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(b) << 16);
            t[2 * i] = __half2float(a);
            t[2 * i + 1] = __half2float(b);
        }
        if (write) store_chunk<2 * E>(u.head + dv.hi_off + ((long long)ps.m * P + j * E) * 2, hv);
    } else {
        Chunk<E> c;
        pack_codes<SSQ_I8_ASYM, E>(k, c);
        float dq[E];
        scale_row<E>(rp.delta, r, dq);
#pragma unroll
        for (int e = 0; e < E; ++e) t[e] = dq[e];
        if (write) {
            const int i = ps.m - dv.K;
            store_chunk<E>(u.head + dv.codes_off + (long long)i * P + j * E, c);
            if (j == 0) {
                *reinterpret_cast<float2*>(u.head + dv.meta_off + (long long)i * 8) =
                    make_float2(rp.delta, rp.z);
                if (!rp.finite) atomicOr(err, SSQ_DEVERR_NONFINITE);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Hand-off: fp32 S[nl][batch][H][P][N] -> tiers.  One CTA per head; a lane
// group of LPR lanes loads a key channel's column S[.][n] (E values per
// lane, in the order of the rotated index), rotates it with the lane-split
// fast transform in double, rounds once and stores the tier.
// ---------------------------------------------------------------------------
template <int P>
__global__ void __launch_bounds__(kThreads)
damp_quantize_kernel(const __grid_constant__ DampView dv, const __grid_constant__ DampCall dc)
{
    constexpr int E = kDampE, LPR = P / E;
    uint32_t* err = reinterpret_cast<uint32_t*>(dv.pool);
    const int tid = threadIdx.x, lane = tid & 31;
    const int j = tid % LPR;
    const int passes = (dv.N * LPR + kThreads - 1) / kThreads;
    const long long units = (long long)dc.nl * dc.batch * dv.H;
    for (long long uu = blockIdx.x; uu < units; uu += gridDim.x) {
        const DampUnit u = damp_unit(dv, dc, uu);
        if (u.slot < 0 || u.slot >= dv.n_slots) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_SLOT);
            continue;
        }
        if (!damp_chan_ok(dv, u, tid)) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_CHANNEL);
            continue;
        }
        const float* S = dc.S_in + (u.lb * dv.H + u.h) * (long long)P * dv.N;
        for (int pass = 0; pass < passes; ++pass) {
            const DampPos ps = damp_pos<LPR>(dv, u, pass, tid);
            double a[E];
#pragma unroll
            for (int e = 0; e < E; ++e) a[e] = (double)__ldg(S + (long long)(j * E + e) * dv.N + ps.n);
            fwht_lanes<E, LPR>(a, lane);
            float t[E];
#pragma unroll
            for (int e = 0; e < E; ++e) t[e] = __double2float_rn(a[e]);
            damp_store<LPR>(dv, u, ps, j, t, ps.active, err);
        }
    }
}

// ---------------------------------------------------------------------------
// Read-back: tiers -> fp32 S[nl][batch][H][P][N]: reconstruct, rotate back
// with the fast transform in double, scale by the exact 1/P, round once.
// ---------------------------------------------------------------------------
template <int P>
__global__ void __launch_bounds__(kThreads)
damp_dequantize_kernel(const __grid_constant__ DampView dv, const __grid_constant__ DampCall dc)
{
    constexpr int E = kDampE, LPR = P / E;
    uint32_t* err = reinterpret_cast<uint32_t*>(dv.pool);
    const int tid = threadIdx.x, lane = tid & 31;
    const int j = tid % LPR;
    const int passes = (dv.N * LPR + kThreads - 1) / kThreads;
    const long long units = (long long)dc.nl * dc.batch * dv.H;
    for (long long uu = blockIdx.x; uu < units; uu += gridDim.x) {
        const DampUnit u = damp_unit(dv, dc, uu);
        if (u.slot < 0 || u.slot >= dv.n_slots) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_SLOT);
            continue;
        }
        if (!damp_chan_ok(dv, u, tid)) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_CHANNEL);
            continue;
        }
        float* S = dc.S_out + (u.lb * dv.H + u.h) * (long long)P * dv.N;
        for (int pass = 0; pass < passes; ++pass) {
            const DampPos ps = damp_pos<LPR>(dv, u, pass, tid);
            float t[E];
            damp_load(dv, u, ps, j, t);
            double a[E];
#pragma unroll
            for (int e = 0; e < E; ++e) a[e] = (double)t[e];
            fwht_lanes<E, LPR>(a, lane);
            if (ps.active) {
#pragma unroll
                for (int e = 0; e < E; ++e)
                    S[(long long)(j * E + e) * dv.N + ps.n] =
                        __double2float_rn(__dmul_rn(a[e], 1.0 / (double)P));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Decode step: a head's packed state is one contiguous block, so a producer
// warp streams whole blocks (with the head's x, its group's B and C and its
// channel map) into a ring of shared-memory stages with bulk copies; each
// consumer warp takes one head at a time, updates the block in place in
// shared memory and writes it back with one bulk store, while the next
// heads' blocks are in flight.  Heads are dealt to the consumer warps in
// turn; a stage is released once the bulk store of its head has read it.
// ---------------------------------------------------------------------------
constexpr int kDampCWarps = 8;                       // consumer warps per CTA (at most)
constexpr int kDampStages = 16;                      // ring stages (at most)
constexpr int kDampPipeThreads = (kDampCWarps + 1) * 32;
constexpr int kDampSmemBudget = 227 * 1024;

struct DampGeom {
    int off_x, off_B, off_C, off_chan, stage_bytes;
    int S, Wc;                 // stages, consumer warps (S > Wc)
    int off_scr;               // per-warp scratch: fl(dt * xr[k]), P floats
    int off_bar, smem_bytes;
};

inline DampGeom damp_geom(int head_bytes, int P, int N, int S, int Wc)
{
    DampGeom g;
    g.off_x = head_bytes;                       // head_bytes is a multiple of 16
    g.off_B = g.off_x + P * 4;
    g.off_C = g.off_B + N * 4;
    g.off_chan = g.off_C + N * 4;
    g.stage_bytes = (g.off_chan + N * 4 + 127) / 128 * 128;
    g.S = S;
    g.Wc = Wc;
    g.off_scr = S * g.stage_bytes;
    g.off_bar = g.off_scr + Wc * P * 4;
    g.smem_bytes = g.off_bar + 2 * S * 8;
    return g;
}

// xr = H x over one warp: lane L holds indices L + 32r (P >= 32; for P = 16
// lanes L and L+16 both hold index L & 15).  Stages h < 32 pair lanes L and
// L^h, stages h >= 32 pair a lane's own values; h = 1, 2, ..., P/2 in turn.
template <int P>
__device__ __forceinline__ void fwht_warp(double (&a)[(P + 31) / 32], int lane)
{
    constexpr int V = (P + 31) / 32;
    constexpr int HL = P < 32 ? P : 32;
#pragma unroll
    for (int h = 1; h < HL; h *= 2) {
        const bool up = (lane & h) != 0;
#pragma unroll
        for (int r = 0; r < V; ++r) {
            const double other = __shfl_xor_sync(0xffffffffu, a[r], h);
            a[r] = up ? __dsub_rn(other, a[r]) : __dadd_rn(a[r], other);
        }
    }
#pragma unroll
    for (int hr = 1; hr < V; hr *= 2) {
#pragma unroll
        for (int r = 0; r < V; ++r)
            if ((r & hr) == 0) {
                const double x = a[r], y = a[r + hr];
                a[r] = __dadd_rn(x, y);
                a[r + hr] = __dsub_rn(x, y);
            }
    }
}

// k-bit B of a lane's readout value after reduce_scatter: 0 when the bit
// indexes the lane's own KEEP values, else the lane mask of the partner.
template <int E, int LPR, int KEEP, int B>
__host__ __device__ constexpr int kbit_lane()
{
    return B < ilog2<KEEP>() ? 0
           : B < ilog2<E>() ? (LPR << (ilog2<E>() - 1 - B))
                            : (1 << (B - ilog2<E>()));
}

// Fast transform (fp32) of the readout left by reduce_scatter: v[i] holds
// index j*E + base + i; stages h = 1, 2, ..., P/2 in turn.
template <int E, int LPR, int KEEP, int B, int NB>
__device__ __forceinline__ void fwht_readout(float (&v)[KEEP], int lane)
{
    if constexpr (B < NB) {
        constexpr int M = kbit_lane<E, LPR, KEEP, B>();
        if constexpr (M == 0) {
            constexpr int h = 1 << B;
#pragma unroll
            for (int i = 0; i < KEEP; ++i)
                if ((i & h) == 0) {
                    const float a = v[i], b = v[i + h];
                    v[i] = __fadd_rn(a, b);
                    v[i + h] = __fsub_rn(a, b);
                }
        } else {
            const bool up = (lane & M) != 0;
#pragma unroll
            for (int i = 0; i < KEEP; ++i) {
                const float o = __shfl_xor_sync(0xffffffffu, v[i], M);
                v[i] = up ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
            }
        }
        fwht_readout<E, LPR, KEEP, B + 1, NB>(v, lane);
    }
}

template <int P>
__global__ void __launch_bounds__(kDampPipeThreads, 1)
damp_decode_pipe(const __grid_constant__ DampView dv, const __grid_constant__ DampCall dc,
                 const DampGeom g)
{
    constexpr int E = P >= 32 ? 32 : 16;
    constexpr int LPR = P / E, PPW = 32 / LPR;
    constexpr int ROUNDS = ilog2<PPW>();
    constexpr int KEEP = (E >> ROUNDS) > 0 ? (E >> ROUNDS) : 1;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + g.off_bar);
    uint64_t* empty = full + g.S;
    uint32_t* err = reinterpret_cast<uint32_t*>(dv.pool);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = dv.H, N = dv.N, K = dv.K;
    const long long units = (long long)dc.nl * dc.batch * H;
    const long long per = (units + gridDim.x - 1) / gridDim.x;
    const long long u0 = (long long)blockIdx.x * per;
    const long long u1 = u0 + per < units ? u0 + per : units;
    const int n = u1 > u0 ? (int)(u1 - u0) : 0;
    const unsigned head_bytes = (unsigned)dv.head_bytes;

    if (threadIdx.x == 0) {
        for (int s = 0; s < g.S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == kDampCWarps) {
        // ---- producer ---------------------------------------------------
        if (lane != 0) return;
        long long last_lb = -1;
        int slot = 0, filled = 0;
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            const long long u = u0 + i;
            const int s = i % g.S;
            const unsigned f = (unsigned)(i / g.S);
            if (!mbar_wait<kProducerSleep>(&empty[s], (f & 1) ^ 1)) {
                ok = false;
                break;
            }
            const long long lb = u / H;
            const int h = (int)(u - lb * H);
            const int l = (int)(lb / dc.batch);
            const int b = (int)(lb - (long long)l * dc.batch);
            if (lb != last_lb) {
                slot = dc.slot_idx ? __ldg(dc.slot_idx + b) : b;
                last_lb = lb;
            }
            filled = i + 1;
            if (slot < 0 || slot >= dv.n_slots) {
                mbar_arrive(&full[s]);             // nothing to copy; consumers skip it
                continue;
            }
            const int layer = dc.layer0 + l;
            const int grp = h / dv.hpg;
            uint8_t* st = smem + (long long)s * g.stage_bytes;
            const uint8_t* head = dv.pool + dv.header_bytes + (long long)slot * dv.slot_bytes
                                  + (long long)layer * dv.layer_bytes + (long long)h * dv.head_bytes;
            mbar_arrive_tx(&full[s], head_bytes + (unsigned)(P * 4 + 3 * N * 4));
            bulk_g2s(st, head, head_bytes, &full[s]);
            bulk_g2s(st + g.off_x, dc.x + (lb * H + h) * P, P * 4, &full[s]);
            bulk_g2s(st + g.off_B, dc.B + (lb * dv.G + grp) * N, N * 4, &full[s]);
            bulk_g2s(st + g.off_C, dc.C + (lb * dv.G + grp) * N, N * 4, &full[s]);
            bulk_g2s(st + g.off_chan, dv.chan + ((long long)layer * H + h) * N, N * 4, &full[s]);
        }
        if (!ok) {
            atomicOr(err, SSQ_DEVERR_TIMEOUT);
            // copies still in flight land before this CTA's shared memory goes
            for (int i = filled - g.S > 0 ? filled - g.S : 0; i < filled; ++i)
                mbar_wait<kProducerSleep>(&full[i % g.S], (unsigned)(i / g.S) & 1);
        }
        return;
    }
    if (warp >= g.Wc) return;

    // ---- consumers ------------------------------------------------------
    const int j = lane % LPR, q = lane / LPR;
    const int passes = (N + PPW - 1) / PPW;
    int prev_s = -1;
    // scalars of the warp's next head, loaded one head ahead
    auto scalars = [&](int i, int& slot, float& dtv, float& Av, float& Dh) {
        const long long u = u0 + i;
        const long long lb = u / H;
        const int h = (int)(u - lb * H);
        const int l = (int)(lb / dc.batch);
        const int b = (int)(lb - (long long)l * dc.batch);
        slot = dc.slot_idx ? __ldg(dc.slot_idx + b) : b;
        dtv = __ldg(dc.dt + lb * H + h);
        Av = __ldg(dc.A + (long long)l * H + h);
        Dh = __ldg(dc.D + (long long)l * H + h);
    };
    int nslot = 0;
    float ndt = 0.0f, nA = 0.0f, nD = 0.0f;
    if (warp < n) scalars(warp, nslot, ndt, nA, nD);
    for (int i = warp; i < n; i += g.Wc) {
        const int slot = nslot;
        const float dtv = ndt, Av = nA, Dh = nD;
        if (i + g.Wc < n) scalars(i + g.Wc, nslot, ndt, nA, nD);
        const long long u = u0 + i;
        const long long lb = u / H;
        const int h = (int)(u - lb * H);
        const int l = (int)(lb / dc.batch);
        const int s = i % g.S;
        // the whole warp takes the same decision
        if (!__all_sync(0xffffffffu, mbar_wait<kConsumerSleep>(&full[s], (unsigned)(i / g.S) & 1))) {
            if (lane == 0) atomicOr(err, SSQ_DEVERR_TIMEOUT);
            break;
        }
        uint8_t* st = smem + (long long)s * g.stage_bytes;
        bool valid = slot >= 0 && slot < dv.n_slots;
        if (!valid) {
            if (lane == 0) atomicOr(err, SSQ_DEVERR_SLOT);
        } else {
            const int* chs = reinterpret_cast<const int*>(st + g.off_chan);
            bool bad = false;
            for (int m = lane; m < N; m += 32) bad |= (chs[m] < 0 || chs[m] >= N);
            if (__any_sync(0xffffffffu, bad)) {
                valid = false;
                if (lane == 0) atomicOr(err, SSQ_DEVERR_CHANNEL);
            }
        }
        bool stored = false;
        if (valid) {
            const float lam = decay(dtv, Av);
            const float* xs = reinterpret_cast<const float*>(st + g.off_x);
            const float* Bs = reinterpret_cast<const float*>(st + g.off_B);
            const float* Cs = reinterpret_cast<const float*>(st + g.off_C);
            const int* chs = reinterpret_cast<const int*>(st + g.off_chan);
            // fl(dt * xr[k]) for the lane's E rotated indices k = j*E + e:
            // the transform once per warp, handed round through shared memory
            float* dtxs = reinterpret_cast<float*>(smem + g.off_scr) + warp * P;
            {
                constexpr int V = (P + 31) / 32;
                double a[V];
#pragma unroll
                for (int r = 0; r < V; ++r) a[r] = (double)xs[P >= 32 ? lane + 32 * r : (lane & (P - 1))];
                fwht_warp<P>(a, lane);
#pragma unroll
                for (int r = 0; r < V; ++r)
                    if (P >= 32 || lane < P)
                        dtxs[P >= 32 ? lane + 32 * r : lane] = __fmul_rn(dtv, __double2float_rn(a[r]));
            }
            __syncwarp();
            const float* dtxj = dtxs + j * E;     // read per pass (frees registers)
            const float2 lam2 = make_float2(lam, lam);
            float acc[E];
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = 0.0f;
            // B and C of the lane's channel, one pass ahead (the channel map
            // lookup and the two reads behind it are a dependent chain)
            float nbn, ncn;
            {
                const int m = q < N ? q : 0;
                const int nch = chs[m];
                nbn = Bs[nch];
                ncn = q < N ? Cs[nch] : 0.0f;
            }
            // One pass: the lane's channel m = pass*PPW + q.  MODE 0: every
            // lane of the pass in the FP16 tier; 1: every lane in the INT8
            // tier and active; 2: anything (per-lane tier, inactive lanes).
            auto pass_body = [&](auto mode, int pass) {
                constexpr int MODE = decltype(mode)::value;
                const int m0 = pass * PPW + q;
                const bool active = MODE == 1 || m0 < N;
                const int m = active ? m0 : 0;
                const float bn = nbn, cn = ncn;
                if (pass + 1 < passes) {
                    const int m1 = m0 + PPW;
                    const int mm = m1 < N ? m1 : 0;
                    const int nch = chs[mm];
                    nbn = Bs[nch];
                    ncn = m1 < N ? Cs[nch] : 0.0f;
                }
                const bool hi = MODE == 0 || (MODE == 2 && m < K);
                float t[E];
                uint8_t* hp = st + dv.hi_off + (m * P + j * E) * 2;
                uint8_t* cp = st + dv.codes_off + (m - K) * P + j * E;
                uint8_t* mp = st + dv.meta_off + (m - K) * 8;
                if (hi) {
#pragma unroll
                    for (int w4 = 0; w4 < E / 8; ++w4) {
                        const uint4 v = reinterpret_cast<const uint4*>(hp)[w4];
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            t[8 * w4 + 2 * c] = __half2float(__ushort_as_half((unsigned short)(w[c] & 0xffffu)));
                            t[8 * w4 + 2 * c + 1] = __half2float(__ushort_as_half((unsigned short)(w[c] >> 16)));
                        }
                    }
                }
                if constexpr (MODE != 0) {
                    Chunk<E> c;
                    float delta = 0.0f, z = 0.0f;
                    if (!hi) {
#pragma unroll
                        for (int w4 = 0; w4 < E / 16; ++w4) {
                            const uint4 v = reinterpret_cast<const uint4*>(cp)[w4];
                            c.w[4 * w4] = v.x; c.w[4 * w4 + 1] = v.y;
                            c.w[4 * w4 + 2] = v.z; c.w[4 * w4 + 3] = v.w;
                        }
                        const float2 mz = *reinterpret_cast<const float2*>(mp);
                        delta = mz.x;
                        z = mz.y;
                    } else {
#pragma unroll
                        for (int w = 0; w < E / 4; ++w) c.w[w] = 0u;
                    }
                    float sd[E];
                    decode_row<SSQ_I8_ASYM, E>(c, delta, z, sd);   // warp-uniform inside
                    if (!hi) {
#pragma unroll
                        for (int e = 0; e < E; ++e) t[e] = sd[e];
                    }
                }
                // the recurrence on the rotated state: fma(lambda, t, fl(dtx * B_n))
                const float2 b2 = make_float2(bn, bn);
#pragma unroll
                for (int e = 0; e < E; e += 4) {
                    const float4 d4 = *reinterpret_cast<const float4*>(dtxj + e);
                    const float2 w0 = mul2(make_float2(d4.x, d4.y), b2);
                    const float2 w1 = mul2(make_float2(d4.z, d4.w), b2);
                    const float2 r0 = fma2(lam2, make_float2(t[e], t[e + 1]), w0);
                    const float2 r1 = fma2(lam2, make_float2(t[e + 2], t[e + 3]), w1);
                    t[e] = r0.x; t[e + 1] = r0.y; t[e + 2] = r1.x; t[e + 3] = r1.y;
                }
                if constexpr (MODE != 0) {
                    const RowParams rp = refit_row<SSQ_I8_ASYM, E, LPR>(t);
                    float rr[E];
                    uint32_t kk[E];
                    round_row<SSQ_I8_ASYM, E>(rp, t, rr, kk);
                    if (!hi) {
                        Chunk<E> c;
                        pack_codes<SSQ_I8_ASYM, E>(kk, c);
                        // readout of the stored value (q - z) * Delta as
                        // (C * Delta) * (q - z): y is fp32 with a tolerance
                        const float cd = __fmul_rn(cn, rp.delta);
                        const float2 cd2 = make_float2(cd, cd);
#pragma unroll
                        for (int e = 0; e < E; e += 2) {
                            const float2 r = fma2(cd2, make_float2(rr[e], rr[e + 1]),
                                                  make_float2(acc[e], acc[e + 1]));
                            acc[e] = r.x;
                            acc[e + 1] = r.y;
                        }
                        if (active) {
#pragma unroll
                            for (int w4 = 0; w4 < E / 16; ++w4)
                                reinterpret_cast<uint4*>(cp)[w4] =
                                    make_uint4(c.w[4 * w4], c.w[4 * w4 + 1], c.w[4 * w4 + 2],
                                               c.w[4 * w4 + 3]);
                            if (j == 0) {
                                *reinterpret_cast<float2*>(mp) = make_float2(rp.delta, rp.z);
                                if (!rp.finite) atomicOr(err, SSQ_DEVERR_NONFINITE);
                            }
                        }
                    }
                }
                if (hi) {
                    uint32_t hv[E / 2];
#pragma unroll
                    for (int w2 = 0; w2 < E / 2; ++w2) {
                        const __half a = __float2half_rn(t[2 * w2]);
                        const __half bb = __float2half_rn(t[2 * w2 + 1]);
                        hv[w2] = (uint32_t)__half_as_ushort(a) | ((uint32_t)__half_as_ushort(bb) << 16);
                        t[2 * w2] = __half2float(a);
                        t[2 * w2 + 1] = __half2float(bb);
                    }
                    if (active) {
#pragma unroll
                        for (int w4 = 0; w4 < E / 8; ++w4)
                            reinterpret_cast<uint4*>(hp)[w4] =
                                make_uint4(hv[4 * w4], hv[4 * w4 + 1], hv[4 * w4 + 2], hv[4 * w4 + 3]);
                    }
                    const float2 c2 = make_float2(cn, cn);
#pragma unroll
                    for (int e = 0; e < E; e += 2) {
                        const float2 r = fma2(c2, make_float2(t[e], t[e + 1]),
                                              make_float2(acc[e], acc[e + 1]));
                        acc[e] = r.x;
                        acc[e + 1] = r.y;
                    }
                }
            };
            // the passes that touch the FP16 tier, then the passes wholly in
            // the INT8 tier, then a ragged tail (d_state not a multiple of
            // the channels per pass)
            const int lo_begin = (K + PPW - 1) / PPW;
            const int lo_end = N / PPW > lo_begin ? N / PPW : lo_begin;
            for (int pass = 0; pass < passes; ++pass) {
                if (pass >= lo_begin && pass < lo_end)
                    pass_body(std::integral_constant<int, 1>(), pass);
                else
                    pass_body(std::integral_constant<int, 2>(), pass);
            }
            // readout: sum over the warp's positions, rotate back, add D x
            int base = 0;
            reduce_scatter<E, LPR, ROUNDS, E>(acc, lane, base);
            float v[KEEP];
#pragma unroll
            for (int e = 0; e < KEEP; ++e) v[e] = acc[e];
            fwht_readout<E, LPR, KEEP, 0, ilog2<P>()>(v, lane);
            // lanes that hold the same indices (KEEP = 1 with a spare reduce
            // round) write the same values
#pragma unroll
            for (int e = 0; e < KEEP; ++e) {
                const int p = j * E + base + e;
                dc.y[(lb * H + h) * P + p] = __fmaf_rn(Dh, xs[p], __fmul_rn(v[e], 1.0f / (float)P));
            }
            // the updated block goes back with one bulk store
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                uint8_t* head = dv.pool + dv.header_bytes + (long long)slot * dv.slot_bytes
                                + (long long)(dc.layer0 + l) * dv.layer_bytes
                                + (long long)h * dv.head_bytes;
                bulk_s2g(head, st, head_bytes);
                bulk_commit();
            }
            stored = true;
        }
        // release the previous head's stage once its store has read it
        if (lane == 0 && prev_s >= 0) {
            if (stored) bulk_wait_read<1>(); else bulk_wait_read<0>();
            mbar_arrive(&empty[prev_s]);
        }
        prev_s = s;
        __syncwarp();
    }
    if (lane == 0) {
        bulk_wait<0>();
        if (prev_s >= 0) mbar_arrive(&empty[prev_s]);
    }
}

template <int P>
cudaError_t launch_damp_p(const DampView& dv, const DampCall& dc, int which, cudaStream_t st)
{
    const long long units = (long long)dc.nl * dc.batch * dv.H;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (which == 0) {
        int optin = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        const int budget = optin < kDampSmemBudget ? optin : kDampSmemBudget;
        // as many stages as fit (at most kDampStages); a consumer holds its
        // stage while it computes, so the consumer warps take at most the
        // stages beyond 8 heads in flight (half the stages on a small ring)
        DampGeom g = damp_geom((int)dv.head_bytes, P, dv.N, 1, 1);
        int S = (budget - 256 - kDampCWarps * P * 4) / (g.stage_bytes + 16);
        if (S > kDampStages) S = kDampStages;
        if (S < 2) return cudaErrorInvalidConfiguration;
        int Wc = S >= 16 ? S - 8 : S / 2;
        if (Wc > kDampCWarps) Wc = kDampCWarps;
        g = damp_geom((int)dv.head_bytes, P, dv.N, S, Wc);
        auto k = damp_decode_pipe<P>;
        e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 g.smem_bytes);
        if (e != cudaSuccess) return e;
        const long long grid = units < sms ? units : sms;
        k<<<(int)grid, kDampPipeThreads, g.smem_bytes, st>>>(dv, dc, g);
    } else if (which == 1) {
        auto k = damp_quantize_kernel<P>;
        const int grid = grid_for((const void*)k, kThreads, units);
        if (grid <= 0) return cudaErrorInvalidConfiguration;
        k<<<grid, kThreads, 0, st>>>(dv, dc);
    } else {
        auto k = damp_dequantize_kernel<P>;
        const int grid = grid_for((const void*)k, kThreads, units);
        if (grid <= 0) return cudaErrorInvalidConfiguration;
        k<<<grid, kThreads, 0, st>>>(dv, dc);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_damp(const DampView& dv, const DampCall& dc, int which, cudaStream_t st)
{
    switch (dv.P) {
    case 16: return launch_damp_p<16>(dv, dc, which, st);
    case 32: return launch_damp_p<32>(dv, dc, which, st);
    case 64: return launch_damp_p<64>(dv, dc, which, st);
    case 128: return launch_damp_p<128>(dv, dc, which, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssq
