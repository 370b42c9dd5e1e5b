// ssq_damp.cu -- the DAMP mixed-tier state: decode step, hand-off from fp32,
// read-back.
//
// "Mamba state quantization for inference", "Mixed precision spends bits on
// persistent channels": a Hadamard transform along each key channel's value
// dimension; the protected key channels kept in FP16, the rest in INT8 with a
// scale and a zero point; the tiers permuted into contiguous regions so one
// fused kernel loads both without a per-token gather; per token the kernel
// reconstructs the low tier, runs the recurrence in FP32, derives new
// quantization parameters and writes the packed state back.
//
// Per head the state is N key channels ("positions" m = 0..N-1 after the
// caller's channel permutation chan[layer][h][m]; positions < K form the
// FP16 tier) of P rotated values t[m][k] = sum_p H[k][p] S[p][chan[m]], H the
// +-1 Sylvester-Hadamard matrix.  The recurrence is linear, so it runs on the
// rotated state with the rotated input xr = H x:
//   t'[m][k] = fma(lambda, t[m][k], fl(fl(dt * xr[k]) * B[chan[m]]))
// and the readout rotates back once per head:
//   y[p] = D x[p] + (1/P) sum_k H[p][k] sum_m C[chan[m]] stored'[m][k].
// xr[k] is summed in double in the order p = 0..P-1 and rounded once, so
// every stored code, step, zero point and FP16 value is bit-identical to a
// plain scalar evaluation; y accumulates in fp32.
//
// Thread mapping: one CTA of 256 threads per (layer, request, head) unit in
// a grid-stride loop; a position's P values sit on LPR = P/16 consecutive
// lanes, 16 per lane; a warp covers 32/LPR positions per pass.
#include <cuda_fp16.h>

#include "ssq_common.cuh"
#include "ssq_params.h"

namespace ssq {

namespace {

constexpr int kDampE = 16;   // rotated entries per lane

__device__ __forceinline__ bool hneg(int a, int b) { return (__popc(a & b) & 1) != 0; }

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
// Decode step
// ---------------------------------------------------------------------------
template <int P>
__global__ void __launch_bounds__(kThreads, 2)
damp_decode_kernel(const __grid_constant__ DampView dv, const __grid_constant__ DampCall dc)
{
    constexpr int E = kDampE, LPR = P / E, PPW = 32 / LPR;
    constexpr int ROUNDS = ilog2<PPW>();
    constexpr int NW = kThreads / 32;
    __shared__ float s_x[P];         // x of the head
    __shared__ float s_dtx[P];       // fl(dt * xr[k])
    __shared__ float s_red[NW][P];   // per-warp readout partials (rotated)
    __shared__ float s_yr[P];        // rotated readout

    uint32_t* err = reinterpret_cast<uint32_t*>(dv.pool);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int j = tid % LPR;
    const int passes = (dv.N * LPR + kThreads - 1) / kThreads;
    const long long units = (long long)dc.nl * dc.batch * dv.H;

    for (long long uu = blockIdx.x; uu < units; uu += gridDim.x) {
        const DampUnit u = damp_unit(dv, dc, uu);
        if (u.slot < 0 || u.slot >= dv.n_slots) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_SLOT);
            continue;   // uniform over the CTA
        }
        if (!damp_chan_ok(dv, u, tid)) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_CHANNEL);
            continue;
        }
        const float dtv = __ldg(dc.dt + u.lb * dv.H + u.h);
        const float lam = decay(dtv, __ldg(dc.A + (long long)u.l * dv.H + u.h));
        const float* xh = dc.x + (u.lb * dv.H + u.h) * P;
        if (tid < P) s_x[tid] = __ldg(xh + tid);
        __syncthreads();
        if (tid < P) {
            // xr[k] = sum_p H[k][p] x[p], double, order p, rounded once
            double acc = 0.0;
#pragma unroll 8
            for (int p = 0; p < P; ++p) {
                const double v = (double)s_x[p];
                acc = hneg(tid, p) ? __dsub_rn(acc, v) : __dadd_rn(acc, v);
            }
            s_dtx[tid] = __fmul_rn(dtv, __double2float_rn(acc));
        }
        __syncthreads();

        float acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.0f;
        for (int pass = 0; pass < passes; ++pass) {
            const DampPos ps = damp_pos<LPR>(dv, u, pass, tid);
            const float bn = __ldg(dc.B + (u.lb * dv.G + u.g) * dv.N + ps.n);
            const float cn = ps.active ? __ldg(dc.C + (u.lb * dv.G + u.g) * dv.N + ps.n) : 0.0f;
            float t[E];
            damp_load(dv, u, ps, j, t);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float w = __fmul_rn(s_dtx[j * E + e], bn);
                t[e] = __fmaf_rn(lam, t[e], w);
            }
            damp_store<LPR>(dv, u, ps, j, t, ps.active, err);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = ps.active ? __fmaf_rn(cn, t[e], acc[e]) : acc[e];
        }
        // readout: sum over positions (warp butterfly, then across warps)
        int base = 0;
        reduce_scatter<E, LPR, ROUNDS, E>(acc, lane, base);
        constexpr int KEEP = (E >> ROUNDS) > 0 ? (E >> ROUNDS) : 1;
#pragma unroll
        for (int i = 0; i < KEEP; ++i) s_red[warp][j * E + base + i] = acc[i];
        __syncthreads();
        if (tid < P) {
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < NW; ++w) v = __fadd_rn(v, s_red[w][tid]);
            s_yr[tid] = v;
        }
        __syncthreads();
        if (tid < P) {
            float v = 0.0f;
#pragma unroll 8
            for (int k = 0; k < P; ++k)
                v = hneg(tid, k) ? __fsub_rn(v, s_yr[k]) : __fadd_rn(v, s_yr[k]);
            const float Dh = __ldg(dc.D + (long long)u.l * dv.H + u.h);
            dc.y[(u.lb * dv.H + u.h) * P + tid] =
                __fmaf_rn(Dh, s_x[tid], __fmul_rn(v, 1.0f / (float)P));
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Hand-off: fp32 S[nl][batch][H][P][N] -> tiers
// ---------------------------------------------------------------------------
template <int P>
__global__ void __launch_bounds__(kThreads)
damp_quantize_kernel(const __grid_constant__ DampView dv, const __grid_constant__ DampCall dc)
{
    constexpr int E = kDampE, LPR = P / E;
    uint32_t* err = reinterpret_cast<uint32_t*>(dv.pool);
    const int tid = threadIdx.x;
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
            // t[k] = sum_p H[k][p] S[p][n], double, order p, rounded once
            double a[E];
#pragma unroll
            for (int e = 0; e < E; ++e) a[e] = 0.0;
            for (int p = 0; p < P; ++p) {
                const double v = (double)__ldg(S + (long long)p * dv.N + ps.n);
#pragma unroll
                for (int e = 0; e < E; ++e)
                    a[e] = hneg(j * E + e, p) ? __dsub_rn(a[e], v) : __dadd_rn(a[e], v);
            }
            float t[E];
#pragma unroll
            for (int e = 0; e < E; ++e) t[e] = __double2float_rn(a[e]);
            damp_store<LPR>(dv, u, ps, j, t, ps.active, err);
        }
    }
}

// ---------------------------------------------------------------------------
// Read-back: tiers -> fp32 S[nl][batch][H][P][N]
// ---------------------------------------------------------------------------
template <int P>
__global__ void __launch_bounds__(kThreads)
damp_dequantize_kernel(const __grid_constant__ DampView dv, const __grid_constant__ DampCall dc)
{
    constexpr int E = kDampE, LPR = P / E;
    extern __shared__ float s_t[];   // [N][P] stored (rotated) values
    uint32_t* err = reinterpret_cast<uint32_t*>(dv.pool);
    const int tid = threadIdx.x;
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
        for (int pass = 0; pass < passes; ++pass) {
            const DampPos ps = damp_pos<LPR>(dv, u, pass, tid);
            float t[E];
            damp_load(dv, u, ps, j, t);
            if (ps.active) {
#pragma unroll
                for (int e = 0; e < E; ++e) s_t[ps.m * P + j * E + e] = t[e];
            }
        }
        __syncthreads();
        float* S = dc.S_out + (u.lb * dv.H + u.h) * (long long)P * dv.N;
        for (int idx = tid; idx < dv.N * P; idx += kThreads) {
            const int m = idx / P, p = idx - m * P;
            const int n = __ldg(u.chan + m);
            // S[p][n] = (1/P) sum_k H[p][k] t[m][k], double, order k
            double a = 0.0;
            for (int k = 0; k < P; ++k) {
                const double v = (double)s_t[m * P + k];
                a = hneg(p, k) ? __dsub_rn(a, v) : __dadd_rn(a, v);
            }
            S[(long long)p * dv.N + n] = __double2float_rn(__dmul_rn(a, 1.0 / (double)P));
        }
        __syncthreads();
    }
}

template <int P>
cudaError_t launch_damp_p(const DampView& dv, const DampCall& dc, int which, cudaStream_t st)
{
    const long long units = (long long)dc.nl * dc.batch * dv.H;
    if (which == 0) {
        auto k = damp_decode_kernel<P>;
        const int grid = grid_for((const void*)k, kThreads, units);
        if (grid <= 0) return cudaErrorInvalidConfiguration;
        k<<<grid, kThreads, 0, st>>>(dv, dc);
    } else if (which == 1) {
        auto k = damp_quantize_kernel<P>;
        const int grid = grid_for((const void*)k, kThreads, units);
        if (grid <= 0) return cudaErrorInvalidConfiguration;
        k<<<grid, kThreads, 0, st>>>(dv, dc);
    } else {
        auto k = damp_dequantize_kernel<P>;
        const size_t smem = (size_t)dv.N * P * sizeof(float);
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute((const void*)k,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (e != cudaSuccess) return e;
        }
        int dev = 0, sms = 0, occ = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, (const void*)k, kThreads, smem);
        if (e != cudaSuccess) return e;
        long long grid = (long long)sms * (occ < 1 ? 1 : occ);
        if (grid > units) grid = units;
        k<<<(int)grid, kThreads, smem, st>>>(dv, dc);
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
