// ssq_scan.cu -- the per-token scan with the state rounded at every token.
//
// "ssm-state-quantization" README, Setup: a sequential per-token scan
// replaces the chunked library scan so that the state can be rounded at
// every step.  Here each CTA owns a fixed tile of rows of one request for
// all T tokens; the state stays in registers between tokens as the value the
// stored codes decode to (fl((q - z) * Delta)), so T tokens of the scan equal
// T decode steps bit for bit.  Only the final codes and metadata are written
// back.  The per-token inputs (x, dt, B, C) of a chunk of K tokens are staged
// into shared memory with cp.async one chunk ahead of the compute; lambda for
// each (token, head) is computed once per CTA.
#include "ssq_common.cuh"
#include "ssq_params.h"

namespace ssq {

namespace {

constexpr int kScanThreads = 64;
constexpr int kChunk = 8;  // tokens staged per shared-memory buffer

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem)
{
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;\n" ::);
}
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

struct ScanGeom {
    int rpc;    // rows per CTA
    int nh;     // max heads a tile touches (B/C are staged per touched head)
};

__host__ __device__ inline ScanGeom scan_geom(int N, int P, int H)
{
    ScanGeom g;
    const int E = N >= 32 ? 32 : N;
    g.rpc = kScanThreads / (N / E);
    // tiles start at multiples of rpc: when rpc divides P a tile lies in one
    // head, otherwise it spans at most floor((rpc-1)/P) + 2 heads
    g.nh = (P % g.rpc == 0) ? 1 : min(H, (g.rpc - 1) / P + 2);
    return g;
}

// Floats per shared-memory buffer: B and C [kChunk][nh][N], x [kChunk][rpc],
// dt and lambda [kChunk][nh].  A multiple of 8 floats, so both buffers stay
// 16-byte aligned.
__host__ __device__ inline int scan_buf_floats(const ScanGeom& g, int N)
{
    return 2 * kChunk * g.nh * N + kChunk * g.rpc + 2 * kChunk * g.nh;
}

template <int FMT, int N>
__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const __grid_constant__ PoolView pv, const __grid_constant__ CallView cv)
{
    using S = Shape<N>;
    using F = Fmt<FMT>;
    constexpr int E = S::E, LPR = S::LPR;
    constexpr int CB = F::quant ? E * F::bits / 8 : 4;
    constexpr bool kBf16 = (FMT == SSQ_BF16);
    extern __shared__ __align__(16) float smem[];

    const int P = pv.P, H = pv.H, G = pv.G, T = cv.T;
    const ScanGeom geo = scan_geom(N, P, H);
    const int bufsz = scan_buf_floats(geo, N);
    uint32_t* err = reinterpret_cast<uint32_t*>(pv.pool);

    // tile -> (request, region, first row)
    const int per_b = cv.qtiles + cv.ftiles;
    const int b = blockIdx.x / per_b;
    const int k = blockIdx.x - b * per_b;
    const bool quant = k < cv.qtiles;
    const int rbase = (quant ? k : k - cv.qtiles) * geo.rpc;
    const int nrows = (quant ? pv.Hq : pv.Hf) * P;
    const int regbase = quant ? 0 : pv.Hq;
    const int slot = cv.slot_idx ? __ldg(cv.slot_idx + b) : b;
    if (slot < 0 || slot >= pv.n_slots) {
        if (threadIdx.x == 0) atomicOr(err, SSQ_DEVERR_SLOT);
        return;  // block-uniform, before any barrier
    }
    const int rlast = min(rbase + geo.rpc, nrows) - 1;
    const int hr0 = rbase / P;
    const int nh = rlast / P - hr0 + 1;   // <= geo.nh

    const int tid = threadIdx.x;
    const int grow = tid / LPR;
    const int j = tid % LPR;
    const int r = rbase + grow;
    const bool active = r < nrows;
    const int rr = active ? r : rbase;
    const int hrl = rr / P;
    const int p = rr - hrl * P;
    const int h = pv.perm[regbase + hrl];
    const int hl = hrl - hr0;
    const float Av = __ldg(cv.A + h);
    const float Dv = __ldg(cv.D + h);

    // Stage the inputs of tokens [t0, t0 + kChunk) into buffer `bi`.
    auto stage = [&](int t0, int bi) {
        float* base = smem + bi * bufsz;
        float* sB = base;
        float* sC = sB + kChunk * geo.nh * N;
        float* sx = sC + kChunk * geo.nh * N;
        float* sdt = sx + kChunk * geo.rpc;
        const int nt = min(kChunk, T - t0);
        const int nvec = nt * nh * (N / 4);
        for (int i = tid; i < nvec; i += kScanThreads) {
            const int tt = i / (nh * (N / 4));
            const int rem = i - tt * nh * (N / 4);
            const int hh = rem / (N / 4);
            const int v = rem - hh * (N / 4);
            const int gg = pv.perm[regbase + hr0 + hh] / pv.hpg;
            const long long src = (((long long)b * T + t0 + tt) * G + gg) * N + 4 * v;
            const int dst = (tt * geo.nh + hh) * N + 4 * v;
            cp_async16(sB + dst, cv.B + src);
            cp_async16(sC + dst, cv.C + src);
        }
        const int nx = nt * geo.rpc;
        for (int i = tid; i < nx; i += kScanThreads) {
            const int tt = i / geo.rpc;
            const int row = rbase + (i - tt * geo.rpc);
            if (row < nrows) {
                const int hh = pv.perm[regbase + row / P];
                const int pp = row % P;
                cp_async4(sx + i, cv.x + (((long long)b * T + t0 + tt) * H + hh) * P + pp);
            }
        }
        const int nd = nt * nh;
        for (int i = tid; i < nd; i += kScanThreads) {
            const int tt = i / nh;
            const int hh = pv.perm[regbase + hr0 + (i - tt * nh)];
            cp_async4(sdt + tt * geo.nh + (i - tt * nh),
                      cv.dt + ((long long)b * T + t0 + tt) * H + hh);
        }
        cp_async_commit();
    };
    // lambda of every (token, head) of a staged buffer
    auto decays = [&](int t0, int bi) {
        float* base = smem + bi * bufsz;
        float* sdt = base + 2 * kChunk * geo.nh * N + kChunk * geo.rpc;
        float* slam = sdt + kChunk * geo.nh;
        const int nt = min(kChunk, T - t0);
        for (int i = tid; i < nt * nh; i += kScanThreads) {
            const int tt = i / nh;
            const int hh2 = i - tt * nh;
            const int hn = pv.perm[regbase + hr0 + hh2];
            slam[tt * geo.nh + hh2] = decay(sdt[tt * geo.nh + hh2], __ldg(cv.A + hn));
        }
    };

    uint8_t* slot_base = pv.pool + pv.header_bytes + (long long)slot * pv.slot_bytes;
    const int layer = cv.layer0;
    uint8_t* crow = nullptr;
    uint8_t* mrow = nullptr;
    uint8_t* frow = nullptr;
    constexpr int EB = kBf16 ? 2 : 4;

    // Initial state, decoded once.
    float s[E];
    bool qrow = false;
    if constexpr (F::quant) qrow = quant;
    if constexpr (F::quant) {
      if (qrow) {
        crow = slot_base + pv.codes_off + (long long)layer * pv.codes_layer_bytes
               + (long long)rr * (N * F::bits / 8) + j * CB;
        mrow = slot_base + pv.meta_off + (long long)layer * pv.meta_layer_bytes
               + (long long)rr * F::meta_bytes;
        Chunk<CB> c;
        load_chunk<CB>(c, crow);
        float delta0, z0 = 0.0f;
        if constexpr (F::sym) {
            delta0 = *reinterpret_cast<const float*>(mrow);
        } else {
            const float2 m = *reinterpret_cast<const float2*>(mrow);
            delta0 = m.x;
            z0 = m.y;
        }
        decode_row<FMT, E>(c, delta0, z0, s);
      }
    }
    if (!qrow) {
        frow = slot_base + pv.fp_off + (long long)layer * pv.fp_layer_bytes
               + ((long long)rr * N + j * E) * EB;
        if constexpr (kBf16) {
            Chunk<E * 2> c;
            load_chunk<E * 2>(c, frow);
#pragma unroll
            for (int n = 0; n < E; ++n)
                s[n] = __uint_as_float((c.w[n / 2] >> (16 * (n % 2))) << 16);
        } else {
            Chunk<E * 4> c;
            load_chunk<E * 4>(c, frow);
#pragma unroll
            for (int n = 0; n < E; ++n) s[n] = __uint_as_float(c.w[n]);
        }
    }

    stage(0, 0);
    cp_async_wait_all();
    __syncthreads();
    decays(0, 0);
    __syncthreads();

    RowParams rp{};
    uint32_t kfin[E];
    bool finite_all = true;
    const int nchunks = (T + kChunk - 1) / kChunk;
    for (int c = 0; c < nchunks; ++c) {
        const int bi = c & 1;
        const int t0 = c * kChunk;
        if (c + 1 < nchunks) stage(t0 + kChunk, bi ^ 1);
        const float* base = smem + bi * bufsz;
        const float* sB = base;
        const float* sC = sB + kChunk * geo.nh * N;
        const float* sx = sC + kChunk * geo.nh * N;
        const float* sdt = sx + kChunk * geo.rpc;
        const float* slam = sdt + kChunk * geo.nh;
        const int nt = min(kChunk, T - t0);
        for (int tt = 0; tt < nt; ++tt) {
            const float lam = slam[tt * geo.nh + hl];
            const float xv = sx[tt * geo.rpc + (active ? grow : 0)];
            const float dtx = __fmul_rn(sdt[tt * geo.nh + hl], xv);
            float Bv[E], Cv[E];
            const float* bp = sB + (tt * geo.nh + hl) * N + j * E;
            const float* cp = sC + (tt * geo.nh + hl) * N + j * E;
#pragma unroll
            for (int i = 0; i < E / 4; ++i) {
                const float4 vb = reinterpret_cast<const float4*>(bp)[i];
                Bv[4 * i] = vb.x; Bv[4 * i + 1] = vb.y; Bv[4 * i + 2] = vb.z; Bv[4 * i + 3] = vb.w;
            }
            update_row<E>(lam, dtx, Bv, s);
            if constexpr (F::quant) {
                if (qrow) {
                    rp = refit_row<FMT, E, LPR>(s);
                    finite_all = finite_all && rp.finite;
                    float rq[E];
                    round_row<FMT, E>(rp, s, rq, kfin, pv.neg_zero);
                    scale_row<E>(rp.delta, rq, s);
                }
            } else if constexpr (kBf16) {
#pragma unroll
                for (int n = 0; n < E; ++n)
                    s[n] = __bfloat162float(__float2bfloat16_rn(s[n]));
            }
#pragma unroll
            for (int i = 0; i < E / 4; ++i) {
                const float4 vc = reinterpret_cast<const float4*>(cp)[i];
                Cv[4 * i] = vc.x; Cv[4 * i + 1] = vc.y; Cv[4 * i + 2] = vc.z; Cv[4 * i + 3] = vc.w;
            }
            const float ysum = grp_sum<LPR>(dot_row<E>(Cv, s));
            if (active && j == 0) {
                const float yv = __fadd_rn(ysum, __fmul_rn(Dv, xv));
                __stcs(cv.y + (((long long)b * T + t0 + tt) * H + h) * P + p, yv);
            }
        }
        if (c + 1 < nchunks) {
            cp_async_wait_all();
            __syncthreads();               // staged data visible; old buffer free
            decays(t0 + kChunk, bi ^ 1);
            __syncthreads();
        }
    }

    // Final state back to the pool.
    if (active && qrow) {
        if constexpr (F::quant) {
            Chunk<CB> c;
            pack_codes<FMT, E>(kfin, c);
            store_chunk<CB>(crow, c);
            if (j == 0) {
                if constexpr (F::sym) {
                    *reinterpret_cast<float*>(mrow) = rp.delta;
                } else {
                    *reinterpret_cast<float2*>(mrow) = make_float2(rp.delta, rp.z);
                }
                if (!finite_all) atomicOr(err, SSQ_DEVERR_NONFINITE);
            }
        }
    } else if (active) {
        if constexpr (kBf16) {
            Chunk<E * 2> c;
#pragma unroll
            for (int n = 0; n < E; n += 2)
                c.w[n / 2] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(s[n]))
                             | ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(s[n + 1])) << 16);
            store_chunk<E * 2>(frow, c);
        } else {
            Chunk<E * 4> c;
#pragma unroll
            for (int n = 0; n < E; ++n) c.w[n] = __float_as_uint(s[n]);
            store_chunk<E * 4>(frow, c);
        }
    }
}

template <int FMT, int N>
cudaError_t launch_scan_n(const PoolView& pv, const CallView& cv, int grid,
                          cudaStream_t st)
{
    const ScanGeom g = scan_geom(N, pv.P, pv.H);
    const size_t smem = 2 * (size_t)scan_buf_floats(g, N) * sizeof(float);
    auto kern = scan_kernel<FMT, N>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, kScanThreads, smem, st>>>(pv, cv);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_scan_fmt(const PoolView& pv, const CallView& cv, int grid,
                            cudaStream_t st)
{
    switch (pv.N) {
    case 16: return launch_scan_n<FMT, 16>(pv, cv, grid, st);
    case 32: return launch_scan_n<FMT, 32>(pv, cv, grid, st);
    case 64: return launch_scan_n<FMT, 64>(pv, cv, grid, st);
    case 128: return launch_scan_n<FMT, 128>(pv, cv, grid, st);
    case 256: return launch_scan_n<FMT, 256>(pv, cv, grid, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int scan_rows_per_cta(int d_state)
{
    const int E = d_state >= 32 ? 32 : d_state;
    return kScanThreads / (d_state / E);
}

cudaError_t launch_scan(const PoolView& pv, const CallView& cv, int fmt,
                        cudaStream_t st)
{
    const long long grid = (long long)cv.batch * (cv.qtiles + cv.ftiles);
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    switch (fmt) {
    case SSQ_F32: return launch_scan_fmt<SSQ_F32>(pv, cv, (int)grid, st);
    case SSQ_BF16: return launch_scan_fmt<SSQ_BF16>(pv, cv, (int)grid, st);
    case SSQ_I8_SYM: return launch_scan_fmt<SSQ_I8_SYM>(pv, cv, (int)grid, st);
    case SSQ_I8_ASYM: return launch_scan_fmt<SSQ_I8_ASYM>(pv, cv, (int)grid, st);
    case SSQ_I4_SYM: return launch_scan_fmt<SSQ_I4_SYM>(pv, cv, (int)grid, st);
    case SSQ_I4_ASYM: return launch_scan_fmt<SSQ_I4_ASYM>(pv, cv, (int)grid, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssq
