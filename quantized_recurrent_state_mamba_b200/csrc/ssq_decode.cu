// ssq_decode.cu -- the fused decode-step kernel.
//
// One launch updates the state of nl layers x batch requests by one token:
// read the packed row, decode, apply the recurrence in fp32, refit the row
// scale, requantize, write the packed row and its metadata back, and read y
// from the newly stored row -- the single fused pass that "Mamba state
// quantization for inference" describes for a low-bit state ("reconstructs
// the low tier, computes the recurrence in FP32, derives new quantization
// parameters, and writes the packed state back"), with the quantizer of
// "ssm-state-quantization" README, Setup.
//
// Structure (persistent, warp-specialised, two CTAs per SM):
//   - work is a sequence of tiles (up to RPT rows of one region of one
//     (layer, request)); each CTA owns a contiguous range of that sequence;
//   - a producer warp streams each tile's packed rows and metadata from HBM
//     into a ring of shared-memory stages with bulk asynchronous copies
//     (cp.async.bulk, completion counted in bytes on an mbarrier) and the
//     tile's x values with cp.async; once per (layer, request, region)
//     "unit" it stages B, C, dt, A, D into one of two unit buffers;
//   - 8 consumer warps compute from shared memory and store the new rows,
//     metadata and y straight to global memory;
//   - every wait is bounded: a wait that runs out sets SSQ_DEVERR_TIMEOUT in
//     the pool's error word and the CTA winds down (the producer first waits
//     for its own copies in flight).
#include "ssq_common.cuh"
#include "ssq_params.h"

namespace ssq {

namespace {

constexpr int kCWarps = 7;  // + 1 producer: 8-warp CTAs, two per SM
constexpr int kCThreads = kCWarps * 32;
constexpr int kDThreads = kCThreads + 32;
constexpr int kMaxStages = 8;
constexpr long long kWaitLimit = 2000000000LL;  // clock cycles, about one second

// ---- PTX wrappers -------------------------------------------------------
__device__ __forceinline__ unsigned saddr(const void* p)
{
    return (unsigned)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* b, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(saddr(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, unsigned parity)
{
    unsigned ok;
    asm volatile("{\n .reg .pred p;\n"
                 " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
                 " selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok) : "r"(saddr(b)), "r"(parity) : "memory");
    return ok != 0;
}
// Wait for the phase of the given parity to complete; false after about a
// second without progress.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, unsigned parity)
{
    if (mbar_try(b, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try(b, parity))
        if (clock64() - t0 > kWaitLimit) return false;
    return true;
}
// Bulk copy global -> shared; completion counted in bytes on `bar`.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(saddr(dst)), "l"(src), "r"(bytes), "r"(saddr(bar)) : "memory");
}
__device__ __forceinline__ void cpa4(void* dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(saddr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa16(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr(dst)), "l"(src) : "memory");
}
// The mbarrier's current phase also waits for this thread's earlier cp.async.
__device__ __forceinline__ void cpa_arrive(uint64_t* b)
{
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(saddr(b)) : "memory");
}

__host__ __device__ inline int r16(int v) { return (v + 15) & ~15; }

// ---- tile sequence -----------------------------------------------------
// Tiles are ordered (layer, request, region, row block).  A CTA walks a
// contiguous range of them with counters (one division at the start).
struct TileWalk {
    long long lb;   // layer * batch + request
    int l, b, k;    // k: tile within (layer, request)
    bool quant;
    int rbase, n;   // first region row, rows in this tile
    long long key;  // unit key: (lb, region)

    __device__ __forceinline__ void fill(const PoolView& pv, const CallView& cv)
    {
        quant = k < cv.qtiles;
        rbase = (quant ? k : k - cv.qtiles) * cv.rows_per_tile;
        const int nrows = (quant ? pv.Hq : pv.Hf) * pv.P;
        n = min(cv.rows_per_tile, nrows - rbase);
        key = lb * 2 + (quant ? 0 : 1);
    }
    __device__ __forceinline__ void start(const PoolView& pv, const CallView& cv, long long t)
    {
        const int per_lb = cv.qtiles + cv.ftiles;
        lb = t / per_lb;
        k = (int)(t - lb * per_lb);
        l = (int)(lb / cv.batch);
        b = (int)(lb - (long long)l * cv.batch);
        fill(pv, cv);
    }
    __device__ __forceinline__ void next(const PoolView& pv, const CallView& cv)
    {
        if (++k == cv.qtiles + cv.ftiles) {
            k = 0;
            ++lb;
            if (++b == cv.batch) {
                b = 0;
                ++l;
            }
        }
        fill(pv, cv);
    }
};

// ---- shared-memory geometry (host and device agree on it) --------------
struct DecodeGeom {
    int S;            // stages
    int RPT;          // rows per tile
    int x_bytes;      // x area of a stage
    int qcodes_bytes; // codes area of a quantized tile
    int pay_bytes;    // payload area of a stage
    int stage_bytes;
    int ub_B, ub_C, ub_dt, ub_A, ub_D, unit_bytes;  // unit buffer layout
    int Hpad;         // floats per lambda array
    int off_units, off_lam, off_stages, smem_bytes;
};

__host__ __device__ inline DecodeGeom decode_geom(int S, int RPT, int RB, int MB, int fpEB,
                                                  bool has_fp, int N, int H, int G)
{
    DecodeGeom g;
    g.S = S;
    g.RPT = RPT;
    g.x_bytes = r16(RPT * 4);
    g.qcodes_bytes = r16(RPT * RB);
    const int qpay = g.qcodes_bytes + r16(RPT * MB);
    const int fpay = has_fp ? RPT * N * fpEB : 0;
    g.pay_bytes = qpay > fpay ? qpay : fpay;
    g.stage_bytes = g.x_bytes + g.pay_bytes;
    g.Hpad = (H + 3) & ~3;
    g.ub_B = 16;  // 16-byte header: slot, bad flag
    g.ub_C = g.ub_B + G * N * 4;
    g.ub_dt = g.ub_C + G * N * 4;
    g.ub_A = g.ub_dt + g.Hpad * 4;
    g.ub_D = g.ub_A + g.Hpad * 4;
    g.unit_bytes = r16(g.ub_D + g.Hpad * 4);
    const int bars = r16((2 * kMaxStages + 4) * 8);
    g.off_units = bars;
    g.off_lam = g.off_units + 2 * g.unit_bytes;
    g.off_stages = r16(g.off_lam + kCWarps * 2 * g.Hpad * 4);
    g.smem_bytes = g.off_stages + S * g.stage_bytes;
    return g;
}

// Lane shape of the decode kernel: quantized rows give each lane 64 entries
// (two lanes per 128-entry row), which halves the per-row and per-tile
// bookkeeping per entry; fp rows keep 32 entries per lane.
template <int FMT, int N>
struct DShape {
    static constexpr int E = Fmt<FMT>::quant ? (N >= 64 ? 64 : N) : (N >= 32 ? 32 : N);
    static constexpr int LPR = N / E;
};

template <int FMT, int N>
__global__ void __launch_bounds__(kDThreads, 2)
decode_kernel(const __grid_constant__ PoolView pv, const __grid_constant__ CallView cv,
              const __grid_constant__ DecodeGeom geo)
{
    using F = Fmt<FMT>;
    constexpr int E = DShape<FMT, N>::E, LPR = DShape<FMT, N>::LPR;
    constexpr bool kBf16 = (FMT == SSQ_BF16);
    constexpr int RB = F::quant ? N * F::bits / 8 : 0;      // code bytes per row
    constexpr int CB = F::quant ? E * F::bits / 8 : 16;     // code bytes per lane
    constexpr int MB = F::meta_bytes;
    constexpr int FEB = kBf16 ? 2 : 4;                       // fp element bytes
    constexpr int CPL = E / 4;                               // B/C 16-byte chunks per lane

    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* ufull = empty + kMaxStages;
    uint64_t* uempty = ufull + 2;
    uint32_t* err = reinterpret_cast<uint32_t*>(pv.pool);

    const int S = geo.S;
    const int H = pv.H, P = pv.P, G = pv.G;
    const long long total = cv.total_tiles;
    const long long t0 = total * blockIdx.x / gridDim.x;
    const long long t1 = total * (blockIdx.x + 1) / gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCWarps);
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(&ufull[u], 1);
            mbar_init(&uempty[u], kCWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    uint8_t* const units = smem + geo.off_units;
    uint8_t* const stages = smem + geo.off_stages;

    if (warp == kCWarps) {
        // ================= producer warp =================
        int si = 0, sph = 0, k = 0, uk = -1;
        long long prev = -1;
        bool bad = false, ok = true;
        const uint8_t* codes_u = nullptr;
        const uint8_t* meta_u = nullptr;
        const uint8_t* fp_u = nullptr;
        const float* x_u = nullptr;
        TileWalk ti;
        ti.start(pv, cv, t0);
        for (long long t = t0; t < t1; ++t, ti.next(pv, cv)) {
            const int regbase = ti.quant ? 0 : pv.Hq;
            if (ti.key != prev) {
                prev = ti.key;
                ++uk;
                const int u = uk & 1;
                if (!mbar_wait(&uempty[u], ((uk >> 1) & 1) ^ 1)) { ok = false; break; }
                const int slot = cv.slot_idx ? __ldg(cv.slot_idx + ti.b) : ti.b;
                bad = slot < 0 || slot >= pv.n_slots;
                uint8_t* ub = units + u * geo.unit_bytes;
                if (lane == 0) {
                    reinterpret_cast<int*>(ub)[0] = slot;
                    reinterpret_cast<int*>(ub)[1] = bad ? 1 : 0;
                    if (bad) atomicOr(err, SSQ_DEVERR_SLOT);
                }
                if (!bad) {
                    const int layer = cv.layer0 + ti.l;
                    const uint8_t* sb = pv.pool + pv.header_bytes + (long long)slot * pv.slot_bytes;
                    codes_u = sb + pv.codes_off + (long long)layer * pv.codes_layer_bytes;
                    meta_u = sb + pv.meta_off + (long long)layer * pv.meta_layer_bytes;
                    fp_u = sb + pv.fp_off + (long long)layer * pv.fp_layer_bytes;
                    x_u = cv.x + ti.lb * H * P;
                    // B and C in 16-byte chunks.  In quantized units lane j
                    // of a row owns chunks j*CPL .. j*CPL+CPL-1; chunk i of
                    // lane j is stored at i*LPR + j, so at each step the
                    // lanes of a row read consecutive chunks (distinct banks)
                    // at compile-time offsets from a per-lane base.
                    float* dB = reinterpret_cast<float*>(ub + geo.ub_B);
                    float* dC = reinterpret_cast<float*>(ub + geo.ub_C);
                    const float* sB = cv.B + ti.lb * G * N;
                    const float* sC = cv.C + ti.lb * G * N;
                    for (int m = lane; m < G * N / 4; m += 32) {
                        int pos = m;
                        if (ti.quant) {
                            const int gi = m / (N / 4), mm = m - gi * (N / 4);
                            const int jj = mm / CPL, ii = mm - jj * CPL;
                            pos = gi * (N / 4) + ii * LPR + jj;
                        }
                        cpa16(dB + 4 * pos, sB + 4 * m);
                        cpa16(dC + 4 * pos, sC + 4 * m);
                    }
                    float* ddt = reinterpret_cast<float*>(ub + geo.ub_dt);
                    float* dA = reinterpret_cast<float*>(ub + geo.ub_A);
                    float* dD = reinterpret_cast<float*>(ub + geo.ub_D);
                    for (int h = lane; h < H; h += 32) {
                        cpa4(ddt + h, cv.dt + ti.lb * H + h);
                        cpa4(dA + h, cv.A + (long long)ti.l * H + h);
                        cpa4(dD + h, cv.D + (long long)ti.l * H + h);
                    }
                }
                cpa_arrive(&ufull[u]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&ufull[u]);
            }
            if (bad) continue;
            if (!mbar_wait(&empty[si], sph ^ 1)) { ok = false; break; }
            uint8_t* st = stages + si * geo.stage_bytes;
            float* sx = reinterpret_cast<float*>(st);
            for (int i = lane; i < ti.n; i += 32) {
                const int rr = ti.rbase + i;
                const int hr = fdiv(rr, pv.mP);
                const int hh = pv.perm[regbase + hr];
                cpa4(sx + i, x_u + hh * P + (rr - hr * P));
            }
            cpa_arrive(&full[si]);
            __syncwarp();
            if (lane == 0) {
                uint8_t* pay = st + geo.x_bytes;
                if (F::quant && ti.quant) {
                    const unsigned cb = (unsigned)r16(ti.n * RB), mb = (unsigned)r16(ti.n * MB);
                    mbar_arrive_tx(&full[si], cb + mb);
                    bulk_g2s(pay, codes_u + (long long)ti.rbase * RB, cb, &full[si]);
                    bulk_g2s(pay + geo.qcodes_bytes, meta_u + (long long)ti.rbase * MB, mb,
                             &full[si]);
                } else {
                    const unsigned fb = (unsigned)(ti.n * N * FEB);
                    mbar_arrive_tx(&full[si], fb);
                    bulk_g2s(pay, fp_u + (long long)ti.rbase * N * FEB, fb, &full[si]);
                }
            }
            ++k;
            if (++si == S) { si = 0; sph ^= 1; }
        }
        if (!ok && lane == 0) atomicOr(err, SSQ_DEVERR_TIMEOUT);
        // No copy may still be writing shared memory when the CTA exits.
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0) {
            for (int jj = (k > S ? k - S : 0); jj < k; ++jj)
                mbar_wait(&full[jj % S], (jj / S) & 1);
        }
        return;
    }

    // ================= consumer warps =================
    const int ct = threadIdx.x;
    const int grow = ct / LPR;
    const int j = ct % LPR;
    int si = 0, sph = 0, uk = -1;
    long long prev = -1;
    bool bad = false;
    const uint8_t* ub = units;
    float* lam = nullptr;
    uint8_t* codes_u = nullptr;
    uint8_t* meta_u = nullptr;
    uint8_t* fp_u = nullptr;
    float* y_u = nullptr;

    TileWalk ti;
    ti.start(pv, cv, t0);
    for (long long t = t0; t < t1; ++t, ti.next(pv, cv)) {
        if (ti.key != prev) {
            if (uk >= 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&uempty[uk & 1]);
            }
            prev = ti.key;
            ++uk;
            const int u = uk & 1;
            if (!mbar_wait(&ufull[u], (uk >> 1) & 1)) {
                if (lane == 0) atomicOr(err, SSQ_DEVERR_TIMEOUT);
                break;
            }
            ub = units + u * geo.unit_bytes;
            const int slot = reinterpret_cast<const int*>(ub)[0];
            bad = reinterpret_cast<const int*>(ub)[1] != 0;
            lam = reinterpret_cast<float*>(smem + geo.off_lam) + (warp * 2 + u) * geo.Hpad;
            if (!bad) {
                const int layer = cv.layer0 + ti.l;
                uint8_t* sb = pv.pool + pv.header_bytes + (long long)slot * pv.slot_bytes;
                codes_u = sb + pv.codes_off + (long long)layer * pv.codes_layer_bytes;
                meta_u = sb + pv.meta_off + (long long)layer * pv.meta_layer_bytes;
                fp_u = sb + pv.fp_off + (long long)layer * pv.fp_layer_bytes;
                y_u = cv.y + ti.lb * H * P;
                const float* udt = reinterpret_cast<const float*>(ub + geo.ub_dt);
                const float* uA = reinterpret_cast<const float*>(ub + geo.ub_A);
                for (int h = lane; h < H; h += 32) lam[h] = decay(udt[h], uA[h]);
                __syncwarp();
            }
        }
        if (bad) continue;
        if (!mbar_wait(&full[si], sph)) {
            if (lane == 0) atomicOr(err, SSQ_DEVERR_TIMEOUT);
            break;
        }
        const uint8_t* st = stages + si * geo.stage_bytes;
        const float* sx = reinterpret_cast<const float*>(st);
        const uint8_t* pay = st + geo.x_bytes;
        const int regbase = ti.quant ? 0 : pv.Hq;
        const bool active = grow < ti.n;
        const int rl = active ? grow : 0;          // inactive rows shadow row 0
        const int rr = ti.rbase + rl;
        const int hrl = fdiv(rr, pv.mP);
        const int p = rr - hrl * P;
        const int h = pv.perm[regbase + hrl];
        const int g = fdiv(h, pv.mHpg);
        const float xv = sx[rl];
        const float lamv = lam[h];
        const float dtv = reinterpret_cast<const float*>(ub + geo.ub_dt)[h];
        const float Dv = reinterpret_cast<const float*>(ub + geo.ub_D)[h];
        const float dtx = __fmul_rn(dtv, xv);
        const float* gB = reinterpret_cast<const float*>(ub + geo.ub_B) + g * N;
        const float* gC = reinterpret_cast<const float*>(ub + geo.ub_C) + g * N;
        float ysum = 0.0f;
        bool done = false;

        if constexpr (F::quant) {
            if (ti.quant) {
                done = true;
                constexpr int PW = Piece<FMT>::words;        // words per 16 entries
                constexpr int NP = E / 16;                   // 16-entry pieces per lane
                uint32_t cw[CB / 4];
                {
                    const uint8_t* cs = pay + rl * RB + j * CB;
                    if constexpr (CB % 16 == 0) {
#pragma unroll
                        for (int i = 0; i < CB / 16; ++i) {
                            const uint4 v = reinterpret_cast<const uint4*>(cs)[i];
                            cw[4 * i] = v.x; cw[4 * i + 1] = v.y; cw[4 * i + 2] = v.z; cw[4 * i + 3] = v.w;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < CB / 8; ++i) {
                            const uint2 v = reinterpret_cast<const uint2*>(cs)[i];
                            cw[2 * i] = v.x; cw[2 * i + 1] = v.y;
                        }
                    }
                }
                float delta0, z0 = 0.0f;
                {
                    const uint8_t* ms = pay + geo.qcodes_bytes + rl * MB;
                    if constexpr (F::sym) {
                        delta0 = *reinterpret_cast<const float*>(ms);
                    } else {
                        const float2 m = *reinterpret_cast<const float2*>(ms);
                        delta0 = m.x;
                        z0 = m.y;
                    }
                }
                // decode + update, 16 entries at a time, tracking min / max
                float s[E];
                float plo[NP], phi[NP];                      // per-piece min / max
                const bool dfast = F::sym || __all_sync(0xffffffffu, fabsf(z0) < kFastLimit);
                const float c0 = __fadd_rn(kTwo23, __fadd_rn(z0, F::bias));
                const float4* b4 = reinterpret_cast<const float4*>(gB) + j;
#pragma unroll
                for (int pc = 0; pc < NP; ++pc) {
                    float* sp = s + 16 * pc;
                    if (dfast) {
                        float f[16];
                        unpack16_biased<FMT>(cw + PW * pc, f);
                        const float2 nc02 = make_float2(-c0, -c0);
                        const float2 d2 = make_float2(delta0, delta0);
#pragma unroll
                        for (int n = 0; n < 16; n += 2) {
                            float2 v = mul2(add2(make_float2(f[n], f[n + 1]), nc02), d2);
                            sp[n] = v.x; sp[n + 1] = v.y;
                        }
                    } else {
                        int q[16];
                        unpack16_int<FMT>(cw + PW * pc, q);
#pragma unroll
                        for (int n = 0; n < 16; ++n)
                            sp[n] = __fmul_rn(__fsub_rn((float)q[n], z0), delta0);
                    }
                    float Bv[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float4 v = b4[(4 * pc + i) * LPR];
                        Bv[4 * i] = v.x; Bv[4 * i + 1] = v.y; Bv[4 * i + 2] = v.z; Bv[4 * i + 3] = v.w;
                    }
                    const float2 l2 = make_float2(lamv, lamv);
                    const float2 x2 = make_float2(dtx, dtx);
#pragma unroll
                    for (int n = 0; n < 16; n += 2) {
                        const float2 w = mul2(x2, make_float2(Bv[n], Bv[n + 1]));
                        const float2 v = fma2(l2, make_float2(sp[n], sp[n + 1]), w);
                        sp[n] = v.x; sp[n + 1] = v.y;
                    }
                    minmax16(sp, plo[pc], phi[pc]);
                }
                float lo = plo[0], hi = phi[0];
#pragma unroll
                for (int pc = 1; pc < NP; ++pc) {
                    lo = fminf(lo, plo[pc]);
                    hi = fmaxf(hi, phi[pc]);
                }
                const RowParams rp = refit_from_minmax<FMT, LPR>(lo, hi);
                const bool fast = __all_sync(0xffffffffu, rp.fast && !rp.clamp);
                // round, pack and read back, 16 entries at a time
                const float4* c4 = reinterpret_cast<const float4*>(gC) + j;
                float2 accp[NP];                             // one accumulator per piece
#pragma unroll
                for (int pc = 0; pc < NP; ++pc) {
                    float2& acc = accp[pc];
                    acc = make_float2(0.0f, 0.0f);
                    float r[16];
                    uint32_t kk[16];
                    if (fast) {
                        round16_fast<FMT>(rp, s + 16 * pc, r, kk, pv.neg_zero);
                    } else {
                        round16_slow<FMT>(rp, s + 16 * pc, r, kk);
#pragma unroll
                        for (int n = 0; n < 16; ++n) r[n] = __fmul_rn(r[n], rp.delta);
                    }
                    pack16<FMT>(kk, cw + PW * pc);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float4 v = c4[(4 * pc + i) * LPR];
                        acc = fma2(make_float2(v.x, v.y), make_float2(r[4 * i], r[4 * i + 1]), acc);
                        acc = fma2(make_float2(v.z, v.w), make_float2(r[4 * i + 2], r[4 * i + 3]), acc);
                    }
                }
                // fast: acc = sum C (q - z), scaled by Delta once; slow: acc
                // already sums C * fl((q - z) * Delta)
                float2 acc = accp[0];
#pragma unroll
                for (int pc = 1; pc < NP; ++pc) acc = add2(acc, accp[pc]);
                const float part = __fadd_rn(acc.x, acc.y);
                ysum = fast ? __fmul_rn(rp.delta, grp_sum<LPR>(part)) : grp_sum<LPR>(part);
                if (active) {
                    uint8_t* crow = codes_u + (long long)rr * RB + j * CB;
                    if constexpr (CB % 16 == 0) {
#pragma unroll
                        for (int i = 0; i < CB / 16; ++i)
                            __stcs(reinterpret_cast<uint4*>(crow) + i,
                                   make_uint4(cw[4 * i], cw[4 * i + 1], cw[4 * i + 2], cw[4 * i + 3]));
                    } else {
#pragma unroll
                        for (int i = 0; i < CB / 8; ++i)
                            __stcs(reinterpret_cast<uint2*>(crow) + i, make_uint2(cw[2 * i], cw[2 * i + 1]));
                    }
                    if (j == 0) {
                        uint8_t* mrow = meta_u + (long long)rr * MB;
                        if constexpr (F::sym) {
                            __stcs(reinterpret_cast<float*>(mrow), rp.delta);
                        } else {
                            __stcs(reinterpret_cast<float2*>(mrow), make_float2(rp.delta, rp.z));
                        }
                        if (!rp.finite) atomicOr(err, SSQ_DEVERR_NONFINITE);
                    }
                }
            }
        }
        if (!done) {
            // fp row (fp32, or bf16 for the bf16 format), streamed one 16-byte
            // storage chunk at a time.  Lane j owns chunks LPR*c + j, so the
            // lanes of a row touch consecutive chunks.
            constexpr int EPC = 16 / FEB;           // elements per chunk
            constexpr int NCH = E / EPC;            // chunks per lane
            const uint8_t* fs = pay + (long long)rl * N * FEB;
            uint8_t* frow = fp_u + (long long)rr * N * FEB;
            const float2 l2 = make_float2(lamv, lamv);
            const float2 x2 = make_float2(dtx, dtx);
            float2 acc = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int m = LPR * c + j;
                const uint4 v = reinterpret_cast<const uint4*>(fs)[m];
                uint32_t w[4] = {v.x, v.y, v.z, v.w};
                float sv[EPC];
                if constexpr (kBf16) {
#pragma unroll
                    for (int n = 0; n < EPC; ++n)
                        sv[n] = __uint_as_float((w[n / 2] >> (16 * (n % 2))) << 16);
                } else {
#pragma unroll
                    for (int n = 0; n < EPC; ++n) sv[n] = __uint_as_float(w[n]);
                }
#pragma unroll
                for (int q = 0; q < EPC / 4; ++q) {
                    const float4 vb = reinterpret_cast<const float4*>(gB)[m * (EPC / 4) + q];
                    const float4 vc = reinterpret_cast<const float4*>(gC)[m * (EPC / 4) + q];
                    float2 a = fma2(l2, make_float2(sv[4 * q], sv[4 * q + 1]),
                                    mul2(x2, make_float2(vb.x, vb.y)));
                    float2 b = fma2(l2, make_float2(sv[4 * q + 2], sv[4 * q + 3]),
                                    mul2(x2, make_float2(vb.z, vb.w)));
                    if constexpr (kBf16) {
                        a = make_float2(__bfloat162float(__float2bfloat16_rn(a.x)),
                                        __bfloat162float(__float2bfloat16_rn(a.y)));
                        b = make_float2(__bfloat162float(__float2bfloat16_rn(b.x)),
                                        __bfloat162float(__float2bfloat16_rn(b.y)));
                    }
                    sv[4 * q] = a.x; sv[4 * q + 1] = a.y; sv[4 * q + 2] = b.x; sv[4 * q + 3] = b.y;
                    acc = fma2(make_float2(vc.x, vc.y), a, acc);
                    acc1 = fma2(make_float2(vc.z, vc.w), b, acc1);
                }
                if constexpr (kBf16) {
#pragma unroll
                    for (int n = 0; n < EPC; n += 2)
                        w[n / 2] = (__float_as_uint(sv[n]) >> 16) | (__float_as_uint(sv[n + 1]) & 0xffff0000u);
                } else {
#pragma unroll
                    for (int n = 0; n < EPC; ++n) w[n] = __float_as_uint(sv[n]);
                }
                if (active)
                    __stcs(reinterpret_cast<uint4*>(frow) + m, make_uint4(w[0], w[1], w[2], w[3]));
            }
            acc = add2(acc, acc1);
            ysum = grp_sum<LPR>(__fadd_rn(acc.x, acc.y));
        }
        if (active && j == 0) {
            const float yv = __fadd_rn(ysum, __fmul_rn(Dv, xv));
            __stcs(y_u + h * P + p, yv);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[si]);
        if (++si == S) { si = 0; sph ^= 1; }
    }
}

template <int FMT, int N>
cudaError_t launch_n(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    using F = Fmt<FMT>;
    constexpr int LPR = DShape<FMT, N>::LPR;
    constexpr int RPT = kCThreads / LPR;
    constexpr int RB = F::quant ? N * F::bits / 8 : 0;
    const bool has_fp = pv.Hf > 0;
    const int fpEB = FMT == SSQ_BF16 ? 2 : 4;
    // stages: as many as fit a budget that leaves room for two CTAs per SM
    const int budget = 110 * 1024;
    DecodeGeom g = decode_geom(2, RPT, RB, F::meta_bytes, fpEB, has_fp, N, pv.H, pv.G);
    int S = (budget - g.off_stages) / g.stage_bytes;
    if (S > kMaxStages) S = kMaxStages;
    if (S < 2) S = 2;
    g = decode_geom(S, RPT, RB, F::meta_bytes, fpEB, has_fp, N, pv.H, pv.G);
    if (g.smem_bytes > 227 * 1024) return cudaErrorInvalidConfiguration;
    auto kern = decode_kernel<FMT, N>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         g.smem_bytes);
    if (e != cudaSuccess) return e;
    // ask for the largest shared-memory carveout so two CTAs fit per SM
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, occ = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kDThreads,
                                                           g.smem_bytes)) != cudaSuccess)
        return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    long long grid = (long long)sms * occ;
    if (grid > cv.total_tiles) grid = cv.total_tiles;
    kern<<<(int)grid, kDThreads, g.smem_bytes, st>>>(pv, cv, g);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_fmt(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    switch (pv.N) {
    case 16: return launch_n<FMT, 16>(pv, cv, st);
    case 32: return launch_n<FMT, 32>(pv, cv, st);
    case 64: return launch_n<FMT, 64>(pv, cv, st);
    case 128: return launch_n<FMT, 128>(pv, cv, st);
    case 256: return launch_n<FMT, 256>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int decode_rows_per_tile(int fmt, int d_state)
{
    const bool quant = fmt >= SSQ_I8_SYM;
    const int E = quant ? (d_state >= 64 ? 64 : d_state) : (d_state >= 32 ? 32 : d_state);
    return kCThreads / (d_state / E);
}

bool decode_fits(int fmt, int d_state, int nheads, int ngroups)
{
    // B and C of every group plus the lambda arrays must leave room for two
    // pipeline stages within one CTA's shared memory
    const int rpt = decode_rows_per_tile(fmt, d_state);
    const DecodeGeom g = decode_geom(2, rpt, d_state, 8, 4, true, d_state, nheads, ngroups);
    return g.smem_bytes <= 227 * 1024;
}

cudaError_t launch_decode(const PoolView& pv, const CallView& cv, int fmt,
                          cudaStream_t st)
{
    switch (fmt) {
    case SSQ_F32: return launch_fmt<SSQ_F32>(pv, cv, st);
    case SSQ_BF16: return launch_fmt<SSQ_BF16>(pv, cv, st);
    case SSQ_I8_SYM: return launch_fmt<SSQ_I8_SYM>(pv, cv, st);
    case SSQ_I8_ASYM: return launch_fmt<SSQ_I8_ASYM>(pv, cv, st);
    case SSQ_I4_SYM: return launch_fmt<SSQ_I4_SYM>(pv, cv, st);
    case SSQ_I4_ASYM: return launch_fmt<SSQ_I4_ASYM>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssq
