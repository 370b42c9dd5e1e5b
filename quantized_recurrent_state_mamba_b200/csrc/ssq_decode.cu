// ssq_decode.cu -- the fused decode-step kernel.
//
// One launch updates the state of nl layers x batch requests by one token:
// read the packed row, decode, apply the recurrence in fp32, refit the row
// scale, requantize, write the packed row and its metadata back, and read y
// from the newly stored row: one kernel does all of it, as "Mamba state
// quantization for inference" ("Mixed precision spends bits on persistent
// channels") lays out for a low-bit state (decode, fp32 update, new scale,
// packed write-back in one pass), with the quantizer of
// "ssm-state-quantization" README, Setup.
//
// Structure (persistent, warp-specialised, one CTA of 12 warps per SM):
//   - work is a sequence of tiles (up to RPT rows of one region of one
//     (layer, request)); each CTA owns a contiguous range of that sequence;
//   - a producer warp streams each tile's packed rows and metadata from HBM
//     (prefetched into L2 as soon as the tile is next in line) into a ring
//     of shared-memory stages with bulk asynchronous copies
//     (cp.async.bulk, completion counted in bytes on an mbarrier) and the
//     tile's x values with cp.async.  Once per (layer, request, region)
//     "unit" it stages B and C and builds a head table (lambda, dt, D, the
//     y offset and the B/C group of every head of the region), so a
//     consumer row finds everything it needs with two shared loads;
//   - 11 consumer warps compute from shared memory; with nearest rounding a
//     quantized row's new codes and metadata go back into its stage, in
//     place, and the producer stores the finished tile with bulk copies
//     (the stochastic-rounding variant stores each lane's pieces directly);
//     y goes straight to global memory.  A row of a quantized head is held
//     by one lane (two at d_state 256) of up to 128 entries, streamed 16 at
//     a time;
//   - B and C are staged with lane j's 16-byte chunks interleaved, so the
//     lanes of a row read distinct banks;
//   - waits sleep between tries of the mbarrier, and every wait is
//     bounded: one that runs out sets SSQ_DEVERR_TIMEOUT in the pool's error
//     word and the CTA winds down (the producer first waits for its own
//     copies in flight).
#include "ssq_common.cuh"
#include "ssq_params.h"
#include "ssq_pipe.cuh"

#include <type_traits>

namespace ssq {

namespace {

// One CTA of 12 warps per SM: three warps per SM sub-partition, so each
// thread may hold up to 168 registers (the row of 64 entries plus the f32x2
// operand pairs stay in registers).
constexpr int kCWarps = 11;    // + 1 producer
constexpr int kMinBlocks = 1;  // CTAs per SM
constexpr int kCThreads = kCWarps * 32;
constexpr int kDThreads = kCThreads + 32;
constexpr int kMaxStages = 8;
// Shared-memory vector loads / stores at 32-bit shared addresses (the
// quantized path forms its addresses with one XOR each).
template <int OFF>
__device__ __forceinline__ uint4 lds128(unsigned a)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a), "n"(OFF) : "memory");
    return v;
}
template <int OFF>
__device__ __forceinline__ uint2 lds64(unsigned a)
{
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2+%3];"
                 : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF) : "memory");
    return v;
}
template <int OFF>
__device__ __forceinline__ float4 lds128f(unsigned a)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a), "n"(OFF) : "memory");
    return v;
}
template <int OFF>
__device__ __forceinline__ void sts128f(unsigned a, float4 v)
{
    asm volatile("st.shared.v4.f32 [%0+%1], {%2, %3, %4, %5};"
                 :: "r"(a), "n"(OFF), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

template <int OFF>
__device__ __forceinline__ void sts128u(unsigned a, uint4 v)
{
    asm volatile("st.shared.v4.b32 [%0+%1], {%2, %3, %4, %5};"
                 :: "r"(a), "n"(OFF), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
template <int OFF>
__device__ __forceinline__ void sts64u(unsigned a, uint2 v)
{
    asm volatile("st.shared.v2.b32 [%0+%1], {%2, %3};"
                 :: "r"(a), "n"(OFF), "r"(v.x), "r"(v.y) : "memory");
}

// Write `bytes` of shared memory to global memory: the 16-byte multiple as
// one bulk store (in this thread's current bulk group), the rest (a multiple
// of 4 bytes) word by word.  dst and src 16-byte aligned.
__device__ __forceinline__ void store_back(uint8_t* dst, const uint8_t* src, int bytes)
{
    const int b16 = bytes & ~15;
    if (b16 > 0) bulk_s2g(dst, src, (unsigned)b16);
    for (int i = b16; i < bytes; i += 4)
        *reinterpret_cast<uint32_t*>(dst + i) = *reinterpret_cast<const uint32_t*>(src + i);
}

__host__ __device__ inline int r16(int v) { return (v + 15) & ~15; }
__host__ __device__ inline int r256(int v) { return (v + 255) & ~255; }

// ---- tile sequence -----------------------------------------------------
// Tiles are ordered (layer, request, region, row block).  A CTA walks a
// contiguous range of them with counters (one division at the start).
struct TileWalk {
    long long lb;   // layer * batch + request
    int l, b, k;    // k: tile within (layer, request)
    bool quant;
    int rbase, n;   // first region row, rows in this tile

    __device__ __forceinline__ void fill(const PoolView& pv, const CallView& cv)
    {
        quant = k < cv.qtiles;
        const int rpt = quant ? cv.rows_per_tile : cv.rows_per_tile_f;
        rbase = (quant ? k : k - cv.qtiles) * rpt;
        const int nrows = (quant ? pv.Hq : pv.Hf) * pv.P;
        n = min(rpt, nrows - rbase);
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
    // Advance; true when the next tile starts a new unit.
    __device__ __forceinline__ bool next(const PoolView& pv, const CallView& cv)
    {
        const bool was_quant = quant;
        if (++k == cv.qtiles + cv.ftiles) {
            k = 0;
            ++lb;
            if (++b == cv.batch) {
                b = 0;
                ++l;
            }
            fill(pv, cv);
            return true;
        }
        fill(pv, cv);
        return quant != was_quant;
    }
};

// ---- shared-memory geometry (host and device agree on it) --------------
// Unit buffer: [16 B header: slot, bad][B: G*N f32][C: G*N f32]
//              [head table: Hpad x float4 {lambda, dt, D, y offset}]
//              [group table: Hpad x int (g*N)]
// Stage:       [x: RPT f32, padded to 128 B][payload: codes + meta, or fp rows]
struct DecodeGeom {
    int S;            // stages
    int RPTq, RPTf;   // rows per tile in the quantized / fp region
    int x_bytes;      // x area of a stage
    int qcodes_bytes; // codes area of a quantized tile
    int pay_bytes;    // payload area of a stage
    int stage_bytes;
    int ub_B, ub_C, ub_ht, ub_gt, unit_bytes;  // unit buffer layout
    int Hpad;
    int off_units, off_stages, off_scr, scr_warp_bytes, smem_bytes;
};

// Offsets are from a 256-byte aligned base inside the dynamic shared memory
// (the launch adds 256 bytes of slack); B, C and every stage start on a
// 256-byte boundary, so per-lane addresses can be permuted with one XOR.
// scr_lane_bytes: per lane spill area of a consumer warp (0: none).
__host__ __device__ inline DecodeGeom decode_geom(int S, int RPTq, int RPTf, int RB, int MB,
                                                  int fpEB, bool has_q, bool has_fp, int N,
                                                  int H, int G, int scr_lane_bytes)
{
    DecodeGeom g;
    g.S = S;
    g.RPTq = RPTq;
    g.RPTf = RPTf;
    g.x_bytes = r256((RPTq > RPTf ? RPTq : RPTf) * 4);
    g.qcodes_bytes = has_q ? r256(RPTq * RB) : 0;
    const int qpay = has_q ? g.qcodes_bytes + r16(RPTq * MB) : 0;
    const int fpay = has_fp ? RPTf * N * fpEB : 0;
    g.pay_bytes = qpay > fpay ? qpay : fpay;
    g.stage_bytes = r256(g.x_bytes + g.pay_bytes);
    g.Hpad = (H + 3) & ~3;
    g.ub_B = 256;                      // [0, 16): slot, bad flag
    g.ub_C = g.ub_B + G * N * 4;
    g.ub_ht = r256(g.ub_C + G * N * 4);
    g.ub_gt = g.ub_ht + g.Hpad * 16;
    g.unit_bytes = r256(g.ub_gt + g.Hpad * 4);
    const int bars = r256((2 * kMaxStages + 4) * 8);
    g.off_units = bars;
    g.off_stages = g.off_units + 2 * g.unit_bytes;
    g.off_scr = g.off_stages + S * g.stage_bytes;
    g.scr_warp_bytes = has_q ? 32 * scr_lane_bytes : 0;
    g.smem_bytes = g.off_scr + kCWarps * g.scr_warp_bytes + 256;
    return g;
}

// Lane shapes.  A quantized row is held by one lane (the whole row for
// d_state <= 128; two lanes at 256): the per-row work (refit, addresses,
// metadata, the tile bookkeeping) is spread over 128 entries and the row
// reductions need no shuffles.  Of the lane's 8 pieces of 16 entries, the
// first kRegPieces stay in registers between the update and the rounding
// and the rest wait in a per-lane shared-memory area, which keeps the kernel
// within the register budget of three warps per SM sub-partition.  An fp
// row (the fp32 / bf16 formats, and unmasked heads of the integer formats)
// is streamed by N/32 lanes of 32 entries.
constexpr int kQuantE = 128;
constexpr int kRegPieces = 5;
template <int N>
struct QShape {
    static constexpr int E = N >= kQuantE ? kQuantE : N;
    static constexpr int LPR = N / E;
    static constexpr int RPT = kCThreads / LPR;   // rows per tile
    static constexpr int NP = E / 16;             // pieces per lane
    static constexpr int NREG = NP < kRegPieces ? NP : kRegPieces;
    static constexpr int SCR = (NP - NREG) * 16 * 4;   // spill bytes per lane
};
template <int N>
struct FShape {
    static constexpr int E = N >= 32 ? 32 : N;
    static constexpr int LPR = N / E;
    static constexpr int RPT = kCThreads / LPR;
};

// A whole quantized row by the formulas verbatim (every fp32 operation one
// IEEE rounding in the order of the definition), for warps where some row
// falls outside the magic-number paths: a zero point or scaled values of
// 2^22 or more in magnitude (rows far from zero relative to their range).  Every lane of the warp
// calls it together (the row reductions are shuffles).  Codes are read from
// and written in natural order; B and C come from the interleaved layout.
template <int FMT, int N, bool SR>
__device__ __noinline__ float row_exact(const uint8_t* __restrict__ cs, float delta0, float z0,
                                        float lam, float dtx, const float* __restrict__ gB,
                                        const float* __restrict__ gC, int j, bool active,
                                        uint8_t* __restrict__ crow, uint8_t* __restrict__ mrow,
                                        uint32_t* err, SrKey srk)
{
    using F = Fmt<FMT>;
    constexpr int E = QShape<N>::E, LPR = QShape<N>::LPR;
    constexpr int NP = E / 16;
    constexpr int CB = E * F::bits / 8;
    float s[E];
    float lo = 0.0f, hi = 0.0f;
#pragma unroll 1
    for (int n = 0; n < E; ++n) {
        int q;
        if constexpr (F::bits == 8) {
            const uint32_t bb = cs[n];
            q = F::sym ? (int)(int8_t)bb : (int)bb;
        } else {
            const uint32_t bb = (cs[n / 2] >> (4 * (n % 2))) & 0xFu;
            q = F::sym ? (int)((bb ^ 8u) - 8u) : (int)bb;
        }
        const float v = __fmul_rn(__fsub_rn((float)q, z0), delta0);
        const int pc = n / 16, i = (n % 16) / 4, e = n % 4;
        const int bi = ((i * NP + pc) * LPR + j) * 4 + e;
        const float w = __fmul_rn(dtx, gB[bi]);
        const float sv = __fmaf_rn(lam, v, w);
        s[n] = sv;
        lo = n == 0 ? sv : fminf(lo, sv);
        hi = n == 0 ? sv : fmaxf(hi, sv);
    }
    const RowParams rp = refit_from_minmax<FMT, LPR>(lo, hi);
    float acc = 0.0f;
    uint32_t words[CB / 4];
#pragma unroll
    for (int i = 0; i < CB / 4; ++i) words[i] = 0u;
#pragma unroll 1
    for (int n = 0; n < E; ++n) {
        float c, r;
        if constexpr (SR) {
            const int ng = j * E + n;                   // entry within the row
            const uint4 w = philox4x32_10(
                make_uint4(srk.row_block + (uint32_t)(ng / 8), srk.layer, srk.slot, srk.step),
                srk.key);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
            const uint32_t d = (ww[(ng % 8) / 2] >> (16 * (ng % 2))) & 0xFFFFu;
            c = round1_sr_exact<FMT>(s[n], rp.inv, rp.z, (float)d * (1.0f / 65536.0f), &r);
        } else {
            const float rr = rint_prod(s[n], rp.inv);
            if constexpr (F::sym) {
                c = fminf(fmaxf(rr, -F::qmax), F::qmax);
                r = c;
            } else {
                c = fminf(__fadd_rn(rr, rp.z), F::qmax);
                r = __fsub_rn(c, rp.z);
            }
        }
        const uint32_t code = (uint32_t)(int)c & ((1u << F::bits) - 1u);
        words[n * F::bits / 32] |= code << ((n * F::bits) % 32);
        const int pc = n / 16, i = (n % 16) / 4, e = n % 4;
        const int ci = ((i * NP + pc) * LPR + j) * 4 + e;
        acc = __fmaf_rn(gC[ci], __fmul_rn(r, rp.delta), acc);
    }
    const float ysum = grp_sum<LPR>(acc);
    if (active) {
#pragma unroll
        for (int i = 0; i < CB / 4; ++i) reinterpret_cast<uint32_t*>(crow)[i] = words[i];
        if (j == 0) {
            if constexpr (F::sym) {
                *reinterpret_cast<float*>(mrow) = rp.delta;
            } else {
                *reinterpret_cast<float2*>(mrow) = make_float2(rp.delta, rp.z);
            }
            if (!rp.finite) atomicOr(err, SSQ_DEVERR_NONFINITE);
        }
    }
    return ysum;
}

// SR: round the quantized rows stochastically (draws keyed by cv.sr_seed
// and countered by row block, layer, slot and cv.sr_step).
template <int FMT, int N, bool SR>
__global__ void __launch_bounds__(kDThreads, kMinBlocks)
decode_kernel(const __grid_constant__ PoolView pv, const __grid_constant__ CallView cv,
              const __grid_constant__ DecodeGeom geo)
{
    using F = Fmt<FMT>;
    // quantized rows: EQ entries per lane, LQ lanes per row; fp rows: EF, LF
    constexpr int EQ = QShape<N>::E, LQ = QShape<N>::LPR;
    constexpr int EF = FShape<N>::E, LF = FShape<N>::LPR;
    constexpr bool kBf16 = (FMT == SSQ_BF16);
    constexpr int RB = F::quant ? N * F::bits / 8 : 0;      // code bytes per row
    constexpr int CB = F::quant ? EQ * F::bits / 8 : 16;    // code bytes per lane
    constexpr int MB = F::meta_bytes;
    constexpr int FEB = kBf16 ? 2 : 4;                       // fp element bytes
    constexpr int NP = EQ / 16;                              // 16-entry pieces per lane
    constexpr int NREG = QShape<N>::NREG;                    // pieces kept in registers
    constexpr int PW = F::quant ? Piece<FMT>::words : 1;     // code words per piece
    constexpr int PB = PW * 4;                               // code bytes per piece
    // Nearest rounding writes a quantized tile's new codes and metadata back
    // into its stage and the producer stores the tile with bulk copies
    // (coalesced); the stochastic-rounding variant, at its register limit,
    // stores each lane's pieces directly.
    constexpr bool kWB = !SR;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* const smem = smem_raw + ((256u - (saddr(smem_raw) & 255u)) & 255u);
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
        // The consumers leave a quantized tile's new codes and metadata in
        // its stage, laid out as in the pool; lane 0 writes them back with
        // bulk stores once the consumers release the stage, before the
        // stage is filled again.  Per stage: destination and bytes of the
        // tile waiting there (pend_cb < 0: none) and the phase it was
        // loaded in.
        uint8_t* pend_c[kMaxStages];
        uint8_t* pend_m[kMaxStages];
        int pend_cb[kMaxStages], pend_mb[kMaxStages], pend_ph[kMaxStages];
#pragma unroll
        for (int s = 0; s < kMaxStages; ++s) pend_cb[s] = -1;
        auto flush = [&](int s) {
            if (pend_cb[s] < 0) return;
            const uint8_t* pay = stages + s * geo.stage_bytes + geo.x_bytes;
            store_back(pend_c[s], pay, pend_cb[s]);
            store_back(pend_m[s], pay + geo.qcodes_bytes, pend_mb[s]);
            bulk_commit();
            bulk_wait_read<0>();        // the stage may be refilled after this
            pend_cb[s] = -1;
        };
        int si = 0, sph = 0, k = 0, uk = -1;
        bool bad = false, ok = true, newunit = true;
        const uint8_t* codes_u = nullptr;
        const uint8_t* meta_u = nullptr;
        const uint8_t* fp_u = nullptr;
        const float* x_u = nullptr;
        TileWalk ti;
        ti.start(pv, cv, t0);
        for (long long t = t0; t < t1; ++t, newunit = ti.next(pv, cv)) {
            const int regbase = ti.quant ? 0 : pv.Hq;
            if (newunit) {
                ++uk;
                const int u = uk & 1;
                if (!mbar_wait<kProducerSleep>(&uempty[u], ((uk >> 1) & 1) ^ 1)) { ok = false; break; }
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
                    // B and C in 16-byte chunks.  In quantized units lane j's
                    // chunk i of piece pc (its entries 16*pc + 4*i .. +3) is
                    // stored at (i*NP + pc)*LPR + j, so the lanes of a warp,
                    // visiting different pieces, read distinct banks.
                    float* dB = reinterpret_cast<float*>(ub + geo.ub_B);
                    float* dC = reinterpret_cast<float*>(ub + geo.ub_C);
                    const float* sB = cv.B + ti.lb * G * N;
                    const float* sC = cv.C + ti.lb * G * N;
                    for (int m = lane; m < G * N / 4; m += 32) {
                        int pos = m;
                        if (F::quant && ti.quant) {
                            const int gi = m / (N / 4), mm = m - gi * (N / 4);
                            const int jj = mm / (EQ / 4), rest = mm - jj * (EQ / 4);
                            const int pc = rest / 4, ii = rest - pc * 4;
                            pos = gi * (N / 4) + (ii * NP + pc) * LQ + jj;
                        }
                        cpa16(dB + 4 * pos, sB + 4 * m);
                        cpa16(dC + 4 * pos, sC + 4 * m);
                    }
                    // head table of the region: lambda = exp(dt*A) once per
                    // head, dt, D, the head's y offset and B/C group
                    float4* ht = reinterpret_cast<float4*>(ub + geo.ub_ht);
                    int* gt = reinterpret_cast<int*>(ub + geo.ub_gt);
                    const int nreg = ti.quant ? pv.Hq : pv.Hf;
                    for (int hr = lane; hr < nreg; hr += 32) {
                        const int h = pv.perm[regbase + hr];
                        const float dtv = __ldg(cv.dt + ti.lb * H + h);
                        const float Av = __ldg(cv.A + (long long)ti.l * H + h);
                        const float Dv = __ldg(cv.D + (long long)ti.l * H + h);
                        ht[hr] = make_float4(decay(dtv, Av), dtv, Dv, __int_as_float(h * P));
                        gt[hr] = fdiv(h, pv.mHpg) * N;
                    }
                }
                cpa_arrive(&ufull[u]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&ufull[u]);
            }
            if (bad) continue;
            // start the tile's HBM reads into L2 now; the copy into the stage,
            // issued once the consumers release it, then reads from L2
            if (lane == 0) {
                if (F::quant && ti.quant) {
                    bulk_prefetch_l2(codes_u + (long long)ti.rbase * RB, (unsigned)r16(ti.n * RB));
                    bulk_prefetch_l2(meta_u + (long long)ti.rbase * MB, (unsigned)r16(ti.n * MB));
                } else {
                    bulk_prefetch_l2(fp_u + (long long)ti.rbase * N * FEB, (unsigned)(ti.n * N * FEB));
                }
            }
            if (!mbar_wait<kProducerSleep>(&empty[si], sph ^ 1)) { ok = false; break; }
            if (lane == 0) flush(si);
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
                    if (kWB) {
                        pend_c[si] = const_cast<uint8_t*>(codes_u) + (long long)ti.rbase * RB;
                        pend_m[si] = const_cast<uint8_t*>(meta_u) + (long long)ti.rbase * MB;
                        pend_cb[si] = ti.n * RB;
                        pend_mb[si] = ti.n * MB;
                        pend_ph[si] = sph;
                    }
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
        // the last tiles' write-backs, in the order they were loaded
        if (lane == 0) {
            for (int jj = (k > S ? k - S : 0); jj < k; ++jj) {
                const int s = jj % S;
                if (pend_cb[s] < 0) continue;
                if (ok && mbar_wait<kProducerSleep>(&empty[s], (unsigned)pend_ph[s])) {
                    flush(s);
                } else {
                    ok = false;
                    pend_cb[s] = -1;
                }
            }
            if (!ok) atomicOr(err, SSQ_DEVERR_TIMEOUT);
            bulk_wait<0>();
        }
        // No copy may still be writing shared memory when the CTA exits.
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0) {
            for (int jj = (k > S ? k - S : 0); jj < k; ++jj)
                mbar_wait<kConsumerSleep>(&full[jj % S], (jj / S) & 1);
        }
        return;
    }

    // ================= consumer warps =================
    const int ct = threadIdx.x;
    int si = 0, sph = 0, uk = -1;
    bool bad = false, newunit = true;
    const uint8_t* ub = units;
    uint8_t* codes_u = nullptr;
    uint8_t* meta_u = nullptr;
    uint8_t* fp_u = nullptr;
    float* y_u = nullptr;
    int cur_slot = 0;

    TileWalk ti;
    ti.start(pv, cv, t0);
    for (long long t = t0; t < t1; ++t, newunit = ti.next(pv, cv)) {
        if (newunit) {
            if (uk >= 0) {
                __syncwarp();
                mbar_arrive_if(&uempty[uk & 1], lane == 0);
            }
            ++uk;
            const int u = uk & 1;
            if (!mbar_wait<kConsumerSleep>(&ufull[u], (uk >> 1) & 1)) {
                if (lane == 0) atomicOr(err, SSQ_DEVERR_TIMEOUT);
                break;
            }
            ub = units + u * geo.unit_bytes;
            const int slot = reinterpret_cast<const int*>(ub)[0];
            cur_slot = slot;
            bad = reinterpret_cast<const int*>(ub)[1] != 0;
            if (!bad) {
                const int layer = cv.layer0 + ti.l;
                uint8_t* sb = pv.pool + pv.header_bytes + (long long)slot * pv.slot_bytes;
                codes_u = sb + pv.codes_off + (long long)layer * pv.codes_layer_bytes;
                meta_u = sb + pv.meta_off + (long long)layer * pv.meta_layer_bytes;
                fp_u = sb + pv.fp_off + (long long)layer * pv.fp_layer_bytes;
                y_u = cv.y + ti.lb * H * P;
            }
        }
        if (bad) continue;
        if (!mbar_wait<kConsumerSleep>(&full[si], sph)) {
            if (lane == 0) atomicOr(err, SSQ_DEVERR_TIMEOUT);
            break;
        }
        const uint8_t* st = stages + si * geo.stage_bytes;
        const float* sx = reinterpret_cast<const float*>(st);
        const uint8_t* pay = st + geo.x_bytes;
        // row within the tile and lane within the row, by the region's shape
        const int grow = ti.quant ? ct / LQ : ct / LF;
        const int j = ti.quant ? ct % LQ : ct % LF;
        const bool active = grow < ti.n;
        // Rows past the end of a partial tile shadow its row 0: they read
        // row 0's inputs and so compute and store exactly row 0's bytes,
        // which lets every store go without a branch.
        const int rl = active ? grow : 0;
        const int rr = ti.rbase + rl;
        const int hr = fdiv(rr, pv.mP);
        const int p = rr - hr * P;
        const float4 hti = reinterpret_cast<const float4*>(ub + geo.ub_ht)[hr];
        const int gN = reinterpret_cast<const int*>(ub + geo.ub_gt)[hr];
        const float xv = sx[rl];
        const float lamv = hti.x;
        const float dtx = __fmul_rn(hti.y, xv);
        const float* gB = reinterpret_cast<const float*>(ub + geo.ub_B) + gN;
        const float* gC = reinterpret_cast<const float*>(ub + geo.ub_C) + gN;
        float ysum = 0.0f;
        bool done = false;

        if constexpr (F::quant) {
            if (ti.quant) {
                done = true;
                // this lane's codes and the row's metadata in shared memory.
                // The lane visits its pieces in the order pc = sp ^ rot, rot
                // being its 128-byte line, so the lanes of a warp reading
                // one step touch every bank group; its code block, B and C
                // and its row in the pool are aligned so that each permuted
                // address is a single XOR.
                const int loff = rl * RB + j * CB;
                const uint8_t* cs = pay + loff;
                const unsigned rot = (unsigned)(loff >> 7) & (NP - 1);
                const unsigned cs_x = saddr(cs) | (rot * PB);
                const unsigned bx = (saddr(gB) + j * 16) | (rot * LQ * 16);
                const unsigned cx = (saddr(gC) + j * 16) | (rot * LQ * 16);
                // With kWB the new codes and metadata go back into the stage,
                // in place (the producer writes the tile back), and rows past
                // the end of the tile store nothing, as the row they shadow
                // may already hold new codes; otherwise they go straight to
                // the pool (a shadow row stores row 0's bytes again).
                uint8_t* const ms = const_cast<uint8_t*>(pay) + geo.qcodes_bytes + rl * MB;
                uint8_t* const crow = kWB ? const_cast<uint8_t*>(cs)
                                          : codes_u + (long long)rr * RB + j * CB;
                uint8_t* const mrow = kWB ? ms : meta_u + (long long)rr * MB;
                const uintptr_t crow_x = reinterpret_cast<uintptr_t>(crow) | (rot * PB);
                float delta0, z0 = 0.0f;
                {
                    if constexpr (F::sym) {
                        delta0 = *reinterpret_cast<const float*>(ms);
                    } else {
                        const float2 m = *reinterpret_cast<const float2*>(ms);
                        delta0 = m.x;
                        z0 = m.y;
                    }
                }
                // pieces NREG.. of the updated row wait in this lane's spill
                // area: chunk k of lane l at scr + (k * 32 + l) * 16
                const unsigned scr = saddr(smem + geo.off_scr) + warp * geo.scr_warp_bytes + lane * 16;
                // decode + update, one 16-entry piece at a time, with
                // per-piece min / max.  The decode is exact for |z| < 2^22;
                // rows beyond that take the exact path below.
                float s[NREG * 16];
                float lo, hi;
                {
                    const float c0 = __fadd_rn(kTwo23, __fadd_rn(z0, F::bias));
                    const float2 nc02 = make_float2(-c0, -c0);
                    const float2 d2 = make_float2(delta0, delta0);
                    const float2 l2 = make_float2(lamv, lamv);
                    const float2 x2 = make_float2(dtx, dtx);
#pragma unroll
                    for (int sp = 0; sp < NP; ++sp) {
                        uint32_t w[PW];
                        if constexpr (PW == 4) {
                            const uint4 v = lds128<0>(cs_x ^ (sp * PB));
                            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
                        } else {
                            const uint2 v = lds64<0>(cs_x ^ (sp * PB));
                            w[0] = v.x; w[1] = v.y;
                        }
                        float f[16];
                        unpack16_biased<FMT>(w, f);
                        const unsigned bp = bx ^ (sp * LQ * 16);
                        float v16[16];
                        auto bq = [&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            const float4 bv = lds128f<i * NP * LQ * 16>(bp);
                            const float2 v0 = mul2(add2(make_float2(f[4 * i], f[4 * i + 1]), nc02), d2);
                            const float2 v1 = mul2(add2(make_float2(f[4 * i + 2], f[4 * i + 3]), nc02), d2);
                            const float2 u0 = fma2(l2, v0, mul2(x2, make_float2(bv.x, bv.y)));
                            const float2 u1 = fma2(l2, v1, mul2(x2, make_float2(bv.z, bv.w)));
                            v16[4 * i] = u0.x; v16[4 * i + 1] = u0.y;
                            v16[4 * i + 2] = u1.x; v16[4 * i + 3] = u1.y;
                        };
                        bq(std::integral_constant<int, 0>{});
                        bq(std::integral_constant<int, 1>{});
                        bq(std::integral_constant<int, 2>{});
                        bq(std::integral_constant<int, 3>{});
                        float plo, phi;
                        minmax16(v16, plo, phi);
                        lo = sp == 0 ? plo : fminf(lo, plo);
                        hi = sp == 0 ? phi : fmaxf(hi, phi);
                        if (sp < NREG) {
#pragma unroll
                            for (int n = 0; n < 16; ++n) s[(sp < NREG ? sp : 0) * 16 + n] = v16[n];
                        } else {
                            const unsigned a = scr + (sp - NREG) * 4 * 512;
                            sts128f<0>(a, make_float4(v16[0], v16[1], v16[2], v16[3]));
                            sts128f<512>(a, make_float4(v16[4], v16[5], v16[6], v16[7]));
                            sts128f<1024>(a, make_float4(v16[8], v16[9], v16[10], v16[11]));
                            sts128f<1536>(a, make_float4(v16[12], v16[13], v16[14], v16[15]));
                        }
                    }
                }
                const RowParams rp = refit_from_minmax<FMT, LQ>(lo, hi);
                // the magic-number paths are exact for every row of the warp;
                // rows whose top code must be capped take the clamped loop
                const bool fast = __all_sync(0xffffffffu, (F::sym || fabsf(z0) < kFastLimit)
                                                          && rp.fast);
                // the stochastic-rounding key of this row (unused for RTN)
                SrKey srk;
                if constexpr (SR) {
                    srk.key = make_uint2((uint32_t)cv.sr_seed, (uint32_t)(cv.sr_seed >> 32));
                    srk.layer = (uint32_t)(cv.layer0 + ti.l);
                    srk.slot = (uint32_t)cur_slot;
                    srk.step = cv.sr_step;
                    srk.row_block = (uint32_t)(__float_as_int(hti.w) + p) * (uint32_t)(N / 8);
                }
                if (fast) {
                    const float2 inv2 = make_float2(rp.inv, rp.inv);
                    const float2 z2 = make_float2(rp.z, rp.z);
                    const float mz = F::sym ? -kMagic : -__fadd_rn(kMagic, rp.z);
                    const float2 mz2 = make_float2(mz, mz);
                    // round, pack, store and read back, piece by piece; the
                    // readout sums C (q - z) and scales by Delta once
                    float2 acc = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
                    auto piece = [&](auto clamp_tag, int sp) {
                        float v16[16];
                        if (sp < NREG) {
#pragma unroll
                            for (int n = 0; n < 16; ++n) v16[n] = s[(sp < NREG ? sp : 0) * 16 + n];
                        } else {
                            const unsigned a = scr + (sp - NREG) * 4 * 512;
                            const float4 q0 = lds128f<0>(a), q1 = lds128f<512>(a);
                            const float4 q2 = lds128f<1024>(a), q3 = lds128f<1536>(a);
                            v16[0] = q0.x; v16[1] = q0.y; v16[2] = q0.z; v16[3] = q0.w;
                            v16[4] = q1.x; v16[5] = q1.y; v16[6] = q1.z; v16[7] = q1.w;
                            v16[8] = q2.x; v16[9] = q2.y; v16[10] = q2.z; v16[11] = q2.w;
                            v16[12] = q3.x; v16[13] = q3.y; v16[14] = q3.z; v16[15] = q3.w;
                        }
                        float r[16];
                        uint32_t kk[16];
                        if constexpr (SR) {
                            float u[16];
                            sr_draws16(srk, j * EQ + 16 * (int)((unsigned)sp ^ rot), u);
                            round16_sr<FMT>(inv2, z2, mz2, v16, u, r, kk);
                        } else {
                            round16_carry<FMT, decltype(clamp_tag)::value>(inv2, z2, mz2, v16, r, kk);
                        }
                        uint32_t w[PW];
                        pack16<FMT>(kk, w);
                        if constexpr (kWB) {
                            if (active) {
                                if constexpr (PW == 4)
                                    sts128u<0>(cs_x ^ (sp * PB), make_uint4(w[0], w[1], w[2], w[3]));
                                else
                                    sts64u<0>(cs_x ^ (sp * PB), make_uint2(w[0], w[1]));
                            }
                        } else {
                            void* dst = reinterpret_cast<void*>(crow_x ^ (uintptr_t)(sp * PB));
                            if constexpr (PW == 4)
                                __stcs(reinterpret_cast<uint4*>(dst), make_uint4(w[0], w[1], w[2], w[3]));
                            else
                                __stcs(reinterpret_cast<uint2*>(dst), make_uint2(w[0], w[1]));
                        }
                        const unsigned cp = cx ^ (sp * LQ * 16);
                        auto cq = [&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            const float4 cv4 = lds128f<i * NP * LQ * 16>(cp);
                            acc = fma2(make_float2(cv4.x, cv4.y), make_float2(r[4 * i], r[4 * i + 1]), acc);
                            acc1 = fma2(make_float2(cv4.z, cv4.w), make_float2(r[4 * i + 2], r[4 * i + 3]), acc1);
                        };
                        cq(std::integral_constant<int, 0>{});
                        cq(std::integral_constant<int, 1>{});
                        cq(std::integral_constant<int, 2>{});
                        cq(std::integral_constant<int, 3>{});
                    };
                    if (SR || F::sym || !__any_sync(0xffffffffu, rp.clamp)) {
#pragma unroll
                        for (int sp = 0; sp < NP; ++sp) piece(std::false_type{}, sp);
                    } else {
#pragma unroll
                        for (int sp = 0; sp < NP; ++sp) piece(std::true_type{}, sp);
                    }
                    acc = add2(acc, acc1);
                    ysum = __fmul_rn(rp.delta, grp_sum<LQ>(__fadd_rn(acc.x, acc.y)));
                    if constexpr (kWB) {
                        if (active && j == 0) {
                            if constexpr (F::sym) {
                                *reinterpret_cast<float*>(ms) = rp.delta;
                            } else {
                                *reinterpret_cast<float2*>(ms) = make_float2(rp.delta, rp.z);
                            }
                        }
                    } else {
                        // every lane of the row writes the same metadata
                        if constexpr (F::sym) {
                            __stcs(reinterpret_cast<float*>(mrow), rp.delta);
                        } else {
                            __stcs(reinterpret_cast<float2*>(mrow), make_float2(rp.delta, rp.z));
                        }
                    }
                    if (__any_sync(0xffffffffu, !rp.finite) && lane == 0)
                        atomicOr(err, SSQ_DEVERR_NONFINITE);
                } else {
                    ysum = row_exact<FMT, N, SR>(cs, delta0, z0, lamv, dtx, gB, gC, j, active,
                                                 crow, mrow, err, srk);
                }
            }
        }
        if (!done) {
            // fp row (fp32, or bf16 for the bf16 format), streamed one 16-byte
            // storage chunk at a time.  Lane j owns chunks LF*c + j; a lane
            // starts at chunk `rot` so a warp's reads of one step spread over
            // every bank group while B and C stay within one 128-byte line.
            constexpr int EPC = 16 / FEB;           // elements per chunk
            constexpr int NCH = EF / EPC;            // chunks per lane
            constexpr int RW = (8 / LF) < NCH ? (8 / LF) : NCH;   // rotation width
            const int rot = RW > 1 ? grow % RW : 0;
            const uint8_t* fs = pay + (long long)rl * N * FEB;
            uint8_t* frow = fp_u + (long long)rr * N * FEB;
            const float2 l2 = make_float2(lamv, lamv);
            const float2 x2 = make_float2(dtx, dtx);
            float2 acc = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int c0 = 0; c0 < NCH; ++c0) {
                const int c = RW > 1 ? ((c0 + rot) & (NCH - 1)) : c0;
                const int m = LF * c + j;
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
                __stcs(reinterpret_cast<uint4*>(frow) + m, make_uint4(w[0], w[1], w[2], w[3]));
            }
            acc = add2(acc, acc1);
            ysum = grp_sum<LF>(__fadd_rn(acc.x, acc.y));
        }
        // every lane of the row writes the same y (after the row sum all
        // hold it); a row past the end of the tile writes nothing (with the
        // in-place write-back it may have read its shadowed row's new codes)
        if (active)
            __stcs(y_u + __float_as_int(hti.w) + p, __fadd_rn(ysum, __fmul_rn(hti.z, xv)));
        // the stage's new codes must be visible to the producer's bulk store
        if (kWB && F::quant && ti.quant) fence_proxy_async();
        __syncwarp();
        mbar_arrive_if(&empty[si], lane == 0);
        if (++si == S) { si = 0; sph ^= 1; }
    }
}

template <int FMT, int N, bool SR>
cudaError_t launch_n(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    using F = Fmt<FMT>;
    constexpr int RPTq = QShape<N>::RPT, RPTf = FShape<N>::RPT;
    constexpr int RB = F::quant ? N * F::bits / 8 : 0;
    const bool has_q = pv.Hq > 0, has_fp = pv.Hf > 0;
    const int fpEB = FMT == SSQ_BF16 ? 2 : 4;
    // stages: as many as fit a budget that leaves room for kMinBlocks CTAs per SM
    const int budget = (kMinBlocks == 1 ? 225 : 110) * 1024;
    constexpr int SCR = F::quant ? QShape<N>::SCR : 0;
    DecodeGeom g = decode_geom(2, RPTq, RPTf, RB, F::meta_bytes, fpEB, has_q, has_fp, N, pv.H, pv.G, SCR);
    int S = (budget - (g.smem_bytes - 2 * g.stage_bytes)) / g.stage_bytes;
    if (S > kMaxStages) S = kMaxStages;
    if (S < 2) S = 2;
    g = decode_geom(S, RPTq, RPTf, RB, F::meta_bytes, fpEB, has_q, has_fp, N, pv.H, pv.G, SCR);
    if (g.smem_bytes > 227 * 1024) return cudaErrorInvalidConfiguration;
    auto kern = decode_kernel<FMT, N, SR>;
    // per-device launch facts, looked up once per kernel instantiation and device
    thread_local int s_dev = -1, s_grid = 0, s_smem = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (s_dev != dev || s_smem != g.smem_bytes) {
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      g.smem_bytes)) != cudaSuccess)
            return e;
        // the largest shared-memory carveout, so two CTAs fit per SM
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                      (int)cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
            return e;
        int sms = 0, occ = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kDThreads,
                                                               g.smem_bytes)) != cudaSuccess)
            return e;
        if (occ < 1) return cudaErrorInvalidConfiguration;
        s_dev = dev;
        s_smem = g.smem_bytes;
        s_grid = sms * occ;
    }
    long long grid = s_grid;
    if (grid > cv.total_tiles) grid = cv.total_tiles;
    kern<<<(int)grid, kDThreads, g.smem_bytes, st>>>(pv, cv, g);
    return cudaGetLastError();
}

template <int FMT, bool SR>
cudaError_t launch_fmt(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    switch (pv.N) {
    case 16: return launch_n<FMT, 16, SR>(pv, cv, st);
    case 32: return launch_n<FMT, 32, SR>(pv, cv, st);
    case 64: return launch_n<FMT, 64, SR>(pv, cv, st);
    case 128: return launch_n<FMT, 128, SR>(pv, cv, st);
    case 256: return launch_n<FMT, 256, SR>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

void decode_tile_rows(int fmt, int d_state, int* rows_q, int* rows_f)
{
    const int eq = d_state >= kQuantE ? kQuantE : d_state;
    const int ef = d_state >= 32 ? 32 : d_state;
    *rows_q = kCThreads / (d_state / eq);
    *rows_f = kCThreads / (d_state / ef);
    (void)fmt;
}

bool decode_fits(int fmt, int d_state, int nheads, int ngroups)
{
    // B and C of every group plus the head tables must leave room for two
    // pipeline stages (of either region) within one CTA's shared memory
    int rq = 0, rf = 0;
    decode_tile_rows(fmt, d_state, &rq, &rf);
    const bool q = fmt >= SSQ_I8_SYM;
    const int eq = d_state >= kQuantE ? kQuantE : d_state;
    const int np = eq / 16, nreg = np < kRegPieces ? np : kRegPieces;
    const DecodeGeom g = decode_geom(2, rq, rf, d_state, 8, 4, q, true, d_state, nheads, ngroups,
                                     (np - nreg) * 64);
    return g.smem_bytes <= 227 * 1024;
}

cudaError_t launch_decode(const PoolView& pv, const CallView& cv, int fmt, bool sr,
                          cudaStream_t st)
{
    // stochastic rounding changes only the integer formats
    switch (fmt) {
    case SSQ_F32: return launch_fmt<SSQ_F32, false>(pv, cv, st);
    case SSQ_BF16: return launch_fmt<SSQ_BF16, false>(pv, cv, st);
    case SSQ_I8_SYM:
        return sr ? launch_fmt<SSQ_I8_SYM, true>(pv, cv, st) : launch_fmt<SSQ_I8_SYM, false>(pv, cv, st);
    case SSQ_I8_ASYM:
        return sr ? launch_fmt<SSQ_I8_ASYM, true>(pv, cv, st) : launch_fmt<SSQ_I8_ASYM, false>(pv, cv, st);
    case SSQ_I4_SYM:
        return sr ? launch_fmt<SSQ_I4_SYM, true>(pv, cv, st) : launch_fmt<SSQ_I4_SYM, false>(pv, cv, st);
    case SSQ_I4_ASYM:
        return sr ? launch_fmt<SSQ_I4_ASYM, true>(pv, cv, st) : launch_fmt<SSQ_I4_ASYM, false>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssq
