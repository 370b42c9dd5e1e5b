// ssq_scan.cu -- the per-token scan with the state rounded at every token.
//
// "ssm-state-quantization" README, Setup: a sequential per-token scan
// replaces the chunked library scan so that the state can be rounded at
// every step.  The state of a row lives in registers for all T tokens as the
// value its stored codes decode to, fl((q - z) * Delta), so T tokens of the
// scan equal T decode steps bit for bit; only the final codes and metadata
// go back to the pool.
//
// Work split: a CTA of W warps owns W * RPW consecutive head_dim rows of ONE
// head of one request, so lambda, dt, B and C are uniform across the CTA.
// A row of N entries is held by LPR = N / E lanes, E consecutive entries
// each.  The per-token inputs of K tokens (B and C of the head's group, x of
// the CTA's rows, dt) are staged into shared memory with cp.async one chunk
// ahead of the compute; B and C go in chunk-interleaved order (16-byte chunk
// i of lane j at position i * LPR + j), so the lanes of a warp read
// consecutive 16-byte words.  lambda = exp(dt * A) is computed once per
// token per CTA.  The token loop streams each lane's entries in pieces of 16:
// the readout of the previous token and the update of this one in one pass,
// min / max, refit, then round and rescale.
#include "ssq_common.cuh"
#include "ssq_params.h"

#include <type_traits>

namespace ssq {

namespace {

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

// Geometry of one scan instantiation.
template <int N, int E>
struct SGeom {
    static constexpr int LPR = N / E;                 // lanes per row
    static constexpr int RPW = 32 / LPR;              // rows per warp
    static constexpr int NP = E / 16;                 // 16-entry pieces per lane
    static_assert(E % 16 == 0 && N % E == 0 && LPR <= 32, "bad scan shape");
};

// Staging buffers: chunk c is read from buffer c % 3 while chunk c + 1 is
// staged into the next; the third keeps chunk c - 1, whose last token's C the
// first token of chunk c still reads (the readout of token t is fused into
// the update of token t + 1).
constexpr int kScanBufs = 3;

// Floats of one staging buffer: B, C [K][N]; x [K][rows]; dt, lambda [K].
__host__ __device__ inline int scan_buf_floats(int N, int K, int rows)
{
    const int f = 2 * K * N + K * rows + 2 * K;
    return (f + 3) / 4 * 4;   // keep the next buffer 16-byte aligned
}

// Entries a lane owns for a given d_state: 64 when the batch gives at least
// one warp per SM sub-partition, else 32 (more warps for small batches).
__host__ __device__ inline int scan_entries(int N, bool wide)
{
    if (N < 64) return N;
    return wide ? 64 : 32;
}

// Round 16 entries of a row on the fast path: s <- fl(rint(s*inv) * Delta),
// the product s*inv exact (one FMA with the magic number); with CODES also
// the carriers of the stored codes.
template <int FMT, bool CODES>
__device__ __forceinline__ void round_piece_fast(const RowParams& rp, float* s,
                                                 uint32_t (&k)[16])
{
    using F = Fmt<FMT>;
    const float2 inv2 = make_float2(rp.inv, rp.inv);
    const float2 d2 = make_float2(rp.delta, rp.delta);
    const float2 m2 = make_float2(kMagic, kMagic);
    const float2 nm2 = make_float2(-kMagic, -kMagic);
    const float2 z2 = make_float2(rp.z, rp.z);
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
        const float2 t = fma2(make_float2(s[n], s[n + 1]), inv2, m2);   // 1.5*2^23 + rint(s*inv)
        const float2 r = add2(t, nm2);         // rint(p) = q - z, exact
        const float2 v = mul2(r, d2);
        s[n] = v.x; s[n + 1] = v.y;
        if constexpr (CODES) {
            if constexpr (F::sym) {
                k[n] = __float_as_uint(t.x);
                k[n + 1] = __float_as_uint(t.y);
            } else {
                const float2 u = add2(t, z2);  // 1.5*2^23 + q, exact
                k[n] = __float_as_uint(u.x);
                k[n + 1] = __float_as_uint(u.y);
            }
        }
    }
}

// Stochastic rounding of 16 entries on the fast path (see round16_sr): s <-
// fl((q - z) * Delta) with q = clamp(floor(s*inv + u) (+ z)); with CODES also
// the carriers of the stored codes.
template <int FMT, bool CODES>
__device__ __forceinline__ void round_piece_sr(const RowParams& rp, float* s,
                                               const float (&u)[16], uint32_t (&k)[16])
{
    using F = Fmt<FMT>;
    const float2 inv2 = make_float2(rp.inv, rp.inv);
    const float2 z2 = make_float2(rp.z, rp.z);
    const float mz = F::sym ? -kMagic : -__fadd_rn(kMagic, rp.z);
    const float2 mz2 = make_float2(mz, mz);
    const float2 d2 = make_float2(rp.delta, rp.delta);
    float r[16];
    uint32_t kk[16];
    round16_sr<FMT>(inv2, z2, mz2, s, u, r, kk);
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
        const float2 v = mul2(make_float2(r[n], r[n + 1]), d2);
        s[n] = v.x; s[n + 1] = v.y;
        if constexpr (CODES) {
            k[n] = kk[n];
            k[n + 1] = kk[n + 1];
        }
    }
}

// The stochastic rounding by the formulas verbatim.
template <int FMT>
__device__ __forceinline__ void round_piece_sr_slow(const RowParams& rp, float* s,
                                                    const float (&u)[16], uint32_t (&k)[16])
{
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        float r;
        const float c = round1_sr_exact<FMT>(s[n], rp.inv, rp.z, u[n], &r);
        s[n] = __fmul_rn(r, rp.delta);
        k[n] = (uint32_t)(int)c;
    }
}

// The scalar formulas verbatim, for rows the fast path does not cover.
template <int FMT>
__device__ __forceinline__ void round_piece_slow(const RowParams& rp, float* s,
                                                 uint32_t (&k)[16])
{
    using F = Fmt<FMT>;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const float rr = rint_prod(s[n], rp.inv);
        float c, r;
        if constexpr (F::sym) {
            c = fminf(fmaxf(rr, -F::qmax), F::qmax);
            r = c;
        } else {
            c = fminf(__fadd_rn(rr, rp.z), F::qmax);
            r = __fsub_rn(c, rp.z);
        }
        s[n] = __fmul_rn(r, rp.delta);
        k[n] = (uint32_t)(int)c;
    }
}

// PF (prefill hand-off): the state stays fp32 for all T tokens (y read from
// it) and is quantized, or bf16-rounded, once after the last token.
// SR: round stochastically at every token (draws keyed by cv.sr_seed,
// countered by row block, layer, slot and cv.sr_step + t).
template <int FMT, int N, int E, bool PF, bool SR>
__global__ void __launch_bounds__(64, E >= 64 ? 6 : 8)
scan_kernel(const __grid_constant__ PoolView pv, const __grid_constant__ CallView cv)
{
    using F = Fmt<FMT>;
    using SG = SGeom<N, E>;
    constexpr int LPR = SG::LPR, RPW = SG::RPW, NP = SG::NP;
    constexpr int CB = F::quant ? E * F::bits / 8 : 4;   // code bytes per lane
    constexpr int PW = Piece<FMT>::words;
    constexpr bool kBf16 = (FMT == SSQ_BF16);
    extern __shared__ __align__(16) float smem[];

    const int P = pv.P, H = pv.H, G = pv.G, T = cv.T;
    const int K = cv.scan_chunk;                         // tokens per staged chunk
    const int nthreads = blockDim.x;
    const int rows = (nthreads / 32) * RPW;             // rows per CTA
    const int bufsz = scan_buf_floats(N, K, rows);
    uint32_t* err = reinterpret_cast<uint32_t*>(pv.pool);

    // CTA -> (request, region, head, first row)
    const int per_b = cv.qtiles + cv.ftiles;
    const int b = blockIdx.x / per_b;
    const int k = blockIdx.x - b * per_b;
    const bool quant = k < cv.qtiles;
    const int kk = quant ? k : k - cv.qtiles;
    const int tph = cv.tiles_per_head;
    const int hrl = kk / tph;
    const int p0 = (kk - hrl * tph) * rows;
    const int regbase = quant ? 0 : pv.Hq;
    const int h = pv.perm[regbase + hrl];
    const int g = h / pv.hpg;
    const int slot = cv.slot_idx ? __ldg(cv.slot_idx + b) : b;
    if (slot < 0 || slot >= pv.n_slots) {
        if (threadIdx.x == 0) atomicOr(err, SSQ_DEVERR_SLOT);
        return;  // block-uniform, before any barrier
    }

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int rowc = (tid >> 5) * RPW + lane / LPR;      // row within the CTA
    const int j = lane % LPR;
    const bool active = p0 + rowc < P;
    const int rowe = active ? rowc : 0;                  // inactive rows shadow row p0
    const int p = p0 + rowe;
    const int rr = hrl * P + p;                          // row within its region
    const float Av = __ldg(cv.A + h);
    const float Dv = __ldg(cv.D + h);
    const long long bT = (long long)b * T;
    SrKey srk;
    if constexpr (SR) {
        srk.key = make_uint2((uint32_t)cv.sr_seed, (uint32_t)(cv.sr_seed >> 32));
        srk.layer = (uint32_t)cv.layer0;
        srk.slot = (uint32_t)slot;
        srk.step = cv.sr_step;
        srk.row_block = (uint32_t)(h * P + p) * (uint32_t)(N / 8);
    }

    // Stage tokens [t0, t0 + nt) into buffer `bi`.
    auto stage = [&](int t0, int bi) {
        float* sB = smem + bi * bufsz;
        float* sC = sB + K * N;
        float* sx = sC + K * N;
        float* sdt = sx + K * rows;
        const int nt = min(K, T - t0);
        constexpr int NC = N / 4;            // 16-byte chunks per row
        constexpr int CPL = E / 4;           // chunks per lane
        for (int i = tid; i < nt * NC; i += nthreads) {
            const int tt = i / NC, c = i % NC;
            const int dst = tt * N + ((c % CPL) * LPR + c / CPL) * 4;
            const long long src = ((bT + t0 + tt) * G + g) * N + 4 * c;
            cp_async16(sB + dst, cv.B + src);
            cp_async16(sC + dst, cv.C + src);
        }
        for (int i = tid; i < nt * rows; i += nthreads) {
            const int tt = i / rows, r = i - tt * rows;
            const int pr = p0 + (p0 + r < P ? r : 0);
            cp_async4(sx + i, cv.x + ((bT + t0 + tt) * H + h) * P + pr);
        }
        if (tid < nt) cp_async4(sdt + tid, cv.dt + (bT + t0 + tid) * H + h);
        cp_async_commit();
    };

    uint8_t* slot_base = pv.pool + pv.header_bytes + (long long)slot * pv.slot_bytes;
    const int layer = cv.layer0;
    uint8_t* crow = nullptr;
    uint8_t* mrow = nullptr;
    uint8_t* frow = nullptr;
    constexpr int EB = kBf16 ? 2 : 4;

    // The initial state, decoded once.
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

    RowParams rp{};
    uint32_t cw[F::quant ? CB / 4 : 1];
    bool finite_all = true;
    const long long HP = (long long)H * P;
    float* const yrow = cv.y + (bT * H + h) * P + p;   // y of this row at token 0
    const bool ylane = active && j == 0;
    const int nchunks = (T + K - 1) / K;
    // The readout of token t, y_t = C_t . s_t + D x_t, is formed while token
    // t + 1 updates the state: one pass over the entries reads s_t for both,
    // and the row sum of y_t overlaps the refit of token t + 1.
    const float* cprev = nullptr;     // C row of token t - 1 in shared memory
    float xprev = 0.0f;               // x of this row at token t - 1
    auto emit_y = [&](int t, float ysum, float xv) {
        if (ylane) __stcs(yrow + (long long)t * HP, __fadd_rn(ysum, __fmul_rn(Dv, xv)));
    };
    // C . s over the lane's entries, reduced over the row's lanes
    auto readout = [&](const float* crow_s) {
        const float4* c4 = reinterpret_cast<const float4*>(crow_s) + j;
        float2 accp[NP];
#pragma unroll
        for (int pc = 0; pc < NP; ++pc) {
            const float* sp = s + 16 * pc;
            float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 v = c4[(4 * pc + i) * LPR];
                acc = fma2(make_float2(v.x, v.y), make_float2(sp[4 * i], sp[4 * i + 1]), acc);
                acc = fma2(make_float2(v.z, v.w), make_float2(sp[4 * i + 2], sp[4 * i + 3]), acc);
            }
            accp[pc] = acc;
        }
        float2 acc = accp[0];
#pragma unroll
        for (int pc = 1; pc < NP; ++pc) acc = add2(acc, accp[pc]);
        return grp_sum<LPR>(__fadd_rn(acc.x, acc.y));
    };
    stage(0, 0);
    for (int c = 0; c < nchunks; ++c) {
        const int bi = c % kScanBufs;
        const int t0 = c * K;
        const int nt = min(K, T - t0);
        cp_async_wait_all();
        __syncthreads();   // chunk c visible to all; everyone is done with chunk c-2
        if (c + 1 < nchunks) stage(t0 + K, (c + 1) % kScanBufs);
        const float* sB = smem + bi * bufsz;
        const float* sC = sB + K * N;
        const float* sx = sC + K * N;
        float* sdt = const_cast<float*>(sx + K * rows);
        float* slam = sdt + K;
        if (tid < nt) slam[tid] = decay(sdt[tid], Av);
        __syncthreads();

        // Update one token's state (s <- lambda s + dt x B) with the min /
        // max of the result; with READ also the readout of the previous
        // token from the state before the update.  Returns x of this row.
        auto update = [&](auto read_tag, auto quant_tag, int tt, float& lo, float& hi,
                          float& yprev) {
            constexpr bool READ = decltype(read_tag)::value;
            constexpr bool MINMAX = decltype(quant_tag)::value;
            const float xv = sx[tt * rows + rowe];
            const float dtx = __fmul_rn(sdt[tt], xv);
            const float2 l2 = make_float2(slam[tt], slam[tt]);
            const float2 x2 = make_float2(dtx, dtx);
            const float4* b4 = reinterpret_cast<const float4*>(sB + tt * N) + j;
            const float4* c4 = reinterpret_cast<const float4*>(cprev) + j;
            float plo[NP], phi[NP];
            float2 accp[NP];
#pragma unroll
            for (int pc = 0; pc < NP; ++pc) {
                float* sp = s + 16 * pc;
                float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 v = b4[(4 * pc + i) * LPR];
                    const float2 s0 = make_float2(sp[4 * i], sp[4 * i + 1]);
                    const float2 s1 = make_float2(sp[4 * i + 2], sp[4 * i + 3]);
                    if constexpr (READ) {
                        const float4 cq = c4[(4 * pc + i) * LPR];
                        acc = fma2(make_float2(cq.x, cq.y), s0, acc);
                        acc = fma2(make_float2(cq.z, cq.w), s1, acc);
                    }
                    float2 u0 = fma2(l2, s0, mul2(x2, make_float2(v.x, v.y)));
                    float2 u1 = fma2(l2, s1, mul2(x2, make_float2(v.z, v.w)));
                    if constexpr (kBf16 && !PF) {
                        u0 = __bfloat1622float2(__float22bfloat162_rn(u0));
                        u1 = __bfloat1622float2(__float22bfloat162_rn(u1));
                    }
                    sp[4 * i] = u0.x; sp[4 * i + 1] = u0.y;
                    sp[4 * i + 2] = u1.x; sp[4 * i + 3] = u1.y;
                }
                accp[pc] = acc;
                if constexpr (MINMAX) minmax16(sp, plo[pc], phi[pc]);
            }
            if constexpr (MINMAX) {
                lo = plo[0];
                hi = phi[0];
#pragma unroll
                for (int pc = 1; pc < NP; ++pc) {
                    lo = fminf(lo, plo[pc]);
                    hi = fmaxf(hi, phi[pc]);
                }
            }
            if constexpr (READ) {
                float2 acc = accp[0];
#pragma unroll
                for (int pc = 1; pc < NP; ++pc) acc = add2(acc, accp[pc]);
                yprev = grp_sum<LPR>(__fadd_rn(acc.x, acc.y));
            }
            return xv;
        };
        // one token of a quantized row; CODES: also pack the stored codes
        auto qtoken = [&](auto codes_tag, int tt) {
            constexpr bool CODES = decltype(codes_tag)::value;
            float lo, hi, yprev = 0.0f;
            const int t = t0 + tt;
            float xv;
            if (t > 0) {
                xv = update(std::true_type{}, std::true_type{}, tt, lo, hi, yprev);
                emit_y(t - 1, yprev, xprev);
            } else {
                xv = update(std::false_type{}, std::true_type{}, tt, lo, hi, yprev);
            }
            rp = refit_from_minmax<FMT, LPR>(lo, hi);
            finite_all = finite_all && rp.finite;
            uint32_t kc[16];
            if constexpr (SR) {
                srk.step = cv.sr_step + (uint32_t)t;
                const bool sfast = __all_sync(0xffffffffu, rp.fast);
#pragma unroll
                for (int pc = 0; pc < NP; ++pc) {
                    float u[16];
                    sr_draws16(srk, j * E + 16 * pc, u);
                    if (sfast)
                        round_piece_sr<FMT, CODES>(rp, s + 16 * pc, u, kc);
                    else
                        round_piece_sr_slow<FMT>(rp, s + 16 * pc, u, kc);
                    if constexpr (CODES) pack16<FMT>(kc, cw + PW * pc);
                }
            } else if (__all_sync(0xffffffffu, rp.fast && !rp.clamp)) {
#pragma unroll
                for (int pc = 0; pc < NP; ++pc) {
                    round_piece_fast<FMT, CODES>(rp, s + 16 * pc, kc);
                    if constexpr (CODES) pack16<FMT>(kc, cw + PW * pc);
                }
            } else {
#pragma unroll
                for (int pc = 0; pc < NP; ++pc) {
                    round_piece_slow<FMT>(rp, s + 16 * pc, kc);
                    if constexpr (CODES) pack16<FMT>(kc, cw + PW * pc);
                }
            }
            cprev = sC + tt * N;
            xprev = xv;
        };
        // one token of an fp row (fp32 update, rounded to bf16 for bf16)
        auto ftoken = [&](int tt) {
            float lo, hi, yprev = 0.0f;
            const int t = t0 + tt;
            float xv;
            if (t > 0) {
                xv = update(std::true_type{}, std::false_type{}, tt, lo, hi, yprev);
                emit_y(t - 1, yprev, xprev);
            } else {
                xv = update(std::false_type{}, std::false_type{}, tt, lo, hi, yprev);
            }
            cprev = sC + tt * N;
            xprev = xv;
        };

        bool qdone = false;
        if constexpr (F::quant && !PF) {
            if (qrow) {
                qdone = true;
                // the final token also packs the codes that go back to the pool
                const int nmain = (t0 + nt == T) ? nt - 1 : nt;
                for (int tt = 0; tt < nmain; ++tt) qtoken(std::false_type{}, tt);
                if (nmain < nt) qtoken(std::true_type{}, nmain);
            }
        }
        if (!qdone)
            for (int tt = 0; tt < nt; ++tt) ftoken(tt);
    }
    // the readout of the last token
    emit_y(T - 1, readout(cprev), xprev);

    if constexpr (PF && F::quant) {
        // the hand-off: one refit and rounding of the final fp32 state (all
        // lanes of the warp take part in the row reductions)
        if (qrow) {
            float lo = s[0], hi = s[0];
#pragma unroll
            for (int pc = 0; pc < NP; ++pc) {
                float plo, phi;
                minmax16(s + 16 * pc, plo, phi);
                lo = fminf(lo, plo);
                hi = fmaxf(hi, phi);
            }
            rp = refit_from_minmax<FMT, LPR>(lo, hi);
            finite_all = rp.finite;
            uint32_t kc[16];
            if (__all_sync(0xffffffffu, rp.fast && !rp.clamp)) {
#pragma unroll
                for (int pc = 0; pc < NP; ++pc) {
                    round_piece_fast<FMT, true>(rp, s + 16 * pc, kc);
                    pack16<FMT>(kc, cw + PW * pc);
                }
            } else {
#pragma unroll
                for (int pc = 0; pc < NP; ++pc) {
                    round_piece_slow<FMT>(rp, s + 16 * pc, kc);
                    pack16<FMT>(kc, cw + PW * pc);
                }
            }
        }
    }

    // The final state back to the pool.
    if (!active) return;
    if (qrow) {
        if constexpr (F::quant) {
            Chunk<CB> c;
#pragma unroll
            for (int i = 0; i < CB / 4; ++i) c.w[i] = cw[i];
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
    } else {
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

template <int FMT, int N, int E, bool PF, bool SR>
cudaError_t launch_scan_ne(const PoolView& pv, const CallView& cv, int warps, int grid,
                           cudaStream_t st)
{
    using SG = SGeom<N, E>;
    const size_t smem =
        kScanBufs * (size_t)scan_buf_floats(N, cv.scan_chunk, warps * SG::RPW) * sizeof(float);
    auto kern = scan_kernel<FMT, N, E, PF, SR>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, 32 * warps, smem, st>>>(pv, cv);
    return cudaGetLastError();
}

template <int FMT, bool PF, bool SR>
cudaError_t launch_scan_fmt(const PoolView& pv, const CallView& cv, int E, int warps,
                            int grid, cudaStream_t st)
{
    switch (pv.N) {
    case 16: return launch_scan_ne<FMT, 16, 16, PF, SR>(pv, cv, warps, grid, st);
    case 32: return launch_scan_ne<FMT, 32, 32, PF, SR>(pv, cv, warps, grid, st);
    case 64:
        return E == 64 ? launch_scan_ne<FMT, 64, 64, PF, SR>(pv, cv, warps, grid, st)
                       : launch_scan_ne<FMT, 64, 32, PF, SR>(pv, cv, warps, grid, st);
    case 128:
        return E == 64 ? launch_scan_ne<FMT, 128, 64, PF, SR>(pv, cv, warps, grid, st)
                       : launch_scan_ne<FMT, 128, 32, PF, SR>(pv, cv, warps, grid, st);
    case 256:
        return E == 64 ? launch_scan_ne<FMT, 256, 64, PF, SR>(pv, cv, warps, grid, st)
                       : launch_scan_ne<FMT, 256, 32, PF, SR>(pv, cv, warps, grid, st);
    default: return cudaErrorInvalidValue;
    }
}

template <bool PF>
cudaError_t launch_scan_pf(const PoolView& pv, const CallView& cv, int fmt, int E, int w,
                           int g, cudaStream_t st)
{
    switch (fmt) {
    case SSQ_F32: return launch_scan_fmt<SSQ_F32, PF, false>(pv, cv, E, w, g, st);
    case SSQ_BF16: return launch_scan_fmt<SSQ_BF16, PF, false>(pv, cv, E, w, g, st);
    case SSQ_I8_SYM: return launch_scan_fmt<SSQ_I8_SYM, PF, false>(pv, cv, E, w, g, st);
    case SSQ_I8_ASYM: return launch_scan_fmt<SSQ_I8_ASYM, PF, false>(pv, cv, E, w, g, st);
    case SSQ_I4_SYM: return launch_scan_fmt<SSQ_I4_SYM, PF, false>(pv, cv, E, w, g, st);
    case SSQ_I4_ASYM: return launch_scan_fmt<SSQ_I4_ASYM, PF, false>(pv, cv, E, w, g, st);
    default: return cudaErrorInvalidValue;
    }
}

// stochastic rounding at every token: the integer formats only
cudaError_t launch_scan_sr(const PoolView& pv, const CallView& cv, int fmt, int E, int w,
                           int g, cudaStream_t st)
{
    switch (fmt) {
    case SSQ_I8_SYM: return launch_scan_fmt<SSQ_I8_SYM, false, true>(pv, cv, E, w, g, st);
    case SSQ_I8_ASYM: return launch_scan_fmt<SSQ_I8_ASYM, false, true>(pv, cv, E, w, g, st);
    case SSQ_I4_SYM: return launch_scan_fmt<SSQ_I4_SYM, false, true>(pv, cv, E, w, g, st);
    case SSQ_I4_ASYM: return launch_scan_fmt<SSQ_I4_ASYM, false, true>(pv, cv, E, w, g, st);
    default: return launch_scan_pf<false>(pv, cv, fmt, E, w, g, st);
    }
}

}  // namespace

ScanPlan scan_plan(int d_state, int headdim, long long batch_heads, int sms)
{
    // Wide rows (64 entries per lane: half the per-row refit and bookkeeping
    // per entry) unless that leaves fewer than one warp per SM
    // sub-partition; on the 370M-shaped batch of 8 (1024 warps) wide rows
    // measured 7 % faster than 32 entries per lane with twice the warps.
    const int N = d_state;
    const int rpw64 = 32 / (N / scan_entries(N, true));
    const long long warps64 = batch_heads * ((headdim + rpw64 - 1) / rpw64);
    const bool wide = (N < 64) || warps64 >= 4LL * sms;
    ScanPlan sp;
    sp.E = scan_entries(N, wide);
    const int rpw = 32 / (N / sp.E);
    // Two warps per CTA (one when the head has rows for only one): small
    // CTAs spread evenly over the SMs, and two warps halve the staging.
    const int wneed = (headdim + rpw - 1) / rpw;
    sp.warps = wneed < 2 ? 1 : 2;
    sp.rows = sp.warps * rpw;
    sp.tiles_per_head = (headdim + sp.rows - 1) / sp.rows;
    // Tokens per staged chunk: three buffers of B and C of K tokens stay
    // near 26 KB per CTA (eight CTAs fit an SM's shared memory).
    sp.chunk = N <= 128 ? 8 : 4;
    sp.smem_bytes = kScanBufs * (size_t)scan_buf_floats(N, sp.chunk, sp.rows) * sizeof(float);
    return sp;
}

cudaError_t launch_scan(const PoolView& pv, const CallView& cv, int fmt, const ScanPlan& sp,
                        bool prefill, bool sr, cudaStream_t st)
{
    const long long grid = (long long)cv.batch * (cv.qtiles + cv.ftiles);
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int g = (int)grid, E = sp.E, w = sp.warps;
    if (sr) return launch_scan_sr(pv, cv, fmt, E, w, g, st);
    return prefill ? launch_scan_pf<true>(pv, cv, fmt, E, w, g, st)
                   : launch_scan_pf<false>(pv, cv, fmt, E, w, g, st);
}

}  // namespace ssq
