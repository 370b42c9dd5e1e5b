// ssq_api.cu -- the extern "C" entry points of libssq: argument validation,
// pool layout, and dispatch to the kernel launchers.  Every check that can
// be made on the host is made here, before anything is launched; nothing in
// this file allocates device memory.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "ssq.h"
#include "ssq_params.h"

namespace {

thread_local char g_detail[256] = "";

// Test support (ssq_test_hooks): applied to the decode launches of this host
// thread.
thread_local int g_test_withhold = 0;
thread_local long long g_test_wait_limit = 0;

ssq_status fail(ssq_status s, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return s;
}

ssq_status cuda_fail(cudaError_t e, const char* what)
{
    return fail(SSQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool is_quant(ssq_format f) { return f >= SSQ_I8_SYM && f <= SSQ_I4_ASYM; }
bool is_sym(ssq_format f) { return f == SSQ_I8_SYM || f == SSQ_I4_SYM; }
int bits_of(ssq_format f)
{
    switch (f) {
    case SSQ_I8_SYM: case SSQ_I8_ASYM: return 8;
    case SSQ_I4_SYM: case SSQ_I4_ASYM: return 4;
    case SSQ_BF16: return 16;
    default: return 32;
    }
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Validate a config and fill the layout and the region permutation.
ssq_status layout_of(const ssq_config* cfg, ssq_layout* L, int32_t* perm)
{
    if (!cfg) return fail(SSQ_ERR_INVALID_ARG, "cfg is NULL");
    if (cfg->fmt < SSQ_F32 || cfg->fmt > SSQ_I4_ASYM)
        return fail(SSQ_ERR_INVALID_ARG, "unknown format %d", (int)cfg->fmt);
    if (cfg->n_layers < 1) return fail(SSQ_ERR_INVALID_ARG, "n_layers %d < 1", cfg->n_layers);
    if (cfg->n_slots < 1) return fail(SSQ_ERR_INVALID_ARG, "n_slots %d < 1", cfg->n_slots);
    if (cfg->nheads < 1 || cfg->nheads > SSQ_MAX_HEADS)
        return fail(SSQ_ERR_UNSUPPORTED, "nheads %d outside [1, %d]", cfg->nheads, SSQ_MAX_HEADS);
    if (cfg->headdim < 1) return fail(SSQ_ERR_INVALID_ARG, "headdim %d < 1", cfg->headdim);
    if (cfg->headdim > 2048)
        return fail(SSQ_ERR_UNSUPPORTED, "headdim %d > 2048", cfg->headdim);
    const int N = cfg->d_state;
    if (N != 16 && N != 32 && N != 64 && N != 128 && N != 256)
        return fail(SSQ_ERR_UNSUPPORTED, "d_state %d not in {16,32,64,128,256}", N);
    if (cfg->ngroups < 1 || cfg->nheads % cfg->ngroups != 0)
        return fail(SSQ_ERR_INVALID_ARG, "ngroups %d does not divide nheads %d",
                    cfg->ngroups, cfg->nheads);

    const bool q = is_quant(cfg->fmt);
    int hq = 0;
    for (int h = 0; h < cfg->nheads; ++h)
        if (q && (!cfg->head_mask || cfg->head_mask[h])) ++hq;
    const int hf = cfg->nheads - hq;
    if (perm) {
        int iq = 0, ifp = hq;
        for (int h = 0; h < cfg->nheads; ++h) {
            const bool hq_row = q && (!cfg->head_mask || cfg->head_mask[h]);
            perm[hq_row ? iq++ : ifp++] = h;
        }
    }

    const size_t P = (size_t)cfg->headdim, Nz = (size_t)N, Ly = (size_t)cfg->n_layers;
    memset(L, 0, sizeof(*L));
    L->header_bytes = SSQ_POOL_HEADER_BYTES;
    L->n_quant_heads = hq;
    L->n_fp_heads = hf;
    L->row_code_bytes = q ? Nz * bits_of(cfg->fmt) / 8 : 0;
    L->row_meta_bytes = q ? (is_sym(cfg->fmt) ? 4 : 8) : 0;
    L->fp_elem_bytes = cfg->fmt == SSQ_BF16 ? 2 : 4;
    // each layer's block starts on a SSQ_POOL_ALIGN boundary (bulk copies
    // need 16-byte aligned sources)
    L->codes_layer_bytes = round_up((size_t)hq * P * L->row_code_bytes, SSQ_POOL_ALIGN);
    L->meta_layer_bytes = round_up((size_t)hq * P * L->row_meta_bytes, SSQ_POOL_ALIGN);
    L->fp_layer_bytes = round_up((size_t)hf * P * Nz * L->fp_elem_bytes, SSQ_POOL_ALIGN);
    L->codes_off = 0;
    L->meta_off = round_up(L->codes_off + Ly * L->codes_layer_bytes, SSQ_POOL_ALIGN);
    L->fp_off = round_up(L->meta_off + Ly * L->meta_layer_bytes, SSQ_POOL_ALIGN);
    L->slot_bytes = round_up(L->fp_off + Ly * L->fp_layer_bytes, SSQ_POOL_ALIGN);
    // overflow guard: the pool must fit in 2^62 bytes
    const double total = (double)L->header_bytes + (double)L->slot_bytes * cfg->n_slots;
    if (total > 4.0e18) return fail(SSQ_ERR_INVALID_ARG, "pool size overflows");
    L->pool_bytes = L->header_bytes + L->slot_bytes * (size_t)cfg->n_slots;
    return SSQ_OK;
}

ssq_status make_pool_view(const ssq_config* cfg, void* pool, ssq::PoolView* pv,
                          ssq_layout* L)
{
    int32_t perm[SSQ_MAX_HEADS];
    ssq_status st = layout_of(cfg, L, perm);
    if (st != SSQ_OK) return st;
    if (!pool) return fail(SSQ_ERR_INVALID_ARG, "pool is NULL");
    if (!aligned(pool, SSQ_POOL_ALIGN))
        return fail(SSQ_ERR_ALIGNMENT, "pool not %d-byte aligned", SSQ_POOL_ALIGN);
    memset(pv, 0, sizeof(*pv));
    pv->pool = static_cast<uint8_t*>(pool);
    pv->header_bytes = (long long)L->header_bytes;
    pv->slot_bytes = (long long)L->slot_bytes;
    pv->codes_off = (long long)L->codes_off;
    pv->meta_off = (long long)L->meta_off;
    pv->fp_off = (long long)L->fp_off;
    pv->codes_layer_bytes = (long long)L->codes_layer_bytes;
    pv->meta_layer_bytes = (long long)L->meta_layer_bytes;
    pv->fp_layer_bytes = (long long)L->fp_layer_bytes;
    pv->n_slots = cfg->n_slots;
    pv->n_layers = cfg->n_layers;
    pv->H = cfg->nheads;
    pv->P = cfg->headdim;
    pv->N = cfg->d_state;
    pv->G = cfg->ngroups;
    pv->hpg = cfg->nheads / cfg->ngroups;
    pv->Hq = L->n_quant_heads;
    pv->Hf = L->n_fp_heads;
    pv->mP = ssq::fdiv_magic(pv->P);
    pv->mHpg = ssq::fdiv_magic(pv->hpg);
    for (int i = 0; i < cfg->nheads; ++i) pv->perm[i] = (uint16_t)perm[i];
    return SSQ_OK;
}

// Common checks of (slot_idx, batch, layer range).
ssq_status check_batch(const ssq_config* cfg, const int32_t* slot_idx, int batch,
                       int layer0, int nl)
{
    if (batch < 0) return fail(SSQ_ERR_INVALID_ARG, "batch %d < 0", batch);
    if (nl < 1) return fail(SSQ_ERR_INVALID_ARG, "nl %d < 1", nl);
    if (layer0 < 0 || (long long)layer0 + nl > cfg->n_layers)
        return fail(SSQ_ERR_INVALID_ARG, "layers [%d, %d) outside [0, %d)", layer0,
                    layer0 + nl, cfg->n_layers);
    if (!slot_idx && batch > cfg->n_slots)
        return fail(SSQ_ERR_INVALID_ARG, "batch %d > n_slots %d with identity slots",
                    batch, cfg->n_slots);
    if (slot_idx && !aligned(slot_idx, 4))
        return fail(SSQ_ERR_ALIGNMENT, "slot_idx not 4-byte aligned");
    return SSQ_OK;
}

ssq_status need(const void* p, const char* name, size_t align)
{
    if (!p) return fail(SSQ_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned(p, align)) return fail(SSQ_ERR_ALIGNMENT, "%s not %zu-byte aligned", name, align);
    return SSQ_OK;
}

#define SSQ_TRY(x)                         \
    do {                                   \
        ssq_status _s = (x);               \
        if (_s != SSQ_OK) return _s;       \
    } while (0)

void fill_tiles(const ssq::PoolView& pv, ssq::CallView* cv, int rows_q, int rows_f)
{
    const long long qrows = (long long)pv.Hq * pv.P, frows = (long long)pv.Hf * pv.P;
    cv->rows_per_tile = rows_q;
    cv->rows_per_tile_f = rows_f;
    cv->qtiles = (int)((qrows + rows_q - 1) / rows_q);
    cv->ftiles = (int)((frows + rows_f - 1) / rows_f);
    cv->total_tiles = (long long)cv->nl * cv->batch * (cv->qtiles + cv->ftiles);
}

}  // namespace

namespace ssq {

int grid_for(const void* kernel, int threads, long long tiles)
{
    int dev = 0, sms = 0, occ = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, 0) != cudaSuccess)
        return 0;
    if (occ < 1) occ = 1;
    long long g = (long long)sms * occ;
    if (g > tiles) g = tiles;
    return (int)g;
}

}  // namespace ssq

extern "C" {

const char* ssq_status_string(ssq_status s)
{
    switch (s) {
    case SSQ_OK: return "SSQ_OK";
    case SSQ_ERR_INVALID_ARG: return "SSQ_ERR_INVALID_ARG";
    case SSQ_ERR_UNSUPPORTED: return "SSQ_ERR_UNSUPPORTED";
    case SSQ_ERR_ALIGNMENT: return "SSQ_ERR_ALIGNMENT";
    case SSQ_ERR_CUDA: return "SSQ_ERR_CUDA";
    default: return "SSQ_ERR_UNKNOWN";
    }
}

const char* ssq_last_error_detail(void) { return g_detail; }

ssq_status ssq_test_hooks(int withhold_first_tile, long long wait_limit_cycles)
{
    if (wait_limit_cycles < 0)
        return fail(SSQ_ERR_INVALID_ARG, "wait_limit_cycles %lld < 0", wait_limit_cycles);
    g_test_withhold = withhold_first_tile ? 1 : 0;
    g_test_wait_limit = wait_limit_cycles;
    return SSQ_OK;
}

ssq_status ssq_pool_layout(const ssq_config* cfg, ssq_layout* out, int32_t* head_perm)
{
    if (!out) return fail(SSQ_ERR_INVALID_ARG, "out is NULL");
    return layout_of(cfg, out, head_perm);
}

ssq_status ssq_pool_init(const ssq_config* cfg, void* pool, cudaStream_t stream)
{
    ssq_layout L;
    SSQ_TRY(layout_of(cfg, &L, nullptr));
    SSQ_TRY(need(pool, "pool", SSQ_POOL_ALIGN));
    cudaError_t e = cudaMemsetAsync(pool, 0, L.pool_bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    return SSQ_OK;
}

ssq_status ssq_pool_error(const ssq_config* cfg, void* pool, uint32_t* flags,
                          cudaStream_t stream)
{
    ssq_layout L;
    SSQ_TRY(layout_of(cfg, &L, nullptr));
    SSQ_TRY(need(pool, "pool", SSQ_POOL_ALIGN));
    if (!flags) return fail(SSQ_ERR_INVALID_ARG, "flags is NULL");
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, pool, sizeof(v), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(pool, 0, sizeof(v), stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "reading the pool error word");
    *flags = v;
    return SSQ_OK;
}

ssq_status ssq_quantize_rows(const ssq_config* cfg, void* pool, const int32_t* slot_idx,
                             int batch, int layer0, int nl, const float* S,
                             cudaStream_t stream)
{
    ssq::PoolView pv;
    ssq_layout L;
    SSQ_TRY(make_pool_view(cfg, pool, &pv, &L));
    SSQ_TRY(check_batch(cfg, slot_idx, batch, layer0, nl));
    SSQ_TRY(need(S, "S", 16));
    if (batch == 0) return SSQ_OK;
    ssq::CallView cv;
    memset(&cv, 0, sizeof(cv));
    cv.slot_idx = slot_idx;
    cv.batch = batch;
    cv.layer0 = layer0;
    cv.nl = nl;
    cv.S_in = S;
    fill_tiles(pv, &cv, ssq::rows_per_tile(cfg->d_state), ssq::rows_per_tile(cfg->d_state));
    cudaError_t e = ssq::launch_quantize(pv, cv, (int)cfg->fmt, stream);
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    return SSQ_OK;
}

ssq_status ssq_dequantize_rows(const ssq_config* cfg, const void* pool,
                               const int32_t* slot_idx, int batch, int layer0, int nl,
                               float* S_out, cudaStream_t stream)
{
    ssq::PoolView pv;
    ssq_layout L;
    SSQ_TRY(make_pool_view(cfg, const_cast<void*>(pool), &pv, &L));
    SSQ_TRY(check_batch(cfg, slot_idx, batch, layer0, nl));
    SSQ_TRY(need(S_out, "S_out", 16));
    if (batch == 0) return SSQ_OK;
    ssq::CallView cv;
    memset(&cv, 0, sizeof(cv));
    cv.slot_idx = slot_idx;
    cv.batch = batch;
    cv.layer0 = layer0;
    cv.nl = nl;
    cv.S_out = S_out;
    fill_tiles(pv, &cv, ssq::rows_per_tile(cfg->d_state), ssq::rows_per_tile(cfg->d_state));
    cudaError_t e = ssq::launch_dequantize(pv, cv, (int)cfg->fmt, stream);
    if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
    return SSQ_OK;
}

ssq_status ssq_decode_diag(const ssq_config* cfg, const void* pool, const int32_t* slot_idx,
                           int batch, int layer0, int nl, const float* x, const float* B,
                           const float* C, const float* dt, const float* A, float* diag,
                           cudaStream_t stream)
{
    ssq::PoolView pv;
    ssq_layout L;
    SSQ_TRY(make_pool_view(cfg, const_cast<void*>(pool), &pv, &L));
    SSQ_TRY(check_batch(cfg, slot_idx, batch, layer0, nl));
    SSQ_TRY(need(x, "x", 4));
    SSQ_TRY(need(B, "B", 16));
    SSQ_TRY(need(C, "C", 16));
    SSQ_TRY(need(dt, "dt", 4));
    SSQ_TRY(need(A, "A", 4));
    SSQ_TRY(need(diag, "diag", 16));
    if (batch == 0) return SSQ_OK;
    ssq::CallView cv;
    memset(&cv, 0, sizeof(cv));
    cv.slot_idx = slot_idx;
    cv.batch = batch;
    cv.layer0 = layer0;
    cv.nl = nl;
    cv.x = x;
    cv.B = B;
    cv.C = C;
    cv.dt = dt;
    cv.A = A;
    cv.diag = diag;
    cv.wait_limit = g_test_wait_limit;
    if (!ssq::decode_fits((int)cfg->fmt, cfg->d_state, cfg->nheads, cfg->ngroups))
        return fail(SSQ_ERR_UNSUPPORTED, "ngroups*d_state %d too large for the decode kernel",
                    cfg->ngroups * cfg->d_state);
    int rows_q = 0, rows_f = 0;
    ssq::decode_tile_rows((int)cfg->fmt, cfg->d_state, &rows_q, &rows_f);
    fill_tiles(pv, &cv, rows_q, rows_f);
    cudaError_t e = ssq::launch_decode_diag(pv, cv, (int)cfg->fmt, stream);
    if (e != cudaSuccess) return cuda_fail(e, "diag launch");
    return SSQ_OK;
}

}  // extern "C"

namespace {

// ssq_decode_step and ssq_decode_step_sr: sr rounds the quantized rows
// stochastically with draws keyed by seed at step counter `step`.
ssq_status decode_common(const ssq_config* cfg, void* pool, const int32_t* slot_idx,
                         int batch, int layer0, int nl, const float* x, const float* B,
                         const float* C, const float* dt, const float* A, const float* D,
                         float* y, bool sr, uint64_t seed, uint32_t step, cudaStream_t stream)
{
    ssq::PoolView pv;
    ssq_layout L;
    SSQ_TRY(make_pool_view(cfg, pool, &pv, &L));
    SSQ_TRY(check_batch(cfg, slot_idx, batch, layer0, nl));
    SSQ_TRY(need(x, "x", 16));
    SSQ_TRY(need(B, "B", 16));
    SSQ_TRY(need(C, "C", 16));
    SSQ_TRY(need(dt, "dt", 4));
    SSQ_TRY(need(A, "A", 4));
    SSQ_TRY(need(D, "D", 4));
    SSQ_TRY(need(y, "y", 16));
    if (batch == 0) return SSQ_OK;
    ssq::CallView cv;
    memset(&cv, 0, sizeof(cv));
    cv.slot_idx = slot_idx;
    cv.batch = batch;
    cv.layer0 = layer0;
    cv.nl = nl;
    cv.x = x;
    cv.B = B;
    cv.C = C;
    cv.dt = dt;
    cv.A = A;
    cv.D = D;
    cv.y = y;
    cv.sr_seed = seed;
    cv.sr_step = step;
    cv.wait_limit = g_test_wait_limit;
    cv.test_withhold = g_test_withhold;
    if (!ssq::decode_fits((int)cfg->fmt, cfg->d_state, cfg->nheads, cfg->ngroups))
        return fail(SSQ_ERR_UNSUPPORTED, "ngroups*d_state %d too large for the decode kernel",
                    cfg->ngroups * cfg->d_state);
    int rows_q = 0, rows_f = 0;
    ssq::decode_tile_rows((int)cfg->fmt, cfg->d_state, &rows_q, &rows_f);
    fill_tiles(pv, &cv, rows_q, rows_f);
    cudaError_t e = ssq::launch_decode(pv, cv, (int)cfg->fmt, sr, stream);
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return SSQ_OK;
}


// ssq_scan, ssq_scan_sr and ssq_prefill: the same launch geometry; prefill
// keeps the state fp32 across the tokens and quantizes it once at the end;
// sr rounds stochastically at every token (token t at step counter
// step0 + t).
ssq_status scan_common(const ssq_config* cfg, void* pool, const int32_t* slot_idx, int batch,
                       int layer, int T, const float* x, const float* B, const float* C,
                       const float* dt, const float* A, const float* D, float* y,
                       bool prefill, bool sr, uint64_t seed, uint32_t step0,
                       cudaStream_t stream)
{
    ssq::PoolView pv;
    ssq_layout L;
    SSQ_TRY(make_pool_view(cfg, pool, &pv, &L));
    SSQ_TRY(check_batch(cfg, slot_idx, batch, layer, 1));
    if (T < 0) return fail(SSQ_ERR_INVALID_ARG, "T %d < 0", T);
    SSQ_TRY(need(x, "x", 16));
    SSQ_TRY(need(B, "B", 16));
    SSQ_TRY(need(C, "C", 16));
    SSQ_TRY(need(dt, "dt", 4));
    SSQ_TRY(need(A, "A", 4));
    SSQ_TRY(need(D, "D", 4));
    SSQ_TRY(need(y, "y", 16));
    if (batch == 0 || T == 0) return SSQ_OK;
    ssq::CallView cv;
    memset(&cv, 0, sizeof(cv));
    cv.slot_idx = slot_idx;
    cv.batch = batch;
    cv.layer0 = layer;
    cv.nl = 1;
    cv.T = T;
    cv.x = x;
    cv.B = B;
    cv.C = C;
    cv.dt = dt;
    cv.A = A;
    cv.D = D;
    cv.y = y;
    cv.sr_seed = seed;
    cv.sr_step = step0;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    const ssq::ScanPlan sp = ssq::scan_plan(cfg->d_state, cfg->headdim,
                                            (long long)batch * cfg->nheads, sms);
    cv.tiles_per_head = sp.tiles_per_head;
    cv.scan_chunk = sp.chunk;
    cv.qtiles = pv.Hq * sp.tiles_per_head;
    cv.ftiles = pv.Hf * sp.tiles_per_head;
    cv.total_tiles = (long long)batch * (cv.qtiles + cv.ftiles);
    e = ssq::launch_scan(pv, cv, (int)cfg->fmt, sp, prefill, sr, stream);
    if (e != cudaSuccess) return cuda_fail(e, prefill ? "prefill launch" : "scan launch");
    return SSQ_OK;
}

}  // namespace

extern "C" {

ssq_status ssq_decode_step(const ssq_config* cfg, void* pool, const int32_t* slot_idx,
                           int batch, int layer0, int nl, const float* x, const float* B,
                           const float* C, const float* dt, const float* A, const float* D,
                           float* y, cudaStream_t stream)
{
    return decode_common(cfg, pool, slot_idx, batch, layer0, nl, x, B, C, dt, A, D, y, false,
                         0, 0, stream);
}

ssq_status ssq_decode_step_sr(const ssq_config* cfg, void* pool, const int32_t* slot_idx,
                              int batch, int layer0, int nl, const float* x, const float* B,
                              const float* C, const float* dt, const float* A,
                              const float* D, float* y, uint64_t seed, uint32_t step,
                              cudaStream_t stream)
{
    return decode_common(cfg, pool, slot_idx, batch, layer0, nl, x, B, C, dt, A, D, y, true,
                         seed, step, stream);
}

ssq_status ssq_scan(const ssq_config* cfg, void* pool, const int32_t* slot_idx, int batch,
                    int layer, int T, const float* x, const float* B, const float* C,
                    const float* dt, const float* A, const float* D, float* y,
                    cudaStream_t stream)
{
    return scan_common(cfg, pool, slot_idx, batch, layer, T, x, B, C, dt, A, D, y, false,
                       false, 0, 0, stream);
}

ssq_status ssq_scan_sr(const ssq_config* cfg, void* pool, const int32_t* slot_idx, int batch,
                       int layer, int T, const float* x, const float* B, const float* C,
                       const float* dt, const float* A, const float* D, float* y,
                       uint64_t seed, uint32_t step0, cudaStream_t stream)
{
    return scan_common(cfg, pool, slot_idx, batch, layer, T, x, B, C, dt, A, D, y, false,
                       true, seed, step0, stream);
}

ssq_status ssq_prefill(const ssq_config* cfg, void* pool, const int32_t* slot_idx, int batch,
                       int layer, int T, const float* x, const float* B, const float* C,
                       const float* dt, const float* A, const float* D, float* y,
                       cudaStream_t stream)
{
    return scan_common(cfg, pool, slot_idx, batch, layer, T, x, B, C, dt, A, D, y, true,
                       false, 0, 0, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// DAMP mixed-tier pool
// ---------------------------------------------------------------------------
namespace {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

ssq_status damp_layout_of(const ssq_damp_config* c, ssq_damp_layout* L)
{
    if (!c) return fail(SSQ_ERR_INVALID_ARG, "cfg is NULL");
    if (c->n_layers < 1 || c->n_slots < 1)
        return fail(SSQ_ERR_INVALID_ARG, "n_layers %d / n_slots %d < 1", c->n_layers, c->n_slots);
    if (c->nheads < 1 || c->nheads > SSQ_MAX_HEADS)
        return fail(SSQ_ERR_INVALID_ARG, "nheads %d outside [1, %d]", c->nheads, SSQ_MAX_HEADS);
    if (c->headdim != 16 && c->headdim != 32 && c->headdim != 64 && c->headdim != 128)
        return fail(SSQ_ERR_UNSUPPORTED, "headdim %d not 16, 32, 64 or 128", c->headdim);
    if (c->d_state < 16 || c->d_state > 256 || c->d_state % 16 != 0)
        return fail(SSQ_ERR_UNSUPPORTED, "d_state %d not a multiple of 16 in [16, 256]",
                    c->d_state);
    if (c->ngroups < 1 || c->nheads % c->ngroups != 0)
        return fail(SSQ_ERR_INVALID_ARG, "ngroups %d does not divide nheads %d", c->ngroups,
                    c->nheads);
    if (c->n_protected < 0 || c->n_protected > c->d_state)
        return fail(SSQ_ERR_INVALID_ARG, "n_protected %d outside [0, %d]", c->n_protected,
                    c->d_state);
    const size_t P = (size_t)c->headdim, N = (size_t)c->d_state, K = (size_t)c->n_protected;
    memset(L, 0, sizeof(*L));
    L->header_bytes = SSQ_POOL_HEADER_BYTES;
    L->hi_off = 0;
    L->codes_off = align_up(2 * K * P, 16);
    L->meta_off = L->codes_off + align_up((N - K) * P, 16);
    L->head_bytes = align_up(L->meta_off + 8 * (N - K), 16);
    L->layer_bytes = L->head_bytes * (size_t)c->nheads;
    L->slot_bytes = align_up(L->layer_bytes * (size_t)c->n_layers, SSQ_POOL_ALIGN);
    L->pool_bytes = L->header_bytes + L->slot_bytes * (size_t)c->n_slots;
    L->bits_per_value = (16.0 * K * P + 8.0 * (N - K) * P + 64.0 * (N - K)) / (double)(N * P);
    return SSQ_OK;
}

ssq_status damp_view(const ssq_damp_config* c, void* pool, const int32_t* chan,
                     ssq::DampView* dv)
{
    ssq_damp_layout L;
    SSQ_TRY(damp_layout_of(c, &L));
    SSQ_TRY(need(pool, "pool", SSQ_POOL_ALIGN));
    SSQ_TRY(need(chan, "chan", 4));
    memset(dv, 0, sizeof(*dv));
    dv->pool = static_cast<uint8_t*>(pool);
    dv->header_bytes = (long long)L.header_bytes;
    dv->slot_bytes = (long long)L.slot_bytes;
    dv->layer_bytes = (long long)L.layer_bytes;
    dv->head_bytes = (long long)L.head_bytes;
    dv->hi_off = (int)L.hi_off;
    dv->codes_off = (int)L.codes_off;
    dv->meta_off = (int)L.meta_off;
    dv->n_slots = c->n_slots;
    dv->n_layers = c->n_layers;
    dv->H = c->nheads;
    dv->P = c->headdim;
    dv->N = c->d_state;
    dv->G = c->ngroups;
    dv->hpg = c->nheads / c->ngroups;
    dv->K = c->n_protected;
    dv->chan = chan;
    return SSQ_OK;
}

ssq_status damp_check_batch(const ssq_damp_config* c, const int32_t* slot_idx, int batch,
                            int layer0, int nl)
{
    if (batch < 0) return fail(SSQ_ERR_INVALID_ARG, "batch %d < 0", batch);
    if (nl < 1) return fail(SSQ_ERR_INVALID_ARG, "nl %d < 1", nl);
    if (layer0 < 0 || (long long)layer0 + nl > c->n_layers)
        return fail(SSQ_ERR_INVALID_ARG, "layers [%d, %d) outside [0, %d)", layer0,
                    layer0 + nl, c->n_layers);
    if (!slot_idx && batch > c->n_slots)
        return fail(SSQ_ERR_INVALID_ARG, "batch %d > n_slots %d with identity slots", batch,
                    c->n_slots);
    if (slot_idx && !aligned(slot_idx, 4))
        return fail(SSQ_ERR_ALIGNMENT, "slot_idx not 4-byte aligned");
    return SSQ_OK;
}

ssq::DampCall damp_call(const int32_t* slot_idx, int batch, int layer0, int nl)
{
    ssq::DampCall dc;
    memset(&dc, 0, sizeof(dc));
    dc.slot_idx = slot_idx;
    dc.batch = batch;
    dc.layer0 = layer0;
    dc.nl = nl;
    return dc;
}

}  // namespace

extern "C" {

ssq_status ssq_damp_pool_layout(const ssq_damp_config* cfg, ssq_damp_layout* out)
{
    if (!out) return fail(SSQ_ERR_INVALID_ARG, "out is NULL");
    return damp_layout_of(cfg, out);
}

ssq_status ssq_damp_quantize(const ssq_damp_config* cfg, void* pool, const int32_t* chan,
                             const int32_t* slot_idx, int batch, int layer0, int nl,
                             const float* S, cudaStream_t stream)
{
    ssq::DampView dv;
    SSQ_TRY(damp_view(cfg, pool, chan, &dv));
    SSQ_TRY(damp_check_batch(cfg, slot_idx, batch, layer0, nl));
    SSQ_TRY(need(S, "S", 16));
    if (batch == 0) return SSQ_OK;
    ssq::DampCall dc = damp_call(slot_idx, batch, layer0, nl);
    dc.S_in = S;
    cudaError_t e = ssq::launch_damp(dv, dc, 1, stream);
    if (e != cudaSuccess) return cuda_fail(e, "damp quantize launch");
    return SSQ_OK;
}

ssq_status ssq_damp_dequantize(const ssq_damp_config* cfg, const void* pool,
                               const int32_t* chan, const int32_t* slot_idx, int batch,
                               int layer0, int nl, float* S_out, cudaStream_t stream)
{
    ssq::DampView dv;
    SSQ_TRY(damp_view(cfg, const_cast<void*>(pool), chan, &dv));
    SSQ_TRY(damp_check_batch(cfg, slot_idx, batch, layer0, nl));
    SSQ_TRY(need(S_out, "S_out", 16));
    if (batch == 0) return SSQ_OK;
    ssq::DampCall dc = damp_call(slot_idx, batch, layer0, nl);
    dc.S_out = S_out;
    cudaError_t e = ssq::launch_damp(dv, dc, 2, stream);
    if (e != cudaSuccess) return cuda_fail(e, "damp dequantize launch");
    return SSQ_OK;
}

ssq_status ssq_damp_decode_step(const ssq_damp_config* cfg, void* pool, const int32_t* chan,
                                const int32_t* slot_idx, int batch, int layer0, int nl,
                                const float* x, const float* B, const float* C,
                                const float* dt, const float* A, const float* D, float* y,
                                cudaStream_t stream)
{
    ssq::DampView dv;
    SSQ_TRY(damp_view(cfg, pool, chan, &dv));
    SSQ_TRY(damp_check_batch(cfg, slot_idx, batch, layer0, nl));
    SSQ_TRY(need(x, "x", 4));
    SSQ_TRY(need(B, "B", 4));
    SSQ_TRY(need(C, "C", 4));
    SSQ_TRY(need(dt, "dt", 4));
    SSQ_TRY(need(A, "A", 4));
    SSQ_TRY(need(D, "D", 4));
    SSQ_TRY(need(y, "y", 4));
    if (batch == 0) return SSQ_OK;
    ssq::DampCall dc = damp_call(slot_idx, batch, layer0, nl);
    dc.x = x;
    dc.B = B;
    dc.C = C;
    dc.dt = dt;
    dc.A = A;
    dc.D = D;
    dc.y = y;
    cudaError_t e = ssq::launch_damp(dv, dc, 0, stream);
    if (e != cudaSuccess) return cuda_fail(e, "damp decode launch");
    return SSQ_OK;
}

ssq_status ssq_damp_pool_error(const ssq_damp_config* cfg, void* pool, uint32_t* flags,
                               cudaStream_t stream)
{
    ssq_damp_layout L;
    SSQ_TRY(damp_layout_of(cfg, &L));
    SSQ_TRY(need(pool, "pool", SSQ_POOL_ALIGN));
    if (!flags) return fail(SSQ_ERR_INVALID_ARG, "flags is NULL");
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, pool, sizeof(v), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(pool, 0, sizeof(v), stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "reading the pool error word");
    *flags = v;
    return SSQ_OK;
}

}  // extern "C"
