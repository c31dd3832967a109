// C ABI of the PD-SSM scan library: argument checks, workspace planning and
// the launch sequence of each call.  Every call is asynchronous on the
// caller's stream unless its declaration in pdssm.h says otherwise.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"

using namespace pdssm;

namespace {

thread_local char g_last_error[256] = "";

pdssm_status cuda_fail(cudaError_t e, const char *where) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
    return PDSSM_ERR_CUDA;
}

pdssm_status arg_fail(pdssm_status st, const char *why) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", why);
    return st;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

int stage_override() {
    static const int v = [] {
        const char *e = getenv("PDSSM_STAGES");
        const int n = e ? atoi(e) : 0;
        return (n >= 2 && n <= kMaxStages) ? n : 0;
    }();
    return v;
}

size_t dtype_size(pdssm_dtype t) { return t == PDSSM_BF16 ? 2 : 4; }

// Shape checks shared by the scan calls.
pdssm_status check_scan_dims(const pdssm_dims *dm, int64_t pi_hs, int64_t chunk) {
    if (!dm) return arg_fail(PDSSM_ERR_INVALID_ARG, "dims is NULL");
    if (dm->B < 1 || dm->H < 1 || dm->L < 0 || dm->N < 1 || dm->K < 1)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "need B, H, N, K >= 1 and L >= 0");
    if (chunk < 1) return arg_fail(PDSSM_ERR_INVALID_ARG, "chunk must be >= 1");
    if (dm->N > kMaxN) return arg_fail(PDSSM_ERR_UNSUPPORTED, "N > 64");
    if (dm->K > 32) return arg_fail(PDSSM_ERR_UNSUPPORTED, "K > 32");
    if (pi_hs != 0 && pi_hs < dm->K * dm->N)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "pi_head_stride must be 0 or >= K*N");
    if (dm->B * dm->H * dm->L > ((int64_t)1 << 40))
        return arg_fail(PDSSM_ERR_UNSUPPORTED, "B*H*L too large");
    return PDSSM_OK;
}

pdssm_status check_dtype(pdssm_dtype t) {
    if (t != PDSSM_F32 && t != PDSSM_BF16)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "unknown dtype");
    return PDSSM_OK;
}

// Fill the parameters shared by all chunk kernels.
ChunkParams make_params(const pdssm_dims *dm, const WsLayout &w, void *ws, int64_t chunk,
                        const int32_t *k, const void *d, const void *b, const void *c,
                        pdssm_dtype dt) {
    ChunkParams p;
    memset(&p, 0, sizeof(p));
    p.B = dm->B;
    p.H = dm->H;
    p.L = dm->L;
    p.N = dm->N;
    p.K = dm->K;
    p.C = w.C;
    p.chunk = chunk;
    p.units = dm->B * dm->H * w.C;
    p.dict_hs = w.Hd > 1 ? dm->K * dm->N : 0;
    unsigned char *base = reinterpret_cast<unsigned char *>(ws);
    p.dict = reinterpret_cast<const int32_t *>(base + w.dict);
    p.tab = reinterpret_cast<const uint8_t *>(base + w.tab);
    p.fan = reinterpret_cast<const int32_t *>(base + w.fan);
    p.seg = reinterpret_cast<const uint2 *>(base + w.seg);
    p.dict_stats = reinterpret_cast<const int *>(base + w.status) + 1;
    p.k = k;
    p.d = d;
    p.b = b;
    p.c = c;
    p.Pi = reinterpret_cast<int32_t *>(base + w.Pi);
    p.Dl = reinterpret_cast<float *>(base + w.Dl);
    p.v = reinterpret_cast<float *>(base + w.v);
    p.Hc = reinterpret_cast<float *>(base + w.Hc);
    if (w.wc) p.wc = reinterpret_cast<float *>(base + w.wc);
    if (w.lam) p.lam = reinterpret_cast<float *>(base + w.lam);
    p.status = reinterpret_cast<int *>(base + w.status);
    const int es = (int)dtype_size(dt);
    const int rowb = (int)dm->N * es;
    const bool vec_ok = (rowb % 16) == 0;
    const bool ptr_ok = (!d || aligned(d, 16)) && (!b || aligned(b, 16)) && (!c || aligned(c, 16));
    p.bulk = (vec_ok && ptr_ok) ? 1 : 0;
    // double-buffered tiles (plus L2 prefetch further ahead); PDSSM_STAGES
    // overrides the depth (2..4) for tuning
    p.ns = stage_override() > 0 ? stage_override() : 2;
    return p;
}

}  // namespace

// The tensor-core selection path is the default where it applies;
// PDSSM_SELECT_FMA=1 forces the plain fma-chain kernel (for comparisons).
bool pdssm::select_tc_enabled() {
    static const bool on = [] {
        const char *e = getenv("PDSSM_SELECT_FMA");
        return !(e && atoi(e) != 0);
    }();
    return on;
}

extern "C" {

const char *pdssm_status_str(int status) {
    switch (status) {
        case PDSSM_OK: return "PDSSM_OK";
        case PDSSM_ERR_INVALID_ARG: return "PDSSM_ERR_INVALID_ARG";
        case PDSSM_ERR_UNSUPPORTED: return "PDSSM_ERR_UNSUPPORTED";
        case PDSSM_ERR_BAD_INDEX: return "PDSSM_ERR_BAD_INDEX";
        case PDSSM_ERR_CUDA: return "PDSSM_ERR_CUDA";
        case PDSSM_ERR_TIMEOUT: return "PDSSM_ERR_TIMEOUT";
        case PDSSM_ERR_WORKSPACE: return "PDSSM_ERR_WORKSPACE";
        default: return "PDSSM_ERR_UNKNOWN";
    }
}

const char *pdssm_last_error(void) { return g_last_error; }

int pdssm_version(void) { return 100; }

size_t pdssm_workspace_bytes(const pdssm_dims *dims, int64_t pi_head_stride, int64_t chunk,
                             int for_bwd) {
    if (check_scan_dims(dims, pi_head_stride, chunk) != PDSSM_OK) return 0;
    return ws_layout(*dims, pi_head_stride, chunk, for_bwd != 0).total;
}

pdssm_status pdssm_select(const pdssm_dims *dims, const void *u, pdssm_dtype u_dtype,
                          const float *W_sel, int32_t *k_out, void *stream) {
    if (!dims) return arg_fail(PDSSM_ERR_INVALID_ARG, "dims is NULL");
    if (check_dtype(u_dtype) != PDSSM_OK) return PDSSM_ERR_INVALID_ARG;
    if (dims->B < 1 || dims->H < 1 || dims->L < 0 || dims->K < 1 || dims->D_in < 1)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "need B, H, K, D_in >= 1 and L >= 0");
    if (dims->K > 32) return arg_fail(PDSSM_ERR_UNSUPPORTED, "K > 32");
    if (dims->D_in > 256) return arg_fail(PDSSM_ERR_UNSUPPORTED, "D_in > 256");
    if (dims->L == 0) return PDSSM_OK;
    if (!u || !W_sel || !k_out) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(W_sel, 16)) return arg_fail(PDSSM_ERR_INVALID_ARG, "W_sel not 16-byte aligned");
    cudaError_t e = launch_select(*dims, u, u_dtype, W_sel, k_out, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "select");
    return PDSSM_OK;
}

static pdssm_status fwd_common(const pdssm_dims *dims, const int32_t *pi_dict,
                               int64_t pi_head_stride, const int32_t *k, const void *d,
                               const void *b, pdssm_dtype in_dtype, int64_t chunk, void *ws,
                               size_t ws_bytes, bool for_bwd, WsLayout *wout) {
    pdssm_status st = check_scan_dims(dims, pi_head_stride, chunk);
    if (st != PDSSM_OK) return st;
    if (check_dtype(in_dtype) != PDSSM_OK) return PDSSM_ERR_INVALID_ARG;
    if (!pi_dict || !ws) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL dictionary or workspace");
    if (dims->L > 0 && (!k || !d || !b))
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(ws, 256)) return arg_fail(PDSSM_ERR_INVALID_ARG, "ws not 256-byte aligned");
    const WsLayout w = ws_layout(*dims, pi_head_stride, chunk, for_bwd);
    if (ws_bytes < w.total) return arg_fail(PDSSM_ERR_WORKSPACE, "workspace too small");
    *wout = w;
    return PDSSM_OK;
}

static pdssm_status run_prep(const pdssm_dims *dims, const int32_t *pi_dict,
                             int64_t pi_head_stride, const WsLayout &w, void *ws,
                             cudaStream_t st) {
    unsigned char *base = reinterpret_cast<unsigned char *>(ws);
    // status word and the dictionary statistics (largest segment lane
    // distance, largest fan-in)
    cudaError_t e = cudaMemsetAsync(base + w.status, 0, 16, st);
    if (e != cudaSuccess) return cuda_fail(e, "status reset");
    e = launch_prep(*dims, pi_dict, pi_head_stride, reinterpret_cast<int32_t *>(base + w.dict),
                    reinterpret_cast<uint2 *>(base + w.seg),
                    reinterpret_cast<int *>(base + w.status) + 1,
                    reinterpret_cast<uint8_t *>(base + w.tab),
                    reinterpret_cast<int32_t *>(base + w.fan), w.Hd,
                    reinterpret_cast<int *>(base + w.status), st);
    if (e != cudaSuccess) return cuda_fail(e, "prep");
    return PDSSM_OK;
}

pdssm_status pdssm_scan_fwd(const pdssm_dims *dims, const int32_t *pi_dict,
                            int64_t pi_head_stride, const int32_t *k, const void *d,
                            const void *b, const void *c, pdssm_dtype in_dtype, const float *h0,
                            float *y, float *h_last, int64_t chunk, void *ws, size_t ws_bytes,
                            void *stream) {
    WsLayout w;
    pdssm_status st = fwd_common(dims, pi_dict, pi_head_stride, k, d, b, in_dtype, chunk, ws,
                                 ws_bytes, false, &w);
    if (st != PDSSM_OK) return st;
    if (dims->L > 0 && (!c || !y)) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL c or y");
    cudaStream_t s = (cudaStream_t)stream;
    st = run_prep(dims, pi_dict, pi_head_stride, w, ws, s);
    if (st != PDSSM_OK) return st;
    if (dims->L == 0) {
        if (h_last) {
            const size_t bytes = (size_t)(dims->B * dims->H * dims->N) * 4;
            cudaError_t e = h0 ? cudaMemcpyAsync(h_last, h0, bytes, cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(h_last, 0, bytes, s);
            if (e != cudaSuccess) return cuda_fail(e, "h_last for L = 0");
        }
        return PDSSM_OK;
    }
    ChunkParams p = make_params(dims, w, ws, chunk, k, d, b, c, in_dtype);
    p.h0 = h0;
    p.y = y;
    p.h_last = h_last;
    cudaError_t e = launch_phaseA(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "phase A");
    e = launch_phaseB(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "phase B");
    e = launch_phaseC(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "phase C");
    return PDSSM_OK;
}

pdssm_status pdssm_scan_bwd(const pdssm_dims *dims, const int32_t *pi_dict,
                            int64_t pi_head_stride, const int32_t *k, const void *d,
                            const void *b, const void *c, pdssm_dtype in_dtype, const float *h0,
                            const float *g_y, const float *g_hlast, float *g_b, float *g_d,
                            float *g_c, float *g_h0, int64_t chunk, void *ws, size_t ws_bytes,
                            void *stream) {
    WsLayout w;
    pdssm_status st = fwd_common(dims, pi_dict, pi_head_stride, k, d, b, in_dtype, chunk, ws,
                                 ws_bytes, true, &w);
    if (st != PDSSM_OK) return st;
    if (chunk > kBwdMaxChunk && dims->L > kBwdMaxChunk)
        return arg_fail(PDSSM_ERR_UNSUPPORTED, "backward needs chunk <= 256");
    if (dims->L > 0 && (!c || !g_y || !g_b || !g_d || !g_c))
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL tensor pointer");
    cudaStream_t s = (cudaStream_t)stream;
    if (dims->L == 0) {
        if (g_h0) {
            const size_t bytes = (size_t)(dims->B * dims->H * dims->N) * 4;
            cudaError_t e = g_hlast
                                ? cudaMemcpyAsync(g_h0, g_hlast, bytes, cudaMemcpyDeviceToDevice, s)
                                : cudaMemsetAsync(g_h0, 0, bytes, s);
            if (e != cudaSuccess) return cuda_fail(e, "g_h0 for L = 0");
        }
        return PDSSM_OK;
    }
    ChunkParams p = make_params(dims, w, ws, chunk, k, d, b, c, in_dtype);
    p.h0 = h0;
    p.g_y = g_y;
    p.g_hlast = g_hlast;
    p.g_b = g_b;
    p.g_d = g_d;
    p.g_c = g_c;
    p.g_h0 = g_h0;
    cudaError_t e = launch_bwdA(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "bwd phase A");
    e = launch_bwdB(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "bwd phase B");
    e = launch_bwdC(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "bwd phase C");
    return PDSSM_OK;
}

pdssm_status pdssm_chunk_transfers(const pdssm_dims *dims, const int32_t *pi_dict,
                                   int64_t pi_head_stride, const int32_t *k, const void *d,
                                   const void *b, pdssm_dtype in_dtype, int64_t chunk,
                                   int32_t *Pi_out, float *Delta_out, float *v_out, void *ws,
                                   size_t ws_bytes, void *stream) {
    WsLayout w;
    pdssm_status st = fwd_common(dims, pi_dict, pi_head_stride, k, d, b, in_dtype, chunk, ws,
                                 ws_bytes, false, &w);
    if (st != PDSSM_OK) return st;
    if (dims->L > 0 && (!Pi_out || !Delta_out || !v_out))
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL output pointer");
    cudaStream_t s = (cudaStream_t)stream;
    st = run_prep(dims, pi_dict, pi_head_stride, w, ws, s);
    if (st != PDSSM_OK) return st;
    if (dims->L == 0) return PDSSM_OK;
    ChunkParams p = make_params(dims, w, ws, chunk, k, d, b, nullptr, in_dtype);
    p.Pi = Pi_out;
    p.Dl = Delta_out;
    p.v = v_out;
    p.y = nullptr;
    cudaError_t e = launch_phaseA(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "phase A");
    return PDSSM_OK;
}

pdssm_status pdssm_validate(const pdssm_dims *dims, const int32_t *pi_dict,
                            int64_t pi_head_stride, const int32_t *k, void *ws, size_t ws_bytes,
                            void *stream) {
    pdssm_status st = check_scan_dims(dims, pi_head_stride, 1);
    if (st != PDSSM_OK) return st;
    if (!pi_dict || !ws || ws_bytes < 256)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL dictionary or workspace < 256 bytes");
    if (dims->L > 0 && !k) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL k");
    cudaStream_t s = (cudaStream_t)stream;
    int *counts = reinterpret_cast<int *>(reinterpret_cast<unsigned char *>(ws) + 64);
    cudaError_t e = cudaMemsetAsync(counts, 0, 8, s);
    if (e != cudaSuccess) return cuda_fail(e, "validate reset");
    e = launch_validate(*dims, pi_dict, pi_head_stride, dims->L > 0 ? k : nullptr, counts, s);
    if (e != cudaSuccess) return cuda_fail(e, "validate");
    int host[2] = {0, 0};
    e = cudaMemcpyAsync(host, counts, 8, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "validate copy");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "validate sync");
    if (host[0] || host[1]) {
        snprintf(g_last_error, sizeof(g_last_error),
                 "%d dictionary entries outside [0, N), %d selections outside [0, K)", host[0],
                 host[1]);
        return PDSSM_ERR_BAD_INDEX;
    }
    return PDSSM_OK;
}

pdssm_status pdssm_ws_status(void *ws, size_t ws_bytes, void *stream) {
    if (!ws || ws_bytes < 256) return arg_fail(PDSSM_ERR_INVALID_ARG, "bad workspace");
    cudaStream_t s = (cudaStream_t)stream;
    int host = 0;
    cudaError_t e = cudaMemcpyAsync(&host, ws, 4, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "status copy");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "status sync");
    e = cudaMemsetAsync(ws, 0, 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    if (host & kStTimeout) return arg_fail(PDSSM_ERR_TIMEOUT, "a staging wait gave up");
    if (host & kStBadIndex) return arg_fail(PDSSM_ERR_BAD_INDEX, "an index was clamped");
    return PDSSM_OK;
}

}  // extern "C"
