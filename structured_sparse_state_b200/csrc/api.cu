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
}  // namespace

namespace pdssm {

pdssm_status cuda_fail(cudaError_t e, const char *where) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
    return PDSSM_ERR_CUDA;
}

pdssm_status arg_fail(pdssm_status st, const char *why) {
    snprintf(g_last_error, sizeof(g_last_error), "%s", why);
    return st;
}

}  // namespace pdssm

namespace {

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

size_t dtype_size(pdssm_dtype t) { return t == PDSSM_BF16 ? 2 : 4; }

}  // namespace

// Shape checks shared by the scan calls.
pdssm_status pdssm::check_scan_dims(const pdssm_dims *dm, int64_t pi_hs, int64_t chunk) {
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

namespace {

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
    p.segw = reinterpret_cast<const uint2 *>(base + w.segw);
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
    p.ticket = reinterpret_cast<unsigned long long *>(base + w.look);
    p.look = reinterpret_cast<int *>(base + w.look + kLookHeader);
    p.wait_ns = kWaitCapNs;
    const int es = (int)dtype_size(dt);
    const int rowb = (int)dm->N * es;
    const bool vec_ok = (rowb % 16) == 0;
    const bool ptr_ok = (!d || aligned(d, 16)) && (!b || aligned(b, 16)) && (!c || aligned(c, 16));
    p.bulk = (vec_ok && ptr_ok) ? 1 : 0;
    // double-buffered tiles (the general kernels add an L2 prefetch further ahead)
    p.ns = kFastStages;
    return p;
}

}  // namespace

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

static pdssm_status select_common(const pdssm_dims *dims, const void *u, pdssm_dtype u_dtype,
                                  const float *W_sel, int32_t *k_out, int method,
                                  float *logits_out, float *scale_out, void *stream) {
    if (!dims) return arg_fail(PDSSM_ERR_INVALID_ARG, "dims is NULL");
    if (check_dtype(u_dtype) != PDSSM_OK) return PDSSM_ERR_INVALID_ARG;
    if (dims->B < 1 || dims->H < 1 || dims->L < 0 || dims->K < 1 || dims->D_in < 1)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "need B, H, K, D_in >= 1 and L >= 0");
    if (dims->K > 32) return arg_fail(PDSSM_ERR_UNSUPPORTED, "K > 32");
    if (dims->D_in > 256) return arg_fail(PDSSM_ERR_UNSUPPORTED, "D_in > 256");
    if (dims->L == 0) return PDSSM_OK;
    if (!u || !W_sel || !k_out) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(W_sel, 16)) return arg_fail(PDSSM_ERR_INVALID_ARG, "W_sel not 16-byte aligned");
    if (method != PDSSM_SELECT_AUTO && method != PDSSM_SELECT_FMA_CHAIN &&
        method != PDSSM_SELECT_TENSOR_CORE)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "unknown selection method");
    const bool tc_ok = select_tc_supported(*dims, u_dtype, u, W_sel);
    if (method == PDSSM_SELECT_TENSOR_CORE && !tc_ok)
        return arg_fail(PDSSM_ERR_UNSUPPORTED,
                        "tensor-core selection needs bf16 u, D_in a multiple of 16, K a power "
                        "of two and H*K <= 256");
    const bool use_tc = method == PDSSM_SELECT_TENSOR_CORE || (method == PDSSM_SELECT_AUTO && tc_ok);
    cudaError_t e = launch_select(*dims, u, u_dtype, W_sel, k_out, use_tc, logits_out, scale_out,
                                  (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "select");
    return PDSSM_OK;
}

pdssm_status pdssm_select(const pdssm_dims *dims, const void *u, pdssm_dtype u_dtype,
                          const float *W_sel, int32_t *k_out, void *stream) {
    return select_common(dims, u, u_dtype, W_sel, k_out, PDSSM_SELECT_AUTO, nullptr, nullptr,
                         stream);
}

pdssm_status pdssm_select_with(const pdssm_dims *dims, const void *u, pdssm_dtype u_dtype,
                               const float *W_sel, int32_t *k_out, int method, void *stream) {
    return select_common(dims, u, u_dtype, W_sel, k_out, method, nullptr, nullptr, stream);
}

pdssm_status pdssm_select_tc_logits(const pdssm_dims *dims, const void *u, const float *W_sel,
                                    int32_t *k_out, float *logits_out, float *scale_out,
                                    void *stream) {
    if (!logits_out || !scale_out)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL logits or scale output");
    return select_common(dims, u, PDSSM_BF16, W_sel, k_out, PDSSM_SELECT_TENSOR_CORE, logits_out,
                         scale_out, stream);
}

static pdssm_status fwd_common(const pdssm_dims *dims, const int32_t *pi_dict,
                               int64_t pi_head_stride, const int32_t *k, const void *d,
                               const void *b, pdssm_dtype in_dtype, int64_t chunk, void *ws,
                               size_t ws_bytes, bool for_bwd, WsLayout *wout,
                               bool k_given = true) {
    pdssm_status st = check_scan_dims(dims, pi_head_stride, chunk);
    if (st != PDSSM_OK) return st;
    if (check_dtype(in_dtype) != PDSSM_OK) return PDSSM_ERR_INVALID_ARG;
    if (!pi_dict || !ws) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL dictionary or workspace");
    if (dims->L > 0 && ((k_given && !k) || !d || !b))
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(ws, 256)) return arg_fail(PDSSM_ERR_INVALID_ARG, "ws not 256-byte aligned");
    const WsLayout w = ws_layout(*dims, pi_head_stride, chunk, for_bwd);
    if (ws_bytes < w.total) return arg_fail(PDSSM_ERR_WORKSPACE, "workspace too small");
    *wout = w;
    return PDSSM_OK;
}

// look: also clear the single-pass forward's ticket counter and per-chunk
// flags (only that kernel reads them).
static pdssm_status run_prep(const pdssm_dims *dims, const int32_t *pi_dict,
                             int64_t pi_head_stride, const WsLayout &w, void *ws,
                             cudaStream_t st, bool look) {
    unsigned char *base = reinterpret_cast<unsigned char *>(ws);
    // status word and the dictionary statistics (largest segment lane
    // distance, largest fan-in, largest window back-span)
    cudaError_t e = cudaMemsetAsync(base + w.status, 0, 16, st);
    if (e != cudaSuccess) return cuda_fail(e, "status reset");
    // the single-pass forward's ticket counter and per-chunk flags
    if (look) {
        e = cudaMemsetAsync(base + w.look, 0, kLookHeader + (size_t)(dims->B * dims->H * w.C) * 4,
                            st);
        if (e != cudaSuccess) return cuda_fail(e, "look-back reset");
    }
    e = launch_prep(*dims, pi_dict, pi_head_stride, reinterpret_cast<int32_t *>(base + w.dict),
                    reinterpret_cast<uint2 *>(base + w.seg),
                    reinterpret_cast<uint2 *>(base + w.segw),
                    reinterpret_cast<int *>(base + w.status) + 1,
                    reinterpret_cast<uint8_t *>(base + w.tab),
                    reinterpret_cast<int32_t *>(base + w.fan), w.Hd,
                    reinterpret_cast<int *>(base + w.status), st);
    if (e != cudaSuccess) return cuda_fail(e, "prep");
    return PDSSM_OK;
}

}  // extern "C"

namespace {

// Records the caller's events between the kernels of a traced call: mark()
// before each kernel (with its name), finish() after the last one.
struct Tracer {
    pdssm_trace *t;
    cudaStream_t s;
    cudaError_t mark(const char *name) {
        if (!t) return cudaSuccess;
        if (t->n_kernels + 1 >= t->max_events || t->n_kernels >= PDSSM_TRACE_MAX_KERNELS)
            return cudaSuccess;
        t->names[t->n_kernels] = name;
        return cudaEventRecord((cudaEvent_t)t->events[t->n_kernels++], s);
    }
    cudaError_t finish() {
        if (!t || t->n_kernels == 0) return cudaSuccess;
        return cudaEventRecord((cudaEvent_t)t->events[t->n_kernels], s);
    }
};

pdssm_status scan_fwd_impl(const pdssm_dims *dims, const int32_t *pi_dict, int64_t pi_head_stride,
                           const int32_t *k, const void *d, const void *b, const void *c,
                           pdssm_dtype in_dtype, const float *h0, float *y, float *h_last,
                           int64_t chunk, void *ws, size_t ws_bytes, void *stream,
                           pdssm_trace *trace, bool single_pass = false) {
    WsLayout w;
    pdssm_status st = fwd_common(dims, pi_dict, pi_head_stride, k, d, b, in_dtype, chunk, ws,
                                 ws_bytes, false, &w);
    if (st != PDSSM_OK) return st;
    if (dims->L > 0 && (!c || !y)) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL c or y");
    if (trace) {
        if (!trace->events || trace->max_events < 2)
            return arg_fail(PDSSM_ERR_INVALID_ARG, "trace needs at least two events");
        trace->n_kernels = 0;
    }
    cudaStream_t s = (cudaStream_t)stream;
    Tracer tr{trace, s};
    cudaError_t e = tr.mark("prep");
    if (e != cudaSuccess) return cuda_fail(e, "trace event");
    st = run_prep(dims, pi_dict, pi_head_stride, w, ws, s, single_pass);
    if (st != PDSSM_OK) return st;
    if (dims->L == 0) {
        if (h_last) {
            const size_t bytes = (size_t)(dims->B * dims->H * dims->N) * 4;
            e = h0 ? cudaMemcpyAsync(h_last, h0, bytes, cudaMemcpyDeviceToDevice, s)
                   : cudaMemsetAsync(h_last, 0, bytes, s);
            if (e != cudaSuccess) return cuda_fail(e, "h_last for L = 0");
        }
        e = tr.finish();
        return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "trace event");
    }
    ChunkParams p = make_params(dims, w, ws, chunk, k, d, b, c, in_dtype);
    p.h0 = h0;
    p.y = y;
    p.h_last = h_last;
    if (single_pass) {
        if (!fused_path(p))
            return arg_fail(PDSSM_ERR_UNSUPPORTED,
                            "the single-pass forward needs N = 32 or 64 with 16-byte aligned rows");
        if ((e = tr.mark("single pass")) != cudaSuccess) return cuda_fail(e, "trace event");
        e = launch_scan_fused(p, in_dtype, s, false);
        if (e != cudaSuccess) return cuda_fail(e, "single-pass forward");
        e = tr.finish();
        return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "trace event");
    }
    if ((e = tr.mark("phase A")) != cudaSuccess) return cuda_fail(e, "trace event");
    e = launch_phaseA(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "phase A");
    if ((e = tr.mark("phase B")) != cudaSuccess) return cuda_fail(e, "trace event");
    e = launch_phaseB(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "phase B");
    if ((e = tr.mark("phase C")) != cudaSuccess) return cuda_fail(e, "trace event");
    e = launch_phaseC(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "phase C");
    e = tr.finish();
    return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "trace event");
}

pdssm_status scan_bwd_impl(const pdssm_dims *dims, const int32_t *pi_dict, int64_t pi_head_stride,
                           const int32_t *k, const void *d, const void *b, const void *c,
                           pdssm_dtype in_dtype, const float *h0, const float *g_y,
                           const float *g_hlast, float *g_b, float *g_d, float *g_c, float *g_h0,
                           int64_t chunk, void *ws, size_t ws_bytes, void *stream,
                           pdssm_trace *trace) {
    WsLayout w;
    pdssm_status st = fwd_common(dims, pi_dict, pi_head_stride, k, d, b, in_dtype, chunk, ws,
                                 ws_bytes, true, &w);
    if (st != PDSSM_OK) return st;
    if (chunk > kBwdMaxChunk && dims->L > kBwdMaxChunk)
        return arg_fail(PDSSM_ERR_UNSUPPORTED, "backward needs chunk <= 256");
    if (dims->L > 0 && (!c || !g_y || !g_b || !g_d || !g_c))
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL tensor pointer");
    if (trace) {
        if (!trace->events || trace->max_events < 2)
            return arg_fail(PDSSM_ERR_INVALID_ARG, "trace needs at least two events");
        trace->n_kernels = 0;
    }
    cudaStream_t s = (cudaStream_t)stream;
    Tracer tr{trace, s};
    cudaError_t e;
    if (dims->L == 0) {
        if (g_h0) {
            const size_t bytes = (size_t)(dims->B * dims->H * dims->N) * 4;
            e = g_hlast ? cudaMemcpyAsync(g_h0, g_hlast, bytes, cudaMemcpyDeviceToDevice, s)
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
    if ((e = tr.mark("bwd phase A")) != cudaSuccess) return cuda_fail(e, "trace event");
    e = launch_bwdA(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "bwd phase A");
    if ((e = tr.mark("bwd phase B")) != cudaSuccess) return cuda_fail(e, "trace event");
    e = launch_bwdB(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "bwd phase B");
    if ((e = tr.mark("bwd phase C")) != cudaSuccess) return cuda_fail(e, "trace event");
    e = launch_bwdC(p, in_dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "bwd phase C");
    e = tr.finish();
    return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "trace event");
}

}  // namespace

extern "C" {

pdssm_status pdssm_scan_fwd(const pdssm_dims *dims, const int32_t *pi_dict,
                            int64_t pi_head_stride, const int32_t *k, const void *d,
                            const void *b, const void *c, pdssm_dtype in_dtype, const float *h0,
                            float *y, float *h_last, int64_t chunk, void *ws, size_t ws_bytes,
                            void *stream) {
    return scan_fwd_impl(dims, pi_dict, pi_head_stride, k, d, b, c, in_dtype, h0, y, h_last,
                         chunk, ws, ws_bytes, stream, nullptr);
}

pdssm_status pdssm_scan_fwd_single_pass(const pdssm_dims *dims, const int32_t *pi_dict,
                                        int64_t pi_head_stride, const int32_t *k, const void *d,
                                        const void *b, const void *c, pdssm_dtype in_dtype,
                                        const float *h0, float *y, float *h_last, int64_t chunk,
                                        void *ws, size_t ws_bytes, void *stream) {
    return scan_fwd_impl(dims, pi_dict, pi_head_stride, k, d, b, c, in_dtype, h0, y, h_last,
                         chunk, ws, ws_bytes, stream, nullptr, true);
}

pdssm_status pdssm_scan_fwd_traced(const pdssm_dims *dims, const int32_t *pi_dict,
                                   int64_t pi_head_stride, const int32_t *k, const void *d,
                                   const void *b, const void *c, pdssm_dtype in_dtype,
                                   const float *h0, float *y, float *h_last, int64_t chunk,
                                   void *ws, size_t ws_bytes, void *stream, pdssm_trace *trace) {
    if (!trace) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL trace");
    return scan_fwd_impl(dims, pi_dict, pi_head_stride, k, d, b, c, in_dtype, h0, y, h_last,
                         chunk, ws, ws_bytes, stream, trace);
}

pdssm_status pdssm_select_scan_fwd(const pdssm_dims *dims, const void *u, pdssm_dtype u_dtype,
                                   const float *W_sel, const int32_t *pi_dict,
                                   int64_t pi_head_stride, const void *d, const void *b,
                                   const void *c, pdssm_dtype in_dtype, const float *h0, float *y,
                                   float *h_last, int32_t *k_out, int64_t chunk, void *ws,
                                   size_t ws_bytes, void *stream) {
    if (!dims) return arg_fail(PDSSM_ERR_INVALID_ARG, "dims is NULL");
    if (dims->L < 1) return arg_fail(PDSSM_ERR_INVALID_ARG, "need L >= 1");
    if (!u || !W_sel) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL u or W_sel");
    WsLayout w;
    pdssm_status st = fwd_common(dims, pi_dict, pi_head_stride, nullptr, d, b, in_dtype, chunk,
                                 ws, ws_bytes, false, &w, false);
    if (st != PDSSM_OK) return st;
    if (!c || !y) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL c or y");
    ChunkParams p = make_params(dims, w, ws, chunk, nullptr, d, b, c, in_dtype);
    p.u = u;
    p.W_sel = W_sel;
    p.D_in = (int)dims->D_in;
    p.k_out = k_out;
    if (u_dtype != PDSSM_BF16 || !fused_select_ok(p, u, W_sel))
        return arg_fail(PDSSM_ERR_UNSUPPORTED,
                        "the selection runs inside the forward for bf16 u, D_in a multiple of 16 "
                        "(<= 256), K <= 16, N = 32 or 64 with 16-byte aligned rows and chunk <= "
                        "1024; use pdssm_select and pdssm_scan_fwd otherwise");
    cudaStream_t s = (cudaStream_t)stream;
    st = run_prep(dims, pi_dict, pi_head_stride, w, ws, s, true);
    if (st != PDSSM_OK) return st;
    p.h0 = h0;
    p.y = y;
    p.h_last = h_last;
    cudaError_t e = launch_scan_fused(p, in_dtype, s, true);
    return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "selection + single-pass forward");
}

pdssm_status pdssm_scan_bwd(const pdssm_dims *dims, const int32_t *pi_dict,
                            int64_t pi_head_stride, const int32_t *k, const void *d,
                            const void *b, const void *c, pdssm_dtype in_dtype, const float *h0,
                            const float *g_y, const float *g_hlast, float *g_b, float *g_d,
                            float *g_c, float *g_h0, int64_t chunk, void *ws, size_t ws_bytes,
                            void *stream) {
    return scan_bwd_impl(dims, pi_dict, pi_head_stride, k, d, b, c, in_dtype, h0, g_y, g_hlast,
                         g_b, g_d, g_c, g_h0, chunk, ws, ws_bytes, stream, nullptr);
}

pdssm_status pdssm_scan_bwd_traced(const pdssm_dims *dims, const int32_t *pi_dict,
                                   int64_t pi_head_stride, const int32_t *k, const void *d,
                                   const void *b, const void *c, pdssm_dtype in_dtype,
                                   const float *h0, const float *g_y, const float *g_hlast,
                                   float *g_b, float *g_d, float *g_c, float *g_h0,
                                   int64_t chunk, void *ws, size_t ws_bytes, void *stream,
                                   pdssm_trace *trace) {
    if (!trace) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL trace");
    return scan_bwd_impl(dims, pi_dict, pi_head_stride, k, d, b, c, in_dtype, h0, g_y, g_hlast,
                         g_b, g_d, g_c, g_h0, chunk, ws, ws_bytes, stream, trace);
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
    st = run_prep(dims, pi_dict, pi_head_stride, w, ws, s, false);
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

pdssm_status pdssm_ws_transfers(const pdssm_dims *dims, int64_t pi_head_stride, int64_t chunk,
                                const void *ws, size_t ws_bytes, int32_t *Pi_out,
                                float *Delta_out, float *v_out, float *H_out, void *stream) {
    pdssm_status st = check_scan_dims(dims, pi_head_stride, chunk);
    if (st != PDSSM_OK) return st;
    if (!ws || !Pi_out || !Delta_out || !v_out || !H_out)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL pointer");
    const WsLayout w = ws_layout(*dims, pi_head_stride, chunk, false);
    if (ws_bytes < w.total) return arg_fail(PDSSM_ERR_WORKSPACE, "workspace too small");
    const size_t bytes = (size_t)(dims->B * dims->H * w.C * dims->N) * 4;
    if (bytes == 0) return PDSSM_OK;
    const unsigned char *base = reinterpret_cast<const unsigned char *>(ws);
    cudaStream_t s = (cudaStream_t)stream;
    void *dst[4] = {Pi_out, Delta_out, v_out, H_out};
    const size_t src[4] = {w.Pi, w.Dl, w.v, w.Hc};
    for (int i = 0; i < 4; ++i) {
        cudaError_t e = cudaMemcpyAsync(dst[i], base + src[i], bytes, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_fail(e, "transfer copy");
    }
    return PDSSM_OK;
}

pdssm_status pdssm_dict_hardmax(int64_t n_mats, int64_t N, const float *A, int32_t *pi_out,
                                void *stream) {
    if (n_mats < 0 || N < 1 || N > kMaxN)
        return arg_fail(N > kMaxN ? PDSSM_ERR_UNSUPPORTED : PDSSM_ERR_INVALID_ARG,
                        "need n_mats >= 0 and 1 <= N <= 64");
    if (n_mats == 0) return PDSSM_OK;
    if (!A || !pi_out) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL pointer");
    cudaError_t e = launch_dict_hardmax(n_mats, (int)N, A, pi_out, (cudaStream_t)stream);
    return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "dictionary hardmax");
}

pdssm_status pdssm_soft_maps(const pdssm_dims *dims, const void *u, pdssm_dtype u_dtype,
                             const float *W_sel, const float *A, int64_t a_head_stride,
                             float inv_tau, int32_t *maps_out, void *stream) {
    if (!dims) return arg_fail(PDSSM_ERR_INVALID_ARG, "dims is NULL");
    if (check_dtype(u_dtype) != PDSSM_OK) return PDSSM_ERR_INVALID_ARG;
    if (dims->B < 1 || dims->H < 1 || dims->L < 0 || dims->N < 1 || dims->K < 1 ||
        dims->D_in < 1)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "need B, H, N, K, D_in >= 1 and L >= 0");
    if (dims->N > kMaxN || dims->K > 32 || dims->D_in > 256)
        return arg_fail(PDSSM_ERR_UNSUPPORTED, "N > 64, K > 32 or D_in > 256");
    if (a_head_stride != 0 && a_head_stride < dims->K * dims->N * dims->N)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "a_head_stride must be 0 or >= K*N*N");
    if (!(inv_tau > 0.f) || inv_tau > 3.0e38f)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "inv_tau must be positive and finite");
    if (dims->L == 0) return PDSSM_OK;
    if (!u || !W_sel || !A || !maps_out) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL pointer");
    cudaError_t e = launch_soft_maps(*dims, u, u_dtype, W_sel, A, a_head_stride, inv_tau,
                                     maps_out, (cudaStream_t)stream);
    return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "soft maps");
}

pdssm_status pdssm_scan_fwd_maps(const pdssm_dims *dims, const int32_t *maps, const void *d,
                                 const void *b, const void *c, pdssm_dtype in_dtype,
                                 const float *h0, float *y, float *h_last, void *stream) {
    pdssm_status st = check_scan_dims(dims, 0, 1);
    if (st != PDSSM_OK) return st;
    if (check_dtype(in_dtype) != PDSSM_OK) return PDSSM_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (dims->L == 0) {
        if (h_last) {
            const size_t bytes = (size_t)(dims->B * dims->H * dims->N) * 4;
            cudaError_t e = h0 ? cudaMemcpyAsync(h_last, h0, bytes, cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(h_last, 0, bytes, s);
            if (e != cudaSuccess) return cuda_fail(e, "h_last for L = 0");
        }
        return PDSSM_OK;
    }
    if (!maps || !d || !b || !c || !y) return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL pointer");
    cudaError_t e = launch_scan_maps(*dims, maps, d, b, c, in_dtype, h0, y, h_last, s);
    return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "scan with per-step maps");
}

static pdssm_status check_surrogate_dims(const pdssm_dims *dims, int64_t a_hs) {
    if (!dims) return arg_fail(PDSSM_ERR_INVALID_ARG, "dims is NULL");
    if (dims->B < 1 || dims->H < 1 || dims->L < 0 || dims->N < 1 || dims->K < 1 ||
        dims->D_in < 1)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "need B, H, N, K, D_in >= 1 and L >= 0");
    if (dims->N > kMaxN || dims->K > 32 || dims->D_in > 256)
        return arg_fail(PDSSM_ERR_UNSUPPORTED, "N > 64, K > 32 or D_in > 256");
    if (a_hs != 0 && a_hs < dims->K * dims->N * dims->N)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "a_head_stride must be 0 or >= K*N*N");
    return PDSSM_OK;
}

size_t pdssm_surrogate_scratch_bytes(const pdssm_dims *dims, int64_t a_head_stride) {
    if (check_surrogate_dims(dims, a_head_stride) != PDSSM_OK) return 0;
    return surrogate_scratch_bytes(*dims, a_head_stride);
}

pdssm_status pdssm_surrogate_bwd(const pdssm_dims *dims, const void *u, pdssm_dtype u_dtype,
                                 const float *W_sel, const float *A, int64_t a_head_stride,
                                 const int32_t *pi_dict, const int32_t *k, const void *d,
                                 const void *b, pdssm_dtype in_dtype, const float *h0,
                                 const float *lambda, int64_t chunk, const void *ws,
                                 size_t ws_bytes, float inv_tau_s, float inv_tau_a,
                                 void *scratch, size_t scratch_bytes, float *g_logits,
                                 float *g_W, float *g_A, void *stream) {
    pdssm_status st = check_surrogate_dims(dims, a_head_stride);
    if (st != PDSSM_OK) return st;
    if (check_dtype(u_dtype) != PDSSM_OK || check_dtype(in_dtype) != PDSSM_OK)
        return PDSSM_ERR_INVALID_ARG;
    if (chunk < 1) return arg_fail(PDSSM_ERR_INVALID_ARG, "chunk must be >= 1");
    if (!(inv_tau_s > 0.f) || !(inv_tau_a > 0.f) || inv_tau_s > 3.0e38f || inv_tau_a > 3.0e38f)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "inverse temperatures must be positive and finite");
    if (!W_sel || !A || !pi_dict || !g_W || !g_A || !ws || !scratch)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL pointer");
    if (dims->L > 0 && (!u || !k || !d || !b || !lambda || !g_logits))
        return arg_fail(PDSSM_ERR_INVALID_ARG, "NULL tensor pointer");
    const int64_t pi_hs = a_head_stride ? dims->K * dims->N : 0;
    const WsLayout w = ws_layout(*dims, pi_hs, chunk, false);
    if (ws_bytes < w.total) return arg_fail(PDSSM_ERR_WORKSPACE, "forward workspace too small");
    if (scratch_bytes < surrogate_scratch_bytes(*dims, a_head_stride))
        return arg_fail(PDSSM_ERR_WORKSPACE, "surrogate scratch too small");
    if (!aligned(scratch, 256)) return arg_fail(PDSSM_ERR_INVALID_ARG, "scratch not 256-byte aligned");
    const float *Hc = reinterpret_cast<const float *>(reinterpret_cast<const unsigned char *>(ws) + w.Hc);
    cudaError_t e = launch_surrogate(*dims, u, u_dtype, W_sel, A, a_head_stride, pi_dict, k, d, b,
                                     in_dtype, h0, Hc, chunk, lambda, inv_tau_s, inv_tau_a,
                                     scratch, g_logits, g_W, g_A, (cudaStream_t)stream);
    return e == cudaSuccess ? PDSSM_OK : cuda_fail(e, "surrogate backward");
}

pdssm_status pdssm_wait_selftest(int which, int64_t cap_ns, void *ws, size_t ws_bytes,
                                 void *stream) {
    if (which != 0 && which != 1) return arg_fail(PDSSM_ERR_INVALID_ARG, "which must be 0 or 1");
    if (cap_ns < 1 || cap_ns > (int64_t)kWaitCapNs)
        return arg_fail(PDSSM_ERR_INVALID_ARG, "cap_ns must lie in [1, 2e9]");
    // a one-sequence, two-chunk layout whose flags are all zero
    const pdssm_dims dm = {1, 1, 2, 32, 1, 0};
    const WsLayout w = ws_layout(dm, 0, 1, false);
    if (!ws || ws_bytes < w.total || !aligned(ws, 256))
        return arg_fail(PDSSM_ERR_WORKSPACE, "workspace too small or not 256-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    unsigned char *base = reinterpret_cast<unsigned char *>(ws);
    cudaError_t e = cudaMemsetAsync(base, 0, w.total, s);
    if (e != cudaSuccess) return cuda_fail(e, "self-test reset");
    ChunkParams p = make_params(&dm, w, ws, 1, nullptr, nullptr, nullptr, nullptr, PDSSM_F32);
    p.wait_ns = (uint64_t)cap_ns;
    e = launch_wait_selftest(p, which, s);
    if (e != cudaSuccess) return cuda_fail(e, "wait self-test");
    return PDSSM_OK;
}

size_t pdssm_wait_selftest_ws_bytes(void) {
    const pdssm_dims dm = {1, 1, 2, 32, 1, 0};
    return ws_layout(dm, 0, 1, false).total;
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
