// api.cu -- the C ABI of libsparse_attn.so: argument checks, workspace
// sizing, dispatch to the kernels, status word.  See include/sparse_attn.h.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "lsa.cuh"

using namespace sa;

static std::atomic<unsigned long long> g_launches{0};
void sa::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

sa::WsLayout sa::ws_layout(const Shape &s) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t units = (size_t)s.B * s.Hsel;
    const size_t ktiles = (size_t)s.B * s.Hkv * ((s.nb * s.bs + 127) / 128);
    WsLayout L;
    size_t o = kStatusBytes;
    L.sel_chunk = o;  o += al(units * s.nb * 4);
    L.sel_decode = o; o += al(units * 4);
    L.sel_ready = o;  o += al(units * 4);
    L.dec = o;        o += al(units * 8);
    L.bwd_kv = o;     o += al(ktiles * 8 * 4);
    L.scratch = o;
    return L;
}

int sa::sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Numbers that tell one decode step's published lists from every earlier
// step's (never 0, the value of a fresh workspace).
std::atomic<unsigned> g_epoch{0};
unsigned next_epoch() {
    unsigned e;
    do e = g_epoch.fetch_add(1u, std::memory_order_relaxed) + 1u;
    while (e == 0u);
    return e;
}

// Resolves and checks a parameter block.  Returns SA_OK or an error code.
int resolve(const sa_params *p, Shape &s) {
    if (!p) return SA_ERR_ARG;
    if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->N <= 0 || p->block <= 0) return SA_ERR_ARG;
    if (p->Hq % p->Hkv) return SA_ERR_ARG;
    if (p->dtype != SA_BF16 && p->dtype != SA_FP32) return SA_ERR_ARG;
    if (p->top_k < 0 || p->top_k > 256) return SA_ERR_ARG;
    if (p->flags & ~(SA_SINK | SA_LOCAL | SA_GATE | SA_HIER | SA_CAUSAL | SA_SELECT_PER_QHEAD)) return SA_ERR_ARG;
    if (!(p->scale >= 0.f) || isinf(p->scale)) return SA_ERR_ARG;
    if (p->d != 64 && p->d != 128) return SA_ERR_UNSUPPORTED;
    if (p->block < 16 || p->block > 128 || p->block % 16) return SA_ERR_UNSUPPORTED;
    if ((p->flags & SA_GATE) && (p->flags & SA_HIER)) return SA_ERR_UNSUPPORTED;
    if ((p->flags & SA_GATE) && !(p->flags & SA_LOCAL)) return SA_ERR_UNSUPPORTED;
    s.B = p->B;
    s.Hq = p->Hq;
    s.Hkv = p->Hkv;
    s.G = p->Hq / p->Hkv;
    s.d = p->d;
    s.N = p->N;
    s.bs = p->block;
    s.nb = (p->N + p->block - 1) / p->block;
    s.top_k = p->top_k;
    s.cap = p->top_k + 2;
    s.flags = p->flags;
    s.dtype = p->dtype;
    const bool perq = p->flags & SA_SELECT_PER_QHEAD;
    s.Hsel = perq ? p->Hq : p->Hkv;
    s.heads_per = perq ? 1 : s.G;
    s.scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
    s.seq_len = nullptr;
    s.first_block = nullptr;
    if ((long long)s.B * s.Hq * s.nb > (1ll << 31) - 1) return SA_ERR_UNSUPPORTED;
    if (s.heads_per * s.d > 2048) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

// Resolves and checks a flat-index parameter block.
int resolve_lsa(const sa_lsa_params *p, LsaShape &s) {
    if (!p) return SA_ERR_ARG;
    if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->N <= 0 || p->pool <= 0) return SA_ERR_ARG;
    if (p->Hq % p->Hkv) return SA_ERR_ARG;
    if (p->dtype != SA_BF16 && p->dtype != SA_FP32) return SA_ERR_ARG;
    if (p->seg < 2 || p->clusters < 1 || p->clusters > p->seg) return SA_ERR_ARG;
    if (p->top_clusters < 0 || p->sink < 0 || p->window < 0) return SA_ERR_ARG;
    if (!(p->scale >= 0.f) || isinf(p->scale)) return SA_ERR_ARG;
    if (p->d != 64 && p->d != 128) return SA_ERR_UNSUPPORTED;
    if (p->seg > 64 || p->N > (1 << 20) || p->top_clusters > 4096) return SA_ERR_UNSUPPORTED;
    if ((long long)p->pool * p->seg > (1ll << 30)) return SA_ERR_UNSUPPORTED;
    s.B = p->B;
    s.Hq = p->Hq;
    s.Hkv = p->Hkv;
    s.G = p->Hq / p->Hkv;
    s.d = p->d;
    s.N = p->N;
    s.pool = p->pool;
    s.seg = p->seg;
    s.clusters = p->clusters;
    s.top_clusters = p->top_clusters;
    s.sink = p->sink;
    s.window = p->window;
    s.dtype = p->dtype;
    s.scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
    s.nseg = p->N / (p->pool * p->seg);
    s.ctotal = s.nseg * p->clusters;
    if ((long long)s.B * s.Hkv * s.nseg > (1ll << 31) - 1) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

thread_local int t_last_cuda_error = 0;

int launch_result(cudaError_t e) {
    if (e == cudaSuccess) return SA_OK;
    t_last_cuda_error = (int)e;
    return SA_ERR_LAUNCH;
}

}  // namespace

// Decode on a fixed scratch buffer (the no-allocation entry point): the
// status word, the per-unit completion counters and this call's split
// partials, packed from the buffer's start.  The status word and the
// counters are cleared on the stream first; the partials need no clearing
// (every split writes its own slot before the merge reads it).
int sa::decode_on_scratch(const sa_params *p, const void *q, const void *K, const void *V, const int32_t *idx,
                          const float *score, const int32_t *count, void *o, float *lse, void *scratch,
                          size_t scratch_bytes, size_t *need, cudaStream_t st) {
    Shape s;
    const int r = resolve(p, s);
    if (r != SA_OK) return r;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t cnt_bytes = al((size_t)s.B * s.Hsel * 8);
    const size_t total = kStatusBytes + cnt_bytes + al(decode_workspace(s));
    if (need) *need = total;
    if (total > scratch_bytes) return SA_ERR_WORKSPACE;
    if (!q || !K || !V || !idx || !score || !count || !o || !lse || !scratch) return SA_ERR_ARG;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(o) || !aligned16(scratch)) return SA_ERR_ARG;
    unsigned char *w = static_cast<unsigned char *>(scratch);
    if (cudaMemsetAsync(w, 0, kStatusBytes + cnt_bytes, st) != cudaSuccess) return SA_ERR_LAUNCH;
    return launch_result(launch_decode(s, q, K, V, idx, score, count, o, lse, reinterpret_cast<unsigned *>(w),
                                       reinterpret_cast<unsigned *>(w + kStatusBytes),
                                       reinterpret_cast<float *>(w + kStatusBytes + cnt_bytes), st));
}

extern "C" {

size_t sparse_attn_workspace_size(const sa_params *p, int op) {
    Shape s;
    if (resolve(p, s) != SA_OK) return 0;
    size_t extra = 0;
    switch (op) {
        case SA_OP_SELECT: extra = select_workspace(s, false); break;
        case SA_OP_SELECT_DECODE: extra = select_workspace(s, true); break;
        case SA_OP_DECODE: extra = decode_workspace(s); break;
        case SA_OP_PREFILL_BACKWARD: extra = prefill_backward_workspace(s); break;
        case SA_OP_SELECT_BACKWARD: extra = select_backward_workspace(s); break;
        default: break;
    }
    return ws_layout(s).scratch + ((extra + 255) & ~(size_t)255);
}

int sparse_attn_landmarks(const sa_params *p, const void *K, void *L, void *stream) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    if (!K || !L || !aligned16(K) || !aligned16(L)) return SA_ERR_ARG;
    return launch_result(launch_landmarks(s, K, L, (cudaStream_t)stream));
}

int sparse_attn_landmarks_update(const sa_params *p, const void *K, void *L, const int32_t *seq_len,
                                 const int32_t *first_block, void *stream) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    if (!K || !L || !aligned16(K) || !aligned16(L)) return SA_ERR_ARG;
    s.seq_len = seq_len;
    s.first_block = first_block;
    return launch_result(launch_landmarks(s, K, L, (cudaStream_t)stream));
}

static int select_common(const sa_params *p, bool decode, const void *Q, const void *L, int32_t *idx, float *score,
                         int32_t *count, void *ws, size_t ws_bytes, void *stream, const int32_t *seq_len = nullptr) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    s.seq_len = seq_len;
    if (!Q || !L || !idx || !score || !count || !ws) return SA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(L) || !aligned16(ws)) return SA_ERR_ARG;
    if (ws_bytes < sparse_attn_workspace_size(p, decode ? SA_OP_SELECT_DECODE : SA_OP_SELECT)) return SA_ERR_WORKSPACE;
    return launch_result(launch_select(s, decode, Q, L, idx, score, count, ws, ws_bytes, (cudaStream_t)stream));
}

int sparse_attn_select(const sa_params *p, const void *Q, const void *L, int32_t *idx, float *score,
                       int32_t *count, void *ws, size_t ws_bytes, void *stream) {
    return select_common(p, false, Q, L, idx, score, count, ws, ws_bytes, stream);
}

int sparse_attn_select_decode(const sa_params *p, const void *q, const void *L, int32_t *idx, float *score,
                              int32_t *count, void *ws, size_t ws_bytes, void *stream) {
    return select_common(p, true, q, L, idx, score, count, ws, ws_bytes, stream);
}

int sparse_attn_select_decode_varlen(const sa_params *p, const void *q, const void *L, const int32_t *seq_len,
                                     int32_t *idx, float *score, int32_t *count, void *ws, size_t ws_bytes,
                                     void *stream) {
    if (!seq_len) return SA_ERR_ARG;
    return select_common(p, true, q, L, idx, score, count, ws, ws_bytes, stream, seq_len);
}

int sparse_attn_prefill(const sa_params *p, const void *Q, const void *K, const void *V, const int32_t *idx,
                        const float *score, const int32_t *count, void *O, float *lse, void *ws,
                        size_t ws_bytes, void *stream) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    if (!Q || !K || !V || !idx || !score || !count || !O || !lse || !ws) return SA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(ws)) return SA_ERR_ARG;
    if (ws_bytes < sparse_attn_workspace_size(p, SA_OP_PREFILL)) return SA_ERR_WORKSPACE;
    if (prefill_tc2_supported(s))
        return launch_result(
            launch_prefill_tc2(s, Q, K, V, idx, score, count, O, lse, (unsigned *)ws, (cudaStream_t)stream));
    if (prefill_tc_supported(s))
        return launch_result(
            launch_prefill_tc(s, Q, K, V, idx, score, count, O, lse, (unsigned *)ws, (cudaStream_t)stream));
    return launch_result(
        launch_prefill_simt(s, Q, K, V, idx, score, count, O, lse, (unsigned *)ws, (cudaStream_t)stream));
}

int sparse_attn_prefill_kernel(const sa_params *p) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    return prefill_tc2_supported(s) ? 2 : prefill_tc_supported(s) ? 1 : 0;
}

static int decode_common(const sa_params *p, const void *q, const void *K, const void *V, const int32_t *seq_len,
                         const int32_t *idx, const float *score, const int32_t *count, void *o, float *lse,
                         void *ws, size_t ws_bytes, void *stream) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    s.seq_len = seq_len;
    if (!q || !K || !V || !idx || !score || !count || !o || !lse || !ws) return SA_ERR_ARG;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(o) || !aligned16(ws)) return SA_ERR_ARG;
    if (ws_bytes < sparse_attn_workspace_size(p, SA_OP_DECODE)) return SA_ERR_WORKSPACE;
    const WsLayout L = ws_layout(s);
    unsigned char *w = static_cast<unsigned char *>(ws);
    return launch_result(launch_decode(s, q, K, V, idx, score, count, o, lse, reinterpret_cast<unsigned *>(w),
                                       reinterpret_cast<unsigned *>(w + L.dec),
                                       reinterpret_cast<float *>(w + L.scratch), (cudaStream_t)stream));
}

int sparse_attn_decode(const sa_params *p, const void *q, const void *K, const void *V, const int32_t *idx,
                       const float *score, const int32_t *count, void *o, float *lse, void *ws, size_t ws_bytes,
                       void *stream) {
    return decode_common(p, q, K, V, nullptr, idx, score, count, o, lse, ws, ws_bytes, stream);
}

int sparse_attn_decode_step(const sa_params *p, const void *q, const void *L, const void *K, const void *V,
                            const int32_t *seq_len, int32_t *idx, float *score, int32_t *count, void *o,
                            float *lse, void *ws, size_t ws_bytes, void *stream) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    s.seq_len = seq_len;
    if (!q || !L || !K || !V || !idx || !score || !count || !o || !lse || !ws) return SA_ERR_ARG;
    if (!aligned16(q) || !aligned16(L) || !aligned16(K) || !aligned16(V) || !aligned16(o) || !aligned16(ws))
        return SA_ERR_ARG;
    if (ws_bytes < sparse_attn_workspace_size(p, SA_OP_SELECT_DECODE) ||
        ws_bytes < sparse_attn_workspace_size(p, SA_OP_DECODE))
        return SA_ERR_WORKSPACE;
    const WsLayout Lw = ws_layout(s);
    unsigned char *w = static_cast<unsigned char *>(ws);
    const cudaStream_t st = (cudaStream_t)stream;
    // overlap when the selection publishes lists and the decode can wait on them
    const bool overlap = select_decode_supported(s) && !select_force_chunked() && decode_mma_supported(s);
    unsigned *ready = overlap ? reinterpret_cast<unsigned *>(w + Lw.sel_ready) : nullptr;
    const unsigned epoch = overlap ? next_epoch() : 0u;
    const cudaError_t e = overlap ? launch_select_decode(s, q, L, idx, score, count, ws, st, ready, epoch)
                                  : launch_select(s, true, q, L, idx, score, count, ws, ws_bytes, st);
    if (e != cudaSuccess) return launch_result(e);
    return launch_result(launch_decode(s, q, K, V, idx, score, count, o, lse, reinterpret_cast<unsigned *>(w),
                                       reinterpret_cast<unsigned *>(w + Lw.dec),
                                       reinterpret_cast<float *>(w + Lw.scratch), st, ready, epoch));
}

int sparse_attn_decode_varlen(const sa_params *p, const void *q, const void *K, const void *V, const int32_t *seq_len,
                              const int32_t *idx, const float *score, const int32_t *count, void *o, float *lse,
                              void *ws, size_t ws_bytes, void *stream) {
    if (!seq_len) return SA_ERR_ARG;
    return decode_common(p, q, K, V, seq_len, idx, score, count, o, lse, ws, ws_bytes, stream);
}

int sparse_attn_prefill_backward(const sa_params *p, const void *Q, const void *K, const void *V, const void *O,
                                 const float *lse, const void *dO, const int32_t *idx, const float *score,
                                 const int32_t *count, float *dQ, float *dK, float *dV, float *dscore, void *ws,
                                 size_t ws_bytes, void *stream) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    if (!backward_supported(s)) return SA_ERR_UNSUPPORTED;
    if (!Q || !K || !V || !O || !lse || !dO || !idx || !score || !count || !dQ || !dK || !dV || !dscore || !ws)
        return SA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(dQ) ||
        !aligned16(dK) || !aligned16(dV) || !aligned16(ws))
        return SA_ERR_ARG;
    if (ws_bytes < sparse_attn_workspace_size(p, SA_OP_PREFILL_BACKWARD)) return SA_ERR_WORKSPACE;
    return launch_result(launch_prefill_backward(s, Q, K, V, O, lse, dO, idx, score, count, dQ, dK, dV, dscore, ws,
                                                 (cudaStream_t)stream));
}

int sparse_attn_select_backward(const sa_params *p, const void *Q, const void *L, const int32_t *idx,
                                const float *dscore, const int32_t *count, float *dQ, float *dK, void *ws,
                                size_t ws_bytes, void *stream) {
    Shape s;
    int r = resolve(p, s);
    if (r != SA_OK) return r;
    if (!backward_supported(s)) return SA_ERR_UNSUPPORTED;
    if (!Q || !L || !idx || !dscore || !count || !dQ || !dK || !ws) return SA_ERR_ARG;
    if (!aligned16(Q) || !aligned16(L) || !aligned16(dQ) || !aligned16(dK) || !aligned16(ws)) return SA_ERR_ARG;
    if (ws_bytes < sparse_attn_workspace_size(p, SA_OP_SELECT_BACKWARD)) return SA_ERR_WORKSPACE;
    return launch_result(launch_select_backward(s, Q, L, idx, dscore, count, dQ, dK, ws, (cudaStream_t)stream));
}

int sparse_attn_lsa_clusters(const sa_lsa_params *p) {
    LsaShape s;
    const int r = resolve_lsa(p, s);
    return r != SA_OK ? r : s.ctotal;
}

size_t sparse_attn_lsa_workspace_size(const sa_lsa_params *p) {
    LsaShape s;
    LsaDecPlan pl;
    if (resolve_lsa(p, s) != SA_OK || !lsa_decode_plan(s, pl)) return 0;
    return pl.bytes;
}

int sparse_attn_lsa_build(const sa_lsa_params *p, const void *K, double *centres, int32_t *members, int32_t *sizes,
                          void *stream) {
    LsaShape s;
    const int r = resolve_lsa(p, s);
    if (r != SA_OK) return r;
    if (!K || !aligned16(K)) return SA_ERR_ARG;
    if (s.ctotal > 0 && (!centres || !members || !sizes)) return SA_ERR_ARG;
    return launch_result(launch_lsa_build(s, K, centres, members, sizes, (cudaStream_t)stream));
}

int sparse_attn_lsa_decode(const sa_lsa_params *p, const void *q, const void *K, const void *V,
                           const double *centres, const int32_t *members, const int32_t *sizes, void *o, float *lse,
                           int32_t *kept, void *ws, size_t ws_bytes, void *stream) {
    LsaShape s;
    LsaDecPlan pl;
    const int r = resolve_lsa(p, s);
    if (r != SA_OK) return r;
    if (!lsa_decode_plan(s, pl)) return SA_ERR_UNSUPPORTED;
    if (!q || !K || !V || !o || !lse || !ws) return SA_ERR_ARG;
    if (s.ctotal > 0 && (!centres || !members || !sizes)) return SA_ERR_ARG;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(ws)) return SA_ERR_ARG;
    if (s.ctotal > 0 && !aligned16(centres)) return SA_ERR_ARG;
    if (ws_bytes < pl.bytes) return SA_ERR_WORKSPACE;
    return launch_result(launch_lsa_decode(s, pl, q, K, V, centres, members, sizes, ws, o, lse, kept,
                                           (cudaStream_t)stream));
}

static int resolve_tree(const sa_lsa_params *p, int fanout, LsaShape &s, LsaTreePlan &tp) {
    const int r = resolve_lsa(p, s);
    if (r != SA_OK) return r;
    if (fanout < 2) return SA_ERR_ARG;
    if (!lsa_tree_plan(s, fanout, tp)) return SA_ERR_UNSUPPORTED;
    return SA_OK;
}

size_t sparse_attn_lsa_tree_size(const sa_lsa_params *p, int fanout, int *levels) {
    LsaShape s;
    LsaTreePlan tp;
    if (resolve_tree(p, fanout, s, tp) != SA_OK) return 0;
    if (levels) *levels = tp.L;
    return tp.bytes;
}

size_t sparse_attn_lsa_tree_workspace_size(const sa_lsa_params *p, int fanout) {
    LsaShape s;
    LsaTreePlan tp;
    LsaDecPlan pl;
    if (resolve_tree(p, fanout, s, tp) != SA_OK || !lsa_decode_plan(s, pl, false)) return 0;
    return pl.bytes + tp.work_bytes;     // the decode's regions, then the build's working centres
}

int sparse_attn_lsa_tree_build(const sa_lsa_params *p, int fanout, const double *centres, const int32_t *sizes,
                               void *tree, void *ws, size_t ws_bytes, void *stream) {
    LsaShape s;
    LsaTreePlan tp;
    LsaDecPlan pl;
    const int r = resolve_tree(p, fanout, s, tp);
    if (r != SA_OK) return r;
    if (!lsa_decode_plan(s, pl, false)) return SA_ERR_UNSUPPORTED;
    if (!centres || !sizes || !tree || !ws) return SA_ERR_ARG;
    if (!aligned16(centres) || !aligned16(tree) || !aligned16(ws)) return SA_ERR_ARG;
    if (ws_bytes < sparse_attn_lsa_tree_workspace_size(p, fanout)) return SA_ERR_WORKSPACE;
    double *work = reinterpret_cast<double *>(static_cast<unsigned char *>(ws) + pl.bytes);
    return launch_result(launch_lsa_tree_build(s, tp, centres, sizes, tree, work, (cudaStream_t)stream));
}

int sparse_attn_lsa_tree_decode(const sa_lsa_params *p, int fanout, int beam, const void *q, const void *K,
                                const void *V, const double *centres, const int32_t *members, const int32_t *sizes,
                                const void *tree, void *o, float *lse, int32_t *kept, int32_t *compared, void *ws,
                                size_t ws_bytes, void *stream) {
    LsaShape s;
    LsaTreePlan tp;
    LsaDecPlan pl;
    const int r = resolve_tree(p, fanout, s, tp);
    if (r != SA_OK) return r;
    if (beam < 1) return SA_ERR_ARG;
    if (!lsa_decode_plan(s, pl, false)) return SA_ERR_UNSUPPORTED;
    if (!q || !K || !V || !centres || !members || !sizes || !tree || !o || !lse || !ws) return SA_ERR_ARG;
    if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(ws) || !aligned16(centres) || !aligned16(tree))
        return SA_ERR_ARG;
    if (ws_bytes < sparse_attn_lsa_tree_workspace_size(p, fanout)) return SA_ERR_WORKSPACE;
    return launch_result(launch_lsa_tree_decode(s, pl, tp, beam, q, K, V, centres, members, sizes, tree, ws, o, lse,
                                                kept, compared, (cudaStream_t)stream));
}

int sparse_attn_check_status(void *ws, void *stream, int *detail) {
    if (!ws) return SA_ERR_ARG;
    unsigned word = 0;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return SA_ERR_LAUNCH;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_LAUNCH;
    if (detail) *detail = (int)word;
    if (word) {
        if (cudaMemsetAsync(ws, 0, sizeof(word), st) != cudaSuccess) return SA_ERR_LAUNCH;
        if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_LAUNCH;
        return SA_ERR_DEVICE;
    }
    return SA_OK;
}

const char *sparse_attn_status_string(int code) {
    switch (code) {
        case SA_OK: return "ok";
        case SA_ERR_ARG: return "invalid argument (null or misaligned pointer, bad shape or flag)";
        case SA_ERR_UNSUPPORTED: return "unsupported combination of shape, dtype or flags";
        case SA_ERR_WORKSPACE: return "workspace missing or too small";
        case SA_ERR_LAUNCH: return "CUDA launch or copy failed";
        case SA_ERR_DEVICE: return "device-side problem recorded in the status word";
        default: return "unknown status code";
    }
}

int sparse_attn_version(void) { return 100; }

int sparse_attn_last_cuda_error(void) { return t_last_cuda_error; }

const char *sparse_attn_cuda_error_string(int err) { return cudaGetErrorString((cudaError_t)err); }

unsigned long long sparse_attn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
