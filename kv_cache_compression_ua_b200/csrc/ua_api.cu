// ua_api.cu -- the C ABI of libua: argument validation, workspace carving and launches.
// Formulas, layouts and error behaviour are documented in include/ua.h.
#include <algorithm>
#include <vector>
#include <math.h>
#include <string.h>

#include <mutex>

#include "ua_common.cuh"
#include "ua_kernels.h"

namespace ua {
__device__ int g_status = 0;
__device__ unsigned long long g_wait_limit_ns = UA_WAIT_LIMIT_DEFAULT_NS;
}

using namespace ua;

namespace {

constexpr int kVersion = 100;   // 0.1.0
constexpr int kBq = 64;         // query tile height of the SIMT attention path
constexpr int kMaxCapacity = 1 << 20;   // decode keeps a capacity/32-word bitmap in shared memory

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool group_ok(int G) { return G == 1 || G == 2 || G == 3 || G == 4 || G == 8; }

// Known bits only, and at least one decay mechanism left on.
bool variant_ok(int v) { return (v & ~(kVarMech | kVarQNorm)) == 0 && (v & kVarMech) != kVarMech; }
bool prefill_variant_ok(int v) { return variant_ok(v & ~kVarPerHead); }

ua_status check_shape(const ua_shape* s) {
    if (!s) return UA_ERR_INVALID_ARG;
    if (s->B < 1 || s->T < 1 || s->H < 1 || s->Hkv < 1) return UA_ERR_INVALID_ARG;
    if (s->H % s->Hkv != 0) return UA_ERR_INVALID_ARG;
    if (!(s->rope_theta > 0.0) || !isfinite(s->scale)) return UA_ERR_INVALID_ARG;
    if (s->d != 64 && s->d != 128) return UA_ERR_UNSUPPORTED;
    if (!group_ok(s->H / s->Hkv)) return UA_ERR_UNSUPPORTED;
    if (s->dtype != UA_F32 && s->dtype != UA_BF16) return UA_ERR_UNSUPPORTED;
    if (!prefill_variant_ok(s->variant)) return UA_ERR_INVALID_ARG;
    if (!(s->prune_p >= 0.f && s->prune_p <= 1.f)) return UA_ERR_INVALID_ARG;
    return UA_OK;
}

// Per-query-head decay runs the per-KV-head path with one decay unit per query head, on keys
// and values repeated for the G query heads of each group (k_per_head.cu).
bool per_head(const ua_shape* s) { return (s->variant & kVarPerHead) != 0; }

ua_shape per_head_inner(const ua_shape* s) {
    ua_shape i = *s;
    i.Hkv = s->H;
    i.variant = s->variant & ~kVarPerHead;
    return i;
}

// bytes of one repeated key or value tensor [B,T,H,d], rounded to 256
size_t rep_bytes(const ua_shape* s) {
    const size_t e = s->dtype == UA_BF16 ? 2 : 4;
    return ((size_t)s->B * s->T * s->H * s->d * e + 255) / 256 * 256;
}

// Chunked pruned prefill: a key is evicted when its boundary prefix Pb exceeds -log p.
float prune_thr(const ua_shape* s) { return s->prune_p > 0.f ? -logf(s->prune_p) : INFINITY; }

// Workspace of the SIMT prefill forward: f32 rotated/normalised copies, rates, prefixes.
struct FwdWs {
    size_t qr, kh, kr, rq, rk, pb, mq, qmax, total;
};

FwdWs fwd_ws_layout(const ua_shape* s) {
    const size_t B = s->B, T = s->T, H = s->H, Hkv = s->Hkv, d = s->d;
    const size_t nqt = (T + kBq - 1) / kBq;
    FwdWs w;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = round_up(off + bytes, 256); return o; };
    w.qr = take(B * H * T * d * 4);
    w.kh = take(B * Hkv * T * d * 4);
    w.kr = take(B * Hkv * T * d * 4);
    w.rq = take(B * Hkv * T * 4);
    w.rk = take(B * Hkv * T * 4);
    w.pb = take(B * Hkv * nqt * T * 4);
    w.mq = take(B * H * T * 4);
    w.qmax = take(B * Hkv * nqt * 4);
    w.total = off;
    return w;
}

// Workspace of the tensor-core prefill forward: bf16 rotated/normalised copies (TMA
// sources), log2-rates and row bounds (rows padded to Tp), prefixes at 128-row query tiles.
// head_dim 64 cuts 128-row query tiles; head_dim 128 cuts 64-row query tiles (its prefix rows
// are then padded to whole 128-key tiles, Tpk) and counts its publications per 128-key tile.
struct TcWs {
    size_t qr, kh, kr, lq2, lk2, mq, pb, flags, flags_bytes, fix_list, fix_scratch, total;
    int Tp, Tpk, nqt, nkt;
    size_t fix_count_word, fix_state_word;   // word offsets inside the zeroed flags region
};

TcWs tc_ws_layout(const ua_shape* s) {
    const size_t B = s->B, T = s->T, H = s->H, Hkv = s->Hkv, d = s->d;
    TcWs w;
    w.Tp = (int)round_up(T, 4);
    const size_t bq = d == 128 ? 64 : 128;
    w.nqt = (int)((T + bq - 1) / bq);
    w.nkt = (int)((T + 127) / 128);
    w.Tpk = d == 128 ? (int)round_up(T, 128) : w.Tp;
    const size_t Tp = w.Tp;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = round_up(off + bytes, 1024); return o; };
    w.qr = take(B * H * T * d * 2);
    w.kh = take(B * Hkv * T * d * 2);
    w.kr = take(B * Hkv * T * d * 2);
    w.lq2 = take(B * Hkv * Tp * 4);
    w.lk2 = take(B * Hkv * Tp * 4);
    w.mq = take(B * H * Tp * 4);
    w.pb = take(B * Hkv * (size_t)w.nqt * w.Tpk * 4);
    // publication counters, the work ticket, the skip counter, the count of rows listed for
    // the exact recomputation, a spare word, then one recomputation state per unit
    w.fix_count_word = B * Hkv * (size_t)w.nqt * w.nkt + 2;
    w.fix_state_word = B * Hkv * (size_t)w.nqt * w.nkt + 4;
    w.flags_bytes = (B * Hkv * (size_t)w.nqt * w.nkt + 4 + B * Hkv) * 4;
    w.flags = take(w.flags_bytes);
    w.fix_list = take(B * H * T * 4);
    w.fix_scratch = take((size_t)kFixGrid * T * 4);
    w.total = off;
    return w;
}

// The tensor-core forward evaluates the three-rate geometric mean only (its decay runs in
// log2 units with the cube root folded in); a shape with a mechanism switched off runs SIMT.
bool use_tc(const ua_shape* s) {
    // (the rows listed for the exact recomputation are indexed by (b*H + h)*T + i in an int)
    return s->dtype == UA_BF16 && fwd_tc_supported(s->d, s->H / s->Hkv) && (s->variant & kVarMech) == 0 &&
           (size_t)s->B * s->H * s->T < (size_t)INT32_MAX;
}

size_t prefill_ws_bytes(const ua_shape* s) {
    size_t n = fwd_ws_layout(s).total;
    if (use_tc(s)) {
        const size_t t = tc_ws_layout(s).total;
        // the debug Lambda output (T <= 1024) runs the SIMT path, so small T reserve both
        n = s->T <= 1024 ? (n > t ? n : t) : t;
    }
    return n;
}

ua_status cuda_status(cudaError_t e) { return e == cudaSuccess ? UA_OK : UA_ERR_CUDA; }

// RoPE frequencies theta^(-2m/d), m < d/2, in double precision.
RopeFreq rope_freq(double theta, int d) {
    RopeFreq r;
    for (int m = 0; m < 64; ++m) r.f[m] = (m < d / 2) ? pow(theta, -2.0 * (double)m / (double)d) : 0.0;
    return r;
}

char* at(void* base, size_t off) { return static_cast<char*>(base) + off; }

ua_status check_cache(const ua_cache* c) {
    if (!c) return UA_ERR_INVALID_ARG;
    if (c->B < 1 || c->Hkv < 1 || c->capacity < 1) return UA_ERR_INVALID_ARG;
    if (c->capacity > kMaxCapacity) return UA_ERR_UNSUPPORTED;
    if (c->d != 64 && c->d != 128) return UA_ERR_UNSUPPORTED;
    if (c->dtype != UA_F32 && c->dtype != UA_BF16) return UA_ERR_UNSUPPORTED;
    if (c->kv_rep < 0 || (c->kv_rep > 1 && c->Hkv % c->kv_rep != 0)) return UA_ERR_INVALID_ARG;
    if (!c->khat || !c->v || !c->bias || !c->rk || !c->pos || !c->n_kept) return UA_ERR_INVALID_ARG;
    const void* ps[] = {c->khat, c->v, c->bias, c->rk, c->pos, c->n_kept};
    for (const void* p : ps)
        if (!aligned(p, 16)) return UA_ERR_ALIGNMENT;
    if (c->page_table) {                      // paged storage
        const int sz = c->page_size;
        if (sz < 128 || sz > kMaxCapacity || (sz & (sz - 1)) != 0) return UA_ERR_INVALID_ARG;
        if (c->max_pages < 1 || c->pool_pages < 1) return UA_ERR_INVALID_ARG;
        if ((long long)c->max_pages * sz != c->capacity) return UA_ERR_INVALID_ARG;
        if ((long long)c->pool_pages * sz >= (long long)INT32_MAX) return UA_ERR_UNSUPPORTED;
        if (!aligned(c->page_table, 4)) return UA_ERR_ALIGNMENT;
    }
    return UA_OK;
}

CacheView view(const ua_cache* c) {
    CacheView v;
    v.B = c->B; v.Hkv = c->Hkv; v.d = c->d; v.cap = c->capacity; v.rep = c->kv_rep > 1 ? c->kv_rep : 1;
    v.khat = c->khat; v.v = c->v; v.bias = c->bias; v.rk = c->rk;
    v.pos = c->pos; v.n_kept = c->n_kept;
    v.pt = c->page_table;
    v.ps_shift = 0;
    v.max_pages = v.pool_pages = 0;
    if (c->page_table) {
        while ((1 << v.ps_shift) < c->page_size) ++v.ps_shift;
        v.max_pages = c->max_pages;
        v.pool_pages = c->pool_pages;
    }
    return v;
}

}  // namespace

extern "C" {

int ua_version(void) { return kVersion; }

const char* ua_status_string(ua_status s) {
    switch (s) {
        case UA_OK: return "UA_OK";
        case UA_ERR_INVALID_ARG: return "UA_ERR_INVALID_ARG";
        case UA_ERR_UNSUPPORTED: return "UA_ERR_UNSUPPORTED";
        case UA_ERR_ALIGNMENT: return "UA_ERR_ALIGNMENT";
        case UA_ERR_WORKSPACE: return "UA_ERR_WORKSPACE";
        case UA_ERR_CAPACITY: return "UA_ERR_CAPACITY";
        case UA_ERR_CUDA: return "UA_ERR_CUDA";
        case UA_ERR_TIMEOUT: return "UA_ERR_TIMEOUT";
        case UA_ERR_RANGE: return "UA_ERR_RANGE";
    }
    return "UA_ERR_UNKNOWN";
}

// Whole workspace of a forward call (per-query-head decay: two repeated tensors first).
size_t fwd_call_ws_bytes(const ua_shape* s) {
    if (!per_head(s)) return prefill_ws_bytes(s);
    const ua_shape in = per_head_inner(s);
    return 2 * rep_bytes(s) + prefill_ws_bytes(&in);
}

ua_status ua_prefill_workspace_size(const ua_shape* shape, size_t* bytes) {
    ua_status st = check_shape(shape);
    if (st != UA_OK) return st;
    if (!bytes) return UA_ERR_INVALID_ARG;
    *bytes = fwd_call_ws_bytes(shape);
    return UA_OK;
}

static ua_status prefill_fwd_simt(const ua_shape* s, const void* q, const void* k, const void* v, const void* g,
                                  const float* a_q, const float* a_k, const float* alpha, const float* beta,
                                  void* o, float* lse, float* b_final, float* lambda_dbg, void* ws,
                                  cudaStream_t cs) {
    ua_status st;
    const FwdWs w = fwd_ws_layout(s);
    const bool bf = s->dtype == UA_BF16;
    const int nqt = (s->T + kBq - 1) / kBq;
    PrepParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.B = s->B; pp.T = s->T; pp.H = s->H; pp.Hkv = s->Hkv; pp.d = s->d; pp.theta = s->rope_theta;
    pp.q = q; pp.k = k; pp.a_q = a_q; pp.a_k = a_k;
    pp.qr = at(ws, w.qr); pp.kh = at(ws, w.kh); pp.kr = at(ws, w.kr);
    pp.rq = reinterpret_cast<float*>(at(ws, w.rq)); pp.rk = reinterpret_cast<float*>(at(ws, w.rk));
    pp.rf = rope_freq(s->rope_theta, s->d);
    pp.mq = reinterpret_cast<float*>(at(ws, w.mq)); pp.Tp = s->T; pp.mq_scale = s->scale;
    pp.variant = s->variant;
    if ((st = cuda_status(launch_prep(pp, bf, false, cs))) != UA_OK) return st;
    TileQmaxParams tq;
    tq.B = s->B; tq.T = s->T; tq.H = s->H; tq.Hkv = s->Hkv; tq.nqt = nqt; tq.mq = pp.mq;
    tq.qmax = reinterpret_cast<float*>(at(ws, w.qmax));
    if ((st = cuda_status(launch_tile_qmax(tq, cs))) != UA_OK) return st;

    BoundaryParams bp;
    bp.B = s->B; bp.T = s->T; bp.Hkv = s->Hkv; bp.d = s->d; bp.bq = kBq; bp.nqt = nqt;
    bp.kh = reinterpret_cast<const float*>(pp.kh); bp.rq = pp.rq; bp.rk = pp.rk;
    bp.alpha = alpha; bp.beta = beta;
    bp.pb = reinterpret_cast<float*>(at(ws, w.pb)); bp.bfinal = b_final; bp.variant = s->variant;
    if ((st = cuda_status(launch_boundary_simt(bp, cs))) != UA_OK) return st;

    if (lambda_dbg) {
        const size_t n = (size_t)s->B * s->Hkv * s->T * s->T * sizeof(float);
        if ((st = cuda_status(cudaMemsetAsync(lambda_dbg, 0, n, cs))) != UA_OK) return st;
    }
    FwdParams fp;
    fp.B = s->B; fp.T = s->T; fp.H = s->H; fp.Hkv = s->Hkv; fp.d = s->d; fp.G = s->H / s->Hkv; fp.nqt = nqt;
    fp.scale = s->scale;
    fp.qr = reinterpret_cast<const float*>(pp.qr); fp.kh = reinterpret_cast<const float*>(pp.kh);
    fp.kr = reinterpret_cast<const float*>(pp.kr);
    fp.v = v; fp.g = g; fp.rq = pp.rq; fp.rk = pp.rk; fp.alpha = alpha; fp.beta = beta; fp.pb = bp.pb;
    fp.qmax = tq.qmax;
    fp.o = o; fp.lse = lse; fp.lambda_dbg = lambda_dbg; fp.variant = s->variant; fp.prune_thr = prune_thr(s);
    return cuda_status(launch_fwd_simt(fp, bf, cs));
}

static ua_status prefill_fwd_tc(const ua_shape* s, const void* q, const void* k, const void* v, const void* g,
                                const float* a_q, const float* a_k, const float* alpha, const float* beta,
                                void* o, float* lse, float* b_final, void* ws, cudaStream_t cs) {
    ua_status st;
    const TcWs w = tc_ws_layout(s);
    PrepParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.B = s->B; pp.T = s->T; pp.H = s->H; pp.Hkv = s->Hkv; pp.d = s->d; pp.theta = s->rope_theta;
    pp.q = q; pp.k = k; pp.a_q = a_q; pp.a_k = a_k;
    pp.qr = at(ws, w.qr); pp.kh = at(ws, w.kh); pp.kr = at(ws, w.kr);
    pp.rq = nullptr; pp.rk = nullptr;
    pp.Tp = w.Tp; pp.mq_scale = s->scale * 1.4426950408889634f;
    pp.lq2 = reinterpret_cast<float*>(at(ws, w.lq2)); pp.lk2 = reinterpret_cast<float*>(at(ws, w.lk2));
    pp.mq = reinterpret_cast<float*>(at(ws, w.mq));
    pp.rf = rope_freq(s->rope_theta, s->d);
    pp.variant = s->variant;   // the query norm only: use_tc excludes the mechanism bits
    if ((st = cuda_status(launch_prep(pp, true, true, cs))) != UA_OK) return st;

    // the fused forward zeroes its publication counters and ticket itself (stream-ordered)
    if ((st = cuda_status(cudaMemsetAsync(at(ws, w.flags), 0, w.flags_bytes, cs))) != UA_OK) return st;
    FwdTcLaunch L;
    L.B = s->B; L.T = s->T; L.Tp = w.Tp; L.Tpk = w.Tpk; L.H = s->H; L.Hkv = s->Hkv; L.nqt = w.nqt;
    L.scale = s->scale;
    L.kh = pp.kh; L.kr = pp.kr; L.qr = pp.qr; L.v = v; L.lq2 = pp.lq2; L.lk2 = pp.lk2; L.mq = pp.mq;
    L.pincl = reinterpret_cast<float*>(at(ws, w.pb));
    L.flags = reinterpret_cast<unsigned*>(at(ws, w.flags));
    L.alpha = alpha; L.beta = beta; L.g = g; L.o = o; L.lse = lse; L.b_final = b_final; L.prune_thr = prune_thr(s);
    unsigned* fl = reinterpret_cast<unsigned*>(at(ws, w.flags));
    L.fix_count = fl + w.fix_count_word;
    L.fix_list = reinterpret_cast<int*>(at(ws, w.fix_list));
    if ((st = cuda_status(s->d == 128 ? launch_fwd_tc128(L, cs) : launch_fwd_tc(L, cs))) != UA_OK) return st;
    // rows whose shifted row sum fell out of range are recomputed exactly (an empty list costs
    // one launch whose CTAs return at once)
    FixParams fx;
    fx.B = s->B; fx.T = s->T; fx.H = s->H; fx.Hkv = s->Hkv; fx.G = s->H / s->Hkv; fx.d = s->d;
    fx.QT = s->d == 128 ? 64 : 128; fx.nqt = w.nqt; fx.Tp = w.Tp; fx.Tpk = w.Tpk;
    fx.scale = s->scale;
    fx.qr = pp.qr; fx.kh = pp.kh; fx.kr = pp.kr; fx.lq2 = pp.lq2; fx.lk2 = pp.lk2; fx.pincl = L.pincl;
    fx.alpha = alpha; fx.beta = beta; fx.v = v; fx.g = g; fx.o = o; fx.lse = lse;
    fx.prune_thr = L.prune_thr; fx.prefix_exact = b_final != nullptr ? 1 : 0;
    fx.fix_count = L.fix_count; fx.fix_list = L.fix_list; fx.fix_state = fl + w.fix_state_word;
    fx.scratch = reinterpret_cast<float*>(at(ws, w.fix_scratch));
    return cuda_status(launch_fwd_fix(fx, kFixGrid, cs));
}

// A validated forward: per-query-head decay repeats K and V into the head of the workspace and
// runs the per-KV-head path on the rest of it.
static ua_status prefill_fwd_dispatch(const ua_shape* s, const void* q, const void* k, const void* v, const void* g,
                                      const float* a_q, const float* a_k, const float* alpha, const float* beta,
                                      void* o, float* lse, float* b_final, float* lambda_dbg, void* ws,
                                      cudaStream_t cs) {
    if (per_head(s)) {
        const ua_shape in = per_head_inner(s);
        const size_t rb = rep_bytes(s);
        void* kr = ws;
        void* vr = at(ws, rb);
        const bool bf = s->dtype == UA_BF16;
        const int G = s->H / s->Hkv;
        ua_status st;
        if ((st = cuda_status(launch_repeat_kv(k, kr, s->B, s->T, s->H, G, s->d, bf, cs))) != UA_OK) return st;
        if ((st = cuda_status(launch_repeat_kv(v, vr, s->B, s->T, s->H, G, s->d, bf, cs))) != UA_OK) return st;
        return prefill_fwd_dispatch(&in, q, kr, vr, g, a_q, a_k, alpha, beta, o, lse, b_final, lambda_dbg,
                                    at(ws, 2 * rb), cs);
    }
    if (use_tc(s) && !lambda_dbg) return prefill_fwd_tc(s, q, k, v, g, a_q, a_k, alpha, beta, o, lse, b_final, ws, cs);
    return prefill_fwd_simt(s, q, k, v, g, a_q, a_k, alpha, beta, o, lse, b_final, lambda_dbg, ws, cs);
}

ua_status ua_prefill_fwd(const ua_shape* s, const void* q, const void* k, const void* v, const void* g,
                         const float* a_q, const float* a_k, const float* alpha, const float* beta,
                         void* o, float* lse, float* b_final, float* lambda_dbg, void* ws, size_t ws_bytes,
                         void* stream) {
    ua_status st = check_shape(s);
    if (st != UA_OK) return st;
    if (!q || !k || !v || !g || !a_q || !a_k || !alpha || !beta || !o || !ws) return UA_ERR_INVALID_ARG;
    const void* ps[] = {q, k, v, g, a_q, a_k, alpha, beta, o, lse, b_final, lambda_dbg};
    for (const void* p : ps)
        if (p && !aligned(p, 16)) return UA_ERR_ALIGNMENT;
    if (!aligned(ws, 256)) return UA_ERR_ALIGNMENT;
    if (lambda_dbg && s->T > 1024) return UA_ERR_INVALID_ARG;
    if (ws_bytes < fwd_call_ws_bytes(s)) return UA_ERR_WORKSPACE;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    return prefill_fwd_dispatch(s, q, k, v, g, a_q, a_k, alpha, beta, o, lse, b_final, lambda_dbg, ws, cs);
}

// ---------------------------------------------------------------------------------------
// Allocation-free prefill forward.  Some callers cannot allocate device memory at all: a
// plug-in whose host application (an inference server, a game engine) has already carved
// the whole GPU into its own memory pool and forbids further cudaMalloc calls, or a caller
// that must not pay cudaMalloc's latency and device-wide synchronisation.  Such callers use
// ua_prefill_fwd_noalloc, whose scratch is this fixed file-scope device array instead of a
// caller workspace.  Every device that loads the library holds the array until exit.
namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;   // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the array on the current device, resolved once per device.  The array's
// host-side symbol is only a handle and must never be handed to a kernel.
ua_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return UA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return UA_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return UA_OK;
}
}  // namespace

ua_status ua_prefill_fwd_noalloc(const ua_shape* s, const void* q, const void* k, const void* v, const void* g,
                                 const float* a_q, const float* a_k, const float* alpha, const float* beta,
                                 void* o, float* lse, float* b_final, void* stream) {
    ua_status st = check_shape(s);
    if (st != UA_OK) return st;
    if (!q || !k || !v || !g || !a_q || !a_k || !alpha || !beta || !o) return UA_ERR_INVALID_ARG;
    const void* ps[] = {q, k, v, g, a_q, a_k, alpha, beta, o, lse, b_final};
    for (const void* p : ps)
        if (p && !aligned(p, 16)) return UA_ERR_ALIGNMENT;
    if (fwd_call_ws_bytes(s) > kNoAllocScratchBytes) return UA_ERR_WORKSPACE;
    void* ws = nullptr;
    if ((st = noalloc_scratch(&ws)) != UA_OK) return st;
    // Every part of the scratch is written before it is read within a call, so nothing has
    // to be cleared between calls.
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    return prefill_fwd_dispatch(s, q, k, v, g, a_q, a_k, alpha, beta, o, lse, b_final, nullptr, ws, cs);
}

size_t ua_prefill_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

// Workspace of the backward: the f32 token preparation and decay prefixes of the SIMT
// forward, then f32 gradient intermediates.
struct BwdWs {
    FwdWs f;
    size_t delta, dpb, dqr, dkh, dkh_rows, dkr, dv32, daq, dak, dab, total;
    int nqt, nkt;
};

BwdWs bwd_ws_layout(const ua_shape* s) {
    BwdWs w;
    w.f = fwd_ws_layout(s);
    const size_t B = s->B, T = s->T, H = s->H, Hkv = s->Hkv, d = s->d;
    w.nqt = (int)((T + kBq - 1) / kBq);
    w.nkt = (int)((T + 31) / 32);
    size_t off = w.f.total;
    auto take = [&](size_t bytes) { size_t o = off; off = round_up(off + bytes, 256); return o; };
    w.delta = take(B * H * T * 4);
    w.dpb = take(B * Hkv * (size_t)w.nqt * T * 4);
    w.dqr = take(B * H * T * d * 4);
    w.dkh = take(B * Hkv * T * d * 4);
    w.dkh_rows = take(B * Hkv * T * d * 4);
    w.dkr = take(B * Hkv * T * d * 4);
    w.dv32 = take(B * Hkv * T * d * 4);
    w.daq = take(B * Hkv * T * 4);
    w.dak = take(B * Hkv * T * 4);
    w.dab = take(B * Hkv * (size_t)w.nkt * 2 * 4);
    w.total = off;
    return w;
}

// Workspace of the tensor-core backward: the bf16 token preparation of the tensor-core forward,
// dA, Delta and lse in log2 units, the decay prefixes above every 32-row step, the stored bf16
// dZ^T / dX^T tiles of the causal band, and f32 gradient intermediates.
struct BwdTcWs {
    size_t qr, kh, kr, lq2, lk2, mq, ad, lse2, delta, pb, tiles, daq, cmax, slast, dab, dv32, dkr, dkh, dkh_rows,
        dqr, dak, total, ntiles;
    int Tp, Tpk, nkt, nst;
};

BwdTcWs bwd_tc_ws_layout(const ua_shape* s) {
    const size_t B = s->B, T = s->T, H = s->H, Hkv = s->Hkv, d = s->d, G = s->H / s->Hkv;
    BwdTcWs w;
    w.Tp = (int)round_up(T, 4);
    w.nkt = (int)((T + 127) / 128);
    w.Tpk = w.nkt * 128;
    w.nst = 4 * w.nkt;
    w.ntiles = (size_t)2 * w.nkt * (w.nkt + 1);
    const size_t Tp = w.Tp, Tpk = w.Tpk, nkt = w.nkt;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = round_up(off + bytes, 1024); return o; };
    w.qr = take(B * H * T * d * 2);
    w.kh = take(B * Hkv * T * d * 2);
    w.kr = take(B * Hkv * T * d * 2);
    w.lq2 = take(B * Hkv * Tp * 4);
    w.lk2 = take(B * Hkv * Tp * 4);
    w.mq = take(B * H * Tp * 4);
    w.ad = take(B * H * T * d * 2);
    w.lse2 = take(B * H * Tp * 4);
    w.delta = take(B * H * Tp * 4);
    w.pb = take(B * Hkv * (size_t)w.nst * Tpk * 4);
    w.tiles = take(B * Hkv * (G + 1) * w.ntiles * 8192);
    w.daq = take(B * Hkv * nkt * 4 * Tpk * 4);
    w.cmax = take(B * Hkv * Tpk * 4);
    w.slast = take(B * Hkv * nkt * 4);
    w.dab = take(B * Hkv * nkt * 2 * 4);
    w.dv32 = take(B * Hkv * T * d * 4);
    w.dkr = take(B * Hkv * T * d * 4);
    w.dkh = take(B * Hkv * T * d * 4);
    w.dkh_rows = take(B * Hkv * T * d * 4);
    w.dqr = take(B * H * T * d * 4);
    w.dak = take(B * Hkv * T * 4);
    w.total = off;
    return w;
}

// bf16 problems of the three-rate method (or with the query norm) whose head_dim and group size
// the tensor-core kernels take run the tensor-core backward; the others the fp32 SIMT one.
bool use_bwd_tc(const ua_shape* s) {
    return s->dtype == UA_BF16 && bwd_tc_supported(s->d, s->H / s->Hkv) && (s->variant & kVarMech) == 0;
}

size_t bwd_inner_ws_bytes(const ua_shape* s) {
    return use_bwd_tc(s) ? bwd_tc_ws_layout(s).total : bwd_ws_layout(s).total;
}

// Whole workspace of a backward call (per-query-head decay: repeated K, V and their gradient
// copies first).
size_t bwd_call_ws_bytes(const ua_shape* s) {
    if (!per_head(s)) return bwd_inner_ws_bytes(s);
    const ua_shape in = per_head_inner(s);
    return 4 * rep_bytes(s) + bwd_inner_ws_bytes(&in);
}

ua_status ua_prefill_bwd_workspace_size(const ua_shape* shape, size_t* bytes) {
    ua_status st = check_shape(shape);
    if (st != UA_OK) return st;
    if (!bytes || shape->prune_p != 0.f) return UA_ERR_INVALID_ARG;   // training is dense
    *bytes = bwd_call_ws_bytes(shape);
    return UA_OK;
}

static ua_status prefill_bwd_tc(const ua_shape* s, const void* q, const void* k, const void* v, const void* g,
                                const float* a_q, const float* a_k, const float* alpha, const float* beta,
                                const void* o, const float* lse, const void* d_o, void* dq, void* dk, void* dv,
                                void* dg, float* da_q, float* da_k, float* dalpha, float* dbeta, void* ws,
                                cudaStream_t cs) {
    ua_status st;
    const BwdTcWs w = bwd_tc_ws_layout(s);
    PrepParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.B = s->B; pp.T = s->T; pp.H = s->H; pp.Hkv = s->Hkv; pp.d = s->d; pp.theta = s->rope_theta;
    pp.q = q; pp.k = k; pp.a_q = a_q; pp.a_k = a_k;
    pp.qr = at(ws, w.qr); pp.kh = at(ws, w.kh); pp.kr = at(ws, w.kr);
    pp.rq = nullptr; pp.rk = nullptr;
    pp.Tp = w.Tp; pp.mq_scale = s->scale * 1.4426950408889634f;
    pp.lq2 = reinterpret_cast<float*>(at(ws, w.lq2)); pp.lk2 = reinterpret_cast<float*>(at(ws, w.lk2));
    pp.mq = reinterpret_cast<float*>(at(ws, w.mq));
    pp.rf = rope_freq(s->rope_theta, s->d);
    pp.variant = s->variant;   // the query norm only: use_bwd_tc excludes the mechanism bits
    if ((st = cuda_status(launch_prep(pp, true, true, cs))) != UA_OK) return st;
    BwdTcParams p;
    p.B = s->B; p.T = s->T; p.Tp = w.Tp; p.Tpk = w.Tpk; p.H = s->H; p.Hkv = s->Hkv; p.d = s->d;
    p.G = s->H / s->Hkv; p.nkt = w.nkt; p.nst = w.nst; p.scale = s->scale; p.rf = pp.rf; p.variant = s->variant;
    p.qr = pp.qr; p.kh = pp.kh; p.kr = pp.kr; p.lq2 = pp.lq2; p.lk2 = pp.lk2; p.mq = pp.mq;
    p.q = q; p.k = k; p.v = v; p.g = g; p.o = o; p.d_o = d_o;
    p.a_q = a_q; p.a_k = a_k; p.alpha = alpha; p.beta = beta; p.lse = lse;
    p.ad = at(ws, w.ad);
    p.lse2 = reinterpret_cast<float*>(at(ws, w.lse2));
    p.delta = reinterpret_cast<float*>(at(ws, w.delta));
    p.pb = reinterpret_cast<float*>(at(ws, w.pb));
    p.tiles = at(ws, w.tiles);
    p.ntiles = w.ntiles;
    p.daq_part = reinterpret_cast<float*>(at(ws, w.daq));
    p.cmax = reinterpret_cast<float*>(at(ws, w.cmax));
    p.slast = reinterpret_cast<int*>(at(ws, w.slast));
    p.dab = reinterpret_cast<float*>(at(ws, w.dab));
    p.dv32 = reinterpret_cast<float*>(at(ws, w.dv32));
    p.dkr = reinterpret_cast<float*>(at(ws, w.dkr));
    p.dkh_keys = reinterpret_cast<float*>(at(ws, w.dkh));
    p.dkh_rows = reinterpret_cast<float*>(at(ws, w.dkh_rows));
    p.dqr = reinterpret_cast<float*>(at(ws, w.dqr));
    p.dak32 = reinterpret_cast<float*>(at(ws, w.dak));
    p.dq = dq; p.dk = dk; p.dv = dv; p.dg = dg; p.da_q = da_q; p.da_k = da_k; p.dalpha = dalpha; p.dbeta = dbeta;
    return cuda_status(launch_bwd_tc(p, cs));
}

ua_status ua_prefill_bwd(const ua_shape* s, const void* q, const void* k, const void* v, const void* g,
                         const float* a_q, const float* a_k, const float* alpha, const float* beta, const void* o,
                         const float* lse, const float* b_final, const void* d_o, void* dq, void* dk, void* dv,
                         void* dg, float* da_q, float* da_k, float* dalpha, float* dbeta, void* ws, size_t ws_bytes,
                         void* stream) {
    ua_status st = check_shape(s);
    if (st != UA_OK) return st;
    if (s->prune_p != 0.f) return UA_ERR_INVALID_ARG;   // training is dense
    (void)b_final;   // the backward recomputes the decay prefixes; b_final is not read
    const void* need[] = {q, k, v, g, a_q, a_k, alpha, beta, o, lse, d_o, dq, dk, dv, dg, da_q, da_k, dalpha, dbeta, ws};
    for (const void* p : need)
        if (!p) return UA_ERR_INVALID_ARG;
    for (const void* p : need)
        if (!aligned(p, 16)) return UA_ERR_ALIGNMENT;
    if (!aligned(ws, 256)) return UA_ERR_ALIGNMENT;
    if (ws_bytes < bwd_call_ws_bytes(s)) return UA_ERR_WORKSPACE;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (per_head(s)) {
        // per-query-head decay: the per-KV-head backward on repeated K and V, whose key and
        // value gradients are then summed over each group's copies
        const ua_shape in = per_head_inner(s);
        const size_t rb = rep_bytes(s);
        void* kr = ws;
        void* vr = at(ws, rb);
        void* dkr = at(ws, 2 * rb);
        void* dvr = at(ws, 3 * rb);
        const bool bfa = s->dtype == UA_BF16;
        const int G = s->H / s->Hkv;
        if ((st = cuda_status(launch_repeat_kv(k, kr, s->B, s->T, s->H, G, s->d, bfa, cs))) != UA_OK) return st;
        if ((st = cuda_status(launch_repeat_kv(v, vr, s->B, s->T, s->H, G, s->d, bfa, cs))) != UA_OK) return st;
        if ((st = ua_prefill_bwd(&in, q, kr, vr, g, a_q, a_k, alpha, beta, o, lse, b_final, d_o, dq, dkr, dvr, dg,
                                 da_q, da_k, dalpha, dbeta, at(ws, 4 * rb), ws_bytes - 4 * rb, stream)) != UA_OK)
            return st;
        if ((st = cuda_status(launch_sum_copies(dkr, dk, s->B, s->T, s->Hkv, G, s->d, bfa, cs))) != UA_OK) return st;
        return cuda_status(launch_sum_copies(dvr, dv, s->B, s->T, s->Hkv, G, s->d, bfa, cs));
    }
    if (use_bwd_tc(s)) {
        return prefill_bwd_tc(s, q, k, v, g, a_q, a_k, alpha, beta, o, lse, d_o, dq, dk, dv, dg, da_q, da_k, dalpha,
                              dbeta, ws, cs);
    }
    const BwdWs w = bwd_ws_layout(s);
    if (ws_bytes < w.total) return UA_ERR_WORKSPACE;
    const bool bf = s->dtype == UA_BF16;

    PrepParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.B = s->B; pp.T = s->T; pp.H = s->H; pp.Hkv = s->Hkv; pp.d = s->d; pp.theta = s->rope_theta;
    pp.q = q; pp.k = k; pp.a_q = a_q; pp.a_k = a_k;
    pp.qr = at(ws, w.f.qr); pp.kh = at(ws, w.f.kh); pp.kr = at(ws, w.f.kr);
    pp.rq = reinterpret_cast<float*>(at(ws, w.f.rq)); pp.rk = reinterpret_cast<float*>(at(ws, w.f.rk));
    pp.rf = rope_freq(s->rope_theta, s->d);
    pp.mq = reinterpret_cast<float*>(at(ws, w.f.mq)); pp.Tp = s->T; pp.mq_scale = s->scale;
    pp.variant = s->variant;
    if ((st = cuda_status(launch_prep(pp, bf, false, cs))) != UA_OK) return st;
    TileQmaxParams tq;
    tq.B = s->B; tq.T = s->T; tq.H = s->H; tq.Hkv = s->Hkv; tq.nqt = w.nqt; tq.mq = pp.mq;
    tq.qmax = reinterpret_cast<float*>(at(ws, w.f.qmax));
    if ((st = cuda_status(launch_tile_qmax(tq, cs))) != UA_OK) return st;
    BoundaryParams bp;
    bp.B = s->B; bp.T = s->T; bp.Hkv = s->Hkv; bp.d = s->d; bp.bq = kBq; bp.nqt = w.nqt;
    bp.kh = reinterpret_cast<const float*>(pp.kh); bp.rq = pp.rq; bp.rk = pp.rk; bp.alpha = alpha; bp.beta = beta;
    bp.pb = reinterpret_cast<float*>(at(ws, w.f.pb)); bp.bfinal = nullptr; bp.variant = s->variant;
    if ((st = cuda_status(launch_boundary_simt(bp, cs))) != UA_OK) return st;

    BwdParams p;
    p.B = s->B; p.T = s->T; p.H = s->H; p.Hkv = s->Hkv; p.d = s->d; p.G = s->H / s->Hkv; p.nqt = w.nqt; p.nkt = w.nkt;
    p.scale = s->scale; p.theta = s->rope_theta; p.rf = pp.rf;
    p.qr = reinterpret_cast<const float*>(pp.qr); p.kh = reinterpret_cast<const float*>(pp.kh);
    p.kr = reinterpret_cast<const float*>(pp.kr); p.rq = pp.rq; p.rk = pp.rk; p.pb = bp.pb; p.qmax = tq.qmax;
    p.k = k; p.v = v; p.g = g; p.o = o; p.d_o = d_o; p.a_q = a_q; p.a_k = a_k; p.alpha = alpha; p.beta = beta;
    p.lse = lse;
    p.delta = reinterpret_cast<float*>(at(ws, w.delta)); p.dpb = reinterpret_cast<float*>(at(ws, w.dpb));
    p.dqr = reinterpret_cast<float*>(at(ws, w.dqr)); p.dkh = reinterpret_cast<float*>(at(ws, w.dkh));
    p.dkh_rows = reinterpret_cast<float*>(at(ws, w.dkh_rows)); p.dkr = reinterpret_cast<float*>(at(ws, w.dkr));
    p.dv32 = reinterpret_cast<float*>(at(ws, w.dv32)); p.daq32 = reinterpret_cast<float*>(at(ws, w.daq));
    p.dak32 = reinterpret_cast<float*>(at(ws, w.dak)); p.dab = reinterpret_cast<float*>(at(ws, w.dab));
    p.dq = dq; p.dk = dk; p.dv = dv; p.dg = dg; p.da_q = da_q; p.da_k = da_k; p.dalpha = dalpha; p.dbeta = dbeta;
    p.q = q; p.variant = s->variant;
    return cuda_status(launch_bwd_simt(p, bf, cs));
}

ua_status ua_cache_fill(const ua_cache* c, int T, const void* k, const void* v, const float* a_k,
                        const float* b_final, double rope_theta, void* stream) {
    ua_status st = check_cache(c);
    if (st != UA_OK) return st;
    if (T < 1 || !k || !v || !a_k || !b_final || !(rope_theta > 0.0)) return UA_ERR_INVALID_ARG;
    if (T > c->capacity) return UA_ERR_CAPACITY;
    const void* ps[] = {k, v, a_k, b_final};
    for (const void* p : ps)
        if (!aligned(p, 16)) return UA_ERR_ALIGNMENT;
    FillParams fp;
    fp.c = view(c); fp.T = T; fp.theta = rope_theta; fp.k = k; fp.v = v; fp.a_k = a_k; fp.bfinal = b_final;
    fp.rf = rope_freq(rope_theta, c->d);
    return cuda_status(launch_cache_fill(fp, c->dtype == UA_BF16, static_cast<cudaStream_t>(stream)));
}

ua_status ua_cache_compact(const ua_cache* c, const uint8_t* keep, float p, int32_t* kept_idx, void* stream) {
    ua_status st = check_cache(c);
    if (st != UA_OK) return st;
    if (!keep && !(p >= 0.f && p <= 1.f)) return UA_ERR_INVALID_ARG;
    if ((keep && !aligned(keep, 16)) || (kept_idx && !aligned(kept_idx, 16))) return UA_ERR_ALIGNMENT;
    CompactParams cp;
    cp.c = view(c); cp.keep = keep; cp.logp = p > 0.f ? logf(p) : -INFINITY; cp.kept_idx = kept_idx;
    return cuda_status(launch_cache_compact(cp, c->dtype == UA_BF16, static_cast<cudaStream_t>(stream)));
}

ua_status ua_decode_step(const ua_cache* c, int H, const void* q, const void* k, const void* v, const void* g,
                         const float* a_q, const float* a_k, const float* alpha, const float* beta, int pos_t,
                         float p, float scale, double rope_theta, void* o, uint32_t* evict_bits,
                         int32_t* kept_idx, int flags, void* stream) {
    ua_status st = check_cache(c);
    if (st != UA_OK) return st;
    const int defer = flags & UA_DECODE_DEFER_COMPACT;
    // per-query-head decay: a cache of one head per query head; the kernels see the method itself
    int var = flags & ~UA_DECODE_DEFER_COMPACT;
    if ((var & kVarPerHead) && H != c->Hkv) return UA_ERR_INVALID_ARG;
    var &= ~kVarPerHead;
    if (H < 1 || H % c->Hkv != 0 || pos_t < 0 || !variant_ok(var)) return UA_ERR_INVALID_ARG;
    if (!group_ok(H / c->Hkv)) return UA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !a_q || !a_k || !alpha || !beta || !o) return UA_ERR_INVALID_ARG;
    if (!(p >= 0.f && p <= 1.f) || !isfinite(scale) || !(rope_theta > 0.0)) return UA_ERR_INVALID_ARG;
    const void* ps[] = {q, k, v, g, a_q, a_k, alpha, beta, o, evict_bits, kept_idx};
    for (const void* x : ps)
        if (x && !aligned(x, 16)) return UA_ERR_ALIGNMENT;
    DecodeParams dp;
    dp.c = view(c); dp.H = H; dp.G = H / c->Hkv; dp.pos_t = pos_t; dp.scale = scale;
    dp.logp = p > 0.f ? logf(p) : -INFINITY; dp.theta = rope_theta; dp.rf = rope_freq(rope_theta, c->d);
    dp.q = q; dp.k = k; dp.v = v; dp.g = g; dp.a_q = a_q; dp.a_k = a_k; dp.alpha = alpha; dp.beta = beta;
    dp.o = o; dp.evict_bits = evict_bits; dp.kept_idx = kept_idx;
    dp.variant = var; dp.defer = defer ? 1 : 0;
    dp.split_cnt = nullptr; dp.split_state = nullptr;
    return cuda_status(launch_decode(dp, c->dtype == UA_BF16, static_cast<cudaStream_t>(stream)));
}

// Split decode: a counter per cache (256-byte block), then kDecodeSplitMax partial states of
// G*(d+2) floats per cache.
static size_t decode_ws_bytes(const ua_cache* c, int H) {
    const size_t units = (size_t)c->B * c->Hkv, G = (size_t)H / c->Hkv;
    return round_up(units * 4, 256) + units * kDecodeSplitMax * G * (c->d + 2) * 4;
}

ua_status ua_decode_workspace_size(const ua_cache* c, int H, size_t* bytes) {
    ua_status st = check_cache(c);
    if (st != UA_OK) return st;
    if (!bytes || H < 1 || H % c->Hkv != 0) return UA_ERR_INVALID_ARG;
    if (!group_ok(H / c->Hkv)) return UA_ERR_UNSUPPORTED;
    *bytes = decode_ws_bytes(c, H);
    return UA_OK;
}

ua_status ua_decode_step_split(const ua_cache* c, int H, const void* q, const void* k, const void* v, const void* g,
                               const float* a_q, const float* a_k, const float* alpha, const float* beta, int pos_t,
                               float p, float scale, double rope_theta, void* o, uint32_t* evict_bits,
                               int32_t* kept_idx, int flags, void* ws, size_t ws_bytes, void* stream) {
    ua_status st = check_cache(c);
    if (st != UA_OK) return st;
    int var = flags & ~UA_DECODE_DEFER_COMPACT;
    if ((var & kVarPerHead) && H != c->Hkv) return UA_ERR_INVALID_ARG;
    var &= ~kVarPerHead;
    if (H < 1 || H % c->Hkv != 0 || pos_t < 0 || !variant_ok(var)) return UA_ERR_INVALID_ARG;
    if (!group_ok(H / c->Hkv)) return UA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !a_q || !a_k || !alpha || !beta || !o || !ws) return UA_ERR_INVALID_ARG;
    if (!(p >= 0.f && p <= 1.f) || !isfinite(scale) || !(rope_theta > 0.0)) return UA_ERR_INVALID_ARG;
    const void* ps[] = {q, k, v, g, a_q, a_k, alpha, beta, o, evict_bits, kept_idx};
    for (const void* x : ps)
        if (x && !aligned(x, 16)) return UA_ERR_ALIGNMENT;
    if (!aligned(ws, 256)) return UA_ERR_ALIGNMENT;
    if (ws_bytes < decode_ws_bytes(c, H)) return UA_ERR_WORKSPACE;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const size_t units = (size_t)c->B * c->Hkv;
    // the per-cache arrival counters at the start of ws are zero before the first step (the
    // caller zeroes the workspace once) and every step leaves them zero, so consecutive steps
    // need no memset between their kernels
    DecodeParams dp;
    dp.c = view(c); dp.H = H; dp.G = H / c->Hkv; dp.pos_t = pos_t; dp.scale = scale;
    dp.logp = p > 0.f ? logf(p) : -INFINITY; dp.theta = rope_theta; dp.rf = rope_freq(rope_theta, c->d);
    dp.q = q; dp.k = k; dp.v = v; dp.g = g; dp.a_q = a_q; dp.a_k = a_k; dp.alpha = alpha; dp.beta = beta;
    dp.o = o; dp.evict_bits = evict_bits; dp.kept_idx = kept_idx; dp.variant = var; dp.defer = 1;
    dp.split_cnt = static_cast<unsigned*>(ws);
    dp.split_state = reinterpret_cast<float*>(at(ws, round_up(units * 4, 256)));
    // bf16 caches on the tensor cores (their TMA row coordinate must fit an int)
    const size_t rows = c->page_table ? (size_t)c->pool_pages * c->page_size : units * (size_t)c->capacity;
    if (c->dtype == UA_BF16 && rows < (size_t)INT32_MAX)
        return cuda_status(launch_decode_tc(dp, cs));
    return cuda_status(launch_decode_split(dp, c->dtype == UA_BF16, cs));
}

ua_status ua_prefill_tile_stats(const ua_shape* s, const void* ws, size_t ws_bytes, unsigned long long* tiles,
                                unsigned long long* skipped, void* stream) {
    if (!s || !tiles || !skipped) return UA_ERR_INVALID_ARG;
    if (s->B <= 0 || s->T <= 0 || s->Hkv <= 0) return UA_ERR_INVALID_ARG;
    if (s->d == 128 && (s->T + 63) / 64 > 0) {
        // 64-row query tiles: query tile t meets key tiles 0 .. t/2
        unsigned long long n = 0;
        for (long long t = 0; t < (s->T + 63) / 64; ++t) n += (unsigned long long)(t / 2 + 1);
        *tiles = (unsigned long long)s->B * s->Hkv * n;
    } else {
        const unsigned long long n = (unsigned long long)((s->T + 127) / 128);
        *tiles = (unsigned long long)s->B * s->Hkv * n * (n + 1) / 2;
    }
    *skipped = 0;
    if (!use_tc(s)) return UA_OK;
    const TcWs w = tc_ws_layout(s);
    if (!ws) return UA_ERR_INVALID_ARG;
    if (ws_bytes < w.total) return UA_ERR_WORKSPACE;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    unsigned host = 0;
    const size_t off = w.flags + ((size_t)s->B * s->Hkv * w.nqt * w.nkt + 1) * sizeof(unsigned);
    cudaError_t e = cudaMemcpyAsync(&host, static_cast<const uint8_t*>(ws) + off, sizeof(unsigned),
                                    cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return UA_ERR_CUDA;
    *skipped = host;
    return UA_OK;
}

ua_status ua_prefill_bwd_band_stats(const ua_shape* s, const void* ws, size_t ws_bytes, unsigned long long* steps,
                                    unsigned long long* walked, void* stream) {
    if (!s || !steps || !walked) return UA_ERR_INVALID_ARG;
    ua_status st = check_shape(s);
    if (st != UA_OK) return st;
    if (s->prune_p != 0.f) return UA_ERR_INVALID_ARG;
    if (per_head(s)) {
        // the per-KV-head backward on repeated K and V, whose workspace follows the four copies
        const ua_shape in = per_head_inner(s);
        const size_t rb = 4 * rep_bytes(s);
        if (!ws) return UA_ERR_INVALID_ARG;
        if (ws_bytes < rb) return UA_ERR_WORKSPACE;
        return ua_prefill_bwd_band_stats(&in, static_cast<const uint8_t*>(ws) + rb, ws_bytes - rb, steps, walked,
                                         stream);
    }
    // 32-row steps of the causal band: key tile kt meets steps 4kt .. nst-1
    const long long nkt = ((long long)s->T + 127) / 128, nst = 4 * nkt;
    const unsigned long long per_unit = (unsigned long long)(nkt * nst - 4 * nkt * (nkt - 1) / 2);
    *steps = (unsigned long long)s->B * s->Hkv * per_unit;
    *walked = *steps;
    if (!use_bwd_tc(s)) return UA_OK;                 // the SIMT backward walks the whole band
    const BwdTcWs w = bwd_tc_ws_layout(s);
    if (!ws) return UA_ERR_INVALID_ARG;
    if (ws_bytes < w.total) return UA_ERR_WORKSPACE;
    const size_t n = (size_t)s->B * s->Hkv * w.nkt;
    std::vector<int> last(n);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(last.data(), static_cast<const uint8_t*>(ws) + w.slast, n * sizeof(int),
                                    cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return UA_ERR_CUDA;
    unsigned long long sum = 0;
    for (size_t i = 0; i < n; ++i) {
        // the bound the kernels use: at least the diagonal block, at most the last step
        const int kt = (int)(i % w.nkt);
        const int sd = std::min(4 * kt + 3, w.nst - 1);
        const int sl = std::max(std::min(last[i], w.nst - 1), sd);
        sum += (unsigned long long)(sl - 4 * kt + 1);
    }
    *walked = sum;
    return UA_OK;
}

ua_status ua_prefill_fixed_rows(const ua_shape* s, const void* ws, size_t ws_bytes, unsigned long long* rows,
                                void* stream) {
    if (!s || !rows) return UA_ERR_INVALID_ARG;
    if (s->B <= 0 || s->T <= 0 || s->Hkv <= 0 || s->H <= 0) return UA_ERR_INVALID_ARG;
    *rows = 0;
    if (!use_tc(s)) return UA_OK;
    const TcWs w = tc_ws_layout(s);
    if (!ws) return UA_ERR_INVALID_ARG;
    if (ws_bytes < w.total) return UA_ERR_WORKSPACE;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    unsigned host = 0;
    const size_t off = w.flags + w.fix_count_word * sizeof(unsigned);
    cudaError_t e = cudaMemcpyAsync(&host, static_cast<const uint8_t*>(ws) + off, sizeof(unsigned),
                                    cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return UA_ERR_CUDA;
    *rows = host;
    return UA_OK;
}

ua_status ua_set_wait_limit_ns(unsigned long long ns) {
    // synchronous copy to the current device's symbol: every later launch sees the new limit
    if (cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns)) != cudaSuccess) return UA_ERR_CUDA;
    return UA_OK;
}

ua_status ua_get_device_status(void* stream, int* code) {
    if (!code) return UA_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    int host = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&host, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    const int zero = 0;
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return UA_ERR_CUDA;
    *code = host;
    return UA_OK;
}

}  // extern "C"
