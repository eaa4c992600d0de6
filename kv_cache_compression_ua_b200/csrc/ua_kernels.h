// ua_kernels.h -- internal launch interface between ua_api.cu and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "ua_common.cuh"

namespace ua {

// Launch with programmatic stream serialisation: the kernel may be scheduled before the
// previous kernel on the stream has finished; it must call grid_dep_wait() before touching
// global memory (see ua_common.cuh).
template <typename... Args, typename... Act>
cudaError_t launch_dependent(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Act&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

// Token preparation: normalised keys, RoPE'd queries/keys, per-token rates.
struct PrepParams {
    int B, T, H, Hkv, d;
    double theta;
    const void* q;      // [B,T,H,d] act
    const void* k;      // [B,T,Hkv,d] act
    const float* a_q;   // [B,T,Hkv]
    const float* a_k;   // [B,T,Hkv]
    void* qr;           // [B,H,T,d] work type: RoPE(q)
    void* kh;           // [B,Hkv,T,d] work type: khat
    void* kr;           // [B,Hkv,T,d] work type: RoPE(khat)
    float* rq;          // [B,Hkv,T] softplus(a_q), or NULL
    float* rk;          // [B,Hkv,T] softplus(a_k), or NULL
    // tensor-core path extras (NULL when unused); rows padded to Tp
    int Tp;
    float mq_scale;     // scale * log2(e)
    float* lq2;         // [B*Hkv][Tp] log2(softplus(a_q)) / 3
    float* lk2;         // [B*Hkv][Tp] log2(softplus(a_k)) / 3
    float* mq;          // [B*H][Tp]  scale * ||q|| * log2(e): bound of every logit of the row
    RopeFreq rf;
    int variant;        // UA_VAR_* bits: query norm; rq / rk = 1 for a switched-off mechanism
};

// Boundary pass: per-query-tile column prefixes of the decay and the final biases.
struct BoundaryParams {
    int B, T, Hkv, d;
    int bq;             // query tile height the prefixes are cut at
    int nqt;            // ceil(T / bq)
    const float* kh;    // [B,Hkv,T,d] f32
    const float* rq;    // [B,Hkv,T]
    const float* rk;    // [B,Hkv,T]
    const float* alpha; // [Hkv]
    const float* beta;  // [Hkv]
    float* pb;          // [B,Hkv,nqt,T]: sum_{j < l < t*bq} D[l,j]  (>= 0)
    float* bfinal;      // [B,Hkv,T] = -sum_{l > j} D[l,j], or NULL
    int variant;        // UA_VAR_* bits (decay_var)
};

// Fused biased attention (SIMT path).
struct FwdParams {
    int B, T, H, Hkv, d, G, nqt;
    float scale;
    const float* qr;    // [B,H,T,d]
    const float* kh;    // [B,Hkv,T,d]
    const float* kr;    // [B,Hkv,T,d]
    const void* v;      // [B,T,Hkv,d] act
    const void* g;      // [B,T,H,d] act
    const float* rq;
    const float* rk;
    const float* alpha;
    const float* beta;
    const float* pb;    // [B,Hkv,nqt,T] with bq = 64
    const float* qmax;  // [B,Hkv,nqt] largest scale*||q_i|| of each query tile and group, or NULL
    void* o;            // [B,T,H,d] act
    float* lse;         // [B,H,T] or NULL
    float* lambda_dbg;  // [B,Hkv,T,T] or NULL (pre-zeroed)
    int variant;        // UA_VAR_* bits (decay_var)
    float prune_thr;    // chunked pruned prefill: a key whose Pb at its chunk boundary exceeds
                        // this (-log p) is evicted; +inf = dense
};

// A 64-row query tile and a key tile of the SIMT paths contribute exactly nothing (every
// probability underflows to 0 in fp32, expf below -103.98) when min_j Pb[j] exceeds
// 2 * max_i scale*||q_i|| by this much: the logit of (i, j) is at most scale*||q_i|| - Pb[j]
// and row i's normaliser at least its diagonal logit, -scale*||q_i||.
constexpr float kSimtSkipMargin = 105.f;

// qmax[unit][t] = max over the 64 rows of query tile t and the G heads of the group of mq.
struct TileQmaxParams {
    int B, T, H, Hkv, nqt;
    const float* mq;    // [B,H,T] scale*||q_i||
    float* qmax;        // [B,Hkv,nqt]
};
cudaError_t launch_tile_qmax(const TileQmaxParams& p, cudaStream_t s);

struct CacheView {
    int B, Hkv, d, cap;
    int rep;             // cache heads per KV head of the step's / prefill's k and v (>= 1)
    void* khat;          // pair-interleaved unit keys (see il_index)
    void* v;
    float* bias;
    float* rk;
    int32_t* pos;
    int32_t* n_kept;
    // paged storage (pt == nullptr: cache u's slot s is at u * cap + s)
    const int32_t* pt;   // [B*Hkv][max_pages] page ids
    int ps_shift;        // log2(page size)
    int max_pages, pool_pages;
};

// Physical slot (row of khat and v, index of bias, rk and pos) of slot s of cache u.  A page id
// outside the pool gives -1: RAISE records UA_ERR_INVALID_ARG (a slot the call must touch), else
// the caller only skips the access (a speculative read).
template <bool RAISE = true>
__device__ __forceinline__ long long phys_slot(const CacheView& c, int u, int s) {
    if (c.pt == nullptr) return (long long)u * c.cap + s;
    const int pg = __ldg(c.pt + (size_t)u * c.max_pages + (s >> c.ps_shift));
    if ((unsigned)pg >= (unsigned)c.pool_pages) {
        if (RAISE) raise_status(UA_ERR_INVALID_ARG);
        return -1;
    }
    return ((long long)pg << c.ps_shift) | (long long)(s & ((1 << c.ps_shift) - 1));
}

struct FillParams {
    CacheView c;
    int T;
    double theta;
    RopeFreq rf;
    const void* k;       // [B,T,Hkv,d] act
    const void* v;       // [B,T,Hkv,d] act
    const float* a_k;    // [B,T,Hkv]
    const float* bfinal; // [B,Hkv,T]
};

struct CompactParams {
    CacheView c;
    const uint8_t* keep; // [B,Hkv,cap] or NULL
    float logp;
    int32_t* kept_idx;   // or NULL
};

struct DecodeParams {
    CacheView c;
    int H, G, pos_t;
    float scale, logp;
    double theta;
    RopeFreq rf;
    const void* q;       // [B,H,d] act
    const void* k;       // [B,Hkv,d] act
    const void* v;       // [B,Hkv,d] act
    const void* g;       // [B,H,d] act
    const float* a_q;    // [B,Hkv]
    const float* a_k;    // [B,Hkv]
    const float* alpha;
    const float* beta;
    void* o;             // [B,H,d] act
    uint32_t* evict_bits;
    int32_t* kept_idx;
    int variant;         // UA_VAR_* bits
    int defer;           // 1: no compaction (pairs stay in their slots; append at n_kept)
    // split walk (launch_decode_split): per cache a counter, then per (cache, slice) the partial
    // softmax state [G maxima][G sums][G x d weighted values]
    unsigned* split_cnt;
    float* split_state;
};

// Split decode step: the walk of each cache is cut into slices, one CTA each (up to
// kDecodeSplitMax; the CUDA-core kernel takes up to 16 slices of at least kDecodeSplitSlice pairs,
// the tensor-core one up to 64 of at least kDecodeTcSlice); compaction is deferred.
constexpr int kDecodeSplitMax = 64;
constexpr int kDecodeSplitSimt = 16;
constexpr int kDecodeSplitSlice = 512;
constexpr int kDecodeTcSlice = 256;
cudaError_t launch_decode_split(const DecodeParams& p, bool bf16, cudaStream_t s);
// Exact recomputation of the rows a tensor-core forward listed as out of its shift's range
// (k_fwd_fix.cu).  The forward's workspace operands, its published prefixes and the caller's
// v, g, o, lse.
struct FixParams {
    int B, T, H, Hkv, G, d;
    int QT, nqt, Tp, Tpk;          // query tile rows (128 at d = 64, 64 at d = 128), prefix strides
    float scale;
    const void* qr;                // [B*H][T][d] bf16 RoPE(q)
    const void* kh;                // [B*Hkv][T][d] bf16 khat
    const void* kr;                // [B*Hkv][T][d] bf16 RoPE(khat)
    const float* lq2;              // [B*Hkv][Tp] log2 rates / 3
    const float* lk2;
    float* pincl;                  // [B*Hkv][nqt][Tpk] published inclusive prefixes (made exact here if needed)
    const float* alpha;
    const float* beta;
    const void* v;                 // [B,T,Hkv,d] bf16
    const void* g;                 // [B,T,H,d] bf16
    void* o;                       // [B,T,H,d] bf16
    float* lse;                    // [B,H,T] or NULL
    float prune_thr;               // -log p of the chunked pruning, +inf when dense
    int prefix_exact;              // 1: every decay tile was evaluated (b_final requested)
    const unsigned* fix_count;     // rows listed by the forward
    const int* fix_list;           // (b*H + h)*T + i per listed row
    unsigned* fix_state;           // [B*Hkv] 0 / 1 / 2: prefixes not recomputed / in progress / exact
    float* scratch;                // [grid][T]
};
cudaError_t launch_fwd_fix(const FixParams& p, int grid, cudaStream_t s);
constexpr int kFixGrid = 64;

// The split step of a bf16 cache on the tensor cores (k_decode_tc.cu): same contract and
// workspace as launch_decode_split; group sizes 1-4 and 8.
cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t s);

// Backward (SIMT path).  Inputs from the f32 token preparation and boundary pass (query
// tiles of 64 rows); f32 intermediates in the workspace; outputs in the caller's layouts.
struct BwdParams {
    int B, T, H, Hkv, d, G, nqt, nkt;
    float scale;
    double theta;
    RopeFreq rf;
    const float* qr;     // [B,H,T,d]  RoPE(q)
    const float* kh;     // [B,Hkv,T,d] khat
    const float* kr;     // [B,Hkv,T,d] RoPE(khat)
    const float* qmax;   // [B,Hkv,nqt] tile row bounds (see TileQmaxParams), or NULL
    const float* rq;     // [B,Hkv,T]
    const float* rk;     // [B,Hkv,T]
    const float* pb;     // [B,Hkv,nqt,T] decay prefixes
    const void* k;       // [B,T,Hkv,d] act (raw keys, for the normalisation Jacobian)
    const void* v;
    const void* g;
    const void* o;
    const void* d_o;
    const float* a_q;
    const float* a_k;
    const float* alpha;
    const float* beta;
    const float* lse;    // [B,H,T]
    float* delta;        // [B,H,T]
    float* dpb;          // [B,Hkv,nqt,T] suffix sums of dLambda per query tile
    float* dqr;          // [B,H,T,d]
    float* dkh;          // [B,Hkv,T,d] key-side similarity gradient
    float* dkh_rows;     // [B,Hkv,T,d] row-side similarity gradient
    float* dkr;          // [B,Hkv,T,d]
    float* dv32;         // [B,Hkv,T,d]
    float* daq32;        // [B,Hkv,T]
    float* dak32;        // [B,Hkv,T]
    float* dab;          // [B*Hkv*nkt][2]
    void* dq; void* dk; void* dv; void* dg;
    float* da_q; float* da_k; float* dalpha; float* dbeta;
    const void* q;       // [B,T,H,d] act (raw queries, for the query-norm Jacobian)
    int variant;         // UA_VAR_* bits
};

struct FwdTcLaunch {
    int B, T, Tp, H, Hkv, nqt;
    int Tpk;             // row stride of pincl (head_dim 128: T rounded up to 128)
    float scale;
    const void* kh;      // [B*Hkv][T][64] bf16 khat
    const void* kr;      // [B*Hkv][T][64] bf16 RoPE(khat)
    const void* qr;      // [B*H][T][64] bf16 RoPE(q)
    const void* v;       // [B,T,Hkv,64] bf16 (caller's layout)
    const float* lq2;
    const float* lk2;
    const float* mq;
    float* pincl;        // [B*Hkv][nqt][Tp]: per query tile, the inclusive column prefix it publishes
    unsigned* flags;     // [B*Hkv][nqt][nqt] publication counters, then one ticket counter (zeroed here)
    const float* alpha;
    const float* beta;
    const void* g;
    void* o;
    float* lse;
    float* b_final;      // [B*Hkv][T] or NULL
    float prune_thr;     // chunked pruned prefill (chunks = the 128-row query tiles): -log p, +inf = dense
    unsigned* fix_count; // rows out of the softmax shift's range, listed for k_fwd_fix
    int* fix_list;
};

// Backward on the tensor cores (bf16, head_dim 64 or 128, H/Hkv <= 4, the three-rate method or
// the query norm).  Rows are cut into 32-row steps, keys into 128-key tiles; nst = 4 * nkt steps
// (the last ones may lie past T and are then all zero).
struct BwdTcParams {
    int B, T, Tp, Tpk, H, Hkv, d, G, nkt, nst;
    float scale;
    RopeFreq rf;
    int variant;          // UA_VAR_QUERY_NORM or 0
    // token preparation of the tensor-core forward (bf16 copies, log2 rates / 3)
    const void* qr;       // [B*H][T][d] RoPE(q)
    const void* kh;       // [B*Hkv][T][d] khat (bf16)
    const void* kr;       // [B*Hkv][T][d] RoPE(khat)
    const float* lq2;     // [B*Hkv][Tp]
    const float* lk2;     // [B*Hkv][Tp]
    const float* mq;      // [B*H][Tp] scale * log2(e) * |qrot| (fp32, after the query norm)
    // the caller's tensors
    const void* q; const void* k; const void* v; const void* g; const void* o; const void* d_o;
    const float* a_q; const float* a_k; const float* alpha; const float* beta; const float* lse;
    // workspace
    void* ad;             // [B*H][T][d] bf16: dA = dO * sigmoid(g)
    float* lse2;          // [B*H][Tp] lse * log2(e)
    float* delta;         // [B*H][Tp] sum_c dO * O
    float* pb;            // [B*Hkv][nst][Tpk] decay prefix above each step
    void* tiles;          // [B*Hkv][G+1][ntiles][8 KB]: dZ^T of each head, then dX^T (bf16)
    size_t ntiles;        // 32-row x 128-key tiles of the causal band: 2 * nkt * (nkt + 1)
    float* daq_part;      // [B*Hkv][Tpk][nkt][4] row sums of w over each quarter of each key tile
    float* cmax;          // [B*Hkv][Tpk] per row: max over the group's heads of s|qrot|(1 + 2^-6) - lse (nats)
    int* slast;           // [B*Hkv][nkt] last 32-row step of each key tile with a possibly nonzero probability
    float* dab;           // [B*Hkv*nkt][2] dalpha / dbeta partials
    float* dv32;          // [B*Hkv][T][d]
    float* dkr;           // [B*Hkv][T][d] scale * dkrot
    float* dkh_keys;      // [B*Hkv][T][d] key-side similarity gradient (alpha applied)
    float* dkh_rows;      // [B*Hkv][T][d] row-side similarity gradient (alpha applied)
    float* dqr;           // [B*H][T][d] scale * dqrot
    float* dak32;         // [B*Hkv][T]
    // outputs
    void* dq; void* dk; void* dv; void* dg;
    float* da_q; float* da_k; float* dalpha; float* dbeta;
};
bool bwd_tc_supported(int d, int G);
cudaError_t launch_bwd_tc(const BwdTcParams& p, cudaStream_t s);
// reduction of the per-CTA dalpha / dbeta partials (k_backward_simt.cu)
__global__ void k_bwd_dab(const float* dab, int B, int Hkv, int nkt, float* dalpha, float* dbeta);

// per-query-head decay: repeat K / V for the G query heads of each group; sum gradients back
cudaError_t launch_repeat_kv(const void* in, void* out, int B, int T, int H, int G, int d, bool bf16, cudaStream_t s);
cudaError_t launch_sum_copies(const void* in, void* out, int B, int T, int Hkv, int G, int d, bool bf16,
                              cudaStream_t s);

bool fwd_tc_supported(int d, int G);
cudaError_t launch_fwd_tc(const FwdTcLaunch& L, cudaStream_t s);
// head_dim 128: 64-row query tiles (nqt = ceil(T/64)), flags [B*Hkv][nqt][ceil(T/128)] + 4,
// pincl [B*Hkv][nqt][Tpk]
cudaError_t launch_fwd_tc128(const FwdTcLaunch& L, cudaStream_t s);

cudaError_t launch_prep(const PrepParams& p, bool bf16_in, bool bf16_work, cudaStream_t s);
cudaError_t launch_boundary_simt(const BoundaryParams& p, cudaStream_t s);
cudaError_t launch_fwd_simt(const FwdParams& p, bool bf16_act, cudaStream_t s);
cudaError_t launch_cache_fill(const FillParams& p, bool bf16, cudaStream_t s);
cudaError_t launch_cache_compact(const CompactParams& p, bool bf16, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams& p, bool bf16, cudaStream_t s);
cudaError_t launch_bwd_simt(const BwdParams& p, bool bf16_act, cudaStream_t s);

}  // namespace ua
