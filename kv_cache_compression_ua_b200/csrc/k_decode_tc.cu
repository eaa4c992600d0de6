// k_decode_tc.cu -- the split decode step of a bf16 cache on the tensor cores.
//
// One decode step per (batch, KV head) cache (paperlayer.ai summary §4.2: every live pair j
// takes the new row's decay, b_j -= D[t, j], is evicted once b_j < log p, and the query heads
// attend over the survivors with the bias added to their logits; ai4snews synopsis, eviction
// paragraph).  The pages name fused kernels for the pruned cache as missing (summary §6,
// App. H); this is the long-cache one.  A cache walked entry by entry on the CUDA cores spends
// ~140 warp instructions per entry (one similarity and G logit dot products spread over lanes
// with shuffle reductions, G online-softmax updates), several times its memory time, so here a
// 128-entry tile is one thread per entry plus two small tcgen05 products:
//
//   thread j:  x_j = <khat_t, khat_j> (fp32, from the bf16 entry in shared memory), and the
//              entry rotated in place to RoPE(khat_j, pos_j) (the cache keeps no rotated copy:
//              unit keys are stored pair-interleaved, so a 16-byte chunk holds whole pairs)
//   S   = RoPE(khat) . [q_h high parts | q_h residuals]^T        (M = 128 entries, N = 16)
//   thread j:  decay D, bias update, eviction bit, probabilities P_hj (bf16) from x_j and S
//   O^T += V^T . P                                                (M = head dims, N = 16)
//
// Each query enters as a bf16 high part and its bf16 residual, so the logits carry the query
// to ~16 bits (the cache itself is bf16).  Softmax shift: probabilities are exp(logit - shift_h),
// one shift per head, started at the new token's own logit (a lower bound of the row maximum)
// and raised, with the accumulated values rescaled in TMEM, whenever a tile's maximum exceeds it
// by more than 16; so no probability exceeds e^16 and none that matters underflows.
//
// Work split: grid (slices, B*Hkv), two or four 128-thread CTAs per SM.  Cache (b, h)
// with n live slots is cut into slices of whole 128-entry tiles; each CTA with a slice leaves a
// partial softmax state (shift, sum, weighted values) in the workspace, and the CTA that arrives
// last (a counter per cache that every CTA of the grid increments, a fence before every
// arrival) merges them with the new token, gates, writes o and appends the token.  A CTA without
// a slice arrives at once and only builds the new token if it turns out to be last.  Counting
// every CTA means the merge (which changes n) happens only after all of them have read n.
// Compaction is deferred (pairs keep their slots; ua_cache_compact removes the evicted ones).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "tc_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

using namespace tc;

namespace {

constexpr int kDecTile = 128;
constexpr float kLog2eDec = 1.4426950408889634f;
constexpr float kRescaleGap = 16.f;     // raise the shift when a logit exceeds it by more than this

template <int DH, int G>
struct DecTc {
    static constexpr int NB = DH / 64;                       // 64-column (128-byte) boxes per row
    static constexpr int CTAS = DH == 64 ? 4 : 2;            // CTAs per SM the footprint allows
    static constexpr int COL_S = 0, COL_O = 16, TMEM_COLS = 32;
    static constexpr int SS = G * (DH + 2);                  // floats of one partial state
};

template <int DH, int G>
struct DecTcSmem {
    using C = DecTc<DH, G>;
    // per stage: NB boxes of v then NB boxes of khat (rotated in place), each [128 entries][64]
    // bf16 with the 128-byte swizzle.  The second product's M = 128 rows are the head dims in
    // 64-row atoms one box apart; when DH = 64 its upper atom reads the stage's khat box, whose
    // rows of the result are never read.
    alignas(1024) uint8_t stage[1][2 * C::NB][16384];
    alignas(1024) uint8_t bq[16 * DH * 2];                   // no-swizzle K-major B of S
    alignas(128) uint8_t pt[2][kDecTile][16];                // P: MN-major no-swizzle, heads 0-7 | 8-15
    double gtf[DH / 2];                                       // RoPE frequencies / (2 pi)
    alignas(16) float ff[DH / 2];                            // RoPE frequencies (fp32)
    float bcs[2][DH / 2][2];                                 // per tile parity: cos, sin of pos_base * f_m
    int wd[2][4];                                            // per tile parity and warp: pos_j - j, or a
                                                             // sentinel when the warp's positions are not contiguous
    alignas(16) float kt[DH];                                // khat_t, pair-interleaved
    float ktr[DH];                                           // RoPE(khat_t, pos_t), pair-interleaved
    float vt[DH];
    float q[G][DH];                                          // RoPE(q_h, pos_t), pair-interleaved
    float own[G];                                            // the new token's own logits
    float qn[G];
    float shift[G];
    float red[G][4];
    float red2[4];
    unsigned tflag[2];                                       // per tile parity: bit 0 abort, bit 1 raise the shift
    int scp[2][kDecTile];                                    // per tile parity: pos, bias, r_k of the entries
    float scb[2][kDecTile];
    float scr[2][kDecTile];
    uint64_t full_k, full_v;                                 // khat and v of the tile landed
    uint64_t sfull, pfree;
    uint32_t tmem_base;
    int abort;
    int last;
};

// The new token's inputs, loaded into registers at the kernel's start (the loads go out before
// anything waits): element tid of k_t and v_t, the two components of this thread's query pairs
// (item e = tid + 128 r is pair m = e % (DH/2) of head e / (DH/2)), and the rates.
template <int DH, int G>
struct TokIn {
    static constexpr int QI = (G * (DH / 2) + 127) / 128;
    float kx, vx;
    float qa[QI], qb[QI];
    float aq, ak, al, be;
};

template <int DH, int G>
__device__ __forceinline__ void load_token(TokIn<DH, G>& t, const DecodeParams& p, int unit, int b, int kvh) {
    constexpr int half = DH / 2;
    const int tid = threadIdx.x;
    const size_t tok = (size_t)b * (p.c.Hkv / p.c.rep) + kvh / p.c.rep;   // head kvh / rep of the step's k, v
    const __nv_bfloat16* kin = static_cast<const __nv_bfloat16*>(p.k) + tok * DH;
    const __nv_bfloat16* vin = static_cast<const __nv_bfloat16*>(p.v) + tok * DH;
    const __nv_bfloat16* qin = static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
    t.kx = t.vx = 0.f;
    if (tid < DH) {
        t.kx = __bfloat162float(kin[tid]);
        t.vx = __bfloat162float(vin[tid]);
    }
#pragma unroll
    for (int r = 0; r < TokIn<DH, G>::QI; ++r) {
        const int e = tid + 128 * r;
        t.qa[r] = t.qb[r] = 0.f;
        if (e < G * half) {
            const int h = e / half, m = e % half;
            t.qa[r] = __bfloat162float(qin[h * DH + m]);
            t.qb[r] = __bfloat162float(qin[h * DH + m + half]);
        }
    }
    t.aq = p.a_q[unit];
    t.ak = p.a_k[unit];
    t.al = p.alpha[kvh];
    t.be = p.beta[kvh];
}

// New token of the cache: khat_t, RoPE(khat_t), v_t, RoPE(q_h) (query norm applied) and the own
// logits, into shared memory, from the preloaded inputs.  All 128 threads; ends with a barrier.
template <int DH, int G>
__device__ void new_token(DecTcSmem<DH, G>& S, const DecodeParams& p, const TokIn<DH, G>& tk) {
    constexpr int half = DH / 2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < DH) S.vt[tid] = tk.vx;
    float ss = tk.kx * tk.kx;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) S.red2[warp] = ss;
    // the RoPE frequencies, a quarter per warp (a kernel-parameter array read at a different
    // index by each lane serialises those reads)
    static_assert(half % 4 == 0, "frequencies split over the four warps");
    if (lane < half / 4) {
        const int m = warp * (half / 4) + lane;
        const double f = p.rf.f[m];
        S.gtf[m] = f * 0.15915494309189535;
        S.ff[m] = (float)f;
    }
    __syncthreads();
    const float den = fmaxf(sqrtf(S.red2[0] + S.red2[1] + S.red2[2] + S.red2[3]), 1e-12f);
    if (tid < DH) S.kt[il_index(tid, half)] = tk.kx / den;
    __syncthreads();
    const double pt = (double)p.pos_t;
#pragma unroll
    for (int r = 0; r < TokIn<DH, G>::QI; ++r) {
        const int e = tid + 128 * r;
        if (e < G * half) {
            const int h = e / half, m = e % half;
            float cs, sn;
            rope_cs_turns(pt, S.gtf[m], &cs, &sn);
            S.q[h][2 * m] = tk.qa[r] * cs - tk.qb[r] * sn;
            S.q[h][2 * m + 1] = tk.qb[r] * cs + tk.qa[r] * sn;
        }
    }
    for (int m = tid; m < half; m += blockDim.x) {
        float cs, sn;
        rope_cs_turns(pt, S.gtf[m], &cs, &sn);
        const float x0 = S.kt[2 * m], x1 = S.kt[2 * m + 1];
        S.ktr[2 * m] = x0 * cs - x1 * sn;
        S.ktr[2 * m + 1] = x1 * cs + x0 * sn;
    }
    __syncthreads();
    if (p.variant & kVarQNorm) {                     // query RMS norm (RoPE keeps the norm)
        for (int h = warp; h < G; h += 4) {
            float qq = 0.f;
            for (int x = lane; x < DH; x += 32) qq = fmaf(S.q[h][x], S.q[h][x], qq);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) qq += __shfl_xor_sync(0xffffffffu, qq, o);
            if (lane == 0) S.qn[h] = 1.f / sqrtf(qq * (1.f / DH) + kQNormEps);
        }
        __syncthreads();
        for (int e = tid; e < G * DH; e += blockDim.x) S.q[e / DH][e % DH] *= S.qn[e / DH];
        __syncthreads();
    }
    for (int h = warp; h < G; h += 4) {              // the new token's own logits (its bias is 0)
        float a = 0.f;
        for (int x = lane; x < DH; x += 32) a = fmaf(S.q[h][x], S.ktr[x], a);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) S.own[h] = a * p.scale;
    }
    __syncthreads();
}

// The last CTA of a cache: merge the partial states of the nsl slices that walked pairs with the
// new token, gate, write o, clear the eviction words past the live pairs and append the token.
// One round of loads brings every slice's shift and sum (and the gate); a warp per head forms
// the common shift, the weights and the normaliser; the weighted values are then read once.
template <int DH, int G>
__device__ void merge_append(DecTcSmem<DH, G>& S, const DecodeParams& p, const TokIn<DH, G>& tk, int unit, int b,
                             int kvh, int n, int nsl) {
    using C = DecTc<DH, G>;
    constexpr int GE = (G * DH + 127) / 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const CacheView& c = p.c;
    const int words = (c.cap + 31) / 32;
    const size_t base = (size_t)unit * c.cap;
    const __nv_bfloat16* gin = static_cast<const __nv_bfloat16*>(p.g) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
    __nv_bfloat16* oout = static_cast<__nv_bfloat16*>(p.o) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
    const float* st0 = p.split_state + (size_t)unit * kDecodeSplitMax * C::SS;
    float* s_ml = reinterpret_cast<float*>(S.stage[0][0]);         // [nsl][2G]: shifts, sums
    float* s_w = s_ml + kDecodeSplitMax * 2 * G;                     // [nsl][G] merge weights
    float* s_wt = s_w + kDecodeSplitMax * G;                         // [G] weight of the new token
    float* s_inv = s_wt + G;                                         // [G] 1 / normaliser
    for (int e = tid; e < nsl * 2 * G; e += blockDim.x)
        s_ml[e] = __ldcg(st0 + (size_t)(e / (2 * G)) * C::SS + e % (2 * G));
    float gv[GE];
#pragma unroll
    for (int r = 0; r < GE; ++r) {
        const int e = tid + 128 * r;
        gv[r] = e < G * DH ? __bfloat162float(gin[e]) : 0.f;
    }
    __syncthreads();
    for (int h = warp; h < G; h += 4) {
        float mq[2], lq[2];
        float M = S.own[h];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int q = lane + 32 * i;
            lq[i] = q < nsl ? s_ml[q * 2 * G + G + h] : 0.f;
            mq[i] = lq[i] > 0.f ? s_ml[q * 2 * G + h] : -INFINITY;
            M = fmaxf(M, mq[i]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int q = lane + 32 * i;
            const float w = lq[i] > 0.f ? expf(mq[i] - M) : 0.f;
            if (q < nsl) s_w[q * G + h] = w;
            L = fmaf(lq[i], w, L);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) {
            const float wt = expf(S.own[h] - M);
            s_wt[h] = wt;
            s_inv[h] = 1.f / (L + wt);
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < GE; ++r) {
        const int e = tid + 128 * r;
        if (e >= G * DH) break;
        const int h = e / DH, x = e % DH;
        float A0 = s_wt[h] * S.vt[x], A1 = 0.f;
        int q = 0;
        for (; q + 2 <= nsl; q += 2) {
            const float w0 = s_w[q * G + h], w1 = s_w[(q + 1) * G + h];
            if (w0 != 0.f) A0 = fmaf(__ldcg(st0 + (size_t)q * C::SS + 2 * G + e), w0, A0);
            if (w1 != 0.f) A1 = fmaf(__ldcg(st0 + (size_t)(q + 1) * C::SS + 2 * G + e), w1, A1);
        }
        if (q < nsl) {
            const float w0 = s_w[q * G + h];
            if (w0 != 0.f) A0 = fmaf(__ldcg(st0 + (size_t)q * C::SS + 2 * G + e), w0, A0);
        }
        oout[e] = __float2bfloat16_rn((A0 + A1) * s_inv[h] * sigmoid_f(gv[r]));
    }
    if (p.evict_bits)
        for (int w = ((n + 31) >> 5) + tid; w < words; w += blockDim.x) p.evict_bits[(size_t)unit * words + w] = 0u;
    __nv_bfloat16* khat = static_cast<__nv_bfloat16*>(c.khat);
    __nv_bfloat16* vc = static_cast<__nv_bfloat16*>(c.v);
    if (n < c.cap) {
        const long long pa = phys_slot(c, unit, n);
        if (pa >= 0) {
            const size_t e = (size_t)pa * DH;
            for (int x = tid; x < DH; x += blockDim.x) {
                khat[e + x] = __float2bfloat16_rn(S.kt[x]);
                vc[e + x] = __float2bfloat16_rn(S.vt[x]);
            }
            if (tid == 0) {
                c.bias[pa] = 0.f;
                c.rk[pa] = softplus_f(tk.ak);
                c.pos[pa] = p.pos_t;
            }
        }
        if (tid == 0) {
            c.n_kept[unit] = n + 1;
            if (p.kept_idx) p.kept_idx[base + n] = -1;
        }
    } else if (tid == 0) {
        raise_status(UA_ERR_CAPACITY);
    }
    if (tid == 0) p.split_cnt[unit] = 0u;            // back to zero for the next step
}

// Dense tiles: when a tile's positions are contiguous (pos_j = pos_base + (j - first slot), as in a
// cache that has evicted nothing since the slots were written), an entry's rotation angle is
// pos_base*f + tid*f, so the exact reduction (double precision) is needed once per frequency and
// tile, and each thread adds its small offset angle tid*f (|tid*f| < 128, fp32 and the fast
// sine/cosine unit) by the angle-addition formulas.  Each warp records pos_j - j for its entries
// (kNotDense if they disagree); warp 0 forms cos/sin of pos_base*f for the tile.
constexpr int kNotDense = -2147483647;

template <int DH, int G>
__device__ __forceinline__ void tile_density(DecTcSmem<DH, G>& S, int par, int pj, int j, bool valid, int warp,
                                             int lane) {
    const int dj = pj - j;
    const int ref = __shfl_sync(0xffffffffu, dj, 0);             // lane 0 holds the warp's first entry
    const bool same = __all_sync(0xffffffffu, !valid || dj == ref);
    const bool any = __any_sync(0xffffffffu, valid);
    if (lane == 0) S.wd[par][warp] = !any ? ref : (same ? ref : kNotDense);
    if (warp == 0) {                                              // base angles: pos of the first slot
        const double pb = (double)__shfl_sync(0xffffffffu, pj, 0);
        for (int m = lane; m < DH / 2; m += 32) rope_cs_turns(pb, S.gtf[m], &S.bcs[par][m][0], &S.bcs[par][m][1]);
    }
}

template <int DH, int G, bool PAGED>
__global__ void __launch_bounds__(128, DecTc<DH, G>::CTAS)
    k_decode_tc(const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_v, DecodeParams p) {
    using C = DecTc<DH, G>;
    using Sm = DecTcSmem<DH, G>;
    constexpr int NB = C::NB;
    extern __shared__ uint8_t dsm_raw[];
    Sm& S = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const CacheView& c = p.c;
    const int unit = blockIdx.y, sl = blockIdx.x, b = unit / c.Hkv, kvh = unit % c.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int variant = p.variant;
    const size_t base = (size_t)unit * c.cap;
    const int words = (c.cap + 31) / 32;

    grid_dep_wait();
    grid_dep_release();
    TokIn<DH, G> tk;
    load_token<DH, G>(tk, p, unit, b, kvh);
    int n = c.n_kept[unit];
    if (n < 0 || n > c.cap) {                 // corrupt count: never read past the cache
        if (tid == 0 && sl == 0) raise_status(UA_ERR_CAPACITY);
        n = n < 0 ? 0 : c.cap;
    }
    const int nsl = min((int)gridDim.x, max(1, (n + kDecodeTcSlice - 1) / kDecodeTcSlice));
    const int chunk = (((n + nsl - 1) / nsl) + kDecTile - 1) / kDecTile * kDecTile;
    const int lo = sl < nsl ? min(n, sl * chunk) : n;
    const int hi = sl < nsl ? min(n, lo + chunk) : n;
    const int ntiles = (hi - lo + kDecTile - 1) / kDecTile;
    const int nwalk = chunk > 0 ? min(nsl, (n + chunk - 1) / chunk) : 0;   // slices 0 .. nwalk-1 hold pairs

    // Arrival on the cache's counter (zero before the step; the merging CTA zeroes it again):
    // every CTA of the grid counts, so the merge -- which changes n -- comes after all of them
    // have read n.  A count already at the grid's size means the workspace was not zeroed.
    auto arrive = [&]() {
        if (tid == 0) {
            const unsigned old = atomicAdd(p.split_cnt + unit, 1u);
            if (old >= gridDim.x) raise_status(UA_ERR_INVALID_ARG);
            S.last = old == gridDim.x - 1;
        }
        __syncthreads();
    };
    if (ntiles == 0) {
        // nothing to walk (the merge reads only the slices that walked pairs): arrival, and
        // the merge if this CTA is the last one
        arrive();
        if (!S.last) return;
        __threadfence();
        new_token<DH, G>(S, p, tk);
        merge_append<DH, G>(S, p, tk, unit, b, kvh, n, nwalk);
        return;
    }

    if (tid == 0) {
        S.abort = 0;
        mbar_init(&S.full_k, 1);
        mbar_init(&S.full_v, 1);
        mbar_init(&S.sfull, 1);
        mbar_init(&S.pfree, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    const bool leader = tid == 0;
    // One stage.  A tile's keys are reloaded as soon as its first product has read them (mid
    // tile), its values once the second product is done (at the start of the next tile), so both
    // loads overlap the work of a tile instead of following it.
    // a tile's first physical row: a tile lies within one page (pages hold a power of two >= 128
    // slots, tiles start at multiples of 128); a page outside the pool (raised) reads row 0
    auto tile_row = [&](int tt) -> int {
        if constexpr (PAGED) {
            const long long r = phys_slot(c, unit, lo + tt * kDecTile);
            return r >= 0 ? (int)r : 0;
        } else {
            return (int)(base + lo + (size_t)tt * kDecTile);
        }
    };
    auto issue_k = [&](int tt) {
        const int row = tile_row(tt);
        mbar_expect_tx(&S.full_k, NB * 16384);
        for (int bx = 0; bx < NB; ++bx) tma_load_2d(S.stage[0][NB + bx], &tm_kh, &S.full_k, 64 * bx, row);
    };
    auto issue_v = [&](int tt) {
        const int row = tile_row(tt);
        mbar_expect_tx(&S.full_v, NB * 16384);
        for (int bx = 0; bx < NB; ++bx) tma_load_2d(S.stage[0][bx], &tm_v, &S.full_v, 64 * bx, row);
    };
    // a tile's scalars (pos, bias, r_k) go to shared memory by asynchronous copies, a tile ahead;
    // each thread copies and later reads only its own entry's
    auto load_scalars = [&](int tt) {
        const int jj = lo + tt * kDecTile + tid, par = tt & 1;
        if constexpr (PAGED) {
            const long long ps = jj < hi ? phys_slot(c, unit, jj) : -1;
            if (ps >= 0) {
                cp_async4(&S.scp[par][tid], c.pos + ps);
                cp_async4(&S.scb[par][tid], c.bias + ps);
                cp_async4(&S.scr[par][tid], c.rk + ps);
            }
        } else if (jj < hi) {
            cp_async4(&S.scp[par][tid], c.pos + base + jj);
            cp_async4(&S.scb[par][tid], c.bias + base + jj);
            cp_async4(&S.scr[par][tid], c.rk + base + jj);
        }
        cp_async_commit();
    };
    __syncthreads();                                  // barriers initialised
    if (leader) {
        issue_k(0);
        issue_v(0);
    }
    load_scalars(0);
    tc_fence_before();
    new_token<DH, G>(S, p, tk);                       // ends with __syncthreads
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    volatile int* abort = &S.abort;

    // ---- B of S: rows q_h (high parts), then q_h (residuals), then zeros; no swizzle, K-major:
    // element (row r, column k) at (k/8)*128 + (r/8)*(DH*16) + (r%8)*16 + (k%8)*2
    for (int idx = tid; idx < 16 * DH; idx += blockDim.x) {
        const int r = idx / DH, k = idx % DH;
        float x = 0.f;
        if (r < 2 * G) {
            const float v = S.q[r % G][k];
            const float hi_ = __bfloat162float(__float2bfloat16_rn(v));
            x = r < G ? hi_ : v - hi_;
        }
        *reinterpret_cast<__nv_bfloat16*>(S.bq + (k >> 3) * 128 + (r >> 3) * (DH * 16) + (r & 7) * 16 + (k & 7) * 2) =
            __float2bfloat16_rn(x);
    }
    // the second block of P columns (heads 8-15) stays zero when G <= 8
    for (int idx = tid; idx < kDecTile * 4; idx += blockDim.x) reinterpret_cast<uint32_t*>(S.pt[1])[idx] = 0u;
    if (tid < G) S.shift[tid] = S.own[tid];
    if (tid == 0) S.tflag[0] = S.tflag[1] = 0u;
    cp_async_wait_all();
    tile_density<DH, G>(S, 0, S.scp[0][tid], lo + tid, lo + tid < hi, warp, lane);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();

    const float scale = p.scale, logp = p.logp;
    const float rq_t = (variant & kVarNoQ) ? 1.f : softplus_f(tk.aq);
    const float al = tk.al, be = tk.be;
    const uint32_t ID1 = idesc_bf16(128, 16, 0, 0);
    const uint32_t ID2 = idesc_bf16(128, 16, 1, 1);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float lsum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) lsum[h] = 0.f;
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
        const int j = lo + t * kDecTile + tid;
        const bool valid = j < hi;
        const int pj = S.scp[t & 1][tid];
        const float bj = S.scb[t & 1][tid], rkj = S.scr[t & 1][tid];
        if (t + 1 < ntiles) load_scalars(t + 1);
        // values of this tile: the previous tile's second product must be done with the buffer
        if (tid == 96 && t >= 1 && mbar_wait(&S.pfree, (t - 1) & 1, abort)) issue_v(t);
        if (!__all_sync(0xffffffffu, mbar_wait(&S.full_k, t & 1, abort))) ok = false;
        // ---- x_j = <khat_t, khat_j> (four partial sums: short dependency chains), and khat_j
        // rotated in place (16-byte chunks, swizzled)
        float xp[4] = {0.f, 0.f, 0.f, 0.f};
        const int par = t & 1;
        bool dense = true;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int dw = S.wd[par][w];
            dense = dense && (lo + t * kDecTile + w * 32 >= hi || (dw != kNotDense && dw == S.wd[par][0]));
        }
        if (ok && dense) {
            const float tf = (float)tid;
#pragma unroll 1
            for (int bx = 0; bx < NB; ++bx) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint8_t* ptr = S.stage[0][NB + bx] + (uint32_t)tid * 128u + ((uint32_t)(ch ^ (tid & 7)) << 4);
                    float xa[8], xb[8];
                    Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(ptr), xa);
                    const float4 k0 = *reinterpret_cast<const float4*>(&S.kt[bx * 64 + ch * 8]);
                    const float4 k1 = *reinterpret_cast<const float4*>(&S.kt[bx * 64 + ch * 8 + 4]);
                    xp[0] = fmaf(k0.x, xa[0], xp[0]); xp[1] = fmaf(k0.y, xa[1], xp[1]);
                    xp[2] = fmaf(k0.z, xa[2], xp[2]); xp[3] = fmaf(k0.w, xa[3], xp[3]);
                    xp[0] = fmaf(k1.x, xa[4], xp[0]); xp[1] = fmaf(k1.y, xa[5], xp[1]);
                    xp[2] = fmaf(k1.z, xa[6], xp[2]); xp[3] = fmaf(k1.w, xa[7], xp[3]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int m = bx * 32 + ch * 4 + i;
                        float co, so;
                        __sincosf(tf * S.ff[m], &so, &co);
                        const float cb = S.bcs[par][m][0], sb = S.bcs[par][m][1];
                        const float cs = cb * co - sb * so, sn = fmaf(sb, co, cb * so);
                        xb[2 * i] = xa[2 * i] * cs - xa[2 * i + 1] * sn;
                        xb[2 * i + 1] = xa[2 * i + 1] * cs + xa[2 * i] * sn;
                    }
                    Vec16<__nv_bfloat16>::st(reinterpret_cast<__nv_bfloat16*>(ptr), xb);
                }
            }
        } else if (ok) {
            const double pd = (double)pj;
#pragma unroll 1
            for (int bx = 0; bx < NB; ++bx) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint8_t* ptr = S.stage[0][NB + bx] + (uint32_t)tid * 128u + ((uint32_t)(ch ^ (tid & 7)) << 4);
                    float xa[8], xb[8];
                    Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(ptr), xa);
                    const float4 k0 = *reinterpret_cast<const float4*>(&S.kt[bx * 64 + ch * 8]);
                    const float4 k1 = *reinterpret_cast<const float4*>(&S.kt[bx * 64 + ch * 8 + 4]);
                    xp[0] = fmaf(k0.x, xa[0], xp[0]); xp[1] = fmaf(k0.y, xa[1], xp[1]);
                    xp[2] = fmaf(k0.z, xa[2], xp[2]); xp[3] = fmaf(k0.w, xa[3], xp[3]);
                    xp[0] = fmaf(k1.x, xa[4], xp[0]); xp[1] = fmaf(k1.y, xa[5], xp[1]);
                    xp[2] = fmaf(k1.z, xa[6], xp[2]); xp[3] = fmaf(k1.w, xa[7], xp[3]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float cs, sn;
                        rope_cs_turns(pd, S.gtf[bx * 32 + ch * 4 + i], &cs, &sn);
                        xb[2 * i] = xa[2 * i] * cs - xa[2 * i + 1] * sn;
                        xb[2 * i + 1] = xa[2 * i + 1] * cs + xa[2 * i] * sn;
                    }
                    Vec16<__nv_bfloat16>::st(reinterpret_cast<__nv_bfloat16*>(ptr), xb);
                }
            }
        }
        const float x = (xp[0] + xp[1]) + (xp[2] + xp[3]);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (__syncthreads_or(!ok)) { ok = false; break; }
        // ---- S of the tile
        if (leader) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk) {
                const uint64_t a = smem_desc(smem_u32(S.stage[0][NB + (kk >> 2)]) + (uint32_t)(kk & 3) * 32u, 16,
                                             1024, kSwizzle128B);
                const uint64_t bd = smem_desc(smem_u32(S.bq) + (uint32_t)kk * 256u, 128, DH * 16, kSwizzleNone);
                umma_f16(tmem + C::COL_S, a, bd, ID1, kk > 0 ? 1u : 0u);
            }
            umma_commit(&S.sfull);
        }
        // ---- decay, bias update, eviction (while the product runs)
        const float D = decay_var(rq_t, (variant & kVarNoK) ? 1.f : rkj, fmaf(al, x, be), variant);
        const float bnew = bj - D;
        const bool keep = valid && bnew >= logp;
        if (valid) {
            if constexpr (PAGED) {
                const long long ps = phys_slot(c, unit, j);
                if (ps >= 0) c.bias[ps] = bnew;
            } else {
                c.bias[base + j] = bnew;
            }
            if (p.kept_idx) p.kept_idx[base + j] = j;
        }
        const unsigned ev = __ballot_sync(0xffffffffu, valid && !keep);
        const int wj0 = lo + t * kDecTile + warp * 32;
        if (p.evict_bits && lane == 0 && wj0 < hi) p.evict_bits[(size_t)unit * words + (wj0 >> 5)] = ev;
        if (!__all_sync(0xffffffffu, mbar_wait(&S.sfull, t & 1, abort))) ok = false;
        tc_fence_after();
        if (leader && ok && t + 1 < ntiles) issue_k(t + 1);      // the first product has read the keys
        float xs[2 * G <= 8 ? 8 : 16];
        if (2 * G <= 8) tmem_ld8(tmem + lane_base + C::COL_S, xs);
        else tmem_ld16(tmem + lane_base + C::COL_S, xs);
        float lg[G], nsh[G];
        bool over = false;                            // a logit above its head's shift by > kRescaleGap
#pragma unroll
        for (int h = 0; h < G; ++h) {
            lg[h] = keep ? fmaf(scale, xs[h] + xs[G + h], bnew) : -INFINITY;
            nsh[h] = S.shift[h];
            over |= lg[h] > nsh[h] + kRescaleGap;
        }
        // the previous tile's second product must be done before P and O are touched, and before
        // its stage is refilled
        if (t >= 1 && !__all_sync(0xffffffffu, mbar_wait(&S.pfree, (t - 1) & 1, abort))) ok = false;
        {   // one barrier for both votes: bit 0 abort, bit 1 a logit above its shift's headroom
            const unsigned ba = __ballot_sync(0xffffffffu, !ok), bo = __ballot_sync(0xffffffffu, over);
            if (lane == 0 && (ba | bo)) atomicOr(&S.tflag[t & 1], (ba ? 1u : 0u) | (bo ? 2u : 0u));
        }
        __syncthreads();
        const unsigned fl = S.tflag[t & 1];
        if (fl & 1u) { ok = false; break; }
        const bool any = (fl & 2u) != 0;
        if (tid == 0) S.tflag[(t + 1) & 1] = 0u;      // the next tile's word (its writers come after
                                                      // this tile's last barrier)
        // the next tile's contiguity and base angles (read after this tile's last barrier)
        if (t + 1 < ntiles) {
            cp_async_wait_all();
            tile_density<DH, G>(S, (t + 1) & 1, S.scp[(t + 1) & 1][tid], j + kDecTile, j + kDecTile < hi, warp,
                                lane);
        }
        tc_fence_after();
        // ---- shift: raised (and the accumulated values rescaled) when a logit of the tile
        // exceeds it by more than kRescaleGap (rare: the per-head maxima are formed only then)
        float fac[G];
#pragma unroll
        for (int h = 0; h < G; ++h) fac[h] = 1.f;
        if (any) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float m = lg[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0) S.red[h][warp] = m;
            }
            __syncthreads();
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float tm = fmaxf(fmaxf(S.red[h][0], S.red[h][1]), fmaxf(S.red[h][2], S.red[h][3]));
                if (tm > nsh[h] + kRescaleGap) {
                    fac[h] = expf(nsh[h] - tm);
                    nsh[h] = tm;
                }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) lsum[h] *= fac[h];
            if (t >= 1) {                             // O holds earlier tiles: scale its columns
                float o[16];
                tmem_ld16(tmem + lane_base + C::COL_O, o);
#pragma unroll
                for (int h = 0; h < G; ++h) o[h] *= fac[h];
                tmem_st16(tmem + lane_base + C::COL_O, o);
                tmem_wait_st();
            }
        }
        if (!valid) {
            // a ragged last tile: this row of V enters the second product with P = 0; zero it, as
            // slots past the live pairs may hold anything and 0 x NaN would poison O
            if (!mbar_wait(&S.full_v, t & 1, abort)) ok = false;
#pragma unroll
            for (int bx = 0; bx < NB; ++bx)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4*>(S.stage[0][bx] + (uint32_t)tid * 128u + ((uint32_t)ch << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
        }
        // ---- probabilities into P (bf16, heads 0-7 in block 0, 8-15 in block 1)
        float pr[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) pr[h] = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float pe = keep ? ex2f((lg[h] - nsh[h]) * kLog2eDec) : 0.f;
            const float pb = __bfloat162float(__float2bfloat16_rn(pe));
            pr[h] = pb;
            lsum[h] += pb;
        }
        Vec16<__nv_bfloat16>::st(reinterpret_cast<__nv_bfloat16*>(S.pt[0][tid]), pr);
        if (G > 8) Vec16<__nv_bfloat16>::st(reinterpret_cast<__nv_bfloat16*>(S.pt[1][tid]), pr + 8);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();                              // every thread has read the old shifts and red
        if (any && tid < G) S.shift[tid] = nsh[tid];
        // ---- O^T += V^T P
        if (leader) {
            if (!mbar_wait(&S.full_v, t & 1, abort)) ok = false;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kDecTile / 16; ++kk) {
                const uint64_t a = smem_desc(smem_u32(S.stage[0][0]) + (uint32_t)kk * 2048u, 16384, 1024,
                                             kSwizzle128B);
                const uint64_t bd = smem_desc(smem_u32(S.pt[0]) + (uint32_t)kk * 256u, 128, 2048, kSwizzleNone);
                umma_f16(tmem + C::COL_O, a, bd, ID2, (t > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&S.pfree);
        }
    }
    // ---- the slice's partial state
    if (ok && !__all_sync(0xffffffffu, mbar_wait(&S.pfree, (ntiles - 1) & 1, abort))) ok = false;
    ok = !__syncthreads_or(!ok);
    tc_fence_after();
    float* st = p.split_state + ((size_t)unit * kDecodeSplitMax + sl) * C::SS;
    {
        float o[16];
        tmem_ld16(tmem + lane_base + C::COL_O, o);
        const int d = warp * 32 + lane;
        if (d < DH)
#pragma unroll
            for (int h = 0; h < G; ++h) st[2 * G + h * DH + d] = ok ? o[h] : 0.f;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float l = lsum[h];
#pragma unroll
        for (int k = 16; k > 0; k >>= 1) l += __shfl_xor_sync(0xffffffffu, l, k);
        if (lane == 0) S.red[h][warp] = l;
    }
    __syncthreads();
    if (tid < G) {
        st[tid] = S.shift[tid];
        st[G + tid] = ok ? S.red[tid][0] + S.red[tid][1] + S.red[tid][2] + S.red[tid][3] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    if (*abort && tid == 0) drain_pause(10000000ull);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    // ---- arrival; the last CTA of the cache merges
    __threadfence();
    __syncthreads();
    arrive();
    if (!S.last) return;
    __threadfence();
    merge_append<DH, G>(S, p, tk, unit, b, kvh, n, nwalk);
}

template <int DH>
bool map_cache_rows(CUtensorMap* m, const void* base, size_t rows) {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    cuuint64_t dims[2] = {(cuuint64_t)DH, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)DH * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kDecTile};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Slices per cache (the grid's x extent; a cache uses fewer when it is short): the count that
// minimises (waves of resident CTAs) x (a CTA's fixed cost + its tiles), with the tiles taken
// from the capacity and a CTA's fixed cost (new token, setup, arrival) counted as two tiles.
// Few caches get many slices (up to kDecodeSplitMax), hundreds of long ones a handful, sized so
// the last wave is nearly full.
int decode_tc_slices(int units, int cap, int ctas_per_sm) {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            sms = 148;
    }
    const long long slots = (long long)ctas_per_sm * sms;
    const long long tiles = (cap + kDecTile - 1) / kDecTile;
    int best = 1;
    long long best_cost = -1;
    for (int n = 1; n <= kDecodeSplitMax; ++n) {
        const long long waves = ((long long)std::max(1, units) * n + slots - 1) / slots;
        const long long cost = waves * (2 + (tiles + n - 1) / n);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = n;
        }
    }
    return best;
}

template <int DH, int G>
cudaError_t decode_tc_inst(const DecodeParams& p, cudaStream_t s) {
    const size_t rows = p.c.pt ? (size_t)p.c.pool_pages << p.c.ps_shift : (size_t)p.c.B * p.c.Hkv * p.c.cap;
    CUtensorMap mk, mv;
    if (!map_cache_rows<DH>(&mk, p.c.khat, rows) || !map_cache_rows<DH>(&mv, p.c.v, rows))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(DecTcSmem<DH, G>) + 1024;
    auto kern = p.c.pt != nullptr ? k_decode_tc<DH, G, true> : k_decode_tc<DH, G, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    UA_PROFILE("k_decode_tc", s);
    const int units = p.c.B * p.c.Hkv;
    return launch_dependent(kern, dim3(decode_tc_slices(units, p.c.cap, DecTc<DH, G>::CTAS), units),
                            dim3(128), smem, s, mk, mv, p);
}

template <int DH>
cudaError_t decode_tc_g(const DecodeParams& p, cudaStream_t s) {
    switch (p.G) {
        case 1: return decode_tc_inst<DH, 1>(p, s);
        case 2: return decode_tc_inst<DH, 2>(p, s);
        case 3: return decode_tc_inst<DH, 3>(p, s);
        case 4: return decode_tc_inst<DH, 4>(p, s);
        case 8: return decode_tc_inst<DH, 8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

// Footprints: DH = 64 four CTAs per SM, DH = 128 two (227 KB of shared memory per SM); the merge
// reuses the first stage for 3 x kDecodeSplitMax x G + 2 G floats.
static_assert(4 * (sizeof(DecTcSmem<64, 8>) + 1024) <= 232448, "decode tiles: four CTAs per SM at d = 64");
static_assert(2 * (sizeof(DecTcSmem<128, 8>) + 1024) <= 232448, "decode tiles: two CTAs per SM at d = 128");
static_assert((3 * kDecodeSplitMax * 8 + 2 * 8) * 4 <= 16384, "the merge's scratch fits the first stage box");

}  // namespace

cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t s) {
    return p.c.d == 64 ? decode_tc_g<64>(p, s) : decode_tc_g<128>(p, s);
}

}  // namespace ua
