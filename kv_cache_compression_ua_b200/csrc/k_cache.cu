// k_cache.cu -- the self-pruning KV cache: fill from a prefill, stable compaction, and the
// fused decode step (bias update, eviction, attention, compaction, append) in one pass.
//
// The pages keep a scalar bias per cached key/value pair that the learned decay lowers at
// every step, and evict a pair once exp(b_j) < p; b_j only decreases, so evicted pairs never
// come back, and each head keeps its own, input-dependent number of pairs (paperlayer.ai
// summary §4.2; ai4snews synopsis, eviction paragraph).  The pages report that their own
// implementation lacked a fused dynamic cache manager and name specialised kernels for the
// pruned cache as future work (paperlayer.ai summary §6, App. H) -- this file is that part.
//
// Layout: one structure-of-arrays cache per (batch, KV head), slots in ascending token
// order.  An entry is read by a group of LPE lanes, each moving 16 bytes of khat and v
// (128-bit coalesced loads); dot products reduce across the group with shuffles.  The cache
// holds no rotated copy of the keys: khat is stored pair-interleaved (il_index), so each lane
// holds whole RoPE pairs and rotates them by its entry's position while the next pass loads
// (268 bytes per bf16 entry at d = 64 instead of 396).
#include <algorithm>

#include "ua_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

template <typename TC, int DH>
struct EntryLayout {
    static constexpr int VEC = Vec16<TC>::N;   // elements per 16-byte vector
    static constexpr int LPE = DH / VEC;       // lanes per entry
    static constexpr int EPW = 32 / LPE;       // entries per warp
    static constexpr int NW = 8;               // warps per block
    static constexpr int EPB = EPW * NW;       // entries per block pass
};

template <int LPE>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int o = LPE / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// RoPE of a cached key's VEC/2 pairs (pair-interleaved khat) at its position pos, the lane's
// frequencies given in turns (gt = f / (2 pi)).
template <int VEC>
__device__ __forceinline__ void rotate_pairs(const float (&xa)[VEC], float (&xb)[VEC], double pos,
                                             const double (&gt)[VEC / 2]) {
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) {
        float cs, sn;
        rope_cs_turns(pos, gt[i], &cs, &sn);
        xb[2 * i] = xa[2 * i] * cs - xa[2 * i + 1] * sn;
        xb[2 * i + 1] = xa[2 * i + 1] * cs + xa[2 * i] * sn;
    }
}

// Block-wide stable compaction bookkeeping for one pass: returns the destination of this
// lane's entry (valid only when keep) and the number of survivors in the pass.
template <int LPE, int NW>
__device__ __forceinline__ int pass_scan(bool keep, int warp, int lane, int* s_wcnt, int* total) {
    const int grp_lane0 = (lane / LPE) * LPE;
    const unsigned bal = __ballot_sync(0xffffffffu, keep && (lane % LPE) == 0);
    const int wpre = __popc(bal & ((1u << grp_lane0) - 1u));
    if (lane == 0) s_wcnt[warp] = __popc(bal);
    __syncthreads();
    int bpre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int c = s_wcnt[w];
        bpre += (w < warp) ? c : 0;
        tot += c;
    }
    *total = tot;
    return bpre + wpre;
}

// ------------------------------------------------------------------ fill from a prefill
// grid (T, B), 256 threads; warp per KV head.
template <typename TC, int DH>
__global__ void __launch_bounds__(256) k_cache_fill(FillParams p) {
    const int t = blockIdx.x, b = blockIdx.y, T = p.T;
    const CacheView& c = p.c;
    constexpr int half = DH / 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TC* kin = static_cast<const TC*>(p.k);
    const TC* vin = static_cast<const TC*>(p.v);
    for (int h = warp; h < c.Hkv; h += 8) {
        const size_t src = (((size_t)b * T + t) * (c.Hkv / c.rep) + h / c.rep) * DH;
        const long long ps = phys_slot(c, b * c.Hkv + h, t);    // uniform over the warp
        if (ps < 0) {
            if (lane == 0 && t == 0) c.n_kept[(size_t)b * c.Hkv + h] = T;
            continue;
        }
        const size_t slot = (size_t)ps;
        float x0[2] = {0.f, 0.f}, x1[2] = {0.f, 0.f};
        float ss = 0.f;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int m = lane + 32 * r;
            if (m < half) {
                x0[r] = Elem<TC>::ld(kin + src + m);
                x1[r] = Elem<TC>::ld(kin + src + m + half);
                ss += x0[r] * x0[r] + x1[r] * x1[r];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float den = fmaxf(sqrtf(ss), 1e-12f);
        TC* kh = static_cast<TC*>(c.khat) + slot * DH;
        TC* vv = static_cast<TC*>(c.v) + slot * DH;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int m = lane + 32 * r;
            if (m < half) {                               // the pair (m, m + half), interleaved
                Elem<TC>::st(kh + 2 * m, x0[r] / den);
                Elem<TC>::st(kh + 2 * m + 1, x1[r] / den);
            }
        }
        for (int x = lane; x < DH; x += 32) vv[x] = vin[src + x];
        if (lane == 0) {
            c.bias[slot] = p.bfinal[((size_t)b * c.Hkv + h) * T + t];
            c.rk[slot] = softplus_f(p.a_k[((size_t)b * T + t) * c.Hkv + h]);
            c.pos[slot] = t;
            if (t == 0) c.n_kept[(size_t)b * c.Hkv + h] = T;
        }
    }
}

// ------------------------------------------------------------------ compaction
// grid (B*Hkv), 256 threads.
template <typename TC, int DH>
__global__ void __launch_bounds__(256) k_cache_compact(CompactParams p) {
    using L = EntryLayout<TC, DH>;
    __shared__ int s_wcnt[L::NW];
    const CacheView& c = p.c;
    const int unit = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = lane / L::LPE, gl = lane % L::LPE;
    grid_dep_wait();
    grid_dep_release();
    int n = c.n_kept[unit];
    if (n < 0 || n > c.cap) {                 // corrupt count: never read past the cache
        if (threadIdx.x == 0) raise_status(UA_ERR_CAPACITY);
        n = n < 0 ? 0 : c.cap;
    }
    const size_t base = (size_t)unit * c.cap;
    TC* khat = static_cast<TC*>(c.khat);
    TC* vc = static_cast<TC*>(c.v);
    int out = 0;
    for (int c0 = 0; c0 < n; c0 += L::EPB) {
        const int j = c0 + warp * L::EPW + grp;
        const bool valid = j < n;
        uint4 a = make_uint4(0, 0, 0, 0), vv = a;
        float bj = 0.f, rkj = 0.f;
        int pj = 0;
        bool keep = false;
        const long long ps = valid ? phys_slot(c, unit, j) : -1;
        if (ps >= 0) {
            const size_t e = (size_t)ps * DH + gl * L::VEC;
            a = *reinterpret_cast<const uint4*>(khat + e);
            vv = *reinterpret_cast<const uint4*>(vc + e);
            bj = c.bias[ps];
            rkj = c.rk[ps];
            pj = c.pos[ps];
            keep = p.keep ? (p.keep[base + j] != 0) : (bj >= p.logp);
        }
        int tot;
        const int dst = out + pass_scan<L::LPE, L::NW>(keep, warp, lane, s_wcnt, &tot);
        if (keep) {
            const long long pd = dst != j ? phys_slot(c, unit, dst) : -1;
            if (pd >= 0) {
                const size_t e = (size_t)pd * DH + gl * L::VEC;
                *reinterpret_cast<uint4*>(khat + e) = a;
                *reinterpret_cast<uint4*>(vc + e) = vv;
                if (gl == 0) {
                    c.bias[pd] = bj;
                    c.rk[pd] = rkj;
                    c.pos[pd] = pj;
                }
            }
            if (gl == 0 && p.kept_idx) p.kept_idx[base + dst] = j;
        }
        out += tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) c.n_kept[unit] = out;
}

// ------------------------------------------------------------------ decode step
// grid (B*Hkv), 256 threads.  Dynamic shared memory: eviction bitmap (ceil(cap/32) words)
// followed by the per-group softmax partials.
// DEFER: deferred compaction (UA_DECODE_DEFER_COMPACT).  VAR: an ablation variant is set; without
// it the variant is the constant 0 and every variant branch folds away.  Both are separate
// instantiations so that the method's own per-step path keeps its registers and instructions.
template <typename TC, int DH, int G, bool DEFER, bool VAR, bool PAGED>
__global__ void __launch_bounds__(256, G <= 4 ? 2 : 1) k_decode(DecodeParams p) {
    const int variant = VAR ? p.variant : 0;
    using L = EntryLayout<TC, DH>;
    constexpr int VEC = L::VEC, LPE = L::LPE, EPB = L::EPB, NW = L::NW;
    constexpr int half = DH / 2;
    __shared__ float s_kt[DH], s_ktr[DH], s_vt[DH], s_q[G][DH], s_g[G * DH], s_qn[G];
    __shared__ float s_red[NW];
    __shared__ double s_rf[DH / 2];
    __shared__ int s_wcnt[NW];
    extern __shared__ float dsm[];
    const CacheView& c = p.c;
    const int words = (c.cap + 31) / 32;
    uint32_t* s_ev = reinterpret_cast<uint32_t*>(dsm);
    float* s_m = dsm + ((words + 3) & ~3);          // [EPB][G]
    float* s_l = s_m + EPB * G;                       // [EPB][G]
    float* s_acc = s_l + EPB * G;                     // [EPB][G][DH]

    const int unit = blockIdx.x, b = unit / c.Hkv, kvh = unit % c.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = lane / LPE, gl = lane % LPE;
    const int gidx = warp * L::EPW + grp;             // entry group index in the pass
    const size_t base = (size_t)unit * c.cap;
    TC* khat = static_cast<TC*>(c.khat);
    TC* vc = static_cast<TC*>(c.v);

    grid_dep_wait();
    grid_dep_release();
    // ---- Every load that depends on no other goes out first: the live count, the first pass
    // of cache entries, the new token, its gate and the rates, so a step over a pruned, tiny
    // cache pays one memory round trip before its arithmetic.  The first pass is read within
    // the capacity whatever the count (which is still in flight); entries past the count are
    // masked out below.
    int n = c.n_kept[unit];
    // Software pipeline: the entries of the next pass are loaded before this pass is processed,
    // so two passes of loads are in flight.  Safe with the in-place compaction: a survivor of
    // this pass only ever moves to a slot at or below its own, never into the next pass.
    uint4 na = make_uint4(0, 0, 0, 0), nv = na;
    float nbj = 0.f, nrk = 0.f;
    int npj = 0;
    long long nps = -1;                               // paged: the loaded entry's physical slot
    auto load_entry = [&](int jj, int lim) {
        if constexpr (PAGED) {
            nps = jj < lim ? phys_slot(c, unit, jj) : -1;
            if (nps >= 0) {
                const size_t e = (size_t)nps * DH + gl * VEC;
                na = *reinterpret_cast<const uint4*>(khat + e);
                nv = *reinterpret_cast<const uint4*>(vc + e);
                nbj = c.bias[nps];
                nrk = c.rk[nps];
                npj = c.pos[nps];
            }
        } else if (jj < lim) {
            const size_t e = (base + jj) * DH + gl * VEC;
            na = *reinterpret_cast<const uint4*>(khat + e);
            nv = *reinterpret_cast<const uint4*>(vc + e);
            nbj = c.bias[base + jj];
            nrk = c.rk[base + jj];
            npj = c.pos[base + jj];
        }
    };
    // (paged storage reads the first pass once the count is known: slots past it may have no page)
    if (!PAGED) load_entry(gidx, c.cap);
    // the step's key and value: head kvh / rep of [B, Hkv / rep, d]
    const size_t tok = (size_t)b * (c.Hkv / c.rep) + kvh / c.rep;
    const TC* kin = static_cast<const TC*>(p.k) + tok * DH;
    const TC* vin = static_cast<const TC*>(p.v) + tok * DH;
    const TC* qin = static_cast<const TC*>(p.q) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
    const TC* gin = static_cast<const TC*>(p.g) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
    constexpr int QE = (G * half + 255) / 256, GE = (G * DH + 255) / 256;
    float kx = 0.f, vx = 0.f;
    if (tid < DH) {
        kx = Elem<TC>::ld(kin + tid);
        vx = Elem<TC>::ld(vin + tid);
    }
    float qa[QE], qb[QE];
#pragma unroll
    for (int r = 0; r < QE; ++r) {
        const int e = tid + 256 * r;
        qa[r] = qb[r] = 0.f;
        if (e < G * half) {
            const int vecid = e / half, m = e % half;
            qa[r] = Elem<TC>::ld(qin + vecid * DH + m);
            qb[r] = Elem<TC>::ld(qin + vecid * DH + m + half);
        }
    }
    // the gate goes to shared memory: loaded now, held in no register through the entry loop
#pragma unroll
    for (int r = 0; r < GE; ++r) {
        const int e = tid + 256 * r;
        if (e < G * DH) s_g[e] = Elem<TC>::ld(gin + e);
    }
    const float aq_t = p.a_q[unit], ak_t = p.a_k[unit];
    const float al = p.alpha[kvh], be = p.beta[kvh];


    // ---- new token: khat_t, RoPE(khat_t), v_t, RoPE(q_h), rates
    float ss = kx * kx;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_red[warp] = ss;
    for (int w = tid; w < words; w += blockDim.x) s_ev[w] = 0u;
    // the RoPE frequencies go to shared memory once, a few per warp (a kernel-parameter array
    // read at a different index by each lane serialises those reads)
    static_assert(half % NW == 0, "frequencies split evenly over the warps");
    if (lane < half / NW) s_rf[warp * (half / NW) + lane] = p.rf.f[warp * (half / NW) + lane];
    __syncthreads();
    float tot_ss = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) tot_ss += s_red[w];
    const float den = fmaxf(sqrtf(tot_ss), 1e-12f);
    // khat_t, RoPE(q_h) and RoPE(khat_t) are held pair-interleaved, as the cache stores keys
    if (tid < DH) {
        s_kt[il_index(tid, half)] = kx / den;
        s_vt[tid] = vx;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < QE; ++r) {
        const int e = tid + 256 * r;
        if (e < G * half) {
            const int vecid = e / half, m = e % half;
            float cs, sn;
            rope_cs((double)p.pos_t, s_rf[m], &cs, &sn);
            s_q[vecid][2 * m] = qa[r] * cs - qb[r] * sn;
            s_q[vecid][2 * m + 1] = qb[r] * cs + qa[r] * sn;
        }
    }
    for (int m = tid; m < half; m += blockDim.x) {
        float cs, sn;
        rope_cs((double)p.pos_t, s_rf[m], &cs, &sn);
        const float x0 = s_kt[2 * m], x1 = s_kt[2 * m + 1];
        s_ktr[2 * m] = x0 * cs - x1 * sn;
        s_ktr[2 * m + 1] = x1 * cs + x0 * sn;
    }
    __syncthreads();
    if (variant & kVarQNorm) {                    // query RMS norm (RoPE keeps the norm)
        if (tid < G) {
            float qq = 0.f;
            for (int x = 0; x < DH; ++x) qq = fmaf(s_q[tid][x], s_q[tid][x], qq);
            s_qn[tid] = 1.f / sqrtf(qq * (1.f / DH) + kQNormEps);
        }
        __syncthreads();
        for (int e = tid; e < G * DH; e += blockDim.x) s_q[e / DH][e % DH] *= s_qn[e / DH];
        __syncthreads();
    }
    const float rq_t = (variant & kVarNoQ) ? 1.f : softplus_f(aq_t);
    const float rk_t = softplus_f(ak_t);          // stored in the cache as is

    // the new key stays in registers; the rotated queries are read from shared memory per
    // entry, which leaves the registers for the next pass's entries (loaded one pass ahead)
    float kq[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) kq[e] = s_kt[gl * VEC + e];
    double gt[VEC / 2];                               // this lane's RoPE frequencies / (2 pi)
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) gt[i] = s_rf[gl * (VEC / 2) + i] * 0.15915494309189535;
    float m_h[G], l_h[G], acc[G][VEC];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m_h[h] = -INFINITY;
        l_h[h] = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[h][e] = 0.f;
    }

    if (n < 0 || n > c.cap) {                 // corrupt count: never read past the cache
        if (tid == 0) raise_status(UA_ERR_CAPACITY);
        n = n < 0 ? 0 : c.cap;
    }
    int out = 0;
    const bool multi_pass = n > 4 * EPB;   // block-uniform
    if (PAGED) load_entry(gidx, n);
    for (int c0 = 0; c0 < n; c0 += EPB) {
        const int j = c0 + gidx;
        const bool valid = j < n;
        // long caches: ask L2 for the entries of the next two passes now (no registers held);
        // one lane per entry covers its whole 128-byte row; a cache of four passes or fewer skips this
        if (multi_pass && gl == 0) {
#pragma unroll
            for (int ahead = 1; ahead <= 2; ++ahead) {
                const int jn = j + ahead * EPB;
                if constexpr (PAGED) {
                    const long long pn = jn < n ? phys_slot<false>(c, unit, jn) : -1;
                    if (pn >= 0) {
                        const size_t e = (size_t)pn * DH;
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(khat + e));
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(vc + e));
                        if ((jn & 31) == 0) {
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(c.bias + pn));
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(c.rk + pn));
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(c.pos + pn));
                        }
                    }
                } else if (jn < n) {
                    const size_t e = (base + jn) * DH;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(khat + e));
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(vc + e));
                    if ((jn & 31) == 0) {
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(c.bias + base + jn));
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(c.rk + base + jn));
                        asm volatile("prefetch.global.L2 [%0];" ::"l"(c.pos + base + jn));
                    }
                }
            }
        }
        const uint4 ra = na, rv = nv;
        const float bj = nbj, rkj = nrk;
        const int pj = npj;
        const long long psj = nps;                    // paged only
        load_entry(j + EPB, n);
        float xa[VEC], xb[VEC], xv[VEC];
        Vec16<TC>::unpack(ra, xa);
        Vec16<TC>::unpack(rv, xv);
        rotate_pairs<VEC>(xa, xb, (double)pj, gt);
        float sim = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) sim = fmaf(kq[e], xa[e], sim);
        sim = group_sum<LPE>(sim);
        const float D = decay_var(rq_t, (variant & kVarNoK) ? 1.f : rkj, fmaf(al, sim, be), variant);
        const float bnew = bj - D;
        const bool keep = PAGED ? valid && psj >= 0 && (bnew >= p.logp) : valid && (bnew >= p.logp);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float lg = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) lg = fmaf(s_q[h][gl * VEC + e], xb[e], lg);
            lg = group_sum<LPE>(lg);
            if (keep) {
                lg = fmaf(lg, p.scale, bnew);
                const float mn = fmaxf(m_h[h], lg);
                const float corr = expf(m_h[h] - mn);
                const float pe = expf(lg - mn);
                l_h[h] = l_h[h] * corr + pe;
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[h][e] = fmaf(pe, xv[e], acc[h][e] * corr);
                m_h[h] = mn;
            }
        }
        if (valid && !keep && gl == 0) atomicOr(&s_ev[j >> 5], 1u << (j & 31));
        if (DEFER) {                              // every pair keeps its slot
            if (valid && gl == 0) {
                if constexpr (PAGED) {
                    if (psj >= 0) c.bias[psj] = bnew;
                } else {
                    c.bias[base + j] = bnew;
                }
                if (p.kept_idx) p.kept_idx[base + j] = j;
            }
            __syncthreads();
            continue;
        }
        int tot;
        const int dst = out + pass_scan<LPE, NW>(keep, warp, lane, s_wcnt, &tot);
        if (keep) {
            if constexpr (PAGED) {
                const long long pd = dst != j ? phys_slot(c, unit, dst) : psj;
                if (pd >= 0 && dst != j) {
                    const size_t e = (size_t)pd * DH + gl * VEC;
                    *reinterpret_cast<uint4*>(khat + e) = ra;
                    *reinterpret_cast<uint4*>(vc + e) = rv;
                    if (gl == 0) {
                        c.rk[pd] = rkj;
                        c.pos[pd] = pj;
                    }
                }
                if (gl == 0) {
                    if (pd >= 0) c.bias[pd] = bnew;
                    if (p.kept_idx) p.kept_idx[base + dst] = j;
                }
            } else {
                if (dst != j) {
                    const size_t e = (base + dst) * DH + gl * VEC;
                    *reinterpret_cast<uint4*>(khat + e) = ra;
                    *reinterpret_cast<uint4*>(vc + e) = rv;
                    if (gl == 0) {
                        c.rk[base + dst] = rkj;
                        c.pos[base + dst] = pj;
                    }
                }
                if (gl == 0) {
                    c.bias[base + dst] = bnew;
                    if (p.kept_idx) p.kept_idx[base + dst] = j;
                }
            }
        }
        out += tot;
        __syncthreads();
    }

    if (DEFER) out = n;                           // append after every pair, evicted ones included
    // ---- merge the per-group online-softmax states, add the new token, gate, store
    if (gl == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            s_m[gidx * G + h] = m_h[h];
            s_l[gidx * G + h] = l_h[h];
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < VEC; e += 4)
            *reinterpret_cast<float4*>(s_acc + ((size_t)gidx * G + h) * DH + gl * VEC + e) =
                make_float4(acc[h][e], acc[h][e + 1], acc[h][e + 2], acc[h][e + 3]);
    __syncthreads();
    const int qn = min(EPB, n);                       // entry groups that saw an entry (short caches: few)
    // Warp h merges head h's states: the common maximum with the new token's own logit, the
    // weight of each group's state (left in s_m) and of the new token, and 1 / (the total sum).
    static_assert(EPB <= 32, "a lane per entry group in the merge");
    __shared__ float s_wt[G], s_inv[G];
    if (warp < G) {
        const int h = warp;
        // the new token's own logit (its bias is 0)
        float lt = 0.f;
#pragma unroll
        for (int x = lane; x < DH; x += 32) lt = fmaf(s_q[h][x], s_ktr[x], lt);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, o);
        lt *= p.scale;
        const float mq = lane < qn ? s_m[lane * G + h] : -INFINITY;
        float M = fmaxf(mq, lt);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float w = lane < qn ? expf(mq - M) : 0.f;
        float L = lane < qn ? s_l[lane * G + h] * w : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        const float wt = expf(lt - M);
        __syncwarp();
        if (lane < qn) s_m[lane * G + h] = w;
        if (lane == 0) {
            s_wt[h] = wt;
            s_inv[h] = 1.f / (L + wt);
        }
    }
    __syncthreads();
    TC* oout = static_cast<TC*>(p.o) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
#pragma unroll
    for (int r = 0; r < GE; ++r) {
        const int e = tid + 256 * r;
        if (e >= G * DH) break;
        const int h = e / DH, x = e % DH;
        // four partial sums over the groups' states (independent loads and adds)
        const float* ac = s_acc + (size_t)h * DH + x;     // group q at + q * G * DH
        const float* wq = s_m + h;                         // group q at + q * G
        float A0 = s_wt[h] * s_vt[x], A1 = 0.f, A2 = 0.f, A3 = 0.f;
        int q = 0;
        for (; q + 4 <= qn; q += 4) {
            A0 = fmaf(ac[(size_t)q * G * DH], wq[q * G], A0);
            A1 = fmaf(ac[(size_t)(q + 1) * G * DH], wq[(q + 1) * G], A1);
            A2 = fmaf(ac[(size_t)(q + 2) * G * DH], wq[(q + 2) * G], A2);
            A3 = fmaf(ac[(size_t)(q + 3) * G * DH], wq[(q + 3) * G], A3);
        }
        for (; q < qn; ++q) A0 = fmaf(ac[(size_t)q * G * DH], wq[q * G], A0);
        Elem<TC>::st(oout + e, ((A0 + A1) + (A2 + A3)) * s_inv[h] * sigmoid_f(s_g[e]));
    }
    // ---- eviction bits, append the new token
    if (p.evict_bits)
        for (int w = tid; w < words; w += blockDim.x) p.evict_bits[(size_t)unit * words + w] = s_ev[w];
    if (out < c.cap) {
        if constexpr (PAGED) {
            const long long pa = phys_slot(c, unit, out);
            if (pa >= 0) {
                const size_t e = (size_t)pa * DH;
                for (int x = tid; x < DH; x += blockDim.x) {
                    Elem<TC>::st(khat + e + x, s_kt[x]);
                    Elem<TC>::st(vc + e + x, s_vt[x]);
                }
                if (tid == 0) {
                    c.bias[pa] = 0.f;
                    c.rk[pa] = rk_t;
                    c.pos[pa] = p.pos_t;
                }
            }
            if (tid == 0) {
                c.n_kept[unit] = out + 1;
                if (p.kept_idx) p.kept_idx[base + out] = -1;
            }
        } else {
            const size_t e = (base + out) * DH;
            for (int x = tid; x < DH; x += blockDim.x) {
                Elem<TC>::st(khat + e + x, s_kt[x]);
                Elem<TC>::st(vc + e + x, s_vt[x]);
            }
            if (tid == 0) {
                c.bias[base + out] = 0.f;
                c.rk[base + out] = rk_t;
                c.pos[base + out] = p.pos_t;
                c.n_kept[unit] = out + 1;
                if (p.kept_idx) p.kept_idx[base + out] = -1;
            }
        }
    } else if (tid == 0) {
        c.n_kept[unit] = out;
        raise_status(UA_ERR_CAPACITY);
    }
}

// ------------------------------------------------------------------ split decode step
// grid (kDecodeSplitSimt, B*Hkv), 256 threads.  A long cache is walked by several CTAs at once:
// slice s of S = min(kDecodeSplitSimt, ceil(n / kDecodeSplitSlice)) covers pairs [lo, hi) (whole
// 32-pair words); CTAs past S get an empty slice.  Each CTA updates its pairs' biases in place,
// marks its evictions, and leaves its partial online-softmax state (per head: maximum, sum,
// weighted values) in the workspace; the CTA that arrives last (a counter per cache counting
// every CTA of the grid; a fence before every arrival) merges the states with the new token's
// own term, gates, writes o and appends the token.  Counting every CTA, not only those with
// pairs, means the merge -- which changes n -- happens only after all of them have read n.
// Compaction is deferred: pairs keep their slots, evicted ones are excluded by their bias until
// ua_cache_compact removes them.  No CTA ever waits on another.
template <typename TC, int DH, int G, bool VAR>
__global__ void __launch_bounds__(256, G <= 4 ? 2 : 1) k_decode_split(DecodeParams p) {
    const int variant = VAR ? p.variant : 0;
    using L = EntryLayout<TC, DH>;
    constexpr int VEC = L::VEC, LPE = L::LPE, EPB = L::EPB, NW = L::NW;
    constexpr int half = DH / 2;
    constexpr int SS = G * (DH + 2);                  // floats of one partial state
    __shared__ float s_kt[DH], s_ktr[DH], s_vt[DH], s_q[G][DH], s_lt[G], s_g[G * DH], s_qn[G];
    __shared__ float s_red[NW];
    __shared__ float s_m[EPB * G], s_l[EPB * G];
    __shared__ int s_last;
    extern __shared__ float dsm[];
    float* s_acc = dsm;                               // [EPB][G][DH]
    uint32_t* s_ev = reinterpret_cast<uint32_t*>(dsm + (size_t)EPB * G * DH);   // the slice's words
    const CacheView& c = p.c;
    const int words = (c.cap + 31) / 32;
    const int unit = blockIdx.y, sl = blockIdx.x, b = unit / c.Hkv, kvh = unit % c.Hkv;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int grp = lane / LPE, gl = lane % LPE;
    const int gidx = warp * L::EPW + grp;
    const size_t base = (size_t)unit * c.cap;
    TC* khat = static_cast<TC*>(c.khat);
    TC* vc = static_cast<TC*>(c.v);

    grid_dep_wait();
    grid_dep_release();
    int n = c.n_kept[unit];
    if (n < 0 || n > c.cap) {                 // corrupt count: never read past the cache
        if (tid == 0 && sl == 0) raise_status(UA_ERR_CAPACITY);
        n = n < 0 ? 0 : c.cap;
    }
    const int nsl = min((int)gridDim.x, max(1, (n + kDecodeSplitSlice - 1) / kDecodeSplitSlice));
    const int chunk = (((n + nsl - 1) / nsl) + 31) & ~31;
    const int lo = sl < nsl ? min(n, sl * chunk) : n;
    const int hi = sl < nsl ? min(n, lo + chunk) : n;
    const int w0 = lo >> 5, nw = (hi - lo + 31) >> 5;

    // ---- new token (every CTA of the cache forms it; only the last one uses v, g)
    // the step's key and value: head kvh / rep of [B, Hkv / rep, d]
    const size_t tok = (size_t)b * (c.Hkv / c.rep) + kvh / c.rep;
    const TC* kin = static_cast<const TC*>(p.k) + tok * DH;
    const TC* vin = static_cast<const TC*>(p.v) + tok * DH;
    const TC* qin = static_cast<const TC*>(p.q) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
    const TC* gin = static_cast<const TC*>(p.g) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
    float kx = 0.f;
    if (tid < DH) {
        kx = Elem<TC>::ld(kin + tid);
        s_vt[tid] = Elem<TC>::ld(vin + tid);
    }
    for (int e = tid; e < G * DH; e += blockDim.x) s_g[e] = Elem<TC>::ld(gin + e);
    for (int w = tid; w < nw; w += blockDim.x) s_ev[w] = 0u;
    float ss = kx * kx;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    float tot_ss = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) tot_ss += s_red[w];
    const float den = fmaxf(sqrtf(tot_ss), 1e-12f);
    if (tid < DH) s_kt[il_index(tid, half)] = kx / den;     // pair-interleaved, as cached
    __syncthreads();
    for (int e = tid; e < G * half; e += blockDim.x) {
        const int vecid = e / half, m = e % half;
        float cs, sn;
        rope_cs((double)p.pos_t, p.rf.f[m], &cs, &sn);
        const float qa = Elem<TC>::ld(qin + vecid * DH + m), qb = Elem<TC>::ld(qin + vecid * DH + m + half);
        s_q[vecid][2 * m] = qa * cs - qb * sn;
        s_q[vecid][2 * m + 1] = qb * cs + qa * sn;
    }
    for (int m = tid; m < half; m += blockDim.x) {
        float cs, sn;
        rope_cs((double)p.pos_t, p.rf.f[m], &cs, &sn);
        const float x0 = s_kt[2 * m], x1 = s_kt[2 * m + 1];
        s_ktr[2 * m] = x0 * cs - x1 * sn;
        s_ktr[2 * m + 1] = x1 * cs + x0 * sn;
    }
    __syncthreads();
    if (variant & kVarQNorm) {
        if (tid < G) {
            float qq = 0.f;
            for (int x = 0; x < DH; ++x) qq = fmaf(s_q[tid][x], s_q[tid][x], qq);
            s_qn[tid] = 1.f / sqrtf(qq * (1.f / DH) + kQNormEps);
        }
        __syncthreads();
        for (int e = tid; e < G * DH; e += blockDim.x) s_q[e / DH][e % DH] *= s_qn[e / DH];
        __syncthreads();
    }
    if (tid < G) {
        float a = 0.f;
        for (int x = 0; x < DH; ++x) a = fmaf(s_q[tid][x], s_ktr[x], a);
        s_lt[tid] = a * p.scale;
    }
    const float aq_t = p.a_q[unit], ak_t = p.a_k[unit];
    const float al = p.alpha[kvh], be = p.beta[kvh];
    const float rq_t = (variant & kVarNoQ) ? 1.f : softplus_f(aq_t);
    float kq[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) kq[e] = s_kt[gl * VEC + e];
    double gt[VEC / 2];                               // this lane's RoPE frequencies / (2 pi)
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) gt[i] = p.rf.f[gl * (VEC / 2) + i] * 0.15915494309189535;
    float m_h[G], l_h[G], acc[G][VEC];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m_h[h] = -INFINITY;
        l_h[h] = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[h][e] = 0.f;
    }

    // ---- the slice: pairs [lo, hi), next pass loaded one pass ahead
    uint4 na = make_uint4(0, 0, 0, 0), nv = na;
    float nbj = 0.f, nrk = 0.f;
    int npj = 0;
    long long nps = -1;                               // the loaded entry's physical slot
    auto load_entry = [&](int jj) {
        nps = jj < hi ? phys_slot(c, unit, jj) : -1;
        if (nps >= 0) {
            const size_t e = (size_t)nps * DH + gl * VEC;
            na = *reinterpret_cast<const uint4*>(khat + e);
            nv = *reinterpret_cast<const uint4*>(vc + e);
            nbj = c.bias[nps];
            nrk = c.rk[nps];
            npj = c.pos[nps];
        }
    };
    load_entry(lo + gidx);
    for (int c0 = lo; c0 < hi; c0 += EPB) {
        const int j = c0 + gidx;
        const bool valid = j < hi;
        const uint4 ra = na, rv = nv;
        const float bj = nbj, rkj = nrk;
        const int pj = npj;
        const long long psj = nps;
        load_entry(j + EPB);
        float xa[VEC], xb[VEC], xv[VEC];
        Vec16<TC>::unpack(ra, xa);
        Vec16<TC>::unpack(rv, xv);
        rotate_pairs<VEC>(xa, xb, (double)pj, gt);
        float sim = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) sim = fmaf(kq[e], xa[e], sim);
        sim = group_sum<LPE>(sim);
        const float D = decay_var(rq_t, (variant & kVarNoK) ? 1.f : rkj, fmaf(al, sim, be), variant);
        const float bnew = bj - D;
        const bool keep = valid && psj >= 0 && (bnew >= p.logp);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float lg = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) lg = fmaf(s_q[h][gl * VEC + e], xb[e], lg);
            lg = group_sum<LPE>(lg);
            if (keep) {
                lg = fmaf(lg, p.scale, bnew);
                const float mn = fmaxf(m_h[h], lg);
                const float corr = expf(m_h[h] - mn);
                const float pe = expf(lg - mn);
                l_h[h] = l_h[h] * corr + pe;
#pragma unroll
                for (int e = 0; e < VEC; ++e) acc[h][e] = fmaf(pe, xv[e], acc[h][e] * corr);
                m_h[h] = mn;
            }
        }
        if (valid && gl == 0) {
            if (psj >= 0) c.bias[psj] = bnew;
            if (p.kept_idx) p.kept_idx[base + j] = j;
            if (!keep) atomicOr(&s_ev[(j >> 5) - w0], 1u << (j & 31));
        }
    }
    // ---- the CTA's partial state: merge its entry groups
    if (gl == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            s_m[gidx * G + h] = m_h[h];
            s_l[gidx * G + h] = l_h[h];
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < VEC; ++e) s_acc[((size_t)gidx * G + h) * DH + gl * VEC + e] = acc[h][e];
    __syncthreads();
    if (p.evict_bits)
        for (int w = tid; w < nw; w += blockDim.x) p.evict_bits[(size_t)unit * words + w0 + w] = s_ev[w];
    float* st = p.split_state + ((size_t)unit * kDecodeSplitMax + sl) * SS;
    for (int e = tid; e < G * DH; e += blockDim.x) {
        const int h = e / DH, x = e % DH;
        float M = -INFINITY;
        for (int q = 0; q < EPB; ++q) M = fmaxf(M, s_m[q * G + h]);
        float Ls = 0.f, A = 0.f;
        if (M > -INFINITY) {
            for (int q = 0; q < EPB; ++q) {
                const float w = expf(s_m[q * G + h] - M);
                Ls = fmaf(s_l[q * G + h], w, Ls);
                A = fmaf(s_acc[((size_t)q * G + h) * DH + x], w, A);
            }
        }
        st[2 * G + e] = A;
        if (x == 0) {
            st[h] = M;
            st[G + h] = Ls;
        }
    }
    __threadfence();                                   // the state, biases and bits before the arrival
    __syncthreads();
    if (tid == 0) {
        const unsigned old = atomicAdd(p.split_cnt + unit, 1u);
        if (old >= gridDim.x) raise_status(UA_ERR_INVALID_ARG);   // the workspace was not zeroed
        s_last = old == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // ---- last CTA of the cache: merge the slices with the new token, gate, append
    TC* oout = static_cast<TC*>(p.o) + ((size_t)b * p.H + (size_t)kvh * G) * DH;
    const float* st0 = p.split_state + (size_t)unit * kDecodeSplitMax * SS;
    for (int e = tid; e < G * DH; e += blockDim.x) {
        const int h = e / DH, x = e % DH;
        float M = s_lt[h];
        for (int q = 0; q < (int)gridDim.x; ++q) M = fmaxf(M, __ldcg(st0 + (size_t)q * SS + h));
        float Ls = expf(s_lt[h] - M);
        float A = Ls * s_vt[x];
        for (int q = 0; q < (int)gridDim.x; ++q) {
            const float mq = __ldcg(st0 + (size_t)q * SS + h);
            if (mq > -INFINITY) {
                const float w = expf(mq - M);
                Ls = fmaf(__ldcg(st0 + (size_t)q * SS + G + h), w, Ls);
                A = fmaf(__ldcg(st0 + (size_t)q * SS + 2 * G + e), w, A);
            }
        }
        Elem<TC>::st(oout + e, A / Ls * sigmoid_f(s_g[e]));
    }
    // words past the live pairs carry no eviction
    if (p.evict_bits)
        for (int w = ((n + 31) >> 5) + tid; w < words; w += blockDim.x) p.evict_bits[(size_t)unit * words + w] = 0u;
    if (n < c.cap) {
        const long long pa = phys_slot(c, unit, n);
        if (pa >= 0) {
            const size_t e = (size_t)pa * DH;
            for (int x = tid; x < DH; x += blockDim.x) {
                Elem<TC>::st(khat + e + x, s_kt[x]);
                Elem<TC>::st(vc + e + x, s_vt[x]);
            }
            if (tid == 0) {
                c.bias[pa] = 0.f;
                c.rk[pa] = softplus_f(ak_t);
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
    if (tid == 0) p.split_cnt[unit] = 0u;            // ready for the next step
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_cache_fill(const FillParams& p, bool bf16, cudaStream_t s) {
    dim3 grid(p.T, p.c.B);
    UA_PROFILE("k_cache_fill", s);
    if (bf16) {
        if (p.c.d == 64) k_cache_fill<__nv_bfloat16, 64><<<grid, 256, 0, s>>>(p);
        else k_cache_fill<__nv_bfloat16, 128><<<grid, 256, 0, s>>>(p);
    } else {
        if (p.c.d == 64) k_cache_fill<float, 64><<<grid, 256, 0, s>>>(p);
        else k_cache_fill<float, 128><<<grid, 256, 0, s>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_cache_compact(const CompactParams& p, bool bf16, cudaStream_t s) {
    dim3 grid(p.c.B * p.c.Hkv);
    UA_PROFILE("k_cache_compact", s);
    if (bf16) {
        return p.c.d == 64 ? launch_dependent(k_cache_compact<__nv_bfloat16, 64>, grid, dim3(256), 0, s, p)
                           : launch_dependent(k_cache_compact<__nv_bfloat16, 128>, grid, dim3(256), 0, s, p);
    } else {
        return p.c.d == 64 ? launch_dependent(k_cache_compact<float, 64>, grid, dim3(256), 0, s, p)
                           : launch_dependent(k_cache_compact<float, 128>, grid, dim3(256), 0, s, p);
    }
}

template <typename TC, int DH, int G, bool DEFER, bool VAR>
static cudaError_t decode_launch(const DecodeParams& p, size_t smem, cudaStream_t s) {
    auto kern = p.c.pt != nullptr ? k_decode<TC, DH, G, DEFER, VAR, true> : k_decode<TC, DH, G, DEFER, VAR, false>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    UA_PROFILE("k_decode", s);
    return launch_dependent(kern, dim3(p.c.B * p.c.Hkv), dim3(256), smem, s, p);
}

template <typename TC, int DH, int G>
static cudaError_t decode_inst(const DecodeParams& p, cudaStream_t s) {
    using L = EntryLayout<TC, DH>;
    const int words = (p.c.cap + 31) / 32;
    const size_t smem = sizeof(float) * ((size_t)((words + 3) & ~3) + 2 * L::EPB * G + (size_t)L::EPB * G * DH);
    if (p.variant != 0)
        return p.defer ? decode_launch<TC, DH, G, true, true>(p, smem, s) : decode_launch<TC, DH, G, false, true>(p, smem, s);
    return p.defer ? decode_launch<TC, DH, G, true, false>(p, smem, s) : decode_launch<TC, DH, G, false, false>(p, smem, s);
}

template <typename TC, int DH>
static cudaError_t decode_g(const DecodeParams& p, cudaStream_t s) {
    switch (p.G) {
        case 1: return decode_inst<TC, DH, 1>(p, s);
        case 2: return decode_inst<TC, DH, 2>(p, s);
        case 3: return decode_inst<TC, DH, 3>(p, s);
        case 4: return decode_inst<TC, DH, 4>(p, s);
        case 8: return decode_inst<TC, DH, 8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

template <typename TC, int DH, int G>
static cudaError_t decode_split_inst(const DecodeParams& p, cudaStream_t s) {
    using L = EntryLayout<TC, DH>;
    // the largest slice: at most kDecodeSplitSlice pairs while the cache is short enough to be
    // split into whole slices, else a kDecodeSplitSimt-th of the capacity (whole 32-pair words)
    const int max_chunk = std::max(kDecodeSplitSlice, ((p.c.cap + kDecodeSplitSimt - 1) / kDecodeSplitSimt + 31) & ~31);
    const size_t smem = sizeof(float) * (size_t)L::EPB * G * DH + sizeof(uint32_t) * (size_t)(max_chunk / 32 + 1);
    dim3 grid(kDecodeSplitSimt, p.c.B * p.c.Hkv);
    auto kern = p.variant != 0 ? k_decode_split<TC, DH, G, true> : k_decode_split<TC, DH, G, false>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    UA_PROFILE("k_decode_split", s);
    return launch_dependent(kern, grid, dim3(256), smem, s, p);
}

template <typename TC, int DH>
static cudaError_t decode_split_g(const DecodeParams& p, cudaStream_t s) {
    switch (p.G) {
        case 1: return decode_split_inst<TC, DH, 1>(p, s);
        case 2: return decode_split_inst<TC, DH, 2>(p, s);
        case 3: return decode_split_inst<TC, DH, 3>(p, s);
        case 4: return decode_split_inst<TC, DH, 4>(p, s);
        case 8: return decode_split_inst<TC, DH, 8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_split(const DecodeParams& p, bool bf16, cudaStream_t s) {
    if (bf16) return p.c.d == 64 ? decode_split_g<__nv_bfloat16, 64>(p, s) : decode_split_g<__nv_bfloat16, 128>(p, s);
    return p.c.d == 64 ? decode_split_g<float, 64>(p, s) : decode_split_g<float, 128>(p, s);
}

cudaError_t launch_decode(const DecodeParams& p, bool bf16, cudaStream_t s) {
    if (bf16) return p.c.d == 64 ? decode_g<__nv_bfloat16, 64>(p, s) : decode_g<__nv_bfloat16, 128>(p, s);
    return p.c.d == 64 ? decode_g<float, 64>(p, s) : decode_g<float, 128>(p, s);
}

}  // namespace ua
