// k_prefill_simt.cu -- token preparation, the decay boundary pass and the fused biased
// attention forward, written as plain fp32 SIMT CUDA.  This is the exact-arithmetic path
// (fp32 activations); bf16 activations take the tensor-core path in k_prefill_tc.cu.
//
// Structure followed (see ua.h for the formulas): keys L2-normalised and RoPE kept
// (ai4snews synopsis, Fig. 1 caption); three rates combined by a geometric mean and
// accumulated causally (paperlayer.ai summary §4, §4.1); the decay applied inside a fused
// online softmax without materialising the T x T mask (paperlayer.ai summary App. C).
// Lambda is built as a chunked scan: the boundary pass writes, for every query tile t and
// key j, the column prefix Pb_t[j] = sum_{j<l<t*bq} D[l,j]; the attention kernel adds the
// in-tile triangular cumulative sum on top.
#include "ua_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

constexpr int kPrepTokens = 16;   // tokens per CTA of the token preparation

// ------------------------------------------------------------------ token preparation
// 8 consecutive activations <-> float registers (16-byte bf16 or 2 x 16-byte f32 accesses).
template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void ld(const __nv_bfloat16* p, float* x) { Vec16<__nv_bfloat16>::ld(p, x); }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, const float* x) { Vec16<__nv_bfloat16>::st(p, x); }
};
template <> struct Vec8<float> {
    static __device__ __forceinline__ void ld(const float* p, float* x) {
        Vec16<float>::ld(p, x);
        Vec16<float>::ld(p + 4, x + 4);
    }
    static __device__ __forceinline__ void st(float* p, const float* x) {
        Vec16<float>::st(p, x);
        Vec16<float>::st(p + 4, x + 4);
    }
};

// grid (ceil(T/TB), B), 256 threads.  A task is one 8-element chunk c of one (query or key)
// head of one token: elements 8c..8c+7 of the first half and their RoPE partners d/2 + 8c...;
// the CH = d/16 tasks of a head sit on consecutive lanes, which reduce the head's norm.
template <typename TI, typename TW, int DH>
__global__ void __launch_bounds__(256) k_prep(PrepParams p) {
    constexpr int TB = kPrepTokens, HALF = DH / 2, CH = HALF / 8;
    __shared__ float s_cos[TB][HALF], s_sin[TB][HALF];
    __shared__ double s_f[HALF];
    const int t0 = blockIdx.x * TB, b = blockIdx.y, T = p.T;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the RoPE frequencies, a few per warp (a kernel-parameter array read at a different index by
    // each lane serialises those reads)
    static_assert(HALF % 8 == 0, "frequencies split over the eight warps");
    if (lane < HALF / 8) s_f[warp * (HALF / 8) + lane] = p.rf.f[warp * (HALF / 8) + lane];
    __syncthreads();
    for (int e = tid; e < TB * HALF; e += blockDim.x) {
        const int tk = e / HALF, m = e % HALF;
        rope_cs((double)(t0 + tk), s_f[m], &s_cos[tk][m], &s_sin[tk][m]);
    }
    __syncthreads();
    const int nh = p.H + p.Hkv;
    const int ntask = TB * nh * CH;
    const TI* q = static_cast<const TI*>(p.q);
    const TI* k = static_cast<const TI*>(p.k);
    for (int base = 0; base < ntask; base += blockDim.x) {
        const int task = base + tid;
        const int c = task % CH, hh = (task / CH) % nh, tk = task / (CH * nh);
        const int t = t0 + tk;
        const bool valid = task < ntask && t < T;
        const bool is_q = hh < p.H;
        const int h = is_q ? hh : hh - p.H;
        float x0[8], x1[8];
        if (valid) {
            const TI* src = is_q ? q + (((size_t)b * T + t) * p.H + h) * DH : k + (((size_t)b * T + t) * p.Hkv + h) * DH;
            Vec8<TI>::ld(src + 8 * c, x0);
            Vec8<TI>::ld(src + HALF + 8 * c, x1);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) x0[e] = x1[e] = 0.f;
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x0[e], x0[e], fmaf(x1[e], x1[e], ss));
#pragma unroll
        for (int o = CH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (!valid) continue;
        TW* dst_rot;
        if (is_q) {
            if (p.variant & kVarQNorm) {              // Qwen3-style RMS norm, unit gain
                const float r = 1.f / sqrtf(ss * (1.f / DH) + kQNormEps);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x0[e] *= r;
                    x1[e] *= r;
                }
                ss *= r * r;
            }
            if (p.mq && c == 0) p.mq[((size_t)b * p.H + h) * p.Tp + t] = p.mq_scale * sqrtf(ss);
            dst_rot = static_cast<TW*>(p.qr) + (((size_t)b * p.H + h) * T + t) * DH;
        } else {
            const float den = fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                x0[e] = x0[e] / den;
                x1[e] = x1[e] / den;
            }
            TW* dst_hat = static_cast<TW*>(p.kh) + (((size_t)b * p.Hkv + h) * T + t) * DH;
            Vec8<TW>::st(dst_hat + 8 * c, x0);
            Vec8<TW>::st(dst_hat + HALF + 8 * c, x1);
            dst_rot = static_cast<TW*>(p.kr) + (((size_t)b * p.Hkv + h) * T + t) * DH;
        }
        float y0[8], y1[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float cs = s_cos[tk][8 * c + e], sn = s_sin[tk][8 * c + e];
            y0[e] = x0[e] * cs - x1[e] * sn;
            y1[e] = x1[e] * cs + x0[e] * sn;
        }
        Vec8<TW>::st(dst_rot + 8 * c, y0);
        Vec8<TW>::st(dst_rot + HALF + 8 * c, y1);
    }
    for (int e = tid; e < TB * p.Hkv; e += blockDim.x) {
        const int tk = e / p.Hkv, h = e % p.Hkv, t = t0 + tk;
        if (t >= T) continue;
        const size_t src = ((size_t)b * T + t) * p.Hkv + h;
        const size_t dst = ((size_t)b * p.Hkv + h) * T + t;
        // a switched-off mechanism contributes the neutral rate 1 to the geometric mean
        const float sq = (p.variant & kVarNoQ) ? 1.f : softplus_f(p.a_q[src]);
        const float sk = (p.variant & kVarNoK) ? 1.f : softplus_f(p.a_k[src]);
        if (p.rq) p.rq[dst] = sq;
        if (p.rk) p.rk[dst] = sk;
        if (p.lq2) {
            const size_t dp = ((size_t)b * p.Hkv + h) * p.Tp + t;
            p.lq2[dp] = log2f(sq) * (1.f / 3.f);      // log2(0) = -inf keeps the veto
            p.lk2[dp] = log2f(sk) * (1.f / 3.f);
        }
    }
}

// ------------------------------------------------------------------ tile row bounds
// grid (nqt, B*Hkv), 256 threads: the largest scale*||q_i|| over the 64 rows of a query tile and
// the G heads of a KV group.
__global__ void __launch_bounds__(256) k_tile_qmax(TileQmaxParams p) {
    const int qt = blockIdx.x, unit = blockIdx.y, b = unit / p.Hkv, kvh = unit % p.Hkv, G = p.H / p.Hkv;
    __shared__ float red[8];
    float m = 0.f;
    for (int e = threadIdx.x; e < 64 * G; e += blockDim.x) {
        const int hh = e / 64, i = qt * 64 + e % 64;
        if (i < p.T) m = fmaxf(m, p.mq[((size_t)b * p.H + kvh * G + hh) * p.T + i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
        p.qmax[(size_t)unit * p.nqt + qt] = m;
    }
}

cudaError_t launch_tile_qmax(const TileQmaxParams& p, cudaStream_t s) {
    UA_PROFILE("k_tile_qmax", s);
    k_tile_qmax<<<dim3(p.nqt, p.B * p.Hkv), 256, 0, s>>>(p);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ boundary pass
// grid (ceil(T/128), Hkv, B), 128 threads; thread = key j, sweeping the rows l > j in
// order.  At every query-tile boundary l = t*bq it writes the prefix sum so far.
// VAR: an ablation variant is set (without it the variant is the constant 0 and folds away).
template <int DH, bool VAR>
__global__ void __launch_bounds__(128) k_boundary_simt(BoundaryParams p) {
    const int variant = VAR ? p.variant : 0;
    constexpr int RC = 32;
    __shared__ float s_k[RC][DH];
    __shared__ float s_rq[RC];
    const int T = p.T;
    const int kt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int j = kt * 128 + threadIdx.x;
    const bool valid = j < T;
    const size_t unit = (size_t)b * p.Hkv + kvh;
    const float* kh = p.kh + unit * T * DH;
    float kj[DH];
#pragma unroll
    for (int c = 0; c < DH; ++c) kj[c] = valid ? kh[(size_t)j * DH + c] : 0.f;
    const float rkj = valid ? p.rk[unit * T + j] : 0.f;
    const float al = p.alpha[kvh], be = p.beta[kvh];
    float* pb = p.pb + unit * (size_t)p.nqt * T;
    const int l0 = kt * 128;
    if (valid)
        for (int t = 0; t * p.bq < l0; ++t) pb[(size_t)t * T + j] = 0.f;
    float acc = 0.f;
    for (int c0 = l0; c0 < T; c0 += RC) {
        __syncthreads();
        const int nrow = min(RC, T - c0);
        for (int e = threadIdx.x; e < RC * DH; e += 128) {
            const int r = e / DH, c = e % DH;
            s_k[r][c] = r < nrow ? kh[(size_t)(c0 + r) * DH + c] : 0.f;
        }
        if (threadIdx.x < RC) s_rq[threadIdx.x] = threadIdx.x < nrow ? p.rq[unit * T + c0 + threadIdx.x] : 0.f;
        __syncthreads();
        for (int r = 0; r < nrow; ++r) {
            const int l = c0 + r;
            if (valid && (l % p.bq) == 0) pb[(size_t)(l / p.bq) * T + j] = acc;
            if (valid && l > j) {
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < DH; ++c) s = fmaf(s_k[r][c], kj[c], s);
                acc += decay_var(s_rq[r], rkj, fmaf(al, s, be), variant);
            }
        }
    }
    if (valid && p.bfinal) p.bfinal[unit * T + j] = -acc;
}

// ------------------------------------------------------------------ fused forward
// grid (nqt, H, B), 256 threads = 16 x 16; 64 query rows x 64 keys per tile.  Thread
// (ty, tx) owns rows ty + 16*rr and columns tx + 16*cc (rr, cc < 4), which keeps the
// padded shared-memory reads conflict-free.
// FULL: an ablation variant or the chunked pruning is on.  Without it both fold away at
// compile time, so the method's own forward carries neither branch.
template <int DH, typename TI, bool FULL>
__global__ void __launch_bounds__(256) k_fwd_simt(FwdParams p) {
    const int variant = FULL ? p.variant : 0;
    const float prune_thr = FULL ? p.prune_thr : INFINITY;
    constexpr int BM = 64, BN = 64, LD = DH + 1, LP = BN + 1, ND = DH / 16;
    extern __shared__ float sm[];
    float* sQ = sm;
    float* sKq = sQ + BM * LD;
    float* sKh = sKq + BM * LD;
    float* sKr = sKh + BN * LD;
    float* sV = sKr + BN * LD;
    float* sL = sV + BN * LD;
    float* sP = sL + BM * LP;
    float* sRq = sP + BM * LP;
    float* sRk = sRq + BM;
    float* sPb = sRk + BN;
    float* sEv = sPb + BN;                            // 1: key evicted at this chunk's boundary

    const int T = p.T;
    const int qt = gridDim.x - 1 - blockIdx.x;        // heaviest (last) query tiles first
    const int h = blockIdx.y, b = blockIdx.z, kvh = h / p.G;
    const int i0 = qt * BM;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const size_t unit = (size_t)b * p.Hkv + kvh;
    const TI* vin = static_cast<const TI*>(p.v);
    const bool write_lambda = p.lambda_dbg != nullptr && (h % p.G) == 0;

    for (int e = tid; e < BM * DH; e += 256) {
        const int r = e / DH, c = e % DH, i = i0 + r;
        sQ[r * LD + c] = i < T ? p.qr[(((size_t)b * p.H + h) * T + i) * DH + c] : 0.f;
        sKq[r * LD + c] = i < T ? p.kh[(unit * T + i) * DH + c] : 0.f;
    }
    for (int r = tid; r < BM; r += 256) sRq[r] = (i0 + r < T) ? p.rq[unit * T + i0 + r] : 0.f;

    float m_r[4], l_r[4], acc[4][ND];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        m_r[rr] = -INFINITY;
        l_r[rr] = 0.f;
#pragma unroll
        for (int dd = 0; dd < ND; ++dd) acc[rr][dd] = 0.f;
    }
    const float al = p.alpha[kvh], be = p.beta[kvh];

    // tiles whose probabilities all underflow are skipped (not when the debug Lambda is written)
    const bool can_skip = p.qmax != nullptr && p.lambda_dbg == nullptr;
    const float thr = can_skip ? kSimtSkipMargin + 2.f * p.qmax[unit * p.nqt + qt] : 0.f;
    // Chunked pruned prefill: the 128-row chunk of this tile starts at query tile qt & ~1, and a
    // key before it is evicted when its bias there, -Pb, is below log p (Pb > prune_thr).
    const int qchunk = qt & ~1;
    for (int kt = 0; kt <= qt; ++kt) {
        const int j0 = kt * BN;
        const bool pruned_tile = FULL && kt < qchunk && prune_thr < INFINITY;
        __syncthreads();
        for (int c = tid; c < BN; c += 256) {
            const int j = j0 + c;
            sRk[c] = j < T ? p.rk[unit * T + j] : 0.f;
            sPb[c] = j < T ? p.pb[(unit * p.nqt + qt) * T + j] : 0.f;
            sEv[c] = (pruned_tile && j < T && p.pb[(unit * p.nqt + qchunk) * T + j] > prune_thr) ? 1.f : 0.f;
        }
        // skip when every key underflows, or (no debug Lambda to write) every key is evicted;
        // thread tid < BN votes on the entries it wrote itself
        if (__syncthreads_and(tid >= BN || (can_skip && sPb[tid] >= thr) ||
                              (pruned_tile && p.lambda_dbg == nullptr && sEv[tid] != 0.f)))
            continue;
        for (int e = tid; e < BN * DH; e += 256) {
            const int c = e / DH, x = e % DH, j = j0 + c;
            const bool ok = j < T;
            sKh[c * LD + x] = ok ? p.kh[(unit * T + j) * DH + x] : 0.f;
            sKr[c * LD + x] = ok ? p.kr[(unit * T + j) * DH + x] : 0.f;
            sV[c * LD + x] = ok ? Elem<TI>::ld(vin + (((size_t)b * T + j) * p.Hkv + kvh) * DH + x) : 0.f;
        }
        __syncthreads();
        // decay D[l = i0 + r, j = j0 + c]
        {
            float s[4][4];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) s[rr][cc] = 0.f;
            for (int x = 0; x < DH; ++x) {
                float a[4], bb[4];
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) a[rr] = sKq[(ty + 16 * rr) * LD + x];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) bb[cc] = sKh[(tx + 16 * cc) * LD + x];
#pragma unroll
                for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) s[rr][cc] = fmaf(a[rr], bb[cc], s[rr][cc]);
            }
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int r = ty + 16 * rr, c = tx + 16 * cc;
                    const int i = i0 + r, j = j0 + c;
                    float D = 0.f;
                    if (i > j && i < T && j < T) D = decay_var(sRq[r], sRk[c], fmaf(al, s[rr][cc], be), variant);
                    sL[r * LP + c] = D;
                }
        }
        __syncthreads();
        // in-tile causal accumulation on top of the boundary prefix
        if (tid < BN) {
            float a = sPb[tid];
            for (int r = 0; r < BM; ++r) {
                a += sL[r * LP + tid];
                sL[r * LP + tid] = -a;
            }
        }
        __syncthreads();
        float sc[4][4];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) sc[rr][cc] = 0.f;
        for (int x = 0; x < DH; ++x) {
            float a[4], bb[4];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) a[rr] = sQ[(ty + 16 * rr) * LD + x];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) bb[cc] = sKr[(tx + 16 * cc) * LD + x];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) sc[rr][cc] = fmaf(a[rr], bb[cc], sc[rr][cc]);
        }
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const int r = ty + 16 * rr, i = i0 + r;
            float mx = -INFINITY;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int c = tx + 16 * cc, j = j0 + c;
                const float lam = sL[r * LP + c];
                if (write_lambda && i < T && j < T)
                    p.lambda_dbg[(unit * T + i) * (size_t)T + j] = (j <= i) ? lam : 0.f;
                sc[rr][cc] = (j <= i && j < T && (!FULL || sEv[c] == 0.f)) ? fmaf(p.scale, sc[rr][cc], lam) : -INFINITY;
                mx = fmaxf(mx, sc[rr][cc]);
            }
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_new = fmaxf(m_r[rr], mx);
            // a row that has seen no visible key yet (every key so far evicted by the chunked
            // pruning) keeps m = -inf; subtracting 0 then gives exp(-inf) = 0, not a NaN
            const float m_use = m_new == -INFINITY ? 0.f : m_new;
            const float corr = expf(m_r[rr] - m_use);
            float rs = 0.f;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const float pe = expf(sc[rr][cc] - m_use);
                rs += pe;
                sP[r * LP + tx + 16 * cc] = pe;
            }
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
            l_r[rr] = l_r[rr] * corr + rs;
            m_r[rr] = m_new;
#pragma unroll
            for (int dd = 0; dd < ND; ++dd) acc[rr][dd] *= corr;
        }
        __syncthreads();
        for (int c = 0; c < BN; ++c) {
            float pv[4], vv[ND];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) pv[rr] = sP[(ty + 16 * rr) * LP + c];
#pragma unroll
            for (int dd = 0; dd < ND; ++dd) vv[dd] = sV[c * LD + tx + 16 * dd];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                for (int dd = 0; dd < ND; ++dd) acc[rr][dd] = fmaf(pv[rr], vv[dd], acc[rr][dd]);
        }
    }
    const TI* gin = static_cast<const TI*>(p.g);
    TI* out = static_cast<TI*>(p.o);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int i = i0 + ty + 16 * rr;
        if (i >= T) continue;
        const float inv = 1.f / l_r[rr];
#pragma unroll
        for (int dd = 0; dd < ND; ++dd) {
            const size_t off = (((size_t)b * T + i) * p.H + h) * DH + tx + 16 * dd;
            Elem<TI>::st(out + off, acc[rr][dd] * inv * sigmoid_f(Elem<TI>::ld(gin + off)));
        }
        if (tx == 0 && p.lse) p.lse[((size_t)b * p.H + h) * T + i] = m_r[rr] + logf(l_r[rr]);
    }
}

// ------------------------------------------------------------------ launchers
template <int DH>
static void prep_inst(const PrepParams& p, bool bf16_in, bool bf16_work, cudaStream_t s) {
    dim3 grid((p.T + kPrepTokens - 1) / kPrepTokens, p.B);
    if (bf16_in && bf16_work) k_prep<__nv_bfloat16, __nv_bfloat16, DH><<<grid, 256, 0, s>>>(p);
    else if (bf16_in) k_prep<__nv_bfloat16, float, DH><<<grid, 256, 0, s>>>(p);
    else if (bf16_work) k_prep<float, __nv_bfloat16, DH><<<grid, 256, 0, s>>>(p);
    else k_prep<float, float, DH><<<grid, 256, 0, s>>>(p);
}

cudaError_t launch_prep(const PrepParams& p, bool bf16_in, bool bf16_work, cudaStream_t s) {
    UA_PROFILE("k_prep", s);
    if (p.d == 64) prep_inst<64>(p, bf16_in, bf16_work, s);
    else prep_inst<128>(p, bf16_in, bf16_work, s);
    return cudaGetLastError();
}

cudaError_t launch_boundary_simt(const BoundaryParams& p, cudaStream_t s) {
    dim3 grid((p.T + 127) / 128, p.Hkv, p.B);
    UA_PROFILE("k_boundary_simt", s);
    if (p.variant != 0) {
        if (p.d == 64) k_boundary_simt<64, true><<<grid, 128, 0, s>>>(p);
        else k_boundary_simt<128, true><<<grid, 128, 0, s>>>(p);
    } else {
        if (p.d == 64) k_boundary_simt<64, false><<<grid, 128, 0, s>>>(p);
        else k_boundary_simt<128, false><<<grid, 128, 0, s>>>(p);
    }
    return cudaGetLastError();
}

template <int DH, typename TI, bool FULL>
static cudaError_t fwd_simt_launch(const FwdParams& p, cudaStream_t s) {
    constexpr int BM = 64, BN = 64, LD = DH + 1, LP = BN + 1;
    const size_t smem = sizeof(float) * (size_t)(2 * BM * LD + 3 * BN * LD + 2 * BM * LP + BM + 3 * BN);
    cudaError_t e = cudaFuncSetAttribute(k_fwd_simt<DH, TI, FULL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.nqt, p.H, p.B);
    UA_PROFILE("k_fwd_simt", s);
    k_fwd_simt<DH, TI, FULL><<<grid, 256, smem, s>>>(p);
    return cudaGetLastError();
}

template <int DH, typename TI>
static cudaError_t fwd_simt_inst(const FwdParams& p, cudaStream_t s) {
    const bool full = p.variant != 0 || p.prune_thr < INFINITY;
    return full ? fwd_simt_launch<DH, TI, true>(p, s) : fwd_simt_launch<DH, TI, false>(p, s);
}

cudaError_t launch_fwd_simt(const FwdParams& p, bool bf16_act, cudaStream_t s) {
    if (p.d == 64) return bf16_act ? fwd_simt_inst<64, __nv_bfloat16>(p, s) : fwd_simt_inst<64, float>(p, s);
    return bf16_act ? fwd_simt_inst<128, __nv_bfloat16>(p, s) : fwd_simt_inst<128, float>(p, s);
}

}  // namespace ua
