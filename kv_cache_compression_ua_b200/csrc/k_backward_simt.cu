// k_backward_simt.cu -- backward of the UA prefill (gradient of sum(dO * O) with respect to
// q, k, v, g, a_q, a_k, alpha, beta), fp32 SIMT, deterministic (no atomics).
//
// The pages describe custom training kernels with activation checkpointing: the quadratic
// decay mask is recomputed rather than stored (paperlayer.ai summary §4.2, App. C).  Here
// the forward's lse and the boundary prefixes Pb are the only saved statistics; D, Lambda, P
// and dS are recomputed tile by tile.
//
// Formulas (per KV group; s = scale, A = O / sigmoid(g) the ungated output):
//   dA = dO * sigmoid(g);  dg = dO * O * (1 - sigmoid(g));  Delta_i = sum_c dO_ic O_ic
//   P_ij = exp(s qrot_i.krot_j + Lambda_ij - lse_i);  dP_ij = dA_i . v_j
//   dS_ij = P_ij (dP_ij - Delta_i);  dLambda_ij = sum over the group's heads of dS_ij
//   dv_j = sum_i P_ij dA_i;  dkrot_j = s sum_i dS_ij qrot_i;  dqrot_i = s sum_j dS_ij krot_j
//   dD[l,j] = -sum_{i>=l} dLambda_ij;  w = dD * D / 3
//   da_q[l] = sum_j w sigmoid(a_q)/softplus(a_q);  da_k[j] = sum_l w sigmoid(a_k)/softplus(a_k)
//   dX = w sigmoid(X)/softplus(X), X = alpha c + beta, c = <khat_l, khat_j>
//   dalpha = sum dX c;  dbeta = sum dX;  dkhat_l += alpha sum_j dX khat_j;  dkhat_j += alpha sum_l dX khat_l
//   dq = RoPE^T dqrot;  dk = (dkhat + RoPE^T dkrot - khat <khat, .>) / ||k||
//
// Passes:
//   k_bwd_rowstats  Delta, dg
//   k_bwd_keys      per (batch, KV head, 32-key tile), query tiles from last to first:
//                   dv, dkrot, key-side decay terms (da_k, dkhat_j, dalpha, dbeta partials),
//                   and the suffix sums dPb_t[j] = sum_{i >= 64(t+1)} dLambda_ij
//   k_bwd_rows      per (batch, KV head, 64-row query tile), key tiles in order:
//                   dqrot for the G heads, row-side decay terms (da_q, dkhat_l)
//   k_bwd_post      RoPE^T, the normalisation Jacobian, casts, dalpha / dbeta reduction
#include "ua_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

namespace {
constexpr int BM = 64;    // query rows per tile
constexpr int BN = 32;    // keys per tile
constexpr int NT = 256;   // threads

// sigmoid(x) / softplus(x), the derivative of log(softplus(x)); 0 where softplus underflows
// (the decay it multiplies is then zero as well).
__device__ __forceinline__ float sig_over_sp(float x) {
    const float sp = softplus_f(x);
    return sp > 0.f ? sigmoid_f(x) / sp : 0.f;
}

template <int DH>
struct Tiles {
    static constexpr int LD = DH + 1;
    float* khq;   // [BM][LD] khat of the query rows
    float* khk;   // [BN][LD] khat of the keys
    float* krk;   // [BN][LD] RoPE(khat) of the keys
    float* vk;    // [BN][LD] values
    float* q;     // [BM][LD] RoPE(q) of one head
    float* da;    // [BM][LD] dA of one head
    float* D;     // [BM][BN+1] decay
    float* L;     // [BM][BN+1] Lambda
    float* P;     // [BM][BN+1] probabilities
    float* dS;    // [BM][BN+1]
    float* dL;    // [BM][BN+1] dLambda (summed over heads)
    float* rowv;  // [4][BM] rq, lse, delta, fq
    float* colv;  // [4][BN] rk, pb, fk, dpb
};

template <int DH>
__device__ __forceinline__ Tiles<DH> carve(float* sm) {
    constexpr int LD = DH + 1, LP = BN + 1;
    Tiles<DH> t;
    t.khq = sm; sm += BM * LD;
    t.khk = sm; sm += BN * LD;
    t.krk = sm; sm += BN * LD;
    t.vk = sm; sm += BN * LD;
    t.q = sm; sm += BM * LD;
    t.da = sm; sm += BM * LD;
    t.D = sm; sm += BM * LP;
    t.L = sm; sm += BM * LP;
    t.P = sm; sm += BM * LP;
    t.dS = sm; sm += BM * LP;
    t.dL = sm; sm += BM * LP;
    t.rowv = sm; sm += 4 * BM;
    t.colv = sm; sm += 4 * BN;
    return t;
}

template <int DH>
constexpr size_t tiles_bytes() {
    return sizeof(float) * ((size_t)(3 * BM + 3 * BN) * (DH + 1) + 5 * BM * (BN + 1) + 4 * BM + 4 * BN);
}

// thread (ty, tx) of 16 x 16 owns rows ty + 16 rr (rr < 4) and columns tx + 16 cc (cc < 2)
// of a BM x BN tile.
template <int DH>
__device__ __forceinline__ void tile_dots(const float* A, const float* Bm, int ty, int tx, float (&acc)[4][2]) {
    constexpr int LD = DH + 1;
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) acc[rr][cc] = 0.f;
    for (int x = 0; x < DH; ++x) {
        float a[4], b[2];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) a[rr] = A[(ty + 16 * rr) * LD + x];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) b[cc] = Bm[(tx + 16 * cc) * LD + x];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) acc[rr][cc] = fmaf(a[rr], b[cc], acc[rr][cc]);
    }
}

struct Ctx {
    int B, T, H, Hkv, d, G, nqt;
    float scale;
    const float *qr, *kh, *kr;
    const void *v, *g, *o, *d_o;
    const float *aq, *ak, *rq, *rk, *alpha, *beta, *lse, *delta, *pb;
    const float* qmax;   // [B,Hkv,nqt] tile row bounds, or NULL (no skipping)
    float *dpb, *dqr, *dkh_rows, *dkh_keys, *dkr, *dv32, *daq32, *dak32, *dab;
    int variant;         // UA_VAR_* bits
    float inv_n;         // 1 / number of decay mechanisms on (1/3 for the method itself)
};

// Decay tile D[l, j] and Lambda for query tile starting at i0 and key tile at j0.  Needs
// khq/khk/rowv(rq)/colv(rk, pb) loaded; leaves D and L filled.
template <int DH>
__device__ void decay_tile(const Tiles<DH>& t, int i0, int j0, int T, float al, float be, int variant, int ty, int tx,
                           int tid) {
    constexpr int LP = BN + 1;
    float acc[4][2];
    tile_dots<DH>(t.khq, t.khk, ty, tx, acc);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int r = ty + 16 * rr, c = tx + 16 * cc, i = i0 + r, j = j0 + c;
            float D = 0.f;
            if (i > j && i < T && j < T) D = decay_var(t.rowv[r], t.colv[c], fmaf(al, acc[rr][cc], be), variant);
            t.D[r * LP + c] = D;
        }
    __syncthreads();
    if (tid < BN) {
        float a = t.colv[BN + tid];   // pb
        for (int r = 0; r < BM; ++r) {
            a += t.D[r * LP + tid];
            t.L[r * LP + tid] = -a;
        }
    }
    __syncthreads();
}

// P and dS for one head (q, da, rowv(lse, delta) loaded); accumulates dL.
template <int DH>
__device__ void head_tile(const Tiles<DH>& t, int i0, int j0, int T, float scale, int ty, int tx, bool first_head) {
    constexpr int LP = BN + 1;
    float s[4][2], dp[4][2];
    tile_dots<DH>(t.q, t.krk, ty, tx, s);
    tile_dots<DH>(t.da, t.vk, ty, tx, dp);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int r = ty + 16 * rr, c = tx + 16 * cc, i = i0 + r, j = j0 + c;
            float P = 0.f;
            if (j <= i && i < T && j < T) P = expf(fmaf(scale, s[rr][cc], t.L[r * LP + c]) - t.rowv[BM + r]);
            const float dS = P * (dp[rr][cc] - t.rowv[2 * BM + r]);
            t.P[r * LP + c] = P;
            t.dS[r * LP + c] = dS;
            t.dL[r * LP + c] = first_head ? dS : t.dL[r * LP + c] + dS;
        }
}

template <typename TI, int DH>
__device__ void load_rows(float* dst, const TI* src_base, size_t row_stride, int i0, int T, int tid) {
    constexpr int LD = DH + 1;
    for (int e = tid; e < BM * DH; e += NT) {
        const int r = e / DH, x = e % DH, i = i0 + r;
        dst[r * LD + x] = i < T ? Elem<TI>::ld(src_base + (size_t)i * row_stride + x) : 0.f;
    }
}

}  // namespace

// ------------------------------------------------------------------ row statistics
// grid (T, B), 128 threads: Delta = sum dO*O per (b, h, t) and dg = dO * O * (1 - sigmoid(g)).
template <typename TI>
__global__ void __launch_bounds__(128) k_bwd_rowstats(Ctx c) {
    const int t = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const TI* o = static_cast<const TI*>(c.o);
    const TI* dO = static_cast<const TI*>(c.d_o);
    const TI* g = static_cast<const TI*>(c.g);
    for (int h = warp; h < c.H; h += 4) {
        const size_t base = (((size_t)b * c.T + t) * c.H + h) * c.d;
        float acc = 0.f;
        for (int x = lane; x < c.d; x += 32) acc = fmaf(Elem<TI>::ld(dO + base + x), Elem<TI>::ld(o + base + x), acc);
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
        if (lane == 0) const_cast<float*>(c.delta)[((size_t)b * c.H + h) * c.T + t] = acc;
    }
}

// ------------------------------------------------------------------ key-side pass
// grid (ceil(T/BN), Hkv, B), 256 threads.
template <typename TI, int DH>
__global__ void __launch_bounds__(NT) k_bwd_keys(Ctx c) {
    extern __shared__ float sm[];
    constexpr int LD = DH + 1, LP = BN + 1;
    constexpr int ND = DH / 8;                        // dims per thread in the key accumulators
    Tiles<DH> t = carve<DH>(sm);
    const int T = c.T;
    const int kt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int j0 = kt * BN;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const size_t unit = (size_t)b * c.Hkv + kvh;
    const float al = c.alpha[kvh], be = c.beta[kvh];
    const bool sim_on = !(c.variant & kVarNoSim);   // similarity mechanism on: dX terms exist
    const TI* vin = static_cast<const TI*>(c.v);
    const TI* gin = static_cast<const TI*>(c.g);
    const TI* doin = static_cast<const TI*>(c.d_o);

    for (int e = tid; e < BN * DH; e += NT) {
        const int cc = e / DH, x = e % DH, j = j0 + cc;
        const bool ok = j < T;
        t.khk[cc * LD + x] = ok ? c.kh[(unit * T + j) * DH + x] : 0.f;
        t.krk[cc * LD + x] = ok ? c.kr[(unit * T + j) * DH + x] : 0.f;
        t.vk[cc * LD + x] = ok ? Elem<TI>::ld(vin + (((size_t)b * T + j) * c.Hkv + kvh) * DH + x) : 0.f;
    }
    if (tid < BN) {
        const int j = j0 + tid;
        t.colv[tid] = j < T ? c.rk[unit * T + j] : 0.f;
        // d log r_k / d a_k; zero when the key mechanism is off (r_k is then the constant 1)
        t.colv[2 * BN + tid] = j < T && !(c.variant & kVarNoK) ? sig_over_sp(c.ak[((size_t)b * T + j) * c.Hkv + kvh]) : 0.f;
    }
    // key accumulators: thread owns key kc = tid / 8 and dims (tid % 8) + 8 m
    const int kc = tid >> 3, kd = tid & 7;
    float aV[ND], aKr[ND], aKh[ND];
#pragma unroll
    for (int m = 0; m < ND; ++m) aV[m] = aKr[m] = aKh[m] = 0.f;
    float sdl = 0.f;                                  // thread tid < BN: suffix of dLambda for key tid
    float dak = 0.f, dal = 0.f, dbe = 0.f;

    const int t_first = j0 / BM;                      // query tiles that reach this key tile
    for (int qt = c.nqt - 1; qt >= t_first; --qt) {
        const int i0 = qt * BM;
        __syncthreads();
        load_rows<float, DH>(t.khq, c.kh + unit * T * DH, DH, i0, T, tid);
        if (tid < BM) {
            const int i = i0 + tid;
            t.rowv[tid] = i < T ? c.rq[unit * T + i] : 0.f;
        }
        if (tid < BN) {
            const int j = j0 + tid;
            t.colv[BN + tid] = j < T ? c.pb[(unit * c.nqt + qt) * T + j] : 0.f;
            if (j < T) c.dpb[(unit * c.nqt + qt) * T + j] = sdl;   // sum of dLambda over rows >= 64(qt+1)
        }
        // Nothing of this (query tile, key tile) reaches any gradient when every probability
        // underflows (then dS = dLambda = 0 here) and the later query tiles fed no dLambda into
        // these keys (then dD = 0 here too): skip it.
        if (c.qmax) {
            const float thr = kSimtSkipMargin + 2.f * c.qmax[unit * c.nqt + qt];
            if (__syncthreads_and(tid >= BN || (t.colv[BN + tid] >= thr && sdl == 0.f))) continue;
        } else {
            __syncthreads();
        }
        decay_tile<DH>(t, i0, j0, T, al, be, c.variant, ty, tx, tid);
        for (int hh = 0; hh < c.G; ++hh) {
            const int h = kvh * c.G + hh;
            __syncthreads();
            load_rows<float, DH>(t.q, c.qr + ((size_t)b * c.H + h) * T * DH, DH, i0, T, tid);
            for (int e = tid; e < BM * DH; e += NT) {
                const int r = e / DH, x = e % DH, i = i0 + r;
                float v = 0.f;
                if (i < T) {
                    const size_t off = (((size_t)b * T + i) * c.H + h) * DH + x;
                    v = Elem<TI>::ld(doin + off) * sigmoid_f(Elem<TI>::ld(gin + off));
                }
                t.da[r * LD + x] = v;
            }
            if (tid < BM) {
                const int i = i0 + tid;
                t.rowv[BM + tid] = i < T ? c.lse[((size_t)b * c.H + h) * T + i] : 0.f;
                t.rowv[2 * BM + tid] = i < T ? c.delta[((size_t)b * c.H + h) * T + i] : 0.f;
            }
            __syncthreads();
            head_tile<DH>(t, i0, j0, T, c.scale, ty, tx, hh == 0);
            __syncthreads();
            // dv_j += sum_i P_ij dA_i ; dkrot_j += s sum_i dS_ij qrot_i
            for (int r = 0; r < BM; ++r) {
                const float p = t.P[r * LP + kc], ds = t.dS[r * LP + kc];
#pragma unroll
                for (int m = 0; m < ND; ++m) {
                    const int x = kd + 8 * m;
                    aV[m] = fmaf(p, t.da[r * LD + x], aV[m]);
                    aKr[m] = fmaf(ds, t.q[r * LD + x], aKr[m]);
                }
            }
        }
        __syncthreads();
        // dD from the suffix of dLambda (bottom row up), then the decay derivatives
        if (tid < BN) {
            const int j = j0 + tid;
            for (int r = BM - 1; r >= 0; --r) {
                sdl += t.dL[r * LP + tid];
                const int i = i0 + r;
                const float D = t.D[r * LP + tid];
                // w = dD * D / n with dD = -sdl (n mechanisms on); stored in dS for the dX pass below
                t.dS[r * LP + tid] = (i > j && D > 0.f) ? -sdl * D * c.inv_n : 0.f;
            }
        }
        __syncthreads();
        {
            float acc[4][2];
            tile_dots<DH>(t.khq, t.khk, ty, tx, acc);   // similarities again
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int r = ty + 16 * rr, cl = tx + 16 * cc;
                    const float w = t.dS[r * LP + cl];
                    const float X = fmaf(al, acc[rr][cc], be);
                    const float dX = w != 0.f && sim_on ? w * sig_over_sp(X) : 0.f;
                    dal = fmaf(dX, acc[rr][cc], dal);
                    dbe += dX;
                    t.P[r * LP + cl] = dX;                // reuse P for dX
                }
        }
        __syncthreads();
        for (int r = 0; r < BM; ++r) {
            const float dX = t.P[r * LP + kc];
#pragma unroll
            for (int m = 0; m < ND; ++m) aKh[m] = fmaf(dX, t.khq[r * LD + kd + 8 * m], aKh[m]);
        }
        if (tid < BN) {
            float s = 0.f;
            for (int r = 0; r < BM; ++r) s += t.dS[r * LP + tid];
            dak += s * t.colv[2 * BN + tid];
        }
    }
    // write key-side results
    const int j = j0 + kc;
    if (j < T) {
#pragma unroll
        for (int m = 0; m < ND; ++m) {
            const int x = kd + 8 * m;
            const size_t off = (unit * T + j) * DH + x;
            c.dv32[off] = aV[m];
            c.dkr[off] = c.scale * aKr[m];
            c.dkh_keys[off] = al * aKh[m];
        }
    }
    if (tid < BN && j0 + tid < T) c.dak32[unit * T + j0 + tid] = dak;
    // dalpha / dbeta partials: block reduction
    __shared__ float red[2][NT / 32];
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
        dal += __shfl_xor_sync(0xffffffffu, dal, s);
        dbe += __shfl_xor_sync(0xffffffffu, dbe, s);
    }
    if ((tid & 31) == 0) {
        red[0][tid >> 5] = dal;
        red[1][tid >> 5] = dbe;
    }
    __syncthreads();
    if (tid == 0) {
        float a = 0.f, bb = 0.f;
        for (int w = 0; w < NT / 32; ++w) {
            a += red[0][w];
            bb += red[1][w];
        }
        const size_t cta = (unit * gridDim.x + kt) * 2;
        c.dab[cta] = a;
        c.dab[cta + 1] = bb;
    }
}

// ------------------------------------------------------------------ row-side pass
// grid (nqt, Hkv, B), 256 threads.  Accumulates dqrot of the G heads and the row-side decay
// terms for one 64-row query tile.
template <typename TI, int DH, int G>
__global__ void __launch_bounds__(NT) k_bwd_rows(Ctx c) {
    extern __shared__ float sm[];
    constexpr int LD = DH + 1, LP = BN + 1;
    constexpr int ND = DH / 16;                       // dims per thread: rows ty + 16 rr, dims tx + 16 m
    Tiles<DH> t = carve<DH>(sm);
    const int T = c.T;
    const int qt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int i0 = qt * BM;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const size_t unit = (size_t)b * c.Hkv + kvh;
    const float al = c.alpha[kvh], be = c.beta[kvh];
    const bool sim_on = !(c.variant & kVarNoSim);   // similarity mechanism on: dX terms exist
    const TI* vin = static_cast<const TI*>(c.v);
    const TI* gin = static_cast<const TI*>(c.g);
    const TI* doin = static_cast<const TI*>(c.d_o);

    load_rows<float, DH>(t.khq, c.kh + unit * T * DH, DH, i0, T, tid);
    if (tid < BM) {
        const int i = i0 + tid;
        t.rowv[tid] = i < T ? c.rq[unit * T + i] : 0.f;
        t.rowv[3 * BM + tid] = i < T && !(c.variant & kVarNoQ) ? sig_over_sp(c.aq[((size_t)b * T + i) * c.Hkv + kvh]) : 0.f;
    }
    float aQ[G][4][ND], aKh[4][ND], daq[4];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        daq[rr] = 0.f;
#pragma unroll
        for (int m = 0; m < ND; ++m) {
            aKh[rr][m] = 0.f;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) aQ[hh][rr][m] = 0.f;
        }
    }
    const int nkt = (min(T, i0 + BM) + BN - 1) / BN;  // key tiles up to the diagonal
    for (int kt = 0; kt < nkt; ++kt) {
        const int j0 = kt * BN;
        __syncthreads();
        for (int e = tid; e < BN * DH; e += NT) {
            const int cc = e / DH, x = e % DH, j = j0 + cc;
            const bool ok = j < T;
            t.khk[cc * LD + x] = ok ? c.kh[(unit * T + j) * DH + x] : 0.f;
            t.krk[cc * LD + x] = ok ? c.kr[(unit * T + j) * DH + x] : 0.f;
            t.vk[cc * LD + x] = ok ? Elem<TI>::ld(vin + (((size_t)b * T + j) * c.Hkv + kvh) * DH + x) : 0.f;
        }
        if (tid < BN) {
            const int j = j0 + tid;
            t.colv[tid] = j < T ? c.rk[unit * T + j] : 0.f;
            t.colv[BN + tid] = j < T ? c.pb[(unit * c.nqt + qt) * T + j] : 0.f;
            t.colv[3 * BN + tid] = j < T ? c.dpb[(unit * c.nqt + qt) * T + j] : 0.f;
        }
        // as in the key pass: no probability survives and no dLambda arrives from later rows
        if (c.qmax) {
            const float thr = kSimtSkipMargin + 2.f * c.qmax[unit * c.nqt + qt];
            if (__syncthreads_and(tid >= BN || (t.colv[BN + tid] >= thr && t.colv[3 * BN + tid] == 0.f))) continue;
        } else {
            __syncthreads();
        }
        decay_tile<DH>(t, i0, j0, T, al, be, c.variant, ty, tx, tid);
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            const int h = kvh * G + hh;
            __syncthreads();
            load_rows<float, DH>(t.q, c.qr + ((size_t)b * c.H + h) * T * DH, DH, i0, T, tid);
            for (int e = tid; e < BM * DH; e += NT) {
                const int r = e / DH, x = e % DH, i = i0 + r;
                float v = 0.f;
                if (i < T) {
                    const size_t off = (((size_t)b * T + i) * c.H + h) * DH + x;
                    v = Elem<TI>::ld(doin + off) * sigmoid_f(Elem<TI>::ld(gin + off));
                }
                t.da[r * LD + x] = v;
            }
            if (tid < BM) {
                const int i = i0 + tid;
                t.rowv[BM + tid] = i < T ? c.lse[((size_t)b * c.H + h) * T + i] : 0.f;
                t.rowv[2 * BM + tid] = i < T ? c.delta[((size_t)b * c.H + h) * T + i] : 0.f;
            }
            __syncthreads();
            head_tile<DH>(t, i0, j0, T, c.scale, ty, tx, hh == 0);
            __syncthreads();
            // dqrot_i += s sum_j dS_ij krot_j
            for (int cl = 0; cl < BN; ++cl) {
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const float ds = t.dS[(ty + 16 * rr) * LP + cl];
#pragma unroll
                    for (int m = 0; m < ND; ++m) aQ[hh][rr][m] = fmaf(ds, t.krk[cl * LD + tx + 16 * m], aQ[hh][rr][m]);
                }
            }
        }
        __syncthreads();
        // dD[l, j] = -(dPb_t[j] + sum over rows i >= l of this tile of dLambda_ij)
        if (tid < BN) {
            const int j = j0 + tid;
            float sd = t.colv[3 * BN + tid];
            for (int r = BM - 1; r >= 0; --r) {
                sd += t.dL[r * LP + tid];
                const int i = i0 + r;
                const float D = t.D[r * LP + tid];
                t.dS[r * LP + tid] = (i > j && D > 0.f) ? -sd * D * c.inv_n : 0.f;   // w
            }
        }
        __syncthreads();
        {
            float acc[4][2];
            tile_dots<DH>(t.khq, t.khk, ty, tx, acc);
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int r = ty + 16 * rr, cl = tx + 16 * cc;
                    const float w = t.dS[r * LP + cl];
                    const float X = fmaf(al, acc[rr][cc], be);
                    t.P[r * LP + cl] = w != 0.f && sim_on ? w * sig_over_sp(X) : 0.f;   // dX
                }
        }
        __syncthreads();
        for (int cl = 0; cl < BN; ++cl) {
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                const int r = ty + 16 * rr;
                const float dX = t.P[r * LP + cl];
                if (tx == 0) daq[rr] += t.dS[r * LP + cl];
#pragma unroll
                for (int m = 0; m < ND; ++m) aKh[rr][m] = fmaf(dX, t.khk[cl * LD + tx + 16 * m], aKh[rr][m]);
            }
        }
    }
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int r = ty + 16 * rr, i = i0 + r;
        if (i >= T) continue;
#pragma unroll
        for (int m = 0; m < ND; ++m) {
            const int x = tx + 16 * m;
            c.dkh_rows[(unit * T + i) * DH + x] = al * aKh[rr][m];
#pragma unroll
            for (int hh = 0; hh < G; ++hh)
                c.dqr[(((size_t)b * c.H + kvh * G + hh) * T + i) * DH + x] = c.scale * aQ[hh][rr][m];
        }
        if (tx == 0) c.daq32[unit * T + i] = daq[rr] * t.rowv[3 * BM + r];
    }
}

// ------------------------------------------------------------------ post pass
// grid (T, B), 256 threads: RoPE^T of dqrot / dkrot, normalisation Jacobian, casts.
template <typename TI>
__global__ void __launch_bounds__(256) k_bwd_post(Ctx c, BwdParams p) {
    const int t = blockIdx.x, b = blockIdx.y;
    const int d = c.d, half = d / 2, T = c.T;
    __shared__ float s_cos[64], s_sin[64];
    for (int m = threadIdx.x; m < half; m += blockDim.x) rope_cs((double)t, p.rf.f[m], &s_cos[m], &s_sin[m]);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    TI* dq = static_cast<TI*>(p.dq);
    TI* dk = static_cast<TI*>(p.dk);
    TI* dv = static_cast<TI*>(p.dv);
    const TI* kin = static_cast<const TI*>(p.k);
    for (int hh = warp; hh < c.H + c.Hkv; hh += 8) {
        const bool is_q = hh < c.H;
        const int h = is_q ? hh : hh - c.H;
        if (is_q && !(p.variant & kVarQNorm)) {
            const float* src = c.dqr + (((size_t)b * c.H + h) * T + t) * d;
            TI* dst = dq + (((size_t)b * T + t) * c.H + h) * d;
            for (int m = lane; m < half; m += 32) {
                const float x0 = src[m], x1 = src[m + half], cs = s_cos[m], sn = s_sin[m];
                Elem<TI>::st(dst + m, x0 * cs + x1 * sn);          // rotation by -angle
                Elem<TI>::st(dst + m + half, x1 * cs - x0 * sn);
            }
        } else if (is_q) {
            // query norm q' = r q, r = 1/sqrt(mean(q^2) + eps):  dq = r (dq' - q' <q', dq'> / d),
            // dq' = RoPE^T dqrot
            const float* src = c.dqr + (((size_t)b * c.H + h) * T + t) * d;
            const TI* qraw = static_cast<const TI*>(p.q) + (((size_t)b * T + t) * c.H + h) * d;
            TI* dst = dq + (((size_t)b * T + t) * c.H + h) * d;
            float y0[2] = {0.f, 0.f}, y1[2] = {0.f, 0.f}, q0[2] = {0.f, 0.f}, q1[2] = {0.f, 0.f};
            float ss = 0.f, qy = 0.f;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int m = lane + 32 * u;
                if (m < half) {
                    const float x0 = src[m], x1 = src[m + half], cs = s_cos[m], sn = s_sin[m];
                    y0[u] = x0 * cs + x1 * sn;
                    y1[u] = x1 * cs - x0 * sn;
                    q0[u] = Elem<TI>::ld(qraw + m);
                    q1[u] = Elem<TI>::ld(qraw + m + half);
                    ss += q0[u] * q0[u] + q1[u] * q1[u];
                    qy += q0[u] * y0[u] + q1[u] * y1[u];
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                ss += __shfl_xor_sync(0xffffffffu, ss, o);
                qy += __shfl_xor_sync(0xffffffffu, qy, o);
            }
            const float r = 1.f / sqrtf(ss / (float)d + kQNormEps);
            const float k = r * r * qy / (float)d;        // <q', dq'> / d, divided by r once more
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int m = lane + 32 * u;
                if (m < half) {
                    Elem<TI>::st(dst + m, r * (y0[u] - q0[u] * k));
                    Elem<TI>::st(dst + m + half, r * (y1[u] - q1[u] * k));
                }
            }
        } else {
            const size_t u = (size_t)b * c.Hkv + h;
            const float* rot = c.dkr + (u * T + t) * d;
            const float* a1 = c.dkh_keys + (u * T + t) * d;
            const float* a2 = c.dkh_rows + (u * T + t) * d;
            const float* khat = c.kh + (u * T + t) * d;
            float g0[2] = {0.f, 0.f}, g1[2] = {0.f, 0.f};
            float proj = 0.f, ss = 0.f;
            const TI* kr = kin + (((size_t)b * T + t) * c.Hkv + h) * d;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int m = lane + 32 * q;
                if (m < half) {
                    const float cs = s_cos[m], sn = s_sin[m];
                    g0[q] = a1[m] + a2[m] + rot[m] * cs + rot[m + half] * sn;
                    g1[q] = a1[m + half] + a2[m + half] + rot[m + half] * cs - rot[m] * sn;
                    proj += g0[q] * khat[m] + g1[q] * khat[m + half];
                    const float k0 = Elem<TI>::ld(kr + m), k1 = Elem<TI>::ld(kr + m + half);
                    ss += k0 * k0 + k1 * k1;
                }
            }
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) {
                proj += __shfl_xor_sync(0xffffffffu, proj, s);
                ss += __shfl_xor_sync(0xffffffffu, ss, s);
            }
            const float n = sqrtf(ss);
            TI* dst = dk + (((size_t)b * T + t) * c.Hkv + h) * d;
            TI* dvd = dv + (((size_t)b * T + t) * c.Hkv + h) * d;
            const float* dvs = c.dv32 + (u * T + t) * d;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int m = lane + 32 * q;
                if (m < half) {
                    if (n > 1e-12f) {
                        Elem<TI>::st(dst + m, (g0[q] - khat[m] * proj) / n);
                        Elem<TI>::st(dst + m + half, (g1[q] - khat[m + half] * proj) / n);
                    } else {
                        Elem<TI>::st(dst + m, g0[q] / 1e-12f);
                        Elem<TI>::st(dst + m + half, g1[q] / 1e-12f);
                    }
                    Elem<TI>::st(dvd + m, dvs[m]);
                    Elem<TI>::st(dvd + m + half, dvs[m + half]);
                }
            }
        }
    }
    for (int h = threadIdx.x; h < c.Hkv; h += blockDim.x) {
        const size_t u = (size_t)b * c.Hkv + h;
        p.da_q[((size_t)b * T + t) * c.Hkv + h] = c.daq32[u * T + t];
        p.da_k[((size_t)b * T + t) * c.Hkv + h] = c.dak32[u * T + t];
    }
    // dg = dO * O * (1 - sigmoid(g))
    const TI* o = static_cast<const TI*>(c.o);
    const TI* dO = static_cast<const TI*>(c.d_o);
    const TI* g = static_cast<const TI*>(c.g);
    TI* dg = static_cast<TI*>(p.dg);
    const size_t base = ((size_t)b * T + t) * c.H * d;
    for (int e = threadIdx.x; e < c.H * d; e += blockDim.x)
        Elem<TI>::st(dg + base + e, Elem<TI>::ld(dO + base + e) * Elem<TI>::ld(o + base + e) *
                                        (1.f - sigmoid_f(Elem<TI>::ld(g + base + e))));
}

// dalpha / dbeta: sum the per-CTA partials of every batch for each KV head.
__global__ void k_bwd_dab(const float* dab, int B, int Hkv, int nkt, float* dalpha, float* dbeta) {
    const int h = blockIdx.x;
    float a = 0.f, bb = 0.f;
    for (int e = threadIdx.x; e < B * nkt; e += blockDim.x) {
        const int b = e / nkt, kt = e % nkt;
        const size_t cta = (((size_t)b * Hkv + h) * nkt + kt) * 2;
        a += dab[cta];
        bb += dab[cta + 1];
    }
    __shared__ float ra[256], rb[256];
    ra[threadIdx.x] = a;
    rb[threadIdx.x] = bb;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) {
            ra[threadIdx.x] += ra[threadIdx.x + s];
            rb[threadIdx.x] += rb[threadIdx.x + s];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        dalpha[h] = ra[0];
        dbeta[h] = rb[0];
    }
}

// ------------------------------------------------------------------ launcher
template <typename TI, int DH, int G>
static cudaError_t bwd_inst(const BwdParams& p, cudaStream_t s) {
    Ctx c;
    c.B = p.B; c.T = p.T; c.H = p.H; c.Hkv = p.Hkv; c.d = p.d; c.G = p.G; c.nqt = p.nqt; c.scale = p.scale;
    c.qr = p.qr; c.kh = p.kh; c.kr = p.kr; c.v = p.v; c.g = p.g; c.o = p.o; c.d_o = p.d_o;
    c.aq = p.a_q; c.ak = p.a_k; c.rq = p.rq; c.rk = p.rk; c.alpha = p.alpha; c.beta = p.beta; c.lse = p.lse;
    c.delta = p.delta; c.pb = p.pb; c.qmax = p.qmax; c.dpb = p.dpb; c.dqr = p.dqr; c.dkh_rows = p.dkh_rows; c.dkh_keys = p.dkh;
    c.dkr = p.dkr; c.dv32 = p.dv32; c.daq32 = p.daq32; c.dak32 = p.dak32; c.dab = p.dab;
    c.variant = p.variant; c.inv_n = var_inv_n(p.variant);
    const size_t smem = tiles_bytes<DH>();
    cudaError_t e;
    {
        UA_PROFILE("k_bwd_rowstats", s);
        k_bwd_rowstats<TI><<<dim3(p.T, p.B), 128, 0, s>>>(c);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k_bwd_keys<TI, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    {
        UA_PROFILE("k_bwd_keys", s);
        k_bwd_keys<TI, DH><<<dim3(p.nkt, p.Hkv, p.B), NT, smem, s>>>(c);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k_bwd_rows<TI, DH, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
        return e;
    {
        UA_PROFILE("k_bwd_rows", s);
        k_bwd_rows<TI, DH, G><<<dim3(p.nqt, p.Hkv, p.B), NT, smem, s>>>(c);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        UA_PROFILE("k_bwd_post", s);
        k_bwd_post<TI><<<dim3(p.T, p.B), 256, 0, s>>>(c, p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        UA_PROFILE("k_bwd_dab", s);
        k_bwd_dab<<<p.Hkv, 256, 0, s>>>(p.dab, p.B, p.Hkv, p.nkt, p.dalpha, p.dbeta);
    }
    return cudaGetLastError();
}

template <typename TI, int DH>
static cudaError_t bwd_g(const BwdParams& p, cudaStream_t s) {
    switch (p.G) {
        case 1: return bwd_inst<TI, DH, 1>(p, s);
        case 2: return bwd_inst<TI, DH, 2>(p, s);
        case 3: return bwd_inst<TI, DH, 3>(p, s);
        case 4: return bwd_inst<TI, DH, 4>(p, s);
        case 8: return bwd_inst<TI, DH, 8>(p, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_bwd_simt(const BwdParams& p, bool bf16_act, cudaStream_t s) {
    if (bf16_act) return p.d == 64 ? bwd_g<__nv_bfloat16, 64>(p, s) : bwd_g<__nv_bfloat16, 128>(p, s);
    return p.d == 64 ? bwd_g<float, 64>(p, s) : bwd_g<float, 128>(p, s);
}

}  // namespace ua
