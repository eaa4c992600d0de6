// k_fwd_fix.cu -- exact recomputation of the rows the tensor-core forward could not normalise.
//
// The tensor-core forwards shift every softmax row by an a-priori bound (scale*||q||, the
// largest over the rows of a quarter and the G heads) instead of a running maximum, which keeps
// the row reductions off the transposed layout (paperlayer.ai summary App. C: the decay applied
// inside a fused online softmax).  A row whose true maximum lies far below that shift -- a large
// query norm with no well-aligned key, or a small-norm row sharing a quarter with a large one --
// would lose probability mass to fp32 underflow.  Such a row shows it in its normaliser: the
// forward lists every row whose shifted sum l is below 2^-60 (or not finite) instead of failing,
// and this kernel recomputes each listed row exactly, with a running maximum, in fp32 from the
// forward's own bf16 operands: l >= 2^-60 means the row maximum is at least 2^-73 after the
// shift, so whatever underflowed (below 2^-126) was below 2^-53 of it, T x 2^-53 at most in all.
//
// One listed row per CTA pass (grid-stride over the list; a launch with an empty list returns at
// once).  The decay of row i is Lambda_ij = -(Pb_t[j] + sum_{l = t*QT .. i, l > j} D[l, j]) with
// t = i / QT: the column prefix up to the row's query tile comes from the prefixes the forward
// published.  Those are exact when the forward evaluated every decay tile (b_final requested);
// otherwise they are lower bounds past the skip threshold for the skipped tiles, and the first
// CTA that needs a unit recomputes all its prefixes exactly (column sweeps, one thread per key)
// while the others wait for it (bounded).
#include <cuda.h>

#include "tc_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

using namespace tc;

namespace {

constexpr int kFixThreads = 256;

// D[l, j] in natural units from the log2 rates / 3 and the similarity logit x (fp32, accurate).
__device__ __forceinline__ float fix_decay(float lq2, float lk2, float x) {
    return exp2f(lq2 + lk2) * cbrtf(softplus_f(x));
}

template <int DH>
__device__ float dot_bf16_row(const __nv_bfloat16* a, const float* b) {
    float s = 0.f;
#pragma unroll 4
    for (int x = 0; x < DH; x += 8) {
        float v[8];
        Vec16<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(a + x), v);
#pragma unroll
        for (int e = 0; e < 8; ++e) s = fmaf(v[e], b[x + e], s);
    }
    return s;
}

// Exact inclusive column prefixes of one unit: for every query tile t and key j below its end,
// Pb[t][j] = sum_{j < l <= last row of t} D[l, j].
template <int DH>
__device__ void fix_unit_prefixes(const FixParams& p, int unit, float* s_k) {
    const int T = p.T;
    const __nv_bfloat16* kh = static_cast<const __nv_bfloat16*>(p.kh) + (size_t)unit * T * DH;
    const float* lq2 = p.lq2 + (size_t)unit * p.Tp;
    const float* lk2 = p.lk2 + (size_t)unit * p.Tp;
    const float al = p.alpha[unit % p.Hkv], be = p.beta[unit % p.Hkv];
    float* pin = p.pincl + (size_t)unit * p.nqt * p.Tpk;
    for (int j0 = 0; j0 < T; j0 += kFixThreads) {
        const int j = j0 + threadIdx.x;
        uint4 kj[DH / 8];                                 // this thread's key, bf16
#pragma unroll
        for (int x = 0; x < DH / 8; ++x)
            kj[x] = j < T ? reinterpret_cast<const uint4*>(kh + (size_t)j * DH)[x] : make_uint4(0, 0, 0, 0);
        float a = 0.f;
        const float lkj = j < T ? lk2[j] : 0.f;
        // rows from the first one below key j0 to the end, 32 at a time through shared memory
        for (int l0 = j0 + 1; l0 < T; l0 += 32) {
            __syncthreads();
            for (int e = threadIdx.x; e < 32 * DH; e += kFixThreads) {
                const int r = e / DH, x = e % DH, l = l0 + r;
                s_k[e] = l < T ? __bfloat162float(kh[(size_t)l * DH + x]) : 0.f;
            }
            __syncthreads();
            for (int r = 0; r < 32 && l0 + r < T; ++r) {
                const int l = l0 + r;
                if (j < T && l > j) {
                    float s = 0.f;
#pragma unroll
                    for (int x = 0; x < DH / 8; ++x) {
                        float kv[8];
                        Vec16<__nv_bfloat16>::unpack(kj[x], kv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) s = fmaf(s_k[r * DH + 8 * x + e], kv[e], s);
                    }
                    a += fix_decay(lq2[l], lkj, fmaf(al, s, be));
                }
                if (j < T && ((l + 1) % p.QT == 0 || l == T - 1)) {
                    const int t = l / p.QT;
                    if (l >= j) pin[(size_t)t * p.Tpk + j] = a;
                }
            }
        }
        if (j < T && j == T - 1) pin[(size_t)((T - 1) / p.QT) * p.Tpk + j] = 0.f;
    }
}

template <int DH>
__global__ void __launch_bounds__(kFixThreads) k_fwd_fix(FixParams p) {
    __shared__ float s_q[DH];
    __shared__ float s_red[kFixThreads / 32];
    __shared__ float s_acc[kFixThreads];
    __shared__ float s_k[4096];     // the row's tile rows (bf16 pairs, <= 16 KB) or 32 sweep rows (f32)
    __shared__ float s_lq[128];
    __shared__ int s_state;
    const unsigned count = *p.fix_count;
    if (count == 0) return;
    const int T = p.T, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (unsigned idx = blockIdx.x; idx < count; idx += gridDim.x) {
        const long long r = p.fix_list[idx];
        const int i = (int)(r % T);
        const long long bh = r / T;
        const int hq = (int)(bh % p.H), b = (int)(bh / p.H);
        const int kvh = hq / p.G, unit = b * p.Hkv + kvh;
        const int t = i / p.QT, r0 = t * p.QT;
        // ---- exact prefixes of the unit, if the forward may have passed lower bounds on
        if (!p.prefix_exact) {
            if (tid == 0) {
                unsigned st = atomicCAS(p.fix_state + unit, 0u, 1u);
                s_state = (int)st;
            }
            __syncthreads();
            if (s_state == 0) {
                fix_unit_prefixes<DH>(p, unit, s_k);
                __threadfence();
                __syncthreads();
                if (tid == 0) atomicExch(p.fix_state + unit, 2u);
            } else {
                if (tid == 0) {
                    const uint64_t t0 = globaltimer();
                    while (atomicAdd(p.fix_state + unit, 0u) != 2u) {
                        if (globaltimer() - t0 > wait_limit_ns()) {
                            raise_status(UA_ERR_TIMEOUT);
                            break;
                        }
                        __nanosleep(1000);
                    }
                }
                __syncthreads();
                __threadfence();
            }
        }
        // ---- the row's query, the tile's key rows and row rates
        const __nv_bfloat16* qr = static_cast<const __nv_bfloat16*>(p.qr) + (((size_t)b * p.H + hq) * T + i) * DH;
        const __nv_bfloat16* kh = static_cast<const __nv_bfloat16*>(p.kh) + (size_t)unit * T * DH;
        const __nv_bfloat16* kr = static_cast<const __nv_bfloat16*>(p.kr) + (size_t)unit * T * DH;
        const float* lq2 = p.lq2 + (size_t)unit * p.Tp;
        const float* lk2 = p.lk2 + (size_t)unit * p.Tp;
        const int nrow = i - r0 + 1;                      // rows of the tile up to and including i
        __nv_bfloat162* s_kt = reinterpret_cast<__nv_bfloat162*>(s_k);
        for (int e = tid; e < DH; e += kFixThreads) s_q[e] = __bfloat162float(qr[e]);
        for (int e = tid; e < nrow * DH / 2; e += kFixThreads)
            s_kt[e] = reinterpret_cast<const __nv_bfloat162*>(kh + (size_t)r0 * DH)[e];
        for (int e = tid; e < nrow; e += kFixThreads) s_lq[e] = lq2[r0 + e];
        __syncthreads();
        const float al = p.alpha[kvh], be = p.beta[kvh];
        const float* pin = p.pincl + ((size_t)unit * p.nqt + (t > 0 ? t - 1 : 0)) * p.Tpk;
        // chunked pruning decides at the start of the row's 128-row chunk, c0: the prefix published
        // by the query tile that ends there (the row's own tile's Pb when the tiles are 128 rows)
        const int c0 = (i / 128) * 128;
        const float* pinc = p.pincl + ((size_t)unit * p.nqt + (c0 > 0 ? c0 / p.QT - 1 : 0)) * p.Tpk;
        float* sc = p.scratch + (size_t)blockIdx.x * T;
        // ---- pass 1: logits (with the row's Lambda) and their maximum
        float mx = -INFINITY;
        for (int j = tid; j <= i; j += kFixThreads) {
            uint4 kj[DH / 8];                             // key j, bf16
#pragma unroll
            for (int x = 0; x < DH / 8; ++x) kj[x] = reinterpret_cast<const uint4*>(kh + (size_t)j * DH)[x];
            const bool before = j < r0;
            const float pb = before ? pin[j] : 0.f;
            float lg;
            if (j < c0 && pinc[j] > p.prune_thr) {
                lg = -INFINITY;                           // evicted at the chunk boundary
            } else {
                float a = pb;
                const float lkj = lk2[j];
                for (int rr = (before ? 0 : j - r0 + 1); rr < nrow; ++rr) {
                    float s = 0.f;
#pragma unroll
                    for (int x = 0; x < DH / 8; ++x) {
                        float kv[8];
                        Vec16<__nv_bfloat16>::unpack(kj[x], kv);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 kk = __bfloat1622float2(s_kt[rr * (DH / 2) + 4 * x + e]);
                            s = fmaf(kk.x, kv[2 * e], fmaf(kk.y, kv[2 * e + 1], s));
                        }
                    }
                    a += fix_decay(s_lq[rr], lkj, fmaf(al, s, be));
                }
                lg = fmaf(p.scale, dot_bf16_row<DH>(kr + (size_t)j * DH, s_q), -a);
            }
            sc[j] = lg;
            mx = fmaxf(mx, lg);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) s_red[warp] = mx;
        __syncthreads();
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kFixThreads / 32; ++w) M = fmaxf(M, s_red[w]);
        __syncthreads();
        // ---- pass 2: probabilities and their sum
        float ls = 0.f;
        for (int j = tid; j <= i; j += kFixThreads) {
            const float pe = expf(sc[j] - M);
            sc[j] = pe;
            ls += pe;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
        if (lane == 0) s_red[warp] = ls;
        __syncthreads();
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kFixThreads / 32; ++w) L += s_red[w];
        // ---- pass 3: weighted values (thread = head dim x, kFixThreads / DH groups of keys)
        const int x = tid % DH, grp = tid / DH;
        constexpr int NG = kFixThreads / DH;
        const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(p.v);
        float acc = 0.f;
        for (int j = grp; j <= i; j += NG)
            acc = fmaf(sc[j], __bfloat162float(v[(((size_t)b * T + j) * p.Hkv + kvh) * DH + x]), acc);
        s_acc[tid] = acc;
        __syncthreads();
        if (grp == 0) {
            float A = 0.f;
#pragma unroll
            for (int g2 = 0; g2 < NG; ++g2) A += s_acc[g2 * DH + x];
            const size_t off = (((size_t)b * T + i) * p.H + hq) * DH + x;
            const float gt = __bfloat162float(static_cast<const __nv_bfloat16*>(p.g)[off]);
            static_cast<__nv_bfloat16*>(p.o)[off] = __float2bfloat16_rn(A / L * sigmoid_f(gt));
        }
        if (tid == 0 && p.lse) p.lse[((size_t)b * p.H + hq) * T + i] = M + logf(L);
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_fwd_fix(const FixParams& p, int grid, cudaStream_t s) {
    UA_PROFILE("k_fwd_fix", s);
    if (p.d == 64) k_fwd_fix<64><<<grid, kFixThreads, 0, s>>>(p);
    else k_fwd_fix<128><<<grid, kFixThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace ua
