// k_backward_tc.cu -- backward of the bf16 UA prefill on the tensor cores (tcgen05 / TMEM / TMA).
//
// The pages describe custom training kernels with activation checkpointing: the decay mask is
// recomputed, not stored (paperlayer.ai summary §4.2, App. C, App. H).  Here the forward's lse is
// the only saved statistic; the decay D, Lambda, P and dS are recomputed tile by tile.
//
// Formulas (per KV group; s = scale, dA = dO * sigmoid(g)):
//   P_ij = exp(s qrot_i.krot_j + Lambda_ij - lse_i);  dP_ij = dA_i . v_j;  dZ_ij = P_ij (dP_ij - Delta_i)
//   dv_j = sum_i P_ij dA_i;  dkrot_j = s sum_i dZ_ij qrot_i;  dqrot_i = s sum_j dZ_ij krot_j
//   dLambda_ij = sum over the G heads of dZ_ij;  dD[l,j] = -sum_{i>=l} dLambda_ij;  w = dD D / 3
//   da_q[l] = sum_j w sigmoid(a_q)/softplus(a_q);  da_k[j] = sum_l w sigmoid(a_k)/softplus(a_k)
//   dX = w sigmoid(X)/softplus(X), X = alpha c + beta, c = <khat_l, khat_j>
//   dalpha = sum dX c;  dbeta = sum dX;  dkhat_l += alpha sum_j dX khat_j;  dkhat_j += alpha sum_l dX khat_l
//
// Passes (rows in 32-row steps, keys in 128-key tiles, everything in the forward's transposed
// layout: one thread per key, which scans its key column in registers):
//   k_bwd_prep_tc    dA (bf16 operand), Delta, lse in log2 units
//   k_bwd_bound_tc   per (batch, KV head, key tile), steps top-down: the decay prefix Pb above
//                    every step (X^T on the tensor cores)
//   k_bwd_key_tc     per (batch, KV head, key tile), steps bottom-up: X^T, S_h^T and dP_h^T on the
//                    tensor cores; decay, P, dZ, the dD suffix scan, w and dX per thread; dv and
//                    dkrot accumulated in TMEM (P_h^T dA_h, dZ_h^T qrot_h); the key-side decay
//                    sums; the row sums of w per key tile; dZ_h^T and dX^T stored as bf16 tiles
//   k_bwd_rowgemm_tc per (batch, KV head, 128-row block, output): dqrot_h = s dZ_h krot and the
//                    row-side dkhat = alpha dX khat, summed over key tiles in a fixed order
//   k_bwd_keygemm_tc per (batch, KV head, key tile): the key-side dkhat = alpha dX^T khat
//   k_bwd_post_tc    RoPE^T, the normalisation Jacobians, casts, da_q / da_k
// Every sum runs in a fixed order (no atomics), so the result is deterministic.
#include <type_traits>
#include <cudaTypedefs.h>

#include "tc_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

using namespace tc;

namespace {
constexpr float kL2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kCbrtLn2b = 0.8849970445005177f;   // (ln 2)^(1/3), the decay's log2-unit factor
constexpr int ST = 32;                              // rows per step
constexpr uint32_t kTileBytes = 128 * ST * 2;       // one stored bf16 tile: 128 keys x 32 rows

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_bwd() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// bf16 [outer][T][d], box = 64 columns x `rows` rows x 1, 128-byte swizzle.
bool map_rows_bwd(CUtensorMap* m, const void* base, int d, int T, int outer, int rows) {
    auto fn = encode_fn_bwd();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)outer};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)T * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// V in the caller's [B][T][Hkv][d] layout, box = 64 x 1 head x 128 tokens x 1.
bool map_v_bwd(CUtensorMap* m, const void* base, int d, int Hkv, int T, int B) {
    auto fn = encode_fn_bwd();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)Hkv, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)Hkv * d * 2, (cuuint64_t)T * Hkv * d * 2};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// f32 rows of logical length n, row stride ld floats (a multiple of 4), box = `box` x 1; reads
// past n are zero-filled.
bool map_vec_bwd(CUtensorMap* m, const void* base, int n, int ld, int outer, int box_n) {
    auto fn = encode_fn_bwd();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
    cuuint32_t box[2] = {(cuuint32_t)box_n, 1};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major SW128 descriptor of a bf16 tile of `rows` rows x d columns stored as 64-column boxes
// of rows*128 bytes: k-step kk (16 columns) lives in box kk/4 at byte offset (kk%4)*32.
__device__ __forceinline__ uint64_t kdesc_rows(uint32_t tile, int rows, int kk) {
    return smem_desc(tile + (uint32_t)(kk >> 2) * (uint32_t)(rows * 128) + (uint32_t)(kk & 3) * 32u, 16, 1024,
                     kSwizzle128B);
}

// mbar_wait taken by every lane of a warp, with one verdict for the whole warp (a warp then
// never diverges around its warp-collective TMEM loads or issue loops).
__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, volatile int* abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort)) != 0;
}

// Bulk copy (no tensor map) global -> shared, completing on an mbarrier.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// First stored tile of key tile kt in the causal band (steps 4kt .. nst-1 of every key tile).
__host__ __device__ __forceinline__ size_t band_off(int kt, int nkt) {
    return (size_t)4 * ((size_t)kt * nkt - (size_t)kt * (kt - 1) / 2);
}

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// For t2 = X log2(e): log2(softplus(X) / ln 2), the decay's inner term (the forward's
// log2_softplus_over_ln2, same arithmetic), and sigmoid(X) / softplus(X), both from one exp2
// e = 2^-|t2|.  softplus / ln2 = max(t2, 0) + e q(e) with q the degree-7 fit of log2(1 + e) / e;
// sigmoid = 1 / (1 + e) for t2 >= 0 (where softplus / ln2 >= 1) and e / (1 + e) below, where
// the factor e cancels against softplus = e q ln2.  So the ratio never divides by a tiny number
// (its limit 1 as X -> -inf included).
__device__ __forceinline__ float log2sp_and_ratio(float t2, float& ratio) {
    const float e = ex2f(-fabsf(t2));
    float q = -0.012319492176175117f;
    q = fmaf(q, e, 0.06360796093940735f);
    q = fmaf(q, e, -0.15535196661949158f);
    q = fmaf(q, e, 0.2560097873210907f);
    q = fmaf(q, e, -0.35339486598968506f);
    q = fmaf(q, e, 0.48006370663642883f);
    q = fmaf(q, e, -0.7213100790977478f);
    q = fmaf(q, e, 1.4426947832107544f);
    const float sp2 = fmaf(e, q, fmaxf(t2, 0.f));
    ratio = rcp_approx(fmaf(e, kLn2, kLn2) * (t2 >= 0.f ? sp2 : q));
    return lg2f(sp2);
}

// sigmoid(x) / softplus(x), 0 where softplus underflows (the decay it multiplies is then 0 too).
__device__ __forceinline__ float sig_over_sp_f(float x) {
    const float sp = softplus_f(x);
    return sp > 0.f ? sigmoid_f(x) / sp : 0.f;
}

// Sum over the 32 lanes of a warp of v[0..7] (lane t's 8 values), transposed: lane t gets the sum
// of v[t % 8] over all lanes.  A butterfly that halves the vector at every level (each lane keeps
// the half its bit selects and sends the other), then the four 8-lane groups added.
__device__ __forceinline__ float warp_transpose_sum8(float (&v)[8], int lane) {
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1) {
        const bool upper = (lane & w) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float send = upper ? v[i] : v[i + w];
            const float keep = upper ? v[i + w] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    float t = v[0] + __shfl_xor_sync(0xffffffffu, v[0], 8);
    return t + __shfl_xor_sync(0xffffffffu, t, 16);
}

// Key-major pass: threads per key (each takes kKeyRows of a step's 32 rows).
constexpr int kKeyQ = 4, kKeyRows = 32 / kKeyQ;
}  // namespace

// =========================================================================== prep
// N consecutive bf16 (N = 2 or 4; 4N-byte aligned) to and from fp32.
template <int N>
__device__ __forceinline__ void ld_bf16(const __nv_bfloat16* src, float (&f)[N]) {
    static_assert(N == 2 || N == 4, "two or four elements");
    if constexpr (N == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(src);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
        f[0] = lo.x, f[1] = lo.y, f[2] = hi.x, f[3] = hi.y;
    } else {
        const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src));
        f[0] = v.x, f[1] = v.y;
    }
}
template <int N>
__device__ __forceinline__ void st_bf16(__nv_bfloat16* dst, const float (&f)[N]) {
    static_assert(N % 2 == 0, "pairs");
#pragma unroll
    for (int e = 0; e < N; e += 2) *reinterpret_cast<__nv_bfloat162*>(dst + e) = __floats2bfloat162_rn(f[e], f[e + 1]);
}

// grid (T, B), 256 threads: dA = dO * sigmoid(g) (bf16, [B*H][T][d] rows), the gate's gradient
// dg = dO * O * (1 - sigmoid(g)) (bf16, laid out like g), Delta = sum_c dO*O and lse * log2(e) per
// (b, h, t); per (b, KV head, t) the bound c = max over the group's heads of s|qrot|(1 + 2^-6) - lse
// on the log-probability of row t before its decay (|qrot| from the token preparation in fp32;
// the bf16 copies the products read are within 1 + 2^-9 of it, and |krot| of 1).  A warp per KV
// group, its heads in turn.
template <int DH>
__global__ void __launch_bounds__(256) k_bwd_prep_tc(BwdTcParams p) {
    constexpr int PER = DH / 32;
    const int t = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const __nv_bfloat16* o = static_cast<const __nv_bfloat16*>(p.o);
    const __nv_bfloat16* dO = static_cast<const __nv_bfloat16*>(p.d_o);
    const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(p.g);
    __nv_bfloat16* ad = static_cast<__nv_bfloat16*>(p.ad);
    __nv_bfloat16* dg = static_cast<__nv_bfloat16*>(p.dg);
    for (int u = warp; u < p.Hkv; u += 8) {
        float cm = -INFINITY;
        for (int hg = 0; hg < p.G; ++hg) {
            const int h = u * p.G + hg;
            const size_t r = (size_t)b * p.H + h;
            const size_t src = (((size_t)b * p.T + t) * p.H + h) * DH + lane * PER;
            float fo[PER], fd[PER], fg[PER];
            ld_bf16<PER>(dO + src, fd);
            ld_bf16<PER>(o + src, fo);
            ld_bf16<PER>(g + src, fg);
            float acc = 0.f;
            float a[PER], dgv[PER];
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                acc = fmaf(fd[e], fo[e], acc);
                const float sg = sigmoid_f(fg[e]);
                a[e] = fd[e] * sg;
                dgv[e] = fd[e] * fo[e] * (1.f - sg);
            }
            st_bf16<PER>(ad + (r * p.T + t) * DH + lane * PER, a);
            st_bf16<PER>(dg + src, dgv);
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
            const float lse = p.lse[r * p.T + t];
            cm = fmaxf(cm, p.mq[r * p.Tp + t] * kLn2 * (1.f + 1.f / 64.f) - lse);
            if (lane == 0) {
                p.delta[r * p.Tp + t] = acc;
                p.lse2[r * p.Tp + t] = lse * kL2e;
            }
        }
        if (lane == 0) p.cmax[((size_t)b * p.Hkv + u) * p.Tpk + t] = cm;
    }
}

// =========================================================================== boundary pass
// grid (B*Hkv, nkt), 128 threads = one thread per key of the tile.  Steps s = 4kt .. nst-1 top
// down: Pb[s][j] = sum_{j < l < 32 s} D[l, j] is written, then the step's X^T tile (tensor cores,
// two TMEM slots so the next step's MMA overlaps this step's decay) adds its rows.
// Exact underflow: Lambda only decreases down a column, so every probability of key j in step s
// is at most exp(c_s - Pb[s][j]), c_s the rows' bound from the prep pass.  Below -88 nats the
// kernels' exp2 (flush to zero under 2^-126) returns exactly 0, and so do dZ, dLambda, dD, w and
// dX for every step from there down.  The key tile's last step that fails the test (at least its
// diagonal block) bounds the key-major pass and the GEMMs; what lies below contributes zeros.
constexpr float kUnderflowNats = -88.f;
namespace bnd {
template <int DH>
struct Smem {
    alignas(1024) uint8_t khk[DH / 64][16384];      // khat of the key tile, boxes [128][64]
    alignas(1024) uint8_t kq[2][DH / 64][4096];     // khat of the step's rows, boxes [32][64]
    alignas(128) float lq[2][ST];
    alignas(128) float lk[128];
    alignas(8) uint64_t kfull, qfull[2], xfull[2];
    uint32_t tmem;
    int abort;
    int last[4];
    float cw[4];
};
}  // namespace bnd

template <int DH>
__global__ void __launch_bounds__(128) k_bwd_bound_tc(const __grid_constant__ CUtensorMap tm_khk,
                                                      const __grid_constant__ CUtensorMap tm_khq,
                                                      const __grid_constant__ CUtensorMap tm_lq,
                                                      const __grid_constant__ CUtensorMap tm_lk, BwdTcParams p) {
    constexpr uint32_t ID_X = idesc_bf16(128, ST, 0, 0);
    constexpr int NB = DH / 64;
    extern __shared__ uint8_t smem_raw[];
    using SM = bnd::Smem<DH>;
    SM& S = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int kt = blockIdx.y, unit = blockIdx.x, kvh = unit % p.Hkv;   // longest key tiles first
    const int T = p.T;
    const int s0 = 4 * kt, nsteps = p.nst - s0;
    volatile int* abort = &S.abort;
    if (tid == 0) {
        mbar_init(&S.kfull, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.qfull[i], 1);
            mbar_init(&S.xfull[i], 1);
        }
        S.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem, 64);
        tmem_relinquish();
    }
    // the unit's largest row bound: once every key's prefix is past it, so is every later step
    const float* crow = p.cmax + (size_t)unit * p.Tpk;
    {
        float c = -INFINITY;
        for (int r = tid; r < T; r += 128) c = fmaxf(c, crow[r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, o));
        if ((tid & 31) == 0) S.cw[warp] = c;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const float call = fmaxf(fmaxf(S.cw[0], S.cw[1]), fmaxf(S.cw[2], S.cw[3]));
    const bool leader = warp == 0 && elect_one();
    auto load_step = [&](int it) {
        const int st = it & 1, s = s0 + it;
        mbar_expect_tx(&S.qfull[st], NB * 4096 + ST * 4);
        for (int c = 0; c < NB; ++c) tma_load_3d(S.kq[st][c], &tm_khq, &S.qfull[st], 64 * c, s * ST, unit);
        tma_load_2d(S.lq[st], &tm_lq, &S.qfull[st], s * ST, unit);
    };
    auto issue_x = [&](int it) {
        const int st = it & 1;
        const uint32_t a = smem_u32(S.khk[0]), bq = smem_u32(S.kq[st][0]);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk)
            umma_f16(tmem + st * 32, kdesc_rows(a, 128, kk), kdesc_rows(bq, ST, kk), ID_X, kk > 0);
        umma_commit(&S.xfull[st]);
    };
    if (leader) {
        mbar_expect_tx(&S.kfull, NB * 16384 + 512);
        for (int c = 0; c < NB; ++c) tma_load_3d(S.khk[c], &tm_khk, &S.kfull, 64 * c, kt * 128, unit);
        tma_load_2d(S.lk, &tm_lk, &S.kfull, kt * 128, unit);
        load_step(0);
        if (nsteps > 1) load_step(1);
    }
    bool ok = mbar_wait(&S.kfull, 0, abort);
    if (leader && ok && mbar_wait(&S.qfull[0], 0, abort)) {
        tc_fence_after();
        issue_x(0);
    }
    const int j = kt * 128 + tid;
    const float rk3 = ex2f(S.lk[tid]) * kCbrtLn2b;
    const float al2 = p.alpha[kvh] * kL2e, be2 = p.beta[kvh] * kL2e;
    float run = 0.f;                                  // sum of D / rk3 over the rows so far
    float* pbrow = p.pb + (size_t)unit * p.nst * p.Tpk + (size_t)kt * 128 + tid;
    int last = min(s0 + 3, p.nst - 1);                // the diagonal block is always walked
    const uint32_t tl = (uint32_t)(warp * 32) << 16;
    for (int it = 0; it < nsteps; ++it) {
        const int st = it & 1, s = s0 + it;
        const float pb = rk3 * run;
        pbrow[(size_t)s * p.Tpk] = pb;
        {
            const int row = s * ST + (tid & 31);
            float c = row < T ? crow[row] : -INFINITY;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, o));
            if (j < T && c - pb >= kUnderflowNats) last = s;
        }
        // below the diagonal block, once this step and all later ones are past the threshold for
        // every key: stop (after this step's product and the next step's copy have landed)
        if (it >= 4 && __syncthreads_and(j >= T || call - pb < kUnderflowNats)) {
            if (ok) {
                ok = mbar_wait(&S.xfull[st], (it >> 1) & 1, abort);
                if (ok && it + 1 < nsteps) ok = mbar_wait(&S.qfull[(it + 1) & 1], ((it + 1) >> 1) & 1, abort);
            }
            break;
        }
        if (leader && ok && it + 1 < nsteps) {
            if (mbar_wait(&S.qfull[(it + 1) & 1], ((it + 1) >> 1) & 1, abort)) {
                tc_fence_after();
                issue_x(it + 1);
            } else {
                ok = false;
            }
        }
        ok = __all_sync(0xffffffffu, ok && mbar_wait(&S.xfull[st], (it >> 1) & 1, abort)) != 0;
        uint32_t x[32];
        float lqv[32];
        if (ok) {
            tc_fence_after();
            uint32_t (&x0)[16] = *reinterpret_cast<uint32_t(*)[16]>(&x[0]);
            uint32_t (&x1)[16] = *reinterpret_cast<uint32_t(*)[16]>(&x[16]);
            tmem_ld16_async(tmem + tl + st * 32, x0);
            tmem_ld16_async(tmem + tl + st * 32 + 16, x1);
            tmem_wait16(x0);
            tmem_wait16(x1);
#pragma unroll
            for (int r = 0; r < 32; r += 4) {
                const float4 v = *reinterpret_cast<const float4*>(&S.lq[st][r]);
                lqv[r] = v.x; lqv[r + 1] = v.y; lqv[r + 2] = v.z; lqv[r + 3] = v.w;
            }
        }
        tc_fence_before();
        ok = __syncthreads_and(ok) != 0;                // slot st and lq[st] read by everyone
        if (leader && ok && it + 2 < nsteps) load_step(it + 2);
        if (ok) {
            const int l0 = s * ST;
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                const float dq = ex2f(fmaf(log2_softplus_over_ln2(fmaf(al2, __uint_as_float(x[r]), be2)),
                                           0.33333334f, lqv[r]));
                const int l = l0 + r;
                run += (l > j && l < T) ? dq : 0.f;
            }
        }
    }
    last = __reduce_max_sync(0xffffffffu, last);
    if ((tid & 31) == 0) S.last[warp] = last;
    tc_fence_before();
    __syncthreads();
    if (tid == 0)
        p.slast[(size_t)unit * p.nkt + kt] = max(max(S.last[0], S.last[1]), max(S.last[2], S.last[3]));
    if (*abort && tid == 0) drain_pause(10000000ull);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

// =========================================================================== key-major pass
// grid (B*Hkv, nkt), 544 threads: warps 0-15 compute (four threads per key j, TMEM lane j % 128:
// warps 4q .. 4q+3 rows 8q .. 8q+7 of each step), warp 16 issues the TMA loads and the MMAs.  Steps s = nst-1 down to 4kt.  TMEM: dV (DH columns), dKrot (DH),
// the X^T slot (32), two slots for the S_h^T / dP_h^T pair of a head (64 each).
// Last step of key tile kt walked by the key-major pass and summed by the GEMMs: the boundary
// pass's bound, kept within [the diagonal block, nst - 1].
__device__ __forceinline__ int last_step(const BwdTcParams& p, int unit, int kt) {
    const int sd = min(4 * kt + 3, p.nst - 1);
    return max(min(p.slast[(size_t)unit * p.nkt + kt], p.nst - 1), sd);
}

namespace key {
template <int DH, int G>
struct Smem {
    alignas(1024) uint8_t khk[DH / 64][16384];   // khat / krot / v of the key tile, boxes [128][64]
    alignas(1024) uint8_t krk[DH / 64][16384];
    alignas(1024) uint8_t vk[DH / 64][16384];
    alignas(1024) uint8_t kq[DH / 64][4096];     // khat of the step's rows, boxes [32][64]
    alignas(1024) uint8_t qh[G][DH / 64][4096];  // qrot / dA of the step's rows, per head
    alignas(1024) uint8_t ah[G][DH / 64][4096];
    alignas(1024) uint8_t tp[2][kTileBytes];     // P_h^T and dZ_h^T tiles (K-major, no swizzle),
    alignas(1024) uint8_t tz[2][kTileBytes];     // by head parity
    alignas(128) float lq[ST];                   // log2 rate / 3 of the step's rows (with kq)
    alignas(128) float pbv[128];                 // decay prefix above the step (with kq)
    alignas(128) float lse2[G][ST];              // per head (with qh / ah)
    alignas(128) float dlt[G][ST];
    alignas(128) float lk[128];
    alignas(16) float red[2][4 * kKeyQ];
    alignas(16) float ca[2][kKeyQ][128];         // each row group's decay totals, by step parity
    alignas(16) float tv[2][kKeyQ][128];         // each row group's dLambda totals, by step parity
    alignas(16) float dakx[kKeyQ][128];          // each row group's d a_k sums
    alignas(8) uint64_t kfull, qfull, qempty, xfull, xempty, hfull[G], hdone[G], pfull[2], pempty[2],
        tfull[2], tempty[2], accdone, cafull[2], tvfull[2];
    uint32_t tmem;
    int abort;
};
}  // namespace key

template <int DH, int G>
__global__ void __launch_bounds__(128 * kKeyQ + 32, 1)
k_bwd_key_tc(const __grid_constant__ CUtensorMap tm_khk, const __grid_constant__ CUtensorMap tm_krk,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_khq,
             const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ad,
             const __grid_constant__ CUtensorMap tm_lq, const __grid_constant__ CUtensorMap tm_lk,
             const __grid_constant__ CUtensorMap tm_pb, const __grid_constant__ CUtensorMap tm_lse2,
             const __grid_constant__ CUtensorMap tm_dlt, BwdTcParams p) {
    constexpr int NB = DH / 64;
    constexpr uint32_t ID_L = idesc_bf16(128, ST, 0, 0);      // logits: keys x rows, both K-major
    constexpr uint32_t ID_ACC = idesc_bf16(128, DH, 0, 1);    // tile^T (K-major) x rows (MN-major)
    constexpr uint32_t COL_DV = 0, COL_DK = DH, COL_X = 2 * DH, COL_P = 2 * DH + 32;
    static_assert(COL_P + 128 <= 512, "TMEM budget");
    extern __shared__ uint8_t smem_raw[];
    using SM = key::Smem<DH, G>;
    SM& S = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kt = blockIdx.y, unit = blockIdx.x, kvh = unit % p.Hkv, b = unit / p.Hkv;   // longest first
    const int T = p.T;
    // steps sfin down to 4kt; the ones below sfin hold no nonzero probability
    const int s0 = 4 * kt, sfin = last_step(p, unit, kt), nsteps = sfin - s0 + 1;
    volatile int* abort = &S.abort;
    if (tid == 0) {
        mbar_init(&S.kfull, 1);
        mbar_init(&S.xfull, 1);
        mbar_init(&S.xempty, 4 * kKeyQ);              // every compute warp, in each of these
        mbar_init(&S.accdone, 1);
        mbar_init(&S.qfull, 1);
        mbar_init(&S.qempty, 4 * kKeyQ);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.tfull[i], 4 * kKeyQ);
            mbar_init(&S.tempty[i], 1);
            mbar_init(&S.pfull[i], 1);
            mbar_init(&S.pempty[i], 4 * kKeyQ);
            mbar_init(&S.cafull[i], 4 * kKeyQ);
            mbar_init(&S.tvfull[i], 4 * kKeyQ);
        }
        for (int h = 0; h < G; ++h) {
            mbar_init(&S.hfull[h], 1);
            mbar_init(&S.hdone[h], 1);
        }
        S.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;

    if (warp == 4 * kKeyQ) {
        // ------------------------------------------------ TMA + MMA issue (one elected lane)
        const bool leader = elect_one();
        bool ok = true;
        // step it covers rows of step s = nst-1-it.  The step's khat rows, lq and the prefix
        // vector have one buffer: X^T is the first MMA of a step, so they are free
        // early and the next step's copy overlaps the rest of this one.
        auto load_q = [&](int it) {
            const int s = sfin - it;
            if (leader) {
                mbar_expect_tx(&S.qfull, NB * 4096 + ST * 4 + 128 * 4);
                for (int c = 0; c < NB; ++c) tma_load_3d(S.kq[c], &tm_khq, &S.qfull, 64 * c, s * ST, unit);
                tma_load_2d(S.lq, &tm_lq, &S.qfull, s * ST, unit);
                tma_load_2d(S.pbv, &tm_pb, &S.qfull, kt * 128, unit * p.nst + s);
            }
            __syncwarp();
        };
        auto load_h = [&](int it, int h) {
            const int s = sfin - it, row = b * p.H + kvh * G + h;
            if (leader) {
                mbar_expect_tx(&S.hfull[h], 2 * NB * 4096 + 2 * ST * 4);
                for (int c = 0; c < NB; ++c) {
                    tma_load_3d(S.qh[h][c], &tm_q, &S.hfull[h], 64 * c, s * ST, row);
                    tma_load_3d(S.ah[h][c], &tm_ad, &S.hfull[h], 64 * c, s * ST, row);
                }
                tma_load_2d(S.lse2[h], &tm_lse2, &S.hfull[h], s * ST, row);
                tma_load_2d(S.dlt[h], &tm_dlt, &S.hfull[h], s * ST, row);
            }
            __syncwarp();
        };
        if (leader) {
            mbar_expect_tx(&S.kfull, 3 * NB * 16384 + 512);
            for (int c = 0; c < NB; ++c) {
                tma_load_3d(S.khk[c], &tm_khk, &S.kfull, 64 * c, kt * 128, unit);
                tma_load_3d(S.krk[c], &tm_krk, &S.kfull, 64 * c, kt * 128, unit);
                tma_load_4d(S.vk[c], &tm_v, &S.kfull, 64 * c, kvh, kt * 128, b);
            }
            tma_load_2d(S.lk, &tm_lk, &S.kfull, kt * 128, unit);
        }
        __syncwarp();
        load_q(0);
        for (int h = 0; h < G; ++h) load_h(0, h);
        ok = wwait(&S.kfull, 0, abort);
        const uint32_t akh = smem_u32(S.khk[0]), akr = smem_u32(S.krk[0]), av = smem_u32(S.vk[0]);
        const uint32_t bq = smem_u32(S.kq[0]);
        bool first_acc = true;
        // Head operands of the next step are copied once the head's accumulation has completed;
        // the copy waits until the next head's products are issued (so their round trip is not
        // behind the accumulation's), and before that head's own products at the latest.
        int pend = -1, pit = 0;
        auto reload = [&]() -> bool {
            if (pend < 0) return true;
            const int hh = pend;
            pend = -1;
            if (!wwait(&S.hdone[hh], pit & 1, abort)) return false;
            load_h(pit + 1, hh);
            return true;
        };
        for (int it = 0; ok && it < nsteps; ++it) {
            // X^T of the step (the same bf16 unit keys as the forward, whose row normalisers the
            // probabilities are divided by)
            if (!wwait(&S.qfull, it & 1, abort)) break;
            if (it >= 1 && !wwait(&S.xempty, (it - 1) & 1, abort)) break;
            tc_fence_after();
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < DH / 16; ++kk)
                    umma_f16(tmem + COL_X, kdesc_rows(akh, 128, kk), kdesc_rows(bq, ST, kk), ID_L, kk > 0);
                umma_commit(&S.xfull);
            }
            __syncwarp();
            // accumulation of head hh of this step: dV += P^T dA, dKrot += dZ^T qrot
            auto accum = [&](int hh) -> bool {
                const uint32_t v = (uint32_t)(it * G + hh), tb = v & 1;
                if (!wwait(&S.tfull[tb], (v >> 1) & 1, abort)) return false;
                tc_fence_after();
                if (leader) {
                    const uint32_t tpa = smem_u32(S.tp[tb]), tza = smem_u32(S.tz[tb]);
                    const uint32_t ba = smem_u32(S.ah[hh][0]), bqh = smem_u32(S.qh[hh][0]);
#pragma unroll
                    for (int kk = 0; kk < ST / 16; ++kk) {
                        // A: tile^T, K-major no swizzle (8 keys x 16 B core matrices; 128 B apart
                        // along the keys, 2048 B apart along the rows); B: rows of the step,
                        // MN-major SW128 (64-dim atoms 4096 B apart, 8-row groups 1024 B apart)
                        const uint64_t da = smem_desc(tpa + kk * 4096u, 2048, 128, kSwizzleNone);
                        const uint64_t dz = smem_desc(tza + kk * 4096u, 2048, 128, kSwizzleNone);
                        const uint64_t db = smem_desc(ba + kk * 2048u, 4096, 1024, kSwizzle128B);
                        const uint64_t dq = smem_desc(bqh + kk * 2048u, 4096, 1024, kSwizzle128B);
                        const uint32_t acc = (first_acc && kk == 0) ? 0u : 1u;
                        umma_f16(tmem + COL_DV, da, db, ID_ACC, acc);
                        umma_f16(tmem + COL_DK, dz, dq, ID_ACC, acc);
                    }
                    umma_commit(&S.tempty[tb]);
                    umma_commit(&S.hdone[hh]);
                }
                __syncwarp();
                first_acc = false;
                return true;
            };
            for (int h = 0; h < G && ok; ++h) {
                const uint32_t u = (uint32_t)(it * G + h), pp = u & 1;
                if (pend == h && !reload()) { ok = false; break; }
                if (!wwait(&S.hfull[h], it & 1, abort)) { ok = false; break; }
                if (u >= 2 && !wwait(&S.pempty[pp], ((u >> 1) - 1) & 1, abort)) { ok = false; break; }
                tc_fence_after();
                if (leader) {
                    const uint32_t bqh = smem_u32(S.qh[h][0]), bah = smem_u32(S.ah[h][0]);
#pragma unroll
                    for (int kk = 0; kk < DH / 16; ++kk) {
                        umma_f16(tmem + COL_P + pp * 64, kdesc_rows(akr, 128, kk), kdesc_rows(bqh, ST, kk), ID_L,
                                 kk > 0);
                        umma_f16(tmem + COL_P + pp * 64 + 32, kdesc_rows(av, 128, kk), kdesc_rows(bah, ST, kk),
                                 ID_L, kk > 0);
                    }
                    umma_commit(&S.pfull[pp]);
                }
                __syncwarp();
                if (!reload()) { ok = false; break; }
                if (h == 0 && it + 1 < nsteps) {
                    // the step's khat rows, lq and prefixes are free once the compute warps have
                    // read X^T and the vectors: copy the next step's
                    if (!wwait(&S.qempty, it & 1, abort)) { ok = false; break; }
                    load_q(it + 1);
                }
                if (h >= 1) {
                    if (!accum(h - 1)) { ok = false; break; }
                    if (it + 1 < nsteps) {
                        pend = h - 1;
                        pit = it;
                    }
                }
            }
            if (!ok) break;
            if (!reload()) break;
            if (!accum(G - 1)) break;
            if (it + 1 < nsteps) {
                pend = G - 1;
                pit = it;
            }
        }
        if (leader) umma_commit(&S.accdone);
        __syncwarp();
    } else {
        // ------------------------------------------------ compute warps: kKeyQ threads per key j
        // (TMEM lane jl): warps 4q .. 4q+3 take rows kKeyRows*q .. of each 32-row step.  Two
        // exchanges per step join them: the decay totals of the row groups above, where a
        // group's prefixes start, and every group's dLambda total, from which each forms its
        // rows' suffix sums (bottom up: the lowest group's rows first).
        constexpr int RQ = kKeyRows;
        const int jl = tid & 127, qi = tid >> 7, rb = RQ * qi;   // this thread: rows rb .. rb+RQ-1
        const int j = kt * 128 + jl;
        const uint32_t tl = (uint32_t)((warp & 3) * 32) << 16;
        const float al = p.alpha[kvh], be = p.beta[kvh];
        const float al2 = al * kL2e, be2 = be * kL2e;
        const float sl = p.scale * kL2e;
        bool ok = wwait(&S.kfull, 0, abort);
        const float rk3 = ok ? ex2f(S.lk[jl]) * kCbrtLn2b : 0.f;   // r_k^(1/3) (ln 2)^(1/3)
        float carry = 0.f;                            // sum of dLambda over the rows below the step
        float dak = 0.f, dal = 0.f, dbe = 0.f;
        const size_t tstride = (size_t)p.ntiles * kTileBytes;      // bytes per stored tile set
        uint8_t* tile_base = static_cast<uint8_t*>(p.tiles) + (size_t)unit * (G + 1) * tstride;
        const size_t band = band_off(kt, p.nkt);
        {
            // below sfin: the rest of its 128-row block of stored tiles is zero (the GEMMs sum whole
            // blocks; the post pass reads the rows' w sums of walked steps only)
            const int zend = min(4 * (sfin / 4) + 3, p.nst - 1);
            const int nz = (zend - sfin) * (int)(kTileBytes / 16);
            for (int g2 = 0; g2 <= G; ++g2) {
                uint4* z = reinterpret_cast<uint4*>(tile_base + (size_t)g2 * tstride +
                                                    (band + (sfin + 1 - s0)) * kTileBytes);
                for (int i = tid; i < nz; i += 128 * kKeyQ) z[i] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        for (int it = 0; ok && it < nsteps; ++it) {
            const int s = sfin - it;
            const int i0 = s * ST;
            const int xb = it & 1;                    // exchange buffer and its phase
            const uint32_t xph = (uint32_t)(it >> 1) & 1u;
            if (!wwait(&S.qfull, it & 1, abort)) { ok = false; break; }
            const float pbj = S.pbv[jl];
            if (!wwait(&S.xfull, it & 1, abort)) { ok = false; break; }
            tc_fence_after();
            uint32_t x[RQ];
            tmem_ld8_async(tmem + tl + COL_X + rb, x);
            tmem_wait8(x);
            // Steps below the key tile's diagonal, inside the sequence, of a key tile inside it carry
            // no causal or end mask (one uniform choice per step).
            const bool interior = i0 >= kt * 128 + 128 && i0 + ST <= T && kt * 128 + 128 <= T;
            // decay of this group's rows: Dq = D / rk3, and their running sum from its first row;
            // sigmoid / softplus of X for dX
            float dqv[RQ], csum[RQ], rto[RQ];
            float c = 0.f;
            auto decay = [&](auto masked) {
#pragma unroll
                for (int r = 0; r < RQ; r += 4) {
                    const float4 lv = *reinterpret_cast<const float4*>(&S.lq[rb + r]);
                    const float l4[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float dq = ex2f(fmaf(log2sp_and_ratio(fmaf(al2, __uint_as_float(x[r + e]), be2), rto[r + e]),
                                             0.33333334f, l4[e]));
                        if constexpr (decltype(masked)::value) {
                            const int l = i0 + rb + r + e;
                            dq = (l > j && l < T) ? dq : 0.f;
                        }
                        dqv[r + e] = dq;
                        c += dq;
                        csum[r + e] = c;
                    }
                }
            };
            if (interior) decay(std::false_type{});
            else decay(std::true_type{});
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&S.xempty);
                mbar_arrive(&S.qempty);
            }
            // the decay of the step's rows above this group: the totals of the groups above
            S.ca[xb][qi][jl] = c;
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.cafull[xb]);
            if (!wwait(&S.cafull[xb], xph, abort)) { ok = false; break; }
            float cbase = 0.f;
#pragma unroll
            for (int q = 0; q < kKeyQ - 1; ++q)
                if (q < qi) cbase += S.ca[xb][q][jl];
            float lam[RQ];                            // Lambda * log2(e)
#pragma unroll
            for (int r = 0; r < RQ; ++r) lam[r] = -fmaf(rk3, cbase + csum[r], pbj) * kL2e;
            float dlam[RQ];
#pragma unroll
            for (int r = 0; r < RQ; ++r) dlam[r] = 0.f;
            const bool jv = j < T;
            for (int h = 0; h < G && ok; ++h) {
                const uint32_t u = (uint32_t)(it * G + h), pp = u & 1;
                if (!wwait(&S.hfull[h], it & 1, abort)) { ok = false; break; }
                if (!wwait(&S.pfull[pp], (u >> 1) & 1, abort)) { ok = false; break; }
                tc_fence_after();
                uint32_t sv[RQ], dpv[RQ];
                {
                    const uint32_t base = tmem + tl + COL_P + pp * 64;
                    tmem_ld8_async(base + rb, sv);
                    tmem_ld8_async(base + 32 + rb, dpv);
                    tmem_wait8(sv);
                    tmem_wait8(dpv);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.pempty[pp]);
                uint4* gz = reinterpret_cast<uint4*>(tile_base + (size_t)h * tstride + (band + (s - s0)) * kTileBytes);
                uint4 vp[RQ / 8], vz[RQ / 8];
                auto probs = [&](auto masked) {
#pragma unroll
                    for (int c2 = 0; c2 < RQ / 8; ++c2) {
                        uint32_t wp[4], wz[4];
                        float ls[8], dl[8];
#pragma unroll
                        for (int e = 0; e < 8; e += 4) {
                            const float4 a4 = *reinterpret_cast<const float4*>(&S.lse2[h][rb + c2 * 8 + e]);
                            const float4 d4 = *reinterpret_cast<const float4*>(&S.dlt[h][rb + c2 * 8 + e]);
                            ls[e] = a4.x, ls[e + 1] = a4.y, ls[e + 2] = a4.z, ls[e + 3] = a4.w;
                            dl[e] = d4.x, dl[e + 1] = d4.y, dl[e + 2] = d4.z, dl[e + 3] = d4.w;
                        }
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            float pz[2], zz[2];
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                const int r = c2 * 8 + e + q;     // this group's row r = step row rb + r
                                float pv = ex2f(fmaf(__uint_as_float(sv[r]), sl, lam[r] - ls[e + q]));
                                if constexpr (decltype(masked)::value) {
                                    const int i = i0 + rb + r;
                                    pv = (jv && i >= j && i < T) ? pv : 0.f;
                                }
                                const float z = pv * (__uint_as_float(dpv[r]) - dl[e + q]);
                                dlam[r] += z;
                                pz[q] = pv;
                                zz[q] = z;
                            }
                            __nv_bfloat162 bp = __floats2bfloat162_rn(pz[0], pz[1]);
                            __nv_bfloat162 bz = __floats2bfloat162_rn(zz[0], zz[1]);
                            wp[e >> 1] = *reinterpret_cast<uint32_t*>(&bp);
                            wz[e >> 1] = *reinterpret_cast<uint32_t*>(&bz);
                        }
                        vp[c2] = make_uint4(wp[0], wp[1], wp[2], wp[3]);
                        vz[c2] = make_uint4(wz[0], wz[1], wz[2], wz[3]);
                        gz[(rb / 8 + c2) * 128 + jl] = vz[c2];
                    }
                };
                if (interior) probs(std::false_type{});
                else probs(std::true_type{});
                // the tile pair of this parity is free once the accumulation of head u-2 completed
                const uint32_t tb = u & 1;
                if (u >= 2 && !wwait(&S.tempty[tb], ((u >> 1) - 1) & 1, abort)) { ok = false; break; }
                uint8_t* ttp = S.tp[tb];
                uint8_t* ttz = S.tz[tb];
#pragma unroll
                for (int c2 = 0; c2 < RQ / 8; ++c2) {
                    // core matrix (8 keys x 8 rows): rows 8*c8.., this key's 16-byte line
                    const int c8 = rb / 8 + c2;
                    *reinterpret_cast<uint4*>(ttp + c8 * 2048 + jl * 16) = vp[c2];
                    *reinterpret_cast<uint4*>(ttz + c8 * 2048 + jl * 16) = vz[c2];
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.tfull[tb]);
            }
            if (!ok) break;
            // dD = -(sum of dLambda over the rows at and below l), bottom up; w = dD D / 3.  Each
            // group totals its rows' dLambda; with every total each thread of the key carries the
            // same running sum below the step (summed in the same order everywhere).
            float tmine = 0.f;
#pragma unroll
            for (int r = RQ - 1; r >= 0; --r) tmine += dlam[r];
            S.tv[xb][qi][jl] = tmine;
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.tvfull[xb]);
            if (!wwait(&S.tvfull[xb], xph, abort)) { ok = false; break; }
            float cin = carry;
            {
                float acc = carry;
#pragma unroll
                for (int q = kKeyQ - 1; q >= 0; --q) {
                    if (q == qi) cin = acc;
                    acc += S.tv[xb][q][jl];
                }
                carry = acc;
            }
            float wv[RQ];
#pragma unroll
            for (int r = RQ - 1; r >= 0; --r) {
                cin += dlam[r];
                wv[r] = -cin * rk3 * dqv[r] * 0.33333334f;      // zero where D was masked
                dak += wv[r];
            }
            {
                uint4* gx = reinterpret_cast<uint4*>(tile_base + (size_t)G * tstride + (band + (s - s0)) * kTileBytes);
#pragma unroll
                for (int c2 = 0; c2 < RQ / 8; ++c2) {
                    const int c8 = rb / 8 + c2;
                    uint32_t wx[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        float xx[2];
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int r = c2 * 8 + e + q;
                            const float xs = __uint_as_float(x[r]);
                            const float dX = wv[r] * rto[r];
                            dal = fmaf(dX, xs, dal);
                            dbe += dX;
                            xx[q] = dX;
                        }
                        __nv_bfloat162 bx = __floats2bfloat162_rn(xx[0], xx[1]);
                        wx[e >> 1] = *reinterpret_cast<uint32_t*>(&bx);
                    }
                    gx[c8 * 128 + jl] = make_uint4(wx[0], wx[1], wx[2], wx[3]);
                }
            }
            // row sums of w over this warp's 32 keys: lane t < RQ gets row rb + t's sum (the post pass
            // sums the key tiles' four quarters per row)
            const float rs = warp_transpose_sum8(wv, lane);
            if (lane < RQ) p.daq_part[(((size_t)unit * p.Tpk + i0 + rb + lane) * p.nkt + kt) * 4 + (warp & 3)] = rs;
        }
        // ---- results of the key tile: each group reads DH / kKeyQ of the dV / dKrot columns
        const bool done = ok && wwait(&S.accdone, 0, abort);
        if (done) {
            tc_fence_after();
            float* dv = p.dv32 + ((size_t)unit * T + j) * DH;
            float* dk = p.dkr + ((size_t)unit * T + j) * DH;
#pragma unroll 1
            for (int c = qi * (DH / kKeyQ); c < (qi + 1) * (DH / kKeyQ); c += 16) {
                float a[16], k2[16];
                tmem_ld16(tmem + tl + COL_DV + c, a);      // warp-collective: every lane loads
                tmem_ld16(tmem + tl + COL_DK + c, k2);
                if (j < T) {
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        *reinterpret_cast<float4*>(dv + c + e) = make_float4(a[e], a[e + 1], a[e + 2], a[e + 3]);
                        *reinterpret_cast<float4*>(dk + c + e) = make_float4(p.scale * k2[e], p.scale * k2[e + 1],
                                                                             p.scale * k2[e + 2], p.scale * k2[e + 3]);
                    }
                }
            }
        }
        // d a_k of the key (the groups' sums) and the CTA's dalpha / dbeta partials
        S.dakx[qi][jl] = dak;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            dal += __shfl_xor_sync(0xffffffffu, dal, o);
            dbe += __shfl_xor_sync(0xffffffffu, dbe, o);
        }
        if (lane == 0) {
            S.red[0][warp] = dal;
            S.red[1][warp] = dbe;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(128 * kKeyQ) : "memory");
        if (done && qi == 0 && j < T) {
            float dsum = 0.f;
#pragma unroll
            for (int q = 0; q < kKeyQ; ++q) dsum += S.dakx[q][jl];
            const float ak = p.a_k[((size_t)b * T + j) * p.Hkv + kvh];
            p.dak32[(size_t)unit * T + j] = dsum * sig_over_sp_f(ak);
        }
        if (tid == 0) {
            const size_t o = ((size_t)unit * p.nkt + kt) * 2;
            float sa = 0.f, sb = 0.f;
#pragma unroll
            for (int w = 0; w < 4 * kKeyQ; ++w) {
                sa += S.red[0][w];
                sb += S.red[1][w];
            }
            p.dab[o] = sa;
            p.dab[o + 1] = sb;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort && tid == 0) drain_pause(10000000ull);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// =========================================================================== GEMMs over stored tiles
// Row side: per (128-row block rb, output o, unit): C^T[dims x 128 rows] = sum_{kt <= rb} K_kt^T T_kt,
// with K the key tile's krot (o < G, T = dZ_o^T tiles) or khat (o = G, T = dX^T tiles); the 128
// dims run along the TMEM lanes (head_dim 64 uses the lower 64: the upper half of the A operand
// points at a zero block).  Key side: per (key tile kt, unit): C[128 keys x dims] = sum_{rb >= kt}
// dX^T_(kt, rb) khat_rb.  128 threads: warp 0 loads, warp 1 issues, all four write the result.
// Grids (row blocks from the last, G + 1, units) and (key tiles, units).  One operand stage per
// CTA (64 KB), so two to three CTAs share an SM and overlap each other's copies, products and
// epilogues: most sums are short once the underflowing band is skipped, and a three-stage ring in
// one CTA per SM was slower (row GEMM 0.92 -> 0.71 ms on the 3B workload with one stage).
namespace gemm {
constexpr int NS = 1;
template <int DH>
struct Smem {
    alignas(1024) uint8_t a[NS][2][16384];       // operand tile boxes [128][64] (rows side: keys; key side: rows)
    alignas(1024) uint8_t t[NS][4 * kTileBytes]; // four stored tiles (128 rows)
    alignas(1024) uint8_t zero[DH == 64 ? 16384 : 16];
    alignas(8) uint64_t full[NS], empty[NS], done;
    uint32_t tmem;
    int abort;
};
}  // namespace gemm

template <int DH, bool ROWS>
__global__ void __launch_bounds__(128, 1)
k_bwd_gemm_tc(const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_kr, BwdTcParams p) {
    constexpr int NB = DH / 64;
    constexpr int NCOL = ROWS ? 128 : DH;             // accumulator columns
    extern __shared__ uint8_t smem_raw[];
    using SM = gemm::Smem<DH>;
    SM& S = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NS = gemm::NS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // row blocks from the last (the longest sums first within each unit and output)
    const int blk = ROWS ? p.nkt - 1 - (int)blockIdx.x : (int)blockIdx.x, unit = ROWS ? blockIdx.z : blockIdx.y;
    const int o = ROWS ? (int)blockIdx.y : p.G;       // output: head o's dqrot, or the dkhat part
    const int kvh = unit % p.Hkv, b = unit / p.Hkv;
    const int T = p.T;
    // operand pairs to sum: key tiles kt <= blk whose walked steps reach the row block (the
    // diagonal one always does), or row blocks blk .. the one of the key tile's last walked step
    int n = 0;
    if (ROWS) {
        for (int kt = 0; kt <= blk; ++kt) n += last_step(p, unit, kt) >= 4 * blk;
    } else {
        n = last_step(p, unit, blk) / 4 - blk + 1;
    }
    volatile int* abort = &S.abort;
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&S.full[i], 1);
            mbar_init(&S.empty[i], 1);
        }
        mbar_init(&S.done, 1);
        S.abort = 0;
        fence_barrier_init();
    }
    if (DH == 64 && ROWS) {
        uint32_t* z = reinterpret_cast<uint32_t*>(S.zero);
        for (int i = tid; i < (int)(sizeof(S.zero) / 4); i += 128) z[i] = 0u;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem, NCOL);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const size_t tstride = (size_t)p.ntiles * kTileBytes;
    const uint8_t* tiles = static_cast<const uint8_t*>(p.tiles) + ((size_t)unit * (p.G + 1) + o) * tstride;
    if (warp == 0) {
        const bool leader = elect_one();
        int ktn = 0;                                  // rows side: next key tile to test
        for (int i = 0; i < n; ++i) {
            const int stg = i % NS;
            if (i >= NS && !wwait(&S.empty[stg], ((i / NS) - 1) & 1, abort)) break;
            // rows side: the i-th key tile of row block blk with walked steps there; key side: row
            // block rb = blk + i of key tile blk
            if (ROWS)
                while (last_step(p, unit, ktn) < 4 * blk) ++ktn;
            const int kt = ROWS ? ktn++ : blk, rb = ROWS ? blk : blk + i;
            if (leader) {
                mbar_expect_tx(&S.full[stg], NB * 16384 + 4 * kTileBytes);
                const CUtensorMap* m = (ROWS && o < p.G) ? &tm_kr : &tm_kh;
                const int r0 = ROWS ? kt * 128 : rb * 128;
                for (int c = 0; c < NB; ++c) tma_load_3d(S.a[stg][c], m, &S.full[stg], 64 * c, r0, unit);
                const size_t ti = band_off(kt, p.nkt) + (size_t)(4 * rb - 4 * kt);
                bulk_load(S.t[stg], tiles + ti * kTileBytes, 4 * kTileBytes, &S.full[stg]);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        const bool leader = elect_one();
        // rows side: A = K^T (MN-major SW128, M = dims: 64-dim atoms 16384 B apart = the leading
        // byte offset, or the zero block), B = tiles as [128 rows x 128 keys] (MN-major, no swizzle:
        // there the leading byte offset is the K-direction step, 8-key groups 128 B apart, and the
        // stride byte offset the MN-direction step, 8-row groups 2048 B apart); key side: A = tiles
        // as [128 keys x 128 rows] (K-major, no swizzle: leading = K step, 8-row groups 2048 B
        // apart; stride = M step, 8-key groups 128 B apart), B = khat rows (MN-major SW128, N = dims).
        constexpr uint32_t ID = ROWS ? idesc_bf16(128, 128, 1, 1) : idesc_bf16(128, DH, 0, 1);
        bool ok = true;
        for (int i = 0; i < n && ok; ++i) {
            const int stg = i % NS;
            if (!wwait(&S.full[stg], (i / NS) & 1, abort)) { ok = false; break; }
            tc_fence_after();
            if (leader) {
                const uint32_t aa = smem_u32(S.a[stg][0]), ta = smem_u32(S.t[stg]);
                const uint32_t lbo_a = (DH == 64) ? smem_u32(S.zero) - aa : 16384u;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                    if (ROWS) {
                        const uint64_t da = smem_desc(aa + kk * 2048u, lbo_a, 1024, kSwizzle128B);
                        const uint64_t db = smem_desc(ta + kk * 256u, 128, 2048, kSwizzleNone);
                        umma_f16(tmem, da, db, ID, acc);
                    } else {
                        const uint64_t da = smem_desc(ta + kk * 4096u, 2048, 128, kSwizzleNone);
                        const uint64_t db = smem_desc(aa + kk * 2048u, 16384, 1024, kSwizzle128B);
                        umma_f16(tmem, da, db, ID, acc);
                    }
                }
                umma_commit(&S.empty[stg]);
            }
            __syncwarp();
        }
        if (leader && ok) umma_commit(&S.done);
        __syncwarp();
    }
    // ---- epilogue
    const bool ok = wwait(&S.done, 0, abort);
    if (ok) {
        tc_fence_after();
        const uint32_t tl = (uint32_t)(warp * 32) << 16;
        if (ROWS) {
            // lane = dim d, columns = the block's 128 rows
            const int d = warp * 32 + lane;
            const float f = o < p.G ? p.scale : p.alpha[kvh];
#pragma unroll 1
            for (int c = 0; c < 128; c += 16) {
                float v[16];
                tmem_ld16(tmem + tl + c, v);
                if (d < DH) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int i = blk * 128 + c + e;
                        if (i < T) {
                            if (o < p.G)
                                p.dqr[(((size_t)b * p.H + kvh * p.G + o) * T + i) * DH + d] = f * v[e];
                            else
                                p.dkh_rows[((size_t)unit * T + i) * DH + d] = f * v[e];
                        }
                    }
                }
            }
        } else {
            // lane = key, columns = dims
            const int j = blk * 128 + warp * 32 + lane;
            const float f = p.alpha[kvh];
#pragma unroll 1
            for (int c = 0; c < DH; c += 16) {
                float v[16];
                tmem_ld16(tmem + tl + c, v);
                if (j < T) {
                    float* dst = p.dkh_keys + ((size_t)unit * T + j) * DH + c;
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4*>(dst + e) = make_float4(f * v[e], f * v[e + 1], f * v[e + 2], f * v[e + 3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort && tid == 0) drain_pause(10000000ull);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, NCOL);
    }
}

// =========================================================================== post pass
// N consecutive floats (N = 1 or 2).
template <int N>
__device__ __forceinline__ void ld_f(const float* src, float (&f)[N]) {
    if constexpr (N == 2) {
        const float2 v = *reinterpret_cast<const float2*>(src);
        f[0] = v.x, f[1] = v.y;
    } else {
        f[0] = src[0];
    }
}
template <int N>
__device__ __forceinline__ void st_bf(__nv_bfloat16* dst, const float (&f)[N]) {
    if constexpr (N == 2) *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(f[0], f[1]);
    else dst[0] = __float2bfloat16_rn(f[0]);
}

// grid (T, B), 256 threads: RoPE^T of dqrot / dkrot, the query-norm and key-normalisation
// Jacobians (khat recomputed from the raw key in fp32), casts; da_q (row sums of w over the key
// tiles and their quarters), da_k.  A warp per head; lane l takes the rotation pairs
// (m, m + d/2) for m = l*PH .. l*PH+PH-1.
template <int DH>
__global__ void __launch_bounds__(256) k_bwd_post_tc(BwdTcParams p) {
    constexpr int HALF = DH / 2, PH = HALF / 32;
    const int t = blockIdx.x, b = blockIdx.y, T = p.T;
    __shared__ float s_cos[64], s_sin[64];
    __shared__ double s_f[HALF];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the RoPE frequencies, a few per warp (a kernel-parameter array read at a different index by
    // each lane serialises those reads)
    static_assert(HALF % 8 == 0, "frequencies split over the eight warps");
    if (lane < HALF / 8) s_f[warp * (HALF / 8) + lane] = p.rf.f[warp * (HALF / 8) + lane];
    __syncthreads();
    for (int m = threadIdx.x; m < HALF; m += blockDim.x) rope_cs((double)t, s_f[m], &s_cos[m], &s_sin[m]);
    __syncthreads();
    using bf = __nv_bfloat16;
    bf* dq = static_cast<bf*>(p.dq);
    bf* dk = static_cast<bf*>(p.dk);
    bf* dv = static_cast<bf*>(p.dv);
    const int m0 = lane * PH;
    float cs[PH], sn[PH];
#pragma unroll
    for (int e = 0; e < PH; ++e) cs[e] = s_cos[m0 + e], sn[e] = s_sin[m0 + e];
    for (int hh = warp; hh < p.H + p.Hkv; hh += 8) {
        const bool is_q = hh < p.H;
        const int h = is_q ? hh : hh - p.H;
        if (is_q) {
            const float* src = p.dqr + (((size_t)b * p.H + h) * T + t) * DH;
            bf* dst = dq + (((size_t)b * T + t) * p.H + h) * DH;
            float x0[PH], x1[PH], y0[PH], y1[PH], q0[PH], q1[PH];
            ld_f<PH>(src + m0, x0);
            ld_f<PH>(src + m0 + HALF, x1);
            float ss = 0.f, qy = 0.f;
#pragma unroll
            for (int e = 0; e < PH; ++e) {
                y0[e] = x0[e] * cs[e] + x1[e] * sn[e];          // rotation by -angle
                y1[e] = x1[e] * cs[e] - x0[e] * sn[e];
                q0[e] = q1[e] = 0.f;
            }
            float r = 1.f, k = 0.f;
            if (p.variant & kVarQNorm) {
                // q' = r q, r = 1/sqrt(mean(q^2) + eps): dq = r (dq' - q' <q', dq'> / d)
                const bf* qraw = static_cast<const bf*>(p.q) + (((size_t)b * T + t) * p.H + h) * DH;
#pragma unroll
                for (int e = 0; e < PH; ++e) {
                    q0[e] = __bfloat162float(qraw[m0 + e]);
                    q1[e] = __bfloat162float(qraw[m0 + e + HALF]);
                    ss += q0[e] * q0[e] + q1[e] * q1[e];
                    qy += q0[e] * y0[e] + q1[e] * y1[e];
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    ss += __shfl_xor_sync(0xffffffffu, ss, o);
                    qy += __shfl_xor_sync(0xffffffffu, qy, o);
                }
                r = 1.f / sqrtf(ss / (float)DH + kQNormEps);
                k = r * r * qy / (float)DH;
            }
            float z0[PH], z1[PH];
#pragma unroll
            for (int e = 0; e < PH; ++e) {
                z0[e] = r * (y0[e] - q0[e] * k);
                z1[e] = r * (y1[e] - q1[e] * k);
            }
            st_bf<PH>(dst + m0, z0);
            st_bf<PH>(dst + m0 + HALF, z1);
        } else {
            const size_t u = (size_t)b * p.Hkv + h;
            const size_t row = (u * T + t) * DH;
            const bf* kraw = static_cast<const bf*>(p.k) + (((size_t)b * T + t) * p.Hkv + h) * DH;
            float r0[PH], r1[PH], a0[PH], a1[PH], c0[PH], c1[PH], v0[PH], v1[PH];
            ld_f<PH>(p.dkr + row + m0, r0);
            ld_f<PH>(p.dkr + row + m0 + HALF, r1);
            ld_f<PH>(p.dkh_keys + row + m0, a0);
            ld_f<PH>(p.dkh_keys + row + m0 + HALF, a1);
            ld_f<PH>(p.dkh_rows + row + m0, c0);
            ld_f<PH>(p.dkh_rows + row + m0 + HALF, c1);
            ld_f<PH>(p.dv32 + row + m0, v0);
            ld_f<PH>(p.dv32 + row + m0 + HALF, v1);
            float g0[PH], g1[PH], k0[PH], k1[PH];
            float proj = 0.f, ss = 0.f;
#pragma unroll
            for (int e = 0; e < PH; ++e) {
                g0[e] = a0[e] + c0[e] + r0[e] * cs[e] + r1[e] * sn[e];
                g1[e] = a1[e] + c1[e] + r1[e] * cs[e] - r0[e] * sn[e];
                k0[e] = __bfloat162float(kraw[m0 + e]);
                k1[e] = __bfloat162float(kraw[m0 + e + HALF]);
                ss += k0[e] * k0[e] + k1[e] * k1[e];
                proj += g0[e] * k0[e] + g1[e] * k1[e];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                proj += __shfl_xor_sync(0xffffffffu, proj, o);
                ss += __shfl_xor_sync(0xffffffffu, ss, o);
            }
            const float n = fmaxf(sqrtf(ss), 1e-12f);
            const float inv = 1.f / n;
            // khat = k / n:  dk = (g - khat <khat, g>) / n
            const float pr = proj * inv * inv;
            float z0[PH], z1[PH];
#pragma unroll
            for (int e = 0; e < PH; ++e) {
                z0[e] = (g0[e] - k0[e] * pr) * inv;
                z1[e] = (g1[e] - k1[e] * pr) * inv;
            }
            bf* dst = dk + (((size_t)b * T + t) * p.Hkv + h) * DH;
            bf* dvd = dv + (((size_t)b * T + t) * p.Hkv + h) * DH;
            st_bf<PH>(dst + m0, z0);
            st_bf<PH>(dst + m0 + HALF, z1);
            st_bf<PH>(dvd + m0, v0);
            st_bf<PH>(dvd + m0 + HALF, v1);
        }
    }
    // da_q: the row sums of w over the key tiles up to the row's and their four quarters (one
    // float4 per key tile, contiguous per row), a warp per KV head; key tiles whose walked steps
    // stop above the row contribute 0 (their entries are not written); da_k from the key pass
    const int nk = t / 128 + 1;
    for (int h = warp; h < p.Hkv; h += 8) {
        const size_t u = (size_t)b * p.Hkv + h;
        const float4* part = reinterpret_cast<const float4*>(p.daq_part + (u * p.Tpk + t) * p.nkt * 4);
        float sw = 0.f;
        for (int kt = lane; kt < nk; kt += 32) {
            if (last_step(p, (int)u, kt) < t / ST) continue;
            const float4 v = part[kt];
            sw += (v.x + v.y) + (v.z + v.w);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sw += __shfl_xor_sync(0xffffffffu, sw, o);
        if (lane == 0) {
            const size_t src = ((size_t)b * T + t) * p.Hkv + h;
            p.da_q[src] = sw * sig_over_sp_f(p.a_q[src]);
            p.da_k[src] = p.dak32[u * T + t];
        }
    }
}

// =========================================================================== launcher
// head_dim 128 with four query heads per KV head does not fit the key-major pass's shared
// memory (the step's query and dA rows of four heads beside the key tile's four operands)
bool bwd_tc_supported(int d, int G) { return (d == 64 && G >= 1 && G <= 4) || (d == 128 && G >= 1 && G <= 3); }

template <int DH, int G>
static cudaError_t bwd_tc_inst(const BwdTcParams& p, cudaStream_t s) {
    static_assert(sizeof(key::Smem<DH, G>) + 1024 <= 232448, "key-major pass: shared memory budget");
    const int BH = p.B * p.H, BK = p.B * p.Hkv;
    cudaError_t e;
    {
        UA_PROFILE("k_bwd_prep_tc", s);
        k_bwd_prep_tc<DH><<<dim3(p.T, p.B), 256, 0, s>>>(p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CUtensorMap m_khk, m_krk, m_v, m_khq, m_q, m_ad, m_lq, m_lk, m_pb, m_lse2, m_dlt, m_kh128;
    if (!map_rows_bwd(&m_khk, p.kh, DH, p.T, BK, 128) || !map_rows_bwd(&m_krk, p.kr, DH, p.T, BK, 128) ||
        !map_v_bwd(&m_v, p.v, DH, p.Hkv, p.T, p.B) || !map_rows_bwd(&m_khq, p.kh, DH, p.T, BK, ST) ||
        !map_rows_bwd(&m_q, p.qr, DH, p.T, BH, ST) || !map_rows_bwd(&m_ad, p.ad, DH, p.T, BH, ST) ||
        !map_vec_bwd(&m_lq, p.lq2, p.T, p.Tp, BK, ST) || !map_vec_bwd(&m_lk, p.lk2, p.T, p.Tp, BK, 128) ||
        !map_vec_bwd(&m_pb, p.pb, p.Tpk, p.Tpk, BK * p.nst, 128) ||
        !map_vec_bwd(&m_lse2, p.lse2, p.T, p.Tp, BH, ST) || !map_vec_bwd(&m_dlt, p.delta, p.T, p.Tp, BH, ST) ||
        !map_rows_bwd(&m_kh128, p.kh, DH, p.T, BK, 128))
        return cudaErrorInvalidValue;
    {
        const size_t smem = sizeof(bnd::Smem<DH>) + 1024;
        if ((e = cudaFuncSetAttribute(k_bwd_bound_tc<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return e;
        UA_PROFILE("k_bwd_bound_tc", s);
        k_bwd_bound_tc<DH><<<dim3(BK, p.nkt), 128, smem, s>>>(m_khk, m_khq, m_lq, m_lk, p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        const size_t smem = sizeof(key::Smem<DH, G>) + 1024;
        if ((e = cudaFuncSetAttribute(k_bwd_key_tc<DH, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
            cudaSuccess)
            return e;
        UA_PROFILE("k_bwd_key_tc", s);
        k_bwd_key_tc<DH, G><<<dim3(BK, p.nkt), 128 * kKeyQ + 32, smem, s>>>(m_khk, m_krk, m_v, m_khq, m_q, m_ad, m_lq, m_lk,
                                                               m_pb, m_lse2, m_dlt, p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        const size_t smem = sizeof(gemm::Smem<DH>) + 1024;
        if ((e = cudaFuncSetAttribute(k_bwd_gemm_tc<DH, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(k_bwd_gemm_tc<DH, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        {
            UA_PROFILE("k_bwd_rowgemm_tc", s);
            k_bwd_gemm_tc<DH, true><<<dim3(p.nkt, G + 1, BK), 128, smem, s>>>(m_kh128, m_krk, p);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        {
            UA_PROFILE("k_bwd_keygemm_tc", s);
            k_bwd_gemm_tc<DH, false><<<dim3(p.nkt, BK), 128, smem, s>>>(m_kh128, m_krk, p);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        UA_PROFILE("k_bwd_post_tc", s);
        k_bwd_post_tc<DH><<<dim3(p.T, p.B), 256, 0, s>>>(p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        UA_PROFILE("k_bwd_dab", s);
        k_bwd_dab<<<p.Hkv, 256, 0, s>>>(p.dab, p.B, p.Hkv, p.nkt, p.dalpha, p.dbeta);
    }
    return cudaGetLastError();
}

template <int DH>
static cudaError_t bwd_tc_g(const BwdTcParams& p, cudaStream_t s) {
    switch (p.G) {
        case 1: return bwd_tc_inst<DH, 1>(p, s);
        case 2: return bwd_tc_inst<DH, 2>(p, s);
        case 3: return bwd_tc_inst<DH, 3>(p, s);
        case 4:
            if constexpr (DH == 64) return bwd_tc_inst<DH, 4>(p, s);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_bwd_tc(const BwdTcParams& p, cudaStream_t s) {
    return p.d == 64 ? bwd_tc_g<64>(p, s) : bwd_tc_g<128>(p, s);
}

}  // namespace ua
