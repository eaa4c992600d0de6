// k_prefill_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) kernels of the bf16 prefill:
// the decay boundary pass and the fused biased attention forward.
//
// Decay structure (see ua.h for the formulas): L2-normalised keys, three rates combined by
// a geometric mean, log space, causal accumulation into Lambda (ai4snews synopsis, Fig. 1
// caption; paperlayer.ai summary §4, §4.1), applied inside the softmax without writing the
// T x T mask (paperlayer.ai summary App. C).
//
// Both kernels compute key-key and key-query products TRANSPOSED: the 128 keys j of a key
// tile sit on the 128 TMEM lanes and the query rows l (or i) run along the columns.  One
// thread then owns one key column, so the causal sum of D[l, j] over l is a sequential
// scan in that thread's registers, with no cross-lane traffic.
#include <cudaTypedefs.h>

#include "tc_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

using namespace tc;

namespace {
constexpr float kLog2e = 1.4426950408889634f;

// --------------------------------------------------------------- tensor maps (host)
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// bf16 tensor viewed as [outer][T][d] (d contiguous), box = 64 columns x 128 rows x 1,
// 128-byte swizzle: one box is a K-major SW128 operand tile of 128 rows.
bool map_rows_bf16(CUtensorMap* m, const void* base, int d, int T, int outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)outer};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)T * d * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 activation in the caller's [B][T][Hkv][d] layout, box = 64 x 1 head x 128 tokens x 1.
bool map_act_bf16(CUtensorMap* m, const void* base, int d, int Hkv, int T, int B) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)Hkv, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)Hkv * d * 2, (cuuint64_t)T * Hkv * d * 2};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// f32 rows of logical length T stored with row stride Tp (a multiple of 4), box = 128 x 1,
// no swizzle; reads past T are zero-filled.
bool map_vec_f32(CUtensorMap* m, const void* base, int T, int Tp, int outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)T, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)Tp * 4};
    cuuint32_t box[2] = {128, 1};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major SW128 descriptor of a 128-row bf16 tile stored as 64-column boxes of 16 KB:
// k-step kk (16 columns) lives in box kk/4 at byte offset (kk%4)*32 within each row.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kk) {
    return smem_desc(tile + (uint32_t)(kk >> 2) * 16384u + (uint32_t)(kk & 3) * 32u, 16, 1024, kSwizzle128B);
}

// Decay D[l, j] = 2^(lq2_l + lk2_j + log2(softplus(alpha*x + beta))/3), x = <khat_l, khat_j>;
// lq2 / lk2 are log2 of the rates over 3, so a zero rate (-inf) vetoes the product.
__device__ __forceinline__ float decay_tc(float x, float al, float be, float lq2, float lk2) {
    return ex2f(fmaf(log2_softplus(fmaf(al, x, be)), 0.33333334f, lq2 + lk2));
}

}  // namespace

// ================================================================ boundary pass
// grid (ceil(T/128) key tiles, Hkv, B); 192 threads: warps 0-3 decay (one key per thread,
// TMEM lanes 0-127), warp 4 TMA producer, warp 5 MMA issuer.  For key tile kt it sweeps the
// query tiles t = kt .. nqt-1: X^T = Khat_k * Khat_t^T (M=128 keys, N=128 rows) into one of
// two TMEM buffers, and each thread sums D over its row of X^T.
namespace bnd {
constexpr int NS = 3;   // query-tile stages
struct Smem {
    alignas(1024) uint8_t a[2][16384];          // Khat of the key tile (1 or 2 boxes)
    alignas(1024) uint8_t b[NS][2][16384];      // Khat of query tile (1 or 2 boxes)
    alignas(16) float lq[NS][128];              // lq2 of the query tile rows
    alignas(8) uint64_t full[NS], empty[NS], tfull[2], tempty[2], abar;
    uint32_t tmem;
    int abort;
};
}  // namespace bnd

struct BoundaryTcParams {
    int B, T, Tp, Hkv, d, nqt;
    const float* lk2;    // [B*Hkv][Tp]
    const float* alpha;
    const float* beta;
    float* pb;           // [B*Hkv][nqt][Tp]
    float* bfinal;       // [B*Hkv][T] or NULL
};

template <int DH>
__global__ void __launch_bounds__(192, 1)
k_boundary_tc(const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_lq,
              BoundaryTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    bnd::Smem& S = *reinterpret_cast<bnd::Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int NB = DH / 64;                  // 64-column boxes per tile
    constexpr int KSTEPS = DH / 16;
    constexpr uint32_t IDESC = idesc_bf16(128, 128, 0, 0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kt = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int unit = b * p.Hkv + kvh;
    const int T = p.T;
    const int ntile = p.nqt - kt;                // query tiles kt .. nqt-1
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < bnd::NS; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], 1 + 4);       // MMA commit + 4 decay warps (lq reads)
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.tfull[i], 1);
            mbar_init(&S.tempty[i], 4);
        }
        mbar_init(&S.abar, 1);
        S.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tmap(&tm_kh);
            prefetch_tmap(&tm_lq);
            mbar_expect_tx(&S.abar, NB * 16384);
            for (int bx = 0; bx < NB; ++bx) tma_load_3d(S.a[bx], &tm_kh, &S.abar, bx * 64, kt * 128, unit);
            for (int it = 0; it < ntile; ++it) {
                const int s = it % bnd::NS;
                if (it >= bnd::NS && !mbar_wait(&S.empty[s], ((it / bnd::NS) - 1) & 1, abort)) break;
                const int t = kt + it;
                mbar_expect_tx(&S.full[s], NB * 16384 + 512);
                for (int bx = 0; bx < NB; ++bx) tma_load_3d(S.b[s][bx], &tm_kh, &S.full[s], bx * 64, t * 128, unit);
                tma_load_2d(S.lq[s], &tm_lq, &S.full[s], t * 128, unit);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            if (mbar_wait(&S.abar, 0, abort)) {
                for (int it = 0; it < ntile; ++it) {
                    const int s = it % bnd::NS, buf = it & 1;
                    if (!mbar_wait(&S.full[s], (it / bnd::NS) & 1, abort)) break;
                    if (it >= 2 && !mbar_wait(&S.tempty[buf], ((it >> 1) - 1) & 1, abort)) break;
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(S.a[0]), b0 = smem_u32(S.b[s][0]);
                    for (int kk = 0; kk < KSTEPS; ++kk)
                        umma_f16(tmem + buf * 128, kmajor_desc(a0, kk), kmajor_desc(b0, kk), IDESC, kk > 0);
                    umma_commit(&S.empty[s]);
                    umma_commit(&S.tfull[buf]);
                }
            }
        }
    } else {
        // decay warps: thread owns key j
        const int jl = warp * 32 + lane;
        const int j = kt * 128 + jl;
        const bool jvalid = j < T;
        const float al = p.alpha[kvh], be = p.beta[kvh];
        const float lk2 = jvalid ? p.lk2[(size_t)unit * p.Tp + j] : -INFINITY;
        float* pb = p.pb + (size_t)unit * p.nqt * p.Tp;
        if (jvalid)
            for (int t = 0; t < kt; ++t) pb[(size_t)t * p.Tp + j] = 0.f;
        float acc = 0.f;
        for (int it = 0; it < ntile; ++it) {
            const int s = it % bnd::NS, buf = it & 1;
            const int t = kt + it;
            if (!mbar_wait(&S.tfull[buf], (it >> 1) & 1, abort)) break;
            if (!mbar_wait(&S.full[s], (it / bnd::NS) & 1, abort)) break;   // lq of this stage landed
            tc_fence_after();
            float tile = 0.f;
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
                float x[32];
                tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + buf * 128 + ch * 32, x);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int l = t * 128 + ch * 32 + c;
                    const float D = decay_tc(x[c], al, be, S.lq[s][ch * 32 + c], lk2);
                    tile += (l > j && l < T) ? D : 0.f;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&S.tempty[buf]);
                mbar_arrive(&S.empty[s]);
            }
            if (jvalid) pb[(size_t)t * p.Tp + j] = acc;
            acc += tile;
        }
        if (jvalid && p.bfinal && !*abort) p.bfinal[(size_t)unit * T + j] = -acc;
    }

    __syncthreads();
    if (*abort && threadIdx.x == 0) drain_pause(10000000ull);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ================================================================ launchers

size_t boundary_tc_smem() { return sizeof(bnd::Smem) + 1024; }

cudaError_t launch_boundary_tc(const BoundaryParams& bp, const void* kh_bf16, const float* lq2, const float* lk2,
                               int Tp, cudaStream_t s) {
    CUtensorMap tm_kh, tm_lq;
    if (!map_rows_bf16(&tm_kh, kh_bf16, bp.d, bp.T, bp.B * bp.Hkv)) return cudaErrorInvalidValue;
    if (!map_vec_f32(&tm_lq, lq2, bp.T, Tp, bp.B * bp.Hkv)) return cudaErrorInvalidValue;
    BoundaryTcParams p;
    p.B = bp.B; p.T = bp.T; p.Tp = Tp; p.Hkv = bp.Hkv; p.d = bp.d; p.nqt = bp.nqt;
    p.lk2 = lk2; p.alpha = bp.alpha; p.beta = bp.beta; p.pb = bp.pb; p.bfinal = bp.bfinal;
    const size_t smem = boundary_tc_smem();
    dim3 grid((bp.T + 127) / 128, bp.Hkv, bp.B);
    UA_PROFILE("k_boundary_tc", s);
    if (bp.d == 64) {
        cudaError_t e = cudaFuncSetAttribute(k_boundary_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k_boundary_tc<64><<<grid, 192, smem, s>>>(tm_kh, tm_lq, p);
    } else {
        cudaError_t e = cudaFuncSetAttribute(k_boundary_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k_boundary_tc<128><<<grid, 192, smem, s>>>(tm_kh, tm_lq, p);
    }
    return cudaGetLastError();
}


// ================================================================ fused forward
// grid (nqt, Hkv, B): one CTA per (batch, KV head, 128-row query tile) serving all G query
// heads of the group, so the decay tile is built once for the G heads.  224 threads:
// warps 0-3 decay/softmax/epilogue (thread = key j while streaming key tiles, thread =
// query row i in the epilogue), warp 4 TMA producer, warp 5 MMA issuer, warp 6 idle helper.
//
// Per key tile kt <= qt:
//   X^T = Khat_k Khat_q^T and S_h^T = Krope_k Qrope_h^T in two 64-row halves (TMEM ping-pong);
//   thread j turns X^T into D, scans it down its column on top of the boundary prefix Pb,
//   and keeps Lambda (log2 units) for the 128 rows in registers; then for each head
//   P = 2^(S*scale*log2e + Lambda - M_i), written MN-major (rows i contiguous) to smem.
//   M_i = scale*||q_i||*log2e bounds every logit of row i (keys are unit vectors, Lambda <= 0),
//   so no running max and no rescaling are needed.  O_h += P V and l_h += P 1 on the tensor
//   cores (accumulators in TMEM).
namespace fwd {
constexpr int NKK = 2;   // key-tile stages
template <int G>
struct Smem {
    alignas(1024) uint8_t kq[16384];             // Khat of the query tile rows
    alignas(1024) uint8_t q[G][16384];           // Qrope of the G heads
    alignas(1024) uint8_t kh[NKK][16384];        // Khat of the key tile
    alignas(1024) uint8_t kr[NKK][16384];        // Krope of the key tile
    alignas(1024) uint8_t v[NKK][16384];         // V of the key tile
    alignas(1024) uint8_t p[32768];              // P, MN-major SW128: [2 row blocks][16 k groups][8][128 B]
    alignas(1024) uint8_t ones[1024];            // all-ones bf16 operand for the row sums
    alignas(16) float lq[128];                   // lq2 of the query rows
    alignas(16) float mq[G][128];                // row bound M_i (log2 units) per head
    alignas(16) float lk[NKK][128];              // lk2 of the key tile
    alignas(16) float pb[NKK][128];              // boundary prefix of the key tile at this query tile
    alignas(8) uint64_t qfull, kkfull[NKK], kkempty[NKK], xsfull[2], xsempty[2], pfull, pempty, ofull;
    uint32_t tmem;
    int abort;
};
}  // namespace fwd

struct FwdTcParams {
    int B, T, Tp, H, Hkv, nqt;
    float scale_log2e;
    const float* alpha;
    const float* beta;
    const void* g;       // [B,T,H,64] bf16
    void* o;             // [B,T,H,64] bf16
    float* lse;          // [B,H,T] or NULL
};

template <int G>
__global__ void __launch_bounds__(224, 1)
k_fwd_tc(const __grid_constant__ CUtensorMap tm_kh, const __grid_constant__ CUtensorMap tm_kr,
         const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_v,
         const __grid_constant__ CUtensorMap tm_lq, const __grid_constant__ CUtensorMap tm_lk,
         const __grid_constant__ CUtensorMap tm_mq, const __grid_constant__ CUtensorMap tm_pb, FwdTcParams p) {
    constexpr int DH = 64;
    constexpr uint32_t ID_XS = idesc_bf16(128, 64, 0, 0);
    constexpr uint32_t ID_PV = idesc_bf16(128, 64, 1, 1);
    constexpr uint32_t ID_L = idesc_bf16(128, 16, 1, 0);
    constexpr uint32_t COL_O = 0, COL_L = G * DH, COL_XS = G * DH + G * 16;
    constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_XS + 128 <= TMEM_COLS, "TMEM budget");
    extern __shared__ uint8_t smem_raw[];
    using SM = fwd::Smem<G>;
    SM& S = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt = gridDim.x - 1 - blockIdx.x;          // heaviest query tiles first
    const int kvh = blockIdx.y, b = blockIdx.z;
    const int unit = b * p.Hkv + kvh;
    const int T = p.T;
    const int ntile = qt + 1;
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        mbar_init(&S.qfull, 1);
        for (int s = 0; s < fwd::NKK; ++s) {
            mbar_init(&S.kkfull[s], 1);
            mbar_init(&S.kkempty[s], 1 + 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.xsfull[i], 1);
            mbar_init(&S.xsempty[i], 4);
        }
        mbar_init(&S.pfull, 4);
        mbar_init(&S.pempty, 1);
        mbar_init(&S.ofull, 1);
        S.abort = 0;
        fence_barrier_init();
    }
    if (warp == 6) {
        // all-ones operand (bf16 1.0 = 0x3F80); any layout of it reads as ones
        uint32_t* o32 = reinterpret_cast<uint32_t*>(S.ones);
        for (int i = lane; i < 256; i += 32) o32[i] = 0x3F803F80u;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const CUtensorMap* maps[8] = {&tm_kh, &tm_kr, &tm_q, &tm_v, &tm_lq, &tm_lk, &tm_mq, &tm_pb};
            for (int m = 0; m < 8; ++m) prefetch_tmap(maps[m]);
            mbar_expect_tx(&S.qfull, 16384 * (1 + G) + 512 * (1 + G));
            tma_load_3d(S.kq, &tm_kh, &S.qfull, 0, qt * 128, unit);
            for (int h = 0; h < G; ++h) tma_load_3d(S.q[h], &tm_q, &S.qfull, 0, qt * 128, b * p.H + kvh * G + h);
            tma_load_2d(S.lq, &tm_lq, &S.qfull, qt * 128, unit);
            for (int h = 0; h < G; ++h) tma_load_2d(S.mq[h], &tm_mq, &S.qfull, qt * 128, b * p.H + kvh * G + h);
            for (int kt = 0; kt < ntile; ++kt) {
                const int s = kt % fwd::NKK;
                if (kt >= fwd::NKK && !mbar_wait(&S.kkempty[s], ((kt / fwd::NKK) - 1) & 1, abort)) break;
                mbar_expect_tx(&S.kkfull[s], 3 * 16384 + 2 * 512);
                tma_load_3d(S.kh[s], &tm_kh, &S.kkfull[s], 0, kt * 128, unit);
                tma_load_3d(S.kr[s], &tm_kr, &S.kkfull[s], 0, kt * 128, unit);
                tma_load_4d(S.v[s], &tm_v, &S.kkfull[s], 0, kvh, kt * 128, b);
                tma_load_2d(S.lk[s], &tm_lk, &S.kkfull[s], kt * 128, unit);
                tma_load_2d(S.pb[s], &tm_pb, &S.kkfull[s], kt * 128, unit * p.nqt + qt);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t xs_use = 0, p_use = 0;
            bool ok = mbar_wait(&S.qfull, 0, abort);
            const uint32_t a_ones = smem_u32(S.ones);
            const uint64_t d_ones = smem_desc(a_ones, 256, 128, kSwizzleNone);
            for (int kt = 0; ok && kt < ntile; ++kt) {
                const int s = kt % fwd::NKK;
                if (!mbar_wait(&S.kkfull[s], (kt / fwd::NKK) & 1, abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t akh = smem_u32(S.kh[s]), akr = smem_u32(S.kr[s]), av = smem_u32(S.v[s]);
                const uint32_t ap = smem_u32(S.p);
                // issue one 64-row half of X^T (src = Khat_q) or S_h^T (src = Qrope_h)
                auto issue_half = [&](uint32_t a_tile, uint32_t b_tile, int half) -> bool {
                    const uint32_t buf = xs_use & 1;
                    if (xs_use >= 2 && !mbar_wait(&S.xsempty[buf], ((xs_use >> 1) - 1) & 1, abort)) return false;
                    tc_fence_after();
                    const uint32_t bt = b_tile + (uint32_t)half * 8192u;
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem + COL_XS + buf * 64, kmajor_desc(a_tile, kk), kmajor_desc(bt, kk), ID_XS, kk > 0);
                    umma_commit(&S.xsfull[buf]);
                    ++xs_use;
                    return true;
                };
                auto issue_pv = [&](int h) -> bool {
                    if (!mbar_wait(&S.pfull, p_use & 1, abort)) return false;
                    tc_fence_after();
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
                        const uint64_t dp = smem_desc(ap + (uint32_t)kk * 2048u, 16384, 1024, kSwizzle128B);
                        const uint64_t dv = smem_desc(av + (uint32_t)kk * 2048u, 16384, 1024, kSwizzle128B);
                        umma_f16(tmem + COL_O + h * DH, dp, dv, ID_PV, acc);
                        umma_f16(tmem + COL_L + h * 16, dp, d_ones, ID_L, acc);
                    }
                    umma_commit(&S.pempty);
                    ++p_use;
                    return true;
                };
                const uint32_t akq = smem_u32(S.kq);
                if (!issue_half(akh, akq, 0) || !issue_half(akh, akq, 1)) { ok = false; break; }
                for (int h = 0; h <= G && ok; ++h) {
                    if (h < G) {
                        const uint32_t aq = smem_u32(S.q[h]);
                        if (!issue_half(akr, aq, 0) || !issue_half(akr, aq, 1)) { ok = false; break; }
                    }
                    if (h >= 1 && !issue_pv(h - 1)) { ok = false; break; }
                }
                if (!ok) break;
                umma_commit(&S.kkempty[s]);
                if (kt == ntile - 1) umma_commit(&S.ofull);
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------------ decay / softmax warps
        const int jl = warp * 32 + lane;
        const uint32_t tlane = (uint32_t)(warp * 32) << 16;
        const float al = p.alpha[kvh], be = p.beta[kvh];
        const float sl = p.scale_log2e;
        uint32_t xs_use = 0, p_use = 0;
        bool ok = mbar_wait(&S.qfull, 0, abort);
        uint8_t* pbase = S.p + (jl >> 3) * 1024 + (jl & 7) * 128;
        const int sw = jl & 7;
        for (int kt = 0; ok && kt < ntile; ++kt) {
            const int s = kt % fwd::NKK;
            const int j = kt * 128 + jl;
            if (!mbar_wait(&S.kkfull[s], (kt / fwd::NKK) & 1, abort)) { ok = false; break; }
            const float lk2 = S.lk[s][jl];
            float c = S.pb[s][jl];
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.kkempty[s]);
            const bool jv = j < T;
            // ---- Lambda (log2 units) for the 128 query rows of this tile
            float lam[128];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint32_t buf = xs_use & 1;
                if (ok && !mbar_wait(&S.xsfull[buf], (xs_use >> 1) & 1, abort)) ok = false;
                tc_fence_after();
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    float x[32];
                    tmem_ld32(tmem + tlane + COL_XS + buf * 64 + ch * 32, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int r = half * 64 + ch * 32 + e;
                        const int i = qt * 128 + r;
                        const float D = decay_tc(x[e], al, be, S.lq[r], lk2);
                        c += (i > j) ? D : 0.f;
                        lam[r] = -c * kLog2e;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.xsempty[buf]);
                ++xs_use;
            }
            if (!ok) break;
            // ---- per head: P = 2^(S*scale*log2e + Lambda - M_i), rows i > ... masked causally
            for (int h = 0; h < G && ok; ++h) {
                uint32_t packed[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t buf = xs_use & 1;
                    if (ok && !mbar_wait(&S.xsfull[buf], (xs_use >> 1) & 1, abort)) ok = false;
                    tc_fence_after();
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch) {
                        float x[32];
                        tmem_ld32(tmem + tlane + COL_XS + buf * 64 + ch * 32, x);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int r = half * 64 + ch * 32 + e;
                            const int i = qt * 128 + r;
                            float p0 = ex2f(fmaf(x[e], sl, lam[r] - S.mq[h][r]));
                            float p1 = ex2f(fmaf(x[e + 1], sl, lam[r + 1] - S.mq[h][r + 1]));
                            p0 = (jv && j <= i) ? p0 : 0.f;
                            p1 = (jv && j <= i + 1) ? p1 : 0.f;
                            __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
                            packed[(ch * 32 + e) >> 1] = *reinterpret_cast<uint32_t*>(&pr);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.xsempty[buf]);
                    ++xs_use;
                    if (half == 0) {
                        // the single P buffer must be free: PV of the previous use has completed
                        if (ok && p_use >= 1 && !mbar_wait(&S.pempty, (p_use - 1) & 1, abort)) ok = false;
                    }
                    // rows half*64 .. +63 of column j: 8 chunks of 8 rows, SW128 chunk swizzle
                    uint8_t* rowblk = pbase + half * 16384;
#pragma unroll
                    for (int ck = 0; ck < 8; ++ck) {
                        uint4 w4 = make_uint4(packed[ck * 4], packed[ck * 4 + 1], packed[ck * 4 + 2], packed[ck * 4 + 3]);
                        *reinterpret_cast<uint4*>(rowblk + ((ck ^ sw) << 4)) = w4;
                    }
                }
                if (!ok) break;
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.pfull);
                ++p_use;
            }
        }
        // ---- epilogue: thread = query row i; O_h / l_h * sigmoid(g), lse
        if (ok && mbar_wait(&S.ofull, 0, abort)) {
            tc_fence_after();
            const int i = qt * 128 + jl;
            for (int h = 0; h < G; ++h) {
                float o[64], l16[16];
                tmem_ld32(tmem + tlane + COL_O + h * DH, o);
                tmem_ld32(tmem + tlane + COL_O + h * DH + 32, o + 32);
                tmem_ld16(tmem + tlane + COL_L + h * 16, l16);
                tmem_wait_ld();
                if (i < T) {
                    const int hq = kvh * G + h;
                    const float l = l16[0];
                    if (!(l > 0.f) || !isfinite(l)) raise_status(UA_ERR_RANGE);
                    const float inv = 1.f / l;
                    const size_t off = (((size_t)b * T + i) * p.H + hq) * DH;
                    const __nv_bfloat16* gi = static_cast<const __nv_bfloat16*>(p.g) + off;
                    __nv_bfloat16* oi = static_cast<__nv_bfloat16*>(p.o) + off;
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        float gv[8], ov[8];
                        Vec16<__nv_bfloat16>::ld(gi + c8 * 8, gv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) ov[e] = o[c8 * 8 + e] * inv * sigmoid_f(gv[e]);
                        Vec16<__nv_bfloat16>::st(oi + c8 * 8, ov);
                    }
                    if (p.lse) p.lse[((size_t)b * p.H + hq) * T + i] = (S.mq[h][jl] + lg2f(l)) * 0.6931471805599453f;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort && threadIdx.x == 0) drain_pause(10000000ull);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

size_t fwd_tc_smem(int G) {
    switch (G) {
        case 1: return sizeof(fwd::Smem<1>) + 1024;
        case 2: return sizeof(fwd::Smem<2>) + 1024;
        case 3: return sizeof(fwd::Smem<3>) + 1024;
        default: return sizeof(fwd::Smem<4>) + 1024;
    }
}

bool fwd_tc_supported(int d, int G) { return d == 64 && G >= 1 && G <= 4; }

template <int G>
static cudaError_t fwd_tc_inst(const CUtensorMap* m, const FwdTcParams& p, cudaStream_t s) {
    const size_t smem = fwd_tc_smem(G);
    cudaError_t e = cudaFuncSetAttribute(k_fwd_tc<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.nqt, p.Hkv, p.B);
    UA_PROFILE("k_fwd_tc", s);
    k_fwd_tc<G><<<grid, 224, smem, s>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], p);
    return cudaGetLastError();
}

cudaError_t launch_fwd_tc(const FwdTcLaunch& L, cudaStream_t s) {
    CUtensorMap m[8];
    const int BH = L.B * L.H, BK = L.B * L.Hkv;
    if (!map_rows_bf16(&m[0], L.kh, 64, L.T, BK)) return cudaErrorInvalidValue;
    if (!map_rows_bf16(&m[1], L.kr, 64, L.T, BK)) return cudaErrorInvalidValue;
    if (!map_rows_bf16(&m[2], L.qr, 64, L.T, BH)) return cudaErrorInvalidValue;
    if (!map_act_bf16(&m[3], L.v, 64, L.Hkv, L.T, L.B)) return cudaErrorInvalidValue;
    if (!map_vec_f32(&m[4], L.lq2, L.T, L.Tp, BK)) return cudaErrorInvalidValue;
    if (!map_vec_f32(&m[5], L.lk2, L.T, L.Tp, BK)) return cudaErrorInvalidValue;
    if (!map_vec_f32(&m[6], L.mq, L.T, L.Tp, BH)) return cudaErrorInvalidValue;
    if (!map_vec_f32(&m[7], L.pb, L.T, L.Tp, BK * L.nqt)) return cudaErrorInvalidValue;
    FwdTcParams p;
    p.B = L.B; p.T = L.T; p.Tp = L.Tp; p.H = L.H; p.Hkv = L.Hkv; p.nqt = L.nqt;
    p.scale_log2e = L.scale * kLog2e;
    p.alpha = L.alpha; p.beta = L.beta; p.g = L.g; p.o = L.o; p.lse = L.lse;
    switch (L.H / L.Hkv) {
        case 1: return fwd_tc_inst<1>(m, p, s);
        case 2: return fwd_tc_inst<2>(m, p, s);
        case 3: return fwd_tc_inst<3>(m, p, s);
        case 4: return fwd_tc_inst<4>(m, p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ua
