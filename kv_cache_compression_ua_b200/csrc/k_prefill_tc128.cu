// k_prefill_tc128.cu -- tensor-core (tcgen05 / TMEM / TMA) fused forward of the bf16 prefill
// for head_dim 128: the 3B-shaped layer (24 query heads over 8 KV heads).
//
// Decay structure (see ua.h for the formulas): L2-normalised keys, three rates combined by a
// geometric mean in log space and accumulated causally into Lambda (ai4snews synopsis, Fig. 1
// caption; paperlayer.ai summary §4, §4.1), applied inside the softmax without writing the T x T
// mask (paperlayer.ai summary App. C).
//
// Same scheme as the head_dim-64 kernel (k_prefill_tc.cu): key-key and key-query products are
// computed TRANSPOSED, so one thread owns one key column of the decay and scans it in registers;
// one CTA serves the G query heads of a KV group so the decay is evaluated once per KV head; the
// boundary prefixes are handed from query tile to query tile inside the launch.  What head_dim
// 128 changes:
//   * The query tile is 64 rows.  With 128 rows the G = 3 query tiles (96 KB), the query-side
//     keys (32 KB), two key tiles (64 KB), V (32 KB) and the P tiles do not fit in 227 KB of
//     shared memory; with 64 rows they take 192 KB.
//   * The output is accumulated transposed, O_h^T = V^T P_h^T: 128 TMEM lanes = the 128 head
//     dimensions, 64 columns = the query rows, so the G accumulators take G * 64 columns
//     instead of G * 128 (three 128 x 128 accumulators, a row-sum accumulator and a ring of
//     logit tiles would need more than the 512 columns of an SM).
//   * The row sums l_h = P_h 1 are one accumulator for all heads: l_h^T = e_h^T P_h^T with a
//     one-hot operand e_h (row h all ones) puts head h's sums on TMEM lane h of 64 shared
//     columns.
#include <cudaTypedefs.h>

#include "tc_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

using namespace tc;

namespace {
constexpr float kLog2e128 = 1.4426950408889634f;
constexpr float kCbrtLn2_128 = 0.8849970445005177f;   // (ln 2)^(1/3): decay evaluated in log2 units
// Every P of a (query tile, key tile) underflows to exactly 0 when min_j Pb[j] * log2(e) >= 128
// (see the head_dim-64 kernel: the exponent of every probability is then <= -126).
constexpr float kSkipLog2_128 = 128.f;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn128() {
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

// bf16 [outer][T][128] (head dim contiguous), box = 64 columns x `rows` rows x 1, 128-byte
// swizzle: a tile is two boxes (head dims 0-63 and 64-127), each a K-major SW128 operand.
bool map_rows128(CUtensorMap* m, const void* base, int T, int outer, int rows) {
    auto fn = encode_fn128();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)outer};
    cuuint64_t strides[2] = {256, (cuuint64_t)T * 256};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// V in the caller's [B][T][Hkv][128] layout, box = 64 x 1 head x 128 tokens x 1.
bool map_v128(CUtensorMap* m, const void* base, int Hkv, int T, int B) {
    auto fn = encode_fn128();
    if (!fn) return false;
    cuuint64_t dims[4] = {128, (cuuint64_t)Hkv, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {256, (cuuint64_t)Hkv * 256, (cuuint64_t)T * Hkv * 256};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// f32 rows of logical length T, row stride Tp (a multiple of 4), box = `n` x 1; reads past T
// are zero-filled.
bool map_vec128(CUtensorMap* m, const void* base, int T, int Tp, int outer, int n) {
    auto fn = encode_fn128();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)T, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)Tp * 4};
    cuuint32_t box[2] = {(cuuint32_t)n, 1};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major SW128 descriptor of a bf16 tile of `rows` rows x 128 columns stored as two 64-column
// boxes: k-step kk (16 columns) lives in box kk/4 at byte offset (kk%4)*32 within each row.
__device__ __forceinline__ uint64_t kdesc128(uint32_t tile, int rows, int kk) {
    return smem_desc(tile + (uint32_t)(kk >> 2) * (uint32_t)(rows * 128) + (uint32_t)(kk & 3) * 32u, 16, 1024,
                     kSwizzle128B);
}
}  // namespace

namespace fwd128 {
constexpr int NWG = 4;      // decay warpgroups, 16 query rows each
constexpr int QR = 64;      // query rows per CTA
template <int G>
struct Cfg {
    // TMEM: O^T (G x 64 columns), row sums (64), then the ring of 64-column logit tiles
    static constexpr int NSLOT = (7 - G) < 4 ? (7 - G) : 4;
};
template <int G>
struct Smem {
    alignas(1024) uint8_t kq[16384];         // Khat of the 64 query rows: 2 boxes [64][64 d]
    alignas(1024) uint8_t q[G][16384];       // Qrope of the G heads, same layout
    alignas(1024) uint8_t kh[32768];         // Khat of the key tile: 2 boxes [128][64 d]
    alignas(1024) uint8_t kr[32768];         // Krope of the key tile
    alignas(1024) uint8_t v[32768];          // V of the key tile
    alignas(1024) uint8_t p[2][16384];       // P_h^T tiles, MN-major SW128 [16 key groups][8 keys][64 rows]
    alignas(1024) uint8_t onehot[4096 + 64]; // zeros except row 0 of a K-major 128 x 16 operand at +64
    alignas(128) float lq[QR];               // lq2 of the query rows
    alignas(128) float mq[G][QR];            // row bound M_i (log2 units) per head
    alignas(128) float lk[128];              // lk2 of the key tile
    alignas(16) float pb[2][128];            // boundary prefix Pb of the key tile, two stages
    alignas(16) float pbc[2][128];           // chunked pruning: the prefix at the 128-row chunk's start
    int pbskip[2];                           // 0 compute; 1 softmax skipped; 2 decay skipped too
    alignas(16) float pinc[2][128];          // inclusive prefix handed to the publisher warp
    alignas(16) float tot[3][NWG][128];      // per-quarter column sums (without the key factor), ring of 3
    float shift[4 * NWG];                    // per decay warp: max M_i over its quarter and the G heads
    float lsum[G][QR];                       // row sums, staged for the epilogue
    alignas(8) uint64_t qfull, khfull, khempty, krfull, krempty, vfull, vempty, xsfull[4], xsempty[4], pfull[2],
        pempty[2], ofull, cfull[3][NWG], pbfull[2], pbempty[2], pubfull[2], pubempty[2], lfull[NWG];
    uint32_t tmem;
    int ticket;
    int abort;
};
#define UA_TMA_DST(G_, m, a) static_assert(offsetof(Smem<G_>, m) % (a) == 0, "TMA destination alignment")
#define UA_TMA_DSTS(G_) UA_TMA_DST(G_, kq, 1024); UA_TMA_DST(G_, q, 1024); UA_TMA_DST(G_, kh, 1024); \
    UA_TMA_DST(G_, kr, 1024); UA_TMA_DST(G_, v, 1024); UA_TMA_DST(G_, p, 1024); UA_TMA_DST(G_, lq, 128); \
    UA_TMA_DST(G_, mq, 128); UA_TMA_DST(G_, lk, 128); UA_TMA_DST(G_, onehot, 16)
UA_TMA_DSTS(1);
UA_TMA_DSTS(2);
UA_TMA_DSTS(3);
UA_TMA_DSTS(4);
#undef UA_TMA_DSTS
#undef UA_TMA_DST
static_assert(sizeof(Smem<4>) + 1024 <= 232448, "shared memory budget");
}  // namespace fwd128

struct FwdTc128Params {
    int B, T, Tp, Tpk, H, Hkv, nqt, nkt;
    float scale_log2e;
    const float* alpha;
    const float* beta;
    const void* g;       // [B,T,H,128] bf16
    void* o;             // [B,T,H,128] bf16
    float* lse;          // [B,H,T] or NULL
    float* pincl;        // [B*Hkv*nqt][Tpk] inclusive column prefixes published per 64-row query tile
    unsigned* flags;     // [B*Hkv][nqt][nkt] publication counters; then ticket, skip counter
    float* b_final;      // [B*Hkv][T] or NULL
    int nunits;          // B * Hkv
    float prune_thr;     // chunked pruned prefill (128-row chunks): -log p, +inf = dense
    unsigned* fix_count; // rows whose shifted row sum fell below 2^-60, listed for k_fwd_fix
    int* fix_list;       // (b*H + h)*T + i per listed row
};

// Wait (all lanes) until *f >= target, acquire semantics, bounded.
__device__ __forceinline__ bool wait_counter128(const unsigned* f, unsigned target, volatile int* abort, int lane) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 0;; ++it) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
        if (__all_sync(0xffffffffu, v >= target)) return true;
        if ((it & 63u) == 63u) {
            const bool stop = __shfl_sync(0xffffffffu, (int)(*abort != 0 || globaltimer() - t0 > wait_limit_ns()), 0);
            if (stop) {
                if (lane == 0 && !*abort) {
                    raise_status(UA_ERR_TIMEOUT);
                    *abort = 1;
                }
                return false;
            }
        }
        __nanosleep(64);
    }
}

// 16 rows of one key column of the decay tile: D / (r_k^(1/3) (ln 2)^(1/3)) from the
// similarity x and the row's lq2 = log2(r_q)/3, scanned into c; lam[r] = running sum after
// row r.  MASK: only rows rlo <= r < rhi accumulate (the causal diagonal, the sequence end).
template <bool MASK>
__device__ __forceinline__ void decay16r(const uint32_t (&x)[16], const float* lq, int rlo, int rhi, float al2,
                                         float be2, float& c, float (&lam)[16]) {
#pragma unroll
    for (int r4 = 0; r4 < 16; r4 += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(lq + r4);   // shared memory broadcast
        const float lv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = r4 + e;
            const float dq =
                ex2f(fmaf(log2_softplus_over_ln2(fmaf(al2, __uint_as_float(x[r]), be2)), 0.33333334f, lv[e]));
            if (MASK) c += (r >= rlo && r < rhi) ? dq : 0.f;
            else c += dq;
            lam[r] = c;
        }
    }
}

// 16 rows of one key column of P_h: P = 2^(S*scale*log2e + lam), packed to bf16 and stored as
// two 16-byte chunks (8 rows each) of the key's 128-byte row of the MN-major P^T tile.  MASK:
// only rows r >= rlo are kept (the causal diagonal).
template <bool MASK>
__device__ __forceinline__ void probs16r(const uint32_t (&x)[16], float sl, const float (&lam)[16], int rlo,
                                         uint8_t* prow, int ck0, int sw) {
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const int r = cc * 8 + e;
            float p0 = ex2f(fmaf(__uint_as_float(x[r]), sl, lam[r]));
            float p1 = ex2f(fmaf(__uint_as_float(x[r + 1]), sl, lam[r + 1]));
            if (MASK) {
                p0 = (r >= rlo) ? p0 : 0.f;
                p1 = (r + 1 >= rlo) ? p1 : 0.f;
            }
            __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
            w4[e >> 1] = *reinterpret_cast<uint32_t*>(&pr);
        }
        *reinterpret_cast<uint4*>(prow + (((ck0 + cc) ^ sw) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
}

// One CTA per (batch, KV head, 64-row query tile) for all G query heads; 640 threads:
//   warps 0-15  decay/softmax: warpgroup w = warp/4 owns query rows 16w .. 16w+15; while
//               streaming key tiles, thread = key j (TMEM lane)
//   warp 16     TMA producer
//   warp 17     MMA issuer of the logit ring (X^T, then S_h^T of each head: M 128 keys, N 64 rows)
//   warp 18     boundary look-back (Pb of each key tile from the previous query tile) and publisher
//   warp 19     MMA issuer of O_h^T += V^T P_h^T and of the row sums
// Key tile kt (128 keys) runs from 0 to qt/2, the tile holding the CTA's rows.  Pb(qt, kt) is the
// inclusive prefix published by query tile qt-1 for kt; for the tile holding the CTA's rows when
// qt is even, no earlier row lies below any of its keys and Pb = 0.
template <int G, bool EARLY>
__global__ void __launch_bounds__(640, 1)
k_fwd_tc128(const __grid_constant__ CUtensorMap tm_khk, const __grid_constant__ CUtensorMap tm_khq,
            const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_q,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_lq,
            const __grid_constant__ CUtensorMap tm_lk, const __grid_constant__ CUtensorMap tm_mq, FwdTc128Params p) {
    constexpr int NWG = fwd128::NWG, QR = fwd128::QR;
    constexpr int NSLOT = fwd128::Cfg<G>::NSLOT;
    constexpr uint32_t ID_XS = idesc_bf16(128, 64, 0, 0);   // keys x rows, both K-major
    constexpr uint32_t ID_PV = idesc_bf16(128, 64, 1, 1);   // head dims x rows, both MN-major
    constexpr uint32_t ID_L = idesc_bf16(128, 64, 0, 1);    // one-hot (K-major) x P^T (MN-major)
    constexpr uint32_t COL_O = 0, COL_L = G * 64, COL_XS = G * 64 + 64;
    constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_XS + NSLOT * 64 <= TMEM_COLS, "TMEM budget");
    extern __shared__ uint8_t smem_raw[];
    using SM = fwd128::Smem<G>;
    SM& S = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = p.T;
    volatile int* abort = &S.abort;

    if (threadIdx.x == 0) {
        mbar_init(&S.qfull, 1);
        mbar_init(&S.khfull, 1);
        mbar_init(&S.khempty, 1 + 4 * NWG);            // X MMA done + every decay warp read lk
        mbar_init(&S.krfull, 1);
        mbar_init(&S.krempty, 1);
        mbar_init(&S.vfull, 1);
        mbar_init(&S.vempty, 1);
        mbar_init(&S.ofull, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.pfull[i], 4 * NWG);
            mbar_init(&S.pempty[i], 1);
            mbar_init(&S.pbfull[i], 1);
            mbar_init(&S.pbempty[i], 4 * NWG + 2 + (EARLY ? 1 : 0));
            mbar_init(&S.pubfull[i], 4);
            mbar_init(&S.pubempty[i], 1);
        }
        for (int w = 0; w < NSLOT; ++w) {
            mbar_init(&S.xsfull[w], 1);
            mbar_init(&S.xsempty[w], 4 * NWG);          // every decay warp reads its 16 columns
        }
        for (int i = 0; i < 3; ++i)
            for (int w = 0; w < NWG; ++w) mbar_init(&S.cfull[i][w], 4);
        for (int w = 0; w < NWG; ++w) mbar_init(&S.lfull[w], 1);
        S.abort = 0;
        // work tickets in launch order, query tile major (see the head_dim-64 kernel)
        S.ticket = (int)atomicAdd(p.flags + (size_t)p.nunits * p.nqt * p.nkt, 1u);
        fence_barrier_init();
    }
    if (warp == 16) {
        // one-hot operand: zero, then bf16 1.0 in both 16-byte K chunks of row 0 (at +64 and
        // +64+2048); shifting the descriptor start down by 16 h bytes moves the ones to row h
        uint32_t* o32 = reinterpret_cast<uint32_t*>(S.onehot);
        for (int i = lane; i < (4096 + 64) / 4; i += 32) o32[i] = 0u;
        __syncwarp();
        if (lane < 4) {
            o32[(64 >> 2) + lane] = 0x3F803F80u;
            o32[((64 + 2048) >> 2) + lane] = 0x3F803F80u;
        }
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
    const int qt = S.ticket / p.nunits, unit = S.ticket % p.nunits;
    const int kvh = unit % p.Hkv, b = unit / p.Hkv;
    const int ktd = qt >> 1;                            // key tile holding this CTA's rows
    const int ntile = ktd + 1;
    const int i0 = qt * QR;                             // first query row of the CTA

    if (warp == 16) {
        // ------------------------------------------------ TMA producer
        const bool leader = elect_one();
        if (leader) {
            const CUtensorMap* maps[8] = {&tm_khk, &tm_khq, &tm_kr, &tm_q, &tm_v, &tm_lq, &tm_lk, &tm_mq};
            for (int m = 0; m < 8; ++m) prefetch_tmap(maps[m]);
            mbar_expect_tx(&S.qfull, 16384 * (1 + G) + 256 * (1 + G));
            tma_load_3d(S.kq, &tm_khq, &S.qfull, 0, i0, unit);
            tma_load_3d(S.kq + 8192, &tm_khq, &S.qfull, 64, i0, unit);
            for (int h = 0; h < G; ++h) {
                const int row = b * p.H + kvh * G + h;
                tma_load_3d(S.q[h], &tm_q, &S.qfull, 0, i0, row);
                tma_load_3d(S.q[h] + 8192, &tm_q, &S.qfull, 64, i0, row);
                tma_load_2d(S.mq[h], &tm_mq, &S.qfull, i0, row);
            }
            tma_load_2d(S.lq, &tm_lq, &S.qfull, i0, unit);
        }
        __syncwarp();
        uint32_t nk = 0;
        for (int kt = 0; kt < ntile; ++kt) {
            if (EARLY) {
                if (!mbar_wait(&S.pbfull[kt & 1], (kt >> 1) & 1, abort)) break;
                const int code = S.pbskip[kt & 1];
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.pbempty[kt & 1]);
                if (code == 2) continue;
            }
            if (nk >= 1 && !mbar_wait(&S.khempty, (nk - 1) & 1, abort)) break;
            if (leader) {
                mbar_expect_tx(&S.khfull, 32768 + 512);
                tma_load_3d(S.kh, &tm_khk, &S.khfull, 0, kt * 128, unit);
                tma_load_3d(S.kh + 16384, &tm_khk, &S.khfull, 64, kt * 128, unit);
                tma_load_2d(S.lk, &tm_lk, &S.khfull, kt * 128, unit);
            }
            __syncwarp();
            if (nk >= 1 && !mbar_wait(&S.krempty, (nk - 1) & 1, abort)) break;
            if (leader) {
                mbar_expect_tx(&S.krfull, 32768);
                tma_load_3d(S.kr, &tm_kr, &S.krfull, 0, kt * 128, unit);
                tma_load_3d(S.kr + 16384, &tm_kr, &S.krfull, 64, kt * 128, unit);
            }
            __syncwarp();
            // V last: it is needed only after this tile's decay and first softmax
            if (nk >= 1 && !mbar_wait(&S.vempty, (nk - 1) & 1, abort)) break;
            if (leader) {
                mbar_expect_tx(&S.vfull, 32768);
                tma_load_4d(S.v, &tm_v, &S.vfull, 0, kvh, kt * 128, b);
                tma_load_4d(S.v + 16384, &tm_v, &S.vfull, 64, kvh, kt * 128, b);
            }
            __syncwarp();
            ++nk;
        }
    } else if (warp == 18) {
        // ------------------------------------------------ boundary look-back and publisher
        auto fetch = [&](int kt) -> bool {
            const int sb = kt & 1;
            if (kt >= 2 && !mbar_wait(&S.pbempty[sb], ((kt >> 1) - 1) & 1, abort)) return false;
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f), c4 = v4;
            int skip = 0;
            if (qt >= 1 && kt <= ((qt - 1) >> 1)) {      // the previous query tile covered kt
                const size_t row = (size_t)unit * p.nqt + (qt - 1);
                if (!wait_counter128(p.flags + row * p.nkt + kt, 1u, abort, lane)) return false;
                v4 = __ldcg(reinterpret_cast<const float4*>(p.pincl + row * p.Tpk + (size_t)kt * 128) + lane);
                // Chunked pruning decides at the start of the 128-row chunk: for the chunk's first
                // 64-row tile that is Pb itself; the second reads what the tile two back published
                // (complete: the tile before waited on it for this key tile before publishing).
                // The chunk's own key tile (kt = qt / 2) is never pruned.
                c4 = v4;
                if ((qt & 1) && kt < (qt >> 1))
                    c4 = qt >= 3 ? __ldcg(reinterpret_cast<const float4*>(
                                       p.pincl + (row - 1) * p.Tpk + (size_t)kt * 128) + lane)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                float mn = fminf(fminf(v4.x, v4.y), fminf(v4.z, v4.w));
                float mc = fminf(fminf(c4.x, c4.y), fminf(c4.z, c4.w));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                    mc = fminf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
                }
                const bool pruned = kt < (qt >> 1) && mc > p.prune_thr;   // every key of the tile evicted
                skip = (mn * kLog2e128 >= kSkipLog2_128 || pruned) ? (EARLY ? 2 : 1) : 0;
            }
            *reinterpret_cast<float4*>(&S.pb[sb][lane * 4]) = v4;
            *reinterpret_cast<float4*>(&S.pbc[sb][lane * 4]) = c4;
            if (lane == 0) {
                S.pbskip[sb] = skip;
                if (skip) atomicAdd(p.flags + (size_t)p.nunits * p.nqt * p.nkt + 1, 1u);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.pbfull[sb]);
            return true;
        };
        uint32_t npub = 0;
        auto publish = [&](int kt) -> bool {
            float4 v4;
            if (S.pbskip[kt & 1] == 2) {
                v4 = *reinterpret_cast<const float4*>(&S.pb[kt & 1][lane * 4]);
            } else {
                const int sb = npub & 1;
                if (!mbar_wait(&S.pubfull[sb], (npub >> 1) & 1, abort)) return false;
                v4 = *reinterpret_cast<const float4*>(&S.pinc[sb][lane * 4]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.pubempty[sb]);
                ++npub;
            }
            const size_t row = (size_t)unit * p.nqt + qt;
            __stcg(reinterpret_cast<float4*>(p.pincl + row * p.Tpk + (size_t)kt * 128) + lane, v4);
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(p.flags + row * p.nkt + kt, 1u);
            return true;
        };
        bool ok = true;
        for (int kt = 0; ok && kt < ntile && kt < 2; ++kt) ok = fetch(kt);
        for (int kt = 0; ok && kt < ntile; ++kt) {
            if (qt < p.nqt - 1) ok = publish(kt);
            if (ok && kt + 2 < ntile) ok = fetch(kt + 2);
        }
    } else if (warp == 17 || warp == 19) {
        // ------------------------------------------------ MMA issuers
        const bool leader = elect_one();
        bool ok = true;
        if (warp == 17) {
            ok = mbar_wait(&S.qfull, 0, abort);
            const uint32_t akq = smem_u32(S.kq), akh = smem_u32(S.kh), akr = smem_u32(S.kr);
            uint32_t nh = 0;
            // one logit tile: D[128 keys][64 rows] = A (key tile) x B (query rows)^T, K = 128
            auto issue = [&](uint32_t a_tile, uint32_t b_tile) -> bool {
                const uint32_t slot = nh % NSLOT;
                if (nh >= NSLOT && !mbar_wait(&S.xsempty[slot], ((nh / NSLOT) - 1) & 1, abort)) return false;
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16(tmem + COL_XS + slot * 64, kdesc128(a_tile, 128, kk), kdesc128(b_tile, 64, kk),
                                 ID_XS, kk > 0);
                    umma_commit(&S.xsfull[slot]);
                }
                __syncwarp();
                ++nh;
                return true;
            };
            uint32_t nk = 0;
            for (int kt = 0; ok && kt < ntile; ++kt) {
                int code = 0;
                auto take_code = [&]() -> bool {
                    if (!mbar_wait(&S.pbfull[kt & 1], (kt >> 1) & 1, abort)) return false;
                    code = S.pbskip[kt & 1];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.pbempty[kt & 1]);
                    return true;
                };
                if (EARLY && !take_code()) break;
                if (code == 2) continue;
                if (!mbar_wait(&S.khfull, nk & 1, abort)) break;
                tc_fence_after();
                if (!issue(akh, akq)) break;
                if (leader) umma_commit(&S.khempty);
                __syncwarp();
                if (!EARLY && !take_code()) break;
                const bool skip = code != 0;
                if (!mbar_wait(&S.krfull, nk & 1, abort)) break;
                tc_fence_after();
#pragma unroll 1
                for (int h = 0; h < G && ok && !skip; ++h) ok = issue(akr, smem_u32(S.q[h]));
                if (!ok) break;
                if (leader) umma_commit(&S.krempty);
                __syncwarp();
                ++nk;
            }
        } else {
            // A = V^T (MN-major: two 64-dim atoms 16 KB apart, 8-key groups 1024 B apart),
            // B = P_h^T (MN-major, one 64-row atom); k-step kk (16 keys) adds 2048 B to both
            const uint64_t dva = smem_desc(smem_u32(S.v), 16384, 1024, kSwizzle128B);
            const uint64_t dpa = smem_desc(smem_u32(S.p[0]), 16384, 1024, kSwizzle128B);
            const uint64_t dpb = smem_desc(smem_u32(S.p[1]), 16384, 1024, kSwizzle128B);
            const uint32_t oh = smem_u32(S.onehot) + 64;
            uint32_t p_use = 0, nk = 0;
            bool first = true;
            for (int kt = 0; ok && kt < ntile; ++kt) {
                if (!mbar_wait(&S.pbfull[kt & 1], (kt >> 1) & 1, abort)) break;
                const int code = S.pbskip[kt & 1];
                const bool skip = code != 0;
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.pbempty[kt & 1]);
                if (code == 2) continue;
                if (!mbar_wait(&S.vfull, nk & 1, abort)) break;
#pragma unroll 1
                for (int h = 0; h < G && ok && !skip; ++h) {
                    const uint32_t pbuf = p_use & 1;
                    if (!mbar_wait(&S.pfull[pbuf], (p_use >> 1) & 1, abort)) { ok = false; break; }
                    tc_fence_after();
                    if (leader) {
                        const uint64_t dp = pbuf ? dpb : dpa;
                        // one-hot operand of head h: K-major, no swizzle, core matrices of
                        // 8 rows x 16 B, 128 B apart along M (SBO) and 2048 B apart along K (LBO)
                        const uint64_t dl = smem_desc(oh - 16u * (uint32_t)h, 2048, 128, kSwizzleNone);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t acc_o = (!first || kk > 0) ? 1u : 0u;
                            const uint32_t acc_l = (!first || h > 0 || kk > 0) ? 1u : 0u;
                            umma_f16(tmem + COL_O + h * 64, dva + (uint64_t)(kk * 128), dp + (uint64_t)(kk * 128),
                                     ID_PV, acc_o);
                            umma_f16(tmem + COL_L, dl, dp + (uint64_t)(kk * 128), ID_L, acc_l);
                        }
                        umma_commit(&S.pempty[pbuf]);
                    }
                    __syncwarp();
                    ++p_use;
                }
                if (!ok) break;
                if (!skip) first = false;
                if (leader) {
                    umma_commit(&S.vempty);
                    if (kt == ntile - 1) umma_commit(&S.ofull);
                }
                __syncwarp();
                ++nk;
            }
        }
    } else {
        // ------------------------------------------------ decay / softmax warpgroups
        const int wg = warp >> 2;                        // quarter: rows 16*wg .. 16*wg+15
        const int wq = warp & 3;
        const int jl = wq * 32 + lane;                   // key within the tile = TMEM lane
        const uint32_t tlane = (uint32_t)(wq * 32) << 16;
        const uint32_t xcol0 = tmem + tlane + COL_XS + wg * 16;   // + slot * 64
        const float al = p.alpha[kvh], be = p.beta[kvh];
        const float sl = p.scale_log2e;
        const int r0 = wg * 16;                          // first row of this quarter within the tile
        uint32_t use = 0, p_use = 0, nd = 0, npub = 0, nk = 0;
        bool ok = mbar_wait(&S.qfull, 0, abort);
        if (ok) {
            float m = (lane < 16) ? S.mq[0][r0 + lane] : -INFINITY;
            for (int h = 1; h < G; ++h) m = fmaxf(m, (lane < 16) ? S.mq[h][r0 + lane] : -INFINITY);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) S.shift[warp] = m;
            __syncwarp();
        }
        const float al2 = al * kLog2e128, be2 = be * kLog2e128;
        // this thread's key row of a P^T tile: 8-key group jl/8, row jl%8; chunks r0/8 + c
        const uint32_t prow_off = (jl >> 3) * 1024 + (jl & 7) * 128;
        const int ck0 = r0 >> 3, sw = jl & 7;
        auto slot_read = [&](uint32_t (&x)[16]) -> bool {
            const uint32_t slot = use % NSLOT;
            if (!mbar_wait(&S.xsfull[slot], (use / NSLOT) & 1, abort)) return false;
            tc_fence_after();
            tmem_ld16_async(xcol0 + slot * 64, x);
            tmem_wait16(x);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.xsempty[slot]);
            ++use;
            return true;
        };
        for (int kt = 0; ok && kt < ntile; ++kt) {
            const int j = kt * 128 + jl;
            const bool diag = (kt == ktd);
            const bool tailq = i0 + QR > T;
            int code = 0;
            float pbj = 0.f, pbcj = 0.f;
            auto take_pb = [&]() -> bool {
                if (!mbar_wait(&S.pbfull[kt & 1], (kt >> 1) & 1, abort)) return false;
                pbj = S.pb[kt & 1][jl];
                pbcj = S.pbc[kt & 1][jl];
                code = S.pbskip[kt & 1];
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.pbempty[kt & 1]);
                return true;
            };
            if (EARLY && !take_pb()) { ok = false; break; }
            if (code == 2) continue;
            if (!mbar_wait(&S.khfull, nk & 1, abort)) { ok = false; break; }
            const float rk3 = ex2f(S.lk[jl]) * kCbrtLn2_128;
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.khempty);
            ++nk;
            // ---- decay over this quarter's 16 rows, scanned down the key column
            float lam[16];
            float above = 0.f;
            {
                uint32_t x[16];
                if (!slot_read(x)) { ok = false; break; }
                float c = 0.f;
                const bool masked = diag || tailq;
                const int rlo = diag ? j - (i0 + r0) + 1 : 0;
                const int rhi = tailq ? T - (i0 + r0) : 16;
                if (masked) decay16r<true>(x, S.lq + r0, rlo, rhi, al2, be2, c, lam);
                else decay16r<false>(x, S.lq + r0, rlo, rhi, al2, be2, c, lam);
                // carry across quarters (ring of three buffers, as in the head_dim-64 kernel)
                const int tb = nd % 3;
                const uint32_t tph = (nd / 3) & 1;
                S.tot[tb][wg][jl] = c;
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.cfull[tb][wg]);
                for (int w = 0; w < wg && ok; ++w) {
                    if (!mbar_wait(&S.cfull[tb][w], tph, abort)) { ok = false; break; }
                    above += S.tot[tb][w][jl];
                }
                if (!ok) break;
                ++nd;
            }
            if (!EARLY && !take_pb()) { ok = false; break; }
            const bool skip = code != 0;
            if (wg == NWG - 1) {
                const float pinc = fmaf(rk3, above + lam[15], pbj);
                if (qt == p.nqt - 1) {
                    if (p.b_final && j < T) p.b_final[(size_t)unit * T + j] = -pinc;
                } else {
                    const int sb = npub & 1;
                    if (npub >= 2 && !mbar_wait(&S.pubempty[sb], ((npub >> 1) - 1) & 1, abort)) { ok = false; break; }
                    S.pinc[sb][jl] = pinc;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&S.pubfull[sb]);
                    ++npub;
                }
            }
            if (skip) continue;
            const float ka = -rk3 * kLog2e128, kb = -fmaf(rk3, above, pbj) * kLog2e128 - S.shift[warp];
#pragma unroll
            for (int r = 0; r < 16; ++r) lam[r] = fmaf(lam[r], ka, kb);
            if (!diag && pbcj > p.prune_thr) {           // key evicted at this chunk's start
#pragma unroll
                for (int r = 0; r < 16; ++r) lam[r] = -INFINITY;
            }
            // ---- per head: P = 2^(S*scale*log2e + Lambda - shift), causally masked
#pragma unroll 1
            for (int h = 0; h < G && ok; ++h) {
                uint32_t x[16];
                if (!slot_read(x)) { ok = false; break; }
                const uint32_t pbuf = p_use & 1;
                if (p_use >= 2 && !mbar_wait(&S.pempty[pbuf], ((p_use >> 1) - 1) & 1, abort)) { ok = false; break; }
                uint8_t* prow = S.p[pbuf] + prow_off;
                if (diag) probs16r<true>(x, sl, lam, j - (i0 + r0), prow, ck0, sw);
                else probs16r<false>(x, sl, lam, 0, prow, ck0, sw);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.pfull[pbuf]);
                ++p_use;
            }
        }
        // ---- epilogue: thread = head dim (TMEM lane) d = jl; warpgroup wg finishes rows 16wg .. 16wg+15
        if (ok && mbar_wait(&S.ofull, 0, abort)) {
            tc_fence_after();
            if (wq == 0) {
                float l16[16];
                tmem_ld16(tmem + COL_L + wg * 16, l16);   // lane h holds head h's sums
                if (lane < G) {
#pragma unroll
                    for (int r = 0; r < 16; ++r) S.lsum[lane][r0 + r] = l16[r];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&S.lfull[wg]);
            }
            // the row sums of this quarter, staged by its first warp (a bounded wait, so a warp
            // that gave up elsewhere can never leave the others blocked here)
            const bool lok = mbar_wait(&S.lfull[wg], 0, abort);
            const float sh = S.shift[4 * wg];
#pragma unroll 1
            for (int h = 0; h < G && lok; ++h) {
                const int hq = kvh * G + h;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float o[8];
                    tmem_ld8(tmem + tlane + COL_O + h * 64 + wg * 16 + half * 8, o);
#pragma unroll
                    for (int r8 = 0; r8 < 8; ++r8) {
                        const int r = half * 8 + r8;
                        const int i = i0 + r0 + r;
                        if (i < T) {
                            const float l = S.lsum[h][r0 + r];
                            const size_t off = (((size_t)b * T + i) * p.H + hq) * 128 + jl;
                            const float gv = __bfloat162float(static_cast<const __nv_bfloat16*>(p.g)[off]);
                            static_cast<__nv_bfloat16*>(p.o)[off] = __float2bfloat16_rn(o[r8] / l * sigmoid_f(gv));
                        }
                    }
                }
                if (wq == 0 && lane < 16) {
                    const int i = i0 + r0 + lane;
                    if (i < T) {
                        const float l = S.lsum[h][r0 + lane];
                        if (!(l >= 0x1p-60f) || !isfinite(l))  // out of the shift's range: recomputed exactly
                            p.fix_list[atomicAdd(p.fix_count, 1u)] = (int)(((size_t)b * p.H + hq) * T + i);
                        if (p.lse) p.lse[((size_t)b * p.H + hq) * T + i] = (sh + lg2f(l)) * 0.6931471805599453f;
                    }
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

static size_t fwd_tc128_smem(int G) {
    switch (G) {
        case 1: return sizeof(fwd128::Smem<1>) + 1024;
        case 2: return sizeof(fwd128::Smem<2>) + 1024;
        case 3: return sizeof(fwd128::Smem<3>) + 1024;
        default: return sizeof(fwd128::Smem<4>) + 1024;
    }
}

template <int G, bool EARLY>
static cudaError_t fwd_tc128_launch(const CUtensorMap* m, const FwdTc128Params& p, cudaStream_t s) {
    const size_t smem = fwd_tc128_smem(G);
    cudaError_t e = cudaFuncSetAttribute(k_fwd_tc128<G, EARLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    UA_PROFILE("k_fwd_tc128", s);
    k_fwd_tc128<G, EARLY><<<p.nqt * p.nunits, 640, smem, s>>>(m[0], m[1], m[2], m[3], m[4], m[5], m[6], m[7], p);
    return cudaGetLastError();
}

template <int G>
static cudaError_t fwd_tc128_inst(const CUtensorMap* m, const FwdTc128Params& p, cudaStream_t s) {
    return p.b_final ? fwd_tc128_launch<G, false>(m, p, s) : fwd_tc128_launch<G, true>(m, p, s);
}

cudaError_t launch_fwd_tc128(const FwdTcLaunch& L, cudaStream_t s) {
    CUtensorMap m[8];
    const int BH = L.B * L.H, BK = L.B * L.Hkv;
    if (!map_rows128(&m[0], L.kh, L.T, BK, 128)) return cudaErrorInvalidValue;
    if (!map_rows128(&m[1], L.kh, L.T, BK, 64)) return cudaErrorInvalidValue;
    if (!map_rows128(&m[2], L.kr, L.T, BK, 128)) return cudaErrorInvalidValue;
    if (!map_rows128(&m[3], L.qr, L.T, BH, 64)) return cudaErrorInvalidValue;
    if (!map_v128(&m[4], L.v, L.Hkv, L.T, L.B)) return cudaErrorInvalidValue;
    if (!map_vec128(&m[5], L.lq2, L.T, L.Tp, BK, 64)) return cudaErrorInvalidValue;
    if (!map_vec128(&m[6], L.lk2, L.T, L.Tp, BK, 128)) return cudaErrorInvalidValue;
    if (!map_vec128(&m[7], L.mq, L.T, L.Tp, BH, 64)) return cudaErrorInvalidValue;
    FwdTc128Params p;
    p.B = L.B; p.T = L.T; p.Tp = L.Tp; p.Tpk = L.Tpk; p.H = L.H; p.Hkv = L.Hkv; p.nqt = L.nqt;
    p.nkt = (L.T + 127) / 128;
    p.scale_log2e = L.scale * kLog2e128;
    p.alpha = L.alpha; p.beta = L.beta; p.g = L.g; p.o = L.o; p.lse = L.lse;
    p.pincl = L.pincl; p.flags = L.flags; p.b_final = L.b_final; p.nunits = BK; p.prune_thr = L.prune_thr;
    p.fix_count = L.fix_count; p.fix_list = L.fix_list;
    switch (L.H / L.Hkv) {
        case 1: return fwd_tc128_inst<1>(m, p, s);
        case 2: return fwd_tc128_inst<2>(m, p, s);
        case 3: return fwd_tc128_inst<3>(m, p, s);
        case 4: return fwd_tc128_inst<4>(m, p, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ua
