// k_per_head.cu -- per-query-head decay (UA_VAR_PER_HEAD_DECAY) as a composition of the
// per-KV-head kernels.  With rates, similarity parameters and eviction per query head, query
// head h behaves exactly as multi-head Universal Attention over its group's shared keys and
// values (paperlayer.ai summary §4.2: retention decided head by head).  So the library repeats
// each KV head's keys and values for the G query heads of its group, runs the ordinary path with
// one decay unit per query head, and sums the key and value gradients back over the copies.
#include <algorithm>

#include "ua_common.cuh"
#include "ua_kernels.h"
#include "ua_profile.h"

namespace ua {

// out[b, t, h, :] = in[b, t, h / G, :]; one 16-byte vector per thread.
template <typename TA>
__global__ void __launch_bounds__(256) k_repeat_kv(const TA* in, TA* out, size_t rows_out, int H, int G, int d) {
    constexpr int V = 16 / sizeof(TA);
    const int vpr = d / V;                            // vectors per head row
    const size_t total = rows_out * vpr;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        const size_t row = e / vpr;                   // (b*T + t) * H + h
        const int c = (int)(e % vpr);
        const int h = (int)(row % H);
        const size_t src = (row / H) * (H / G) + h / G;
        reinterpret_cast<uint4*>(out)[row * vpr + c] = reinterpret_cast<const uint4*>(in)[src * vpr + c];
    }
}

// out[b, t, kh, :] = sum over the G copies in[b, t, kh*G + g, :] (fp32 sum in copy order).
template <typename TA>
__global__ void __launch_bounds__(256) k_sum_copies(const TA* in, TA* out, size_t rows_out, int G, int d) {
    const size_t total = rows_out * d;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        const size_t row = e / d;
        const int x = (int)(e % d);
        float s = 0.f;
        for (int g = 0; g < G; ++g) s += Elem<TA>::ld(in + (row * G + g) * d + x);
        Elem<TA>::st(out + e, s);
    }
}

cudaError_t launch_repeat_kv(const void* in, void* out, int B, int T, int H, int G, int d, bool bf16, cudaStream_t s) {
    const size_t rows = (size_t)B * T * H;
    const int grid = (int)std::min<size_t>((rows * d / 8 + 255) / 256, 148 * 16);
    UA_PROFILE("k_repeat_kv", s);
    if (bf16)
        k_repeat_kv<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(in),
                                                        static_cast<__nv_bfloat16*>(out), rows, H, G, d);
    else
        k_repeat_kv<float><<<grid, 256, 0, s>>>(static_cast<const float*>(in), static_cast<float*>(out), rows, H, G, d);
    return cudaGetLastError();
}

cudaError_t launch_sum_copies(const void* in, void* out, int B, int T, int Hkv, int G, int d, bool bf16, cudaStream_t s) {
    const size_t rows = (size_t)B * T * Hkv;
    const int grid = (int)std::min<size_t>((rows * d + 255) / 256, 148 * 16);
    UA_PROFILE("k_sum_copies", s);
    if (bf16)
        k_sum_copies<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(in),
                                                         static_cast<__nv_bfloat16*>(out), rows, G, d);
    else
        k_sum_copies<float><<<grid, 256, 0, s>>>(static_cast<const float*>(in), static_cast<float*>(out), rows, G, d);
    return cudaGetLastError();
}

}  // namespace ua
