// ua_common.cuh -- small device helpers shared by the libua kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ua.h"

namespace ua {

// Device status word: the first ua_status code a kernel raises sticks until
// ua_get_device_status reads and clears it.  Defined in ua_api.cu.
extern __device__ int g_status;

__device__ __forceinline__ void raise_status(int code) { atomicCAS(&g_status, 0, code); }

// Limit of every bounded device-side wait, in ns of %globaltimer (ua_set_wait_limit_ns; default
// UA_WAIT_LIMIT_DEFAULT_NS).  Defined in ua_api.cu.
extern __device__ unsigned long long g_wait_limit_ns;

// ------------------------------------------------------------------ dependent launches
// Kernels of the decode step are launched with programmatic stream serialisation (one decode
// step after another, in a CUDA graph or not): the next kernel's blocks may be scheduled while
// this one finishes.  grid_dep_wait() blocks until every kernel the grid depends on has
// completed and its writes are visible -- each kernel calls it before its first access to
// global memory; it returns at once for a grid launched without the attribute.
// grid_dep_release() lets the next grid be scheduled (its blocks still wait for this grid's
// completion before touching memory).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ scalar math
// softplus(x) = log(1 + e^x) in its overflow-free form.
__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

// Geometric mean of the three decay rates (veto: a zero factor gives exactly zero).
__device__ __forceinline__ float decay_geo(float rq, float rk, float rsim) {
    return cbrtf(rq * rk * rsim);
}

// Variant bits of ua_shape.variant (the ablations; 0 = the method itself).
constexpr int kVarNoQ = 1, kVarNoK = 2, kVarNoSim = 4, kVarQNorm = 8, kVarPerHead = 16;
constexpr int kVarMech = kVarNoQ | kVarNoK | kVarNoSim;
constexpr float kQNormEps = 1e-6f;

// Decay rate of a variant: the geometric mean of the rates whose mechanisms are on.
// rq and rk arrive as 1 when their mechanism is off; x is the similarity logit
// alpha * <khat_l, khat_j> + beta, whose softplus enters only when that mechanism is on.
__device__ __forceinline__ float decay_var(float rq, float rk, float x, int variant) {
    const int off = variant & kVarMech;
    if (off == 0) return decay_geo(rq, rk, softplus_f(x));
    const float prod = rq * rk * ((off & kVarNoSim) ? 1.f : softplus_f(x));
    return __popc(off) == 1 ? sqrtf(prod) : prod;     // two rates on, or one
}

// 1 / number of mechanisms on: the exponent of the geometric mean, d log D / d log r.
__host__ __device__ __forceinline__ float var_inv_n(int variant) {
    const int n = 3 - (((variant & kVarNoQ) != 0) + ((variant & kVarNoK) != 0) + ((variant & kVarNoSim) != 0));
    return n == 3 ? 1.f / 3.f : (n == 2 ? 0.5f : 1.f);
}

// RoPE frequencies theta^(-2m/d), computed on the host in double precision (m < d/2 <= 64).
struct RopeFreq {
    double f[64];
};

// cos / sin of the RoPE angle pos * f.  The angle is formed in double precision and reduced
// to [-pi, pi] with a two-constant Cody-Waite split of 2*pi (exact to ~1e-16 relative for the
// positions used here), then the fp32 sincosf of the reduced angle is taken.
__device__ __forceinline__ void rope_cs(double pos, double f, float* c, float* s) {
    const double a = pos * f;
    const double k = rint(a * 0.15915494309189535);            // 1 / (2 pi)
    double r = fma(-k, 6.283185307179586, a);                   // 2 pi, high part
    r = fma(-k, 2.4492935982947064e-16, r);                     // 2 pi, low part
    sincosf((float)r, s, c);
}

// cos / sin of the RoPE angle pos * f for a cached key, given gt = f / (2 pi) in double.  The
// reduction works in turns: pos * gt is formed in double precision and its nearest integer
// removed exactly, so the fraction (|r| <= 1/2) keeps ~1e-16 relative accuracy whatever the
// position; the fp32 angle 2 pi r in [-pi, pi] then goes to the fast sine / cosine unit, whose
// absolute error there is ~1e-6 (far below the 2^-8 relative rounding of a bf16 key).
__device__ __forceinline__ void rope_cs_turns(double pos, double gt, float* c, float* s) {
    const double a = pos * gt;
    const float th = (float)(a - rint(a)) * 6.28318530717958648f;
    __sincosf(th, s, c);
}

// Cached keys are stored pair-interleaved: element 2m holds component m and element 2m + 1
// component m + d/2, the two components one RoPE frequency rotates together, so a lane that
// loads 16 bytes of a key holds whole rotation pairs.
__host__ __device__ __forceinline__ int il_index(int x, int half) {
    return x < half ? 2 * x : 2 * (x - half) + 1;
}

// ------------------------------------------------------------------ element access
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float ld(const float* p) { return *p; }
    static __device__ __forceinline__ void st(float* p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};

// 16-byte vector of activations <-> float registers.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void ld(const float* p, float* x) {
        float4 u = *reinterpret_cast<const float4*>(p);
        x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
    }
    static __device__ __forceinline__ void st(float* p, const float* x) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
    static __device__ __forceinline__ uint4 raw(const float* p) { return *reinterpret_cast<const uint4*>(p); }
    static __device__ __forceinline__ void unpack(uint4 u, float* x) {
        x[0] = __uint_as_float(u.x); x[1] = __uint_as_float(u.y);
        x[2] = __uint_as_float(u.z); x[3] = __uint_as_float(u.w);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void unpack(uint4 u, float* x) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void ld(const __nv_bfloat16* p, float* x) {
        unpack(*reinterpret_cast<const uint4*>(p), x);
    }
    static __device__ __forceinline__ uint4 raw(const __nv_bfloat16* p) { return *reinterpret_cast<const uint4*>(p); }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, const float* x) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

}  // namespace ua
