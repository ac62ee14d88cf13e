// lbq_ldg.cuh -- pieces shared by the register-streaming GEMV kernels (sm_100a): weight
// streaming, the 16-bit fixed-point activation planes, programmatic dependent launches.
#pragma once
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

constexpr int kLdgChunk = 256;                 // k per unit (one superblock)
constexpr int kLdgPlaneMax = 32639;            // |v| bound so that (v + 128) >> 8 fits in int8

// Smallest E with maxabs * 2^-E <= kLdgPlaneMax (E = 0 for an all-zero chunk), from the
// exponent and significand fields (maxabs = m * 2^e, m in [1, 2)).
__device__ __forceinline__ int ldg_fixed_point_exponent(float maxabs) {
    if (!(maxabs > 0.0f)) return 0;
    uint32_t u = __float_as_uint(maxabs);
    int bias = 0;
    if ((u >> 23) == 0) {                       // subnormal: scale up exactly by 2^64 first
        u = __float_as_uint(maxabs * 18446744073709551616.0f);
        bias = 64;
    }
    const int e = (int)(u >> 23) - 127 - bias;
    const float m = __uint_as_float((u & 0x007FFFFFu) | 0x3F800000u);
    return e - 14 + (m * 16384.0f > (float)kLdgPlaneMax ? 1 : 0);
}

// 2^p as a float (exact for every p a normal float holds).
__device__ __forceinline__ float ldg_exp2i(int p) {
    if (p >= -126 && p <= 127) return __uint_as_float((uint32_t)(p + 127) << 23);
    return ldexpf(1.0f, p);
}

// 16 bytes of streamed weights: read once, so no L1 allocation and evict-first in L2.
__device__ __forceinline__ uint4 ldg_stream(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// Byte offset, inside a 256-wide chunk of a plane row, of the 8 bytes prepared by lane l
// (elements 8l..8l+7): k-step l / 4, lane-group l mod 4; two consecutive k-steps of a
// lane-group sit side by side so that one 16-byte load fetches both B fragments.
__host__ __device__ __forceinline__ int plane_off(int l) { return 64 * (l >> 3) + 16 * (l & 3) + 8 * ((l >> 2) & 1); }

struct PrepOut {
    uint2 hi, lo;   // this lane's 8 bytes of the hi and lo planes
    int gsum;       // exact sum of q over the lane's group of LPG lanes (on every lane of it)
    int E;
};

// max |v| over the warp's 32 x 8 values.
__device__ __forceinline__ float warp_max_abs8(const float (&v)[8]) {
    float mx = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; e++) mx = fmaxf(mx, fabsf(v[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    return mx;
}

// The lane's 8 values as q = rint(v * 2^-E) split into hi/lo plane bytes (v = 256 hi + lo;
// even elements in .x, odd in .y), and sum(q) over groups of LPG consecutive lanes.
template <int LPG>
__device__ __forceinline__ PrepOut prep_quantize8(const float (&v)[8], int E) {
    PrepOut r;
    r.E = E;
    // v * 2^-E in at most two exact power-of-two multiplications
    const int e1 = max(-126, min(127, -E));
    const float f1 = ldg_exp2i(e1), f2 = ldg_exp2i(-E - e1);
    uint32_t hev = 0, hod = 0, lev = 0, lod = 0;
    int sum = 0;
#pragma unroll
    for (int e = 0; e < 8; e++) {
        const int q = __float2int_rn((v[e] * f1) * f2);
        const int h = (q + 128) >> 8;
        const int l = q - 256 * h;
        sum += q;
        const int sh = 8 * (e >> 1);
        if (e & 1) {
            hod |= (uint32_t)(h & 0xFF) << sh;
            lod |= (uint32_t)(l & 0xFF) << sh;
        } else {
            hev |= (uint32_t)(h & 0xFF) << sh;
            lev |= (uint32_t)(l & 0xFF) << sh;
        }
    }
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    r.hi = make_uint2(hev, hod);
    r.lo = make_uint2(lev, lod);
    r.gsum = sum;
    return r;
}

// ------------------------------------------------------------------ host side

// Programmatic-dependent launch; cluster > 1 groups the CTAs into thread-block clusters of
// that many (grid a multiple of it).
template <class Kern, class... Args>
inline lbq_status launch_pdl_cluster(Kern kern, int grid, int cluster, int threads, size_t smem, cudaStream_t st,
                                     const Args&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int na = 1;
    if (cluster > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        na = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) return LBQ_ERR_CUDA;
    return launch_status();
}
template <class Kern, class... Args>
inline lbq_status launch_pdl(Kern kern, int grid, int threads, size_t smem, cudaStream_t st, const Args&... args) {
    return launch_pdl_cluster(kern, grid, 1, threads, smem, st, args...);
}

template <auto KERN>
inline lbq_status ldg_smem_attr(int bytes) {
    static bool set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LBQ_ERR_CUDA;
    if (dev >= 0 && dev < 64 && set[dev]) return LBQ_OK;
    if (cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return LBQ_ERR_CUDA;
    if (dev >= 0 && dev < 64) set[dev] = true;
    return LBQ_OK;
}

}  // namespace lbq
