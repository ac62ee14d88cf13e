// lbq_gemv_group_tma.cu -- dequant-fused group GEMV on integer tensor cores (sm_100a), M = 1..16.
//
//   y[m, i] = sum_k x[m, k] * s[i, k/g] * (q[i, k] - z[i, k/g])
//
// Decode time per token is the bytes read over the read bandwidth ("AirLLM corre un
// modelo 70B en una GPU de 4GB...", section "Por qué es lento"): the kernel must keep
// HBM streaming while spending as few instructions per weight as possible.
//
//  * One launch serves up to kMaxProblems independent products of the same bit width
//    and group size (e.g. the q/k/v or gate/up projections of a decoder block); their
//    (128-row block, 256-wide k chunk) units form one list that the CTAs split evenly
//    ("stream-K"), so the SMs finish together.  A row block split between CTAs is
//    finished by the last CTA to arrive (tile_epilogue, deterministic).
//  * A producer warp streams every unit into a shared-memory ring with the Tensor
//    Memory Accelerator: the eight 16-row tiles' packed codes (1-D bulk copies,
//    evict-first in L2) on one transaction-count mbarrier; the activation rows (1-D bulk
//    copies) and 128 x 8 tiles of the fp16 scales and zeros (2-D tensor copies) on a
//    second one, so that the activation prep starts while the weights are in flight.
//  * Launched as a programmatic dependent of the previous kernel in the stream, the
//    producer issues the first stages' weight and scale copies before waiting for that
//    kernel (griddepcontrol.wait); only the activation copies, the prep and the stores
//    depend on it.  Packed weights, scales and zeros must therefore not be written by a
//    kernel that signals programmatic completion early.
//  * Two prep warps turn each activation chunk into 16-bit fixed point with one
//    power-of-two scale 2^E per token and chunk (|v| <= 32639), split into int8 planes
//    hi, lo (v = 256 hi + lo) laid out for the B fragment, plus per-group sums of v.
//  * Eight consumer warps (one 16-row tile each) mask the packed words into u8 A
//    fragments (one LOP per four codes) and run mma.m16n8k32 u8 x s8 -> s32 with the hi
//    and lo planes side by side in N.  Per group the exact integer sum
//    S = sum q v is corrected to sum (q - z) v = S - z sum(v) and scaled by s into an
//    fp32 chunk accumulator, which is scaled by 2^E once per chunk.
//  * Every wait is bounded; on expiry the kernel records kErrTimeout, stops issuing,
//    waits (bounded) for its own copies in flight and returns.
// Group codes: "TurboQuant: cuantizar modelos grandes para que quepan en local",
// section "Compresión por bloques"; RTN codes: "Métodos de cuantización de LLM para
// ejecutar un modelo de 70B en una sola GPU", section "RTN (Round-To-Nearest)".
#include <cuda.h>
#include <cstring>
#include "lbq_common.cuh"
#include "lbq_internal.h"
#include "lbq_group_frag.cuh"

namespace lbq {

constexpr int kConsumers = 8;
constexpr int kPrepWarps = 2;
constexpr int kProducerWarp = kConsumers;
constexpr int kGemvThreads = (kConsumers + 1 + kPrepWarps) * 32;
constexpr int kChunk = 256;                            // k per pipeline stage
constexpr int kPlanePitch = kChunk + 16;                // bytes per int8 plane row in smem (bank pad)
constexpr int kScaleBox = 8;                            // groups per scale-tile row (a chunk never spans more)
constexpr int kScaleTile = 128 * kScaleBox * 2;         // bytes of one 128 x 8 fp16 tile
constexpr int kBarBytes = 512;                          // mbarriers + abort flag
constexpr int kGemvSmemBudget = 110 * 1024;             // two CTAs per SM
constexpr int kPlaneMaxAbs = 32639;                     // |v| bound so that (v + 128) >> 8 fits in int8

struct GemvProblemDev {
    const uint16_t* x;
    const uint8_t* packed;
    uint16_t* y;
    int64_t n, k, n_tiles, kch, unit_begin, tile_begin;
};

struct alignas(64) GemvArgs {
    CUtensorMap ms[kMaxGemvProblems];
    CUtensorMap mz[kMaxGemvProblems];
    GemvProblemDev p[kMaxGemvProblems];
    float* partials;
    unsigned* counters;
    unsigned* err;
    int64_t total_units;
    int count, M, maxc, nstage;
};

struct StageLayout {
    int xraw, planes, xsum, expo, sc, zr, bytes;
    __host__ __device__ StageLayout(int B, int M) {
        xraw = 128 * kChunk * B / 8;
        planes = xraw + up(M * 2 * kChunk, 16);
        xsum = planes + up(2 * M * kPlanePitch, 16);
        expo = xsum + up(M * 8 * 4, 16);
        sc = up(expo + up(M * 4, 16), 128);
        zr = sc + kScaleTile;
        bytes = zr + kScaleTile;
    }
    __host__ __device__ static int up(int v, int a) { return (v + a - 1) / a * a; }
};

// Smallest E with maxabs * 2^-E <= kPlaneMaxAbs (E = 0 for an all-zero chunk),
// from the exponent and significand fields (maxabs = m * 2^e, m in [1, 2)).
__device__ __forceinline__ int fixed_point_exponent(float maxabs) {
    if (!(maxabs > 0.0f)) return 0;
    uint32_t u = __float_as_uint(maxabs);
    int bias = 0;
    if ((u >> 23) == 0) {                       // subnormal: scale up exactly by 2^64 first
        u = __float_as_uint(maxabs * 18446744073709551616.0f);
        bias = 64;
    }
    const int e = (int)(u >> 23) - 127 - bias;
    const float m = __uint_as_float((u & 0x007FFFFFu) | 0x3F800000u);
    return e - 14 + (m * 16384.0f > (float)kPlaneMaxAbs ? 1 : 0);
}

// 2^p as a float (exact); the bit pattern path covers every p a normal float can hold.
__device__ __forceinline__ float exp2i(int p) {
    if (p >= -126 && p <= 127) return __uint_as_float((uint32_t)(p + 127) << 23);
    return ldexpf(1.0f, p);
}

// Position of a unit of the launch's list: problem, row block, k chunk.
struct UnitCursor {
    int p = 0;
    __device__ __forceinline__ void seek(const GemvArgs& a, int64_t u) {
        while (p + 1 < a.count && u >= a.p[p + 1].unit_begin) p++;
    }
};

// Load NG consecutive fp16 values from shared memory (NG in 2, 4, 8; 4-byte aligned).
template <int NG>
__device__ __forceinline__ void lds_halves(const uint16_t* p, uint32_t (&d)[NG / 2]) {
    if constexpr (NG == 2) d[0] = *reinterpret_cast<const uint32_t*>(p);
    else if constexpr (NG == 4) { const uint2 v = *reinterpret_cast<const uint2*>(p); d[0] = v.x; d[1] = v.y; }
    else { const uint4 v = *reinterpret_cast<const uint4*>(p); d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w; }
}

template <int B, int GROUP, int NB, bool BF16>
__global__ void __launch_bounds__(kGemvThreads, 2) k_gemv_group_tc(const __grid_constant__ GemvArgs a) {
    using G = GroupGeom<B>;
    using F = IFrag<B>;
    constexpr int TILE_BYTES = G::SB_BYTES;            // one tile's codes per stage (512 * B)
    constexpr int KPG = GROUP / 32;                    // k-steps per group
    constexpr int NGC = kChunk / GROUP;                // groups per chunk

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBarBytes - 4);
    const int M = a.M, nstage = a.nstage;
    const StageLayout L(B, M);
    uint8_t* stage0 = smem + kBarBytes;
    unsigned* err = a.err;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t S_total = a.total_units;
    const int64_t NC = gridDim.x;
    const int64_t u_begin = (int64_t)blockIdx.x * S_total / NC;
    const int64_t u_end = ((int64_t)blockIdx.x + 1) * S_total / NC;

    // barriers: wfull[s] (weights), afull[s] (activations + scales), empty[s], xready[s]
    auto wfull = [&](int s) { return smem_u32(&bars[s]); };
    auto afull = [&](int s) { return smem_u32(&bars[nstage + s]); };
    auto empty = [&](int s) { return smem_u32(&bars[2 * nstage + s]); };
    auto xready = [&](int s) { return smem_u32(&bars[3 * nstage + s]); };
    if (threadIdx.x == 0) {
        for (int s = 0; s < nstage; s++) {
            mbar_init(wfull(s), 1);
            mbar_init(afull(s), 1);
            mbar_init(empty(s), kConsumers);
            mbar_init(xready(s), kPrepWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    griddep_launch_dependents();

    // ------------------------------------------------------------ producer warp
    if (warp == kProducerWarp) {
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            UnitCursor cur;
            auto issue = [&](int64_t u, int s, bool static_part, bool with_x) {
                cur.seek(a, u);
                const GemvProblemDev& P = a.p[cur.p];
                const int64_t lu = u - P.unit_begin;
                const int64_t rb = lu / P.kch, kc = lu % P.kch;
                uint8_t* st = stage0 + (size_t)s * L.bytes;
                if (static_part) {
                    const int64_t tiles_left = P.n_tiles - rb * kConsumers;
                    const int tiles = (int)(tiles_left < kConsumers ? tiles_left : kConsumers);
                    mbar_arrive_expect_tx(wfull(s), (uint32_t)(tiles * TILE_BYTES));
                    for (int t = 0; t < tiles; t++)
                        tma_load_1d_hint(smem_u32(st + t * TILE_BYTES),
                                         P.packed + ((rb * kConsumers + t) * P.kch + kc) * (int64_t)TILE_BYTES,
                                         TILE_BYTES, wfull(s), pol);
                    mbar_arrive_expect_tx(afull(s), (uint32_t)(M * 2 * kChunk + 2 * kScaleTile));
                    const int j0 = (int)((kc * kChunk) / GROUP) & ~7;
                    tma_load_2d(smem_u32(st + L.sc), &a.ms[cur.p], j0, (int)(rb * 128), afull(s));
                    tma_load_2d(smem_u32(st + L.zr), &a.mz[cur.p], j0, (int)(rb * 128), afull(s));
                }
                if (with_x)
                    for (int m = 0; m < M; m++)
                        tma_load_1d(smem_u32(st + L.xraw + m * 2 * kChunk), P.x + (int64_t)m * P.k + kc * kChunk,
                                    2 * kChunk, afull(s));
            };
            // prologue: weights and scales of the first stages do not depend on the previous kernel
            const int64_t pro = min((int64_t)nstage, u_end - u_begin);
            for (int64_t j = 0; j < pro; j++) issue(u_begin + j, (int)j, true, false);
            griddep_wait();
            cur.p = 0;
            for (int64_t j = 0; j < pro; j++) issue(u_begin + j, (int)j, false, true);
            int64_t it = pro;
            for (int64_t u = u_begin + pro; u < u_end; u++, it++) {
                const int s = (int)(it % nstage);
                const uint32_t ph = (uint32_t)((it / nstage) & 1);
                if (!mbar_wait_bounded(empty(s), ph ^ 1u, err)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                issue(u, s, true, true);
            }
            for (int64_t j = (it > nstage ? it - nstage : 0); j < it; j++) {
                mbar_wait_bounded(wfull((int)(j % nstage)), (uint32_t)((j / nstage) & 1), err);
                mbar_wait_bounded(afull((int)(j % nstage)), (uint32_t)((j / nstage) & 1), err);
            }
        }
        return;
    }

    // ------------------------------------------------------------ activation prep warps
    if (warp > kProducerWarp) {
        const int pw = warp - kProducerWarp - 1;
        int64_t it = 0;
        for (int64_t u = u_begin; u < u_end; u++, it++) {
            const int s = (int)(it % nstage);
            const uint32_t ph = (uint32_t)((it / nstage) & 1);
            if (*abort_flag || !mbar_wait_bounded(afull(s), ph, err)) {
                *abort_flag = 1;
                return;
            }
            uint8_t* st = stage0 + (size_t)s * L.bytes;
            for (int m = pw; m < M; m += kPrepWarps) {
                const uint4 raw = *reinterpret_cast<const uint4*>(st + L.xraw + m * 2 * kChunk + 16 * lane);
                const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
                float v[8];
                float mx = 0.0f;
#pragma unroll
                for (int e = 0; e < 8; e++) {
                    v[e] = to_f32<BF16>((uint16_t)(rw[e / 2] >> (16 * (e & 1))));
                    mx = fmaxf(mx, fabsf(v[e]));
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const int E = fixed_point_exponent(mx);
                // v * 2^-E in at most two exact power-of-two multiplications
                const int e1 = max(-126, min(127, -E));
                const float f1 = exp2i(e1), f2 = exp2i(-E - e1);
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
                *reinterpret_cast<uint2*>(st + L.planes + (2 * m) * kPlanePitch + 8 * lane) = make_uint2(hev, hod);
                *reinterpret_cast<uint2*>(st + L.planes + (2 * m + 1) * kPlanePitch + 8 * lane) = make_uint2(lev, lod);
                constexpr int LPG = GROUP / 8;                 // lanes per group
#pragma unroll
                for (int o = 1; o < LPG; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                // group sums are exact in fp32 (|sum| <= 128 * 32639 < 2^24)
                if (lane % LPG == 0) reinterpret_cast<float*>(st + L.xsum)[m * 8 + lane / LPG] = (float)sum;
                if (lane == 0) reinterpret_cast<int*>(st + L.expo)[m] = E;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(xready(s));
        }
        return;
    }

    // ------------------------------------------------------------ consumer warps
    const int g = lane >> 2, c = lane & 3;
    const int rl = warp * 16 + g;                        // row inside the 128-row block
    UnitCursor cur;
    int64_t it = 0;
    for (int64_t u0 = u_begin; u0 < u_end;) {
        cur.seek(a, u0);
        const GemvProblemDev& P = a.p[cur.p];
        const int64_t lu0 = u0 - P.unit_begin;
        const int64_t rb = lu0 / P.kch;
        const int64_t kc0 = lu0 % P.kch;
        const int64_t kc1 = min(P.kch, kc0 + (u_end - u0));
        u0 += kc1 - kc0;
        const int64_t tile = rb * kConsumers + warp;
        const bool active = tile < P.n_tiles;

        float acc[NB][2];
#pragma unroll
        for (int nb = 0; nb < NB; nb++) acc[nb][0] = acc[nb][1] = 0.0f;

        for (int64_t kc = kc0; kc < kc1; kc++, it++) {
            const int s = (int)(it % nstage);
            const uint32_t ph = (uint32_t)((it / nstage) & 1);
            if (!mbar_wait_bounded(wfull(s), ph, err) || !mbar_wait_bounded(xready(s), ph, err)) {
                *abort_flag = 1;
                return;
            }
            if (active) {
                const uint8_t* st = stage0 + (size_t)s * L.bytes;
                const uint8_t* wt = st + warp * TILE_BYTES + lane * 16;
                uint32_t lo[F::NLO], hi[F::NHI];
#pragma unroll
                for (int i = 0; i < G::W0; i++) {
                    const uint4 v = *reinterpret_cast<const uint4*>(wt + i * 512);
                    lo[4 * i] = v.x; lo[4 * i + 1] = v.y; lo[4 * i + 2] = v.z; lo[4 * i + 3] = v.w;
                }
#pragma unroll
                for (int i = 0; i < G::W1; i++) {
                    const uint4 v = *reinterpret_cast<const uint4*>(wt + 512 * G::W0 + i * 512);
                    hi[4 * i] = v.x; hi[4 * i + 1] = v.y; hi[4 * i + 2] = v.z; hi[4 * i + 3] = v.w;
                }
                if constexpr (G::W1 == 0) hi[0] = 0;
                // scales and zeros of this chunk's NGC groups, rows g and g+8 (fp16 -> fp32)
                const int jb = (int)((kc * kChunk) / GROUP) & 7;
                const uint16_t* ss = reinterpret_cast<const uint16_t*>(st + L.sc);
                const uint16_t* zz = reinterpret_cast<const uint16_t*>(st + L.zr);
                uint32_t sh0[NGC / 2], sh1[NGC / 2], zh0[NGC / 2], zh1[NGC / 2];
                lds_halves<NGC>(ss + rl * kScaleBox + jb, sh0);
                lds_halves<NGC>(ss + (rl + 8) * kScaleBox + jb, sh1);
                lds_halves<NGC>(zz + rl * kScaleBox + jb, zh0);
                lds_halves<NGC>(zz + (rl + 8) * kScaleBox + jb, zh1);
                // B-fragment source rows: plane 8*nb + g (token (8*nb + g)/2, hi or lo)
                const uint8_t* prow[NB];
                bool pval[NB];
#pragma unroll
                for (int nb = 0; nb < NB; nb++) {
                    const int pl = 8 * nb + g;
                    pval[nb] = pl < 2 * M;
                    prow[nb] = st + L.planes + (pval[nb] ? pl : 0) * kPlanePitch + 8 * c;
                }
                const float* xs = reinterpret_cast<const float*>(st + L.xsum);
                float cacc[NB][2];
#pragma unroll
                for (int nb = 0; nb < NB; nb++) cacc[nb][0] = cacc[nb][1] = 0.0f;
                int ci[NB][4];
                static_for<0, 8>([&](auto kap_c) {
                    constexpr int kap = decltype(kap_c)::value;
                    const uint32_t a0 = F::template reg<kap, 0, 0>(lo, hi);
                    const uint32_t a1 = F::template reg<kap, 1, 0>(lo, hi);
                    const uint32_t a2 = F::template reg<kap, 0, 1>(lo, hi);
                    const uint32_t a3 = F::template reg<kap, 1, 1>(lo, hi);
#pragma unroll
                    for (int nb = 0; nb < NB; nb++) {
                        uint2 bv = make_uint2(0u, 0u);
                        if (pval[nb]) bv = *reinterpret_cast<const uint2*>(prow[nb] + 32 * kap);
                        if constexpr (kap % KPG == 0) mma_16832_u8s8_zc(ci[nb], a0, a1, a2, a3, bv.x, bv.y);
                        else mma_16832_u8s8(ci[nb], a0, a1, a2, a3, bv.x, bv.y);
                    }
                    if constexpr (kap % KPG == KPG - 1) {
                        constexpr int gi = kap / KPG;
                        const float sg = __half2float(__ushort_as_half((uint16_t)(sh0[gi / 2] >> (16 * (gi & 1)))));
                        const float sg8 = __half2float(__ushort_as_half((uint16_t)(sh1[gi / 2] >> (16 * (gi & 1)))));
                        const float zg = __half2float(__ushort_as_half((uint16_t)(zh0[gi / 2] >> (16 * (gi & 1)))));
                        const float zg8 = __half2float(__ushort_as_half((uint16_t)(zh1[gi / 2] >> (16 * (gi & 1)))));
#pragma unroll
                        for (int nb = 0; nb < NB; nb++) {
                            const int tok = 4 * nb + c;
                            const float X = tok < M ? xs[tok * 8 + gi] : 0.0f;
                            const float f0 = fmaf(-zg, X, (float)(256 * ci[nb][0] + ci[nb][1]));
                            const float f1 = fmaf(-zg8, X, (float)(256 * ci[nb][2] + ci[nb][3]));
                            cacc[nb][0] = fmaf(sg, f0, cacc[nb][0]);
                            cacc[nb][1] = fmaf(sg8, f1, cacc[nb][1]);
                        }
                    }
                });
                const int* ex = reinterpret_cast<const int*>(st + L.expo);
#pragma unroll
                for (int nb = 0; nb < NB; nb++) {
                    const int tok = 4 * nb + c;
                    const float sc = tok < M ? exp2i(ex[tok]) : 0.0f;
                    acc[nb][0] = fmaf(sc, cacc[nb][0], acc[nb][0]);
                    acc[nb][1] = fmaf(sc, cacc[nb][1], acc[nb][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(s));
        }
        if (active)
            tile_epilogue<NB>(acc, (kc0 == 0) && (kc1 == P.kch), M, P.n, tile, P.tile_begin + tile,
                              P.unit_begin + rb * P.kch, P.kch, S_total, NC, blockIdx.x, a.partials, a.counters,
                              a.maxc, P.y);
    }
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// [rows x cols] fp16 array, box of 128 rows x kScaleBox columns, zero fill outside.
static bool encode_scale_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {kScaleBox, 128};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int gemv_nstage(int bits, int64_t M) {
    const int sb = StageLayout(bits, (int)M).bytes;
    const int ns = (kGemvSmemBudget - kBarBytes) / sb;
    return ns > 12 ? 12 : ns;
}

bool gemv_group_tma_supported(int64_t M, int64_t n, int64_t k, int bits, int group) {
    if (M < 1 || M > 16 || k % kChunk != 0 || n % 16 != 0 || bits < 2 || bits > 6) return false;
    if ((k / group) % 8 != 0) return false;              // 16-byte row stride of the scale arrays
    if (n / 16 > kMaxTiles || k / group > ((int64_t)1 << 31)) return false;
    return gemv_nstage(bits, M) >= 2;
}

struct GemvPlan {
    int64_t total_units = 0, total_tiles = 0;
    int grid = 1, maxc = 2;
};

static GemvPlan plan_gemv(const int64_t* n, const int64_t* k, int count) {
    GemvPlan pl;
    int64_t max_kch = 1;
    for (int i = 0; i < count; i++) {
        const int64_t n_tiles = n[i] / 16;
        const int64_t kch = k[i] / kChunk;
        pl.total_units += ceil_div(n_tiles, kConsumers) * kch;
        pl.total_tiles += n_tiles;
        max_kch = std::max(max_kch, kch);
    }
    pl.grid = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)sm_count() * 2, pl.total_units));
    // contributors to one row block: at most ceil(kch * grid / total_units) + 1
    pl.maxc = (int)(ceil_div(max_kch * pl.grid, std::max<int64_t>(pl.total_units, 1)) + 1);
    return pl;
}

size_t gemv_group_tma_ws_bytes_multi(const int64_t* n, const int64_t* k, int count, int64_t M) {
    const GemvPlan pl = plan_gemv(n, k, count);
    return kCounterBytes + (size_t)(pl.total_tiles * pl.maxc * 16 * M * 4);
}

size_t gemv_group_tma_ws_bytes(int64_t M, int64_t n, int64_t k) { return gemv_group_tma_ws_bytes_multi(&n, &k, 1, M); }

template <int B, int GROUP, int NB, bool BF16>
static lbq_status launch_inst(int grid, size_t smem, cudaStream_t st, const GemvArgs& args) {
    auto kern = k_gemv_group_tc<B, GROUP, NB, BF16>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemvSmemBudget) != cudaSuccess)
            return LBQ_ERR_CUDA;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kGemvThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, args) != cudaSuccess) return LBQ_ERR_CUDA;
    return launch_status();
}

template <int B, bool BF16>
static lbq_status launch_b(int group, int NB, int grid, size_t smem, cudaStream_t st, const GemvArgs& args) {
#define LBQ_I(GR, NBV) launch_inst<B, GR, NBV, BF16>(grid, smem, st, args)
#define LBQ_NB(GR) (NB == 1 ? LBQ_I(GR, 1) : NB == 2 ? LBQ_I(GR, 2) : NB == 3 ? LBQ_I(GR, 3) : LBQ_I(GR, 4))
    if (group == 32) return LBQ_NB(32);
    if (group == 64) return LBQ_NB(64);
    return LBQ_NB(128);
#undef LBQ_NB
#undef LBQ_I
}

lbq_status launch_gemv_group_tma_multi(const lbq_gemv_problem* probs, int count, bool bf16, int64_t M, int bits,
                                       int group, void* ws, size_t ws_bytes, cudaStream_t st) {
    int64_t n[kMaxGemvProblems], k[kMaxGemvProblems];
    for (int i = 0; i < count; i++) {
        n[i] = probs[i].n;
        k[i] = probs[i].k;
    }
    const GemvPlan pl = plan_gemv(n, k, count);
    if (pl.total_units == 0) return LBQ_OK;
    if (ws == nullptr || ws_bytes < gemv_group_tma_ws_bytes_multi(n, k, count, M)) return LBQ_ERR_WORKSPACE;
    if (pl.total_tiles > kMaxTiles) return LBQ_ERR_UNSUPPORTED;
    if (encode_fn() == nullptr) return LBQ_ERR_CUDA;
    GemvArgs args;
    memset(&args, 0, sizeof args);
    int64_t ub = 0, tb = 0;
    for (int i = 0; i < count; i++) {
        if (!encode_scale_map(&args.ms[i], probs[i].scales, n[i], k[i] / group) ||
            !encode_scale_map(&args.mz[i], probs[i].zeros, n[i], k[i] / group))
            return LBQ_ERR_CUDA;
        GemvProblemDev& P = args.p[i];
        P.x = (const uint16_t*)probs[i].x;
        P.packed = (const uint8_t*)probs[i].packed;
        P.y = (uint16_t*)probs[i].y;
        P.n = n[i];
        P.k = k[i];
        P.n_tiles = n[i] / 16;
        P.kch = k[i] / kChunk;
        P.unit_begin = ub;
        P.tile_begin = tb;
        ub += ceil_div(P.n_tiles, kConsumers) * P.kch;
        tb += P.n_tiles;
    }
    args.partials = (float*)((char*)ws + kCounterBytes);
    args.counters = (unsigned*)ws;
    args.err = device_error_word();
    args.total_units = pl.total_units;
    args.count = count;
    args.M = (int)M;
    args.maxc = pl.maxc;
    args.nstage = gemv_nstage(bits, M);
    const size_t smem = kBarBytes + (size_t)args.nstage * StageLayout(bits, (int)M).bytes;
    const int NB = (int)((2 * M + 7) / 8);
#define LBQ_TB(BB, BF) launch_b<BB, BF>(group, NB, pl.grid, smem, st, args)
    if (bf16) {
        switch (bits) {
            case 2: return LBQ_TB(2, true);
            case 3: return LBQ_TB(3, true);
            case 4: return LBQ_TB(4, true);
            case 5: return LBQ_TB(5, true);
            default: return LBQ_TB(6, true);
        }
    }
    switch (bits) {
        case 2: return LBQ_TB(2, false);
        case 3: return LBQ_TB(3, false);
        case 4: return LBQ_TB(4, false);
        case 5: return LBQ_TB(5, false);
        default: return LBQ_TB(6, false);
    }
#undef LBQ_TB
}

lbq_status launch_gemv_group_tma(const void* x, bool bf16, int64_t M, const void* packed, const void* scales,
                                 const void* zeros, int64_t n, int64_t k, int bits, int group, void* y, void* ws,
                                 size_t ws_bytes, cudaStream_t st) {
    lbq_gemv_problem p;
    p.x = x;
    p.packed = packed;
    p.scales = scales;
    p.zeros = zeros;
    p.y = y;
    p.n = n;
    p.k = k;
    return launch_gemv_group_tma_multi(&p, 1, bf16, M, bits, group, ws, ws_bytes, st);
}

}  // namespace lbq
