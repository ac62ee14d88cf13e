// lbq_binlr.cu -- binary low-rank GEMV  y = s1 ⊙ U (V^T (s2 ⊙ x))  (sm_100a).
//
// Form: "70B en 4GB de VRAM: la compresión neural de 2026, ¿es real?" (nramos.dev),
// section "1. NanoQuant — sub-1-bit PTQ", bullet "Formulación":
// W ≈ s1 ⊙ (U±1 · V±1ᵀ) ⊙ s2ᵀ with binary low-rank factors.  The page's own binary
// GEMV/GEMM kernels (same bullet list) are not used; this is a B200 design.
//
// Fast path (LBQ_LAYOUT_KERNEL), one ±1 matrix-vector product per stage:
//   sum_k sign[i,k] v[k] = 2 * sum_{bit=1} v[k] - sum_k v[k]
//  * v (s2 ⊙ x for stage 1, t for stage 2) is turned into a 16-bit fixed-point
//    integer with one power-of-two scale 2^E per token (|v_q| <= 32639) and split
//    into two int8 planes hi, lo with v_q = 256*hi + lo;
//  * a 32-bit word of signs masked with 0x01010101 << p gives four u8 A-fragment
//    bytes equal to 2^p * bit (one LOP per four signs); integer tensor cores
//    (mma m16n8k32 u8 x s8 -> s32) multiply them by the planes, one accumulator set
//    per p, and the sets are combined exactly as acc_p >> p at the end.  For M > 4
//    tokens the bytes are shifted down to 0/1 instead and one set suffices;
//  * every partial sum is an exact int32, so split-K contributions are added with
//    integer atomics in any order and the result stays deterministic;
//  * five launches: quantize v -> stage 1 -> t and quantize t -> stage 2 -> scale.
// Canonical path: CUDA-core fp32 sign-select sums, two launches.
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

constexpr int kBinWarps = 8;
constexpr int kPlaneMax = 32639;   // |v_q| bound so that hi = (v_q + 128) >> 8 fits in int8

// ------------------------------------------------------------------ workspace
struct BinWs {
    int8_t* planes1;   // [2M][Kp1]
    int8_t* planes2;   // [2M][Kp2]
    int* S1;           // [M][r]
    int* S2;           // [M][d_out]
    int* meta;         // [M][4]: E1, vsum1, E2, vsum2
    float* t;          // canonical path: [M][r]
    size_t bytes;
};


static BinWs bin_ws(void* base, int64_t M, int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout) {
    BinWs w{};
    char* p = (char*)base;
    size_t off = kCounterBytes;
    if (layout == LBQ_LAYOUT_CANONICAL) {
        w.t = (float*)(p + off);
        off += al256((size_t)(M * r * 4));
        w.bytes = off;
        return w;
    }
    const int64_t kp1 = sign_cols_pad(d_in), kp2 = sign_cols_pad(r);
    w.planes1 = (int8_t*)(p + off); off += al256((size_t)(2 * M * kp1));
    w.planes2 = (int8_t*)(p + off); off += al256((size_t)(2 * M * kp2));
    w.S1 = (int*)(p + off); off += al256((size_t)(M * r * 4));
    w.S2 = (int*)(p + off); off += al256((size_t)(M * d_out * 4));
    w.meta = (int*)(p + off); off += al256((size_t)(M * 16));
    w.bytes = off;
    return w;
}

size_t gemv_binlr_ws_bytes(int64_t M, int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout) {
    size_t b = bin_ws(nullptr, M, d_out, d_in, r, layout).bytes;
    if (layout == LBQ_LAYOUT_KERNEL && gemv_binlr_ldg_supported(M, d_out, d_in, r))
        b = std::max(b, gemv_binlr_ldg_ws_bytes(M, d_out, d_in, r));
    return b;
}

// ------------------------------------------------------------------ fixed-point planes
__device__ __forceinline__ float block_max(float v, float* red) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0f;
    if (w == 0)
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (threadIdx.x == 0) red[0] = v;
    __syncthreads();
    return red[0];
}
__device__ __forceinline__ int block_sum(int v, int* red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0;
    if (w == 0)
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
    __syncthreads();
    return red[0];
}

// Smallest E with maxabs * 2^-E <= kPlaneMax (E = 0 for an all-zero vector).
__device__ __forceinline__ int plane_exponent(float maxabs) {
    if (!(maxabs > 0.0f)) return 0;
    const int e0 = ilogbf(maxabs) - 14;
    return e0 + (ldexpf(maxabs, -e0) > (float)kPlaneMax ? 1 : 0);
}

// Stage-1 input: v[k] = s2[k] * x[m][k] (exact fp32 product of two 11-bit values).
// Stage-2 input: v[k] = 2^E1 * (2*S1[m][k] - vsum1[m]).
// Blocks [0, M) quantize token blockIdx.x; the rest zero `zero_a`/`zero_b`.
template <bool BF16, bool STAGE2>
__global__ void __launch_bounds__(1024)
k_bin_prep(int M, int64_t K, int64_t Kp, const uint16_t* __restrict__ x, const uint16_t* __restrict__ s2,
           const int* __restrict__ S1, int* __restrict__ meta, int8_t* __restrict__ planes, int* zero_a,
           int64_t n_zero_a, int* zero_b, int64_t n_zero_b) {
    __shared__ float redf[32];
    __shared__ int redi[32];
    if ((int)blockIdx.x >= M) {
        const int64_t nb = gridDim.x - M;
        const int64_t tid = (blockIdx.x - M) * (int64_t)blockDim.x + threadIdx.x;
        for (int64_t i = tid; i < n_zero_a; i += nb * blockDim.x) zero_a[i] = 0;
        for (int64_t i = tid; i < n_zero_b; i += nb * blockDim.x) zero_b[i] = 0;
        return;
    }
    const int m = blockIdx.x;
    auto value = [&](int64_t kk) -> float {
        if constexpr (STAGE2) {
            const int I = 2 * S1[(int64_t)m * K + kk] - meta[m * 4 + 1];
            return ldexpf((float)I, meta[m * 4 + 0]);
        } else {
            return __half2float(__ushort_as_half(s2[kk])) * to_f32<BF16>(x[(int64_t)m * K + kk]);
        }
    };
    float mx = 0.0f;
    for (int64_t kk = threadIdx.x; kk < K; kk += blockDim.x) mx = fmaxf(mx, fabsf(value(kk)));
    mx = block_max(mx, redf);
    const int E = plane_exponent(mx);
    int vs = 0;
    int8_t* hi = planes + (int64_t)(2 * m) * Kp;
    int8_t* lo = hi + Kp;
    for (int64_t kk = threadIdx.x; kk < Kp; kk += blockDim.x) {
        int q = 0;
        if (kk < K) q = __float2int_rn(ldexpf(value(kk), -E));
        const int h = (q + 128) >> 8;
        hi[kk] = (int8_t)h;
        lo[kk] = (int8_t)(q - 256 * h);
        vs += q;
    }
    vs = block_sum(vs, redi);
    if (threadIdx.x == 0) {
        meta[m * 4 + (STAGE2 ? 2 : 0)] = E;
        meta[m * 4 + (STAGE2 ? 3 : 1)] = vs;
    }
}

// ------------------------------------------------------------------ sign x planes product
// S[m][row] += sum over the CTA's k-range of bit[row][k] * v_q[m][k]  (int32 atomics).
// PMASK: per-p accumulators with bytes 2^p*bit (M <= 4); else 0/1 bytes, NB n-blocks.
template <int NB, bool PMASK>
__global__ void __launch_bounds__(kBinWarps * 32)
k_bin_stage(int M, int64_t rows, int64_t Kp, const uint8_t* __restrict__ signs, const int8_t* __restrict__ planes,
            int* __restrict__ S) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int64_t KSB = Kp / 256;
    const int64_t n_tiles = rows / 16;
    const int64_t n_rb = ceil_div(n_tiles, kBinWarps);
    const int64_t S_total = n_rb * KSB;
    const int64_t NC = gridDim.x;
    const int64_t u_begin = (int64_t)blockIdx.x * S_total / NC;
    const int64_t u_end = ((int64_t)blockIdx.x + 1) * S_total / NC;

    // plane rows this lane feeds as B column g of n-block nb: plane index 8*nb + g
    const int8_t* prow[NB];
    bool pval[NB];
#pragma unroll
    for (int nb = 0; nb < NB; nb++) {
        const int pl = 8 * nb + g;
        pval[nb] = pl < 2 * M;
        prow[nb] = planes + (int64_t)(pval[nb] ? pl : 0) * Kp + 4 * c;
    }

    for (int64_t u0 = u_begin; u0 < u_end;) {
        const int64_t rb = u0 / KSB;
        const int64_t ks0 = u0 % KSB;
        const int64_t ks1 = min(KSB, ks0 + (u_end - u0));
        u0 += ks1 - ks0;
        const int64_t tile = rb * kBinWarps + warp;
        if (tile >= n_tiles) continue;
        const uint8_t* tp = signs + (tile * KSB) * 512 + lane * 16;

        constexpr int NSET = PMASK ? 8 : 1;
        int acc[NSET][NB][4];
#pragma unroll
        for (int s = 0; s < NSET; s++)
#pragma unroll
            for (int nb = 0; nb < NB; nb++)
#pragma unroll
                for (int e = 0; e < 4; e++) acc[s][nb][e] = 0;

        uint4 cur = ldg_stream(tp + ks0 * 512);
        for (int64_t ks = ks0; ks < ks1; ks++) {
            uint4 nxt = cur;
            if (ks + 1 < ks1) nxt = ldg_stream(tp + (ks + 1) * 512);
            const int64_t kb = ks * 256;
#pragma unroll
            for (int p = 0; p < 8; p++) {
                uint32_t a0, a1, a2, a3;
                if constexpr (PMASK) {
                    const uint32_t msk = 0x01010101u << p;
                    a0 = cur.x & msk; a1 = cur.y & msk; a2 = cur.z & msk; a3 = cur.w & msk;
                } else {
                    a0 = (cur.x >> p) & 0x01010101u; a1 = (cur.y >> p) & 0x01010101u;
                    a2 = (cur.z >> p) & 0x01010101u; a3 = (cur.w >> p) & 0x01010101u;
                }
#pragma unroll
                for (int nb = 0; nb < NB; nb++) {
                    uint32_t b0 = 0, b1 = 0;
                    if (pval[nb]) {
                        b0 = ldg_u32(prow[nb] + kb + 32 * p);
                        b1 = ldg_u32(prow[nb] + kb + 32 * p + 16);
                    }
                    mma_16832_u8s8(acc[PMASK ? p : 0][nb], a0, a1, a2, a3, b0, b1);
                }
            }
            cur = nxt;
        }
        // combine and add: lane (g, c) holds columns 2c (hi) and 2c+1 (lo) of token 4*nb + c
#pragma unroll
        for (int nb = 0; nb < NB; nb++) {
            int v[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                int s = 0;
#pragma unroll
                for (int q = 0; q < NSET; q++) s += PMASK ? (acc[q][nb][e] >> q) : acc[q][nb][e];
                v[e] = s;
            }
            const int tok = 4 * nb + c;
            if (tok < M) {
                const int64_t row = tile * 16 + g;
                atomicAdd(S + (int64_t)tok * rows + row, 256 * v[0] + v[1]);
                atomicAdd(S + (int64_t)tok * rows + row + 8, 256 * v[2] + v[3]);
            }
        }
    }
}

// y[m][i] = s1[i] * 2^E2 * (2*S2[m][i] - vsum2[m])
template <bool BF16>
__global__ void k_bin_finish(int M, int64_t d_out, const int* __restrict__ S2, const int* __restrict__ meta,
                             const uint16_t* __restrict__ s1, uint16_t* __restrict__ y) {
    const int64_t total = (int64_t)M * d_out;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int m = (int)(i / d_out);
        const int64_t row = i % d_out;
        const int I = 2 * S2[i] - meta[m * 4 + 3];
        const float t = ldexpf((float)I, meta[m * 4 + 2]);
        y[i] = from_f32<false>(__half2float(__ushort_as_half(s1[row])) * t);
    }
}

// ------------------------------------------------------------------ canonical path
// Stage 1: t[m][j] = sum_k sign(Vt[j,k]) * s2[k] * x[m][k]; warp per row j.
template <bool BF16>
__global__ void __launch_bounds__(256)
k_bin_canon_stage1(int M, int64_t d_in, int64_t r, const uint32_t* __restrict__ Vt, const uint16_t* __restrict__ s2,
                   const uint16_t* __restrict__ x, float* __restrict__ t) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t wpr = d_in / 32;
    for (int64_t j = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; j < r; j += nw) {
        float acc[16];
#pragma unroll
        for (int m = 0; m < 16; m++) acc[m] = 0.0f;
        for (int64_t wi = lane; wi < wpr; wi += 32) {
            const uint32_t w = Vt[j * wpr + wi];
            for (int b = 0; b < 32; b++) {
                const int64_t kk = wi * 32 + b;
                const float s = __half2float(__ushort_as_half(s2[kk]));
                const bool plus = (w >> b) & 1u;
#pragma unroll
                for (int m = 0; m < 16; m++)
                    if (m < M) {
                        const float v = s * to_f32<BF16>(x[(int64_t)m * d_in + kk]);
                        acc[m] += plus ? v : -v;
                    }
            }
        }
#pragma unroll
        for (int m = 0; m < 16; m++)
            if (m < M) {
                float v = acc[m];
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) t[(int64_t)m * r + j] = v;
            }
    }
}

// Stage 2: y[m][i] = s1[i] * sum_j sign(U[i,j]) * t[m][j]; warp per row i.
template <bool BF16>
__global__ void __launch_bounds__(256)
k_bin_canon_stage2(int M, int64_t d_out, int64_t r, const uint32_t* __restrict__ U, const uint16_t* __restrict__ s1,
                   const float* __restrict__ t, uint16_t* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t wpr = r / 32;
    for (int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; i < d_out; i += nw) {
        float acc[16];
#pragma unroll
        for (int m = 0; m < 16; m++) acc[m] = 0.0f;
        for (int64_t wi = lane; wi < wpr; wi += 32) {
            const uint32_t w = U[i * wpr + wi];
            for (int b = 0; b < 32; b++) {
                const int64_t j = wi * 32 + b;
                const bool plus = (w >> b) & 1u;
#pragma unroll
                for (int m = 0; m < 16; m++)
                    if (m < M) {
                        const float v = t[(int64_t)m * r + j];
                        acc[m] += plus ? v : -v;
                    }
            }
        }
        const float sc = __half2float(__ushort_as_half(s1[i]));
#pragma unroll
        for (int m = 0; m < 16; m++)
            if (m < M) {
                float v = acc[m];
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) y[(int64_t)m * d_out + i] = from_f32<false>(sc * v);
            }
    }
}

// ------------------------------------------------------------------ host side
static int bin_grid(int64_t rows, int64_t Kp) {
    const int64_t n_rb = ceil_div(rows / 16, kBinWarps);
    const int64_t S_total = n_rb * (Kp / 256);
    return (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)sm_count() * 2, S_total));
}

static void launch_stage(int M, int64_t rows, int64_t Kp, const uint8_t* signs, const int8_t* planes, int* S,
                         cudaStream_t st) {
    const int grid = bin_grid(rows, Kp);
    const int th = kBinWarps * 32;
    if (M <= 4) k_bin_stage<1, true><<<grid, th, 0, st>>>(M, rows, Kp, signs, planes, S);
    else if (M <= 8) k_bin_stage<2, false><<<grid, th, 0, st>>>(M, rows, Kp, signs, planes, S);
    else if (M <= 12) k_bin_stage<3, false><<<grid, th, 0, st>>>(M, rows, Kp, signs, planes, S);
    else k_bin_stage<4, false><<<grid, th, 0, st>>>(M, rows, Kp, signs, planes, S);
}

lbq_status launch_gemv_binlr(const void* x, bool bf16, int64_t M, const void* U, const void* Vt, const void* s1,
                             const void* s2, int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout, void* y,
                             void* ws, size_t ws_bytes, cudaStream_t st) {
    if (M == 0 || d_out == 0) return LBQ_OK;
    // few tokens: the two-launch register-streaming path (lbq_binlr_ldg.cu)
    // (16-byte vector loads of x and s2)
    if (layout == LBQ_LAYOUT_KERNEL && gemv_binlr_ldg_supported(M, d_out, d_in, r) &&
        ((uintptr_t)x | (uintptr_t)s2) % 16 == 0)
        return launch_gemv_binlr_ldg(x, bf16, M, U, Vt, s1, s2, d_out, d_in, r, y, ws, ws_bytes, st);
    const BinWs w = bin_ws(ws, M, d_out, d_in, r, layout);
    if (ws == nullptr || ws_bytes < w.bytes) return LBQ_ERR_WORKSPACE;
    auto* xp = (const uint16_t*)x;
    auto* s1p = (const uint16_t*)s1;
    auto* s2p = (const uint16_t*)s2;
    auto* yp = (uint16_t*)y;
    if (layout == LBQ_LAYOUT_CANONICAL) {
        const int g1 = (int)std::min<int64_t>(ceil_div(r, 8), (int64_t)sm_count() * 8);
        const int g2 = (int)std::min<int64_t>(ceil_div(d_out, 8), (int64_t)sm_count() * 8);
        if (bf16) {
            k_bin_canon_stage1<true><<<g1, 256, 0, st>>>((int)M, d_in, r, (const uint32_t*)Vt, s2p, xp, w.t);
            k_bin_canon_stage2<true><<<g2, 256, 0, st>>>((int)M, d_out, r, (const uint32_t*)U, s1p, w.t, yp);
        } else {
            k_bin_canon_stage1<false><<<g1, 256, 0, st>>>((int)M, d_in, r, (const uint32_t*)Vt, s2p, xp, w.t);
            k_bin_canon_stage2<false><<<g2, 256, 0, st>>>((int)M, d_out, r, (const uint32_t*)U, s1p, w.t, yp);
        }
        return launch_status();
    }
    const int64_t kp1 = sign_cols_pad(d_in), kp2 = sign_cols_pad(r);
    const int zb = (int)std::min<int64_t>(ceil_div(M * (r + d_out), 1024), 64) + 1;
    if (bf16)
        k_bin_prep<true, false><<<(int)M + zb, 1024, 0, st>>>((int)M, d_in, kp1, xp, s2p, nullptr, w.meta, w.planes1,
                                                             w.S1, M * r, w.S2, M * d_out);
    else
        k_bin_prep<false, false><<<(int)M + zb, 1024, 0, st>>>((int)M, d_in, kp1, xp, s2p, nullptr, w.meta,
                                                              w.planes1, w.S1, M * r, w.S2, M * d_out);
    launch_stage((int)M, r, kp1, (const uint8_t*)Vt, w.planes1, w.S1, st);
    k_bin_prep<false, true><<<(int)M, 1024, 0, st>>>((int)M, r, kp2, nullptr, nullptr, w.S1, w.meta, w.planes2,
                                                    nullptr, 0, nullptr, 0);
    launch_stage((int)M, d_out, kp2, (const uint8_t*)U, w.planes2, w.S2, st);
    const int gf = (int)std::min<int64_t>(ceil_div(M * d_out, 256), (int64_t)sm_count() * 8);
    if (bf16) k_bin_finish<true><<<gf, 256, 0, st>>>((int)M, d_out, w.S2, w.meta, s1p, yp);
    else k_bin_finish<false><<<gf, 256, 0, st>>>((int)M, d_out, w.S2, w.meta, s1p, yp);
    return launch_status();
}

}  // namespace lbq
