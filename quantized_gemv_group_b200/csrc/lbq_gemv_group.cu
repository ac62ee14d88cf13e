// lbq_gemv_group.cu -- dequant-fused group GEMV, y = x * W_hat^T, M = 1..16 (sm_100a).
//
//   y[m, i] = sum_k x[m, k] * s[i, k/g] * (q[i, k] - z[i, k/g])
//
// Group format: "TurboQuant: cuantizar modelos grandes para que quepan en local"
// (quellm.com), section "Compresión por bloques" (blocks share a scale and an
// offset); RTN codes from "Métodos de cuantización de LLM para ejecutar un modelo de
// 70B en una sola GPU" (gotburnout.io), section "RTN (Round-To-Nearest)".  Decode is
// bound by the bytes read per token ("AirLLM corre un modelo 70B en una GPU de 4GB",
// section "Por qué es lento"), so the kernel streams the packed codes once, at the
// HBM rate, and does all dequantization in registers.
//
// LBQ_LAYOUT_KERNEL runs on integer tensor cores with the weights streamed straight
// into registers (lbq_gemv_group_ldg.cu).  This file holds the canonical-layout path --
// one warp per row, CUDA-core fp32 FMA, any shape with k % 32 == 0 -- and the dispatch.
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

// ------------------------------------------------------------------ canonical kernel
// One warp per row; each lane takes 32-code chunks (b words) and accumulates in fp32.
template <int B, bool BF16>
__global__ void __launch_bounds__(256)
k_gemv_group_canonical(const uint16_t* __restrict__ x, int M, const uint32_t* __restrict__ packed,
                       const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros, int64_t n,
                       int64_t k, int group, uint16_t* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t chunks = k / 32;
    const int64_t G = k / group;
    for (int64_t row = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; row < n; row += nwarps) {
        float acc[16];
#pragma unroll
        for (int m = 0; m < 16; m++) acc[m] = 0.0f;
        const uint32_t* rp = packed + row * chunks * B;
        for (int64_t ch = lane; ch < chunks; ch += 32) {
            uint32_t w[B];
#pragma unroll
            for (int i = 0; i < B; i++) w[i] = rp[ch * B + i];
            const int64_t gi = (ch * 32) / group;
            const float s = __half2float(__ushort_as_half(scales[row * G + gi]));
            const float z = __half2float(__ushort_as_half(zeros[row * G + gi]));
            float wv[32];
#pragma unroll
            for (int j = 0; j < 32; j++) {
                const int pos = j * B;
                uint32_t v = w[pos / 32] >> (pos % 32);
                if ((pos % 32) + B > 32) v |= w[pos / 32 + 1] << (32 - pos % 32);
                wv[j] = (float)(v & ((1u << B) - 1)) - z;
            }
#pragma unroll
            for (int m = 0; m < 16; m++) {
                if (m < M) {
                    const uint16_t* xr = x + (int64_t)m * k + ch * 32;
                    float d = 0.0f;
#pragma unroll
                    for (int j = 0; j < 32; j++) d = fmaf(wv[j], to_f32<BF16>(xr[j]), d);
                    acc[m] = fmaf(s, d, acc[m]);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < 16; m++) {
            if (m < M) {
                float v = acc[m];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) y[(int64_t)m * n + row] = from_f32<false>(v);
            }
        }
    }
}

// ------------------------------------------------------------------ host side
size_t gemv_group_ws_bytes(int64_t M, int64_t n, int64_t k, int bits, int group, lbq_layout layout) {
    if (layout != LBQ_LAYOUT_KERNEL) return 0;
    if (gemv_group_ldg_supported(M, n, k, bits, group)) return gemv_group_ldg_ws_bytes(M, n, k);
    return 0;
}

template <bool BF16>
static void launch_canonical(int bits, int grid, cudaStream_t st, const uint16_t* x, int M, const uint32_t* packed,
                             const uint16_t* s, const uint16_t* z, int64_t n, int64_t k, int group, uint16_t* y) {
    switch (bits) {
        case 2: k_gemv_group_canonical<2, BF16><<<grid, 256, 0, st>>>(x, M, packed, s, z, n, k, group, y); break;
        case 3: k_gemv_group_canonical<3, BF16><<<grid, 256, 0, st>>>(x, M, packed, s, z, n, k, group, y); break;
        case 4: k_gemv_group_canonical<4, BF16><<<grid, 256, 0, st>>>(x, M, packed, s, z, n, k, group, y); break;
        case 5: k_gemv_group_canonical<5, BF16><<<grid, 256, 0, st>>>(x, M, packed, s, z, n, k, group, y); break;
        default: k_gemv_group_canonical<6, BF16><<<grid, 256, 0, st>>>(x, M, packed, s, z, n, k, group, y); break;
    }
}

lbq_status launch_gemv_group(const void* x, bool bf16, int64_t M, const void* packed, const void* scales,
                             const void* zeros, int64_t n, int64_t k, int bits, int group, lbq_layout layout,
                             void* y, void* ws, size_t ws_bytes, cudaStream_t st) {
    if (M == 0 || n == 0) return LBQ_OK;
    auto* xp = (const uint16_t*)x;
    auto* sp = (const uint16_t*)scales;
    auto* zp = (const uint16_t*)zeros;
    auto* yp = (uint16_t*)y;
    if (layout == LBQ_LAYOUT_CANONICAL) {
        const int grid = (int)std::min<int64_t>(ceil_div(n, 8), (int64_t)sm_count() * 8);
        if (bf16) launch_canonical<true>(bits, grid, st, xp, (int)M, (const uint32_t*)packed, sp, zp, n, k, group, yp);
        else launch_canonical<false>(bits, grid, st, xp, (int)M, (const uint32_t*)packed, sp, zp, n, k, group, yp);
        return launch_status();
    }
    if (!gemv_group_ldg_supported(M, n, k, bits, group)) return LBQ_ERR_UNSUPPORTED;
    return launch_gemv_group_ldg(x, bf16, M, packed, scales, zeros, n, k, bits, group, y, ws, ws_bytes, st);
}

}  // namespace lbq
