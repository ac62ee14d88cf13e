// lbq_quant.cu -- RTN group quantization and bit packing (sm_100a).
//
// Quantizer: "Métodos de cuantización de LLM para ejecutar un modelo de 70B en una
// sola GPU" (gotburnout.io), section "RTN (Round-To-Nearest)" -- round every weight
// to the nearest grid level, no calibration; blocks that share a scale and an offset
// from "TurboQuant: cuantizar modelos grandes para que quepan en local" (quellm.com),
// section "Compresión por bloques".  Every step is one IEEE-correct operation
// (division __fdiv_rn, round-up conversion __float2half_ru, round-half-even
// __float2int_rn), so codes, scales and zeros are bit-exact with any IEEE
// implementation of the same steps.
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

// One warp per group (group = 32 * EPL elements, EPL elements per lane).
template <bool BF16, int EPL>
__global__ void __launch_bounds__(256) k_quantize_rtn(const uint16_t* __restrict__ W, int64_t n_groups,
                                                     int bits, uint8_t* __restrict__ codes,
                                                     uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros,
                                                     unsigned* err) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int qmax = (1 << bits) - 1;
    const float qmaxf = (float)qmax;
    for (int64_t gi = warp; gi < n_groups; gi += nwarps) {
        const int64_t base = gi * (32 * EPL);
        float w[EPL];
        float lo = 0.0f, hi = 0.0f;
        bool finite = true;
#pragma unroll
        for (int e = 0; e < EPL; e++) {
            w[e] = to_f32<BF16>(W[base + e * 32 + lane]);
            finite &= isfinite(w[e]);
            lo = fminf(lo, w[e]);
            hi = fmaxf(hi, w[e]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        if (!__all_sync(0xffffffffu, finite) && lane == 0) atomicOr(err, kErrNonFinite);
        const float d = __fsub_rn(hi, lo);
        const float s32 = __fdiv_rn(d, qmaxf);
        __half sh = __float2half_ru(s32);
        float s = __half2float(sh);
        if (s == 0.0f) { sh = __float2half_rn(1.0f); s = 1.0f; }
        int z = __float2int_rn(__fdiv_rn(-lo, s));
        z = min(max(z, 0), qmax);
#pragma unroll
        for (int e = 0; e < EPL; e++) {
            int q = __float2int_rn(__fdiv_rn(w[e], s)) + z;
            q = min(max(q, 0), qmax);
            codes[base + e * 32 + lane] = (uint8_t)q;
        }
        if (lane == 0) {
            scales[gi] = __half_as_ushort(sh);
            zeros[gi] = __half_as_ushort(__int2half_rn(z));
        }
    }
}

lbq_status launch_quantize_rtn(const void* W, bool bf16, int64_t n, int64_t k, int bits, int group,
                               uint8_t* codes, void* scales, void* zeros, cudaStream_t st) {
    const int64_t n_groups = n * (k / group);
    if (n_groups == 0) return LBQ_OK;
    const int threads = 256;
    const int64_t want = ceil_div(n_groups, threads / 32);
    const int grid = (int)std::min<int64_t>(want, (int64_t)sm_count() * 32);
    auto* w = (const uint16_t*)W;
    auto* s = (uint16_t*)scales;
    auto* z = (uint16_t*)zeros;
    unsigned* err = device_error_word();
#define LBQ_Q(BF, EPL) k_quantize_rtn<BF, EPL><<<grid, threads, 0, st>>>(w, n_groups, bits, codes, s, z, err)
    if (bf16) {
        if (group == 32) LBQ_Q(true, 1); else if (group == 64) LBQ_Q(true, 2); else LBQ_Q(true, 4);
    } else {
        if (group == 32) LBQ_Q(false, 1); else if (group == 64) LBQ_Q(false, 2); else LBQ_Q(false, 4);
    }
#undef LBQ_Q
    return launch_status();
}

// ---------------------------------------------------------------- canonical packing
// One thread per 32 codes of a row (k % 32 == 0): reads 32 bytes, writes `bits` words.
template <int B>
__global__ void k_pack_canonical(const uint8_t* __restrict__ codes, int64_t nchunks, uint32_t* __restrict__ out) {
    for (int64_t ch = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; ch < nchunks;
         ch += (int64_t)gridDim.x * blockDim.x) {
        const uint4 lo = *reinterpret_cast<const uint4*>(codes + ch * 32);
        const uint4 hi = *reinterpret_cast<const uint4*>(codes + ch * 32 + 16);
        const uint32_t src[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        uint32_t w[B];
#pragma unroll
        for (int i = 0; i < B; i++) w[i] = 0;
#pragma unroll
        for (int j = 0; j < 32; j++) {
            const uint32_t v = (src[j / 4] >> (8 * (j % 4))) & ((1u << B) - 1);
            const int pos = j * B;
            w[pos / 32] |= v << (pos % 32);
            if ((pos % 32) + B > 32) w[pos / 32 + 1] |= v >> (32 - pos % 32);
        }
#pragma unroll
        for (int i = 0; i < B; i++) out[ch * B + i] = w[i];
    }
}

template <int B>
__global__ void k_unpack_canonical(const uint32_t* __restrict__ in, int64_t nchunks, uint8_t* __restrict__ codes) {
    for (int64_t ch = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; ch < nchunks;
         ch += (int64_t)gridDim.x * blockDim.x) {
        uint32_t w[B];
#pragma unroll
        for (int i = 0; i < B; i++) w[i] = in[ch * B + i];
        uint32_t dst[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 32; j++) {
            const int pos = j * B;
            uint32_t v = w[pos / 32] >> (pos % 32);
            if ((pos % 32) + B > 32) v |= w[pos / 32 + 1] << (32 - pos % 32);
            v &= (1u << B) - 1;
            dst[j / 4] |= v << (8 * (j % 4));
        }
        *reinterpret_cast<uint4*>(codes + ch * 32) = make_uint4(dst[0], dst[1], dst[2], dst[3]);
        *reinterpret_cast<uint4*>(codes + ch * 32 + 16) = make_uint4(dst[4], dst[5], dst[6], dst[7]);
    }
}

// ---------------------------------------------------------------- kernel layout
// Word-centric: each 32-bit output word gathers (or scatters, when unpacking) its
// codes.  Word of (tile T, superblock S, plane p of width w, chunk i, lane L = 4g+c,
// word wi): it holds octets eta = O*omega + o (omega = 4i + wi, O = 4/w, o < O);
// octet eta is row 16T + g + 8*(eta%2), columns 256S + 32*(eta/2) + 8c + nu, and
// code nu = 2j + e sits at bits 8j + 2w*o + w*e.
template <int B, bool UNPACK>
__global__ void k_kernel_layout(const uint8_t* __restrict__ codes_in, uint32_t* __restrict__ words, int64_t n,
                                int64_t k, uint8_t* __restrict__ codes_out) {
    using G = GroupGeom<B>;
    const int64_t nwords = n * k * B / 32;
    const int64_t ksb = k / 256;
    for (int64_t wi_all = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; wi_all < nwords;
         wi_all += (int64_t)gridDim.x * blockDim.x) {
        const int64_t byte = wi_all * 4;
        const int64_t sbi = byte / G::SB_BYTES;
        const int64_t T = sbi / ksb, S = sbi % ksb;
        const int off = (int)(byte % G::SB_BYTES);
        const int plane = off < 512 * G::W0 ? 0 : 1;
        const int poff = plane ? off - 512 * G::W0 : off;
        const int w = plane ? G::W1 : G::W0;
        const int O = 4 / w;
        const int i = poff / 512, L = (poff % 512) / 16, wi = (poff % 16) / 4;
        const int g = L / 4, c = L % 4;
        const int omega = 4 * i + wi;
        const uint32_t vmask = (1u << w) - 1;
        uint32_t word = UNPACK ? words[wi_all] : 0u;
        for (int o = 0; o < O; o++) {
            const int eta = O * omega + o;
            const int64_t row = T * 16 + g + 8 * (eta % 2);
            const int64_t kb = S * 256 + 32 * (eta / 2) + 8 * c;
            for (int nu = 0; nu < 8; nu++) {
                const int sh = 8 * (nu / 2) + 2 * w * o + w * (nu % 2);
                uint8_t* dst = codes_out ? codes_out + row * k + kb + nu : nullptr;
                if (!UNPACK) {
                    const uint32_t q = codes_in[row * k + kb + nu];
                    const uint32_t v = plane ? (q >> G::W0) : (q & ((1u << G::W0) - 1));
                    word |= (v & vmask) << sh;
                } else {
                    const uint32_t v = ((word >> sh) & vmask) << (plane ? G::W0 : 0);
                    // low and high planes of a code live in different words: OR into place
                    atomicOr(reinterpret_cast<unsigned*>((uintptr_t)dst & ~(uintptr_t)3),
                             v << (8 * ((uintptr_t)dst & 3)));
                }
            }
        }
        if (!UNPACK) words[wi_all] = word;
    }
}

lbq_status launch_pack(const uint8_t* codes, int64_t n, int64_t k, int bits, lbq_layout layout, void* packed,
                       cudaStream_t st) {
    const int threads = 256;
    const int gmax = sm_count() * 16;
    if (layout == LBQ_LAYOUT_CANONICAL) {
        const int64_t nch = n * k / 32;
        if (nch == 0) return LBQ_OK;
        const int grid = (int)std::min<int64_t>(ceil_div(nch, threads), gmax);
        auto* o = (uint32_t*)packed;
        switch (bits) {
            case 2: k_pack_canonical<2><<<grid, threads, 0, st>>>(codes, nch, o); break;
            case 3: k_pack_canonical<3><<<grid, threads, 0, st>>>(codes, nch, o); break;
            case 4: k_pack_canonical<4><<<grid, threads, 0, st>>>(codes, nch, o); break;
            case 5: k_pack_canonical<5><<<grid, threads, 0, st>>>(codes, nch, o); break;
            default: k_pack_canonical<6><<<grid, threads, 0, st>>>(codes, nch, o); break;
        }
    } else {
        const int64_t nw = n * k * bits / 32;
        if (nw == 0) return LBQ_OK;
        const int grid = (int)std::min<int64_t>(ceil_div(nw, threads), gmax);
        auto* o = (uint32_t*)packed;
        switch (bits) {
            case 2: k_kernel_layout<2, false><<<grid, threads, 0, st>>>(codes, o, n, k, nullptr); break;
            case 3: k_kernel_layout<3, false><<<grid, threads, 0, st>>>(codes, o, n, k, nullptr); break;
            case 4: k_kernel_layout<4, false><<<grid, threads, 0, st>>>(codes, o, n, k, nullptr); break;
            case 5: k_kernel_layout<5, false><<<grid, threads, 0, st>>>(codes, o, n, k, nullptr); break;
            default: k_kernel_layout<6, false><<<grid, threads, 0, st>>>(codes, o, n, k, nullptr); break;
        }
    }
    return launch_status();
}

lbq_status launch_unpack(const void* packed, int64_t n, int64_t k, int bits, lbq_layout layout, uint8_t* codes,
                         cudaStream_t st) {
    const int threads = 256;
    const int gmax = sm_count() * 16;
    if (layout == LBQ_LAYOUT_CANONICAL) {
        const int64_t nch = n * k / 32;
        if (nch == 0) return LBQ_OK;
        const int grid = (int)std::min<int64_t>(ceil_div(nch, threads), gmax);
        auto* in = (const uint32_t*)packed;
        switch (bits) {
            case 2: k_unpack_canonical<2><<<grid, threads, 0, st>>>(in, nch, codes); break;
            case 3: k_unpack_canonical<3><<<grid, threads, 0, st>>>(in, nch, codes); break;
            case 4: k_unpack_canonical<4><<<grid, threads, 0, st>>>(in, nch, codes); break;
            case 5: k_unpack_canonical<5><<<grid, threads, 0, st>>>(in, nch, codes); break;
            default: k_unpack_canonical<6><<<grid, threads, 0, st>>>(in, nch, codes); break;
        }
    } else {
        const int64_t nw = n * k * bits / 32;
        if (nw == 0) return LBQ_OK;
        if (cudaMemsetAsync(codes, 0, (size_t)(n * k), st) != cudaSuccess) return LBQ_ERR_CUDA;
        const int grid = (int)std::min<int64_t>(ceil_div(nw, threads), gmax);
        auto* w = (uint32_t*)packed;
        switch (bits) {
            case 2: k_kernel_layout<2, true><<<grid, threads, 0, st>>>(nullptr, w, n, k, codes); break;
            case 3: k_kernel_layout<3, true><<<grid, threads, 0, st>>>(nullptr, w, n, k, codes); break;
            case 4: k_kernel_layout<4, true><<<grid, threads, 0, st>>>(nullptr, w, n, k, codes); break;
            case 5: k_kernel_layout<5, true><<<grid, threads, 0, st>>>(nullptr, w, n, k, codes); break;
            default: k_kernel_layout<6, true><<<grid, threads, 0, st>>>(nullptr, w, n, k, codes); break;
        }
    }
    return launch_status();
}

// ---------------------------------------------------------------- signs
// +-1 int8 rows -> canonical words: one thread per output word (32 bytes in).
__global__ void k_pack_signs_canonical(const int8_t* __restrict__ pm1, int64_t nwords, uint32_t* __restrict__ out) {
    for (int64_t wi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; wi < nwords;
         wi += (int64_t)gridDim.x * blockDim.x) {
        const uint4 a = *reinterpret_cast<const uint4*>(pm1 + wi * 32);
        const uint4 b = *reinterpret_cast<const uint4*>(pm1 + wi * 32 + 16);
        const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 32; j++) {
            const int8_t s = (int8_t)((v[j / 4] >> (8 * (j % 4))) & 0xFF);
            word |= (s > 0 ? 1u : 0u) << j;
        }
        out[wi] = word;
    }
}

// canonical words -> kernel sign layout: one thread per output word.
// Output word (tile T, superblock S, lane L = 4g + c, word widx): row 16T + g + 8*(widx&1);
// bit 8j + p is column 256S + 32p + 16*(widx>>1) + 4c + j (zero beyond cols).
__global__ void k_repack_signs(const uint32_t* __restrict__ canon, int64_t rows, int64_t cols, int64_t cols_pad,
                               uint32_t* __restrict__ out) {
    const int64_t nwords = rows * cols_pad / 32;
    const int64_t wpr = cols / 32;
    const int64_t nsb = cols_pad / 256;
    for (int64_t wi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; wi < nwords;
         wi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = wi / 128;  // 512-byte block
        const int64_t T = blk / nsb, S = blk % nsb;
        const int inb = (int)(wi % 128);
        const int L = inb / 4, widx = inb % 4;
        const int g = L / 4, c = L % 4;
        const int64_t row = T * 16 + g + 8 * (widx & 1);
        const int half = widx >> 1;
        uint32_t word = 0;
#pragma unroll
        for (int p = 0; p < 8; p++) {
            const int64_t cw = S * 8 + p;  // canonical word holding columns 256S + 32p ..
            const uint32_t src = (cw < wpr) ? canon[row * wpr + cw] : 0u;
            const uint32_t nib = (src >> (16 * half + 4 * c)) & 0xFu;
#pragma unroll
            for (int j = 0; j < 4; j++) word |= ((nib >> j) & 1u) << (8 * j + p);
        }
        out[wi] = word;
    }
}

// +-1 int8 rows -> kernel sign layout directly (same word geometry as k_repack_signs).
__global__ void k_pack_signs_kernel(const int8_t* __restrict__ pm1, int64_t rows, int64_t cols, int64_t cols_pad,
                                    uint32_t* __restrict__ out) {
    const int64_t nwords = rows * cols_pad / 32;
    const int64_t nsb = cols_pad / 256;
    for (int64_t wi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; wi < nwords;
         wi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = wi / 128;
        const int64_t T = blk / nsb, S = blk % nsb;
        const int inb = (int)(wi % 128);
        const int L = inb / 4, widx = inb % 4;
        const int g = L / 4, c = L % 4;
        const int64_t row = T * 16 + g + 8 * (widx & 1);
        const int half = widx >> 1;
        uint32_t word = 0;
        for (int p = 0; p < 8; p++) {
            const int64_t col0 = S * 256 + 32 * p + 16 * half + 4 * c;
            if (col0 < cols) {
                const uint32_t v = *reinterpret_cast<const uint32_t*>(pm1 + row * cols + col0);
#pragma unroll
                for (int j = 0; j < 4; j++)
                    word |= (((int8_t)((v >> (8 * j)) & 0xFF) > 0) ? 1u : 0u) << (8 * j + p);
            }
        }
        out[wi] = word;
    }
}

lbq_status launch_pack_signs(const int8_t* pm1, int64_t rows, int64_t cols, lbq_layout layout, void* out,
                             cudaStream_t st) {
    const int threads = 256;
    const int gmax = sm_count() * 16;
    if (layout == LBQ_LAYOUT_CANONICAL) {
        const int64_t nw = rows * cols / 32;
        if (nw == 0) return LBQ_OK;
        const int grid = (int)std::min<int64_t>(ceil_div(nw, threads), gmax);
        k_pack_signs_canonical<<<grid, threads, 0, st>>>(pm1, nw, (uint32_t*)out);
    } else {
        const int64_t cp = sign_cols_pad(cols);
        const int64_t nw = rows * cp / 32;
        if (nw == 0) return LBQ_OK;
        const int grid = (int)std::min<int64_t>(ceil_div(nw, threads), gmax);
        k_pack_signs_kernel<<<grid, threads, 0, st>>>(pm1, rows, cols, cp, (uint32_t*)out);
    }
    return launch_status();
}

lbq_status launch_repack_signs(const uint32_t* canon, int64_t rows, int64_t cols, void* out, cudaStream_t st) {
    const int threads = 256;
    const int64_t cp = sign_cols_pad(cols);
    const int64_t nw = rows * cp / 32;
    if (nw == 0) return LBQ_OK;
    const int grid = (int)std::min<int64_t>(ceil_div(nw, threads), (int64_t)sm_count() * 16);
    k_repack_signs<<<grid, threads, 0, st>>>(canon, rows, cols, cp, (uint32_t*)out);
    return launch_status();
}

}  // namespace lbq
