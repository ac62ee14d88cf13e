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
// Fast path (LBQ_LAYOUT_KERNEL):
//  * each warp owns a 16-row tile; per 512-byte block every lane issues ONE 128-bit
//    streaming load that already holds its m16n8k16 A-fragment codes for two rows;
//  * codes become exact fp16/bf16 values (q - z) with one LOP3 per pair (magic
//    exponent 1024 / 128) and one half2 subtraction; the tensor core multiplies them
//    by the fp16/bf16 activations with exact products and fp32 accumulation;
//  * the group scale is applied in fp32 once per group (4 FFMA per lane);
//  * work is split "stream-K" style: every CTA gets the same number of
//    (128-row block, k-superblock) units, so all SMs finish together; a row block
//    split between CTAs is reduced by the last CTA to arrive (atomic ticket, fixed
//    summation order => deterministic), which also resets the ticket.
// Canonical path: one warp per row, CUDA-core fp32 FMA (correctness path for any shape).
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

constexpr int kGemvWarps = 8;                 // warps per CTA = 16-row tiles per row block
constexpr int kRowBlock = 16 * kGemvWarps;    // rows per CTA work unit

// ------------------------------------------------------------------ A-fragment builder
template <int B, bool BF16>
struct FragDeq {
    using G = GroupGeom<B>;
    static constexpr uint32_t MAGIC = BF16 ? 0x43004300u : 0x64006400u;   // 128.0 / 1024.0
    static constexpr uint32_t MASK0 = ((1u << G::W0) - 1u) * 0x00010001u;
    static constexpr uint32_t MASK1 = (((1u << (G::W1 > 0 ? G::W1 : 1)) - 1u) << G::W0) * 0x00010001u;
    static constexpr int P0 = 16 / G::W0;
    static constexpr int P1 = G::W1 > 0 ? 16 / G::W1 : 1;

    // half2 of (MAGIC + q) for row half `upper` (0: row g, 1: row g+8), sub-slot pair `sub`
    template <int SIG, int UPPER, int SUB>
    __device__ __forceinline__ static uint32_t pair(const uint4 (&blk)[G::NBLK]) {
        constexpr int b0 = SIG / P0, sb0 = SIG % P0;
        constexpr bool second0 = sb0 >= P0 / 2;
        constexpr int pi0 = 2 * (sb0 % (P0 / 2)) + SUB;
        const uint4& v0 = blk[b0];
        const uint32_t w0 = second0 ? (UPPER ? v0.w : v0.z) : (UPPER ? v0.y : v0.x);
        uint32_t h = and_or(shift_right_signed<G::W0 * pi0>(w0), MASK0, MAGIC);
        if constexpr (G::W1 > 0) {
            constexpr int b1 = G::NB0 + SIG / P1, sb1 = SIG % P1;
            constexpr bool second1 = sb1 >= P1 / 2;
            constexpr int pi1 = 2 * (sb1 % (P1 / 2)) + SUB;
            const uint4& v1 = blk[b1];
            const uint32_t w1 = second1 ? (UPPER ? v1.w : v1.z) : (UPPER ? v1.y : v1.x);
            h = and_or(shift_right_signed<G::W1 * pi1 - G::W0>(w1), MASK1, h);
        }
        return h;
    }
};

template <bool BF16>
__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
    if constexpr (BF16) return hsub2_bf16(a, b);
    else return hsub2_f16(a, b);
}

// (MAGIC + z) replicated in both halves, from the fp16 zero-point bits.
template <bool BF16>
__device__ __forceinline__ uint32_t zero_sub(uint16_t zbits) {
    const float zf = __half2float(__ushort_as_half(zbits));
    uint16_t v;
    if constexpr (BF16) v = __bfloat16_as_ushort(__float2bfloat16_rn(128.0f + zf));
    else v = __half_as_ushort(__float2half_rn(1024.0f + zf));
    return (uint32_t)v | ((uint32_t)v << 16);
}

// Load NG consecutive fp16 values (NG in 1,2,4,8) as packed halves.
template <int NG>
__device__ __forceinline__ void load_halves(const uint16_t* p, uint32_t (&d)[(NG + 1) / 2]) {
    if constexpr (NG == 1) d[0] = ldg_u16(p);
    else if constexpr (NG == 2) d[0] = ldg_u32(p);
    else if constexpr (NG == 4) { uint2 v = ldg_u64(p); d[0] = v.x; d[1] = v.y; }
    else { uint4 v = ldg_u128(p); d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w; }
}
template <int NG>
__device__ __forceinline__ uint16_t half_at(const uint32_t (&d)[(NG + 1) / 2], int i) {
    return (uint16_t)(d[i / 2] >> (16 * (i & 1)));
}

// ------------------------------------------------------------------ fast kernel
template <int B, int GROUP, int NT, bool BF16, int PF>
__global__ void __launch_bounds__(kGemvWarps * 32)
k_gemv_group_frag(const uint16_t* __restrict__ x, int M, const uint8_t* __restrict__ packed,
                  const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros, int64_t n, int64_t k,
                  uint16_t* __restrict__ y, float* __restrict__ partials, unsigned* __restrict__ counters,
                  int maxc) {
    using G = GroupGeom<B>;
    using D = FragDeq<B, BF16>;
    constexpr int SB = G::SB;
    constexpr int F = GROUP < SB ? GROUP : SB;        // k covered by one scale application
    constexpr int NG = SB / F;                         // scale applications per superblock
    constexpr int NGW = (NG + 1) / 2;
    constexpr int SPF = F / 16;                        // slices per scale application

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int64_t KSB = k / SB;
    const int64_t G_per_row = k / GROUP;
    const int64_t n_tiles = n / 16;
    const int64_t n_rb = ceil_div(n_tiles, kGemvWarps);
    const int64_t S_total = n_rb * KSB;
    const int64_t NC = gridDim.x;
    const int64_t u_begin = (int64_t)blockIdx.x * S_total / NC;
    const int64_t u_end = ((int64_t)blockIdx.x + 1) * S_total / NC;

    for (int64_t u0 = u_begin; u0 < u_end;) {
        const int64_t rb = u0 / KSB;
        const int64_t ks0 = u0 % KSB;
        const int64_t ks1 = min(KSB, ks0 + (u_end - u0));
        u0 += ks1 - ks0;
        const int64_t tile = rb * kGemvWarps + warp;
        if (tile >= n_tiles) continue;                 // warp-uniform; no block-level syncs below

        const int64_t row_g = tile * 16 + g;
        const uint8_t* tile_ptr = packed + (tile * KSB) * G::SB_BYTES + lane * 16;
        const uint16_t* s_g = scales + row_g * G_per_row;
        const uint16_t* z_g = zeros + row_g * G_per_row;
        const uint16_t* s_g8 = s_g + 8 * G_per_row;
        const uint16_t* z_g8 = z_g + 8 * G_per_row;

        float acc[NT][4];
        float cg[NT][4];
#pragma unroll
        for (int t = 0; t < NT; t++)
#pragma unroll
            for (int e = 0; e < 4; e++) acc[t][e] = cg[t][e] = 0.0f;

        // token rows of x this lane feeds into the B fragment (zero beyond M)
        const uint16_t* xrow[NT];
        bool xval[NT];
#pragma unroll
        for (int t = 0; t < NT; t++) {
            const int tok = 8 * t + g;
            xval[t] = tok < M;
            xrow[t] = x + (int64_t)(xval[t] ? tok : 0) * k + 2 * c;
        }

        uint4 wbuf[PF][G::NBLK];
        uint32_t sbuf[PF][4][NGW];
        auto load_stage = [&](int st, int64_t ks) {
            const uint8_t* p = tile_ptr + ks * G::SB_BYTES;
#pragma unroll
            for (int b = 0; b < G::NBLK; b++) wbuf[st][b] = ldg_stream(p + b * 512);
            const int64_t j0 = (ks * SB) / GROUP;
            load_halves<NG>(s_g + j0, sbuf[st][0]);
            load_halves<NG>(z_g + j0, sbuf[st][1]);
            load_halves<NG>(s_g8 + j0, sbuf[st][2]);
            load_halves<NG>(z_g8 + j0, sbuf[st][3]);
        };
#pragma unroll
        for (int st = 0; st < PF; st++)
            if (ks0 + st < ks1) load_stage(st, ks0 + st);

        for (int64_t base = ks0; base < ks1; base += PF) {
#pragma unroll
            for (int st = 0; st < PF; st++) {
                const int64_t ks = base + st;
                if (ks < ks1) {
                    const int64_t kbase = ks * SB;
                    static_for<0, NG>([&](auto gi_c) {
                        constexpr int gi = decltype(gi_c)::value;
                        const uint32_t zs_g = zero_sub<BF16>(half_at<NG>(sbuf[st][1], gi));
                        const uint32_t zs_g8 = zero_sub<BF16>(half_at<NG>(sbuf[st][3], gi));
                        static_for<0, SPF>([&](auto sl_c) {
                            constexpr int sig = gi * SPF + decltype(sl_c)::value;
                            uint32_t a[4];
                            a[0] = hsub2<BF16>(D::template pair<sig, 0, 0>(wbuf[st]), zs_g);
                            a[1] = hsub2<BF16>(D::template pair<sig, 1, 0>(wbuf[st]), zs_g8);
                            a[2] = hsub2<BF16>(D::template pair<sig, 0, 1>(wbuf[st]), zs_g);
                            a[3] = hsub2<BF16>(D::template pair<sig, 1, 1>(wbuf[st]), zs_g8);
                            const int64_t kk = kbase + 16 * sig;
#pragma unroll
                            for (int t = 0; t < NT; t++) {
                                uint32_t b0 = 0, b1 = 0;
                                if (xval[t]) {
                                    b0 = ldg_u32(xrow[t] + kk);
                                    b1 = ldg_u32(xrow[t] + kk + 8);
                                }
                                mma_16816<BF16>(cg[t], a, b0, b1);
                            }
                        });
                        const float sg = __half2float(__ushort_as_half(half_at<NG>(sbuf[st][0], gi)));
                        const float sg8 = __half2float(__ushort_as_half(half_at<NG>(sbuf[st][2], gi)));
#pragma unroll
                        for (int t = 0; t < NT; t++) {
                            acc[t][0] = fmaf(sg, cg[t][0], acc[t][0]);
                            acc[t][1] = fmaf(sg, cg[t][1], acc[t][1]);
                            acc[t][2] = fmaf(sg8, cg[t][2], acc[t][2]);
                            acc[t][3] = fmaf(sg8, cg[t][3], acc[t][3]);
                            cg[t][0] = cg[t][1] = cg[t][2] = cg[t][3] = 0.0f;
                        }
                    });
                    if (ks + PF < ks1) load_stage(st, ks + PF);
                }
            }
        }

        // ---- epilogue: direct store, or partial + last-arriver reduction
        const bool full = (ks0 == 0) && (ks1 == KSB);
        if (full) {
#pragma unroll
            for (int t = 0; t < NT; t++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int tok = 8 * t + 2 * c + (e & 1);
                    const int64_t row = row_g + 8 * (e >> 1);
                    if (tok < M) y[(int64_t)tok * n + row] = from_f32<false>(acc[t][e]);
                }
        } else {
            // contributors of this row block: CTAs owning its first and last superblock
            const int64_t first_u = rb * KSB, last_u = rb * KSB + KSB - 1;
            const int64_t own_first = ((first_u + 1) * NC - 1) / S_total;
            const int64_t own_last = ((last_u + 1) * NC - 1) / S_total;
            const int count = (int)(own_last - own_first + 1);
            const int slot = (int)(blockIdx.x - own_first);
            float* pslot = partials + ((tile * maxc) + slot) * (int64_t)(16 * M);
#pragma unroll
            for (int t = 0; t < NT; t++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int tok = 8 * t + 2 * c + (e & 1);
                    const int r = g + 8 * (e >> 1);
                    if (tok < M) __stcg(pslot + tok * 16 + r, acc[t][e]);
                }
            __syncwarp();
            unsigned old = 0;
            if (lane == 0) {
                __threadfence();
                old = atomicAdd(counters + tile, 1u);
            }
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old == (unsigned)(count - 1)) {
                __threadfence();
                const float* p0 = partials + (tile * maxc) * (int64_t)(16 * M);
                for (int e = lane; e < 16 * M; e += 32) {
                    float s = 0.0f;
                    for (int sl = 0; sl < count; sl++) s += __ldcg(p0 + sl * (int64_t)(16 * M) + e);
                    const int tok = e / 16, r = e % 16;
                    y[(int64_t)tok * n + tile * 16 + r] = from_f32<false>(s);
                }
                if (lane == 0) counters[tile] = 0u;
            }
        }
    }
}

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
struct GemvPlan {
    int64_t n_rb, KSB, S_total;
    int NC;
    int maxc;
    size_t counters_bytes, partial_bytes;
};

static constexpr int kCtasPerSm = 2;

static GemvPlan plan_frag(int64_t M, int64_t n, int64_t k, int bits) {
    GemvPlan p{};
    const int64_t SB = group_superblock(bits);
    const int64_t n_tiles = n / 16;
    p.n_rb = ceil_div(n_tiles, kGemvWarps);
    p.KSB = k / SB;
    p.S_total = p.n_rb * p.KSB;
    p.NC = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)sm_count() * kCtasPerSm, p.S_total));
    p.maxc = (int)(p.NC / std::max<int64_t>(p.n_rb, 1) + 2);
    p.counters_bytes = kCounterBytes;
    p.partial_bytes = (size_t)(n_tiles * p.maxc * 16 * M * 4);
    return p;
}

size_t gemv_group_ws_bytes(int64_t M, int64_t n, int64_t k, int bits, lbq_layout layout) {
    if (layout != LBQ_LAYOUT_KERNEL) return 0;
    const GemvPlan p = plan_frag(M, n, k, bits);
    return p.counters_bytes + p.partial_bytes;
}

template <int B, int GROUP, bool BF16>
static void launch_frag_bg(int NT, int grid, cudaStream_t st, const uint16_t* x, int M, const uint8_t* packed,
                           const uint16_t* s, const uint16_t* z, int64_t n, int64_t k, uint16_t* y, float* part,
                           unsigned* cnt, int maxc) {
    constexpr int NBLK = GroupGeom<B>::NBLK;
    constexpr int PF = NBLK == 1 ? 4 : (NBLK <= 3 ? 2 : 1);
    if (NT == 1)
        k_gemv_group_frag<B, GROUP, 1, BF16, PF><<<grid, kGemvWarps * 32, 0, st>>>(x, M, packed, s, z, n, k, y,
                                                                                 part, cnt, maxc);
    else
        k_gemv_group_frag<B, GROUP, 2, BF16, PF><<<grid, kGemvWarps * 32, 0, st>>>(x, M, packed, s, z, n, k, y,
                                                                                 part, cnt, maxc);
}

template <int B, bool BF16>
static void launch_frag_b(int group, int NT, int grid, cudaStream_t st, const uint16_t* x, int M,
                          const uint8_t* packed, const uint16_t* s, const uint16_t* z, int64_t n, int64_t k,
                          uint16_t* y, float* part, unsigned* cnt, int maxc) {
    if (group == 32) launch_frag_bg<B, 32, BF16>(NT, grid, st, x, M, packed, s, z, n, k, y, part, cnt, maxc);
    else if (group == 64) launch_frag_bg<B, 64, BF16>(NT, grid, st, x, M, packed, s, z, n, k, y, part, cnt, maxc);
    else launch_frag_bg<B, 128, BF16>(NT, grid, st, x, M, packed, s, z, n, k, y, part, cnt, maxc);
}

template <bool BF16>
static void launch_frag(int bits, int group, int NT, int grid, cudaStream_t st, const uint16_t* x, int M,
                        const uint8_t* packed, const uint16_t* s, const uint16_t* z, int64_t n, int64_t k,
                        uint16_t* y, float* part, unsigned* cnt, int maxc) {
    switch (bits) {
        case 2: launch_frag_b<2, BF16>(group, NT, grid, st, x, M, packed, s, z, n, k, y, part, cnt, maxc); break;
        case 3: launch_frag_b<3, BF16>(group, NT, grid, st, x, M, packed, s, z, n, k, y, part, cnt, maxc); break;
        case 4: launch_frag_b<4, BF16>(group, NT, grid, st, x, M, packed, s, z, n, k, y, part, cnt, maxc); break;
        case 5: launch_frag_b<5, BF16>(group, NT, grid, st, x, M, packed, s, z, n, k, y, part, cnt, maxc); break;
        default: launch_frag_b<6, BF16>(group, NT, grid, st, x, M, packed, s, z, n, k, y, part, cnt, maxc); break;
    }
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
    const GemvPlan p = plan_frag(M, n, k, bits);
    if (ws_bytes < p.counters_bytes + p.partial_bytes || (ws == nullptr && p.partial_bytes > 0))
        return LBQ_ERR_WORKSPACE;
    auto* cnt = (unsigned*)ws;
    auto* part = (float*)((char*)ws + p.counters_bytes);
    const int NT = M <= 8 ? 1 : 2;
    if (bf16) launch_frag<true>(bits, group, NT, p.NC, st, xp, (int)M, (const uint8_t*)packed, sp, zp, n, k, yp,
                                part, cnt, p.maxc);
    else launch_frag<false>(bits, group, NT, p.NC, st, xp, (int)M, (const uint8_t*)packed, sp, zp, n, k, yp, part,
                            cnt, p.maxc);
    return launch_status();
}

}  // namespace lbq
