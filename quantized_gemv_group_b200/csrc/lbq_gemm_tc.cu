// lbq_gemm_tc.cu -- batched GEMMs on tcgen05 tensor cores (sm_100a), M >= 64 tokens.
//
//   group codes:  y[m, i] = sum_k x[m, k] * s[i, k/g] * (q[i, k] - z[i, k/g])
//   +-1 signs:    the two stages of the binary low-rank form (end of this file)
//
// With many tokens one loaded weight serves all of them ("AirLLM corre un modelo 70B en
// una GPU de 4GB...", section "Es genuinamente excelente para trabajo batch offline"),
// and the product becomes a dense contraction worth the 5th-generation tensor cores.
// One CTA computes a 128-row x NT-token tile of y^T in tensor memory (TMEM):
//
//  * warps 2..9 (one per 16-row tile) each stream their tile's packed codes and its 16 x 8
//    scale and zero boxes, superblock by superblock, into a ring of their own with cp.async
//    (one 16-byte piece per lane and 512-byte block: the bulk-copy engine's throughput per
//    CTA follows the number of copies, plain async loads do not), expand them to fp16
//    weights w = fp16(s * (q - z)) for the 128 x 64 A piece, K-major with 128-byte swizzle,
//    and at the end read the fp32 accumulator back from TMEM and store y in fp16;
//  * warp 10 streams the activations x (fp16) in 64-wide k pieces through a 2-D tensor
//    map (TMA) with 128-byte swizzle, the K-major layout the tensor core reads;
//  * warp 1 allocates TMEM and one of its threads issues tcgen05.mma.kind::f16
//    (M = 128, N = NT, K = 16) from shared-memory descriptors; tcgen05.commit frees the
//    A and x buffers and finally signals the epilogue.
// A and B are both fp16 (kind::f16 takes one type for both): bf16 activations are first
// converted to fp16, exact for values in fp16's normal range.  The weights are rounded
// to fp16 once (relative error 2^-11 per weight).  Every wait is bounded: on expiry the
// kernel records kErrTimeout, drains its tensor-core work, frees TMEM and returns.
#include <cuda.h>
#include <cstring>
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

constexpr int kGemmDq = 8;                         // dequant warps, one per 16-row tile
constexpr int kGemmDq0 = 2;                        // first dequant warp
constexpr int kGemmThreads = (3 + kGemmDq) * 32;   // codes producer, MMA, dequant x8, x producer
constexpr int kXWarp = 2 + kGemmDq;
constexpr int kPiece = 64;                         // k per A piece = one 128-byte swizzle row
constexpr int kWarpRing = 3;                       // superblocks in flight per dequant warp
constexpr int kMaxXStages = 8;                     // activation ring depth: as deep as shared memory allows
constexpr int kAStages = 4;                        // A pieces between dequant and tensor core
constexpr int kGScaleBox = 8;                      // groups per scale/zero box
constexpr int kAStageBytes = 128 * kPiece * 2;     // 16 KB

// B = 2..6: group codes with scale/zero boxes; B = 1: a +-1 sign matrix (no scales).
// Each dequant warp owns a ring of kWarpRing slots: its tile's 512 * B bytes of one
// superblock, then (group codes) the tile's 16 rows x 8 groups of scales and of zeros.
struct GemmSmem {
    int x, a, codes, slot, bars, bytes;
    __host__ __device__ GemmSmem(int B, int NT, int XS) {
        x = 0;                                           // every stage 1024-byte aligned
        a = x + XS * NT * 128;
        codes = a + kAStages * kAStageBytes;
        slot = 512 * B + (B > 1 ? 2 * 16 * kGScaleBox * 2 : 0);
        bars = codes + kGemmDq * kWarpRing * slot;
        bytes = bars + 512;
    }
};

struct GemmArgs {
    CUtensorMap mx;        // B operand (fp16) [M x k], box 64 x NT, 128-byte swizzle
    const uint16_t* scales;    // group codes: [n x ngroups] fp16 scales and zeros
    const uint16_t* zeros;
    int64_t ngroups;
    const uint8_t* packed; // A in its kernel layout: 16-row tiles x 256-wide k superblocks
    const uint16_t* rowscale;  // optional fp16 factor per output row (signs: s1), else null
    uint16_t* y;           // fp16 [M x ldy]
    int64_t n, ksb, M, ldy;    // rows of A, k superblocks, tokens, output row stride
    unsigned* err;
    float* partials;           // split-K: [tile][split][128][NT] fp32 (splits > 1)
    unsigned* counters;        // split-K tickets, one per output tile (zero between calls)
    int xs, splits;            // activation ring depth, k slices per output tile
};

// Byte offset of the 16-byte chunk (row r, k-octet k8) in a 128-row x 64-k fp16 piece,
// K-major with 128-byte swizzle: 8-row atoms of 1024 bytes, chunk index XOR (r mod 8).
__device__ __forceinline__ uint32_t a_sw128(int r, int k8) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((k8 ^ (r & 7)) << 4));
}

// Half2 holding (1024 + code(j), 1024 + code(j + 2)) for the codes whose low bits sit at
// bit `sh0` of w0 (bytes j and j+2) and high bits at `sh1` of w1.
template <int W0, int W1>
__device__ __forceinline__ uint32_t code_pair_f16(uint32_t w0, uint32_t w1, int sh0, int sh1) {
    constexpr uint32_t m0 = ((1u << W0) - 1u) * 0x00010001u;
    uint32_t v = ((w0 >> sh0) & m0) | 0x64006400u;
    if constexpr (W1 > 0) {
        constexpr uint32_t m1 = ((1u << W1) - 1u) * 0x00010001u;
        v |= ((w1 >> sh1) & m1) << W0;
    }
    return v;
}

// Eight consecutive-k weights (one 16-byte A chunk) from one octet of a lane's codes:
// w0/w1 hold the octet's plane words, o0/o1 its slot inside them.
template <int W0, int W1>
__device__ __forceinline__ uint4 dequant_octet(uint32_t w0, uint32_t w1, int o0, int o1, uint32_t zz2, uint32_t ss2) {
    uint32_t pr[4];
#pragma unroll
    for (int jp = 0; jp < 2; jp++) {
        const uint32_t h0 = code_pair_f16<W0, W1>(w0, w1, 8 * jp + 2 * W0 * o0, 8 * jp + 2 * W1 * o1);
        const uint32_t h1 = code_pair_f16<W0, W1>(w0, w1, 8 * jp + 2 * W0 * o0 + W0, 8 * jp + 2 * W1 * o1 + W1);
        pr[jp] = __byte_perm(h0, h1, 0x5410);        // codes 2j, 2j+1 with j = jp
        pr[jp + 2] = __byte_perm(h0, h1, 0x7632);    // j = jp + 2
    }
    uint4 r;
    uint32_t* rr = &r.x;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        // (1024 + q) - (1024 + z) is exact in fp16; one rounding in the product with s.
        const __half2 d = __hsub2(*reinterpret_cast<const __half2*>(&pr[j]), *reinterpret_cast<const __half2*>(&zz2));
        const __half2 w = __hmul2(d, *reinterpret_cast<const __half2*>(&ss2));
        rr[j] = *reinterpret_cast<const uint32_t*>(&w);
    }
    return r;
}

// Eight fp16 +-1 values from bit p of each byte of two sign words (bit 1 = +1): byte
// 0xBC - 0x80 * bit is the high byte of -1.0 / +1.0, and a byte permute places it.
__device__ __forceinline__ uint4 signs_octet(uint32_t wa, uint32_t wb, int p) {
    const uint32_t xa = 0xBCBCBCBCu - ((wa >> p) & 0x01010101u) * 0x80u;
    const uint32_t xb = 0xBCBCBCBCu - ((wb >> p) & 0x01010101u) * 0x80u;
    return make_uint4(__byte_perm(xa, 0, 0x1404), __byte_perm(xa, 0, 0x3424), __byte_perm(xb, 0, 0x1404),
                      __byte_perm(xb, 0, 0x3424));
}

template <int B, int GROUP, int NT>
__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm_group_tc05(const __grid_constant__ GemmArgs a) {
    constexpr bool kSigns = (B == 1);
    using G = GroupGeom<kSigns ? 4 : B>;
    constexpr int W0 = G::W0, W1 = G::W1;
    constexpr uint32_t kTmemCols = NT < 32 ? 32 : NT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int XS = a.xs;
    const GemmSmem S(B, NT, XS);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S.bars);
    // x_full[8] x_empty[8] a_full[4] a_empty[4] d_full | tmem address | abort flag | split
    // ticket result
    constexpr int kXb = kMaxXStages, kAb = kAStages;
    const uint32_t x_full0 = smem_u32(&bars[0]), x_empty0 = smem_u32(&bars[kXb]);
    const uint32_t a_full0 = smem_u32(&bars[2 * kXb]), a_empty0 = smem_u32(&bars[2 * kXb + kAb]);
    const uint32_t d_full = smem_u32(&bars[2 * kXb + 2 * kAb]);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[2 * kXb + 2 * kAb + 1]);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(&bars[2 * kXb + 2 * kAb + 2]);
    volatile int* last_flag = reinterpret_cast<volatile int*>(&bars[2 * kXb + 2 * kAb + 3]);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_tt = (a.M + NT - 1) / NT;
    const int splits = a.splits;
    const int64_t tile_id = blockIdx.x / splits;      // output tile (row block, token tile)
    const int ks = (int)(blockIdx.x % splits);        // k slice of this CTA
    const int64_t rb = tile_id / n_tt, tt = tile_id % n_tt;
    const int64_t sb0 = ks * a.ksb / splits, sb1 = (ks + 1) * a.ksb / splits;
    const int64_t KSB = sb1 - sb0;                    // superblocks of this CTA
    const int64_t n_pieces = KSB * (256 / kPiece);
    unsigned* err = a.err;

    if (threadIdx.x == 0) {
        for (int i = 0; i < XS; i++) {
            mbar_init(x_full0 + 8 * i, 1);
            mbar_init(x_empty0 + 8 * i, 1);
        }
        for (int i = 0; i < kAStages; i++) {
            mbar_init(a_full0 + 8 * i, kGemmDq);
            mbar_init(a_empty0 + 8 * i, 1);
        }
        mbar_init(d_full, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;

    if (warp == 0) {
        // (idle: the dequant warps fetch their own codes, scales and zeros)
    } else if (warp == kXWarp) {
        // ------------------------------------------------------------ activation producer
        if (lane == 0) {
            // ring slot xs, and the parity of the slot's previous use (incremental, no divisions)
            int xs = 0;
            uint32_t xph = 1;
            const int np = (int)n_pieces, pk0 = (int)(sb0 * 4);
            for (int p = 0; p < np && !*abort_flag; p++) {
                if (p >= XS && !mbar_wait_bounded(x_empty0 + 8 * xs, xph, err)) {
                    *abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(x_full0 + 8 * xs, (uint32_t)(NT * 128));
                tma_load_2d(smem_u32(smem + S.x + xs * NT * 128), &a.mx, (pk0 + p) * kPiece, (int)(tt * NT),
                            x_full0 + 8 * xs);
                if (++xs == XS) {
                    xs = 0;
                    xph ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // kind::f16 instruction descriptor: D fp32, A/B fp16, both K-major, N = NT, M = 128.
            constexpr uint32_t idesc = (1u << 4) | ((uint32_t)(NT >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
            // ring slots and the parities to wait for (incremental: this thread is on the
            // critical path once the tensor core is the bound)
            int as = 0, xs = 0;
            uint32_t aph = 0, xph = 0;
            const int np = (int)n_pieces;
            for (int p = 0; p < np; p++) {
                if (*abort_flag || !mbar_wait_bounded(a_full0 + 8 * as, aph, err) ||
                    !mbar_wait_bounded(x_full0 + 8 * xs, xph, err)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + S.a + as * kAStageBytes);
                const uint32_t x_base = smem_u32(smem + S.x + xs * NT * 128);
#pragma unroll
                for (int kk = 0; kk < kPiece / 16; kk++) {
                    // 128-byte swizzle, K-major: 8-row atoms 1024 bytes apart; the k step of
                    // 16 fp16 advances the start address by 32 bytes inside the atom.
                    const uint64_t da = umma_smem_desc(a_base + kk * 32, 16, 1024, 2);
                    const uint64_t dx = umma_smem_desc(x_base + kk * 32, 16, 1024, 2);
                    umma_f16(tmem_d, da, dx, idesc, (p > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(a_empty0 + 8 * as);
                umma_commit(x_empty0 + 8 * xs);
                if (++as == kAStages) {
                    as = 0;
                    aph ^= 1u;
                }
                if (++xs == XS) {
                    xs = 0;
                    xph ^= 1u;
                }
            }
            umma_commit(d_full);
            // All issued MMAs must finish before TMEM is freed, on the error path too.
            mbar_wait_bounded(d_full, 0u, err, 1u << 26);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ dequant warps
        const int T = warp - 2;                         // 16-row tile inside the 128-row block
        const int g = lane >> 2, c = lane & 3;
        const int flip = g & 1;                         // store order that keeps 8-lane phases conflict-free
        constexpr int O0 = 4 / W0;
        constexpr int O1 = W1 > 0 ? 4 / W1 : 1;
        // This warp's ring: cp.async of its tile's superblock (one 16-byte piece per lane per
        // 512-byte plane block) and of 16 rows x 8 groups of scales and zeros (lane i: row
        // i mod 16 of the scales, i < 16, or of the zeros), kWarpRing superblocks ahead.
        uint8_t* cring = smem + S.codes + T * kWarpRing * S.slot;
        const bool tile_live = rb * 8 + T < a.n / 16;
        auto issue_ring = [&](int slot, int64_t sb) {
            if (!tile_live) return;
            uint8_t* dst = cring + slot * S.slot;
            const uint8_t* src = a.packed + ((rb * 8 + T) * a.ksb + sb0 + sb) * (int64_t)(512 * B) + 16 * lane;
#pragma unroll
            for (int i = 0; i < B; i++) cp_async_cg16(smem_u32(dst + 512 * i + 16 * lane), src + 512 * i);
            if constexpr (!kSigns) {
                const int r = lane & 15, arr = lane >> 4;
                const int64_t j0 = (((sb0 + sb) * 256) / GROUP) & ~(int64_t)7;
                const uint16_t* sp = (arr ? a.zeros : a.scales) + (rb * 128 + 16 * T + r) * a.ngroups + j0;
                cp_async_cg16(smem_u32(dst + 512 * B + arr * (16 * kGScaleBox * 2) + r * (kGScaleBox * 2)), sp);
            }
        };
#pragma unroll 1
        for (int i = 0; i < kWarpRing; i++) {
            if (i < KSB) issue_ring(i, i);
            cp_async_commit();
        }
        int ring_slot = 0;
        for (int64_t sb = 0; sb < KSB && !*abort_flag; sb++) {
            cp_async_wait<kWarpRing - 1>();
            __syncwarp();
            const uint8_t* st = cring + ring_slot * S.slot;
            if constexpr (kSigns) {
                // Sign layout: lane L = 4g + c holds words (row g, cols 4c..4c+3 of each
                // 32-column block p at bit 8j + p), (row g+8, same), (row g, cols 16 + ...),
                // (row g+8, cols 16 + ...).  The octet 8c..8c+7 of a block comes from lanes
                // 4g + 2(c mod 2) and 4g + 2(c mod 2) + 1, word u + 2(c / 2).
                const uint32_t* tw = reinterpret_cast<const uint32_t*>(st);
                const int la = 4 * g + 2 * (c & 1);
                uint32_t wa[2], wb[2];
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    wa[u] = tw[4 * la + u + 2 * (c >> 1)];
                    wb[u] = tw[4 * (la + 1) + u + 2 * (c >> 1)];
                }
                bool ok = true;
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const int64_t p = sb * 4 + q;
                    const int as = (int)(p % kAStages);
                    if (p >= kAStages &&
                        !mbar_wait_bounded(a_empty0 + 8 * as, (uint32_t)(((p / kAStages) - 1) & 1), err)) {
                        ok = false;
                        break;
                    }
                    uint8_t* abuf = smem + S.a + as * kAStageBytes;
#pragma unroll
                    for (int u = 0; u < 2; u++) {
                        const int row = 16 * T + g + 8 * u;
#pragma unroll
                        for (int i = 0; i < 2; i++) {
                            const int kl = i ^ flip;            // 32-column block 2q + kl of the superblock
                            sts128(smem_u32(abuf + a_sw128(row, 4 * kl + c)), signs_octet(wa[u], wb[u], 2 * q + kl));
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(a_full0 + 8 * as);
                }
                if (!ok) {
                    *abort_flag = 1;
                    break;
                }
                __syncwarp();
                if (sb + kWarpRing < KSB) issue_ring(ring_slot, sb + kWarpRing);
                cp_async_commit();
                ring_slot = ring_slot + 1 == kWarpRing ? 0 : ring_slot + 1;
                continue;
            }
            const uint8_t* tb = st + 16 * lane;
            const uint16_t* ss = reinterpret_cast<const uint16_t*>(st + 512 * B);   // [16 rows][8 groups]
            const uint16_t* zs = ss + 16 * kGScaleBox;
            const int jbase = (int)(((sb0 + sb) * 256) / GROUP) & ~7;
            uint4 pl0 = make_uint4(0, 0, 0, 0), pl1 = make_uint4(0, 0, 0, 0);
            bool ok = true;
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int64_t p = sb * 4 + q;
                const int as = (int)(p % kAStages);
                // Plane words of this lane: octet eta = 4q + 2kl + u lives in word eta / O.
                if (q % (4 / W0) == 0) pl0 = *reinterpret_cast<const uint4*>(tb + (q / (4 / W0)) * 512);
                if constexpr (W1 > 0)
                    if (q % (4 / W1) == 0) pl1 = *reinterpret_cast<const uint4*>(tb + 512 * W0 + (q / (4 / W1)) * 512);
                if (p >= kAStages &&
                    !mbar_wait_bounded(a_empty0 + 8 * as, (uint32_t)(((p / kAStages) - 1) & 1), err)) {
                    ok = false;
                    break;
                }
                uint8_t* abuf = smem + S.a + as * kAStageBytes;
                uint4 out[2][2];
#pragma unroll
                for (int kl = 0; kl < 2; kl++) {
                    const int jj = (int)(((sb0 + sb) * 256 + 64 * q + 32 * kl) / GROUP) - jbase;
#pragma unroll
                    for (int u = 0; u < 2; u++) {
                        const int eta = 4 * q + 2 * kl + u;
                        const int wi0 = (eta / O0) & 3, o0 = eta % O0;
                        const uint32_t* p0 = &pl0.x;
                        const uint32_t* p1 = &pl1.x;
                        const uint32_t w0 = p0[wi0];
                        uint32_t w1 = 0;
                        int o1 = 0;
                        if constexpr (W1 > 0) {
                            w1 = p1[(eta / O1) & 3];
                            o1 = eta % O1;
                        }
                        const int lrow = g + 8 * u;                   // row inside the warp's tile
                        const uint16_t sh = ss[lrow * kGScaleBox + jj];
                        const __half zh = __hadd(__ushort_as_half(zs[lrow * kGScaleBox + jj]), __float2half(1024.f));
                        const uint32_t zz2 = (uint32_t)__half_as_ushort(zh) * 0x00010001u;
                        const uint32_t ss2 = (uint32_t)sh * 0x00010001u;
                        out[u][kl] = dequant_octet<W0, W1>(w0, w1, o0, o1, zz2, ss2);
                    }
                }
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    const int row = 16 * T + g + 8 * u;
#pragma unroll
                    for (int i = 0; i < 2; i++) {
                        const int kl = i ^ flip;
                        const uint4 v = flip ? out[u][i ^ 1] : out[u][i];
                        sts128(smem_u32(abuf + a_sw128(row, 4 * kl + c)), v);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(a_full0 + 8 * as);
            }
            if (!ok) {
                *abort_flag = 1;
                break;
            }
            __syncwarp();
            if (sb + kWarpRing < KSB) issue_ring(ring_slot, sb + kWarpRing);
            cp_async_commit();
            ring_slot = ring_slot + 1 == kWarpRing ? 0 : ring_slot + 1;
        }
        cp_async_wait<0>();
        // ------------------------------------------------------------ epilogue
        // All eight warps take every named barrier (id 1) below, whatever happened before.
        if (!mbar_wait_bounded(d_full, 0u, err, 1u << 26)) *abort_flag = 1;
        named_barrier(1, kGemmDq * 32);
        const bool ok = !*abort_flag;
        tc_fence_after();
        const int quarter = warp & 3;                  // TMEM lanes this warp may access
        const int half = (warp - 2) >> 2;              // which half of the NT columns
        const int rloc = 32 * quarter + lane;          // row inside the 128-row block
        const int64_t row = rb * 128 + rloc;
        float rs = 1.0f;
        if (a.rowscale != nullptr && row < a.n) rs = __half2float(__ushort_as_half(a.rowscale[row]));
        if (splits == 1) {
            if (ok) {
#pragma unroll 1
                for (int c0 = half * (NT / 2); c0 < (half + 1) * (NT / 2); c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem_d + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0, v);
                    tmem_wait_ld();
                    if (row < a.n) {
#pragma unroll
                        for (int j = 0; j < 16; j++) {
                            const int64_t tok = tt * NT + c0 + j;
                            if (tok < a.M) a.y[tok * a.ldy + row] = from_f32<false>(__uint_as_float(v[j]) * rs);
                        }
                    }
                }
            }
        } else {
            // split-K: this slice's fp32 tile to its partial slot; the last slice to arrive
            // (ticket) adds the slots in slice order and stores y (deterministic)
            float* slot = a.partials + (tile_id * splits + ks) * (int64_t)(128 * NT);
            if (ok) {
#pragma unroll 1
                for (int c0 = half * (NT / 2); c0 < (half + 1) * (NT / 2); c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(tmem_d + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        __stcg(reinterpret_cast<float4*>(slot + rloc * NT + c0 + j),
                               make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                                           __uint_as_float(v[j + 3])));
                }
            }
            __threadfence();
            named_barrier(1, kGemmDq * 32);
            if (threadIdx.x == kGemmDq0 * 32) {
                // every slice takes its ticket, also after an error, so the counter returns to zero
                const unsigned old = atomicAdd(a.counters + tile_id, 1u);
                *last_flag = old == (unsigned)(splits - 1);
            }
            named_barrier(1, kGemmDq * 32);
            if (*last_flag) {
                __threadfence();
                const float* p0 = a.partials + tile_id * splits * (int64_t)(128 * NT);
                if (ok && row < a.n) {
#pragma unroll 1
                    for (int c0 = half * (NT / 2); c0 < (half + 1) * (NT / 2); c0 += 4) {
                        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int sl = 0; sl < splits; sl++) {
                            const float4 t = __ldcg(reinterpret_cast<const float4*>(p0 + sl * (int64_t)(128 * NT) +
                                                                                   rloc * NT + c0));
                            acc.x += t.x;
                            acc.y += t.y;
                            acc.z += t.z;
                            acc.w += t.w;
                        }
                        const float vv[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            const int64_t tok = tt * NT + c0 + j;
                            if (tok < a.M) a.y[tok * a.ldy + row] = from_f32<false>(vv[j] * rs);
                        }
                    }
                }
                if (threadIdx.x == kGemmDq0 * 32) a.counters[tile_id] = 0u;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_d, kTmemCols);
    }
}

// fp16 copy of the activations [M x k], optionally times a per-column fp16 factor
// (s2 of the binary form).  bf16 -> fp16 alone is exact in fp16's normal range.
template <bool BF16>
__global__ void k_to_f16(const uint16_t* __restrict__ in, const uint16_t* __restrict__ colscale, int64_t k,
                         uint16_t* __restrict__ out, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        float v = to_f32<BF16>(in[i]);
        if (colscale != nullptr) v *= __half2float(__ushort_as_half(colscale[i % k]));
        out[i] = __half_as_ushort(__float2half_rn(v));
    }
}

static lbq_status to_f16(const void* x, bool bf16, const void* colscale, int64_t M, int64_t k, void* out,
                         cudaStream_t st) {
    const int64_t cnt = M * k;
    const int grid = (int)std::min<int64_t>(ceil_div(cnt, (int64_t)256), (int64_t)sm_count() * 16);
    if (bf16)
        k_to_f16<true><<<grid, 256, 0, st>>>((const uint16_t*)x, (const uint16_t*)colscale, k, (uint16_t*)out, cnt);
    else
        k_to_f16<false><<<grid, 256, 0, st>>>((const uint16_t*)x, (const uint16_t*)colscale, k, (uint16_t*)out, cnt);
    return cudaGetLastError() == cudaSuccess ? LBQ_OK : LBQ_ERR_CUDA;
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn gemm_encode_fn() {
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

// Row-major [rows x cols] 16-bit matrix with row stride ld elements, box box_c (inner) x box_r.
static bool encode_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, uint32_t box_c,
                      uint32_t box_r, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = gemm_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    cuuint32_t box[2] = {box_c, box_r};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token tile: the smallest of 64 / 128 / 256 that holds M, 256 beyond.
static int gemm_nt(int64_t M) { return M <= 64 ? 64 : (M <= 128 ? 128 : 256); }

// Deepest activation ring (<= 8 stages) that fits the 227 KB of shared memory.
static int gemm_xs(int B, int NT) {
    int xs = kMaxXStages;
    while (xs > 2 && GemmSmem(B, NT, xs).bytes + 1024 > 227 * 1024) xs--;
    return xs;
}

// k slices per output tile.  Only grids smaller than one wave are split (each slice's fp32
// partial tile is written and read back once, which larger grids cannot repay): as many
// slices as keep the CTAs within one wave of the SMs, at most 8 and at least 4
// superblocks a slice.
static int gemm_splits(int64_t rows, int64_t M, int64_t ksb) {
    const int64_t tiles = ceil_div(rows, (int64_t)128) * ceil_div(M, (int64_t)gemm_nt(M));
    const int64_t sms = sm_count();
    if (tiles >= sms) return 1;
    int64_t s = sms / tiles;
    s = std::min<int64_t>(s, 8);
    s = std::min<int64_t>(s, std::max<int64_t>(1, ksb / 4));
    return (int)std::max<int64_t>(1, s);
}

static size_t gemm_partials_bytes(int64_t rows, int64_t M, int64_t ksb) {
    const int s = gemm_splits(rows, M, ksb);
    if (s == 1) return 0;
    const int64_t tiles = ceil_div(rows, (int64_t)128) * ceil_div(M, (int64_t)gemm_nt(M));
    return (size_t)(tiles * s * 128 * gemm_nt(M) * 4);
}

// counter header | fp16 copy of bf16 activations | split-K partials
size_t gemm_group_tc_ws_bytes(int64_t M, int64_t n, int64_t k) {
    return kCounterBytes + al256((size_t)(M * k * 2)) + gemm_partials_bytes(n, M, k / 256);
}

bool gemm_group_tc_supported(int64_t M, int64_t n, int64_t k, int bits, int group) {
    if (M < 64 || n % 16 != 0 || k % 256 != 0 || bits < 2 || bits > 6) return false;
    if (group != 32 && group != 64 && group != 128) return false;
    if ((k / group) % 8 != 0 || M > ((int64_t)1 << 31) || n > ((int64_t)1 << 31)) return false;
    if (ceil_div(n, (int64_t)128) * ceil_div(M, (int64_t)gemm_nt(M)) > kCounterBytes / 4) return false;
    return GemmSmem(bits, gemm_nt(M), 2).bytes + 1024 <= 227 * 1024;
}

template <int B, int GROUP, int NT>
static lbq_status launch_gemm_inst(const GemmArgs& args, int64_t grid, size_t smem, cudaStream_t st) {
    auto kern = k_gemm_group_tc05<B, GROUP, NT>;
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LBQ_ERR_CUDA;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return LBQ_ERR_CUDA;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    kern<<<(unsigned)grid, kGemmThreads, smem, st>>>(args);
    return launch_status();
}

template <int B, int NT>
static lbq_status launch_gemm_g(int group, const GemmArgs& args, int64_t grid, size_t smem, cudaStream_t st) {
    if constexpr (B == 1) {
        return launch_gemm_inst<1, 32, NT>(args, grid, smem, st);   // signs: no groups
    } else {
        if (group == 32) return launch_gemm_inst<B, 32, NT>(args, grid, smem, st);
        if (group == 64) return launch_gemm_inst<B, 64, NT>(args, grid, smem, st);
        return launch_gemm_inst<B, 128, NT>(args, grid, smem, st);
    }
}

template <int B>
static lbq_status launch_gemm_b(int group, GemmArgs& args, cudaStream_t st) {
    const int NT = gemm_nt(args.M);
    args.xs = gemm_xs(B, NT);
    args.splits = gemm_splits(args.n, args.M, args.ksb);
    const int64_t grid = ceil_div(args.n, (int64_t)128) * ceil_div(args.M, (int64_t)NT) * args.splits;
    const size_t smem = (size_t)GemmSmem(B, NT, args.xs).bytes + 1024;   // + room to align the base to 1024
    if (NT == 64) return launch_gemm_g<B, 64>(group, args, grid, smem, st);
    if (NT == 128) return launch_gemm_g<B, 128>(group, args, grid, smem, st);
    return launch_gemm_g<B, 256>(group, args, grid, smem, st);
}

lbq_status launch_gemm_group_tc(const void* x, bool bf16, int64_t M, const void* packed, const void* scales,
                                const void* zeros, int64_t n, int64_t k, int bits, int group, void* y, void* ws,
                                size_t ws_bytes, cudaStream_t st) {
    if (ws == nullptr || ws_bytes < gemm_group_tc_ws_bytes(M, n, k)) return LBQ_ERR_WORKSPACE;
    if (gemm_encode_fn() == nullptr) return LBQ_ERR_CUDA;
    const void* xf = x;
    if (bf16) {
        void* conv = (char*)ws + kCounterBytes;
        const lbq_status s = to_f16(x, true, nullptr, M, k, conv, st);
        if (s != LBQ_OK) return s;
        xf = conv;
    }
    GemmArgs args;
    memset(&args, 0, sizeof args);
    if (!encode_2d(&args.mx, xf, M, k, k, 64, (uint32_t)gemm_nt(M), CU_TENSOR_MAP_SWIZZLE_128B)) return LBQ_ERR_CUDA;
    args.scales = (const uint16_t*)scales;
    args.zeros = (const uint16_t*)zeros;
    args.ngroups = k / group;
    args.packed = (const uint8_t*)packed;
    args.rowscale = nullptr;
    args.y = (uint16_t*)y;
    args.n = n;
    args.ksb = k / 256;
    args.M = M;
    args.ldy = n;
    args.err = device_error_word();
    args.counters = (unsigned*)ws;
    args.partials = (float*)((char*)ws + kCounterBytes + al256((size_t)(M * k * 2)));
    switch (bits) {
        case 2: return launch_gemm_b<2>(group, args, st);
        case 3: return launch_gemm_b<3>(group, args, st);
        case 4: return launch_gemm_b<4>(group, args, st);
        case 5: return launch_gemm_b<5>(group, args, st);
        default: return launch_gemm_b<6>(group, args, st);
    }
}

// ------------------------------------------------------------------ binary low-rank GEMM
// y = s1 . U (V^T (s2 . x)) as two tensor-core GEMMs over the sign kernel layout
// ("70B en 4GB de VRAM: la compresion neural de 2026, es real?", section
// "1. NanoQuant", bullet "Formulacion"):
//   stage 1: t[m, j] = sum_i V^T[j, i] * fp16(s2[i] x[m, i])     rows r,     k = d_in
//   stage 2: y[m, i] = s1[i] * sum_j U[i, j] * t[m, j]           rows d_out, k = r
// t is kept in fp16 (11-bit significand) between the stages; the sign bits of the
// 256-column padding are 0 (-1) and meet zero-filled activation columns.
struct BinGemmWs {
    uint16_t* xs;      // fp16(s2 . x) [M x d_in]
    uint16_t* t;       // fp16 [M x ldt]
    float* partials;   // split-K partial tiles
    int64_t ldt;
    size_t bytes;
};

static BinGemmWs bin_gemm_ws(void* base, int64_t M, int64_t d_out, int64_t d_in, int64_t r) {
    BinGemmWs w{};
    const size_t xs_bytes = al256((size_t)(M * d_in * 2));
    w.ldt = sign_cols_pad(r);
    w.xs = (uint16_t*)((char*)base + kCounterBytes);
    w.t = (uint16_t*)((char*)base + kCounterBytes + xs_bytes);
    const size_t t_bytes = al256((size_t)(M * w.ldt * 2));
    w.partials = (float*)((char*)base + kCounterBytes + xs_bytes + t_bytes);
    // the stages run one after the other and share the partials region
    w.bytes = kCounterBytes + xs_bytes + t_bytes +
              std::max(gemm_partials_bytes(r, M, sign_cols_pad(d_in) / 256),
                       gemm_partials_bytes(d_out, M, sign_cols_pad(r) / 256));
    return w;
}

size_t gemm_binlr_tc_ws_bytes(int64_t M, int64_t d_out, int64_t d_in, int64_t r) {
    return bin_gemm_ws(nullptr, M, d_out, d_in, r).bytes;
}

bool gemm_binlr_tc_supported(int64_t M, int64_t d_out, int64_t d_in, int64_t r) {
    if (M < 64 || d_out % 16 != 0 || r % 32 != 0 || d_in % 32 != 0) return false;
    if (M > ((int64_t)1 << 31) || d_out > ((int64_t)1 << 31) || r > ((int64_t)1 << 31)) return false;
    if (ceil_div(std::max(d_out, r), (int64_t)128) * ceil_div(M, (int64_t)gemm_nt(M)) > kCounterBytes / 4) return false;
    return GemmSmem(1, gemm_nt(M), 2).bytes + 1024 <= 227 * 1024;
}

lbq_status launch_gemm_binlr_tc(const void* x, bool bf16, int64_t M, const void* U, const void* Vt, const void* s1,
                                const void* s2, int64_t d_out, int64_t d_in, int64_t r, void* y, void* ws,
                                size_t ws_bytes, cudaStream_t st) {
    if (ws == nullptr || ws_bytes < gemm_binlr_tc_ws_bytes(M, d_out, d_in, r)) return LBQ_ERR_WORKSPACE;
    if (gemm_encode_fn() == nullptr) return LBQ_ERR_CUDA;
    const BinGemmWs w = bin_gemm_ws(ws, M, d_out, d_in, r);
    lbq_status s = to_f16(x, bf16, s2, M, d_in, w.xs, st);
    if (s != LBQ_OK) return s;
    const int NT = gemm_nt(M);
    GemmArgs a1;
    memset(&a1, 0, sizeof a1);
    if (!encode_2d(&a1.mx, w.xs, M, d_in, d_in, 64, (uint32_t)NT, CU_TENSOR_MAP_SWIZZLE_128B)) return LBQ_ERR_CUDA;
    a1.packed = (const uint8_t*)Vt;
    a1.rowscale = nullptr;
    a1.y = w.t;
    a1.n = r;
    a1.ksb = sign_cols_pad(d_in) / 256;
    a1.M = M;
    a1.ldy = w.ldt;
    a1.err = device_error_word();
    a1.counters = (unsigned*)ws;
    a1.partials = w.partials;
    s = launch_gemm_b<1>(32, a1, st);
    if (s != LBQ_OK) return s;
    GemmArgs a2;
    memset(&a2, 0, sizeof a2);
    if (!encode_2d(&a2.mx, w.t, M, r, w.ldt, 64, (uint32_t)NT, CU_TENSOR_MAP_SWIZZLE_128B)) return LBQ_ERR_CUDA;
    a2.packed = (const uint8_t*)U;
    a2.rowscale = (const uint16_t*)s1;
    a2.y = (uint16_t*)y;
    a2.n = d_out;
    a2.ksb = sign_cols_pad(r) / 256;
    a2.M = M;
    a2.ldy = d_out;
    a2.err = a1.err;
    a2.counters = (unsigned*)ws;
    a2.partials = w.partials;
    return launch_gemm_b<1>(32, a2, st);
}

}  // namespace lbq
