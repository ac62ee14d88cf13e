// lbq_binlr_ldg.cu -- binary low-rank GEMV y = s1 . U (V^T (s2 . x)), M = 1..4 tokens (sm_100a).
//
// Form: "70B en 4GB de VRAM: la compresión neural de 2026, ¿es real?" (nramos.dev),
// section "1. NanoQuant — sub-1-bit PTQ", bullet "Formulación".  Two chained launches,
// each one +-1 matrix times a vector with the machinery of the group GEMV:
//
//   stage 1: t[m, j] = sum_i V^T[j, i] * s2[i] * x[m, i]       rows r,     columns d_in
//   stage 2: y[m, i] = s1[i] * sum_j U[i, j] * t[m, j]         rows d_out, columns r
//
//  * Every CTA prepares the stage input v (s2 . x, or t) in its shared memory right after
//    waiting for the previous kernel, in one pass: one power-of-two scale 2^E per token and
//    256-column chunk (|v| <= 32639 after scaling), int8 planes hi, lo (v = 256 hi + lo) in
//    B-fragment order and the exact chunk sums of v.
//  * Warps split the (16-row tile, 256-column superblock) units evenly (warp-level
//    stream-K) and stream the lanes' 16-byte sign words straight into registers, several
//    units ahead.  Per k-step p the word's bits p of each byte give four 0/1 u8 A-fragment
//    bytes; mma.m16n8k32 u8 x s8 gives S = sum bit * v over the unit exactly.
//  * sum_k sign * v = 2 S - sum v; each unit adds 2^E (2 S - chunk sum) to the warp's fp32
//    partial (times s1 in stage 2); tiles split between warps are added in shared memory
//    after one CTA barrier, and tiles split between CTAs by the last CTA to arrive, both in
//    a fixed order (cta_fix_finish), so the result is deterministic.
//  * Both launches are programmatic dependents; only their first weight loads precede the
//    wait for the previous kernel.
#include <cstring>
#include <type_traits>
#include "lbq_common.cuh"
#include "lbq_internal.h"
#include "lbq_group_frag.cuh"
#include "lbq_ldg.cuh"

namespace lbq {

constexpr int kBinPrepBatch = 4;             // prep chunks whose loads a warp issues together

struct BinStageArgs {
    const uint8_t* signs;       // kernel sign layout, rows x cpad
    const uint16_t* x;          // stage 1: [M x cols] activations
    const uint16_t* s2;         // stage 1: [cols] column scales
    const float* tin;           // stage 2: [M x cols] stage-1 result
    float* tout;                // stage 1 output [M x rows]
    const uint16_t* s1;         // stage 2: [rows] row scales
    uint16_t* y;                // stage 2 output [M x rows]
    float* partials;
    unsigned* counters;
    int64_t rows, cols, cpad, ksb, n_tiles, total_units, total_warps;
    int M, maxc;
    int sp, sv, se, szero;      // shared-memory offsets: planes, chunk sums, exponents, zero chunk,
    int sfix;                   // CTA-level tile finish (CtaFix)
    int cluster2;               // 1: clusters of two CTAs that share the input prep
};

// Byte offset, in a 256-column chunk of a plane row, of column 32p + 16h + 4c + j: the
// B-fragment bytes (b0: h = 0, b1: h = 1) of k-steps p and p + 1 of lane-group c are one
// 16-byte piece.
__device__ __forceinline__ int bin_plane_off(int p, int h, int c) { return 64 * (p >> 1) + 16 * c + 8 * (p & 1) + 4 * h; }

// The lane's 8 consecutive values as q = rint(v * 2^-E) in natural order: hi/lo bytes of
// elements 0..3 in .x, 4..7 in .y; sum(q) over the whole warp.
__device__ __forceinline__ PrepOut bin_quantize8(const float (&v)[8], int E) {
    PrepOut r;
    r.E = E;
    const int e1 = max(-126, min(127, -E));
    const float f1 = ldg_exp2i(e1), f2 = ldg_exp2i(-E - e1);
    uint32_t h0 = 0, h1 = 0, l0 = 0, l1 = 0;
    int sum = 0;
#pragma unroll
    for (int e = 0; e < 8; e++) {
        const int q = __float2int_rn((v[e] * f1) * f2);
        const int h = (q + 128) >> 8;
        const int l = q - 256 * h;
        sum += q;
        const int sh = 8 * (e & 3);
        if (e < 4) {
            h0 |= (uint32_t)(h & 0xFF) << sh;
            l0 |= (uint32_t)(l & 0xFF) << sh;
        } else {
            h1 |= (uint32_t)(h & 0xFF) << sh;
            l1 |= (uint32_t)(l & 0xFF) << sh;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    r.hi = make_uint2(h0, h1);
    r.lo = make_uint2(l0, l1);
    r.gsum = sum;
    return r;
}

// Raw bits of the lane's 8 stage-input values of token m, columns k0..k0+7 (zero past the
// last column): stage 1 x (r0) and s2 (r1), stage 2 the fp32 t (r0: 0..3, r1: 4..7).
// The inputs may come from the previous kernel of the stream: read through L2.
template <bool STAGE2>
__device__ __forceinline__ void bin_load_raw(const BinStageArgs& a, int m, int64_t k0, uint4& r0, uint4& r1) {
    if (k0 >= a.cols) {
        r0 = r1 = make_uint4(0, 0, 0, 0);
    } else if constexpr (STAGE2) {
        r0 = __ldcg(reinterpret_cast<const uint4*>(a.tin + (int64_t)m * a.cols + k0));
        r1 = __ldcg(reinterpret_cast<const uint4*>(a.tin + (int64_t)m * a.cols + k0 + 4));
    } else {
        r0 = __ldcg(reinterpret_cast<const uint4*>(a.x + (int64_t)m * a.cols + k0));
        r1 = __ldg(reinterpret_cast<const uint4*>(a.s2 + k0));
    }
}

template <bool STAGE2, bool BF16>
__device__ __forceinline__ void bin_convert(const uint4& r0, const uint4& r1, float (&v)[8]) {
    if constexpr (STAGE2) {
        v[0] = __uint_as_float(r0.x); v[1] = __uint_as_float(r0.y); v[2] = __uint_as_float(r0.z); v[3] = __uint_as_float(r0.w);
        v[4] = __uint_as_float(r1.x); v[5] = __uint_as_float(r1.y); v[6] = __uint_as_float(r1.z); v[7] = __uint_as_float(r1.w);
    } else {
        const uint32_t xw[4] = {r0.x, r0.y, r0.z, r0.w};
        const uint32_t sw[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int e = 0; e < 8; e++) {
            const float xv = to_f32<BF16>((uint16_t)(xw[e / 2] >> (16 * (e & 1))));
            const float sv = __half2float(__ushort_as_half((uint16_t)(sw[e / 2] >> (16 * (e & 1)))));
            v[e] = xv * sv;       // exact: a product of two 11- (or 8-) bit significands
        }
    }
}

template <bool STAGE2, int D, int NW, bool BF16>
__global__ void __launch_bounds__(NW * 32, 1) k_binlr_ldg(const __grid_constant__ BinStageArgs a) {
    constexpr int NB = 1;                      // M <= 4: hi/lo planes of 4 tokens in one n-block
    constexpr int PF = 16;                     // units prefetched into L2 before the wait
    extern __shared__ __align__(16) uint8_t smem[];
    griddep_launch_dependents();
    // clusters of two: each CTA prepares half of the stage input, into both shared
    // memories; the partner must have started before the first remote store
    const bool c2 = a.cluster2 != 0;
    if (c2) cluster_arrive_relaxed();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int64_t W = a.total_warps, S = a.total_units;
    const int64_t wid = (int64_t)blockIdx.x * NW + warp;
    const int u_begin = (int)(wid < W ? wid * S / W : S);
    const int u_end = (int)(wid < W ? (wid + 1) * S / W : S);
    const bool has_work = u_begin < u_end;
    const int M = a.M;
    const int ksb = (int)a.ksb;
    const uint64_t pol = l2_policy_evict_first();

    int ct = 0, csb = 0;
    if (has_work) {
        ct = u_begin / ksb;
        csb = u_begin % ksb;
    }
    const uint8_t* lptr = a.signs + (int64_t)u_begin * 512 + 16 * lane;
    uint4 wb[D];
#pragma unroll
    for (int d = 0; d < D; d++)
        if (u_begin + d < u_end) wb[d] = ldg_stream(lptr + d * 512, pol);
    lptr += D * 512;
    if (lane < PF && u_begin + D + lane < u_end) l2_prefetch_bulk(lptr - 16 * lane + lane * 512, 512);
    if (threadIdx.x < 16) reinterpret_cast<uint4*>(smem + a.szero)[threadIdx.x] = make_uint4(0, 0, 0, 0);
    // stage 2: the row scales of the warp's first tile (a weight, like the signs)
    uint16_t s1h0 = 0, s1h1 = 0;
    if constexpr (STAGE2) {
        if (has_work) {
            s1h0 = __ldg(a.s1 + (int64_t)ct * 16 + g);
            s1h1 = __ldg(a.s1 + (int64_t)ct * 16 + g + 8);
        }
    }
    griddep_wait();

    // ---- prepare the stage input in one pass: per 256-column chunk one power-of-two scale,
    // the int8 planes and the exact chunk sum; the chunk order is rotated by the CTA (pair)
    // index so that the CTAs do not all read the same lines at once
    if (c2) cluster_wait();
    const uint32_t peer = (blockIdx.x & 1) ^ 1u;
    const int pw = c2 ? 2 * NW : NW;                                // warps sharing the prep
    const int pwi = c2 ? (int)(blockIdx.x & 1) * NW + warp : warp;
    const int kch = (int)(a.cpad / kLdgChunk);
    const int ntask = M * kch;                   // (token, chunk) pairs
    const int rot = (int)((c2 ? blockIdx.x >> 1 : blockIdx.x) % (unsigned)kch);
    int* expo = reinterpret_cast<int*>(smem + a.se);
    int* vsum = reinterpret_cast<int*>(smem + a.sv);
    // a warp's chunks are independent: issue the loads of kBinPrepBatch of them together
    for (int t0 = pwi; t0 < ntask; t0 += pw * kBinPrepBatch) {
        uint4 r0[kBinPrepBatch], r1[kBinPrepBatch];
#pragma unroll
        for (int j = 0; j < kBinPrepBatch; j++) {
            const int t = t0 + j * pw;
            if (t < ntask) {
                const int m = t / kch, cw = t - m * kch;
                const int ch = cw + rot < kch ? cw + rot : cw + rot - kch;
                bin_load_raw<STAGE2>(a, m, (int64_t)ch * kLdgChunk + 8 * lane, r0[j], r1[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < kBinPrepBatch; j++) {
            const int t = t0 + j * pw;
            if (t < ntask) {
                const int m = t / kch, cw = t - m * kch;
                const int ch = cw + rot < kch ? cw + rot : cw + rot - kch;
                float v[8];
                bin_convert<STAGE2, BF16>(r0[j], r1[j], v);
                const PrepOut r = bin_quantize8(v, ldg_fixed_point_exponent(warp_max_abs8(v)));
                // elements 8 lane + 0..3 and + 4..7: columns 32p + 16h + 4c' + j
                const int p = lane >> 2, h = (lane & 3) >> 1, c0 = 2 * (lane & 1);
                int8_t* base = reinterpret_cast<int8_t*>(smem + a.sp) + (int64_t)(2 * m) * a.cpad + ch * kLdgChunk;
                uint32_t* q[4] = {reinterpret_cast<uint32_t*>(base + bin_plane_off(p, h, c0)),
                                  reinterpret_cast<uint32_t*>(base + bin_plane_off(p, h, c0 + 1)),
                                  reinterpret_cast<uint32_t*>(base + a.cpad + bin_plane_off(p, h, c0)),
                                  reinterpret_cast<uint32_t*>(base + a.cpad + bin_plane_off(p, h, c0 + 1))};
                const uint32_t qv[4] = {r.hi.x, r.hi.y, r.lo.x, r.lo.y};
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    *q[i] = qv[i];
                    if (c2) st_cluster_s32(cluster_map_smem(smem_u32(q[i]), peer), (int)qv[i]);
                }
                if (lane == 0) {
                    vsum[m * kch + ch] = r.gsum;
                    expo[m * kch + ch] = r.E;
                    if (c2) {
                        st_cluster_s32(cluster_map_smem(smem_u32(vsum + m * kch + ch), peer), r.gsum);
                        st_cluster_s32(cluster_map_smem(smem_u32(expo + m * kch + ch), peer), r.E);
                    }
                }
            }
        }
    }
    if (c2) cluster_sync_all();                  // both halves of the input are in place
    else __syncthreads();
    const CtaFix fix = cta_fix_at(smem + a.sfix, NW, M);
    cta_fix_clear(fix, warp, lane);
    const int head_tile = ct;

    // B-fragment row of this lane (plane g: token g / 2, hi or lo) and its token's sums
    const bool pv = g < 2 * M;
    const int8_t* prow = pv ? reinterpret_cast<const int8_t*>(smem + a.sp) + (int64_t)g * a.cpad + 16 * c
                            : reinterpret_cast<const int8_t*>(smem + a.szero) + 16 * c;
    const int pstep = pv ? kLdgChunk : 0;
    const bool tv = c < M;
    const int* vrow = tv ? vsum + c * kch : reinterpret_cast<const int*>(smem + a.szero);
    const int* erow = tv ? expo + c * kch : reinterpret_cast<const int*>(smem + a.szero);
    const int vstep = tv ? 1 : 0;

    float part0 = 0.0f, part1 = 0.0f;                // rows g and g + 8 of token c, this warp's slice
    int tile_first_u = u_begin - csb;

    for (int base = u_begin; base < u_end; base += D) {
#pragma unroll
        for (int d = 0; d < D; d++) {
            const int u = base + d;
            if (u < u_end) {
                const uint4 w = wb[d];
                if (u + D < u_end) {
                    wb[d] = ldg_stream(lptr, pol);
                    lptr += 512;
                }
                const int8_t* pr = prow + csb * pstep;
                // S = sum over the unit of bit * v, exactly: 0/1 A bytes of k-step p; the even
                // and the odd k-steps accumulate in two independent chains
                int se[4], so[4];
#pragma unroll
                for (int p = 0; p < 8; p += 2) {
                    const uint4 bq = *reinterpret_cast<const uint4*>(pr + 64 * (p >> 1));
                    const uint32_t a0 = (w.x >> p) & 0x01010101u, a1 = (w.y >> p) & 0x01010101u;
                    const uint32_t a2 = (w.z >> p) & 0x01010101u, a3 = (w.w >> p) & 0x01010101u;
                    const uint32_t b0 = (w.x >> (p + 1)) & 0x01010101u, b1 = (w.y >> (p + 1)) & 0x01010101u;
                    const uint32_t b2 = (w.z >> (p + 1)) & 0x01010101u, b3 = (w.w >> (p + 1)) & 0x01010101u;
                    if (p == 0) {
                        mma_16832_u8s8_zc(se, a0, a1, a2, a3, bq.x, bq.y);
                        mma_16832_u8s8_zc(so, b0, b1, b2, b3, bq.z, bq.w);
                    } else {
                        mma_16832_u8s8(se, a0, a1, a2, a3, bq.x, bq.y);
                        mma_16832_u8s8(so, b0, b1, b2, b3, bq.z, bq.w);
                    }
                }
                // sum_k sign * v = 2 S - sum v, times this chunk's 2^E; columns 2c (hi), 2c + 1 (lo)
                const int vs = vrow[csb * vstep];
                const float sc = ldg_exp2i(erow[csb * vstep]);
                part0 = fmaf(sc, (float)(2 * (256 * (se[0] + so[0]) + se[1] + so[1]) - vs), part0);
                part1 = fmaf(sc, (float)(2 * (256 * (se[2] + so[2]) + se[3] + so[3]) - vs), part1);
                if (csb == ksb - 1 || u == u_end - 1) {
                    float part[NB][2];   // [0][0]: row g, [0][1]: row g + 8 of token c
                    part[0][0] = tv ? part0 : 0.0f;
                    part[0][1] = tv ? part1 : 0.0f;
                    if constexpr (STAGE2) {
                        part[0][0] *= __half2float(__ushort_as_half(s1h0));
                        part[0][1] *= __half2float(__ushort_as_half(s1h1));
                        // the next tile's row scales, a tile ahead of their use
                        if (ct + 1 < a.n_tiles) {
                            s1h0 = __ldg(a.s1 + (int64_t)(ct + 1) * 16 + g);
                            s1h1 = __ldg(a.s1 + (int64_t)(ct + 1) * 16 + g + 8);
                        }
                    }
                    const bool full = tile_first_u >= u_begin && csb == ksb - 1;
                    if (full) {
                        if constexpr (STAGE2) tile_store_full<NB>(part, M, a.rows, ct, a.y);
                        else tile_store_full<NB>(part, M, a.rows, ct, a.tout);
                    } else {
                        cta_fix_put<NB>(fix, warp, ct == head_tile ? 0 : 1, ct, part, M);
                    }
                    part0 = part1 = 0.0f;
                    tile_first_u = u + 1;
                }
                if (++csb == ksb) {
                    csb = 0;
                    ct++;
                }
            }
        }
    }

    // ---- partial tiles: CTA sums in shared memory, CTA-crossing tiles by ticket
    __syncthreads();
    const int64_t cw0 = (int64_t)blockIdx.x * NW, cw1 = min(cw0 + NW, W);
    const int64_t C0 = cw0 < W ? cw0 * S / W : S, C1 = cw0 < W ? cw1 * S / W : S;
    using Y = typename std::conditional<STAGE2, uint16_t, float>::type;
    Y* yout;
    if constexpr (STAGE2) yout = a.y;
    else yout = a.tout;
    cta_fix_finish<Y>(fix, NW, warp, M, u_begin, C0, C1, S, W, blockIdx.x, a.partials, a.counters, a.maxc,
                      [&](int T, int64_t& first_u, int64_t& units, Y*& y, int64_t& n, int64_t& row0) {
                          first_u = (int64_t)T * ksb;
                          units = ksb;
                          y = yout;
                          n = a.rows;
                          row0 = (int64_t)T * 16;
                      });
}

// ------------------------------------------------------------------ host side
struct BinLdgPlan {
    int64_t units1, units2, warps1, warps2;
    int grid1, grid2, maxc1, maxc2;
    size_t part1, part2, t_off, bytes;
};

// Warps per CTA and register ring depth of the sign stream (one CTA per SM: the stage
// input is prepared once per SM).
constexpr int kBinNW = 16, kBinD = 8;
// Launches of at least this many CTAs run as clusters of two that prepare half of the
// stage input each (the prep is latency-bound: a 28672-wide input costs ~7 us per CTA).
constexpr int kBinClusterMinGrid = 32;

static void bin_stage_plan(int64_t rows, int64_t cpad, int64_t& units, int64_t& warps, int& grid, int& maxc) {
    const int64_t ksb = cpad / kLdgChunk;
    units = rows / 16 * ksb;
    constexpr int64_t kMinUnitsPerWarp = 4;
    grid = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)sm_count(), ceil_div(units, kBinNW * kMinUnitsPerWarp)));
    if (grid >= kBinClusterMinGrid) grid &= ~1;    // clusters of two share the input prep
    warps = std::min<int64_t>((int64_t)grid * kBinNW, std::max<int64_t>(units, 1));
    maxc = (int)(ceil_div(ksb * warps, std::max<int64_t>(units, 1)) + 2);
}

static BinLdgPlan bin_ldg_plan(int64_t M, int64_t d_out, int64_t d_in, int64_t r) {
    BinLdgPlan pl;
    bin_stage_plan(r, sign_cols_pad(d_in), pl.units1, pl.warps1, pl.grid1, pl.maxc1);
    bin_stage_plan(d_out, sign_cols_pad(r), pl.units2, pl.warps2, pl.grid2, pl.maxc2);
    pl.part1 = kCounterBytes;
    pl.part2 = pl.part1 + al256((size_t)(r / 16 * pl.maxc1 * 16 * M * 4));
    pl.t_off = pl.part2 + al256((size_t)(d_out / 16 * pl.maxc2 * 16 * M * 4));
    pl.bytes = pl.t_off + al256((size_t)(M * r * 4));
    return pl;
}

static int bin_fix_bytes(int64_t M) { return al16((int64_t)cta_fix_bytes(kBinNW, (int)M)); }

static int bin_smem_bytes(int64_t M, int64_t cpad) {
    // planes [2M][cpad] | chunk sums [M][cpad/256] | chunk exponents [M][cpad/256] | zero chunk | CTA finish
    return al16(2 * M * cpad) + 2 * al16(M * (cpad / kLdgChunk) * 4) + 256 + bin_fix_bytes(M);
}

bool gemv_binlr_ldg_supported(int64_t M, int64_t d_out, int64_t d_in, int64_t r) {
    if (M < 1 || M > 4 || d_out % 16 != 0 || r % 32 != 0 || d_in % 32 != 0) return false;
    // int32 sums: |sum over a tile of bit * v| <= 32639 * columns must stay below 2^30
    if (d_out / 16 + r / 16 > kMaxTiles || d_in > 32768 || r > 32768) return false;
    const int budget = 200 * 1024;                 // one CTA per SM
    return bin_smem_bytes(M, sign_cols_pad(d_in)) <= budget && bin_smem_bytes(M, sign_cols_pad(r)) <= budget;
}

size_t gemv_binlr_ldg_ws_bytes(int64_t M, int64_t d_out, int64_t d_in, int64_t r) {
    return bin_ldg_plan(M, d_out, d_in, r).bytes;
}

template <bool STAGE2, bool BF16>
static lbq_status launch_bin_stage(const BinStageArgs& a, int grid, int smem, cudaStream_t st) {
    constexpr auto kern = k_binlr_ldg<STAGE2, kBinD, kBinNW, BF16>;
    const lbq_status s = ldg_smem_attr<kern>(200 * 1024);
    if (s != LBQ_OK) return s;
    return launch_pdl_cluster(kern, grid, a.cluster2 ? 2 : 1, kBinNW * 32, (size_t)smem, st, a);
}

lbq_status launch_gemv_binlr_ldg(const void* x, bool bf16, int64_t M, const void* U, const void* Vt, const void* s1,
                                 const void* s2, int64_t d_out, int64_t d_in, int64_t r, void* y, void* ws,
                                 size_t ws_bytes, cudaStream_t st) {
    const BinLdgPlan pl = bin_ldg_plan(M, d_out, d_in, r);
    if (ws == nullptr || ws_bytes < pl.bytes) return LBQ_ERR_WORKSPACE;
    char* base = (char*)ws;
    float* t = (float*)(base + pl.t_off);
    for (int stage = 0; stage < 2; stage++) {
        BinStageArgs a;
        memset(&a, 0, sizeof a);
        const bool st2 = stage == 1;
        a.signs = (const uint8_t*)(st2 ? U : Vt);
        a.rows = st2 ? d_out : r;
        a.cols = st2 ? r : d_in;
        a.cpad = sign_cols_pad(a.cols);
        a.ksb = a.cpad / kLdgChunk;
        a.n_tiles = a.rows / 16;
        a.x = (const uint16_t*)x;
        a.s2 = (const uint16_t*)s2;
        a.tin = t;
        a.tout = t;
        a.s1 = (const uint16_t*)s1;
        a.y = (uint16_t*)y;
        a.partials = (float*)(base + (st2 ? pl.part2 : pl.part1));
        // the two stages' tickets are disjoint ranges of the counter header
        a.counters = (unsigned*)base + (st2 ? r / 16 : 0);
        a.total_units = st2 ? pl.units2 : pl.units1;
        a.total_warps = st2 ? pl.warps2 : pl.warps1;
        a.M = (int)M;
        a.maxc = st2 ? pl.maxc2 : pl.maxc1;
        a.sp = 0;
        a.sv = al16(2 * M * a.cpad);
        a.se = a.sv + al16(M * a.ksb * 4);
        a.szero = a.se + al16(M * a.ksb * 4);
        a.sfix = a.szero + 256;
        const int smem = bin_smem_bytes(M, a.cpad);
        const int grid = st2 ? pl.grid2 : pl.grid1;
        a.cluster2 = grid >= kBinClusterMinGrid ? 1 : 0;
        lbq_status s;
        if (st2) s = bf16 ? launch_bin_stage<true, true>(a, grid, smem, st) : launch_bin_stage<true, false>(a, grid, smem, st);
        else s = bf16 ? launch_bin_stage<false, true>(a, grid, smem, st) : launch_bin_stage<false, false>(a, grid, smem, st);
        if (s != LBQ_OK) return s;
    }
    return LBQ_OK;
}

}  // namespace lbq
