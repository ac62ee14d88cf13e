// lbq_gemv_group_ldg.cu -- dequant-fused group GEMV on integer tensor cores (sm_100a), M = 1..16.
//
//   y[m, i] = sum_k x[m, k] * s[i, k/g] * (q[i, k] - z[i, k/g])
//
// Decode time per token is the bytes read over the read bandwidth ("AirLLM corre un
// modelo 70B en una GPU de 4GB...", section "Por qué es lento"), so the packed weights
// must stream from HBM at full rate while every other cost hides under that stream.
//
//  * Work list: the (16-row tile, 256-wide k superblock) units of up to kMaxGemvProblems
//    products of one bit width and group size (e.g. the q/k/v or gate/up projections of
//    a decoder block), tile-major.  Every warp of the grid takes an equal contiguous
//    slice of it ("stream-K" at warp granularity), so all warps finish together.  A tile
//    split between warps of one CTA is added in shared memory after one CTA barrier; a
//    tile split between CTAs by the last CTA to arrive at its ticket (cta_fix_finish):
//    fixed order, deterministic, at most two GPU-scope tickets per CTA.
//  * Each warp streams its units' packed words straight into registers with 128-bit
//    non-coherent loads (evict-first in L2), keeping D units in flight: one unit is the
//    lane's 16 * B bytes of a tile's 512 * B-byte superblock block, already in mma
//    fragment order.  Warps never wait for one another, so a warp stalled on compute or
//    on a scale load leaves the other warps' loads in flight.
//  * Every distinct activation row becomes 16-bit fixed point with one power-of-two
//    scale 2^E per token and 256-wide chunk (|v| <= 32639), stored as two int8 planes
//    hi, lo (v = 256 hi + lo) in B-fragment order, plus exact per-group sums of v.  For
//    one token block each CTA prepares them in its own shared memory right after the
//    wait; otherwise a prep kernel writes them to the workspace, read through L2.
//  * Per k-step the lane masks its words into u8 A fragments (one LOP per four codes)
//    and runs mma.m16n8k32 u8 x s8 -> s32 with the hi and lo planes side by side in N.
//    Per group the exact integer sum S = sum q v becomes sum (q - z) v = S - z sum(v),
//    scaled by s into an fp32 chunk accumulator, which is scaled by 2^E once per chunk.
//  * The kernels are launched as programmatic dependents: the GEMV's first weight
//    loads are issued before it waits for the previous kernel (griddepcontrol.wait), and
//    x is read only after that wait.  Packed
//    weights, scales and zeros must therefore not be written by a kernel that signals
//    programmatic completion early.
// Group codes: "TurboQuant: cuantizar modelos grandes para que quepan en local",
// section "Compresión por bloques"; RTN codes: "Métodos de cuantización de LLM para
// ejecutar un modelo de 70B en una sola GPU", section "RTN (Round-To-Nearest)".
#include <cstring>
#include "lbq_common.cuh"
#include "lbq_internal.h"
#include "lbq_group_frag.cuh"
#include "lbq_ldg.cuh"

namespace lbq {


struct LdgProblem {
    const uint8_t* packed;
    const uint16_t* scales;
    const uint16_t* zeros;
    uint16_t* y;
    int64_t n, k, ksb, n_tiles, ngroups, unit_begin, tile_begin;
    int slot;               // activation prep slot (products that share x share one)
};

struct LdgArgs {
    LdgProblem p[kMaxGemvProblems];
    float* partials;
    unsigned* counters;
    int64_t total_units, total_warps, total_tiles;
    int count, M, maxc;
    int pair;               // 1: clusters of two CTAs, each pair a whole number of tiles
    int sring;              // byte offset of the scale/zero rings in shared memory
    int szero;              // byte offset of a 256-byte zero chunk in shared memory
    int sfix;               // byte offset of the CTA-level tile finish (CtaFix)
};

// First unit of launch-wide tile T (total_units for T = total_tiles).
__device__ __forceinline__ int64_t ldg_tile_first_unit(const LdgArgs& a, int64_t T) {
    if (T >= a.total_tiles) return a.total_units;
    int q = 0;
    while (q + 1 < a.count && T >= a.p[q + 1].tile_begin) q++;
    return a.p[q].unit_begin + (T - a.p[q].tile_begin) * a.p[q].ksb;
}

constexpr int kScaleRing = 6;               // units of scales/zeros in flight per warp
constexpr int kPrepBatch = 4;               // activation chunks whose loads a warp issues together

// Bytes of one unit's scale/zero slot: 2 arrays x 16 rows x (256 / GROUP) fp16.
constexpr int scale_slot_bytes(int group) { return 64 * (kLdgChunk / group); }

// Prepared activations of one distinct x: planes [2M][k] (row 2m = hi plane of token m,
// 2m + 1 = lo plane, B-fragment byte order), exact group sums [M][k / GROUP] and
// exponents [M][k / 256], in global memory (planes/xsum/expo) or at byte offsets of the
// CTA's shared memory (sp/sx/se).
struct PrepSlot {
    const uint16_t* x;
    int8_t* planes;
    float* xsum;
    int* expo;
    int64_t k, warp_begin;
    int sp, sx, se;
};

struct PrepArgs {
    PrepSlot s[kMaxGemvProblems];
    int8_t* zero;           // 256 zero bytes in global memory (written by k_gemv_prep)
    int64_t total_warps;
    int count, M;
};

// NG consecutive fp16 values (NG in 4, 8, 16; 2 * NG-byte aligned) from shared memory.
template <int NG>
__device__ __forceinline__ void lds_halves_ldg(const uint16_t* p, uint32_t (&d)[NG / 2]) {
    if constexpr (NG == 4) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        d[0] = v.x;
        d[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < NG / 8; i++) {
            const uint4 v = reinterpret_cast<const uint4*>(p)[i];
            d[4 * i] = v.x;
            d[4 * i + 1] = v.y;
            d[4 * i + 2] = v.z;
            d[4 * i + 3] = v.w;
        }
    }
}

// ------------------------------------------------------------------ activation prep
// One warp per (distinct activation row set, token m, 256-wide chunk); lane l holds
// elements 8l..8l+7 of the chunk and stores them as the B-fragment bytes of k-slots
// 4(l mod 4).. (even elements) and 16 + 4(l mod 4).. (odd elements) of k-step l / 4.
// x may have been written by the previous kernel of the stream, so it is read through
// L2 (ld.global.cg), never through the non-coherent path.
__device__ __forceinline__ uint4 prep_load(const uint16_t* xc, int lane) {
    return __ldcg(reinterpret_cast<const uint4*>(xc + 8 * lane));
}

template <int GROUP, bool BF16>
__device__ __forceinline__ PrepOut prep_convert(const uint4 raw) {
    const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; e++) v[e] = to_f32<BF16>((uint16_t)(rw[e / 2] >> (16 * (e & 1))));
    return prep_quantize8<GROUP / 8>(v, ldg_fixed_point_exponent(warp_max_abs8(v)));
}

template <int GROUP, bool BF16>
__device__ __forceinline__ PrepOut prep_chunk(const uint16_t* xc, int lane) {
    return prep_convert<GROUP, BF16>(prep_load(xc, lane));
}

// Warp task wi of the prep list -> (slot, token, chunk).
__device__ __forceinline__ int prep_task(const PrepArgs& a, int64_t wi, int& m, int64_t& ch) {
    int s = 0;
    while (s + 1 < a.count && wi >= a.s[s + 1].warp_begin) s++;
    const int64_t kch = a.s[s].k / kLdgChunk;
    const int64_t li = wi - a.s[s].warp_begin;
    m = (int)(li / kch);
    ch = li % kch;
    return s;
}

// Stand-alone prep into global memory, for activations too large for shared memory.
template <int GROUP, bool BF16>
__global__ void __launch_bounds__(256) k_gemv_prep(const __grid_constant__ PrepArgs a) {
    griddep_launch_dependents();
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t wi = ((int64_t)blockIdx.x * 256 + threadIdx.x) >> 5;
    if (wi >= a.total_warps) return;
    int m;
    int64_t ch;
    const PrepSlot& S = a.s[prep_task(a, wi, m, ch)];
    const PrepOut r = prep_chunk<GROUP, BF16>(S.x + (int64_t)m * S.k + ch * kLdgChunk, lane);
    int8_t* row_h = S.planes + (int64_t)(2 * m) * S.k + ch * kLdgChunk;
    *reinterpret_cast<uint2*>(row_h + plane_off(lane)) = r.hi;
    *reinterpret_cast<uint2*>(row_h + S.k + plane_off(lane)) = r.lo;
    if (wi == 0 && lane < 16) reinterpret_cast<uint4*>(a.zero)[lane] = make_uint4(0, 0, 0, 0);
    constexpr int LPG = GROUP / 8;
    if (lane % LPG == 0) S.xsum[(int64_t)m * (S.k / GROUP) + ch * (kLdgChunk / GROUP) + lane / LPG] = (float)r.gsum;
    if (lane == 0) S.expo[(int64_t)m * (S.k / kLdgChunk) + ch] = r.E;
}

// Prepared-activation reads: shared memory (plain loads) or global memory written by the
// prep kernel of this launch (L2 only: data another grid wrote during this grid's life).
template <bool SMEMP>
__device__ __forceinline__ uint4 ld_plane16(const int8_t* p) {
    if constexpr (SMEMP) return *reinterpret_cast<const uint4*>(p);
    else return __ldcg(reinterpret_cast<const uint4*>(p));
}
template <bool SMEMP, int N>
__device__ __forceinline__ void ld_floats(const float* p, float (&v)[N]) {
    if constexpr (N == 2) {
        const float2 t = SMEMP ? *reinterpret_cast<const float2*>(p) : __ldcg(reinterpret_cast<const float2*>(p));
        v[0] = t.x;
        v[1] = t.y;
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 t =
                SMEMP ? *reinterpret_cast<const float4*>(p + i) : __ldcg(reinterpret_cast<const float4*>(p + i));
            v[i] = t.x;
            v[i + 1] = t.y;
            v[i + 2] = t.z;
            v[i + 3] = t.w;
        }
    }
}
template <bool SMEMP, class T>
__device__ __forceinline__ T ld_prep(const T* p) {
    if constexpr (SMEMP) return *p;
    else return __ldcg(p);
}

// ------------------------------------------------------------------ GEMV
// D units in flight per warp; NW warps per CTA, one CTA per SM (NW = 16: up to 128 registers
// a thread, NW = 8: up to 255);
// SMEMP: every CTA prepares the activations itself, in its shared memory, right after
// waiting for the previous kernel (else they come from k_gemv_prep via L2).
template <int B, int GROUP, int NB, int D, int NW, bool SMEMP, bool BF16>
__global__ void __launch_bounds__(NW * 32, 1)
    k_gemv_group_ldg(const __grid_constant__ LdgArgs a, const __grid_constant__ PrepArgs pa) {
    using G = GroupGeom<B>;
    using F = IFrag<B>;
    constexpr int KPG = GROUP / 32;                // k-steps per group
    constexpr int NGC = kLdgChunk / GROUP;         // groups per unit
    // units prefetched into L2 before the wait (about 16 KB a warp): HBM keeps streaming
    // while the activations are prepared
    constexpr int PF = 16384 / (512 * B);
    extern __shared__ __align__(16) uint8_t smem[];
    griddep_launch_dependents();
    // pair mode: the two CTAs prepare half of the activations each, into both shared
    // memories; the partner must have started before the first remote store
    const bool pairp = SMEMP && a.pair != 0;
    if (pairp) cluster_arrive_relaxed();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int64_t W = a.total_warps, S = a.total_units;
    // this warp's units [u_begin, u_end) and the CTA's [C0, C1); unit indices fit 32 bits
    // (the host caps the list)
    int64_t ub, ue, C0, C1;
    if (a.pair) {
        // pair p of P takes tiles [p NT / P, (p + 1) NT / P); min(2 NW, its units) warps of
        // the pair split them evenly, the other warps take none
        const int64_t P = gridDim.x >> 1, p = blockIdx.x >> 1, rank = blockIdx.x & 1;
        const int64_t U0 = ldg_tile_first_unit(a, p * a.total_tiles / P);
        const int64_t U1 = ldg_tile_first_unit(a, (p + 1) * a.total_tiles / P);
        const int64_t n = U1 - U0, Wp = n < 2 * NW ? n : (int64_t)(2 * NW), wp = rank * NW + warp;
        if (n == 0) {
            ub = ue = C0 = C1 = U0;
        } else {
            ub = wp < Wp ? U0 + wp * n / Wp : U1;
            ue = wp < Wp ? U0 + (wp + 1) * n / Wp : U1;
            C0 = U0 + (rank * NW < Wp ? rank * NW : Wp) * n / Wp;
            C1 = U0 + ((rank + 1) * NW < Wp ? (rank + 1) * NW : Wp) * n / Wp;
        }
    } else {
        // warps past the W that share the list take no units
        const int64_t wid = (int64_t)blockIdx.x * NW + warp;
        ub = wid < W ? wid * S / W : S;
        ue = wid < W ? (wid + 1) * S / W : S;
        const int64_t cw0 = (int64_t)blockIdx.x * NW, cw1 = min(cw0 + NW, W);
        C0 = cw0 < W ? cw0 * S / W : S;
        C1 = cw0 < W ? cw1 * S / W : S;
    }
    const int u_begin = (int)ub;
    const int u_end = (int)ue;
    const int M = a.M;
    const uint64_t pol = l2_policy_evict_first();

    const bool has_work = u_begin < u_end;
    const int arr = lane >> 4, srow = lane & 15;     // this lane's row of the scale ring fill

    // compute cursor (problem cp, tile ct, superblock csb), weight-load cursor (pointer,
    // units left in its problem) and scale-fill cursor (row pointer, tile, superblock)
    int cp = 0;
    while (cp + 1 < a.count && u_begin >= a.p[cp + 1].unit_begin) cp++;
    int ct = 0, csb = 0;
    if (has_work) {
        const int lu = u_begin - (int)a.p[cp].unit_begin;
        ct = lu / (int)a.p[cp].ksb;
        csb = lu % (int)a.p[cp].ksb;
    }
    int lp = cp;
    const uint8_t* lptr = a.p[cp].packed + ((int64_t)ct * a.p[cp].ksb + csb) * (512 * B) + 16 * lane;
    int lleft = (int)(a.p[cp].n_tiles * a.p[cp].ksb) - (ct * (int)a.p[cp].ksb + csb);
    int sp = cp;
    int st_ = ct, ssb = csb;
    const uint16_t* sbase = (arr ? a.p[cp].zeros : a.p[cp].scales) + ((int64_t)ct * 16 + srow) * a.p[cp].ngroups;

    uint4 wb[D][B];
    auto load_next = [&](uint4 (&dst)[B]) {
#pragma unroll
        for (int i = 0; i < B; i++) dst[i] = ldg_stream(lptr + 512 * i, pol);
        lptr += 512 * B;
        if (--lleft == 0 && lp + 1 < a.count) {
            lp++;
            lptr = a.p[lp].packed + 16 * lane;
            lleft = (int)(a.p[lp].n_tiles * a.p[lp].ksb);
        }
    };
    // scale/zero ring: lane i copies, for one unit, row i mod 16 of the scales (i < 16)
    // or of the zeros into the warp's slot, rows interleaved [row][scales, zeros]
    constexpr int SCB = scale_slot_bytes(GROUP);
    uint8_t* sring = smem + a.sring + warp * kScaleRing * SCB;
    auto issue_scales = [&](int slot) {
        cp_async_ca<2 * NGC>(smem_u32(sring + slot * SCB + (srow * 2 + arr) * 2 * NGC), sbase + ssb * NGC);
        if (++ssb == a.p[sp].ksb) {
            ssb = 0;
            if (++st_ == a.p[sp].n_tiles && sp + 1 < a.count) {
                sp++;
                st_ = 0;
                sbase = (arr ? a.p[sp].zeros : a.p[sp].scales) + srow * a.p[sp].ngroups;
            } else {
                sbase += 16 * a.p[sp].ngroups;
            }
        }
    };
#pragma unroll 1
    for (int i = 0; i < kScaleRing; i++) {
        if (u_begin + i < u_end) issue_scales(i);
        cp_async_commit();
    }
    // prologue: the first D + PF units into L2.  Bulk prefetches hold no registers and block
    // no issue slot, so the wait and the activation prep start at once while HBM streams;
    // the register ring is filled (from L2) after the prep
    if (lane < D + PF && u_begin + lane < u_end && lleft > lane)
        l2_prefetch_bulk(lptr - 16 * lane + (int64_t)lane * (512 * B), 512 * B);
    // zeroed chunk that padded plane rows and tokens read instead of branching
    const int8_t* zero;
    if constexpr (SMEMP) {
        if (threadIdx.x < 16) reinterpret_cast<uint4*>(smem + a.szero)[threadIdx.x] = make_uint4(0, 0, 0, 0);
        zero = reinterpret_cast<const int8_t*>(smem + a.szero);
    } else {
        zero = pa.zero;
    }
    griddep_wait();
    if constexpr (SMEMP) {
        // this CTA's copy of the prepared activations: warp w takes chunks w, w + NW, ...
        // of every token of every slot (in pair mode the pair's 2 NW warps split them and
        // each chunk is stored into both CTAs), rotated by the CTA (pair) index so that the
        // CTAs do not all read the same lines of x at once (no divisions on the way)
        if (pairp) cluster_wait();
        const uint32_t peer = (blockIdx.x & 1) ^ 1u;
        const int pw = pairp ? 2 * NW : NW;
        const int pwi = pairp ? (int)(blockIdx.x & 1) * NW + warp : warp;
        const unsigned pidx = pairp ? blockIdx.x >> 1 : blockIdx.x;
        for (int si = 0; si < pa.count; si++) {
            const PrepSlot& Q = pa.s[si];
            const int kch = (int)(Q.k / kLdgChunk);
            const int k32 = (int)Q.k;
            const int rot = (int)(pidx % (unsigned)kch);
            for (int m = 0; m < M; m++) {
                const uint16_t* xm = Q.x + (int64_t)m * k32;
                int8_t* row_h = reinterpret_cast<int8_t*>(smem + Q.sp) + (int64_t)(2 * m) * k32;
                float* xs = reinterpret_cast<float*>(smem + Q.sx) + m * (k32 / GROUP);
                int* ex = reinterpret_cast<int*>(smem + Q.se) + m * kch;
                // a warp's chunks are independent: issue kPrepBatch loads of x together
                constexpr int PB = kPrepBatch;
                for (int cw0 = pwi; cw0 < kch; cw0 += pw * PB) {
                    uint4 raw[PB];
#pragma unroll
                    for (int j = 0; j < PB; j++) {
                        const int cw = cw0 + j * pw;
                        const int ch = cw + rot < kch ? cw + rot : cw + rot - kch;
                        if (cw < kch) raw[j] = prep_load(xm + ch * kLdgChunk, lane);
                    }
#pragma unroll
                    for (int j = 0; j < PB; j++) {
                        const int cw = cw0 + j * pw;
                        if (cw < kch) {
                            const int ch = cw + rot < kch ? cw + rot : cw + rot - kch;
                            const PrepOut r = prep_convert<GROUP, BF16>(raw[j]);
                            int8_t* ph = row_h + ch * kLdgChunk + plane_off(lane);
                            *reinterpret_cast<uint2*>(ph) = r.hi;
                            *reinterpret_cast<uint2*>(ph + k32) = r.lo;
                            constexpr int LPG = GROUP / 8;
                            float* px = xs + ch * (kLdgChunk / GROUP) + lane / LPG;
                            if (lane % LPG == 0) *px = (float)r.gsum;
                            if (lane == 0) ex[ch] = r.E;
                            if (pairp) {
                                st_cluster_u32x2(cluster_map_smem(smem_u32(ph), peer), r.hi);
                                st_cluster_u32x2(cluster_map_smem(smem_u32(ph + k32), peer), r.lo);
                                if (lane % LPG == 0)
                                    st_cluster_f32(cluster_map_smem(smem_u32(px), peer), (float)r.gsum);
                                if (lane == 0) st_cluster_s32(cluster_map_smem(smem_u32(ex + ch), peer), r.E);
                            }
                        }
                    }
                }
            }
        }
    }
    if (pairp) cluster_sync_all();        // both halves of the activations are in place
    else __syncthreads();
#pragma unroll
    for (int d = 0; d < D; d++)
        if (u_begin + d < u_end) load_next(wb[d]);
    const CtaFix fix = cta_fix_at(smem + a.sfix, NW, M);
    cta_fix_clear(fix, warp, lane);
    const int head_gtile = (int)a.p[cp].tile_begin + ct;

    // per-problem byte offsets, from one base, of this lane's plane rows, group sums and
    // exponents; padded rows and tokens point at the zero chunk with a zero stride
    const char* pbase = nullptr;
    int prow0[NB], xrow0[NB], erow0[NB], pstep[NB], xstep[NB];
    auto set_problem_bases = [&]() {
        const LdgProblem& P = a.p[cp];
        const PrepSlot& PS = pa.s[P.slot];
        const char* planes = SMEMP ? reinterpret_cast<const char*>(smem + PS.sp) : reinterpret_cast<const char*>(PS.planes);
        const char* xsum = SMEMP ? reinterpret_cast<const char*>(smem + PS.sx) : reinterpret_cast<const char*>(PS.xsum);
        const char* expo = SMEMP ? reinterpret_cast<const char*>(smem + PS.se) : reinterpret_cast<const char*>(PS.expo);
        pbase = planes;
        const int zoff = (int)(reinterpret_cast<const char*>(zero) - planes);
        const int xoff = (int)(xsum - planes), eoff = (int)(expo - planes);
#pragma unroll
        for (int nb = 0; nb < NB; nb++) {
            const int pl = 8 * nb + g;
            const bool pv = pl < 2 * M;
            prow0[nb] = pv ? pl * (int)P.k + 16 * c : zoff + 16 * c;
            pstep[nb] = pv ? kLdgChunk : 0;
            const int tok = 4 * nb + c;
            const bool tv = tok < M;
            xrow0[nb] = tv ? xoff + 4 * tok * (int)P.ngroups : zoff;
            erow0[nb] = tv ? eoff + 4 * tok * (int)P.ksb : zoff;
            xstep[nb] = tv ? 4 : 0;
        }
    };
    set_problem_bases();

    float acc[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; nb++) acc[nb][0] = acc[nb][1] = 0.0f;
    int tile_first_u = u_begin - csb;              // first unit of the tile being accumulated
    int rs = 0;                                    // ring slot of the unit being computed

    for (int base = u_begin; base < u_end; base += D) {
#pragma unroll
        for (int d = 0; d < D; d++) {
            const int u = base + d;
            if (u < u_end) {
                uint32_t lo[F::NLO], hi[F::NHI];
#pragma unroll
                for (int i = 0; i < G::W0; i++) {
                    lo[4 * i] = wb[d][i].x;
                    lo[4 * i + 1] = wb[d][i].y;
                    lo[4 * i + 2] = wb[d][i].z;
                    lo[4 * i + 3] = wb[d][i].w;
                }
#pragma unroll
                for (int i = 0; i < G::W1; i++) {
                    hi[4 * i] = wb[d][G::W0 + i].x;
                    hi[4 * i + 1] = wb[d][G::W0 + i].y;
                    hi[4 * i + 2] = wb[d][G::W0 + i].z;
                    hi[4 * i + 3] = wb[d][G::W0 + i].w;
                }
                if constexpr (G::W1 == 0) hi[0] = 0;
                // refill this register slot with the unit D ahead
                if (u + D < u_end) load_next(wb[d]);
                // scales and zeros of this unit's NGC groups, rows g and g+8, from the ring
                cp_async_wait<kScaleRing - 1>();
                __syncwarp();
                const uint16_t* sslot = reinterpret_cast<const uint16_t*>(sring + rs * SCB);
                uint32_t sz0[NGC], sz1[NGC];        // [scales NGC/2 words | zeros NGC/2 words]
                lds_halves_ldg<2 * NGC>(sslot + (2 * g) * NGC, sz0);
                lds_halves_ldg<2 * NGC>(sslot + (2 * (g + 8)) * NGC, sz1);
                // exponent of each token of this lane, this unit
                int E[NB];
#pragma unroll
                for (int nb = 0; nb < NB; nb++)
                    E[nb] = ld_prep<SMEMP>(reinterpret_cast<const int*>(pbase + erow0[nb] + csb * xstep[nb]));
                float cacc[NB][2];
#pragma unroll
                for (int nb = 0; nb < NB; nb++) cacc[nb][0] = cacc[nb][1] = 0.0f;
                int ci[NB][4];
                uint4 bq[NB];
                static_for<0, 8>([&](auto kap_c) {
                    constexpr int kap = decltype(kap_c)::value;
                    const uint32_t a0 = F::template reg<kap, 0, 0>(lo, hi);
                    const uint32_t a1 = F::template reg<kap, 1, 0>(lo, hi);
                    const uint32_t a2 = F::template reg<kap, 0, 1>(lo, hi);
                    const uint32_t a3 = F::template reg<kap, 1, 1>(lo, hi);
#pragma unroll
                    for (int nb = 0; nb < NB; nb++) {
                        // one 16-byte load holds the B fragments of k-steps kap and kap + 1
                        if constexpr (kap % 2 == 0)
                            bq[nb] = ld_plane16<SMEMP>(reinterpret_cast<const int8_t*>(pbase + prow0[nb] + csb * pstep[nb] +
                                                                                        64 * (kap / 2)));
                        const uint32_t b0 = kap % 2 ? bq[nb].z : bq[nb].x;
                        const uint32_t b1 = kap % 2 ? bq[nb].w : bq[nb].y;
                        if constexpr (kap % KPG == 0) mma_16832_u8s8_zc(ci[nb], a0, a1, a2, a3, b0, b1);
                        else mma_16832_u8s8(ci[nb], a0, a1, a2, a3, b0, b1);
                    }
                    if constexpr (kap % KPG == KPG - 1) {
                        constexpr int gi = kap / KPG;
                        constexpr int wz = NGC / 2 + gi / 2, ws = gi / 2, sh = 16 * (gi & 1);
                        const float sg = __half2float(__ushort_as_half((uint16_t)(sz0[ws] >> sh)));
                        const float sg8 = __half2float(__ushort_as_half((uint16_t)(sz1[ws] >> sh)));
                        const float zg = __half2float(__ushort_as_half((uint16_t)(sz0[wz] >> sh)));
                        const float zg8 = __half2float(__ushort_as_half((uint16_t)(sz1[wz] >> sh)));
#pragma unroll
                        for (int nb = 0; nb < NB; nb++) {
                            const float X = ld_prep<SMEMP>(
                                reinterpret_cast<const float*>(pbase + xrow0[nb] + (csb * NGC + gi) * xstep[nb]));
                            const float f0 = fmaf(-zg, X, (float)(256 * ci[nb][0] + ci[nb][1]));
                            const float f1 = fmaf(-zg8, X, (float)(256 * ci[nb][2] + ci[nb][3]));
                            cacc[nb][0] = fmaf(sg, f0, cacc[nb][0]);
                            cacc[nb][1] = fmaf(sg8, f1, cacc[nb][1]);
                        }
                    }
                });
                // the ring slot's values are consumed: refill it with the unit kScaleRing ahead
                __syncwarp();
                if (u + kScaleRing < u_end) issue_scales(rs);
                cp_async_commit();
                rs = rs + 1 == kScaleRing ? 0 : rs + 1;
#pragma unroll
                for (int nb = 0; nb < NB; nb++) {
                    const float sc = ldg_exp2i(E[nb]);
                    acc[nb][0] = fmaf(sc, cacc[nb][0], acc[nb][0]);
                    acc[nb][1] = fmaf(sc, cacc[nb][1], acc[nb][1]);
                }
                // the tile ends here, or this warp's slice does
                const LdgProblem& P = a.p[cp];
                if (csb == P.ksb - 1 || u == u_end - 1) {
                    const bool full = tile_first_u >= u_begin && csb == P.ksb - 1;
                    const int gt = (int)P.tile_begin + ct;
                    if (full) tile_store_full<NB>(acc, M, P.n, ct, P.y);
                    else cta_fix_put<NB>(fix, warp, gt == head_gtile ? 0 : 1, gt, acc, M);
#pragma unroll
                    for (int nb = 0; nb < NB; nb++) acc[nb][0] = acc[nb][1] = 0.0f;
                    tile_first_u = u + 1;
                }
                if (++csb == P.ksb) {
                    csb = 0;
                    if (++ct == P.n_tiles && cp + 1 < a.count) {
                        cp++;
                        ct = 0;
                        set_problem_bases();
                    }
                }
            }
        }
    }

    // ---- partial tiles: CTA sums in shared memory; a tile shared with another CTA goes
    // by ticket, or in pair mode across the cluster barrier to rank 0
    __syncthreads();
    auto info = [&](int T, int64_t& first_u, int64_t& units, uint16_t*& y, int64_t& n, int64_t& row0) {
        int q = 0;
        while (q + 1 < a.count && T >= a.p[q + 1].tile_begin) q++;
        const LdgProblem& Q = a.p[q];
        const int64_t t = T - Q.tile_begin;
        first_u = Q.unit_begin + t * Q.ksb;
        units = Q.ksb;
        y = Q.y;
        n = Q.n;
        row0 = t * 16;
    };
    PairKeep keep;
    cta_fix_finish<uint16_t>(fix, NW, warp, M, u_begin, C0, C1, S, W, blockIdx.x, a.partials, a.counters, a.maxc,
                             info, a.pair ? 1 + (int)(blockIdx.x & 1) : 0, &keep);
    if (a.pair) {
        __syncwarp();
        cluster_sync_all();          // every thread of both CTAs: no thread returns earlier
        pair_finish<uint16_t>(fix, M, keep, info);
    }
}

// ------------------------------------------------------------------ host side
// Units in flight per warp and warps per CTA (one CTA per SM, so that the activations are
// prepared once per SM).  16 warps (<= 128 registers a thread) with about 12 x 16 bytes in
// flight per lane where the registers allow it; otherwise 8 warps with twice the depth.
// Either way each SM keeps about 96 KB of weights in flight, twice what 1 us of HBM
// latency at full rate needs.
struct LdgShape {
    int D, NW;
};
constexpr LdgShape ldg_shape(int bits, int group, int nb) {
    const int d = bits == 2 ? 4 : bits == 3 ? 3 : bits == 4 ? 3 : 2;
    const bool wide = nb == 1 && !(group == 32 && bits >= 5);
    if (wide) return {(group == 32 && bits == 4) ? 2 : d, 16};
    return {nb >= 4 ? d + d / 2 : 2 * d, 8};
}

struct LdgPlan {
    int64_t total_units = 0, total_tiles = 0, total_warps = 0;
    int grid = 1, maxc = 2;
    bool pair = false;
};

// Pair mode: clusters of two CTAs that each get a whole number of tiles, so that no tile
// is shared outside a cluster and no GPU-scope ticket is left at the end of the launch;
// chosen for the 16-warp shapes of 4 bits or more when the grid is full and the largest
// pair has at most kPairSlack more units than the average.  (On the 8-warp shapes, and on
// the 2- and 3-bit ones, whose units are shorter, pairs measured slower than tickets.)
constexpr bool kLdgPairMode = true;
constexpr double kPairSlack = 0.06;

static LdgPlan plan_ldg(const int64_t* n, const int64_t* k, int count, int nw, int bits = 0) {
    LdgPlan pl;
    int64_t max_ksb = 1;
    for (int i = 0; i < count; i++) {
        const int64_t n_tiles = n[i] / 16;
        const int64_t ksb = k[i] / kLdgChunk;
        pl.total_units += n_tiles * ksb;
        pl.total_tiles += n_tiles;
        max_ksb = std::max(max_ksb, ksb);
    }
    // at least kMinUnitsPerWarp units a warp: small products then split each tile over
    // fewer warps (cheaper fixups) and still keep several units in flight per warp
    constexpr int64_t kMinUnitsPerWarp = 4;
    pl.grid = (int)std::max<int64_t>(
        1, std::min<int64_t>((int64_t)sm_count(), ceil_div(pl.total_units, nw * kMinUnitsPerWarp)));
    // no more warps than units: every participating warp then owns at least one unit,
    // so each warp counted as a contributor to a tile also arrives at its ticket
    pl.total_warps = std::min<int64_t>((int64_t)pl.grid * nw, std::max<int64_t>(pl.total_units, 1));
    // warps that share one tile: the slices are floor(w S / W), so a window of ksb units
    // meets at most ceil(ksb W / S) + 1 of them; one more slot of margin
    pl.maxc = (int)(ceil_div(max_ksb * pl.total_warps, std::max<int64_t>(pl.total_units, 1)) + 2);
    const int64_t P = sm_count() / 2;
    if (kLdgPairMode && nw == 16 && bits >= 4 && P >= 1 && pl.grid == sm_count() && pl.total_tiles >= P) {
        auto first_unit = [&](int64_t T) {
            int64_t u = 0;
            for (int i = 0; i < count; i++) {
                const int64_t nt = n[i] / 16, ksb = k[i] / kLdgChunk;
                if (T < nt) return u + T * ksb;
                T -= nt;
                u += nt * ksb;
            }
            return u;
        };
        int64_t worst = 0;
        for (int64_t p = 0; p < P; p++)
            worst = std::max(worst, first_unit((p + 1) * pl.total_tiles / P) - first_unit(p * pl.total_tiles / P));
        if ((double)worst * (double)P <= (1.0 + kPairSlack) * (double)pl.total_units) {
            pl.pair = true;
            pl.grid = (int)(2 * P);
        }
    }
    return pl;
}

// Workspace: ticket header, partial tiles, then per product the planes [2M][k], the
// group sums [M][k/32] (enough for every group size) and the exponents [M][k/256].

static size_t prep_bytes(int64_t k, int64_t M) {
    return al256((size_t)(2 * M * k)) + al256((size_t)(M * (k / 32) * 4)) + al256((size_t)(M * (k / kLdgChunk) * 4));
}

// The workspace is sized for the larger warp count (16 a CTA), which every shape fits.
size_t gemv_group_ldg_ws_bytes_multi(const int64_t* n, const int64_t* k, int count, int64_t M) {
    const LdgPlan pl = plan_ldg(n, k, count, 16);
    size_t b = kCounterBytes + al256((size_t)(pl.total_tiles * pl.maxc * 16 * M * 4));
    for (int i = 0; i < count; i++) b += prep_bytes(k[i], M);
    return b + 256;                                      // zero chunk
}

size_t gemv_group_ldg_ws_bytes(int64_t M, int64_t n, int64_t k) { return gemv_group_ldg_ws_bytes_multi(&n, &k, 1, M); }

bool gemv_group_ldg_supported(int64_t M, int64_t n, int64_t k, int bits, int group) {
    if (M < 1 || M > 16 || k % kLdgChunk != 0 || n % 16 != 0 || bits < 2 || bits > 6) return false;
    if (group != 32 && group != 64 && group != 128) return false;
    if ((k / group) % 8 != 0) return false;              // 16-byte aligned scale rows
    // 32-bit unit indices and prepared-activation offsets inside the kernel
    return n / 16 <= kMaxTiles && k <= ((int64_t)1 << 22);
}

// Shared memory a CTA may spend on prepared activations (two CTAs per SM share 228 KB).
constexpr int kLdgSmemBudget = 200 * 1024;     // one CTA per SM


template <int B, int GROUP, int NB>
static lbq_status launch_ldg_inst(int grid, bool smemp, bool bf16, int smem, cudaStream_t st, const LdgArgs& args,
                                  const PrepArgs& prep) {
    constexpr LdgShape sh = ldg_shape(B, GROUP, NB);
    if constexpr (NB == 1) {
        if (smemp) {
            constexpr auto kb = k_gemv_group_ldg<B, GROUP, NB, sh.D, sh.NW, true, true>;
            constexpr auto kh = k_gemv_group_ldg<B, GROUP, NB, sh.D, sh.NW, true, false>;
            const lbq_status s = bf16 ? ldg_smem_attr<kb>(kLdgSmemBudget) : ldg_smem_attr<kh>(kLdgSmemBudget);
            if (s != LBQ_OK) return s;
            return launch_pdl_cluster(bf16 ? kb : kh, grid, args.pair ? 2 : 1, sh.NW * 32, (size_t)smem, st, args, prep);
        }
    }
    constexpr auto kg = k_gemv_group_ldg<B, GROUP, NB, sh.D, sh.NW, false, false>;
    const lbq_status s = ldg_smem_attr<kg>(kLdgSmemBudget);
    if (s != LBQ_OK) return s;
    return launch_pdl_cluster(kg, grid, args.pair ? 2 : 1, sh.NW * 32, (size_t)smem, st, args, prep);
}

template <int B, int GROUP>
static lbq_status launch_ldg_nb(int NB, int grid, bool smemp, bool bf16, int smem, cudaStream_t st,
                                const LdgArgs& args, const PrepArgs& prep) {
    if (NB == 1) return launch_ldg_inst<B, GROUP, 1>(grid, smemp, bf16, smem, st, args, prep);
    if (NB == 2) return launch_ldg_inst<B, GROUP, 2>(grid, smemp, bf16, smem, st, args, prep);
    if (NB == 3) return launch_ldg_inst<B, GROUP, 3>(grid, smemp, bf16, smem, st, args, prep);
    return launch_ldg_inst<B, GROUP, 4>(grid, smemp, bf16, smem, st, args, prep);
}

template <int B>
static lbq_status launch_ldg_b(int group, int NB, int grid, bool smemp, bool bf16, int smem, cudaStream_t st,
                               const LdgArgs& args, const PrepArgs& prep) {
    if (group == 32) return launch_ldg_nb<B, 32>(NB, grid, smemp, bf16, smem, st, args, prep);
    if (group == 64) return launch_ldg_nb<B, 64>(NB, grid, smemp, bf16, smem, st, args, prep);
    return launch_ldg_nb<B, 128>(NB, grid, smemp, bf16, smem, st, args, prep);
}


lbq_status launch_gemv_group_ldg_multi(const lbq_gemv_problem* probs, int count, bool bf16, int64_t M, int bits,
                                       int group, void* ws, size_t ws_bytes, cudaStream_t st) {
    int64_t n[kMaxGemvProblems], k[kMaxGemvProblems];
    for (int i = 0; i < count; i++) {
        n[i] = probs[i].n;
        k[i] = probs[i].k;
    }
    const int NB = (int)((2 * M + 7) / 8);
    const LdgShape shape = ldg_shape(bits, group, NB);
    const LdgPlan pl = plan_ldg(n, k, count, shape.NW, bits);
    if (pl.total_units == 0) return LBQ_OK;
    if (ws == nullptr || ws_bytes < gemv_group_ldg_ws_bytes_multi(n, k, count, M)) return LBQ_ERR_WORKSPACE;
    if (pl.total_tiles > kMaxTiles || pl.total_units >= ((int64_t)1 << 31)) return LBQ_ERR_UNSUPPORTED;

    LdgArgs args;
    memset(&args, 0, sizeof args);
    PrepArgs prep;
    memset(&prep, 0, sizeof prep);
    char* base = (char*)ws;
    args.counters = (unsigned*)base;
    args.partials = (float*)(base + kCounterBytes);
    size_t off = kCounterBytes + al256((size_t)(pl.total_tiles * pl.maxc * 16 * M * 4));
    int64_t ub = 0, tb = 0, pw = 0;
    int soff = 0;
    for (int i = 0; i < count; i++) {
        // products that read the same activations share one prep slot
        int slot = -1;
        for (int j = 0; j < prep.count; j++)
            if (prep.s[j].x == (const uint16_t*)probs[i].x && prep.s[j].k == k[i]) slot = j;
        if (slot < 0) {
            PrepSlot& s = prep.s[prep.count];
            s.x = (const uint16_t*)probs[i].x;
            s.k = k[i];
            s.planes = (int8_t*)(base + off);
            s.xsum = (float*)(base + off + al256((size_t)(2 * M * k[i])));
            s.expo = (int*)(base + off + al256((size_t)(2 * M * k[i])) + al256((size_t)(M * (k[i] / 32) * 4)));
            s.sp = soff;
            s.sx = s.sp + al16(2 * M * k[i]);
            s.se = s.sx + al16(M * (k[i] / group) * 4);
            soff = s.se + al16(M * (k[i] / kLdgChunk) * 4);
            s.warp_begin = pw;
            pw += M * (k[i] / kLdgChunk);
            off += prep_bytes(k[i], M);
            slot = prep.count++;
        }
        LdgProblem& P = args.p[i];
        P.packed = (const uint8_t*)probs[i].packed;
        P.scales = (const uint16_t*)probs[i].scales;
        P.zeros = (const uint16_t*)probs[i].zeros;
        P.y = (uint16_t*)probs[i].y;
        P.slot = slot;
        P.n = n[i];
        P.k = k[i];
        P.ksb = k[i] / kLdgChunk;
        P.n_tiles = n[i] / 16;
        P.ngroups = k[i] / group;
        P.unit_begin = ub;
        P.tile_begin = tb;
        ub += P.n_tiles * P.ksb;
        tb += P.n_tiles;
    }
    prep.zero = (int8_t*)(base + off);                   // 256 zero bytes after the prep slots
    prep.total_warps = pw;
    prep.M = (int)M;
    args.total_units = pl.total_units;
    args.total_warps = pl.total_warps;
    args.total_tiles = pl.total_tiles;
    args.pair = pl.pair ? 1 : 0;
    args.count = count;
    args.M = (int)M;
    args.maxc = pl.maxc;

    // prepared activations in each CTA's shared memory when they fit, else one prep launch;
    // the scale/zero rings follow them (or start the shared memory)
    const int ring = shape.NW * kScaleRing * scale_slot_bytes(group);
    const int fixb = al16((int64_t)cta_fix_bytes(shape.NW, (int)M));
    const bool smemp = NB == 1 && soff + ring + 256 + fixb <= kLdgSmemBudget;
    args.sring = smemp ? al16(soff) : 0;
    args.szero = args.sring + ring;
    args.sfix = args.szero + 256;
    const int smem = args.sfix + fixb;
    if (!smemp) {
        const int pgrid = (int)ceil_div(pw, (int64_t)8);
        lbq_status s;
#define LBQ_PREP(GR) (bf16 ? launch_pdl(k_gemv_prep<GR, true>, pgrid, 256, 0, st, prep) \
                           : launch_pdl(k_gemv_prep<GR, false>, pgrid, 256, 0, st, prep))
        if (group == 32) s = LBQ_PREP(32);
        else if (group == 64) s = LBQ_PREP(64);
        else s = LBQ_PREP(128);
#undef LBQ_PREP
        if (s != LBQ_OK) return s;
    }
    switch (bits) {
        case 2: return launch_ldg_b<2>(group, NB, pl.grid, smemp, bf16, smem, st, args, prep);
        case 3: return launch_ldg_b<3>(group, NB, pl.grid, smemp, bf16, smem, st, args, prep);
        case 4: return launch_ldg_b<4>(group, NB, pl.grid, smemp, bf16, smem, st, args, prep);
        case 5: return launch_ldg_b<5>(group, NB, pl.grid, smemp, bf16, smem, st, args, prep);
        default: return launch_ldg_b<6>(group, NB, pl.grid, smemp, bf16, smem, st, args, prep);
    }
}

lbq_status launch_gemv_group_ldg(const void* x, bool bf16, int64_t M, const void* packed, const void* scales,
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
    return launch_gemv_group_ldg_multi(&p, 1, bf16, M, bits, group, ws, ws_bytes, st);
}

}  // namespace lbq
