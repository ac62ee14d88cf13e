// lbq_group_frag.cuh -- fragment helpers for the group GEMV kernels (sm_100a).
#pragma once
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

// ------------------------------------------------------------------ u8 A fragments
// Lane words of one (tile, 256-k superblock): lo[4*W0] low-plane words and
// hi[4*W1] high-plane words (see GroupGeom).  reg<KAPPA, U, E>() is the
// m16n8k32 A register of k-step KAPPA (32 k), row half U (0: row g, 1: row g+8),
// code parity E (0: codes 0,2,4,6 of the lane's octet -> k-slots 4c..4c+3,
// 1: codes 1,3,5,7 -> k-slots 4c+16..4c+19), one code per byte.
template <int B>
struct IFrag {
    using G = GroupGeom<B>;
    static constexpr int W0 = G::W0, W1 = G::W1;
    static constexpr int NLO = 4 * W0;
    static constexpr int NHI = W1 > 0 ? 4 * W1 : 1;
    static constexpr uint32_t LOMASK = ((1u << W0) - 1u) * 0x01010101u;
    static constexpr uint32_t HIMASK = (((1u << (W1 > 0 ? W1 : 1)) - 1u) << W0) * 0x01010101u;

    template <int KAPPA, int U, int E>
    __device__ __forceinline__ static uint32_t reg(const uint32_t (&lo)[NLO], const uint32_t (&hi)[NHI]) {
        constexpr int eta = 2 * KAPPA + U;
        constexpr int O0 = 4 / W0;
        uint32_t r = shift_right_signed<2 * W0 * (eta % O0) + W0 * E>(lo[eta / O0]) & LOMASK;
        if constexpr (W1 > 0) {
            constexpr int O1 = 4 / W1;
            r = and_or(shift_right_signed<2 * W1 * (eta % O1) + W1 * E - W0>(hi[eta / O1]), HIMASK, r);
        }
        return r;
    }
};

// ------------------------------------------------------------------ tile stores
// A warp owns a 16-row tile; acc[nb][0] is row g and acc[nb][1] row g+8 of token 4*nb + c.
// Y is uint16_t (fp16 output) or float.
__device__ __forceinline__ void store_out(uint16_t* p, float v) { *p = from_f32<false>(v); }
__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }

// ------------------------------------------------------------------ CTA-level tile finish
// Warp-level stream-K over a CTA's contiguous unit range leaves each warp at most two
// partial tiles: the tile of its first unit (slot 0) and, if different, the tile of its
// last unit (slot 1).  The warps park those partial sums in shared memory; after one CTA
// barrier the CTA's first contributing warp of each tile adds them in warp order.  A tile
// that lies inside the CTA's range is stored at once; one shared with other CTAs goes
// through the global ticket (the last of its CTAs adds the CTA sums in CTA order), so at
// most two tiles per CTA pay for a GPU-scope atomic, and the sum order is fixed.
//
// Pair mode (clusters of two CTAs, each pair given a whole number of tiles) has no
// GPU-scope ticket: the one tile the pair's two CTAs share is finished by rank 0, which
// receives rank 1's sum in its shared memory (recv) across the cluster barrier.
struct CtaFix {
    float* val;     // [NW][2][16 * M] partial sums, element tok * 16 + row
    int* tile;      // [NW][2] tile index of each slot, -1 if unused
    float* recv;    // [16 * M] pair mode: rank 1's sum of the shared tile (in rank 0)
};

__host__ __device__ __forceinline__ size_t cta_fix_bytes(int nw, int M) {
    return (size_t)nw * 2 * 16 * M * 4 + (size_t)nw * 2 * 4 + (size_t)16 * M * 4;
}
__device__ __forceinline__ CtaFix cta_fix_at(uint8_t* base, int nw, int M) {
    CtaFix f;
    f.val = reinterpret_cast<float*>(base);
    f.recv = reinterpret_cast<float*>(base + (size_t)nw * 2 * 16 * M * 4);
    f.tile = reinterpret_cast<int*>(base + (size_t)nw * 2 * 16 * M * 4 + (size_t)16 * M * 4);
    return f;
}
// Rank 0's share of the pair's shared tile, kept in registers across the cluster barrier.
struct PairKeep {
    int T = -1;
    float v[8];     // elements lane, lane + 32, ... (16 * M <= 256)
};
__device__ __forceinline__ void cta_fix_clear(const CtaFix& f, int warp, int lane) {
    if (lane < 2) f.tile[warp * 2 + lane] = -1;
}
// Park a warp's partial tile (fragment layout above) in slot k.
template <int NB>
__device__ __forceinline__ void cta_fix_put(const CtaFix& f, int warp, int k, int64_t tile, const float (&acc)[NB][2],
                                            int M) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    float* v = f.val + (warp * 2 + k) * 16 * M;
#pragma unroll
    for (int nb = 0; nb < NB; nb++) {
        const int tok = 4 * nb + c;
        if (tok < M) {
            v[tok * 16 + g] = acc[nb][0];
            v[tok * 16 + g + 8] = acc[nb][1];
        }
    }
    if (lane == 0) f.tile[warp * 2 + k] = (int)tile;
}
// Store a full tile straight from the fragments.
template <int NB, class Y>
__device__ __forceinline__ void tile_store_full(const float (&acc)[NB][2], int M, int64_t n, int64_t tile, Y* y) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int nb = 0; nb < NB; nb++) {
        const int tok = 4 * nb + c;
        if (tok < M) {
            store_out(y + (int64_t)tok * n + tile * 16 + g, acc[nb][0]);
            store_out(y + (int64_t)tok * n + tile * 16 + g + 8, acc[nb][1]);
        }
    }
}
// After the CTA barrier: finish the tiles this warp owns.  info(T, first_u, units, y, n, row0)
// describes tile T: its units [first_u, first_u + units) in the launch's unit list, and the
// output rows y[tok * n + row0 + 0..15].  The launch's W warps split S units evenly
// (warp w: [w S / W, (w + 1) S / W)), NW per CTA; u_begin is this warp's first unit,
// [C0, C1) the CTA's range and cta its index.
// pair: 0 = tickets, 1 = pair mode in rank 0 (the shared tile goes to keep), 2 = pair mode
// in rank 1 (the shared tile's sum is stored into rank 0's recv).
template <class Y, class Info>
__device__ __forceinline__ void cta_fix_finish(const CtaFix& f, int NW, int warp, int M, int64_t u_begin, int64_t C0,
                                               int64_t C1, int64_t S, int64_t W, int64_t cta,
                                               float* __restrict__ partials, unsigned* __restrict__ counters, int maxc,
                                               Info info, int pair = 0, PairKeep* keep = nullptr) {
    const int lane = threadIdx.x & 31;
    const int E = 16 * M;
#pragma unroll 1
    for (int k = 0; k < 2; k++) {
        const int T = f.tile[warp * 2 + k];
        if (T < 0) continue;
        int64_t first_u, units, n, row0;
        Y* y;
        info(T, first_u, units, y, n, row0);
        if (k == 0 && warp > 0 && first_u < u_begin) continue;   // an earlier warp of this CTA owns it
        int w_end = warp + 1;
        while (w_end < NW && f.tile[w_end * 2] == T) w_end++;
        const bool inside = first_u >= C0 && first_u + units <= C1;
        if (!inside && pair != 0) {
            const uint32_t rr = pair == 2 ? cluster_map_smem(smem_u32(f.recv), 0) : 0u;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int e = lane + 32 * j;
                if (e < E) {
                    float s = f.val[(warp * 2 + k) * E + e];
                    for (int w2 = warp + 1; w2 < w_end; w2++) s += f.val[(w2 * 2) * E + e];
                    if (pair == 2) st_cluster_f32(rr + 4u * (uint32_t)e, s);
                    else keep->v[j] = s;
                }
            }
            if (pair == 1) keep->T = T;
            continue;
        }
        int64_t cf = 0, count = 1;
        float* p0 = nullptr;
        if (!inside) {
            cf = (((first_u + 1) * W - 1) / S) / NW;
            const int64_t cl = (((first_u + units) * W - 1) / S) / NW;
            count = cl - cf + 1;
            p0 = partials + (int64_t)T * maxc * E;
        }
        for (int e = lane; e < E; e += 32) {
            float s = f.val[(warp * 2 + k) * E + e];
            for (int w2 = warp + 1; w2 < w_end; w2++) s += f.val[(w2 * 2) * E + e];
            if (inside) store_out(y + (int64_t)(e / 16) * n + row0 + (e % 16), s);
            else __stcg(p0 + (cta - cf) * E + e, s);
        }
        if (inside) continue;
        __syncwarp();
        unsigned old = 0;
        if (lane == 0) old = atomic_add_acq_rel_gpu(counters + T, 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == (unsigned)(count - 1)) {
            __syncwarp();   // orders every lane's slot loads after lane 0's acquire
            // the slots' loads are independent: batches of 8, added in CTA order
            for (int e = lane; e < E; e += 32) {
                float s = 0.0f;
                int sl = 0;
                for (; sl + 8 <= count; sl += 8) {
                    float v[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) v[j] = __ldcg(p0 + (sl + j) * (int64_t)E + e);
#pragma unroll
                    for (int j = 0; j < 8; j++) s += v[j];
                }
                for (; sl < count; sl++) s += __ldcg(p0 + sl * (int64_t)E + e);
                store_out(y + (int64_t)(e / 16) * n + row0 + (e % 16), s);
            }
            __syncwarp();
            if (lane == 0) counters[T] = 0u;
        }
    }
}

// Pair mode, after the cluster barrier: rank 0 adds rank 1's sum and stores the shared tile.
template <class Y, class Info>
__device__ __forceinline__ void pair_finish(const CtaFix& f, int M, const PairKeep& keep, Info info) {
    if (keep.T < 0) return;
    const int lane = threadIdx.x & 31;
    int64_t first_u, units, n, row0;
    Y* y;
    info(keep.T, first_u, units, y, n, row0);
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const int e = lane + 32 * j;
        if (e < 16 * M) store_out(y + (int64_t)(e / 16) * n + row0 + (e % 16), keep.v[j] + f.recv[e]);
    }
}

}  // namespace lbq
