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

// ------------------------------------------------------------------ tile epilogue
// A warp owns a 16-row tile; acc[nb][0] is row g and acc[nb][1] row g+8 of token
// 4*nb + c.  If the CTA covered the tile's whole k-range (full) the result is stored
// directly; otherwise it is written to this CTA's partial slot and the last of the
// `count` contributing CTAs (atomic ticket) sums the slots in CTA order, stores y and
// resets the ticket.  The row block's units are [first_u, first_u + units_per_rb) of
// the launch's unit list, split evenly over NC CTAs (start(b) = b * S_total / NC);
// `gtile` indexes the launch-wide ticket and partial arrays, `tile` the rows of y.
// Y is uint16_t (fp16 output) or float.
__device__ __forceinline__ void store_out(uint16_t* p, float v) { *p = from_f32<false>(v); }
__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }

template <int NB, class Y>
__device__ __forceinline__ void tile_epilogue_any(const float (&acc)[NB][2], bool full, int M, int64_t n, int64_t tile,
                                                  int64_t gtile, int64_t first_u, int64_t units_per_rb,
                                                  int64_t S_total, int64_t NC, int64_t cta, float* __restrict__ partials,
                                                  unsigned* __restrict__ counters, int maxc, Y* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int64_t row_g = tile * 16 + g;
    if (full) {
#pragma unroll
        for (int nb = 0; nb < NB; nb++) {
            const int tok = 4 * nb + c;
            if (tok < M) {
                store_out(y + (int64_t)tok * n + row_g, acc[nb][0]);
                store_out(y + (int64_t)tok * n + row_g + 8, acc[nb][1]);
            }
        }
        return;
    }
    const int64_t last_u = first_u + units_per_rb - 1;
    const int64_t own_first = ((first_u + 1) * NC - 1) / S_total;
    const int64_t own_last = ((last_u + 1) * NC - 1) / S_total;
    const int count = (int)(own_last - own_first + 1);
    const int slot = (int)(cta - own_first);
    float* pslot = partials + ((gtile * maxc) + slot) * (int64_t)(16 * M);
#pragma unroll
    for (int nb = 0; nb < NB; nb++) {
        const int tok = 4 * nb + c;
        if (tok < M) {
            __stcg(pslot + tok * 16 + g, acc[nb][0]);
            __stcg(pslot + tok * 16 + g + 8, acc[nb][1]);
        }
    }
    __syncwarp();
    unsigned old = 0;
    if (lane == 0) {
        __threadfence();
        old = atomicAdd(counters + gtile, 1u);
    }
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old == (unsigned)(count - 1)) {
        __threadfence();
        const float* p0 = partials + (gtile * maxc) * (int64_t)(16 * M);
        // The slots' loads are independent: issue them in batches of 8 so that their L2
        // latencies overlap, and add the slots in their fixed order.
        for (int e = lane; e < 16 * M; e += 32) {
            float s = 0.0f;
            int sl = 0;
            for (; sl + 8 <= count; sl += 8) {
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; j++) v[j] = __ldcg(p0 + (sl + j) * (int64_t)(16 * M) + e);
#pragma unroll
                for (int j = 0; j < 8; j++) s += v[j];
            }
            for (; sl < count; sl++) s += __ldcg(p0 + sl * (int64_t)(16 * M) + e);
            store_out(y + (int64_t)(e / 16) * n + tile * 16 + (e % 16), s);
        }
        __syncwarp();
        if (lane == 0) counters[gtile] = 0u;
    }
}

template <int NB>
__device__ __forceinline__ void tile_epilogue(const float (&acc)[NB][2], bool full, int M, int64_t n, int64_t tile,
                                              int64_t gtile, int64_t first_u, int64_t units_per_rb, int64_t S_total,
                                              int64_t NC, int64_t cta, float* __restrict__ partials,
                                              unsigned* __restrict__ counters, int maxc, uint16_t* __restrict__ y) {
    tile_epilogue_any<NB, uint16_t>(acc, full, M, n, tile, gtile, first_u, units_per_rb, S_total, NC, cta, partials,
                                    counters, maxc, y);
}
template <int NB>
__device__ __forceinline__ void tile_epilogue_f32(const float (&acc)[NB][2], bool full, int M, int64_t n,
                                                  int64_t tile, int64_t gtile, int64_t first_u, int64_t units_per_rb,
                                                  int64_t S_total, int64_t NC, int64_t cta, float* __restrict__ partials,
                                                  unsigned* __restrict__ counters, int maxc, float* __restrict__ y) {
    tile_epilogue_any<NB, float>(acc, full, M, n, tile, gtile, first_u, units_per_rb, S_total, NC, cta, partials,
                                 counters, maxc, y);
}

}  // namespace lbq
