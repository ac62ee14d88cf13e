// lbq_internal.h -- host-side launchers and layout geometry shared inside liblbq.
#pragma once
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>
#include "../../include/lbq.h"

namespace lbq {

unsigned* device_error_word();
int sm_count();

// Geometry of the fragment-interleaved group-code layout (LBQ_LAYOUT_KERNEL).
// A b-bit code is a low plane of W0 bits and a high plane of W1 = b - W0 bits.
// Rows come in tiles of 16 and k in superblocks of 256; one (tile, superblock)
// holds 512*b bytes: the low plane (W0 chunks of 512 B) then the high plane
// (W1 chunks).  In a plane of width w each 32-bit word holds O = 4/w "octets"
// (8 consecutive codes of one row) so that byte-masking the word yields the
// m16n8k32 u8 A-fragment registers of one lane.
template <int B>
struct GroupGeom {
    static constexpr int W0 = (B == 2 || B == 3) ? 2 : 4;
    static constexpr int W1 = B - W0;
    static constexpr int SB = 256;
    static constexpr int NB0 = W0;          // 512-byte chunks of the low plane
    static constexpr int NB1 = W1;
    static constexpr int NBLK = NB0 + NB1;
    static constexpr int SB_BYTES = 512 * B;
};

inline int64_t group_superblock(int bits) { return (bits >= 2 && bits <= 6) ? 256 : 0; }

inline int64_t sign_cols_pad(int64_t cols) { return (cols + 255) / 256 * 256; }
inline size_t al256(size_t v) { return (v + 255) / 256 * 256; }
inline int al16(int64_t v) { return (int)((v + 15) / 16 * 16); }

// Every workspace starts with a fixed header of ticket counters (one per 16-row
// tile, at most kMaxTiles).  It must be zero before the first call; every call
// leaves it zero.  The bytes after it are scratch, always written before read.
constexpr int64_t kMaxTiles = 16384;
constexpr int kMaxGemvProblems = LBQ_MAX_GEMV_PROBLEMS;
constexpr size_t kCounterBytes = (size_t)kMaxTiles * 4;

lbq_status launch_quantize_rtn(const void* W, bool bf16, int64_t n, int64_t k, int bits, int group,
                               uint8_t* codes, void* scales, void* zeros, cudaStream_t st);
lbq_status launch_pack(const uint8_t* codes, int64_t n, int64_t k, int bits, lbq_layout layout, void* packed,
                       cudaStream_t st);
lbq_status launch_unpack(const void* packed, int64_t n, int64_t k, int bits, lbq_layout layout, uint8_t* codes,
                         cudaStream_t st);
lbq_status launch_pack_signs(const int8_t* pm1, int64_t rows, int64_t cols, lbq_layout layout, void* out,
                             cudaStream_t st);
lbq_status launch_repack_signs(const uint32_t* canon, int64_t rows, int64_t cols, void* out, cudaStream_t st);

// Group GEMV (M <= 16).  ws layout and size: gemv_group_ws_bytes.
size_t gemv_group_ws_bytes(int64_t M, int64_t n, int64_t k, int bits, int group, lbq_layout layout);
lbq_status launch_gemv_group(const void* x, bool bf16, int64_t M, const void* packed, const void* scales,
                             const void* zeros, int64_t n, int64_t k, int bits, int group, lbq_layout layout,
                             void* y, void* ws, size_t ws_bytes, cudaStream_t st);

// Group GEMV with weights streamed into registers (M <= 16, kernel layout).
bool gemv_group_ldg_supported(int64_t M, int64_t n, int64_t k, int bits, int group);
size_t gemv_group_ldg_ws_bytes(int64_t M, int64_t n, int64_t k);
size_t gemv_group_ldg_ws_bytes_multi(const int64_t* n, const int64_t* k, int count, int64_t M);
lbq_status launch_gemv_group_ldg_multi(const lbq_gemv_problem* probs, int count, bool bf16, int64_t M, int bits,
                                       int group, void* ws, size_t ws_bytes, cudaStream_t st);
lbq_status launch_gemv_group_ldg(const void* x, bool bf16, int64_t M, const void* packed, const void* scales,
                                 const void* zeros, int64_t n, int64_t k, int bits, int group, void* y, void* ws,
                                 size_t ws_bytes, cudaStream_t st);

// Batched group GEMM on tcgen05 (M >= 64, kernel layout).
size_t gemm_group_tc_ws_bytes(int64_t M, int64_t n, int64_t k);
bool gemm_group_tc_supported(int64_t M, int64_t n, int64_t k, int bits, int group);
lbq_status launch_gemm_group_tc(const void* x, bool bf16, int64_t M, const void* packed, const void* scales,
                                const void* zeros, int64_t n, int64_t k, int bits, int group, void* y, void* ws,
                                size_t ws_bytes, cudaStream_t st);

// Binary low-rank GEMM on tcgen05 (M >= 64, sign kernel layout).
size_t gemm_binlr_tc_ws_bytes(int64_t M, int64_t d_out, int64_t d_in, int64_t r);
bool gemm_binlr_tc_supported(int64_t M, int64_t d_out, int64_t d_in, int64_t r);
lbq_status launch_gemm_binlr_tc(const void* x, bool bf16, int64_t M, const void* U, const void* Vt, const void* s1,
                                const void* s2, int64_t d_out, int64_t d_in, int64_t r, void* y, void* ws,
                                size_t ws_bytes, cudaStream_t st);

// Binary low-rank GEMV streaming the signs into registers (M <= 4, sign kernel layout).
bool gemv_binlr_ldg_supported(int64_t M, int64_t d_out, int64_t d_in, int64_t r);
size_t gemv_binlr_ldg_ws_bytes(int64_t M, int64_t d_out, int64_t d_in, int64_t r);
lbq_status launch_gemv_binlr_ldg(const void* x, bool bf16, int64_t M, const void* U, const void* Vt, const void* s1,
                                 const void* s2, int64_t d_out, int64_t d_in, int64_t r, void* y, void* ws,
                                 size_t ws_bytes, cudaStream_t st);

// Binary low-rank GEMV (M <= 16).
size_t gemv_binlr_ws_bytes(int64_t M, int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout);
lbq_status launch_gemv_binlr(const void* x, bool bf16, int64_t M, const void* U, const void* Vt, const void* s1,
                             const void* s2, int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout, void* y,
                             void* ws, size_t ws_bytes, cudaStream_t st);

}  // namespace lbq
