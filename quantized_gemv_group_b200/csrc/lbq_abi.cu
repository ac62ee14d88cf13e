// lbq_abi.cu -- the extern "C" boundary of liblbq: argument checks and dispatch.
// Every check happens on the host before anything is launched (see include/lbq.h).
#include <mutex>
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

constexpr int kMaxDevices = 64;
__device__ unsigned g_error_word;   // one per device (each device gets its own copy)

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    unsigned* err = nullptr;
};
static DeviceInfo g_dev[kMaxDevices];
static std::mutex g_dev_mu;

static DeviceInfo& dev_info() {
    int d = 0;
    cudaGetDevice(&d);
    if (d < 0 || d >= kMaxDevices) d = 0;
    DeviceInfo& info = g_dev[d];
    if (!info.ready) {
        std::lock_guard<std::mutex> lock(g_dev_mu);
        if (!info.ready) {
            cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, d);
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_error_word) == cudaSuccess) info.err = (unsigned*)p;
            info.ready = true;
        }
    }
    return info;
}

unsigned* device_error_word() { return dev_info().err; }
int sm_count() {
    const int s = dev_info().sms;
    return s > 0 ? s : 148;
}

static bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }
static bool valid_bits(int b) { return b >= 2 && b <= 6; }
static bool valid_group(int g) { return g == 32 || g == 64 || g == 128; }

static lbq_status check_group_gemv_args(const void* x, int64_t M, const void* packed, const void* scales,
                                        const void* zeros, int64_t n, int64_t k, int bits, int group,
                                        lbq_layout layout, const void* y) {
    if (M < 0 || n < 0 || k <= 0) return LBQ_ERR_INVALID_ARG;
    if (!valid_bits(bits) || !valid_group(group) || k % group != 0) return LBQ_ERR_INVALID_ARG;
    if (layout != LBQ_LAYOUT_CANONICAL && layout != LBQ_LAYOUT_KERNEL) return LBQ_ERR_INVALID_ARG;
    if (M == 0 || n == 0) return LBQ_OK;
    if (!x || !packed || !scales || !zeros || !y) return LBQ_ERR_INVALID_ARG;
    if (layout == LBQ_LAYOUT_KERNEL) {
        if (n % 16 != 0 || k % group_superblock(bits) != 0 || n / 16 > kMaxTiles) return LBQ_ERR_UNSUPPORTED;
        if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(scales, 16) || !aligned(zeros, 16))
            return LBQ_ERR_MISALIGNED;
    } else {
        if (!aligned(x, 4) || !aligned(packed, 4) || !aligned(scales, 2) || !aligned(zeros, 2))
            return LBQ_ERR_MISALIGNED;
    }
    if (!aligned(y, 2)) return LBQ_ERR_MISALIGNED;
    return LBQ_OK;
}

static lbq_status check_binlr_args(const void* x, int64_t M, const void* U, const void* Vt, const void* s1,
                                   const void* s2, int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout,
                                   const void* y) {
    if (M < 0 || d_out < 0 || d_in <= 0 || r <= 0) return LBQ_ERR_INVALID_ARG;
    if (r % 32 != 0 || d_in % 32 != 0) return LBQ_ERR_INVALID_ARG;
    if (layout != LBQ_LAYOUT_CANONICAL && layout != LBQ_LAYOUT_KERNEL) return LBQ_ERR_INVALID_ARG;
    if (M == 0 || d_out == 0) return LBQ_OK;
    if (!x || !U || !Vt || !s1 || !s2 || !y) return LBQ_ERR_INVALID_ARG;
    if (layout == LBQ_LAYOUT_KERNEL && d_out % 16 != 0) return LBQ_ERR_UNSUPPORTED;
    if (!aligned(U, 16) || !aligned(Vt, 16) || !aligned(x, 4) || !aligned(s1, 2) || !aligned(s2, 2) ||
        !aligned(y, 2))
        return LBQ_ERR_MISALIGNED;
    return LBQ_OK;
}

}  // namespace lbq

using namespace lbq;

extern "C" {

const char* lbq_version(void) { return "0.1.0"; }

const char* lbq_status_string(lbq_status s) {
    switch (s) {
        case LBQ_OK: return "ok";
        case LBQ_ERR_INVALID_ARG: return "invalid argument";
        case LBQ_ERR_UNSUPPORTED: return "unsupported combination of arguments";
        case LBQ_ERR_MISALIGNED: return "misaligned pointer";
        case LBQ_ERR_WORKSPACE: return "workspace missing or too small";
        case LBQ_ERR_CUDA: return "CUDA error";
        case LBQ_ERR_TIMEOUT: return "bounded device wait expired";
        case LBQ_ERR_DEVICE: return "kernel reported a data error";
        case LBQ_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the fixed buffer holds";
    }
    return "unknown status";
}

size_t lbq_packed_bytes(int64_t n, int64_t k, int bits, lbq_layout layout) {
    if (n < 0 || k < 0 || !valid_bits(bits) || k % 32 != 0) return 0;
    if (layout == LBQ_LAYOUT_KERNEL && (n % 16 != 0 || k % group_superblock(bits) != 0)) return 0;
    if (layout != LBQ_LAYOUT_KERNEL && layout != LBQ_LAYOUT_CANONICAL) return 0;
    return (size_t)(n * k * bits / 8);
}

lbq_status lbq_quantize_rtn(const void* W, lbq_dtype w_dtype, int64_t n, int64_t k, int bits, int group,
                            uint8_t* codes, void* scales, void* zeros, void* stream) {
    if (n < 0 || k < 0 || !valid_bits(bits) || !valid_group(group) || k % group != 0) return LBQ_ERR_INVALID_ARG;
    if (w_dtype != LBQ_F16 && w_dtype != LBQ_BF16) return LBQ_ERR_INVALID_ARG;
    if (n == 0 || k == 0) return LBQ_OK;
    if (!W || !codes || !scales || !zeros) return LBQ_ERR_INVALID_ARG;
    if (!aligned(W, 2) || !aligned(scales, 2) || !aligned(zeros, 2)) return LBQ_ERR_MISALIGNED;
    if (!device_error_word()) return LBQ_ERR_CUDA;
    return launch_quantize_rtn(W, w_dtype == LBQ_BF16, n, k, bits, group, codes, scales, zeros,
                               (cudaStream_t)stream);
}

lbq_status lbq_pack(const uint8_t* codes, int64_t n, int64_t k, int bits, lbq_layout layout, void* packed,
                    void* stream) {
    if (n < 0 || k < 0 || !valid_bits(bits) || k % 32 != 0) return LBQ_ERR_INVALID_ARG;
    if (layout != LBQ_LAYOUT_CANONICAL && layout != LBQ_LAYOUT_KERNEL) return LBQ_ERR_INVALID_ARG;
    if (n == 0 || k == 0) return LBQ_OK;
    if (!codes || !packed) return LBQ_ERR_INVALID_ARG;
    if (layout == LBQ_LAYOUT_KERNEL && (n % 16 != 0 || k % group_superblock(bits) != 0)) return LBQ_ERR_UNSUPPORTED;
    if (!aligned(codes, 16) || !aligned(packed, 16)) return LBQ_ERR_MISALIGNED;
    return launch_pack(codes, n, k, bits, layout, packed, (cudaStream_t)stream);
}

lbq_status lbq_unpack(const void* packed, int64_t n, int64_t k, int bits, lbq_layout layout, uint8_t* codes,
                      void* stream) {
    if (n < 0 || k < 0 || !valid_bits(bits) || k % 32 != 0) return LBQ_ERR_INVALID_ARG;
    if (layout != LBQ_LAYOUT_CANONICAL && layout != LBQ_LAYOUT_KERNEL) return LBQ_ERR_INVALID_ARG;
    if (n == 0 || k == 0) return LBQ_OK;
    if (!codes || !packed) return LBQ_ERR_INVALID_ARG;
    if (layout == LBQ_LAYOUT_KERNEL && (n % 16 != 0 || k % group_superblock(bits) != 0)) return LBQ_ERR_UNSUPPORTED;
    if (!aligned(codes, 16) || !aligned(packed, 16)) return LBQ_ERR_MISALIGNED;
    return launch_unpack(packed, n, k, bits, layout, codes, (cudaStream_t)stream);
}

size_t lbq_sign_packed_bytes(int64_t rows, int64_t cols, lbq_layout layout) {
    if (rows < 0 || cols < 0 || cols % 32 != 0) return 0;
    if (layout == LBQ_LAYOUT_CANONICAL) return (size_t)(rows * cols / 8);
    if (layout == LBQ_LAYOUT_KERNEL) return rows % 16 ? 0 : (size_t)(rows * sign_cols_pad(cols) / 8);
    return 0;
}

lbq_status lbq_pack_signs(const int8_t* pm1, int64_t rows, int64_t cols, lbq_layout layout, void* out,
                          void* stream) {
    if (rows < 0 || cols < 0 || cols % 32 != 0) return LBQ_ERR_INVALID_ARG;
    if (layout != LBQ_LAYOUT_CANONICAL && layout != LBQ_LAYOUT_KERNEL) return LBQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return LBQ_OK;
    if (!pm1 || !out) return LBQ_ERR_INVALID_ARG;
    if (layout == LBQ_LAYOUT_KERNEL && rows % 16 != 0) return LBQ_ERR_UNSUPPORTED;
    if (!aligned(pm1, 16) || !aligned(out, 16)) return LBQ_ERR_MISALIGNED;
    return launch_pack_signs(pm1, rows, cols, layout, out, (cudaStream_t)stream);
}

lbq_status lbq_repack_signs(const uint32_t* canonical, int64_t rows, int64_t cols, void* out_kernel, void* stream) {
    if (rows < 0 || cols < 0 || cols % 32 != 0) return LBQ_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return LBQ_OK;
    if (!canonical || !out_kernel) return LBQ_ERR_INVALID_ARG;
    if (rows % 16 != 0) return LBQ_ERR_UNSUPPORTED;
    if (!aligned(canonical, 4) || !aligned(out_kernel, 16)) return LBQ_ERR_MISALIGNED;
    return launch_repack_signs(canonical, rows, cols, out_kernel, (cudaStream_t)stream);
}

size_t lbq_workspace_bytes(lbq_op op, int64_t M, int64_t n, int64_t k, int64_t r) {
    if (M <= 0) return 0;
    switch (op) {
        case LBQ_OP_GEMV_GROUP: {
            size_t best = kCounterBytes;
            for (int b = 2; b <= 6; b++)
                for (int g = 32; g <= 128; g *= 2)
                    if (k % group_superblock(b) == 0 && k % g == 0 && n % 16 == 0)
                        best = std::max(best, gemv_group_ws_bytes(std::min<int64_t>(M, 16), n, k, b, g,
                                                                  LBQ_LAYOUT_KERNEL));
            return best;
        }
        case LBQ_OP_GEMM_GROUP: {
            size_t best = lbq_workspace_bytes(LBQ_OP_GEMV_GROUP, std::min<int64_t>(M, 16), n, k, r);
            if (M >= 64) best = std::max(best, gemm_group_tc_ws_bytes(M, n, k));
            return best;
        }
        case LBQ_OP_GEMV_BINLR:
        case LBQ_OP_GEMM_BINLR: {
            const int64_t m = std::min<int64_t>(M, 16);
            size_t best = std::max(gemv_binlr_ws_bytes(m, n, k, r, LBQ_LAYOUT_KERNEL),
                                   gemv_binlr_ws_bytes(m, n, k, r, LBQ_LAYOUT_CANONICAL));
            if (op == LBQ_OP_GEMM_BINLR && M >= 64) best = std::max(best, gemm_binlr_tc_ws_bytes(M, n, k, r));
            return best;
        }
    }
    return 0;
}

lbq_status lbq_gemv_group(const void* x, lbq_dtype x_dtype, int64_t M, const void* packed, const void* scales,
                          const void* zeros, int64_t n, int64_t k, int bits, int group, lbq_layout layout, void* y,
                          void* ws, size_t ws_bytes, void* stream) {
    if (M > 16 || (x_dtype != LBQ_F16 && x_dtype != LBQ_BF16)) return LBQ_ERR_INVALID_ARG;
    const lbq_status s = check_group_gemv_args(x, M, packed, scales, zeros, n, k, bits, group, layout, y);
    if (s != LBQ_OK || M == 0 || n == 0) return s;
    return launch_gemv_group(x, x_dtype == LBQ_BF16, M, packed, scales, zeros, n, k, bits, group, layout, y, ws,
                             ws_bytes, (cudaStream_t)stream);
}

static lbq_status check_multi(const lbq_gemv_problem* problems, int count, lbq_dtype x_dtype, int64_t M,
                              int bits, int group) {
    if (!problems || count < 1 || count > LBQ_MAX_GEMV_PROBLEMS) return LBQ_ERR_INVALID_ARG;
    if (M < 0 || M > 16 || (x_dtype != LBQ_F16 && x_dtype != LBQ_BF16)) return LBQ_ERR_INVALID_ARG;
    int64_t tiles = 0;
    for (int i = 0; i < count; i++) {
        const lbq_gemv_problem& p = problems[i];
        const lbq_status s =
            check_group_gemv_args(p.x, M, p.packed, p.scales, p.zeros, p.n, p.k, bits, group, LBQ_LAYOUT_KERNEL, p.y);
        if (s != LBQ_OK) return s;
        if (M > 0 && p.n > 0 && !gemv_group_ldg_supported(M, p.n, p.k, bits, group)) return LBQ_ERR_UNSUPPORTED;
        tiles += p.n / 16;
    }
    return tiles > kMaxTiles ? LBQ_ERR_UNSUPPORTED : LBQ_OK;
}

size_t lbq_gemv_group_multi_workspace_bytes(const lbq_gemv_problem* problems, int count, int64_t M) {
    if (!problems || count < 1 || count > LBQ_MAX_GEMV_PROBLEMS || M <= 0) return 0;
    int64_t n[LBQ_MAX_GEMV_PROBLEMS], k[LBQ_MAX_GEMV_PROBLEMS];
    for (int i = 0; i < count; i++) {
        n[i] = problems[i].n;
        k[i] = problems[i].k;
    }
    return gemv_group_ldg_ws_bytes_multi(n, k, count, std::min<int64_t>(M, 16));
}

lbq_status lbq_gemv_group_multi(const lbq_gemv_problem* problems, int count, lbq_dtype x_dtype, int64_t M, int bits,
                                int group, void* ws, size_t ws_bytes, void* stream) {
    const lbq_status s = check_multi(problems, count, x_dtype, M, bits, group);
    if (s != LBQ_OK || M == 0) return s;
    lbq_gemv_problem live[LBQ_MAX_GEMV_PROBLEMS];
    int nlive = 0;
    for (int i = 0; i < count; i++)
        if (problems[i].n > 0) live[nlive++] = problems[i];
    if (nlive == 0) return LBQ_OK;
    return launch_gemv_group_ldg_multi(live, nlive, x_dtype == LBQ_BF16, M, bits, group, ws, ws_bytes,
                                       (cudaStream_t)stream);
}

lbq_status lbq_gemm_group(const void* x, lbq_dtype x_dtype, int64_t M, const void* packed, const void* scales,
                          const void* zeros, int64_t n, int64_t k, int bits, int group, lbq_layout layout, void* y,
                          void* ws, size_t ws_bytes, void* stream) {
    if (x_dtype != LBQ_F16 && x_dtype != LBQ_BF16) return LBQ_ERR_INVALID_ARG;
    const lbq_status s = check_group_gemv_args(x, M, packed, scales, zeros, n, k, bits, group, layout, y);
    if (s != LBQ_OK || M == 0 || n == 0) return s;
    const bool bf16 = x_dtype == LBQ_BF16;
    if (M >= 64 && layout == LBQ_LAYOUT_KERNEL && gemm_group_tc_supported(M, n, k, bits, group))
        return launch_gemm_group_tc(x, bf16, M, packed, scales, zeros, n, k, bits, group, y, ws, ws_bytes,
                                    (cudaStream_t)stream);
    // token blocks of 16 through the GEMV kernels (weights are re-read per block)
    for (int64_t m0 = 0; m0 < M; m0 += 16) {
        const int64_t mb = std::min<int64_t>(16, M - m0);
        const lbq_status r = launch_gemv_group((const uint16_t*)x + m0 * k, bf16, mb, packed, scales, zeros, n, k,
                                               bits, group, layout, (uint16_t*)y + m0 * n, ws, ws_bytes,
                                               (cudaStream_t)stream);
        if (r != LBQ_OK) return r;
    }
    return LBQ_OK;
}

lbq_status lbq_gemv_binlr(const void* x, lbq_dtype x_dtype, int64_t M, const void* U, const void* Vt, const void* s1,
                          const void* s2, int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout, void* y,
                          void* ws, size_t ws_bytes, void* stream) {
    if (M > 16 || (x_dtype != LBQ_F16 && x_dtype != LBQ_BF16)) return LBQ_ERR_INVALID_ARG;
    const lbq_status s = check_binlr_args(x, M, U, Vt, s1, s2, d_out, d_in, r, layout, y);
    if (s != LBQ_OK || M == 0 || d_out == 0) return s;
    return launch_gemv_binlr(x, x_dtype == LBQ_BF16, M, U, Vt, s1, s2, d_out, d_in, r, layout, y, ws, ws_bytes,
                             (cudaStream_t)stream);
}

lbq_status lbq_gemm_binlr(const void* x, lbq_dtype x_dtype, int64_t M, const void* U, const void* Vt, const void* s1,
                          const void* s2, int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout, void* y,
                          void* ws, size_t ws_bytes, void* stream) {
    if (x_dtype != LBQ_F16 && x_dtype != LBQ_BF16) return LBQ_ERR_INVALID_ARG;
    const lbq_status s = check_binlr_args(x, M, U, Vt, s1, s2, d_out, d_in, r, layout, y);
    if (s != LBQ_OK || M == 0 || d_out == 0) return s;
    if (M >= 64 && layout == LBQ_LAYOUT_KERNEL && gemm_binlr_tc_supported(M, d_out, d_in, r))
        return launch_gemm_binlr_tc(x, x_dtype == LBQ_BF16, M, U, Vt, s1, s2, d_out, d_in, r, y, ws, ws_bytes,
                                    (cudaStream_t)stream);
    for (int64_t m0 = 0; m0 < M; m0 += 16) {
        const int64_t mb = std::min<int64_t>(16, M - m0);
        const lbq_status st = launch_gemv_binlr((const uint16_t*)x + m0 * d_in, x_dtype == LBQ_BF16, mb, U, Vt, s1,
                                                s2, d_out, d_in, r, layout, (uint16_t*)y + m0 * d_out, ws, ws_bytes,
                                                (cudaStream_t)stream);
        if (st != LBQ_OK) return st;
    }
    return LBQ_OK;
}

int lbq_schedule_bits(int layer, int proj, int n_layers) {
    if (n_layers <= 0 || layer < 0 || layer >= n_layers || proj < 0 || proj > 6) return 0;
    if (proj <= 3) return (layer < 8 || layer >= n_layers - 8) ? 6 : 5;
    return (layer % 2 == 0) ? 3 : 2;
}

lbq_status lbq_last_device_error(void* stream, int* code) {
    if (!code) return LBQ_ERR_INVALID_ARG;
    unsigned* err = device_error_word();
    if (!err) return LBQ_ERR_CUDA;
    unsigned v = 0;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&v, err, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess) return LBQ_ERR_CUDA;
    if (cudaMemsetAsync(err, 0, sizeof v, st) != cudaSuccess) return LBQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return LBQ_ERR_CUDA;
    *code = (int)v;
    return LBQ_OK;
}

}  // extern "C"
