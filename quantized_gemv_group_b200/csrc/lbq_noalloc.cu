// lbq_noalloc.cu -- group GEMV entry point that allocates nothing and takes no workspace.
//
// For callers that cannot allocate device memory at the point where they multiply:
// engine plugins whose interface hands them no workspace, code that runs after a pool
// allocator has reserved all device memory at start-up, or a host callback on a CUDA
// stream, where CUDA API calls such as cudaMalloc are not permitted.  Such callers
// cannot provide the scratch that lbq_gemv_group needs (split-K tickets and partial
// sums), so this entry point keeps that scratch in a fixed array in device memory
// that the library owns.
//
// The array (kScratchBytes, 8 MiB) is a file-scope __device__ variable: every GPU that
// loads the library holds it until the process exits.  Host code cannot use the
// array's name as a device address, so the first call on each device looks the address
// up with cudaGetSymbolAddress (with that device current) and caches it.
#include <mutex>
#include "lbq_common.cuh"
#include "lbq_internal.h"

namespace lbq {

constexpr size_t kScratchBytes = (size_t)8 << 20;       // counters header + partial sums
static_assert(kScratchBytes > kCounterBytes, "scratch must hold the ticket counters");

static __device__ __align__(256) unsigned char g_gemv_scratch[kScratchBytes];

struct ScratchSlot {
    bool ready = false;
    void* ptr = nullptr;
};
static ScratchSlot g_scratch[64];
static std::mutex g_scratch_mu;

// Device address of this device's scratch array (set up on the first call per device).
static void* scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot& s = g_scratch[dev];
    if (!s.ready) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_gemv_scratch) != cudaSuccess) return nullptr;
        s.ptr = p;
        s.ready = true;
    }
    return s.ptr;
}

}  // namespace lbq

using namespace lbq;

extern "C" lbq_status lbq_gemv_group_noalloc(const void* x, lbq_dtype x_dtype, int64_t M, const void* packed,
                                             const void* scales, const void* zeros, int64_t n, int64_t k, int bits,
                                             int group, void* y, void* stream) {
    if (M < 0 || M > 16 || (x_dtype != LBQ_F16 && x_dtype != LBQ_BF16)) return LBQ_ERR_INVALID_ARG;
    if (n < 0 || k <= 0 || bits < 2 || bits > 6 || (group != 32 && group != 64 && group != 128) || k % group)
        return LBQ_ERR_INVALID_ARG;
    if (M == 0 || n == 0) return LBQ_OK;
    if (!x || !packed || !scales || !zeros || !y) return LBQ_ERR_INVALID_ARG;
    if (!gemv_group_ldg_supported(M, n, k, bits, group)) return LBQ_ERR_UNSUPPORTED;
    const uintptr_t al = (uintptr_t)x | (uintptr_t)packed | (uintptr_t)scales | (uintptr_t)zeros;
    if ((al % 16) != 0 || ((uintptr_t)y % 2) != 0) return LBQ_ERR_MISALIGNED;
    const size_t need = gemv_group_ldg_ws_bytes(M, n, k);
    if (need > kScratchBytes) return LBQ_ERR_SCRATCH_LIMIT;
    void* ws = scratch_address();
    if (!ws) return LBQ_ERR_CUDA;
    // The tickets of the row blocks this call uses must start at zero.  A call leaves
    // them zero, but the array keeps whatever the previous call left, so clear them.
    const size_t used_counters = (size_t)(n / 16) * sizeof(unsigned);
    if (cudaMemsetAsync(ws, 0, used_counters, (cudaStream_t)stream) != cudaSuccess) return LBQ_ERR_CUDA;
    return launch_gemv_group_ldg(x, x_dtype == LBQ_BF16, M, packed, scales, zeros, n, k, bits, group, y, ws,
                                 kScratchBytes, (cudaStream_t)stream);
}
