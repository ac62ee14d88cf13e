/*
 * lbq.h -- C ABI of liblbq: low-bit weight-only GEMV/GEMM for NVIDIA B200 (sm_100a).
 *
 * The library computes the decode-time product of an activation block x with a
 * compressed weight matrix, in two weight formats:
 *
 *  (1) group-wise RTN integers.  "Métodos de cuantización de LLM para ejecutar un
 *      modelo de 70B en una sola GPU" (gotburnout.io), section "RTN
 *      (Round-To-Nearest)": each weight is rounded to the nearest level of its
 *      grid with no calibration data.  "TurboQuant: cuantizar modelos grandes
 *      para que quepan en local" (quellm.com), section "Compresión por bloques":
 *      blocks of 32 or 64 weights share one scale and one offset (this library
 *      also takes 128); section "Asignación de bits por capa": the bit width is
 *      chosen per layer (2 to 6 bits here).
 *      Format: W[n x k] (out x in, row-major) -> codes q in [0, 2^b - 1],
 *      fp16 scale s and fp16 integer zero-point z per (row, group of g along k);
 *      dequantized weight  w_hat = s * (q - z).
 *
 *  (2) binary low-rank.  "70B en 4GB de VRAM: la compresión neural de 2026, ¿es
 *      real?" (nramos.dev), section "1. NanoQuant — sub-1-bit PTQ", bullet
 *      "Formulación": W ≈ s1 ⊙ (U±1 · V±1ᵀ) ⊙ s2ᵀ, computed here as
 *      y = s1 ⊙ U (Vᵀ (s2 ⊙ x)).  The same bullet list says the method ships its
 *      own binary GEMV/GEMM kernels; those are not used here.
 *
 * Conventions for every entry point:
 *  * All tensor arguments are DEVICE pointers on the current CUDA device; the
 *    caller allocates, owns and frees them.  The library never allocates, frees
 *    or synchronises (except lbq_last_device_error, which synchronises `stream`).
 *  * `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls are stream-ordered and may be captured into CUDA graphs.
 *  * Arguments are checked on the host before anything is launched; a bad
 *    argument returns an error status and launches nothing.  A launch failure
 *    returns LBQ_ERR_CUDA.  Kernels never trap: data errors they detect (a
 *    non-finite weight) set a device error word read by lbq_last_device_error.
 *  * Half-precision buffers hold IEEE binary16 (LBQ_F16) or bfloat16 (LBQ_BF16).
 *  * Row-major everywhere; sizes in elements unless stated.
 */
#ifndef LBQ_H
#define LBQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LBQ_OK = 0,
    LBQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bits or group */
    LBQ_ERR_UNSUPPORTED = 2,   /* valid but not implemented combination (e.g. layout vs shape) */
    LBQ_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    LBQ_ERR_WORKSPACE = 4,     /* workspace missing or smaller than lbq_workspace_bytes() */
    LBQ_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
    LBQ_ERR_TIMEOUT = 6,       /* a bounded device-side wait expired */
    LBQ_ERR_DEVICE = 7,        /* a kernel reported a data error (see lbq_last_device_error) */
    LBQ_ERR_SCRATCH_LIMIT = 8  /* the problem needs more scratch than the library's fixed buffer holds */
} lbq_status;

typedef enum { LBQ_F16 = 0, LBQ_BF16 = 1 } lbq_dtype;

/* LBQ_LAYOUT_CANONICAL: per row, an LSB-first bitstream of b-bit codes (bit t of
 *   code j at stream bit j*b + t; at b = 4 two codes per byte, low nibble first).
 *   Row stride k*b/8 bytes.  Needs k % 32 == 0.  Sign matrices: element c at bit
 *   c%32 of 32-bit word c/32, bit 1 meaning +1, row stride cols/32 words.
 * LBQ_LAYOUT_KERNEL: the same bits permuted into the tensor-core fragment order
 *   the fast kernels read with one 128-bit load per lane (index maps in the
 *   DESIGN notes "Kernel layout" and "Kernel layout, signs").  Group codes need
 *   n % 16 == 0 and k % SB == 0 with SB = 64 (b=4), 128 (b=2,6), 256 (b=3,5);
 *   sign matrices need rows % 16 == 0 and are padded to a multiple of 256
 *   columns. */
typedef enum { LBQ_LAYOUT_CANONICAL = 0, LBQ_LAYOUT_KERNEL = 1 } lbq_layout;

typedef enum {
    LBQ_OP_GEMV_GROUP = 0,
    LBQ_OP_GEMM_GROUP = 1,
    LBQ_OP_GEMV_BINLR = 2,
    LBQ_OP_GEMM_BINLR = 3
} lbq_op;

/* Bytes of packed codes for an [n x k] matrix of b-bit codes (n*k*b/8 in both
 * layouts), or 0 if the shape is not supported by `layout`. */
size_t lbq_packed_bytes(int64_t n, int64_t k, int bits, lbq_layout layout);

/* Group-wise asymmetric round-to-nearest quantization (RTN section of the
 * gotburnout.io page; shared per-block scale and offset of the quellm.com page).
 * For every row i and group j of `group` consecutive k:
 *   lo = min(0, min w), hi = max(0, max w)           (fp32, exact)
 *   s  = fp16_round_up((hi - lo) / (2^b - 1))        (fp32 IEEE division; s = 1 if 0)
 *   z  = clamp(rint(-lo / s), 0, 2^b - 1)            (stored as fp16)
 *   q  = clamp(rint(w / s) + z, 0, 2^b - 1)          (rint = round half to even)
 * so that |w - s*(q - z)| <= s/2.
 * W: [n x k] f16 or bf16.  codes: [n x k] u8.  scales, zeros: [n x k/group] f16.
 * bits in 2..6, group in {32, 64, 128}, k % group == 0.  W, scales, zeros must be
 * 2-byte aligned.  A non-finite weight sets the device error word (its group's
 * outputs are unspecified). */
lbq_status lbq_quantize_rtn(const void* W, lbq_dtype w_dtype, int64_t n, int64_t k,
                            int bits, int group, uint8_t* codes, void* scales,
                            void* zeros, void* stream);

/* Bit-pack u8 codes [n x k] (values < 2^bits) into `layout`.  packed must hold
 * lbq_packed_bytes() bytes and be 16-byte aligned; codes 16-byte aligned. */
lbq_status lbq_pack(const uint8_t* codes, int64_t n, int64_t k, int bits,
                    lbq_layout layout, void* packed, void* stream);

/* Inverse of lbq_pack (used to check layouts; not on the hot path). */
lbq_status lbq_unpack(const void* packed, int64_t n, int64_t k, int bits,
                      lbq_layout layout, uint8_t* codes, void* stream);

/* Bytes of a packed [rows x cols] sign matrix in `layout`. */
size_t lbq_sign_packed_bytes(int64_t rows, int64_t cols, lbq_layout layout);

/* Pack a +-1 int8 matrix [rows x cols] (cols % 32 == 0) into `layout`
 * (binary factors U and V^T of the nramos.dev page's "Formulación" bullet). */
lbq_status lbq_pack_signs(const int8_t* pm1, int64_t rows, int64_t cols,
                          lbq_layout layout, void* out, void* stream);

/* Re-lay canonical sign words [rows x cols/32] u32 into LBQ_LAYOUT_KERNEL. */
lbq_status lbq_repack_signs(const uint32_t* canonical, int64_t rows, int64_t cols,
                            void* out_kernel, void* stream);

/* Workspace bytes needed by `op` for the given sizes on the current device
 * (n = output rows, k = input features, r = rank; unused sizes are ignored).
 * The workspace is caller-owned device memory.  Its first 64 KiB hold ticket
 * counters: they must be zero before the first call (zero-fill the buffer once)
 * and every call leaves them zero again, so one workspace serves every op and
 * shape in turn.  The rest is scratch.  Calls that share a workspace must not
 * run concurrently (use one workspace per stream). */
size_t lbq_workspace_bytes(lbq_op op, int64_t M, int64_t n, int64_t k, int64_t r);

/* Dequant-fused group GEMV, y[m, i] = sum_k x[m, k] * s[i, k/g] * (q[i, k] - z[i, k/g]),
 * fp32 accumulation, for M = 1..16 tokens.  This is the hot loop of decode
 * ("AirLLM corre un modelo 70B en una GPU de 4GB...", section "Por qué es lento":
 * time per token is model bytes over read bandwidth, so fewer bytes per weight
 * means proportionally faster decode).
 * x: [M x k] in x_dtype (f16 or bf16); y: [M x n] f16 (fp16 outputs for either
 * activation type).  packed in `layout` (lbq_pack),
 * scales/zeros [n x k/group] f16 as written by lbq_quantize_rtn.  x, packed,
 * scales, zeros 16-byte aligned (LBQ_LAYOUT_KERNEL) or 4-byte (canonical).
 * ws: lbq_workspace_bytes(LBQ_OP_GEMV_GROUP, M, n, k, 0) bytes.
 * Launches of the kernel layout use one CTA per SM and, when they fill the GPU, may run
 * as thread-block clusters of two CTAs (no CTA of a launch waits for another cluster).
 * Results are deterministic: every split sum is added in a fixed order. */
lbq_status lbq_gemv_group(const void* x, lbq_dtype x_dtype, int64_t M,
                          const void* packed, const void* scales, const void* zeros,
                          int64_t n, int64_t k, int bits, int group, lbq_layout layout,
                          void* y, void* ws, size_t ws_bytes, void* stream);

/* One product of a grouped GEMV launch.  All products of one launch share M, the
 * activation dtype, the bit width and the group size; each has its own shapes. */
typedef struct {
    const void* x;        /* [M x k] activations (x_dtype), 16-byte aligned */
    const void* packed;   /* codes of W [n x k] in LBQ_LAYOUT_KERNEL, 16-byte aligned */
    const void* scales;   /* [n x k/group] f16, 16-byte aligned */
    const void* zeros;    /* [n x k/group] f16, 16-byte aligned */
    void* y;              /* [M x n] f16 output */
    int64_t n, k;         /* n % 16 == 0, k % 256 == 0, (k/group) % 8 == 0 */
} lbq_gemv_problem;

#define LBQ_MAX_GEMV_PROBLEMS 8

/* Grouped group GEMV: computes every product of `problems` (1..LBQ_MAX_GEMV_PROBLEMS)
 * in ONE launch, e.g. the q/k/v or gate/up projections of a decoder block, which
 * read the same activations (the fused decode step of the dojofullstack page's
 * "El truco, en un párrafo": a block's layers run one after another, so the GEMVs
 * that do not depend on each other can share a launch).  Same arithmetic, layout and
 * error rules as lbq_gemv_group with LBQ_LAYOUT_KERNEL; the launches of one stream
 * overlap their ramp with the previous kernel's tail, so packed weights, scales and
 * zeros must not be written by a kernel that signals programmatic completion early.
 * ws: lbq_gemv_group_multi_workspace_bytes(problems, count, M) bytes. */
size_t lbq_gemv_group_multi_workspace_bytes(const lbq_gemv_problem* problems, int count, int64_t M);
lbq_status lbq_gemv_group_multi(const lbq_gemv_problem* problems, int count, lbq_dtype x_dtype, int64_t M,
                                int bits, int group, void* ws, size_t ws_bytes, void* stream);

/* Group GEMV for callers that cannot allocate device memory where they multiply
 * (engine plugins handed no workspace, code running after a pool allocator has
 * reserved all device memory, host callbacks on a stream, where CUDA API calls are not
 * allowed).  The pages describe no such variant; this is a library convenience.
 * Same arguments, arithmetic and rules as lbq_gemv_group with LBQ_LAYOUT_KERNEL, but
 * no workspace: the scratch lives in a fixed 8 MiB device array owned by the library,
 * which every GPU that loads the library holds until exit.  The first call on each
 * device looks up the array's address (make that first call before any stream
 * capture).  Problems needing more scratch than the array holds (lbq_workspace_bytes
 * of the kernel path above 8 MiB, e.g. M = 16 on very wide layers) return
 * LBQ_ERR_SCRATCH_LIMIT.  Every call uses the same array, so calls that overlap on the
 * GPU (other streams, or other host threads) race and must be serialised by the
 * caller.  It allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
lbq_status lbq_gemv_group_noalloc(const void* x, lbq_dtype x_dtype, int64_t M, const void* packed,
                                  const void* scales, const void* zeros, int64_t n, int64_t k, int bits,
                                  int group, void* y, void* stream);

/* Same product for any M >= 1 (prefill / batched decode; the batching of the
 * dojofullstack page's "trabajo batch offline" section, where one loaded layer
 * serves many prompts).  M >= 64 with LBQ_LAYOUT_KERNEL uses the tcgen05
 * tensor-core path (weights dequantized into shared memory); smaller M runs the
 * GEMV kernels over blocks of 16 tokens. */
lbq_status lbq_gemm_group(const void* x, lbq_dtype x_dtype, int64_t M,
                          const void* packed, const void* scales, const void* zeros,
                          int64_t n, int64_t k, int bits, int group, lbq_layout layout,
                          void* y, void* ws, size_t ws_bytes, void* stream);

/* Binary low-rank GEMV (nramos.dev page, "Formulación" bullet):
 *   y = s1 ⊙ U (V^T (s2 ⊙ x))  for M = 1..16 tokens.
 * U: [d_out x r] signs, Vt = V^T: [r x d_in] signs, both packed in `layout`
 * (canonical: u32 words, bit 1 = +1).  s1 [d_out], s2 [d_in] f16.
 * x: [M x d_in] in x_dtype, y: [M x d_out] f16.  r % 32 == 0, d_in % 32 == 0.
 * The LBQ_LAYOUT_KERNEL path converts s2 ⊙ x and the intermediate t to 16-bit
 * fixed point with one power-of-two scale per token and 256-column chunk (integer
 * tensor cores, exact int32 sums per chunk); relative error of y stays below 1e-3.
 * ws: lbq_workspace_bytes(LBQ_OP_GEMV_BINLR, M, d_out, d_in, r) bytes. */
lbq_status lbq_gemv_binlr(const void* x, lbq_dtype x_dtype, int64_t M,
                          const void* U, const void* Vt, const void* s1, const void* s2,
                          int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout,
                          void* y, void* ws, size_t ws_bytes, void* stream);

/* Same for any M >= 1.  M >= 64 with LBQ_LAYOUT_KERNEL runs two tcgen05 GEMMs
 * (fp16 +-1 signs expanded in shared memory, fp32 accumulation in tensor memory):
 * t = V^T (s2 ⊙ x) kept in fp16 in the workspace, then y = s1 ⊙ (U t).  Other
 * cases run the GEMV path over blocks of 16 tokens.
 * ws: lbq_workspace_bytes(LBQ_OP_GEMM_BINLR, M, d_out, d_in, r) bytes. */
lbq_status lbq_gemm_binlr(const void* x, lbq_dtype x_dtype, int64_t M,
                          const void* U, const void* Vt, const void* s1, const void* s2,
                          int64_t d_out, int64_t d_in, int64_t r, lbq_layout layout,
                          void* y, void* ws, size_t ws_bytes, void* stream);

/* Fixed per-layer bit allocation for an n_layers-deep Llama-2-70B-shaped stack
 * (quellm.com page, "Asignación de bits por capa": 5-6 bits for attention, 2 for
 * MLP, 2.7-3.2 bits per weight on average).  proj: 0 q, 1 k, 2 v, 3 o, 4 gate,
 * 5 up, 6 down.  Attention: 6 bits in the first and last 8 layers, else 5; MLP:
 * 3 bits on even layers, 2 on odd ones.  Returns 0 for a bad argument. */
int lbq_schedule_bits(int layer, int proj, int n_layers);

/* Synchronises `stream`, returns the device error word of the current device
 * in *code (0 = none; bit 0: non-finite weight seen by lbq_quantize_rtn;
 * bit 1: a bounded wait expired) and clears it. */
lbq_status lbq_last_device_error(void* stream, int* code);

const char* lbq_status_string(lbq_status status);

/* Library version string ("major.minor.patch"). */
const char* lbq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LBQ_H */
