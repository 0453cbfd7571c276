/*
 * qgemm: low-bit mixed-precision matrix multiplication for NVIDIA B200 (sm_100a).
 *
 *     C[M, N] = A[M, K] . dequant(W[N, K])^T        ("nt": A and W both K-contiguous)
 *
 * Operand types follow the BitBLAS Matmul benchmark configuration listing
 * (microsoft/BitBLAS issue #252, "Default Backend Should be changed into tilelang",
 * op_configs and the MatmulConfig tuple M, N, K, A_dtype, W_dtype, out_dtype, accum_dtype,
 * layout "nt", group_size, with_scaling, with_zeros):
 *   W4A16  fp16 activations x unsigned int4 weights with per-group fp16 scale and optional
 *          fp16 zero point, fp32 accumulation, fp16 output;
 *   W8A8   int8 x int8, int32 accumulation and int32 output (an int8 dot product returns
 *          int32: triton-lang/triton PR #3595, "Convert INT8 MMAV2 accumulator layout",
 *          review discussion);
 *   W2A8   int8 activations x two's-complement int2 weights, int32 accumulation and output;
 *   dense  fp16 x fp16 with fp32 accumulation, fp16 output (the in-library baseline).
 * Parallel-k (split-K) follows hidet-org/hidet issue #364, "Multi-stage software pipelining
 * and update parallel k rule": the K reduction is cut into split_k parts whose partial results
 * are added into C with atomic red.global instructions.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers owned by the caller (for example PyTorch tensors); the
 *     library never frees or retains them. All operands are row-major and densely packed.
 *   - Calls are asynchronous and ordered on `stream` (0 = legacy default stream).
 *   - Arguments are validated before any work is queued; on error nothing is launched and
 *     no memory is touched. Launch failures return QG_ERR_CUDA. Errors raised by a kernel
 *     after it started (a bounded wait that ran out) are reported by qgemm_sync_check().
 *   - split_k > 1 makes the call zero C on `stream` first, then add each part into it
 *     atomically; fp16 results then depend on the (unspecified) order of the additions,
 *     int32 results do not. split_k <= 0 selects the tuned or heuristic value for the shape;
 *     for W4A16 at M <= 16 that may be the persistent path (QG_PATH_STREAM), which also zeroes
 *     C and adds partial row blocks atomically. split_k >= 1 keeps to paths that split K into
 *     exactly that many parts.
 *   - The library allocates no per-call memory. It allocates once per device at first use a
 *     4-byte device error word; qgemm_tune() allocates nothing either (it times the caller's
 *     buffers).
 *   - Nothing throws across this interface.
 *   - Every pointer argument named below must be 16-byte aligned, except scales and zeros
 *     (2-byte aligned).
 */
#ifndef QGEMM_H_
#define QGEMM_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum qg_status {
    QG_OK = 0,
    QG_ERR_INVALID_ARG = 1,       /* null pointer, non-positive size, bad flag value        */
    QG_ERR_ALIGNMENT = 2,         /* a pointer is not aligned as required                  */
    QG_ERR_UNSUPPORTED_SHAPE = 3, /* K or group_size violates the divisibility rules       */
    QG_ERR_CUDA = 4,              /* a CUDA runtime call or a kernel launch failed          */
    QG_ERR_DEVICE_TIMEOUT = 5,    /* a kernel gave up a bounded wait (qgemm_sync_check)     */
    QG_ERR_NOT_SM100 = 6,         /* the current device is not compute capability 10.0     */
    QG_ERR_BAD_CONFIG = 7,        /* a config passed to qgemm_set_config cannot run        */
    QG_ERR_SCRATCH_TOO_SMALL = 8  /* the problem needs more than the fixed scratch buffer   */
} qg_status;

typedef enum qg_op {
    QG_OP_W4A16 = 0,
    QG_OP_W8A8 = 1,
    QG_OP_W2A8 = 2,
    QG_OP_DENSE_F16 = 3,
    QG_OP_W4A16_INTERLEAVED = 4,  /* W4A16 with weights from quant_pack_int4_interleaved */
    QG_OP_W2A8_INTERLEAVED = 5    /* W2A8 with weights from quant_pack_int2_interleaved  */
} qg_op;

typedef enum qg_path {
    QG_PATH_AUTO = 0, /* let the library choose                                               */
    QG_PATH_GEMV = 1, /* small-M streaming kernels (weights read once with 128-bit loads)      */
    QG_PATH_TC = 2,   /* tcgen05 tensor-core GEMM with a TMA multi-stage pipeline (large M)   */
    QG_PATH_STREAM = 3 /* W4A16, M <= 16: persistent grid, every CTA streams an equal run of
                          (row block, K stage) units through a TMA ring (a copy warp keeps it
                          full, a prep warp turns the activations into MMA operands); partial
                          row blocks meet in C through atomics (C is zeroed first). Fields:
                          rows (16 rows per consumer warp), bk (256, 512 or 1024 K values a
                          stage), stages (ring depth, 2..16), bm (row warps WR, <= 16), bn (K
                          warps WK sharing a row block: 1, 2 or 4, dividing bk / 128;
                          WR * WK <= 14); split_k unused. */
} qg_path;

/* One launch configuration. Fields a path does not use are ignored (set them to 0). */
typedef struct qgemm_config_t {
    int32_t path;    /* qg_path                                                             */
    int32_t rows;    /* GEMV: weight rows per warp (16, 32 or 64 for W4A16; 1..8 otherwise).
                        TC (one CTA per tile, split_k = 1): 1 = stream-K schedule: the
                        (tile, K) work is cut into one equal share per persistent CTA and
                        partial tiles are added into the zeroed output (fp16 / int32 atomics,
                        so fp16 results can differ in the last bits from run to run); not for
                        qgemm_w8a8_requant. 0 = one whole tile (or K part) per work unit.   */
    int32_t bm;      /* TC: tile extent along the MMA's M: 128 (one CTA), or 256 for the
                        weight-major tile shared by a CTA pair (one cta_group::2 MMA over
                        two SMs: 256 weight rows, bn = 128 or 256 tokens, stages 3, 4, 5 or 8) */
    int32_t bn;      /* TC: tile extent along the MMA's N. GEMV (W4A16, stages > 0):
                        1 = one token, exact fp16 products summed in fp32 on the FMA pipe;
                        2 = 1..8 tokens on the packed fp16 FMA pipe (rows 32 or 64 per CTA,
                        stages 2..6, group size a multiple of 128): products of the centred
                        codes summed in fp16 over 16 per lane and K run of 32, fp32 across
                        runs, so the absolute error grows with |A| (keep |A| < 512)        */
    int32_t bk;      /* TC: tile extent along K                                              */
    int32_t stages;  /* TC: activation ring depth (2..5; 8 for bn <= 128, 16 for bn <= 64;
                        2..4 when swap_ab = 0; 2 or 4 half-tile stages when bn = 512)         */
    int32_t split_k; /* number of K parts (1 = no atomics)                                   */
    int32_t swap_ab; /* TC: 1 = weights fill the MMA's M side (bm = 128 weight rows), tokens
                        its N side (bn = 16..256 tokens, or 512 for packed W4A16 / W2A8:
                        two 256-token accumulators that share each upcast weight slab, no
                        double-buffered accumulator); 0 = token-major, W4A16 with a group
                        size that is a multiple of 64: bm = 128 tokens, bn = 256 weight rows
                        (an MMA from shared memory reaches its full rate only at N = 256)    */
} qgemm_config_t;

/* ---- matmuls ----------------------------------------------------------------------------- */

/*
 * W4A16. A: fp16 [M, K]. Wq: uint32 [N, K/8], code k of row n at bits 4*(k%8) of word k/8
 * (unsigned 0..15). scales, zeros: fp16 [N, G], G = K / group_size; zeros must be NULL iff
 * has_zero == 0 (then z = 0). C: fp16 [M, N].
 *     C[m, n] = sum_k A[m, k] * (q[n, k] - z[n, k/gs]) * s[n, k/gs]
 * accumulated in fp32, rounded to fp16 (round-to-nearest-even).
 * group_size: a multiple of 32 that divides K, or -1 / 0 for one group spanning K.
 * Requires K % 32 == 0.
 */
qg_status qgemm_w4a16(const void *A, const uint32_t *Wq, const void *scales, const void *zeros,
                      void *C, int M, int N, int K, int group_size, int split_k, int has_zero,
                      cudaStream_t stream);

/*
 * W4A16 with weights in the interleaved (pre-shuffled) layout that quant_pack_int4_interleaved
 * writes: within each uint32 word the codes k = 8j .. 8j+7 sit in nibbles 0, 4, 1, 5, 2, 6, 3, 7
 * (nibbles 0..7 hold codes 0, 2, 4, 6, 1, 3, 5, 7), so that the upcast finds codes adjacent in k
 * in nibbles i and i+4 and needs no byte permutes. Everything else as qgemm_w4a16; the result
 * is that of qgemm_w4a16 on the naturally packed weights of the same codes, up to the order of
 * the fp32 additions inside the small-M kernels' MMAs (the tensor-core path gives identical
 * bits). Configurations are kept under QG_OP_W4A16_INTERLEAVED.
 */
qg_status qgemm_w4a16_interleaved(const void *A, const uint32_t *Wq, const void *scales,
                                  const void *zeros, void *C, int M, int N, int K, int group_size,
                                  int split_k, int has_zero, cudaStream_t stream);

/*
 * W4A16 with deterministic split-K: the fp32-workspace form of parallel-k (hidet-org/hidet issue
 * #364, parallel-k discussion; qgemm_w4a16 with split_k > 1 is the atomic form). Operands and
 * result as qgemm_w4a16. Each of the split_k (>= 1, given explicitly) parts of the K reduction
 * writes its fp32 partial tile into `workspace`; the last part to finish a tile adds all partial
 * tiles in part order and rounds once to fp16. The result is bit-identical from run to run and
 * carries no fp16 rounding of partial sums.
 * Runs on the small-M streaming kernel: requires group_size % 128 == 0 (or -1 / 0 with
 * K % 128 == 0); any M is accepted, M <= 16 is what it is built for.
 * workspace: caller-owned device memory, 256-byte aligned, at least
 * qgemm_w4a16_workspace_bytes(M, N, K, group_size, split_k) bytes. Its contents on entry do not
 * matter (the call clears the part that must start at zero). Calls that share a workspace must
 * not overlap on the GPU.
 */
qg_status qgemm_w4a16_splitk_f32(const void *A, const uint32_t *Wq, const void *scales,
                                 const void *zeros, void *C, int M, int N, int K, int group_size,
                                 int split_k, int has_zero, void *workspace,
                                 size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes qgemm_w4a16_splitk_f32 needs for these arguments (0 if they are invalid). */
size_t qgemm_w4a16_workspace_bytes(int M, int N, int K, int group_size, int split_k);

/*
 * qgemm_w4a16_splitk_f32 for callers that cannot allocate device memory: code that runs where
 * cudaMalloc is not allowed or not wanted (inside a memory pool's or a framework's own
 * allocator, in a process whose device memory is fully reserved up front, or on a path that
 * must never block on the allocator). It takes no workspace: the scratch lives in one
 * statically sized buffer inside the library, QGEMM_NOALLOC_SCRATCH_BYTES bytes of device
 * memory that every GPU which loads the library holds until the process exits. The source
 * pages have no counterpart to this entry point.
 *   - Same arguments and result as qgemm_w4a16_splitk_f32 minus the workspace; the result is
 *     bit-identical to it.
 *   - Needs qgemm_w4a16_workspace_bytes(M, N, K, group_size, split_k) <= the buffer size; larger
 *     problems return QG_ERR_SCRATCH_TOO_SMALL before anything is queued.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call. The first call
 *     on each device looks up the buffer's device address (cudaGetSymbolAddress, with that
 *     device current); make that first call before any stream capture.
 *   - Every call on a device shares the one buffer and leaves its contents behind; each call
 *     clears the part that must start at zero. Calls that overlap on the GPU (on different
 *     streams, or from different host threads) race on the buffer: order them.
 */
#define QGEMM_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
qg_status qgemm_w4a16_splitk_f32_noalloc(const void *A, const uint32_t *Wq, const void *scales,
                                         const void *zeros, void *C, int M, int N, int K,
                                         int group_size, int split_k, int has_zero,
                                         cudaStream_t stream);

/*
 * W4A16 with the activations and the result in page-locked host memory: one end-to-end call for
 * a caller whose tokens live on the host. A goes in and C comes out in chunks of tokens through
 * `workspace`, so that the host-to-device copy of one chunk, the matmul of the one before and
 * the device-to-host copy of the one before that run at the same time (the two directions use
 * separate copy engines). Each chunk is computed as qgemm_w4a16 computes it.
 *   A_host: fp16 [M, K] row-major; C_host: fp16 [M, N] row-major; both page-locked
 *   (cudaHostAlloc or cudaHostRegister; pageable memory returns QG_ERR_INVALID_ARG).
 *   Wq, scales, zeros, group_size, split_k, has_zero: as qgemm_w4a16 (device memory).
 *   workspace: caller-owned device memory, 256-byte aligned, holding two A chunks and two C
 *   chunks; chunk = the largest multiple of 256 tokens (or M, or fewer than 256 tokens when
 *   that is all that fits) with 4 * chunk * (K + N) bytes <= workspace_bytes (plus rounding of
 *   each buffer to 256 bytes); qgemm_w4a16_host_workspace_bytes gives the size for a chunk.
 *   With more than two chunks the first and the last are a quarter of a chunk (at least 256
 *   tokens): their copies are the ones nothing else overlaps.
 * Stream order as for every call: the copies start after the work already queued on `stream`,
 * and work queued on `stream` later starts after the last copy into C_host has finished (wait
 * on `stream` before reading C_host on the host). The library creates two copy streams and a
 * few events per device on first use (no device memory). Calls that share a workspace must be
 * ordered on one stream. On an error return the contents of C_host are undefined.
 */
qg_status qgemm_w4a16_host(const void *A_host, const uint32_t *Wq, const void *scales,
                           const void *zeros, void *C_host, int M, int N, int K, int group_size,
                           int split_k, int has_zero, void *workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* Workspace bytes for qgemm_w4a16_host with chunks of chunk_tokens tokens (0: min(M, 1024));
 * 0 if the arguments are invalid. */
size_t qgemm_w4a16_host_workspace_bytes(int M, int N, int K, int chunk_tokens);

/*
 * W8A8. A: int8 [M, K]. W: int8 [N, K]. C: int32 [M, N] = sum_k A[m,k] * W[n,k], exact
 * (it wraps modulo 2^32 only if |C| >= 2^31, impossible for K <= 131072).
 * group_size must be -1 or 0 (no scales) and has_zero 0. Requires K % 16 == 0.
 */
qg_status qgemm_w8a8(const int8_t *A, const int8_t *W, int32_t *C, int M, int N, int K,
                     int group_size, int split_k, int has_zero, cudaStream_t stream);

/*
 * W8A8 with int8 output. A: int8 [M, K]. W: int8 [N, K]. mult: fp32 [N] (one multiplier per
 * output channel). C: int8 [M, N],
 *     C[m, n] = clamp(rint(float(acc[m, n]) * mult[n]), -128, 127),   acc = sum_k A[m,k] W[n,k],
 * acc exact in int32, its conversion to binary32 and the product correctly rounded, rint half to
 * even. microsoft/BitBLAS issue #252's configuration listing has int8 x int8 configurations
 * with an int8 output type; the pages do not state the requantisation, this per-channel form
 * is the reading. The K reduction is never split (the rounding needs the whole sum).
 * Requires K % 16 == 0; A, W 16-byte aligned, mult 4-byte aligned, C any alignment.
 */
qg_status qgemm_w8a8_requant(const int8_t *A, const int8_t *W, const float *mult, int8_t *C,
                             int M, int N, int K, cudaStream_t stream);

/*
 * W2A8. A: int8 [M, K]. Wq: uint32 [N, K/16], value k of row n is the two's-complement
 * 2-bit field at bits 2*(k%16) of word k/16 (values -2..1). C: int32 [M, N], exact.
 * group_size must be -1 or 0 and has_zero 0. Requires K % 64 == 0.
 */
qg_status qgemm_w2a8(const int8_t *A, const uint32_t *Wq, int32_t *C, int M, int N, int K,
                     int group_size, int split_k, int has_zero, cudaStream_t stream);

/*
 * W2A8 with weights in the interleaved (pre-shuffled) layout that quant_pack_int2_interleaved
 * writes: within each uint32 word the values k = 16j .. 16j+15 sit in 2-bit fields
 * 0, 2, 4, 6, 1, 3, 5, 7, 8, 10, 12, 14, 9, 11, 13, 15 (fields 0..15 hold values 0, 4, 1, 5, 2,
 * 6, 3, 7, 8, 12, 9, 13, 10, 14, 11, 15), so that the tensor-core path's upcast (a byte-table
 * PRMT on the low 3 bits of each nibble of w, w >> 2, w >> 16 and w >> 18) yields four int8
 * registers already in K order, with no byte transpose. pytorch/ao issue #2752 ("Migrating from
 * AffineQuantizedTensor + Layouts to tensor subclasses"), packing-format list: pre-shuffled
 * layouts that move the permutation out of the hot loop. Result and every other argument as
 * qgemm_w2a8 on the naturally packed weights of the same values (exact, bit-identical).
 * Configurations are kept under QG_OP_W2A8_INTERLEAVED.
 */
qg_status qgemm_w2a8_interleaved(const int8_t *A, const uint32_t *Wq, int32_t *C, int M, int N,
                                 int K, int group_size, int split_k, int has_zero,
                                 cudaStream_t stream);

/*
 * Dense fp16 baseline. A: fp16 [M, K]; W: fp16 [N, K]; C: fp16 [M, N] = A . W^T with fp32
 * accumulation. Requires K % 8 == 0.
 */
qg_status qgemm_dense_f16(const void *A, const void *W, void *C, int M, int N, int K,
                          int split_k, cudaStream_t stream);

/* ---- weight packing ------------------------------------------------------------------------ */

/*
 * Round-to-nearest int4 quantisation of fp16 weights W [N, K] into packed codes Wq [N, K/8]
 * (the layout of quant_pack_int4) and fp16 scales, zeros [N, K/group_size], so that
 * qgemm_w4a16 with these operands computes A . W~^T for the quantised W~ = (q - z) * s.
 * The pytorch/ao issue's workflow table names int4 weight-only quantisation
 * (Int4WeightOnlyConfig) without a formula; the rule implemented, per group of group_size
 * consecutive K values of a row:
 *     lo = min(0, min w), hi = max(0, max w),
 *     s  = fp16_rn((hi - lo) / 15)   (1 when hi == lo; the smallest subnormal if it rounds to 0)
 *     z  = clamp(rint(0 - lo / s), 0, 15),   q = clamp(rint(w / s) + z, 0, 15),
 * rint rounding half to even; the divisions and rint are binary32 operations (correctly
 * rounded). So |w - (q - z) s| <= s / 2 wherever q is not clamped.
 *   - has_zero must be 1 and zeros non-NULL (unsigned codes need the zero point).
 *   - group_size: 32, 64, 128 or a multiple of 256 dividing K; -1 / 0 for one group over K.
 *   - Requires K % 32 == 0; W and Wq 16-byte aligned, scales and zeros 2-byte aligned.
 *   - Weights are expected finite.
 */
qg_status quant_rtn_int4(const void *W, uint32_t *Wq, void *scales, void *zeros, int N, int K,
                         int group_size, int has_zero, cudaStream_t stream);

/*
 * codes: uint8 [N, K] (only the low 4 bits are used) -> packed: uint32 [N, K/8],
 *     packed[n, j] = sum_{i<8} (codes[n, 8j+i] & 0xF) << 4i.
 * M, group_size, split_k and has_zero are accepted for a uniform call shape and ignored.
 * Requires K % 32 == 0.
 */
qg_status quant_pack_int4(const uint8_t *codes, uint32_t *packed, int M, int N, int K,
                          int group_size, int split_k, int has_zero, cudaStream_t stream);

/*
 * codes: uint8 [N, K] -> packed: uint32 [N, K/8] in the interleaved layout of
 * qgemm_w4a16_interleaved: packed[n, j] = sum_e (codes[n, 8j+e] & 0xF) << 4 * pos(e) with
 * pos = (0, 4, 1, 5, 2, 6, 3, 7). Requires K % 32 == 0. Other arguments as quant_pack_int4.
 */
qg_status quant_pack_int4_interleaved(const uint8_t *codes, uint32_t *packed, int M, int N, int K,
                                      int group_size, int split_k, int has_zero,
                                      cudaStream_t stream);

/*
 * vals: int8 [N, K] holding values -2..1 (only the low 2 bits are used) -> packed: uint32
 * [N, K/16], packed[n, j] = sum_{i<16} (vals[n, 16j+i] & 3) << 2i. Requires K % 64 == 0.
 */
qg_status quant_pack_int2(const int8_t *vals, uint32_t *packed, int M, int N, int K,
                          int group_size, int split_k, int has_zero, cudaStream_t stream);

/*
 * vals: int8 [N, K] holding values -2..1 (only the low 2 bits are used) -> packed: uint32
 * [N, K/16] in the interleaved layout of qgemm_w2a8_interleaved:
 *     packed[n, j] = sum_i (vals[n, 16j+i] & 3) << 2 * pos(i),
 *     pos(i) = 8 * (i / 8) + 2 * (i % 4) + (i % 8) / 4.
 * Requires K % 64 == 0. Other arguments as quant_pack_int2.
 */
qg_status quant_pack_int2_interleaved(const int8_t *vals, uint32_t *packed, int M, int N, int K,
                                      int group_size, int split_k, int has_zero,
                                      cudaStream_t stream);

/* ---- configuration ---------------------------------------------------------------------------- */

/*
 * Fill *out with the configuration a call with these arguments would launch on the current
 * device (or on a 148-SM B200 if no device is visible). split_k > 0 overrides the split.
 * Host-only: launches nothing.
 */
qg_status qgemm_plan(int op, int M, int N, int K, int group_size, int has_zero, int split_k,
                     qgemm_config_t *out);

/* Pin *cfg for this exact problem (NULL removes the entry). Checked before it is stored. */
qg_status qgemm_set_config(int op, int M, int N, int K, int group_size, int has_zero,
                           const qgemm_config_t *cfg);

/*
 * Time every candidate configuration for this problem on the caller's buffers (same meaning
 * as the matching matmul entry point; C is overwritten, W is read only) and pin the fastest.
 * `reps` timed launches per candidate (<= 0: 20). The winner is copied to *best if non-NULL.
 * Synchronises `stream`.
 */
qg_status qgemm_tune(int op, const void *A, const void *W, const void *scales,
                     const void *zeros, void *C, int M, int N, int K, int group_size,
                     int has_zero, int reps, cudaStream_t stream, qgemm_config_t *best);

/* Pinned configurations as text, one per line; load merges into the table. */
qg_status qgemm_save_configs(const char *path);
qg_status qgemm_load_configs(const char *path);
void qgemm_clear_configs(void);

/* ---- errors ------------------------------------------------------------------------------------ */

/*
 * Synchronise `stream`, then read and clear the current device's error word. Returns
 * QG_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait since the last check,
 * QG_ERR_CUDA if the synchronisation failed, QG_OK otherwise.
 */
qg_status qgemm_sync_check(cudaStream_t stream);

/*
 * Self-test of the failure path (no counterpart in the pages): queues on `stream` a kernel whose
 * bounded mbarrier wait can never be satisfied. The wait gives up after limit_us microseconds
 * (1 .. 2000000), raises the device error word exactly as a stalled matmul pipeline would, and the
 * kernel returns: no trap, no fault, the context stays usable. The next qgemm_sync_check reports
 * QG_ERR_DEVICE_TIMEOUT and clears the word.
 */
qg_status qgemm_selftest_bounded_wait(int limit_us, cudaStream_t stream);

const char *qgemm_status_string(qg_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int qgemm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QGEMM_H_ */
