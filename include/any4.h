/*
 * any4.h - C ABI of the any4 mixed-precision linear layer for NVIDIA B200 (sm_100a).
 *
 * any4 stores every weight of a linear layer W (N x K, one row per output
 * channel) as a 4-bit index into a per-row table (LUT) of 16 bf16 values; each
 * row is split into contiguous groups of G columns with a bf16 scale alpha and
 * offset beta per group. The dequantized weight is
 *
 *     w_hat[n][k] = fma(alpha[n][k/G], LUT[n][idx[n][k]], beta[n][k/G])
 *
 * Sources: the any4 explainer (10100.com, article 149119421), section 2 (per-row
 * 16-entry FP16/BF16 table, 4-bit index per weight, table read at inference),
 * section 2.1 (per-group scale and offset), section 3 (tinygemm: table held in
 * registers, weights pre-arranged in the compute format, batch 1-16 decode);
 * "any4: Learned 4-bit Numeric Representation for LLMs" (arXiv 2507.04610,
 * abstract).
 *
 * Conventions for every call:
 *  - All data pointers are DEVICE pointers owned by the caller. The library
 *    never allocates, frees or keeps a reference to caller memory.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and never synchronize the device.
 *  - bf16 values are passed as their 16-bit patterns (uint16_t).
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call returns a negative any4_status and launches nothing.
 *  - A failed kernel launch returns ANY4_ECUDA; the CUDA error code is kept
 *    per thread and returned by any4_last_cuda_error().
 *  - Accepted shapes: N > 0 and N % 16 == 0; K > 0 and K % 64 == 0;
 *    G in {64, 128, 256, 512, 1024} and K % G == 0; 1 <= M <= 16.
 *    Anything else returns ANY4_ESHAPE.
 */
#ifndef ANY4_H
#define ANY4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the shared library are exported explicitly (it is built with
 * hidden default visibility). */
#if defined(__GNUC__)
#define ANY4_API __attribute__((visibility("default")))
#else
#define ANY4_API
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* any4_stream_t;

typedef enum {
    ANY4_OK = 0,
    ANY4_EINVAL = -1,      /* null pointer or a negative / zero size           */
    ANY4_EALIGN = -2,      /* a pointer misses its required alignment          */
    ANY4_ESHAPE = -3,      /* M, N, K or G outside the accepted set            */
    ANY4_EWORKSPACE = -4,  /* packed buffer or workspace smaller than required */
    ANY4_ECUDA = -5        /* a CUDA runtime call or kernel launch failed      */
} any4_status;

/*
 * Size in bytes of the device-layout buffer any4_pack writes for an N x K
 * weight with group size G; 0 if the shape is not accepted. With Np = N
 * rounded up to a multiple of 32 (the padding rows are zeros), the size is
 * Np*K/2 (indices) + 32*Np (LUT) + 4*Np*(K/G) (alpha and beta), each section
 * padded to 256 bytes. At K = 4096 the LUT adds 16*16/4096 = 0.0625 bit per
 * weight (explainer section 2.3).
 */
ANY4_API size_t any4_packed_bytes(int n, int k, int group);

/*
 * any4_pack - reorder canonical any4 tensors into the device layout
 * (explainer section 3: weights pre-arranged in the hardware compute format).
 *
 *   idx_nib  [N][K/2] uint8: byte j of row n holds the index of column 2j in
 *            its low nibble and of column 2j+1 in its high nibble.
 *   lut      [N][16]  bf16 table of each row (section 2).
 *   alpha    [N][K/G] bf16 group scales; beta [N][K/G] bf16 group offsets
 *            (section 2.1).
 *   packed   output, packed_bytes >= any4_packed_bytes(n, k, group); 16-byte
 *            aligned. The layout is opaque and immutable once written; it may
 *            be read by any number of calls and streams.
 * Inputs need no particular alignment. Returns ANY4_OK or an error status.
 */
ANY4_API int any4_pack(const uint8_t* idx_nib, const uint16_t* lut, const uint16_t* alpha,
              const uint16_t* beta, int n, int k, int group, void* packed,
              size_t packed_bytes, any4_stream_t stream);

/*
 * any4_dequant - debug call: write the dequantized weight matrix.
 *   w  output [N][K] bf16, row-major, 4-byte aligned.
 * w_hat[n][k] is alpha*LUT[idx]+beta evaluated as one fp32 fused
 * multiply-add rounded to nearest-even, then rounded to bf16 nearest-even
 * (subnormals kept). Bit-exact by construction.
 */
ANY4_API int any4_dequant(const void* packed, int n, int k, int group, uint16_t* w,
                 any4_stream_t stream);

/*
 * Bytes of workspace any4_linear needs for this shape on the CURRENT device
 * (the launch is sized by the device's SM count); 0 if the shape is not
 * accepted. The workspace holds a fixed header of 65536 arrival counters (one
 * per possible 16-row tile) and a reserved 256-byte area, then the fp32
 * partial sums of output blocks split along K between thread blocks. For
 * M > 512 (prefill beyond the fused decode) the header is followed by a bf16
 * N x K scratch for the dequantized weight (N*K*2 bytes, rounded up to 256),
 * then the partial sums.
 */
ANY4_API size_t any4_linear_workspace_bytes(int m, int n, int k, int group);

/*
 * any4_linear_grid - the launch geometry any4_linear / any4_linear_bits use
 * for this shape on the current device (introspection; no launch).
 *
 *   bits       2, 3 or 4.
 *   blocks     out: thread blocks of the decode kernel (M <= 16) or of the
 *              GEMM (M > 16).
 *   cluster    out: thread blocks per cluster. > 1 when every 32-row panel is
 *              split along K between the blocks of one cluster, which finish
 *              it through distributed shared memory (a shape with fewer
 *              panels than SMs); 1 otherwise.
 *
 * Returns ANY4_EINVAL for null outputs, ANY4_ESHAPE for a shape or bit width
 * the calls reject, ANY4_ECUDA if the device cannot be queried.
 */
ANY4_API int any4_linear_grid(int bits, int m, int n, int k, int group, int* blocks, int* cluster);

/* Kernels of any4_linear / any4_linear_bits (any4_linear_kernel). */
typedef enum {
    ANY4_KERNEL_SHARED_TABLES = 1,    /* M <= 16: row-pair tables in shared memory (the general decode) */
    ANY4_KERNEL_REGISTER_TABLES = 2,  /* M <= 16, any4, a short K split per cluster block: row tables in
                                         registers, byte-permute decode */
    ANY4_KERNEL_PREFILL_FUSED = 3,    /* 16 < M <= 512, any4: decode into the tcgen05 GEMM's shared memory */
    ANY4_KERNEL_PREFILL_GEMM = 4,     /* other M > 16: dequantize into the workspace, then the GEMM */
    ANY4_KERNEL_SHARED_TABLES_DIRECT = 5  /* M <= 4, any4, few chunks per block: the shared row-pair tables
                                             with each warp loading its own operands */
} any4_kernel;

/*
 * any4_linear_kernel - which kernel any4_linear / any4_linear_bits run for
 * this shape on the current device (introspection; no launch). The explainer
 * (10100.com article 149119421, section 3) keeps each row's table next to the
 * arithmetic; which form of it a shape gets is a launch decision of this
 * library, fixed by the shape and the device's SM count.
 *
 * Returns an any4_kernel value (> 0), ANY4_ESHAPE for a shape or bit width
 * the calls reject, or ANY4_ECUDA if the device cannot be queried.
 */
ANY4_API int any4_linear_kernel(int bits, int m, int n, int k, int group);

/*
 * any4_linear - y = x . W_hat^T, the any4 mixed-precision linear layer.
 *
 *   m          tokens, 1 .. 2^20. M <= 16 (decode, explainer section 3's
 *              batch 1-16) runs a fused dequant-and-contract kernel, as
 *              below; which one (the streaming shared-table kernel, or for
 *              shapes with few chunks per thread block the shared tables
 *              with per-warp loads at M <= 4 or the register tables at
 *              M = 5-16) depends on the shape and is reported by
 *              any4_linear_kernel.
 *              M > 16 (prefill) runs a tensor-core GEMM (tcgen05, fp32
 *              accumulation in tensor memory): up to M = 512 its A tiles are
 *              decoded from the packed weight straight into shared memory
 *              (w_hat rounded once to bf16, as below); beyond that W is
 *              dequantized once into the workspace (the bit-exact
 *              any4_dequant values) and the GEMM reads it back.
 *   x          [M][K] bf16 activations, row-major, 16-byte aligned.
 *   packed     the any4_pack output for W (N x K, group G).
 *   y          [M][N] bf16 output, row-major, 4-byte aligned.
 *   workspace  >= any4_linear_workspace_bytes(m, n, k, group) bytes, 16-byte
 *              aligned, owned by the caller. It MUST be zero-filled before its
 *              first use: it starts with the per-tile arrival counters, and
 *              every call that runs to completion sets them back to zero (the
 *              partial-sum area behind them needs no initialization). After a
 *              failed launch, zero-fill it again. Calls that may overlap on
 *              the device need separate workspaces.
 *
 * Each weight is dequantized as w_hat = fma(alpha, LUT[idx], beta) in bf16
 * (fma.rn.bf16x2: the exact value rounded once to bf16) and contracted on the
 * tensor cores (mma.sync m16n8k16) with fp32 accumulation; the fp32 result
 * is rounded to bf16 nearest-even. Output rows split along K between thread
 * blocks (at most one block per SM, all resident at once; for shapes with
 * few 32-row panels, the 2-8 blocks of a thread-block cluster) are finished
 * by the block that holds their first columns: it waits for the others' fp32
 * partials (through the workspace, or within a cluster through distributed
 * shared memory) and adds them in a fixed order, so the result is
 * deterministic (every kernel adds in a fixed order; two calls of the same
 * shape on the same device give the same bits).
 * Every wait in the kernels is bounded (~2-4 s); if one gives up, the kernel
 * completes without hanging and the first 32-bit word of the workspace's
 * reserved area (byte offset 65536*4) is set non-zero. It is zero after
 * every normal call.
 */
ANY4_API int any4_linear(const uint16_t* x, const void* packed, int m, int n, int k, int group,
                uint16_t* y, void* workspace, size_t workspace_bytes, any4_stream_t stream);

/*
 * any3 / any2: the same calls for b = 3 or 2 bits per index (the lower-bit
 * variants named in the abstract of the "any4: Learned 4-bit Numeric
 * Representation for LLMs" summary page). The canonical inputs are as for
 * any4_pack, with every index < 2^b (an 8- or 4-entry table per row; only the
 * first 2^b LUT entries are read, the rest may be anything); any4_quantize
 * with bits = 3 or 2 produces them. The packed buffer stores each row pair's
 * two indices as one 2b-bit code, densely (N*K*b/8 bytes of indices) and is
 * only valid for the *_bits calls with the same b. bits = 4 is the same as
 * the plain calls. any4_linear_bits needs any4_linear_workspace_bytes_bits
 * bytes of workspace: for M > 16, b = 3 and 2 dequantize W into the
 * workspace (N*K*2 bytes more than any4, whose prefill decodes on the fly up
 * to 512 tokens). Errors as for the plain calls, plus ANY4_ESHAPE for bits
 * not in {2, 3, 4}; the size query returns 0 for those.
 */
ANY4_API size_t any4_linear_workspace_bytes_bits(int bits, int m, int n, int k, int group);
ANY4_API size_t any4_packed_bytes_bits(int bits, int n, int k, int group);
ANY4_API int any4_pack_bits(int bits, const uint8_t* idx_nib, const uint16_t* lut,
                            const uint16_t* alpha, const uint16_t* beta, int n, int k, int group,
                            void* packed, size_t packed_bytes, any4_stream_t stream);
ANY4_API int any4_dequant_bits(int bits, const void* packed, int n, int k, int group, uint16_t* w,
                               any4_stream_t stream);
ANY4_API int any4_linear_bits(int bits, const uint16_t* x, const void* packed, int m, int n, int k,
                              int group, uint16_t* y, void* workspace, size_t workspace_bytes,
                              any4_stream_t stream);

/*
 * any4_linear_noalloc - any4_linear for callers that cannot allocate device
 * memory. The source pages have no counterpart of this call; it exists for
 * callers such as operators running inside a serving runtime that owns all
 * device memory and passes a kernel only its inputs and outputs, and
 * latency-critical loops that must not call cudaMalloc because it can
 * synchronize the device.
 *
 * Same arguments, result and rounding as any4_linear for 1 <= M <= 16, minus
 * the workspace (M > 16, the prefill path, returns ANY4_ESHAPE): the partial
 * sums, counters and status word live in a fixed 8 MiB array of device memory
 * that this library reserves on every GPU that loads it, until the process
 * exits. A shape whose launch needs more than that returns ANY4_EWORKSPACE;
 * the largest need is 256 KiB + 256 B plus 2,048 bytes per SM (M = 9..16),
 * 0.56 MB on a 148-SM B200, so every accepted shape fits. The call allocates
 * and frees nothing. The first call on a
 * device (of this function or any4_noalloc_status_word) looks up the array's
 * address with that device current, so make it before any stream capture on
 * that device. All calls on a device share the array: each call first clears
 * its header (counters and status word) on `stream`, and calls that can run
 * at the same time on the GPU race and must be ordered by the caller.
 * A bounded wait inside the kernel that gave up leaves y incomplete and sets
 * the status word non-zero; the call itself still returns ANY4_OK (it only
 * enqueues work). Read the word through any4_noalloc_status_word() after the
 * call's work on `stream` has completed.
 */
ANY4_API int any4_linear_noalloc(const uint16_t* x, const void* packed, int m, int n, int k,
                                 int group, uint16_t* y, any4_stream_t stream);

/*
 * any4_noalloc_status_word - device address (on the current device) of the
 * 32-bit status word of any4_linear_noalloc: 0 after a call that completed
 * normally, non-zero (bit 0: a bounded wait timed out) otherwise, until the
 * next any4_linear_noalloc call on that device clears it. Host-only lookup;
 * copy the word with any device-to-host copy of the caller's choice.
 * Returns ANY4_OK, ANY4_EINVAL for a NULL status, ANY4_ECUDA if the device
 * cannot be queried.
 */
ANY4_API int any4_noalloc_status_word(const uint32_t** status);

/*
 * any4_quantize - the any4 quantizer on the GPU (explainer sections 2.1 and
 * 2.2): group scaling, then per-row weighted k-means with 2^bits centres.
 *
 *   w        [N][K] bf16 weights (device).
 *   ex       [K] float64 E|x| per input channel from a calibration sample
 *            (section 2.1); the k-means weight of column k is alpha * ex[k].
 *   bits     4 (any4), 3 (any3) or 2 (any2); iters: E/M rounds, 0..1000
 *            (10 in this library's tests).
 *   outputs  the canonical tensors any4_pack consumes: idx_nib [N][K/2]
 *            (even column in the low nibble; codes < 2^bits), lut [N][16]
 *            bf16 (2^bits learned entries, padded by repeating the last),
 *            alpha and beta [N][K/G] bf16.
 * Group scaling is asymmetric min-max onto [-2^(bits-1), 2^(bits-1)-1]:
 * alpha = (max-min)/(2^bits-1), beta = min + 2^(bits-1)*alpha, both rounded
 * to bf16. The start table is the row's distinct scaled values when there
 * are at most 2^bits of them, else the integer map; E-step ties go to the
 * lowest index; an empty cluster keeps its value; after the rounds the table
 * is rounded to bf16 and a last E-step assigns against it. All arithmetic is
 * float64 with each cluster sum taken in column order, so the output is a
 * deterministic function of the inputs. One thread per row: meant for
 * model preparation, not for the per-token path.
 * Returns ANY4_OK, ANY4_EINVAL (null pointer, bits or iters out of range) or
 * ANY4_ESHAPE (N, K, G as for any4_pack).
 */
ANY4_API int any4_quantize(const uint16_t* w, const double* ex, int n, int k, int group, int bits,
                           int iters, uint8_t* idx_nib, uint16_t* lut, uint16_t* alpha,
                           uint16_t* beta, any4_stream_t stream);

/*
 * Fixed-table 4-bit formats (explainer section 1, comparison table: int4,
 * NF4 and FP4 against any4). Each is one 16-entry table shared by every row,
 * so a weight in one of these formats is an any4 weight whose row tables are
 * all equal, and it runs through any4_dequant and any4_linear unchanged.
 *   ANY4_FORMAT_INT4  -8, -7, ..., 7 (code q -> q - 8)
 *   ANY4_FORMAT_NF4   4-bit NormalFloat: 7 negative and 8 positive quantiles
 *                     of the standard normal plus 0, in [-1, 1], ascending
 *   ANY4_FORMAT_FP4   E2M1 element type: code bit 3 = sign, bits 2..1 =
 *                     exponent (bias 1), bit 0 = mantissa; code 8 is -0
 * Values are rounded to bf16 nearest-even.
 */
typedef enum { ANY4_FORMAT_INT4 = 1, ANY4_FORMAT_NF4 = 2, ANY4_FORMAT_FP4 = 3 } any4_format;

/*
 * any4_format_lut - the 16 bf16 values (bit patterns) of a format, by code.
 * Host only, no GPU needed. lut: host array of 16 uint16_t written by the
 * call. Returns ANY4_OK, or ANY4_EINVAL for a NULL lut or an unknown format.
 */
ANY4_API int any4_format_lut(int format, uint16_t* lut);

/*
 * any4_pack_format - any4_pack with the format's table in every row.
 * idx_nib, alpha, beta, n, k, group, packed, packed_bytes and stream are as
 * for any4_pack (the indices are the format's 4-bit codes); no LUT input.
 * Returns as any4_pack; ANY4_EINVAL also for an unknown format.
 */
ANY4_API int any4_pack_format(int format, const uint8_t* idx_nib, const uint16_t* alpha,
                              const uint16_t* beta, int n, int k, int group, void* packed,
                              size_t packed_bytes, any4_stream_t stream);

/* Static description of a status code (never NULL). */
ANY4_API const char* any4_strerror(int status);

/* The cudaError_t value of the last ANY4_ECUDA returned on this host thread. */
ANY4_API int any4_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ANY4_H */
