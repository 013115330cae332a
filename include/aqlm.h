/*
 * aqlm.h -- C ABI of the B200 (sm_100a) AQLM inference library.
 *
 * AQLM ("Extreme Compression of Large Language Models via Additive
 * Quantization", ICML 2024; explained in "The AQLM Quantization Algorithm,
 * Explained", section "What is Multi-Codebook Quantization (MCQ)?") stores a
 * weight matrix W of shape d_out x d_in as
 *   - M codebooks of K = 2^B codewords, each codeword g = 8 values (16-bit);
 *   - one 16-bit scale per output channel (row) i;
 *   - for every group of g consecutive inputs of every row, M codes of B bits,
 *     the indices of the codewords that are summed to approximate the group.
 * The dequantised weight is
 *   W^[i][8j + t] = s_i * sum_{m<M} C_m[ b(i, j, m) ][t],
 * and a layer computes y = W^ . x for the activations of T tokens (W.X
 * convention: rows of W are output channels).  The formats are named MxB
 * after the naming scheme of section "Key AQLM quantization parameters":
 * 1x16, 2x8 and 2x16 are supported.
 *
 * Memory layout (all row-major, every pointer is DEVICE memory unless stated):
 *   codes      [d_out][d_in/8][M]   B = 8: uint8; B = 16: 16-bit words whose
 *                                   index is the UNSIGNED value 0..65535
 *                                   (pass int16 or uint16 storage alike)
 *   codebooks  [M][2^B][8]          IEEE binary16 (fp16) bit patterns
 *   scales     [d_out]              fp16
 *   x, y       [T][d_in], [T][d_out] fp16           (aqlm_gemv)
 *   X, Y       [T][d_in], [T][d_out] bfloat16       (aqlm_gemm)
 *   W_out      [d_out][d_in]        bfloat16        (aqlm_dequant)
 *
 * Conventions for every entry point:
 *   - The caller owns all memory.  The library allocates nothing, keeps no
 *     pointer after a call returns and holds no mutable host state, so calls
 *     from several host threads are safe.
 *   - Work is enqueued on `stream` (NULL = the legacy default stream) and the
 *     call returns without synchronising.  Outputs must not alias inputs.
 *   - Validation happens on the host before any launch; a call that returns
 *     anything but AQLM_OK has launched nothing, except AQLM_ERR_CUDA, which
 *     reports the CUDA error of a launch (query it with cudaGetLastError
 *     semantics: the library does not clear unrelated errors).
 *   - No entry point prints, exits, throws or traps.
 *   - Supported shapes: group == 8, (M, B) in {(1,16), (2,8), (2,16)},
 *     d_out >= 1, d_in >= 8, d_in % 8 == 0 (else AQLM_ERR_UNSUPPORTED).
 *   - Alignment: codes, codebooks, x/X, y/Y and W_out 16-byte aligned, and a
 *     row of codes (d_in/8 * M * B/8 bytes) a multiple of 16 bytes, i.e.
 *     d_in % 64 == 0 for 1x16 and 2x8, d_in % 32 == 0 for 2x16 (else
 *     AQLM_ERR_MISALIGNED).  Scales need 2-byte alignment.
 */
#ifndef AQLM_B200_H
#define AQLM_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AQLM_API __attribute__((visibility("default")))
#else
#define AQLM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's cudaStream_t is `struct CUstream_st *`; declaring the
 * same type here keeps this header free of CUDA includes. */
struct CUstream_st;
typedef struct CUstream_st *aqlm_stream_t;

typedef enum {
    AQLM_OK = 0,
    AQLM_ERR_INVALID_ARG = 1,  /* null pointer, tokens out of range, bad sizes */
    AQLM_ERR_UNSUPPORTED = 2,  /* format or shape outside the supported set   */
    AQLM_ERR_MISALIGNED = 3,   /* pointer or row stride not 16-byte aligned   */
    AQLM_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required  */
    AQLM_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed         */
    AQLM_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up           */
} aqlm_status;

typedef struct {
    int32_t d_out;          /* output channels (rows of W)                   */
    int32_t d_in;           /* input features (columns of W)                 */
    int32_t group;          /* g, inputs per group: must be 8                */
    int32_t num_codebooks;  /* M                                             */
    int32_t codebook_bits;  /* B: log2 of the codewords per codebook (8|16) */
} aqlm_shape;

/* Largest token count of the matrix-vector path. */
#define AQLM_GEMV_MAX_TOKENS 16

/* Most layers of one aqlm_gemv_multi call. */
#define AQLM_MULTI_MAX_LAYERS 4

/* One layer of an aqlm_gemv_multi call: a host struct whose pointers are
 * device memory, laid out as above. */
typedef struct {
    const void *codes;          /* [d_out][d_in/8][M]                       */
    const uint16_t *codebooks;  /* [M][2^B][8] fp16                         */
    const uint16_t *scales;     /* [d_out] fp16                             */
    uint16_t *y;                /* [tokens][d_out] fp16, written            */
    int32_t d_out;              /* rows of this layer                       */
} aqlm_layer;

/*
 * aqlm_gemv -- decode-time layer product, y = W^ . x, for 1 <= tokens <= 16.
 *
 * Defined by section "What is Multi-Codebook Quantization (MCQ)?": each
 * group's codes select M codewords that are summed, the sum is scaled by the
 * row's scale, and the product with the activations is taken.  Computed with
 * fp32 accumulation; each y value is rounded once to fp16 (nearest even).
 * The scale is applied to the row's accumulated sum (the same value in exact
 * arithmetic as scaling every group).
 *   codes, codebooks, scales: the layer, layout above.
 *   x: [tokens][d_in] fp16.   y: [tokens][d_out] fp16 (written).
 *   workspace/workspace_bytes: device scratch for fp32 partial sums and
 *   arrival counters, used when a row's input range is split over several
 *   CTAs, and (4 to 16 tokens) a status word; aqlm_gemv_workspace_bytes()
 *   gives the size for this device (0 = none needed, NULL allowed).  Too
 *   small or not 16-byte aligned -> AQLM_ERR_WORKSPACE.  The workspace must be
 *   zero-filled before its first use; every completed call leaves it ready for
 *   the next one.  Calls that share a workspace must not overlap on the GPU.
 * Up to AQLM_GEMV_ROW_TOKENS(shape) tokens (1x16: 2, 2x16: 3, 2x8: 4) the
 * product runs on the CUDA cores with no device waits.  Past that it runs on
 * the tensor cores with producer/consumer waits inside each CTA, each bounded
 * in time: a wait that gives up records AQLM_ERR_TIMEOUT in the workspace's
 * status word (y is then not valid, and the workspace must be zero-filled
 * again); aqlm_gemv_check() reads it.
 * Launch: with programmatic dependent launch.  codes, codebooks and scales
 * are treated as constant weights and may be read before the preceding
 * kernel in the stream has finished; x is read, and y and the workspace are
 * written, only after it has finished.
 */
AQLM_API aqlm_status aqlm_gemv(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                      const uint16_t *x, uint16_t *y, int32_t tokens, aqlm_shape shape,
                      void *workspace, size_t workspace_bytes, aqlm_stream_t stream);

/* Bytes of device workspace aqlm_gemv needs for this shape and token count
 * on the current device (0 if none); returns 0 for invalid arguments too. */
AQLM_API size_t aqlm_gemv_workspace_bytes(aqlm_shape shape, int32_t tokens);

/* Most tokens for which aqlm_gemv and aqlm_gemv_multi run on the CUDA cores
 * with no device waits (1x16: 2, 2x16: 3, 2x8: 4); 0 for an unsupported
 * shape.  The value may change between library versions (it follows
 * measurements of both kernels), so ask rather than hard-code it. */
AQLM_API int32_t aqlm_gemv_row_tokens(aqlm_shape shape);

/*
 * aqlm_gemv_lut -- the 2x8 decode product for one token through lookup
 * tables: y = W^ . x computed as y_i = s_i * sum_j (L_0[j][b(i,j,0)] +
 * L_1[j][b(i,j,1)]) with L_m[j][k] = <C_m[k], x_j>, which equals the product
 * of section "What is Multi-Codebook Quantization (MCQ)?" because it is
 * linear in the codewords.  Each table entry is an fp32 sum of eight exact
 * fp16 products, each row the fp32 sum of its entries in a fixed order, y
 * rounded once to fp16: reproducible bit for bit, within the stated tolerance
 * of the exact product (not bit-identical to aqlm_gemv, whose summation order
 * differs).  Only shape 2x8 (else AQLM_ERR_UNSUPPORTED); x [1][d_in], y
 * [1][d_out]; workspace as aqlm_gemv's (size from
 * aqlm_gemv_lut_workspace_bytes, zero-filled before its first use, left ready
 * for the next call; calls sharing one must not overlap).  Launch with
 * programmatic dependent launch as aqlm_gemv; no device waits.  aqlm_gemv
 * does not use this kernel: on B200 it measured slower than the row kernel
 * at every tested shape.
 */
AQLM_API aqlm_status aqlm_gemv_lut(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                                   const uint16_t *x, uint16_t *y, aqlm_shape shape, void *workspace,
                                   size_t workspace_bytes, aqlm_stream_t stream);

/* Bytes of workspace aqlm_gemv_lut needs on the current device (0 if none,
 * or for a shape it does not take). */
AQLM_API size_t aqlm_gemv_lut_workspace_bytes(aqlm_shape shape);

/*
 * aqlm_gemv_multi -- the products y_l = W^_l . x of 1 to AQLM_MULTI_MAX_LAYERS
 * layers that read the SAME activations x, in one launch: e.g. the query, key
 * and value projections of an attention block, or the gate and up
 * projections of a feed-forward block.  Each layer is computed exactly as
 * aqlm_gemv computes it (same section of the pages, same arithmetic and the
 * same order of every addition, so each y_l is bit-for-bit aqlm_gemv's);
 * one launch instead of n_layers saves the launch-to-launch gaps, and the
 * layers' CTAs share the SMs in proportion to their rows.  Not a counterpart
 * of anything on the pages: a batching of their product.
 *   layers[n_layers]: HOST array; every layer has the format of `shape`
 *   (shape.d_in, group, num_codebooks, codebook_bits; shape.d_out is ignored)
 *   and its own codes, codebooks, scales, output and d_out >= 1.
 *   x: [tokens][d_in] fp16, read by every layer.
 *   tokens: 1 .. 16.  Up to aqlm_gemv_row_tokens(shape) the row kernel runs
 *   the layers with no device waits; past that the tensor-core kernel runs
 *   them (its row tiles of all layers share one work split), with bounded
 *   waits whose timeout status aqlm_gemv_multi_check() reads.
 *   workspace: as aqlm_gemv's, sized by aqlm_gemv_multi_workspace_bytes()
 *   (0 = none needed, NULL allowed); zero-filled before its first use, left
 *   ready for the next call; calls sharing it must not overlap on the GPU.
 * Errors: n_layers outside 1..AQLM_MULTI_MAX_LAYERS, a NULL pointer or tokens
 * outside 1..16 -> AQLM_ERR_INVALID_ARG; alignment as aqlm_gemv (per layer)
 * -> AQLM_ERR_MISALIGNED; no launch happens on any error but AQLM_ERR_CUDA.
 * Launch: programmatic dependent launch, as aqlm_gemv.
 */
AQLM_API aqlm_status aqlm_gemv_multi(const aqlm_layer *layers, int32_t n_layers, const uint16_t *x, int32_t tokens,
                                     aqlm_shape shape, void *workspace, size_t workspace_bytes,
                                     aqlm_stream_t stream);

/* Bytes of device workspace aqlm_gemv_multi needs for these layers (only
 * their d_out is read), format and token count on the current device (0 if
 * none); returns 0 for invalid arguments too. */
AQLM_API size_t aqlm_gemv_multi_workspace_bytes(const aqlm_layer *layers, int32_t n_layers, aqlm_shape shape,
                                                int32_t tokens);

/* aqlm_gemv_check for aqlm_gemv_multi calls with these layers (only their
 * d_out is read), format, token count and workspace. */
AQLM_API aqlm_status aqlm_gemv_multi_check(const aqlm_layer *layers, int32_t n_layers, aqlm_shape shape,
                                           int32_t tokens, void *workspace, size_t workspace_bytes,
                                           aqlm_stream_t stream);

/*
 * aqlm_gemv_check -- synchronise `stream` and return the status that the
 * aqlm_gemv calls with this shape, token count and workspace recorded:
 * AQLM_OK, or AQLM_ERR_TIMEOUT (the word is then cleared).  Paths without
 * device waits (up to AQLM_GEMV_ROW_TOKENS(shape) tokens) have no status word:
 * AQLM_OK after the synchronisation.  Not a counterpart of anything on the pages: library
 * plumbing for the bounded waits.
 */
AQLM_API aqlm_status aqlm_gemv_check(aqlm_shape shape, int32_t tokens, void *workspace, size_t workspace_bytes,
                                     aqlm_stream_t stream);

/*
 * aqlm_dequant -- the runtime dequantisation of section "Why and what do we
 * quantize?" (weights fetched compressed, turned back into native precision
 * before the matmul) with the decode of section "What is Multi-Codebook
 * Quantization (MCQ)?":
 *   W_out[i][8j+t] = bf16_rn( fp32(s_i) * ( fp32(C_0[b0][t]) + ... + fp32(C_{M-1}[b][t]) ) )
 * as separate IEEE binary32 operations in codebook order (no fused
 * multiply-add), then one round-to-nearest-even to bfloat16.  The result is
 * therefore bit-exact and deterministic.
 *   W_out: [d_out][d_in] bf16 (written), 16-byte aligned.
 */
AQLM_API aqlm_status aqlm_dequant(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                         uint16_t *W_out, aqlm_shape shape, aqlm_stream_t stream);

/*
 * aqlm_gemm -- prefill product Y = X . W^T for many tokens: aqlm_dequant into
 * the workspace (W^, bf16), then the tcgen05 tensor-core GEMM of
 * aqlm_bf16_gemm (bf16 operands, fp32 accumulation in tensor memory, bf16
 * output rounded to nearest even; CTA pairs past 128 tokens, see
 * aqlm_bf16_gemm_plan), launched early so that its set-up overlaps the
 * dequantisation's end.  Past 128 tokens, aqlm_gemm_overlap's path instead
 * where it was measured faster on B200: two 16-bit codebooks always, the
 * other formats when the bands its first wave of tiles needs are at most a
 * third of the layer.  Either way Y equals aqlm_bf16_gemm on aqlm_dequant's W^.
 *   X: [tokens][d_in] bf16.  Y: [tokens][d_out] bf16 (written).  tokens >= 1.
 *   workspace: at least aqlm_gemm_workspace_bytes(shape, tokens) bytes,
 *   16-byte aligned: a 256-byte status word, the counters aqlm_gemm_overlap
 *   uses, and W^ in the last 2 * d_out * d_in bytes.
 *   Every device-side wait of the GEMM is bounded; a wait that gives up
 *   records AQLM_ERR_TIMEOUT in the workspace's status word (read it with
 *   aqlm_gemm_check) and the kernel returns without trapping.
 * Extra requirement: d_out % 8 == 0 (else AQLM_ERR_UNSUPPORTED).
 */
AQLM_API aqlm_status aqlm_gemm(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                      const uint16_t *X, uint16_t *Y, int32_t tokens, aqlm_shape shape,
                      void *workspace, size_t workspace_bytes, aqlm_stream_t stream);

AQLM_API size_t aqlm_gemm_workspace_bytes(aqlm_shape shape, int32_t tokens);

/*
 * aqlm_gemm_overlap -- the product of aqlm_gemm with the decoding overlapped
 * with the MMAs, each W^ block decoded once: aqlm_dequant's kernel first
 * decodes the bands of W^ that the GEMM's first wave of tiles needs, then ONE
 * kernel does the rest: the CTA-pair
 * GEMM (aqlm_bf16_gemm_plan's width for more than 128 tokens; the same
 * kernel with half-empty pair tiles below) with eight decoder warps and a
 * publisher warp in every CTA.  The decoders write W^ into the workspace in
 * the order the tiles need it (units of 16 rows x 64 inputs, claimed from
 * global counters) with the binary32 steps of aqlm_dequant; a CTA's TMA load
 * of a W^ tile waits (bounded) until the counters say every unit that writes
 * it is done.  The page this follows, "The AQLM Quantization Algorithm,
 * Explained", section "Why and what do we quantize?": the weights are
 * fetched compressed and dequantised at runtime before the matmul.  W^ left
 * in the workspace equals aqlm_dequant's output and Y equals
 * aqlm_bf16_gemm_config on it with the CTA pair at the same width, bit for
 * bit.  Arguments, workspace (aqlm_gemm_workspace_bytes) and errors as
 * aqlm_gemm; a bounded wait that gives up records AQLM_ERR_TIMEOUT in the
 * status word (aqlm_gemm_check).  Every CTA of the grid must be resident
 * for the decoding to be shared: the grid is the device's co-resident pair
 * count at most, and a unit is always claimed by a running warp.  On B200 it
 * runs as fast as aqlm_gemm's two kernels, within a few per cent either way.
 */
AQLM_API aqlm_status aqlm_gemm_overlap(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                                       const uint16_t *X, uint16_t *Y, int32_t tokens, aqlm_shape shape,
                                       void *workspace, size_t workspace_bytes, aqlm_stream_t stream);

/*
 * aqlm_gemm_fused -- the prefill product of aqlm_gemm, Y = bf16(X . W^T),
 * with the dequantisation fused into the GEMM: extra warps of every GEMM CTA
 * decode the W^ rows of its own output tiles, 64 inputs at a time, straight
 * into the tensor cores' shared-memory operand tiles, with the same binary32
 * steps as aqlm_dequant (so Y equals aqlm_gemm's, bit for bit).  No W^ is
 * written to global memory: the workspace is only the 256-byte status word
 * (aqlm_gemm_fused_workspace_bytes), for callers that cannot hold the bf16
 * copy of a layer (90 MB for 11008 x 4096).  The page this follows, "The
 * AQLM Quantization Algorithm, Explained", section "Why and what do we
 * quantize?": weights are fetched compressed and dequantised at runtime.
 * Each 128-token tile decodes its W^ rows again (16 times for 2048 tokens),
 * so on B200 it is slower than aqlm_gemm (the decoding competes with the
 * tensor cores for shared-memory bandwidth; 1x16 and 2x16 also gather their
 * codewords from L2).  Arguments, alignment, waits and aqlm_gemm_check as for
 * aqlm_gemm.
 */
AQLM_API aqlm_status aqlm_gemm_fused(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                                     const uint16_t *X, uint16_t *Y, int32_t tokens, aqlm_shape shape,
                                     void *workspace, size_t workspace_bytes, aqlm_stream_t stream);

AQLM_API size_t aqlm_gemm_fused_workspace_bytes(aqlm_shape shape, int32_t tokens);

/*
 * aqlm_gemm_check -- synchronises `stream`, reads and clears the status word
 * that aqlm_gemm calls with this workspace recorded.  Returns AQLM_OK,
 * AQLM_ERR_TIMEOUT, or AQLM_ERR_CUDA if the stream itself reports an error.
 */
AQLM_API aqlm_status aqlm_gemm_check(void *workspace, size_t workspace_bytes, aqlm_stream_t stream);

/*
 * aqlm_bf16_gemm -- the tensor-core GEMM of aqlm_gemm on its own, for a dense
 * bf16 weight: Y[tokens][n] = X[tokens][k] . W[n][k]^T.  n % 8 == 0, k % 8
 * == 0, all matrices 16-byte aligned; `status` is a device int32 that
 * receives AQLM_ERR_TIMEOUT if a bounded wait gives up (it is only ever
 * written with a non-zero value; clear it yourself).
 */
AQLM_API aqlm_status aqlm_bf16_gemm(const uint16_t *X, const uint16_t *W, uint16_t *Y, int32_t tokens,
                           int32_t n, int32_t k, int32_t *status, aqlm_stream_t stream);

/*
 * aqlm_bf16_gemm_tile_n -- the output tile width (columns of W per tile:
 * 256, 240, 224 or 192) that aqlm_bf16_gemm and aqlm_gemm use for `tokens`
 * x `n` on a device with `sms` streaming multiprocessors: the width with the
 * least waves x (128 + width), ties to the wider.  Host only; returns 0 if an
 * argument is below 1.
 */
AQLM_API int32_t aqlm_bf16_gemm_tile_n(int32_t tokens, int32_t n, int32_t sms);

/*
 * aqlm_bf16_gemm_plan -- the kernel aqlm_bf16_gemm and aqlm_gemm choose for
 * `tokens` x `n` on a device with `sms` streaming multiprocessors, written to
 * *cta_pair and *tile_n.  More than 128 tokens: the CTA-pair kernel
 * (*cta_pair = 1; one MMA of 256 x tile_n on the tensor cores of two SMs, a
 * cluster of two CTAs), whose width is the one with the least waves x width
 * over sms / 2 pairs, ties to the wider.  Otherwise the single-CTA kernel
 * (*cta_pair = 0) with the width of aqlm_bf16_gemm_tile_n.  The launch uses
 * the pair count the device reports for the kernel, which on a device whose
 * SMs all pair up is sms / 2.  Host only.  Errors: AQLM_ERR_INVALID_ARG
 * (null pointer, tokens or n below 1, sms below 2; both outputs then 0).
 */
AQLM_API aqlm_status aqlm_bf16_gemm_plan(int32_t tokens, int32_t n, int32_t sms, int32_t *cta_pair,
                                         int32_t *tile_n);

/*
 * aqlm_bf16_gemm_config -- aqlm_bf16_gemm with the kernel chosen by the
 * caller, for measurements and tests of each variant: cta_pair 1 = the
 * CTA-pair kernel (256-token tiles), 0 = the single-CTA kernel (128-token
 * tiles), -1 = the rule of aqlm_bf16_gemm_plan; tile_n one of 256, 240, 224,
 * 192, or 0 for the rule's width.  Every variant computes the same products
 * with the same fp32 accumulation order within a tile column (16 k values
 * per MMA step, k steps in order), so the results agree bit for bit.
 * Arguments and errors as aqlm_bf16_gemm, plus AQLM_ERR_INVALID_ARG for
 * another cta_pair or tile_n, and AQLM_ERR_CUDA when the device cannot
 * hold a CTA pair.
 */
AQLM_API aqlm_status aqlm_bf16_gemm_config(const uint16_t *X, const uint16_t *W, uint16_t *Y, int32_t tokens,
                                           int32_t n, int32_t k, int32_t *status, int32_t cta_pair,
                                           int32_t tile_n, aqlm_stream_t stream);

/*
 * aqlm_decode_indices -- the code unpacking step on its own, for bit-exact
 * checks: idx_out[(i*G + j)*M + m] = index of codebook m for group j of row
 * i, as uint16 (G = d_in/8).  idx_out: d_out*G*M uint16, 2-byte aligned.
 * Storing an index of B bits per codebook per group is the code
 * representation of section "What is Multi-Codebook Quantization (MCQ)?".
 */
AQLM_API aqlm_status aqlm_decode_indices(const void *codes, uint16_t *idx_out, aqlm_shape shape,
                                aqlm_stream_t stream);

/*
 * aqlm_test_gemm_timeout -- test hook for the GEMM's failure detection: runs
 * the kernel of aqlm_bf16_gemm with its loads withheld, so that the first
 * bounded wait runs out after `limit_ns` nanoseconds (1 ns .. 1 s).  The
 * kernel must then write AQLM_ERR_TIMEOUT to *status, free its tensor
 * memory and return; nothing faults or hangs.  cta_pair selects the kernel
 * as in aqlm_bf16_gemm_config (with the CTA pair, the timeout of the
 * leader's wait also ends the other CTA's waits).  Other arguments as
 * aqlm_bf16_gemm.
 */
AQLM_API aqlm_status aqlm_test_gemm_timeout(const uint16_t *X, const uint16_t *W, uint16_t *Y, int32_t tokens, int32_t n,
                                   int32_t k, int32_t *status, uint64_t limit_ns, int32_t cta_pair,
                                   aqlm_stream_t stream);

/*
 * aqlm_gemv_noalloc -- aqlm_gemv without a caller-provided workspace, for
 * callers that cannot allocate device memory (for example a plugin that its
 * host engine hands only input and output pointers, or an engine that fixes
 * its device memory at start-up and allows no allocation afterwards).  The
 * paper has no counterpart of this entry point; it is a library convenience.
 *
 * The scratch it needs lives in a fixed array inside the library, 8 MiB per
 * GPU (aqlm_gemv_noalloc_max_scratch_bytes()), held by every GPU that loads
 * the library until the process exits.  Arguments are checked as aqlm_gemv
 * checks them before anything is enqueued.  The first call on a device looks
 * up the array's
 * device address there (cudaGetSymbolAddress); make that first call before
 * any stream capture (a lookup that fails is not kept: the next call tries
 * again).  Each call clears the array's arrival counters on `stream`; the
 * status word (the array's last 16 bytes, which no call's other data ever
 * reaches) is left alone, so a bounded wait that gave up (4 tokens and more,
 * see aqlm_gemv) stays recorded, whatever calls follow, until
 * aqlm_gemv_noalloc_check reads it.  A shape and token count whose scratch
 * exceeds the array (less those 16 bytes where the path has no status word)
 * is rejected with AQLM_ERR_WORKSPACE.  All calls on a device share the one
 * array and it keeps the last call's contents: calls that overlap on the GPU
 * (other streams, other host threads) race and must be avoided.  No
 * cudaMalloc, cudaFree or other allocating routine is called.  Results and
 * errors otherwise as aqlm_gemv.
 */
AQLM_API aqlm_status aqlm_gemv_noalloc(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                                       const uint16_t *x, uint16_t *y, int32_t tokens, aqlm_shape shape,
                                       aqlm_stream_t stream);

/* Size of aqlm_gemv_noalloc's built-in scratch array, in bytes. */
AQLM_API size_t aqlm_gemv_noalloc_max_scratch_bytes(void);

/* aqlm_gemv_check for aqlm_gemv_noalloc: synchronise `stream`, then read and
 * clear the status word of the current device's built-in array: AQLM_OK, or
 * AQLM_ERR_TIMEOUT if a bounded wait of any aqlm_gemv_noalloc call since the
 * last check gave up (that call's y is not valid).  No counterpart on the
 * pages. */
AQLM_API aqlm_status aqlm_gemv_noalloc_check(aqlm_stream_t stream);

/* Test only: write `value` into that status word and synchronise, so that
 * tests can check the reporting without making a device wait run out. */
AQLM_API aqlm_status aqlm_test_gemv_noalloc_set_status(int32_t value, aqlm_stream_t stream);

/* ===========================================================================
 * Encoding: scales, codebooks and codes of a layer from its weights.
 *
 * Section "AQLM quantization process" of "The AQLM Quantization Algorithm,
 * Explained": codes are learned with the codebooks and scales fixed, the
 * codebooks initialised "with a residual k-means approach".  The pages give
 * no loss, search or update rule beyond that; the readings taken here are:
 *   scale s_i   root mean square of row i rounded to fp16 (1.0 if it rounds to
 *               0); the sum of squares is taken in double, so the result is
 *               the correctly rounded one unless the root mean square lies
 *               within (d_in + 4) 2^-53 (relative) of a rounding boundary;
 *   groups      v = W[i][8j .. 8j+7] / s_i (binary32 division), [d_out*d_in/8][8];
 *   nearest     least squared Euclidean distance |v - c|^2, ties to the lowest
 *               index.  Evaluated in binary32 as the score |c|^2 - 2<v, c>
 *               (|v|^2 is common to every codeword), whose error is at most
 *               beta(c) = gamma_9 (|c|^2 + 2 sum_t |v_t c_t|), gamma_n =
 *               n u / (1 - n u), u = 2^-24: the chosen codeword k satisfies
 *               |v - c_k|^2 <= min_c |v - c|^2 + beta(c_k) + beta(c_min), and is
 *               the exact nearest wherever no other codeword lies that close;
 *   distance    (reported for the chosen codeword) its squared distance in
 *               binary32, within gamma_10 (relative) of the exact value;
 *   k-means     a centroid becomes the mean of its groups (sums in double, one
 *               rounding), one without groups keeps its value; codebook m is
 *               k-means of the residuals left by codebooks 0..m-1;
 *   codes       greedy, codebook by codebook: the nearest codeword of the
 *               residual, which then loses that codeword (binary32).
 * Every integer result (index, code, count) is deterministic; centroids sum
 * in double with atomics, so their last binary32 bit may depend on order.
 * The workspace of each call is device scratch of the size its
 * *_workspace_bytes query gives; nothing needs to be zero beforehand.
 * All float arrays are fp32, 16-byte aligned.
 * ======================================================================== */

/* E1/E2: scales[d_out] (fp16) and groups [d_out*d_in/8][8] (fp32) of W
 * [d_out][d_in] (fp32).  d_in % 8 == 0. */
AQLM_API aqlm_status aqlm_encode_scales(const float *W, int32_t d_out, int32_t d_in, uint16_t *scales, float *groups,
                                        aqlm_stream_t stream);

/* Nearest codeword of each of n groups [n][8] in a codebook [K][8]:
 * idx[n] (int32) and, if dist is not NULL, its distance. */
AQLM_API size_t aqlm_nearest_workspace_bytes(int64_t n);
AQLM_API aqlm_status aqlm_nearest_codeword(const float *groups, int64_t n, const float *codebook, int32_t K,
                                           int32_t *idx, float *dist, void *workspace, size_t workspace_bytes,
                                           aqlm_stream_t stream);

/* One k-means update: centroids_out[K][8] from the groups and their
 * assignments idx[n] (indices outside 0..K-1 are ignored); counts (int32
 * [K], may be NULL) receives the group count of every centroid. */
AQLM_API size_t aqlm_kmeans_workspace_bytes(int32_t K);
AQLM_API aqlm_status aqlm_kmeans_update(const float *groups, const int32_t *idx, int64_t n, const float *centroids,
                                        int32_t K, float *centroids_out, int32_t *counts, void *workspace,
                                        size_t workspace_bytes, aqlm_stream_t stream);

/* Residual k-means: M codebooks [M][K][8] (fp32) of the n groups, `iters`
 * updates each.  init_idx is a HOST array [M][K] of group indices (0..n-1,
 * else AQLM_ERR_INVALID_ARG): codebook m starts from the residuals they name
 * (the random draw of the initialisation, made by the caller).  Copies
 * init_idx from pageable host memory, so it is not for stream capture. */
AQLM_API size_t aqlm_residual_kmeans_workspace_bytes(int64_t n, int32_t M, int32_t K);
AQLM_API aqlm_status aqlm_residual_kmeans(const float *groups, int64_t n, int32_t M, int32_t K,
                                          const int32_t *init_idx, int32_t iters, float *codebooks, void *workspace,
                                          size_t workspace_bytes, aqlm_stream_t stream);

/* Greedy codes of the d_out*d_in/8 groups against fp16 codebooks
 * [M][2^B][8], written as the codes of `shape` ([d_out][d_in/8][M], uint8 or
 * 16-bit) -- the layout aqlm_gemv, aqlm_dequant and aqlm_gemm read. */
AQLM_API size_t aqlm_encode_codes_workspace_bytes(aqlm_shape shape);
AQLM_API aqlm_status aqlm_encode_codes(const float *groups, const uint16_t *codebooks, void *codes, aqlm_shape shape,
                                       void *workspace, size_t workspace_bytes, aqlm_stream_t stream);

/* The whole encoding of a layer W [d_out][d_in] (fp32): scales, residual
 * k-means codebooks (iters updates each, started from init_idx, a HOST array
 * [M][2^B] of group indices below d_out*d_in/8) rounded to fp16, greedy codes.
 * Outputs in the inference layout: codes, codebooks [M][2^B][8] fp16, scales
 * [d_out] fp16.  Not for stream capture (see aqlm_residual_kmeans). */
AQLM_API size_t aqlm_encode_layer_workspace_bytes(aqlm_shape shape);
AQLM_API aqlm_status aqlm_encode_layer(const float *W, aqlm_shape shape, const int32_t *init_idx, int32_t iters,
                                       void *codes, uint16_t *codebooks, uint16_t *scales, void *workspace,
                                       size_t workspace_bytes, aqlm_stream_t stream);

/* ===========================================================================
 * Measurement: the random 16-byte gather rate.
 *
 * Not part of the method.  At one token a decode product gathers one random
 * 16-byte codeword per group and codebook ("The AQLM Quantization Algorithm,
 * Explained", section "Key AQLM quantization parameters": more codewords make
 * decoding slower); aqlm_probe_gather launches ctas_per_sm (1..8) CTAs of
 * 256 threads per SM that each make `iters` x 8 random 16-byte reads of
 * `table` (table_bytes, a multiple of 16), through the load the 1x16 / 2x16
 * decode kernels use for codewords (L1 evict-last, L2 evict-last; source 0)
 * or from a copy of the table in shared memory (source 1, table_bytes <=
 * 64 KiB; the 2x8 kernels' path).  *gathers (host) receives the number of
 * reads the launch makes; time it with events on `stream`.  `sink` (device,
 * aqlm_probe_gather_sink_bytes(ctas_per_sm) bytes, 16-byte aligned) receives
 * one word per thread so the reads are not optimised away.
 * ======================================================================== */
AQLM_API size_t aqlm_probe_gather_sink_bytes(int32_t ctas_per_sm);
AQLM_API aqlm_status aqlm_probe_gather(const void *table, size_t table_bytes, int32_t source, int32_t ctas_per_sm,
                                       int32_t iters, void *sink, size_t sink_bytes, uint64_t *gathers,
                                       aqlm_stream_t stream);

/* ===========================================================================
 * Debug bounds checks.
 *
 * Not part of the method.  The library built with -DAQLM_DEBUG_BOUNDS
 * (libaqlm_b200_debug_bounds.so, `python -m additive_codebook_b200.build
 * --debug-bounds`) tests, in every kernel, the computed indices of its global
 * and shared-memory accesses before making them; an index out of range is
 * recorded -- the first one, as (site << 48 | index), the sites numbered in
 * csrc/common.cuh -- in a device word, and the access is skipped.  Nothing
 * traps.  aqlm_debug_bounds_read stores that word (0: no violation since the
 * last clear) in *word (host memory), clearing it if `clear`; it
 * synchronises the device.  The product build returns AQLM_ERR_UNSUPPORTED.
 * aqlm_test_debug_bounds_trip records a violation at site 23 with `index` on
 * purpose, touching no memory (a test of the mechanism; AQLM_ERR_UNSUPPORTED
 * in the product build).
 * ======================================================================== */
AQLM_API aqlm_status aqlm_debug_bounds_read(uint64_t *word, int32_t clear);
AQLM_API aqlm_status aqlm_test_debug_bounds_trip(uint64_t index, aqlm_stream_t stream);

/* A static, human-readable name of a status code. */
AQLM_API const char *aqlm_status_string(aqlm_status status);

/* Library version, e.g. "0.1.0". */
AQLM_API const char *aqlm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AQLM_B200_H */
