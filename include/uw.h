/*
 * uw.h -- C ABI of libuw: lossless BF16 exponent compression with fused
 * decode-matmul kernels for NVIDIA B200 (sm_100a).
 *
 * The method follows the web page "Unweight：Cloudflare 如何在不损失精度的情况下
 * 把大模型压缩 22%" (cited below as "the Unweight page", by section number):
 *   §三  a BF16 weight is 1 sign, 8 exponent and 7 mantissa bits; only the
 *        exponent is predictable (few values dominate, ~2.6 bits of entropy).
 *   §四  the sign+mantissa byte stays raw, the exponent byte is Huffman coded;
 *        any row of 64 weights holding an exponent outside the matrix's top-16
 *        palette is stored raw, so the hot loop needs no per-element branch.
 *   §五  decompress next to the compute, never back to HBM, to save bandwidth.
 *   §六  four pipelines: full decode + GEMM, exponent-only decode, runtime
 *        Huffman -> 4-bit palette transcode, and pre-transcoded palette; here
 *        also a fifth, the runtime transcode done inside the matmul kernel.
 *   §七  reconstructive matmul: compressed tiles are staged into shared memory,
 *        rebuilt to BF16 there and fed straight to the tensor cores.
 *   §九  an autotuner measures the pipelines, the kernel variants and the
 *        decode/compute SM split per projection and batch size and writes a
 *        per-model plan.
 *   §十一 mixture-of-experts models are the next target (many small
 *        expert matrices).
 *
 * Conventions for every entry point:
 *   - Returns a uw_status; nothing throws across the ABI.
 *   - Matrices are row-major.  W is [n, k] (one output feature per row), X is
 *     [m, k] BF16, Y is [m, n] float32, Y = X * W^T.  BF16 values are passed
 *     as their raw 16-bit patterns (uint16_t).
 *   - n and k must be positive multiples of 64 (UW_ERR_UNSUPPORTED_SHAPE).
 *     Null required pointers, m <= 0 and bad plans give UW_ERR_INVALID_ARG.
 *   - Device work is launched asynchronously on the given stream (a
 *     cudaStream_t passed as void*; NULL = legacy default stream).  Argument
 *     errors are reported synchronously.  Errors found by a kernel (corrupt
 *     stream, spin-wait time-out) are OR-ed into the matrix's device status
 *     word and returned by uw_device_status() after the stream is drained.
 *   - The caller owns every device buffer: the device copy of a blob, its
 *     status word, X, Y, decode/transcode outputs and workspaces.  The library
 *     allocates no device memory.  It owns only the host blobs that uw_encode
 *     returns; free them with uw_blob_free.
 *   - Calls are thread-safe as long as no two calls write the same buffers.
 *   - Early start: a direct-palette matmul on the blob's own 4-bit plane
 *     (pipeline 4, no separate palette plane) with the warp-MMA or tcgen05
 *     kernel is launched with programmatic stream serialization.  Its CTAs
 *     may be scheduled, and may read the blob's compressed planes, while the
 *     previous libuw kernel on the stream is still draining; X is read, and
 *     Y and the workspace are written, only after that kernel has completed.
 *     Kernels of other libraries on the stream end before it starts, as
 *     usual.  The library never writes a blob's device copy.
 */
#ifndef UW_H
#define UW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum uw_status {
    UW_OK = 0,
    UW_ERR_INVALID_ARG = 1,        /* null pointer, non-positive size, bad plan field */
    UW_ERR_UNSUPPORTED_SHAPE = 2,  /* n or k not a multiple of 64, or too large */
    UW_ERR_CORRUPT = 3,            /* blob header/CRC/section check failed, or a kernel
                                      found an inconsistent bitstream */
    UW_ERR_CUDA = 4,               /* a CUDA runtime call failed */
    UW_ERR_NOMEM = 5,              /* host allocation failed */
    UW_ERR_TIMEOUT = 6,            /* a kernel's bounded spin-wait ran out */
    UW_ERR_WORKSPACE = 7           /* workspace missing or smaller than uw_workspace_size */
} uw_status;

/* Human-readable name of a status code (static string). */
const char *uw_status_str(int status);
/* Library version string, e.g. "uw 1.1 (blob v2, sm_100a)". */
const char *uw_version(void);

/* ------------------------------------------------------------------------ */
/* Host encoder (Unweight page §三, §四, §六).                                */

#define UW_EMIT_HUFFMAN 1u   /* Huffman exponent stream (pipelines 1, 2, 3)    */
#define UW_EMIT_PALETTE 2u   /* pre-transcoded 4-bit palette plane (pipeline 4) */

/* Sections of a blob (each 256-byte aligned inside the blob). */
enum {
    UW_SEC_SM = 0,        /* uint8[n*k]   sign<<7 | mantissa of every weight          */
    UW_SEC_RAWEXP = 1,    /* uint8[n_raw*64] exponents of raw groups, group order      */
    UW_SEC_FLAGS = 2,     /* uint32[] bit g%32 of word g/32 = group g is raw           */
    UW_SEC_RAWBASE = 3,   /* uint32[] raw groups before word w of FLAGS (prefix count) */
    UW_SEC_STREAM = 4,    /* uint32[] Huffman bits, MSB of each word first, 0-padded   */
    UW_SEC_CHUNKOFF = 5,  /* uint32[n_chunks+1] start bit of each 4-group chunk        */
    UW_SEC_DLUT = 6,      /* uint32[4096] 12-bit-window multi-symbol decode table:
                             bits 0..19 up to 5 symbols (first lowest), bits 20..24
                             4 x their count, bit 25 no code matches, bits 28..31
                             stream bits they use (12 when none matches)        */
    UW_SEC_PAL = 7,       /* uint8[n*k/2] 4-bit palette indices: each little-endian
                             u32 word holds 8 consecutive weights; weight j's index v
                             has v&7 at bits 4j..4j+2 and v>>3 at bit 8j+7 (j<4) or
                             bit 8(j-4)+3 (j>=4); raw groups hold 0                */
    UW_NUM_SECTIONS = 8
};

typedef struct uw_blob uw_blob;   /* opaque host-side serialized matrix */

typedef struct uw_blob_info {
    int64_t n, k;
    uint32_t flags;              /* UW_EMIT_* present in the blob */
    int32_t palette_size;        /* 1..16 */
    uint8_t palette[16];         /* exponent values, ascending; index = position */
    uint8_t code_len[16];        /* Huffman code length per palette index (0 = unused) */
    int64_t n_groups;            /* n*k/64 */
    int64_t n_raw;               /* raw groups */
    int64_t n_chunks;            /* ceil(n_groups/4) */
    uint64_t stream_bits;
    double entropy_bits;         /* Shannon entropy of the 256-bin exponent histogram */
    double top16_coverage;       /* fraction of weights whose exponent is in the palette */
    uint64_t total_bytes;        /* serialized size */
    uint64_t huffman_bytes;      /* bytes needed to keep the Huffman form */
    uint64_t palette_bytes;      /* bytes needed to keep the palette form */
    uint64_t section_offset[UW_NUM_SECTIONS];
    uint64_t section_bytes[UW_NUM_SECTIONS];
} uw_blob_info;

/* Encode one BF16 matrix w[n,k] (host memory, raw bit patterns).
 * flags: UW_EMIT_HUFFMAN and/or UW_EMIT_PALETTE (0 means both).
 * On success *out owns a new blob (free with uw_blob_free).  Bit-exact and
 * deterministic: the same input always gives the same bytes.
 * Errors: INVALID_ARG (null), UNSUPPORTED_SHAPE (n,k not multiples of 64, or a
 * Huffman stream that would exceed 2^32 bits), NOMEM.                        */
uw_status uw_encode(const uint16_t *w, int64_t n, int64_t k, uint32_t flags, uw_blob **out);

/* Pointer to the serialized bytes of a blob and their count (owned by blob). */
const void *uw_blob_data(const uw_blob *blob, size_t *bytes);
void uw_blob_free(uw_blob *blob);

/* Parse and check a serialized blob held in host memory (e.g. read from
 * disk).  Checks magic, version, header CRC and section bounds; with
 * verify_payload != 0 also the CRC over all sections.  Fills *info.        */
uw_status uw_blob_info_get(const void *host_blob, size_t bytes, int verify_payload,
                           uw_blob_info *info);

/* ------------------------------------------------------------------------ */
/* Device view of a blob.                                                     */

typedef struct uw_dmat {
    int64_t n, k;
    uint32_t flags;
    int32_t palette_size;
    uint8_t palette[16];
    uint8_t code_len[16];
    int64_t n_groups, n_raw, n_chunks;
    uint64_t stream_bits;
    uint64_t stream_words;          /* padded word count of the stream section */
    const uint8_t *sm;              /* device pointers into the device blob */
    const uint8_t *rawexp;
    const uint32_t *flagbits;
    const uint32_t *rawbase;
    const uint32_t *stream;
    const uint32_t *chunk_off;
    const uint32_t *dlut;
    const uint8_t *pal;             /* NULL if the blob has no palette plane */
    uint32_t *dev_status;           /* caller's device word for kernel error flags */
} uw_dmat;

/* Bind a device copy of a blob.  host_blob/bytes is a host copy used to read
 * the header (no device read happens); dev_blob must hold the same bytes and
 * be 256-byte aligned.  dev_status points to one caller-owned device uint32
 * (zero it before use) that kernels OR error bits into.  verify_payload as in
 * uw_blob_info_get.  Fills *out; keeps no reference to host_blob.            */
uw_status uw_matrix_bind(const void *host_blob, size_t bytes, const void *dev_blob,
                         uint32_t *dev_status, int verify_payload, uw_dmat *out);

/* Device error bits OR-ed into *dev_status by kernels. */
#define UW_DEVERR_CORRUPT 1u
#define UW_DEVERR_TIMEOUT 2u

/* Synchronize `stream`, read and clear *w->dev_status.  Returns UW_OK,
 * UW_ERR_CORRUPT or UW_ERR_TIMEOUT (CORRUPT wins if both are set).           */
uw_status uw_device_status(const uw_dmat *w, void *stream);

/* ------------------------------------------------------------------------ */
/* Preprocessing kernels (Unweight page §六, pipelines 1, 2 and 3).           */

/* Full Huffman decode to BF16: out_dev is uint16[n*k] (caller-owned, device,
 * 16-byte aligned).  Needs UW_EMIT_HUFFMAN.  Bit-exact inverse of uw_encode. */
uw_status uw_decode_to_bf16(const uw_dmat *w, uint16_t *out_dev, void *stream);

/* Exponent-only Huffman decode: exp_dev is uint8[n*k] (device, 16-byte
 * aligned) and receives every weight's exponent byte, (bits >> 7) & 0xFF, in
 * weight order (raw groups included), i.e. half the bytes of a full decode.
 * Needs UW_EMIT_HUFFMAN.                                                      */
uw_status uw_decode_exponents(const uw_dmat *w, uint8_t *exp_dev, void *stream);

/* Runtime transcode of the Huffman stream to the 4-bit palette plane:
 * pal_dev is uint8[n*k/2] (device, 16-byte aligned), byte-identical to the
 * blob's own UW_SEC_PAL section.  Needs UW_EMIT_HUFFMAN.                     */
uw_status uw_transcode_palette(const uw_dmat *w, uint8_t *pal_dev, void *stream);

/* ------------------------------------------------------------------------ */
/* Matmul (Unweight page §六-§七).                                            */

typedef enum uw_pipeline {
    UW_PIPE_DECODE_GEMM = 1,      /* decode to BF16 in the workspace, then the plain kernel */
    UW_PIPE_DECODE_EXP_FUSED = 2, /* decode only the exponents (n*k bytes) into the
                                     workspace, then the fused kernel rebuilding BF16
                                     from the sign/mantissa and exponent bytes      */
    UW_PIPE_TRANSCODE_FUSED = 3,  /* transcode to the palette plane in the workspace, then
                                     the fused kernel                                    */
    UW_PIPE_DIRECT_PALETTE = 4,   /* fused kernel on the blob's (or a given) palette plane */
    UW_PIPE_HUFFMAN_FUSED = 5     /* the fused stream-K kernel decodes the Huffman stream to
                                     palette indices in shared memory as it goes (pipeline 3's
                                     transcode inside the matmul's producer): no preprocessing
                                     pass and no workspace beyond the stream-K scratch.  Needs
                                     UW_EMIT_HUFFMAN, kernel UW_KERNEL_TC_SK with bn <= 32 and
                                     k a multiple of 256 (a 4-group stream chunk never
                                     straddles two rows); UW_ERR_INVALID_ARG otherwise       */
} uw_pipeline;

typedef enum uw_kernel {
    UW_KERNEL_FMA = 1,   /* CUDA-core FMA GEMV, one warp per `bn` rows, m <= 8       */
    UW_KERNEL_TC = 2,    /* tcgen05 MMA with a TMEM accumulator, token tile `bn`      */
    UW_KERNEL_MMA = 3,   /* m <= 16: W rebuilt in registers straight into warp-level
                            MMA fragments; one CTA per 16-row tile, whose `bn`
                            warps split K (summed in a fixed order)               */
    UW_KERNEL_TC_SK = 4, /* any m: persistent stream-K tcgen05 kernel, token tile
                            `bn`, one CTA per SM, each owning an equal contiguous
                            run of (128-row x bn tile, 64-wide K-step) units; a
                            tile cut between CTAs is summed in CTA (= K) order by
                            the CTA that finishes its last piece.  Needs a
                            workspace whose tile counters are zero (see
                            uw_workspace_size); split_k must be 1             */
    UW_KERNEL_MMA_SK = 5 /* m <= 16, k a multiple of 128, n*k < 2^32 (a larger matrix
                            fails at launch, UW_ERR_CUDA): persistent stream-K form of
                            UW_KERNEL_MMA, one CTA of `bn` (1..16) warps per SM;
                            every warp owns an equal contiguous run of (16-row
                            tile, 128-wide K chunk) units and stages its loads
                            in a shared-memory ring filled by 2-D TMA boxes; a tile
                            cut between warps is summed in warp (= K) order by
                            the warp that finishes its last piece.  Needs a
                            workspace whose tile counters are zero, as TC_SK;
                            split_k must be 1                                 */
} uw_kernel;

#define UW_DEBUG_NEVER_ARRIVE 1u   /* TC kernel: wait on a barrier nobody signals, so
                                      the bounded wait runs out (time-out test)      */

typedef struct uw_plan {
    int32_t pipeline;     /* uw_pipeline */
    int32_t kernel;       /* uw_kernel */
    int32_t bn;           /* TC: tokens per tile, one of 16,32,64,128,256;
                             FMA: weight rows per warp, 1 or 2;
                             MMA: warps per CTA = K slices per 16-row tile, 1..8;
                             MMA_SK: warps per CTA (one CTA per SM), 1..16 */
    int32_t split_k;      /* TC: K split into this many slices (>= 1), reduced in a
                             fixed order; FMA, MMA, TC_SK, MMA_SK: must be 1 */
    int32_t stages;       /* TC: shared-memory ring depth (0 = default: 4 for the plain
                             kernel, the largest that fits for the fused one);
                             TC_SK: compressed-tile ring depth of the fused kernel
                             (W-tile ring of the plain one), 0 = the largest that
                             fits (at most 6 / 8);
                             MMA: weights per lane and row per step, 1 = 16, 2 = 32
                             (K a multiple of 128), 0 = 32 when K allows, else 16;
                             MMA_SK: ring slots per warp (2..8) of 5128 + 256 m
                             bytes each, bn x stages slots within 227 KB less
                             128 bytes; 0 = the deepest that fits, at most 8 */
    uint32_t debug_flags; /* UW_DEBUG_* (0 in production) */
    int64_t timeout_ns;   /* spin-wait limit inside kernels (0 = 2 s) */
} uw_plan;

/* A reasonable plan without measuring: the warp-MMA kernel (4 warps per
 * tile) for m <= 8, the tcgen05 kernel otherwise.  uw_plan_autotune measures. */
uw_status uw_plan_default(int64_t m, int64_t n, int64_t k, int32_t pipeline, uw_plan *plan);

/* Workspace bytes uw_fused_matmul needs for this plan (0 is possible): the
 * preprocessing output (pipeline 1: 2nk bytes of BF16; pipeline 2: the nk-byte
 * exponent plane plus two nk/2048-word index arrays; pipeline 3: nk/2 bytes;
 * pipeline 4: none), each part rounded up to 256 bytes, plus split_k*m*n
 * floats of partial sums for a TC plan with split_k > 1, or for a TC_SK plan
 * one uint32 counter per 128 x bn tile (256-byte rounded) followed by two
 * 128 x bn float tiles per CTA (one CTA per SM of the current device), or
 * for an MMA_SK plan one uint32 counter per 16-row tile (256-byte rounded)
 * followed by two sets of 128 (m <= 8) or 256 floats per warp of the grid
 * (bn warps per SM of the current device, at most one per unit).
 * TC_SK, MMA_SK: the counters must be zero when a call starts.  Zero the whole
 * workspace once after allocating it; every call that completes leaves its
 * counters and partial tiles zero again, so the same workspace serves any
 * later direct-palette (pipeline 4) TC_SK or MMA_SK call, of any shape,
 * without clearing.  A call
 * of pipelines 1-3 writes its preprocessing output at the start of the
 * workspace, where a pipeline-4 call keeps its counters: zero the workspace
 * again after such a call before a stream-K call of another pipeline or
 * shape uses it (uw_stack_run keeps its counters in a region of their own).
 * After a call whose uw_device_status reports an error, zero the workspace
 * again before reusing it.                                                  */
uw_status uw_workspace_size(int64_t m, int64_t n, int64_t k, const uw_plan *plan,
                            size_t *bytes);

/* Y = X * W^T with W compressed.  x_dev: uint16[m,k] BF16 (16-byte aligned
 * rows); y_dev: float[m,n]; pal_dev: a palette plane to use instead of the
 * blob's (pipeline 4 only; may be NULL).  ws/ws_bytes: caller workspace of at
 * least uw_workspace_size bytes (256-byte aligned).  For every plan the
 * result is bit-identical to uw_matmul_bf16 with the same kernel, bn and
 * split_k on the decoded weights.                                            */
uw_status uw_fused_matmul(const uint16_t *x_dev, int64_t m, const uw_dmat *w,
                          const uint8_t *pal_dev, float *y_dev, const uw_plan *plan,
                          void *ws, size_t ws_bytes, void *stream);

/* The same kernels on plain BF16 weights w_dev[n,k] (the parity twin and the
 * uncompressed baseline).  plan->pipeline is ignored.  dev_status: a device
 * uint32 for kernel error bits (may be NULL when no error reporting is wanted). */
uw_status uw_matmul_bf16(const uint16_t *x_dev, int64_t m, const uint16_t *w_dev,
                         int64_t n, int64_t k, float *y_dev, const uw_plan *plan,
                         void *ws, size_t ws_bytes, uint32_t *dev_status, void *stream);

/* ------------------------------------------------------------------------ */
/* Many small matmuls in one launch (the experts of a mixture-of-experts      */
/* layer, which the Unweight page §十一 names as the next target).            */

/* One matmul of a batch: y_dev[m, w->n] = x_dev[m, w->k] * W^T. */
typedef struct uw_batch_item {
    const uw_dmat *w;        /* palette form (UW_EMIT_PALETTE) */
    const uint16_t *x_dev;   /* [m, k] BF16, 16-byte aligned */
    int64_t m;               /* 0..16 tokens; 0 = nothing to do (an expert nobody routed to) */
    float *y_dev;            /* [m, n] float32, 16-byte aligned */
} uw_batch_item;

/* Run every item with the warp-MMA fused kernel, up to 32 items per launch
 * instead of one launch per item.  plan: UW_PIPE_DIRECT_PALETTE and
 * UW_KERNEL_MMA (bn warps per tile, as for uw_fused_matmul); stages 0 takes 32
 * weights per lane and step only if every item's k is a multiple of 128.
 * Each item's y is bit-identical to uw_fused_matmul on that item with the
 * same plan (and stages resolved the same way).  Items may differ in n, k, m
 * and palette; no workspace.  All arguments are checked before anything is
 * launched; errors as in uw_fused_matmul.                                    */
uw_status uw_fused_matmul_batched(const uw_batch_item *items, int n_items, const uw_plan *plan,
                                  void *stream);

/* ------------------------------------------------------------------------ */
/* Matmul without a caller workspace (no counterpart on the Unweight page).   */

/* Bytes of the library-owned scratch array used by uw_fused_matmul_noalloc,
 * and how many of them (at its start) hold stream-K tile counters, one
 * uint32 per 128 x bn tile (TC_SK) or per 16-row tile (MMA_SK).              */
#define UW_NOALLOC_SCRATCH_BYTES (16u << 20)
#define UW_NOALLOC_COUNTER_BYTES (64u << 10)

/* uw_fused_matmul for callers that cannot give the library device memory
 * (an engine that hands its plug-ins no allocator and forbids cudaMalloc
 * after start-up, or a process whose device memory is already reserved by
 * another allocator).  Same arguments and results as uw_fused_matmul with
 * pal_dev = NULL, but no workspace: the split-K partial sums go to a fixed
 * array of UW_NOALLOC_SCRATCH_BYTES in the library's own device memory, which
 * every GPU that loads the library holds until the process exits.  Nothing is
 * allocated per call (no cudaMalloc, no allocating library routine).
 *   - plan->pipeline must be UW_PIPE_DIRECT_PALETTE (INVALID_ARG otherwise);
 *     a plan whose scratch (uw_workspace_size) does not fit is rejected with
 *     UW_ERR_WORKSPACE before anything is launched: partial sums beyond
 *     UW_NOALLOC_SCRATCH_BYTES - UW_NOALLOC_COUNTER_BYTES, or (TC_SK, MMA_SK) more
 *     tile counters than UW_NOALLOC_COUNTER_BYTES hold.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: do not call this
 *     entry point on a device after cudaDeviceReset.  Devices with an
 *     ordinal of 64 or more are refused (UW_ERR_INVALID_ARG).
 *   - All calls on a device share the one array: calls that may overlap on
 *     the GPU (other streams, other threads) race and must be serialised by
 *     the caller.  Partial sums do not carry over: in a call whose kernels
 *     complete, every partial sum read was written by that same call.  A
 *     call whose uw_device_status then reports an error may have left stale
 *     values in y, and (TC_SK, MMA_SK) non-zero tile counters, after which the
 *     entry point should not be used again in the process.                 */
uw_status uw_fused_matmul_noalloc(const uint16_t *x_dev, int64_t m, const uw_dmat *w,
                                  float *y_dev, const uw_plan *plan, void *stream);

/* ------------------------------------------------------------------------ */
/* Autotuner (Unweight page §九).                                             */

/* For every matrix mats[i] and batch size ms[j], time the candidate
 * (pipeline, kernel, bn, split_k) plans with CUDA events on `stream` and
 * store the fastest in plans_out[i*n_ms + j].  The candidates cover every
 * kernel but UW_KERNEL_MMA_SK, which occupies whole SMs and so cannot start
 * while the previous call drains: it can win such isolated timings and still
 * slow a sequence of calls down, so it is used by explicit plan only.  Every
 * timed call is preceded
 * by a 192 MB read of the end of the workspace, so the weights come from HBM
 * (not from the 126 MB L2), as they do when a model's layers run in turn.
 * x_dev must hold at least max(ms) x max(k) BF16 values, y_dev max(ms) x
 * max(n) floats, and ws (256-byte aligned) at least
 * uw_autotune_workspace_size bytes: the largest uw_workspace_size of any
 * candidate plus the 192 MB scratch.  If json_out is non-NULL a JSON plan
 * file (per matrix, per m: the chosen plan and the measured microseconds of
 * every candidate) is written into it.                                      */
uw_status uw_autotune_workspace_size(const uw_dmat *const *mats, int n_mats,
                                     const int64_t *ms, int n_ms, size_t *bytes);
uw_status uw_plan_autotune(const uw_dmat *const *mats, int n_mats, const int64_t *ms,
                           int n_ms, const uint16_t *x_dev, float *y_dev, void *ws,
                           size_t ws_bytes, int reps, uw_plan *plans_out, char *json_out,
                           size_t json_cap, void *stream);

/* ------------------------------------------------------------------------ */
/* Layer stacks with cross-layer overlap (Unweight page §八).                 */

/* One matmul of a stack: y_dev[m, w->n] = x_dev[m, w->k] * W^T with `plan`
 * (any pipeline).  pal_dev as in uw_fused_matmul (pipeline 4 only).        */
typedef struct uw_stack_step {
    const uw_dmat *w;
    const uint16_t *x_dev;
    int64_t m;
    float *y_dev;
    uw_plan plan;
    const uint8_t *pal_dev;
} uw_stack_step;

/* Workspace of uw_stack_run: two preprocessing slots, each the largest
 * preprocessing buffer of the stack (decode 2nk bytes, exponent decode a bit
 * over nk, transcode nk/2), plus the largest split-K scratch of any step,
 * plus (for TC_SK and MMA_SK steps) a region of stream-K tile counters kept
 * apart from the partial sums.  Zero the workspace once after allocating it (the
 * counters must start at zero; completed runs leave them zero).             */
uw_status uw_stack_workspace_size(const uw_stack_step *steps, int n_steps, size_t *bytes);

/* Run the steps in order on `stream`.  The decode (pipelines 1 and 2) or
 * transcode (pipeline 3) of a step is issued on `side_stream` into one of the two
 * workspace slots as soon as that slot is free, so it overlaps the matmuls
 * of the steps before it; the step's matmul waits for it.  Each step's result
 * is bit-identical to uw_fused_matmul with the same plan.  A step may read
 * an earlier step's y (matmuls keep step order on `stream`); no step may
 * write any weights.  side_stream NULL or equal to `stream`: everything runs
 * on `stream`.  All work, side stream included, is complete once `stream`
 * has completed it.  ws: >= uw_stack_workspace_size bytes, 256-byte aligned.
 * Arguments are checked before anything is launched; errors as in
 * uw_fused_matmul.  Device errors are OR-ed into each matrix's dev_status. */
uw_status uw_stack_run(const uw_stack_step *steps, int n_steps, void *ws, size_t ws_bytes,
                       void *stream, void *side_stream);

/* ------------------------------------------------------------------------ */
/* Decode/compute SM split (Unweight page §九: the autotuner also measures how */
/* the SMs are divided between decoding and compute).                         */

/* A split of one device's SMs into two green contexts with one stream each:
 * a preprocessing partition and a compute partition.  Work on a partition's
 * stream runs only on its SMs.  Both streams belong to the device's primary
 * context, so every entry point of this library (and the caller's device
 * memory and events) works on them.                                          */
typedef struct uw_sm_split uw_sm_split;

/* Split device `device`: at least prep_sms SMs (rounded up by the driver to
 * whole granules, 8 SMs on this GPU) for preprocessing, the rest for compute.
 * prep_sms <= 0, or a split that leaves the compute partition empty, gives
 * UW_ERR_INVALID_ARG; a driver without green contexts (or no driver) gives
 * UW_ERR_CUDA.  Typical use: uw_stack_run(..., compute_stream, prep_stream). */
uw_status uw_sm_split_create(int device, int prep_sms, uw_sm_split **out);

/* The split's streams (cudaStream_t as void*) and actual SM counts; any
 * output pointer may be NULL.                                                */
uw_status uw_sm_split_get(const uw_sm_split *s, void **prep_stream, void **compute_stream,
                          int *prep_sms, int *compute_sms);

/* Destroy the streams and green contexts.  All work queued on the split's
 * streams must have completed.  NULL is ignored.                             */
void uw_sm_split_destroy(uw_sm_split *s);

/* Choose the split for a stack: for every candidate cand[c] (preprocessing
 * SMs; 0 = no split, the two streams share all SMs) run the stack once to
 * warm up and then `reps` times (0 = 5) with the matmuls on the compute
 * stream and the preprocessing on the other, timed with CUDA events, and
 * return the fastest candidate in *best and every candidate's microseconds
 * per run in us_out[c] (may be NULL).  The caller's `stream` is synchronized
 * first (the steps' inputs may be produced there); all candidates run on
 * streams created and destroyed here, and no work is left in flight on
 * return.  The stack's weights are re-read every run: a stack larger than
 * the 126 MB L2 times as in a model's layer sequence.  ws as in uw_stack_run.
 * Errors as in uw_stack_run and uw_sm_split_create.                          */
uw_status uw_stack_tune_split(const uw_stack_step *steps, int n_steps, void *ws, size_t ws_bytes,
                              int device, const int *cand, int n_cand, int reps, int *best,
                              float *us_out, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* UW_H */
