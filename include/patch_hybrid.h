/*
 * patch_hybrid.h - C ABI of the B200 (sm_100a) hybrid dense / 2:4 linear layer.
 *
 * The layer is PATCH's inference hot path: a frozen weight W[N,K] is cut into
 * tiles, each tile either dense or 2:4 sparse (two kept in every group of four
 * consecutive k), and the output is Y = X . (W (.) Mask)^T.
 *   - Tiles dense or 2:4, global sparsity continuous in 0..50%: abstract of
 *     "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs"; model card
 *     "llama_3.2_1b-PATCH-45Sparse", method paragraph.
 *   - The mask is a bit-packed keep/prune mask; applying it zeroes the pruned
 *     weights: the same card, release paragraph and "How to use"
 *     (apply_patch_mask).
 *   - Tile shapes 128x128, 128x64, 64x128, 64x64: the same card,
 *     "Training hyper-parameters" table, mask tile size row.
 *   - A hybrid sparse kernel is what turns the mask into speed: the same
 *     card, last sentence of "How to use".
 *
 * Conventions for every call:
 *   - W, X, Y are bf16, row-major (K contiguous for W and X, N contiguous
 *     for Y). "dev" pointers are CUDA device pointers on the current device;
 *     "host" pointers are host memory (pinned is fastest).
 *   - stream is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream. Calls are stream-ordered and asynchronous unless stated.
 *   - No call throws, aborts or traps. Each returns a patch_status; the
 *     message of the last failure on the calling thread is patch_last_error().
 *   - The caller owns every buffer it passes. A handle owns the packed copy
 *     of the weights, its tables, its cached schedules and the decode
 *     kernel's split-K workspaces.
 *   - Concurrency: patch_linear, patch_linear_path and patch_group_linear
 *     calls on one handle or group may overlap on the GPU when they are
 *     issued on different streams or threads. The decode kernel (M <= 64)
 *     keeps its split-K partial sums in a workspace per stream (per thread
 *     for the per-thread default stream); the other kernels keep no per-call
 *     state. Three exceptions: patch_linear_host calls on one handle share a
 *     staging buffer; all patch_linear_noalloc calls share one array; and
 *     every CUDA graph that captured decode calls of one handle or group uses
 *     that handle's or group's one capture workspace. Calls in each of these
 *     three classes must not overlap on the GPU (order them on one stream, or
 *     synchronise between them).
 */
#ifndef PATCH_HYBRID_H
#define PATCH_HYBRID_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct patch_handle_s* patch_handle;
typedef struct patch_group_s* patch_group;

typedef enum {
    PATCH_OK = 0,
    PATCH_ERR_ARG = 1,         /* null pointer, bad enum value, negative size */
    PATCH_ERR_SHAPE = 2,       /* a dimension does not fit the tiling rules */
    PATCH_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
    PATCH_ERR_MASK = 4,        /* a group inside a 2:4 tile does not keep exactly two */
    PATCH_ERR_CUDA = 5,        /* a CUDA runtime call failed */
    PATCH_ERR_TIMEOUT = 6,     /* a device-side wait ran past its limit */
    PATCH_ERR_NOMEM = 7,       /* device or host allocation failed */
    PATCH_ERR_UNSUPPORTED = 8  /* the current device is not compute capability 10.x, or is
                                  larger than a fixed limit of patch_linear_noalloc */
} patch_status;

/* Which kernel patch_linear_path runs. AUTO picks by M: GEMV for M <= 64,
 * GEMM_SINGLE below M = 256, and above it GEMM_WIDE (GEMM_WIDE_24 for pure
 * 2:4 weights) when the call (or group) has at least two 512-row x 240-token
 * tiles per co-resident CTA pair, otherwise GEMM_PAIR. GEMM is AUTO
 * restricted to the tensor-core GEMMs. */
typedef enum {
    PATCH_PATH_AUTO = 0,
    PATCH_PATH_GEMM = 1,         /* tcgen05 tensor-core GEMM, variant chosen as for AUTO */
    PATCH_PATH_GEMV = 2,         /* decode kernel (M <= 64): tcgen05 with N = M rounded up
                                    to 16, split-K over the weight stream */
    PATCH_PATH_GEMM_SINGLE = 3,  /* tcgen05, one CTA per 128-row x 128-token tile */
    PATCH_PATH_GEMM_PAIR = 4,    /* tcgen05 cta_group::2, one CTA pair per 256 x 256 tile */
    PATCH_PATH_GEMV_SIMT = 5,    /* decode on CUDA cores (M <= 16), no workspace */
    PATCH_PATH_GEMM_WIDE = 6,    /* tcgen05 cta_group::2, two strips per CTA: one CTA pair
                                    per 512-row x 240-token tile (each activation tile feeds
                                    both strip pairs); strips padded to a multiple of four */
    PATCH_PATH_GEMM_WIDE_24 = 7  /* the GEMM_WIDE kernel's instance for pure 2:4 weights
                                    (every slab of every member runs on the sparse MMA, the
                                    MaskLLM end of the range): it computes each record's
                                    place instead of reading the tables. GEMM_WIDE, GEMM and
                                    AUTO run it whenever the weights allow; requesting it for
                                    other weights gives PATCH_ERR_ARG */
} patch_path;

typedef struct {
    int64_t N, K;               /* weight shape */
    int32_t tile_rows, tile_cols;
    int64_t tiles_total;        /* (N/tile_rows) * (K/tile_cols) */
    int64_t tiles_sparse;       /* tiles flagged 2:4 */
    int64_t slabs_total;        /* (N/128) * (K/64) storage slabs */
    int64_t slabs_sparse;       /* slabs stored compressed */
    int64_t slabs_pair_sparse;  /* slabs the CTA-pair kernel runs on the sparse MMA */
    int64_t meta_blocks;        /* 2048-byte metadata blocks */
    int64_t dense_images;       /* dense images of 2:4 slabs whose partner strip is dense
                                   (partners: patch_plan_pairs) */
    int64_t packed_bytes;       /* device bytes of the packed weights */
    int64_t pruned;             /* mask zeros over all N*K elements */
    int64_t stray_zeros;        /* mask zeros inside tiles flagged dense */
    double sparsity;            /* pruned / (N*K) */
} patch_info_t;

/*
 * patch_pack - validate the mask and build the packed weights (one-time).
 *
 * Realises apply_patch_mask ("How to use" on the PATCH model cards) for one
 * weight matrix, storing each dense tile as a bf16 block of W (.) Mask and
 * each 2:4 tile as its kept values plus 2-bit position codes.
 *
 *   W_bf16      dev, N*K bf16, row-major, 16-byte aligned. Not retained.
 *   N, K        weight rows (outputs) and columns (inputs). N % 128 == 0,
 *               K % 64 == 0, N % tile_rows == 0, K % tile_cols == 0.
 *   mask_bits   dev, ceil(N*K/8) bytes: bit (n*K + k) is the keep bit of
 *               W[n][k]; it lives in byte (n*K+k)/8 at bit 7-((n*K+k)%8)
 *               when bitorder == 0 (MSB first, numpy packbits default) or at
 *               bit (n*K+k)%8 when bitorder == 1. Not retained.
 *   tile_flags  host, (N/tile_rows)*(K/tile_cols) bytes, row-major over the
 *               tile grid: 0 = dense tile, 1 = 2:4 tile. Not retained.
 *   tile_rows, tile_cols  one of 128x128, 128x64, 64x128, 64x64.
 *   stream      stream for the pack kernel.
 *   out         receives the new handle (NULL on failure).
 *
 * Every group of four consecutive k inside a tile flagged 2:4 must keep
 * exactly two weights, else PATCH_ERR_MASK (nothing is allocated on return).
 * Pruned weights inside dense tiles are allowed and counted (stray_zeros).
 * Synchronises the stream once to read the validation counters.
 */
patch_status patch_pack(const void* W_bf16, int64_t N, int64_t K, const uint8_t* mask_bits,
                        int bitorder, const uint8_t* tile_flags, int tile_rows,
                        int tile_cols, void* stream, patch_handle* out);

/*
 * patch_plan - the tables and packed size patch_pack would produce for these
 * tile flags, computed on the host without touching any device.
 *
 *   N, K, tile_flags, tile_rows, tile_cols  as for patch_pack.
 *   slab_table  host, (N/128)*(K/64) uint32, or NULL.
 *   meta_table  host, (N/128)*ceil(K/128) uint32, or NULL.
 *   gemm_table  host, (N/128)*(K/64) uint32, or NULL.
 *   packed_bytes  receives the device bytes of the packed weights, or NULL.
 * Table layouts: see patch_copy_packed. Same shape rules and errors as
 * patch_pack; no mask is read.
 */
patch_status patch_plan(int64_t N, int64_t K, const uint8_t* tile_flags, int tile_rows, int tile_cols,
                        uint32_t* slab_table, uint32_t* meta_table, uint32_t* gemm_table,
                        int64_t* packed_bytes);

/*
 * patch_plan_pairs - which strips patch_pack makes partners for the CTA-pair
 * kernels, computed on the host without touching any device.
 *
 * The pages fix no kernel; this is the packed format's own rule. A CTA-pair
 * MMA covers two 128-row strips and is either dense or 2:4 for both, so a
 * 2:4 slab whose partner's slab is dense runs from a dense image at dense
 * cost (the tiles' dense / 2:4 choices are learned independently: abstract of
 * "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs"). Strips are paired
 * by agreement: score(i, j) = number of 64-column slabs 2:4 in both strips;
 * the two unpaired strips of highest score are paired first (ties: smallest
 * i, then smallest j); pairs are listed in the order of their first strip and
 * an odd strip out comes last as its own partner. Linears of more than 2048
 * strips keep the order 0, 1, 2, ...
 *
 *   N, K, tile_flags, tile_rows, tile_cols  as for patch_pack.
 *   order       host, N/128 int32: pair i is strips order[2i], order[2i+1].
 * Same shape rules and errors as patch_plan.
 */
patch_status patch_plan_pairs(int64_t N, int64_t K, const uint8_t* tile_flags, int tile_rows,
                              int tile_cols, int32_t* order);

/*
 * patch_classify_tiles - the tile flags a keep/prune mask implies, computed
 * on the host, for a mask that comes without them (a released mask file
 * holds the mask only: model card "llama_3.2_1b-PATCH-45Sparse", release
 * paragraph and "How to use").
 *
 *   mask_bits  host, ceil(N*K/8) bytes, the keep bits of W[N,K] row-major,
 *              8 per byte, in either bit order (the rule below reads whole
 *              groups of four, which never straddle a byte).
 *   N, K, tile_rows, tile_cols  as for patch_pack.
 *   tile_flags  host, (N/tile_rows)*(K/tile_cols) bytes written, row-major
 *              over the tile grid: 1 when every group of four consecutive k
 *              in every row of the tile keeps exactly two (a 2:4 tile), else
 *              0 (dense; the method's dense tiles keep every weight:
 *              "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs",
 *              abstract, and the card's method paragraph).
 *   dense_with_pruned  receives the number of dense tiles that still prune
 *              some weight (patch_pack stores W (.) Mask for those, so the
 *              product stays exact, at dense cost), or NULL.
 * Same shape errors as patch_pack; PATCH_ERR_ARG for a NULL buffer.
 */
patch_status patch_classify_tiles(const uint8_t* mask_bits, int64_t N, int64_t K, int tile_rows,
                                  int tile_cols, uint8_t* tile_flags, int64_t* dense_with_pruned);

/*
 * patch_partition_rows - split W's rows into `parts` contiguous shards of
 * balanced tensor-core cost, for a tensor-parallel (output-feature) split of
 * one linear across ranks. Computed on the host; touches no device.
 *
 * Why: each tile's dense / 2:4 choice is learned on its own, and the
 * abstract of "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs" notes
 * that the learned sparsity is non-uniform across layers; rows of one weight
 * differ in the same way, so equal row counts would leave the ranks with the
 * sparsest rows idle.
 *
 *   N, K, tile_flags, tile_rows, tile_cols  as for patch_pack (the whole W).
 *   parts       number of shards (ranks), >= 1.
 *   align_rows  every bound is a multiple of this many rows, or N; a
 *               positive multiple of 256 so that no strip pair is cut.
 *   bounds      host, parts + 1 int64: shard r is rows [bounds[r], bounds[r+1])
 *               of W (and columns of Y); bounds[0] = 0, bounds[parts] = N,
 *               non-decreasing. A shard is empty only when there are fewer
 *               aligned blocks than parts (the trailing shards then are).
 * Cost of a strip pair (256 rows): for each 64-column slab, 1 when dense and
 * 1/2 when 2:4 in both strips, plus 1 for its epilogue. The split minimises
 * the largest shard's cost over all contiguous aligned splits. Each shard
 * W[bounds[r]:bounds[r+1]] with its rows of mask bits and tile flags is a
 * valid patch_pack input. Same shape and flag errors as patch_plan;
 * PATCH_ERR_ARG for a NULL pointer, parts < 1 or a bad align_rows.
 */
patch_status patch_partition_rows(int64_t N, int64_t K, const uint8_t* tile_flags, int tile_rows,
                                  int tile_cols, int parts, int64_t align_rows, int64_t* bounds);

/*
 * patch_linear - Y = X . (W (.) Mask)^T for the packed weights of h.
 *
 *   X_bf16  dev, M*K bf16 row-major, 16-byte aligned.
 *   M       number of tokens (rows of X), M >= 0. M == 0 is a no-op.
 *   Y_bf16  dev, M*N bf16 row-major, 16-byte aligned. Every element is
 *           written: fp32 accumulation, one round-to-nearest-even to bf16.
 * Picks the tensor-core kernel or the decode kernel by M. The first call for
 * a new value of M builds that M's work schedule and uploads it
 * asynchronously on `stream` (it allocates device and pinned host memory);
 * a call on another stream waits for that upload on the device. The first
 * uncaptured decode call (M <= 64) on a stream allocates that stream's
 * workspace (a few MB, held until the handle or group is freed); the first
 * with 16 < M <= 64 adds four times that for the wider partial sums. Before
 * capturing later calls in a CUDA graph, make one call with the same M and
 * let it complete.
 */
patch_status patch_linear(patch_handle h, const void* X_bf16, int64_t M, void* Y_bf16,
                          void* stream);

/* patch_linear with an explicit kernel choice (patch_path). GEMV requires
 * M <= 64 and GEMV_SIMT M <= 16 (PATCH_ERR_SHAPE otherwise). Any M works on
 * the tensor-core GEMM variants. */
patch_status patch_linear_path(patch_handle h, const void* X_bf16, int64_t M, void* Y_bf16,
                               int path, void* stream);

/*
 * patch_linear_host - the same product from and to HOST memory.
 *
 *   X_host  host, M*K bf16 row-major.  Y_host  host, M*N bf16 row-major.
 * Copies X to a device staging buffer owned by h (grown on demand), runs
 * patch_linear on it, copies Y back, and synchronises the stream before it
 * returns. Calls on one handle must not overlap (shared staging buffer).
 */
patch_status patch_linear_host(patch_handle h, const void* X_host, int64_t M, void* Y_host,
                               void* stream);

/*
 * patch_linear_noalloc - patch_linear for callers that cannot allocate device
 * memory during the call.
 *
 * The pages describe no counterpart; this entry point exists for deployment.
 * patch_linear uploads each new M's tile schedule into device memory it
 * allocates on first use. Callers whose device memory is owned by someone
 * else (a frozen allocator, another framework's memory pool, a thread that
 * may not call cudaMalloc) use this call instead: it allocates nothing and
 * keeps the schedule in one fixed array inside this library's device image.
 * Every GPU that loads the library holds that array (about 257 KiB) until
 * the process exits.
 *
 *   Arguments and layouts as for patch_linear. Kernel per M:
 *     M <= 8         CUDA-core decode kernel (GEMV_SIMT), no schedule;
 *     9 <= M < 256   single-CTA tensor-core kernel, 128-row x 128-token tiles;
 *     M >= 256       the CTA-pair kernel patch_linear would run for this M:
 *                    GEMM_WIDE (512-row x 240-token tiles) or GEMM_PAIR
 *                    (256-row x 256-token tiles).
 *   For M >= 65 the result is bit-identical to patch_linear's (same kernel,
 *   same schedule); for M <= 64 patch_linear runs the tensor-core decode
 *   kernel instead, which sums in another order (both within the tolerance
 *   of the fp32 product).
 * Limits: at most 65536 output tiles per call (tiles as above;
 * PATCH_ERR_SHAPE beyond that) and at most 256 persistent CTAs or CTA pairs
 * on the device (PATCH_ERR_UNSUPPORTED beyond that).
 * The first call on each device looks up the array's device address
 * (set-up); make that first call before any stream capture begins. All calls
 * share the one array and each overwrites it, so calls that overlap on the
 * GPU (different streams, or several handles at once) race: order them on
 * one stream or synchronise between them.
 */
patch_status patch_linear_noalloc(patch_handle h, const void* X_bf16, int64_t M, void* Y_bf16,
                                  void* stream);

/*
 * patch_group_create - bind several packed linears that are run with the same
 * token count M (for example the q, k, v, o, gate, up and down projections of
 * one layer) so that one persistent launch computes all of them.
 *
 *   handles  host array of n handles, all on the current device; 1 <= n <= 8.
 *            The handles must outlive the group.
 *   out      receives the group.
 * The group owns only a small device descriptor array and its cached
 * schedules (allocated on the first call for each M, like patch_linear).
 */
patch_status patch_group_create(const patch_handle* handles, int n, patch_group* out);

/*
 * patch_group_linear - Y_i = X_i . (W_i (.) Mask_i)^T for every member i in
 * one launch (the GEMV_SIMT path runs one launch per member).
 *
 *   X  host array of n dev pointers, X_i: M x K_i bf16, 16-byte aligned.
 *   Y  host array of n dev pointers, Y_i: M x N_i bf16, 16-byte aligned.
 *      Inputs may be shared between members (q, k, v read the same X).
 *   M, path, stream as for patch_linear_path.
 * Device timeouts are reported through patch_check on the first member.
 */
patch_status patch_group_linear(patch_group g, const void* const* X, int64_t M, void* const* Y, int path,
                                void* stream);

/*
 * patch_group_linear_host - patch_group_linear from and to HOST memory, with
 * the copies overlapped with the product.
 *
 *   X  host array of n host pointers, X_i: M x K_i bf16 row-major. Members
 *      that pass the same pointer (q, k, v) share one upload.
 *   Y  host array of n host pointers, Y_i: M x N_i bf16 row-major.
 *   M, path as for patch_group_linear; stream is where the product runs.
 * The tokens are cut into up to four chunks, each a whole number of token
 * tiles of the kernel patch_group_linear would run for this M (so Y is bit
 * for bit the device call's): the inputs of chunk c go up on one copy stream
 * while chunk c-1 is computed on `stream` and the outputs of chunk c-2 come
 * back on another, so both copy directions and the tensor cores work at
 * once. Pinned host memory gives
 * asynchronous copies; pageable memory works, with copies that block the
 * host. Asynchronous: the call returns once everything is enqueued; the Y
 * buffers are complete when `stream` is (it waits for the last copy back),
 * and X and Y must stay valid until then. The group owns the device staging
 * buffers (grown on demand: the first call for a larger M allocates and
 * waits for the group's previous host call). Calls on one group are ordered
 * among themselves on the device; issue them from one host thread at a time.
 * A call that fails part-way may have enqueued some copies: synchronise
 * `stream` before the next call on the group.
 */
patch_status patch_group_linear_host(patch_group g, const void* const* X, int64_t M, void* const* Y,
                                     int path, void* stream);

/*
 * patch_group_path - the explicit path (GEMV, GEMV_SIMT, GEMM_SINGLE,
 * GEMM_PAIR, GEMM_WIDE or GEMM_WIDE_24) that patch_group_linear would run for this M and
 * requested path; nothing is launched. *out receives the value.
 * Errors: PATCH_ERR_ARG for a NULL group or out, M < 0 or an unknown path.
 */
patch_status patch_group_path(patch_group g, int64_t M, int path, int* out);

/* patch_group_free - release a group (not its handles). NULL is ignored. */
void patch_group_free(patch_group g);

/* patch_unpack - write W (.) Mask (N*K bf16, dev, row-major, 16-byte aligned)
 * decoded from the packed weights. */
patch_status patch_unpack(patch_handle h, void* W_masked_bf16, void* stream);

/* patch_info - shape, tile and sparsity figures of a handle (host struct). */
patch_status patch_info(patch_handle h, patch_info_t* info);

/*
 * patch_copy_packed - copy the packed bytes and the three tables to the host.
 *   packed_host  host, packed_cap bytes (>= info.packed_bytes), or NULL.
 *   slab_host, meta_host, gemm_host  host tables with their capacities in
 *                entries, or NULL. A too-small buffer gives PATCH_ERR_ARG.
 * With S = N/128 strips, KB = K/64 slabs and KC = ceil(KB/2) chunks:
 *   slab[s*KB+b] = (offset/16)<<2 | first<<1 | sparse: the slab's own record,
 *     a 16384-byte dense block or 8192 bytes of kept 2:4 values; first marks
 *     the first 2:4 slab of its 128-column chunk.
 *   meta[s*KC+c] = offset/16 of the chunk's 2048-byte metadata block, or
 *     0xFFFFFFFF when the chunk has no 2:4 slab.
 *   gemm[s*KB+b] = (offset/16)<<2 | first<<1 | pair_sparse: the record the
 *     CTA-pair kernels load (a strip and its partner, patch_plan_pairs, agree
 *     on every slab; a 2:4 slab whose partner's slab is dense points at its
 *     dense image).
 * Synchronous.
 */
patch_status patch_copy_packed(patch_handle h, void* packed_host, int64_t packed_cap,
                               uint32_t* slab_host, int64_t slab_cap, uint32_t* meta_host,
                               int64_t meta_cap, uint32_t* gemm_host, int64_t gemm_cap);

/*
 * patch_check - synchronise the stream and report device-side failures of
 * earlier calls on h (a wait that ran past its limit gives PATCH_ERR_TIMEOUT).
 * Clears the handle's device status word.
 */
patch_status patch_check(patch_handle h, void* stream);

/* patch_free - release a handle and its device memory (synchronises the
 * device first). NULL is ignored. */
void patch_free(patch_handle h);

/*
 * patch_selftest_wait - exercise the device-side failure path on the current
 * device: one CTA waits on a barrier that nothing completes, using the bounded
 * wait every kernel uses (limit 1 s of %globaltimer). The wait gives up, the
 * kernel records a timeout in a status word and returns; no fault, trap or
 * hang is involved and the context stays usable. Synchronises `stream`.
 * Returns PATCH_ERR_TIMEOUT when the path behaves as designed, PATCH_OK if the
 * wait unexpectedly completed, PATCH_ERR_CUDA / NOMEM on a runtime failure,
 * PATCH_ERR_UNSUPPORTED on a device that is not compute capability 10.x.
 * Not part of the product: a check for tests and deployment health probes.
 */
patch_status patch_selftest_wait(void* stream);

/* Message of the last failed call on this thread ("" if none). */
const char* patch_last_error(void);

/* ABI version, bumped on any incompatible change. */
int patch_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PATCH_HYBRID_H */
