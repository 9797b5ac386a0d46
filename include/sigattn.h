/*
 * sigattn -- sigmoid attention over padded variable-length batches, sm_100a (B200).
 *
 * C ABI of libsigattn.so.  Plain pointers and sizes only; no framework types.
 *
 * What it computes (per batch b, head h, query row i with key set J(i)):
 *     s_ij = scale * (q_i . k_j) + bias_i
 *     SIGMOID   o_i = sum_{j in J(i)} sigma(s_ij) v_j
 *     SOFTMAX   o_i = sum_j exp(s_ij) v_j / sum_j exp(s_ij)
 *     SOFTMAX1  o_i = sum_j exp(s_ij) v_j / (1 + sum_j exp(s_ij))
 * Sigmoid attention with b = -log(n): "Better Models, Faster Training: Sigmoid
 * Attention for single-cell Foundation Models", section 2A; its backward with
 * sigma' = sigma (1 - sigma) and no row-sum term: same page, section 2B, split into a
 * dQ kernel and a dK/dV kernel with sigma recomputed tile by tile: section 2C.
 * softmax_1: the QuietAttention page, section "Proposition : softmax_1 et
 * QuietAttention".  Rows with no key, and pad rows, give exactly 0 in every output.
 *
 * Tiles.  The attention matrix of each batch entry is cut into 128 x 128 tiles.  A
 * plan lists the tiles that hold at least one unmasked (query, key) pair ("Binary
 * Block Masking for FlashAttention", section "Comment ça marche ?"; "Better Models,
 * Faster Training", section 2C, blocks that are padding on either side are skipped).
 * Only listed tiles are computed.  A tile is FULL (every pair unmasked, no masking
 * work) or PARTIAL (it carries a 128 x 128 bitmask).
 *
 * Conventions for every call:
 *   - Tensors Q, K, V, O, dO, dQ, dK, dV are bf16 with layout [B, N, H, d]: d is
 *     contiguous; the three element strides (batch, token, head) are passed in
 *     that order.  Every device pointer must be 16-byte aligned and every stride
 *     a multiple of 8 elements (16 bytes).  Q/O/dO/dQ have N = Nq rows, K/V/dK/dV
 *     have N = Nk rows.  Supported head dims: d = 64 and d = 128.
 *   - Extents are the caller's promise, as with BLAS leading dimensions: the library
 *     sees pointers and strides only, so every tensor must hold the B x N x H x d (or
 *     T x H x d) elements its strides address, for the plan's B and N; a smaller buffer
 *     is read out of bounds, not reported.  (The Python binding compares each tensor's
 *     shape with the plan's B, Nq, Nk before it calls in, and raises on a short one.)
 *   - bias is fp32 [B, Nq] (per query row; row stride 1, batch stride given); NULL
 *     means 0.  For sigmoid attention the caller fills -log(n), e.g. with
 *     sigattn_bias_from_counts.
 *   - Ownership: the caller owns every tensor; a plan owns its own device buffers.
 *   - Asynchrony: every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) unless its comment says it synchronises.
 *   - Errors: 0 on success, a negative SIGATTN_ERR_* code otherwise; nothing is
 *     launched when an argument check fails.  Kernels never trap: a device-side wait
 *     that runs past its time limit records SIGATTN_ERR_TIMEOUT in a device status
 *     word, read (and cleared) by sigattn_get_status.
 */
#ifndef SIGATTN_H_
#define SIGATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SIGATTN_TILE 128

#if defined(__GNUC__)
#define SIGATTN_API __attribute__((visibility("default")))
#else
#define SIGATTN_API
#endif

typedef struct sigattn_plan sigattn_plan;
typedef void* sigattn_stream; /* cudaStream_t */

enum sigattn_epilogue {
  SIGATTN_SIGMOID = 0,  /* sigma(s), no normalisation */
  SIGATTN_SOFTMAX = 1,  /* online softmax (comparison mode) */
  SIGATTN_SOFTMAX1 = 2  /* online softmax_1: 1 + sum exp in the denominator */
};

enum sigattn_status {
  SIGATTN_OK = 0,
  SIGATTN_ERR_INVALID = -1,     /* null pointer, negative size, bad enum */
  SIGATTN_ERR_UNSUPPORTED = -2, /* head dim other than 64 / 128, sizes past limits */
  SIGATTN_ERR_ALIGNMENT = -3,   /* pointer not 16-byte aligned or stride not a multiple of 8 */
  SIGATTN_ERR_SHAPE = -4,       /* the plan belongs to another device than the current one */
  SIGATTN_ERR_CUDA = -5,        /* a CUDA runtime / driver call failed */
  SIGATTN_ERR_TIMEOUT = -6,     /* a device-side bounded wait expired (see sigattn_get_status) */
  SIGATTN_ERR_NO_DEVICE = -7,   /* no sm_100 device is current */
  SIGATTN_ERR_NOMEM = -8,       /* device allocation failed */
  SIGATTN_ERR_PLAN = -9         /* a tile list failed a structural check (sigattn_plan_validate) */
};

/* Sizes of a plan.  QT = ceil(Nq / 128), KT = ceil(Nk / 128). */
typedef struct sigattn_plan_sizes {
  int32_t B, Nq, Nk, QT, KT;
  int64_t nonempty;     /* listed tiles (FULL + PARTIAL) */
  int64_t full;         /* FULL tiles */
  int64_t partial;      /* PARTIAL tiles (each owns 512 uint32 of bitmask) */
  int64_t grid_total;   /* B * QT * KT: tiles of the padded grid */
  int32_t rows_nonempty;  /* (b, q-tile) rows with at least one tile */
  int32_t cols_nonempty;  /* (b, k-tile) columns with at least one tile */
} sigattn_plan_sizes;

/*
 * Plan for a padded batch: query i of batch entry b sees key j iff i < n_b and
 * j < n_b (Nq = Nk = Npad).  d_lengths: device int32 [B], each in [0, Npad].
 * Builds the tile list on the device: a classification kernel and one cooperative launch
 * (grid-wide barriers with a time limit) on `stream`.  Plan memory: the tile arrays are
 * sized for the worst case (every block listed; for lengths, two PARTIAL tile strips per
 * sequence, for a mask every block PARTIAL at 4 KB each) when that is at most 256 MB (one
 * allocation, which also keeps the build's scratch: 5 bytes per block of the grid and 8 per
 * possible PARTIAL block); then the call returns as soon as the work is queued, without
 * waiting for the device: the attention calls on any stream wait for the build (an
 * event; inside a stream capture, an external-event wait node of the graph),
 * sigattn_plan_get_sizes / the exports wait for it on the host, and
 * sigattn_plan_destroy releases the memory after it; d_lengths (d_mask) must stay valid
 * until the build has run on `stream`.  A larger worst case synchronises `stream` to read
 * the counts, sizes the arrays exactly and synchronises once more at the end.  On success *out owns device memory until sigattn_plan_destroy.
 * Errors: INVALID (null, B < 1, Npad < 1), UNSUPPORTED (B * QT * KT > 2^28, or a device
 * without cooperative launches), CUDA, NOMEM; TIMEOUT (a barrier of the build gave up:
 * reported by the call when it synchronises, else by sigattn_plan_get_sizes, the exports
 * and sigattn_get_status).  Lengths outside [0, Npad] are clamped into it.
 */
SIGATTN_API int sigattn_plan_from_lengths(const int32_t* d_lengths, int B, int Npad, sigattn_stream stream,
                              sigattn_plan** out);

/*
 * Plan for an element mask: d_mask is device uint8 [B, Nq, Nk], nonzero = attend;
 * element (b, i, j) at d_mask[b * stride_b + i * stride_q + j].  The mask is shared by
 * all heads.  Reads the mask once to classify blocks and once more for the PARTIAL
 * blocks' bitmasks.  Asynchrony, plan memory and errors as for the lengths plan.
 */
SIGATTN_API int sigattn_plan_from_mask(const uint8_t* d_mask, int B, int Nq, int Nk, int64_t stride_b,
                           int64_t stride_q, sigattn_stream stream, sigattn_plan** out);

/*
 * Plan for a PACKED batch (no padding): sequence b occupies rows cu[b] .. cu[b+1] of
 * tensors laid out [T, H, d] (T = cu[B]); d_cu: device int32 [B + 1], non-decreasing, each
 * length cu[b+1] - cu[b] in [0, max_seqlen].  The tile list is that of the padded batch
 * with these lengths and Npad = max_seqlen ("Better Models, Faster Training", section 1:
 * ragged cells; here without the padding), so the kernels skip the same tiles; they address
 * row r of sequence b at packed row cu[b] + r and write only the sequence's own rows.  With
 * such a plan, every tensor argument of the attention calls is [T, H, d]: pass strides
 * {any, token, head} (the batch stride is ignored), bias is fp32 [T] (bias_stride_b
 * ignored), and lse / the softmax workspace keep their [B, H, max_seqlen] layout.  The plan
 * keeps a copy of cu.  Synchronises `stream` once (the argument checks and T are read on
 * the host).  Errors: INVALID (null, B < 1, max_seqlen < 1, a length outside
 * [0, max_seqlen], T < 1), UNSUPPORTED, CUDA, NOMEM, TIMEOUT.
 */
SIGATTN_API int sigattn_plan_from_cu_seqlens(const int32_t* d_cu, int B, int max_seqlen,
                                             sigattn_stream stream, sigattn_plan** out);

/* Fills *sizes (host struct).  The first call on a plan whose build returned without
 * synchronising waits for the build and reads its counts (TIMEOUT if a barrier of the
 * build gave up); later calls do no device work. */
SIGATTN_API int sigattn_plan_get_sizes(const sigattn_plan* plan, sigattn_plan_sizes* sizes);

/*
 * Copies the tile list to HOST buffers (any may be NULL to skip it); synchronises.
 *   row_ptr  int32 [B*QT + 1]  CSR offsets by q-tile row r = b*QT + qt
 *   col_idx  int32 [nonempty]  k-tile of each entry, ascending within a row
 *   kind     uint8 [nonempty]  1 = FULL, 2 = PARTIAL
 *   pidx     int32 [nonempty]  bitmask number of a PARTIAL entry (CSR order), -1 if FULL
 *   colT_ptr int32 [B*KT + 1]  CSC offsets by k-tile column c = b*KT + kt
 *   rowT_idx int32 [nonempty]  q-tile of each CSC entry, ascending within a column
 *   csc_map  int32 [nonempty]  CSR index of each CSC entry
 *   bits     uint32 [partial * 512]  bit (k % 32) of word (q*4 + k/32) = mask(qt*128+q, kt*128+k)
 */
SIGATTN_API int sigattn_plan_export(const sigattn_plan* plan, int32_t* row_ptr, int32_t* col_idx,
                        uint8_t* kind, int32_t* pidx, int32_t* colT_ptr, int32_t* rowT_idx,
                        int32_t* csc_map, uint32_t* bits);

/*
 * Copies the two work lists to HOST buffers (either may be NULL); synchronises.
 *   row_work int32 [B*QT]  every q-tile row r, ordered by tile count descending, ties by r
 *   col_work int32 [B*KT]  every k-tile column c, ordered the same way
 * Rows / columns with no tile come last.  Counts past 4094 are ordered as equal.
 */
SIGATTN_API int sigattn_plan_export_work(const sigattn_plan* plan, int32_t* row_work, int32_t* col_work);

/*
 * Copies the runs of the tile list to HOST buffers (any may be NULL); synchronises.  A run
 * is a maximal range of consecutive k-tiles of one kind within a q-tile row: the kernels
 * walk a run without a per-tile list lookup ("Binary Block Masking for FlashAttention",
 * section "Comment ça marche ?": consecutive non-zero blocks skip the redundant checks and
 * reads).  The entries of a run are consecutive in the CSR list, and so are the bitmask
 * numbers of a PARTIAL run.
 *   run_ptr int32 [B*QT + 1]     runs of row r: runs[run_ptr[r] .. run_ptr[r+1])
 *   runs    int32 [nruns * 4]    {first k-tile, number of tiles, kind (1 / 2), first CSR entry}
 *   nruns   int64, one value     number of runs
 */
SIGATTN_API int sigattn_plan_export_runs(const sigattn_plan* plan, int32_t* run_ptr, int32_t* runs,
                                         int64_t* nruns);

/* Releases the plan's device memory, in the order of the legacy default stream and after
 * the plan's own build.  Safe on NULL.  The caller must ensure that no attention kernel that
 * uses the plan is still running on a non-blocking stream. */
SIGATTN_API void sigattn_plan_destroy(sigattn_plan* plan);

/*
 * Debug checks of a tile list (never called by the attention path; a plan the library built
 * always passes).  The properties are those of the block list of "Binary Block Masking for
 * FlashAttention", section "Comment ça marche ?" (each row's non-empty blocks, FULL or
 * PARTIAL with a 128 x 128 block mask), in this library's layout (sigattn_plan_export):
 *   1 row_ptr   CSR offsets non-decreasing, from 0 to `nonempty`
 *   2 col_idx   k-tiles in [0, KT), strictly ascending within a row
 *   3 kind      1 (FULL) or 2 (PARTIAL)
 *   4 pidx      -1 for FULL; PARTIAL entries numbered 0, 1, ... in CSR order
 *   5 colT_ptr  CSC offsets as row_ptr
 *   6 rowT_idx  q-tiles in [0, QT), strictly ascending within a column
 *   7 csc_map   each CSC entry names the CSR entry of the same (b, q-tile, k-tile)
 *   8 bits      each PARTIAL bitmask has a set and a clear bit
 *   9 runs      each row's runs cover its entries in maximal ranges of consecutive k-tiles
 *               of one kind, {first k-tile, tiles, kind, first entry}
 *  10 bitsT     (plan only) the transposed bitmasks match the bitmasks
 *  11 work      (plan only) the longest-first work lists name rows / columns in range with
 *               non-increasing lengths, and their 16-byte records match the offsets
 * Both return SIGATTN_OK, or SIGATTN_ERR_PLAN with *first_bad (may be NULL; -1 when the list
 * passes) = (check number << 40) | index of the failing row, column, entry, bitmask or slot,
 * the smallest such value found.
 *
 * sigattn_plan_validate: checks 1-11 on the plan's device arrays with one kernel on `stream`
 * and synchronises (it waits for the build first; PARTIAL numbering is checked within each
 * row).  Allocates and frees 8 bytes of device memory.  Errors: INVALID, SHAPE (the plan
 * belongs to another device), CUDA, TIMEOUT (the build gave up).
 *
 * sigattn_tile_list_check_host: checks 1-9 on HOST arrays sized as the caller says
 * (nonempty entries, partial * 512 bitmask words, nruns runs of 4 int32; run_ptr NULL skips
 * check 9), sequentially and with the PARTIAL numbering checked across the whole list.
 * Needs no GPU.  Errors: INVALID (bad sizes or a needed array NULL).
 */
SIGATTN_API int sigattn_plan_validate(const sigattn_plan* plan, sigattn_stream stream,
                                      int64_t* first_bad);
SIGATTN_API int sigattn_tile_list_check_host(int B, int QT, int KT, int64_t nonempty,
                                             int64_t partial, const int32_t* row_ptr,
                                             const int32_t* col_idx, const uint8_t* kind,
                                             const int32_t* pidx, const int32_t* colT_ptr,
                                             const int32_t* rowT_idx, const int32_t* csc_map,
                                             const uint32_t* bits, const int32_t* run_ptr,
                                             const int32_t* runs, int64_t nruns,
                                             int64_t* first_bad);

/*
 * bias[i] = -log(counts[i]) for counts[i] > 0, else 0 (b = -log(n) of "Better Models,
 * Faster Training", section 2A; counts[i] is the n of query row i: its sequence's
 * valid length, or its document's length).  Device int32 in, device fp32 out, n items.
 */
SIGATTN_API int sigattn_bias_from_counts(const int32_t* d_counts, int64_t n, float* d_bias,
                             sigattn_stream stream);

/*
 * Forward.  O[b, i, h, :] for every b < B, i < Nq, h < H (pad rows and rows with no key
 * are written as 0).  lse: fp32 [B, H, Nq] natural-log normaliser of each row
 * (log sum exp, or log(1 + sum exp) for SOFTMAX1; -inf for a SOFTMAX row with no key);
 * required for SOFTMAX / SOFTMAX1 (the backward reads it), ignored for SIGMOID (may be
 * NULL).  scale is usually 1/sqrt(d).
 * Errors: INVALID, UNSUPPORTED (d), ALIGNMENT, CUDA.
 */
SIGATTN_API int sigattn_fwd(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                const void* q, const int64_t q_strides[3],
                const void* k, const int64_t k_strides[3],
                const void* v, const int64_t v_strides[3],
                const float* bias, int64_t bias_stride_b,
                void* o, const int64_t o_strides[3],
                float* lse, sigattn_stream stream);

/*
 * Backward of L = sum(dO * O): writes dQ, dK, dV (bf16, fp32 accumulation; pad rows 0).
 * Two kernels, no atomics: a dK/dV kernel walks each k-tile column of the plan, a dQ
 * kernel walks each q-tile row; both recompute the attention weights tile by tile.
 * SOFTMAX / SOFTMAX1 also need o, lse (from sigattn_fwd) and workspace: fp32
 * [B * H * Nq] for D_i = dO_i . O_i; SIGMOID ignores o, lse and workspace (may be NULL).
 * Errors: as sigattn_fwd.
 */
SIGATTN_API int sigattn_bwd(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                const void* q, const int64_t q_strides[3],
                const void* k, const int64_t k_strides[3],
                const void* v, const int64_t v_strides[3],
                const void* o, const int64_t o_strides[3],
                const void* dout, const int64_t do_strides[3],
                const float* bias, int64_t bias_stride_b,
                const float* lse, float* workspace,
                void* dq, const int64_t dq_strides[3],
                void* dk, const int64_t dk_strides[3],
                void* dv, const int64_t dv_strides[3],
                sigattn_stream stream);

/* Parts of the backward for sigattn_bwd_ex (bit mask). */
enum sigattn_bwd_parts {
  SIGATTN_BWD_PREP = 1, /* D_i = dO_i . O_i into workspace (softmax modes only; no-op for SIGMOID) */
  SIGATTN_BWD_DKDV = 2, /* the dK / dV kernel */
  SIGATTN_BWD_DQ = 4,   /* the dQ kernel */
  SIGATTN_BWD_ALL = 7
};

/*
 * sigattn_bwd restricted to the parts in `parts` (launched in the order PREP, DKDV, DQ),
 * so that a caller can time or overlap the two kernels.  DKDV and DQ of the softmax modes
 * read the workspace that PREP wrote.  Arguments and errors as sigattn_bwd; parts outside
 * SIGATTN_BWD_ALL give INVALID.
 */
SIGATTN_API int sigattn_bwd_ex(const sigattn_plan* plan, int epilogue, int H, int d, float scale,
                               const void* q, const int64_t q_strides[3],
                               const void* k, const int64_t k_strides[3],
                               const void* v, const int64_t v_strides[3],
                               const void* o, const int64_t o_strides[3],
                               const void* dout, const int64_t do_strides[3],
                               const float* bias, int64_t bias_stride_b,
                               const float* lse, float* workspace,
                               void* dq, const int64_t dq_strides[3],
                               void* dk, const int64_t dk_strides[3],
                               void* dv, const int64_t dv_strides[3],
                               int parts, sigattn_stream stream);

/*
 * Fused backward (d = 64 only): the same dQ, dK, dV as sigattn_bwd from ONE walk over the
 * k-tile columns of the plan, so the attention weights and dP of each tile are computed
 * once instead of once per kernel.  Each tile's dQ contribution (dS K, tensor cores) is
 * added into an fp32 accumulator in `workspace` with TMA bulk reduce-adds; a small kernel
 * zeroes the accumulator rows of listed q-tiles first and one converts them to bf16 dQ
 * (times scale; rows of q-tiles with no tile get 0) at the end.  This is the variant the
 * two-kernel split of "Better Models, Faster Training", section 2C, avoids (there the
 * accumulation would need atomics); here the TMA unit does the additions.
 *
 * workspace: device memory of at least sigattn_bwd_fused_workspace_size() bytes, 16-byte
 * aligned, owned by the caller; its contents on entry do not matter and are undefined after.
 * Layout: fp32 dQ accumulator [B, Nq, H, 64], then (softmax modes) D [B, H, Nq].  Calls
 * sharing a workspace must not overlap on the GPU.  The order of the fp32 additions varies
 * from run to run, so dQ can differ in the last bits between runs; dK and dV are
 * deterministic.  Other arguments, results and errors as sigattn_bwd; d != 64 gives
 * UNSUPPORTED, a missing or too small workspace INVALID.
 */
SIGATTN_API int sigattn_bwd_fused_workspace_size(const sigattn_plan* plan, int epilogue, int H,
                                                 int d, size_t* bytes);
SIGATTN_API int sigattn_bwd_fused(const sigattn_plan* plan, int epilogue, int H, int d,
                                  float scale, const void* q, const int64_t q_strides[3],
                                  const void* k, const int64_t k_strides[3],
                                  const void* v, const int64_t v_strides[3],
                                  const void* o, const int64_t o_strides[3],
                                  const void* dout, const int64_t do_strides[3],
                                  const float* bias, int64_t bias_stride_b, const float* lse,
                                  void* workspace, size_t workspace_bytes,
                                  void* dq, const int64_t dq_strides[3],
                                  void* dk, const int64_t dk_strides[3],
                                  void* dv, const int64_t dv_strides[3],
                                  sigattn_stream stream);

/*
 * Backward that allocates nothing, for callers that cannot call cudaMalloc: code running
 * under a memory manager that owns all device memory (a framework's caching allocator, or a
 * fixed budget set by a host application that loads this library as a plug-in), and step
 * loops that cannot afford cudaMalloc's implicit device-wide synchronisation and
 * unpredictable latency.  The paper has no counterpart to this entry point.
 *
 * Same arguments, results and errors as sigattn_bwd, without `workspace`: the fp32 D_i =
 * dO_i . O_i values of the softmax modes go into a scratch array that the library keeps in
 * device memory (a file-scope __device__ array of SIGATTN_NOALLOC_MAX_ROWS floats, 8 MiB, held
 * by every GPU that loads the library until the process exits).  B * H * Nq above
 * SIGATTN_NOALLOC_MAX_ROWS gives SIGATTN_ERR_UNSUPPORTED for SOFTMAX / SOFTMAX1 (SIGMOID uses
 * no scratch and has no limit).  The first call on a device looks up the array's device
 * address (once per device, with that device current) and keeps it for the life of the
 * process, so a cudaDeviceReset after that is not supported; make that first call before
 * any stream capture.  All calls share the one array and it keeps the last call's contents;
 * every value a call reads is written by that same call first, so nothing has to be cleared,
 * but calls whose kernels overlap on the GPU (other streams, other threads) race on it.
 */
#define SIGATTN_NOALLOC_MAX_ROWS (1 << 21)
SIGATTN_API int sigattn_bwd_noalloc(const sigattn_plan* plan, int epilogue, int H, int d,
                                    float scale, const void* q, const int64_t q_strides[3],
                                    const void* k, const int64_t k_strides[3],
                                    const void* v, const int64_t v_strides[3],
                                    const void* o, const int64_t o_strides[3],
                                    const void* dout, const int64_t do_strides[3],
                                    const float* bias, int64_t bias_stride_b, const float* lse,
                                    void* dq, const int64_t dq_strides[3],
                                    void* dk, const int64_t dk_strides[3],
                                    void* dv, const int64_t dv_strides[3],
                                    sigattn_stream stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of the current
 * device: SIGATTN_OK, or SIGATTN_ERR_TIMEOUT if a kernel's bounded wait expired since the
 * last call (that kernel's outputs are then undefined), or SIGATTN_ERR_CUDA.
 */
SIGATTN_API int sigattn_get_status(sigattn_stream stream);

/* Device-side wait limit in nanoseconds for all kernels of this library on the current
 * device (default 2e9).  A wait that exceeds it records SIGATTN_ERR_TIMEOUT and the
 * kernel returns early. */
SIGATTN_API int sigattn_set_wait_limit_ns(uint64_t ns);

/* Self-test of the bounded wait: launches one CTA that waits on a barrier nothing
 * arrives at, with a limit of `ns`; the kernel gives up, records SIGATTN_ERR_TIMEOUT and
 * returns.  Used by the tests of the failure path; never faults or hangs. */
SIGATTN_API int sigattn_selftest_wait_timeout(uint64_t ns, sigattn_stream stream);

/* Static description of an error code. */
SIGATTN_API const char* sigattn_error_string(int code);

/* Name of the CUDA error behind the most recent SIGATTN_ERR_CUDA / NOMEM returned by any
 * call of this library (process-wide), e.g. "cudaErrorInvalidValue"; "no CUDA error" if none. */
SIGATTN_API const char* sigattn_last_cuda_error(void);

/* Library version, e.g. 100 for 0.1.0. */
SIGATTN_API int sigattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SIGATTN_H_ */
