/*
 * gptq.h -- C ABI of the B200 (sm_100a) GPTQ layer-quantization library
 * (libgptq.so).
 *
 * The operation is GPTQ layer-wise weight quantization as described on the
 * pages "GPTQ / AWQ / SqueezeLLM" (sec. 一: H = 2 X^T X / n from the
 * calibration inputs, damping, block-wise processing, importance order),
 * "INT4/INT8 量化推理：从 GPTQ 到 AWQ 的取舍" (sec. 一: groups of 128
 * consecutive weights with an fp16 scale and a 4-bit zero point, 66.5 bytes
 * per 128 weights; sec. 三: quantize column by column and push each column's
 * error onto the not-yet-quantized columns through H^-1) and
 * "大模型量化的“校准”艺术" (sec. 2.1 min-max mapping; sec. 2.2 the loop).
 *
 * Conventions shared by every call:
 *  - All array arguments are DEVICE pointers to caller-owned memory (the
 *    library never allocates, frees or synchronizes).  Scratch memory, where
 *    a call needs it, is passed as (ws, ws_bytes); the matching
 *    *_workspace_bytes() call gives the size.
 *  - Matrices are row-major and densely packed (leading dimension = number of
 *    columns).  W is d_out x d_in like a torch Linear weight: a "column" is an
 *    input channel.  X is n_tokens x d_in (token-major).
 *  - fp16 data is passed as its 16-bit IEEE pattern (uint16_t).
 *  - `stream` is a cudaStream_t (0 = legacy default stream).  Every call is
 *    asynchronous on it; device-side outcomes (non-positive pivot) are
 *    reported through a device int the caller may read after synchronizing.
 *  - Pointers must be 16-byte aligned.  Arguments are validated before any
 *    launch; on error nothing is launched and the status says why.
 *  - Return value: a gptq_status.  GPTQ_ERR_CUDA means a launch failed; the
 *    CUDA error is left for the caller to inspect with cudaGetLastError().
 */
#ifndef GPTQ_B200_GPTQ_H
#define GPTQ_B200_GPTQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GPTQ_OK = 0,
    GPTQ_ERR_INVALID_ARG = 1,   /* null pointer, bad enum, misaligned pointer */
    GPTQ_ERR_SHAPE = 2,         /* sizes outside what the call supports */
    GPTQ_ERR_NOT_PD = 3,        /* (host-detectable) no positive definite H */
    GPTQ_ERR_UNSUPPORTED = 4,   /* valid but not implemented (e.g. bits=5) */
    GPTQ_ERR_CUDA = 5,          /* a kernel launch failed */
    GPTQ_ERR_TIMEOUT = 6        /* reserved: a bounded device wait expired */
} gptq_status;

enum { GPTQ_DTYPE_F32 = 0, GPTQ_DTYPE_F16 = 1 };

/* Human-readable name of a status code (static string, never NULL). */
const char* gptq_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int gptq_abi_version(void);

/* Diagnostics: number of kernel launches this process has issued through the
 * library so far (all devices, all calls).  Host-only, never synchronizes. */
uint64_t gptq_debug_launch_count(void);

/* Device status of the current device: 0, or the code a bounded device-side
 * wait recorded when it gave up (the kernel then returned early and its
 * outputs are invalid).  Synchronous (reads a device word); reset != 0 clears
 * it.  Returns GPTQ_OK or GPTQ_ERR_CUDA / GPTQ_ERR_INVALID_ARG. */
int gptq_device_status(int32_t* status_out, int reset);

/*
 * Launch configuration (no counterpart on the pages): caps the CTAs of the
 * library's persistent kernels of one kind -- GPTQ_CTAS_HESSIAN (the Hessian
 * accumulation), GPTQ_CTAS_PREPARE (the factorization in gptq_prepare_hinv)
 * or GPTQ_CTAS_QUANTIZE (the tensor-core updates in gptq_quantize_layer) --
 * at max_ctas (0: one per SM, the default).  A caller that runs one layer's
 * preparation beside the next layer's Hessian and quantization on two
 * streams gives each a share of the SMs this way (a persistent grid larger
 * than the SMs left to it would run its last CTAs after the others); every
 * kernel is correct for any count.  Process-wide, read at each launch; not
 * synchronized with launches in flight.  Returns GPTQ_OK or
 * GPTQ_ERR_INVALID_ARG.
 */
enum { GPTQ_CTAS_HESSIAN = 0, GPTQ_CTAS_PREPARE = 1, GPTQ_CTAS_QUANTIZE = 2 };
int gptq_set_max_ctas(int kind, int max_ctas);

/*
 * Hessian accumulation -- "GPTQ / AWQ / SqueezeLLM" sec. 一 (H from the
 * calibration inputs; the 2/n factor is applied later by gptq_prepare_hinv).
 *
 *   S[i][j] += sum_t X[t][i] * X[t][j]      for 0 <= i <= j < d
 *
 * S: d x d fp32, in/out.  Only the upper triangle (i <= j) is read and
 *    written; the strictly-lower triangle is left untouched.  Zero S before
 *    the first batch; call once per calibration batch.
 * X: n_tokens x d fp16 (token-major).
 * n_seen: optional HOST counter, incremented by n_tokens on success.
 * Requires d % 128 == 0, 128 <= d <= 32768, n_tokens >= 0 (0: no-op).
 * Accumulation is fp32 on the tensor cores with fp16 inputs.
 */
int gptq_hessian_accumulate(float* S, const uint16_t* X, int64_t n_tokens, int64_t d,
                            int64_t* n_seen, void* stream);

/*
 * Hessian accumulation from HOST memory -- the same sum as
 * gptq_hessian_accumulate ("GPTQ / AWQ / SqueezeLLM" sec. 一), for
 * calibration inputs that live in host memory.  The pages have no
 * counterpart: streaming the batch is an interface convenience.
 *
 * X_host is cut into chunks of chunk_tokens tokens.  Chunk k is copied into
 * slot k % 2 of the device ring `stage` on copy_stream while chunk k - 1 is
 * accumulated into S on `stream`, so the PCIe copy overlaps the tensor-core
 * work.  Two caller-owned CUDA events order the ring:
 *   ev_filled: recorded on copy_stream after each chunk's copy; `stream`
 *              waits on it before accumulating that chunk;
 *   ev_freed:  recorded on `stream` after each chunk's accumulation;
 *              copy_stream waits on it before overwriting a slot.
 * Reuse the same (stage, ev_filled, ev_freed) for consecutive calls: the
 * first copy of a call waits for the last accumulation of the previous one,
 * so the next batch's copies overlap whatever the caller queues on `stream`
 * in between (e.g. the rest of a layer's quantization).
 *
 * S: d x d fp32 device, in/out (upper triangle, as gptq_hessian_accumulate).
 * X_host: n_tokens x d fp16 host memory, token-major.  Page-locked memory is
 *    needed for the copies to run asynchronously (pageable memory works but
 *    each copy then blocks the calling thread).  It is read after the call
 *    returns: keep it alive and unchanged until `stream` has passed the call.
 * stage: device buffer of at least 2 * chunk_tokens * d fp16 (stage_bytes).
 * chunk_tokens: tokens per chunk, 1 <= chunk_tokens <= 2^31.
 * stream, copy_stream: cudaStream_t; create copy_stream non-blocking for the
 *    copies to overlap (the same stream twice is allowed: no overlap).
 * ev_filled, ev_freed: cudaEvent_t, created by the caller (timing disabled
 *    is enough), on the device of S.
 * n_seen: optional HOST counter, incremented by n_tokens on success.
 * Requires the conditions of gptq_hessian_accumulate.  On GPTQ_ERR_CUDA
 * part of the work may have been queued; S is then undefined.
 */
int gptq_hessian_accumulate_host(float* S, const uint16_t* X_host, int64_t n_tokens, int64_t d,
                                 int64_t* n_seen, uint16_t* stage, size_t stage_bytes,
                                 int64_t chunk_tokens, void* stream, void* copy_stream,
                                 void* ev_filled, void* ev_freed);

/*
 * Grouped Hessian accumulation -- the sum of gptq_hessian_accumulate ("GPTQ /
 * AWQ / SqueezeLLM" sec. 一) for several independent groups of tokens at
 * once: the experts of a mixture-of-experts layer, each calibrated on the
 * tokens routed to it ("INT4/INT8 量化推理" sec. 五).
 *
 *   S_e[i][j] += sum_{offsets[e] <= t < offsets[e+1]} X[t][i] * X[t][j]
 *                                          0 <= i <= j < d, 0 <= e < n_groups
 *
 * S: n_groups x d x d fp32, in/out (S_e at S + e d^2; upper triangles only,
 *    as gptq_hessian_accumulate).
 * X: n_rows x d fp16, the groups' rows one after the other (e.g. the output
 *    of gptq_gather_rows).
 * offsets: HOST array of n_groups + 1 int64: offsets[0] == 0, non-decreasing,
 *    offsets[n_groups] == n_rows.  Empty groups are allowed (S_e unchanged).
 * n_seen: optional HOST array of n_groups counters, each incremented by its
 *    group's row count on success.
 * One kernel launch per 64 groups; its work items run over (group, token
 * split, output tile), so small and large groups share the SMs.  A group's
 * last box of 64 rows is cut at the group's end on the device (the next
 * group's rows never enter its sum).
 * Requires the d limits of gptq_hessian_accumulate, 0 <= n_rows <= 2^31,
 * 1 <= n_groups <= 2^20.
 */
int gptq_hessian_accumulate_grouped(float* S, const uint16_t* X, int64_t n_rows, int64_t d,
                                    const int64_t* offsets, int64_t n_groups, int64_t* n_seen,
                                    void* stream);

/*
 * Row gather -- the dispatch of routed tokens to experts that precedes the
 * per-expert Hessians ("INT4/INT8 量化推理" sec. 五):
 *   out[r][:] = X[idx[r]][:]      0 <= r < n_idx
 * X: n_rows x d fp16; idx: n_idx int32 (device, 4-byte aligned); out:
 * n_idx x d fp16.  An index outside [0, n_rows) is not followed: its row of
 * `out` is written as zeros and the device status (gptq_device_status)
 * records 0x201.  Requires d % 8 == 0, 8 <= d <= 32768.
 */
int gptq_gather_rows(const uint16_t* X, int64_t n_rows, int64_t d, const int32_t* idx,
                     int64_t n_idx, uint16_t* out, void* stream);

/*
 * Prepare the inverse-Hessian factor -- "GPTQ / AWQ / SqueezeLLM" sec. 一
 * (H = 2 X^T X / n, damping, decomposition of H^-1, importance order) and
 * "INT4/INT8 量化推理" sec. 三 (rows of H^-1 carry the error feedback).
 *
 *   H   = (2 / n) * S, symmetric (upper triangle of S mirrored)
 *   perm = stable descending argsort of diag(H) if act_order, else identity
 *   H   <- H[perm][:, perm];  lambda = damp_rel * mean(diag H);  Hd = H + lambda I
 *   U   = upper-triangular Cholesky factor of Hd^-1  (U^T U = Hd^-1)
 *
 * S: d x d fp32 from gptq_hessian_accumulate (upper triangle read, not written).
 * n_tokens: total tokens accumulated into S (> 0).
 * perm: d int32 output (written whenever non-NULL; required if act_order).
 * U: d x d fp32 output, row-major; strictly-lower triangle written as 0.
 * info: device int32 output: 0 on success, else a 1-based pivot index of Hd
 *       where the factorization met a non-positive pivot (U then undefined).
 * ws: scratch of gptq_prepare_workspace_bytes(d) bytes.
 * Requires d % 128 == 0, 128 <= d <= 32768, damp_rel >= 0.
 */
size_t gptq_prepare_workspace_bytes(int64_t d);
int gptq_prepare_hinv(const float* S, int64_t d, int64_t n_tokens, float damp_rel,
                      int act_order, int32_t* perm, float* U, int32_t* info,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * gptq_prepare_hinv without a workspace argument, for callers that cannot
 * allocate device memory (code running while a stream is captured into a
 * CUDA graph, where cudaMalloc is not allowed, or a plug-in inside an engine
 * that owns the whole device memory pool).  The pages have no counterpart:
 * this is an interface convenience of the library.
 *
 * Same arguments, results and errors as gptq_prepare_hinv, minus (ws,
 * ws_bytes).  Scratch is a fixed 16 MiB array inside the library that every
 * GPU loading the library holds until the process exits; it limits d to
 * 1024 (larger d returns GPTQ_ERR_SHAPE before anything is launched).  The
 * first call on a device looks up the array's device address (make it before
 * any stream capture begins).  All calls share the one array, so calls that
 * overlap on the GPU (e.g. on two streams at once) race: serialize them.
 * Nothing is allocated or freed.
 */
int gptq_prepare_hinv_static(const float* S, int64_t d, int64_t n_tokens, float damp_rel,
                             int act_order, int32_t* perm, float* U, int32_t* info,
                             void* stream);

/*
 * Batched preparation -- gptq_prepare_hinv ("GPTQ / AWQ / SqueezeLLM"
 * sec. 一) for n_mats independent Hessians of the same size, e.g. the
 * experts of a mixture-of-experts layer ("INT4/INT8 量化推理" sec. 五).
 * Every matrix gets exactly the result gptq_prepare_hinv gives it; the
 * factorizations of all matrices run in ONE persistent launch whose task
 * queue interleaves the matrices, so their latency chains overlap.
 *
 * S: n_mats x d x d fp32 (S_e at S + e d^2, upper triangles read).
 * n_tokens: HOST array of n_mats token counts (each > 0).
 * perm: n_mats x d int32 output or NULL (required if act_order).
 * U: n_mats x d x d fp32 output; info: n_mats device int32 outputs.
 * ws: gptq_prepare_batched_workspace_bytes(d, n_mats) bytes of scratch
 *    (n_mats times the single-matrix workspace, about 2 d^2 fp32 each).
 * Requires the d limits of gptq_prepare_hinv, 1 <= n_mats <= 4096 and
 * 2 n_mats d < 2^31.
 */
size_t gptq_prepare_batched_workspace_bytes(int64_t d, int64_t n_mats);
int gptq_prepare_hinv_batched(const float* S, int64_t n_mats, int64_t d, const int64_t* n_tokens,
                              float damp_rel, int act_order, int32_t* perm, float* U,
                              int32_t* info, void* ws, size_t ws_bytes, void* stream);

/*
 * Quantize one layer -- "INT4/INT8 量化推理" sec. 三 (column loop with error
 * compensation), "GPTQ / AWQ / SqueezeLLM" sec. 一 (blocks), "校准艺术"
 * sec. 2.1 (min-max), "INT4/INT8 量化推理" sec. 一 (group layout).
 *
 * For every row r, columns j = 0..d_in-1 in sweep order (W's columns taken
 * through perm when non-NULL):
 *   at a group start: mn = min(0, min w[j:j+g]), mx = max(0, max w[j:j+g])
 *                     (all zero: [-1, 1]); s = fp16(fp32(mx - mn) / maxq)
 *                     clamped to [2^-24, 65504]; z = clamp(rne(-mn / s), 0, maxq)
 *   c = clamp(rne(w_j / s) + z, 0, maxq);   e = w_j - s (c - z)
 *   E_j = e / U[j][j];  w[k] -= E_j U[j][k] for k > j;  row_loss[r] += E_j^2
 * (decisions in IEEE fp32; maxq = 2^bits - 1).  The feedback inside each
 * block of block_size columns is applied column by column on the CUDA cores;
 * the feedback onto later blocks is applied on the tensor cores in two
 * levels: after each block onto the rest of its 512-column outer block
 * (K = 128), and once per outer block onto every column beyond it (K = 512).
 *
 * W: d_out x d_in, dtype GPTQ_DTYPE_F16 or GPTQ_DTYPE_F32 (read only).
 * U: d_in x d_in fp32 from gptq_prepare_hinv (upper triangle read).
 * perm: d_in int32 or NULL (identity).
 * codes: d_out x d_in uint8 output, sweep order (code of column perm[k] at k).
 * scales: d_out x G fp16 output (G = d_in / group_size), zeros: d_out x G uint8.
 * row_loss: d_out fp32 output or NULL: sum_j E_j^2 (= tr(D Hd D^T) per row).
 * bits in {2,3,4,8}; group_size in {32, 64, 128}; or a multiple of 128
 * dividing d_in that divides 512 or is a multiple of 512 (256, 512, 1024,
 * ...: such a group never straddles the 512-column deferred-update block,
 * so at its first column every column of the group holds every earlier
 * column's correction and its parameters are taken there, as in the
 * unblocked sweep); or -1 (or d_in) for one group per row (G = 1: its
 * parameters come from the row before any correction, which is what "at the
 * group's first column" means for column 0); block_size == 128.
 * Requires d_in % 128 == 0, 128 <= d_in <= 32768, 1 <= d_out <= 2^24.
 */
size_t gptq_quantize_workspace_bytes(int64_t d_out, int64_t d_in, int block_size);
int gptq_quantize_layer(const void* W, int w_dtype, int64_t d_out, int64_t d_in,
                        const float* U, const int32_t* perm, int bits, int group_size,
                        int block_size, uint8_t* codes, uint16_t* scales, uint8_t* zeros,
                        float* row_loss, void* ws, size_t ws_bytes, void* stream);

/*
 * gptq_quantize_layer with STATIC groups: every group's scale and zero point
 * are taken, by the same min-max rule ("校准艺术" sec. 2.1), from the row as
 * it is before the sweep (W's columns in sweep order, no correction yet),
 * instead of from the corrected values at the group's first column.  The
 * codes, the error feedback and every other output are as in
 * gptq_quantize_layer.  The pages fix the group parameters only by the
 * min-max rule; this is the reading that parameterizes before correcting.
 * Same arguments and errors as gptq_quantize_layer, except group_size: 32,
 * 64, any multiple of 128 that divides d_in, or -1 (one group per row).
 */
int gptq_quantize_layer_static(const void* W, int w_dtype, int64_t d_out, int64_t d_in,
                               const float* U, const int32_t* perm, int bits, int group_size,
                               int block_size, uint8_t* codes, uint16_t* scales, uint8_t* zeros,
                               float* row_loss, void* ws, size_t ws_bytes, void* stream);

/*
 * Batched quantization -- gptq_quantize_layer ("INT4/INT8 量化推理" sec. 三)
 * for n_mats stacked layers of the same shape (the experts of a
 * mixture-of-experts layer, sec. 五 of the same page), each with its own U
 * and perm:
 *   W: n_mats x d_out x d_in (layer e at e d_out d_in elements),
 *   U: n_mats x d_in x d_in, perm: n_mats x d_in or NULL,
 *   codes: n_mats x d_out x d_in, scales / zeros: n_mats x d_out x G,
 *   row_loss: n_mats x d_out or NULL.
 * Each layer gets exactly the result of gptq_quantize_layer.  Workspace:
 * with ws_bytes >= n_mats * gptq_quantize_workspace_bytes(d_out, d_in,
 * block_size) (layer e's part at e times that size) the layers run
 * together: each 512-column outer block of every layer is swept in one
 * launch (their row tiles fill the SMs' waves together), then each layer's
 * columns beyond it are updated; with a smaller workspace (at least one
 * layer's) the layers run one after the other and share it.  Dynamic
 * 256-column groups always take the second schedule.
 * Dynamic groups only (group_size as gptq_quantize_layer).  Every layer's
 * slice must stay 16-byte aligned (GPTQ_ERR_SHAPE otherwise).
 * Pack the stacked codes and zero points with one gptq_pack_int4 call of
 * n_mats * d_out rows.
 */
int gptq_quantize_layer_batched(const void* W, int w_dtype, int64_t n_mats, int64_t d_out,
                                int64_t d_in, const float* U, const int32_t* perm, int bits,
                                int group_size, int block_size, uint8_t* codes, uint16_t* scales,
                                uint8_t* zeros, float* row_loss, void* ws, size_t ws_bytes,
                                void* stream);

/*
 * Pack INT4 -- "INT4/INT8 量化推理" sec. 一 (64 B of codes + 0.5 B zero point
 * + 2 B fp16 scale per 128 weights).
 *   qweight[r][w] = sum_k codes[r][8w + k] << 4k        (uint32, k = 0..7)
 *   qzeros[r][b]  = zeros[r][2b] | zeros[r][2b+1] << 4   (odd G: high nibble 0)
 * codes: d_out x d_in uint8 (values 0..15), zeros: d_out x G uint8.
 * qweight: d_out x d_in/8 uint32 out, qzeros: d_out x ceil(G/2) uint8 out.
 * Requires d_in % 8 == 0, G >= 1.
 */
int gptq_pack_int4(const uint8_t* codes, const uint8_t* zeros, int64_t d_out, int64_t d_in,
                   int64_t n_groups, uint32_t* qweight, uint8_t* qzeros, void* stream);

/* Inverse of gptq_pack_int4 (bit-exact round trip). */
int gptq_unpack_int4(const uint32_t* qweight, const uint8_t* qzeros, int64_t d_out,
                     int64_t d_in, int64_t n_groups, uint8_t* codes, uint8_t* zeros,
                     void* stream);

/*
 * Pack b-bit codes -- the storage of "INT4/INT8 量化推理" sec. 一 for the
 * page's other widths (INT8 beside INT4; 2 and 3 bits for the low-bit
 * cases), read as one little-endian bit stream per row:
 *   code k of row r occupies bits [b k, b k + b) of row r's stream, stored
 *   as d_in * b / 32 uint32 words (word w = bits [32 w, 32 w + 32));
 *   zero point g of row r occupies bits [b g, b g + b) of a second stream,
 *   stored as ceil(G b / 8) bytes (the last byte padded with zero bits).
 * For b = 4 this is exactly gptq_pack_int4's layout (66.5 B per 128 weights
 * with the fp16 scale); b = 3 gives 50.375 B, b = 8 131 B per 128 weights.
 * codes: d_out x d_in uint8 (values masked to b bits), zeros: d_out x G.
 * qweight: d_out x (d_in b / 32) uint32 out (4-byte aligned), qzeros:
 * d_out x ceil(G b / 8) uint8 out.  bits in 2..8 (else UNSUPPORTED);
 * requires d_in % 32 == 0, 1 <= G <= d_in, codes 16-byte aligned.
 */
int gptq_pack_bits(const uint8_t* codes, const uint8_t* zeros, int64_t d_out, int64_t d_in,
                   int64_t n_groups, int bits, uint32_t* qweight, uint8_t* qzeros, void* stream);

/* Inverse of gptq_pack_bits (bit-exact round trip). */
int gptq_unpack_bits(const uint32_t* qweight, const uint8_t* qzeros, int64_t d_out, int64_t d_in,
                     int64_t n_groups, int bits, uint8_t* codes, uint8_t* zeros, void* stream);

/*
 * Weight-only INT4 product on the packed layer (W4A16) -- "INT4/INT8 量化推理"
 * sec. 六 (weights in 4 bits, activations in fp16), on the storage of sec. 一
 * of the same page:
 *   y[b][r] = sum_j x[b][j] Q[r][j],  Q[r][perm[k]] = s[r][k/g] (c[r][k] - z[r][k/g])
 * with c, z unpacked from qweight / qzeros (gptq_pack_int4's layout, codes in
 * sweep order) and s the fp16 scales.  Products and sums are fp32 (the
 * products on the tensor cores, m16n8k16, exact); the dequantized weights
 * are exact.  Decode-sized: every CTA requests its rows' packed bytes for
 * one 2048-column slice at once (bulk copies), the slices' partial sums
 * meet in y by atomic adds.
 * x: batch x d_in fp16 (original column order); y: batch x d_out fp32 output
 * (overwritten).  perm: d_in int32 or NULL (identity), as gptq_prepare_hinv
 * returned it.  group_size: a multiple of 32 dividing d_in, or -1 (one group
 * per row).  batch in 1..8 (decode-sized; larger batches are UNSUPPORTED).
 * Requires d_in % 128 == 0, 128 <= d_in <= 32768, 1 <= d_out <= 2^24.
 */
int gptq_w4a16_gemm(const uint16_t* x, int64_t batch, const uint32_t* qweight,
                    const uint16_t* scales, const uint8_t* qzeros, const int32_t* perm,
                    int64_t d_out, int64_t d_in, int group_size, float* y, void* stream);

/*
 * W4A16 product on the tensor cores for any batch -- the same product as
 * gptq_w4a16_gemm ("INT4/INT8 量化推理" sec. 六 on the storage of sec. 一):
 *   y[b][r] = sum_j x[b][j] Q[r][j],  Q[r][perm[k]] = s[r][k/g] (c[r][k] - z[r][k/g])
 * The packed words are turned into exact fp16 (c - z) operands in shared
 * memory and multiplied with the fp16 activations by tcgen05 kind::f16
 * (fp32 accumulation in TMEM, at most 512 products per accumulation, each
 * group's sum scaled by its fp16 scale in fp32).
 * x: batch x d_in fp16 (original column order); y: batch x d_out fp32 out.
 * perm: d_in int32 or NULL.  ws: gptq_w4a16_matmul_workspace_bytes(batch,
 * d_in) bytes, always (the activations are first gathered into the order in
 * which the kernel lays out each packed word's columns, through perm when
 * given).
 * group_size: a multiple of 64 dividing d_in, or -1 (smaller groups:
 * gptq_w4a16_gemm).  1 <= batch <= 2^24; the d limits of gptq_w4a16_gemm.
 */
size_t gptq_w4a16_matmul_workspace_bytes(int64_t batch, int64_t d_in);
int gptq_w4a16_matmul(const uint16_t* x, int64_t batch, const uint32_t* qweight,
                      const uint16_t* scales, const uint8_t* qzeros, const int32_t* perm,
                      int64_t d_out, int64_t d_in, int group_size, float* y, void* ws,
                      size_t ws_bytes, void* stream);

/*
 * Round-to-nearest baseline -- "大模型量化实战（上）" (RTN: every weight
 * rounded on its own) with the min-max group quantizer of "校准艺术" sec. 2.1:
 * the same group parameters and codes as gptq_quantize_layer, taken on the
 * original W with no error feedback.  Same argument meaning and limits as
 * gptq_quantize_layer (natural column order, no U, no workspace), except
 * group_size: 32, 64, 128, any multiple of 128 dividing d_in, or -1.
 */
int rtn_quantize(const void* W, int w_dtype, int64_t d_out, int64_t d_in, int bits,
                 int group_size, uint8_t* codes, uint16_t* scales, uint8_t* zeros,
                 void* stream);

/*
 * Channel magnitudes for activation-aware scaling -- "GPTQ / AWQ /
 * SqueezeLLM" sec. 二 (the mean absolute activation of each input channel):
 *   abs_sum[j] += sum_t |X[t][j]|      (fp64 accumulation; mean = abs_sum / n)
 * X: n_tokens x d fp16; abs_sum: d fp64 device, in/out (zero it first; call
 * once per calibration batch).  Requires d % 8 == 0, 8 <= d <= 32768.
 */
int gptq_channel_abs_sum(const uint16_t* X, int64_t n_tokens, int64_t d, double* abs_sum,
                         void* stream);

/*
 * Activation-aware channel scaling chosen by output error -- "GPTQ / AWQ /
 * SqueezeLLM" sec. 二 (scale input channels by activation magnitude, pick
 * among candidate scalings the one with the smallest output error, then
 * GPTQ) and "INT4/INT8 量化推理" sec. 四 (W diag(s) with X diag(s)^-1 is exact
 * before quantization).  The pages give no candidate set; the reading is:
 *   a_j = abs_sum_j / n_tokens, raised to the smallest positive a where 0
 *   (all zero: a = 1); r = a / mean(a); for k = 0 .. n_grid - 1,
 *   alpha = k / n_grid, s = r^alpha (alpha = 0 is no scaling);
 *   W' = W diag(s) (fp64, rounded once to fp32), Q' = the group round-to-
 *   nearest of W' (the quantizer of rtn_quantize), D = Q' diag(s)^-1 - W,
 *   losses[k] = tr(D H D^T) with H = 2 S / n_tokens;
 *   *best = the first k with the smallest loss; scales = s of that k.
 * Optionally W_scaled = fp32(W diag(s)) and S_scaled = fp32(diag(s)^-1 S
 * diag(s)^-1) (upper triangle, the strictly-lower part written as 0): the
 * inputs of gptq_prepare_hinv / gptq_quantize_layer for GPTQ in the scaled
 * coordinates (dequantize with Q diag(s)^-1).
 * W: d_out x d_in (GPTQ_DTYPE_F16 / F32); S: d_in x d_in fp32 (upper
 * triangle, from gptq_hessian_accumulate); abs_sum: d_in fp64 from
 * gptq_channel_abs_sum; losses: n_grid fp64 out; best: 1 int32 out; scales:
 * d_in fp64 out; W_scaled: d_out x d_in fp32 or NULL; S_scaled: d_in x d_in
 * fp32 or NULL (all device).  ws: gptq_awq_workspace_bytes(d_out, d_in).
 * The losses' products D H run on the tensor cores in split-TF32 (fp32-level
 * accuracy), their sums in fp64.  bits in {2,3,4,8}; group_size a multiple
 * of 32 dividing d_in, or -1; 1 <= n_grid <= 1000; the d limits of
 * gptq_quantize_layer.
 */
size_t gptq_awq_workspace_bytes(int64_t d_out, int64_t d_in);
int gptq_awq_search(const void* W, int w_dtype, int64_t d_out, int64_t d_in, const float* S,
                    int64_t n_tokens, const double* abs_sum, int n_grid, int bits, int group_size,
                    double* losses, int32_t* best, double* scales, float* W_scaled,
                    float* S_scaled, void* ws, size_t ws_bytes, void* stream);

/*
 * Test hook (no counterpart on the pages): a stand-alone split-TF32
 * tensor-core GEMM.  It takes every product the way the factorization and
 * the block update do (x = x_hi + x_lo, x_hi rounded to TF32; three
 * kind::tf32 MMAs A_hi B_hi + A_hi B_lo + A_lo B_hi accumulated in TMEM), so
 * a test can check on its own that this arithmetic keeps fp32-level accuracy
 * on the hardware.  The library's kernels do not call it.
 *   C = beta * C + alpha * A * B^T
 * A: M x K (lda), B: N x K (ldb), C: M x N (ldc), dense row-major fp32 device
 * arrays; K % 32 == 0; leading dimensions multiples of 4.  lower != 0
 * computes only 128x128 output tiles on or below the diagonal (M == N).
 */
int gptq_debug_gemm_nt(const float* A, int64_t lda, const float* B, int64_t ldb, float* C,
                       int64_t ldc, int64_t M, int64_t N, int64_t K, float alpha, float beta,
                       int lower, void* stream);

/*
 * Diagnostics (no counterpart on the pages): per-kind kernel timing.
 * gptq_debug_kernel_timing(1) makes every later launch of the library
 * bracket itself with two CUDA events on its stream; gptq_debug_kernel_times
 * waits for the recorded events, returns per kind the summed milliseconds
 * (ms[k]) and the number of timed launch sites (spans[k]), and forgets the
 * records.  Kinds, in order (n_kinds >= 16): hessian, gather, finalize,
 * factorization, init_work, split_u, static_params, sweep, update_near,
 * update_far, pack, unpack, rtn, w4a16, probe, awq (names from
 * gptq_debug_kernel_kind_name).  Use it on eager launches only, never while
 * a stream is being captured; it creates two CUDA events per launch site
 * while enabled.  Disabled (the default) it costs one flag test per launch.
 */
int gptq_debug_kernel_timing(int enable);
int gptq_debug_kernel_times(double* ms, int64_t* spans, int n_kinds);
const char* gptq_debug_kernel_kind_name(int kind);

/*
 * Test hooks (host only, no GPU needed; no counterpart on the pages).
 *
 * gptq_debug_chol_task_order: the tiled factorization's tasks of a d x d
 * preparation in the order CTAs claim them: out[3t .. 3t+2] = (type, i, j)
 * for task t, type 0 = diagonal tile j (factor + invert), 1 = tile (i, j) of
 * L, 2 = tile (i, j) of L^-1.  Needs cap >= 3 (d/128)^2 int32s.  Returns the
 * task count, or minus a status code.
 *
 * gptq_debug_div_rn: out[i] = the quantizer's division-free quotient
 * x[i] / s[i] (reciprocal plus two FMA corrections) for s[i] > 0 finite,
 * computed by the function the sweep kernel uses.  Returns a status code.
 */
int64_t gptq_debug_chol_task_order(int64_t d, int32_t* out, int64_t cap);
int gptq_debug_div_rn(const float* x, const float* s, int64_t n, float* out);

/*
 * Test hook (no counterpart on the pages): failure detection without a GPU
 * fault.  Runs one of the library's bounded waits against a condition that
 * never comes true, with a wait limit of limit_ns nanoseconds instead of
 * the kernels' 4 s:
 *   which = 0: the completion-flag wait tasks use for their dependencies,
 *              on the device int32 *flag (returns at once when it is
 *              non-zero; otherwise gives up and records 0x105);
 *   which = 1: the mbarrier wait of the TMA pipelines, on a fresh barrier
 *              nobody arrives on (gives up and records 0x101; flag unused).
 * The recorded code is read (and cleared) with gptq_device_status; the
 * kernel returns normally either way.  Asynchronous on `stream`.
 * Requires 1e6 <= limit_ns <= 1e9; flag 4-byte aligned when which = 0.
 */
int gptq_debug_bounded_wait(const int32_t* flag, int which, int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_GPTQ_H */
